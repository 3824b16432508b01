"""VSA-style 3-D block-sparse attention for B200 (sm_100a).

The latent grid (T, Hh, W) of a video DiT is cut into spatio-temporal tiles;
each query tile keeps the top-k key/value tiles by mean-pooled Q.K score and
attends only to their tokens.  The work runs in libvsa.so (C ABI in
include/vsa.h); ``api`` wraps it for torch tensors.
"""
from . import api  # noqa: F401
from .api import attn_fwd, device_error, forward, select, tile_count  # noqa: F401
