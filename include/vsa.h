/*
 * vsa.h -- C ABI of libvsa: VSA-style 3-D block-sparse attention on B200 (sm_100a).
 *
 * The method (FastVideo VSA user guide, intro): the post-patch latent grid
 * (T, Hh, W) of a video DiT is cut into spatio-temporal tiles; each query tile
 * scores every key/value tile and attends only to the tokens of its top-k
 * tiles.  Two calls make the forward pass:
 *
 *   vsa_select    mean-pool Q and K per tile, score every tile pair,
 *                 keep the top-k key tiles per query tile   -> idx
 *   vsa_attn_fwd  exact softmax attention of each query tile over the
 *                 tokens of its kept tiles                  -> O, LSE
 *
 * Conventions shared by every call
 * --------------------------------
 * Tensors are dense, row-major, on the current CUDA device, in one of two
 * layouts (vsa_shape.layout):
 *   VSA_LAYOUT_BHND  Q : [B, H, Nq, d]   K, V : [B, H, Nk, d]   O like Q
 *   VSA_LAYOUT_BNHD  Q : [B, Nq, H, d]   K, V : [B, Nk, H, d]   O like Q
 *                (the token-major layout a DiT's projections produce)
 *   element type bfloat16 or float16 (vsa_shape.dtype); Nq = T*Hh*W over the
 *   query grid, Nk = Tk*Hk*Wk over the key/value grid; token n = (t*Hh + y)*W
 *   + x (raster order over its grid; no permutation to tile order is needed
 *   -- the kernels evaluate the tile index map themselves, as the fastbsa
 *   page's "How it works" describes)
 *   idx        : int32 [B, H, nTq, topk], kept key/value tiles of each query
 *                tile, strictly ascending, each in [0, nTk)
 *   LSE        : float32 [B, H, Nq] in both layouts, natural log of the
 *                softmax denominator
 *
 * Always-kept prefix tiles (FastVideo guide, "Choose top-k": the H3 route
 * uses 64-token blocks and keeps all prefix blocks): with prefix_tiles = P,
 * key/value tiles 0 .. P-1 (the first in raster order -- e.g. the tiles of
 * leading conditioning frames) are in every query tile's kept list whatever
 * their scores, and the other topk - P are the best-scoring of the rest;
 * P <= topk.
 *
 * Query and key/value grids (fastbsa page, "Use": separate latent and chunk
 * shapes for q and k): by default both sides use the query grid and tile
 * (self-attention with equal lengths, the Wan route of the FastVideo guide).
 * Setting Tk, Hk, Wk and/or tk, hk, wk gives the key/value side its own grid
 * and tile; the two tiles must hold the same number of tokens.
 *
 * Tiles: nT = ceil(T/tt) * ceil(Hh/th) * ceil(W/tw) per side (the user
 * guide's routing log: grid (31,22,40), tile (4,8,8) -> 120 tiles); edge tiles
 * are partial and their missing tokens are left out of pooling and of the
 * softmax.  Tile j = (bt * ceil(Hh/th) + by) * ceil(W/tw) + bx (raster over
 * tile coordinates).
 *
 * Supported: bf16 or fp16 inputs (O has the input type; pooling, scores,
 * softmax and accumulation are float32); d in {64, 128}; tile extents powers
 * of two with tt*th*tw in {64, 128, 256} (the guide's 4x4x4 = 64 and 4x8x8 =
 * 256 blocks), the same volume on both sides, and tt >= 2 when it is 256;
 * H_q = H_kv; non-causal attention, no mask.  Inputs must be finite (NaN/Inf
 * give unspecified results, never a fault; in the [B, N, H, d] layout a box
 * past the last frame reads the next batch's first frames and masks them,
 * so those must be finite too).
 *
 * Ownership: the caller allocates every buffer (including the select
 * workspace); no call allocates device memory.  (The one piece of device
 * memory the library owns is the fixed scratch array of vsa_select_noalloc,
 * reserved when the library's device code is first loaded on a GPU.)  Calls
 * are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 * stream).  Every call checks its arguments before launching anything and
 * returns a vsa_status; nothing is launched on error.  Faults inside a
 * kernel are reported through vsa_device_error() (bounded waits in the
 * kernels turn a stall into an error code instead of a hang).
 */
#ifndef VSA_H_
#define VSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct vsa_shape {
  int32_t B, H;          /* batch, heads (query heads == key/value heads)     */
  int32_t T, Hh, W;      /* query post-patch latent grid                      */
  int32_t d;             /* head dimension: 64 or 128                         */
  int32_t tt, th, tw;    /* query tile extents along T, Hh, W                  */
  int32_t dtype;         /* element type of Q, K, V, O: VSA_DTYPE_BF16 (0, the
                            default of a zeroed struct) or VSA_DTYPE_F16      */
  int32_t layout;        /* VSA_LAYOUT_BHND (0, default) or VSA_LAYOUT_BNHD   */
  int32_t Tk, Hk, Wk;    /* key/value grid; all 0 (default): the query grid   */
  int32_t tk, hk, wk;    /* key/value tile; all 0 (default): the query tile   */
  int32_t prefix_tiles;  /* key/value tiles 0 .. prefix_tiles-1 are kept for
                            every query tile (counted in topk); 0: none        */
} vsa_shape;

/* Element types (FastVideo VSA guide, "Verify routing and fallback": the
 * Wan route takes FP16 or BF16 tensors). */
#define VSA_DTYPE_BF16 0
#define VSA_DTYPE_F16 1

/* Memory layouts of Q, K, V and O (see the conventions above). */
#define VSA_LAYOUT_BHND 0
#define VSA_LAYOUT_BNHD 1

typedef enum vsa_status {
  VSA_OK = 0,
  VSA_ERR_INVALID_ARG = 1,  /* NULL pointer, non-positive extent (incl. a key/
                               value grid or tile given in part), bad scale,
                               prefix_tiles outside [0, nTk]                    */
  VSA_ERR_TOPK_RANGE = 2,   /* topk <= 0, topk > nTk or topk < prefix_tiles
                               (guide: topk must be positive; topk >
                               num_blocks is invalid), or a sparsity outside
                               [0, 1)                                           */
  VSA_ERR_UNSUPPORTED = 3,  /* d, dtype, layout or tile shape outside the
                               supported set (incl. unequal tile volumes)       */
  VSA_ERR_ALIGNMENT = 4,    /* a tensor pointer not 16-byte aligned            */
  VSA_ERR_WORKSPACE = 5,    /* workspace NULL or smaller than required         */
  VSA_ERR_ARCH = 6,         /* current device is not sm_100                    */
  VSA_ERR_CUDA = 7,         /* a CUDA runtime/driver call failed               */
  VSA_ERR_TOO_LARGE = 8     /* more than 1536 tiles per head on a side, B*H >
                               65535, or (64-token tiles) topk too large for
                               shared memory                                    */
} vsa_status;

/* Query tile count of a shape (FastVideo VSA guide, "Wan top-k behavior":
 * num_blocks).  num_tiles: out, nTq.  tiles_per_axis: out [3] (ceil per
 * axis) or NULL.  Host only; touches no device. */
int vsa_tile_count(const vsa_shape* shape, int32_t* num_tiles, int32_t* tiles_per_axis);

/* Key/value tile count nTk (equal to nTq unless the shape gives the key/value
 * side its own grid or tile).  Same arguments as vsa_tile_count. */
int vsa_kv_tile_count(const vsa_shape* shape, int32_t* num_tiles, int32_t* tiles_per_axis);

/* Kept tiles per query tile for a sparsity (fastbsa page, "Use": sparsity =
 * the fraction of key/value tiles left out, 0.9375 keeping 45 of 720):
 * topk = round((1 - sparsity) * nTk) (halves round up), clamped to
 * [max(1, prefix_tiles), nTk].
 * sparsity must lie in [0, 1).  Host only. */
int vsa_topk_from_sparsity(const vsa_shape* shape, float sparsity, int32_t* topk);

/* Bytes of device workspace vsa_select needs for `shape`: the pooled tile
 * means, float32, channel-major so the score kernel reads contiguous tile
 * rows: Q means [B*H, d, ldq] then K means [B*H, d, ldk], ldq and ldk = nTq
 * and nTk rounded up to a multiple of 4.  Returns 0 for an invalid shape. */
size_t vsa_select_workspace_bytes(const vsa_shape* shape);

/* Tile selection (FastVideo VSA guide intro and "Wan top-k behavior"; fastbsa
 * page "How it works": selection kept on chip, no score matrix in HBM).
 *   q, k      : device Q and K in shape->layout and shape->dtype, 16-byte aligned
 *   topk      : kept key tiles per query tile, max(1, prefix_tiles) <= topk <= nTk
 *               (topk == nTk keeps every tile: the dense case)
 *   idx_out   : device int32 [B, H, nTq, topk]; row i gets the topk tiles j with
 *               the largest s_ij = mean_i(Q) . mean_j(K) (float32 means over the
 *               tile's valid tokens, float32 dot), ties to the lower j, written
 *               in ascending j order
 *   workspace : device buffer of at least vsa_select_workspace_bytes(shape)
 *               bytes, 16-byte aligned; contents on entry are ignored
 * Two kernel launches on `stream`. */
int vsa_select(const vsa_shape* shape, const void* q, const void* k, int32_t topk,
               int32_t* idx_out, void* workspace, size_t workspace_bytes, void* stream);

/* Tile selection for callers that cannot allocate device memory (no
 * counterpart in the paper; an addition of this library).
 *
 * Same arguments and results as vsa_select, minus the workspace: the pooled
 * tile means live in a fixed scratch array inside the library
 * (VSA_SELECT_NOALLOC_SCRATCH_BYTES per GPU, held until the process exits).
 * Meant for callers that must not call cudaMalloc -- a host framework that
 * owns all device memory through its own pool, code running inside a region
 * where allocation is forbidden, or a plugin with no allocator handle.  This
 * call itself allocates nothing (no cudaMalloc, no cudaFree, no allocating
 * library routine).
 *   - The scratch array is reserved when the library's device code is first
 *     loaded on a GPU.  With CUDA's lazy module loading (the default) that
 *     happens inside the first vsa_* call that touches the device, which may
 *     be this one: make one call on each device early -- vsa_device_error
 *     will do -- before a memory pool takes the device's memory and before
 *     any CUDA stream capture.
 *   - The scratch needs vsa_select_workspace_bytes(shape) bytes (about
 *     2*B*H*nT*d*4); larger shapes are rejected with VSA_ERR_WORKSPACE before
 *     anything is launched.
 *   - The first call on a device (with that device current) looks up the
 *     scratch array's device address (again after a cudaDeviceReset, which
 *     makes a new context); make that first call before any stream capture.
 *   - Every call on a device shares the one scratch array: calls that can
 *     overlap on the GPU (different streams, no ordering) race and give
 *     wrong indices.  Nothing needs clearing between calls: every mean a
 *     call uses is written by that call first (the score kernel also reads
 *     the row padding past nT, left from earlier calls, but masks those
 *     columns out).
 * Two kernel launches on `stream`. */
#define VSA_SELECT_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int vsa_select_noalloc(const vsa_shape* shape, const void* q, const void* k, int32_t topk,
                       int32_t* idx_out, void* stream);

/* Block-sparse attention forward (FastVideo VSA guide intro: attention only
 * against the selected top-k blocks; "Verify routing and fallback": scale
 * head_size ** -0.5 by default, non-causal, no mask).
 *   q, k, v       : device Q, K, V in shape->layout and shape->dtype, 16-byte
 *                   aligned
 *   idx           : device int32 [B, H, nTq, topk], strictly ascending tiles
 *                   (as vsa_select writes them); an entry outside [0, nTk)
 *                   sets VSA_DEVERR_BAD_INDEX and is read as tile 0 instead,
 *                   a row that is not strictly ascending sets
 *                   VSA_DEVERR_BAD_ORDER (the row is still attended, with an
 *                   unspecified result); neither faults
 *   softmax_scale : > 0 and finite; pass d ** -0.5 for the standard scale
 *   o             : device O out, layout and type of q, 16-byte aligned
 *   lse           : device float32 [B, H, Nq] out, natural log
 * For every token n of query tile i: O[n] = softmax_m(scale * Q[n].K[m]) V[m]
 * over the valid tokens m of the tiles idx[i, :]; LSE[n] = log of the
 * denominator.  One kernel launch on `stream`. */
int vsa_attn_fwd(const vsa_shape* shape, const void* q, const void* k, const void* v,
                 const int32_t* idx, int32_t topk, float softmax_scale,
                 void* o, float* lse, void* stream);

/* Pooled coarse branch (FastVideo VSA guide, "Checkpoint behavior": Wan
 * checkpoints that carry learned to_gate_compress weights add a gated
 * compensation to the sparse branch; without them the sparse branch runs
 * alone).  The pages give no formula; this library's reading: attention at
 * tile granularity,
 *   o_coarse[i] = sum_j softmax_j(scale * qbar_i . kbar_j) vbar_j
 * over every key/value tile j (one softmax entry per tile, whatever its
 * token count), with qbar, kbar, vbar the tiles' means over their valid
 * tokens, and O[n] = O_sparse[n] + gate[n] * o_coarse[tile of n], the gate
 * being the caller's projection output (same shape and type as O).
 *
 * Bytes of workspace vsa_select_coarse needs: the Q, K and V tile means,
 * float32, channel-major ([B*H, d, ldq], then [B*H, d, ldk] twice).
 * Returns 0 for an invalid shape. */
size_t vsa_select_coarse_workspace_bytes(const vsa_shape* shape);

/* vsa_select plus the coarse branch's tile-level attention.
 *   q, k, v       : device Q, K, V as for vsa_attn_fwd
 *   softmax_scale : > 0 and finite (the fine branch's scale)
 *   idx_out       : as vsa_select
 *   coarse_out    : device float32 [B, H, nTq, d], o_coarse of every query
 *                   tile (16-byte aligned for vsa_attn_fwd_gated)
 *   workspace     : at least vsa_select_coarse_workspace_bytes(shape) bytes,
 *                   16-byte aligned
 * Three kernel launches on `stream`. */
int vsa_select_coarse(const vsa_shape* shape, const void* q, const void* k, const void* v, int32_t topk,
                      float softmax_scale, int32_t* idx_out, float* coarse_out, void* workspace,
                      size_t workspace_bytes, void* stream);

/* vsa_attn_fwd whose output also carries the gated coarse branch:
 * O[n] = sparse attention (as vsa_attn_fwd) + gate[n] * coarse[tile of n],
 * added in float32 before O is rounded to the input type; LSE is the sparse
 * branch's.  coarse: device float32 [B, H, nTq, d] (from vsa_select_coarse),
 * gate: device tensor of O's layout and type; both 16-byte aligned and both
 * required (VSA_ERR_INVALID_ARG otherwise).  One kernel launch on `stream`. */
int vsa_attn_fwd_gated(const vsa_shape* shape, const void* q, const void* k, const void* v,
                       const int32_t* idx, int32_t topk, float softmax_scale, const float* coarse,
                       const void* gate, void* o, float* lse, void* stream);

/* Host-to-host forward (the per-call, end-to-end figure of the fastbsa page,
 * "The number"): vsa_select + vsa_attn_fwd on Q, K, V in HOST memory, with
 * O, LSE and idx written back to host memory.  The (batch, head) pairs go
 * through the GPU in chunks of chunk_heads heads: while chunk i runs its
 * kernels, chunk i+1 is uploaded and chunk i-1 downloaded (three streams
 * of the library, created on the first call on a device; the caller's
 * stream waits for all of it, so the host outputs are complete once the
 * caller synchronizes that stream).  Every vsa_shape field applies; in the
 * [B, N, H, d] layout a chunk is heads of one batch, copied as strided 2-D
 * blocks.
 *   q, k, v      : host Q, K, V in shape->layout and shape->dtype (pinned
 *                  memory for the copies to overlap the kernels)
 *   o, lse, idx  : host outputs, layouts as for vsa_attn_fwd / vsa_select
 *   chunk_heads  : heads per chunk (clamped to [1, H] in [B, N, H, d], to
 *                  [1, B*H] otherwise)
 *   workspace    : device buffer of at least
 *                  vsa_forward_host_workspace_bytes(shape, topk, chunk_heads)
 *                  bytes, 16-byte aligned: two sets of chunk buffers
 * A failure part-way returns VSA_ERR_CUDA with some chunks enqueued. */
size_t vsa_forward_host_workspace_bytes(const vsa_shape* shape, int32_t topk, int32_t chunk_heads);
int vsa_forward_host(const vsa_shape* shape, const void* q, const void* k, const void* v, int32_t topk,
                     float softmax_scale, void* o, float* lse, int32_t* idx, int32_t chunk_heads,
                     void* workspace, size_t workspace_bytes, void* stream);

/* Reads (and with reset != 0 clears) the kernels' device error word on the
 * current device: 0 = no error; otherwise a VSA_DEVERR_* code.  Synchronizes
 * the device.  Returns a vsa_status for the read itself. */
int vsa_device_error(uint32_t* code, int32_t reset);

#define VSA_DEVERR_NONE 0u
#define VSA_DEVERR_WAIT_TIMEOUT 1u   /* an mbarrier wait ran past its bound     */
#define VSA_DEVERR_BAD_INDEX 2u      /* idx entry outside [0, nTk)             */
#define VSA_DEVERR_BAD_ORDER 3u      /* idx row not strictly ascending (a
                                        repeated or out-of-order tile)         */

/* Human-readable name of a vsa_status value.  Never NULL. */
const char* vsa_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H_ */
