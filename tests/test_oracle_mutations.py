"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin fails.

Each case swaps one oracle function for a subtly wrong version -- the kind of
slip a restatement of the method could make -- and runs the pin that should
catch it.  A pin that still passed would not be pinning anything.
"""
import numpy as np
import pytest

from oracle import vsa_oracle as vo
import tests.test_oracle_pins as pins


def _zero_padded_pool(X, grid, tile):
    vol = tile[0] * tile[1] * tile[2]
    return np.stack([X[t].sum(axis=0) / vol for t in vo.tile_tokens(grid, tile)])


def _transposed_scores(qbar, kbar):
    return kbar @ qbar.T


def _ties_to_higher(s_row, topk):
    order = np.lexsort((-np.arange(s_row.shape[0]), -s_row))
    return np.sort(order[:topk])


_orig_attend = vo.attend_head


def _drop_last_kept(Q, K, V, grid, tile, idx, scale, query_tiles=None):
    return _orig_attend(Q, K, V, grid, tile, idx[:, :-1], scale, query_tiles)


def _dense_no_scale(Q, K, V, scale):
    z = Q @ K.T
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    l = e.sum(axis=1, keepdims=True)
    return (e @ V) / l, (m + np.log(l))[:, 0]


def _attend_log2_lse(Q, K, V, grid, tile, idx, scale, query_tiles=None):
    O, L = _orig_attend(Q, K, V, grid, tile, idx, scale, query_tiles)
    return O, L / np.log(2.0)


_orig_tokens = vo.tile_tokens


def _floor_tiles(grid, tile):
    return [t for t in _orig_tokens(grid, tile) if t.size == tile[0] * tile[1] * tile[2]]


_orig_select_head = vo.select_head


def _select_kv_with_query_tile(Q, K, grid, tile, topk, grid_k=None, tile_k=None):
    return _orig_select_head(Q, K, grid, tile, topk, grid_k, tile)


def _attend_kv_with_query_tiles(Q, K, V, grid, tile, idx, scale, query_tiles=None, grid_k=None, tile_k=None):
    return _orig_attend(Q, K, V, grid, tile, idx, scale, query_tiles)


def _prefix_dropped(scores, prefix):
    s = np.array(scores, dtype=np.float64, copy=True)
    s[..., :prefix] = -np.inf
    return s


def _coarse_unscaled(Q, K, V, grid, tile, scale, grid_k=None, tile_k=None):
    return _orig_coarse(Q, K, V, grid, tile, 1.0, grid_k, tile_k)


def _coarse_token_weighted(Q, K, V, grid, tile, scale, grid_k=None, tile_k=None):
    """Softmax weights multiplied by each key block's token count."""
    qbar, kbar, vbar = vo.pool(Q, grid, tile), vo.pool(K, grid, tile), vo.pool(V, grid, tile)
    cnt = np.array([t.size for t in vo.tile_tokens(grid, tile)], dtype=np.float64)
    z = scale * (qbar @ kbar.T)
    e = np.exp(z - z.max(axis=1, keepdims=True)) * cnt[None, :]
    return (e @ vbar) / e.sum(axis=1, keepdims=True)


def _coarse_softmax_wrong_axis(Q, K, V, grid, tile, scale, grid_k=None, tile_k=None):
    qbar, kbar, vbar = vo.pool(Q, grid, tile), vo.pool(K, grid, tile), vo.pool(V, grid, tile)
    z = scale * (qbar @ kbar.T)
    e = np.exp(z - z.max(axis=0, keepdims=True))
    return (e @ vbar) / e.sum(axis=0, keepdims=True)


_orig_coarse = vo.coarse_head


def _gate_next_block(O, gate, oc, grid, tile):
    return _orig_gated(O, gate, np.roll(oc, 1, axis=0), grid, tile)


_orig_gated = vo.gated_output

CASES = [
    ("pool", _zero_padded_pool, lambda: pins.test_pool_constant_per_block_partial_edges()),
    ("tile_scores", _transposed_scores, lambda: pins.test_scores_hand_example()),
    ("topk_row", _ties_to_higher, lambda: pins.test_ties_go_to_lower_index()),
    ("attend_head", _drop_last_kept,
     lambda: pins.test_all_blocks_equals_dense((5, 6, 7), (4, 4, 4))),
    ("dense_bruteforce", _dense_no_scale, lambda: pins.test_dense_vs_library_sdpa()),
    ("attend_head", _attend_log2_lse, lambda: pins.test_lse_normalises_weights()),
    ("tile_tokens", _floor_tiles, lambda: pins.test_block_token_counts(
        pins.WAN5B, {256: 70, 192: 45, 144: 5})),
    ("select_head", _select_kv_with_query_tile, lambda: pins.test_kv_pool_uses_kv_tiles()),
    ("attend_head", _attend_kv_with_query_tiles,
     lambda: pins.test_kv_grid_all_blocks_equals_dense(*pins.KV_CASES[0])),
    ("keep_prefix", _prefix_dropped, lambda: pins.test_prefix_blocks_always_kept(3, 5)),
    ("bf16_to_f64", vo.f16_to_f64, lambda: pins.test_bf16_widening_textbook_values()),
    ("coarse_head", _coarse_unscaled, lambda: pins.test_coarse_scale_matters()),
    ("coarse_head", _coarse_token_weighted,
     lambda: pins.test_coarse_uniform_keys_average_block_values(*pins.RAGGED_COARSE)),
    ("coarse_head", _coarse_softmax_wrong_axis, lambda: pins.test_coarse_constant_values_pass_through()),
    ("gated_output", _gate_next_block, lambda: pins.test_coarse_and_gate_vs_loops(*pins.RAGGED_COARSE)),
]


@pytest.mark.parametrize("name,bad,pin", CASES, ids=[f"{c[0]}:{c[1].__name__}" for c in CASES])
def test_pin_catches_planted_mistake(monkeypatch, name, bad, pin):
    monkeypatch.setattr(vo, name, bad)
    with pytest.raises((AssertionError, ValueError, IndexError)):
        pin()
