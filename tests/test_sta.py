"""Sliding tile attention (STA) as PAB's spatial kind: the fp64 oracle pinned
to things other than itself (CPU), and the tcgen05 kernel against the oracle
(GPU).

The method (sgqg.cn summary of "Fast Video Generation with Sliding Tile
Attention", section "Sliding Tile Attention (STA)"): non-overlapping tiles,
each query tile attends to the key tiles inside a window around it, frame and
window sizes are whole numbers of tiles.  2-D reading per frame: tiles of
tile x tile tokens, a window of an odd number of tiles in each direction
centred on the query's tile and cut off at the frame edge.

Pins: torch's fp64 scaled_dot_product_attention with the window written as a
boolean mask (a library routine and a different formulation: dense scores
with masked entries, no gather), a window that covers the frame reducing to
full spatial attention, a one-tile window reducing to attention inside each
tile, Q = 0 giving the mean of V over the clipped window, keys outside a
tile's window leaving its output bit-for-bit unchanged, and argument checks.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

TILE = 16


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def window_mask(H, W, tile, win_h, win_w):
    """[N, N] bool: key m is inside query n's window (tile distance test)."""
    ys, xs = np.divmod(np.arange(H * W), W)
    ty, tx = ys // tile, xs // tile
    rh, rw = (win_h // tile - 1) // 2, (win_w // tile - 1) // 2
    return (np.abs(ty[:, None] - ty[None, :]) <= rh) & (np.abs(tx[:, None] - tx[None, :]) <= rw)


def sdpa_masked(q, k, v, heads, mask):
    """torch fp64 SDPA with a boolean mask; q/k/v [T, N, C]."""
    T, N, C = q.shape
    d = C // heads
    def split(x):
        return torch.from_numpy(x).view(T, N, heads, d).permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(split(q), split(k), split(v), attn_mask=torch.from_numpy(mask))
    return o.permute(0, 2, 1, 3).reshape(T, N, C).numpy()


@pytest.mark.parametrize("H,W,win_h,win_w", [
    (32, 48, 48, 48),   # 2 x 3 tiles, 3 x 3 window: clipped on every side
    (48, 32, 16, 48),   # one tile high, three wide
    (64, 64, 48, 80),   # interior tiles see the whole window
])
def test_sta_matches_masked_sdpa(oracle_mod, H, W, win_h, win_w):
    T, heads, d = 2, 2, 8
    q, k, v = (rnd((T, H * W, heads * d), s) for s in (1, 2, 3))
    got = oracle_mod.sta_attention(q, k, v, H, W, heads, TILE, win_h, win_w)
    want = sdpa_masked(q, k, v, heads, window_mask(H, W, TILE, win_h, win_w))
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_frame_covering_window_is_full_spatial_attention(oracle_mod):
    T, H, W, heads, d = 2, 32, 48, 2, 8
    q, k, v = (rnd((T, H * W, heads * d), s) for s in (4, 5, 6))
    got = oracle_mod.sta_attention(q, k, v, H, W, heads, TILE, 48, 80)  # reaches every tile
    assert np.allclose(got, oracle_mod.spatial_attention(q, k, v, heads), rtol=0, atol=1e-13)


def test_one_tile_window_is_attention_inside_each_tile(oracle_mod):
    T, H, W, heads, d = 1, 32, 32, 2, 8
    q, k, v = (rnd((T, H * W, heads * d), s) for s in (7, 8, 9))
    got = oracle_mod.sta_attention(q, k, v, H, W, heads, TILE, TILE, TILE)
    grid = lambda x: x.reshape(T, H, W, -1)
    for ty in range(H // TILE):
        for tx in range(W // TILE):
            sl = (slice(None), slice(ty * TILE, (ty + 1) * TILE), slice(tx * TILE, (tx + 1) * TILE))
            sub = [np.ascontiguousarray(grid(x)[sl]).reshape(T, TILE * TILE, -1) for x in (q, k, v)]
            want = oracle_mod.spatial_attention(*sub, heads)
            assert np.allclose(grid(got)[sl].reshape(T, TILE * TILE, -1), want, rtol=0, atol=1e-13)


def test_zero_queries_give_window_mean_of_v(oracle_mod):
    """Q = 0: every key in the window gets the same weight, so each output is
    the mean of V over the window's tokens (clipped at the frame edge)."""
    T, H, W, heads, d = 1, 48, 64, 2, 4
    v = rnd((T, H * W, heads * d), 10)
    k = rnd((T, H * W, heads * d), 11)
    q = np.zeros_like(v)
    got = oracle_mod.sta_attention(q, k, v, H, W, heads, TILE, 48, 48).reshape(T, H, W, -1)
    vg = v.reshape(T, H, W, -1)
    for ty in range(H // TILE):
        for tx in range(W // TILE):
            y0, y1 = max(ty - 1, 0) * TILE, min(ty + 2, H // TILE) * TILE
            x0, x1 = max(tx - 1, 0) * TILE, min(tx + 2, W // TILE) * TILE
            mean = vg[:, y0:y1, x0:x1].mean(axis=(1, 2))
            blk = got[:, ty * TILE:(ty + 1) * TILE, tx * TILE:(tx + 1) * TILE]
            assert np.allclose(blk, mean[:, None, None, :], rtol=0, atol=1e-13)


def test_keys_outside_the_window_do_not_matter(oracle_mod):
    """Changing keys and values outside tile (0, 0)'s 3 x 3 window leaves its
    outputs bit-identical; changing one key inside changes them."""
    T, H, W, heads, d = 1, 64, 64, 1, 8
    q, k, v = (rnd((T, H * W, heads * d), s) for s in (12, 13, 14))
    base = oracle_mod.sta_attention(q, k, v, H, W, heads, TILE, 48, 48).reshape(T, H, W, -1)
    inside = np.zeros((H, W), bool)
    inside[:2 * TILE, :2 * TILE] = True  # tiles (0..1, 0..1): the clipped window of tile (0, 0)
    k2, v2 = k.copy(), v.copy()
    out = ~inside.ravel()
    k2[:, out] += 3.0
    v2[:, out] -= 5.0
    moved = oracle_mod.sta_attention(q, k2, v2, H, W, heads, TILE, 48, 48).reshape(T, H, W, -1)
    assert np.array_equal(moved[:, :TILE, :TILE], base[:, :TILE, :TILE])
    assert not np.allclose(moved[:, 2 * TILE:, 2 * TILE:], base[:, 2 * TILE:, 2 * TILE:])
    k3 = k.copy()
    k3[:, (TILE + 3) * W + TILE + 5] += 4.0  # a token of tile (1, 1), inside the window
    hit = oracle_mod.sta_attention(q, k3, v, H, W, heads, TILE, 48, 48).reshape(T, H, W, -1)
    assert not np.array_equal(hit[:, :TILE, :TILE], base[:, :TILE, :TILE])


@pytest.mark.parametrize("H,W,win_h,win_w", [
    (30, 32, 48, 48),   # frame height not whole tiles
    (32, 32, 32, 48),   # even tile count: no centred window
    (32, 32, 40, 48),   # window not whole tiles
])
def test_bad_sta_arguments_are_rejected(oracle_mod, H, W, win_h, win_w):
    x = np.zeros((1, H * W, 8))
    with pytest.raises(ValueError):
        oracle_mod.sta_attention(x, x, x, H, W, 1, TILE, win_h, win_w)
