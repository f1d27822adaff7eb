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


# ------------------------------------------------------------------ GPU kernel vs oracle
def _randn(shape, seed, scale=1.0):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (scale * torch.randn(shape, generator=g)).to(torch.bfloat16).cuda()


@pytest.fixture(scope="module")
def pab():
    import step_reuse_b200
    assert torch.cuda.is_available()
    return step_reuse_b200


def _no_device_errors(pab):
    torch.cuda.synchronize()
    assert pab.device_errors(clear=True) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("T,H,W,heads,d,win_h,win_w", [
    (2, 32, 48, 2, 64, 48, 48),     # every tile's window clipped
    (1, 48, 64, 3, 72, 16, 48),     # d = 72 (V's padding column carries the row sums)
    (2, 64, 32, 2, 128, 48, 16),
    (1, 16, 16, 2, 32, 16, 16),     # one tile: four 64-key blocks
    (1, 48, 80, 2, 128, 48, 48),    # the 48 x 80 frame of the sliding-tile workload
    (1, 32, 32, 1, 8, 80, 80),      # window beyond the frame on every side
    (1, 80, 48, 2, 40, 48, 80),
    (1, 96, 96, 1, 64, 80, 80),     # interior tiles see 25 key tiles (100 blocks)
])
def test_sta_kernel_parity(pab, oracle_mod, T, H, W, heads, d, win_h, win_w):
    from parity import assert_attn_close, check_guards, guarded_empty, to_f64
    C = heads * d
    q, k, v = (_randn((T, H * W, C), s) for s in (21, 22, 23))
    base, out = guarded_empty((T, H * W, C), torch.bfloat16)
    pab.sta_attention(q, k, v, H, W, heads, TILE, win_h, win_w, out=out)
    want = oracle_mod.sta_attention(to_f64(q), to_f64(k), to_f64(v), H, W, heads, TILE, win_h, win_w)
    assert_attn_close(out, want, f"sta T={T} {H}x{W} h={heads} d={d} win {win_h}x{win_w}")
    check_guards(base)
    _no_device_errors(pab)


@pytest.mark.gpu
def test_sta_frame_covering_window_is_spatial_attention(pab, oracle_mod):
    from parity import assert_attn_close, to_f64
    T, H, W, heads, d = 2, 32, 64, 2, 64
    C = heads * d
    q, k, v = (_randn((T, H * W, C), s) for s in (24, 25, 26))
    out = pab.sta_attention(q, k, v, H, W, heads, TILE, 48, 112)
    want = oracle_mod.spatial_attention(to_f64(q), to_f64(k), to_f64(v), heads)
    assert_attn_close(out, want, "sta, window covering the frame")


@pytest.mark.gpu
@pytest.mark.parametrize("H,W,tile,win_h,win_w,code", [
    (30, 32, 16, 48, 48, "PAB_ERR_ARG"),          # frame not whole tiles
    (32, 32, 16, 32, 48, "PAB_ERR_ARG"),          # even tile count
    (32, 32, 16, 40, 48, "PAB_ERR_ARG"),          # window not whole tiles
    (32, 32, 8, 24, 24, "PAB_ERR_UNSUPPORTED"),   # another tile size
])
def test_sta_rejects_bad_geometry(pab, H, W, tile, win_h, win_w, code):
    x = _randn((1, H * W, 64), 27)
    with pytest.raises(pab.PabError) as e:
        pab.sta_attention(x, x, x, H, W, 1, tile, win_h, win_w)
    assert e.value.code == getattr(pab, code)


@pytest.mark.gpu
def test_plan_spatial_window_runs_sta_under_the_schedule(pab):
    """A plan with a spatial window computes sliding tile attention at its
    computing steps (bit-identical to the stateless call) and serves the
    cached slot at its broadcast steps."""
    T, H, W, heads, d, steps = 2, 32, 48, 2, 64, 10
    C = heads * d
    plan = pab.Plan(T, H, W, heads, d, 16, steps, (2, 3, 4), dtype=torch.bfloat16)
    try:
        plan.set_spatial_window(TILE, 48, 48)
        last = None
        for i in range(steps):
            q, k, v = (_randn((T, H * W, C), 100 * i + s) for s in (1, 2, 3))
            got = plan.attention("spatial", i, q, k, v)
            if plan.is_compute("spatial", i):
                want = pab.sta_attention(q, k, v, H, W, heads, TILE, 48, 48)
                assert torch.equal(got, want), i
            else:
                assert got.data_ptr() == last.data_ptr() and torch.equal(got, last_val), i
            last, last_val = got, got.clone()
        plan.reset()
        plan.set_spatial_window(TILE, 0, 0)  # back to full attention
        q, k, v = (_randn((T, H * W, C), s) for s in (7, 8, 9))
        assert torch.equal(plan.attention("spatial", 0, q, k, v), pab.spatial_attention(q, k, v, heads))
        with pytest.raises(pab.PabError):
            plan.set_spatial_window(TILE, 32, 48)
    finally:
        plan.close()
    _no_device_errors(pab)


@pytest.mark.gpu
def test_sta_full_size_sampled(pab, oracle_mod):
    """The sliding-tile workload at full size (24 frames of 48 x 80 tokens,
    24 heads of d = 128, 3 x 3-tile windows) in the launch the benchmark
    times; two frames (all heads) against the oracle."""
    from parity import assert_attn_close, to_f64
    T, H, W, heads, d = 24, 48, 80, 24, 128
    C = heads * d
    q, k, v = (_randn((T, H * W, C), s) for s in (31, 32, 33))
    out = pab.sta_attention(q, k, v, H, W, heads, TILE, 48, 48)
    torch.cuda.synchronize()
    for fr in (0, T - 1):
        want = oracle_mod.sta_attention(to_f64(q[fr:fr + 1]), to_f64(k[fr:fr + 1]), to_f64(v[fr:fr + 1]),
                                        H, W, heads, TILE, 48, 48)
        assert_attn_close(out[fr:fr + 1], want, f"sta full size, frame {fr}")
    _no_device_errors(pab)


@pytest.mark.parametrize("H,W,win_h,win_w", [(48, 80, 48, 48), (32, 48, 16, 80), (64, 96, 80, 48), (16, 16, 48, 48)])
def test_bench_window_pair_count_is_the_mask_count(H, W, win_h, win_w):
    """The benchmark's algorithmic flops count query-key pairs in closed form;
    they equal the pairs the window mask admits."""
    import dataclasses

    import bench
    import synth
    w = dataclasses.replace(synth.WORKLOADS["sta_48x80"], H=H, W=W, spatial_window=(TILE, win_h, win_w))
    assert bench.sta_pairs(w) == int(window_mask(H, W, TILE, win_h, win_w).sum())
