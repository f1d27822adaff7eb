"""Draft attention as PAB's spatial kind: the fp64 oracle pinned to things
other than itself (CPU), and the library's select + region-sparse kernels
against it (GPU).

The method (crisp3r.com article on "Draft Attention", steps 1-4): average-
pool the latent frame into a low-resolution sketch of the queries and keys,
rank regions with the draft attention map of the sketch, keep the best
regions as a structured sparse mask of the full-resolution attention, group
tokens so the kept blocks are contiguous.  Readings: 16 x 16-token regions
per frame, per query region the `keep` key regions with the highest draft
scores (ties to the lower index), listed in ascending index.

Pins: the sketch and the ranking recomputed with numpy (reshape-mean pooling,
einsum scores, a stable lexsort), ties resolved to the lower index, a planted
key region that every query region must keep, keep = R reducing to full
spatial attention, the attention under a given selection against torch's
fp64 scaled_dot_product_attention with the selection as a boolean mask, a
selection of each region's own tokens reducing to attention inside the
region, and argument checks.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

REGION = 16


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def np_sketch(x, H, W, heads):
    """[T, H*W, C] -> [T, heads, R, d]: the mean over each 16 x 16 region."""
    T, N, C = x.shape
    d = C // heads
    g = x.reshape(T, H // REGION, REGION, W // REGION, REGION, heads, d).mean(axis=(2, 4))
    return g.reshape(T, -1, heads, d).transpose(0, 2, 1, 3)


def np_select(q, k, H, W, heads, keep):
    qb, kb = np_sketch(q, H, W, heads), np_sketch(k, H, W, heads)
    d = qb.shape[-1]
    s = np.einsum("thid,thjd->thij", qb, kb) / np.sqrt(d)
    T, h, R, _ = s.shape
    out = np.zeros((T, h, R, keep), np.int32)
    for t in range(T):
        for hh in range(h):
            for i in range(R):
                order = np.lexsort((np.arange(R), -s[t, hh, i]))  # score desc, index asc
                out[t, hh, i] = np.sort(order[:keep])
    return out


def selection_mask(sel, H, W):
    """[T, heads, N, N] bool from a region selection [T, heads, R, keep]."""
    rw = W // REGION
    ys, xs = np.divmod(np.arange(H * W), W)
    reg = (ys // REGION) * rw + xs // REGION
    T, h, R, keep = sel.shape
    allowed = np.zeros((T, h, R, R), bool)
    for t in range(T):
        for hh in range(h):
            for i in range(R):
                allowed[t, hh, i, sel[t, hh, i]] = True
    return allowed[:, :, reg][:, :, :, reg]


def sdpa_masked(q, k, v, heads, mask):
    T, N, C = q.shape
    d = C // heads
    def split(x):
        return torch.from_numpy(x).view(T, N, heads, d).permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(split(q), split(k), split(v), attn_mask=torch.from_numpy(mask))
    return o.permute(0, 2, 1, 3).reshape(T, N, C).numpy()


@pytest.mark.parametrize("H,W,heads,keep", [(32, 48, 2, 2), (48, 80, 3, 4), (64, 64, 1, 16)])
def test_selection_matches_numpy_sketch_and_ranking(oracle_mod, H, W, heads, keep):
    T, d = 2, 8
    q, k = rnd((T, H * W, heads * d), 1), rnd((T, H * W, heads * d), 2)
    got = oracle_mod.draft_select(q, k, H, W, heads, REGION, keep)
    assert np.array_equal(got, np_select(q, k, H, W, heads, keep))


def test_ties_go_to_the_lower_region_index(oracle_mod):
    """k = 0: every draft score is 0, so each row keeps regions 0..keep-1."""
    T, H, W, heads, d, keep = 1, 32, 64, 2, 8, 3
    q = rnd((T, H * W, heads * d), 3)
    sel = oracle_mod.draft_select(q, np.zeros_like(q), H, W, heads, REGION, keep)
    assert (sel == np.arange(keep)).all()


def test_a_planted_region_is_kept_by_every_query_region(oracle_mod):
    """Queries share a direction u; key region 5's tokens point along it far
    more than any other region, so every row keeps region 5."""
    T, H, W, heads, d, keep = 1, 48, 64, 1, 16, 2
    u = rnd((d,), 4)
    q = rnd((T, H * W, d), 5, 0.3) + u
    k = rnd((T, H * W, d), 6)
    rw = W // REGION
    ry, rx = divmod(5, rw)
    grid = k.reshape(T, H, W, d)
    grid[:, ry * REGION:(ry + 1) * REGION, rx * REGION:(rx + 1) * REGION] += 4.0 * u
    sel = oracle_mod.draft_select(q, grid.reshape(T, H * W, d), H, W, heads, REGION, keep)
    assert (sel == 5).any(axis=-1).all()


def test_keeping_every_region_is_full_spatial_attention(oracle_mod):
    T, H, W, heads, d = 2, 32, 48, 2, 8
    q, k, v = (rnd((T, H * W, heads * d), s) for s in (7, 8, 9))
    R = (H // REGION) * (W // REGION)
    got = oracle_mod.draft_attention(q, k, v, H, W, heads, REGION, R)
    assert np.allclose(got, oracle_mod.spatial_attention(q, k, v, heads), rtol=0, atol=1e-13)


@pytest.mark.parametrize("keep", [1, 3, 5])
def test_attention_under_a_selection_matches_masked_sdpa(oracle_mod, keep):
    T, H, W, heads, d = 2, 48, 48, 2, 8
    q, k, v = (rnd((T, H * W, heads * d), s) for s in (10, 11, 12))
    R = (H // REGION) * (W // REGION)
    rng = np.random.default_rng(13)
    sel = np.stack([np.stack([np.stack([np.sort(rng.permutation(R)[:keep]) for _ in range(R)])
                              for _ in range(heads)]) for _ in range(T)]).astype(np.int32)
    got = oracle_mod.region_sparse_attention(q, k, v, H, W, heads, REGION, sel)
    want = np.stack([sdpa_masked(q[t:t + 1], k[t:t + 1], v[t:t + 1], heads,
                                 selection_mask(sel[t:t + 1], H, W)[0])[0] for t in range(T)])
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_own_region_selection_is_attention_inside_each_region(oracle_mod):
    T, H, W, heads, d = 1, 32, 32, 2, 8
    q, k, v = (rnd((T, H * W, heads * d), s) for s in (14, 15, 16))
    R = (H // REGION) * (W // REGION)
    sel = np.broadcast_to(np.arange(R, dtype=np.int32)[None, None, :, None], (T, heads, R, 1))
    got = oracle_mod.region_sparse_attention(q, k, v, H, W, heads, REGION, sel)
    grid = lambda x: x.reshape(T, H, W, -1)
    for ry in range(H // REGION):
        for rx in range(W // REGION):
            sl = (slice(None), slice(ry * REGION, (ry + 1) * REGION), slice(rx * REGION, (rx + 1) * REGION))
            sub = [np.ascontiguousarray(grid(x)[sl]).reshape(T, REGION * REGION, -1) for x in (q, k, v)]
            want = oracle_mod.spatial_attention(*sub, heads)
            assert np.allclose(grid(got)[sl].reshape(T, REGION * REGION, -1), want, rtol=0, atol=1e-13)


@pytest.mark.parametrize("H,W,keep", [(30, 32, 1), (32, 32, 0), (32, 32, 5)])
def test_bad_draft_arguments_are_rejected(oracle_mod, H, W, keep):
    x = np.zeros((1, H * W, 8))
    with pytest.raises(ValueError):
        oracle_mod.draft_select(x, x, H, W, 1, REGION, keep)


# ------------------------------------------------------------------ GPU kernels vs oracle
# Draft scores on the GPU are fp32 (means of 256 bf16 values, then a d-term
# dot product); the oracle's are fp64.  Both are far below 1e-6 apart for
# these inputs (scores ~4e-3, fp32 rounding ~1e-9), so a selection is judged
# valid when no dropped region beats a kept one by more than SCORE_EPS, and
# must equal the oracle's wherever the oracle's ranking gap exceeds it.
SCORE_EPS = 1e-6


def _randn(shape, seed, scale=1.0):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (scale * torch.randn(shape, generator=g)).to(torch.bfloat16).cuda()


@pytest.fixture(scope="module")
def pab():
    import step_reuse_b200
    assert torch.cuda.is_available()
    return step_reuse_b200


def _f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check_selection(sel_gpu, q, k, H, W, heads, keep, oracle_mod):
    qb, kb = np_sketch(q, H, W, heads), np_sketch(k, H, W, heads)
    s = np.einsum("thid,thjd->thij", qb, kb) / np.sqrt(qb.shape[-1])
    want = oracle_mod.draft_select(q, k, H, W, heads, REGION, keep)
    T, h, R, _ = s.shape
    for t in range(T):
        for hh in range(h):
            for i in range(R):
                got = sel_gpu[t, hh, i]
                assert (np.diff(got) > 0).all() and got.min() >= 0 and got.max() < R, (t, hh, i, got)
                kept = np.zeros(R, bool)
                kept[got] = True
                if keep < R:
                    assert s[t, hh, i, kept].min() >= s[t, hh, i, ~kept].max() - SCORE_EPS, (t, hh, i)
                    srt = np.sort(s[t, hh, i])[::-1]
                    if srt[keep - 1] - srt[keep] > SCORE_EPS:
                        assert np.array_equal(got, want[t, hh, i]), (t, hh, i)


@pytest.mark.gpu
@pytest.mark.parametrize("T,H,W,heads,d,keep", [
    (2, 32, 48, 2, 64, 2),
    (1, 48, 80, 3, 128, 4),    # the 48 x 80 frame of the sliding-tile workload, 75% sparsity
    (1, 64, 64, 2, 72, 3),     # d = 72: V's padding column carries the row sums
    (2, 16, 32, 1, 32, 1),
    (1, 48, 48, 2, 40, 9),     # keep every region
    (1, 96, 96, 1, 64, 6),
])
def test_draft_kernels_parity(pab, oracle_mod, T, H, W, heads, d, keep):
    from parity import assert_attn_close, check_guards, guarded_empty
    C = heads * d
    q, k, v = (_randn((T, H * W, C), s) for s in (31, 32, 33))
    sel = pab.draft_select(q, k, H, W, heads, keep)
    torch.cuda.synchronize()
    sel_np = sel.cpu().numpy()
    check_selection(sel_np, _f64(q), _f64(k), H, W, heads, keep, oracle_mod)
    base, out = guarded_empty((T, H * W, C), torch.bfloat16)
    pab.region_sparse_attention(q, k, v, H, W, heads, sel, out=out)
    want = oracle_mod.region_sparse_attention(_f64(q), _f64(k), _f64(v), H, W, heads, REGION, sel_np)
    assert_attn_close(out, want, f"draft T={T} {H}x{W} h={heads} d={d} keep={keep}")
    check_guards(base)
    _no_device_errors(pab)


def _no_device_errors(pab):
    torch.cuda.synchronize()
    assert pab.device_errors(clear=True) == 0


@pytest.mark.gpu
def test_region_sparse_attention_under_a_given_selection(pab, oracle_mod):
    """A caller's selection (random, unsorted, one region repeated across
    rows) runs exactly as listed."""
    from parity import assert_attn_close
    T, H, W, heads, d, keep = 2, 48, 64, 2, 64, 5
    C = heads * d
    R = (H // REGION) * (W // REGION)
    q, k, v = (_randn((T, H * W, C), s) for s in (34, 35, 36))
    rng = np.random.default_rng(37)
    sel = np.stack([np.stack([np.stack([rng.permutation(R)[:keep] for _ in range(R)]) for _ in range(heads)])
                    for _ in range(T)]).astype(np.int32)
    out = pab.region_sparse_attention(q, k, v, H, W, heads, torch.from_numpy(sel).cuda())
    want = oracle_mod.region_sparse_attention(_f64(q), _f64(k), _f64(v), H, W, heads, REGION, sel)
    assert_attn_close(out, want, "region-sparse, given selection")
    _no_device_errors(pab)


@pytest.mark.gpu
def test_out_of_range_region_index_is_flagged_not_faulted(pab):
    T, H, W, heads, d, keep = 1, 32, 32, 1, 64, 2
    q = _randn((T, H * W, heads * d), 38)
    sel = torch.tensor([[[[0, 1], [1, 99], [2, 3], [-5, 0]]]], dtype=torch.int32, device="cuda")
    pab.region_sparse_attention(q, q, q, H, W, heads, sel)
    torch.cuda.synchronize()
    assert pab.device_errors(clear=True) & 4
    assert pab.device_errors(clear=True) == 0


@pytest.mark.gpu
def test_keeping_every_region_matches_spatial_attention(pab, oracle_mod):
    from parity import assert_attn_close
    T, H, W, heads, d = 1, 48, 64, 2, 128
    C = heads * d
    q, k, v = (_randn((T, H * W, C), s) for s in (39, 40, 41))
    out = pab.draft_attention(q, k, v, H, W, heads, (H // REGION) * (W // REGION))
    want = oracle_mod.spatial_attention(_f64(q), _f64(k), _f64(v), heads)
    assert_attn_close(out, want, "draft, keep = R")


@pytest.mark.gpu
@pytest.mark.parametrize("H,W,region,keep,code", [
    (30, 32, 16, 1, "PAB_ERR_ARG"),
    (32, 32, 16, 0, "PAB_ERR_ARG"),
    (32, 32, 16, 5, "PAB_ERR_ARG"),
    (32, 32, 8, 2, "PAB_ERR_UNSUPPORTED"),
])
def test_draft_rejects_bad_arguments(pab, H, W, region, keep, code):
    x = _randn((1, H * W, 64), 42)
    with pytest.raises(pab.PabError) as e:
        pab.draft_select(x, x, H, W, 1, keep, region, sel=torch.empty(64, dtype=torch.int32, device="cuda"),
                         workspace=torch.empty(1 << 16, dtype=torch.uint8, device="cuda"))
    assert e.value.code == getattr(pab, code)


@pytest.mark.gpu
def test_plan_spatial_draft_runs_under_the_schedule(pab):
    T, H, W, heads, d, steps, keep = 2, 32, 48, 2, 64, 10, 2
    C = heads * d
    plan = pab.Plan(T, H, W, heads, d, 16, steps, (2, 3, 4), dtype=torch.bfloat16)
    try:
        plan.set_spatial_draft(REGION, keep)
        last = last_val = None
        for i in range(steps):
            q, k, v = (_randn((T, H * W, C), 200 * i + s) for s in (1, 2, 3))
            got = plan.attention("spatial", i, q, k, v)
            if plan.is_compute("spatial", i):
                assert torch.equal(got, pab.draft_attention(q, k, v, H, W, heads, keep)), i
            else:
                assert got.data_ptr() == last.data_ptr() and torch.equal(got, last_val), i
            last, last_val = got, got.clone()
        plan.reset()
        plan.set_spatial_window(REGION, 48, 48)  # replaces the draft setting
        q, k, v = (_randn((T, H * W, C), s) for s in (4, 5, 6))
        assert torch.equal(plan.attention("spatial", 0, q, k, v),
                           pab.sta_attention(q, k, v, H, W, heads, REGION, 48, 48))
    finally:
        plan.close()
    _no_device_errors(pab)


@pytest.mark.gpu
def test_draft_full_size_sampled(pab, oracle_mod):
    """The 48 x 80-frame workload at full size (24 frames, 24 heads of
    d = 128), 75% sparsity (keep 4 of 15 regions) in the launches the
    benchmark times; the selection of every frame checked, two frames' output
    against the oracle under that selection."""
    from parity import assert_attn_close
    T, H, W, heads, d, keep = 24, 48, 80, 24, 128, 4
    C = heads * d
    q, k, v = (_randn((T, H * W, C), s) for s in (43, 44, 45))
    sel = pab.draft_select(q, k, H, W, heads, keep)
    out = pab.region_sparse_attention(q, k, v, H, W, heads, sel)
    torch.cuda.synchronize()
    sel_np = sel.cpu().numpy()
    for fr in (0, T - 1):
        qf, kf, vf = (_f64(x[fr:fr + 1]) for x in (q, k, v))
        check_selection(sel_np[fr:fr + 1], qf, kf, H, W, heads, keep, oracle_mod)
        want = oracle_mod.region_sparse_attention(qf, kf, vf, H, W, heads, REGION, sel_np[fr:fr + 1])
        assert_attn_close(out[fr:fr + 1], want, f"draft full size, frame {fr}")
    _no_device_errors(pab)
