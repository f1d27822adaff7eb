"""Pins for the fp64 oracle, against things other than itself.

Attention (the textbook softmax(QK^T/sqrt(d))V of each PAB attention kind):
  torch's fp64 scaled_dot_product_attention (a library routine), a pure-Python
  brute force on tiny inputs, a hand-worked two-key example, rows of the
  softmax summing to one, Q = 0 giving mean(V), a dominant key giving its V
  row, L = 1 giving V, key-permutation invariance, head isolation.
Schedule (PAB report, "Implementation" / Fig. 2): hand-worked counts, the
  closed form, a per-step rule, structural properties.
MSE (Fig. 1 diagnostic): numpy, MSE(a, a) = 0, exact MSE(a, a + c) = c^2.
Layout: torch.permute and the round trip.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def sdpa_heads(q, k, v, heads):
    """torch fp64 SDPA; q: [B, Lq, C], k/v: [B, Lk, C] -> [B, Lq, C]."""
    B, Lq, C = q.shape
    Lk = k.shape[1]
    d = C // heads
    tq = torch.from_numpy(q).reshape(B, Lq, heads, d).transpose(1, 2)
    tk = torch.from_numpy(k).reshape(B, Lk, heads, d).transpose(1, 2)
    tv = torch.from_numpy(v).reshape(B, Lk, heads, d).transpose(1, 2)
    o = F.scaled_dot_product_attention(tq, tk, tv)
    return o.transpose(1, 2).reshape(B, Lq, C).numpy()


# ----------------------------------------------------------------- attention
@pytest.mark.parametrize("T,N,heads,d", [(3, 17, 2, 8), (2, 40, 3, 24), (1, 5, 1, 72)])
def test_spatial_matches_torch_sdpa(oracle_mod, T, N, heads, d):
    C = heads * d
    q, k, v = (rnd((T, N, C), s) for s in (1, 2, 3))
    got = oracle_mod.spatial_attention(q, k, v, heads)
    ref = sdpa_heads(q, k, v, heads)  # frames are the batch
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("N,T,heads,d", [(7, 16, 2, 8), (5, 24, 3, 16), (3, 64, 1, 64)])
def test_temporal_matches_torch_sdpa(oracle_mod, N, T, heads, d):
    C = heads * d
    q, k, v = (rnd((N, T, C), s) for s in (4, 5, 6))
    got = oracle_mod.temporal_attention(q, k, v, heads)
    ref = sdpa_heads(q, k, v, heads)  # positions are the batch
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("R,Lt,heads,d", [(33, 16, 2, 8), (100, 120, 4, 12), (9, 1, 2, 4)])
def test_cross_matches_torch_sdpa(oracle_mod, R, Lt, heads, d):
    C = heads * d
    q = rnd((R, C), 7)
    kt, vt = rnd((Lt, C), 8), rnd((Lt, C), 9)
    got = oracle_mod.cross_attention(q, kt, vt, heads)
    ref = sdpa_heads(q[None], kt[None], vt[None], heads)[0]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_spatial_layout_indices_by_torch_views(oracle_mod):
    """The spatial oracle on [T, N, C] equals the temporal oracle on the permuted
    tensor's permutation back -- i.e. frames and positions are not swapped."""
    T, N, heads, d = 4, 6, 2, 4
    C = heads * d
    q, k, v = (rnd((T, N, C), s) for s in (11, 12, 13))
    sp = oracle_mod.spatial_attention(q, k, v, heads)
    # the temporal oracle treats axis 0 as the batch axis: feed [T, N, C] as-is
    tm = oracle_mod.temporal_attention(q, k, v, heads)
    np.testing.assert_allclose(sp, tm, rtol=1e-13, atol=1e-13)
    # and temporal attention on the spatial view differs from spatial attention
    tm2 = oracle_mod.temporal_attention(np.transpose(q, (1, 0, 2)), np.transpose(k, (1, 0, 2)),
                                        np.transpose(v, (1, 0, 2)), heads)
    assert np.abs(np.transpose(tm2, (1, 0, 2)) - sp).max() > 1e-3


def test_brute_force_tiny(oracle_mod):
    """Pure-Python loops, scores and weights written out per element."""
    T, N, heads, d = 2, 3, 2, 3
    C = heads * d
    q, k, v = (rnd((T, N, C), s) for s in (21, 22, 23))
    got = oracle_mod.spatial_attention(q, k, v, heads)
    for t in range(T):
        for h in range(heads):
            cs = slice(h * d, (h + 1) * d)
            for n in range(N):
                scores = [sum(q[t, n, cs][c] * k[t, m, cs][c] for c in range(d)) / math.sqrt(d)
                          for m in range(N)]
                w = [math.exp(s) for s in scores]  # small inputs: no overflow
                tot = sum(w)
                for c in range(d):
                    want = sum(w[m] * v[t, m, cs][c] for m in range(N)) / tot
                    assert abs(got[t, n, h * d + c] - want) < 1e-13


def test_two_key_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "attention_two_keys.json")))
    d = g["d"]
    q = np.array(g["q"], float).reshape(1, 1, d)
    k = np.array(g["k"], float).reshape(1, 2, d)
    v = np.array(g["v"], float).reshape(1, 2, d)
    got = oracle_mod.cross_attention(q[0], k[0], v[0], heads=1)[0]
    np.testing.assert_allclose(got, g["out"], rtol=0, atol=1e-15)
    assert abs(g["p0"] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16


def test_rows_sum_to_one(oracle_mod):
    """With V = identity the output rows are the softmax weights themselves."""
    Lk, d = 24, 32
    q = rnd((50, d), 31, scale=2.0)
    kt = rnd((Lk, d), 32, scale=2.0)
    vt = np.zeros((Lk, d))
    vt[np.arange(Lk), np.arange(Lk)] = 1.0
    p = oracle_mod.cross_attention(q, kt, vt, heads=1)
    assert (p[:, :Lk] >= 0).all() and (p[:, Lk:] == 0).all()
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    # the weights are ordered like the scores
    s = q @ kt.T
    assert (np.argmax(p[:, :Lk], axis=1) == np.argmax(s, axis=1)).all()


def test_q_zero_gives_mean_v(oracle_mod):
    T, N, heads, d = 2, 9, 3, 8
    C = heads * d
    q = np.zeros((T, N, C))
    k, v = rnd((T, N, C), 41), rnd((T, N, C), 42)
    out = oracle_mod.spatial_attention(q, k, v, heads)
    want = np.broadcast_to(v.mean(axis=1, keepdims=True), out.shape)
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-15)


def test_one_hot_key_gives_its_value(oracle_mod):
    """One key aligned with the query and far above the rest: output -> V_j, with
    error <= (L - 1) * exp(-gap) * max|V| where gap is the score margin."""
    rng = np.random.default_rng(51)
    L, d = 40, 16
    q = rng.standard_normal(d)
    k = rng.standard_normal((L, d)) * 0.1
    j = 17
    k[j] = 20.0 * q / np.linalg.norm(q)
    v = rng.standard_normal((L, d))
    out = oracle_mod.cross_attention(q[None], k, v, heads=1)[0]
    s = k @ q / math.sqrt(d)
    gap = s[j] - np.max(np.delete(s, j))
    bound = (L - 1) * math.exp(-gap) * np.abs(v).max() * 2
    assert gap > 10
    assert np.abs(out - v[j]).max() <= bound


def test_single_key_gives_v(oracle_mod):
    N, T, heads, d = 5, 1, 2, 8
    C = heads * d
    q, k, v = (rnd((N, T, C), s) for s in (61, 62, 63))
    out = oracle_mod.temporal_attention(q, k, v, heads)
    np.testing.assert_array_equal(out, v)


def test_key_permutation_invariance(oracle_mod):
    R, Lt, heads, d = 20, 30, 2, 8
    C = heads * d
    q, kt, vt = rnd((R, C), 71), rnd((Lt, C), 72), rnd((Lt, C), 73)
    perm = np.random.default_rng(74).permutation(Lt)
    a = oracle_mod.cross_attention(q, kt, vt, heads)
    b = oracle_mod.cross_attention(q, kt[perm], vt[perm], heads)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)
    qperm = np.random.default_rng(75).permutation(R)
    c = oracle_mod.cross_attention(q[qperm], kt, vt, heads)
    np.testing.assert_allclose(c, a[qperm], rtol=0, atol=0)


def test_head_isolation(oracle_mod):
    """Head h's output depends only on channels [h*d, (h+1)*d)."""
    T, N, heads, d = 2, 7, 3, 4
    C = heads * d
    q, k, v = (rnd((T, N, C), s) for s in (81, 82, 83))
    a = oracle_mod.spatial_attention(q, k, v, heads)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for x in (q2, k2, v2):
        x[..., d:] += rnd(x[..., d:].shape, 84)  # perturb heads 1..
    b = oracle_mod.spatial_attention(q2, k2, v2, heads)
    np.testing.assert_array_equal(a[..., :d], b[..., :d])
    assert np.abs(a[..., d:] - b[..., d:]).max() > 1e-3


def test_scale_is_inverse_sqrt_d(oracle_mod):
    """Scaling q by sqrt(d) equals unit-scale softmax(q k^T) v (torch, fp64)."""
    R, Lt, d = 6, 9, 16
    q, kt, vt = rnd((R, d), 91), rnd((Lt, d), 92), rnd((Lt, d), 93)
    out = oracle_mod.cross_attention(q, kt, vt, heads=1)
    w = torch.softmax(torch.from_numpy(q) @ torch.from_numpy(kt).T / 4.0, dim=-1)
    np.testing.assert_allclose(out, (w @ torch.from_numpy(vt)).numpy(), rtol=1e-12, atol=1e-13)


def test_large_scores_stable(oracle_mod):
    """Scores far beyond exp's range still give a finite convex combination."""
    R, Lt, d = 4, 5, 8
    q, kt, vt = rnd((R, d), 94, 60.0), rnd((Lt, d), 95, 60.0), rnd((Lt, d), 96)
    out = oracle_mod.cross_attention(q, kt, vt, heads=1)
    assert np.isfinite(out).all()
    assert (out <= vt.max(axis=0) + 1e-12).all() and (out >= vt.min(axis=0) - 1e-12).all()


# ----------------------------------------------------------------- schedule
def closed_form_counts(S, r, edge_pct=15):
    e = -(-edge_pct * S // 100)
    M = max(S - 2 * e, 0)
    computes = (S - M) + (-(-M // r))
    return computes, S - computes


def test_schedule_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "pab_schedule_counts.json")))
    for row in g["rows"]:
        S, r = row["S"], row["r"]
        assert oracle_mod.edge_steps(S) == row["lo"]
        assert S - oracle_mod.edge_steps(S) == row["hi"]
        comp, src = oracle_mod.schedule(S, r)
        assert int(comp.sum()) == row["computes"], row
        assert S - int(comp.sum()) == row["hits"], row
        if "compute_steps" in row:
            assert list(np.nonzero(comp)[0]) == row["compute_steps"]


def test_schedule_closed_form_exhaustive(oracle_mod):
    for S in range(0, 201):
        for r in range(1, 13):
            comp, src = oracle_mod.schedule(S, r)
            assert (int(comp.sum()), S - int(comp.sum())) == closed_form_counts(S, r), (S, r)
            e = -(-15 * S // 100)
            lo, hi = e, S - e
            for i in range(S):
                rule = i < lo or i >= hi or (i - lo) % r == 0
                assert bool(comp[i]) == rule, (S, r, i)


def test_schedule_structure(oracle_mod):
    for S in (1, 2, 7, 10, 30, 50, 97):
        for r in (1, 2, 3, 6, 9):
            comp, src = oracle_mod.schedule(S, r)
            e = oracle_mod.edge_steps(S)
            for i in range(S):
                if i < e or i >= S - e:
                    assert comp[i] == 1
                if comp[i]:
                    assert src[i] == i
                else:
                    # served by the latest compute, at most r - 1 steps back,
                    # never from an edge step
                    j = src[i]
                    assert comp[j] == 1 and 0 < i - j < r and j >= e
                    assert not comp[j + 1:i + 1].any()
            if r == 1:
                assert comp.all()


def test_schedule_edge_pct_param(oracle_mod):
    assert oracle_mod.edge_steps(30, 0) == 0
    assert oracle_mod.edge_steps(30, 50) == 15
    comp, _ = oracle_mod.schedule(30, 4, edge_pct=0)
    assert list(np.nonzero(comp)[0]) == list(range(0, 30, 4))
    with pytest.raises(ValueError):
        oracle_mod.schedule(30, 0)


# ----------------------------------------------------------------- MSE
def test_mse_matches_numpy(oracle_mod):
    a, b = rnd(10007, 101), rnd(10007, 102)
    assert oracle_mod.mse(a, b) == pytest.approx(float(np.mean((a - b) ** 2)), rel=1e-14)


def test_mse_exact_cases(oracle_mod):
    rng = np.random.default_rng(103)
    a = rng.integers(-8192, 8192, size=4096) / 1024.0  # exact binary fractions
    assert oracle_mod.mse(a, a) == 0.0
    for c in (0.25, 2.0, 1.0 / 64):
        assert oracle_mod.mse(a, a + c) == c * c
        assert oracle_mod.mse(a + c, a) == c * c
    assert oracle_mod.mse(np.zeros(0), np.zeros(0)) == 0.0


# ----------------------------------------------------------------- layout
def test_layout_matches_torch_permute(oracle_mod):
    T, N, C = 5, 7, 24
    x = (np.arange(T * N * C, dtype=np.int32).reshape(T, N, C)).astype(np.uint16)
    y = oracle_mod.layout(x, to_temporal=True)
    np.testing.assert_array_equal(y, torch.from_numpy(x.astype(np.int32)).permute(1, 0, 2).numpy())
    z = oracle_mod.layout(y, to_temporal=False)
    np.testing.assert_array_equal(z, x)
