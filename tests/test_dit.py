"""The synthetic DiT block around PAB: the fp64 oracle pinned to closed forms
and invariants (CPU), and the GPU block (library attention + cuBLAS
projections) against the oracle over whole sampling runs (GPU).

The block (PAB report, "Implementation": the three attention kinds inside a
video DiT block, each kind's output broadcast over its range):
    x <- x + A_s(LN(x)); x <- x + A_t(LN(x)); x <- x + A_c(LN(x), text);
    x <- x + GELU(LN(x) W1) W2,  A_kind(h) = Attn_kind(h Wq, h Wk, h Wv) Wo.
"""
import math

import numpy as np
import pytest
import torch

import synth

C_TINY = 16


def rand_weights(C, seed=0, scale=1.0):
    rng = np.random.default_rng(seed)
    w = {f"{k}.{n}": scale * rng.standard_normal((C, C)) / np.sqrt(C)
         for k in ("spatial", "temporal", "cross") for n in ("wq", "wk", "wv", "wo")}
    w["mlp.w1"] = rng.standard_normal((C, 4 * C)) / np.sqrt(C)
    w["mlp.w2"] = rng.standard_normal((4 * C, C)) / np.sqrt(4 * C)
    return w


# ------------------------------------------------------------------ oracle pins (CPU)
def test_layer_norm_hand_example():
    from oracle import dit
    got = dit.layer_norm(np.array([[1.0, 2.0, 3.0]]))
    s = math.sqrt(2.0 / 3.0 + dit.LN_EPS)  # mean 2, population variance 2/3
    assert np.allclose(got, [[-1 / s, 0.0, 1 / s]], rtol=0, atol=1e-15)


def test_layer_norm_rows_are_standardised():
    from oracle import dit
    x = np.random.default_rng(1).standard_normal((7, 33)) * 5 + 3
    y = dit.layer_norm(x)
    assert np.allclose(y.mean(axis=-1), 0, atol=1e-12)
    assert np.allclose((y ** 2).mean(axis=-1), 1, atol=1e-5)


def test_gelu_tanh_against_erf_gelu():
    """The tanh form stays within 1e-3 of x * Phi(x) (Phi via math.erf)."""
    from oracle import dit
    xs = np.linspace(-8, 8, 2001)
    exact = np.array([0.5 * x * (1 + math.erf(x / math.sqrt(2))) for x in xs])
    got = dit.gelu_tanh(xs)
    assert np.max(np.abs(got - exact)) < 1e-3
    assert dit.gelu_tanh(np.array([0.0]))[0] == 0.0


def test_identity_projections_give_attention_of_the_norm():
    """Wq = Wk = Wv = Wo = I: the module is the attention of LN(x)."""
    import oracle
    from oracle import dit
    rng = np.random.default_rng(2)
    T, N, heads = 3, 10, 2
    x = rng.standard_normal((T, N, C_TINY))
    eye = np.eye(C_TINY)
    w = {f"spatial.{n}": eye for n in ("wq", "wk", "wv", "wo")}
    h = dit.layer_norm(x)
    want = oracle.spatial_attention(h, h, h, heads)
    assert np.allclose(dit.attention_module("spatial", x, None, w, heads), want, atol=1e-12)


def test_temporal_module_single_frame_is_value_path():
    """T = 1: softmax over one key is 1, so A_t(h) = LN(x) Wv Wo."""
    from oracle import dit
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 9, C_TINY))
    w = rand_weights(C_TINY, 3)
    want = dit.layer_norm(x) @ w["temporal.wv"] @ w["temporal.wo"]
    assert np.allclose(dit.attention_module("temporal", x, None, w, 2), want, atol=1e-12)


def test_cross_module_single_text_token_is_value_row():
    """One text token: every video token gets (y Wv) Wo."""
    from oracle import dit
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 5, C_TINY))
    y = rng.standard_normal((1, C_TINY))
    w = rand_weights(C_TINY, 4)
    want = np.broadcast_to(y @ w["cross.wv"] @ w["cross.wo"], (2, 5, C_TINY))
    assert np.allclose(dit.attention_module("cross", x, y, w, 2), want, atol=1e-12)


def test_zero_output_projections_leave_only_the_mlp():
    from oracle import dit
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 6, C_TINY))
    y = rng.standard_normal((3, C_TINY))
    w = rand_weights(C_TINY, 5)
    for k in dit.KINDS:
        w[f"{k}.wo"] = np.zeros((C_TINY, C_TINY))
    got = dit.block_step(x, y, w, 2, {k: True for k in dit.KINDS}, {})
    assert np.allclose(got, x + dit.mlp(x, w), atol=1e-12)


def test_broadcast_steps_add_the_source_steps_module_output():
    """Under PAB a broadcasting kind adds exactly the module output of its
    latest computing step (the schedule's source step) and a computing kind a
    fresh module output of the current residual stream; run() agrees with the
    step-by-step walk; with ranges (1, 1, 1) every step computes."""
    import oracle
    from oracle import dit
    rng = np.random.default_rng(6)
    T, N, heads, steps, ranges = 2, 6, 2, 10, (2, 3, 4)
    w = rand_weights(C_TINY, 6)
    xs = [rng.standard_normal((T, N, C_TINY)) for _ in range(steps)]
    y = rng.standard_normal((3, C_TINY))
    sched = {k: oracle.schedule(steps, r) for k, r in zip(dit.KINDS, ranges)}
    cache, snaps, walk = {}, [], []
    for i in range(steps):
        x = xs[i].copy()
        for kind in dit.KINDS:
            if sched[kind][0][i]:
                fresh = dit.attention_module(kind, x, y, w, heads)
                cache[kind] = fresh
            else:
                src = int(sched[kind][1][i])
                assert src < i and sched[kind][0][src]
                assert np.array_equal(cache[kind], snaps[src][kind])
            x = x + cache[kind]
        walk.append(x + dit.mlp(x, w))
        snaps.append(dict(cache))
    outs, table = dit.run(xs, [y] * steps, w, heads, steps, ranges)
    for kind in dit.KINDS:
        assert table[kind] == [bool(c) for c in sched[kind][0]]
    for i in range(steps):
        assert np.array_equal(outs[i], walk[i]), i
    full, table1 = dit.run(xs, [y] * steps, w, heads, steps, (1, 1, 1))
    assert all(all(v) for v in table1.values())
    for i in range(steps):
        assert np.allclose(full[i], dit.block_step(xs[i], y, w, heads, {k: True for k in dit.KINDS}, {}))


# ------------------------------------------------------------------ GPU block vs oracle
def _close(got, want, what, rel=1e-2, abs_=0.1):
    diff = got - want
    r = np.linalg.norm(diff) / np.linalg.norm(want)
    assert np.abs(diff).max() <= abs_ and r <= rel, (what, float(np.abs(diff).max()), r)


@pytest.mark.gpu
@pytest.mark.parametrize("T,H,W,heads,d,text_len,steps,ranges", [
    (4, 8, 8, 2, 32, 16, 10, (2, 3, 4)),   # the tiny workload's shapes
    (4, 16, 16, 4, 72, 120, 8, (2, 4, 6)),  # 480p-like head dim and text length
])
def test_dit_block_matches_oracle_over_a_run(oracle_mod, T, H, W, heads, d, text_len, steps, ranges):
    import step_reuse_b200 as pab
    from oracle import dit as odit
    from step_reuse_b200 import dit
    C = heads * d
    wl = synth.Workload("dit-test", T, H, W, heads, d, text_len, steps, ranges, "bf16", 0.05)
    xs, text = synth.dit_inputs(wl, device="cuda", seed=7)
    wts = dit.make_weights(C, seed=8)
    block = dit.DiTBlock(pab, T, H, W, heads, d, text_len, steps, ranges, wts)
    got, mods = [], []
    try:
        for i in range(steps):
            got.append(block.step(i, xs[i], text).cpu().numpy())
            mods.append({k: block.cache[k].clone() for k in dit.KINDS})
    finally:
        block.close()
    w64 = {k: v.double().cpu().numpy() for k, v in wts.items()}
    want, table = odit.run([x.cpu().numpy() for x in xs], [text.double().cpu().numpy()] * steps,
                           w64, heads, steps, ranges)
    for i in range(steps):
        _close(got[i], want[i], f"step {i}")
        for k in dit.KINDS:
            if not table[k][i]:  # broadcast: the module output is the previous step's, bit for bit
                assert torch.equal(mods[i][k], mods[i - 1][k]), (k, i)
