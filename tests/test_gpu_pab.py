"""GPU parity of whole PAB sampling runs through the plan API (C ABI
pab_attention): every synthetic workload, every kind, every step.

 * schedule: which steps launched work must equal the oracle's walk
   (PAB report, "Implementation" / Fig. 2) exactly;
 * broadcast hits: the returned pointer is the latest compute's slot and its
   bytes are identical to that compute's output;
 * computed outputs: within max-abs 2e-2 / rel-L2 5e-3 of the fp64 oracle on
   the same bf16 inputs -- full tensors for the tiny workload and for two
   480p steps, seeded samples (whole frames' rows, positions, video tokens)
   at the larger workloads;
 * the attention-difference MSE (Fig. 1) between consecutive steps' outputs
   against the oracle's, to 1e-5 relative.
"""
import numpy as np
import pytest
import torch

import synth
from parity import MSE_REL, assert_attn_close, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pab():
    import step_reuse_b200
    assert torch.cuda.is_available()
    return step_reuse_b200


def oracle_kind(oracle_mod, kind, q, k, v, heads):
    if kind == "spatial":
        return oracle_mod.spatial_attention(q, k, v, heads)
    if kind == "temporal":
        return oracle_mod.temporal_attention(q, k, v, heads)
    return oracle_mod.cross_attention(q, k, v, heads)


SAMPLES = (256, 512, 4096)  # spatial rows per sampled frame, temporal positions, cross rows


def sampled_check(oracle_mod, kind, w, x, out, rng, what, sizes=SAMPLES):
    """Compare seeded samples of the output with the oracle computed on just
    those rows (each query row's result depends only on its keys).  Rows are
    gathered on the device first, so only the samples cross to the host."""
    q, k, v = x["q"], x["k"], x["v"]
    dev = q.device
    n_rows, n_pos, n_cross = sizes
    if kind == "spatial":
        for t in rng.choice(w.T, size=min(2, w.T), replace=False):
            rows = torch.from_numpy(np.sort(rng.choice(w.N, size=min(n_rows, w.N), replace=False))).to(dev)
            t = int(t)
            # rows of frame t against all keys of frame t
            want = oracle_mod.cross_attention(to_f64(q[t].index_select(0, rows)), to_f64(k[t]),
                                              to_f64(v[t]), w.heads)
            assert_attn_close(out[t].index_select(0, rows), want, f"{what} frame {t}")
    elif kind == "temporal":
        pos = torch.from_numpy(np.sort(rng.choice(w.N, size=min(n_pos, w.N), replace=False))).to(dev)
        want = oracle_mod.temporal_attention(to_f64(q.index_select(0, pos)), to_f64(k.index_select(0, pos)),
                                             to_f64(v.index_select(0, pos)), w.heads)
        assert_attn_close(out.index_select(0, pos), want, what)
    else:
        rows = torch.from_numpy(np.sort(rng.choice(w.T * w.N, size=min(n_cross, w.T * w.N), replace=False))).to(dev)
        want = oracle_mod.cross_attention(to_f64(q.index_select(0, rows)), to_f64(k), to_f64(v), w.heads)
        assert_attn_close(out.index_select(0, rows), want, what)


def run_pab(pab, oracle_mod, w, ranges, check_steps, full_steps=(), mse_steps=None, seed=0, sizes=SAMPLES):
    """Run one sampling run; returns per-kind lists of (step, computed, mse)."""
    plan = pab.Plan(w.T, w.H, w.W, w.heads, w.d, w.text_len, w.steps, ranges,
                    dtype=w.torch_dtype)
    plan.prepare()
    x = synth.initial_inputs(w, device="cuda", seed=seed)
    g = synth.generator(seed + 1, "cuda")
    edge = oracle_mod.edge_steps(w.steps)
    sched = {kind: oracle_mod.schedule(w.steps, r) for kind, r in zip(synth.KINDS, ranges)}
    rng = np.random.default_rng(seed)
    saved = {}       # kind -> (step, ptr, clone) of the latest compute
    prev_out = {}    # kind -> clone of previous step's output (for MSE)
    log = {kind: [] for kind in synth.KINDS}
    for i in range(w.steps):
        if i > 0:
            synth.drift_(x, synth.sigma_at(w, i, edge), g)
        for kind in synth.KINDS:
            comp = bool(sched[kind][0][i])
            assert plan.is_compute(kind, i) == comp
            xs = x[kind]
            ptr = plan.attention_ptr(kind, i, xs["q"], xs["k"], xs["v"])
            shape = {"spatial": (w.T, w.N, w.C), "temporal": (w.N, w.T, w.C),
                     "cross": (w.T * w.N, w.C)}[kind]
            out = pab._wrap(ptr, shape, w.torch_dtype, xs["q"].device)
            if comp:
                if kind in saved:
                    # the new compute never overwrites the slot of the previous one
                    assert ptr != saved[kind][1]
                saved[kind] = (i, ptr, out.clone())
                if i in full_steps:
                    want = oracle_kind(oracle_mod, kind, *(to_f64(xs[n].to(torch.bfloat16))
                                                         for n in ("q", "k", "v")), w.heads)
                    assert_attn_close(out, want, f"{w.name} {kind} step {i} (full)")
                elif i in check_steps:
                    bx = {n: xs[n].to(torch.bfloat16) for n in ("q", "k", "v")}
                    sampled_check(oracle_mod, kind, w, bx, out, rng, f"{w.name} {kind} step {i}", sizes)
            else:
                src = int(sched[kind][1][i])
                s_step, s_ptr, s_clone = saved[kind]
                assert s_step == src and ptr == s_ptr
                assert torch.equal(out.view(torch.int16), s_clone.view(torch.int16))
            mse = None
            if kind in prev_out and (mse_steps is None or i in mse_steps):
                mse = pab.attn_diff_mse(out, prev_out[kind])
                if mse_steps is not None:
                    want = oracle_mod.mse(to_f64(out), to_f64(prev_out[kind]))
                    assert abs(mse - want) <= MSE_REL * max(abs(want), 1e-300), (mse, want)
            prev_out[kind] = out.clone()
            log[kind].append((i, comp, mse))
    torch.cuda.synchronize()
    assert pab.device_errors(clear=True) == 0
    plan.close()
    return log


def test_tiny_full_run(pab, oracle_mod):
    w = synth.WORKLOADS["tiny"]
    run_pab(pab, oracle_mod, w, w.ranges, check_steps=(), full_steps=set(range(w.steps)),
            mse_steps=set(range(1, w.steps)))


def test_480p_run(pab, oracle_mod):
    w = synth.WORKLOADS["480p"]
    e = oracle_mod.edge_steps(w.steps)
    run_pab(pab, oracle_mod, w, w.ranges,
            check_steps={1, e + 2, e + 6, e + 12, w.steps - e, w.steps - 1},
            full_steps={0, e}, mse_steps={1, e + 1, w.steps - 1})


@pytest.mark.parametrize("name", ["720p", "temporal_heavy"])
def test_large_runs_sampled(pab, oracle_mod, name):
    """Every computed step of every kind checked on seeded samples: 2 frames
    x 256 rows spatial, 512 positions temporal and 4096 rows cross at the
    temporal-heavy workload; at 720p (3600-token frames, 24 heads of 128,
    where the fp64 oracle of a sample costs the most) 2 frames x 32 rows,
    128 positions and 1024 rows, so all 49 computes stay affordable.  Every
    broadcast step's schedule and bytes are checked exactly."""
    w = synth.WORKLOADS[name]
    sizes = (32, 128, 1024) if name == "720p" else SAMPLES
    run_pab(pab, oracle_mod, w, w.ranges, check_steps=set(range(w.steps)), mse_steps={1, w.steps - 1},
            sizes=sizes)


def test_plan_temporal_spatial_view(pab, oracle_mod):
    """A plan set to the spatial view takes [T, N, C] temporal inputs and
    returns [T, N, C]; hits still serve the cached slot bit-identically."""
    w = synth.WORKLOADS["480p"]
    plan = pab.Plan(w.T, w.H, w.W, w.heads, w.d, w.text_len, w.steps, w.ranges, dtype=w.torch_dtype)
    plan.set_temporal_view(True)
    x = synth.initial_inputs(w, device="cuda")
    q, k, v = (x["temporal"][n].reshape(w.N, w.T, w.C).permute(1, 0, 2).contiguous() for n in ("q", "k", "v"))
    out = plan.attention("temporal", 0, q, k, v)
    assert out.shape == (w.T, w.N, w.C)
    rng = np.random.default_rng(5)
    pos = np.sort(rng.choice(w.N, size=256, replace=False))
    want = oracle_mod.temporal_attention(*(np.transpose(to_f64(t[:, pos]), (1, 0, 2)) for t in (q, k, v)), w.heads)
    assert_attn_close(out[:, pos], np.transpose(want, (1, 0, 2)), "plan temporal spatial view")
    saved = out.clone()
    e = oracle_mod.edge_steps(w.steps)
    for i in range(1, e + 1):
        plan.attention("temporal", i, q, k, v)
    hit = plan.attention("temporal", e + 1)
    assert not plan.is_compute("temporal", e + 1) and hit.shape == (w.T, w.N, w.C)
    plan.close()


def test_sweep_u_shape_and_counts(pab, oracle_mod):
    """Sweep workload (480p shapes, 50 steps, drift 0.2 on edge steps, 0.02 in
    the middle): the compute counts follow the ranges, and with no broadcast
    the step-to-step MSE is larger on the edges than in the middle (the U
    shape is built into the synthetic drift; this checks the pipeline
    reports it)."""
    w = synth.WORKLOADS["sweep"]
    e = oracle_mod.edge_steps(w.steps)
    for ranges in w.extra_ranges:
        log = run_pab(pab, oracle_mod, w, ranges, check_steps={e + 3} if ranges == (3, 6, 9) else set(),
                      mse_steps=None)
        for kind, r in zip(synth.KINDS, ranges):
            comp = [c for _, c, _ in log[kind]]
            assert sum(comp) == int(oracle_mod.schedule(w.steps, r)[0].sum())
        if ranges == (1, 1, 1):
            for kind in synth.KINDS:
                m = {i: v for i, _, v in log[kind] if v is not None}
                edge_mse = np.mean([m[i] for i in range(1, e)] + [m[i] for i in range(w.steps - e + 1, w.steps)])
                mid_mse = np.mean([m[i] for i in range(e + 1, w.steps - e)])
                assert edge_mse > 5 * mid_mse, (kind, edge_mse, mid_mse)


def _run_plan_mse(pab, w, ranges, setup=None, seed=0, side=None):
    """One run with the plan's MSE table on (its launches on the stream
    `side` when given): (mse table, outputs of every compute)."""
    plan = pab.Plan(w.T, w.H, w.W, w.heads, w.d, w.text_len, w.steps, ranges, dtype=w.torch_dtype)
    if setup:
        setup(plan)
    table = torch.full((3, w.steps), -1.0, dtype=torch.float64, device="cuda")
    plan.set_diff_mse(table)
    if side is not None:
        plan.set_diff_mse_stream(side)
    x = synth.initial_inputs(w, device="cuda", seed=seed)
    g = synth.generator(seed + 1, "cuda")
    edge = _edge(w)
    outs = {kind: [] for kind in synth.KINDS}
    for i in range(w.steps):
        if i > 0:
            synth.drift_(x, synth.sigma_at(w, i, edge), g)
        for kind in synth.KINDS:
            xs = x[kind]
            q, k, v = xs["q"], xs["k"], xs["v"]
            if kind == "temporal" and getattr(plan, "temporal_sv", False):
                q, k, v = (t.reshape(w.N, w.T, w.C).permute(1, 0, 2).contiguous() for t in (q, k, v))
            comp = plan.is_compute(kind, i)
            out = plan.attention(kind, i, q, k, v)
            if comp:
                outs[kind].append((i, out.clone()))
    torch.cuda.synchronize()
    assert pab.device_errors(clear=True) == 0
    plan.close()
    return table.cpu().numpy(), outs


def _edge(w):
    import oracle
    return oracle.edge_steps(w.steps)


@pytest.mark.parametrize("name,view", [("tiny", False), ("480p", False), ("480p", True), ("720p", False)])
def test_plan_diff_mse(pab, oracle_mod, name, view):
    """The plan's attention-difference MSE (PAB report, Fig. 1): every compute
    after a kind's first writes the MSE of its output against the kind's
    previous compute -- equal to the oracle's to 1e-5 relative (checked on
    every pair at the tiny size, on the first and last pair of each kind at
    the large ones, where the host oracle of a pair reads two whole outputs)
    and bit-identical to the stand-alone MSE call on every pair (the same
    reduction over the same data) -- and nothing else is written; a second
    run writes bit-identical values."""
    w = synth.WORKLOADS[name]
    setup = (lambda p: p.set_temporal_view(True)) if view else None
    t1, outs = _run_plan_mse(pab, w, w.ranges, setup)
    t2, _ = _run_plan_mse(pab, w, w.ranges, setup)
    assert np.array_equal(t1, t2)  # bitwise reproducible
    for ki, kind in enumerate(synth.KINDS):
        comps = outs[kind]
        written = {i for i in range(w.steps) if t1[ki, i] != -1.0}
        assert written == {i for i, _ in comps[1:]}, (kind, written)
        for n, ((i, o), (_, prev)) in enumerate(zip(comps[1:], comps[:-1])):
            alone = pab.attn_diff_mse(o, prev)
            assert t1[ki, i] == alone, (kind, i, t1[ki, i], alone)
            if name == "tiny" or n in (0, len(comps) - 2):
                want = oracle_mod.mse(to_f64(o), to_f64(prev))
                assert abs(t1[ki, i] - want) <= MSE_REL * want, (kind, i, t1[ki, i], want)


@pytest.mark.parametrize("name", ["tiny", "480p"])
def test_plan_diff_mse_side_stream(pab, name):
    """The plan's MSE launches on a side stream (pab_plan_set_diff_mse_stream):
    the table is bit-identical to the in-line one and every computed output
    is unchanged -- the kind's next compute waits for the MSE reading the
    slot it overwrites."""
    w = synth.WORKLOADS[name]
    t0, outs0 = _run_plan_mse(pab, w, w.ranges)
    side = torch.cuda.Stream()
    t1, outs1 = _run_plan_mse(pab, w, w.ranges, side=side)
    assert np.array_equal(t0, t1)
    for kind in synth.KINDS:
        assert [i for i, _ in outs0[kind]] == [i for i, _ in outs1[kind]]
        for (_, a), (_, b) in zip(outs0[kind], outs1[kind]):
            assert torch.equal(a, b)


def test_plan_diff_mse_stream_switch(pab):
    """Switching between side-stream and in-line MSE launches mid-run gives
    the same table (an in-line launch waits for the pending side-stream ones:
    they share the plan's scratch)."""
    w = synth.WORKLOADS["tiny"]
    t0, _ = _run_plan_mse(pab, w, w.ranges)
    side = torch.cuda.Stream()
    plan = pab.Plan(w.T, w.H, w.W, w.heads, w.d, w.text_len, w.steps, w.ranges, dtype=w.torch_dtype)
    table = torch.full((3, w.steps), -1.0, dtype=torch.float64, device="cuda")
    plan.set_diff_mse(table)
    x = synth.initial_inputs(w, device="cuda", seed=0)
    g = synth.generator(1, "cuda")
    edge = _edge(w)
    for i in range(w.steps):
        if i > 0:
            synth.drift_(x, synth.sigma_at(w, i, edge), g)
        plan.set_diff_mse_stream(side if i % 2 == 0 else None)
        for kind in synth.KINDS:
            plan.attention(kind, i, x[kind]["q"], x[kind]["k"], x[kind]["v"])
    torch.cuda.synchronize()
    plan.close()
    assert np.array_equal(t0, table.cpu().numpy())


@pytest.mark.parametrize("mode", ["window", "draft"])
def test_plan_diff_mse_spatial_alternatives(pab, oracle_mod, mode):
    """The same diagnostic through the sliding-tile (window) and draft-attention
    (region list) forms of the spatial kind."""
    w = synth.Workload(name="tiles", T=2, H=32, W=48, heads=2, d=64, text_len=16, steps=10, ranges=(2, 3, 4),
                       sigma=0.05, dtype="bf16")
    setup = (lambda p: p.set_spatial_window(16, 48, 48)) if mode == "window" else \
        (lambda p: p.set_spatial_draft(16, 3))
    t1, outs = _run_plan_mse(pab, w, w.ranges, setup)
    t2, _ = _run_plan_mse(pab, w, w.ranges, setup)
    assert np.array_equal(t1, t2)
    comps = outs["spatial"]
    assert len(comps) > 2
    for (i, o), (_, prev) in zip(comps[1:], comps[:-1]):
        want = oracle_mod.mse(to_f64(o), to_f64(prev))
        assert abs(t1[0, i] - want) <= MSE_REL * want, (i, t1[0, i], want)
