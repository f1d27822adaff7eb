"""Broadcast sequence parallel (PAB report, "Parallel", Fig. 3): the
frame-sharded attention stack with its two all-to-all exchanges per temporal
compute, none on a temporal broadcast step.

CPU (gloo, two and four ranks): DSPStack from the product, driven through a stand-in
binding whose plan and block permute are the oracle's functions, must give
every rank exactly the oracle's attention of the whole video restricted to
its frames, at every step of a PAB run; the exchange, collective and byte
counts follow the schedule (two exchanges per temporal compute, none on
broadcast steps -- for a 30-step run with temporal range 4, 15 of the 30
temporal steps compute, so half the exchanges of running without
broadcast).
The block permute's oracle is pinned to numpy's transpose and to the layout
oracle.  GPU: the block-permute kernel against the oracle (bit-exact) and the
one-rank DSP path against the unsharded library calls (bit-identical).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KINDS = ("spatial", "temporal", "cross")


# ------------------------------------------------------------------ oracle pins (CPU)
@pytest.mark.parametrize("P,Q,block,C,dtype", [(3, 4, 5, 8, np.float64), (2, 2, 1, 16, np.uint16),
                                               (1, 5, 3, 4, np.float32), (4, 1, 2, 2, np.int8)])
def test_permute_blocks_oracle_is_a_transpose(oracle_mod, P, Q, block, C, dtype):
    x = (np.arange(P * Q * block * C) % 251).astype(dtype).reshape(P, Q, block, C)
    assert np.array_equal(oracle_mod.permute_blocks(x, P, Q), x.transpose(1, 0, 2, 3))


def test_permute_blocks_with_single_rows_is_the_layout_change(oracle_mod):
    x = np.random.default_rng(0).standard_normal((5, 7, 6))
    assert np.array_equal(oracle_mod.permute_blocks(x, 5, 7)[:, :, 0, :], oracle_mod.layout(x, True))


# ------------------------------------------------------------------ two gloo ranks (CPU)
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(step, T, N, C, L):
    g = torch.Generator().manual_seed(1000 + step)
    full = {k: [torch.randn((T, N, C), generator=g, dtype=torch.float64) for _ in range(3)] for k in KINDS}
    text = [torch.randn((L, C), generator=g, dtype=torch.float64) for _ in range(2)]
    return full, text


def _dsp_worker(rank, world, port, ranges, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import oracle
    from step_reuse_b200 import dsp

    class FakePlan:
        def __init__(self, T, H, W, heads, d, text_len, steps, ranges, dtype=None):
            self.heads, self.sv, self.cache = heads, False, {}
            self.sched = {k: oracle.schedule(steps, r)[0] for k, r in zip(KINDS, ranges)}

        def set_temporal_view(self, sv):
            self.sv = sv

        def is_compute(self, kind, step):
            return bool(self.sched[kind][step])

        def reset(self):
            self.cache = {}

        def close(self):
            pass

        def attention(self, kind, step, q, k, v, stream=None):
            if not self.is_compute(kind, step):
                return self.cache[kind]
            a = [t.contiguous().numpy() for t in (q, k, v)]
            if kind == "spatial":
                o = oracle.spatial_attention(*a, self.heads)
            elif kind == "cross":
                o = oracle.cross_attention(*a, self.heads)
            else:
                assert self.sv  # the sharded stack hands temporal attention the spatial view
                o = oracle.temporal_attention(*[x.transpose(1, 0, 2) for x in a], self.heads).transpose(1, 0, 2)
            self.cache[kind] = torch.from_numpy(np.ascontiguousarray(o))
            return self.cache[kind]

    class FakePab:
        Plan = FakePlan

        @staticmethod
        def permute_blocks(x, P, Q, out=None, stream=None):
            y = oracle.permute_blocks(x.contiguous().numpy(), P, Q)
            out.copy_(torch.from_numpy(y).view(out.shape))
            return out

    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        T, H, W, heads, d, L, steps = 4, 4, 6, 2, 8, 5, 10
        N, C = H * W, heads * d
        st = dsp.DSPStack(FakePab, T, H, W, heads, d, L, steps, ranges, device="cpu", dtype=torch.float64)
        Tl = T // world
        fr = slice(rank * Tl, (rank + 1) * Tl)
        worst = {k: 0.0 for k in KINDS}
        last_full = {}
        for i in range(steps):
            full, text = _inputs(i, T, N, C, L)
            for kind in KINDS:
                qf, kf, vf = full[kind]
                if kind == "cross":
                    got = st.attention(kind, i, qf[fr].reshape(Tl * N, C), text[0], text[1])
                else:
                    got = st.attention(kind, i, qf[fr], kf[fr], vf[fr])
                if st.is_compute(kind, i):  # the oracle of the whole video, this rank's frames
                    a = [x.numpy() for x in (qf, kf, vf)]
                    if kind == "spatial":
                        want = oracle.spatial_attention(*a, heads)
                    elif kind == "cross":
                        want = oracle.cross_attention(a[0].reshape(T * N, C), text[0].numpy(), text[1].numpy(),
                                                      heads).reshape(T, N, C)
                    else:
                        want = oracle.temporal_attention(*[x.transpose(1, 0, 2) for x in a], heads).transpose(1, 0, 2)
                    last_full[kind] = want
                want = last_full[kind][fr].reshape(got.shape)
                worst[kind] = max(worst[kind], float(np.abs(got.numpy() - want).max()))
        q.put((rank, worst, st.exchanges, st.collectives, st.bytes_sent))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _run_ranks(ranges, world=2):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_dsp_worker, args=(r, world, port, ranges, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    return sorted(q.get(timeout=10) for _ in range(world))


@pytest.mark.timeout(300)
@pytest.mark.parametrize("ranges,world", [((2, 3, 4), 2), ((1, 1, 1), 2), ((2, 3, 4), 4)])
def test_sequence_parallel_matches_the_whole_video(oracle_mod, ranges, world):
    res = _run_ranks(ranges, world)
    steps, T, N, C, elem, G = 10, 4, 24, 16, 8, world
    computes = int(oracle_mod.schedule(steps, ranges[1])[0].sum())
    for rank, worst, exchanges, collectives, sent in res:
        for kind, err in worst.items():
            assert err < 1e-12, (rank, kind, err)
        assert exchanges == 2 * computes  # none on a temporal broadcast step
        assert collectives == 4 * computes  # q, k, v in; the output back
        assert sent == computes * 4 * (T // G) * N * C * elem * (G - 1) // G
    if ranges == (2, 3, 4):
        assert computes == 6  # 10 steps, edges 2 + 2, middle 6 with range 3: 2 computes, 4 broadcasts


# ------------------------------------------------------------------ GPU
@pytest.mark.gpu
@pytest.mark.parametrize("P,Q,block,C", [(8, 2, 795, 1152), (3, 4, 5, 64), (1, 1, 7, 8), (16, 1, 1, 72),
                                         (2, 8, 450, 3072)])
def test_permute_blocks_kernel_matches_the_oracle(oracle_mod, P, Q, block, C):
    import step_reuse_b200 as pab
    g = torch.Generator().manual_seed(P * 1000 + Q)
    x = torch.randn((P, Q, block, C), generator=g).to(torch.bfloat16)
    out = pab.permute_blocks(x.cuda(), P, Q)
    torch.cuda.synchronize()
    want = oracle_mod.permute_blocks(x.view(torch.int16).numpy(), P, Q)
    assert np.array_equal(out.cpu().view(torch.int16).numpy(), want)
    assert pab.device_errors(clear=True) == 0


@pytest.mark.gpu
def test_one_rank_sequence_parallel_is_the_unsharded_stack():
    """G = 1: the packing kernels and the temporal plan on the spatial view
    give bit for bit what the unsharded calls give, and a broadcast step
    returns the cached output."""
    import step_reuse_b200 as pab
    from step_reuse_b200 import dsp
    T, H, W, heads, d, L, steps, ranges = 8, 12, 16, 2, 64, 16, 10, (2, 3, 4)
    N, C = H * W, heads * d
    st = dsp.DSPStack(pab, T, H, W, heads, d, L, steps, ranges)
    try:
        g = torch.Generator().manual_seed(5)
        prev = None
        for i in range(steps):
            q, k, v = (torch.randn((T, N, C), generator=g).to(torch.bfloat16).cuda() for _ in range(3))
            got = st.attention("temporal", i, q, k, v)
            if st.is_compute("temporal", i):
                assert torch.equal(got, pab.temporal_attention_sv(q, k, v, heads)), i
            else:
                assert torch.equal(got, prev), i
            prev = got.clone()
            sp = st.attention("spatial", i, q, k, v)
            if st.is_compute("spatial", i):
                assert torch.equal(sp, pab.spatial_attention(q, k, v, heads)), i
        assert st.exchanges == 2 * sum(st.is_compute("temporal", i) for i in range(steps))
        assert st.bytes_sent == 0
    finally:
        st.close()
    torch.cuda.synchronize()
    assert pab.device_errors(clear=True) == 0
