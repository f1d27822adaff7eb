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


def _dsp_worker(rank, world, port, ranges, q, exchange="collective", tmpdir=None):
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
        """Stand-in binding: the oracle's plan and block permute; for the direct
        exchange, buffers other processes can map are shared memory-mapped
        files (the handle is the path) and the block scatter is written out
        from its definition with numpy slicing."""
        Plan = FakePlan
        n_ipc = 0

        @staticmethod
        def permute_blocks(x, P, Q, out=None, stream=None):
            y = oracle.permute_blocks(x.contiguous().numpy(), P, Q)
            out.copy_(torch.from_numpy(y).view(out.shape))
            return out

        @classmethod
        def ipc_tensor(cls, shape, dtype, device):
            cls.n_ipc += 1
            path = os.path.join(tmpdir, f"ipc_{rank}_{cls.n_ipc}.bin")
            arr = np.memmap(path, dtype=np.float64, mode="w+", shape=tuple(shape))
            return torch.from_numpy(arr), path.encode().ljust(64, b"\0"), arr

        @staticmethod
        def ipc_open_tensor(handle, shape, dtype, device):
            arr = np.memmap(handle.rstrip(b"\0").decode(), dtype=np.float64, mode="r+", shape=tuple(shape))
            return torch.from_numpy(arr), arr

        @staticmethod
        def ipc_close(arr):
            arr.flush()

        @staticmethod
        def ipc_free(arr):
            os.remove(arr.filename)

        @staticmethod
        def scatter_blocks(srcs, dsts, G, P, block_rows, src_order, dst_offset_rows, dst_stride_rows,
                           stream=None):
            for t, x in enumerate(srcs):
                C = x.shape[-1]
                xb = x.reshape(-1, C)
                for p in range(P):
                    for g in range(G):
                        bi = p * G + g if src_order == 0 else g * P + p
                        d = dsts[t][g].view(-1, C)
                        r0 = dst_offset_rows + p * dst_stride_rows
                        d[r0:r0 + block_rows] = xb[bi * block_rows:(bi + 1) * block_rows]

    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        T, H, W, heads, d, L, steps = 4, 4, 6, 2, 8, 5, 10
        N, C = H * W, heads * d
        st = dsp.DSPStack(FakePab, T, H, W, heads, d, L, steps, ranges, device="cpu", dtype=torch.float64,
                          exchange=exchange)
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
        st.close()
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _run_ranks(ranges, world=2, exchange="collective", tmpdir=None):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_dsp_worker, args=(r, world, port, ranges, q, exchange, tmpdir))
             for r in range(world)]
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


@pytest.mark.timeout(300)
@pytest.mark.parametrize("ranges,world", [((2, 3, 4), 2), ((2, 3, 4), 4), ((1, 1, 1), 2)])
def test_direct_exchange_matches_the_whole_video(oracle_mod, tmp_path, ranges, world):
    """The direct exchange: every rank writes its blocks straight into the
    other ranks' mapped buffers (shared memory-mapped files standing in for
    CUDA IPC buffers) and a one-element collective after each move orders the
    writes before their readers.  Every rank gets the oracle's attention of
    the whole video for its frames; two barriers per temporal compute, none
    on broadcast steps."""
    res = _run_ranks(ranges, world, exchange="direct", tmpdir=str(tmp_path))
    steps, T, N, C, elem, G = 10, 4, 24, 16, 8, world
    computes = int(oracle_mod.schedule(steps, ranges[1])[0].sum())
    for rank, worst, exchanges, collectives, sent in res:
        for kind, err in worst.items():
            assert err < 1e-12, (rank, kind, err)
        assert exchanges == 2 * computes
        assert collectives == 2 * computes  # one barrier after each move
        assert sent == computes * 4 * (T // G) * N * C * elem * (G - 1) // G
    assert not list(tmp_path.iterdir())  # every rank freed its mapped buffers


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


@pytest.mark.gpu
@pytest.mark.parametrize("G,Tl,Nl,C", [(2, 8, 795, 1152), (4, 4, 300, 1024), (8, 2, 150, 3072), (3, 1, 7, 64),
                                       (1, 16, 1590, 1152)])
def test_scatter_kernel_packs_and_unpacks_like_the_oracle(oracle_mod, G, Tl, Nl, C):
    """The exchange kernel with G local buffers standing in for the G ranks'
    buffers: every rank's pack lands in the receiving ranks' temporal inputs
    exactly as the oracle's block permute places it, and every rank's unpack
    of its output lands in the owning ranks' spatial view -- bit for bit."""
    import step_reuse_b200 as pab
    T, N = G * Tl, G * Nl
    g = torch.Generator().manual_seed(G * 100 + Tl)
    xs = [[torch.randn((Tl, N, C), generator=g).to(torch.bfloat16) for _ in range(3)] for _ in range(G)]
    recv = [[torch.full((T, Nl, C), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
            for _ in range(G)]
    for r in range(G):  # rank r packs its q, k, v into every rank's receive buffers
        pab.scatter_blocks([x.cuda() for x in xs[r]], [[recv[d][t] for d in range(G)] for t in range(3)],
                           G, Tl, Nl, src_order=0, dst_offset_rows=r * Tl * Nl, dst_stride_rows=Nl)
    torch.cuda.synchronize()
    for dst in range(G):
        for t in range(3):
            want = np.concatenate([oracle_mod.permute_blocks(xs[r][t].view(torch.int16).numpy(), Tl, G)[dst]
                                   for r in range(G)])
            assert np.array_equal(recv[dst][t].cpu().view(torch.int16).numpy(), want.reshape(T, Nl, C)), (dst, t)
    # the output of rank g: [T, N/G, C] of its positions; back to every rank's frames
    outs = [torch.randn((T, Nl, C), generator=g).to(torch.bfloat16) for _ in range(G)]
    tout = [torch.full((Tl, N, C), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    for src in range(G):
        pab.scatter_blocks([outs[src].cuda()], [[tout[r] for r in range(G)]], G, Tl, Nl, src_order=1,
                           dst_offset_rows=src * Nl, dst_stride_rows=N)
    torch.cuda.synchronize()
    for r in range(G):
        chunks = np.stack([outs[s].view(torch.int16).numpy().reshape(G, Tl, Nl, C)[r] for s in range(G)])
        want = oracle_mod.permute_blocks(chunks, G, Tl)  # [Tl, G, Nl, C]
        assert np.array_equal(tout[r].cpu().view(torch.int16).numpy(), want.reshape(Tl, N, C)), r
    assert pab.device_errors(clear=True) == 0
