"""Broadcast sequence parallel: the PAB attention stack of one video split
over the ranks of a process group (PAB report, "Parallel", Fig. 3).

Dynamic sequence parallel (DSP) gives each of the G ranks T/G of the video's
frames.  Spatial and cross attention need nothing from other ranks; temporal
attention attends across all T frames of a position, so it needs two
all-to-all exchanges: one that moves every rank's frames of position chunk g
to rank g (after which rank g holds all T frames of N/G positions), and one
that moves the output back.  Under PAB a temporal step that broadcasts
serves the output of its latest computing step and the exchanges are skipped
altogether, which is where the pages' "more than 50% less communication"
comes from.

Two data paths carry the exchanges:

"direct" (the default with CUDA devices): the library's exchange kernel
(pab_scatter_blocks) writes every block straight into its destination --
    pack:   q, k, v [T/G, N, C] -> rank g's temporal inputs [3, T, N/G, C],
            rows of this rank's frames (one launch for the three tensors)
    temporal attention on that spatial view  [T, N/G, C]
    unpack: output [T, N/G, C] -> rank r's spatial view [T/G, N, C],
            columns of this rank's positions
with one stream-ordered one-element collective after each move as the
barrier that orders every rank's writes before their readers.  With G > 1
the destinations are the other ranks' buffers, allocated for CUDA IPC and
mapped into this process (peer stores over NVLink); with G = 1 they are this
process's own buffers.

"collective": the block-permute kernel packs per-destination chunks and
torch.distributed all_to_all_single moves them (NCCL on GPUs, gloo on CPU
ranks); the unpack permutes the returned chunks.

T and H*W must be divisible by G.  Pass torch's current stream (the
collectives run on it).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

KINDS = ("spatial", "temporal", "cross")


class DSPStack:
    """The three attention kinds of one video under PAB, frames sharded over
    `group` (default: the world group; a single process without a group is
    G = 1).  `pab` is the library binding (step_reuse_b200).  `exchange`:
    "direct", "collective" or "auto" (direct with CUDA devices, collective
    otherwise)."""

    def __init__(self, pab, T, H, W, heads, d, text_len, steps, ranges, group=None, device="cuda",
                 dtype=torch.bfloat16, exchange="auto"):
        self.pab, self.group = pab, group
        grouped = dist.is_available() and dist.is_initialized()
        self.G = dist.get_world_size(group) if grouped else 1
        self.rank = dist.get_rank(group) if grouped else 0
        N = H * W
        if T % self.G or N % self.G:
            raise ValueError(f"T={T} frames and H*W={N} positions must both divide by {self.G} ranks")
        if exchange == "auto":
            exchange = "direct" if torch.device(device).type == "cuda" else "collective"
        if exchange not in ("direct", "collective"):
            raise ValueError(f"exchange={exchange!r}")
        self.mode = exchange
        self.T, self.N, self.C, self.steps = T, N, heads * d, steps
        self.Tl, self.Nl = T // self.G, N // self.G
        # spatial and cross on this rank's frames; temporal on all frames of its positions
        self.plan = pab.Plan(self.Tl, H, W, heads, d, text_len, steps, ranges, dtype=dtype)
        self.tplan = pab.Plan(T, 1, self.Nl, heads, d, text_len, steps, ranges, dtype=dtype)
        self.tplan.set_temporal_view(True)
        G, Tl, Nl, C = self.G, self.Tl, self.Nl, self.C
        self._ipc_own, self._ipc_peer = [], []
        if exchange == "direct":
            rshape, oshape = (3, T, Nl, C), (2, Tl, N, C)
            if G == 1:
                self.recv = torch.empty(rshape, dtype=dtype, device=device)
                self.touts = torch.empty(oshape, dtype=dtype, device=device)
                self.peer_recv, self.peer_tout = [self.recv], [self.touts]
            else:
                self.recv, h_recv, p = pab.ipc_tensor(rshape, dtype, device)
                self._ipc_own.append(p)
                self.touts, h_tout, p = pab.ipc_tensor(oshape, dtype, device)
                self._ipc_own.append(p)
                handles = [None] * G
                dist.all_gather_object(handles, (h_recv, h_tout), group=group)
                self.peer_recv, self.peer_tout = [], []
                for g in range(G):
                    if g == self.rank:
                        self.peer_recv.append(self.recv)
                        self.peer_tout.append(self.touts)
                        continue
                    t, p = pab.ipc_open_tensor(handles[g][0], rshape, dtype, device)
                    self._ipc_peer.append(p)
                    self.peer_recv.append(t)
                    t, p = pab.ipc_open_tensor(handles[g][1], oshape, dtype, device)
                    self._ipc_peer.append(p)
                    self.peer_tout.append(t)
            self.tout = [self.touts[0], self.touts[1]]
            self.flag = torch.zeros(1, dtype=torch.float32, device=device)
        else:
            self.send = torch.empty((3, G, Tl, Nl, C), dtype=dtype, device=device)
            self.recv = self.send if G == 1 else torch.empty_like(self.send)
            self.oback = torch.empty((G, Tl, Nl, C), dtype=dtype, device=device)
            self.tout = [torch.empty((Tl, N, C), dtype=dtype, device=device) for _ in range(2)]
        self.cur = -1
        self.exchanges = 0        # all-to-all phases (two per temporal compute)
        self.collectives = 0      # collective calls (data moves or barriers)
        self.bytes_sent = 0       # bytes this rank sent to other ranks
        self._elem = torch.tensor([], dtype=dtype).element_size()

    def close(self):
        self.plan.close()
        self.tplan.close()
        if self._ipc_own or self._ipc_peer:
            # every rank has finished reading and writing the mapped buffers
            if torch.cuda.is_available():
                torch.cuda.synchronize()
            dist.barrier(group=self.group)
            for p in self._ipc_peer:
                self.pab.ipc_close(p)
            for p in self._ipc_own:
                self.pab.ipc_free(p)
            self._ipc_own, self._ipc_peer = [], []

    def reset(self):
        """A new sampling run: schedules restart, caches are dropped."""
        self.plan.reset()
        self.tplan.reset()
        self.cur = -1

    def is_compute(self, kind, step: int) -> bool:
        return self.plan.is_compute(kind, step)

    def _all_to_all(self, out, inp):
        self.collectives += 1
        if self.G == 1:
            if out.data_ptr() != inp.data_ptr():
                out.copy_(inp)
            return
        self.bytes_sent += inp.numel() * self._elem * (self.G - 1) // self.G
        dist.all_to_all_single(out, inp, group=self.group)

    def _barrier(self, payload_elems):
        """Orders every rank's direct writes before their readers: a
        one-element collective on the current stream (each rank joins it
        only after its own writes, in stream order)."""
        if self.G == 1:
            return
        self.collectives += 1
        self.bytes_sent += payload_elems * self._elem * (self.G - 1) // self.G
        dist.all_reduce(self.flag, group=self.group)

    def attention(self, kind, step: int, q=None, k=None, v=None, stream=None) -> torch.Tensor:
        """This rank's output of `kind` at `step`: spatial [T/G, N, C], cross
        [T/G * N, C] (q likewise), temporal [T/G, N, C] (q, k, v in the
        spatial view of this rank's frames).  A broadcast step returns the
        cached output and exchanges nothing."""
        if kind != "temporal":
            return self.plan.attention(kind, step, q, k, v, stream)
        if not self.plan.is_compute("temporal", step):
            if self.cur < 0:
                raise RuntimeError(f"temporal step {step} broadcasts, but no temporal step has computed")
            return self.tout[self.cur]
        slot = 1 if self.cur == 0 else 0
        if self.mode == "direct":
            self._temporal_direct(step, q, k, v, slot, stream)
        else:
            self._temporal_collective(step, q, k, v, slot, stream)
        self.cur = slot
        return self.tout[slot]

    def _temporal_direct(self, step, q, k, v, slot, stream):
        pab, G, Tl, Nl, C, r = self.pab, self.G, self.Tl, self.Nl, self.C, self.rank
        # pack: block (frame p, position chunk g) -> rank g's input, frame r*Tl + p
        pab.scatter_blocks([q, k, v], [[self.peer_recv[g][j] for g in range(G)] for j in range(3)],
                           G, Tl, Nl, src_order=0, dst_offset_rows=r * Tl * Nl, dst_stride_rows=Nl,
                           stream=stream)
        self.exchanges += 1
        self._barrier(3 * Tl * self.N * C)
        o = self.tplan.attention("temporal", step, self.recv[0], self.recv[1], self.recv[2], stream)
        # unpack: block (frame p of rank g, this rank's positions) -> rank g's view, columns r*Nl..
        pab.scatter_blocks([o], [[self.peer_tout[g][slot] for g in range(G)]], G, Tl, Nl, src_order=1,
                           dst_offset_rows=r * Nl, dst_stride_rows=self.N, stream=stream)
        self.exchanges += 1
        self._barrier(self.T * Nl * C)

    def _temporal_collective(self, step, q, k, v, slot, stream):
        pab, G, Tl, Nl, C = self.pab, self.G, self.Tl, self.Nl, self.C
        for j, x in enumerate((q, k, v)):
            pab.permute_blocks(x, Tl, G, out=self.send[j], stream=stream)
        self.exchanges += 1
        for j in range(3):
            self._all_to_all(self.recv[j], self.send[j])
        o = self.tplan.attention("temporal", step, self.recv[0].view(self.T, Nl, C),
                                 self.recv[1].view(self.T, Nl, C), self.recv[2].view(self.T, Nl, C), stream)
        self.exchanges += 1
        self._all_to_all(self.oback, o.view(G, Tl, Nl, C))
        pab.permute_blocks(self.oback, G, Tl, out=self.tout[slot].view(Tl, G, Nl, C), stream=stream)
