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

Data path per temporal compute on each rank (every step in the library):
    q, k, v [T/G, N, C]  --permute_blocks-->  [G, T/G, N/G, C]   (chunk g = positions of rank g)
    all_to_all (one per tensor)          -->  [G, T/G, N/G, C] = [T, N/G, C]  (all frames, own positions)
    temporal attention on that spatial view   [T, N/G, C]
    all_to_all                           -->  [G, T/G, N/G, C]   (chunk g: own frames of rank g's positions)
    permute_blocks                       -->  [T/G, N, C]
The exchanges are torch.distributed all_to_all_single calls (NCCL over
NVLink on GPUs) on torch's current stream; pass that stream to the calls.
T and H*W must be divisible by G.  With G = 1 the exchanges are the
identity and the same packing kernels run.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

KINDS = ("spatial", "temporal", "cross")


class DSPStack:
    """The three attention kinds of one video under PAB, frames sharded over
    `group` (default: the world group; a single process without a group is
    G = 1).  `pab` is the library binding (step_reuse_b200)."""

    def __init__(self, pab, T, H, W, heads, d, text_len, steps, ranges, group=None, device="cuda",
                 dtype=torch.bfloat16):
        self.pab, self.group = pab, group
        grouped = dist.is_available() and dist.is_initialized()
        self.G = dist.get_world_size(group) if grouped else 1
        self.rank = dist.get_rank(group) if grouped else 0
        N = H * W
        if T % self.G or N % self.G:
            raise ValueError(f"T={T} frames and H*W={N} positions must both divide by {self.G} ranks")
        self.T, self.N, self.C, self.steps = T, N, heads * d, steps
        self.Tl, self.Nl = T // self.G, N // self.G
        # spatial and cross on this rank's frames; temporal on all frames of its positions
        self.plan = pab.Plan(self.Tl, H, W, heads, d, text_len, steps, ranges, dtype=dtype)
        self.tplan = pab.Plan(T, 1, self.Nl, heads, d, text_len, steps, ranges, dtype=dtype)
        self.tplan.set_temporal_view(True)
        G, Tl, Nl, C = self.G, self.Tl, self.Nl, self.C
        self.send = torch.empty((3, G, Tl, Nl, C), dtype=dtype, device=device)
        self.recv = self.send if G == 1 else torch.empty_like(self.send)
        self.oback = torch.empty((G, Tl, Nl, C), dtype=dtype, device=device)
        self.tout = [torch.empty((Tl, N, C), dtype=dtype, device=device) for _ in range(2)]
        self.cur = -1
        self.exchanges = 0        # all-to-all phases (two per temporal compute)
        self.collectives = 0      # all_to_all_single calls
        self.bytes_sent = 0       # bytes this rank sent to other ranks
        self._elem = torch.tensor([], dtype=dtype).element_size()

    def close(self):
        self.plan.close()
        self.tplan.close()

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
        slot = 1 if self.cur == 0 else 0
        pab.permute_blocks(self.oback, G, Tl, out=self.tout[slot].view(Tl, G, Nl, C), stream=stream)
        self.cur = slot
        return self.tout[slot]
