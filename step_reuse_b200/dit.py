"""A synthetic video DiT block around the PAB attention library.

The PAB report ("Implementation") places the three attention kinds inside
the DiT blocks of a video diffusion model and broadcasts each kind's
attention output to the following steps of its range; the speedups it
quotes (up to 35% from broadcast alone) are for whole models.  This block
measures that effect on one GPU with random weights, around the library's
own kernels:

    x <- x + A_spatial(LN(x))            A_kind(h) = Attn_kind(h Wq, h Wk, h Wv) Wo
    x <- x + A_temporal(LN(x))           (cross: keys and values from the text)
    x <- x + A_cross(LN(x), text)
    x <- x + GELU(LN(x) W1) W2

LN is a layer norm over C without affine parameters (eps 1e-6), GELU the
tanh form.  The attention runs through the C ABI (pab_attention; temporal
attention on the spatial view, no layout change).  Projections, norms and
the MLP are plain library operations (cuBLAS GEMMs in bf16 with fp32
accumulation, PyTorch's layer norm and GELU); the residual stream is fp32.
A kind that broadcasts at a step adds the module output it computed at its
latest computing step: its norm, projections and attention are all skipped.
"""
from __future__ import annotations

import torch
import torch.nn.functional as F

KINDS = ("spatial", "temporal", "cross")
LN_EPS = 1e-6


def make_weights(C: int, seed: int = 0, device="cuda", dtype=torch.bfloat16) -> dict:
    """Random projection and MLP weights, N(0, 1/fan_in), as [in, out] matrices."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    w = {}
    for kind in KINDS:
        for n in ("wq", "wk", "wv", "wo"):
            w[f"{kind}.{n}"] = torch.randn((C, C), generator=g) / C ** 0.5
    w["mlp.w1"] = torch.randn((C, 4 * C), generator=g) / C ** 0.5
    w["mlp.w2"] = torch.randn((4 * C, C), generator=g) / (4 * C) ** 0.5
    return {k: v.to(dtype).to(device) for k, v in w.items()}


class DiTBlock:
    """One DiT block over a sampling run, PAB-scheduled through a plan."""

    def __init__(self, pab, T, H, W, heads, d, text_len, steps, ranges, weights, device="cuda"):
        self.pab = pab
        self.T, self.N, self.C, self.heads, self.d = T, H * W, heads * d, heads, d
        self.w = weights
        self.plan = pab.Plan(T, H, W, heads, d, text_len, steps, ranges, dtype=torch.bfloat16)
        self.plan.set_temporal_view(True)
        self.plan.prepare()
        self.cache = {}
        self.device = device

    def close(self):
        self.plan.close()

    def reset(self):
        """A new sampling run: the schedule restarts and the module cache is dropped."""
        self.plan.reset()
        self.cache = {}

    def _ln(self, x):
        return F.layer_norm(x, (self.C,), eps=LN_EPS).to(torch.bfloat16)

    def _module(self, kind, step, x, text, stream):
        T, N, C, w = self.T, self.N, self.C, self.w
        h = self._ln(x).view(T * N, C)
        q = (h @ w[f"{kind}.wq"]).view(T, N, C)
        if kind == "cross":
            k, v = text @ w["cross.wk"], text @ w["cross.wv"]
            q = q.view(T * N, C)
        else:
            k = (h @ w[f"{kind}.wk"]).view(T, N, C)
            v = (h @ w[f"{kind}.wv"]).view(T, N, C)
        a = self.plan.attention(kind, step, q, k, v, stream)
        return (a.reshape(T * N, C) @ w[f"{kind}.wo"]).view(T, N, C)

    def step(self, step: int, x: torch.Tensor, text: torch.Tensor, stream=None) -> torch.Tensor:
        """Block output at diffusion step `step` for x [T, N, C] (fp32) and the
        text [text_len, C] (bf16); returns a new fp32 tensor."""
        x = x.float().clone()
        for kind in KINDS:
            if self.plan.is_compute(kind, step):
                self.cache[kind] = self._module(kind, step, x, text, stream)
            x += self.cache[kind].float()
        h = self._ln(x).view(self.T * self.N, self.C)
        y = F.gelu((h @ self.w["mlp.w1"]).float(), approximate="tanh").to(torch.bfloat16) @ self.w["mlp.w2"]
        x += y.view(self.T, self.N, self.C).float()
        return x
