"""A synthetic video DiT block around the PAB attention library.

The PAB report ("Implementation") places the three attention kinds inside
the DiT blocks of a video diffusion model and broadcasts each kind's
attention output to the following steps of its range; the speedups it
quotes (up to 35% from broadcast alone) are for whole models.  This block
measures that effect on one GPU with random weights:

    x <- x + A_spatial(LN(x))            A_kind(h) = Attn_kind(h Wq, h Wk, h Wv) Wo
    x <- x + A_temporal(LN(x))           (cross: keys and values from the text)
    x <- x + A_cross(LN(x), text)
    x <- x + GELU(LN(x) W1) W2

LN is a layer norm over C without affine parameters (eps 1e-6), GELU the
tanh form; the residual stream x is fp32, everything the tensor cores read
is bf16.  Every operation runs in the library's kernels (C ABI):
  * LN -- pab_block_layer_norm, which also adds the cached outputs of the
    kinds that broadcast since the previous norm (up to three) into x;
  * the q, k, v projections -- one pab_block_gemm with Wq | Wk | Wv
    concatenated, its epilogue writing q, k and v as three tensors (cross:
    q from the video tokens, k | v from the text);
  * the attention -- pab_attention (temporal attention on the spatial view);
  * the output projection -- pab_block_gemm whose epilogue adds A_kind into
    x in fp32 and keeps bf16(A_kind) for the broadcast steps;
  * the MLP -- pab_block_gemm with GELU in the epilogue of W1 and the
    residual add in the epilogue of W2.
A kind that broadcasts at a step adds the module output it computed at its
latest computing step: its norm, projections and attention are all skipped.
"""
from __future__ import annotations

import torch

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
        R, C = T * H * W, heads * d
        self.w = weights
        # the projections of each kind as one [C, 3C] (cross: q [C, C] and the
        # text's k | v [C, 2C]) matrix
        cat = lambda *ms: torch.cat([weights[m] for m in ms], dim=1).contiguous()
        self.wqkv = {k: cat(f"{k}.wq", f"{k}.wk", f"{k}.wv") for k in ("spatial", "temporal")}
        self.wq_cross = weights["cross.wq"]
        self.wkv_cross = cat("cross.wk", "cross.wv")
        self.plan = pab.Plan(T, H, W, heads, d, text_len, steps, ranges, dtype=torch.bfloat16)
        self.plan.set_temporal_view(True)
        self.plan.prepare()
        bf = dict(dtype=torch.bfloat16, device=device)
        self.h = torch.empty((R, C), **bf)
        self.q, self.k, self.v = (torch.empty((R, C), **bf) for _ in range(3))
        self.kt, self.vt = (torch.empty((text_len, C), **bf) for _ in range(2))
        self.hid = torch.empty((R, 4 * C), **bf)
        self.mods = {kind: torch.empty((T, H * W, C), **bf) for kind in KINDS}
        self.cache = {}
        self.device = device

    def close(self):
        self.plan.close()

    def reset(self):
        """A new sampling run: the schedule restarts and the module cache is dropped."""
        self.plan.reset()
        self.cache = {}

    def step(self, step: int, x: torch.Tensor, text: torch.Tensor, stream=None) -> torch.Tensor:
        """Block output at diffusion step `step` for x [T, N, C] (fp32) and the
        text [text_len, C] (bf16); returns a new fp32 tensor."""
        pab, T, N, C = self.pab, self.T, self.N, self.C
        R = T * N
        x = x.float().clone()
        xr = x.view(R, C)
        pending = []  # broadcast module outputs not yet added to x
        for kind in KINDS:
            if not self.plan.is_compute(kind, step):
                pending.append(self.cache[kind].view(R, C))
                continue
            pab.block_layer_norm(xr, self.h, ys=pending, stream=stream)
            pending = []
            if kind == "cross":
                pab.block_gemm(self.h, self.wq_cross, outs=[self.q], stream=stream)
                pab.block_gemm(text, self.wkv_cross, outs=[self.kt, self.vt], stream=stream)
                a = self.plan.attention(kind, step, self.q, self.kt, self.vt, stream)
            else:
                pab.block_gemm(self.h, self.wqkv[kind], outs=[self.q, self.k, self.v], stream=stream)
                a = self.plan.attention(kind, step, self.q.view(T, N, C), self.k.view(T, N, C),
                                        self.v.view(T, N, C), stream)
            # x += A_kind in fp32; bf16(A_kind) kept for the broadcast steps
            pab.block_gemm(a.reshape(R, C), self.w[f"{kind}.wo"], pab.GEMM_RESID, X=xr,
                           Y=self.mods[kind].view(R, C), stream=stream)
            self.cache[kind] = self.mods[kind]
        pab.block_layer_norm(xr, self.h, ys=pending, stream=stream)
        pab.block_gemm(self.h, self.w["mlp.w1"], pab.GEMM_GELU, outs=[self.hid], stream=stream)
        pab.block_gemm(self.hid, self.w["mlp.w2"], pab.GEMM_RESID, X=xr, stream=stream)
        return x
