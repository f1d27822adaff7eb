"""Seeded synthetic workloads for the PAB attention stack.

This module holds shapes and random-number recipes only -- none of the
method's arithmetic.  Tests feed the same tensors to the CUDA library and to
the fp64 oracle; the benchmark uses the same recipes on the device.

The pages measure PAB on Open-Sora videos (five 4 s, 192-frame, 480p clips);
those videos and the trained models are not used.  Instead q, k, v are drawn
from N(0, 1) with the latent-video shapes below and drift from step to step
as x_i = x_{i-1} + sigma * N(0, 1), which mimics slowly changing activations
over the denoising trajectory.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int            # latent frames
    H: int            # latent height (tokens)
    W: int            # latent width (tokens)
    heads: int
    d: int            # head dim
    text_len: int
    steps: int        # diffusion steps
    ranges: tuple     # broadcast ranges (spatial, temporal, cross)
    dtype: str        # "bf16" or "fp32" at the library boundary
    sigma: float      # per-step drift in the middle segment
    sigma_edge: float = 0.0  # drift on edge steps (0 -> same as sigma)
    seed: int = 0
    extra_ranges: tuple = field(default_factory=tuple)
    # (tile, win_h, win_w) in tokens when the spatial kind is sliding tile
    # attention; () for full attention within the frame
    spatial_window: tuple = field(default_factory=tuple)
    # (region, keep) when the spatial kind is draft attention; () otherwise
    spatial_draft: tuple = field(default_factory=tuple)

    @property
    def N(self) -> int:
        return self.H * self.W

    @property
    def C(self) -> int:
        return self.heads * self.d

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def flops(self) -> dict:
        """Algorithmic flops per computed invocation of each kind: 4*Lq*Lk*d
        per (batch unit, head) -- 2 for QK^T and 2 for PV per multiply-add."""
        T, N, h, d, L = self.T, self.N, self.heads, self.d, self.text_len
        return {
            "spatial": 4.0 * T * h * N * N * d,
            "temporal": 4.0 * N * h * T * T * d,
            "cross": 4.0 * T * N * h * L * d,
        }

    def elems(self) -> int:
        return self.T * self.N * self.C


WORKLOADS = {
    "tiny": Workload("tiny", T=4, H=8, W=8, heads=2, d=32, text_len=16, steps=10,
                     ranges=(2, 3, 4), dtype="fp32", sigma=0.05),
    "480p": Workload("480p", T=16, H=30, W=53, heads=16, d=72, text_len=120, steps=30,
                     ranges=(2, 4, 6), dtype="bf16", sigma=0.02),
    "720p": Workload("720p", T=24, H=45, W=80, heads=24, d=128, text_len=256, steps=30,
                     ranges=(2, 4, 6), dtype="bf16", sigma=0.02),
    "temporal_heavy": Workload("temporal_heavy", T=64, H=30, W=40, heads=16, d=64,
                               text_len=120, steps=30, ranges=(2, 4, 6), dtype="bf16",
                               sigma=0.02),
    # a 720p-class frame rounded up to whole 16 x 16 tiles (768 x 1280 video),
    # 3 x 3-tile windows: the sliding-tile spatial kind under the PAB schedule
    "sta_48x80": Workload("sta_48x80", T=24, H=48, W=80, heads=24, d=128, text_len=256, steps=30,
                          ranges=(2, 4, 6), dtype="bf16", sigma=0.02, spatial_window=(16, 48, 48)),
    # the same frames under draft attention: 16 x 16 regions (15 per frame),
    # 4 kept per query region (75% sparsity, the low end of the pages' range)
    "draft_48x80": Workload("draft_48x80", T=24, H=48, W=80, heads=24, d=128, text_len=256, steps=30,
                            ranges=(2, 4, 6), dtype="bf16", sigma=0.02, spatial_draft=(16, 4)),
    "sweep": Workload("sweep", T=16, H=30, W=53, heads=16, d=72, text_len=120, steps=50,
                      ranges=(1, 1, 1), dtype="bf16", sigma=0.02, sigma_edge=0.2,
                      extra_ranges=((1, 1, 1), (2, 3, 4), (2, 4, 6), (3, 6, 9))),
}

KINDS = ("spatial", "temporal", "cross")


def shapes(w: Workload) -> dict:
    """Tensor shapes per kind as the library takes them."""
    T, N, C, L = w.T, w.N, w.C, w.text_len
    return {
        "spatial": {"q": (T, N, C), "k": (T, N, C), "v": (T, N, C)},
        "temporal": {"q": (N, T, C), "k": (N, T, C), "v": (N, T, C)},
        "cross": {"q": (T * N, C), "k": (L, C), "v": (L, C)},
    }


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def initial_inputs(w: Workload, device="cpu", seed: int | None = None) -> dict:
    """{kind: {"q","k","v": tensor}} drawn from N(0, 1) in fp32, then cast to the
    boundary dtype.  Each kind draws its own q, k, v."""
    g = generator(w.seed if seed is None else seed, device)
    out = {}
    for kind in KINDS:
        out[kind] = {}
        for name, shp in shapes(w)[kind].items():
            x = torch.randn(shp, generator=g, device=device, dtype=torch.float32)
            out[kind][name] = x.to(w.torch_dtype)
    return out


def sigma_at(w: Workload, step: int, edge: int) -> float:
    """Drift applied before `step` (>= 1): sigma_edge on the edge steps when set."""
    if w.sigma_edge and (step < edge or step >= w.steps - edge):
        return w.sigma_edge
    return w.sigma


def drift_(inputs: dict, sigma: float, g: torch.Generator) -> None:
    """In place: x <- x + sigma * N(0, 1) for every tensor (fp32 math, cast back)."""
    for kind in KINDS:
        for name, x in inputs[kind].items():
            noise = torch.randn(x.shape, generator=g, device=x.device, dtype=torch.float32)
            x.copy_((x.float() + sigma * noise).to(x.dtype))


def randn(shape, seed: int, dtype=torch.float32, device="cpu", scale: float = 1.0):
    g = generator(seed, device)
    return (scale * torch.randn(shape, generator=g, device=device, dtype=torch.float32)).to(dtype)


def dit_inputs(w: Workload, device="cpu", seed: int | None = None, steps: int | None = None):
    """Inputs of the synthetic DiT block over a sampling run: the residual
    stream x_i [T, N, C] (fp32, N(0, 1) at step 0, then drifting by
    sigma * N(0, 1) per step) and one text embedding [text_len, C] (bf16,
    N(0, 1), the same at every step).  Returns (xs, text)."""
    g = generator(w.seed if seed is None else seed)
    x = torch.randn((w.T, w.N, w.C), generator=g)
    text = torch.randn((w.text_len, w.C), generator=g).to(torch.bfloat16)
    xs = [x.clone()]
    for _ in range(1, steps or w.steps):
        x = x + w.sigma * torch.randn(x.shape, generator=g)
        xs.append(x.clone())
    return [t.to(device) for t in xs], text.to(device)
