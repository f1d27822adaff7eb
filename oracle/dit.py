"""fp64 CPU oracle of a synthetic video DiT block under Pyramid Attention
Broadcast -- TEST INFRASTRUCTURE ONLY (the same import rules as the rest of
``oracle``: tests, smoke and the bench's CPU legs only; it never imports the
product library).

The PAB report ("Implementation") places the three attention kinds inside
the DiT blocks of a video diffusion model and reuses each kind's attention
output over several diffusion steps.  The block written out here, in plain
numpy float64 on top of this package's attention and schedule functions:

    x <- x + A_spatial(LN(x))            A_kind(h) = Attn_kind(h Wq, h Wk, h Wv) Wo
    x <- x + A_temporal(LN(x))           (cross: keys and values from the text,
    x <- x + A_cross(LN(x), text)         y Wk and y Wv)
    x <- x + GELU(LN(x) W1) W2

LN is a layer norm over the C channels without affine parameters (eps 1e-6),
GELU the tanh form.  Under PAB a kind that broadcasts at step i adds the
module output A_kind(.) computed at its latest computing step instead of
computing it again (norm, projections and attention are all skipped); the
MLP runs at every step.
"""
from __future__ import annotations

import numpy as np

from . import cross_attention, schedule, spatial_attention, temporal_attention

KINDS = ("spatial", "temporal", "cross")
LN_EPS = 1e-6


def layer_norm(x: np.ndarray) -> np.ndarray:
    """Normalise the last axis to zero mean and unit variance (no affine)."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + LN_EPS)


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def attention_module(kind: str, x: np.ndarray, text: np.ndarray, w: dict, heads: int) -> np.ndarray:
    """A_kind(LN(x)) for x [T, N, C] and text [L, C]; returns [T, N, C]."""
    T, N, C = x.shape
    h = layer_norm(x)
    wq, wk, wv, wo = (np.asarray(w[f"{kind}.{n}"], dtype=np.float64) for n in ("wq", "wk", "wv", "wo"))
    q = h @ wq
    if kind == "cross":
        y = np.asarray(text, dtype=np.float64)
        a = cross_attention(q.reshape(T * N, C), y @ wk, y @ wv, heads).reshape(T, N, C)
    elif kind == "spatial":
        a = spatial_attention(q, h @ wk, h @ wv, heads)
    else:
        # the frames at each position attend to each other: the [N, T, C] view
        perm = lambda t: np.ascontiguousarray(t.transpose(1, 0, 2))
        a = temporal_attention(perm(q), perm(h @ wk), perm(h @ wv), heads).transpose(1, 0, 2)
    return a @ wo


def mlp(x: np.ndarray, w: dict) -> np.ndarray:
    """GELU(LN(x) W1) W2."""
    w1, w2 = (np.asarray(w[n], dtype=np.float64) for n in ("mlp.w1", "mlp.w2"))
    return gelu_tanh(layer_norm(x) @ w1) @ w2


def block_step(x: np.ndarray, text: np.ndarray, w: dict, heads: int, compute: dict, cache: dict):
    """One block evaluation at one diffusion step.

    compute[kind] -- True when the kind computes at this step (else it
    broadcasts cache[kind]); cache is updated in place with the module
    outputs of the computing kinds.  Returns the block output [T, N, C]."""
    x = np.asarray(x, dtype=np.float64).copy()
    for kind in KINDS:
        if compute[kind]:
            cache[kind] = attention_module(kind, x, text, w, heads)
        x = x + cache[kind]
    return x + mlp(x, w)


def run(xs, texts, w: dict, heads: int, steps: int, ranges, edge_pct: int = 15):
    """The block over `steps` diffusion steps under PAB with per-kind ranges
    (spatial, temporal, cross): xs[i] and texts[i] are step i's inputs.
    Returns (outputs, compute table {kind: [bool] * steps})."""
    table = {k: [bool(c) for c in schedule(steps, r, edge_pct)[0]] for k, r in zip(KINDS, ranges)}
    cache, outs = {}, []
    for i in range(steps):
        outs.append(block_step(xs[i], texts[i], w, heads, {k: table[k][i] for k in KINDS}, cache))
    return outs, table
