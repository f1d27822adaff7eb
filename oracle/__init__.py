"""fp64 CPU oracle for the PAB attention stack -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product library
(``step_reuse_b200``) never imports, links or calls it, and this package never
imports the product library: the two share no code.

The arithmetic lives in ``pab_oracle.c`` (plain C, double precision, OpenMP
over independent (batch unit, head) pairs); this module only compiles it with
gcc, loads it with ctypes and marshals numpy float64 arrays.

What each function computes (sources are the PAB pages):
  * spatial / temporal / cross attention -- the three attention kinds of a
    video DiT block (m.sbmmt.com PAB report, "Implementation"): the textbook
    softmax(Q K^T / sqrt(d)) V per head, head h on channels [h*d, (h+1)*d);
  * schedule -- Pyramid Attention Broadcast (same report, Fig. 2, and the
    paper abstract): first and last 15% of steps compute, the middle 70%
    broadcasts each compute to the following (range - 1) steps;
  * mse -- the attention-difference diagnostic of Fig. 1 (MSE between the
    outputs of consecutive diffusion steps);
  * layout -- the spatial view [T, N, C] <-> temporal view [N, T, C];
  * permute_blocks -- [P, Q, block, C] -> [Q, P, block, C], the packing of a
    sequence-parallel all-to-all (PAB report, "Parallel");
  * sta_attention -- sliding tile attention as the spatial kind (sgqg.cn
    summary of "Fast Video Generation with Sliding Tile Attention", section
    "Sliding Tile Attention (STA)"): 2-D tiles per frame, a window of whole
    tiles centred on the query's tile, cut off at the frame edge;
  * draft_select / region_sparse_attention / draft_attention -- draft
    attention as the spatial kind (crisp3r.com article on "Draft Attention",
    steps 1-4): pooled region sketch, draft scores, the best key regions of
    each query region, attention restricted to them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pab_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile pab_oracle.c into liboracle.so beside it (gcc, -O2, OpenMP)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_spatial_attention.argtypes = [_dp, _dp, _dp, _dp] + [ctypes.c_int] * 4
        lib.oracle_temporal_attention.argtypes = [_dp, _dp, _dp, _dp] + [ctypes.c_int] * 4
        lib.oracle_cross_attention.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_long] + [ctypes.c_int] * 3
        lib.oracle_sta_attention.argtypes = [_dp, _dp, _dp, _dp] + [ctypes.c_int] * 8
        lib.oracle_draft_select.argtypes = [_dp, _dp] + [ctypes.c_int] * 7 + [_ip]
        lib.oracle_region_sparse_attention.argtypes = [_dp, _dp, _dp, _dp] + [ctypes.c_int] * 7 + [_ip]
        lib.oracle_pab_edge_steps.argtypes = [ctypes.c_int, ctypes.c_int]
        lib.oracle_pab_schedule.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _ip, _ip]
        lib.oracle_mse.argtypes = [_dp, _dp, ctypes.c_long]
        lib.oracle_mse.restype = ctypes.c_double
        lib.oracle_layout.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 4
        lib.oracle_permute_blocks.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_long, ctypes.c_int, ctypes.c_int]
        lib.oracle_num_threads.restype = ctypes.c_int
        for name in ("oracle_spatial_attention", "oracle_temporal_attention",
                     "oracle_cross_attention", "oracle_sta_attention", "oracle_draft_select",
                     "oracle_region_sparse_attention", "oracle_pab_edge_steps",
                     "oracle_pab_schedule", "oracle_layout", "oracle_permute_blocks", "oracle_num_threads"):
            if getattr(lib, name).restype is not ctypes.c_double:
                getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def num_threads() -> int:
    """OpenMP threads the oracle uses (the host cores it runs on)."""
    return int(_load().oracle_num_threads())


def spatial_attention(q, k, v, heads: int) -> np.ndarray:
    """q, k, v: [T, N, C] -> out [T, N, C]; attention within each frame."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, N, C = q.shape
    assert k.shape == q.shape and v.shape == q.shape and C % heads == 0
    o = np.empty_like(q)
    rc = _load().oracle_spatial_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(o), T, N, heads, C // heads)
    if rc != 0:
        raise RuntimeError(f"oracle_spatial_attention failed ({rc})")
    return o


def temporal_attention(q, k, v, heads: int) -> np.ndarray:
    """q, k, v: [N, T, C] -> out [N, T, C]; attention across frames per position."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, T, C = q.shape
    assert k.shape == q.shape and v.shape == q.shape and C % heads == 0
    o = np.empty_like(q)
    rc = _load().oracle_temporal_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(o), N, T, heads, C // heads)
    if rc != 0:
        raise RuntimeError(f"oracle_temporal_attention failed ({rc})")
    return o


def cross_attention(q, kt, vt, heads: int) -> np.ndarray:
    """q: [R, C] video tokens; kt, vt: [Lt, C] text tokens -> out [R, C]."""
    q, kt, vt = _f64(q), _f64(kt), _f64(vt)
    shape = q.shape
    q2 = q.reshape(-1, shape[-1])
    R, C = q2.shape
    Lt = kt.shape[0]
    assert kt.shape == (Lt, C) and vt.shape == (Lt, C) and C % heads == 0
    o = np.empty_like(q2)
    rc = _load().oracle_cross_attention(_ptr(q2), _ptr(kt), _ptr(vt), _ptr(o), R, Lt, heads, C // heads)
    if rc != 0:
        raise RuntimeError(f"oracle_cross_attention failed ({rc})")
    return o.reshape(shape)


def sta_attention(q, k, v, H: int, W: int, heads: int, tile: int, win_h: int, win_w: int) -> np.ndarray:
    """Sliding tile attention within each frame: q, k, v [T, H*W, C] ->
    out [T, H*W, C].  Each query attends to the keys of the tiles (tile x tile
    tokens) inside a window of win_h x win_w tokens (odd tile counts)
    centred on its own tile, cut off at the frame edge."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, N, C = q.shape
    assert N == H * W and k.shape == q.shape and v.shape == q.shape and C % heads == 0
    o = np.empty_like(q)
    rc = _load().oracle_sta_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(o), T, H, W, heads, C // heads,
                                      tile, win_h, win_w)
    if rc == -1:
        raise ValueError("bad STA arguments (sizes must be whole tiles, windows odd tile counts)")
    if rc != 0:
        raise RuntimeError(f"oracle_sta_attention failed ({rc})")
    return o


def draft_select(q, k, H: int, W: int, heads: int, region: int, keep: int) -> np.ndarray:
    """Draft attention's region selection: q, k [T, H*W, C] -> int32
    [T, heads, R, keep], R = (H/region)(W/region): per query region the
    `keep` key regions with the highest pooled-sketch scores (ties to the
    lower index), listed in ascending region index."""
    q, k = _f64(q), _f64(k)
    T, N, C = q.shape
    assert N == H * W and k.shape == q.shape and C % heads == 0
    R = (H // region) * (W // region) if region > 0 and H % region == 0 and W % region == 0 else 0
    sel = np.zeros((T, heads, max(R, 1), max(keep, 1)), dtype=np.int32)
    rc = _load().oracle_draft_select(_ptr(q), _ptr(k), T, H, W, heads, C // heads, region, keep,
                                     sel.ctypes.data_as(_ip))
    if rc == -1:
        raise ValueError("bad draft-attention arguments")
    if rc != 0:
        raise RuntimeError(f"oracle_draft_select failed ({rc})")
    return sel


def region_sparse_attention(q, k, v, H: int, W: int, heads: int, region: int, sel) -> np.ndarray:
    """Attention of every query region over the key regions sel lists
    ([T, heads, R, keep] int): q, k, v [T, H*W, C] -> out [T, H*W, C]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    sel = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
    T, N, C = q.shape
    assert N == H * W and k.shape == q.shape and v.shape == q.shape and C % heads == 0
    keep = sel.shape[-1]
    o = np.empty_like(q)
    rc = _load().oracle_region_sparse_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(o), T, H, W, heads,
                                                C // heads, region, keep, sel.ctypes.data_as(_ip))
    if rc == -1:
        raise ValueError("bad region-sparse attention arguments")
    if rc != 0:
        raise RuntimeError(f"oracle_region_sparse_attention failed ({rc})")
    return o


def draft_attention(q, k, v, H: int, W: int, heads: int, region: int, keep: int) -> np.ndarray:
    """Draft attention within each frame: the selection of draft_select, then
    region_sparse_attention under it."""
    return region_sparse_attention(q, k, v, H, W, heads, region, draft_select(q, k, H, W, heads, region, keep))


def edge_steps(steps: int, edge_pct: int = 15) -> int:
    e = int(_load().oracle_pab_edge_steps(steps, edge_pct))
    if e < 0:
        raise ValueError("bad schedule arguments")
    return e


def schedule(steps: int, range_: int, edge_pct: int = 15):
    """Per step: (is_compute [steps] int array, source step [steps] int array)."""
    is_compute = np.zeros(max(steps, 1), dtype=np.int32)
    source = np.zeros(max(steps, 1), dtype=np.int32)
    rc = _load().oracle_pab_schedule(steps, edge_pct, range_,
                                     is_compute.ctypes.data_as(_ip), source.ctypes.data_as(_ip))
    if rc != 0:
        raise ValueError("bad schedule arguments")
    return is_compute[:steps].copy(), source[:steps].copy()


def mse(a, b) -> float:
    """Mean over all elements of (a - b)^2, in double precision."""
    a, b = _f64(a).ravel(), _f64(b).ravel()
    assert a.shape == b.shape
    return float(_load().oracle_mse(_ptr(a), _ptr(b), a.size))


def layout(x: np.ndarray, to_temporal: bool) -> np.ndarray:
    """[T, N, C] -> [N, T, C] (to_temporal) or back; bytes moved unchanged."""
    x = np.ascontiguousarray(x)
    A, B, C = x.shape
    out = np.empty((B, A, C), dtype=x.dtype)
    T, N = (A, B) if to_temporal else (B, A)
    rc = _load().oracle_layout(1 if to_temporal else 0, x.ctypes.data, out.ctypes.data,
                               T, N, C, x.dtype.itemsize)
    if rc != 0:
        raise RuntimeError("oracle_layout failed")
    return out


def permute_blocks(x: np.ndarray, P: int, Q: int) -> np.ndarray:
    """x viewed as [P, Q, block, C] -> [Q, P, block, C]; bytes moved unchanged
    (sequence-parallel packing, PAB report, "Parallel")."""
    x = np.ascontiguousarray(x)
    C = x.shape[-1]
    block = x.size // (P * Q * C) if P * Q * C else 0
    assert P * Q * block * C == x.size
    out = np.empty((Q, P, block, C), dtype=x.dtype)
    rc = _load().oracle_permute_blocks(x.ctypes.data, out.ctypes.data, P, Q, block, C, x.dtype.itemsize)
    if rc != 0:
        raise RuntimeError("oracle_permute_blocks failed")
    return out
