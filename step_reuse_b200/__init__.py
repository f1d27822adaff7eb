"""Python binding of libpab.so -- the B200 (sm_100a) Pyramid Attention
Broadcast attention library.

Argument marshalling only: every step of the attention stack runs in the
library's CUDA kernels.  Tensors are torch CUDA tensors (PyTorch supplies the
device memory and the stream); the calls go through the C ABI declared in
include/pab.h with ctypes.  Importing this package fails loudly if
libpab.so has not been built (python step_reuse_b200/build.py); there is no
CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpab.so")

PAB_OK = 0
PAB_ERR_ARG = -1
PAB_ERR_STEP_ORDER = -2
PAB_ERR_NO_CACHE = -3
PAB_ERR_CUDA = -4
PAB_ERR_OOM = -5
PAB_ERR_UNSUPPORTED = -6

SPATIAL, TEMPORAL, CROSS = 0, 1, 2
KIND = {"spatial": SPATIAL, "temporal": TEMPORAL, "cross": CROSS}
BF16, FP32 = 0, 1

# every symbol include/pab.h declares
EXPORTS = (
    "pab_version", "pab_last_error_string", "pab_spatial_attention", "pab_temporal_attention",
    "pab_temporal_attention_sv", "pab_plan_set_temporal_view", "pab_sta_attention",
    "pab_plan_set_spatial_window", "pab_draft_workspace_bytes", "pab_draft_select",
    "pab_region_sparse_attention", "pab_plan_set_spatial_draft", "pab_permute_blocks",
    "pab_scatter_blocks", "pab_block_gemm", "pab_block_layer_norm", "pab_ipc_alloc", "pab_ipc_free", "pab_ipc_open", "pab_ipc_close",
    "pab_cross_attention", "pab_layout", "pab_attn_diff_mse", "pab_attn_diff_mse_async", "pab_attn_diff_mse_noalloc",
    "pab_device_errors", "pab_plan_create", "pab_plan_destroy", "pab_plan_reset",
    "pab_plan_prepare", "pab_plan_set_diff_mse", "pab_plan_set_diff_mse_stream", "pab_schedule_query", "pab_schedule_source", "pab_schedule_count",
    "pab_attention",
)


class PabError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


class pab_ranges(ctypes.Structure):
    _fields_ = [("spatial", ctypes.c_int), ("temporal", ctypes.c_int), ("cross", ctypes.c_int),
                ("edge_pct", ctypes.c_int)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python step_reuse_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
    sig = {
        "pab_version": ([], i),
        "pab_last_error_string": ([], ctypes.c_char_p),
        "pab_spatial_attention": ([vp, vp, vp, vp, i, i, i, i, vp], i),
        "pab_temporal_attention": ([vp, vp, vp, vp, i, i, i, i, vp], i),
        "pab_temporal_attention_sv": ([vp, vp, vp, vp, i, i, i, i, vp], i),
        "pab_plan_set_temporal_view": ([vp, i], i),
        "pab_sta_attention": ([vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp], i),
        "pab_plan_set_spatial_window": ([vp, i, i, i], i),
        "pab_draft_workspace_bytes": ([i, i, i, i, i, i, ctypes.POINTER(ll)], i),
        "pab_draft_select": ([vp, vp, i, i, i, i, i, i, i, vp, vp, ll, vp], i),
        "pab_region_sparse_attention": ([vp, vp, vp, vp, i, i, i, i, i, i, i, vp, vp], i),
        "pab_plan_set_spatial_draft": ([vp, i, i], i),
        "pab_cross_attention": ([vp, vp, vp, vp, ll, i, i, i, vp], i),
        "pab_layout": ([i, vp, vp, i, i, i, i, vp], i),
        "pab_permute_blocks": ([vp, vp, i, i, ll, i, i, vp], i),
        "pab_scatter_blocks": ([ctypes.POINTER(vp), ctypes.POINTER(vp), i, i, i, ll, i, i, ll, ll, i, vp], i),
        "pab_block_gemm": ([vp, vp, i, i, i, i, ctypes.POINTER(vp), i, vp, vp, vp], i),
        "pab_block_layer_norm": ([vp, ctypes.POINTER(vp), i, vp, ll, i, vp], i),
        "pab_ipc_alloc": ([ll, ctypes.POINTER(vp), ctypes.c_char_p], i),
        "pab_ipc_free": ([vp], i),
        "pab_ipc_open": ([ctypes.c_char_p, ctypes.POINTER(vp)], i),
        "pab_ipc_close": ([vp], i),
        "pab_attn_diff_mse": ([vp, vp, ll, i, ctypes.POINTER(ctypes.c_double), vp], i),
        "pab_attn_diff_mse_async": ([vp, vp, ll, i, vp, vp], i),
        "pab_attn_diff_mse_noalloc": ([vp, vp, ll, i, vp, vp], i),
        "pab_device_errors": ([i, ctypes.POINTER(ctypes.c_uint)], i),
        "pab_plan_create": ([i, i, i, i, i, i, i, pab_ranges, i, ctypes.POINTER(vp)], i),
        "pab_plan_destroy": ([vp], i),
        "pab_plan_reset": ([vp], i),
        "pab_plan_prepare": ([vp], i),
        "pab_plan_set_diff_mse": ([vp, vp], i),
        "pab_plan_set_diff_mse_stream": ([vp, i, vp], i),
        "pab_schedule_query": ([vp, i, i, ctypes.POINTER(i)], i),
        "pab_schedule_source": ([vp, i, i, ctypes.POINTER(i)], i),
        "pab_schedule_count": ([vp, i, ctypes.POINTER(i)], i),
        "pab_attention": ([vp, i, i, vp, vp, vp, ctypes.POINTER(vp), vp], i),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def _check(rc: int):
    if rc != PAB_OK:
        raise PabError(rc, lib.pab_last_error_string().decode(errors="replace"))


def _stream(stream=None):
    if stream is None:
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def version() -> int:
    return lib.pab_version()


def spatial_attention(q, k, v, heads: int, out=None, stream=None):
    """q, k, v: [T, N, C] bf16 CUDA tensors -> [T, N, C]."""
    T, N, C = q.shape
    out = torch.empty_like(q) if out is None else out
    _check(lib.pab_spatial_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), T, N, heads, C // heads,
                                     _stream(stream)))
    return out


def sta_attention(q, k, v, H: int, W: int, heads: int, tile: int = 16, win_h: int = 48, win_w: int = 48,
                  out=None, stream=None):
    """Sliding tile attention within each frame: q, k, v [T, H*W, C] bf16
    CUDA tensors -> [T, H*W, C]; tile x tile-token tiles, a win_h x win_w
    window (odd tile counts) centred on each query's tile, cut at the edge."""
    T, N, C = q.shape
    if N != H * W:
        raise ValueError(f"q has {N} tokens per frame, H*W = {H * W}")
    out = torch.empty_like(q) if out is None else out
    _check(lib.pab_sta_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), T, H, W, heads, C // heads,
                                 tile, win_h, win_w, _stream(stream)))
    return out


def draft_workspace_bytes(T: int, H: int, W: int, heads: int, d: int, region: int = 16) -> int:
    n = ctypes.c_longlong(0)
    _check(lib.pab_draft_workspace_bytes(T, H, W, heads, d, region, ctypes.byref(n)))
    return n.value


def draft_select(q, k, H: int, W: int, heads: int, keep: int, region: int = 16, sel=None, workspace=None,
                 stream=None):
    """Draft attention's region selection: q, k [T, H*W, C] bf16 CUDA tensors
    -> int32 [T, heads, R, keep] (per query region the keep key regions with
    the highest pooled-sketch scores, ascending)."""
    T, N, C = q.shape
    if N != H * W:
        raise ValueError(f"q has {N} tokens per frame, H*W = {H * W}")
    R = (H // region) * (W // region)
    if sel is None:
        sel = torch.empty((T, heads, R, keep), dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = torch.empty(draft_workspace_bytes(T, H, W, heads, C // heads, region),
                                dtype=torch.uint8, device=q.device)
    _check(lib.pab_draft_select(_ptr(q), _ptr(k), T, H, W, heads, C // heads, region, keep, _ptr(sel),
                                _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return sel


def region_sparse_attention(q, k, v, H: int, W: int, heads: int, sel, region: int = 16, out=None, stream=None):
    """Attention of every query region over the key regions sel
    ([T, heads, R, keep] int32 CUDA tensor) lists: q, k, v [T, H*W, C]."""
    T, N, C = q.shape
    if N != H * W:
        raise ValueError(f"q has {N} tokens per frame, H*W = {H * W}")
    if sel.dtype != torch.int32 or not sel.is_contiguous():
        raise ValueError("sel must be a contiguous int32 tensor")
    out = torch.empty_like(q) if out is None else out
    _check(lib.pab_region_sparse_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), T, H, W, heads, C // heads,
                                           region, sel.shape[-1], _ptr(sel), _stream(stream)))
    return out


def draft_attention(q, k, v, H: int, W: int, heads: int, keep: int, region: int = 16, stream=None):
    """Draft attention within each frame: draft_select then region_sparse_attention."""
    sel = draft_select(q, k, H, W, heads, keep, region, stream=stream)
    return region_sparse_attention(q, k, v, H, W, heads, sel, region, stream=stream)


def temporal_attention(q, k, v, heads: int, out=None, stream=None):
    """q, k, v: [N, T, C] bf16 CUDA tensors -> [N, T, C]."""
    N, T, C = q.shape
    out = torch.empty_like(q) if out is None else out
    _check(lib.pab_temporal_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), N, T, heads, C // heads,
                                      _stream(stream)))
    return out


def temporal_attention_sv(q, k, v, heads: int, out=None, stream=None):
    """Temporal attention on the spatial view: q, k, v [T, N, C] -> [T, N, C]."""
    T, N, C = q.shape
    out = torch.empty_like(q) if out is None else out
    _check(lib.pab_temporal_attention_sv(_ptr(q), _ptr(k), _ptr(v), _ptr(out), T, N, heads, C // heads,
                                         _stream(stream)))
    return out


def cross_attention(q, kt, vt, heads: int, out=None, stream=None):
    """q: [..., C] video tokens; kt, vt: [text_len, C] -> like q."""
    C = q.shape[-1]
    R = q.numel() // C
    out = torch.empty_like(q) if out is None else out
    _check(lib.pab_cross_attention(_ptr(q), _ptr(kt), _ptr(vt), _ptr(out), R, kt.shape[0], heads,
                                   C // heads, _stream(stream)))
    return out


def layout(x, to_temporal: bool, out=None, stream=None):
    """[T, N, C] -> [N, T, C] when to_temporal, else [N, T, C] -> [T, N, C]."""
    A, B, C = x.shape
    out = x.new_empty((B, A, C)) if out is None else out
    T, N = (A, B) if to_temporal else (B, A)
    _check(lib.pab_layout(1 if to_temporal else 0, _ptr(x), _ptr(out), T, N, C, _dtype_code(x),
                          _stream(stream)))
    return out


def permute_blocks(x, P: int, Q: int, out=None, stream=None):
    """x viewed as [P, Q, block_rows, C] -> out [Q, P, block_rows, C] (same
    total shape as x unless `out` gives one)."""
    C = x.shape[-1]
    block_rows = x.numel() // (P * Q * C) if P * Q * C else 0
    if P * Q * block_rows * C != x.numel():
        raise ValueError(f"{tuple(x.shape)} is not [{P}, {Q}, rows, {C}]")
    out = torch.empty((Q, P, block_rows, C), dtype=x.dtype, device=x.device) if out is None else out
    _check(lib.pab_permute_blocks(_ptr(x), _ptr(out), P, Q, block_rows, C, _dtype_code(x), _stream(stream)))
    return out


def scatter_blocks(srcs, dsts, G: int, P: int, block_rows: int, src_order: int, dst_offset_rows: int,
                   dst_stride_rows: int, stream=None):
    """One move of broadcast sequence parallelism's exchange: every source
    tensor in `srcs` (1..3, each P*G blocks of block_rows rows) has block
    (p, g) written to rows dst_offset_rows + p*dst_stride_rows.. of the
    g-th destination.  `dsts[t]` lists G destinations of tensor t, each a
    CUDA tensor or a raw device address (int) -- e.g. a peer GPU's buffer
    mapped with ipc_open."""
    nt = len(srcs)
    if nt < 1 or nt > 3 or len(dsts) != nt or any(len(d) != G for d in dsts):
        raise ValueError("need 1..3 sources, each with G destinations")
    C = srcs[0].shape[-1]
    for x in srcs:
        if x.dtype != srcs[0].dtype or x.shape[-1] != C or x.numel() != P * G * block_rows * C:
            raise ValueError(f"source {tuple(x.shape)} is not {P * G} blocks of [{block_rows}, {C}]")
    src_arr = (ctypes.c_void_p * nt)(*[x.data_ptr() for x in srcs])
    flat = [d if isinstance(d, int) else d.data_ptr() for row in dsts for d in row]
    dst_arr = (ctypes.c_void_p * len(flat))(*flat)
    _check(lib.pab_scatter_blocks(src_arr, dst_arr, nt, G, P, block_rows, C, src_order, dst_offset_rows,
                                  dst_stride_rows, _dtype_code(srcs[0]), _stream(stream)))


GEMM_STORE, GEMM_GELU, GEMM_RESID = 0, 1, 2


def block_gemm(A, B, epilogue=GEMM_STORE, outs=None, X=None, Y=None, stream=None):
    """A [M, K] @ B [K, N] (bf16 CUDA tensors) on the tensor cores with an
    epilogue: GEMM_STORE writes bf16 column blocks into `outs` (1..3 tensors
    of N / len(outs) columns each; new tensors when None), GEMM_GELU writes
    bf16 GELU(A B) into outs[0], GEMM_RESID adds A B into the fp32 tensor X
    (and writes bf16 A B into Y when given).  Returns the outputs."""
    M, K = A.shape
    N = B.shape[1]
    if epilogue == GEMM_RESID:
        if X is None or X.dtype != torch.float32:
            raise ValueError("GEMM_RESID needs an fp32 X")
        arr = (ctypes.c_void_p * 1)(None)
        _check(lib.pab_block_gemm(_ptr(A), _ptr(B), M, N, K, epilogue, arr, 0, _ptr(X), _ptr(Y), _stream(stream)))
        return X
    if outs is None:
        outs = [torch.empty((M, N), dtype=torch.bfloat16, device=A.device)]
    split = N // len(outs)
    arr = (ctypes.c_void_p * len(outs))(*[o.data_ptr() for o in outs])
    _check(lib.pab_block_gemm(_ptr(A), _ptr(B), M, N, K, epilogue, arr, split if len(outs) > 1 else 0, None, None,
                              _stream(stream)))
    return outs


def block_layer_norm(x, h=None, ys=(), norm=True, stream=None):
    """x += sum of the bf16 tensors in `ys` (written back into the fp32 x),
    then h = bf16(LayerNorm(x)) over the last dim when `norm`."""
    C = x.shape[-1]
    if norm and h is None:
        h = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    arr = (ctypes.c_void_p * max(1, len(ys)))(*[y.data_ptr() for y in ys])
    _check(lib.pab_block_layer_norm(_ptr(x), arr, len(ys), _ptr(h) if norm else None, x.numel() // C, C,
                                    _stream(stream)))
    return h


def ipc_alloc(nbytes: int):
    """(device address, 64-byte handle) of a new buffer that other processes
    of this node can map with ipc_open; release it with ipc_free."""
    ptr = ctypes.c_void_p()
    handle = ctypes.create_string_buffer(64)
    _check(lib.pab_ipc_alloc(nbytes, ctypes.byref(ptr), handle))
    return ptr.value, handle.raw


def ipc_free(ptr: int):
    _check(lib.pab_ipc_free(ctypes.c_void_p(ptr)))


def ipc_open(handle: bytes) -> int:
    """Map another process's ipc_alloc buffer into this process."""
    if len(handle) != 64:
        raise ValueError("IPC handles are 64 bytes")
    ptr = ctypes.c_void_p()
    _check(lib.pab_ipc_open(handle, ctypes.byref(ptr)))
    return ptr.value


def ipc_close(ptr: int):
    _check(lib.pab_ipc_close(ctypes.c_void_p(ptr)))


def ipc_tensor(shape, dtype, device):
    """A new CUDA tensor in a buffer the other processes of this node can map
    (ipc_open_tensor): (tensor, 64-byte handle, address for ipc_free)."""
    n = 1
    for x in shape:
        n *= int(x)
    ptr, handle = ipc_alloc(n * torch.tensor([], dtype=dtype).element_size())
    return _wrap(ptr, shape, dtype, device), handle, ptr


def ipc_open_tensor(handle: bytes, shape, dtype, device):
    """Another process's ipc_tensor mapped into this one: (tensor, address for
    ipc_close)."""
    ptr = ipc_open(handle)
    return _wrap(ptr, shape, dtype, device), ptr


def attn_diff_mse(a, b, stream=None) -> float:
    """mean((a - b)^2) over all elements, fp64; synchronises the stream."""
    assert a.shape == b.shape and a.dtype == b.dtype
    res = ctypes.c_double(0.0)
    _check(lib.pab_attn_diff_mse(_ptr(a), _ptr(b), a.numel(), _dtype_code(a), ctypes.byref(res),
                                 _stream(stream)))
    return res.value


def attn_diff_mse_async(a, b, result_dev, stream=None):
    """Writes mean((a - b)^2) into the fp64 device scalar `result_dev`."""
    assert a.shape == b.shape and a.dtype == b.dtype and result_dev.dtype == torch.float64
    _check(lib.pab_attn_diff_mse_async(_ptr(a), _ptr(b), a.numel(), _dtype_code(a),
                                       ctypes.c_void_p(result_dev.data_ptr()), _stream(stream)))
    return result_dev


def device_errors(clear: bool = True) -> int:
    flags = ctypes.c_uint(0)
    _check(lib.pab_device_errors(1 if clear else 0, ctypes.byref(flags)))
    return flags.value


class _DeviceView:
    """__cuda_array_interface__ wrapper so torch can view library-owned memory."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (ptr, False), "version": 3, "strides": None}


def _wrap(ptr: int, shape, dtype, device) -> torch.Tensor:
    if dtype == torch.bfloat16:
        t = torch.as_tensor(_DeviceView(ptr, shape, "<i2"), device=device)
        return t.view(torch.bfloat16)
    return torch.as_tensor(_DeviceView(ptr, shape, "<f4"), device=device)


class Plan:
    """A PAB plan: the broadcast schedule of one sampling run plus the
    broadcast cache (two output slots per kind, owned by the library).

    Tensors returned by attention() VIEW library memory: they stay valid until
    the second following compute of the same kind, reset() or close()."""

    def __init__(self, T, H, W, heads, d, text_len, steps, ranges, dtype=torch.bfloat16,
                 edge_pct: int = 15):
        self.T, self.H, self.W, self.heads, self.d = T, H, W, heads, d
        self.N, self.C, self.text_len, self.steps = H * W, heads * d, text_len, steps
        self.dtype = dtype
        r = pab_ranges(int(ranges[0]), int(ranges[1]), int(ranges[2]), int(edge_pct))
        h = ctypes.c_void_p()
        _check(lib.pab_plan_create(T, H, W, heads, d, text_len, steps, r,
                                   FP32 if dtype == torch.float32 else BF16, ctypes.byref(h)))
        self._h = h

    def close(self):
        if self._h:
            lib.pab_plan_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def reset(self):
        _check(lib.pab_plan_reset(self._h))

    def set_temporal_view(self, spatial_view: bool):
        """True: TEMPORAL takes and returns [T, N, C] instead of [N, T, C]."""
        _check(lib.pab_plan_set_temporal_view(self._h, 1 if spatial_view else 0))
        self.temporal_sv = bool(spatial_view)

    def set_spatial_window(self, tile: int = 16, win_h: int = 0, win_w: int = 0):
        """Spatial computes become sliding tile attention with this window
        (win_h = win_w = 0: full attention within the frame again)."""
        _check(lib.pab_plan_set_spatial_window(self._h, tile, win_h, win_w))

    def set_spatial_draft(self, region: int = 16, keep: int = 0):
        """Spatial computes become draft attention keeping `keep` key regions
        per query region (keep = 0: full attention within the frame again)."""
        _check(lib.pab_plan_set_spatial_draft(self._h, region, keep))

    def prepare(self):
        _check(lib.pab_plan_prepare(self._h))

    def set_diff_mse(self, results=None):
        """results: a float64 CUDA tensor of 3 * steps elements ([3, steps]);
        every compute after a kind's first writes MSE(out, previous compute)
        at [kind, step] (the MSE kernel runs on the attention's stream right
        after it).  None disables."""
        if results is not None:
            if results.dtype != torch.float64 or results.numel() != 3 * self.steps or not results.is_contiguous():
                raise ValueError(f"need a contiguous float64 tensor of 3 * {self.steps} elements")
            self._mse_results = results  # keep the memory alive while the plan writes to it
            _check(lib.pab_plan_set_diff_mse(self._h, ctypes.c_void_p(results.data_ptr())))
        else:
            _check(lib.pab_plan_set_diff_mse(self._h, None))
            self._mse_results = None

    def set_diff_mse_stream(self, stream=None):
        """Run the plan's MSE launches on `stream` (a torch.cuda.Stream), where
        they overlap the following attention computes; the table is complete
        once that stream has drained.  None: in line on the compute stream."""
        if stream is None:
            _check(lib.pab_plan_set_diff_mse_stream(self._h, 0, None))
            self._mse_stream = None
        else:
            self._mse_stream = stream  # keep the stream alive while the plan launches on it
            _check(lib.pab_plan_set_diff_mse_stream(self._h, 1, _stream(stream)))

    def is_compute(self, kind, step: int) -> bool:
        kind = KIND.get(kind, kind)
        out = ctypes.c_int(0)
        _check(lib.pab_schedule_query(self._h, kind, step, ctypes.byref(out)))
        return bool(out.value)

    def source(self, kind, step: int) -> int:
        kind = KIND.get(kind, kind)
        out = ctypes.c_int(0)
        _check(lib.pab_schedule_source(self._h, kind, step, ctypes.byref(out)))
        return out.value

    def count(self, kind) -> int:
        kind = KIND.get(kind, kind)
        out = ctypes.c_int(0)
        _check(lib.pab_schedule_count(self._h, kind, ctypes.byref(out)))
        return out.value

    def attention_ptr(self, kind, step: int, q=None, k=None, v=None, stream=None) -> int:
        """Raw device pointer of the step's output (compute or broadcast hit)."""
        kind = KIND.get(kind, kind)
        out = ctypes.c_void_p()
        _check(lib.pab_attention(self._h, kind, step, _ptr(q), _ptr(k), _ptr(v), ctypes.byref(out),
                                 _stream(stream)))
        return out.value

    def attention(self, kind, step: int, q=None, k=None, v=None, stream=None) -> torch.Tensor:
        kind = KIND.get(kind, kind)
        ptr = self.attention_ptr(kind, step, q, k, v, stream)
        tshape = (self.T, self.N, self.C) if getattr(self, "temporal_sv", False) else (self.N, self.T, self.C)
        shape = {SPATIAL: (self.T, self.N, self.C), TEMPORAL: tshape,
                 CROSS: (self.T * self.N, self.C)}[kind]
        dev = q.device if q is not None else torch.device("cuda", torch.cuda.current_device())
        return _wrap(ptr, shape, self.dtype, dev)
