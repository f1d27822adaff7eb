"""The dense kernels of the DiT block around the attention kinds (PAB report,
"Implementation": attention modules inside DiT blocks between layer norms,
projections and an MLP): the tensor-core GEMM with its three epilogues and
the row layer norm, against float64 references written from the
definitions (numpy matmul on the same bf16 inputs, the oracle's layer norm
and tanh GELU).

Tolerances: a bf16 output is rounded once (relative 2^-9), so relative L2
<= 4e-3 and max-abs <= 2^-7 of the largest magnitude; an fp32 residual sum
accumulates over K in fp32 (relative L2 <= 1e-5).
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import dit as odit

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pab():
    import step_reuse_b200
    assert torch.cuda.is_available()
    return step_reuse_b200


def _bf(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (scale * torch.randn(shape, generator=g)).to(torch.bfloat16)


def _f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _rel(got, want):
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


@pytest.mark.parametrize("M,K,N,nout", [
    (256, 64, 192, 3),      # the tiny block's q | k | v projection
    (25440, 1152, 3456, 3),  # 480p: q | k | v of 16 frames x 1590 tokens
    (1000, 288, 864, 3),     # K tail (288 = 4.5 x 64), ragged M
    (120, 1152, 2304, 2),    # the text's k | v projection
    (333, 512, 256, 1),      # one output, N a multiple of 256
    (129, 96, 96, 1),        # one 128-row tile and a row, a narrow N
])
def test_gemm_store_split(pab, M, K, N, nout):
    A, B = _bf((M, K), 1), _bf((K, N), 2, scale=K ** -0.5)
    outs = [torch.full((M, N // nout), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(nout)]
    pab.block_gemm(A.cuda(), B.cuda(), outs=outs)
    torch.cuda.synchronize()
    want = _f64(A) @ _f64(B)
    got = np.concatenate([_f64(o) for o in outs], axis=1)
    assert np.isfinite(got).all()
    assert _rel(got, want) <= 4e-3
    assert np.abs(got - want).max() <= 2 ** -7 * np.abs(want).max()
    assert pab.device_errors(clear=True) == 0


@pytest.mark.parametrize("M,K,N", [(25440, 1152, 4608), (300, 288, 1152), (64, 64, 256)])
def test_gemm_gelu(pab, M, K, N):
    A, B = _bf((M, K), 3), _bf((K, N), 4, scale=K ** -0.5)
    out = pab.block_gemm(A.cuda(), B.cuda(), pab.GEMM_GELU)[0]
    torch.cuda.synchronize()
    want = odit.gelu_tanh(_f64(A) @ _f64(B))
    got = _f64(out)
    assert _rel(got, want) <= 4e-3
    assert np.abs(got - want).max() <= 2 ** -7 * np.abs(want).max()


@pytest.mark.parametrize("M,K,N,with_y", [(25440, 4608, 1152, False), (25440, 1152, 1152, True),
                                          (777, 288, 288, True), (5, 64, 32, True)])
def test_gemm_residual(pab, M, K, N, with_y):
    A, B = _bf((M, K), 5), _bf((K, N), 6, scale=K ** -0.5)
    g = torch.Generator().manual_seed(7)
    X0 = torch.randn((M, N), generator=g)
    X = X0.clone().cuda()
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") if with_y else None
    pab.block_gemm(A.cuda(), B.cuda(), pab.GEMM_RESID, X=X, Y=Y)
    torch.cuda.synchronize()
    prod = _f64(A) @ _f64(B)
    assert _rel(_f64(X) - X0.double().numpy(), prod) <= 1e-5
    if with_y:
        assert _rel(_f64(Y), prod) <= 4e-3


@pytest.mark.parametrize("rows,C,ny", [(25440, 1152, 0), (25440, 1152, 3), (1000, 288, 1), (7, 3072, 2),
                                       (33, 64, 0)])
def test_layer_norm_with_adds(pab, rows, C, ny):
    g = torch.Generator().manual_seed(rows + C)
    x0 = 3.0 * torch.randn((rows, C), generator=g) + 0.5
    ys = [_bf((rows, C), 10 + j) for j in range(ny)]
    x = x0.clone().cuda()
    h = pab.block_layer_norm(x, ys=[y.cuda() for y in ys])
    torch.cuda.synchronize()
    want_x = x0.clone()
    for y in ys:  # added in order, in fp32: the same sums bit for bit
        want_x += y.float()
    assert torch.equal(x.cpu(), want_x)
    want_h = odit.layer_norm(want_x.double().numpy())
    got = _f64(h)
    assert _rel(got, want_h) <= 4e-3
    assert np.abs(got - want_h).max() <= 2e-2


def test_layer_norm_adds_only(pab):
    x0 = torch.randn((100, 256))
    y = _bf((100, 256), 3)
    x = x0.clone().cuda()
    assert pab.block_layer_norm(x, ys=[y.cuda()], norm=False) is None
    torch.cuda.synchronize()
    assert torch.equal(x.cpu(), x0 + y.float())


def test_block_argument_errors(pab):
    lib = pab.lib
    a = torch.zeros((128, 64), dtype=torch.bfloat16, device="cuda")
    arr = (ctypes.c_void_p * 3)(a.data_ptr(), a.data_ptr(), a.data_ptr())
    p = ctypes.c_void_p(a.data_ptr())
    assert lib.pab_block_gemm(p, p, 128, 64, 60, 0, arr, 0, None, None, None) == pab.PAB_ERR_UNSUPPORTED  # K % 8
    assert lib.pab_block_gemm(p, p, 128, 40, 64, 0, arr, 0, None, None, None) == pab.PAB_ERR_UNSUPPORTED  # N % 32
    assert lib.pab_block_gemm(p, p, 128, 64, 64, 3, arr, 0, None, None, None) == pab.PAB_ERR_ARG
    assert lib.pab_block_gemm(p, p, 128, 128, 64, 0, arr, 48, None, None, None) == pab.PAB_ERR_ARG  # split % 32
    assert lib.pab_block_gemm(p, p, 128, 64, 64, 2, arr, 0, None, None, None) == pab.PAB_ERR_ARG  # no X
    assert lib.pab_block_layer_norm(None, None, 0, None, 10, 64, None) == pab.PAB_ERR_ARG
    assert lib.pab_block_layer_norm(p, None, 4, None, 10, 64, None) == pab.PAB_ERR_ARG
