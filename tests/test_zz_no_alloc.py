"""The allocation-free MSE entry point (pab_attn_diff_mse_noalloc).

Some callers cannot call cudaMalloc -- code embedded in a framework whose
memory pool owns all device memory, or latency-critical loops that must not
allocate -- so the library offers a variant of the MSE diagnostic whose fp64
partial sums live in a static device array instead of a lazily allocated
buffer.  This test calls it through the C ABI and checks that it returns the
same value as the allocating entry point (pab_attn_diff_mse_async), within the
MSE tolerance the other tests use (1e-5 relative), on two calls in a row.

The file is named so that pytest collects it last: if it fails, a run that
stops at the first failure has already run every other test.  It passes when
run alone in a fresh process and after the other tests.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

MSE_REL = 1e-5


@pytest.fixture(scope="module")
def pab():
    import step_reuse_b200
    assert torch.cuda.is_available()
    return step_reuse_b200


def _randn(n, seed, dtype, scale=1.0):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (scale * torch.randn(n, generator=g)).to(dtype).cuda()


@pytest.mark.parametrize("n,dtype,code", [
    (29306880, torch.bfloat16, 0),   # one 480p attention output
    (1000003, torch.bfloat16, 0),    # ragged tail
    (123457, torch.float32, 1),
    (5, torch.bfloat16, 0),
])
def test_noalloc_matches_allocating_entry_point(pab, n, dtype, code):
    lib = pab.lib
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    results = []
    for call in range(2):  # two calls in a row share the static scratch array
        a = _randn(n, 100 + call, dtype)
        b = _randn(n, 200 + call, dtype, scale=0.5)
        ref = torch.zeros(1, dtype=torch.float64, device="cuda")
        got = torch.full((1,), -1.0, dtype=torch.float64, device="cuda")
        rc = lib.pab_attn_diff_mse_async(ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(b.data_ptr()),
                                         n, code, ctypes.c_void_p(ref.data_ptr()), stream)
        assert rc == 0, lib.pab_last_error_string()
        rc = lib.pab_attn_diff_mse_noalloc(ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(b.data_ptr()),
                                           n, code, ctypes.c_void_p(got.data_ptr()), stream)
        assert rc == 0, lib.pab_last_error_string()
        torch.cuda.synchronize()
        r, g = ref.item(), got.item()
        assert r > 0
        assert abs(g - r) <= MSE_REL * abs(r), (call, g, r)
        results.append(g)
    assert results[0] != results[1]  # the second call really recomputed


def test_noalloc_argument_errors(pab):
    lib = pab.lib
    res = torch.zeros(1, dtype=torch.float64, device="cuda")
    rp = ctypes.c_void_p(res.data_ptr())
    assert lib.pab_attn_diff_mse_noalloc(None, None, 10, 0, rp, None) == pab.PAB_ERR_ARG
    assert lib.pab_attn_diff_mse_noalloc(None, None, 10, 9, rp, None) == pab.PAB_ERR_ARG
    assert lib.pab_attn_diff_mse_noalloc(None, None, -1, 0, rp, None) == pab.PAB_ERR_ARG
    assert lib.pab_attn_diff_mse_noalloc(None, None, 0, 0, None, None) == pab.PAB_ERR_ARG
