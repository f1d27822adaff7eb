"""GPU parity of the stateless kernels against the fp64 oracle, through the
C ABI: spatial / temporal / cross attention (PAB report, "Implementation"),
the layout change between the spatial and temporal views, and the
attention-difference MSE (Fig. 1).  Sizes span several tiles with ragged
tails; edge cases cover single keys, single rows, odd head dims and the
documented maxima."""
import numpy as np
import pytest
import torch

from parity import MSE_REL, assert_attn_close, check_guards, guarded_empty, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pab():
    import step_reuse_b200
    assert torch.cuda.is_available()
    return step_reuse_b200


def randn(shape, seed, dtype=torch.bfloat16, scale=1.0):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (scale * torch.randn(shape, generator=g)).to(dtype).cuda()


def no_device_errors(pab):
    torch.cuda.synchronize()
    assert pab.device_errors(clear=True) == 0


# ------------------------------------------------------------------ spatial
@pytest.mark.parametrize("T,N,heads,d", [
    (2, 300, 2, 64),     # 3 query tiles, ragged 44-row tail
    (1, 1590, 2, 72),    # the 480p frame length, d = 72 (d % 16 == 8)
    (1, 777, 1, 128),
    (3, 129, 4, 32),     # one row past a tile
    (2, 1, 2, 64),       # a single token
    (1, 65, 3, 8),       # smallest head dim
    (1, 200, 2, 120),
    (2, 64, 2, 16),
])
def test_spatial_parity(pab, oracle_mod, T, N, heads, d):
    C = heads * d
    q, k, v = (randn((T, N, C), s) for s in (1, 2, 3))
    base, out = guarded_empty((T, N, C), torch.bfloat16)
    pab.spatial_attention(q, k, v, heads, out=out)
    want = oracle_mod.spatial_attention(to_f64(q), to_f64(k), to_f64(v), heads)
    assert_attn_close(out, want, f"spatial T={T} N={N} h={heads} d={d}")
    check_guards(base)
    no_device_errors(pab)


def test_spatial_large_scores(pab, oracle_mod):
    """Peaked softmax (scores up to ~100): the online max must keep it stable."""
    T, N, heads, d = 1, 333, 2, 64
    C = heads * d
    q, k, v = randn((T, N, C), 4, scale=3.0), randn((T, N, C), 5, scale=3.0), randn((T, N, C), 6)
    out = pab.spatial_attention(q, k, v, heads)
    want = oracle_mod.spatial_attention(to_f64(q), to_f64(k), to_f64(v), heads)
    assert_attn_close(out, want, "spatial peaked")


# ------------------------------------------------------------------ temporal
@pytest.mark.parametrize("N,T,heads,d", [
    (37, 16, 16, 72),   # 480p-like T and d
    (50, 24, 4, 128),   # 720p-like
    (20, 64, 16, 64),   # temporal-heavy-like
    (33, 4, 2, 32),     # tiny-like
    (9, 1, 2, 64),      # a single frame: output = v
    (11, 17, 3, 40),    # ragged key block
    (7, 100, 2, 56),
    (5, 128, 2, 64),    # documented maximum T
    (300, 16, 1, 8),
])
def test_temporal_parity(pab, oracle_mod, N, T, heads, d):
    C = heads * d
    q, k, v = (randn((N, T, C), s) for s in (11, 12, 13))
    base, out = guarded_empty((N, T, C), torch.bfloat16)
    pab.temporal_attention(q, k, v, heads, out=out)
    want = oracle_mod.temporal_attention(to_f64(q), to_f64(k), to_f64(v), heads)
    assert_attn_close(out, want, f"temporal N={N} T={T} h={heads} d={d}")
    check_guards(base)
    if T == 1:
        assert torch.equal(out.view(torch.int16), v.view(torch.int16))


# ------------------------------------------------------------------ cross
@pytest.mark.parametrize("R,Lt,heads,d", [
    (1000, 120, 16, 72),  # 480p text length, ragged rows
    (700, 256, 4, 128),   # 720p text length (4 key tiles of 64)
    (333, 16, 2, 32),
    (129, 1, 2, 64),      # a single text token: output = v row
    (77, 512, 2, 64),     # documented maximum text_len
    (64, 300, 3, 24),
    (5000, 120, 16, 72),  # 640 query tiles: several per CTA, heads change inside a CTA's run
    (100, 64, 300, 8),    # one query tile per head: the head changes at every tile
    (25440, 120, 4, 72),  # a 480p frame stack's rows, 4 heads
    (257, 100, 2, 112),   # d % 16 == 0 at the largest head dim whose ones column fits O (N = 128)
    (130, 128, 3, 96),    # d % 16 == 0: the row-sum column in an extra 16-column chunk; full 128 keys
    (300, 90, 2, 128),    # d = 128 with a short text: the general flash kernel
])
def test_cross_parity(pab, oracle_mod, R, Lt, heads, d):
    C = heads * d
    q = randn((R, C), 21)
    kt, vt = randn((Lt, C), 22), randn((Lt, C), 23)
    base, out = guarded_empty((R, C), torch.bfloat16)
    pab.cross_attention(q, kt, vt, heads, out=out)
    want = oracle_mod.cross_attention(to_f64(q), to_f64(kt), to_f64(vt), heads)
    assert_attn_close(out, want, f"cross R={R} Lt={Lt} h={heads} d={d}")
    check_guards(base)
    if Lt == 1:
        want1 = vt.expand(R, C).contiguous()
        bad = (out.view(torch.int16) != want1.view(torch.int16)).nonzero()
        assert bad.numel() == 0, (f"{bad.shape[0]} elements differ; first {bad[:8].tolist()}; "
                                  f"got {out[bad[:4, 0], bad[:4, 1]].tolist()} want {want1[bad[:4, 0], bad[:4, 1]].tolist()}")


@pytest.mark.parametrize("R,Lt,heads,d", [
    (86400, 256, 24, 128),  # 720p: every video token against 256 text tokens (the flash kernel)
    (76800, 120, 16, 64),   # temporal-heavy: cross_tc at d = 64
])
def test_cross_full_size_sampled(pab, oracle_mod, R, Lt, heads, d):
    """Full-size cross attention, checked on 1024 sampled query rows (rows
    are independent, so the oracle of a row subset is the subset of the
    oracle's output), spread over the whole range including the last row."""
    C = heads * d
    q = randn((R, C), 24)
    kt, vt = randn((Lt, C), 25), randn((Lt, C), 26)
    base, out = guarded_empty((R, C), torch.bfloat16)
    pab.cross_attention(q, kt, vt, heads, out=out)
    rows = torch.cat([torch.randperm(R - 1, generator=torch.Generator().manual_seed(27))[:1023],
                      torch.tensor([R - 1])])
    want = oracle_mod.cross_attention(to_f64(q[rows.cuda()]), to_f64(kt), to_f64(vt), heads)
    assert_attn_close(out[rows.cuda()], want, f"cross full size R={R} Lt={Lt} h={heads} d={d}")
    check_guards(base)


def test_cross_row_order_is_kept(pab):
    R, Lt, heads, d = 500, 120, 4, 64
    C = heads * d
    q, kt, vt = randn((R, C), 31), randn((Lt, C), 32), randn((Lt, C), 33)
    a = pab.cross_attention(q, kt, vt, heads)
    perm = torch.randperm(R, generator=torch.Generator().manual_seed(0)).cuda()
    b = pab.cross_attention(q[perm].contiguous(), kt, vt, heads)
    assert torch.equal(a[perm], b)


# ------------------------------------------------------------------ layout
@pytest.mark.parametrize("T,N,C,dtype", [
    (16, 1590, 1152, torch.bfloat16),
    (24, 333, 3072, torch.bfloat16),
    (64, 120, 1024, torch.bfloat16),
    (4, 64, 64, torch.float32),
    (3, 5, 8, torch.bfloat16),
    (1, 7, 24, torch.bfloat16),
    (7, 1, 4, torch.float32),
])
def test_layout_bit_exact(pab, oracle_mod, T, N, C, dtype):
    x = randn((T, N, C), 41, dtype=dtype)
    base, y = guarded_empty((N, T, C), dtype)
    pab.layout(x, to_temporal=True, out=y)
    want = oracle_mod.layout(x.view(torch.int16 if dtype == torch.bfloat16 else torch.int32).cpu().numpy(), True)
    got = y.view(torch.int16 if dtype == torch.bfloat16 else torch.int32).cpu().numpy()
    np.testing.assert_array_equal(got, want)
    check_guards(base)
    z = pab.layout(y, to_temporal=False)
    assert torch.equal(z.view(torch.int16), x.view(torch.int16))
    no_device_errors(pab)


# ------------------------------------------------------------------ MSE
@pytest.mark.parametrize("n,dtype", [
    (0, torch.bfloat16), (1, torch.bfloat16), (7, torch.bfloat16), (8, torch.float32),
    (1000003, torch.bfloat16), (29306880, torch.bfloat16), (123457, torch.float32),
])
def test_mse_parity(pab, oracle_mod, n, dtype):
    a = randn((n,), 51, dtype=dtype)
    b = randn((n,), 52, dtype=dtype, scale=0.5)
    got = pab.attn_diff_mse(a, b)
    want = oracle_mod.mse(to_f64(a), to_f64(b))
    if n == 0:
        assert got == 0.0
    else:
        assert abs(got - want) <= MSE_REL * abs(want), (got, want)
    # deterministic: bitwise identical on repeat, sync and async agree
    assert pab.attn_diff_mse(a, b) == got
    r = torch.zeros(1, dtype=torch.float64, device="cuda")
    pab.attn_diff_mse_async(a, b, r)
    assert r.item() == got


def test_mse_special_cases(pab):
    a = randn((1 << 20,), 61)
    assert pab.attn_diff_mse(a, a) == 0.0
    # exact: binary fractions in bf16, c a power of two
    ints = torch.randint(-64, 64, (1 << 16,), generator=torch.Generator().manual_seed(1))
    x = (ints.float() / 8).to(torch.bfloat16).cuda()
    y = (x.float() + 0.25).to(torch.bfloat16)
    assert pab.attn_diff_mse(y, x) == 0.0625


# ------------------------------------------------------------------ temporal on the spatial view
@pytest.mark.parametrize("T,N,heads,d", [(16, 37, 16, 72), (24, 50, 4, 128), (64, 20, 16, 64), (4, 33, 2, 32),
                                         (1, 9, 2, 64), (17, 11, 3, 40)])
def test_temporal_spatial_view(pab, oracle_mod, T, N, heads, d):
    """[T, N, C] in and out, no layout change: bit-identical to permuting,
    running the temporal-view kernel and permuting back; and oracle parity."""
    C = heads * d
    q, k, v = (randn((T, N, C), s) for s in (71, 72, 73))
    base, out = guarded_empty((T, N, C), torch.bfloat16)
    pab.temporal_attention_sv(q, k, v, heads, out=out)
    check_guards(base)
    tv = [x.permute(1, 0, 2).contiguous() for x in (q, k, v)]
    ref = pab.temporal_attention(*tv, heads).permute(1, 0, 2).contiguous()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    want = oracle_mod.temporal_attention(*(np.transpose(to_f64(x), (1, 0, 2)) for x in (q, k, v)), heads)
    assert_attn_close(out, np.transpose(want, (1, 0, 2)), f"temporal_sv T={T} N={N} h={heads} d={d}")
    no_device_errors(pab)
