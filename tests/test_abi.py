"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/pab.h declares, and its PAB schedule and argument
checks behave as documented.  The schedule is compared with the oracle's
step-by-step walk (PAB report, "Implementation" / Fig. 2)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names.update(re.findall(r"\b(pab_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def pab():
    import step_reuse_b200
    return step_reuse_b200


def test_library_exports_every_declared_symbol(pab):
    declared = header_functions()
    assert len(declared) >= 15
    raw = ctypes.CDLL(pab.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name
    assert set(pab.EXPORTS) == declared
    assert pab.version() >= 1


def test_library_has_sm100a_code_only():
    """The build targets sm_100a only (no PTX / other arch fallbacks)."""
    src = open(os.path.join(ROOT, "step_reuse_b200", "build.py")).read()
    assert "arch=compute_100a,code=sm_100a" in src
    assert "sm_90" not in src and "compute_90" not in src


@pytest.mark.parametrize("name", ["tiny", "480p", "720p", "temporal_heavy", "sweep"])
def test_schedule_matches_oracle(pab, oracle_mod, name):
    from synth import WORKLOADS
    w = WORKLOADS[name]
    range_sets = w.extra_ranges or (w.ranges,)
    for ranges in range_sets:
        plan = pab.Plan(w.T, w.H, w.W, w.heads, w.d, w.text_len, w.steps, ranges)
        for kind, r in zip(("spatial", "temporal", "cross"), ranges):
            comp, src = oracle_mod.schedule(w.steps, r)
            got = [plan.is_compute(kind, i) for i in range(w.steps)]
            assert got == [bool(c) for c in comp], (name, ranges, kind)
            assert [plan.source(kind, i) for i in range(w.steps)] == list(src)
            assert plan.count(kind) == int(comp.sum())
        plan.close()


def test_schedule_exhaustive_small(pab, oracle_mod):
    for steps in range(1, 61):
        for r in (1, 2, 3, 5, 7):
            plan = pab.Plan(2, 2, 2, 1, 8, 4, steps, (r, r, r))
            comp, src = oracle_mod.schedule(steps, r)
            assert [plan.is_compute(0, i) for i in range(steps)] == [bool(c) for c in comp]
            assert [plan.source(2, i) for i in range(steps)] == list(src)
            plan.close()


def test_edge_pct_parameter(pab, oracle_mod):
    for edge in (0, 5, 15, 25, 50, -1):
        plan = pab.Plan(2, 2, 2, 1, 8, 4, 40, (3, 3, 3), edge_pct=edge)
        # a negative share selects the default 15%; 0 means no edge steps
        comp, _ = oracle_mod.schedule(40, 3, edge_pct=15 if edge < 0 else edge)
        assert [plan.is_compute(1, i) for i in range(40)] == [bool(c) for c in comp]
        plan.close()


def test_argument_errors(pab):
    P = pab.Plan
    with pytest.raises(pab.PabError) as e:
        P(4, 8, 8, 2, 30, 16, 10, (2, 3, 4))  # d % 8 != 0
    assert e.value.code == pab.PAB_ERR_UNSUPPORTED
    with pytest.raises(pab.PabError) as e:
        P(4, 8, 8, 2, 32, 16, 10, (0, 3, 4))
    assert e.value.code == pab.PAB_ERR_ARG
    with pytest.raises(pab.PabError) as e:
        P(4, 8, 8, 2, 32, 16, 0, (2, 3, 4))
    assert e.value.code == pab.PAB_ERR_ARG
    with pytest.raises(pab.PabError) as e:
        P(200, 8, 8, 2, 32, 16, 10, (2, 3, 4))  # T > 128
    assert e.value.code == pab.PAB_ERR_UNSUPPORTED
    with pytest.raises(pab.PabError) as e:
        P(4, 8, 8, 2, 32, 0, 10, (2, 3, 4))
    assert e.value.code == pab.PAB_ERR_UNSUPPORTED
    with pytest.raises(pab.PabError) as e:
        P(4, 8, 8, 2, 32, 16, 10, (2, 3, 4), edge_pct=60)
    assert e.value.code == pab.PAB_ERR_ARG
    plan = P(4, 8, 8, 2, 32, 16, 10, (2, 3, 4))
    with pytest.raises(pab.PabError) as e:
        plan.is_compute(3, 0)
    assert e.value.code == pab.PAB_ERR_ARG
    with pytest.raises(pab.PabError) as e:
        plan.is_compute(0, 10)
    assert e.value.code == pab.PAB_ERR_ARG
    plan.close()


def test_hit_before_compute_and_step_order(pab):
    """Host-side cache rules, exercised on broadcast steps (no device work)."""
    plan = pab.Plan(4, 8, 8, 2, 32, 16, 10, (2, 3, 4))
    assert not plan.is_compute("spatial", 3)
    with pytest.raises(pab.PabError) as e:
        plan.attention_ptr("spatial", 3)  # hit, but step 2 was never computed
    assert e.value.code == pab.PAB_ERR_NO_CACHE
    with pytest.raises(pab.PabError) as e:
        plan.attention_ptr("spatial", 3)  # the failed call did not advance the order
    assert e.value.code == pab.PAB_ERR_NO_CACHE
    plan.reset()
    plan.close()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_compute_without_device_fails_loudly(pab):
    """No GPU: a compute step reports PAB_ERR_CUDA instead of falling back."""
    plan = pab.Plan(4, 8, 8, 2, 32, 16, 10, (2, 3, 4))
    buf = ctypes.create_string_buffer(1 << 16)
    addr = (ctypes.addressof(buf) + 15) // 16 * 16
    out = ctypes.c_void_p()
    rc = pab.lib.pab_attention(plan._h, 0, 0, ctypes.c_void_p(addr), ctypes.c_void_p(addr),
                               ctypes.c_void_p(addr), ctypes.byref(out), None)
    assert rc in (pab.PAB_ERR_CUDA, pab.PAB_ERR_OOM)
    assert pab.lib.pab_last_error_string()
    with pytest.raises(pab.PabError) as e:
        plan.prepare()
    assert e.value.code in (pab.PAB_ERR_CUDA, pab.PAB_ERR_OOM)
    plan.close()
    res = ctypes.c_double()
    rc = pab.lib.pab_attn_diff_mse(ctypes.c_void_p(addr), ctypes.c_void_p(addr), 64, 0,
                                   ctypes.byref(res), None)
    assert rc in (pab.PAB_ERR_CUDA, pab.PAB_ERR_OOM)


def test_stateless_argument_checks(pab):
    lib = pab.lib
    vp = ctypes.c_void_p
    assert lib.pab_spatial_attention(None, None, None, None, 1, 16, 2, 32, None) == pab.PAB_ERR_ARG
    assert lib.pab_spatial_attention(None, None, None, None, 1, 16, 2, 36, None) == pab.PAB_ERR_UNSUPPORTED
    assert lib.pab_temporal_attention(None, None, None, None, 16, 200, 2, 32, None) == pab.PAB_ERR_UNSUPPORTED
    assert lib.pab_cross_attention(None, None, None, None, 10, 0, 2, 32, None) == pab.PAB_ERR_UNSUPPORTED
    assert lib.pab_cross_attention(None, None, None, None, 10, 600, 2, 32, None) == pab.PAB_ERR_UNSUPPORTED
    # empty problems are no-ops
    assert lib.pab_spatial_attention(None, None, None, None, 0, 16, 2, 32, None) == pab.PAB_OK
    assert lib.pab_layout(1, None, None, 4, 0, 64, 0, None) == pab.PAB_OK
    # misaligned pointers
    assert lib.pab_layout(1, vp(8), vp(1 << 20), 4, 4, 64, 0, None) == pab.PAB_ERR_ARG
    assert lib.pab_layout(1, vp(1 << 20), vp(1 << 21), 4, 4, 60, 0, None) == pab.PAB_ERR_UNSUPPORTED
    # overlap
    assert lib.pab_layout(1, vp(1 << 20), vp((1 << 20) + 64), 4, 4, 64, 0, None) == pab.PAB_ERR_ARG
    res = ctypes.c_double(1.0)
    assert lib.pab_attn_diff_mse(None, None, 10, 0, ctypes.byref(res), None) == pab.PAB_ERR_ARG
    assert lib.pab_attn_diff_mse(None, None, 10, 7, ctypes.byref(res), None) == pab.PAB_ERR_ARG
    assert lib.pab_attn_diff_mse(None, None, 10, 0, None, None) == pab.PAB_ERR_ARG
    # side-stream MSE option: null plan, bad flag; disabling needs no device
    assert lib.pab_plan_set_diff_mse_stream(None, 1, None) == pab.PAB_ERR_ARG
    plan = pab.Plan(4, 8, 8, 2, 32, 16, 10, (2, 3, 4))
    assert lib.pab_plan_set_diff_mse_stream(plan._h, 2, None) == pab.PAB_ERR_ARG
    assert lib.pab_plan_set_diff_mse_stream(plan._h, 0, None) == pab.PAB_OK
    plan.close()


def test_spatial_alternatives_argument_checks(pab):
    """Sliding tile and draft attention reject bad geometry before any device
    work (no GPU needed); the plan options validate against the plan's frame."""
    lib = pab.lib
    ARG, UNS = pab.PAB_ERR_ARG, pab.PAB_ERR_UNSUPPORTED
    # pab_sta_attention(q, k, v, out, T, H, W, heads, d, tile, win_h, win_w, stream)
    assert lib.pab_sta_attention(None, None, None, None, 1, 30, 32, 2, 64, 16, 48, 48, None) == ARG  # H not tiles
    assert lib.pab_sta_attention(None, None, None, None, 1, 32, 32, 2, 64, 16, 32, 48, None) == ARG  # even window
    assert lib.pab_sta_attention(None, None, None, None, 1, 32, 32, 2, 64, 16, 40, 48, None) == ARG  # window not tiles
    assert lib.pab_sta_attention(None, None, None, None, 1, 32, 32, 2, 64, 8, 24, 24, None) == UNS   # tile size
    assert lib.pab_sta_attention(None, None, None, None, 1, 32, 32, 2, 64, 16, 48, 48, None) == ARG  # null pointers
    assert lib.pab_sta_attention(None, None, None, None, 0, 32, 32, 2, 64, 16, 48, 48, None) == pab.PAB_OK
    # draft attention
    n = ctypes.c_longlong(0)
    assert lib.pab_draft_workspace_bytes(2, 48, 80, 24, 128, 16, ctypes.byref(n)) == pab.PAB_OK
    assert n.value == 2 * 2 * 15 * 24 * 128 * 4
    assert lib.pab_draft_workspace_bytes(2, 48, 80, 24, 128, 8, ctypes.byref(n)) == UNS
    sel = ctypes.c_void_p(1 << 20)
    assert lib.pab_draft_select(None, None, 1, 30, 32, 1, 64, 16, 1, sel, sel, 1 << 20, None) == ARG
    assert lib.pab_draft_select(None, None, 1, 32, 32, 1, 64, 16, 0, sel, sel, 1 << 20, None) == ARG
    assert lib.pab_draft_select(None, None, 1, 32, 32, 1, 64, 16, 5, sel, sel, 1 << 20, None) == ARG
    assert lib.pab_draft_select(None, None, 1, 32, 32, 1, 64, 8, 1, sel, sel, 1 << 20, None) == UNS
    big = ctypes.c_void_p(1 << 24)
    assert lib.pab_draft_select(big, big, 1, 32, 32, 1, 64, 16, 2, sel, sel, 16, None) == ARG  # workspace too small
    assert lib.pab_region_sparse_attention(big, big, big, big, 1, 32, 32, 1, 64, 16, 2, None, None) == ARG
    # plan options: validated against the plan's 48 x 80 frame
    plan = pab.Plan(2, 48, 80, 2, 64, 16, 10, (2, 3, 4), dtype=torch.bfloat16)
    try:
        plan.set_spatial_window(16, 48, 48)
        plan.set_spatial_draft(16, 4)
        plan.set_spatial_draft(16, 0)
        for bad in ((16, 32, 48), (8, 24, 24)):
            with pytest.raises(pab.PabError):
                plan.set_spatial_window(*bad)
        for bad in ((16, 16), (8, 2)):
            with pytest.raises(pab.PabError):
                plan.set_spatial_draft(*bad)
    finally:
        plan.close()
    odd = pab.Plan(2, 30, 53, 2, 64, 16, 10, (2, 3, 4), dtype=torch.bfloat16)
    try:
        with pytest.raises(pab.PabError):
            odd.set_spatial_window(16, 48, 48)
        with pytest.raises(pab.PabError):
            odd.set_spatial_draft(16, 2)
    finally:
        odd.close()


def test_scatter_blocks_argument_checks(pab):
    """The sequence-parallel exchange's argument checks run on the host before
    any device work (fake aligned addresses: nothing is dereferenced)."""
    lib = pab.lib
    VP = ctypes.c_void_p

    def call(nt=1, G=2, P=4, rows=8, C=64, order=0, off=0, stride=8, dtype=0, src=None, dst=None):
        s = src if src is not None else [0x100000 * (i + 1) for i in range(nt)]
        d = dst if dst is not None else [0x10000000 + 0x100000 * i for i in range(nt * G)]
        sa = (VP * max(1, len(s)))(*s)
        da = (VP * max(1, len(d)))(*d)
        return lib.pab_scatter_blocks(sa, da, nt, G, P, rows, C, order, off, stride, dtype, None)

    assert call(nt=0) == pab.PAB_ERR_ARG
    assert call(nt=4) == pab.PAB_ERR_ARG
    assert call(G=0) == pab.PAB_ERR_ARG
    assert call(G=33) == pab.PAB_ERR_ARG
    assert call(order=2) == pab.PAB_ERR_ARG
    assert call(dtype=7) == pab.PAB_ERR_ARG
    assert call(P=-1) == pab.PAB_ERR_ARG
    assert call(C=60) == pab.PAB_ERR_UNSUPPORTED  # 120-byte rows
    assert call(stride=4) == pab.PAB_ERR_ARG       # destination blocks would overlap
    assert call(src=[0x100008]) == pab.PAB_ERR_ARG  # misaligned
    assert call(dst=[0x10000000, 0]) == pab.PAB_ERR_ARG
    # a destination overlapping the source
    assert call(src=[0x100000], dst=[0x100000 + 4096, 0x20000000]) == pab.PAB_ERR_ARG
    assert call(P=0) == pab.PAB_OK  # nothing to move
    assert lib.pab_scatter_blocks(None, None, 1, 2, 4, 8, 64, 0, 0, 8, 0, None) == pab.PAB_ERR_ARG


def test_ipc_argument_checks(pab):
    lib = pab.lib
    p = ctypes.c_void_p()
    h = ctypes.create_string_buffer(64)
    assert lib.pab_ipc_alloc(0, ctypes.byref(p), h) == pab.PAB_ERR_ARG
    assert lib.pab_ipc_alloc(64, None, h) == pab.PAB_ERR_ARG
    assert lib.pab_ipc_open(None, ctypes.byref(p)) == pab.PAB_ERR_ARG
    assert lib.pab_ipc_free(None) == pab.PAB_OK
    assert lib.pab_ipc_close(None) == pab.PAB_OK
