"""Host-side checks of the native library; no GPU work is launched.

  * the library loads and exports every function include/muon_b200.h declares;
  * the ctypes structs have the C layout;
  * argument validation rejects bad calls before any CUDA call;
  * workspace sizing is consistent.
"""
import ctypes
import os
import re

import pytest

from muon_polar_orthogonalized_b200 import _native as N
from muon_polar_orthogonalized_b200 import api
from muon_polar_orthogonalized_b200.build import LIB_PATH, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon_b200.h")


@pytest.fixture(scope="module")
def L():
    build()
    return N.lib()


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+\**([a-z_][a-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_expected_entry_points():
    names = header_functions()
    for must in ("muon_step", "adamw_step", "muon_orthogonalize", "muon_workspace_size",
                 "muon_query_status", "muon_status_string"):
        assert must in names
    assert set(names) == set(N.SIGNATURES), set(names) ^ set(N.SIGNATURES)


def test_library_exports_every_header_symbol(L):
    out = os.popen(f"nm -D --defined-only {LIB_PATH}").read()
    exported = set(re.findall(r" T (\w+)$", out, flags=re.M))
    for name in header_functions():
        assert name in exported, name
        assert getattr(L, name) is not None


def test_struct_layouts():
    assert ctypes.sizeof(N.MuonGroup) == 24
    assert N.AdamWGroup.count.offset == 40 and N.AdamWGroup.lr.offset == 48
    assert ctypes.sizeof(N.AdamWGroup) == 72


def test_status_strings(L):
    for code, name in [(0, "MUON_OK"), (1, "MUON_ERR_INVALID_ARG"), (3, "MUON_ERR_WORKSPACE"),
                       (5, "MUON_ERR_TIMEOUT")]:
        assert N.status_string(code) == name


def _call_step(L, groups, ptr_count, ns=5, coeffs=True, flags=3, ws=0x1000, wsb=1 << 40,
               beta=0.95, lr=0.02, ptr=0x10000):
    g = api.make_groups(groups)
    arr = (ctypes.c_void_p * max(ptr_count, 1))(*([ptr] * ptr_count))
    ca = (ctypes.c_float * 48)(*([1.0] * 48)) if coeffs else None
    return L.muon_step(arr, arr, arr, g, len(groups), lr, beta, 0.01, ns, ca, flags,
                       ctypes.c_void_p(ws), wsb, None)


@pytest.mark.parametrize("case,expect", [
    (dict(groups=[(0, 4, 1, 0, 0, 1.0)]), N.MUON_ERR_INVALID_ARG),          # rows 0
    (dict(groups=[(4, 4, 1, 0, 7, 1.0)]), N.MUON_ERR_INVALID_ARG),          # dtype
    (dict(groups=[(4, 4, 1, 0, 0, float("nan"))]), N.MUON_ERR_INVALID_ARG),  # lr_scale
    (dict(groups=[(70000, 4, 1, 0, 0, 1.0)]), N.MUON_ERR_INVALID_ARG),      # too large
    (dict(groups=[(4, 8, 2, 0, 0, 1.0), (8, 8, 1, 1, 0, 1.0)]), N.MUON_ERR_INVALID_ARG),  # overlap
    (dict(ns=17), N.MUON_ERR_INVALID_ARG),
    (dict(ns=-1), N.MUON_ERR_INVALID_ARG),
    (dict(coeffs=False), N.MUON_ERR_INVALID_ARG),
    (dict(flags=512), N.MUON_ERR_INVALID_ARG),
    (dict(ws=0), N.MUON_ERR_WORKSPACE),
    (dict(ws=0x1010), N.MUON_ERR_WORKSPACE),                                 # misaligned
    (dict(wsb=100), N.MUON_ERR_WORKSPACE),
    (dict(beta=1.0), N.MUON_ERR_INVALID_ARG),
    (dict(lr=float("inf")), N.MUON_ERR_INVALID_ARG),
    (dict(ptr=0), N.MUON_ERR_INVALID_ARG),                                   # NULL tensor
    (dict(ptr=0x10008), N.MUON_ERR_INVALID_ARG),                             # misaligned tensor
])
def test_muon_step_validation(L, case, expect):
    groups = case.pop("groups", [(64, 128, 2, 0, 0, 1.0)])
    st = _call_step(L, groups, 2, **case)
    assert st == expect, N.last_error()
    assert N.last_error() != ""


def test_row_equilibrate_workspace_holds_one_partial_per_row():
    """MuonEq keeps one Frobenius partial per parameter row: for short rows
    (768 columns, fewer elements per row than a momentum block) the
    workspace grows by the extra partials, never shrinks, and a flag-less
    size is too small for a flagged call."""
    groups = [(768, 768, 48, 0, 1, 1.0), (3072, 768, 12, 48, 1, 1.0)]
    plain = api.muon_workspace_size(groups, 0)
    eq = api.muon_workspace_size(groups, N.MUON_ROW_EQUILIBRATE)
    assert eq > plain
    rows = 48 * 768 + 12 * 3072
    assert eq - plain <= 4 * rows + 2048
    assert api.muon_workspace_min_size(groups, N.MUON_ROW_EQUILIBRATE) > api.muon_workspace_min_size(groups, 0)


def test_replicated_step_validation(L):
    groups = api.make_groups([(64, 128, 2, 0, 0, 1.0)])
    arr = (ctypes.c_void_p * 2)(0x10000, 0x10000)
    ca = (ctypes.c_float * 15)(*([1.0] * 15))
    bad = (ctypes.c_void_p * 2)(0x10000, 0x10008)          # misaligned copy
    good = (ctypes.c_void_p * 2)(0x20000, 0x20000)

    def call(table, n):
        return L.muon_step_replicated(arr, arr, arr, groups, 1, 0.02, 0.95, 0.01, 5, ca, 3,
                                      ctypes.c_void_p(0x1000), 1 << 40, table, n, None)
    T = ctypes.POINTER(ctypes.c_void_p) * 8
    assert call(None, 1) == N.MUON_ERR_INVALID_ARG
    assert call(T(*[ctypes.cast(good, ctypes.POINTER(ctypes.c_void_p))] * 8), 8) == N.MUON_ERR_INVALID_ARG
    assert call(T(ctypes.cast(bad, ctypes.POINTER(ctypes.c_void_p))), 1) == N.MUON_ERR_INVALID_ARG
    assert "replicas[0]" in N.last_error()
    assert call(T(ctypes.cast(good, ctypes.POINTER(ctypes.c_void_p)),
                  ctypes.POINTER(ctypes.c_void_p)()), 2) == N.MUON_ERR_INVALID_ARG
    assert "replicas[1]" in N.last_error()


def test_reduce_mean_validation(L):
    dst = (ctypes.c_void_p * 1)(0x10000)
    src = (ctypes.c_void_p * 1)(0x20000)
    n = (ctypes.c_int64 * 1)(100)
    T = ctypes.POINTER(ctypes.c_void_p) * 9
    tab = T(*[ctypes.cast(src, ctypes.POINTER(ctypes.c_void_p))] * 9)
    assert L.muon_reduce_mean(dst, tab, 0, n, 1, 0, None) == N.MUON_ERR_INVALID_ARG
    assert L.muon_reduce_mean(dst, tab, 9, n, 1, 0, None) == N.MUON_ERR_INVALID_ARG
    assert L.muon_reduce_mean(dst, tab, 2, n, 1, 7, None) == N.MUON_ERR_INVALID_ARG
    bad = (ctypes.c_void_p * 1)(0x10004)
    assert L.muon_reduce_mean(bad, tab, 2, n, 1, 0, None) == N.MUON_ERR_INVALID_ARG
    misal = (ctypes.c_void_p * 1)(0x20008)
    tab2 = T(ctypes.cast(src, ctypes.POINTER(ctypes.c_void_p)), ctypes.cast(misal, ctypes.POINTER(ctypes.c_void_p)))
    assert L.muon_reduce_mean(dst, tab2, 2, n, 1, 0, None) == N.MUON_ERR_INVALID_ARG
    assert "sources[1][0]" in N.last_error()
    neg = (ctypes.c_int64 * 1)(-1)
    assert L.muon_reduce_mean(dst, tab, 2, neg, 1, 0, None) == N.MUON_ERR_INVALID_ARG


def test_adamw_validation(L):
    p = (ctypes.c_void_p * 1)(0x10000)
    n = (ctypes.c_int64 * 1)(16)
    g = N.AdamWGroup(p, p, p, p, n, 1, 0, 1e-3, 0.9, 0.95, 1e-8, 0.0)
    assert L.adamw_step(ctypes.byref(g), 1, 0, None) == N.MUON_ERR_INVALID_ARG  # step 0
    bad = N.AdamWGroup(p, p, p, p, n, 1, 0, 1e-3, 1.5, 0.95, 1e-8, 0.0)
    assert L.adamw_step(ctypes.byref(bad), 1, 1, None) == N.MUON_ERR_INVALID_ARG  # beta1
    q = (ctypes.c_void_p * 1)(0x10004)
    mis = N.AdamWGroup(q, p, p, p, n, 1, 0, 1e-3, 0.9, 0.95, 1e-8, 0.0)
    assert L.adamw_step(ctypes.byref(mis), 1, 1, None) == N.MUON_ERR_INVALID_ARG
    neg = N.AdamWGroup(p, p, p, p, (ctypes.c_int64 * 1)(-1), 1, 0, 1e-3, 0.9, 0.95, 1e-8, 0.0)
    assert L.adamw_step(ctypes.byref(neg), 1, 1, None) == N.MUON_ERR_INVALID_ARG


def test_workspace_sizes(L):
    g = [(768, 768, 48, 0, 1, 1.0), (3072, 768, 12, 48, 1, 1.0), (768, 3072, 12, 60, 1, 1.0)]
    full = api.muon_workspace_size(g)
    mn = api.muon_workspace_min_size(g)
    assert 0 < mn < full
    # X ping-pong (2 x bf16 params) + B (bf16 m x m) per matrix, plus small arrays
    muon_elems = 48 * 768 * 768 + 24 * 768 * 3072
    b_elems = 72 * 768 * 768
    lower = 2 * 2 * muon_elems + 2 * b_elems
    assert lower <= full <= lower * 1.01 + (1 << 20)
    # fp32 debug mode doubles the matrix buffers
    assert api.muon_workspace_size(g, N.MUON_FP32_DEBUG) > 1.9 * full
    # invalid groups -> 0
    assert api.muon_workspace_size([(0, 4, 1, 0, 0, 1.0)]) == 0


def test_profiler_kinds(L):
    names = [L.muon_kernel_kind_name(i).decode() for i in range(L.muon_kernel_kind_count())]
    for k in ("momentum_norm", "ns_gram", "ns_poly", "ns_axpy", "ns_axpy_update", "adamw"):
        assert k in names


def test_selftest_validation(L):
    assert L.muon_selftest_wait_timeout(None, 10**6, None) == N.MUON_ERR_WORKSPACE
    assert L.muon_selftest_wait_timeout(ctypes.c_void_p(0x1010), 10**6, None) == N.MUON_ERR_WORKSPACE
    assert L.muon_selftest_wait_timeout(ctypes.c_void_p(0x1000), 10, None) == N.MUON_ERR_INVALID_ARG
    assert L.muon_selftest_wait_timeout(ctypes.c_void_p(0x1000), 10**10, None) == N.MUON_ERR_INVALID_ARG


def test_schedule_validation(L):
    assert L.muon_schedule_advance(None, 10, 0.1, 0.2, 0.1, None) == N.MUON_ERR_INVALID_ARG
    st = ctypes.c_void_p(0x1000)
    assert L.muon_schedule_advance(st, 0, 0.1, 0.2, 0.1, None) == N.MUON_ERR_INVALID_ARG
    assert L.muon_schedule_advance(st, 10, 0.7, 0.5, 0.1, None) == N.MUON_ERR_INVALID_ARG
    assert L.muon_schedule_advance(ctypes.c_void_p(0x1004), 10, 0.1, 0.2, 0.1, None) == N.MUON_ERR_INVALID_ARG
    assert L.muon_schedule_advance_cosine(None, 10, 1, 0.1, None) == N.MUON_ERR_INVALID_ARG
    assert L.muon_schedule_advance_cosine(st, 0, 0, 0.1, None) == N.MUON_ERR_INVALID_ARG
    assert L.muon_schedule_advance_cosine(st, 10, 11, 0.1, None) == N.MUON_ERR_INVALID_ARG
    assert L.muon_schedule_advance_cosine(st, 10, -1, 0.1, None) == N.MUON_ERR_INVALID_ARG
    assert L.muon_schedule_advance_cosine(st, 10, 1, float("nan"), None) == N.MUON_ERR_INVALID_ARG
    p = (ctypes.c_void_p * 1)(0x10000)
    n = (ctypes.c_int64 * 1)(16)
    g = N.AdamWGroup(p, p, p, p, n, 1, 0, 1e-3, 0.9, 0.95, 1e-8, 0.0)
    assert L.adamw_step_scheduled(ctypes.byref(g), 1, None, None) == N.MUON_ERR_INVALID_ARG


# ------------------------------------------------ binding-side validation
# The C ABI receives bare pointer arrays; the Python binding checks list
# lengths, coefficient rows and tensor layouts before the call, so that a
# short list or a wrong dtype never reaches the library.  Raw integer
# pointers pass through unchecked (fake addresses here: nothing is launched).

GROUPS = [(4, 8, 2, 0, N.MUON_F32, 1.0)]
FAKE = [0x100000, 0x200000]


def test_binding_rejects_short_coefficient_table():
    with pytest.raises(ValueError, match="coeffs"):
        api.muon_step(FAKE, FAKE, FAKE, GROUPS, 0.02, 0.95, 0.0, 3,
                      [(3.4445, -4.7750, 2.0315)] * 2, 0, 0x300000, workspace_bytes=1 << 20)
    with pytest.raises(ValueError, match="triple"):
        api.muon_step(FAKE, FAKE, FAKE, GROUPS, 0.02, 0.95, 0.0, 1, [(1.0, 2.0)], 0, 0x300000,
                      workspace_bytes=1 << 20)


def test_binding_rejects_short_pointer_lists():
    with pytest.raises(ValueError, match="grads: 1 entries"):
        api.muon_step(FAKE, FAKE[:1], FAKE, GROUPS, 0.02, 0.95, 0.0, 0, None, 0, 0x300000,
                      workspace_bytes=1 << 20)
    with pytest.raises(ValueError, match=r"replicas\[0\]"):
        api.muon_step_replicated(FAKE, FAKE, FAKE, GROUPS, 0.02, 0.95, 0.0, 0, None, 0, 0x300000,
                                 [FAKE[:1]], workspace_bytes=1 << 20)


def test_binding_rejects_tensors_the_library_would_misread():
    import torch
    cpu = [torch.zeros(4, 8), torch.zeros(4, 8)]
    with pytest.raises(ValueError, match=r"params\[0\].*CUDA"):
        api.muon_step(cpu, FAKE, FAKE, GROUPS, 0.02, 0.95, 0.0, 0, None, 0, 0x300000,
                      workspace_bytes=1 << 20)
    spec = api.AdamWSpec([torch.zeros(8)], [torch.zeros(8)], [torch.zeros(8)], [], 1e-3, 0.9, 0.95,
                         1e-8, 0.0)
    with pytest.raises(ValueError, match="exp_avg_sq"):
        api.adamw_step([spec], 1)
