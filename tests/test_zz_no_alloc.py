"""muon_step_noalloc: the step for callers that cannot allocate device memory.

Programs whose device memory is fixed at start-up by another runtime, or
code running inside a framework callback that owns every allocation, cannot
hand muon_step a workspace.  muon_step_noalloc takes its scratch from a
built-in device array instead.  These tests call it through the C ABI and
check, over two calls in a row (so the second call starts from the scratch
contents the first one left), that it updates params and momentum exactly as
muon_step with a caller workspace does: the same kernels run on the same
inputs, so the results must agree bit for bit, also when the built-in array
is too small for the whole set and the step runs in several waves.  The
array's status word is read back through muon_noalloc_scratch and
muon_query_status, and a device-side timeout recorded there is reported.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from muon_polar_orthogonalized_b200 import _native as N
from muon_polar_orthogonalized_b200 import api
from muon_polar_orthogonalized_b200 import workloads as wl
from muon_polar_orthogonalized_b200.build import build

pytestmark = pytest.mark.gpu

COEFFS = (3.4445, -4.7750, 2.0315)
FLAGS = N.MUON_NESTEROV | N.MUON_CAUTIOUS_WD
SCRATCH = 32 * 1024 * 1024   # MUON_NOALLOC_SCRATCH_BYTES


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _noalloc_call(L, W, G, M, groups, lr=0.02, beta=0.95, wd=0.01, ns=5):
    g = api.make_groups(groups)
    coeffs = (ctypes.c_float * (3 * ns))(*(list(COEFFS) * ns))
    return L.muon_step_noalloc(api._ptrs(W), api._ptrs(G), api._ptrs(M), g, len(groups), lr, beta,
                               wd, ns, coeffs, FLAGS, _stream())


def _scratch(L):
    ptr, size = ctypes.c_void_p(), ctypes.c_size_t()
    assert L.muon_noalloc_scratch(ctypes.byref(ptr), ctypes.byref(size)) == N.MUON_OK, N.last_error()
    assert ptr.value and ptr.value % 256 == 0 and size.value == SCRATCH
    return ptr


def _state(dev, shapes, counts, gdt, tag):
    groups, first = [], 0
    W_ref, W_na, M_ref, M_na = [], [], [], []
    for gi, ((r, c), n) in enumerate(zip(shapes, counts)):
        groups.append((r, c, n, first, gdt, 1.0))
        first += n
        for j in range(n):
            w = torch.from_numpy(wl.iid_normal((r, c), 0.02, wl.seed_of(tag, gi, j)).astype(np.float32)).to(dev)
            W_ref.append(w.clone())
            W_na.append(w.clone())
            M_ref.append(torch.zeros(r, c, device=dev))
            M_na.append(torch.zeros(r, c, device=dev))
    return groups, W_ref, W_na, M_ref, M_na


@pytest.mark.parametrize("case", ["one_wave", "several_waves"])
def test_noalloc_matches_workspace_step_two_calls(case):
    build()
    assert torch.cuda.is_available(), "GPU test without a visible CUDA device"
    L = N.lib()
    dev = torch.device("cuda:0")
    if case == "one_wave":
        shapes, counts, gdt = [(256, 1024), (1024, 256), (384, 384)], [2, 1, 3], N.MUON_F32
    else:
        # each 2048 x 2048 matrix takes ~24 MiB of scratch: one matrix per wave
        shapes, counts, gdt = [(2048, 2048), (512, 1536)], [3, 2], N.MUON_BF16
    groups, W_ref, W_na, M_ref, M_na = _state(dev, shapes, counts, gdt, "na" + case)
    full = api.muon_workspace_size(groups, FLAGS)
    assert (full <= SCRATCH) == (case == "one_wave")
    ws = torch.empty(full, dtype=torch.uint8, device=dev)
    tdt = torch.bfloat16 if gdt == N.MUON_BF16 else torch.float32
    for call in range(2):
        G = [torch.from_numpy(wl.iid_normal(tuple(w.shape), 1.0, wl.seed_of("naG", case, call, k))
                              .astype(np.float32)).to(dev).to(tdt) for k, w in enumerate(W_ref)]
        api.muon_step(W_ref, G, M_ref, groups, 0.02, 0.95, 0.01, 5, COEFFS, FLAGS, ws)
        st = _noalloc_call(L, W_na, G, M_na, groups)
        assert st == N.MUON_OK, N.last_error()
        assert L.muon_query_status(_scratch(L), _stream()) == N.MUON_OK
        torch.cuda.synchronize()
        for k in range(len(W_ref)):
            assert torch.equal(W_na[k], W_ref[k]), (case, call, k)
            assert torch.equal(M_na[k], M_ref[k]), (case, call, k)


def test_noalloc_status_word_reports_a_device_timeout():
    """The bounded-wait self-test pointed at the built-in array records a
    timeout there; muon_query_status on the array's address reports it, and
    the next muon_step_noalloc clears it and succeeds (the context stays
    usable)."""
    build()
    L = N.lib()
    dev = torch.device("cuda:0")
    scratch = _scratch(L)
    assert L.muon_selftest_wait_timeout(scratch, 50_000_000, _stream()) == N.MUON_OK, N.last_error()
    assert L.muon_query_status(scratch, _stream()) == N.MUON_ERR_TIMEOUT
    groups, W_ref, W_na, M_ref, M_na = _state(dev, [(256, 512)], [1], N.MUON_F32, "na_timeout")
    G = [torch.ones(256, 512, device=dev)]
    assert _noalloc_call(L, W_na, G, M_na, groups) == N.MUON_OK, N.last_error()
    assert L.muon_query_status(scratch, _stream()) == N.MUON_OK
    assert torch.isfinite(W_na[0]).all()


def test_noalloc_rejects_matrix_larger_than_scratch():
    build()
    L = N.lib()
    dev = torch.device("cuda:0")
    # 4096 x 4096 needs 2 x 32 MiB of X buffers alone: more than the 32 MiB scratch
    groups = [(4096, 4096, 1, 0, N.MUON_F32, 1.0)]
    assert api.muon_workspace_min_size(groups, FLAGS) > SCRATCH
    W = [torch.zeros(4096, 4096, device=dev)]
    G = [torch.ones(4096, 4096, device=dev)]
    M = [torch.zeros(4096, 4096, device=dev)]
    st = _noalloc_call(L, W, G, M, groups)
    assert st == N.MUON_ERR_WORKSPACE
    assert "MUON_NOALLOC_SCRATCH_BYTES" in N.last_error()
    torch.cuda.synchronize()
    assert float(M[0].abs().max()) == 0.0 and float(W[0].abs().max()) == 0.0  # untouched
