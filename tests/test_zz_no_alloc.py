"""muon_step_noalloc: the step for callers that cannot allocate device memory.

Programs whose device memory is fixed at start-up by another runtime, or
code running inside a framework callback that owns every allocation, cannot
hand muon_step a workspace.  muon_step_noalloc takes its scratch from a
built-in device array instead.  These tests call it through the C ABI and
check, over two calls in a row (so the second call starts from the scratch
contents the first one left), that it updates params and momentum exactly as
muon_step with a caller workspace does, within the tolerances the other
parity tests use.  This file is collected last on purpose.
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
TOL_STEP = 2e-2    # applied step W_old - W_new (only U carries bf16 error)
TOL_MOM = 1e-6     # momentum


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _noalloc_call(L, W, G, M, groups, lr=0.02, beta=0.95, wd=0.01, ns=5):
    g = api.make_groups(groups)
    coeffs = (ctypes.c_float * (3 * ns))(*(list(COEFFS) * ns))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.muon_step_noalloc(api._ptrs(W), api._ptrs(G), api._ptrs(M), g, len(groups), lr, beta,
                               wd, ns, coeffs, FLAGS, stream)


def test_noalloc_matches_workspace_step_two_calls():
    build()
    assert torch.cuda.is_available(), "GPU test without a visible CUDA device"
    L = N.lib()
    dev = torch.device("cuda:0")
    shapes, counts = [(256, 1024), (1024, 256), (384, 384)], [2, 1, 3]
    groups, first = [], 0
    W_ref, W_na, M_ref, M_na = [], [], [], []
    for gi, ((r, c), n) in enumerate(zip(shapes, counts)):
        groups.append((r, c, n, first, N.MUON_F32, 1.0))
        first += n
        for j in range(n):
            w = torch.from_numpy(wl.iid_normal((r, c), 0.02, wl.seed_of("naW", gi, j)).astype(np.float32)).to(dev)
            W_ref.append(w.clone())
            W_na.append(w.clone())
            M_ref.append(torch.zeros(r, c, device=dev))
            M_na.append(torch.zeros(r, c, device=dev))
    ws = torch.empty(api.muon_workspace_size(groups, FLAGS), dtype=torch.uint8, device=dev)
    for call in range(2):
        G = [torch.from_numpy(wl.iid_normal(tuple(w.shape), 1.0, wl.seed_of("naG", call, k))
                              .astype(np.float32)).to(dev) for k, w in enumerate(W_ref)]
        w_before = [w.double().cpu().numpy() for w in W_ref]
        api.muon_step(W_ref, G, M_ref, groups, 0.02, 0.95, 0.01, 5, COEFFS, FLAGS, ws)
        st = _noalloc_call(L, W_na, G, M_na, groups)
        assert st == N.MUON_OK, N.last_error()
        torch.cuda.synchronize()
        for k in range(len(W_ref)):
            a_w, b_w = W_ref[k].double().cpu().numpy(), W_na[k].double().cpu().numpy()
            assert _rel(w_before[k] - b_w, w_before[k] - a_w) <= TOL_STEP, (call, k)
            assert _rel(M_na[k].double().cpu().numpy(), M_ref[k].double().cpu().numpy()) <= TOL_MOM


def test_noalloc_rejects_matrix_larger_than_scratch():
    build()
    L = N.lib()
    dev = torch.device("cuda:0")
    # 4096 x 4096 needs 2 x 32 MiB of X buffers alone: more than the 32 MiB scratch
    groups = [(4096, 4096, 1, 0, N.MUON_F32, 1.0)]
    assert api.muon_workspace_min_size(groups, FLAGS) > 32 * 1024 * 1024
    W = [torch.zeros(4096, 4096, device=dev)]
    G = [torch.ones(4096, 4096, device=dev)]
    M = [torch.zeros(4096, 4096, device=dev)]
    st = _noalloc_call(L, W, G, M, groups)
    assert st == N.MUON_ERR_WORKSPACE
    assert "MUON_NOALLOC_SCRATCH_BYTES" in N.last_error()
    torch.cuda.synchronize()
    assert float(M[0].abs().max()) == 0.0 and float(W[0].abs().max()) == 0.0  # untouched
