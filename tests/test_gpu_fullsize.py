"""Full-size parity: the transformer parameter sets, run exactly as bench.py
launches them (every matrix of every shape in one wave, CTA-pair tensor-core
GEMMs, the cautious update fused into the last B.X epilogue, one multi-tensor
AdamW launch), checked against the fp64 oracle.

* d=768, 12 layers: every one of the 72 matrices and whole AdamW tables.
* d=1664, 26 layers (rank-64 + noise gradients): sampled matrices of each
  shape group, AdamW row blocks and all 53 norm gains.
* the 32-layer 8B-shaped set: sampled matrices of each of the four shape
  groups (the oracle needs ~13 TFLOP of fp64 for them) and AdamW row blocks.

Tolerances as in test_gpu_parity.py: momentum and AdamW 1e-6, the applied
Muon step 2e-2 (only the bf16 orthogonalised update carries error).
"""
import gc

import numpy as np
import pytest
import torch

import bench
import oracle
from muon_polar_orthogonalized_b200 import _native as N
from muon_polar_orthogonalized_b200 import api
from muon_polar_orthogonalized_b200 import workloads as W
from tests.gpu_helpers import host64, rel

pytestmark = pytest.mark.gpu

FLAGS = N.MUON_NESTEROV | N.MUON_CAUTIOUS_WD


def _f32(x):
    return float(np.float32(x))


def _run_fullsize(name, muon_sample, adam_rows):
    """One step of workload `name` on cuda:0; returns per-check errors."""
    from muon_polar_orthogonalized_b200.build import build
    build()
    dev = torch.device("cuda:0")
    wl = W.get(name)
    D = bench.DeviceWorkload(wl, dev)
    ws = torch.empty(api.muon_workspace_size(D.groups, FLAGS), dtype=torch.uint8, device=dev)
    # snapshot the sampled inputs (momentum starts at zero)
    firsts = [g[3] for g in D.groups]
    picks = []
    for gi, js in muon_sample.items():
        for j in js:
            k = firsts[gi] + j
            picks.append((gi, j, host64(D.params[k]), host64(D.grads[k])))
    adam_picks = []
    for ti, (ps, gs, ms, vs, t) in enumerate(D.adam):
        for j, p in enumerate(ps):
            rows = adam_rows(p.shape[0]) if p.dim() == 2 else [slice(0, p.shape[0])]
            for sl in rows:
                adam_picks.append((ti, j, sl, host64(p[sl]), host64(gs[j][sl]), t))
    api.muon_step(D.params, D.grads, D.mom, D.groups, W.MUON_LR, W.MUON_BETA, W.MUON_WD,
                  wl.ns_steps, W.NS_COEFFS_FIXED, FLAGS, ws)
    if D.adam:
        api.adamw_step(D.adam_specs(), 1)
    torch.cuda.synchronize()
    assert api.muon_query_status(ws) == N.MUON_OK
    errs = []
    for gi, j, w0, g in picks:
        k = firsts[gi] + j
        rw, rm, _ = oracle.muon_step(w0, g, np.zeros_like(w0), W.MUON_LR, W.MUON_BETA, W.MUON_WD,
                                     wl.ns_steps, W.NS_COEFFS_FIXED)
        w1, m1 = host64(D.params[k]), host64(D.mom[k])
        e_m, e_s = rel(m1, rm), rel(w0 - w1, w0 - rw)
        errs.append(("muon", gi, j, e_m, e_s))
        assert e_m <= 1e-6, (name, gi, j, e_m)
        assert e_s <= 2e-2, (name, gi, j, e_s)
    b1, b2 = W.ADAMW_BETAS
    for ti, j, sl, p0, g, t in adam_picks:
        ps, gs, ms, vs, _ = D.adam[ti]
        rp, rm, rv = oracle.adamw_step(p0, g, 0 * p0, 0 * p0, 1, _f32(W.ADAMW_LR), _f32(b1), _f32(b2),
                                       _f32(W.ADAMW_EPS), _f32(t.wd))
        for got, ref in ((ps[j][sl], rp), (ms[j][sl], rm), (vs[j][sl], rv)):
            g64 = host64(got)
            assert rel(g64, ref) <= 1e-6
            assert np.abs(g64 - ref).max() <= 1e-6 * np.abs(ref).max()
        errs.append(("adamw", ti, j))
    del D, ws
    gc.collect()
    torch.cuda.empty_cache()
    return errs


def test_gpt_d768_12l_every_matrix():
    wl = W.get("gpt_d768_12l")
    sample = {gi: list(range(s.count)) for gi, s in enumerate(wl.muon)}
    errs = _run_fullsize("gpt_d768_12l", sample, lambda n: [slice(0, n)])
    worst = max(e[4] for e in errs if e[0] == "muon")
    print(f"gpt_d768_12l: {sum(e[0] == 'muon' for e in errs)} matrices, worst step rel err {worst:.3e}")


def test_gpt_d1664_26l_sampled():
    sample = {0: [0, 57, 103], 1: [0, 25], 2: [7, 25]}
    errs = _run_fullsize("gpt_d1664_26l", sample,
                         lambda n: [slice(0, 256), slice(n // 2, n // 2 + 256), slice(n - 256, n)])
    worst = max(e[4] for e in errs if e[0] == "muon")
    print(f"gpt_d1664_26l: worst sampled step rel err {worst:.3e}")


def test_llama_8b_32l_sampled():
    sample = {0: [63], 1: [0, 37], 2: [5], 3: [31]}
    errs = _run_fullsize("llama_8b_32l", sample,
                         lambda n: [slice(0, 128), slice(77777, 77777 + 128), slice(n - 128, n)])
    worst = max(e[4] for e in errs if e[0] == "muon")
    print(f"llama_8b_32l: worst sampled step rel err {worst:.3e}")
