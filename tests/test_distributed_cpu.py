"""Owner-sharded Muon and ZeRO-1 AdamW across data-parallel ranks, on CPU
with gloo (world 2).

The protocol of muon_polar_orthogonalized_b200.distributed -- one
reduce_scatter of each flat gradient buffer, every rank steps what it owns
(its Muon matrices, its slice of the AdamW tensors), one in-place all_gather
of each flat parameter buffer -- runs on two gloo ranks with the per-rank
compute taken from the fp64 oracle; the result must equal one process
stepping every matrix and every AdamW tensor on the data-parallel mean
gradient.  The peer-buffer variant (every rank's buffers in shared memory
standing in for peer GPU memory: owners average the gradients from every
rank themselves and write every rank's copy of what they update) must give
the same.  Also checks the flat layout, the owner assignment, and that
momentum and AdamW state live only where owned.
"""
import json
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [(64, 128), (128, 64), (96, 96), (32, 256), (256, 32), (48, 80)]
ADAM_SHAPES = [(10, 4), (7,)]          # 40 elements straddle the two ranks' slices
ADAM_LR = [1e-3, 5e-3]
LR, BETA, WD = 0.02, 0.95, 0.01


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _params():
    rng = np.random.default_rng(0)
    return [torch.from_numpy(rng.standard_normal(s) * 0.02) for s in SHAPES]


def _adam_params():
    rng = np.random.default_rng(5)
    return [torch.from_numpy(rng.standard_normal(s) * 0.02) for s in ADAM_SHAPES]


def _grads(rank, step):
    rng = np.random.default_rng(1000 + 10 * step + rank)
    return [torch.from_numpy(rng.standard_normal(s)) for s in SHAPES]


def _adam_grads(rank, step):
    rng = np.random.default_rng(2000 + 10 * step + rank)
    return [torch.from_numpy(rng.standard_normal(s)) for s in ADAM_SHAPES]


def _oracle_fns(oracle, calls):
    def step_fn(ps, gs, ms, replicas=None):
        calls["muon"] += 1
        for k, (p, g, m) in enumerate(zip(ps, gs, ms)):
            w_new, m_new, _ = oracle.muon_step(p.numpy(), g.numpy(), m.numpy(), LR, BETA, WD)
            p.copy_(torch.from_numpy(w_new))
            m.copy_(torch.from_numpy(m_new))
            for rep in replicas or []:
                rep[k].copy_(torch.from_numpy(w_new))

    def adamw_fn(pieces, step):
        calls["adamw"] += 1
        for pc in pieces:
            b1, b2 = pc["betas"]
            for p, g, m, v in zip(pc["params"], pc["grads"], pc["exp_avg"], pc["exp_avg_sq"]):
                pn, mn, vn = oracle.adamw_step(p.numpy(), g.numpy(), m.numpy(), v.numpy(), step, pc["lr"],
                                               b1, b2, pc["eps"], pc["weight_decay"])
                p.copy_(torch.from_numpy(pn))
                m.copy_(torch.from_numpy(mn))
                v.copy_(torch.from_numpy(vn))
    return step_fn, adamw_fn


def _run_steps(opt, rank):
    for step in range(2):
        for k, g in enumerate(_grads(rank, step)):
            opt.muon_grads[k].copy_(g)
        for gi, g in enumerate(_adam_grads(rank, step)):
            opt.adamw_grads[gi][0].copy_(g)
        opt.step()


def _worker(rank, world, port, out_dir, shared):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    from muon_polar_orthogonalized_b200.distributed import DistributedMuonAdamW
    dist.init_process_group("gloo", rank=rank, world_size=world)
    params, adam = _params(), _adam_params()
    groups = [dict(params=[a], lr=lr) for a, lr in zip(adam, ADAM_LR)]
    calls = {"muon": 0, "adamw": 0, "mean": 0}
    step_fn, adamw_fn = _oracle_fns(oracle, calls)
    kw = {}
    if shared is not None:
        peer_grads = shared.get("peer_grads")

        def reduce_fn(dst, sources):
            calls["mean"] += 1
            for i, d in enumerate(dst):
                acc = sources[0][i].clone()
                for src in sources[1:]:
                    acc += src[i]
                d.copy_(acc / len(sources))
        bufs = shared["bufs"]
        kw = dict(buffers=bufs[rank],
                  peer_params={q: (bufs[q]["muon_params"], bufs[q]["adamw_params"])
                               for q in range(world) if q != rank},
                  reduce_fn=reduce_fn)
        if peer_grads:
            kw["peer_grads"] = {q: (bufs[q]["muon_grads"], bufs[q]["adamw_grads"])
                                for q in range(world) if q != rank}
    opt = DistributedMuonAdamW(params, groups, step_fn=step_fn, adamw_fn=adamw_fn, **kw)
    # parameters now live in the flat buffers; gradients are written into them
    assert all(p.grad is g for p, g in zip(params, opt.muon_grads))
    _run_steps(opt, rank)
    state_numel = sum(t.numel() for pc in opt._pieces for t in pc["exp_avg"])
    out = {"params": [p.numpy().tolist() for p in params], "adam": [a.numpy().tolist() for a in adam],
           "owners": opt.owners, "owned": opt.owned, "momentum_keys": sorted(opt.momentum),
           "adam_state_numel": state_numel, "calls": calls}
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(out, f)
    dist.barrier()
    dist.destroy_process_group()


def _reference():
    sys.path.insert(0, ROOT)
    import oracle
    params = [p.numpy() for p in _params()]
    moms = [np.zeros_like(p) for p in params]
    adam = [a.numpy() for a in _adam_params()]
    ms = [np.zeros_like(a) for a in adam]
    vs = [np.zeros_like(a) for a in adam]
    for step in range(2):
        g_mean = [(a.numpy() + b.numpy()) / 2 for a, b in zip(_grads(0, step), _grads(1, step))]
        for i in range(len(params)):
            params[i], moms[i], _ = oracle.muon_step(params[i], g_mean[i], moms[i], LR, BETA, WD)
        ga = [(a.numpy() + b.numpy()) / 2 for a, b in zip(_adam_grads(0, step), _adam_grads(1, step))]
        for t in range(len(adam)):
            adam[t], ms[t], vs[t] = oracle.adamw_step(adam[t], ga[t], ms[t], vs[t], step + 1, ADAM_LR[t],
                                                      0.9, 0.95, 1e-8, 0.0)
    return params, adam


def _check(res, world):
    ref_params, ref_adam = _reference()
    for r in range(world):
        for got, want in zip(res[r]["params"], ref_params):
            np.testing.assert_allclose(np.array(got), want, rtol=0, atol=1e-15)
        for got, want in zip(res[r]["adam"], ref_adam):
            np.testing.assert_allclose(np.array(got), want, rtol=0, atol=1e-15)


def test_sharded_step_equals_single_process(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path), None), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    _check(res, world)
    # every matrix owned by exactly one rank; momentum only where owned
    assert res[0]["owners"] == res[1]["owners"]
    assert sorted(res[0]["owned"] + res[1]["owned"]) == list(range(len(SHAPES)))
    for r in range(world):
        assert res[r]["momentum_keys"] == res[r]["owned"]
    # ZeRO-1: the AdamW state is split, not replicated
    total = sum(math.prod(s) for s in ADAM_SHAPES)
    assert res[0]["adam_state_numel"] + res[1]["adam_state_numel"] == total
    assert 0 < res[0]["adam_state_numel"] < total


@pytest.mark.parametrize("peer_grads", [False, True])
def test_peer_buffers_equal_single_process(tmp_path, peer_grads):
    sys.path.insert(0, ROOT)
    from muon_polar_orthogonalized_b200.distributed import DistributedMuonAdamW
    world, port = 2, _free_port()
    sizes = DistributedMuonAdamW.buffer_numels(SHAPES, [math.prod(s) for s in ADAM_SHAPES], world)
    bufs = []
    for r in range(world):
        b = {k: torch.zeros(n, dtype=torch.float64) for k, n in sizes.items()}
        for t in b.values():
            t.share_memory_()
        bufs.append(b)
    shared = {"bufs": bufs, "peer_grads": peer_grads}
    mp.start_processes(_worker, args=(world, port, str(tmp_path), shared), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    _check(res, world)
    for r in range(world):
        assert res[r]["calls"]["mean"] == (2 * 2 if peer_grads else 0)   # Muon region + AdamW slice


def test_flat_layout():
    sys.path.insert(0, ROOT)
    from muon_polar_orthogonalized_b200.distributed import ALIGN, FlatLayout
    shapes = [(4096, 4096)] * 4 + [(1024, 4096)] * 4 + [(100, 37)] * 3
    numels = [1000003, 17, 64, 5]
    for world in (1, 2, 3, 8):
        L = FlatLayout(shapes, numels, world)
        assert L.muon_region % ALIGN == 0 and L.adamw_slice % ALIGN == 0
        spans = sorted((o, o + math.prod(s)) for o, s in zip(L.muon_offset, shapes))
        for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
            assert a1 <= b0                                   # disjoint
        for i, (o, s) in enumerate(zip(L.muon_offset, shapes)):
            assert o % ALIGN == 0
            r = L.owners[i]
            assert r * L.muon_region <= o and o + math.prod(s) <= (r + 1) * L.muon_region
        covered = [0] * len(numels)
        for r in range(world):
            for t, start, n in L.owned_pieces(r):
                assert (L.adamw_offset[t] + start) % ALIGN == 0
                assert r * L.adamw_slice <= L.adamw_offset[t] + start
                assert L.adamw_offset[t] + start + n <= (r + 1) * L.adamw_slice
                covered[t] += n
        assert covered == numels                              # every element owned once
        assert L.adamw_offset[-1] + numels[-1] <= L.adamw_total


def test_peers_must_cover_other_ranks():
    sys.path.insert(0, ROOT)
    from muon_polar_orthogonalized_b200.distributed import DistributedMuonAdamW
    ps = _params()
    with pytest.raises(ValueError):
        DistributedMuonAdamW(ps, [], step_fn=lambda *a: None,
                             peer_params={1: (torch.zeros(1), torch.zeros(1))})   # world 1: no peers
    seen = []
    opt = DistributedMuonAdamW(_params(), [], step_fn=lambda p, g, m, reps: seen.append(len(reps)),
                               peer_params={})                                    # world 1: none needed
    opt.step()
    assert seen == [0]


def test_owner_assignment_balances_ns_cost():
    sys.path.insert(0, ROOT)
    from muon_polar_orthogonalized_b200.distributed import assign_owners, ns_cost
    shapes = [(4096, 4096)] * 64 + [(1024, 4096)] * 64 + [(14336, 4096)] * 64 + [(4096, 14336)] * 32
    for world in (2, 4, 8):
        owners = assign_owners(shapes, world)
        loads = [sum(ns_cost(*s) for s, o in zip(shapes, owners) if o == r) for r in range(world)]
        assert max(loads) / min(loads) < 1.03, (world, loads)
        assert owners == assign_owners(shapes, world)  # deterministic on every rank
