"""Owner-sharded Muon across data-parallel ranks, on CPU with gloo (world 2).

The protocol of muon_polar_orthogonalized_b200.distributed (reduce each
matrix's gradient to its owner, owner steps, owner broadcasts) runs on two
gloo ranks with the per-rank compute taken from the fp64 oracle; the result
must equal one process stepping every matrix on the data-parallel mean
gradient.  Also checks the owner assignment and that momentum lives only on
owners.
"""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [(64, 128), (128, 64), (96, 96), (32, 256), (256, 32), (48, 80)]
LR, BETA, WD = 0.02, 0.95, 0.01


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _params():
    rng = np.random.default_rng(0)
    return [torch.from_numpy(rng.standard_normal(s) * 0.02) for s in SHAPES]


def _grads(rank, step):
    rng = np.random.default_rng(1000 + 10 * step + rank)
    return [torch.from_numpy(rng.standard_normal(s)) for s in SHAPES]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    from muon_polar_orthogonalized_b200.distributed import DistributedMuonAdamW
    dist.init_process_group("gloo", rank=rank, world_size=world)
    params = _params()
    emb = torch.from_numpy(np.random.default_rng(5).standard_normal((10, 4)) * 0.02)
    state = {"m": torch.zeros_like(emb), "v": torch.zeros_like(emb), "t": 0}

    def step_fn(ps, gs, ms):
        for p, g, m in zip(ps, gs, ms):
            w_new, m_new, _ = oracle.muon_step(p.numpy(), g.numpy(), m.numpy(), LR, BETA, WD)
            p.copy_(torch.from_numpy(w_new))
            m.copy_(torch.from_numpy(m_new))

    def adamw_fn(groups):
        state["t"] += 1
        p = groups[0]["params"][0]
        pn, mn, vn = oracle.adamw_step(p.numpy(), p.grad.numpy(), state["m"].numpy(), state["v"].numpy(),
                                       state["t"], 1e-3, 0.9, 0.95, 1e-8, 0.0)
        p.copy_(torch.from_numpy(pn)); state["m"].copy_(torch.from_numpy(mn)); state["v"].copy_(torch.from_numpy(vn))

    opt = DistributedMuonAdamW(params, [dict(params=[emb])], step_fn=step_fn, adamw_fn=adamw_fn)
    for step in range(2):
        for p, g in zip(params, _grads(rank, step)):
            p.grad = g
        emb.grad = torch.from_numpy(np.random.default_rng(2000 + 10 * step + rank).standard_normal((10, 4)))
        opt.step()
    out = {"params": [p.numpy().tolist() for p in params], "emb": emb.numpy().tolist(),
           "owners": opt.owners, "owned": opt.owned, "momentum_keys": sorted(opt.momentum)}
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(out, f)
    dist.barrier()
    dist.destroy_process_group()


def _reference():
    sys.path.insert(0, ROOT)
    import oracle
    params = [p.numpy() for p in _params()]
    moms = [np.zeros_like(p) for p in params]
    emb = np.random.default_rng(5).standard_normal((10, 4)) * 0.02
    m = v = np.zeros_like(emb)
    for step in range(2):
        g_mean = [(a.numpy() + b.numpy()) / 2 for a, b in zip(_grads(0, step), _grads(1, step))]
        for i in range(len(params)):
            params[i], moms[i], _ = oracle.muon_step(params[i], g_mean[i], moms[i], LR, BETA, WD)
        ge = (np.random.default_rng(2000 + 10 * step).standard_normal((10, 4)) +
              np.random.default_rng(2000 + 10 * step + 1).standard_normal((10, 4))) / 2
        emb, m, v = oracle.adamw_step(emb, ge, m, v, step + 1, 1e-3, 0.9, 0.95, 1e-8, 0.0)
    return params, emb


def test_owner_sharded_step_equals_single_process(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    ref_params, ref_emb = _reference()
    for r in range(world):
        for got, want in zip(res[r]["params"], ref_params):
            np.testing.assert_allclose(np.array(got), want, rtol=0, atol=1e-15)
        np.testing.assert_allclose(np.array(res[r]["emb"]), ref_emb, rtol=0, atol=1e-15)
    # every matrix owned by exactly one rank; momentum only where owned
    assert res[0]["owners"] == res[1]["owners"]
    owned = sorted(res[0]["owned"] + res[1]["owned"])
    assert owned == list(range(len(SHAPES)))
    for r in range(world):
        assert res[r]["momentum_keys"] == res[r]["owned"]


def _worker_peer(rank, world, port, out_dir, all_params, all_grads):
    """As _worker, with every rank's Muon parameters (and, if given, gradients)
    in shared memory standing in for peer GPU memory: owners write the other
    rank's copies in their step (peer_params) instead of broadcasting, and
    average the gradients from every rank themselves (peer_grads) instead of
    the reduces."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    from muon_polar_orthogonalized_b200.distributed import DistributedMuonAdamW
    dist.init_process_group("gloo", rank=rank, world_size=world)
    params = all_params[rank]
    peers = {r: all_params[r] for r in range(world) if r != rank}
    peer_grads = {r: all_grads[r] for r in range(world) if r != rank} if all_grads else None
    calls = {"replicated": 0, "mean": 0}

    def reduce_fn(dst, sources):
        calls["mean"] += 1
        for i, d in enumerate(dst):
            acc = sources[0][i].clone()
            for src in sources[1:]:
                acc += src[i]
            d.copy_(acc / len(sources))

    def step_fn(ps, gs, ms, replicas):
        calls["replicated"] += 1
        for k, (p, g, m) in enumerate(zip(ps, gs, ms)):
            w_new, m_new, _ = oracle.muon_step(p.numpy(), g.numpy(), m.numpy(), LR, BETA, WD)
            p.copy_(torch.from_numpy(w_new))
            m.copy_(torch.from_numpy(m_new))
            for rep in replicas:
                rep[k].copy_(torch.from_numpy(w_new))

    opt = DistributedMuonAdamW(params, [], step_fn=step_fn, peer_params=peers, peer_grads=peer_grads,
                               reduce_fn=reduce_fn)
    for step in range(2):
        for k, (p, g) in enumerate(zip(params, _grads(rank, step))):
            if all_grads:
                all_grads[rank][k].copy_(g)      # the rank's gradient buffer, seen by its peers
                p.grad = all_grads[rank][k]
            else:
                p.grad = g
        opt.step()
    out = {"params": [p.numpy().tolist() for p in params], "calls": calls["replicated"],
           "mean_calls": calls["mean"]}
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(out, f)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("peer_grads", [False, True])
def test_owner_writes_peer_replicas_equals_single_process(tmp_path, peer_grads):
    world, port = 2, _free_port()
    all_params, all_grads = [], []
    for r in range(world):
        ps = [p.clone() for p in _params()]
        gs = [torch.zeros_like(p) for p in ps]
        for t in ps + gs:
            t.share_memory_()
        all_params.append(ps)
        all_grads.append(gs)
    mp.start_processes(_worker_peer, args=(world, port, str(tmp_path), all_params,
                                           all_grads if peer_grads else None),
                       nprocs=world, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    ref_params, _ = _reference()
    for r in range(world):
        assert res[r]["calls"] == 2
        assert res[r]["mean_calls"] == (2 if peer_grads else 0)
        for got, want in zip(res[r]["params"], ref_params):
            np.testing.assert_allclose(np.array(got), want, rtol=0, atol=1e-15)


def test_peer_params_must_cover_other_ranks():
    sys.path.insert(0, ROOT)
    from muon_polar_orthogonalized_b200.distributed import DistributedMuonAdamW
    ps = _params()
    import pytest
    with pytest.raises(ValueError):
        DistributedMuonAdamW(ps, [], step_fn=lambda *a: None, peer_params={1: ps})   # world 1: no peers
    seen = []
    opt = DistributedMuonAdamW(ps, [], step_fn=lambda p, g, m, reps: seen.append(len(reps)),
                               peer_params={})                                    # world 1: none needed
    for p in ps:
        p.grad = torch.zeros_like(p)
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
