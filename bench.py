"""Benchmark: one Muon + AdamW optimizer step over a synthetic parameter set.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one muon_step (momentum + Frobenius norm, 5 quintic Newton-Schulz
iterations as grouped tcgen05 GEMMs, cautious decay + update) over every
hidden matrix plus one adamw_step over the embedding / LM head (/ gains),
all through the C ABI.  Default workload: the 32-layer 8B-shaped set
(Wq, Wo 4096^2; Wk, Wv 1024x4096; gate, up 14336x4096; down 4096x14336;
AdamW on two 128256x4096 tables), fp32 params / momentum, bf16 grads.
Inputs (~84 GB resident) are far larger than L2, so no flush is needed.

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
cuda synchronize on both sides, CUDA events on the launching stream, max
over ranks; then K more steps with a CUDA-event pair around every launch for
the per-kernel breakdown (kept out of the timed steps).  With N > 1 (torchrun), every rank runs its own replica of the
workload on its GPU (matrices are independent problems; there is no data-path
collective), so per-GPU work is fixed: weak scaling.

Rank 0 prints one JSON line.  --impl reference times the CPU fp64 oracle on a
bounded sample of the same workload instead (the reference arm).

--distributed times the data-parallel optimizer instead (DistributedMuonAdamW:
every rank holds the whole parameter set, the matrices are owner-sharded for
Muon and the AdamW tensors ZeRO-1-sliced; per step one reduce_scatter of the
flat gradient buffers, the owners' steps, one all_gather of the flat parameter
buffers over NCCL).  Total work is one optimizer step of one model however
many ranks share it: strong scaling.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Muon+AdamW step ms at 8B shapes; NS TFLOP/s as % of bf16 tensor peak"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic of one pass of a product (its launches over every matrix of
# the step), from one ncu capture of the named sources (the kernel and the
# planner that composes its launches; their fingerprint: sha256 prefix of the
# files listed with comments removed, source_fingerprint).  When the sources
# differ from the captured ones the figure no longer describes the kernel and
# the roofline reports traffic = null.  Captured on the one-layer slice of
# the 8B shapes and scaled x32 (the slice is exactly 1/32 of the set: same
# seven shapes, 1 layer instead of 32).
TRAFFIC_CAPTURES = {
    "ns_axpy": {"sources": ["k_gemm_tc.cu", "sm100.cuh", "common.cuh", "muon_api.cu"], "sha": "253ab92629fdb298",
                "bytes_per_pass": {"llama_8b_32l": 32 * 990843392, "llama_8b_1layer": 990843392}},
}


def source_fingerprint(files) -> str:
    """sha256 prefix of the kernel sources with comments, blank lines and
    trailing blanks removed: changes whenever the compiled code can, not when
    only a comment does."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "muon_polar_orthogonalized_b200", "csrc")
    text = "".join(open(os.path.join(csrc, f)).read() for f in files)
    text = re.sub(r"//[^\n]*|/\*.*?\*/", "", text, flags=re.S)
    # what is left of comment-only lines, and trailing blanks, do not count
    code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def captured_traffic(kernel: str, workload: str):
    """DRAM bytes of one pass of the product from the committed ncu capture,
    or None once the kernel's or the planner's sources have changed since that
    capture."""
    cap = TRAFFIC_CAPTURES.get(kernel)
    if not cap or workload not in cap["bytes_per_pass"]:
        return None
    if source_fingerprint(cap["sources"]) != cap["sha"]:
        return None
    return cap["bytes_per_pass"][workload]


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        out = open(self.path, "w")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        finally:
            out.close()   # the sampler process holds its own descriptor

    def stop(self):
        if self.proc is None:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------- workload
def algorithmic_work(wl):
    """Per-iteration FLOPs and per-step bytes of each kernel kind.  Nominal
    FLOPs as the spec counts them: gram 2 m^2 n, A.A 2 m^3, B.X 2 m^2 n per
    iteration.  Executed FLOPs: the two symmetric products compute only the
    upper half (gram m^2 n, A.A m^3); B.X is not symmetric (2 m^2 n)."""
    gram = poly = axpy = 0.0
    mom_bytes = upd_bytes = 0.0
    for s in wl.muon:
        m, n = min(s.rows, s.cols), max(s.rows, s.cols)
        gram += s.count * 2.0 * m * m * n
        poly += s.count * 2.0 * m ** 3
        axpy += s.count * 2.0 * m * m * n
        gb = 2 if s.grad_dtype == "bf16" else 4
        mom_bytes += s.count * s.rows * s.cols * (gb + 8 + 2)
        upd_bytes += s.count * s.rows * s.cols * (2 + 8)
    adam_bytes = 0.0
    for t in wl.adamw:
        gb = 2 if t.grad_dtype == "bf16" else 4
        adam_bytes += t.count * math.prod(t.shape) * (gb + 24)
    return dict(gram_flops=gram, poly_flops=poly, axpy_flops=axpy,
                gram_flops_executed=gram / 2, poly_flops_executed=poly / 2, axpy_flops_executed=axpy,
                momentum_bytes=mom_bytes, update_bytes=upd_bytes, adamw_bytes=adam_bytes)


class DeviceWorkload:
    """All tensors of a workload resident on one GPU: params / momentum / grads
    as views into one flat buffer per shape group (16-byte aligned views)."""

    def __init__(self, wl, device, e2e_host: bool = False, pinned: bool = True):
        import torch
        from muon_polar_orthogonalized_b200 import _native as N
        from muon_polar_orthogonalized_b200 import workloads as W
        self.wl = wl
        self.device = device
        self.groups, self.params, self.grads, self.mom = [], [], [], []
        self.flat_grads = []
        first = 0
        for gi, s in enumerate(wl.muon):
            numel = s.rows * s.cols
            gdt = torch.bfloat16 if s.grad_dtype == "bf16" else torch.float32
            P = torch.empty(s.count * numel, dtype=torch.float32, device=device)
            Mm = torch.zeros(s.count * numel, dtype=torch.float32, device=device)
            G = torch.empty(s.count * numel, dtype=gdt, device=device)
            gen = W.device_generator(device, wl.name, "W", gi)
            P.normal_(0.0, 0.02, generator=gen)
            for j in range(s.count):
                g = W.device_grad(wl, s.rows, s.cols, gdt, device, gi, j)
                G[j * numel:(j + 1) * numel].copy_(g.reshape(-1))
                del g
            for j in range(s.count):
                sl = slice(j * numel, (j + 1) * numel)
                self.params.append(P[sl].view(s.rows, s.cols))
                self.mom.append(Mm[sl].view(s.rows, s.cols))
                self.grads.append(G[sl].view(s.rows, s.cols))
            self.flat_grads.append(G)
            self.groups.append((s.rows, s.cols, s.count, first,
                                N.MUON_BF16 if s.grad_dtype == "bf16" else N.MUON_F32, 1.0))
            first += s.count
        self.adam = []
        for ti, t in enumerate(wl.adamw):
            gdt = torch.bfloat16 if t.grad_dtype == "bf16" else torch.float32
            ps, gs, ms, vs = [], [], [], []
            for j in range(t.count):
                p = torch.empty(t.shape, dtype=torch.float32, device=device)
                if t.init == "ones":
                    p.fill_(1.0)
                else:
                    p.normal_(0.0, 0.02, generator=W.device_generator(device, wl.name, "aW", ti, j))
                g = torch.randn(t.shape, generator=W.device_generator(device, wl.name, "aG", ti, j),
                                device=device).mul_(wl.grad_std).to(gdt)
                ps.append(p)
                gs.append(g)
                ms.append(torch.zeros_like(p))
                vs.append(torch.zeros_like(p))
                self.flat_grads.append(g.view(-1))
            self.adam.append((ps, gs, ms, vs, t))
        self.host_grads = None
        self.host_pinned = False
        if e2e_host:
            self.host_grads = [torch.empty(g.shape, dtype=g.dtype, pin_memory=pinned) for g in self.flat_grads]
            self.host_pinned = pinned
            for h, g in zip(self.host_grads, self.flat_grads):
                h.copy_(g)

    def adam_specs(self, adam_grads=None):
        from muon_polar_orthogonalized_b200 import api
        from muon_polar_orthogonalized_b200 import workloads as W
        specs = []
        for ti, (ps, gs, ms, vs, t) in enumerate(self.adam):
            g = adam_grads[ti] if adam_grads is not None else gs
            specs.append(api.AdamWSpec(ps, g, ms, vs, W.ADAMW_LR, W.ADAMW_BETAS[0], W.ADAMW_BETAS[1],
                                       W.ADAMW_EPS, t.wd))
        return specs

    def grad_views(self, flats):
        """(muon grads, adam grads per AdamW group) as views of `flats`, a list of
        flat buffers laid out like self.flat_grads."""
        muon, k = [], 0
        for s in self.wl.muon:
            numel = s.rows * s.cols
            muon.extend(flats[k][j * numel:(j + 1) * numel].view(s.rows, s.cols) for j in range(s.count))
            k += 1
        adam = []
        for (ps, gs, ms, vs, t) in self.adam:
            adam.append([flats[k + j].view(p.shape) for j, p in enumerate(ps)])
            k += len(ps)
        return muon, adam


class RankContext:
    """Ranks of one benchmark job (torchrun env: RANK / LOCAL_RANK / WORLD_SIZE /
    MASTER_*).  With one rank nothing is initialised.  The backend is "nccl"
    on GPUs; the CPU tests drive the same logic with "gloo"."""

    def __init__(self, backend: str = "nccl", timeout_s: int = 600):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.dist = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
            self.dist = dist

    @property
    def is_root(self) -> bool:
        return self.rank == 0

    def barrier(self) -> None:
        if self.dist is not None:
            self.dist.barrier()

    def max(self, x: float, device=None) -> float:
        """Max of x over all ranks (every rank gets it)."""
        if self.dist is None:
            return x
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self) -> None:
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def pinned_fits(nbytes: int, ranks_on_host: int) -> bool:
    """Pin host buffers for the end-to-end copies only if all ranks' buffers
    leave a quarter of the host RAM free."""
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        return True
    return nbytes * ranks_on_host < 0.75 * avail


def run_gpu(args):
    import torch
    from muon_polar_orthogonalized_b200 import _native as N
    from muon_polar_orthogonalized_b200 import api
    from muon_polar_orthogonalized_b200 import workloads as W
    from muon_polar_orthogonalized_b200.build import build

    R = RankContext("nccl")
    world, rank, local = R.world, R.rank, R.local
    if rank == 0:
        build()
    R.barrier()
    if rank != 0:
        build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = W.get(args.workload)
    grad_bytes = sum(s.rows * s.cols * s.count * (2 if s.grad_dtype == "bf16" else 4) for s in wl.muon) + \
        sum(math.prod(t.shape) * t.count * (2 if t.grad_dtype == "bf16" else 4) for t in wl.adamw)
    e2e_pinned = pinned_fits(grad_bytes, min(world, torch.cuda.device_count()))
    D = DeviceWorkload(wl, dev, e2e_host=not args.no_e2e, pinned=e2e_pinned)
    flags = (N.MUON_NESTEROV | N.MUON_CAUTIOUS_WD | (N.MUON_TC_SINGLE_CTA if args.single_cta else 0)
             | (N.MUON_NORMUON if args.normuon else 0)
             | (N.MUON_ROW_EQUILIBRATE if args.row_equilibrate else 0)
             | (N.MUON_TC_NARROW_TILES if args.narrow_tiles else 0)
             | (N.MUON_TC_WIDE_TILES if args.wide_tiles else 0))
    ws_bytes = api.muon_workspace_size(D.groups, flags)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    coeffs = W.NS_COEFFS_FIXED
    specs = D.adam_specs()
    stream = torch.cuda.current_stream()
    step_no = [0]

    def step(grads=None, adam_specs=None):
        step_no[0] += 1
        api.muon_step(D.params, D.grads if grads is None else grads, D.mom, D.groups, W.MUON_LR,
                      W.MUON_BETA, W.MUON_WD, wl.ns_steps, coeffs, flags, ws, stream=stream)
        sp = specs if adam_specs is None else adam_specs
        if sp:
            api.adamw_step(sp, step_no[0], stream=stream)

    def barrier():
        torch.cuda.synchronize()
        R.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x: float) -> float:
        return R.max(x, device=dev)

    for _ in range(args.warmup):
        step()
    barrier()
    if api.muon_query_status(ws) != N.MUON_OK:
        raise RuntimeError("device status word reports an error after warm-up")

    # ---------------------------------------------------- device-timed region
    # The K timed steps carry no per-kernel events (an event pair around
    # every launch would add its own gaps to launch-bound steps); the
    # per-kernel breakdown comes from K more steps with the profiler on.
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record(stream)
    for k in range(args.steps):
        step()
        evs[k + 1].record(stream)
    e0, e1 = evs[0], evs[-1]
    barrier()
    clk = clocks.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1))
    per_step = sorted(evs[k].elapsed_time(evs[k + 1]) for k in range(args.steps))
    # ------------------------------------------ per-kernel breakdown (profiled)
    api.muon_profiler_reset()
    api.muon_profiler_enable(True)
    barrier()
    for k in range(args.steps):
        step()
    barrier()
    api.muon_profiler_enable(False)

    def quantile(q):
        x = q * (len(per_step) - 1)
        lo = int(x)
        hi = min(lo + 1, len(per_step) - 1)
        return per_step[lo] + (per_step[hi] - per_step[lo]) * (x - lo)
    step_quantiles = {name: round(max_over_ranks(quantile(q)), 3)
                      for name, q in (("p10", 0.1), ("p50", 0.5), ("p90", 0.9))}
    prof = api.muon_profiler_read()
    ms_step = ms_total / args.steps

    # --------------------------------------------------------- end to end
    # Every step's gradients come from host memory.  They are copied on a copy
    # stream into one of two device gradient buffers while the previous step
    # computes (the next batch's gradients prefetched, as a training loop
    # would); every copy is inside the timed region, which starts before the
    # first copy and ends after the last step's status word is read back.
    e2e = None
    if D.host_grads is not None:
        h2d = sum(h.numel() * h.element_size() for h in D.host_grads)
        status_host = torch.empty(1, dtype=torch.int32, pin_memory=True)
        flats = [D.flat_grads, [torch.empty_like(g) for g in D.flat_grads]]
        views = [D.grad_views(f) for f in flats]
        vspecs = [D.adam_specs(v[1]) for v in views]
        copy_stream = torch.cuda.Stream(device=dev)
        ev_copy = [torch.cuda.Event(), torch.cuda.Event()]
        ev_step = [torch.cuda.Event(), torch.cuda.Event()]

        def copy_grads(b):
            with torch.cuda.stream(copy_stream):
                for g, h in zip(flats[b], D.host_grads):
                    g.copy_(h, non_blocking=True)
            ev_copy[b].record(copy_stream)

        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        copy_stream.wait_event(a0)
        copy_grads(0)
        for t in range(args.steps):
            b = t % 2
            if t + 1 < args.steps:
                if t >= 1:
                    copy_stream.wait_event(ev_step[1 - b])  # buffer last used by step t-1
                copy_grads(1 - b)
            stream.wait_event(ev_copy[b])
            step(views[b][0], vspecs[b])
            ev_step[b].record(stream)
            status_host.copy_(ws[:4].view(torch.int32), non_blocking=True)
        a1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(a0.elapsed_time(a1)) / args.steps
        e2e = {"value": round(e2e_ms, 3), "unit": "ms", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": 4,
               "path": ("pinned" if D.host_pinned else "pageable") +
                       " host grads -> cudaMemcpyAsync on a copy stream, double-buffered (next step's"
                       " grads copied while this step computes) -> muon_step + adamw_step -> status"
                       " word read back"}

    if rank == 0:
        work = algorithmic_work(wl)
        peaks, peak_src = load_peaks()
        ns_nom = wl.ns_flops_nominal()
        ns_exe = wl.ns_flops_executed()
        kinds = {k: v for k, v in prof.items() if v[1] > 0}
        ns_ms = sum(kinds.get(k, (0, 0))[0] for k in ("ns_gram", "ns_poly", "ns_axpy", "ns_axpy_update")) / args.steps
        # dominant kernel and its roofline
        dom = max(kinds.items(), key=lambda kv: kv[1][0])[0] if kinds else None
        launches = sum(v[1] for v in kinds.values())
        per_kernel = {}
        for k, (ms, n) in kinds.items():
            per_kernel[k] = {"ms_per_step": round(ms / args.steps, 4), "launches_per_step": n / args.steps,
                             "avg_launch_ms": round(ms / n, 4)}
        K = wl.ns_steps
        alg = {
            "ns_gram": ("tensor", work["gram_flops_executed"]),
            "ns_poly": ("tensor", work["poly_flops_executed"]),
            "ns_axpy": ("tensor", work["axpy_flops_executed"]),
            "ns_axpy_update": ("tensor", work["axpy_flops_executed"]),
            "momentum_norm": ("hbm", work["momentum_bytes"]),
            "momentum_rowq": ("hbm", work["momentum_bytes"]),
            "update": ("hbm", work["update_bytes"]),
            "normuon_update": ("hbm", work["update_bytes"]),
            "adamw": ("hbm", work["adamw_bytes"]),
        }
        # per-step algorithmic work of each kernel kind: GEMM kinds run once per
        # NS iteration (the last B.X is the fused-update kind), elementwise
        # once.  GEMMs count executed FLOPs (the roofline must not credit the
        # symmetric products with tiles they skip); nominal FLOPs are kept
        # per kernel beside them.
        n_axpy = K - 1 if "ns_axpy_update" in kinds else K
        nominal_step_work = {
            "ns_gram": work["gram_flops"] * K, "ns_poly": work["poly_flops"] * K,
            "ns_axpy": work["axpy_flops"] * n_axpy, "ns_axpy_update": work["axpy_flops"]}
        per_step_work = {
            "ns_gram": work["gram_flops_executed"] * K, "ns_poly": work["poly_flops_executed"] * K,
            "ns_axpy": work["axpy_flops_executed"] * n_axpy,
            "ns_axpy_update": work["axpy_flops_executed"],
            "momentum_norm": work["momentum_bytes"], "momentum_rowq": work["momentum_bytes"],
            "update": work["update_bytes"],
            "normuon_update": work["update_bytes"],
            "adamw": work["adamw_bytes"]}
        roof = None
        if dom in alg:
            bound = alg[dom][0]
            ms, n = kinds[dom]
            launches_per_step = n / args.steps
            per_launch = per_step_work[dom] / launches_per_step
            avg_s = ms / n / 1e3
            # DRAM bytes of an average launch: the captured pass times the
            # passes per step, over the launches per step
            passes = {"ns_axpy": n_axpy, "ns_gram": K, "ns_poly": K, "ns_axpy_update": 1}.get(dom, 1)
            cap_pass = captured_traffic(dom, wl.name)
            traffic = round(cap_pass * passes / launches_per_step) if cap_pass else None
            if bound == "tensor":
                ach = per_launch / avg_s / 1e12
                peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
                roof = {"bound": "tensor", "kernel": dom, "achieved": round(ach, 1), "peak": peak,
                        "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                        "traffic": traffic, "traffic_unit": "bytes per launch",
                        "peak_source": f"{peak_src} (sustained bf16 cuBLAS)",
                        "work_per_launch": per_launch, "work_unit": "executed FLOP"}
            else:
                ach = per_launch / avg_s / 1e9
                peak = peaks["hbm_gbs"]
                roof = {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": peak,
                        "unit": "GB/s", "frac": round(ach / peak, 4),
                        "traffic": traffic, "traffic_unit": "bytes per launch",
                        "peak_source": f"{peak_src} (HBM copy)",
                        "work_per_launch": per_launch, "work_unit": "algorithmic bytes"}
        ew = {}
        for k in ("momentum_norm", "momentum_rowq", "update", "normuon_update", "adamw"):
            if k in kinds:
                ew[k] = round(per_step_work[k] / (kinds[k][0] / args.steps / 1e3) / 1e9, 1)
        sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        for k in ("ns_gram", "ns_poly", "ns_axpy", "ns_axpy_update"):
            if k in kinds:
                sec = kinds[k][0] / args.steps / 1e3
                per_kernel[k]["executed_tflops"] = round(per_step_work[k] / sec / 1e12, 1)
                per_kernel[k]["executed_frac_of_sustained"] = round(per_step_work[k] / sec / 1e12 / sustained, 4)
                per_kernel[k]["nominal_tflops"] = round(nominal_step_work[k] / sec / 1e12, 1)
        res = {
            "metric": METRIC,
            "value": round(ms_step, 3),
            "unit": "ms",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 3),
            "step_ms_quantiles": step_quantiles,
            "higher_is_better": False,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl.name, "muon_params": wl.muon_params(), "adamw_params": wl.adamw_params(),
                       "muon_groups": [[s.rows, s.cols, s.count] for s in wl.muon],
                       "ns_steps": K, "grads": "bf16", "params_state": "fp32",
                       "l2": "inputs larger than L2 (no flush)", "parallelism": f"replicas x{world}",
                       "gemm_tiles": "128x256 single-CTA" if args.single_cta else
                       "CTA pairs: 256x256" if args.narrow_tiles else
                       "CTA pairs: 256x512 (Gram, B'X), 256x256 (A*A, fused update)" if args.wide_tiles else
                       "CTA pairs: Gram and B'X on 256x512 where the output width is a multiple of "
                       "512 and K >= 2048, else 256x256; A*A and the fused update 256x256",
                       "normuon": bool(args.normuon), "row_equilibrate": bool(args.row_equilibrate)},
            "ns_tflops_executed": round(ns_exe / (ns_ms / 1e3) / 1e12, 1) if ns_ms else None,
            "ns_frac_of_peak_executed": round(ns_exe / (ns_ms / 1e3) / 1e12 / sustained, 4) if ns_ms else None,
            "ns_ms_per_step": round(ns_ms, 3),
            # nominal FLOPs (4 m^2 n + 2 m^3 per iteration) credit the symmetric
            # products with the tiles they skip, so this can exceed 1
            "ns_tflops_nominal": round(ns_nom / (ns_ms / 1e3) / 1e12, 1) if ns_ms else None,
            "ns_frac_of_peak_nominal_counting_skipped_tiles":
                round(ns_nom / (ns_ms / 1e3) / 1e12 / sustained, 4) if ns_ms else None,
            "elementwise_gbs": ew,
            "roofline": roof,
            "per_kernel": per_kernel,
            "gpu_launches": launches,
            "clocks": clk,
            "e2e": e2e,
        }
        if not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(wl, samples=3, with_full_reference_step=True)
        print(json.dumps(res), flush=True)
    R.close()


def run_distributed(args):
    """One data-parallel optimizer step of the workload shared by all ranks."""
    import torch
    from muon_polar_orthogonalized_b200 import workloads as W
    from muon_polar_orthogonalized_b200.build import build
    from muon_polar_orthogonalized_b200.distributed import DistributedMuonAdamW

    R = RankContext("nccl")
    world, rank, local = R.world, R.rank, R.local
    if rank == 0:
        build()
    R.barrier()
    if rank != 0:
        build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = W.get(args.workload)
    if any(s.grad_dtype != "bf16" for s in wl.muon) or any(t.grad_dtype != "bf16" for t in wl.adamw):
        raise SystemExit("--distributed takes a workload with bf16 gradients")
    # placeholders of the right shapes (no storage): the optimizer moves every
    # parameter into its flat buffers, which are then filled with the draws
    zero = torch.zeros((), device=dev)
    mats = [zero.expand(s.rows, s.cols) for s in wl.muon for _ in range(s.count)]
    adam = [zero.expand(*t.shape) for t in wl.adamw for _ in range(t.count)]
    groups = [dict(params=adam[i:i + 1], lr=W.ADAMW_LR, betas=W.ADAMW_BETAS, eps=W.ADAMW_EPS,
                   weight_decay=0.0) for i in range(len(adam))]
    opt = DistributedMuonAdamW(mats, groups, process_group=None, grad_dtype=torch.bfloat16,
                               adamw_grad_dtype=torch.bfloat16, lr=W.MUON_LR, momentum=W.MUON_BETA,
                               weight_decay=W.MUON_WD, ns_steps=wl.ns_steps)
    gen = W.device_generator(dev, wl.name, "W", "flat")
    opt.buf["muon_params"].normal_(0.0, 0.02, generator=gen)
    opt.buf["adamw_params"].normal_(0.0, 0.02, generator=gen)
    k = 0
    for gi, s in enumerate(wl.muon):
        for j in range(s.count):
            opt.muon_grads[k].copy_(W.device_grad(wl, s.rows, s.cols, torch.bfloat16, dev, gi, j))
            k += 1
    for gl in opt.adamw_grads:
        for g in gl:
            g.copy_(torch.randn(g.shape, generator=gen, device=dev).mul_(wl.grad_std))
    stream = torch.cuda.current_stream()

    def barrier():
        torch.cuda.synchronize()
        R.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        opt.step()
    barrier()
    ws = opt._local.workspace
    if opt.owned and api_status(ws) != 0:
        raise RuntimeError("device status word reports an error after warm-up")
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        opt.step()
    e1.record(stream)
    barrier()
    clk = clocks.stop()
    ms = R.max(e0.elapsed_time(e1), device=dev) / args.steps
    if rank == 0:
        ns_exe = wl.ns_flops_executed()
        res = {"metric": METRIC, "value": round(ms, 3), "unit": "ms", "n_gpus": world,
               "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
               "higher_is_better": False, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
               "data": "synthetic",
               "config": {"workload": wl.name, "muon_params": wl.muon_params(),
                          "adamw_params": wl.adamw_params(), "ns_steps": wl.ns_steps, "grads": "bf16",
                          "params_state": "fp32", "l2": "inputs larger than L2 (no flush)",
                          "parallelism": f"dp{world}: owner-sharded Muon, ZeRO-1 AdamW; one reduce_scatter "
                                         "and one all_gather per flat buffer (NCCL)",
                          "matrices_per_rank": [opt.owners.count(r) for r in range(world)]},
               "ns_tflops_executed_per_gpu": round(ns_exe / world / (ms / 1e3) / 1e12, 1),
               "clocks": clk, "e2e": None,
               "e2e_note": "the distributed mode times the device step only"}
        print(json.dumps(res), flush=True)
    R.close()


def api_status(ws) -> int:
    from muon_polar_orthogonalized_b200 import api
    return api.muon_query_status(ws)


# --------------------------------------------------------- CPU (oracle)
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_cores() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count()


def oracle_muon_shape_seconds(rows: int, cols: int, ns_steps: int, grad_std: float, seed: int = 0) -> float:
    """Wall seconds of the fp64 oracle's muon_step on one rows x cols matrix."""
    import numpy as np

    import oracle
    from muon_polar_orthogonalized_b200 import workloads as W
    rng = np.random.default_rng(seed)
    Wm = rng.standard_normal((rows, cols)) * 0.02
    G = rng.standard_normal((rows, cols)) * grad_std
    M = np.zeros_like(G)
    t0 = time.perf_counter()
    oracle.muon_step(Wm, G, M, W.MUON_LR, W.MUON_BETA, W.MUON_WD, ns_steps, W.NS_COEFFS_FIXED)
    return time.perf_counter() - t0


def oracle_adamw_seconds(numel: int, grad_std: float, seed: int = 0) -> float:
    import numpy as np

    import oracle
    from muon_polar_orthogonalized_b200 import workloads as W
    rng = np.random.default_rng(seed)
    p = rng.standard_normal(numel) * 0.02
    g = rng.standard_normal(numel) * grad_std
    z = np.zeros(numel)
    t0 = time.perf_counter()
    oracle.adamw_step(p, g, z, z.copy(), 1, W.ADAMW_LR, 0.9, 0.95, 1e-8, 0.0)
    return time.perf_counter() - t0


def oracle_sample_ms(wl) -> float:
    """One bounded sample of the oracle on the workload, scaled to ms per full
    step: one matrix of every oriented shape (m x n, m <= n: a tall group runs
    as its transpose, at the same cost) timed once, times the number of
    matrices of that shape; plus AdamW on up to 4M elements scaled by element
    count."""
    by_shape = {}
    for s in wl.muon:
        key = (min(s.rows, s.cols), max(s.rows, s.cols))
        by_shape[key] = by_shape.get(key, 0) + s.count
    muon_s = sum(n * oracle_muon_shape_seconds(m, nn, wl.ns_steps, wl.grad_std)
                 for (m, nn), n in by_shape.items())
    adam_s = 0.0
    n_adam = wl.adamw_params()
    if n_adam:
        k = min(n_adam, 1 << 22)
        adam_s = oracle_adamw_seconds(k, wl.grad_std) * (n_adam / k)
    return (muon_s + adam_s) * 1e3


def oracle_sample_description(wl) -> str:
    shapes = sorted({(min(s.rows, s.cols), max(s.rows, s.cols)) for s in wl.muon})
    n_adam = wl.adamw_params()
    return (f"fp64 NumPy muon_step timed on one matrix of each oriented shape "
            f"({', '.join(f'{m}x{n}' for m, n in shapes)}), scaled by the count of each to all "
            f"{sum(x.count for x in wl.muon)} matrices, plus AdamW on {min(n_adam, 1 << 22)} "
            f"elements scaled to {n_adam}")


def oracle_full_step_ms(wl) -> float:
    """The oracle's whole step on the workload, every matrix and every AdamW
    tensor, unextrapolated (inputs drawn per matrix, not kept)."""
    muon_s = 0.0
    for s in wl.muon:
        for j in range(s.count):
            muon_s += oracle_muon_shape_seconds(s.rows, s.cols, wl.ns_steps, wl.grad_std, seed=j)
    adam_s = sum(oracle_adamw_seconds(math.prod(t.shape), wl.grad_std, seed=j)
                 for t in wl.adamw for j in range(t.count))
    return (muon_s + adam_s) * 1e3


def cpu_baseline(wl, samples: int = 3, with_full_reference_step: bool = False):
    """The oracle, as it stands, on the host cores: the median of `samples`
    bounded samples (oracle_sample_ms) with their spread; a sample is
    extrapolated to the full step unless it already is the full step.  With
    with_full_reference_step, the d=768 transformer set's whole step is also
    timed unextrapolated beside it."""
    from muon_polar_orthogonalized_b200 import workloads as W
    vals = [oracle_sample_ms(wl) for _ in range(samples)]
    extrapolated = any(s.count > 1 for s in wl.muon) or any(t.count > 1 for t in wl.adamw) or \
        wl.adamw_params() > (1 << 22)
    out = {"value": round(statistics.median(vals), 1), "unit": "ms", "cores": oracle_cores(),
           "kind": "oracle", "cpu_model": cpu_model(),
           "sample": oracle_sample_description(wl) + f"; median of {samples} samples",
           "samples_ms": [round(v, 1) for v in vals],
           "spread_ms": [round(min(vals), 1), round(max(vals), 1)],
           "extrapolated": extrapolated}
    if with_full_reference_step and wl.name != "gpt_d768_12l":
        ref = W.get("gpt_d768_12l")
        out["full_step_unextrapolated"] = {
            "workload": ref.name, "ms": round(oracle_full_step_ms(ref), 1),
            "sample_estimate_ms": round(oracle_sample_ms(ref), 1)}
    return out


def run_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return  # the oracle arm runs on rank 0 only; other ranks exit without work
    from muon_polar_orthogonalized_b200 import workloads as W
    wl = W.get(args.workload)
    for _ in range(args.warmup):
        oracle_sample_ms(wl)
    vals = [oracle_sample_ms(wl) for _ in range(args.steps)]
    v = round(statistics.median(vals), 1)
    cb = {"value": v, "unit": "ms", "cores": oracle_cores(), "kind": "oracle", "cpu_model": cpu_model(),
          "sample": oracle_sample_description(wl) + f"; one sample per step, median of {args.steps}",
          "samples_ms": [round(x, 1) for x in vals], "spread_ms": [round(min(vals), 1), round(max(vals), 1)],
          "extrapolated": True}
    res = {"impl": "reference", "metric": METRIC, "value": v, "unit": "ms", "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": v, "higher_is_better": False,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": wl.name, "parallelism": "cpu oracle"},
           "cpu_baseline": cb,
           "e2e": {"value": v, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama_8b_32l")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--normuon", action="store_true",
                    help="row-normalise the orthogonalised update (NorMuon)")
    ap.add_argument("--row-equilibrate", action="store_true",
                    help="MuonEq row equilibration of the momentum-smoothed matrix before Newton-Schulz")
    ap.add_argument("--narrow-tiles", action="store_true",
                    help="Gram and B'X on 256x256 CTA-pair tiles for every shape")
    ap.add_argument("--wide-tiles", action="store_true",
                    help="Gram and B'X on 256x512 CTA-pair tiles for every shape")
    ap.add_argument("--single-cta", action="store_true",
                    help="Newton-Schulz GEMMs on single-CTA 128x256 tiles instead of CTA pairs")
    ap.add_argument("--distributed", action="store_true",
                    help="time the data-parallel optimizer (owner-sharded Muon, ZeRO-1 AdamW) over the ranks")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    elif args.distributed:
        run_distributed(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
