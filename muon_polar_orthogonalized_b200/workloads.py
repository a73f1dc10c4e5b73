"""Seeded synthetic workloads for the Muon + AdamW optimizer step.

This module only draws random numbers and lays out parameter-set shapes.  It
holds none of the optimizer's arithmetic (no momentum, normalisation,
Newton-Schulz, weight decay or Adam math), so both the CUDA path and the CPU
oracle may take their inputs from it.

Shapes follow the parameter sets the optimizer pages talk about:
  * "Stuck at the optimizer after figuring out backward()" (nanochat
    discussion), mira687's reply: the 256x1024 MLP c_proj matrix of a depth-4
    model, an iid gradient and a "rank-8 plus noise" gradient with a decaying
    spectrum.
  * transformer parameter sets whose hidden matrices go to Muon and whose
    embedding / LM head / norm gains go to AdamW ("Chapter 4: The MuonAdamW
    Optimizer", section "Parameter Dispatch").

Every generator is deterministic in (config, index, step).
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import List, Optional, Sequence, Tuple

import numpy as np

# ----------------------------------------------------------------------------
# hyperparameters shared by the configs
# ----------------------------------------------------------------------------
NS_COEFFS_FIXED = (3.4445, -4.7750, 2.0315)   # one (a, b, c) triple per step
MUON_LR = 0.02
MUON_WD = 0.01
MUON_BETA = 0.95
ADAMW_LR = 3e-4
ADAMW_BETAS = (0.9, 0.95)
ADAMW_EPS = 1e-8


@dataclasses.dataclass(frozen=True)
class MuonShape:
    rows: int
    cols: int
    count: int
    grad_dtype: str          # "f32" or "bf16"
    role: str = ""


@dataclasses.dataclass(frozen=True)
class AdamWTensor:
    shape: Tuple[int, ...]
    count: int
    grad_dtype: str
    role: str = ""
    wd: float = 0.0
    init: str = "normal"     # "normal" (N(0, 0.02^2)) or "ones" (norm gains)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    muon: Tuple[MuonShape, ...]
    adamw: Tuple[AdamWTensor, ...]
    grad_kind: str           # "iid", "lowrank8", "lowrank64"
    grad_std: float
    ns_steps: int = 5

    # -- sizes ---------------------------------------------------------------
    def muon_params(self) -> int:
        return sum(s.rows * s.cols * s.count for s in self.muon)

    def adamw_params(self) -> int:
        return sum(int(np.prod(t.shape)) * t.count for t in self.adamw)

    def ns_flops_nominal(self, ns_steps: Optional[int] = None) -> float:
        """4 m^2 n + 2 m^3 per iteration for the wide orientation (m <= n)."""
        k = self.ns_steps if ns_steps is None else ns_steps
        tot = 0.0
        for s in self.muon:
            m, n = min(s.rows, s.cols), max(s.rows, s.cols)
            tot += s.count * (4.0 * m * m * n + 2.0 * m ** 3)
        return tot * k

    def ns_flops_executed(self, ns_steps: Optional[int] = None) -> float:
        """Symmetric-aware count: m^2 n (Gram, half) + m^3 (A.A, half) + 2 m^2 n."""
        k = self.ns_steps if ns_steps is None else ns_steps
        tot = 0.0
        for s in self.muon:
            m, n = min(s.rows, s.cols), max(s.rows, s.cols)
            tot += s.count * (3.0 * m * m * n + 1.0 * m ** 3)
        return tot * k

    def matrices(self) -> List[Tuple[int, int, int, str]]:
        """Flat list of (group index, rows, cols, grad dtype), one per matrix."""
        out = []
        for gi, s in enumerate(self.muon):
            out.extend([(gi, s.rows, s.cols, s.grad_dtype)] * s.count)
        return out

    def adamw_tensors(self) -> List[Tuple[int, Tuple[int, ...], str, float, str]]:
        out = []
        for ti, t in enumerate(self.adamw):
            out.extend([(ti, t.shape, t.grad_dtype, t.wd, t.init)] * t.count)
        return out


# ----------------------------------------------------------------------------
# the five parameter sets
# ----------------------------------------------------------------------------
def single_256x1024() -> Workload:
    """One fp32 256x1024 c_proj matrix plus a 256x4096 fp32 embedding."""
    return Workload(
        name="single_256x1024",
        muon=(MuonShape(256, 1024, 1, "f32", "c_proj"),),
        adamw=(AdamWTensor((256, 4096), 1, "f32", "wte"),),
        grad_kind="iid", grad_std=1.0)


def illcond_256x1024() -> Workload:
    """Rank-8 + noise gradients at 256x1024 and at its 1024x256 transpose."""
    return Workload(
        name="illcond_256x1024",
        muon=(MuonShape(256, 1024, 1, "f32", "wide"),
              MuonShape(1024, 256, 1, "f32", "tall")),
        adamw=(),
        grad_kind="lowrank8", grad_std=1.0)


def gpt_d768_12l() -> Workload:
    """12-layer d=768 transformer: Wq,Wk,Wv,Wo, MLP up (3072x768), down (768x3072)."""
    L, d = 12, 768
    return Workload(
        name="gpt_d768_12l",
        muon=(MuonShape(d, d, 4 * L, "bf16", "attn"),
              MuonShape(4 * d, d, L, "bf16", "mlp_up"),
              MuonShape(d, 4 * d, L, "bf16", "mlp_down")),
        adamw=(AdamWTensor((50304, d), 2, "bf16", "wte+lm_head"),),
        grad_kind="iid", grad_std=1e-3)


def gpt_d1664_26l() -> Workload:
    """26-layer d=1664 transformer with rank-64 + noise gradients and norm gains."""
    L, d = 26, 1664
    return Workload(
        name="gpt_d1664_26l",
        muon=(MuonShape(d, d, 4 * L, "bf16", "attn"),
              MuonShape(4 * d, d, L, "bf16", "mlp_up"),
              MuonShape(d, 4 * d, L, "bf16", "mlp_down")),
        adamw=(AdamWTensor((65536, d), 2, "bf16", "wte+lm_head"),
               AdamWTensor((d,), 2 * L + 1, "bf16", "norm_gain", init="ones")),
        grad_kind="lowrank64", grad_std=1e-3)


def llama_8b_32l() -> Workload:
    """32-layer 8B-shaped set: Wq,Wo 4096^2; Wk,Wv 1024x4096; gate,up 14336x4096; down 4096x14336."""
    L = 32
    return Workload(
        name="llama_8b_32l",
        muon=(MuonShape(4096, 4096, 2 * L, "bf16", "wq+wo"),
              MuonShape(1024, 4096, 2 * L, "bf16", "wk+wv"),
              MuonShape(14336, 4096, 2 * L, "bf16", "gate+up"),
              MuonShape(4096, 14336, L, "bf16", "down")),
        adamw=(AdamWTensor((128256, 4096), 2, "bf16", "wte+lm_head"),),
        grad_kind="iid", grad_std=1e-3)


def llama_8b_1layer() -> Workload:
    """One layer of the 8B-shaped set plus a 16384x4096 AdamW slice (a few GB;
    for profiler captures of the same kernels on the same shapes)."""
    return Workload(
        name="llama_8b_1layer",
        muon=(MuonShape(4096, 4096, 2, "bf16", "wq+wo"),
              MuonShape(1024, 4096, 2, "bf16", "wk+wv"),
              MuonShape(14336, 4096, 2, "bf16", "gate+up"),
              MuonShape(4096, 14336, 1, "bf16", "down")),
        adamw=(AdamWTensor((16384, 4096), 1, "bf16", "wte slice"),),
        grad_kind="iid", grad_std=1e-3)


WORKLOADS = {
    "single_256x1024": single_256x1024,
    "illcond_256x1024": illcond_256x1024,
    "gpt_d768_12l": gpt_d768_12l,
    "gpt_d1664_26l": gpt_d1664_26l,
    "llama_8b_32l": llama_8b_32l,
    "llama_8b_1layer": llama_8b_1layer,
}


def get(name: str) -> Workload:
    return WORKLOADS[name]()


# ----------------------------------------------------------------------------
# seeding
# ----------------------------------------------------------------------------
def seed_of(*parts) -> int:
    """Stable 63-bit seed from any tuple of printable parts."""
    h = hashlib.sha256("/".join(str(p) for p in parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _orthonormal(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))[None, :]


# ----------------------------------------------------------------------------
# host (NumPy) generators: small cases and sampled matrices
# ----------------------------------------------------------------------------
def lowrank_spectrum_grad(rows: int, cols: int, rank: int, sigma: Sequence[float],
                          noise: float, signal_seed: int, noise_seed: int) -> np.ndarray:
    """G = sum_i sigma_i u_i v_i^T + noise * N(0,1), u and v orthonormal (QR).

    The signal part depends only on signal_seed, so consecutive steps share the
    same singular directions and only the noise is fresh.  Returned as float64;
    callers round to the storage dtype they need.
    """
    rng = np.random.default_rng(signal_seed)
    u = _orthonormal(rng, rows, rank)
    v = _orthonormal(rng, cols, rank)
    g = (u * np.asarray(sigma, dtype=np.float64)[None, :]) @ v.T
    g += noise * np.random.default_rng(noise_seed).standard_normal((rows, cols))
    return g


def illcond_grad(step: int, noise: float = 1e-3, tall: bool = False) -> np.ndarray:
    """Rank-8 gradient with s_i = 10^(-i/2) plus noise at 256x1024.

    The tall variant is exactly the transpose of the wide one.  Signal seed 1,
    noise seed 100 + step.
    """
    sigma = [10.0 ** (-i / 2.0) for i in range(8)]
    g = lowrank_spectrum_grad(256, 1024, 8, sigma, noise, 1, 100 + step)
    return g.T.copy() if tall else g


def iid_normal(shape, std: float, seed: int) -> np.ndarray:
    return std * np.random.default_rng(seed).standard_normal(shape)


def to_bf16_bits_rne(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest even) as uint16 bit patterns.

    Storage conversion only: lets a generator hand both sides identical bf16
    gradients.  NaN is not expected in generated data.
    """
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_through_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Value of x after storing it as `dtype` ("f32" or "bf16"), as float64."""
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_bits_to_f64(to_bf16_bits_rne(x))
    raise ValueError(dtype)


def host_muon_inputs(wl: Workload, mat_index: int, step: int = 0):
    """(W, G, M) as float64 arrays holding exactly the stored values of matrix `mat_index`.

    W ~ N(0, 0.02^2) stored fp32, M = 0 at step 0, G per the workload's kind
    stored in its grad dtype.  Used for host-side cases; device workloads use
    `device_muon_inputs` instead.
    """
    gi, r, c, gd = wl.matrices()[mat_index]
    W = round_through_dtype(iid_normal((r, c), 0.02, seed_of(wl.name, "W", mat_index)), "f32")
    if wl.grad_kind == "iid":
        G = iid_normal((r, c), wl.grad_std, seed_of(wl.name, "G", mat_index, step))
    elif wl.grad_kind == "lowrank8":
        G = illcond_grad(step, tall=(r > c))
    else:
        raise ValueError("host generator supports iid and lowrank8 kinds")
    G = round_through_dtype(G, gd)
    M = np.zeros((r, c))
    return W, G, M


# ----------------------------------------------------------------------------
# device (torch) generators: full-size workloads
# ----------------------------------------------------------------------------
def device_generator(device, *parts):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed_of(*parts))
    return g


def device_grad(wl: Workload, rows: int, cols: int, dtype, device, *parts):
    """A gradient of the workload's kind drawn on `device` (torch), seeded by `parts`."""
    import torch
    gen = device_generator(device, wl.name, "G", *parts)
    if wl.grad_kind == "iid":
        g = torch.randn(rows, cols, generator=gen, device=device, dtype=torch.float32)
        g.mul_(wl.grad_std)
    elif wl.grad_kind == "lowrank64":
        # sum_{i<64} s_i u_i v_i^T with s_i = 10^(-i/32), Gaussian factors
        # (nearly orthonormal at these sizes), plus 1e-3 N(0,1) noise, then
        # rescaled to entry RMS grad_std.
        k = 64
        u = torch.randn(rows, k, generator=gen, device=device) / rows ** 0.5
        v = torch.randn(cols, k, generator=gen, device=device) / cols ** 0.5
        s = 10.0 ** (-torch.arange(k, device=device, dtype=torch.float32) / 32.0)
        g = (u * s[None, :]) @ v.T
        g.add_(torch.randn(rows, cols, generator=gen, device=device), alpha=1e-3)
        g.mul_(wl.grad_std / g.pow(2).mean().sqrt())
    elif wl.grad_kind == "lowrank8":
        g = torch.from_numpy(illcond_grad(int(parts[-1]) if parts else 0,
                                          tall=rows > cols)).to(device=device, dtype=torch.float32)
    else:
        raise ValueError(wl.grad_kind)
    return g.to(dtype)
