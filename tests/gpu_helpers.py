"""Shared helpers of the GPU parity tests: exact host<->device copies of the
seeded inputs, and error measures.  No optimizer arithmetic lives here."""
import numpy as np
import torch

from muon_polar_orthogonalized_b200 import workloads as wl


def dev_tensor(x64: np.ndarray, dtype: str, device) -> torch.Tensor:
    """Device tensor holding x64 stored as dtype ("f32" or "bf16")."""
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(x64, dtype=np.float32)).to(device)
    bits = wl.to_bf16_bits_rne(x64)
    return torch.from_numpy(bits.view(np.int16)).to(device).view(torch.bfloat16)


def host64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a device tensor's stored values."""
    if t.dtype == torch.bfloat16:
        bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        return wl.bf16_bits_to_f64(bits)
    return t.detach().cpu().double().numpy()


def rel(a, b) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
