"""Python binding of the C ABI: same names, torch tensors in, pointers out.

Argument marshalling only: every step of the optimizer runs in the CUDA
library.  Tensors must already live on the current CUDA device; streams are
torch streams (default: the current stream).

The C ABI takes plain pointer arrays and cannot see their lengths or the
tensors behind them, so the binding checks what it marshals: list lengths
against the groups, and each tensor's device, dtype, contiguity and element
count against the layout the library will read and write.  Raw integer
pointers are passed through unchecked.
"""
from __future__ import annotations

import ctypes
from ctypes import c_double, c_float, c_int64, c_void_p
from typing import List, Optional, Sequence, Tuple

from . import _native as N
from ._native import AdamWGroup, MuonGroup, check

GroupSpec = Tuple[int, int, int, int, int, float]  # rows, cols, count, first, grad_dtype, lr_scale


def _stream_handle(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _ptrs(tensors) -> ctypes.Array:
    arr = (c_void_p * max(len(tensors), 1))()
    for i, t in enumerate(tensors):
        arr[i] = t if isinstance(t, int) else t.data_ptr()
    return arr


def _group_fields(s) -> Tuple[int, int, int, int, int]:
    if isinstance(s, MuonGroup):
        return s.rows, s.cols, s.count, s.first, s.grad_dtype
    r, c, n, first, dt, _ = s
    return int(r), int(c), int(n), int(first), int(dt)


def _torch_dtype(code: int):
    import torch
    return torch.bfloat16 if code == N.MUON_BF16 else torch.float32


def _check_tensor(t, what: str, numel: int, dtype) -> None:
    if isinstance(t, int):
        return
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous() and t.numel() == numel):
        raise ValueError(f"{what}: expected a contiguous CUDA {dtype} tensor of {numel} elements, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}"
                         + ("" if t.is_contiguous() else ", not contiguous"))


def _check_group_lists(groups: Sequence, lists) -> None:
    """lists: (name, tensors, dtype) with dtype None meaning the group's grad dtype."""
    for s in groups:
        r, c, n, first, dt = _group_fields(s)
        if n <= 0 or first < 0:
            continue   # the library rejects the group itself
        for name, seq, dtype in lists:
            if len(seq) < first + n:
                raise ValueError(f"{name}: {len(seq)} entries, the groups index up to {first + n - 1}")
            want = _torch_dtype(dt) if dtype is None else dtype
            for j in range(first, first + n):
                _check_tensor(seq[j], f"{name}[{j}]", r * c, want)


def _check_step_args(groups, params, grads, momentum) -> None:
    import torch
    _check_group_lists(groups, (("params", params, torch.float32), ("grads", grads, None),
                                ("momentum", momentum, torch.float32)))


def make_groups(specs: Sequence) -> ctypes.Array:
    arr = (MuonGroup * max(len(specs), 1))()
    for i, s in enumerate(specs):
        if isinstance(s, MuonGroup):
            arr[i] = s
        else:
            r, c, n, first, dt, ls = s
            arr[i] = MuonGroup(int(r), int(c), int(n), int(first), int(dt), float(ls))
    return arr


def _coeff_array(coeffs, ns_steps: int):
    if ns_steps == 0:
        return None
    flat: List[float] = []
    if len(coeffs) == 3 and not hasattr(coeffs[0], "__len__"):
        flat = [float(x) for x in coeffs] * ns_steps
    else:
        for row in list(coeffs)[:ns_steps]:
            vals = [float(x) for x in row]
            if len(vals) != 3:
                raise ValueError("coeffs: every row is one (a, b, c) triple")
            flat.extend(vals)
    if len(flat) != 3 * ns_steps:
        raise ValueError(f"coeffs: {len(flat) // 3} rows of (a, b, c) for ns_steps = {ns_steps}")
    arr = (c_float * len(flat))(*flat)
    return arr


def muon_workspace_size(groups: Sequence, flags: int = 0) -> int:
    g = make_groups(groups)
    return int(N.lib().muon_workspace_size(g, len(groups), flags))


def muon_workspace_min_size(groups: Sequence, flags: int = 0) -> int:
    g = make_groups(groups)
    return int(N.lib().muon_workspace_min_size(g, len(groups), flags))


def muon_step(params, grads, momentum, groups: Sequence, lr: float, beta: float, wd: float,
              ns_steps: int, coeffs, flags: int, workspace, workspace_bytes: Optional[int] = None,
              stream=None) -> None:
    """One Muon step; see include/muon_b200.h.  params/grads/momentum are lists
    of tensors (or raw pointers) in pointer-array order."""
    _check_step_args(groups, params, grads, momentum)
    g = make_groups(groups)
    ca = _coeff_array(coeffs, ns_steps)
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    ws = workspace if isinstance(workspace, int) else workspace.data_ptr()
    st = N.lib().muon_step(_ptrs(params), _ptrs(grads), _ptrs(momentum), g, len(groups),
                           float(lr), float(beta), float(wd), int(ns_steps), ca, int(flags),
                           c_void_p(ws), wsb, c_void_p(_stream_handle(stream)))
    check(st, "muon_step")


def muon_step_replicated(params, grads, momentum, groups: Sequence, lr: float, beta: float, wd: float,
                         ns_steps: int, coeffs, flags: int, workspace, replicas: Sequence[Sequence],
                         workspace_bytes: Optional[int] = None, stream=None) -> None:
    """muon_step that also writes each updated matrix into every replica list
    (replicas[r][i] is copy r of params[i]; tensors or raw device pointers,
    possibly in peer GPUs' memory)."""
    import torch
    _check_step_args(groups, params, grads, momentum)
    for r, rep in enumerate(replicas):
        _check_group_lists(groups, ((f"replicas[{r}]", rep, torch.float32),))
    g = make_groups(groups)
    ca = _coeff_array(coeffs, ns_steps)
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    ws = workspace if isinstance(workspace, int) else workspace.data_ptr()
    rows = [_ptrs(rep) for rep in replicas]
    table = (ctypes.POINTER(c_void_p) * max(len(rows), 1))(
        *[ctypes.cast(r, ctypes.POINTER(c_void_p)) for r in rows])
    st = N.lib().muon_step_replicated(_ptrs(params), _ptrs(grads), _ptrs(momentum), g, len(groups),
                                      float(lr), float(beta), float(wd), int(ns_steps), ca, int(flags),
                                      c_void_p(ws), wsb, table, len(rows), c_void_p(_stream_handle(stream)))
    check(st, "muon_step_replicated")


def muon_reduce_mean(dst: Sequence, sources: Sequence[Sequence], stream=None) -> None:
    """dst[i] <- mean over r of sources[r][i] (fp32 or bf16 tensors of one
    dtype; sources may live in peer GPUs' memory)."""
    import torch
    if not dst:
        return
    if dst[0].dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("muon_reduce_mean: tensors must be fp32 or bf16")
    dt = N.MUON_BF16 if dst[0].dtype == torch.bfloat16 else N.MUON_F32
    for r, src in enumerate(sources):
        if len(src) != len(dst):
            raise ValueError(f"muon_reduce_mean: sources[{r}] has {len(src)} tensors, dst {len(dst)}")
    for i, t in enumerate(dst):
        _check_tensor(t, f"dst[{i}]", t.numel(), dst[0].dtype)
        for r, src in enumerate(sources):
            _check_tensor(src[i], f"sources[{r}][{i}]", t.numel(), dst[0].dtype)
    numel = (c_int64 * len(dst))(*[t.numel() for t in dst])
    rows = [_ptrs(src) for src in sources]
    table = (ctypes.POINTER(c_void_p) * max(len(rows), 1))(
        *[ctypes.cast(r, ctypes.POINTER(c_void_p)) for r in rows])
    st = N.lib().muon_reduce_mean(_ptrs(dst), table, len(rows), numel, len(dst), dt,
                                  c_void_p(_stream_handle(stream)))
    check(st, "muon_reduce_mean")


def muon_step_scheduled(params, grads, momentum, groups: Sequence, lr: float, beta: float, wd: float,
                        ns_steps: int, coeffs, flags: int, workspace, schedule_state,
                        workspace_bytes: Optional[int] = None, stream=None) -> None:
    """muon_step with the learning rate multiplied by the device schedule
    state's lr_mult (schedule_state: a 16-byte device tensor, see
    new_schedule_state)."""
    _check_step_args(groups, params, grads, momentum)
    g = make_groups(groups)
    ca = _coeff_array(coeffs, ns_steps)
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    ws = workspace if isinstance(workspace, int) else workspace.data_ptr()
    st = N.lib().muon_step_scheduled(_ptrs(params), _ptrs(grads), _ptrs(momentum), g, len(groups),
                                     float(lr), float(beta), float(wd), int(ns_steps), ca, int(flags),
                                     c_void_p(ws), wsb, c_void_p(schedule_state.data_ptr()),
                                     c_void_p(_stream_handle(stream)))
    check(st, "muon_step_scheduled")


def new_schedule_state(device, lr_mult: float = 1.0, step: int = 0):
    """A device-resident schedule state {float lr_mult; float reserved; int64 step}."""
    import struct
    import torch
    raw = struct.pack("<ffq", float(lr_mult), 0.0, int(step))
    return torch.frombuffer(bytearray(raw), dtype=torch.uint8).to(device)


def read_schedule_state(state):
    import struct
    lr_mult, _, step = struct.unpack("<ffq", bytes(state.cpu().numpy().tobytes()))
    return lr_mult, step


def muon_schedule_advance(schedule_state, total_steps: int, warmup_frac: float = 0.1,
                          warmdown_frac: float = 0.2, final_frac: float = 0.1, stream=None) -> None:
    st = N.lib().muon_schedule_advance(c_void_p(schedule_state.data_ptr()), int(total_steps),
                                       float(warmup_frac), float(warmdown_frac), float(final_frac),
                                       c_void_p(_stream_handle(stream)))
    check(st, "muon_schedule_advance")


def muon_schedule_advance_cosine(schedule_state, total_steps: int, warmup_steps: int,
                                 final_frac: float = 0.1, stream=None) -> None:
    st = N.lib().muon_schedule_advance_cosine(c_void_p(schedule_state.data_ptr()), int(total_steps),
                                              int(warmup_steps), float(final_frac),
                                              c_void_p(_stream_handle(stream)))
    check(st, "muon_schedule_advance_cosine")


def muon_orthogonalize(inputs, outputs, groups: Sequence, ns_steps: int, coeffs, flags: int,
                       workspace, workspace_bytes: Optional[int] = None, stream=None) -> None:
    import torch
    _check_group_lists(groups, (("inputs", inputs, None), ("outputs", outputs, torch.float32)))
    g = make_groups(groups)
    ca = _coeff_array(coeffs, ns_steps)
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    ws = workspace if isinstance(workspace, int) else workspace.data_ptr()
    st = N.lib().muon_orthogonalize(_ptrs(inputs), _ptrs(outputs), g, len(groups), int(ns_steps), ca,
                                    int(flags), c_void_p(ws), wsb, c_void_p(_stream_handle(stream)))
    check(st, "muon_orthogonalize")


class AdamWSpec:
    """One AdamW group: lists of tensors plus hyperparameters."""

    def __init__(self, params, grads, exp_avg, exp_avg_sq, lr, beta1, beta2, eps, wd,
                 grad_dtype: Optional[int] = None):
        self.params, self.grads, self.exp_avg, self.exp_avg_sq = params, grads, exp_avg, exp_avg_sq
        self.lr, self.beta1, self.beta2, self.eps, self.wd = lr, beta1, beta2, eps, wd
        if grad_dtype is None:
            import torch
            grad_dtype = N.MUON_BF16 if (grads and grads[0].dtype == torch.bfloat16) else N.MUON_F32
        self.grad_dtype = grad_dtype


def _adamw_groups(groups: Sequence[AdamWSpec]):
    n = len(groups)
    arr = (AdamWGroup * max(n, 1))()
    keep = []
    import torch
    for i, g in enumerate(groups):
        n_t = len(g.params)
        for name in ("grads", "exp_avg", "exp_avg_sq"):
            if len(getattr(g, name)) != n_t:
                raise ValueError(f"AdamW group {i}: {len(getattr(g, name))} {name} for {n_t} params")
        for k, t in enumerate(g.params):
            ne = t.numel()
            _check_tensor(t, f"AdamW group {i} params[{k}]", ne, torch.float32)
            _check_tensor(g.grads[k], f"AdamW group {i} grads[{k}]", ne, _torch_dtype(int(g.grad_dtype)))
            _check_tensor(g.exp_avg[k], f"AdamW group {i} exp_avg[{k}]", ne, torch.float32)
            _check_tensor(g.exp_avg_sq[k], f"AdamW group {i} exp_avg_sq[{k}]", ne, torch.float32)
        p, gr, m, v = _ptrs(g.params), _ptrs(g.grads), _ptrs(g.exp_avg), _ptrs(g.exp_avg_sq)
        numel = (c_int64 * max(len(g.params), 1))(*[t.numel() for t in g.params])
        keep.extend([p, gr, m, v, numel])
        arr[i] = AdamWGroup(ctypes.cast(p, ctypes.POINTER(c_void_p)),
                            ctypes.cast(gr, ctypes.POINTER(c_void_p)),
                            ctypes.cast(m, ctypes.POINTER(c_void_p)),
                            ctypes.cast(v, ctypes.POINTER(c_void_p)),
                            numel, len(g.params), int(g.grad_dtype), float(g.lr), float(g.beta1),
                            float(g.beta2), float(g.eps), float(g.wd))
    return arr, keep


def adamw_step(groups: Sequence[AdamWSpec], step: int, stream=None) -> None:
    arr, keep = _adamw_groups(groups)
    st = N.lib().adamw_step(arr, len(groups), int(step), c_void_p(_stream_handle(stream)))
    check(st, "adamw_step")


def adamw_step_scheduled(groups: Sequence[AdamWSpec], schedule_state, stream=None) -> None:
    """adamw_step with lr * lr_mult and t = step read from the device schedule state."""
    arr, keep = _adamw_groups(groups)
    st = N.lib().adamw_step_scheduled(arr, len(groups), c_void_p(schedule_state.data_ptr()),
                                      c_void_p(_stream_handle(stream)))
    check(st, "adamw_step_scheduled")


def muon_query_status(workspace, stream=None) -> int:
    ws = workspace if isinstance(workspace, int) else workspace.data_ptr()
    return int(N.lib().muon_query_status(c_void_p(ws), c_void_p(_stream_handle(stream))))


def adamw_query_status(stream=None) -> int:
    """MUON_ERR_TIMEOUT if a bounded wait in an AdamW kernel on this device ran
    out since the last call (the record is then cleared), else MUON_OK."""
    return int(N.lib().adamw_query_status(c_void_p(_stream_handle(stream))))


# --------------------------------------------------------------- profiler
def muon_profiler_enable(on: bool) -> bool:
    return bool(N.lib().muon_profiler_enable(1 if on else 0))


def muon_profiler_reset() -> None:
    N.lib().muon_profiler_reset()


def muon_profiler_read() -> dict:
    """{kernel kind: (device ms summed, launches)} since the last reset."""
    L = N.lib()
    k = L.muon_kernel_kind_count()
    ms = (c_double * k)()
    cnt = (c_int64 * k)()
    L.muon_profiler_read(ms, cnt, k)
    return {L.muon_kernel_kind_name(i).decode(): (ms[i], int(cnt[i])) for i in range(k)}
