"""B200 (sm_100a) Muon + AdamW optimizer step behind a C ABI.

The compute path is the native library libmuon_b200.so (hand-written CUDA for
sm_100a); this package only marshals arguments to it.  Importing the package
does not load the library; the first call does, and raises if it is missing.
The optimizer classes live in `optimizer` (MuonAdamW) and `distributed`
(DistributedMuonAdamW).
"""
from ._native import (MUON_BF16, MUON_CAUTIOUS_WD, MUON_F32, MUON_FP32_DEBUG,  # noqa: F401
                      MUON_NESTEROV, MUON_NORMUON, MUON_ROW_EQUILIBRATE, MUON_TC_NARROW_TILES,
                      MUON_TC_SINGLE_CTA, MUON_TC_WIDE_TILES, MUON_UNFUSED_UPDATE, MuonError,
                      MuonGroup)
from .api import (AdamWSpec, adamw_query_status, adamw_step, adamw_step_scheduled,  # noqa: F401
                  muon_orthogonalize,
                  muon_profiler_enable, muon_profiler_read, muon_profiler_reset,
                  muon_query_status, muon_reduce_mean, muon_schedule_advance,
                  muon_schedule_advance_cosine, muon_step, muon_step_replicated,
                  muon_step_scheduled, muon_workspace_min_size, muon_workspace_size,
                  new_schedule_state, read_schedule_state)

__all__ = [
    "muon_step", "muon_step_replicated", "muon_step_scheduled", "muon_orthogonalize",
    "muon_reduce_mean", "adamw_step", "adamw_step_scheduled", "adamw_query_status", "muon_workspace_size",
    "muon_workspace_min_size", "muon_query_status", "new_schedule_state", "read_schedule_state",
    "muon_schedule_advance", "muon_schedule_advance_cosine", "AdamWSpec", "MuonError", "MuonGroup",
    "muon_profiler_enable", "muon_profiler_read", "muon_profiler_reset",
]
