"""CPU fp64 oracle for the Muon + AdamW optimizer step.

TEST INFRASTRUCTURE ONLY.  The product path (the CUDA library and its Python
binding) never imports, links or calls anything in this package; only the
tests, the package smoke check and the benchmark's CPU-baseline leg do.

Every function restates a step as the optimizer pages describe it, in plain
NumPy float64 with library matmuls and no blocking or fusion, so that a reader
can check it against the pages by eye.  Each function is pinned by tests in
``tests/test_oracle_pins.py`` against facts the pages or the mathematics fix
(closed forms through an SVD, the classical Newton-Schulz limit, AdamW's
sign-at-step-one property, values the pages print).  No function here is
"parity unpinned".
"""
from .muon_ref import (  # noqa: F401
    NS_COEFFS_FIXED,
    NS_COEFFS_CLASSICAL,
    NS_EPS,
    nesterov_momentum,
    frobenius_normalize,
    ns_polynomial,
    ns_singular_value_map,
    newton_schulz,
    ns_closed_form,
    cautious_mask,
    cautious_weight_decay_update,
    muon_step,
    normuon_rows,
    NORMUON_EPS,
    row_equilibrate,
    ROWEQ_EPS,
    adamw_step,
    trapezoid_lr,
    warmup_cosine_lr,
    round_bf16,
    newton_schulz_bf16_emulated,
)
