"""Plain fp64 restatement of the MuonAdamW optimizer step (oracle).

TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path.

Sources (page title, section):
  [MAC]  "Chapter 4: The MuonAdamW Optimizer" -- sections "The Muon Update
         Rule", "Polar Express: Newton-Schulz Orthogonalization", "The Full
         Muon Step", "The AdamW Step".
  [OPT]  "3.9 Optimizers: SGD, Adam, Adafactor, Lion, Muon & Shampoo" --
         sections "From Gradient Descent to Momentum", "Implementing AdamW
         from scratch", "Muon: Orthogonalizing the Update", "Exercises".
  [NC]   "Stuck at the optimizer after figuring out backward()" (nanochat
         discussion 856), reply by mira687: cautious weight decay mask,
         per-step Polar Express coefficient table.
  [RACE] "Muon vs AdamW, Lion and Sophia: a fair race", section "Muon".
  [TAB]  "A transformer trained with Muon", section "The optimizer, Muon".

Readings taken where the pages are silent or disagree are listed in the
module-level notes of each function.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np

# [MAC] "Polar Express: Newton-Schulz Orthogonalization" and [OPT] "Muon:
# Orthogonalizing the Update" both print this triple, used for every step.
NS_COEFFS_FIXED: Tuple[float, float, float] = (3.4445, -4.7750, 2.0315)
# [TAB] "The optimizer, Muon": the classical quintic with 15/8, -10/8, 3/8
# converges to exactly 1.
NS_COEFFS_CLASSICAL: Tuple[float, float, float] = (15.0 / 8.0, -10.0 / 8.0, 3.0 / 8.0)
# [OPT] newton_schulz5(..., eps=1e-7); [MAC] adds 1e-7 to the norm.
NS_EPS = 1e-7


def _coeff_list(coeffs, steps: int):
    """Per-step (a, b, c) list.  A single triple is repeated for every step;
    a table with one row per step ([NC]: per-iteration Polar Express triples)
    is used row by row."""
    arr = np.asarray(coeffs, dtype=np.float64)
    if arr.ndim == 1:
        return [tuple(arr)] * steps
    if arr.shape[0] < steps:
        raise ValueError("coefficient table shorter than ns_steps")
    return [tuple(row) for row in arr[:steps]]


# ----------------------------------------------------------------------------
# momentum
# ----------------------------------------------------------------------------
def nesterov_momentum(m: np.ndarray, g: np.ndarray, beta: float, nesterov: bool = True):
    """Momentum buffer update and the matrix that gets orthogonalised.

    [MAC] "The Muon Update Rule": m_t = beta*m_{t-1} + G_t, then the Nesterov
    lookahead m~_t = beta*m_t + G_t.  [OPT] "Muon: Orthogonalizing the Update"
    shows the heavy-ball form, which orthogonalises the buffer m_t itself.

    Returns (m_new, matrix_to_orthogonalise).
    """
    m_new = beta * m + g
    if nesterov:
        return m_new, beta * m_new + g
    return m_new, m_new.copy()


# ----------------------------------------------------------------------------
# Newton-Schulz / Polar Express
# ----------------------------------------------------------------------------
def frobenius_normalize(x: np.ndarray, eps: float = NS_EPS) -> np.ndarray:
    """X0 = M / (||M||_F + eps)  ([MAC] "Polar Express ..."; [OPT] newton_schulz5).

    The norm is the square root of the sum of squared entries ([RACE] "Muon").
    eps is added to the norm, not to its square.
    """
    return x / (np.sqrt(np.sum(x * x)) + eps)


def ns_polynomial(sigma, a: float, b: float, c: float):
    """p(s) = a s + b s^3 + c s^5: what one iteration does to each singular value
    ([MAC] "Why 5 Steps?"; [RACE] "Muon": 'on each singular value ... a step is a
    polynomial')."""
    s = np.asarray(sigma, dtype=np.float64)
    return a * s + b * s ** 3 + c * s ** 5


def ns_singular_value_map(sigma, coeffs=NS_COEFFS_FIXED, steps: int = 5):
    """Compose the per-step scalar polynomials: p_k o ... o p_1 (sigma)."""
    s = np.asarray(sigma, dtype=np.float64)
    for a, b, c in _coeff_list(coeffs, steps):
        s = ns_polynomial(s, a, b, c)
    return s


def newton_schulz(g: np.ndarray, coeffs=NS_COEFFS_FIXED, steps: int = 5,
                  eps: float = NS_EPS) -> np.ndarray:
    """Quintic Newton-Schulz orthogonalisation of one matrix, in fp64.

    Steps, in the order [MAC] "Polar Express: Newton-Schulz Orthogonalization"
    gives them:
      1. X = G / (||G||_F + eps)
      2. if rows > cols, iterate on X^T (the smaller Gram product)
      3. for each step k:  A = X X^T;  B = b_k A + c_k A A;  X = a_k X + B X
      4. transpose back if step 2 transposed.
    [OPT] transposes before normalising; the Frobenius norm is transpose
    invariant, so the two orders agree.
    """
    x = frobenius_normalize(np.asarray(g, dtype=np.float64), eps)
    transposed = x.shape[0] > x.shape[1]
    if transposed:
        x = x.T
    for a, b, c in _coeff_list(coeffs, steps):
        A = x @ x.T
        B = b * A + c * (A @ A)
        x = a * x + B @ x
    if transposed:
        x = x.T
    return np.ascontiguousarray(x)


def ns_closed_form(g: np.ndarray, coeffs=NS_COEFFS_FIXED, steps: int = 5,
                   eps: float = NS_EPS) -> np.ndarray:
    """What the iteration must equal, written through an SVD.

    Each step keeps the singular vectors and maps each singular value through
    p ([MAC] "Why 5 Steps?", [RACE] "Muon", [TAB] "The optimizer, Muon").  So
    NS(G) = U diag(p_k o ... o p_1 (s_i / (||G||_F + eps))) V^T with G = U S V^T.
    """
    g = np.asarray(g, dtype=np.float64)
    u, s, vt = np.linalg.svd(g, full_matrices=False)
    scale = 1.0 / (np.sqrt(np.sum(g * g)) + eps)
    return (u * ns_singular_value_map(s * scale, coeffs, steps)[None, :]) @ vt


# ----------------------------------------------------------------------------
# cautious weight decay + update
# ----------------------------------------------------------------------------
def cautious_mask(update: np.ndarray, w: np.ndarray) -> np.ndarray:
    """[NC]: decay only where the update and the parameter agree in sign,
    mask = (update * param) >= 0.  A zero product (either factor +-0) keeps the
    mask on.  Decided from the signs, which is what the product's sign is for
    finite values, so no underflow of a tiny product can flip it."""
    su = np.signbit(update)
    sw = np.signbit(w)
    return (su == sw) | (update == 0) | (w == 0)


def cautious_weight_decay_update(w: np.ndarray, update: np.ndarray, lr: float, wd: float,
                                 cautious: bool = True) -> np.ndarray:
    """W <- W - lr * (U + wd * mask * W).

    [MAC] "The Full Muon Step": decoupled decay p *= (1 - lr*wd) then the
    update.  [NC] gates that decay with the cautious mask.  Reading: the decay
    uses the pre-update W and the same lr as the update; without the cautious
    flag the mask is all ones (plain decoupled decay).
    """
    mask = cautious_mask(update, w) if cautious else np.ones(w.shape, dtype=bool)
    return w - lr * (update + wd * mask * w)


NORMUON_EPS = 1e-8


def normuon_rows(update: np.ndarray, eps: float = NORMUON_EPS) -> np.ndarray:
    """NorMuon ([MAC] "NorMuon: Normalized Muon"): every row of the update is
    divided by (its norm / sqrt(number of columns) + 1e-8), so each row's RMS
    becomes 1 (the learning rate then sets the step's RMS).  Rows are in the
    parameter orientation (the last dimension of the returned update)."""
    u = np.asarray(update, dtype=np.float64)
    rms = np.sqrt(np.sum(u * u, axis=-1, keepdims=True)) / np.sqrt(u.shape[-1])
    return u / (rms + eps)


# ----------------------------------------------------------------------------
# MuonEq row equilibration
# ----------------------------------------------------------------------------
ROWEQ_EPS = NS_EPS


def row_equilibrate(x: np.ndarray, eps: float = ROWEQ_EPS) -> np.ndarray:
    """MuonEq row equilibration.

    [NC] names it as one of the two optional extras layered on the
    orthogonalisation (leaving it out turns the update's direction by a
    cosine of 0.986) but prints no formula.  Reading: each row of the matrix,
    in parameter orientation, is divided by its Euclidean norm plus eps (the
    1e-7 the Frobenius normalisation adds), so every row enters Newton-Schulz
    with norm ~1 and a zero row stays zero.  It acts on the momentum-smoothed
    matrix, before the Frobenius normalisation; the momentum buffer itself is
    not changed.  The one figure the pages print for it (cos 0.986) was
    measured with a coefficient table they do not print, so it is context
    only; the pins are the row norms, the invariance of the result under
    positive row scaling of the input, and the closed form for a row-scaled
    matrix with orthonormal rows.
    """
    x = np.asarray(x, dtype=np.float64)
    n = np.sqrt(np.sum(x * x, axis=1, keepdims=True))
    return x / (n + eps)


def muon_step(w: np.ndarray, g: np.ndarray, m: np.ndarray, lr: float, beta: float, wd: float,
              ns_steps: int = 5, coeffs=NS_COEFFS_FIXED, nesterov: bool = True,
              cautious: bool = True, lr_scale: float = 1.0, eps: float = NS_EPS,
              normuon: bool = False, row_equilibrate_input: bool = False):
    """One Muon step on one matrix: momentum -> (MuonEq) -> NS -> (NorMuon) ->
    cautious decay + update.

    Returns (w_new, m_new, update) in fp64.  lr_scale is the per-matrix shape
    factor some recipes multiply the learning rate by; 1 gives W -= lr*update.
    With normuon the orthogonalised update is row-normalised first ([MAC]
    "The Full Muon Step": normalize_muon_update, then decay, then the step).
    With row_equilibrate_input the momentum-smoothed matrix is row-equilibrated
    before the orthogonalisation (row_equilibrate).
    """
    m_new, mt = nesterov_momentum(m, g, beta, nesterov)
    if row_equilibrate_input:
        mt = row_equilibrate(mt)
    u = newton_schulz(mt, coeffs, ns_steps, eps)
    if normuon:
        u = normuon_rows(u)
    w_new = cautious_weight_decay_update(w, u, lr * lr_scale, wd, cautious)
    return w_new, m_new, u


# ----------------------------------------------------------------------------
# learning-rate schedule (device-resident schedule state)
# ----------------------------------------------------------------------------
def trapezoid_lr(step: int, total_steps: int, max_lr: float, min_lr: float,
                 warmup_frac: float = 0.1, warmdown_frac: float = 0.2) -> float:
    """[MAC] "Learning Rate Schedule: Trapezoidal (Warmup-Flat-Warmdown)":
    linear warmup from 0 over int(total*warmup_frac) steps, max_lr for the
    flat middle, linear warmdown to min_lr over int(total*warmdown_frac)
    steps.  step counts from 0.  Reading for what the page leaves open: with
    no warmdown steps, or at and beyond total_steps, the value is min_lr.
    """
    warmup = int(total_steps * warmup_frac)
    warmdown = int(total_steps * warmdown_frac)
    flat = total_steps - warmup - warmdown
    if step < warmup:
        return max_lr * step / warmup
    if step < warmup + flat:
        return max_lr
    if warmdown == 0 or step >= total_steps:
        return min_lr
    decay = step - warmup - flat
    return min_lr + (max_lr - min_lr) * (1.0 - decay / warmdown)


def warmup_cosine_lr(step: int, total_steps: int, max_lr: float, warmup_steps: int,
                     final_frac: float = 0.1) -> float:
    """[RACE] "Muon vs AdamW, Lion and Sophia: a fair race" (the bake-off's
    learning rate, by step): a climb to the peak over the warmup, then a
    cosine down to a tenth of the peak by the last step.

    Readings for what the page leaves open: step counts from 0; the climb is
    linear from 0, max_lr*step/warmup_steps, as the trapezoidal schedule's; the
    cosine's phase runs from 0 at step == warmup_steps to pi at the last step,
    step == total_steps - 1, so lr = max_lr*(final + (1 - final)*(1 + cos(phase))/2);
    from the last step on (and when no step is left after the warmup) the
    value is final_frac*max_lr.
    """
    if step < warmup_steps:
        return max_lr * step / warmup_steps
    last = total_steps - 1
    if step >= last or last <= warmup_steps:
        return max_lr * final_frac
    phase = np.pi * (step - warmup_steps) / (last - warmup_steps)
    return max_lr * (final_frac + (1.0 - final_frac) * 0.5 * (1.0 + np.cos(phase)))


# ----------------------------------------------------------------------------
# AdamW
# ----------------------------------------------------------------------------
def adamw_step(p: np.ndarray, g: np.ndarray, m: np.ndarray, v: np.ndarray, t: int,
               lr: float, beta1: float, beta2: float, eps: float, wd: float):
    """One AdamW step with bias correction, t >= 1.

    [OPT] "Implementing AdamW from scratch" (and [MAC] "The AdamW Step"):
      p <- p (1 - lr wd)                    decoupled decay, on the weights
      m <- b1 m + (1 - b1) g
      v <- b2 v + (1 - b2) g^2
      p <- p - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
    Returns (p_new, m_new, v_new).
    """
    if t < 1:
        raise ValueError("AdamW step count starts at 1")
    p = p * (1.0 - lr * wd)
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    bc1 = 1.0 - beta1 ** t
    bc2 = 1.0 - beta2 ** t
    denom = np.sqrt(v) / np.sqrt(bc2) + eps
    p = p - (lr / bc1) * m / denom
    return p, m, v


# ----------------------------------------------------------------------------
# bf16 storage emulation (diagnostic only, never a parity gate)
# ----------------------------------------------------------------------------
def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to bfloat16 (nearest, ties to even) via fp32, returned as float64."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def newton_schulz_bf16_emulated(g: np.ndarray, coeffs=NS_COEFFS_FIXED, steps: int = 5,
                                eps: float = NS_EPS, fold_a: bool = False, exact_diag: bool = False,
                                diag_scale: bool = False, rounding=None) -> np.ndarray:
    """The iteration with bf16 rounding wherever a bf16 matrix is stored.

    [MAC] casts to bf16 before iterating and keeps X, A, B in bf16.  Storage
    points here: X0 = bf16(M) with the 1/(||M||+eps) factor carried as a
    scalar into the first Gram product and the first X update, A, B and each
    new X; products are exact (fp64) between roundings.  Used to tell bf16
    precision apart from kernel bugs; the gate is always the fp64 oracle.

    fold_a: the stored B holds a on its diagonal, B' = bf16(a I + b A + c A A),
    and X' = bf16(B' X): the same algebra, a*X + B X = (a I + B) X, with the
    rounding moved.
    exact_diag (with fold_a): the part of B''s diagonal that bf16 cannot hold,
    lo_i = d_i - bf16(d_i), is kept unrounded beside the stored B' and added
    back as lo_i * X_ij, so X' = bf16(B' X + lo * X): B' keeps its diagonal
    exactly and only its off-diagonal entries are rounded.
    diag_scale (with fold_a): row i of the product is multiplied by
    r_i = d_i / bf16(d_i), so X' = bf16(r * (B' X)): the diagonal term
    d_i X_i comes out exact and the off-diagonal terms of row i are scaled by
    r_i = 1 + O(2^-9).
    rounding: the function applied at every storage point (round_bf16 by
    default); the identity turns every mode into the exact iteration.
    """
    rnd = round_bf16 if rounding is None else rounding
    if (exact_diag or diag_scale) and not fold_a:
        raise ValueError("exact_diag and diag_scale apply to the folded B'")
    if exact_diag and diag_scale:
        raise ValueError("exact_diag and diag_scale are alternatives")
    g = np.asarray(g, dtype=np.float64)
    s = 1.0 / (np.sqrt(np.sum(g * g)) + eps)
    x = rnd(g)
    transposed = x.shape[0] > x.shape[1]
    if transposed:
        x = x.T
    for k, (a, b, c) in enumerate(_coeff_list(coeffs, steps)):
        sk = s if k == 0 else 1.0
        A = rnd(sk * sk * (x @ x.T))
        if fold_a:
            Bfull = a * np.eye(A.shape[0]) + b * A + c * (A @ A)
            B = rnd(Bfull)
            if exact_diag:
                lo = np.diag(Bfull) - np.diag(B)
                x = rnd(sk * (B @ x + lo[:, None] * x))
            elif diag_scale:
                d, h = np.diag(Bfull), np.diag(B)
                r = np.where(h != 0, d / np.where(h != 0, h, 1.0), 1.0)
                x = rnd(sk * (B @ x) * r[:, None])
            else:
                x = rnd(sk * (B @ x))
        else:
            B = rnd(b * A + c * (A @ A))
            x = rnd(sk * (a * x + B @ x))
    if steps == 0:
        x = rnd(s * x)
    if transposed:
        x = x.T
    return np.ascontiguousarray(x)
