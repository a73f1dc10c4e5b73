"""Planted mistakes in copies of the oracle must fail its pins.

Each mutant below is a plausible slip in restating the pages (a dropped term,
a flipped sign, an operand on the wrong side, a missing transpose, a missing
bias correction).  The pin checkers of tests/test_oracle_pins.py must reject
every one, which shows the pins constrain each part of the oracle.  All of
this runs on the CPU against the oracle only.
"""
import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import (adamw_pin_failures, cosine_pin_failures, momentum_pin_failures,
                                    normuon_pin_failures, ns_pin_failures, rowq_pin_failures,
                                    schedule_pin_failures, update_pin_failures)


def _coeffs(coeffs, steps):
    arr = np.asarray(coeffs, dtype=np.float64)
    return [tuple(arr)] * steps if arr.ndim == 1 else [tuple(r) for r in arr[:steps]]


def _ns_variant(kind):
    def ns(g, coeffs=oracle.NS_COEFFS_FIXED, steps=5, eps=oracle.NS_EPS):
        x = np.asarray(g, dtype=np.float64)
        if kind == "norm_squared":
            x = x / (np.sum(x * x) + eps)
        elif kind == "norm_maxabs":
            x = x / (np.abs(x).max() + eps)
        else:
            x = x / (np.sqrt(np.sum(x * x)) + eps)
        tr = x.shape[0] > x.shape[1]
        if tr and kind != "no_orient":
            x = x.T
        cl = _coeffs(coeffs, steps)
        if kind == "reversed_table":
            cl = cl[::-1]
        for a, b, c in cl:
            A = x.T @ x if kind == "gram_wrong_side" else x @ x.T
            if kind == "drop_c":
                B = b * A
            elif kind == "sign_c":
                B = b * A - c * (A @ A)
            elif kind == "swap_bc":
                B = c * A + b * (A @ A)
            else:
                B = b * A + c * (A @ A)
            if kind == "x_times_b":
                x = a * x + x @ B
            elif kind == "drop_ax":
                x = B @ x
            else:
                x = a * x + B @ x
        if tr and kind not in ("no_orient", "no_transpose_back"):
            x = x.T
        return x
    return ns


NS_MUTANTS = ["norm_squared", "norm_maxabs", "reversed_table", "drop_c", "sign_c",
              "swap_bc", "drop_ax", "no_transpose_back"]


@pytest.mark.parametrize("kind", NS_MUTANTS)
def test_ns_mutant_caught(kind):
    assert ns_pin_failures(_ns_variant(kind)) != []


@pytest.mark.parametrize("kind", ["gram_wrong_side", "x_times_b"])
def test_ns_shape_mutant_caught(kind):
    """Operands on the wrong side either break shapes or fail a pin."""
    try:
        fails = ns_pin_failures(_ns_variant(kind))
    except ValueError:
        return  # matmul shape mismatch: caught
    assert fails != []


def test_ns_unmutated_copy_passes():
    assert ns_pin_failures(_ns_variant("none")) == []


def test_skipping_orientation_is_not_a_mistake():
    """Iterating on a tall matrix directly gives the same polynomial of the
    singular values (zero singular values stay zero); orientation only picks
    the smaller Gram product.  The pins accept it, as they should."""
    assert ns_pin_failures(_ns_variant("no_orient")) == []


def _mom_variant(kind):
    def mom(m, g, beta, nesterov=True):
        if kind == "ema":
            m_new = beta * m + (1 - beta) * g
        else:
            m_new = beta * m + g
        if not nesterov:
            return m_new, m_new.copy()
        if kind == "lookahead_old_buffer":
            return m_new, beta * m + g
        if kind == "lookahead_no_grad":
            return m_new, beta * m_new
        return m_new, beta * m_new + g
    return mom


@pytest.mark.parametrize("kind", ["ema", "lookahead_old_buffer", "lookahead_no_grad"])
def test_momentum_mutant_caught(kind):
    assert momentum_pin_failures(_mom_variant(kind)) != []


def _upd_variant(kind):
    def upd(w, u, lr, wd, cautious=True):
        if cautious:
            if kind == "strict_mask":
                mask = (u * w) > 0
            elif kind == "inverted_mask":
                mask = (u * w) <= 0
            else:
                mask = (u * w) >= 0
        else:
            mask = np.ones(w.shape, dtype=bool)
        if kind == "decay_sign":
            return w - lr * (u - wd * mask * w)
        if kind == "decay_no_lr":
            return w - lr * u - wd * mask * w
        if kind == "ignore_mask":
            return w - lr * (u + wd * w)
        return w - lr * (u + wd * mask * w)
    return upd


@pytest.mark.parametrize("kind", ["strict_mask", "inverted_mask", "decay_sign",
                                  "decay_no_lr", "ignore_mask"])
def test_update_mutant_caught(kind):
    assert update_pin_failures(_upd_variant(kind)) != []


def _adamw_variant(kind):
    def adamw(p, g, m, v, t, lr, b1, b2, eps, wd):
        if kind != "decay_after":
            p = p * (1 - lr * wd)
        m = b1 * m + (1 - b1) * g
        v = b2 * v + (1 - b2) * (np.abs(g) if kind == "v_uses_abs" else g * g)
        bc1 = 1 - b1 ** t
        bc2 = 1 - b2 ** t
        if kind == "no_bias_correction":
            bc1 = bc2 = 1.0
        if kind == "bc2_not_sqrt":
            denom = np.sqrt(v) / bc2 + eps
        elif kind == "eps_inside_sqrt":
            denom = np.sqrt(v / bc2 + eps)
        else:
            denom = np.sqrt(v) / np.sqrt(bc2) + eps
        p = p - (lr / bc1) * m / denom
        if kind == "decay_after":
            p = p * (1 - lr * wd)
        return p, m, v
    return adamw


@pytest.mark.parametrize("kind", ["no_bias_correction", "bc2_not_sqrt", "eps_inside_sqrt",
                                  "v_uses_abs", "decay_after"])
def test_adamw_mutant_caught(kind):
    assert adamw_pin_failures(_adamw_variant(kind)) != []


def _normuon_variant(kind):
    def norm(u, eps=oracle.NORMUON_EPS):
        u = np.asarray(u, dtype=np.float64)
        if kind == "wrong_axis":
            rms = np.sqrt(np.sum(u * u, axis=0, keepdims=True)) / np.sqrt(u.shape[0])
        elif kind == "no_sqrt_cols":
            rms = np.sqrt(np.sum(u * u, axis=-1, keepdims=True))
        elif kind == "whole_matrix":
            rms = np.sqrt(np.mean(u * u))
        else:
            rms = np.sqrt(np.sum(u * u, axis=-1, keepdims=True)) / np.sqrt(u.shape[-1])
        return u / (rms + eps)
    return norm


@pytest.mark.parametrize("kind", ["wrong_axis", "no_sqrt_cols", "whole_matrix"])
def test_normuon_mutant_caught(kind):
    assert normuon_pin_failures(_normuon_variant(kind)) != []


def test_normuon_unmutated_copy_passes():
    assert normuon_pin_failures(_normuon_variant("none")) == []


def _sched_variant(kind):
    def sched(step, total, max_lr, min_lr, wu=0.1, wd=0.2):
        warm, down = int(total * wu), int(total * wd)
        flat = total - warm - down
        if kind == "no_warmup_ramp" and step < warm:
            return max_lr
        if step < warm:
            return max_lr * step / warm
        if step < warm + flat:
            return max_lr
        if step >= total:
            return min_lr
        dec = step - warm - flat
        if kind == "decay_to_zero":
            return max_lr * (1 - dec / down)
        if kind == "wrong_fraction":
            return min_lr + (max_lr - min_lr) * (1 - dec / total)
        return min_lr + (max_lr - min_lr) * (1 - dec / down)
    return sched


@pytest.mark.parametrize("kind", ["no_warmup_ramp", "decay_to_zero", "wrong_fraction"])
def test_schedule_mutant_caught(kind, pages):
    assert schedule_pin_failures(_sched_variant(kind), pages["trapezoid_chart"]) != []


def _cosine_variant(kind):
    def sched(step, total, max_lr, warmup, final=0.1):
        if step < warmup:
            return max_lr * (step + 1 if kind == "warmup_from_one" else step) / warmup
        last = total if kind == "phase_to_total" else total - 1
        if step >= last or last <= warmup:
            return max_lr * (0.0 if kind == "decay_to_zero" else final)
        p = (step - warmup) / (last - warmup)
        if kind == "linear":
            return max_lr * (final + (1 - final) * (1 - p))
        if kind == "sin_phase":
            return max_lr * (final + (1 - final) * 0.5 * (1 + np.sin(np.pi * p)))
        if kind == "decay_to_zero":
            return max_lr * 0.5 * (1 + np.cos(np.pi * p))
        return max_lr * (final + (1 - final) * 0.5 * (1 + np.cos(np.pi * p)))
    return sched


@pytest.mark.parametrize("kind", ["warmup_from_one", "phase_to_total", "decay_to_zero", "linear",
                                  "sin_phase"])
def test_cosine_mutant_caught(kind, pages):
    assert cosine_pin_failures(_cosine_variant(kind), pages["race_schedule"]) != []


def test_cosine_unmutated_copy_passes(pages):
    assert cosine_pin_failures(_cosine_variant("none"), pages["race_schedule"]) == []


def _rowq_variant(kind):
    """(equilibrate, step) pair with one planted slip."""
    def equil(x, eps=oracle.ROWEQ_EPS):
        x = np.asarray(x, dtype=np.float64)
        if kind == "columns":
            return x / (np.sqrt(np.sum(x * x, axis=0, keepdims=True)) + eps)
        if kind == "squared_norm":
            return x / (np.sum(x * x, axis=1, keepdims=True) + eps)
        if kind == "rms_not_norm":
            return x / (np.sqrt(np.mean(x * x, axis=1, keepdims=True)) + eps)
        if kind == "no_eps":
            return x / np.sqrt(np.sum(x * x, axis=1, keepdims=True))
        return x / (np.sqrt(np.sum(x * x, axis=1, keepdims=True)) + eps)

    def step(w, g, m, lr=0.02, beta=0.95):
        if kind == "on_grad":
            g = equil(g)
        m_new = beta * m + g
        mt = beta * m_new + g
        if kind == "into_momentum":
            m_new = equil(m_new)
            mt = beta * m_new + g
        if kind == "after_frobenius":
            mt = equil(mt / (np.linalg.norm(mt) + oracle.NS_EPS))
        elif kind == "after_orient":
            x = mt.T if mt.shape[0] > mt.shape[1] else mt
            x = equil(x)
            mt = x.T if mt.shape[0] > mt.shape[1] else x
        elif kind != "dropped" and kind != "on_grad":
            mt = equil(mt)
        u = oracle.newton_schulz(mt)
        return w - lr * u, m_new, u
    return equil, step


ROWQ_MUTANTS = ["columns", "squared_norm", "rms_not_norm", "no_eps", "on_grad", "into_momentum",
                "after_frobenius", "after_orient", "dropped"]


@pytest.mark.parametrize("kind", ROWQ_MUTANTS)
def test_rowq_mutant_caught(kind):
    assert rowq_pin_failures(*_rowq_variant(kind)) != []


def test_rowq_unmutated_copy_passes():
    assert rowq_pin_failures(*_rowq_variant("none")) == []
