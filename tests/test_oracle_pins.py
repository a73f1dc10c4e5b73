"""Pins for the CPU oracle: facts the pages and the mathematics fix.

Each pin checker takes the implementation under test as an argument and
returns the names of the pins it fails, so the same checkers also run against
deliberately broken copies of the oracle (tests/test_oracle_mutations.py):
a plausible slip (a dropped term, a wrong sign, a transposed operand, a missing
bias correction) must trip at least one pin.

Sources (page title, section):
  "Chapter 4: The MuonAdamW Optimizer" -- Polar Express, The Full Muon Step,
      The AdamW Step.
  "3.9 Optimizers: SGD, Adam, Adafactor, Lion, Muon & Shampoo" -- From Gradient
      Descent to Momentum, Implementing AdamW from scratch, Muon:
      Orthogonalizing the Update, Exercises 2, 3(b), 6(b).
  "Muon vs AdamW, Lion and Sophia: a fair race" -- Muon (QR test, torch cosine).
  "A transformer trained with Muon" -- The optimizer, Muon (5x8 spreads).
  "Stuck at the optimizer after figuring out backward()" -- mira687's reply
      (cautious mask, AdamW step-1 = sign(g), cos 0.797, ns_steps 1 vs 5).
"""
import math

import numpy as np
import pytest

import oracle
from muon_polar_orthogonalized_b200 import workloads as wl

FIXED = oracle.NS_COEFFS_FIXED
CLASSICAL = oracle.NS_COEFFS_CLASSICAL


def _rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    if a.shape != b.shape:
        return float("inf")
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def _qr_orthonormal(rng, n, k):
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))[None, :]


# ============================================================================
# Newton-Schulz pins
# ============================================================================
def ns_pin_failures(ns, poly_map=oracle.ns_singular_value_map):
    """Pins on an NS implementation ns(G, coeffs, steps) -> X."""
    fails = []
    rng = np.random.default_rng(1234)

    # (1) SVD closed form: each step maps singular values by p and keeps the
    # singular vectors; the closed form is assembled here from numpy's SVD and
    # the scalar polynomial, not from the matrix iteration.
    for shape in [(7, 13), (13, 7), (16, 16), (5, 8), (1, 9), (9, 1)]:
        g = rng.standard_normal(shape)
        for steps in (1, 2, 5):
            u, s, vt = np.linalg.svd(g, full_matrices=False)
            x0 = s / (math.sqrt(float((g * g).sum())) + oracle.NS_EPS)
            ref = (u * poly_map(x0, FIXED, steps)[None, :]) @ vt
            if _rel(ns(g, FIXED, steps), ref) > 1e-10:
                fails.append(f"svd_closed_form{shape}x{steps}")
                break
    # a per-step table is applied in order (Polar Express style rows)
    table = np.array([[3.0, -3.2, 1.2], [2.5, -1.5, 0.5], [1.875, -1.25, 0.375]])
    g = rng.standard_normal((6, 11))
    u, s, vt = np.linalg.svd(g, full_matrices=False)
    x = s / (math.sqrt(float((g * g).sum())) + oracle.NS_EPS)
    for a, b, c in table:
        x = a * x + b * x ** 3 + c * x ** 5
    if _rel(ns(g, table, 3), (u * x[None, :]) @ vt) > 1e-10:
        fails.append("per_step_table_order")

    # (2) classical quintic (15/8, -10/8, 3/8) converges to the polar factor
    # U V^T ("A transformer trained with Muon"), which also equals
    # (M M^T)^(-1/2) M ("3.9 Optimizers", exercise 6(b)).
    for shape in [(6, 10), (10, 6), (8, 8)]:
        k = min(shape)
        uu = _qr_orthonormal(rng, shape[0], k)
        vv = _qr_orthonormal(rng, shape[1], k)
        sig = np.linspace(1.0, 0.4, k)
        m = (uu * sig[None, :]) @ vv.T
        polar = uu @ vv.T
        if _rel(ns(m, CLASSICAL, 40), polar) > 1e-9:
            fails.append(f"classical_limit{shape}")
        if shape[0] <= shape[1]:
            w, q = np.linalg.eigh(m @ m.T)
            inv_sqrt = (q / np.sqrt(w)[None, :]) @ q.T
            if _rel(ns(m, CLASSICAL, 40), inv_sqrt @ m) > 1e-9:
                fails.append(f"shampoo_identity{shape}")

    # (3) "A fair race", Muon: U, V from QR, singular values 0.1 .. 10; the
    # result is diagonal in those directions with entries in [0.6, 1.2].
    n, mcols = 32, 64
    uu = _qr_orthonormal(rng, n, n)
    vv = _qr_orthonormal(rng, mcols, n)
    sig = np.geomspace(0.1, 10.0, n)
    g = (uu * sig[None, :]) @ vv.T
    d = uu.T @ ns(g, FIXED, 5) @ vv
    off = d - np.diag(np.diag(d))
    if np.abs(off).max() > 1e-10:
        fails.append("qr_diagonal")
    if not (0.6 <= np.diag(d).min() and np.diag(d).max() <= 1.2):
        fails.append("qr_band")

    # (4) scalar cases.  Orthonormal rows scaled by alpha: every normalised
    # singular value is 1/sqrt(k), so X = p^5(1/sqrt(k)) Q.
    k, ncols = 4, 12
    q = _qr_orthonormal(rng, ncols, k).T
    out = ns(3.7 * q, FIXED, 5)
    target = 3.7 / (3.7 * math.sqrt(k) + oracle.NS_EPS)
    for _ in range(5):
        a, b, c = FIXED
        target = a * target + b * target ** 3 + c * target ** 5
    if _rel(out, target * q) > 1e-9:
        fails.append("orthonormal_rows")
    # diagonal matrix: elementwise map of |d_i| / ||d|| with sign kept
    dg = np.diag([2.0, -1.0, 0.5])
    nrm = math.sqrt(4 + 1 + 0.25) + oracle.NS_EPS
    want = np.diag([np.sign(v) * poly_map(abs(v) / nrm, FIXED, 5) for v in (2.0, -1.0, 0.5)])
    if _rel(ns(dg, FIXED, 5), want) > 1e-12:
        fails.append("diagonal")

    # (5) zero input stays zero (the eps in the normalisation exists for it)
    if np.abs(ns(np.zeros((3, 5)), FIXED, 5)).max() != 0.0:
        fails.append("zero_input")

    # (6) orientation: a tall matrix is iterated as its transpose, so the
    # result for G^T is the transpose of the result for G.
    g = rng.standard_normal((5, 9))
    if _rel(ns(g.T.copy(), FIXED, 5), ns(g, FIXED, 5).T) > 1e-13:
        fails.append("orientation")
    return fails


def test_ns_pins():
    assert ns_pin_failures(oracle.newton_schulz) == []


def test_ns_closed_form_function_matches_iteration():
    rng = np.random.default_rng(7)
    for shape in [(12, 20), (20, 12), (17, 17)]:
        g = rng.standard_normal(shape)
        assert _rel(oracle.newton_schulz(g), oracle.ns_closed_form(g)) < 1e-11


def test_polynomial_values(pages):
    a, b, c = pages["ns_coeffs_fixed"]
    assert (a, b, c) == FIXED
    # slope at 0 is a: "about three and a half times a step" for small values
    assert abs(a - pages["small_sigma_gain_per_step"]) < 0.1
    # classical quintic: fixed point at 1 with zero slope (converges to exactly 1)
    ca, cb, cc = pages["ns_coeffs_classical"]
    assert (ca, cb, cc) == CLASSICAL
    assert abs(oracle.ns_polynomial(1.0, ca, cb, cc) - 1.0) < 1e-15
    assert abs(ca + 3 * cb + 5 * cc) < 1e-15
    # the fixed triple does not reach 1: p(1) = a + b + c
    assert abs(oracle.ns_polynomial(1.0, a, b, c) - (a + b + c)) < 1e-15


def test_envelope_near_one_band(pages):
    """Five fixed-triple steps keep normalised singular values in a band around 1.

    'A fair race': values near one are kept between about 0.7 and 1.2; small
    values are pushed up.  Over sigma in [1e-3, 1] the 5-step map lands in
    [0.47, 1.21]; over [0.05, 1] (the "near one" region after two steps of
    growth) it stays inside [0.68, 1.21]."""
    s = np.geomspace(1e-3, 1.0, 20001)
    y = oracle.ns_singular_value_map(s, FIXED, 5)
    assert 0.45 < y.min() < 0.48 and 1.19 < y.max() < 1.21
    lo, hi = pages["near_one_band"]
    y2 = oracle.ns_singular_value_map(np.geomspace(0.05, 1.0, 2001), FIXED, 5)
    assert lo - 0.03 <= y2.min() and y2.max() <= hi + 0.01


def test_p4_spread_approximate(pages):
    """'A transformer trained with Muon': a 5x8 matrix with singular values from
    1 down to 0.001.  The page prints a Muon spread of 2.60 (values 0.45-1.17)
    and a classical spread of 45.1.  Its exact singular values are not printed;
    with geometric spacing the oracle gives 2.44 / 43.9, so this is an
    approximate pin (Muon's spread tiny next to the classical one)."""
    rng = np.random.default_rng(5)
    u = _qr_orthonormal(rng, 5, 5)
    v = _qr_orthonormal(rng, 8, 5)
    sig = np.geomspace(*pages["p4_5x8_sigma_range"], 5)
    g = (u * sig[None, :]) @ v.T
    sm = np.linalg.svd(oracle.newton_schulz(g, FIXED, 5), compute_uv=False)
    sc = np.linalg.svd(oracle.newton_schulz(g, CLASSICAL, 5), compute_uv=False)
    spread_m, spread_c = sm.max() / sm.min(), sc.max() / sc.min()
    assert abs(spread_m - pages["p4_muon_spread"]) < 0.35
    assert abs(spread_c - pages["p4_classical_spread"]) < 5.0
    lo, hi = pages["p4_muon_values"]
    assert lo - 0.05 < sm.min() and sm.max() < hi + 0.05


def test_ns_steps_flatten_conditioning():
    """mira687's reply: ns_steps 1 leaves the update's conditioning poor, 5
    flattens it (qualitative; the page's numbers use other coefficients)."""
    for noise in (1e-3, 1e-4):
        g = wl.lowrank_spectrum_grad(256, 1024, 8, [10 ** (-i / 2) for i in range(8)],
                                     noise, 1, 100)
        conds = {}
        for k in (1, 3, 5):
            s = np.linalg.svd(oracle.newton_schulz(g, FIXED, k), compute_uv=False)
            conds[k] = s.max() / s.min()
        assert conds[1] > 5 * conds[5], conds
        assert conds[3] > conds[5], conds
        assert conds[5] < 2.5, conds


def test_iid_condition_matches_page(pages):
    """Input-generator check: an iid 256x1024 Gaussian has condition ~2.98."""
    g = wl.iid_normal((256, 1024), 1.0, 0)
    s = np.linalg.svd(g, compute_uv=False)
    assert abs(s.max() / s.min() - pages["iid_256x1024_condition"]) < 0.1


def test_torch_muon_cross_check(pages):
    """'A fair race', Muon: our update moves each matrix in the direction
    PyTorch's Muon does, to a cosine of 0.99 (PyTorch iterates in bf16)."""
    torch = pytest.importorskip("torch")
    if not hasattr(torch.optim, "Muon"):
        pytest.skip("torch.optim.Muon not available")
    g = wl.iid_normal((256, 1024), 1.0, 11)
    p = torch.nn.Parameter(torch.zeros(256, 1024, dtype=torch.float32))
    p.grad = torch.from_numpy(g.astype(np.float32))
    opt = torch.optim.Muon([p], lr=1.0, weight_decay=0.0, momentum=0.95, nesterov=True)
    opt.step()
    upd_t = -p.detach().double().numpy()
    _, _, u = oracle.muon_step(np.zeros_like(g), g, np.zeros_like(g), 1.0, 0.95, 0.0)
    cos = float((upd_t * u).sum() / (np.linalg.norm(upd_t) * np.linalg.norm(u)))
    assert cos >= pages["torch_muon_cosine"], cos
    assert abs(np.linalg.norm(upd_t) / np.linalg.norm(u) - 1) < 0.05


EMUL_MODES = {"pages": {}, "fold_a": {"fold_a": True},
              "fold_a_exact_diag": {"fold_a": True, "exact_diag": True},
              "fold_a_diag_scale": {"fold_a": True, "diag_scale": True}}


@pytest.mark.parametrize("mode", list(EMUL_MODES))
def test_bf16_emulation_close_to_fp64(mode):
    """Diagnostic mode stays within the bf16 tolerance of the fp64 oracle."""
    kw = EMUL_MODES[mode]
    g = wl.iid_normal((64, 256), 1.0, 3)
    e = _rel(oracle.newton_schulz_bf16_emulated(g, **kw), oracle.newton_schulz(g))
    assert 1e-4 < e < 2e-2
    gt = g.T.copy()
    assert _rel(oracle.newton_schulz_bf16_emulated(gt, **kw), oracle.newton_schulz(gt)) < 2e-2


@pytest.mark.parametrize("mode", list(EMUL_MODES))
def test_bf16_emulation_algebra_is_exact(mode):
    """With rounding switched off, each storage layout is an exact rewriting
    of the pages' iteration (deferred scale; a*X + B X = (a I + B) X; the
    diagonal split B' = bf16(B') + diag(lo); the row scale d/bf16(d) = 1
    without rounding), so it must reproduce the fp64
    oracle -- itself pinned to the SVD closed form -- on wide, tall and
    ragged inputs, for several step counts and a per-step table."""
    kw = EMUL_MODES[mode]
    table = np.array([[3.0, -3.2, 1.2], [2.5, -2.0, 0.6], [1.875, -1.25, 0.375]])
    for shape, seed in [((24, 80), 1), ((80, 24), 2), ((33, 33), 3)]:
        g = wl.iid_normal(shape, 1.0, seed)
        for steps, coeffs in [(0, oracle.NS_COEFFS_FIXED), (1, oracle.NS_COEFFS_FIXED),
                              (5, oracle.NS_COEFFS_FIXED), (3, table)]:
            got = oracle.newton_schulz_bf16_emulated(g, coeffs, steps, rounding=lambda x: x, **kw)
            assert _rel(got, oracle.newton_schulz(g, coeffs, steps)) < 1e-12, (mode, shape, steps)


def test_bf16_emulation_first_order_bound_on_diagonal_input():
    """One step on a diagonal input with bf16-exact entries: every matrix
    stays diagonal and each stored value carries a relative rounding error of
    at most u = 2^-8, so with t = s*sigma, q = b t^2 + c t^4 the first-order
    error of the new diagonal against p(t) = t (a + q) is at most
      pages:      t u (|a + q| + |b| t^2 + 2|c| t^4 + |q|)     (A, B, X' rounded)
      fold_a:     t u (2|a + q| + |b| t^2 + 2|c| t^4)          (A, B', X' rounded)
      exact_diag: t u (|a + q| + |b| t^2 + 2|c| t^4)           (A, X' rounded)
      diag_scale: the same as exact_diag (a diagonal B' has no off-diagonal
                  terms for the row scale to touch)
    (times 1 + 4u for the second-order terms).  Each mode must stay inside its
    own bound; folding without the exact diagonal must leave the exact-diagonal
    bound somewhere (the diagonal of B' is then rounded)."""
    u = 2.0 ** -8
    a, b, c = oracle.NS_COEFFS_FIXED
    sig = oracle.round_bf16(np.geomspace(1.0, 1e-2, 256) * (1.0 + np.arange(256) % 7 / 64.0))
    assert np.array_equal(oracle.round_bf16(sig), sig)
    G = np.diag(sig)
    s = 1.0 / (np.sqrt(np.sum(sig * sig)) + oracle.NS_EPS)
    t = s * sig
    q = b * t ** 2 + c * t ** 4
    common = abs(b) * t ** 2 + 2 * abs(c) * t ** 4
    bound = {"pages": t * u * (np.abs(a + q) + common + np.abs(q)) * (1 + 4 * u),
             "fold_a": t * u * (2 * np.abs(a + q) + common) * (1 + 4 * u),
             "fold_a_exact_diag": t * u * (np.abs(a + q) + common) * (1 + 4 * u)}
    bound["fold_a_diag_scale"] = bound["fold_a_exact_diag"]
    err = {}
    for mode, kw in EMUL_MODES.items():
        x = oracle.newton_schulz_bf16_emulated(G, steps=1, **kw)
        assert np.count_nonzero(x - np.diag(np.diag(x))) == 0
        err[mode] = np.abs(np.diag(x) - t * (a + q))
        assert np.all(err[mode] <= bound[mode]), mode
        assert err[mode].max() > 0.05 * bound[mode].max(), mode   # it does round
    assert np.any(err["fold_a"] > bound["fold_a_exact_diag"])


def test_round_bf16_rne():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 3.0e38])
    got = oracle.round_bf16(vals)
    assert got[0] == 1.0
    assert got[1] == 1.0                    # tie -> even (mantissa ...0)
    assert got[2] == 1.0 + 2 ** -6          # tie -> even (rounds up)
    assert got[3] == -2.5 and got[4] == 0.0
    assert np.isfinite(got[5])


# ============================================================================
# momentum pins
# ============================================================================
def momentum_pin_failures(mom):
    fails = []
    rng = np.random.default_rng(2)
    g = rng.standard_normal((3, 4))
    beta = 0.95
    # constant gradient: m_t = G (1 - beta^t) / (1 - beta)  (geometric series,
    # "3.9 Optimizers" exercise 2); lookahead m~ = beta m_t + G
    m = np.zeros_like(g)
    for t in range(1, 8):
        m, mt = mom(m, g, beta, True)
        want = g * (1 - beta ** t) / (1 - beta)
        if _rel(m, want) > 1e-13:
            fails.append(f"geometric_t{t}")
            break
        if _rel(mt, beta * want + g) > 1e-13:
            fails.append(f"lookahead_t{t}")
            break
    # heavy-ball form orthogonalises the buffer itself
    m2, mt2 = mom(np.ones((2, 2)), np.ones((2, 2)), 0.5, False)
    if not (np.allclose(m2, 1.5) and np.allclose(mt2, 1.5)):
        fails.append("heavy_ball")
    return fails


def test_momentum_pins():
    assert momentum_pin_failures(oracle.nesterov_momentum) == []


# ============================================================================
# cautious weight decay + update pins
# ============================================================================
def update_pin_failures(upd):
    fails = []
    rng = np.random.default_rng(3)
    w = rng.standard_normal((6, 7))
    u = rng.standard_normal((6, 7))
    lr, wd = 0.02, 0.1
    # no decay: W -= lr * update  (the plain update form)
    if _rel(upd(w, u, lr, 0.0, True), w - lr * u) > 1e-15:
        fails.append("no_decay")
    # plain decoupled decay as "Chapter 4 / The Full Muon Step" sequences it:
    # p *= (1 - lr wd), then p += -lr * update
    seq = w * (1 - lr * wd)
    seq = seq - lr * u
    if _rel(upd(w, u, lr, wd, False), seq) > 1e-14:
        fails.append("plain_decay_sequence")
    # cautious: where update and param disagree in sign there is no decay;
    # where they agree the decay is the full decoupled one
    out = upd(w, u, lr, wd, True)
    agree = (u * w) > 0
    if not np.allclose(out[~agree], (w - lr * u)[~agree], rtol=0, atol=1e-15):
        fails.append("cautious_off_where_disagree")
    if not np.allclose(out[agree], seq[agree], rtol=0, atol=1e-15):
        fails.append("cautious_on_where_agree")
    # zero product (update exactly 0, either sign of zero): mask on
    wz = np.array([[1.0, -1.0]])
    uz = np.array([[0.0, -0.0]])
    if not np.array_equal(upd(wz, uz, lr, wd, True), wz * (1 - lr * wd)):
        fails.append("zero_product_keeps_decay")
    return fails


def test_update_pins():
    assert update_pin_failures(oracle.cautious_weight_decay_update) == []


def test_mask_sign_logic_no_underflow():
    u = np.array([1e-200, -1e-200, 1e-200, 0.0])
    w = np.array([1e-200, 1e-200, -1e-200, -3.0])
    # products underflow to +-0 in fp64; the mask follows the signs
    assert oracle.cautious_mask(u, w).tolist() == [True, False, False, True]


def test_full_step_matches_closed_form():
    """beta = 0, wd = 0: one step is W - lr * NS(G), NS from the SVD closed form."""
    rng = np.random.default_rng(9)
    g = rng.standard_normal((24, 40))
    w = rng.standard_normal((24, 40))
    w_new, m_new, _ = oracle.muon_step(w, g, np.zeros_like(g), 0.02, 0.0, 0.0)
    assert np.array_equal(m_new, g)
    assert _rel(w_new, w - 0.02 * oracle.ns_closed_form(g)) < 1e-12


# ============================================================================
# NorMuon pins
# ============================================================================
def normuon_pin_failures(norm):
    """[MAC] "NorMuon: Normalized Muon": the update is scaled so its RMS equals
    lr, row by row (norm over the last dimension, divided by sqrt(cols))."""
    fails = []
    rng = np.random.default_rng(8)
    for shape in [(7, 13), (13, 7), (1, 9), (9, 1), (16, 16)]:
        u = rng.standard_normal(shape) * rng.uniform(0.01, 3.0, size=(shape[0], 1))
        out = norm(u)
        if out.shape != u.shape:
            fails.append(f"shape{shape}")
            continue
        rms = np.sqrt(np.mean(u * u, axis=1))
        got = np.sqrt(np.mean(out * out, axis=1))
        if not np.allclose(got, rms / (rms + oracle.NORMUON_EPS), rtol=1e-12, atol=0):
            fails.append(f"row_rms{shape}")
        # direction of every row unchanged
        if not np.allclose(out * np.linalg.norm(u, axis=1, keepdims=True),
                           u * np.linalg.norm(out, axis=1, keepdims=True), rtol=1e-10, atol=1e-14):
            fails.append(f"row_direction{shape}")
    # orthonormal rows (a wide orthogonal update): every row has norm 1 and RMS
    # 1/sqrt(cols), so the scale is sqrt(cols).  (The page's comment gives the
    # whole matrix's RMS as 1/sqrt(min(m,n)); it is sqrt(min/(m n)) =
    # 1/sqrt(max(m,n)), checked here on the input.)
    q = np.linalg.qr(rng.standard_normal((24, 6)))[0].T  # 6 x 24, orthonormal rows
    want = q * (1.0 / (1.0 / np.sqrt(24) + oracle.NORMUON_EPS))
    if np.abs(norm(q) - want).max() > 1e-12:
        fails.append("orthonormal_rows_scale")
    if abs(np.sqrt(np.mean(q * q)) - 1 / np.sqrt(24)) > 1e-12:
        fails.append("orthogonal_rms")
    # a zero row stays zero
    z = np.zeros((3, 5))
    z[1] = 1.0
    out = norm(z)
    if not (np.all(out[0] == 0) and np.all(out[2] == 0)):
        fails.append("zero_row")
    return fails


def test_normuon_pins():
    assert normuon_pin_failures(oracle.normuon_rows) == []


def test_muon_step_with_normuon_matches_page_sequence():
    """[MAC] "The Full Muon Step": update = normalize_muon_update(NS(m~), lr);
    p *= (1 - lr wd); p -= update  (plain decay, as the page sequences it)."""
    rng = np.random.default_rng(12)
    w, g = rng.standard_normal((20, 36)), rng.standard_normal((20, 36))
    lr, wd = 0.02, 0.1
    got, _, _ = oracle.muon_step(w, g, np.zeros_like(w), lr, 0.95, wd, normuon=True, cautious=False)
    u = oracle.newton_schulz(0.95 * g + g)  # one step from zero momentum
    scale = lr / (np.linalg.norm(u, axis=-1, keepdims=True) / u.shape[-1] ** 0.5 + 1e-8)
    seq = w * (1 - lr * wd)
    seq = seq - u * scale
    assert _rel(got, seq) < 1e-14


# ============================================================================
# MuonEq row-equilibration pins
# ============================================================================
def rowq_step(w, g, m):
    """The oracle's Muon step with row equilibration (lr 0.02, beta 0.95,
    wd 0, the fixed triple five times)."""
    return oracle.muon_step(w, g, m, 0.02, 0.95, 0.0, row_equilibrate_input=True)


def rowq_pin_failures(equil, step):
    """equil(x): the row equilibration; step(w, g, m) -> (w_new, m_new, U): a
    Muon step that applies it (as rowq_step).  The pages name MuonEq row
    equilibration without a formula; these pins fix the reading (each
    parameter row divided by its norm + 1e-7, on the momentum-smoothed matrix,
    before the Frobenius normalisation) by its mathematical consequences."""
    fails = []
    rng = np.random.default_rng(21)
    eps = oracle.ROWEQ_EPS
    for shape in [(7, 13), (13, 7), (1, 9), (9, 1)]:
        x = rng.standard_normal(shape) * rng.uniform(0.01, 3.0, size=(shape[0], 1))
        out = equil(x)
        if np.shape(out) != x.shape:
            fails.append(f"shape{shape}")
            continue
        n = np.linalg.norm(x, axis=1)
        if not np.allclose(np.linalg.norm(out, axis=1), n / (n + eps), rtol=1e-12, atol=0):
            fails.append(f"row_norm{shape}")
        no = np.linalg.norm(out, axis=1)
        if np.any(np.sum(out * x, axis=1) <= 0) or \
                not np.allclose(out * n[:, None], x * no[:, None], rtol=1e-10, atol=1e-14):
            fails.append(f"row_direction{shape}")
    z = np.zeros((3, 5))
    z[1] = 2.0
    out = equil(z)
    if not (np.all(out[0] == 0) and np.all(out[2] == 0)):
        fails.append("zero_row")
    # Closed form: G = D Q with orthonormal rows (wide).  Equilibrated, the
    # step sees Q up to eps; after the Frobenius normalisation every singular
    # value is 1/sqrt(rows), so U = p5(1/sqrt(rows)) Q, whatever D was.
    q = _qr_orthonormal(rng, 24, 6).T
    d = np.array([0.03, 0.2, 1.0, 4.0, 9.0, 50.0])[:, None]
    _, _, u = step(np.zeros((6, 24)), d * q, np.zeros((6, 24)))
    want = oracle.ns_singular_value_map(np.array([1.0 / np.sqrt(6.0)]), FIXED, 5)[0] * q
    if np.shape(u) != want.shape or np.abs(u - want).max() > 1e-5:
        fails.append("closed_form_row_scaled_orthonormal")
    # Rescaling each parameter row of G and m by a positive factor leaves U
    # unchanged (up to eps), for tall and wide matrices alike; in a tall
    # matrix the parameter rows are the columns of the iterated X.
    for shape in [(30, 8), (8, 30)]:
        g = rng.standard_normal(shape)
        m0 = rng.standard_normal(shape)
        dd = rng.uniform(0.05, 20.0, size=(shape[0], 1))
        _, _, u1 = step(np.zeros(shape), g, m0)
        _, _, u2 = step(np.zeros(shape), dd * g, dd * m0)
        if _rel(u2, u1) > 1e-6:
            fails.append(f"row_scale_invariance{shape}")
        # without equilibration the same rescaling does change U
        u3 = oracle.newton_schulz(dd * (0.95 * (0.95 * m0 + g) + g))
        if _rel(u3, u1) < 1e-2:
            fails.append(f"invariance_is_not_trivial{shape}")
    # the momentum buffer itself is not equilibrated
    g = rng.standard_normal((12, 20))
    m0 = rng.standard_normal((12, 20)) * 3.0
    _, m_new, _ = step(np.zeros_like(g), g, m0)
    if _rel(m_new, 0.95 * m0 + g) > 1e-15:
        fails.append("momentum_untouched")
    return fails


def test_rowq_pins():
    assert rowq_pin_failures(oracle.row_equilibrate, rowq_step) == []


def test_rowq_direction_change_is_small(pages):
    """Context for the page's figure (cos 0.986 between the update with and
    without MuonEq, measured with another coefficient table): under this
    reading the fixed triple gives a change of the same small size on the
    page's two inputs (iid 256x1024; rank-8 plus noise)."""
    page_cos = pages["muoneq_drop_direction_cos"]
    cs = []
    for g in [wl.iid_normal((256, 1024), 1.0, 0), wl.illcond_grad(0)]:
        u0 = oracle.newton_schulz(g)
        u1 = oracle.newton_schulz(oracle.row_equilibrate(g))
        cs.append(float(np.sum(u0 * u1) / np.linalg.norm(u0) / np.linalg.norm(u1)))
    assert min(cs) < page_cos < max(cs) + 1e-3, cs
    assert min(cs) > 0.95, cs


# ============================================================================
# schedule pins
# ============================================================================
def schedule_pin_failures(sched, pages_chart):
    fails = []
    c = pages_chart
    total = 1000
    for frac, want in zip(c["x_frac"], c["lr"]):
        got = sched(int(round(frac * total)), total, c["max_lr"], c["min_lr"], c["warmup_frac"],
                    c["warmdown_frac"])
        if abs(got - want) > 1e-12:
            fails.append(f"chart@{frac}")
    # linear warmup from 0, flat, linear warmdown (piecewise-linear, continuous)
    vals = [sched(t, total, 1.0, 0.1, 0.1, 0.2) for t in range(total)]
    if vals[0] != 0.0 or abs(vals[50] - 0.5) > 1e-12:
        fails.append("warmup_linear")
    if any(v != 1.0 for v in vals[100:800]):
        fails.append("flat")
    if abs(vals[900] - (0.1 + 0.9 * 0.5)) > 1e-12:
        fails.append("warmdown_linear")
    if max(abs(a - b) for a, b in zip(vals, vals[1:])) > 0.0101:
        fails.append("continuity")
    return fails


def test_schedule_pins(pages):
    assert schedule_pin_failures(oracle.trapezoid_lr, pages["trapezoid_chart"]) == []


def cosine_pin_failures(sched, race):
    """sched(step, total_steps, max_lr, warmup_steps, final_frac): the
    bake-off's warmup + cosine ("Muon vs AdamW, Lion and Sophia: a fair race":
    a climb to the peak over the warmup, a cosine down to a tenth of the peak
    by the last step)."""
    fails = []
    T, W, f = race["steps"], race["warmup_steps"], race["final_frac"]
    vals = [sched(t, T, 1.0, W, f) for t in range(T)]
    last = T - 1
    if vals[0] != 0.0 or abs(vals[W // 2] - 0.5) > 1e-12:
        fails.append("warmup_linear")
    if abs(vals[W] - 1.0) > 1e-12:
        fails.append("peak_after_warmup")
    if abs(vals[last] - f) > 1e-12:
        fails.append("tenth_at_last_step")
    if any(b > a + 1e-15 for a, b in zip(vals[W:], vals[W + 1:])):
        fails.append("monotone_decay")
    if any(b < a for a, b in zip(vals[:W], vals[1:W + 1])):
        fails.append("monotone_warmup")
    # cos(pi p) + cos(pi (1 - p)) = 0: lr(W + k) + lr(last - k) = (1 + f) peak
    for k in (0, 1, 37, 200, (last - W) // 2):
        if abs(vals[W + k] + vals[last - k] - (1.0 + f)) > 1e-12:
            fails.append(f"symmetry{k}")
    # middle and quarter of a decay of 900 steps: cos(pi/2) = 0, cos(pi/4) = sqrt(1/2)
    if abs(sched(W + 450, W + 901, 1.0, W, f) - (1.0 + f) / 2) > 1e-12:
        fails.append("midpoint")
    if abs(sched(W + 225, W + 901, 1.0, W, f) - (f + (1.0 - f) * (1.0 + math.sqrt(0.5)) / 2)) > 1e-12:
        fails.append("quarter")
    if abs(sched(300, T, 3e-4, W, f) - 3e-4 * vals[300]) > 1e-18:
        fails.append("peak_scale")
    if abs(sched(T + 5, T, 1.0, W, f) - f) > 1e-12:
        fails.append("after_last")
    return fails


def test_cosine_pins(pages):
    assert cosine_pin_failures(oracle.warmup_cosine_lr, pages["race_schedule"]) == []


# ============================================================================
# AdamW pins
# ============================================================================
def adamw_pin_failures(adamw):
    fails = []
    rng = np.random.default_rng(4)
    lr = 1e-3
    # step 1 from zeroed state with eps = 0 is exactly -lr * sign(g)
    g = rng.standard_normal(1000)
    p = rng.standard_normal(1000)
    z = np.zeros_like(g)
    p1, m1, v1 = adamw(p, g, z, z, 1, lr, 0.9, 0.95, 0.0, 0.0)
    if not np.allclose(p1 - p, -lr * np.sign(g), rtol=1e-12, atol=0):
        fails.append("step1_sign")
    # constant gradient: every step is -lr * sign(g), whatever t and betas
    # ("3.9 Optimizers", exercise 3(b))
    m, v, pp = z, z, p
    for t in range(1, 12):
        pn, m, v = adamw(pp, g, m, v, t, lr, 0.8, 0.99, 0.0, 0.0)
        if not np.allclose(pn - pp, -lr * np.sign(g), rtol=1e-9, atol=0):
            fails.append(f"constant_grad_t{t}")
            break
        pp = pn
    # zero gradient at step 1: only the decoupled decay acts
    p2, _, _ = adamw(p, z, z, z, 1, lr, 0.9, 0.95, 1e-8, 0.1)
    if not np.array_equal(p2, p * (1 - lr * 0.1)):
        fails.append("decay_only")
    # agreement with torch.optim.AdamW (float64, CPU) over 5 steps, wd 0.1
    try:
        import torch
    except ImportError:
        return fails
    p0 = rng.standard_normal((17, 9))
    tp = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([tp], lr=3e-3, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1)
    pm, mm, vm = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for t in range(1, 6):
        gt = rng.standard_normal(p0.shape)
        tp.grad = torch.from_numpy(gt.copy())
        opt.step()
        pm, mm, vm = adamw(pm, gt, mm, vm, t, 3e-3, 0.9, 0.95, 1e-8, 0.1)
    if _rel(pm, tp.detach().numpy()) > 1e-12:
        fails.append("torch_adamw_5steps")
    st = opt.state[tp]
    if _rel(mm, st["exp_avg"].numpy()) > 1e-12 or _rel(vm, st["exp_avg_sq"].numpy()) > 1e-12:
        fails.append("torch_adamw_state")
    return fails


def test_adamw_pins():
    assert adamw_pin_failures(oracle.adamw_step) == []


def test_adamw_step1_cosine(pages):
    """mira687's reply: at step 1 the update is sign(g), |update| = 1 per element
    (in units of lr), cos against sign(G) = 1, cos against G = 0.797 = sqrt(2/pi)."""
    g = wl.iid_normal((1 << 20,), 1.0, 21)
    z = np.zeros_like(g)
    p1, _, _ = oracle.adamw_step(z, g, z, z, 1, 1.0, 0.9, 0.95, 1e-8, 0.0)
    upd = -p1
    assert abs(np.abs(upd).mean() - pages["adamw_step1_abs_update"]) < 1e-6
    cs = float(upd @ np.sign(g) / (np.linalg.norm(upd) * np.linalg.norm(np.sign(g))))
    assert abs(cs - pages["adamw_step1_cos_vs_sign"]) < 5e-7  # printed to 6 decimals
    cg = float(upd @ g / (np.linalg.norm(upd) * np.linalg.norm(g)))
    assert abs(cg - math.sqrt(2 / math.pi)) < 3e-3
    assert abs(cg - pages["adamw_step1_cos_vs_gaussian_g"]) < 3e-3
