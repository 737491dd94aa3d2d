"""Pins of the CPU oracle against what the SignMuon summary and mathematics fix.

None of these tests retypes the oracle's formulas: each compares it with an
independent route to the same value (SVD closed forms, a library polar
decomposition, brute-force enumeration, a textbook special case, a closed-form
probability) so that a dropped term, a wrong sign, a swapped coefficient, a
transposed operand or a wrong bit index fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import signmuon_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
QUINTIC = O.NS_QUINTIC


def _rng(seed):
    return np.random.default_rng(seed)


def _phi_k(s, k, a, b, c):
    for _ in range(k):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


# --------------------------------------------------------------------------
# Newton-Schulz
# --------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(5, 7), (7, 5), (6, 6), (1, 4), (4, 1), (3, 9)])
@pytest.mark.parametrize("k", [0, 1, 2, 5])
@pytest.mark.parametrize("coeffs", [QUINTIC, (1.3, -0.7, 0.2), (2.0, -1.5, 0.5)])
def test_ns_equals_svd_closed_form(shape, k, coeffs):
    """k steps map X0 = U S V^T to U phi^k(S) V^T with phi(s) = a s + b s^3 + c s^5."""
    x0 = O.frobenius_normalize(_rng(k * 7 + shape[0]).standard_normal(shape))
    u, s, vt = np.linalg.svd(x0, full_matrices=False)
    expected = (u * _phi_k(s, k, *coeffs)) @ vt
    got = O.newton_schulz(x0, k, *coeffs)
    np.testing.assert_allclose(got, expected, rtol=0, atol=1e-10)


def test_cubic_newton_schulz_converges_to_polar_factor():
    """Textbook case: (1.5, -0.5, 0) is the cubic Newton-Schulz iteration, whose
    fixed point on a full-rank matrix with ||X||_2 < sqrt(3) is the polar
    factor U V^T (compared with scipy's polar decomposition)."""
    rng = _rng(1)
    for shape in [(6, 6), (4, 9), (9, 4)]:
        q1, _ = np.linalg.qr(rng.standard_normal((shape[0], shape[0])))
        q2, _ = np.linalg.qr(rng.standard_normal((shape[1], shape[1])))
        r = min(shape)
        sig = np.linspace(0.25, 1.0, r)
        x0 = q1[:, :r] @ np.diag(sig) @ q2[:, :r].T
        got = O.newton_schulz(x0, 60, 1.5, -0.5, 0.0)
        if shape[0] >= shape[1]:
            polar, _ = scipy.linalg.polar(x0, side="right")
        else:
            polar = scipy.linalg.polar(x0.T, side="right")[0].T
        np.testing.assert_allclose(got, polar, atol=1e-12)


def test_ns_transpose_equivariance():
    """Gram on the small side: NS(X^T) == NS(X)^T for tall and wide inputs."""
    rng = _rng(2)
    for shape in [(8, 20), (20, 8)]:
        x0 = O.frobenius_normalize(rng.standard_normal(shape))
        np.testing.assert_allclose(O.newton_schulz(x0.T, 3), O.newton_schulz(x0, 3).T,
                                   atol=1e-12)


def test_ns_diagonal_and_orthogonal_special_cases():
    d = np.diag([0.9, 0.5, 0.1, 0.01])
    np.testing.assert_allclose(O.newton_schulz(d, 4),
                               np.diag(_phi_k(np.diag(d), 4, *QUINTIC)), atol=1e-13)
    n = 8
    q, _ = np.linalg.qr(_rng(3).standard_normal((n, n)))
    x0 = O.frobenius_normalize(q)          # all singular values 1/sqrt(n) (minus eps)
    s = 1.0 / (math.sqrt(n) + O.NORM_EPS)
    np.testing.assert_allclose(O.newton_schulz(x0, 5), _phi_k(s, 5, *QUINTIC) * q,
                               atol=1e-12)


def test_normalisation_bounds_spectral_norm_by_one():
    """The normalised direction has spectral norm at most 1."""
    rng = _rng(4)
    for shape in [(16, 16), (7, 30), (30, 7)]:
        for scale in [1e-3, 1.0, 1e3]:
            m = scale * rng.standard_normal(shape)
            x0 = O.frobenius_normalize(m)
            assert np.linalg.norm(x0, 2) <= 1.0
            nm = np.linalg.norm(m)
            assert abs(np.linalg.norm(x0) - nm / (nm + O.NORM_EPS)) < 1e-12
    assert np.all(O.frobenius_normalize(np.zeros((3, 4))) == 0)


def test_ns_coefficients_are_the_stated_quintic():
    """The pages print no Newton-Schulz polynomial; the specification fixes
    the quintic (a, b, c) = (3.4445, -4.7750, 2.0315).  The oracle and the
    step class each carry that literal (they share no code), so both are
    pinned to it here: a typo in either would otherwise reach both sides of
    every GPU parity test that takes its coefficients from one of them."""
    from sign_muon_optimizer_momentum_b200 import step as S
    assert O.NS_QUINTIC == (3.4445, -4.7750, 2.0315)
    assert S.NS_QUINTIC == (3.4445, -4.7750, 2.0315)
    # The scalar map of these coefficients: phi(1) = a + b + c = 0.701 and a
    # maximum of 1.2024 on [0, 1] (the orbit band used below).
    s = np.linspace(0.0, 1.0, 200001)
    phi = 3.4445 * s - 4.7750 * s ** 3 + 2.0315 * s ** 5
    assert abs(phi[-1] - 0.701) < 1e-12
    assert abs(phi.max() - 1.2024) < 1e-4


def test_quintic_iterates_land_in_band():
    """Singular values in [1e-3, 1] are driven into [0.6818, 1.2024] after six
    quintic steps (the band of the scalar map's orbit), not onto 1."""
    rng = _rng(5)
    n = 24
    q1, _ = np.linalg.qr(rng.standard_normal((n, n)))
    q2, _ = np.linalg.qr(rng.standard_normal((n, n)))
    sig = np.logspace(-3, 0, n)
    x0 = q1 @ np.diag(sig) @ q2.T
    for k in (6, 7, 10):
        sv = np.linalg.svd(O.newton_schulz(x0, k), compute_uv=False)
        assert sv.min() >= 0.6818 and sv.max() <= 1.2024, (k, sv.min(), sv.max())


# --------------------------------------------------------------------------
# Momentum
# --------------------------------------------------------------------------
def test_momentum_special_cases_and_closed_form():
    rng = _rng(6)
    g = rng.standard_normal((5, 6)).astype(np.float32)
    m0 = rng.standard_normal((5, 6)).astype(np.float32)
    # beta = 0: the momentum is the gradient; beta = 1: it is unchanged.
    assert np.array_equal(O.momentum_update(m0, g, 0.0), g.astype(np.float64))
    assert np.array_equal(O.momentum_update(m0, g, 1.0), m0.astype(np.float64))
    # Constant gradient from zero state: M_t = (1 - beta^t) G.
    beta = float(np.float32(0.9))
    m = np.zeros_like(g, dtype=np.float64)
    for t in range(1, 9):
        m = O.momentum_update(m, g, beta)
        expected = (1 - beta ** t) * g.astype(np.float64)
        np.testing.assert_allclose(m, expected, rtol=4e-7 * t, atol=0)
    # The state is fp32-representable.
    assert np.array_equal(m, m.astype(np.float32).astype(np.float64))


# --------------------------------------------------------------------------
# Sign, packing
# --------------------------------------------------------------------------
def test_sign_conventions():
    u = np.array([-2.0, -1e-30, -0.0, 0.0, 1e-30, 3.0, np.nan, -np.inf, np.inf])
    assert O.sign_entries(u).tolist() == [-1, -1, 1, 1, 1, 1, 1, -1, 1]
    assert O.sign_entries(u).dtype == np.int8


def _brute_pack(s):
    rows, cols = s.shape
    wpr = (cols + 31) // 32
    out = np.zeros((rows, wpr), dtype=np.uint32)
    for r in range(rows):
        for w in range(wpr):
            bits = "".join("1" if (32 * w + j < cols and s[r, 32 * w + j] == 1) else "0"
                           for j in reversed(range(32)))
            out[r, w] = int(bits, 2)
    return out


def test_k0_signs_are_the_momentum_signs_unless_the_norm_is_not_finite():
    """With k = 0 the Newton-Schulz output is X0 = M / (||M||_F + 1e-7): its
    sign equals sign(M) entry by entry (0 and -0 -> +1) whenever the norm is
    finite, and is +1 everywhere when M holds a NaN or an infinity (X0 is
    then NaN, or +-0 beside a NaN).  Checked on values spanning fp32's range,
    subnormals included, so that no entry of X0 underflows in fp64."""
    rng = np.random.default_rng(3)
    m = rng.standard_normal((40, 64)) * np.float64(10.0) ** rng.integers(-44, 30, (40, 64))
    m = m.astype(np.float32).astype(np.float64)
    m[0, :5] = [0.0, -0.0, 1e-45, -1e-45, -3e38]
    x0 = O.newton_schulz(O.frobenius_normalize(m), 0)
    assert np.array_equal(O.sign_entries(x0), O.sign_entries(m))
    for bad in (np.nan, np.inf, -np.inf):
        mb = m.copy()
        mb[7, 9] = bad
        with np.errstate(invalid="ignore", over="ignore"):
            s = O.sign_entries(O.newton_schulz(O.frobenius_normalize(mb), 0))
        assert (s == 1).all(), bad


@pytest.mark.parametrize("shape", [(1, 1), (3, 31), (2, 32), (4, 33), (5, 147), (2, 96)])
def test_pack_against_brute_force_and_roundtrip(shape):
    s = np.where(_rng(sum(shape)).random(shape) < 0.5, -1, 1).astype(np.int8)
    w = O.pack_signs(s)
    assert w.dtype == np.uint32 and w.shape == (shape[0], (shape[1] + 31) // 32)
    assert np.array_equal(w, _brute_pack(s))
    assert np.array_equal(O.unpack_signs(w, shape[1]), s)
    # Pad bits are zero.
    tail = shape[1] % 32
    if tail:
        assert np.all(w[:, -1] >> np.uint32(tail) == 0)


def test_pack_single_bit_positions():
    for j in [0, 1, 31, 32, 63, 64, 70]:
        s = -np.ones((1, 71), dtype=np.int8)
        s[0, j] = 1
        w = O.pack_signs(s)
        expected = np.zeros(3, dtype=np.uint32)
        expected[j // 32] = np.uint32(1) << np.uint32(j % 32)
        assert np.array_equal(w[0], expected)


def test_payload_sizes_match_published_ratios():
    rows = {}
    with open(os.path.join(GOLDEN, "compression_ratios.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, bits, ratio = line.split()
                rows[name] = (int(bits), int(ratio))
    shape = (64, 1024)
    fp32_bytes = shape[0] * shape[1] * 4
    s = np.ones(shape, dtype=np.int8)
    assert fp32_bytes // O.pack_signs(s).nbytes == rows["pack1"][1] == 32
    assert fp32_bytes // s.nbytes == rows["int8"][1] == 4
    assert O.pack_signs(s).nbytes * 8 == rows["pack1"][0] * s.size


# --------------------------------------------------------------------------
# Vote
# --------------------------------------------------------------------------
def _brute_vote(column):
    plus = sum(1 for v in column if v == 1)
    minus = len(column) - plus
    return 1 if plus > minus else (-1 if minus > plus else 0)


@pytest.mark.parametrize("m", [1, 2, 3, 4, 5, 6])
def test_vote_against_brute_force_enumeration(m):
    patterns = list(itertools.product([-1, 1], repeat=m))
    signs = [np.array([[p[i] for p in patterns]], dtype=np.int8) for i in range(m)]
    v = O.majority_vote(signs)[0]
    assert v.tolist() == [_brute_vote(p) for p in patterns]
    # Same through the packed route.
    cols = len(patterns)
    vp = O.majority_vote_packed([O.pack_signs(s) for s in signs], cols)[0]
    assert vp.tolist() == v.tolist()
    if m % 2 == 0:
        assert 0 in v.tolist()        # ties exist and give 0
    else:
        assert 0 not in v.tolist()


def test_vote_degenerate_cases():
    s = np.where(_rng(7).random((4, 40)) < 0.5, -1, 1).astype(np.int8)
    assert np.array_equal(O.majority_vote([s]), s)          # M = 1
    assert np.array_equal(O.majority_vote([s] * 5), s)      # all workers agree
    assert np.all(O.majority_vote([s, -s]) == 0)            # exact tie


@pytest.mark.parametrize("m", [2, 3, 8])
def test_vote_statistics_closed_form(m):
    """With p ~ U(0,1) per entry and Bernoulli(p) bits, P(tie) = 1/(M+1) for even
    M (since int_0^1 C(M,k) p^k (1-p)^(M-k) dp = 1/(M+1)) and P(+1) = P(-1)."""
    from sign_muon_optimizer_momentum_b200 import synthetic
    n = 1 << 17
    signs = [s.numpy() for _, s in synthetic.vote_sweep_signs(n, m, seed=11)]
    v = O.majority_vote(signs)
    p_tie = 1.0 / (m + 1) if m % 2 == 0 else 0.0
    frac_tie = np.mean(v == 0)
    tol = 5 * math.sqrt(max(p_tie * (1 - p_tie), 1e-12) / n)
    assert abs(frac_tie - p_tie) <= tol + 1e-12
    p_plus = (1 - p_tie) / 2
    assert abs(np.mean(v == 1) - p_plus) <= 5 * math.sqrt(p_plus * (1 - p_plus) / n)


# --------------------------------------------------------------------------
# Rounding and update
# --------------------------------------------------------------------------
def _bf16_neighbours_brute(x):
    """All bf16 values whose fp32 bit pattern is near that of float32(x)."""
    f = np.float32(x)
    base = np.array([f], dtype=np.float32).view(np.uint32)[0] & np.uint32(0xFFFF0000)
    cands = []
    for d in range(-2, 3):
        bits = np.uint32((int(base) + d * 0x10000) & 0xFFFFFFFF)
        c = float(np.array([bits], dtype=np.uint32).view(np.float32)[0])
        if np.isfinite(c) and (c == 0 or np.sign(c) == np.sign(f)):
            cands.append(c)
    return cands


def test_round_to_bf16_against_brute_force_nearest():
    rng = _rng(8)
    xs = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-6, 6, 3000),
                         [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8),
                          0.5, 3.0e-39, 1e-40]])
    got = O.round_to_bf16(xs)
    for x, g in zip(xs, got):
        cands = _bf16_neighbours_brute(x)
        dist = [abs(c - x) for c in cands]
        best = min(dist)
        winners = [c for c, d in zip(cands, dist) if d == best]
        if len(winners) == 1:
            assert g == winners[0], (x, g, winners)
        else:  # tie: the candidate with an even last mantissa bit
            even = [c for c in winners
                    if (np.array([c], np.float32).view(np.uint32)[0] >> 16) % 2 == 0]
            assert g == even[0], (x, g, winners)


def test_round_to_bf16_matches_torch_on_fp32_inputs():
    x = torch.randn(100000, dtype=torch.float32) * 3
    ref = x.to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16(x.double().numpy()), ref)


@pytest.mark.parametrize("w_dtype", ["f32", "bf16"])
def test_update_moves_each_weight_by_eta_or_not_at_all(w_dtype):
    rng = _rng(9)
    w = O.round_to_dtype(0.02 * rng.standard_normal((16, 40)), w_dtype)
    v = rng.integers(-1, 2, (16, 40)).astype(np.int8)
    eta = 0.02
    w_new = O.apply_update(w, eta, v, w_dtype)
    assert np.array_equal(w_new[v == 0], w[v == 0])
    step = (w - w_new)[v != 0] * v[v != 0]
    ulp = 2.0 ** -8 if w_dtype == "bf16" else 2.0 ** -24
    assert np.all(np.abs(step - np.float32(eta)) <= ulp * (np.abs(w[v != 0]) + eta) * 2)
    # The result is representable in the weight dtype.
    assert np.array_equal(w_new, O.round_to_dtype(w_new, w_dtype))


def _exact_round_brute(x, w_dtype):
    """Correct rounding of the exact rational x to fp32 or bf16 by brute
    force: the nearest of the representable values around it, compared with
    exact rational distances; a tie goes to the even significand."""
    from fractions import Fraction
    f = np.float32(float(x))
    bits = int(np.array([f], np.float32).view(np.uint32)[0])
    step, cands = (1, []) if w_dtype == "f32" else (0x10000, [])
    base = bits if w_dtype == "f32" else bits & 0xFFFF0000
    for k in range(-3, 4):
        b = (base + k * step) & 0xFFFFFFFF
        c = float(np.array([b], np.uint32).view(np.float32)[0])
        if np.isfinite(c):
            cands.append((abs(Fraction(c) - x), (b // step) % 2, c))
    best = min(d for d, _, _ in cands)
    winners = sorted({(odd, c) for d, odd, c in cands if d == best})
    return winners[0][1]


def test_update_rounds_the_exact_difference_once():
    """W - eta * D is rounded once from its exact value.  Two constructed
    cases put the fp64 difference exactly on a rounding midpoint of the
    target while the exact value lies 2^-54 (bf16) or 2^-70 (fp32) above it:
    rounding the fp64 value would tie to the even neighbour, the correct
    result is the odd one above.  Random fp32 directions (as the device's
    polar step produces) are checked against exact rational arithmetic."""
    from fractions import Fraction
    # bf16: W = 1 + 2^-7, eta = 2^-8 (1 + 2^-23), D = 1 - 2^-23:
    # W - eta D = 1 + 2^-8 + 2^-54, just above the midpoint 1 + 2^-8.
    w, eta, dd = 1.0 + 2.0 ** -7, 2.0 ** -8 * (1 + 2.0 ** -23), 1.0 - 2.0 ** -23
    assert np.float32(eta) == eta and np.float32(dd) == dd
    got = O.apply_update(np.array([w]), eta, np.array([dd]), "bf16")[0]
    assert got == 1.0 + 2.0 ** -7 == _exact_round_brute(Fraction(w) - Fraction(eta) * Fraction(dd), "bf16")
    # fp32: W = 1 + 2^-23, eta = 2^-24 (1 + 2^-23), D = 1 - 2^-23:
    # W - eta D = 1 + 2^-24 + 2^-70.
    w, eta = 1.0 + 2.0 ** -23, 2.0 ** -24 * (1 + 2.0 ** -23)
    got = O.apply_update(np.array([w]), eta, np.array([dd]), "f32")[0]
    assert got == 1.0 + 2.0 ** -23 == _exact_round_brute(Fraction(w) - Fraction(eta) * Fraction(dd), "f32")
    # Mirror images (negative weights, negative direction) round away too.
    got = O.apply_update(np.array([-(1.0 + 2.0 ** -7)]), 2.0 ** -8 * (1 + 2.0 ** -23), np.array([-dd]), "bf16")
    assert got[0] == -(1.0 + 2.0 ** -7)
    rng = _rng(13)
    for w_dtype in ("f32", "bf16"):
        w = O.round_to_dtype(0.02 * rng.standard_normal(400), w_dtype)
        w[:40] = O.round_to_dtype(rng.standard_normal(40) * 10.0 ** rng.integers(-8, 3, 40), w_dtype)
        d = O.round_to_f32(rng.standard_normal(400) * 10.0 ** rng.integers(-4, 1, 400))
        eta = float(np.float32(0.02))
        got = O.apply_update(w, eta, d, w_dtype)
        for wi, di, gi in zip(w, d, got):
            assert gi == _exact_round_brute(Fraction(wi) - Fraction(eta) * Fraction(di), w_dtype), (wi, di)


# --------------------------------------------------------------------------
# Optional local polar step
# --------------------------------------------------------------------------
def _hadamard(n):
    h = np.array([[1]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def test_polar_step_on_hadamard_vote_closed_form():
    """A Hadamard +-1 matrix H (n x n) has nnz = n^2 and H/n orthogonal up to a
    1/sqrt(n) scale, so the polar direction is phi(1/sqrt(n)) H / sqrt(n)."""
    n = 16
    h = _hadamard(n).astype(np.int8)
    assert np.sum(h.astype(np.int64) ** 2) == np.count_nonzero(h) == n * n
    d = O.polar_direction(h, 1)
    np.testing.assert_allclose(d, _phi_k(1 / math.sqrt(n), 1, *QUINTIC) * h / math.sqrt(n),
                               atol=1e-13)


def test_polar_step_zero_vote_leaves_weights():
    w = O.round_to_f32(_rng(10).standard_normal((4, 4)))
    out = O.signmuon_step(w, [np.ones((4, 4)), -np.ones((4, 4))],
                          [np.zeros((4, 4)), np.zeros((4, 4))],
                          beta=0.0, eta=0.1, k=1, w_dtype="f32", polar=True)
    assert np.all(out["vote"] == 0)
    assert np.array_equal(out["w"], w)


def test_whole_step_invariants_small():
    rng = _rng(12)
    shape, m = (8, 12), 3
    w = O.round_to_f32(0.02 * rng.standard_normal(shape))
    gs = [rng.standard_normal(shape) for _ in range(m)]
    ms = [np.zeros(shape) for _ in range(m)]
    out = O.signmuon_step(w, gs, ms, beta=0.9, eta=0.02, k=2, w_dtype="f32",
                          int8_variant=False)
    # Odd M: no ties, every weight moves by eta.
    assert set(np.unique(out["vote"]).tolist()) <= {-1, 1}
    np.testing.assert_allclose(np.abs(out["w"] - w), np.float32(0.02), rtol=1e-5)
    # Each worker's sign is the sign of its own Newton-Schulz output.
    for u, s in zip(out["u"], out["signs"]):
        assert np.array_equal(s, np.where(u < 0, -1, 1))
    # A zero momentum (and zero gradient) gives U = 0 and S = +1 everywhere.
    z = O.signmuon_step(w, [np.zeros(shape)], [np.zeros(shape)], beta=0.9, eta=0.02,
                        k=3, w_dtype="f32")
    assert np.all(z["u"][0] == 0) and np.all(z["signs"][0] == 1)


# --------------------------------------------------------------------------
# Spectral scaling (power iteration)
# --------------------------------------------------------------------------
def test_power_iteration_converges_to_svd_sigma_max():
    rng = _rng(20)
    for shape in [(30, 20), (20, 30), (25, 25)]:
        q1, _ = np.linalg.qr(rng.standard_normal((shape[0], shape[0])))
        q2, _ = np.linalg.qr(rng.standard_normal((shape[1], shape[1])))
        r = min(shape)
        sig = np.concatenate([[3.0, 1.5], np.linspace(1.0, 0.1, r - 2)])
        m = q1[:, :r] @ np.diag(sig) @ q2[:, :r].T
        assert abs(O.spectral_norm_estimate(m, 60) - np.linalg.norm(m, 2)) < 1e-12
        # Never above sigma_max, for any number of iterations.
        for t in range(1, 8):
            assert O.spectral_norm_estimate(m, t) <= np.linalg.norm(m, 2) * (1 + 1e-12)


def test_power_iteration_closed_forms():
    # Rank one u v^T: M^T M w = ||u||^2 (v.w) v, so one step from v0 gives
    # sigma^2 = ||u||^2 ||v|| |v.v0| and every later step is exact, ||u|| ||v||.
    rng = _rng(21)
    u, v = rng.standard_normal(7), rng.standard_normal(5)
    v0 = np.full(5, 1 / math.sqrt(5))
    assert math.isclose(O.spectral_norm_estimate(np.outer(u, v), 1),
                        math.sqrt(np.dot(u, u) * np.linalg.norm(v) * abs(np.dot(v, v0))), rel_tol=1e-13)
    for t in (2, 3):
        assert math.isclose(O.spectral_norm_estimate(np.outer(u, v), t), np.linalg.norm(u) * np.linalg.norm(v),
                            rel_tol=1e-13)
    # Diagonal D from v0 = 1/sqrt(n): after t steps sigma^2 = ||d^(2t)|| / ||d^(2t-2)||.
    d = np.array([2.0, 1.5, 1.0, 0.5])
    for t in (1, 2, 5):
        expected = math.sqrt(np.linalg.norm(d ** (2 * t)) / np.linalg.norm(d ** (2 * t - 2)))
        assert math.isclose(O.spectral_norm_estimate(np.diag(d), t), expected, rel_tol=1e-13)
    # Scale equivariance and the zero matrix.
    m = rng.standard_normal((6, 9))
    assert math.isclose(O.spectral_norm_estimate(-3.0 * m, 4), 3.0 * O.spectral_norm_estimate(m, 4), rel_tol=1e-13)
    assert O.spectral_norm_estimate(np.zeros((4, 4)), 3) == 0.0
    assert np.all(O.spectral_normalize(np.zeros((4, 4)), 3) == 0)


def test_spectral_scaling_bounds_normalised_direction():
    """||X0||_2 = sigma_max / sigma_est >= 1 (slightly above 1 for a partly
    converged estimate) and equal to 1 up to eps once converged."""
    rng = _rng(22)
    m = rng.standard_normal((40, 60))
    x_conv = O.spectral_normalize(m, 200)
    assert abs(np.linalg.norm(x_conv, 2) - 1.0) < 1e-6
    x5 = O.spectral_normalize(m, 5)
    assert 1.0 - 1e-6 <= np.linalg.norm(x5, 2) < 1.25
