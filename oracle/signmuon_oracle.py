"""CPU fp64 oracle of the Sign-Muon optimizer step.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain reference that the
CUDA path is checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or
run it.  The product path (the C-ABI library and its Python binding) never
calls into it, and it shares no code with that path: it imports nothing but
numpy.

Source followed throughout: the technical summary of *SignMuon:
Communication-Efficient Distributed Muon Optimization* (arXiv 2605.16311),
cited below as "SignMuon summary", by section:

* §2 "Core mechanism", items 1-3 (polar direction by Newton-Schulz, 1-bit
  sign aggregation, majority vote as an integer sum followed by sign);
* §2 "Algorithmic flow (distributed)", steps 1-5 (momentum, polar factor,
  entrywise sign, one collective, local vote + update, optional local polar
  step on the voted matrix);
* §2 "Communication efficiency" (1 bit per entry, or 8 bits with int8;
  32x / 4x smaller than fp32);
* §3 "Theory" (the normalisation bounds the spectral norm of the update
  direction by 1);
* §4 "nanoGPT" hyper-parameter note (Frobenius vs spectral scaling; one
  Newton-Schulz iteration often suffices).

Readings where the summary is silent (each is a stated choice, not a fact of
the pages): momentum is the EMA ``beta*M + (1-beta)*G``; the Newton-Schulz
input is ``M / (||M||_F + 1e-7)`` and the momentum buffer itself stays
unnormalised; the quintic coefficients are (3.4445, -4.7750, 2.0315); the Gram
matrix is taken on the smaller side; ``sign(0) = sign(-0) = +1`` and NaN maps
to +1; a vote tie (even number of workers) gives 0; the update is computed
exactly and rounded once to the weight's dtype; the optional local polar step
normalises the voted matrix by its Frobenius norm ``sqrt(nnz)`` and runs one
iteration with the same coefficients.

Every function here is pinned by ``tests/test_oracle.py`` against closed forms
(SVD), a textbook special case (cubic Newton-Schulz -> polar factor),
invariants and brute force.  Nothing here is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

# Quintic Newton-Schulz coefficients (a, b, c) used by the build.  The summary
# gives none; these are the widely used Muon quintic coefficients.
NS_QUINTIC = (3.4445, -4.7750, 2.0315)
# Additive epsilon of the Frobenius normalisation (a stated choice).
NORM_EPS = 1e-7


# ---------------------------------------------------------------------------
# Rounding helpers (to the storage dtypes of the step)
# ---------------------------------------------------------------------------
def round_to_f32(x):
    """Round fp64 values to the nearest fp32 (ties to even); returns fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to_bf16(x):
    """Round fp64 values to the nearest bfloat16 (ties to even); returns fp64.

    bfloat16 keeps 8 significant bits and fp32's exponent range (normal
    numbers down to 2**-126, subnormal spacing 2**-133).  The rounding is done
    in one step from the fp64 value: ``rint`` on the value scaled so that the
    bfloat16 grid spacing becomes 1 (numpy's ``rint`` rounds half to even).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    fin = np.isfinite(x) & (x != 0)
    if np.any(fin):
        xf = x[fin]
        _, e = np.frexp(np.abs(xf))          # |x| = m * 2**e, 0.5 <= m < 1
        e = np.maximum(e, -125)              # below 2**-126: fixed subnormal grid
        spacing = np.ldexp(1.0, e - 8)       # 8 significant bits
        r = np.rint(xf / spacing) * spacing
        bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
        r = np.where(np.abs(r) > bf16_max, np.sign(r) * np.inf, r)
        out[fin] = r
    return out


def round_to_dtype(x, dtype: str):
    if dtype == "f32":
        return round_to_f32(x)
    if dtype == "bf16":
        return round_to_bf16(x)
    raise ValueError(f"unknown dtype {dtype!r}")


# ---------------------------------------------------------------------------
# Step 1: per-worker momentum (SignMuon summary, §2 "Algorithmic flow", step 1)
# ---------------------------------------------------------------------------
def momentum_update(mom, grad, beta):
    """Each worker updates its local momentum from its stochastic gradient.

    The summary says only that worker m "updates the local momentum
    M^(m)_{t+1}" from G^(m)_t; the EMA form ``beta*M + (1-beta)*G`` is the
    reading adopted here.  Computed in fp64 from the stored values, then
    rounded to fp32, the dtype the momentum state is kept in.
    """
    mom = np.asarray(mom, dtype=np.float64)
    grad = np.asarray(grad, dtype=np.float64)
    beta = float(beta)
    return round_to_f32(beta * mom + (1.0 - beta) * grad)


# ---------------------------------------------------------------------------
# Normalisation of the Newton-Schulz input (SignMuon summary, §3 "Theory",
# last item, and §4 "nanoGPT": Frobenius vs spectral scaling)
# ---------------------------------------------------------------------------
def frobenius_normalize(mom, eps=NORM_EPS):
    """X0 = M / (||M||_F + eps), in fp64.

    Frobenius scaling makes ||X0||_2 <= ||X0||_F <= 1, which is the
    "spectral norm at most 1" the theory section asks of the normalised
    direction.
    """
    m = np.asarray(mom, dtype=np.float64)
    return m / (np.sqrt(np.sum(m * m)) + eps)


# ---------------------------------------------------------------------------
# Spectral scaling of the Newton-Schulz input (SignMuon summary, §4
# "nanoGPT": the method is robust to Frobenius vs spectral scaling)
# ---------------------------------------------------------------------------
def spectral_norm_estimate(m, iters):
    """Power-iteration estimate of the largest singular value of M.

    The summary names spectral scaling but not how sigma_max is obtained; the
    reading here is `iters` power iterations on M^T M from the unit start
    vector v0 = 1/sqrt(n) (n = columns): z = M^T M v, v <- z / ||z||, and
    sigma_est = sqrt(||z||) from the last step.  For a unit v,
    ||M^T M v|| <= sigma_max^2, so the estimate never exceeds sigma_max and
    converges to it as iters grows (for a start vector not orthogonal to the
    top right singular vector).  A zero matrix gives 0.
    """
    m = np.asarray(m, dtype=np.float64)
    n = m.shape[1]
    v = np.full(n, 1.0 / np.sqrt(n))
    z_norm = 0.0
    for _ in range(max(int(iters), 1)):
        z = m.T @ (m @ v)
        z_norm = float(np.sqrt(np.sum(z * z)))
        if z_norm == 0.0:
            return 0.0
        v = z / z_norm
    return float(np.sqrt(z_norm))


def spectral_normalize(mom, iters, eps=NORM_EPS):
    """X0 = M / (sigma_est + eps) with sigma_est from spectral_norm_estimate."""
    m = np.asarray(mom, dtype=np.float64)
    return m / (spectral_norm_estimate(m, iters) + eps)


# ---------------------------------------------------------------------------
# Newton-Schulz polar iteration (SignMuon summary, §2 "Core mechanism" item 1
# and "Algorithmic flow" step 1)
# ---------------------------------------------------------------------------
def newton_schulz(x0, k, a=NS_QUINTIC[0], b=NS_QUINTIC[1], c=NS_QUINTIC[2]):
    """k Newton-Schulz steps X <- a X + (b A + c A^2) X with A = X X^T.

    The summary names the iteration (it orthogonalises the momentum toward
    its polar factor) but prints no polynomial; the odd polynomial
    ``a s + b s^3 + c s^5`` applied to the singular values is the standard
    Muon form.  For a tall matrix (rows > cols) the Gram matrix is taken on
    the small side: A = X^T X and X <- a X + X (b A + c A^2), which is the
    same map (it is the wide iteration applied to X^T, transposed back).
    """
    x = np.array(x0, dtype=np.float64, copy=True)
    tall = x.shape[0] > x.shape[1]
    for _ in range(int(k)):
        if tall:
            gram = x.T @ x
            poly = b * gram + c * (gram @ gram)
            x = a * x + x @ poly
        else:
            gram = x @ x.T
            poly = b * gram + c * (gram @ gram)
            x = a * x + poly @ x
    return x


# ---------------------------------------------------------------------------
# Entrywise sign (SignMuon summary, §2 "Algorithmic flow", step 2)
# ---------------------------------------------------------------------------
def sign_entries(u):
    """S = sign(U) in {-1, +1} as int8.

    The summary's sign alphabet is {-1, +1}, so zero needs a side: +1 is
    chosen for 0 and -0, and NaN also maps to +1 (the test is "u < 0").
    """
    u = np.asarray(u, dtype=np.float64)
    return np.where(u < 0, -1, 1).astype(np.int8)


# ---------------------------------------------------------------------------
# 1-bit packing (SignMuon summary, §2 "Algorithmic flow" step 3, all-gather
# variant, and "Communication efficiency": 1 bit per entry)
# ---------------------------------------------------------------------------
def packed_words_per_row(cols):
    return (int(cols) + 31) // 32


def pack_signs(s):
    """Pack a {-1,+1} matrix to uint32 words, one bit per entry.

    Layout (a stated choice; the summary fixes only "1 bit per entry"):
    row-major words, ``ceil(cols/32)`` words per row; bit j of word w in row
    r holds entry (r, 32*w + j); a set bit means +1; bits past the last
    column are 0.
    """
    s = np.asarray(s)
    rows, cols = s.shape
    wpr = packed_words_per_row(cols)
    out = np.zeros((rows, wpr), dtype=np.uint32)
    for j in range(cols):
        bit = (s[:, j] == 1).astype(np.uint32) << np.uint32(j % 32)
        out[:, j // 32] |= bit
    return out


def unpack_signs(words, cols):
    """Inverse of ``pack_signs``: uint32 words -> int8 {-1,+1} matrix."""
    words = np.asarray(words, dtype=np.uint32)
    rows = words.shape[0]
    out = np.empty((rows, cols), dtype=np.int8)
    for j in range(cols):
        bit = (words[:, j // 32] >> np.uint32(j % 32)) & np.uint32(1)
        out[:, j] = np.where(bit == 1, 1, -1)
    return out


# ---------------------------------------------------------------------------
# Majority vote (SignMuon summary, §2 "Core mechanism" item 3 and
# "Algorithmic flow" step 4)
# ---------------------------------------------------------------------------
def majority_vote(signs):
    """S_bar = sign(sum_m S^(m)); a tie (only possible for even M) gives 0.

    ``signs`` is a sequence of M int8 {-1,+1} matrices.  The summary
    implements the vote as an integer SUM over workers followed by a local
    sign; with c = #{m : S^(m) = +1} the sum is 2c - M.
    """
    signs = [np.asarray(s, dtype=np.int64) for s in signs]
    if not signs:
        raise ValueError("majority_vote needs at least one worker")
    total = np.zeros_like(signs[0])
    for s in signs:
        total = total + s
    return np.sign(total).astype(np.int8)


def majority_vote_packed(words_list, cols):
    """Vote over M packed buffers: count the +1 bits per entry, then sign(2c - M)."""
    m = len(words_list)
    count = np.zeros((np.asarray(words_list[0]).shape[0], cols), dtype=np.int64)
    for w in words_list:
        count += (unpack_signs(w, cols) == 1)
    return np.sign(2 * count - m).astype(np.int8)


# ---------------------------------------------------------------------------
# Parameter update (SignMuon summary, §2 "Algorithmic flow", step 4)
# ---------------------------------------------------------------------------
def apply_update(w, eta, direction, w_dtype):
    """W_{t+1} = W_t - eta * D, rounded once (to nearest, ties to even) from
    the exact difference to W's dtype.

    ``w`` holds the stored weights (fp32 or bf16 values, as fp64 or fp32);
    ``eta`` is the fp32 learning rate the device receives.  The summary gives
    the update but not its rounding; the reading here is "exact, then one
    rounding".  The product p = eta * D is exact in fp64 whenever D has at
    most 29 significant bits (the voted signs in {-1, 0, +1}, or the fp32
    values of a polar direction computed on the device).  The difference
    w - p is then split exactly into hi + lo (hi = the fp64 difference, lo
    its rounding error, by the two-sum rule).  Rounding hi gives the correctly
    rounded result unless hi lies exactly on a rounding midpoint of the
    target grid while lo is non-zero: then the exact value lies on lo's side
    of that midpoint (no double and so no midpoint lies strictly between hi
    and the exact value), and the neighbour on that side is taken.
    """
    w = np.asarray(w, dtype=np.float64)
    d = np.asarray(direction, dtype=np.float64)
    eta = float(np.float32(eta))
    p = eta * d
    hi = w - p
    z = hi - w
    lo = (w - (hi - z)) + (-p - z)                    # hi + lo == w - p exactly
    r = round_to_dtype(hi, w_dtype)
    up = round_to_dtype(np.nextafter(hi, np.inf), w_dtype)
    down = round_to_dtype(np.nextafter(hi, -np.inf), w_dtype)
    midpoint = (up != down) & (r != hi)               # hi halfway between two grid values
    r = np.where(midpoint & (lo > 0), up, r)
    r = np.where(midpoint & (lo < 0), down, r)
    return r


# ---------------------------------------------------------------------------
# Optional local polar step (SignMuon summary, §2 "Algorithmic flow", step 5)
# ---------------------------------------------------------------------------
def polar_direction(vote, k=1, a=NS_QUINTIC[0], b=NS_QUINTIC[1], c=NS_QUINTIC[2]):
    """Newton-Schulz applied locally to the aggregated sign matrix.

    Reading: the voted matrix is Frobenius-normalised (its squared Frobenius
    norm is its number of non-zeros) and one iteration with the same
    coefficients is run.  An all-zero vote gives a zero direction.
    """
    v = np.asarray(vote, dtype=np.float64)
    nnz = int(np.count_nonzero(v))
    if nnz == 0:
        return np.zeros_like(v)
    return newton_schulz(v / np.sqrt(nnz), k, a, b, c)


# ---------------------------------------------------------------------------
# Whole step for one weight matrix and its M workers
# ---------------------------------------------------------------------------
def signmuon_step(w, grads, moms, *, beta, eta, k, w_dtype, polar=False,
                  coeffs=NS_QUINTIC, int8_variant=True):
    """One Sign-Muon step of one weight matrix, following steps 1-5 in order.

    Returns a dict with the new weights, new momentum buffers, the
    Newton-Schulz outputs U^(m), the signs S^(m) (and packed words for the
    1-bit variant), the vote and, for the polar variant, the polar direction.
    """
    a, b, c = coeffs
    new_moms, us, signs, packed = [], [], [], []
    for g, mo in zip(grads, moms):
        m_new = momentum_update(mo, g, beta)                     # step 1
        u = newton_schulz(frobenius_normalize(m_new), k, a, b, c)  # step 1
        s = sign_entries(u)                                      # step 2
        new_moms.append(m_new)
        us.append(u)
        signs.append(s)
        if not int8_variant:
            packed.append(pack_signs(s))                         # step 3 (1-bit)
    if int8_variant:
        vote = majority_vote(signs)                              # steps 3-4 (int sum)
    else:
        vote = majority_vote_packed(packed, np.asarray(w).shape[1])
    out = {"mom": new_moms, "u": us, "signs": signs, "packed": packed,
           "vote": vote}
    if polar:
        d = polar_direction(vote, 1, a, b, c)                    # step 5
        out["polar_dir"] = d
        out["w"] = apply_update(w, eta, d, w_dtype)
    else:
        out["w"] = apply_update(w, eta, vote, w_dtype)           # step 4
    return out
