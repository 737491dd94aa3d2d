"""GPU parity of the C-ABI kernels against the CPU oracle.

Every case draws seeded synthetic inputs, runs them through libsignmuon.so
(via the thin binding) and through the fp64 oracle, and compares:
  * sign/pack, vote and update: bit-exact;
  * momentum: bit-exact fp32 state, bf16 copy exact, norm to 1e-5 relative;
  * Newton-Schulz: relative Frobenius error <= 2e-2 against the fp64 oracle
    and sign agreement >= 99.5 % on entries with |U| > 1e-3.
The oracle never consumes a GPU output: both sides start from the same
seeded inputs.
"""
import math

import numpy as np
import pytest
import torch

from oracle import signmuon_oracle as O
from sign_muon_optimizer_momentum_b200 import _lib as L
from sign_muon_optimizer_momentum_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

NS_TOL = 2e-2          # relative Frobenius error of U (bf16 operands, fp32 accumulation)
SIGN_AGREE = 0.995     # on |U_oracle| > 1e-3
A, B, C = O.NS_QUINTIC


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_lib):
    return cuda_lib


def stream():
    return torch.cuda.current_stream().cuda_stream


def f64(t):
    return t.detach().float().cpu().double().numpy()


def ws(nbytes):
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device="cuda")


def assert_no_device_error(w):
    assert L.signmuon_device_error(w.data_ptr(), stream()) == 0


# ---------------------------------------------------------------------------
# helpers running the GPU path
# ---------------------------------------------------------------------------
def gpu_momentum(shapes, M, grads, moms, beta, grad_dtype):
    xs = [torch.empty((r, L.signmuon_x_ld(c)), dtype=torch.bfloat16, device="cuda")
          for (r, c) in shapes for _ in range(M)]
    inv = torch.empty(len(shapes) * M, dtype=torch.float32, device="cuda")
    w = ws(L.signmuon_momentum_workspace_bytes(shapes, M))
    code = L.SIGNMUON_BF16 if grad_dtype == torch.bfloat16 else L.SIGNMUON_F32
    L.signmuon_momentum_norm(shapes, M, code, [g.data_ptr() for g in grads], [m.data_ptr() for m in moms],
                             beta, [x.data_ptr() for x in xs], inv.data_ptr(), w.data_ptr(), w.numel(),
                             stream())
    torch.cuda.synchronize()
    assert_no_device_error(w)
    return xs, inv


def gpu_ns(shapes, M, xs, inv, k, out_mode, outs=None, w_dtype=L.SIGNMUON_F32, weights=None, eta=0.0,
           minimal_ws=False, coeffs=(A, B, C)):
    nbytes = L.signmuon_newton_schulz_workspace_bytes(shapes, M, minimal=minimal_ws)
    w = ws(nbytes)
    L.signmuon_newton_schulz_batched(shapes, M, [x.data_ptr() for x in xs], inv.data_ptr(), k, *coeffs,
                                     out_mode, None if outs is None else [o.data_ptr() for o in outs],
                                     w_dtype, None if weights is None else [x.data_ptr() for x in weights],
                                     eta, w.data_ptr(), w.numel(), stream())
    torch.cuda.synchronize()
    assert_no_device_error(w)


def seeded_state(shapes, M, seed, grad_dtype=torch.float32, mom_std=1.0, g_std=2.0):
    grads, moms = [], []
    for i, s in enumerate(shapes):
        for m in range(M):
            grads.append(syn.gaussian(s, g_std, "cpu", "tg", seed, i, m, dtype=grad_dtype))
            moms.append(syn.gaussian(s, mom_std, "cpu", "tm", seed, i, m))
    return grads, moms


def oracle_u(mom0, grad, beta, k):
    m = O.momentum_update(f64(mom0), f64(grad), float(np.float32(beta)))
    return m, O.newton_schulz(O.frobenius_normalize(m), k)


def unpack_words(words, rows, cols):
    """Decodes a packed sign buffer (bit j of word w in row r = entry (r, 32w+j))."""
    wpr = (cols + 31) // 32
    w = np.ascontiguousarray(words[: rows * wpr].reshape(rows, wpr).astype("<u4"))
    bits = np.unpackbits(w.view(np.uint8), axis=1, bitorder="little")[:, :cols]
    return np.where(bits == 1, 1, -1).astype(np.int8)


def rel_fro(x, ref):
    return np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30)


# ---------------------------------------------------------------------------
# sign + pack
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(1, 1), (3, 31), (31, 33), (64, 147), (5, 96), (300, 1000), (129, 4096)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_sign_pack_bit_exact(shape, dtype):
    u = syn.gaussian(shape, 1.0, "cpu", "u", *shape, dtype=dtype)
    flat = u.view(-1)
    flat[::7] = 0.0
    flat[1::11] = -0.0
    if dtype == torch.float32:
        flat[2::13] = float("nan")
    ud = u.cuda()
    nwords = L.signmuon_packed_words(shape)
    out = torch.full((nwords,), -1, dtype=torch.int32, device="cuda")
    code = L.SIGNMUON_BF16 if dtype == torch.bfloat16 else L.SIGNMUON_F32
    L.signmuon_sign_pack(shape, code, ud.data_ptr(), shape[1], 0, out.data_ptr(), stream())
    o8 = torch.zeros(shape, dtype=torch.int8, device="cuda")
    L.signmuon_sign_pack(shape, code, ud.data_ptr(), shape[1], 1, o8.data_ptr(), stream())
    torch.cuda.synchronize()
    s = O.sign_entries(f64(u))
    ref = O.pack_signs(s).reshape(-1)
    got = out.cpu().numpy().view(np.uint32)
    assert np.array_equal(got[: ref.size], ref)
    assert np.all(got[ref.size:] == 0)          # trailing pad words are zero
    assert np.array_equal(o8.cpu().numpy(), s)


def test_sign_pack_strided_input():
    shape, ld = (17, 40), 56
    u = syn.gaussian((shape[0], ld), 1.0, "cpu", "us")
    out = torch.zeros(L.signmuon_packed_words(shape), dtype=torch.int32, device="cuda")
    L.signmuon_sign_pack(shape, L.SIGNMUON_F32, u.cuda().data_ptr(), ld, 0, out.data_ptr(), stream())
    torch.cuda.synchronize()
    ref = O.pack_signs(O.sign_entries(f64(u)[:, :shape[1]])).reshape(-1)
    assert np.array_equal(out.cpu().numpy().view(np.uint32)[: ref.size], ref)


# ---------------------------------------------------------------------------
# vote + update
# ---------------------------------------------------------------------------
def _signs(shape, M, seed):
    n = shape[0] * shape[1]
    return [s.view(shape) for _, s in syn.vote_sweep_signs(n, M, seed=seed)]


def _packed_device(s_list, shape):
    outs = []
    for s in s_list:
        words = np.zeros(L.signmuon_packed_words(shape), dtype=np.uint32)
        p = O.pack_signs(s.numpy())
        words[: p.size] = p.reshape(-1)
        outs.append(torch.from_numpy(words.view(np.int32)).cuda())
    return outs


# M = 126 and 127: the largest worker counts (even: ties; the byte sums and
# the seven counter planes at their range).
VOTE_CASES = [((4, 32), 1), ((64, 64), 2), ((37, 96), 3), ((256, 256), 8), ((100, 1024), 16),
              ((64, 4096), 64), ((33, 147), 5), ((31, 33), 4), ((2, 1000), 7), ((512, 1024), 64),
              ((16, 512), 126), ((9, 160), 127)]


@pytest.mark.parametrize("shape,M", VOTE_CASES)
@pytest.mark.parametrize("int8_in", [False, True])
@pytest.mark.parametrize("w_dtype", [torch.float32, torch.bfloat16])
def test_vote_update_bit_exact(shape, M, int8_in, w_dtype):
    s_list = _signs(shape, M, seed=M * 1000 + shape[0])
    w0 = syn.gaussian(shape, 0.02, "cpu", "w", *shape, dtype=w_dtype)
    eta = 0.01
    if int8_in:
        dev_signs = [s.cuda() for s in s_list]
    else:
        dev_signs = _packed_device(s_list, shape)
    w = w0.cuda()
    wk = ws(L.signmuon_vote_workspace_bytes([shape], M))
    code = L.SIGNMUON_BF16 if w_dtype == torch.bfloat16 else L.SIGNMUON_F32
    L.signmuon_vote_update([shape], M, int8_in, [s.data_ptr() for s in dev_signs], code, [w.data_ptr()], eta,
                           None, 0, 0, wk.data_ptr(), wk.numel(), stream())
    torch.cuda.synchronize()
    v = O.majority_vote([s.numpy() for s in s_list])
    ref = O.apply_update(f64(w0), eta, v, "bf16" if w_dtype == torch.bfloat16 else "f32")
    assert np.array_equal(f64(w), ref)


def test_vote_update_multi_matrix_and_vote_out():
    shapes = [(64, 147), (128, 256), (33, 64), (7, 5)]
    M = 6
    all_signs = [_signs(s, M, seed=10 + i) for i, s in enumerate(shapes)]
    for int8_in in (False, True):
        flat = []
        for s_list, shp in zip(all_signs, shapes):
            flat += [x.cuda() for x in s_list] if int8_in else _packed_device(s_list, shp)
        votes = [torch.full((r, L.signmuon_x_ld(c)), 7.0, dtype=torch.bfloat16, device="cuda") for r, c in shapes]
        nnz = torch.full((4,), -5, dtype=torch.int64, device="cuda")
        inv = torch.zeros(4, dtype=torch.float32, device="cuda")
        wk = ws(L.signmuon_vote_workspace_bytes(shapes, M))
        L.signmuon_vote_update(shapes, M, int8_in, [x.data_ptr() for x in flat], L.SIGNMUON_F32, None, 0.01,
                               [v.data_ptr() for v in votes], nnz.data_ptr(), inv.data_ptr(), wk.data_ptr(),
                               wk.numel(), stream())
        torch.cuda.synchronize()
        for i, (shp, s_list) in enumerate(zip(shapes, all_signs)):
            ref = O.majority_vote([s.numpy() for s in s_list])
            got = f64(votes[i])[:, : shp[1]]
            assert np.array_equal(got, ref)
            assert nnz[i].item() == np.count_nonzero(ref)
            assert math.isclose(inv[i].item(), 1 / math.sqrt(np.count_nonzero(ref)), rel_tol=1e-6)


# ---------------------------------------------------------------------------
# momentum
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shapes,M", [([(256, 256)], 4), ([(64, 147), (1, 1), (7, 9)], 3),
                                      ([(768, 2304), (3072, 768)], 2)])
@pytest.mark.parametrize("grad_dtype", [torch.float32, torch.bfloat16])
def test_momentum_norm_exact(shapes, M, grad_dtype):
    beta = 0.9
    grads, moms = seeded_state(shapes, M, 3, grad_dtype)
    g_d = [g.cuda() for g in grads]
    m_d = [m.cuda() for m in moms]
    xs, inv = gpu_momentum(shapes, M, g_d, m_d, beta, grad_dtype)
    for u in range(len(grads)):
        r, c = shapes[u // M]
        ref = O.momentum_update(f64(moms[u]), f64(grads[u]), float(np.float32(beta)))
        got = f64(m_d[u])
        assert np.array_equal(got, ref), np.max(np.abs(got - ref))
        assert np.array_equal(f64(xs[u])[:, :c], O.round_to_bf16(ref))
        ref_inv = 1.0 / (math.sqrt(np.sum(ref * ref)) + O.NORM_EPS)
        assert math.isclose(inv[u].item(), ref_inv, rel_tol=1e-5)


@pytest.mark.parametrize("int8_out", [False, True])
@pytest.mark.parametrize("grad_dtype", [torch.float32, torch.bfloat16])
def test_momentum_sign_fused_matches_oracle(int8_out, grad_dtype):
    """k = 0 fused: momentum bit-exact and the signs of X0 = M / (||M|| + eps)
    exactly as the oracle's (a NaN unit gives all +1, a zero unit all +1)."""
    shapes = [(64, 96), (96, 64), (32, 2048)] + ([(33, 147), (5, 40)] if int8_out else [])
    M = 3
    grads, moms = seeded_state(shapes, M, 29, grad_dtype=grad_dtype)
    grads[1][3, 5] = float("nan")                       # unit 1: NaN norm
    grads[2].zero_()
    moms[2].zero_()                                     # unit 2: zero momentum
    grads[4][0, :] = -0.0
    moms[4][0, :] = -0.0                                # a row of zeros: signs +1
    gd = [g.cuda() for g in grads]
    md = [m.cuda() for m in moms]
    if int8_out:
        signs = [torch.zeros(shapes[u // M], dtype=torch.int8, device="cuda") for u in range(len(gd))]
    else:
        signs = [torch.zeros(L.signmuon_packed_words(shapes[u // M]), dtype=torch.int32, device="cuda")
                 for u in range(len(gd))]
    inv = torch.empty(len(gd), dtype=torch.float32, device="cuda")
    w = ws(L.signmuon_momentum_workspace_bytes(shapes, M))
    code = L.SIGNMUON_BF16 if grad_dtype == torch.bfloat16 else L.SIGNMUON_F32
    L.signmuon_momentum_sign(shapes, M, code, [g.data_ptr() for g in gd], [m.data_ptr() for m in md], 0.9,
                             int8_out, [x.data_ptr() for x in signs], inv.data_ptr(), w.data_ptr(), w.numel(),
                             stream())
    torch.cuda.synchronize()
    for u in range(len(gd)):
        r, c = shapes[u // M]
        m_ref = O.momentum_update(f64(moms[u]), f64(grads[u]), float(np.float32(0.9)))
        assert np.array_equal(f64(md[u]), m_ref, equal_nan=True)
        ref = O.sign_entries(O.frobenius_normalize(m_ref))
        if int8_out:
            got = signs[u].cpu().numpy()
        else:
            got = unpack_words(signs[u].cpu().numpy().view(np.uint32), r, c)
        assert np.array_equal(got, ref), (u, shapes[u // M])
        if u in (1, 2):                                 # NaN / zero unit: every sign +1
            assert (got == 1).all()


def test_momentum_zero_gradient_gives_zero_x():
    shapes, M = [(32, 64)], 2
    g = [torch.zeros(32, 64, device="cuda") for _ in range(M)]
    m = [torch.zeros(32, 64, device="cuda") for _ in range(M)]
    xs, inv = gpu_momentum(shapes, M, g, m, 0.9, torch.float32)
    assert all(torch.all(x[:, :64] == 0) for x in xs)
    assert torch.allclose(inv, torch.full_like(inv, 1e7))


# ---------------------------------------------------------------------------
# Newton-Schulz
# ---------------------------------------------------------------------------
NS_CASES = [([(256, 256)], 4, 1), ([(128, 384), (384, 128)], 2, 2), ([(100, 300), (300, 100)], 2, 5),
            ([(64, 147), (147, 64)], 3, 1), ([(768, 2304)], 1, 5), ([(3072, 768)], 1, 5),
            ([(1, 1), (1, 40), (40, 1)], 2, 3), ([(513, 513)], 1, 2), ([(2048, 1000)], 1, 1),
            ([(768, 768), (768, 3072)], 1, 5), ([(512, 4608), (2048, 512), (256, 2304)], 1, 1)]


@pytest.mark.parametrize("shapes,M,k", NS_CASES)
def test_newton_schulz_matches_oracle(shapes, M, k):
    beta = 0.9
    grads, moms = seeded_state(shapes, M, 5)
    g_d = [g.cuda() for g in grads]
    m_d = [m.cuda() for m in moms]
    xs, inv = gpu_momentum(shapes, M, g_d, m_d, beta, torch.float32)
    us = [torch.empty(shapes[u // M], dtype=torch.float32, device="cuda") for u in range(len(xs))]
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, us)
    for u in range(len(xs)):
        _, ref = oracle_u(moms[u], grads[u], beta, k)
        got = f64(us[u])
        err = rel_fro(got, ref)
        assert err <= NS_TOL, (shapes[u // M], k, err)
        big = np.abs(ref) > 1e-3
        if big.sum() > 0:
            agree = np.mean(np.sign(got[big]) == np.sign(ref[big]))
            assert agree >= SIGN_AGREE, (shapes[u // M], agree)


@pytest.mark.parametrize("coeffs", [(1.5, -0.5, 0.0), (2.0, -1.5, 0.5), (1.0, -1.0, 0.01)])
@pytest.mark.parametrize("shapes,M,k", [([(256, 384), (300, 700)], 2, 3), ([(2056, 2100)], 1, 2)])
def test_newton_schulz_other_coefficients(coeffs, shapes, M, k):
    """Coefficients other than the quintic: c = 0 (the cubic iteration,
    B' = a I + b A, the square stage reading A back), c != 0 with another
    moderate diagonal shift (the Gram stage stores A + b/(2c) I and the square
    forms c Q Q + (a - b^2/(4c)) I), and a shift too large for fp16's
    precision (b/(2c) = -50: the unshifted form); short and long-reduction
    launches."""
    grads, moms = seeded_state(shapes, M, 31)
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.clone().cuda() for m in moms], 0.9,
                           torch.float32)
    us = [torch.empty(shapes[u // M], dtype=torch.float32, device="cuda") for u in range(len(xs))]
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, us, coeffs=coeffs)
    a, b, c = coeffs
    for u in range(len(grads)):
        mom = O.momentum_update(f64(moms[u]), f64(grads[u]), float(np.float32(0.9)))
        ref = O.newton_schulz(O.frobenius_normalize(mom), k, a, b, c)
        assert rel_fro(f64(us[u]), ref) <= NS_TOL, (coeffs, shapes[u // M])


def test_newton_schulz_fused_outputs_are_signs_of_u():
    """The packed and int8 epilogues write exactly the signs of the fp32 U the
    same launch configuration produces (sign(0) = +1)."""
    # cols % 16 == 0, % 8 == 0, % 4 == 0 and odd: every store width of the
    # int8 epilogue, wide and tall.
    shapes, M, k = [(96, 300), (300, 96), (64, 147), (200, 1000), (1000, 104)], 2, 2
    grads, moms = seeded_state(shapes, M, 7)
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.cuda() for m in moms], 0.9,
                           torch.float32)
    saved = [x.clone() for x in xs]
    us = [torch.empty(shapes[u // M], dtype=torch.float32, device="cuda") for u in range(len(xs))]
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, us)
    for x, s in zip(xs, saved):
        x.copy_(s)
    packed = [torch.zeros(L.signmuon_packed_words(shapes[u // M]), dtype=torch.int32, device="cuda")
              for u in range(len(xs))]
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_PACK1, packed)
    for x, s in zip(xs, saved):
        x.copy_(s)
    i8 = [torch.zeros(shapes[u // M], dtype=torch.int8, device="cuda") for u in range(len(xs))]
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_INT8, i8)
    for u in range(len(xs)):
        r, c = shapes[u // M]
        uu = us[u].cpu().numpy()
        plus = ~(uu < 0)
        assert np.array_equal(i8[u].cpu().numpy(), np.where(plus, 1, -1))
        words = packed[u].cpu().numpy().view(np.uint32)
        wpr = (c + 31) // 32
        for j in range(c):
            bit = (words[: r * wpr].reshape(r, wpr)[:, j // 32] >> np.uint32(j % 32)) & 1
            assert np.array_equal(bit.astype(bool), plus[:, j])


def test_newton_schulz_waves_match_single_wave():
    shapes, M, k = [(128, 256), (256, 128), (200, 200)], 3, 2
    grads, moms = seeded_state(shapes, M, 9)
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.cuda() for m in moms], 0.9,
                           torch.float32)
    saved = [x.clone() for x in xs]
    u1 = [torch.empty(shapes[u // M], dtype=torch.float32, device="cuda") for u in range(len(xs))]
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, u1)
    for x, s in zip(xs, saved):
        x.copy_(s)
    u2 = [torch.empty_like(t) for t in u1]
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, u2, minimal_ws=True)
    for a, b in zip(u1, u2):
        assert torch.equal(a, b)


@pytest.mark.parametrize("minimal_ws", [False, True])
def test_newton_schulz_plan_run_matches_batched(minimal_ws):
    """plan + run (run repeated, then a re-plan onto other outputs) gives
    bit-identical results to the one-shot entry point."""
    shapes, M, k = [(128, 256), (256, 128), (200, 200), (64, 147)], 3, 2
    grads, moms = seeded_state(shapes, M, 21)
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.cuda() for m in moms], 0.9,
                           torch.float32)
    saved = [x.clone() for x in xs]

    def restore():
        for x, sv in zip(xs, saved):
            x.copy_(sv)

    def new_outs():
        return [torch.full(shapes[u // M], float("nan"), device="cuda") for u in range(len(xs))]

    ref = new_outs()
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, ref, minimal_ws=minimal_ws)
    w = ws(L.signmuon_newton_schulz_workspace_bytes(shapes, M, minimal=minimal_ws))
    xp = [x.data_ptr() for x in xs]
    for _ in range(2):
        outs = new_outs()
        restore()
        plan = L.signmuon_newton_schulz_plan(shapes, M, xp, inv.data_ptr(), L.SIGNMUON_OUT_U_F32,
                                             [o.data_ptr() for o in outs], L.SIGNMUON_F32, None, w.data_ptr(),
                                             w.numel(), stream())
        for _ in range(2):  # the same plan, twice in a row
            restore()
            for o in outs:
                o.fill_(float("nan"))
            L.signmuon_newton_schulz_run(plan, k, A, B, C, 0.0, stream())
            torch.cuda.synchronize()
            assert_no_device_error(w)
            for a, b in zip(ref, outs):
                assert torch.equal(a, b)
    # k = 0 through the same plan equals the one-shot k = 0.
    restore()
    ref0 = new_outs()
    gpu_ns(shapes, M, xs, inv, 0, L.SIGNMUON_OUT_U_F32, ref0, minimal_ws=minimal_ws)
    restore()
    outs = new_outs()
    plan = L.signmuon_newton_schulz_plan(shapes, M, xp, inv.data_ptr(), L.SIGNMUON_OUT_U_F32,
                                         [o.data_ptr() for o in outs], L.SIGNMUON_F32, None, w.data_ptr(),
                                         w.numel(), stream())
    L.signmuon_newton_schulz_run(plan, 0, A, B, C, 0.0, stream())
    torch.cuda.synchronize()
    for a, b in zip(ref0, outs):
        assert torch.equal(a, b)


def test_newton_schulz_k0_and_zero_input():
    shapes, M = [(40, 72), (72, 40)], 2
    grads, moms = seeded_state(shapes, M, 11)
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.cuda() for m in moms], 0.9,
                           torch.float32)
    us = [torch.empty(shapes[u // M], dtype=torch.float32, device="cuda") for u in range(len(xs))]
    gpu_ns(shapes, M, xs, inv, 0, L.SIGNMUON_OUT_U_F32, us)
    for u in range(len(xs)):
        m, ref = oracle_u(moms[u], grads[u], 0.9, 0)
        assert rel_fro(f64(us[u]), ref) < 4e-3     # bf16 rounding of X0 only
    # Zero momentum: U = 0 and every sign is +1.
    z = [torch.zeros(s, device="cuda") for s in shapes for _ in range(M)]
    xs, inv = gpu_momentum(shapes, M, z, [torch.zeros_like(t) for t in z], 0.9, torch.float32)
    packed = [torch.zeros(L.signmuon_packed_words(shapes[u // M]), dtype=torch.int32, device="cuda")
              for u in range(len(xs))]
    gpu_ns(shapes, M, xs, inv, 3, L.SIGNMUON_OUT_PACK1, packed)
    for u in range(len(xs)):
        r, c = shapes[u // M]
        ref = O.pack_signs(np.ones((r, c), dtype=np.int8)).reshape(-1)
        assert np.array_equal(packed[u].cpu().numpy().view(np.uint32)[: ref.size], ref)


@pytest.mark.parametrize("w_dtype", [torch.float32, torch.bfloat16])
def test_polar_step_update(w_dtype):
    """Vote-out, then one Newton-Schulz iteration on the voted matrix fused with
    W <- W - eta * U_V (the optional local polar step)."""
    # Aligned rows (vector update) and ragged ones (cols % 8 != 0, odd).
    shapes, M, eta = [(256, 256), (128, 384), (100, 147), (72, 300)], 4, 0.02
    all_signs = [_signs(s, M, seed=20 + i) for i, s in enumerate(shapes)]
    flat = []
    for s_list, shp in zip(all_signs, shapes):
        flat += _packed_device(s_list, shp)
    votes = [torch.zeros((r, L.signmuon_x_ld(c)), dtype=torch.bfloat16, device="cuda") for r, c in shapes]
    nnz = torch.zeros(len(shapes), dtype=torch.int64, device="cuda")
    inv = torch.zeros(len(shapes), dtype=torch.float32, device="cuda")
    wk = ws(L.signmuon_vote_workspace_bytes(shapes, M))
    L.signmuon_vote_update(shapes, M, False, [x.data_ptr() for x in flat], L.SIGNMUON_F32, None, eta,
                           [v.data_ptr() for v in votes], nnz.data_ptr(), inv.data_ptr(), wk.data_ptr(),
                           wk.numel(), stream())
    w0 = [syn.gaussian(s, 0.02, "cpu", "pw", i, dtype=w_dtype) for i, s in enumerate(shapes)]
    w = [t.cuda() for t in w0]
    code = L.SIGNMUON_BF16 if w_dtype == torch.bfloat16 else L.SIGNMUON_F32
    # The polar direction the update used: the same launch with the fp32 U
    # written out (one iteration reads the vote buffers without writing them).
    u_gpu = gpu_polar_u(shapes, votes, inv)
    gpu_ns(shapes, 1, votes, inv, 1, L.SIGNMUON_OUT_UPDATE_W, None, code, w, eta)
    wd = "bf16" if w_dtype == torch.bfloat16 else "f32"
    for i, s_list in enumerate(all_signs):
        vote = O.majority_vote([s.numpy() for s in s_list])
        assert np.array_equal(f64(votes[i])[:, :shapes[i][1]], vote)
        d = O.polar_direction(vote, 1)
        assert rel_fro(f64(u_gpu[i]), d) <= NS_TOL
        # The update is the exact W - eta * U of the device's own U, rounded
        # once to W's dtype: bit-exact against the oracle's update.
        assert np.array_equal(f64(w[i]), O.apply_update(f64(w0[i]), eta, f64(u_gpu[i]), wd)), shapes[i]


@pytest.mark.parametrize("w_dtype", [torch.float32, torch.bfloat16])
def test_polar_step_all_ties_leaves_weights_bit_identical(w_dtype):
    """Two workers with opposite signs everywhere: every vote ties, nnz = 0,
    1/sqrt(nnz) is taken as 0, the polar step's U is 0 and W stays bit for
    bit (signed zeros included), as the oracle's zero vote does."""
    shapes, eta = [(256, 384), (72, 300)], 0.02
    flat, w0 = [], []
    for i, (r, c) in enumerate(shapes):
        pos = torch.ones((r, c), dtype=torch.int8)
        flat += _packed_device([pos, -pos], (r, c))
        w = syn.gaussian((r, c), 0.02, "cpu", "tiew", i, dtype=w_dtype)
        w[0, :8] = 0.0
        w[0, 8:16] = -0.0
        w0.append(w)
    votes = [torch.full((r, L.signmuon_x_ld(c)), 3.0, dtype=torch.bfloat16, device="cuda") for r, c in shapes]
    nnz = torch.full((len(shapes),), -1, dtype=torch.int64, device="cuda")
    inv = torch.full((len(shapes),), 5.0, dtype=torch.float32, device="cuda")
    wk = ws(L.signmuon_vote_workspace_bytes(shapes, 2))
    L.signmuon_vote_update(shapes, 2, False, [x.data_ptr() for x in flat], L.SIGNMUON_F32, None, eta,
                           [v.data_ptr() for v in votes], nnz.data_ptr(), inv.data_ptr(), wk.data_ptr(), wk.numel(),
                           stream())
    torch.cuda.synchronize()
    assert nnz.tolist() == [0, 0] and inv.tolist() == [0.0, 0.0]
    for v, (r, c) in zip(votes, shapes):
        assert bool((v[:, :c] == 0).all())
    w = [t.cuda() for t in w0]
    code = L.SIGNMUON_BF16 if w_dtype == torch.bfloat16 else L.SIGNMUON_F32
    gpu_ns(shapes, 1, votes, inv, 1, L.SIGNMUON_OUT_UPDATE_W, None, code, w, eta)
    ibits = torch.int16 if w_dtype == torch.bfloat16 else torch.int32
    wd = "bf16" if w_dtype == torch.bfloat16 else "f32"
    for a, b in zip(w, w0):
        assert torch.equal(a.cpu().view(ibits), b.view(ibits))
        ref = O.apply_update(f64(b), eta, O.polar_direction(np.zeros(b.shape), 1), wd)
        assert np.array_equal(f64(a), ref)


def gpu_polar_u(shapes, votes, inv):
    """U of the local polar step (one iteration on the voted matrices), as
    fp32, through the same Newton-Schulz call with the U output."""
    us = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes]
    gpu_ns(shapes, 1, votes, inv, 1, L.SIGNMUON_OUT_U_F32, us)
    return us


# ---------------------------------------------------------------------------
# whole step
# ---------------------------------------------------------------------------
def _run_steps(wl, steps, seed=0, restore_after=None):
    from sign_muon_optimizer_momentum_b200.step import SignMuonStep
    dt = syn.torch_dtype(wl.w_dtype)
    opt = SignMuonStep(wl.shapes, wl.n_workers, wl.ns_iters, wl.variant, wl.beta, wl.eta, dt,
                       polar=wl.polar)
    weights = [w.cuda() for w in syn.initial_weights(wl, seed)]
    signal = syn.gradient_signal(wl, seed)       # drawn on the CPU, like the oracle's inputs
    grads = [torch.empty(s, dtype=dt, device="cuda") for s in wl.shapes for _ in range(wl.n_workers)]
    for t in range(steps):
        for i in range(len(wl.shapes)):
            for m in range(wl.n_workers):
                grads[i * wl.n_workers + m].copy_(syn.worker_gradient(wl, signal[i], i, m, t, seed))
        opt.step(weights, grads)
        if restore_after is not None and t == restore_after:
            sd = opt.state_dict()
            wsave = [w.clone() for w in weights]
            opt = SignMuonStep(wl.shapes, wl.n_workers, wl.ns_iters, wl.variant, wl.beta, wl.eta, dt,
                               polar=wl.polar)
            opt.load_state_dict(sd)
            for w, s in zip(weights, wsave):
                w.copy_(s)
    torch.cuda.synchronize()
    return opt, weights


def test_full_step_single256_against_oracle():
    wl = syn.WORKLOADS["single256"]
    opt, weights = _run_steps(wl, 1)
    w0 = syn.initial_weights(wl, 0)[0]
    signal = syn.gradient_signal(wl, 0)[0]
    grads = [syn.worker_gradient(wl, signal, 0, m, 0, 0) for m in range(wl.n_workers)]
    moms = [np.zeros(wl.shapes[0]) for _ in range(wl.n_workers)]
    ref = O.signmuon_step(f64(w0), [f64(g) for g in grads], moms, beta=float(np.float32(wl.beta)),
                          eta=wl.eta, k=wl.ns_iters, w_dtype=wl.w_dtype, int8_variant=True)
    for m in range(wl.n_workers):
        assert np.array_equal(f64(opt.mom[m]), ref["mom"][m])
        s_gpu = opt.signs[m].cpu().numpy()
        big = np.abs(ref["u"][m]) > 1e-3
        assert np.mean(s_gpu[big] == ref["signs"][m][big]) >= SIGN_AGREE
    got = f64(weights[0])
    # Where the GPU's vote equals the oracle's the update is bit-exact; the
    # votes can differ only where some worker's |U| is tiny.
    same = got == ref["w"]
    assert same.mean() >= 0.99
    steps = np.abs(got - ref["w"])[~same] / np.float32(wl.eta)
    assert np.all((np.abs(steps - 1) < 1e-3) | (np.abs(steps - 2) < 1e-3))


def test_step_is_deterministic_and_resumable():
    wl = syn.Workload("mini", ((96, 160), (160, 96), (64, 147)), 3, 2, "pack1", "bf16", g_noise_std=2.0)
    _, w_a = _run_steps(wl, 4)
    _, w_b = _run_steps(wl, 4)
    _, w_c = _run_steps(wl, 4, restore_after=1)
    for a, b, c in zip(w_a, w_b, w_c):
        assert torch.equal(a, b)
        assert torch.equal(a, c)


def test_polar_workload_small_runs():
    wl = syn.Workload("mini_polar", ((256, 256), (128, 384)), 4, 2, "pack1", "bf16", g_noise_std=4.0,
                      polar=True)
    opt, weights = _run_steps(wl, 2)
    w0 = syn.initial_weights(wl, 0)
    for w, w_init in zip(weights, w0):
        assert torch.isfinite(w.float()).all()
        assert not torch.equal(w.cpu(), w_init)


def test_polar_replans_when_weight_buffers_move():
    """The polar step's plan records the weight addresses: stepping new
    weight tensors (same values) must update those, not the old ones."""
    from sign_muon_optimizer_momentum_b200.step import SignMuonStep
    wl = syn.Workload("mini_polar2", ((128, 256), (256, 128)), 3, 1, "pack1", "f32", g_noise_std=2.0,
                      polar=True)
    signal = syn.gradient_signal(wl, 0)

    def grads(t):
        return [syn.worker_gradient(wl, signal[i], i, m, t, 0).cuda()
                for i in range(len(wl.shapes)) for m in range(wl.n_workers)]

    def run(move):
        opt = SignMuonStep(wl.shapes, wl.n_workers, wl.ns_iters, wl.variant, wl.beta, wl.eta, torch.float32,
                           polar=True)
        w = [x.cuda() for x in syn.initial_weights(wl, 0)]
        opt.step(w, grads(0))
        if move:
            old = w
            w = [x.clone() for x in old]
            for x in old:
                x.fill_(7.0)                      # must stay untouched from here on
        opt.step(w, grads(1))
        torch.cuda.synchronize()
        if move:
            assert all(bool((x == 7.0).all()) for x in old)
        return [x.cpu() for x in w]

    for a, b in zip(run(False), run(True)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("polar,norm", [(False, "frobenius"), (True, "frobenius"), (False, "spectral")])
def test_graph_replay_equals_eager_steps(polar, norm):
    """SignMuonStep.capture: replaying the captured step equals calling step()
    (weights and momentum bit for bit), with new gradient values every step."""
    from sign_muon_optimizer_momentum_b200.step import SignMuonStep
    wl = syn.Workload("graph", ((64, 96), (256, 256), (300, 128)), 3, 2, "pack1", "bf16", g_noise_std=2.0,
                      polar=polar)
    dt = torch.bfloat16
    signal = syn.gradient_signal(wl, 0)
    gvals = [[syn.worker_gradient(wl, signal[i], i, m, t, 0).cuda() for i in range(3) for m in range(3)]
             for t in range(3)]
    results = []
    for use_graph in (False, True):
        opt = SignMuonStep(wl.shapes, 3, 2, "pack1", 0.9, 0.02, dt, polar=polar, norm=norm)
        w = [x.cuda() for x in syn.initial_weights(wl, 0)]
        g = [torch.empty_like(x) for x in gvals[0]]
        graph = opt.capture(w, g) if use_graph else None
        for t in range(3):
            for dst, src in zip(g, gvals[t]):
                dst.copy_(src)
            if graph is not None:
                graph.replay()
            else:
                opt.step(w, g)
        torch.cuda.synchronize()
        results.append(([x.cpu() for x in w], [m.cpu() for m in opt.mom]))
    for a, b in zip(results[0][0] + results[0][1], results[1][0] + results[1][1]):
        assert torch.equal(a, b)


def test_nan_gradient_gives_all_plus_signs():
    """A NaN anywhere in one worker's gradient makes its normalised momentum
    (and U) NaN everywhere; sign(NaN) is +1 (bit = !(u < 0)), as in the
    oracle.  The other workers are unaffected."""
    shapes, M = [(64, 96)], 3
    grads, moms = seeded_state(shapes, M, 17)
    grads[1][5, 7] = float("nan")
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.cuda() for m in moms], 0.9, torch.float32)
    packed = [torch.zeros(L.signmuon_packed_words(shapes[0]), dtype=torch.int32, device="cuda") for _ in range(M)]
    gpu_ns(shapes, M, xs, inv, 2, L.SIGNMUON_OUT_PACK1, packed)
    r, c = shapes[0]
    for m in range(M):
        _, u = oracle_u(moms[m], grads[m], 0.9, 2)
        got = unpack_words(packed[m].cpu().numpy().view(np.uint32), r, c)
        if m == 1:
            assert np.isnan(u).all()
            assert (got == 1).all()
        else:
            big = np.abs(u) > 1e-3
            assert np.mean(got[big] == O.sign_entries(u)[big]) >= SIGN_AGREE


@pytest.mark.slow
def test_nanogpt_full_size_sampled_parity():
    """The nanoGPT-small workload at full size (48 matrices, M = 8, k = 5,
    1-bit vote), one step through the same path bench.py times.  Sampled
    checks on the four matrices of layer 0 (one of each shape): momentum of
    every worker bit-exact; the packed signs against the oracle's Newton-Schulz
    (sign agreement >= 99.5 % on |U| > 1e-3, every worker of the 768 x 768
    matrix, worker 0 of the others); and the vote + update of each of the
    four matrices bit-exact against the oracle's vote and update fed the
    step's own unpacked signs of all M workers."""
    wl = syn.WORKLOADS["nanogpt_small"]
    from sign_muon_optimizer_momentum_b200.step import SignMuonStep
    dt = syn.torch_dtype(wl.w_dtype)
    opt = SignMuonStep(wl.shapes, wl.n_workers, wl.ns_iters, wl.variant, wl.beta, wl.eta, dt)
    weights = [w.cuda() for w in syn.initial_weights(wl, 0)]
    w0 = [weights[i].clone() for i in range(4)]
    signal = [g.cuda() for g in syn.gradient_signal(wl, 0)]
    grads = [syn.worker_gradient(wl, signal[i], i, m, 0, 0).cuda() for i in range(len(wl.shapes))
             for m in range(wl.n_workers)]
    opt.step(weights, grads)
    torch.cuda.synchronize()
    M = wl.n_workers
    for i in range(4):  # one matrix of each shape (layer 0)
        r, c = wl.shapes[i]
        gpu_signs = [unpack_words(opt.signs[i * M + m].cpu().numpy().view(np.uint32), r, c) for m in range(M)]
        for m in (range(M) if i == 1 else [0]):
            u = i * M + m
            mom = O.momentum_update(np.zeros((r, c)), f64(grads[u]), float(np.float32(wl.beta)))
            assert np.array_equal(f64(opt.mom[u]), mom)
            U = O.newton_schulz(O.frobenius_normalize(mom), wl.ns_iters)
            big = np.abs(U) > 1e-3
            assert np.mean(gpu_signs[m][big] == O.sign_entries(U)[big]) >= SIGN_AGREE
        ref_w = O.apply_update(f64(w0[i]), wl.eta, O.majority_vote(gpu_signs), "bf16")
        assert np.array_equal(f64(weights[i]), ref_w), wl.shapes[i]


@pytest.mark.parametrize("int8_in", [False, True])
def test_vote_update_bf16_single_rounding_on_midpoint(int8_in):
    """eta = 2^-9 + 2^-30 puts the fp32 difference 1 - eta exactly on the bf16
    midpoint 1 - 2^-9 although the exact difference lies below it: a
    double-rounded update would give 1.0, the single rounding 0.99609375."""
    # 16 x 64 = 1024 weights: two full 512-weight warps of the int8 path and
    # one 1024-weight warp chunk of the packed path (the vector paths).
    shape, M = (16, 64), 1
    eta = float(np.float32(2.0 ** -9 + 2.0 ** -30))
    assert eta == 2.0 ** -9 + 2.0 ** -30
    w0 = torch.ones(shape, dtype=torch.bfloat16)
    w0[1::4] = -1.0
    w0[2::4] = 2.0
    w0[3::4] = syn.gaussian((4, 64), 1.0, "cpu", "mid", dtype=torch.bfloat16)
    signs = torch.ones(shape, dtype=torch.int8)
    signs[1::4] = -1
    dev = [signs.cuda()] if int8_in else _packed_device([signs], shape)
    w = w0.cuda()
    wk = ws(L.signmuon_vote_workspace_bytes([shape], M))
    L.signmuon_vote_update([shape], M, int8_in, [d.data_ptr() for d in dev], L.SIGNMUON_BF16, [w.data_ptr()], eta,
                           None, 0, 0, wk.data_ptr(), wk.numel(), stream())
    torch.cuda.synchronize()
    ref = O.apply_update(f64(w0), eta, signs.numpy(), "bf16")
    assert ref[0, 0] == 0.99609375
    assert np.array_equal(f64(w), ref)


@pytest.mark.parametrize("int8_in", [False, True])
@pytest.mark.parametrize("w_dtype", [torch.float32, torch.bfloat16])
def test_vote_tie_leaves_weights_bit_identical(int8_in, w_dtype):
    """A tied vote (even M, equal split) leaves W bit for bit, signed zeros
    included; the other entries follow the oracle."""
    shape, M = (16, 64), 2
    w0 = syn.gaussian(shape, 1.0, "cpu", "tie", dtype=w_dtype)
    w0[0, :32] = 0.0
    w0[0, 32:] = -0.0
    s0 = torch.ones(shape, dtype=torch.int8)
    s1 = -torch.ones(shape, dtype=torch.int8)   # every entry ties ...
    s1[8:] = 1                                  # ... except the lower half (+1)
    dev = [s0.cuda(), s1.cuda()] if int8_in else _packed_device([s0, s1], shape)
    w = w0.cuda()
    wk = ws(L.signmuon_vote_workspace_bytes([shape], M))
    code = L.SIGNMUON_BF16 if w_dtype == torch.bfloat16 else L.SIGNMUON_F32
    L.signmuon_vote_update([shape], M, int8_in, [d.data_ptr() for d in dev], code, [w.data_ptr()], 0.01,
                           None, 0, 0, wk.data_ptr(), wk.numel(), stream())
    torch.cuda.synchronize()
    ibits = torch.int16 if w_dtype == torch.bfloat16 else torch.int32
    assert torch.equal(w[:8].cpu().view(ibits), w0[:8].view(ibits))
    ref = O.apply_update(f64(w0), 0.01, O.majority_vote([s0.numpy(), s1.numpy()]),
                         "bf16" if w_dtype == torch.bfloat16 else "f32")
    assert np.array_equal(f64(w), ref)


@pytest.mark.parametrize("shapes,M,k", [([(256, 256), (300, 700)], 2, 2), ([(768, 2304), (3072, 768)], 1, 3),
                                        ([(64, 147), (513, 513)], 2, 1)])
def test_single_and_pair_tile_modes_agree(shapes, M, k, monkeypatch):
    """The one-CTA (128x256) and CTA-pair (256x256, cta_group::2) tile modes
    compute the same products; both stay within the oracle tolerance."""
    grads, moms = seeded_state(shapes, M, 13)
    outs = {}
    for mode in ("single", "pair"):
        monkeypatch.setenv("SIGNMUON_NS_TILE_MODE", mode)
        xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.clone().cuda() for m in moms], 0.9,
                               torch.float32)
        us = [torch.empty(shapes[u // M], dtype=torch.float32, device="cuda") for u in range(len(xs))]
        gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, us)
        outs[mode] = us
    for u in range(len(grads)):
        _, ref = oracle_u(moms[u], grads[u], 0.9, k)
        for mode in ("single", "pair"):
            assert rel_fro(f64(outs[mode][u]), ref) <= NS_TOL, (mode, shapes[u // M])
        assert rel_fro(f64(outs["single"][u]), f64(outs["pair"][u])) <= 1e-2


@pytest.mark.parametrize("variant,w_dtype,M", [("pack1", "bf16", 5), ("pack1", "f32", 4), ("int8", "f32", 3),
                                               ("int8", "bf16", 8)])
def test_signum_majority_vote_step_bit_exact(variant, w_dtype, M):
    """k = 0: the Newton-Schulz output is X0 = M/||M||_F, whose sign is the
    momentum's sign, so the step is the majority-vote Signum baseline the
    SignMuon summary compares against (beta = 0 gives majority-vote SignSGD).
    Momentum, vote and update are all exact, so the whole step is bit-exact."""
    wl = syn.Workload("signum_small", ((64, 96), (96, 64), (33, 147), (128, 256)), M, 0, variant, w_dtype,
                      g_noise_std=2.0)
    for beta in (0.9, 0.0):
        wl_b = syn.Workload(wl.name, wl.shapes, M, 0, variant, w_dtype, beta=beta, g_noise_std=2.0)
        opt, weights = _run_steps(wl_b, 2)
        w = [f64(x) for x in syn.initial_weights(wl_b, 0)]
        moms = [[np.zeros(s) for _ in range(M)] for s in wl_b.shapes]
        signal = syn.gradient_signal(wl_b, 0)
        for t in range(2):
            for i, shape in enumerate(wl_b.shapes):
                grads = [f64(syn.worker_gradient(wl_b, signal[i], i, m, t, 0)) for m in range(M)]
                ref = O.signmuon_step(w[i], grads, moms[i], beta=float(np.float32(beta)), eta=wl_b.eta, k=0,
                                      w_dtype=w_dtype, int8_variant=(variant == "int8"))
                moms[i], w[i] = ref["mom"], ref["w"]
        for i in range(len(wl_b.shapes)):
            assert np.array_equal(f64(weights[i]), w[i]), (beta, wl_b.shapes[i])
            for m in range(M):
                assert np.array_equal(f64(opt.mom[i * M + m]), moms[i][m])


# ---------------------------------------------------------------------------
# spectral scaling (power iteration)
# ---------------------------------------------------------------------------
SPEC_CASES = [([(256, 256)], 2, 5), ([(128, 384), (384, 128)], 2, 3), ([(64, 147), (33, 20)], 3, 1),
              ([(768, 2304), (3072, 768)], 1, 5), ([(1, 1), (1, 40), (40, 1)], 2, 2),
              # 4096 columns (a team of six warps, 3-row groups, ragged last segment) and 768
              # columns over 8 segments whose last group is ragged (one warp per row).
              ([(300, 4096), (1000, 768)], 2, 3),
              # Teams of two (776, 1536), three (2056: 257 chunks, the last one alone in its
              # warp), four (2568) and five warps (3840); the 65- and 33-row units end in a
              # group shorter than a team round.  8 columns: one chunk, lanes 1-31 idle.
              ([(200, 1536), (70, 2056), (130, 776), (65, 2568), (33, 3840), (9, 8)], 2, 2)]


def gpu_spectral(shapes, M, xs, inv, iters):
    w = ws(L.signmuon_spectral_workspace_bytes(shapes, M))
    L.signmuon_spectral_norm(shapes, M, [x.data_ptr() for x in xs], iters, inv.data_ptr(), w.data_ptr(), w.numel(),
                             stream())
    torch.cuda.synchronize()


@pytest.mark.parametrize("shapes,M,iters", SPEC_CASES)
def test_spectral_norm_matches_oracle(shapes, M, iters):
    grads, moms = seeded_state(shapes, M, 17)
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.cuda() for m in moms], 0.9, torch.float32)
    gpu_spectral(shapes, M, xs, inv, iters)
    for u in range(len(xs)):
        m, _ = oracle_u(moms[u], grads[u], 0.9, 0)
        # Same bf16 input as the kernel (rounded by the oracle itself): only
        # the summation order differs.
        ref_bf = 1.0 / (O.spectral_norm_estimate(O.round_to_bf16(m), iters) + O.NORM_EPS)
        assert math.isclose(inv[u].item(), ref_bf, rel_tol=2e-4), (shapes[u // M], inv[u].item(), ref_bf)
        ref = 1.0 / (O.spectral_norm_estimate(m, iters) + O.NORM_EPS)
        assert math.isclose(inv[u].item(), ref, rel_tol=5e-3)


def test_spectral_zero_matrix_and_ns_parity():
    shapes, M, iters, k = [(96, 300), (300, 96)], 2, 5, 5
    z = [torch.zeros(s, device="cuda") for s in shapes for _ in range(M)]
    xs, inv = gpu_momentum(shapes, M, z, [torch.zeros_like(t) for t in z], 0.9, torch.float32)
    gpu_spectral(shapes, M, xs, inv, iters)
    assert torch.allclose(inv, torch.full_like(inv, 1e7))
    grads, moms = seeded_state(shapes, M, 19)
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.cuda() for m in moms], 0.9, torch.float32)
    gpu_spectral(shapes, M, xs, inv, iters)
    us = [torch.empty(shapes[u // M], dtype=torch.float32, device="cuda") for u in range(len(xs))]
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, us)
    for u in range(len(xs)):
        m, _ = oracle_u(moms[u], grads[u], 0.9, 0)
        ref = O.newton_schulz(O.spectral_normalize(m, iters), k)
        got = f64(us[u])
        assert rel_fro(got, ref) <= NS_TOL
        big = np.abs(ref) > 1e-3
        assert np.mean(np.sign(got[big]) == np.sign(ref[big])) >= SIGN_AGREE


def test_spectral_step_runs_and_is_deterministic():
    from sign_muon_optimizer_momentum_b200.step import SignMuonStep
    wl = syn.Workload("spec", ((96, 160), (160, 96)), 3, 3, "pack1", "bf16", g_noise_std=2.0)
    results = []
    for _ in range(2):
        opt = SignMuonStep(wl.shapes, wl.n_workers, wl.ns_iters, wl.variant, wl.beta, wl.eta, torch.bfloat16,
                           norm="spectral", spectral_iters=4)
        weights = [w.cuda() for w in syn.initial_weights(wl, 0)]
        signal = syn.gradient_signal(wl, 0)
        grads = [syn.worker_gradient(wl, signal[i], i, m, 0, 0).cuda() for i in range(2) for m in range(3)]
        opt.step(weights, grads)
        torch.cuda.synchronize()
        results.append([w.clone() for w in weights])
    for a, b in zip(*results):
        assert torch.equal(a, b)


# ---------------------------------------------------------------------------
# full-size workloads (sampled outputs), in the launch configuration bench.py times
# ---------------------------------------------------------------------------
@pytest.mark.slow
def test_resnet50_full_size_sampled_parity():
    """ResNet-50 shapes at full size (54 matrices, M = 4, k = 1, int8 vote):
    momentum of every unit bit-exact; the int8 signs of a sample of matrices
    against the oracle's Newton-Schulz (sign agreement >= 99.5 % on
    |U| > 1e-3); and the vote + update of those matrices bit-exact against
    the oracle's vote and update fed the step's own int8 signs."""
    from sign_muon_optimizer_momentum_b200.step import SignMuonStep
    wl = syn.WORKLOADS["resnet50"]
    M = wl.n_workers
    opt = SignMuonStep(wl.shapes, M, wl.ns_iters, wl.variant, wl.beta, wl.eta, torch.float32)
    w0 = syn.initial_weights(wl, 0)
    weights = [w.cuda() for w in w0]
    signal = syn.gradient_signal(wl, 0)
    grads = [syn.worker_gradient(wl, signal[i], i, m, 0, 0) for i in range(len(wl.shapes)) for m in range(M)]
    opt.step(weights, [g.cuda() for g in grads])
    torch.cuda.synchronize()
    beta = float(np.float32(wl.beta))
    for u, g in enumerate(grads):
        assert np.array_equal(f64(opt.mom[u]), O.momentum_update(np.zeros(g.shape), f64(g), beta))
    for i in (0, 7, 20, 40, 53):   # 64x147, 128x1152-class, 1024x256, 512x2048-class, 2048x1000
        r, c = wl.shapes[i]
        gpu_signs = [opt.signs[i * M + m].cpu().numpy() for m in range(M)]
        for m in range(M):
            mom = O.momentum_update(np.zeros((r, c)), f64(grads[i * M + m]), beta)
            U = O.newton_schulz(O.frobenius_normalize(mom), wl.ns_iters)
            big = np.abs(U) > 1e-3
            if big.sum():
                assert np.mean(gpu_signs[m][big] == O.sign_entries(U)[big]) >= SIGN_AGREE
        ref_w = O.apply_update(f64(w0[i]), wl.eta, O.majority_vote(gpu_signs), "f32")
        assert np.array_equal(f64(weights[i]), ref_w), wl.shapes[i]


@pytest.mark.slow
def test_square4096_batch_full_size_sampled():
    """32 x 4096^2, M = 16, k = 5, 1-bit vote and local polar step, at full
    size through the path bench.py times: sampled momentum bit-exact; sampled
    Newton-Schulz signs against the fp64 oracle; the vote matrix, its nnz and
    1/sqrt(nnz) exact against the majority of the step's own packed signs;
    the polar step's U within 2e-2 of the oracle's polar direction of that
    vote; and the bf16 polar update bit-exact against the oracle's update
    with the device's U."""
    from sign_muon_optimizer_momentum_b200.step import SignMuonStep
    wl = syn.WORKLOADS["square4096x32"]
    M = wl.n_workers
    dt = torch.bfloat16
    opt = SignMuonStep(wl.shapes, M, wl.ns_iters, wl.variant, wl.beta, wl.eta, dt, polar=True)
    weights = [w.cuda() for w in syn.initial_weights(wl, 0, device="cpu")]
    w_before = weights[3].clone()
    signal = [g.cuda() for g in syn.gradient_signal(wl, 0, device="cuda")]
    grads = [torch.empty(s, dtype=dt, device="cuda") for s in wl.shapes for _ in range(M)]
    for i in range(len(wl.shapes)):
        for m in range(M):
            syn.worker_gradient(wl, signal[i], i, m, 0, 0, out=grads[i * M + m])
    opt.step(weights, grads)
    torch.cuda.synchronize()
    beta = float(np.float32(wl.beta))
    u = 3 * M + 5
    mom = O.momentum_update(np.zeros((4096, 4096)), f64(grads[u]), beta)
    assert np.array_equal(f64(opt.mom[u]), mom)
    U = O.newton_schulz(O.frobenius_normalize(mom), wl.ns_iters)
    s_gpu = unpack_words(opt.signs[u].cpu().numpy().view(np.uint32), 4096, 4096)
    big = np.abs(U) > 1e-3
    assert np.mean(s_gpu[big] == O.sign_entries(U)[big]) >= SIGN_AGREE
    # The vote matrix of matrix 3 is the majority of the step's own signs.
    count = sum((unpack_words(opt.signs[3 * M + m].cpu().numpy().view(np.uint32), 4096, 4096) == 1)
                .astype(np.int64) for m in range(M))
    vote = np.sign(2 * count - M)
    assert np.array_equal(f64(opt.vote[3])[:, :4096], vote)
    assert opt.nnz[3].item() == np.count_nonzero(vote)
    # The local polar step on that vote: its U (the same call with the fp32
    # output) within the Newton-Schulz tolerance of the oracle's polar
    # direction, and the bf16 update bit-exact against the oracle's update
    # with the device's own U.
    inv = opt.vote_inv[3:4]
    assert inv.item() == np.float32(1.0 / math.sqrt(np.count_nonzero(vote)))
    u_gpu = f64(gpu_polar_u([(4096, 4096)], [opt.vote[3]], inv)[0])
    d_ref = O.polar_direction(vote, 1)
    assert rel_fro(u_gpu, d_ref) <= NS_TOL
    big = np.abs(d_ref) > 1e-3
    if big.sum():
        assert np.mean(np.sign(u_gpu[big]) == np.sign(d_ref[big])) >= SIGN_AGREE
    assert np.array_equal(f64(weights[3]), O.apply_update(f64(w_before), wl.eta, u_gpu, "bf16"))


@pytest.mark.parametrize("shapes,M,k", [([(2056, 2100)], 1, 2), ([(300, 2100), (2100, 300)], 2, 1)])
def test_long_reduction_layout_ragged_edges(shapes, M, k, monkeypatch):
    """Launches whose every tile has a reduction of 2048 or more use the
    layout that stores its 16-bit outputs from registers (256x512 tiles).  Ragged
    sizes (2056 x 2100: all three products long; 300 x 2100 and its
    transpose: the Gram product long) put row and column edges inside tiles
    and inside 32-column chunks: U within the Newton-Schulz tolerance of the
    oracle, and packed signs equal to the signs of that U."""
    monkeypatch.setenv("SIGNMUON_NS_TILE_MODE", "pair")
    grads, moms = seeded_state(shapes, M, 23)
    us = [torch.empty(shapes[u // M], dtype=torch.float32, device="cuda") for u in range(len(grads))]
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.clone().cuda() for m in moms], 0.9,
                           torch.float32)
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, us)
    packed = [torch.zeros(L.signmuon_packed_words(shapes[u // M]), dtype=torch.int32, device="cuda")
              for u in range(len(grads))]
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.clone().cuda() for m in moms], 0.9,
                           torch.float32)
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_PACK1, packed)
    for u in range(len(grads)):
        r, c = shapes[u // M]
        _, ref = oracle_u(moms[u], grads[u], 0.9, k)
        got = f64(us[u])
        assert rel_fro(got, ref) <= NS_TOL, shapes[u // M]
        big = np.abs(ref) > 1e-3
        assert np.mean((got[big] < 0) == (ref[big] < 0)) >= SIGN_AGREE
        assert np.array_equal(unpack_words(packed[u].cpu().numpy().view(np.uint32), r, c), O.sign_entries(got))


@pytest.mark.parametrize("shapes,M,k", [([(2056, 2100)], 1, 2), ([(300, 2100), (2100, 300)], 2, 1),
                                        ([(2048, 4096), (4096, 2304)], 1, 1), ([(2560, 2560)], 2, 1)])
def test_wide_tiles_equal_256_tiles(shapes, M, k, monkeypatch):
    """The long-reduction launches run 256x512 CTA-pair tiles (two N = 256
    MMAs per K step into the two halves of one TMEM accumulator, the first and
    last k-blocks of a tile issuing half 0 ahead of half 1).  Each output
    entry is accumulated over the same k-blocks in the same order as on
    256x256 tiles, so U is bit-identical to the 256x256 layout's, on ragged
    edges, on symmetric outputs whose tile rows start in the second half of a
    512-column tile, and on tiles whose second half lies past the matrix; and
    within the oracle tolerance."""
    monkeypatch.setenv("SIGNMUON_NS_TILE_MODE", "pair")
    grads, moms = seeded_state(shapes, M, 29)
    outs = {}
    for wide in ("0", "1"):
        monkeypatch.setenv("SIGNMUON_NS_WIDE", wide)
        xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.clone().cuda() for m in moms], 0.9,
                               torch.float32)
        us = [torch.empty(shapes[u // M], dtype=torch.float32, device="cuda") for u in range(len(xs))]
        gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, us)
        outs[wide] = us
    for u in range(len(grads)):
        assert torch.equal(outs["0"][u], outs["1"][u]), shapes[u // M]
        _, ref = oracle_u(moms[u], grads[u], 0.9, k)
        assert rel_fro(f64(outs["1"][u]), ref) <= NS_TOL, shapes[u // M]


@pytest.mark.slow
def test_square4096_two_units_ns_over_waves(monkeypatch):
    """Newton-Schulz at s = 4096 (K = 4096 mainloops, 16 x 16 upper-block
    storage of the symmetric intermediates) on two units of the 4096^2
    batch, k = 5, CTA-pair tiles, with a workspace that holds one unit so the
    call runs in two waves: U within 2e-2 relative Frobenius error of the
    fp64 oracle and sign agreement >= 99.5 % on |U| > 1e-3."""
    monkeypatch.setenv("SIGNMUON_NS_TILE_MODE", "pair")
    shapes, M, k = [(4096, 4096)], 2, 5
    grads, moms = seeded_state(shapes, M, 41, grad_dtype=torch.bfloat16, g_std=4.0)
    xs, inv = gpu_momentum(shapes, M, [g.cuda() for g in grads], [m.clone().cuda() for m in moms], 0.9,
                           torch.bfloat16)
    us = [torch.empty(shapes[0], dtype=torch.float32, device="cuda") for _ in range(M)]
    gpu_ns(shapes, M, xs, inv, k, L.SIGNMUON_OUT_U_F32, us, minimal_ws=True)
    for m in range(M):
        _, ref = oracle_u(moms[m], grads[m], 0.9, k)
        got = f64(us[m])
        assert rel_fro(got, ref) <= NS_TOL, m
        big = np.abs(ref) > 1e-3
        assert np.mean((got[big] < 0) == (ref[big] < 0)) >= SIGN_AGREE


@pytest.mark.slow
@pytest.mark.parametrize("M", [16, 64])
def test_vote_sweep_1b_params_sampled_bit_exact(M):
    """The vote sweep at 2^30 parameters (fp32 W, eta = 0.01): the updated
    weights at 4096 sampled positions equal the oracle's vote and update of
    the same seeded int8 signs, bit for bit."""
    P = 1 << 30
    shape = (P // 1024, 1024)
    rng = np.random.default_rng(M)
    idx = torch.from_numpy(rng.choice(P, 4096, replace=False)).cuda()
    words = L.signmuon_packed_words(shape)
    packed, sampled = [], []
    for m, s8 in syn.vote_sweep_signs(P, M, seed=3, device="cuda"):
        buf = torch.empty(words, dtype=torch.int32, device="cuda")
        L.signmuon_sign_pack(shape, L.SIGNMUON_F32, s8.float().data_ptr(), 1024, 0, buf.data_ptr(), stream())
        torch.cuda.synchronize()
        packed.append(buf)
        sampled.append(s8[idx].cpu().numpy())
        del s8
    w = syn.gaussian(shape, 0.02, "cuda", "W", 3, 0)
    w_s = w.view(-1)[idx].cpu().numpy()
    wk = ws(L.signmuon_vote_workspace_bytes([shape], M))
    L.signmuon_vote_update([shape], M, False, [t.data_ptr() for t in packed], L.SIGNMUON_F32, [w.data_ptr()], 0.01,
                           None, 0, 0, wk.data_ptr(), wk.numel(), stream())
    torch.cuda.synchronize()
    v = O.majority_vote([s[None, :] for s in sampled])[0]
    ref = O.apply_update(w_s.astype(np.float64), 0.01, v, "f32")
    assert np.array_equal(w.view(-1)[idx].cpu().double().numpy(), ref)
