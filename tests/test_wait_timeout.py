"""The bounded waits of the Newton-Schulz kernel and of the spectral segment
pass, made to run out on purpose.

Every mbarrier wait in the kernel gives up after a time limit, records a
wait-timeout code in the first word of the workspace and lets the kernel
return (no trap, no hang).  The library's fault injection
(SIGNMUON_NS_INJECT_WAIT_TIMEOUT_US) makes the producer withhold every
operand load, so the MMA issuer's and the epilogue's waits can only run out,
and shortens the limit to a few milliseconds.  The test checks that the call
returns, that signmuon_device_error reports a wait-timeout code (and clears
it), and that the next normal call on the same context and workspace gives
the oracle's result.  Both tile modes: one-CTA tiles, where each CTA gives
up on its own, and CTA pairs on a long-reduction launch (256x512 tiles),
where the even CTA's MMA issuer and the odd CTA's producer and epilogue each
give up on their own bounded waits before the pair's exit barrier.
"""
import time

import numpy as np
import pytest
import torch

from oracle import signmuon_oracle as O
from sign_muon_optimizer_momentum_b200 import _lib as L
from sign_muon_optimizer_momentum_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

WAIT_TIMEOUT_CODES = {0x101, 0x102, 0x103}   # producer, MMA issuer, epilogue


def _inputs(shapes, M):
    grads = [syn.gaussian(s, 2.0, "cpu", "wt_g", i, m) for i, s in enumerate(shapes) for m in range(M)]
    moms = [syn.gaussian(s, 1.0, "cpu", "wt_m", i, m) for i, s in enumerate(shapes) for m in range(M)]
    return grads, moms


def _momentum(shapes, M, grads, moms, stream):
    xs = [torch.empty((r, L.signmuon_x_ld(c)), dtype=torch.bfloat16, device="cuda") for r, c in shapes
          for _ in range(M)]
    inv = torch.empty(len(shapes) * M, dtype=torch.float32, device="cuda")
    wk = torch.zeros(L.signmuon_momentum_workspace_bytes(shapes, M), dtype=torch.uint8, device="cuda")
    L.signmuon_momentum_norm(shapes, M, L.SIGNMUON_F32, [g.data_ptr() for g in grads],
                             [m.data_ptr() for m in moms], 0.9, [x.data_ptr() for x in xs], inv.data_ptr(),
                             wk.data_ptr(), wk.numel(), stream)
    return xs, inv


@pytest.mark.parametrize("shapes,M,k,mode", [([(256, 256), (96, 300)], 2, 2, "single"),
                                             ([(2048, 2048)], 1, 1, "pair")])
def test_injected_wait_timeout_is_reported_and_the_context_stays_usable(cuda_lib, monkeypatch, shapes, M, k,
                                                                         mode):
    stream = torch.cuda.current_stream().cuda_stream
    grads, moms = _inputs(shapes, M)
    nbytes = L.signmuon_newton_schulz_workspace_bytes(shapes, M)
    wk = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    us = [torch.full(shapes[u // M], 7.0, dtype=torch.float32, device="cuda") for u in range(len(grads))]
    monkeypatch.setenv("SIGNMUON_NS_TILE_MODE", mode)

    # 1. Loads withheld, 20 ms limit: 3k launches, each gives up on its own.
    xs, inv = _momentum(shapes, M, [g.cuda() for g in grads], [m.clone().cuda() for m in moms], stream)
    torch.cuda.synchronize()
    monkeypatch.setenv("SIGNMUON_NS_INJECT_WAIT_TIMEOUT_US", "20000")
    t0 = time.perf_counter()
    L.signmuon_newton_schulz_batched(shapes, M, [x.data_ptr() for x in xs], inv.data_ptr(), k, *O.NS_QUINTIC,
                                     L.SIGNMUON_OUT_U_F32, [u.data_ptr() for u in us], L.SIGNMUON_F32, None, 0.0,
                                     wk.data_ptr(), wk.numel(), stream)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    code = L.signmuon_device_error(wk.data_ptr(), stream)
    assert code in WAIT_TIMEOUT_CODES, hex(code)
    assert elapsed < 1.5, elapsed                  # 3k launches x a few 20 ms waits, far below the 2 s default
    assert L.signmuon_device_error(wk.data_ptr(), stream) == 0     # read and cleared
    assert all(bool((u == 7.0).all()) for u in us)                 # the outputs were not written

    # 2. The same context, workspace and stream, normal operation.
    monkeypatch.delenv("SIGNMUON_NS_INJECT_WAIT_TIMEOUT_US")
    xs, inv = _momentum(shapes, M, [g.cuda() for g in grads], [m.clone().cuda() for m in moms], stream)
    L.signmuon_newton_schulz_batched(shapes, M, [x.data_ptr() for x in xs], inv.data_ptr(), k, *O.NS_QUINTIC,
                                     L.SIGNMUON_OUT_U_F32, [u.data_ptr() for u in us], L.SIGNMUON_F32, None, 0.0,
                                     wk.data_ptr(), wk.numel(), stream)
    torch.cuda.synchronize()
    assert L.signmuon_device_error(wk.data_ptr(), stream) == 0
    for u, (g, m0) in enumerate(zip(grads, moms)):
        mom = O.momentum_update(m0.double().numpy(), g.double().numpy(), float(np.float32(0.9)))
        ref = O.newton_schulz(O.frobenius_normalize(mom), k)
        got = us[u].double().cpu().numpy()
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 2e-2


def test_injected_spectral_wait_timeout_is_reported_and_the_context_stays_usable(cuda_lib, monkeypatch):
    """The spectral segment pass's bounded waits: with its row loads withheld
    (SIGNMUON_SPECTRAL_INJECT_WAIT_TIMEOUT_US) every block gives up after the
    limit and records the spectral wait-timeout code; the next normal call on
    the same context and workspace matches the oracle.  One-warp rows (768
    columns) and three-warp teams (2304 columns)."""
    shapes, M, iters = [(256, 768), (300, 2304)], 2, 2
    stream = torch.cuda.current_stream().cuda_stream
    grads, moms = _inputs(shapes, M)
    nbytes = L.signmuon_spectral_workspace_bytes(shapes, M)
    wk = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    xs, inv = _momentum(shapes, M, [g.cuda() for g in grads], [m.clone().cuda() for m in moms], stream)
    torch.cuda.synchronize()

    # 1. Rows withheld, 20 ms limit: `iters` segment passes, each gives up once.
    monkeypatch.setenv("SIGNMUON_SPECTRAL_INJECT_WAIT_TIMEOUT_US", "20000")
    t0 = time.perf_counter()
    L.signmuon_spectral_norm(shapes, M, [x.data_ptr() for x in xs], iters, inv.data_ptr(), wk.data_ptr(), wk.numel(),
                             stream)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert L.signmuon_device_error(wk.data_ptr(), stream) == 0x105
    assert elapsed < 1.5, elapsed                  # far below the 2 s default limit per pass
    assert L.signmuon_device_error(wk.data_ptr(), stream) == 0     # read and cleared

    # 2. The same context, workspace and stream, normal operation.
    monkeypatch.delenv("SIGNMUON_SPECTRAL_INJECT_WAIT_TIMEOUT_US")
    L.signmuon_spectral_norm(shapes, M, [x.data_ptr() for x in xs], iters, inv.data_ptr(), wk.data_ptr(), wk.numel(),
                             stream)
    torch.cuda.synchronize()
    assert L.signmuon_device_error(wk.data_ptr(), stream) == 0
    for u, (g, m0) in enumerate(zip(grads, moms)):
        mom = O.momentum_update(m0.double().numpy(), g.double().numpy(), float(np.float32(0.9)))
        ref = 1.0 / (O.spectral_norm_estimate(O.round_to_bf16(mom), iters) + O.NORM_EPS)
        assert abs(inv[u].item() - ref) <= 2e-4 * ref, (u, inv[u].item(), ref)
