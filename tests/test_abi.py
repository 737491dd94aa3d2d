"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and its host-side helpers and argument validation behave as
documented (validation returns before anything touches the device)."""
import ctypes
import os
import re

import pytest

from sign_muon_optimizer_momentum_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "signmuon.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(signmuon_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(L.LIB_PATH):
        from sign_muon_optimizer_momentum_b200 import build
        build.build()
    return L.load()


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert declared == sorted(L.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_version_and_layout_helpers(lib):
    assert L.signmuon_abi_version() == 1
    assert [L.signmuon_x_ld(c) for c in (1, 7, 8, 9, 147, 1000, 4096)] == [8, 8, 8, 16, 152, 1000, 4096]
    assert L.signmuon_x_ld(0) == -1
    # rows * ceil(cols/32), rounded up to a multiple of 4 words.
    assert L.signmuon_packed_words((1, 1)) == 4
    assert L.signmuon_packed_words((3, 33)) == 8
    assert L.signmuon_packed_words((64, 147)) == 320
    assert L.signmuon_packed_words((4096, 4096)) == 4096 * 128
    assert L.signmuon_packed_words((0, 5)) == -1


def test_status_strings(lib):
    for code, name in [(0, "SIGNMUON_OK"), (1, "SIGNMUON_ERR_INVALID_ARG"), (2, "SIGNMUON_ERR_ALIGNMENT"),
                       (3, "SIGNMUON_ERR_UNSUPPORTED"), (4, "SIGNMUON_ERR_WORKSPACE"), (5, "SIGNMUON_ERR_CUDA")]:
        assert L.status_string(code) == name
    assert L.status_string(99) == "SIGNMUON_UNKNOWN_STATUS"


def test_workspace_sizes(lib):
    shapes = [(768, 2304), (3072, 768)]
    mom = L.signmuon_momentum_workspace_bytes(shapes, 8)
    blocks = 8 * (-(-768 * 2304 // 4096) + -(-3072 * 768 // 4096))
    assert mom >= 256 + 16 * 56 + 4 * blocks
    full = L.signmuon_newton_schulz_workspace_bytes(shapes, 8)
    minimal = L.signmuon_newton_schulz_workspace_bytes(shapes, 8, minimal=True)
    assert minimal < full
    # One unit of the largest buffers: A and B' (768^2 16-bit each) + an X copy.
    assert minimal >= 256 + 16 * 1152 + 2 * 768 * 768 * 2 + 3072 * 768 * 2
    assert L.signmuon_vote_workspace_bytes(shapes, 8) >= 256 + 2 * 64 + 16 * 8
    assert L.signmuon_momentum_workspace_bytes([], 8) == 0
    assert L.signmuon_momentum_workspace_bytes([(0, 3)], 8) == 0


def _err(fn, *args):
    with pytest.raises(L.SignMuonError) as e:
        fn(*args)
    return e.value.status


def test_argument_validation_returns_status(lib):
    fake = 1 << 20            # a 16-byte-aligned address that is never dereferenced
    odd = fake + 4            # misaligned
    shp = [(4, 8)]
    # Momentum.
    assert _err(L.signmuon_momentum_norm, shp, 0, 0, [fake], [fake], 0.9, [fake], fake, fake, 1 << 20) == 1
    assert _err(L.signmuon_momentum_norm, shp, 1, 7, [fake], [fake], 0.9, [fake], fake, fake, 1 << 20) == 1
    assert _err(L.signmuon_momentum_norm, shp, 1, 0, [0], [fake], 0.9, [fake], fake, fake, 1 << 20) == 1
    assert _err(L.signmuon_momentum_norm, shp, 1, 0, [odd], [fake], 0.9, [fake], fake, fake, 1 << 20) == 2
    assert _err(L.signmuon_momentum_norm, shp, 1, 0, [fake], [fake], 0.9, [fake], fake, 0, 1 << 20) == 4
    assert _err(L.signmuon_momentum_norm, shp, 1, 0, [fake], [fake], 0.9, [fake], fake, fake, 16) == 4
    assert _err(L.signmuon_momentum_norm, [(0, 8)], 1, 0, [fake], [fake], 0.9, [fake], fake, fake, 1 << 20) == 1
    assert _err(L.signmuon_momentum_norm, shp, 128, 0, [fake] * 128, [fake] * 128, 0.9, [fake] * 128, fake,
                fake, 1 << 30) == 1
    # Fused momentum + sign (k = 0): packed output needs cols % 32 == 0.
    ms_ = L.signmuon_momentum_sign
    assert _err(ms_, [(4, 40)], 1, 0, [fake], [fake], 0.9, False, [fake], fake, fake, 1 << 20) == 3
    assert _err(ms_, [(4, 64)], 1, 0, [fake], [fake], 0.9, False, [odd], fake, fake, 1 << 20) == 2
    assert _err(ms_, [(4, 40)], 1, 0, [fake], [fake], 0.9, True, [0], fake, fake, 1 << 20) == 1
    assert _err(ms_, [(4, 40)], 1, 0, [fake], [fake], 0.9, True, [fake], fake, fake, 16) == 4
    # Newton-Schulz.
    a, b, c = 3.4445, -4.7750, 2.0315
    ns = L.signmuon_newton_schulz_batched
    assert _err(ns, shp, 1, [fake], fake, -1, a, b, c, 0, [fake], 0, None, 0.0, fake, 1 << 30) == 1
    assert _err(ns, shp, 1, [fake], fake, 65, a, b, c, 0, [fake], 0, None, 0.0, fake, 1 << 30) == 1
    assert _err(ns, shp, 1, [fake], fake, 1, a, b, c, 9, [fake], 0, None, 0.0, fake, 1 << 30) == 1
    assert _err(ns, shp, 1, [odd], fake, 1, a, b, c, 0, [fake], 0, None, 0.0, fake, 1 << 30) == 2
    assert _err(ns, shp, 1, [fake], fake, 1, a, b, c, 0, [fake], 0, None, 0.0, fake, 64) == 4
    assert _err(ns, shp, 1, [fake], fake, 1, a, b, c, 0, [fake], 0, None, 0.0, fake + 16, 1 << 30) == 2
    # inv_norm needs 4-byte alignment only (one float per unit).
    assert _err(ns, shp, 1, [fake], fake + 2, 1, a, b, c, 0, [fake], 0, None, 0.0, fake, 1 << 30) == 2
    assert _err(ns, shp, 1, [fake], fake + 4, 1, a, b, c, 0, [fake], 0, None, 0.0, fake, 64) == 4
    # UPDATE_W needs one worker and weights.
    assert _err(ns, shp, 2, [fake, fake], fake, 1, a, b, c, 2, None, 0, [fake], 0.1, fake, 1 << 30) == 1
    assert _err(ns, shp, 1, [fake], fake, 1, a, b, c, 2, None, 0, None, 0.1, fake, 1 << 30) == 1
    # Newton-Schulz plan / run.
    assert L.signmuon_newton_schulz_plan_bytes(0, 1) == 0
    assert L.signmuon_newton_schulz_plan_bytes(1, 128) == 0
    assert L.signmuon_newton_schulz_plan_bytes(2, 3) >= 6 * 32
    plan = (ctypes.c_uint64 * 64)()
    pl = L.load().signmuon_newton_schulz_plan
    sh = (L.Shape * 1)(L.Shape(4, 8))
    xp = (ctypes.c_void_p * 1)(fake)
    op = (ctypes.c_void_p * 1)(fake)
    args = [sh, 1, 1, xp, fake, 0, op, 0, None, fake, 1 << 30]
    assert pl(*args, None, 512, None) == 1                              # no plan buffer
    assert pl(*args, ctypes.addressof(plan), 8, None) == 1               # plan buffer too small
    assert pl(*args, ctypes.addressof(plan) + 4, 500, None) == 2         # misaligned plan buffer
    assert pl(sh, 1, 1, xp, fake, 7, op, 0, None, fake, 1 << 30, ctypes.addressof(plan), 512, None) == 1
    assert pl(*args[:-1], 64, ctypes.addressof(plan), 512, None) == 4    # workspace too small
    run = L.load().signmuon_newton_schulz_run
    assert run(None, 1, a, b, c, 0.0, None) == 1
    assert run(ctypes.addressof(plan), 1, a, b, c, 0.0, None) == 1        # never filled (rejected plan)
    assert _err(L.signmuon_newton_schulz_run, plan, 1, a, b, c, 0.0) == 1
    # Sign pack.
    assert _err(L.signmuon_sign_pack, (4, 8), 0, fake, 4, 0, fake) == 1      # ld < cols
    assert _err(L.signmuon_sign_pack, (4, 8), 3, fake, 8, 0, fake) == 1      # bad dtype
    assert _err(L.signmuon_sign_pack, (4, 8), 0, odd, 8, 0, fake) == 2
    assert _err(L.signmuon_sign_pack, (0, 8), 0, fake, 8, 0, fake) == 1
    # Spectral scaling.
    sp = L.signmuon_spectral_norm
    assert _err(sp, shp, 1, [fake], 0, fake, fake, 1 << 20) == 1          # iters < 1
    assert _err(sp, shp, 1, [odd], 3, fake, fake, 1 << 20) == 2
    assert _err(sp, shp, 1, [fake], 3, fake, fake, 64) == 4
    assert _err(sp, shp, 0, [fake], 3, fake, fake, 1 << 20) == 1
    # Vote.
    vu = L.signmuon_vote_update
    assert _err(vu, shp, 0, 0, [], 0, [fake], 0.01, None, 0, 0, fake, 1 << 20) == 1
    assert _err(vu, shp, 2, 0, [fake, 0], 0, [fake], 0.01, None, 0, 0, fake, 1 << 20) == 1
    assert _err(vu, shp, 2, 0, [fake, odd], 0, [fake], 0.01, None, 0, 0, fake, 1 << 20) == 2
    assert _err(vu, shp, 2, 0, [fake, fake], 5, [fake], 0.01, None, 0, 0, fake, 1 << 20) == 1
    assert _err(vu, shp, 2, 0, [fake, fake], 0, [fake], 0.01, [fake], 0, 0, fake, 1 << 20) == 1
    assert _err(vu, shp, 2, 0, [fake, fake], 0, [fake], 0.01, None, 0, 0, fake, 8) == 4


def test_binding_refuses_to_run_without_library(tmp_path, monkeypatch):
    """No fallback: a missing library is a loud error, not a silent CPU path."""
    import importlib
    mod = importlib.reload(L)
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(mod, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        mod.load()
    importlib.reload(L)
