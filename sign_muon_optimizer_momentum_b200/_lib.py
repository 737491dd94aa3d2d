"""ctypes binding of libsignmuon.so (declared in include/signmuon.h).

Argument marshalling only: every function here converts Python ints, lists
and shapes into the C types of the entry point of the same name, calls it and
turns a non-zero status into ``SignMuonError``.  Pointers are plain integers
(device addresses, e.g. ``tensor.data_ptr()``); streams are integers
(``torch.cuda.Stream.cuda_stream``).  No computation happens in Python and
there is no fallback: if the library has not been built, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsignmuon.so")

SIGNMUON_OK = 0
SIGNMUON_ERR_INVALID_ARG = 1
SIGNMUON_ERR_ALIGNMENT = 2
SIGNMUON_ERR_UNSUPPORTED = 3
SIGNMUON_ERR_WORKSPACE = 4
SIGNMUON_ERR_CUDA = 5

SIGNMUON_F32 = 0
SIGNMUON_BF16 = 1

SIGNMUON_OUT_PACK1 = 0
SIGNMUON_OUT_INT8 = 1
SIGNMUON_OUT_UPDATE_W = 2
SIGNMUON_OUT_U_F32 = 3

SIGNMUON_MAX_WORKERS = 127

# Every symbol include/signmuon.h declares.
EXPORTS = (
    "signmuon_status_string", "signmuon_abi_version", "signmuon_x_ld", "signmuon_packed_words",
    "signmuon_device_error", "signmuon_momentum_workspace_bytes", "signmuon_momentum_norm",
    "signmuon_newton_schulz_workspace_bytes", "signmuon_newton_schulz_batched",
    "signmuon_newton_schulz_plan_bytes", "signmuon_newton_schulz_plan", "signmuon_newton_schulz_run",
    "signmuon_sign_pack", "signmuon_vote_workspace_bytes", "signmuon_vote_update",
    "signmuon_momentum_norm_noalloc", "signmuon_last_error_string",
    "signmuon_spectral_workspace_bytes", "signmuon_spectral_norm", "signmuon_momentum_sign",
)


class SignMuonError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        detail = f": {signmuon_last_error_string()}" if status == SIGNMUON_ERR_CUDA else ""
        super().__init__(f"{fn} failed: {status_string(status)} ({status}){detail}")


class Shape(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int32), ("cols", ctypes.c_int32)]


_P = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)
_SZ = ctypes.c_size_t
_I = ctypes.c_int
_F = ctypes.c_float

_SIGS = {
    "signmuon_status_string": (ctypes.c_char_p, [_I]),
    "signmuon_abi_version": (_I, []),
    "signmuon_last_error_string": (ctypes.c_char_p, []),
    "signmuon_x_ld": (ctypes.c_int32, [ctypes.c_int32]),
    "signmuon_packed_words": (ctypes.c_int64, [Shape]),
    "signmuon_device_error": (_I, [_P, ctypes.POINTER(ctypes.c_uint32), _P]),
    "signmuon_momentum_workspace_bytes": (_SZ, [ctypes.POINTER(Shape), _I, _I]),
    "signmuon_momentum_norm": (_I, [ctypes.POINTER(Shape), _I, _I, _I, _PP, _PP, _F, _PP, _P, _P,
                                    _SZ, _P]),
    "signmuon_momentum_sign": (_I, [ctypes.POINTER(Shape), _I, _I, _I, _PP, _PP, _F, _I, _PP, _P, _P, _SZ, _P]),
    "signmuon_newton_schulz_workspace_bytes": (_SZ, [ctypes.POINTER(Shape), _I, _I, _I]),
    "signmuon_newton_schulz_batched": (_I, [ctypes.POINTER(Shape), _I, _I, _PP, _P, _I, _F, _F, _F,
                                            _I, _PP, _I, _PP, _F, _P, _SZ, _P]),
    "signmuon_newton_schulz_plan_bytes": (_SZ, [_I, _I]),
    "signmuon_newton_schulz_plan": (_I, [ctypes.POINTER(Shape), _I, _I, _PP, _P, _I, _PP, _I, _PP, _P, _SZ,
                                         _P, _SZ, _P]),
    "signmuon_newton_schulz_run": (_I, [_P, _I, _F, _F, _F, _F, _P]),
    "signmuon_sign_pack": (_I, [Shape, _I, _P, ctypes.c_int64, _I, _P, _P]),
    "signmuon_vote_workspace_bytes": (_SZ, [ctypes.POINTER(Shape), _I, _I]),
    "signmuon_spectral_workspace_bytes": (_SZ, [ctypes.POINTER(Shape), _I, _I]),
    "signmuon_spectral_norm": (_I, [ctypes.POINTER(Shape), _I, _I, _PP, _I, _P, _P, _SZ, _P]),
    "signmuon_momentum_norm_noalloc": (_I, [ctypes.POINTER(Shape), _I, _I, _I, _PP, _PP, _F, _PP, _P, _P]),
    "signmuon_vote_update": (_I, [ctypes.POINTER(Shape), _I, _I, _I, _PP, _I, _PP, _F, _PP, _P, _P,
                                  _P, _SZ, _P]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Loads libsignmuon.so from the package directory (raises if absent)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m sign_muon_optimizer_momentum_b200.build`"
                " (the Sign-Muon step has no non-CUDA implementation)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().signmuon_status_string(int(status)).decode()


def _check(name: str, status: int) -> None:
    if status != SIGNMUON_OK:
        raise SignMuonError(name, status)


def _shapes(shapes: Sequence[Tuple[int, int]]):
    arr = (Shape * len(shapes))()
    for i, (r, c) in enumerate(shapes):
        arr[i].rows, arr[i].cols = int(r), int(c)
    return arr


def _ptrs(ptrs):
    if ptrs is None:
        return None
    arr = (ctypes.c_void_p * len(ptrs))()
    for i, p in enumerate(ptrs):
        arr[i] = int(p) if p else None
    return arr


def signmuon_last_error_string() -> str:
    return load().signmuon_last_error_string().decode()


def signmuon_abi_version() -> int:
    return load().signmuon_abi_version()


def signmuon_x_ld(cols: int) -> int:
    return load().signmuon_x_ld(int(cols))


def signmuon_packed_words(shape: Tuple[int, int]) -> int:
    return load().signmuon_packed_words(Shape(int(shape[0]), int(shape[1])))


def signmuon_device_error(workspace: int, stream: int = 0) -> int:
    code = ctypes.c_uint32(0)
    _check("signmuon_device_error", load().signmuon_device_error(workspace, ctypes.byref(code), stream))
    return code.value


def signmuon_momentum_workspace_bytes(shapes, n_workers: int) -> int:
    return load().signmuon_momentum_workspace_bytes(_shapes(shapes), len(shapes), n_workers)


def signmuon_momentum_norm(shapes, n_workers, grad_dtype, grad, mom, beta, x_bf16, inv_norm,
                           workspace, ws_bytes, stream=0) -> None:
    st = load().signmuon_momentum_norm(_shapes(shapes), len(shapes), n_workers, grad_dtype, _ptrs(grad),
                                       _ptrs(mom), beta, _ptrs(x_bf16), inv_norm, workspace, ws_bytes,
                                       stream)
    _check("signmuon_momentum_norm", st)


def signmuon_spectral_workspace_bytes(shapes, n_workers: int) -> int:
    return load().signmuon_spectral_workspace_bytes(_shapes(shapes), len(shapes), n_workers)


def signmuon_spectral_norm(shapes, n_workers, x_bf16, iters, inv_norm, workspace, ws_bytes, stream=0) -> None:
    st = load().signmuon_spectral_norm(_shapes(shapes), len(shapes), n_workers, _ptrs(x_bf16), iters, inv_norm,
                                       workspace, ws_bytes, stream)
    _check("signmuon_spectral_norm", st)


def signmuon_momentum_sign(shapes, n_workers, grad_dtype, grad, mom, beta, int8_out, signs, inv_norm, workspace,
                           ws_bytes, stream=0) -> None:
    st = load().signmuon_momentum_sign(_shapes(shapes), len(shapes), n_workers, grad_dtype, _ptrs(grad),
                                       _ptrs(mom), beta, int(bool(int8_out)), _ptrs(signs), inv_norm, workspace,
                                       ws_bytes, stream)
    _check("signmuon_momentum_sign", st)


def signmuon_newton_schulz_workspace_bytes(shapes, n_workers: int, minimal: bool = False) -> int:
    return load().signmuon_newton_schulz_workspace_bytes(_shapes(shapes), len(shapes), n_workers,
                                                         int(bool(minimal)))


def signmuon_newton_schulz_batched(shapes, n_workers, x_bf16, inv_norm, k, a, b, c, out_mode, out,
                                   w_dtype, w, eta, workspace, ws_bytes, stream=0) -> None:
    st = load().signmuon_newton_schulz_batched(_shapes(shapes), len(shapes), n_workers, _ptrs(x_bf16),
                                               inv_norm, k, a, b, c, out_mode, _ptrs(out), w_dtype,
                                               _ptrs(w), eta, workspace, ws_bytes, stream)
    _check("signmuon_newton_schulz_batched", st)


def signmuon_newton_schulz_plan_bytes(n_mats: int, n_workers: int) -> int:
    return load().signmuon_newton_schulz_plan_bytes(n_mats, n_workers)


def signmuon_newton_schulz_plan(shapes, n_workers, x_bf16, inv_norm, out_mode, out, w_dtype, w,
                                workspace, ws_bytes, stream=0, plan=None):
    """Fills `plan` (a host buffer; a new one of the needed size when None)
    and returns it; pass it to signmuon_newton_schulz_run."""
    nbytes = signmuon_newton_schulz_plan_bytes(len(shapes), n_workers)
    if plan is None:
        plan = (ctypes.c_uint64 * max(1, -(-nbytes // 8)))()
    st = load().signmuon_newton_schulz_plan(_shapes(shapes), len(shapes), n_workers, _ptrs(x_bf16), inv_norm,
                                            out_mode, _ptrs(out), w_dtype, _ptrs(w), workspace, ws_bytes,
                                            ctypes.addressof(plan), ctypes.sizeof(plan), stream)
    _check("signmuon_newton_schulz_plan", st)
    return plan


def signmuon_newton_schulz_run(plan, k, a, b, c, eta, stream=0) -> None:
    st = load().signmuon_newton_schulz_run(ctypes.addressof(plan) if plan is not None else None, k, a, b, c,
                                           eta, stream)
    _check("signmuon_newton_schulz_run", st)


def signmuon_sign_pack(shape, u_dtype, u, ld_u, int8_out, out, stream=0) -> None:
    st = load().signmuon_sign_pack(Shape(int(shape[0]), int(shape[1])), u_dtype, u, ld_u,
                                   int(bool(int8_out)), out, stream)
    _check("signmuon_sign_pack", st)


def signmuon_vote_workspace_bytes(shapes, n_workers: int) -> int:
    return load().signmuon_vote_workspace_bytes(_shapes(shapes), len(shapes), n_workers)


def signmuon_vote_update(shapes, n_workers, int8_in, signs, w_dtype, w, eta, vote_bf16, nnz,
                         vote_inv_norm, workspace, ws_bytes, stream=0) -> None:
    st = load().signmuon_vote_update(_shapes(shapes), len(shapes), n_workers, int(bool(int8_in)),
                                     _ptrs(signs), w_dtype, _ptrs(w), eta, _ptrs(vote_bf16), nnz,
                                     vote_inv_norm, workspace, ws_bytes, stream)
    _check("signmuon_vote_update", st)


def signmuon_momentum_norm_noalloc(shapes, n_workers, grad_dtype, grad, mom, beta, x_bf16, inv_norm,
                                   stream=0) -> None:
    """Same as signmuon_momentum_norm with the scratch inside the library
    (for callers that cannot allocate device memory; see the header)."""
    st = load().signmuon_momentum_norm_noalloc(_shapes(shapes), len(shapes), n_workers, grad_dtype,
                                               _ptrs(grad), _ptrs(mom), beta, _ptrs(x_bf16), inv_norm,
                                               stream)
    _check("signmuon_momentum_norm_noalloc", st)
