"""ctypes declarations of libkronq.so (the C ABI in include/kronq.h).

The shared library is loaded from this package directory on first use; if it
is missing or stale that first call fails loudly -- there is no other
implementation to fall back to.  (Loading lazily lets the build module be
imported before the library exists.)
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkronq.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_NOT_PD, ERR_TIMEOUT = range(6)
BF16, F32 = 0, 1
BIIP_MODES = {"full": 0, "no_rescale": 1, "su_only": 2, "sv_only": 3}
U_GIVEN, ORDERED_FP32, WRITE_E, R_FORM = 1, 2, 4, 8

STATUS_NAMES = {0: "KRONQ_OK", 1: "KRONQ_ERR_INVALID_ARG", 2: "KRONQ_ERR_UNSUPPORTED",
                3: "KRONQ_ERR_CUDA", 4: "KRONQ_ERR_NOT_PD", 5: "KRONQ_ERR_TIMEOUT"}


class QuantParams(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group", ctypes.c_int), ("asym", ctypes.c_int),
                ("damp_rel", ctypes.c_float), ("block", ctypes.c_int), ("flags", ctypes.c_uint)]


class KronqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_vp, _i64, _int, _u64, _f32, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                     ctypes.c_uint64, ctypes.c_float, ctypes.c_size_t)
_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_ip = ctypes.POINTER(ctypes.c_int)
_qp = ctypes.POINTER(QuantParams)

# name -> (restype, argtypes)
SIGNATURES = {
    "kronq_accumulate_factors": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _int, _vp]),
    "kronq_sensitivity": (_int, [_vp, _i64, _vp, _i64, _dp, _vp, _sz, _vp]),
    "kronq_trace_tokens_workspace_bytes": (_sz, []),
    "kronq_trace_tokens": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _int, _vp, _sz, _vp]),
    "kronq_sensitivity_from_traces": (_int, [_vp, _dp, _vp]),
    "kronq_allocate_bits": (_int, [_dp, _i64p, _int, ctypes.c_double, _int, _int, _ip]),
    "kronq_allocate_topn_types": (_int, [_dp, _ip, _int, _int, _int, _int, _ip]),
    "kronq_biip_workspace_bytes": (_sz, [_i64, _i64]),
    "kronq_biip_forward": (_int, [_vp, _int, _vp, _i64, _i64, _vp, _vp, _u64, _f32, _int, _vp, _vp,
                                  _vp, _sz, _vp]),
    "kronq_biip_inverse": (_int, [_vp, _i64, _i64, _u64, _int, _vp, _vp, _vp, _sz, _vp]),
    "kronq_quantize_workspace_bytes": (_sz, [_i64, _i64, _qp]),
    "kronq_quantize_layer": (_int, [_vp, _vp, _i64, _i64, _qp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                    _vp]),
    "kronq_quantize_layer_static": (_int, [_vp, _vp, _i64, _i64, _qp, _vp, _vp, _vp, _vp, _vp,
                                           _vp]),
    "kronq_quantize_act_order_workspace_bytes": (_sz, [_i64, _i64, _qp]),
    "kronq_quantize_layer_act_order": (_int, [_vp, _vp, _i64, _i64, _qp, _vp, _vp, _vp, _vp, _vp,
                                              _vp, _vp, _vp, _sz, _vp]),
    "kronq_quantize_two_sided_workspace_bytes": (_sz, [_i64, _i64, _qp]),
    "kronq_quantize_two_sided": (_int, [_vp, _vp, _vp, _i64, _i64, _qp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _sz, _vp]),
    "kronq_pack": (_int, [_vp, _i64, _i64, _int, _vp, _vp]),
    "kronq_unpack": (_int, [_vp, _i64, _i64, _int, _vp, _vp]),
    "kronq_device_status": (_int, [_ip, _vp]),
    "kronq_wait_selftest": (_int, [_int, _u64, _vp, _sz, _vp]),
    "kronq_kfac_loss_workspace_bytes": (_sz, [_i64, _i64]),
    "kronq_kfac_loss": (_int, [_vp, _vp, _i64, _i64, _dp, _vp, _sz, _vp]),
    "kronq_kron_factors_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "kronq_kron_factors": (_int, [_vp, _vp, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _sz,
                                  _vp]),
    "kronq_decode_matvec_workspace_bytes": (_sz, [_i64, _i64]),
    "kronq_decode_matvec": (_int, [_vp, _vp, _vp, _i64, _i64, _int, _int, _u64, _int, _vp, _vp, _vp,
                                   _int, _vp, _vp, _sz, _vp]),
    "kronq_launch_count": (ctypes.c_uint64, []),
    "kronq_last_error": (ctypes.c_char_p, []),
    "kronq_version": (ctypes.c_char_p, []),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"libkronq.so not found at {path}; build it with "
            "`python -m post_quantization_kronq_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


class _LazyLib:
    """Loads libkronq.so at the first attribute access."""

    def __init__(self):
        self._lib = None

    def __getattr__(self, name):
        if self._lib is None:
            self._lib = load()
        return getattr(self._lib, name)


lib = _LazyLib()


def check(status: int) -> None:
    if status != OK:
        raise KronqError(status, lib.kronq_last_error().decode(errors="replace"))
