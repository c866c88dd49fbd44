"""ctypes declarations of the C ABI in include/octopus.h (argument marshalling only).

Loading fails loudly when the compiled library is missing: there is no
Python or CPU fallback for any step of the codec.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboctopus_b200.so")

OCTO_OK, OCTO_EINVAL, OCTO_EUNSUPPORTED, OCTO_ECUDA, OCTO_EWORKSPACE = 0, -1, -2, -3, -4
ROUND_SCALAR, ROUND_JOINT = 0, 1
F32, BF16 = 0, 1


class OctoLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("d", "b", "T", "b_dir", "b_rho", "code_bits", "words", "n_dir", "n_rho",
                 "qjl", "qjl_words", "rounding")]


class OctoTables(ctypes.Structure):
    _fields_ = [("dir_c", ctypes.c_void_p), ("dir_t", ctypes.c_void_p), ("rho_c", ctypes.c_void_p),
                ("rho_t", ctypes.c_void_p), ("signs", ctypes.c_void_p), ("qjl_S", ctypes.c_void_p),
                ("n_heads", ctypes.c_int64)]


class OctoError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


_lib = None

# name -> (restype, argtypes)
_SIGS = {
    "octo_layout_init": (ctypes.c_int, [ctypes.POINTER(OctoLayout), ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "octo_layout_init_delta": (ctypes.c_int, [ctypes.POINTER(OctoLayout), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int]),
    "octo_codebook_build": (ctypes.c_int, [ctypes.POINTER(OctoLayout)] + [ctypes.c_void_p] * 4),
    "octo_rotation_build": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p]),
    "octo_qjl_build": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p]),
    "octo_encode": (ctypes.c_int, [ctypes.POINTER(OctoLayout), ctypes.POINTER(OctoTables), ctypes.c_void_p, ctypes.c_int,
                                   ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p]),
    "octo_decode_attn_workspace": (ctypes.c_size_t, [ctypes.POINTER(OctoLayout), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                     ctypes.c_int, ctypes.c_int64]),
    "octo_decode_attn": (ctypes.c_int, [ctypes.POINTER(OctoLayout), ctypes.POINTER(OctoTables), ctypes.c_void_p, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "octo_decode_attn_static": (ctypes.c_int, [ctypes.POINTER(OctoLayout), ctypes.POINTER(OctoTables), ctypes.c_void_p,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int64, ctypes.c_int64,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p]),
    "octo_decode_attn_static_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]),
    "octo_decode_attn_static_fill": (ctypes.c_int, [ctypes.c_int, ctypes.c_void_p]),
    "octo_dequant": (ctypes.c_int, [ctypes.POINTER(OctoLayout), ctypes.POINTER(OctoTables), ctypes.c_int64, ctypes.c_int64,
                                    ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_int, ctypes.c_void_p]),
    "octo_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "octo_abi_version": (ctypes.c_int, []),
}


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m rotation_preconditioned_quantization_b200.build` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def status_string(status: int) -> str:
    try:
        return lib().octo_status_string(int(status)).decode()
    except Exception:  # pragma: no cover - library missing
        return "unknown"


def check(status: int, what: str) -> None:
    if status != OCTO_OK:
        raise OctoError(status, what)
