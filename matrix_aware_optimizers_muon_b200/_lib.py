"""ctypes declarations of the C ABI in ``include/mo.h``.

Pure argument marshalling: every computation happens in the CUDA library.
Loading fails loudly when ``libmo.so`` is missing; there is no fallback.
"""

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int32, c_int64, c_size_t, c_void_p

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmo.so")

MO_OK = 0
MO_ERR_INVALID_ARG = -1
MO_ERR_UNSUPPORTED = -2
MO_ERR_NO_WORKSPACE = -3
MO_ERR_CUDA = -4
MO_ERR_DEVICE = -5

OP_MUON, OP_SOAP, OP_NS = 0, 1, 2

# kernel kinds reported by mo_profile_read
KINDS = ["prep", "norm", "gram", "poly", "update", "apply", "soap_ew", "soap_rot", "soap_qr", "gemm",
         "soap_ema", "qr_chol", "qr_rowblock", "qr_trail", "ns_small", "tables"]


class MuonMat(ctypes.Structure):
    _fields_ = [("rows", c_int64), ("cols", c_int64), ("W", c_void_p), ("G", c_void_p),
                ("momentum", c_void_p)]


class MuonCfg(ctypes.Structure):
    _fields_ = [("lr", c_float), ("weight_decay", c_float), ("momentum", c_float),
                ("nesterov", c_int), ("momentum_ema", c_int), ("ns_steps", c_int),
                ("a", c_float), ("b", c_float), ("c", c_float), ("eps", c_float),
                ("adjust_lr", c_int), ("nonfinite", c_void_p)]


class NsCfg(ctypes.Structure):
    _fields_ = [("ns_steps", c_int), ("a", c_float), ("b", c_float), ("c", c_float),
                ("eps", c_float), ("nonfinite", c_void_p)]


class SoapMat(ctypes.Structure):
    _fields_ = [("rows", c_int64), ("cols", c_int64), ("W", c_void_p), ("G", c_void_p),
                ("M", c_void_p), ("V", c_void_p), ("L", c_void_p), ("QL", c_void_p),
                ("R", c_void_p), ("QR", c_void_p)]


class SoapCfg(ctypes.Structure):
    _fields_ = [("lr", c_float), ("beta1", c_float), ("beta2", c_float),
                ("shampoo_beta", c_float), ("eps", c_float), ("weight_decay", c_float),
                ("bias_correction", c_int), ("nonfinite", c_void_p), ("skip_refresh", c_int),
                ("damping", c_float)]


class SoapMuonMat(ctypes.Structure):
    _fields_ = [("rows", c_int64), ("cols", c_int64), ("W", c_void_p), ("G", c_void_p),
                ("B", c_void_p), ("V", c_void_p), ("L", c_void_p), ("QL", c_void_p),
                ("R", c_void_p), ("QR", c_void_p)]


class SoapMuonCfg(ctypes.Structure):
    _fields_ = [("lr", c_float), ("weight_decay", c_float), ("momentum", c_float),
                ("nesterov", c_int), ("beta2", c_float), ("shampoo_beta", c_float),
                ("eps", c_float), ("bias_correction", c_int), ("ns_steps", c_int),
                ("a", c_float), ("b", c_float), ("c", c_float), ("ns_eps", c_float),
                ("adjust_lr", c_int), ("damping", c_float), ("nonfinite", c_void_p),
                ("skip_refresh", c_int)]


class GemmDesc(ctypes.Structure):
    _fields_ = [("A", c_void_p), ("lda", c_int64), ("strideA", c_int64), ("a_mn", c_int),
                ("B", c_void_p), ("ldb", c_int64), ("strideB", c_int64), ("b_mn", c_int),
                ("M", c_int), ("N", c_int), ("K", c_int), ("batch", c_int), ("sym", c_int),
                ("alpha", c_float), ("beta", c_float),
                ("scale", c_void_p), ("alpha_pow", c_int), ("beta_pow", c_int),
                ("C", c_void_p), ("ldc", c_int64), ("strideC", c_int64), ("c_f32", c_int),
                ("D", c_void_p), ("ldd", c_int64), ("strideD", c_int64), ("d_f32", c_int),
                ("band", c_int)]


# name -> (restype, argtypes); every entry point declared in include/mo.h
SIGNATURES = {
    "mo_ctx_create": (c_int, [POINTER(c_void_p), c_int]),
    "mo_ctx_destroy": (None, [c_void_p]),
    "mo_last_error": (c_char_p, [c_void_p]),
    "mo_version": (c_char_p, []),
    "mo_workspace_bytes": (c_int, [c_void_p, c_int, POINTER(c_int64), POINTER(c_int64), c_int,
                                   POINTER(c_size_t), POINTER(c_size_t)]),
    "mo_set_workspace": (c_int, [c_void_p, c_void_p, c_size_t, c_void_p]),
    "mo_device_status": (c_int, [c_void_p, c_void_p, POINTER(c_int32)]),
    "muon_step": (c_int, [c_void_p, POINTER(MuonMat), c_int, POINTER(MuonCfg), c_void_p]),
    "ns_orthogonalize": (c_int, [c_void_p, POINTER(c_void_p), POINTER(c_void_p), POINTER(c_int64),
                                 POINTER(c_int64), c_int, POINTER(NsCfg), c_void_p]),
    "soap_step": (c_int, [c_void_p, POINTER(SoapMat), c_int, POINTER(SoapCfg), c_int64, c_void_p]),
    "mo_gemm_bf16": (c_int, [c_void_p, POINTER(GemmDesc), c_void_p]),
    "mo_soap_workspace_bytes": (c_int, [c_void_p, POINTER(SoapMat), c_int, POINTER(c_size_t)]),
    "soap_muon_step": (c_int, [c_void_p, POINTER(SoapMuonMat), c_int, POINTER(SoapMuonCfg), c_int64,
                               c_void_p]),
    "mo_soap_muon_workspace_bytes": (c_int, [c_void_p, POINTER(SoapMuonMat), c_int,
                                             POINTER(c_size_t)]),
    "ns_orthogonalize_static": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_int64,
                                        POINTER(NsCfg), c_void_p]),
    "ns_orthogonalize_strided": (c_int, [c_void_p, c_void_p, c_int64, c_void_p, c_int64, c_int64, c_int64,
                                         c_int, POINTER(NsCfg), c_void_p]),
    "muon_step_strided": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int,
                                  POINTER(MuonCfg), c_void_p]),
    "mo_profile_enable": (c_int, [c_void_p, c_int]),
    "mo_profile_read": (c_int, [c_void_p, POINTER(ctypes.c_double), POINTER(ctypes.c_double),
                                POINTER(c_int64), c_int]),
}

_lib = None


def load():
    """Load libmo.so once; raise if it is missing or lacks a symbol."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m matrix_aware_optimizers_muon_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)          # AttributeError if not exported
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
