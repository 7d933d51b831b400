"""The C-ABI library: it loads, exports every entry point that include/mo.h
declares, and rejects bad arguments on the host before touching a GPU."""
import ctypes
import os
import re

import pytest

from matrix_aware_optimizers_muon_b200 import _lib
from matrix_aware_optimizers_muon_b200 import build as mo_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    mo_build.build()
    return _lib.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "mo.h")).read()
    return sorted(set(re.findall(r"MO_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("muon_step", "soap_step", "ns_orthogonalize", "mo_workspace_bytes",
              "mo_set_workspace", "mo_ctx_create", "mo_gemm_bf16"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, name


def _ctx(lib):
    h = ctypes.c_void_p()
    assert lib.mo_ctx_create(ctypes.byref(h), 0) == 0
    return h


def test_context_and_version(lib):
    h = _ctx(lib)
    assert b"sm_100a" in lib.mo_version()
    assert lib.mo_last_error(h) == b""
    assert lib.mo_ctx_create(None, 0) == _lib.MO_ERR_INVALID_ARG
    lib.mo_ctx_destroy(h)


def test_workspace_sizes(lib):
    h = _ctx(lib)
    rows = (ctypes.c_int64 * 3)(256, 512, 512)
    cols = (ctypes.c_int64 * 3)(512, 256, 1024)
    mn, full = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.mo_workspace_bytes(h, 0, rows, cols, 3, ctypes.byref(mn), ctypes.byref(full)) == 0
    # two 256x512 matrices share a bucket: X0, X1 (bf16 256x512), A, P (bf16 256x256)
    per = 2 * 256 * 512 * 2 + 2 * 256 * 256 * 2
    assert mn.value >= per and full.value >= 2 * per
    assert lib.mo_workspace_bytes(h, 7, rows, cols, 3, None, None) == _lib.MO_ERR_INVALID_ARG
    bad = (ctypes.c_int64 * 1)(0)
    assert lib.mo_workspace_bytes(h, 0, bad, cols, 1, None, None) == _lib.MO_ERR_INVALID_ARG
    lib.mo_ctx_destroy(h)


def _muon_cfg(**kw):
    c = _lib.MuonCfg(0.02, 0.01, 0.95, 1, 0, 5, 3.4445, -4.7750, 2.0315, 1e-7, 0, None)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value", [("lr", -1.0), ("momentum", 1.0), ("ns_steps", 0),
                                         ("ns_steps", 65), ("eps", float("nan")), ("adjust_lr", 2),
                                         ("a", float("inf"))])
def test_muon_rejects_bad_hyperparameters(lib, field, value):
    h = _ctx(lib)
    mats = (_lib.MuonMat * 1)(_lib.MuonMat(4, 4, 16, 16, 16))
    cfg = _muon_cfg(**{field: value})
    assert lib.muon_step(h, mats, 1, ctypes.byref(cfg), None) == _lib.MO_ERR_INVALID_ARG
    assert lib.mo_last_error(h) != b""
    lib.mo_ctx_destroy(h)


def test_muon_rejects_bad_matrices(lib):
    h = _ctx(lib)
    cfg = _muon_cfg()
    for m in (_lib.MuonMat(0, 4, 16, 16, 16), _lib.MuonMat(4, 4, None, 16, 16),
              _lib.MuonMat(4, 4, 16, 16, None), _lib.MuonMat(4, 4, 18, 16, 16)):
        mats = (_lib.MuonMat * 1)(m)
        assert lib.muon_step(h, mats, 1, ctypes.byref(cfg), None) == _lib.MO_ERR_INVALID_ARG
    assert lib.muon_step(h, None, 1, ctypes.byref(cfg), None) == _lib.MO_ERR_INVALID_ARG
    assert lib.muon_step(h, None, 0, ctypes.byref(cfg), None) == 0      # nothing to do
    # a skipped matrix (G == NULL) needs nothing at all
    mats = (_lib.MuonMat * 1)(_lib.MuonMat(4, 4, 16, None, 16))
    assert lib.muon_step(h, mats, 1, ctypes.byref(cfg), None) == 0
    # valid request without a workspace
    mats = (_lib.MuonMat * 1)(_lib.MuonMat(4, 4, 16, 16, 16))
    assert lib.muon_step(h, mats, 1, ctypes.byref(cfg), None) == _lib.MO_ERR_NO_WORKSPACE
    lib.mo_ctx_destroy(h)


def test_ns_rejects_overlap_and_nulls(lib):
    h = _ctx(lib)
    cfg = _lib.NsCfg(5, 3.4445, -4.7750, 2.0315, 1e-7, None)
    ins = (ctypes.c_void_p * 1)(4096)
    outs = (ctypes.c_void_p * 1)(4096 + 32)
    rows = (ctypes.c_int64 * 1)(4)
    cols = (ctypes.c_int64 * 1)(4)
    assert lib.ns_orthogonalize(h, ins, outs, rows, cols, 1, ctypes.byref(cfg), None) == _lib.MO_ERR_INVALID_ARG
    outs[0] = None
    assert lib.ns_orthogonalize(h, ins, outs, rows, cols, 1, ctypes.byref(cfg), None) == _lib.MO_ERR_INVALID_ARG
    lib.mo_ctx_destroy(h)


def test_soap_rejects_bad_arguments(lib):
    h = _ctx(lib)
    cfg = _lib.SoapCfg(3e-3, 0.95, 0.95, 0.95, 1e-8, 0.0, 1, None, 0, 0.0)
    good = _lib.SoapMat(8, 8, 16, 16, 16, 16, 16, 16, None, None)
    mats = (_lib.SoapMat * 1)(good)
    assert lib.soap_step(h, mats, 1, ctypes.byref(cfg), 0, None) == _lib.MO_ERR_INVALID_ARG
    half = _lib.SoapMat(8, 8, 16, 16, 16, 16, 16, None, None, None)
    mats = (_lib.SoapMat * 1)(half)
    assert lib.soap_step(h, mats, 1, ctypes.byref(cfg), 1, None) == _lib.MO_ERR_INVALID_ARG
    bad_cfg = _lib.SoapCfg(3e-3, 1.0, 0.95, 0.95, 1e-8, 0.0, 1, None, 0, 0.0)
    mats = (_lib.SoapMat * 1)(good)
    assert lib.soap_step(h, mats, 1, ctypes.byref(bad_cfg), 1, None) == _lib.MO_ERR_INVALID_ARG
    # damping 0 is the pages' undamped power step (valid); negative, above
    # 1e-2 or NaN is refused
    for damping in (-1e-5, 0.5, float("nan")):
        bad_cfg = _lib.SoapCfg(3e-3, 0.95, 0.95, 0.95, 1e-8, 0.0, 1, None, 0, damping)
        assert lib.soap_step(h, mats, 1, ctypes.byref(bad_cfg), 1, None) == _lib.MO_ERR_INVALID_ARG
        assert b"damping" in lib.mo_last_error(h)
    lib.mo_ctx_destroy(h)


def test_gemm_rejects_misaligned(lib):
    h = _ctx(lib)
    d = _lib.GemmDesc()
    d.A, d.lda, d.B, d.ldb, d.D, d.ldd = 16, 12, 16, 16, 16, 16
    d.M = d.N = d.K = d.batch = 16
    assert lib.mo_gemm_bf16(h, ctypes.byref(d), None) == _lib.MO_ERR_INVALID_ARG
    d.lda = 16
    d.sym, d.N = 1, 32
    assert lib.mo_gemm_bf16(h, ctypes.byref(d), None) == _lib.MO_ERR_INVALID_ARG
    d.sym, d.N, d.band = 0, 16, -1
    assert lib.mo_gemm_bf16(h, ctypes.byref(d), None) == _lib.MO_ERR_INVALID_ARG
    assert b"band" in lib.mo_last_error(h)
    lib.mo_ctx_destroy(h)


def test_soap_muon_rejects_bad_arguments(lib):
    h = _ctx(lib)
    good = _lib.SoapMuonMat(8, 8, 16, 16, 16, 16, 16, 16, None, None)
    mats = (_lib.SoapMuonMat * 1)(good)

    def cfg(**kw):
        base = dict(lr=0.02, weight_decay=0.01, momentum=0.95, nesterov=1, beta2=0.95,
                    shampoo_beta=0.9, eps=1e-8, bias_correction=1, ns_steps=5, a=3.4445,
                    b=-4.7750, c=2.0315, ns_eps=1e-7, adjust_lr=0, damping=0.0,
                    nonfinite=None, skip_refresh=0)
        base.update(kw)
        return _lib.SoapMuonCfg(**base)

    for bad in (dict(momentum=1.0), dict(adjust_lr=2), dict(ns_steps=0), dict(damping=-1e-5),
                dict(beta2=1.0), dict(lr=float("nan"))):
        assert lib.soap_muon_step(h, mats, 1, ctypes.byref(cfg(**bad)), 1, None) == _lib.MO_ERR_INVALID_ARG, bad
        assert lib.mo_last_error(h).startswith(b"soap_muon_step")
    assert lib.soap_muon_step(h, mats, 1, ctypes.byref(cfg()), 0, None) == _lib.MO_ERR_INVALID_ARG
    half = _lib.SoapMuonMat(8, 8, 16, 16, 16, 16, 16, None, None, None)
    mats = (_lib.SoapMuonMat * 1)(half)
    assert lib.soap_muon_step(h, mats, 1, ctypes.byref(cfg()), 1, None) == _lib.MO_ERR_INVALID_ARG
    size = ctypes.c_size_t()
    mats = (_lib.SoapMuonMat * 1)(good)
    assert lib.mo_soap_muon_workspace_bytes(h, mats, 1, ctypes.byref(size)) == 0
    plain = ctypes.c_size_t()
    smats = (_lib.SoapMat * 1)(_lib.SoapMat(8, 8, 16, 16, 16, 16, 16, 16, None, None))
    assert lib.mo_soap_workspace_bytes(h, smats, 1, ctypes.byref(plain)) == 0
    assert size.value > plain.value          # P and the Newton-Schulz scratch on top
    lib.mo_ctx_destroy(h)


def test_strided_batches_validate(lib):
    h = _ctx(lib)
    cfg = _lib.NsCfg(5, 3.4445, -4.7750, 2.0315, 1e-7, None)
    # a stride below rows * cols would overlap the matrices
    assert lib.ns_orthogonalize_strided(h, 16, 100, 4096, 100, 10, 20, 3, ctypes.byref(cfg), None) == \
        _lib.MO_ERR_INVALID_ARG
    assert b"stride" in lib.mo_last_error(h)
    # well formed, but no workspace attached: refused before any launch
    assert lib.ns_orthogonalize_strided(h, 16, 200, 1 << 20, 200, 10, 20, 3, ctypes.byref(cfg), None) == \
        _lib.MO_ERR_NO_WORKSPACE
    mcfg = _lib.MuonCfg(0.02, 0.01, 0.95, 1, 0, 5, 3.4445, -4.7750, 2.0315, 1e-7, 0, None)
    assert lib.muon_step_strided(h, 16, 16, 16, 10, 4, 4, 2, ctypes.byref(mcfg), None) == _lib.MO_ERR_INVALID_ARG
    assert lib.muon_step_strided(h, 16, 1 << 20, 1 << 21, 16, 4, 4, 2, ctypes.byref(mcfg), None) == \
        _lib.MO_ERR_NO_WORKSPACE
    lib.mo_ctx_destroy(h)


def test_detach_without_workspace_is_a_no_op(lib):
    h = _ctx(lib)
    assert lib.mo_set_workspace(h, None, 0, None) == 0
    assert lib.mo_set_workspace(h, None, 64, None) == _lib.MO_ERR_INVALID_ARG
    lib.mo_ctx_destroy(h)
