"""Matrix-aware optimizer steps (Muon, SOAP, Newton-Schulz) on NVIDIA B200.

A thin Python binding of the C ABI in ``include/mo.h``: it turns torch
tensors into device pointers and the current CUDA stream into a handle, and
allocates the workspace with torch.  Every step of the computation runs in the
sm_100a kernels of ``libmo.so``; when that library is missing, importing the
binding's entry points fails.
"""

import ctypes
from ctypes import byref, c_int32, c_int64, c_size_t, c_void_p

from . import _lib
from ._lib import (GemmDesc, MuonCfg, MuonMat, NsCfg, SoapCfg, SoapMat, SoapMuonCfg, SoapMuonMat,
                   OP_MUON, OP_NS, OP_SOAP)

__all__ = ["Context", "MoError", "QUINTIC", "OP_MUON", "OP_SOAP", "OP_NS"]

QUINTIC = (3.4445, -4.7750, 2.0315)


class MoError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"mo status {status}: {message}")
        self.status = status


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _check_f32(t, name):
    import torch
    if t is None:
        return
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")


def _check_state_shapes(i, d, keys):
    """Shapes of one SOAP / SOAP-Muon matrix's tensors: the library gets
    pointers only, so a mismatch here would address memory out of bounds."""
    W = d["W"]
    if W.dim() != 2:
        raise ValueError(f"matrix {i}: W must be 2-D")
    m, n = W.shape
    for k in keys:
        t = d.get(k)
        if t is not None and tuple(t.shape) != (m, n):
            raise ValueError(f"matrix {i}: {k} must have W's shape {(m, n)}")
    for fac, q, side in (("L", "QL", m), ("R", "QR", n)):
        for k in (fac, q):
            t = d.get(k)
            if t is not None and tuple(t.shape) != (side, side):
                raise ValueError(f"matrix {i}: {k} must be {side} x {side}")


def _check_extent(t, name, rows, cols, ld, stride, batch, dtypes):
    """A strided batch of rows x cols matrices (row stride ld, matrix stride
    stride, in elements) must lie inside the contiguous tensor t."""
    import torch
    if not t.is_cuda or not t.is_contiguous() or t.dtype not in dtypes:
        raise ValueError(f"{name} must be a contiguous CUDA tensor of dtype {dtypes}")
    if ld < cols:
        raise ValueError(f"{name}: leading dimension {ld} < row length {cols}")
    last = (batch - 1) * stride + (rows - 1) * ld + cols
    if rows > 0 and cols > 0 and last > t.numel():
        raise ValueError(f"{name}: the {batch} x {rows} x {cols} operand (ld {ld}, stride {stride}) "
                         f"needs {last} elements, the tensor has {t.numel()}")


class Context:
    """One library context on one CUDA device, with a torch-owned workspace."""

    def __init__(self, device=None):
        import torch
        self.lib = _lib.load()
        self.device = torch.cuda.current_device() if device is None else int(device)
        h = c_void_p()
        st = self.lib.mo_ctx_create(byref(h), self.device)
        if st != 0:
            raise MoError(st, "mo_ctx_create failed")
        self.handle = h
        self._workspace = None
        self.retired = []       # workspaces replaced during stream capture, kept alive
        self._batch_reserved = {}

    def close(self):
        if getattr(self, "handle", None):
            self.lib.mo_ctx_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------ workspace
    @property
    def workspace(self):
        """The attached workspace tensor (None when detached)."""
        return self._workspace

    @workspace.setter
    def workspace(self, value):
        """Only None may be assigned: it detaches the workspace in the library
        (reading its status word first) and drops the tensor.  Use
        attach_workspace() or reserve() to attach one."""
        if value is not None:
            raise ValueError("assign None to detach; use attach_workspace() or reserve() to attach")
        if self._workspace is not None:
            self._check(self.lib.mo_set_workspace(self.handle, None, 0, self._stream(None)))
            self._workspace = None
            self._batch_reserved.clear()

    # ------------------------------------------------------------ helpers
    def _stream(self, stream):
        import torch
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        return c_void_p(s.cuda_stream)

    def _check(self, st):
        if st != 0:
            raise MoError(st, self.lib.mo_last_error(self.handle).decode())

    def workspace_bytes(self, op, shapes):
        n = len(shapes)
        rows = (c_int64 * max(n, 1))(*[int(s[0]) for s in shapes])
        cols = (c_int64 * max(n, 1))(*[int(s[1]) for s in shapes])
        mn, full = c_size_t(), c_size_t()
        self._check(self.lib.mo_workspace_bytes(self.handle, op, rows, cols, n, byref(mn), byref(full)))
        return mn.value, full.value

    def attach_workspace(self, nbytes, stream=None):
        """Allocate ``nbytes`` of device memory with torch and attach it.

        Library work already enqueued may still use a workspace this one
        replaces, on any stream, and the switch itself copies the old status
        word on ``stream``.  Outside stream capture the device is synchronised
        before the old buffer goes back to torch's allocator.  During capture
        nothing can be synchronised: eager work enqueued before the capture
        may still be running, and the captured copy reads the old buffer
        whenever the graph replays.  So a buffer replaced during capture is
        kept alive (``retired``) until the next attach outside capture."""
        import torch
        buf = torch.empty(int(nbytes), dtype=torch.uint8, device=f"cuda:{self.device}")
        self._check(self.lib.mo_set_workspace(self.handle, c_void_p(buf.data_ptr()), buf.numel(),
                                              self._stream(stream)))
        old, self._workspace = self._workspace, buf
        if old is not None:
            if torch.cuda.is_current_stream_capturing():
                self.retired.append(old)
            else:
                torch.cuda.synchronize(self.device)
                self.retired.clear()
        del old
        return buf

    def reserve(self, op, shapes, full=True, stream=None):
        """Make sure the attached workspace fits ``op`` on ``shapes``."""
        mn, fb = self.workspace_bytes(op, shapes)
        need = fb if full else mn
        if self.workspace is None or self.workspace.numel() < need:
            self.attach_workspace(need, stream)

    def device_status(self, stream=None):
        v = c_int32()
        st = self.lib.mo_device_status(self.handle, self._stream(stream), byref(v))
        if st not in (0, _lib.MO_ERR_DEVICE):
            self._check(st)
        return v.value

    def profile(self, enable=True):
        self._check(self.lib.mo_profile_enable(self.handle, int(enable)))

    def profile_read(self):
        """{kind: (ms, executed_flops, launches)} since the last read."""
        n = len(_lib.KINDS)
        ms = (ctypes.c_double * n)()
        fl = (ctypes.c_double * n)()
        ln = (c_int64 * n)()
        self._check(self.lib.mo_profile_read(self.handle, ms, fl, ln, n))
        return {k: (ms[i], fl[i], ln[i]) for i, k in enumerate(_lib.KINDS)}

    # ------------------------------------------------------------ entry points
    def muon_step(self, W, G, B, *, lr=0.02, weight_decay=0.01, momentum=0.95, nesterov=True,
                  momentum_ema=False, ns_steps=5, coeffs=QUINTIC, eps=1e-7,
                  adjust_lr="match_rms_adamw", nonfinite=None, stream=None, reserve=True):
        """One Muon step on lists of fp32 CUDA matrices (G entries may be None)."""
        n = len(W)
        if not (len(G) == len(B) == n):
            raise ValueError("W, G and B must have the same length")
        mats = (MuonMat * max(n, 1))()
        for i in range(n):
            for t, nm in ((W[i], "W"), (G[i], "G"), (B[i], "momentum")):
                _check_f32(t, f"{nm}[{i}]")
            if W[i].dim() != 2 or (G[i] is not None and G[i].shape != W[i].shape) or B[i].shape != W[i].shape:
                raise ValueError(f"matrix {i}: W, G and momentum must be 2-D with one shape")
            mats[i] = MuonMat(W[i].shape[0], W[i].shape[1], _ptr(W[i]), _ptr(G[i]), _ptr(B[i]))
        if reserve:
            self.reserve(OP_MUON, [tuple(w.shape) for w in W], stream=stream)
        modes = {"match_rms_adamw": 0, "original": 1}
        cfg = MuonCfg(lr, weight_decay, momentum, int(nesterov), int(momentum_ema), ns_steps,
                      coeffs[0], coeffs[1], coeffs[2], eps, modes[adjust_lr],
                      _ptr(nonfinite))
        self._check(self.lib.muon_step(self.handle, mats, n, byref(cfg), self._stream(stream)))

    def ns_orthogonalize(self, inputs, outputs=None, *, ns_steps=5, coeffs=QUINTIC, eps=1e-7,
                         nonfinite=None, stream=None, reserve=True):
        """O_i = NS(in_i); returns the list of fp32 outputs."""
        import torch
        n = len(inputs)
        if outputs is None:
            outputs = [torch.empty_like(x) for x in inputs]
        ins = (c_void_p * max(n, 1))()
        outs = (c_void_p * max(n, 1))()
        rows = (c_int64 * max(n, 1))()
        cols = (c_int64 * max(n, 1))()
        for i, (x, y) in enumerate(zip(inputs, outputs)):
            _check_f32(x, f"in[{i}]")
            _check_f32(y, f"out[{i}]")
            if x.dim() != 2 or y.shape != x.shape:
                raise ValueError(f"matrix {i}: input and output must be 2-D with one shape")
            ins[i], outs[i] = x.data_ptr(), y.data_ptr()
            rows[i], cols[i] = x.shape
        if reserve:
            self.reserve(OP_NS, [tuple(x.shape) for x in inputs], stream=stream)
        cfg = NsCfg(ns_steps, coeffs[0], coeffs[1], coeffs[2], eps, _ptr(nonfinite))
        self._check(self.lib.ns_orthogonalize(self.handle, ins, outs, rows, cols, n, byref(cfg),
                                              self._stream(stream)))
        return outputs

    def _reserve_batch(self, op, rows, cols, n, stream):
        """reserve() for n matrices of one shape, remembered per workspace so
        that repeated calls on the same batch cost no workspace query."""
        key = (op, rows, cols, n)
        if self.workspace is not None and self._batch_reserved.get(key) == self.workspace.data_ptr():
            return
        self.reserve(op, [(rows, cols)] * n, stream=stream)
        self._batch_reserved[key] = self.workspace.data_ptr()

    @staticmethod
    def _check_batch(t, name, shape=None):
        _check_f32(t, name)
        if t.dim() != 3 or (shape is not None and tuple(t.shape) != tuple(shape)):
            raise ValueError(f"{name} must be a 3-D [n, rows, cols] tensor" +
                             (f" of shape {tuple(shape)}" if shape is not None else ""))

    def ns_orthogonalize_batch(self, X, out=None, *, ns_steps=5, coeffs=QUINTIC, eps=1e-7, nonfinite=None,
                               stream=None, reserve=True):
        """out[i] = NS(X[i]) for a contiguous fp32 tensor X of shape [n, rows,
        cols] (e.g. per-head matrices): one call whatever n is."""
        import torch
        self._check_batch(X, "X")
        if out is None:
            out = torch.empty_like(X)
        self._check_batch(out, "out", X.shape)
        n, r, c = X.shape
        if reserve:
            self._reserve_batch(OP_NS, r, c, n, stream)
        cfg = NsCfg(ns_steps, coeffs[0], coeffs[1], coeffs[2], eps, _ptr(nonfinite))
        self._check(self.lib.ns_orthogonalize_strided(self.handle, _ptr(X), r * c, _ptr(out), r * c, r, c, n,
                                                      byref(cfg), self._stream(stream)))
        return out

    def muon_step_batch(self, W, G, B, *, lr=0.02, weight_decay=0.01, momentum=0.95, nesterov=True,
                        momentum_ema=False, ns_steps=5, coeffs=QUINTIC, eps=1e-7,
                        adjust_lr="match_rms_adamw", nonfinite=None, stream=None, reserve=True):
        """One Muon step on n matrices of one shape held as contiguous fp32
        [n, rows, cols] tensors W, G and B."""
        self._check_batch(W, "W")
        self._check_batch(G, "G", W.shape)
        self._check_batch(B, "B", W.shape)
        n, r, c = W.shape
        if reserve:
            self._reserve_batch(OP_MUON, r, c, n, stream)
        modes = {"match_rms_adamw": 0, "original": 1}
        cfg = MuonCfg(lr, weight_decay, momentum, int(nesterov), int(momentum_ema), ns_steps,
                      coeffs[0], coeffs[1], coeffs[2], eps, modes[adjust_lr], _ptr(nonfinite))
        self._check(self.lib.muon_step_strided(self.handle, _ptr(W), _ptr(G), _ptr(B), r * c, r, c, n,
                                               byref(cfg), self._stream(stream)))

    def soap_step(self, mats, step, *, lr=3e-3, beta1=0.95, beta2=0.95, shampoo_beta=None,
                  eps=1e-8, weight_decay=0.0, bias_correction=True, nonfinite=None, stream=None,
                  reserve=True, refresh=True, damping=0.0):
        """One SOAP step.  ``mats`` is a list of dicts with keys W, G, M, V and
        optionally L, QL, R, QR (missing or None: identity basis on that side).
        ``refresh=False`` keeps the bases this step (factors still update).
        ``damping``: 0 is the pages' power step qr(L Q); a positive value
        runs it on L + damping * trace(L) I instead (an option)."""
        n = len(mats)
        arr = (SoapMat * max(n, 1))()
        for i, d in enumerate(mats):
            for k in ("W", "G", "M", "V", "L", "QL", "R", "QR"):
                _check_f32(d.get(k), f"{k}[{i}]")
            _check_state_shapes(i, d, ("G", "M", "V"))
            W = d["W"]
            arr[i] = SoapMat(W.shape[0], W.shape[1], _ptr(W), _ptr(d.get("G")), _ptr(d["M"]),
                             _ptr(d["V"]), _ptr(d.get("L")), _ptr(d.get("QL")), _ptr(d.get("R")),
                             _ptr(d.get("QR")))
        if reserve:
            need = c_size_t()
            self._check(self.lib.mo_soap_workspace_bytes(self.handle, arr, n, byref(need)))
            if self.workspace is None or self.workspace.numel() < need.value:
                self.attach_workspace(need.value, stream)
        sb = beta2 if shampoo_beta is None else shampoo_beta
        cfg = SoapCfg(lr, beta1, beta2, sb, eps, weight_decay, int(bias_correction), _ptr(nonfinite),
                      0 if refresh else 1, damping)
        self._check(self.lib.soap_step(self.handle, arr, n, byref(cfg), int(step), self._stream(stream)))

    def soap_muon_step(self, mats, step, *, lr=0.02, weight_decay=0.01, momentum=0.95, nesterov=True,
                       beta2=0.95, shampoo_beta=0.9, eps=1e-8, bias_correction=True, ns_steps=5,
                       coeffs=QUINTIC, ns_eps=1e-7, adjust_lr="match_rms_adamw", damping=0.0,
                       nonfinite=None, refresh=True, stream=None, reserve=True):
        """One SOAP-Muon step.  ``mats``: dicts with W, G, B (Muon momentum), V
        and optionally L, QL, R, QR (missing or None: identity basis)."""
        n = len(mats)
        arr = (SoapMuonMat * max(n, 1))()
        for i, d in enumerate(mats):
            for k in ("W", "G", "B", "V", "L", "QL", "R", "QR"):
                _check_f32(d.get(k), f"{k}[{i}]")
            _check_state_shapes(i, d, ("G", "B", "V"))
            W = d["W"]
            arr[i] = SoapMuonMat(W.shape[0], W.shape[1], _ptr(W), _ptr(d.get("G")), _ptr(d["B"]),
                                 _ptr(d["V"]), _ptr(d.get("L")), _ptr(d.get("QL")), _ptr(d.get("R")),
                                 _ptr(d.get("QR")))
        if reserve:
            need = c_size_t()
            self._check(self.lib.mo_soap_muon_workspace_bytes(self.handle, arr, n, byref(need)))
            if self.workspace is None or self.workspace.numel() < need.value:
                self.attach_workspace(need.value, stream)
        modes = {"match_rms_adamw": 0, "original": 1}
        cfg = SoapMuonCfg(lr, weight_decay, momentum, int(nesterov), beta2, shampoo_beta, eps,
                          int(bias_correction), ns_steps, coeffs[0], coeffs[1], coeffs[2], ns_eps,
                          modes[adjust_lr], damping, _ptr(nonfinite), 0 if refresh else 1)
        self._check(self.lib.soap_muon_step(self.handle, arr, n, byref(cfg), int(step),
                                            self._stream(stream)))

    def gemm_bf16(self, A, B, D, *, M, N, K, batch=1, a_mn=False, b_mn=False, sym=False,
                  alpha=1.0, beta=0.0, C=None, scale=None, alpha_pow=0, beta_pow=0,
                  lda=None, ldb=None, ldc=None, ldd=None, strideA=None, strideB=None,
                  strideC=None, strideD=None, band=0, stream=None):
        """Batched bf16 tensor-core GEMM with the fused epilogue (see mo.h)."""
        import torch

        def ld_of(t):
            return t.shape[-1]

        def stride_of(t):
            return t.shape[-1] * t.shape[-2] if t.dim() == 3 else 0

        d = GemmDesc()
        d.A, d.lda, d.strideA, d.a_mn = A.data_ptr(), lda or ld_of(A), strideA or stride_of(A), int(a_mn)
        d.B, d.ldb, d.strideB, d.b_mn = B.data_ptr(), ldb or ld_of(B), strideB or stride_of(B), int(b_mn)
        d.M, d.N, d.K, d.batch, d.sym = M, N, K, batch, int(sym)
        d.alpha, d.beta = alpha, beta
        d.scale = None if scale is None else scale.data_ptr()
        d.alpha_pow, d.beta_pow = alpha_pow, beta_pow
        if C is not None:
            d.C, d.ldc, d.strideC = C.data_ptr(), ldc or ld_of(C), strideC or stride_of(C)
            d.c_f32 = int(C.dtype == torch.float32)
        d.D, d.ldd, d.strideD = D.data_ptr(), ldd or ld_of(D), strideD or stride_of(D)
        d.d_f32 = int(D.dtype == torch.float32)
        d.band = band
        bf16, outs = (torch.bfloat16,), (torch.bfloat16, torch.float32)
        _check_extent(A, "A", K if a_mn else M, M if a_mn else K, d.lda, d.strideA, batch, bf16)
        _check_extent(B, "B", K if b_mn else N, N if b_mn else K, d.ldb, d.strideB, batch, bf16)
        _check_extent(D, "D", M, N, d.ldd, d.strideD, batch, outs)
        if C is not None:
            _check_extent(C, "C", M, N, d.ldc, d.strideC, batch, outs)
        if self.workspace is None:
            self.attach_workspace(4096, stream)
        self._check(self.lib.mo_gemm_bf16(self.handle, byref(d), self._stream(stream)))
