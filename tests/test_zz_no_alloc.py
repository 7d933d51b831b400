"""ns_orthogonalize_static, the entry point for callers that cannot allocate
device memory when they call it (their GPU memory belongs to another
allocator, their runtime forbids allocation after start-up, or they have no
allocator at hand): its scratch is a fixed device array inside the library.

It must give what ns_orthogonalize (the workspace path) gives on the same
input, on two calls in a row that share the array, and must refuse shapes
whose scratch would not fit.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

import workloads as wl
from gates import ns_gate
from gpu_env import context
from oracle import ns as ons

pytestmark = pytest.mark.gpu

QUINTIC = (3.4445, -4.7750, 2.0315)


def _static(ctx, x, y):
    import torch
    from matrix_aware_optimizers_muon_b200 import _lib
    cfg = _lib.NsCfg(5, QUINTIC[0], QUINTIC[1], QUINTIC[2], 1e-7, None)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctx.lib.ns_orthogonalize_static(ctx.handle, ctypes.c_void_p(x.data_ptr()),
                                           ctypes.c_void_p(y.data_ptr()), x.shape[0], x.shape[1],
                                           ctypes.byref(cfg), stream)


def test_static_scratch_matches_workspace_path():
    import torch
    ctx = context()
    rng = wl.rng_of("no-alloc")
    xs = [torch.from_numpy(wl.gaussian(rng, (256, 640), 1e-3)).cuda(),     # wide
          torch.from_numpy(wl.gaussian(rng, (700, 300), 1.0)).cuda()]      # tall, ragged
    refs = [ctx.ns_orthogonalize([x])[0] for x in xs]
    torch.cuda.synchronize()
    outs = [torch.full_like(x, float("nan")) for x in xs]
    # two calls in a row on one stream: the second reuses the array the first left behind
    for x, y in zip(xs, outs):
        assert _static(ctx, x, y) == 0, ctx.lib.mo_last_error(ctx.handle)
    torch.cuda.synchronize()
    for y, r in zip(outs, refs):
        a = y.cpu().numpy().astype(np.float64)
        b = r.cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all()
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-6)


def test_static_scratch_rejects_oversized_shapes():
    import torch
    from matrix_aware_optimizers_muon_b200 import _lib
    ctx = context()
    x = torch.zeros(2048, 4096, device="cuda")
    y = torch.empty_like(x)
    assert _static(ctx, x, y) == _lib.MO_ERR_UNSUPPORTED
    msg = ctx.lib.mo_last_error(ctx.handle).decode()
    assert "scratch" in msg and str(16 << 20) in msg


@pytest.mark.parametrize("m,n", [(96, 200), (200, 96), (5, 7)])
def test_static_small_shapes_against_oracle(m, n):
    """Shapes that the workspace path sends to its fused small-matrix kernel
    take the batched GEMM chain here (a single tile, K below 64, the TMA
    boxes mostly zero fill); gated against the fp64 oracle on the resolved
    subspace, with singular values in [0.6, 1.3], and against the noise
    floor of the oracle's bf16 emulation."""
    import torch
    ctx = context()
    G = wl.gaussian(wl.rng_of("no-alloc-small", m, n), (m, n), 1.0)
    x = torch.from_numpy(G).cuda()
    y = torch.full_like(x, float("nan"))
    assert _static(ctx, x, y) == 0, ctx.lib.mo_last_error(ctx.handle)
    torch.cuda.synchronize()
    O = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(O).all()
    ns_gate(G, O, ons.newton_schulz(G), ons.newton_schulz_bf16(G))


def test_static_status_word_readable_without_workspace():
    """A caller of the static entry point has no workspace: the status word
    of the fixed array is read (and cleared) by mo_device_status all the
    same, and the call leaves the caller's current device as it was."""
    import torch
    from matrix_aware_optimizers_muon_b200 import Context
    ctx = Context(0)                      # no workspace attached
    assert ctx.workspace is None
    dev_before = torch.cuda.current_device()
    x = torch.from_numpy(wl.gaussian(wl.rng_of("no-alloc-status"), (64, 96), 1.0)).cuda()
    y = torch.empty_like(x)
    assert _static(ctx, x, y) == 0, ctx.lib.mo_last_error(ctx.handle)
    assert torch.cuda.current_device() == dev_before
    assert ctx.device_status() == 0
