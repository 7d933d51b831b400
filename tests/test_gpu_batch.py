"""Strided batches of one shape (ns_orthogonalize_strided, muon_step_strided):
the same kernels as the per-matrix lists, so the results are bit-equal to
them; the per-head workload (4096 matrices of 128 x 128) in one call."""
import numpy as np
import pytest

import workloads as wl
from gpu_env import context

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    return context()


@pytest.mark.parametrize("n,m,k", [(5, 96, 200), (3, 300, 160), (300, 128, 128)])
def test_ns_batch_equals_list(ctx, n, m, k):
    import torch
    X = torch.from_numpy(wl.gaussian(wl.rng_of("batch-ns", n, m, k), (n, m, k), 1.0)).cuda()
    out = ctx.ns_orthogonalize_batch(X)
    ref = ctx.ns_orthogonalize([X[i] for i in range(n)])
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    for i in range(n):
        assert torch.equal(out[i], ref[i]), i


def test_muon_batch_equals_list(ctx):
    import torch
    n, m, k = 7, 128, 384
    rng = wl.rng_of("batch-muon")
    W0 = torch.from_numpy(wl.gaussian(rng, (n, m, k), 0.02)).cuda()
    G = torch.from_numpy(wl.gaussian(rng, (n, m, k), 1e-3)).cuda()
    B0 = torch.from_numpy(wl.gaussian(rng, (n, m, k), 1e-3)).cuda()
    W1, B1 = W0.clone(), B0.clone()
    W2, B2 = [W0[i].clone() for i in range(n)], [B0[i].clone() for i in range(n)]
    flags = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    ctx.muon_step_batch(W1, G, B1, nonfinite=flags)
    ctx.muon_step(W2, [G[i] for i in range(n)], B2)
    torch.cuda.synchronize()
    assert (flags.cpu().numpy() == 0).all()
    for i in range(n):
        assert torch.equal(W1[i], W2[i]) and torch.equal(B1[i], B2[i]), i


def test_heads_batch_one_call(ctx):
    """4096 per-head matrices of 128 x 128 in one strided call agree bitwise
    with the same matrices passed as a list."""
    import torch
    n = 4096
    X = torch.randn(n, 128, 128, device="cuda", generator=torch.Generator(device="cuda").manual_seed(3))
    out = ctx.ns_orthogonalize_batch(X)
    ref = ctx.ns_orthogonalize(list(X.unbind(0)))
    torch.cuda.synchronize()
    assert torch.equal(out, torch.stack(ref))
