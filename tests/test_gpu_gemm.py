"""The tcgen05 GEMM building block against float64 products of the same bf16
operands (kernel unit tests: operand majors, ragged tiles, batches, the
symmetric mirror and the fused epilogue)."""
import numpy as np
import pytest

from gpu_env import context

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    return context()


def _bf16(rng, shape, scale=1.0):
    import torch
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * scale)
    return x.to(torch.bfloat16)


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _pad(t, ld):
    import torch
    out = torch.zeros(t.shape[:-1] + (ld,), dtype=t.dtype)
    out[..., : t.shape[-1]] = t
    return out


def _check(D, ref, absprod, d_f32):
    # fp32 accumulation: |err| <= ~K u32 sum|a b|; bf16 output adds half an ulp
    D = _f64(D)
    tol = 1e-5 * absprod + (2.0 ** -8) * np.abs(ref) * (0 if d_f32 else 1) + 1e-30
    bad = np.abs(D - ref) > tol
    assert not bad.any(), (np.abs(D - ref)[bad].max(), int(bad.sum()))


CASES = [
    # M, N, K, batch, a_mn, b_mn
    (256, 512, 320, 1, 0, 0),
    (200, 300, 136, 2, 0, 0),
    (130, 70, 100, 3, 0, 0),
    (256, 384, 192, 1, 0, 1),
    (192, 256, 128, 2, 1, 0),
    (128, 520, 72, 1, 1, 1),
    (96, 96, 256, 5, 0, 1),
    (1, 64, 64, 2, 0, 0),
    # more than 128 rows and N > 128 (256-row tiles when CTA pairs are on)
    (300, 264, 200, 2, 1, 1),
    (640, 768, 512, 3, 0, 1),
    (520, 1000, 136, 1, 1, 0),
]


@pytest.mark.parametrize("M,N,K,batch,a_mn,b_mn", CASES)
@pytest.mark.parametrize("d_f32", [1, 0])
def test_gemm_majors_and_ragged(ctx, M, N, K, batch, a_mn, b_mn, d_f32):
    import torch
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    A = _bf16(rng, (batch, K, M) if a_mn else (batch, M, K))
    B = _bf16(rng, (batch, K, N) if b_mn else (batch, N, K))
    lda = (A.shape[-1] + 7) // 8 * 8
    ldb = (B.shape[-1] + 7) // 8 * 8
    Ap, Bp = _pad(A, lda).cuda(), _pad(B, ldb).cuda()
    ldd = (N + 7) // 8 * 8
    D = torch.zeros((batch, M, ldd), dtype=torch.float32 if d_f32 else torch.bfloat16, device="cuda")
    ctx.gemm_bf16(Ap, Bp, D, M=M, N=N, K=K, batch=batch, a_mn=bool(a_mn), b_mn=bool(b_mn),
                  lda=lda, ldb=ldb, ldd=ldd, strideA=Ap.shape[-2] * lda, strideB=Bp.shape[-2] * ldb,
                  strideD=M * ldd)
    torch.cuda.synchronize()
    a = _f64(A)
    b = _f64(B)
    a = np.swapaxes(a, 1, 2) if a_mn else a            # -> M x K
    b = b if b_mn else np.swapaxes(b, 1, 2)            # -> K x N
    ref = a @ b
    absprod = np.abs(a) @ np.abs(b)
    _check(D[..., :N].cpu(), ref, absprod, d_f32)
    assert ctx.device_status() == 0


@pytest.mark.parametrize("m,k", [(192, 320), (256, 256), (384, 136), (100, 64)])
def test_gemm_symmetric_mirror(ctx, m, k):
    import torch
    rng = np.random.default_rng(m + k)
    X = _bf16(rng, (2, m, k))
    ld = (k + 63) // 64 * 64
    Xp = _pad(X, ld).cuda()
    lda = (m + 63) // 64 * 64
    D = torch.full((2, m, lda), float("nan"), dtype=torch.bfloat16, device="cuda")
    ctx.gemm_bf16(Xp, Xp, D, M=m, N=m, K=k, batch=2, sym=True, lda=ld, ldb=ld, ldd=lda,
                  strideA=m * ld, strideB=m * ld, strideD=m * lda)
    torch.cuda.synchronize()
    out = D[..., :m].cpu()
    x = _f64(X)
    ref = x @ np.swapaxes(x, 1, 2)
    _check(out, ref, np.abs(x) @ np.abs(np.swapaxes(x, 1, 2)), 0)
    o = out.float().numpy()
    np.testing.assert_array_equal(o, np.swapaxes(o, 1, 2))   # bit-equal halves


def test_gemm_epilogue_alpha_beta_scale(ctx):
    import torch
    rng = np.random.default_rng(3)
    M, N, K, batch = 256, 256, 128, 3
    A = _bf16(rng, (batch, M, K))
    B = _bf16(rng, (batch, N, K))
    C = torch.from_numpy(rng.standard_normal((batch, M, N)).astype(np.float32))
    scale = torch.tensor([0.5, 2.0, -1.5], dtype=torch.float32)
    for c_f32, pw in ((1, 1), (0, 2)):
        Cd = (C if c_f32 else C.to(torch.bfloat16)).cuda()
        D = torch.zeros((batch, M, N), dtype=torch.float32, device="cuda")
        ctx.gemm_bf16(A.cuda(), B.cuda(), D, M=M, N=N, K=K, batch=batch, alpha=0.75, beta=-2.0,
                      C=Cd, scale=scale.cuda(), alpha_pow=pw, beta_pow=1)
        torch.cuda.synchronize()
        s = scale.numpy().astype(np.float64)[:, None, None]
        prod = _f64(A) @ np.swapaxes(_f64(B), 1, 2)
        ref = 0.75 * s ** pw * prod - 2.0 * s * _f64(Cd)
        assert np.abs(D.cpu().numpy() - ref).max() <= 1e-4 * np.abs(ref).max()


def test_gemm_in_place_fp32(ctx):
    # C aliases D (the in-place update form used by the SOAP apply)
    import torch
    rng = np.random.default_rng(4)
    M, N, K = 128, 256, 64
    A = _bf16(rng, (M, K)).cuda()
    B = _bf16(rng, (N, K)).cuda()
    W0 = torch.from_numpy(rng.standard_normal((M, N)).astype(np.float32))
    W = W0.clone().cuda()
    ctx.gemm_bf16(A, B, W, M=M, N=N, K=K, alpha=-0.1, beta=0.9, C=W)
    torch.cuda.synchronize()
    ref = -0.1 * (_f64(A.cpu()) @ _f64(B.cpu()).T) + 0.9 * W0.numpy()
    assert np.abs(W.cpu().numpy() - ref).max() <= 1e-5 * np.abs(ref).max()


BAND_CASES = [
    # M, N, K, batch, sym, band, b_mn, with C
    (1000, 1000, 192, 2, 1, 3, 0, 0),    # symmetric, ragged last band
    (904, 904, 256, 1, 1, 1, 0, 0),      # symmetric, one row tile per band
    (700, 520, 136, 1, 0, 2, 1, 1),      # MN-major B, C epilogue
    (640, 384, 128, 3, 0, 4, 0, 0),      # batch, last band of one row tile
]


@pytest.mark.parametrize("M,N,K,batch,sym,band,b_mn,with_c", BAND_CASES)
def test_gemm_banded_tile_order(ctx, M, N, K, batch, sym, band, b_mn, with_c):
    """Bands of row tiles (the order used when A overflows L2) give the same
    bits as the plain column order, and the right product."""
    import torch
    rng = np.random.default_rng(M + N + K + band)
    A = _bf16(rng, (batch, M, K))
    B = A if sym else _bf16(rng, (batch, K, N) if b_mn else (batch, N, K))
    C = _bf16(rng, (batch, M, N)).cuda() if with_c else None
    outs = []
    for bd in (0, band):
        D = torch.full((batch, M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        ctx.gemm_bf16(A.cuda(), B.cuda(), D, M=M, N=N, K=K, batch=batch, b_mn=bool(b_mn), sym=bool(sym),
                      alpha=1.0, beta=0.5 if with_c else 0.0, C=C, band=bd)
        torch.cuda.synchronize()
        outs.append(D.cpu())
    assert ctx.device_status() == 0
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    a = _f64(A)
    b = _f64(B) if b_mn else np.swapaxes(_f64(B), 1, 2)
    ref = a @ b + (0.5 * _f64(C.cpu()) if with_c else 0.0)
    _check(outs[1], ref, np.abs(a) @ np.abs(b) + (0.5 * np.abs(_f64(C.cpu())) if with_c else 0.0), 0)


@pytest.mark.parametrize("sym", [0, 1])
def test_gemm_band_chosen_for_large_panel(ctx, sym):
    """8192 x 8192 x 8192: the 128 MB A panel overflows L2 and the launcher
    takes bands; same bits as the column order forced with a band larger
    than the tile grid, and sampled rows against float64."""
    import torch
    n = 8192
    rng = np.random.default_rng(8192 + sym)
    A = (torch.randn(n, n, generator=torch.Generator().manual_seed(11 + sym)) * 0.02).to(torch.bfloat16)
    B = A if sym else (torch.randn(n, n, generator=torch.Generator().manual_seed(13)) * 0.02).to(torch.bfloat16)
    Ad, Bd = A.cuda(), B.cuda()
    outs = []
    for bd in (0, 1 << 20):
        D = torch.empty(n, n, dtype=torch.bfloat16, device="cuda")
        ctx.gemm_bf16(Ad, Bd, D, M=n, N=n, K=n, b_mn=not sym, sym=bool(sym), band=bd)
        torch.cuda.synchronize()
        outs.append(D)
    assert ctx.device_status() == 0
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    rows = np.sort(rng.choice(n, 6, replace=False))
    a = _f64(A[rows])
    b = _f64(B).T if sym else _f64(B)
    ref = a @ b
    _check(outs[0][rows].cpu(), ref, np.abs(a) @ np.abs(b), 0)
