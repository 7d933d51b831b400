"""Muon and Newton-Schulz parity: the CUDA path through the C ABI against the
fp64 oracle (and its bf16-emulation mode) on the same seeded inputs."""
import numpy as np
import pytest

import workloads as wl
from gates import ns_gate, rel
from gpu_env import context
from oracle import muon as omuon
from oracle import ns as ons

pytestmark = pytest.mark.gpu

LR, WD, BETA = 0.02, 0.01, 0.95


@pytest.fixture(scope="module")
def ctx():
    return context()


def _cuda(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _np(t):
    return t.detach().cpu().numpy().astype(np.float64)


def run_gpu_muon(ctx, Ws, Gs, Bs, **kw):
    import torch
    W = [_cuda(w) for w in Ws]
    G = [None if g is None else _cuda(g) for g in Gs]
    B = [_cuda(b) for b in Bs]
    flags = torch.full((len(Ws),), -1, dtype=torch.int32, device="cuda")
    ctx.muon_step(W, G, B, nonfinite=flags, **kw)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    return [_np(w) for w in W], [_np(b) for b in B], flags.cpu().numpy()


def check_muon(W0, G, B0, Wg, Bg, lr=LR, wd=WD, beta=BETA, **kw):
    ref = omuon.muon_step(W0, G, B0, lr=lr, weight_decay=wd, momentum=beta, **kw)
    emu = omuon.muon_step(W0, G, B0, lr=lr, weight_decay=wd, momentum=beta, precision="bf16", **kw)
    # fp32 path: momentum (one fused multiply-add per element)
    assert rel(Bg, ref["B"]) <= 1e-6
    m, n = G.shape
    s = omuon.shape_scale(m, n, kw.get("adjust_lr", "match_rms_adamw"))
    decay = np.float32(1 - lr * wd)
    # recover the GPU's O from its W update, then gate it against the oracle
    O_gpu = (np.float64(decay) * W0.astype(np.float64) - Wg) / (lr * s)
    gate = ns_gate(ref["N"], O_gpu, ref["O"], emu["O"])
    # fp32 path: the apply itself is exact up to fp32 rounding of W
    dW = Wg - np.float64(decay) * W0
    assert rel(dW, ref["dW"]) <= 2e-2 or gate["k"] < min(m, n)
    return gate


def test_cfg1_single_matrix(ctx):
    W, G, B = wl.cfg1()
    Wg, Bg, flags = run_gpu_muon(ctx, [W], [G], [B])
    gate = check_muon(W, G, B, Wg[0], Bg[0])
    assert gate["k"] == 64 and flags[0] == 0


def test_cfg1_two_steps_deterministic(ctx):
    W, G, B = wl.cfg1()
    G2 = wl.lowrank_sum(wl.rng_of("cfg1-step2"), 256, 512, 64)
    Wg, Bg, _ = run_gpu_muon(ctx, [W], [G], [B])
    Wg2, Bg2, _ = run_gpu_muon(ctx, [Wg[0]], [G2], [Bg[0]])
    # the second step starts from the GPU's own state
    check_muon(Wg[0], G2, Bg[0], Wg2[0], Bg2[0])
    Wr, Br, _ = run_gpu_muon(ctx, [W], [G], [B])
    np.testing.assert_array_equal(Wr[0], Wg[0])      # bitwise repeatable
    np.testing.assert_array_equal(Br[0], Bg[0])


@pytest.mark.parametrize("shape", [(128, 384), (384, 128), (300, 300), (130, 257), (257, 130),
                                   (64, 1000), (7, 3), (1, 40), (40, 1), (3, 1000), (512, 8)])
def test_ragged_shapes_full_rank(ctx, shape):
    m, n = shape
    rng = wl.rng_of("ragged", m, n)
    W = wl.weights(rng, m, n)
    G = wl.gaussian(rng, (m, n), 1e-3)
    B = wl.gaussian(rng, (m, n), 1e-3)
    Wg, Bg, _ = run_gpu_muon(ctx, [W], [G], [B])
    check_muon(W, G, B, Wg[0], Bg[0])


@pytest.mark.parametrize("kw", [dict(nesterov=False), dict(momentum_ema=True),
                                dict(adjust_lr="original"), dict(ns_steps=3)])
def test_options(ctx, kw):
    m, n = 192, 320
    rng = wl.rng_of("options", str(kw))
    W = wl.weights(rng, m, n)
    G = wl.gaussian(rng, (m, n), 1e-3)
    B = wl.gaussian(rng, (m, n), 1e-3)
    Wg, Bg, _ = run_gpu_muon(ctx, [W], [G], [B], **kw)
    check_muon(W, G, B, Wg[0], Bg[0], **kw)


def test_dense_gpt_mini_buckets(ctx):
    """Every matrix kind of the dense GPT workload at reduced width, two
    layers: buckets with mixed orientation (gate/up tall, down wide)."""
    items = wl.cfg2_list(wl.CFG2_MINI)
    Ws, Gs = zip(*[wl.cfg2_matrix(l, nm, m, n, wl.CFG2_MINI, "cfg2-mini") for l, nm, m, n in items])
    Bs = [np.zeros_like(w) for w in Ws]
    Wg, Bg, flags = run_gpu_muon(ctx, list(Ws), list(Gs), Bs)
    for i in range(len(items)):
        check_muon(Ws[i], Gs[i], Bs[i], Wg[i], Bg[i])
    assert (flags == 0).all()


def test_moe_mini_grouped(ctx):
    """Experts with log-normal scales in one grouped batch (96 x 256 each)."""
    cfg = wl.CFG3_MINI
    Ws, Gs = [], []
    for e in range(cfg["experts"]):
        w, g, _ = wl.cfg3_expert(0, e, cfg, "cfg3-mini")
        Ws += w
        Gs += g
    Bs = [np.zeros_like(w) for w in Ws]
    Wg, Bg, _ = run_gpu_muon(ctx, Ws, Gs, Bs)
    for i in range(0, len(Ws), 7):
        check_muon(Ws[i], Gs[i], Bs[i], Wg[i], Bg[i])


def test_skip_and_nonfinite(ctx):
    rng = wl.rng_of("skip")
    Ws = [wl.weights(rng, 64, 128) for _ in range(3)]
    Gs = [wl.gaussian(rng, (64, 128), 1e-3) for _ in range(3)]
    Gs[1] = None
    Gs[2] = Gs[2].copy()
    Gs[2][3, 5] = np.nan
    Bs = [np.zeros_like(w) for w in Ws]
    Wg, Bg, flags = run_gpu_muon(ctx, Ws, Gs, Bs)
    np.testing.assert_array_equal(Wg[1], Ws[1])        # skipped: untouched
    np.testing.assert_array_equal(Bg[1], Bs[1])
    assert flags[0] == 0 and flags[1] == -1 and flags[2] == 1
    assert np.isnan(Wg[2]).any()                       # nonfinite values propagate


def test_min_workspace_chunks_match_full(ctx):
    import torch
    from matrix_aware_optimizers_muon_b200 import OP_MUON
    rng = wl.rng_of("chunks")
    Ws = [wl.weights(rng, 128, 256) for _ in range(5)]
    Gs = [wl.gaussian(rng, (128, 256), 1e-3) for _ in range(5)]
    Bs = [np.zeros_like(w) for w in Ws]
    full, _, _ = run_gpu_muon(ctx, Ws, Gs, Bs)
    mn, _ = ctx.workspace_bytes(OP_MUON, [w.shape for w in Ws])
    saved = ctx.workspace
    ctx.attach_workspace(mn)
    W = [_cuda(w) for w in Ws]
    ctx.muon_step(W, [_cuda(g) for g in Gs], [_cuda(b) for b in Bs], reserve=False)
    torch.cuda.synchronize()
    for a, b in zip(W, full):
        np.testing.assert_array_equal(_np(a), b)
    ctx.attach_workspace(saved.numel())


# ---------------------------------------------------------------- plain NS

def test_ns_dyadic_known_svd(ctx):
    """The sweep's square inputs have a known SVD, so the exact fp64 result
    is the closed form of Lemma 3 (no oracle SVD needed)."""
    for n in (512, 1024):
        G, d = wl.cfg5_square(n)
        O = ctx.ns_orthogonalize([_cuda(G)])[0]
        t = np.abs(d) / (np.linalg.norm(d) + 1e-7)
        exact = wl.dyadic_from_diag(np.sign(d) * ons.scalar_map(t))
        emu = ons.newton_schulz_bf16(G)
        ns_gate(G, _np(O), exact, emu)


def test_ns_heads_batch(ctx):
    mats, factors = wl.cfg5_heads(64, 128)
    outs = ctx.ns_orthogonalize([_cuda(m) for m in mats])
    for i in (0, 17, 63):
        U, s, V = factors[i]
        t = s / (np.linalg.norm(s) + 1e-7)
        exact = (U * ons.scalar_map(t)) @ V.T
        emu = ons.newton_schulz_bf16(mats[i])
        ns_gate(mats[i], _np(outs[i]), exact, emu, svd=(U, s, V.T))


def test_ns_matches_muon_direction(ctx):
    # ns_orthogonalize(N) equals the O inside muon_step for the same N
    rng = wl.rng_of("ns-vs-muon")
    G = wl.gaussian(rng, (96, 160), 1.0)
    O = _np(ctx.ns_orthogonalize([_cuda(G)])[0])
    W = np.zeros_like(G)
    Wg, _, _ = run_gpu_muon(ctx, [W], [G], [np.zeros_like(G)], momentum=0.0, lr=1.0, weight_decay=0.0)
    s = 0.2 * np.sqrt(160)
    np.testing.assert_allclose(-Wg[0] / s, O, rtol=0, atol=1e-6)


@pytest.mark.parametrize("coeffs,steps,band", [
    ((1.5, -0.5, 0.0), 5, None),            # classical cubic (Lesson 12, Lemma 3 text)
    ((2.0, -1.5, 0.5), 12, (0.6, 1.3)),     # exact-at-1 variant run 12 times (mer.dev section 4.3)
    ((3.4445, -4.7750, 2.0315), 3, None),   # fewer quintic steps
])
def test_ns_coefficient_variants(ctx, coeffs, steps, band):
    mats, factors = wl.cfg5_heads(2, 128, tag="variants")
    rng = wl.rng_of("variants-wide")
    Gw = wl.gaussian(rng, (96, 320), 1.0)
    inputs = [mats[0], Gw]
    outs = ctx.ns_orthogonalize([_cuda(m) for m in inputs], ns_steps=steps, coeffs=coeffs)
    for x, o in zip(inputs, outs):
        ref = ons.newton_schulz(x, coeffs, steps)
        emu = ons.newton_schulz_bf16(x, coeffs, steps)
        ns_gate(x, _np(o), ref, emu, band=band)


# ------------------------------------------------ fused small-matrix kernel

@pytest.mark.parametrize("shapes", [
    [(64, 200)] * 170 + [(200, 64)] * 130,    # one bucket, both orientations, > 148 per launch
    [(128, 256), (256, 128), (128, 128)],     # the largest shapes the fused kernel takes
    [(1, 1), (5, 250), (33, 100), (100, 33), (127, 255)],   # ragged tails
    # bulk-copied loads and stores (n' <= 128, rows of 16-byte multiples),
    # wide and tall, more matrices than CTAs (several per CTA)
    [(96, 128)] * 500 + [(128, 96)] * 470 + [(128, 128)] * 460,
])
def test_small_fused_batches(ctx, shapes):
    rng = wl.rng_of("small-fused", len(shapes), shapes[0])
    Ws = [wl.weights(rng, m, n) for m, n in shapes]
    Gs = [wl.gaussian(rng, (m, n), 1e-3) for m, n in shapes]
    Bs = [wl.gaussian(rng, (m, n), 1e-3) for m, n in shapes]
    Wg, Bg, flags = run_gpu_muon(ctx, Ws, Gs, Bs)
    assert (flags == 0).all()
    pick = sorted(set([0, len(shapes) - 1, len(shapes) // 2, 149 % len(shapes), 171 % len(shapes)]))
    for i in pick:
        check_muon(Ws[i], Gs[i], Bs[i], Wg[i], Bg[i])
    Wr, Br, _ = run_gpu_muon(ctx, Ws, Gs, Bs)
    for i in pick:
        np.testing.assert_array_equal(Wr[i], Wg[i])   # bitwise repeatable


def test_small_ns_bulk_many(ctx):
    """Plain NS through the fused kernel's bulk-copy path with several
    matrices per CTA: a padded wide shape, its transpose, and full tiles;
    matrices taken from the first and later rounds of a CTA."""
    rng = wl.rng_of("small-ns-bulk")
    shapes = [(100, 128)] * 500 + [(128, 100)] * 500 + [(128, 128)] * 450
    mats = [wl.gaussian(rng, s, 1.0) for s in shapes]
    outs = ctx.ns_orthogonalize([_cuda(m) for m in mats])
    assert ctx.device_status() == 0
    for i in (0, 449, 499, 500, 950, 999, 1000, 1449):
        G = mats[i]
        U, s, Vt = np.linalg.svd(G.astype(np.float64), full_matrices=False)
        t = s / (np.linalg.norm(s) + 1e-7)
        exact = (U * ons.scalar_map(t)) @ Vt
        ns_gate(G, _np(outs[i]), exact, ons.newton_schulz_bf16(G), svd=(U, s, Vt))


@pytest.mark.parametrize("kw", [dict(nesterov=False), dict(momentum_ema=True), dict(ns_steps=3),
                                dict(adjust_lr="original")])
def test_small_fused_options(ctx, kw):
    rng = wl.rng_of("small-options", str(kw))
    shapes = [(96, 160), (160, 96)]
    Ws = [wl.weights(rng, m, n) for m, n in shapes]
    Gs = [wl.gaussian(rng, (m, n), 1e-3) for m, n in shapes]
    Bs = [wl.gaussian(rng, (m, n), 1e-3) for m, n in shapes]
    Wg, Bg, _ = run_gpu_muon(ctx, Ws, Gs, Bs, **kw)
    for i in range(2):
        check_muon(Ws[i], Gs[i], Bs[i], Wg[i], Bg[i], **kw)


def test_cuda_graph_replay_matches_eager(ctx):
    """A Muon step over both paths (batched GEMMs and the fused small-matrix
    kernel) captured in a CUDA graph gives bitwise the eager result."""
    import torch
    rng = wl.rng_of("graph")
    shapes = [(64, 200), (200, 64), (256, 320), (320, 256)]
    Ws = [wl.weights(rng, m, n) for m, n in shapes]
    Gs = [wl.gaussian(rng, (m, n), 1e-3) for m, n in shapes]
    Bs = [wl.gaussian(rng, (m, n), 1e-3) for m, n in shapes]
    We, Be, _ = run_gpu_muon(ctx, Ws, Gs, Bs)
    W = [_cuda(w) for w in Ws]
    G = [_cuda(g) for g in Gs]
    B = [_cuda(b) for b in Bs]
    ctx.reserve(0, shapes)
    step = lambda: ctx.muon_step(W, G, B, reserve=False)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                                     # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for w, b, w0, b0 in zip(W, B, Ws, Bs):         # reset the state, then replay once
        w.copy_(_cuda(w0))
        b.copy_(_cuda(b0))
    graph.replay()
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    for i in range(len(shapes)):
        np.testing.assert_array_equal(_np(W[i]), We[i])
        np.testing.assert_array_equal(_np(B[i]), Be[i])
    del graph


@pytest.mark.parametrize("shapes", [
    [(192, 512), (512, 192), (256, 256)],     # wide, tall and square in the GEMM path
    [(192, 600), (600, 192)],                 # ragged last tile (600 = 2 x 256 + 88)
    [(200, 518), (518, 200)],                 # rows not 16-byte multiples: scalar W accesses
])
def test_apply_in_update_epilogue(ctx, shapes):
    """Muon's apply runs in the last update product's epilogue.  With zero
    momentum and no Nesterov the NS input is G itself, so ns_orthogonalize on
    the same batch yields the same O; W must then be fma(decay, W0, -step O)
    in fp32 (checked in float64: at most 1 ulp, double rounding aside)."""
    import torch
    rng = wl.rng_of("fused-apply-" + "-".join(f"{m}x{n}" for m, n in shapes))
    Gs = [wl.gaussian(rng, s, 1e-3) for s in shapes]
    W0 = [wl.gaussian(rng, s, 0.02) for s in shapes]
    lr, wd = 0.02, 0.01
    O = [t.cpu().numpy() for t in ctx.ns_orthogonalize([_cuda(g) for g in Gs])]
    W = [_cuda(w) for w in W0]
    B = [torch.zeros_like(w) for w in W]
    ctx.muon_step(W, [_cuda(g) for g in Gs], B, lr=lr, weight_decay=wd, momentum=0.95, nesterov=False)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    lr32, wd32 = np.float64(np.float32(lr)), np.float64(np.float32(wd))
    decay = np.float32(1.0 - lr32 * wd32)
    for (m, n), w0, o, w in zip(shapes, W0, O, W):
        step = np.float32(lr32 * (0.2 * np.sqrt(max(m, n))))
        neg = -(step * o.astype(np.float32))                      # fp32 product, as on the device
        exp = (np.float64(decay) * w0.astype(np.float64) + neg.astype(np.float64)).astype(np.float32)
        got = w.cpu().numpy()
        ulp = np.abs(got.view(np.int32).astype(np.int64) - exp.view(np.int32).astype(np.int64))
        assert ulp.max() <= 1, (m, n, int(ulp.max()))
        assert (ulp == 0).mean() >= 0.999, (m, n, float((ulp == 0).mean()))


def _save_load(tensors):
    """torch.save to memory and back onto the GPU: a checkpoint round trip."""
    import io
    import torch
    buf = io.BytesIO()
    torch.save([t.cpu() for t in tensors], buf)
    buf.seek(0)
    return [t.cuda() for t in torch.load(buf)]


def test_checkpoint_resume_bitwise(ctx):
    """All optimizer state is caller-owned: saving W and the momentum after
    one step, reloading them and stepping again gives the same bits as
    stepping on (Muon, wide and tall matrices in one bucket)."""
    import torch
    rng = wl.rng_of("checkpoint-muon")
    shapes = [(192, 512), (512, 192)]
    W = [_cuda(wl.gaussian(rng, s, 0.02)) for s in shapes]
    B = [torch.zeros_like(w) for w in W]
    G1 = [_cuda(wl.gaussian(rng, s, 1e-3)) for s in shapes]
    G2 = [_cuda(wl.gaussian(rng, s, 1e-3)) for s in shapes]
    ctx.muon_step(W, G1, B)
    W2, B2 = _save_load(W), _save_load(B)
    ctx.muon_step(W, G2, B)
    ctx.muon_step(W2, G2, B2)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    for a, b in zip(W + B, W2 + B2):
        assert torch.equal(a, b)
