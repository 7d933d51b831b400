"""SOAP parity: the CUDA path through the C ABI against the fp64 oracle and
its bf16-emulation mode, from the same seeded warm state."""
import numpy as np
import pytest

import workloads as wl
from gates import basis_gate, rel
from gpu_env import context
from oracle import soap as osoap

pytestmark = pytest.mark.gpu

HP = dict(lr=3e-3, beta1=0.95, beta2=0.95, eps=1e-8, weight_decay=0.0)


@pytest.fixture(scope="module")
def ctx():
    return context()


def _cuda(a):
    import torch
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _np(t):
    return None if t is None else t.detach().cpu().numpy().astype(np.float64)


def warm_state(m, n, left, right, steps, tag, cfg=wl.CFG4_MINI):
    """Oracle (fp64) steps from zero state; returns the float32 state and the
    gradient of the next step."""
    st = wl.SpikeStream(tag, "warm", m * 1000 + n, m, n, cfg)
    S = dict(W=st.W.astype(np.float64), M=np.zeros((m, n)), V=np.zeros((m, n)),
             L=np.zeros((m, m)) if left else None, QL=np.eye(m) if left else None,
             R=np.zeros((n, n)) if right else None, QR=np.eye(n) if right else None)
    for t in range(1, steps + 1):
        G = st.next()
        out = osoap.soap_step(S["W"], G, S["M"], S["V"], S["L"], S["QL"], S["R"], S["QR"], t=t, **HP)
        S = {k: out[k] for k in S}
    f32 = {k: (None if v is None else v.astype(np.float32)) for k, v in S.items()}
    return f32, st.next(), steps + 1


def run_gpu(ctx, S, G, t, flags=None, refresh=True):
    import torch
    d = {k: _cuda(v) for k, v in S.items()}
    d["G"] = _cuda(G)
    ctx.soap_step([d], t, nonfinite=flags, refresh=refresh, **HP)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    return {k: _np(v) for k, v in d.items() if k != "G"}


def check_step(ctx, m, n, left, right, steps=10, tag="soap"):
    S, G, t = warm_state(m, n, left, right, steps, tag)
    out = run_gpu(ctx, S, G, t)
    args = (S["W"], G, S["M"], S["V"], S["L"], S["QL"], S["R"], S["QR"])
    ref = osoap.soap_step(*args, t=t, **HP)
    emu = osoap.soap_step(*args, t=t, precision="bf16", **HP)
    res = {}
    res["M"] = rel(out["M"], ref["M"])
    assert res["M"] <= 1e-6, res                                   # fp32 path
    for side, fac, q in (("L", "L", "QL"), ("R", "R", "QR")):
        if S[fac] is None:
            continue
        res[fac] = rel(out[fac], emu[fac])
        assert res[fac] <= 1e-4, res                               # bf16-operand EMA, fp32 state
        Q = out[q]
        res[q + "_orth"] = float(np.abs(Q.T @ Q - np.eye(Q.shape[0])).max())
        sel, _ = basis_gate(Q, emu[fac], S[q])  # qr(L Q_old), column by column
        assert sel.all(), res                                      # warm factors: every column resolved
        res[q] = rel(Q, emu[q])
        assert res[q] <= 5e-3, res                                 # fp32-accurate refresh
    res["V"] = rel(out["V"], emu["V"])
    assert res["V"] <= 1e-2, res
    decayed = (1 - HP["lr"] * HP["weight_decay"]) * S["W"].astype(np.float64)
    dW = out["W"] - decayed
    res["dW_emu"] = rel(dW, emu["dW"])
    res["dW_fp64"] = rel(dW, ref["dW"])
    assert res["dW_emu"] <= 1e-2, res
    assert res["dW_fp64"] <= 2e-2, res                              # bf16-operand path
    return res


@pytest.mark.parametrize("m,n,left,right", [
    (256, 256, True, True),      # two-sided, square
    (128, 384, True, True),      # two-sided, wide
    (256, 896, True, False),     # right side identity (large axis)
    (160, 96, False, True),      # left side identity
])
def test_warm_step_parity(ctx, m, n, left, right):
    check_step(ctx, m, n, left, right)


def test_identity_bases_is_adamw(ctx):
    rng = wl.rng_of("soap-adamw")
    m, n = 64, 128
    S = dict(W=wl.weights(rng, m, n), M=wl.gaussian(rng, (m, n), 1e-3),
             V=np.abs(wl.gaussian(rng, (m, n), 1e-6)), L=None, QL=None, R=None, QR=None)
    G = wl.gaussian(rng, (m, n), 1e-3)
    out = run_gpu(ctx, S, G, 4)
    ref = osoap.soap_step(S["W"], G, S["M"], S["V"], t=4, **HP)
    assert rel(out["W"] - S["W"], ref["dW"]) <= 1e-5
    assert rel(out["V"], ref["V"]) <= 1e-6


def test_cold_start_properties(ctx):
    """Step 1 from zero state: L_1 is ill-conditioned (kappa ~ 1e4); the basis
    is checked by its defining properties (orthonormal, Q^T Y upper
    triangular with a positive diagonal, Y = L_1 Q_0 = L_1) and against the
    fp64 power step."""
    import torch
    m, n = 256, 896
    st = wl.SpikeStream("soap-cold", "x", 0, m, n, wl.CFG4_MINI)
    G = st.next()
    S = dict(W=st.W, M=np.zeros((m, n), np.float32), V=np.zeros((m, n), np.float32),
             L=np.zeros((m, m), np.float32), QL=np.eye(m, dtype=np.float32), R=None, QR=None)
    flags = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    out = run_gpu(ctx, S, G, 1, flags)
    assert int(flags.item()) == 0
    Q, L1 = out["QL"], out["L"]
    assert np.abs(Q.T @ Q - np.eye(m)).max() <= 1e-4
    Y = L1
    R = Q.T @ Y
    assert np.abs(np.tril(R, -1)).max() <= 1e-4 * np.abs(R).max()
    assert (np.diag(R) > 0).all()
    from oracle.qr import qr_positive
    assert rel(Q, qr_positive(Y)[0]) <= 5e-3
    # first Adam step is a sign-like step: |Dbar| ~ 1 entrywise
    dW = out["W"] - S["W"]
    ratio = np.linalg.norm(dW) / (HP["lr"] * np.sqrt(m * n))
    assert 0.9 <= ratio <= 1.0 + 1e-3


def test_skip_leaves_state(ctx):
    m, n = 64, 64
    rng = wl.rng_of("soap-skip")
    S = dict(W=wl.weights(rng, m, n), M=np.zeros((m, n), np.float32), V=np.zeros((m, n), np.float32),
             L=np.zeros((m, m), np.float32), QL=np.eye(m, dtype=np.float32), R=None, QR=None)
    import torch
    d = {k: _cuda(v) for k, v in S.items()}
    d["G"] = None
    ctx.soap_step([d], 1, **HP)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_np(d["W"]), S["W"])
    np.testing.assert_array_equal(_np(d["QL"]), S["QL"])


@pytest.mark.parametrize("m,n,left,right", [(256, 256, True, True), (256, 896, True, False)])
def test_stale_basis_step(ctx, m, n, left, right):
    """A step between two refreshes: factors update, bases are kept."""
    S, G, t = warm_state(m, n, left, right, 10, "soap-stale")
    out = run_gpu(ctx, S, G, t, refresh=False)
    args = (S["W"], G, S["M"], S["V"], S["L"], S["QL"], S["R"], S["QR"])
    ref = osoap.soap_step(*args, t=t, basis_refresh=False, **HP)
    emu = osoap.soap_step(*args, t=t, basis_refresh=False, precision="bf16", **HP)
    np.testing.assert_array_equal(out["QL"], S["QL"])
    assert rel(out["L"], emu["L"]) <= 1e-4
    dW = out["W"] - S["W"].astype(np.float64)
    assert rel(dW, emu["dW"]) <= 1e-2
    assert rel(dW, ref["dW"]) <= 2e-2


def test_cold_start_square_two_sided(ctx):
    """Steps 1-3 from zero state with both factors square (the factors are
    nearly singular at step 1, cond ~1e8: a rank-8 spike over a square
    Gaussian); each GPU step is checked against the oracle run from the GPU's
    own state.  At step 1 the last columns of qr(L_1) are not determined in
    fp32 (nor by any fp32 QR): the basis is gated column by column on the
    resolved ones, and the update on the entries they resolve."""
    import torch
    m = n = 512
    st = wl.SpikeStream("soap-cold-sq", "x", 0, m, n, wl.CFG4_MINI)
    S = dict(W=st.W, M=np.zeros((m, n), np.float32), V=np.zeros((m, n), np.float32),
             L=np.zeros((m, m), np.float32), QL=np.eye(m, dtype=np.float32),
             R=np.zeros((n, n), np.float32), QR=np.eye(n, dtype=np.float32))
    for t in (1, 2, 3):
        G = st.next()
        flags = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        out = run_gpu(ctx, S, G, t, flags)
        assert int(flags.item()) == 0, t
        emu = osoap.soap_step(S["W"], G, S["M"], S["V"], S["L"], S["QL"], S["R"], S["QR"], t=t,
                              precision="bf16", **HP)
        resolved = {}
        for fac, q in (("L", "QL"), ("R", "QR")):
            Q = out[q]
            resolved[q], _ = basis_gate(Q, emu[fac], S[q])
            if t > 1:
                assert resolved[q].all(), (t, q)
                assert rel(Q, emu[q]) <= 5e-3, (t, q, rel(Q, emu[q]))
        dW = out["W"] - S["W"]
        if t == 1:
            # Dbar = M' / |G'| = sign(G') (to eps) at step 1, so what the
            # update carries is the sign pattern of G' in the new bases.  Where
            # G' is small next to the bases' uncertainty its sign is not
            # determined, so Dbar, recovered from dW with the GPU's own bases,
            # is compared by sign on the entries whose row and column basis
            # vectors are resolved and |G'| >= 1e-3 max|G'|; and the update's
            # size to 1 %.
            Dg = out["QL"].T @ (-dW / HP["lr"]) @ out["QR"]
            mask = np.abs(emu["Gr"]) >= 1e-3 * np.abs(emu["Gr"]).max()
            mask &= resolved["QL"][:, None] & resolved["QR"][None, :]
            assert mask.sum() >= 1000, mask.sum()
            agree = np.mean(np.sign(Dg[mask]) == np.sign(emu["Dbar"][mask]))
            assert agree >= 0.99, agree
            ratio = np.linalg.norm(dW) / (HP["lr"] * np.sqrt(m * n))
            ratio_emu = np.linalg.norm(emu["dW"]) / (HP["lr"] * np.sqrt(m * n))
            assert abs(ratio - ratio_emu) <= 1e-2, (ratio, ratio_emu)
        else:
            # the refresh is gated column by column above; the rest of the
            # step (rotations, Adam in the basis, rotation back, apply) is
            # checked against the emulation run with the GPU's refreshed
            # bases.  (Compared with the emulation's own bases instead, the
            # update would differ by a few percent at these early steps: V is
            # still tiny, so Adam magnifies the fp32-level differences of the
            # bases' ill-determined columns.)
            given = osoap.soap_step(S["W"], G, S["M"], S["V"], S["L"], out["QL"], S["R"], out["QR"], t=t,
                                    precision="bf16", refresh=False, **HP)
            assert rel(dW, given["dW"]) <= 1e-2, (t, rel(dW, given["dW"]))
            assert rel(out["V"], given["V"]) <= 1e-2, (t, rel(out["V"], given["V"]))
        S = {k: out[k].astype(np.float32) for k in S}


def test_rank_one_and_zero_gradients(ctx):
    """A rank-one gradient (factor of rank one at step 1: L Q_old has rank
    one, its QR fixes only the first basis vector) and an all-zero gradient
    (zero factor: qr(0) = I, Householder's completion) in one call."""
    import torch
    m, n = 256, 384
    rng = wl.rng_of("soap-rank1")
    u = rng.standard_normal((m, 1))
    v = rng.standard_normal((1, n))
    grads = [(u @ v * 1e-3).astype(np.float32), np.zeros((m, n), np.float32)]
    states = []
    for i in range(2):
        QL, _ = np.linalg.qr(rng.standard_normal((m, m)))
        states.append(dict(W=wl.weights(rng, m, n), M=np.zeros((m, n), np.float32),
                           V=np.zeros((m, n), np.float32), L=np.zeros((m, m), np.float32),
                           QL=QL.astype(np.float32), R=np.zeros((n, n), np.float32),
                           QR=np.eye(n, dtype=np.float32)))
    ds = []
    for S, G in zip(states, grads):
        d = {k: _cuda(v) for k, v in S.items()}
        d["G"] = _cuda(G)
        ds.append(d)
    flags = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    ctx.soap_step(ds, 1, nonfinite=flags, **HP)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    assert (flags.cpu().numpy() == 0).all()
    for S, G, d in zip(states, grads, ds):
        out = {k: _np(v) for k, v in d.items() if k != "G"}
        emu = osoap.soap_step(S["W"], G, S["M"], S["V"], S["L"], S["QL"], S["R"], S["QR"], t=1,
                              precision="bf16", **HP)
        for fac, q in (("L", "QL"), ("R", "QR")):
            basis_gate(out[q], emu[fac], S[q])
        if not G.any():
            np.testing.assert_array_equal(out["QL"], np.eye(m))  # qr(0) = I
            np.testing.assert_array_equal(out["QR"], np.eye(n))
            np.testing.assert_array_equal(out["W"], S["W"])      # zero step, no decay
        else:
            # the resolved direction: the first left basis vector is u / |u|
            # with the sign of (L Q_old)[:, 0]; the rest of G' is at rounding
            # level, where the sign-like first Adam step is not determined,
            # so dW is only checked to be finite
            y0 = emu["L"] @ S["QL"][:, 0].astype(np.float64)
            c = float(out["QL"][:, 0] @ y0) / np.linalg.norm(y0)
            assert c >= 1 - 1e-6
            assert np.isfinite(out["W"]).all()


def test_checkpoint_resume_bitwise(ctx):
    """SOAP state (W, M, V, L, Q_L, R, Q_R and the step count) saved after a
    step and reloaded steps on to the same bits."""
    import io
    import torch
    m = n = 256
    st = wl.SpikeStream("soap-checkpoint", "x", 0, m, n, wl.CFG4_MINI)
    keys = ("W", "M", "V", "L", "QL", "R", "QR")
    S = dict(W=_cuda(st.W), M=torch.zeros(m, n, device="cuda"), V=torch.zeros(m, n, device="cuda"),
             L=torch.zeros(m, m, device="cuda"), QL=torch.eye(m, device="cuda"),
             R=torch.zeros(n, n, device="cuda"), QR=torch.eye(n, device="cuda"))
    G1, G2 = _cuda(st.next()), _cuda(st.next())
    ctx.soap_step([dict(S, G=G1)], 1, **HP)
    buf = io.BytesIO()
    torch.save({k: S[k].cpu() for k in keys}, buf)
    buf.seek(0)
    S2 = {k: v.cuda() for k, v in torch.load(buf).items()}
    ctx.soap_step([dict(S, G=G2)], 2, **HP)
    ctx.soap_step([dict(S2, G=G2)], 2, **HP)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    for k in keys:
        assert torch.equal(S[k], S2[k]), k


def test_nonfinite_gradient_flags_and_propagates(ctx):
    """A NaN in one matrix's gradient: its factor and weights become
    non-finite, its flag is set (the refresh never reaches an orthonormal
    basis) and it keeps its previous bases; the other matrix of the same
    call is unaffected."""
    import torch
    m = n = 128
    rng = wl.rng_of("soap-nan")
    ds, refs = [], []
    for i in range(2):
        S = dict(W=wl.weights(rng, m, n), M=np.zeros((m, n), np.float32), V=np.zeros((m, n), np.float32),
                 L=np.zeros((m, m), np.float32), QL=np.eye(m, dtype=np.float32),
                 R=np.zeros((n, n), np.float32), QR=np.eye(n, dtype=np.float32))
        G = wl.gaussian(rng, (m, n), 1e-3)
        if i == 0:
            G[5, 7] = np.nan
        d = {k: _cuda(v) for k, v in S.items()}
        d["G"] = _cuda(G)
        ds.append(d)
        refs.append((S, G))
    flags = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    ctx.soap_step(ds, 1, nonfinite=flags, **HP)
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    f = flags.cpu().numpy()
    assert f[0] == 1 and f[1] == 0, f
    assert not np.isfinite(_np(ds[0]["W"])).all()
    np.testing.assert_array_equal(_np(ds[0]["QL"]), np.eye(m))
    np.testing.assert_array_equal(_np(ds[0]["QR"]), np.eye(n))
    S, G = refs[1]
    emu = osoap.soap_step(S["W"], G, S["M"], S["V"], S["L"], S["QL"], S["R"], S["QR"], t=1,
                          precision="bf16", **HP)
    out = {k: _np(v) for k, v in ds[1].items() if k != "G"}
    for fac, q in (("L", "QL"), ("R", "QR")):
        basis_gate(out[q], emu[fac], S[q])
    assert np.isfinite(out["W"]).all()


def test_pass_loop_graph_equals_direct_launches(ctx):
    """The refresh's pass loop runs as a graph with a conditional while node
    in eager calls, and as directly launched gated passes under profiling (or
    a caller's stream capture): the same kernels in the same order, so every
    output is bit-equal, including a cold start that needs several passes."""
    import torch
    for steps, (m, n, left, right) in ((0, (96, 160, True, True)), (6, (128, 96, True, False))):
        if steps == 0:
            st = wl.SpikeStream("graph-vs-direct", "warm", 1, m, n, wl.CFG4_MINI)
            S = dict(W=st.W.astype(np.float32), M=np.zeros((m, n), np.float32), V=np.zeros((m, n), np.float32),
                     L=np.zeros((m, m), np.float32), QL=np.eye(m, dtype=np.float32),
                     R=np.zeros((n, n), np.float32), QR=np.eye(n, dtype=np.float32))
            G, t = st.next(), 1
        else:
            S, G, t = warm_state(m, n, left, right, steps, "graph-vs-direct")
        outs = []
        for prof in (False, True):
            ctx.profile(prof)
            try:
                flags = torch.zeros(1, dtype=torch.int32, device="cuda")
                outs.append((run_gpu(ctx, S, G, t, flags=flags), int(flags.item())))
            finally:
                ctx.profile(False)
        (a, fa), (b, fb) = outs
        assert fa == fb
        for k in a:
            if a[k] is not None:
                np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_cuda_graph_capture_matches_eager(ctx):
    """A SOAP step (refresh included) captured in a caller's CUDA graph and
    replayed gives bitwise the eager result: inside a capture the refresh
    launches its passes directly, gated on the device."""
    import torch
    S, G, t = warm_state(96, 160, True, True, 6, "graph-capture")
    eager = run_gpu(ctx, S, G, t)
    d = {k: _cuda(v) for k, v in S.items()}
    d["G"] = _cuda(G)
    call = lambda: ctx.soap_step([d], t, reserve=False, **HP)
    ctx.soap_step([d], t, **HP)                       # reserves the workspace (state reset below)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()                                        # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for k, v in S.items():                            # reset the state, then replay once
        if v is not None:
            d[k].copy_(_cuda(v))
    graph.replay()
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    for k, v in eager.items():
        if v is not None:
            np.testing.assert_array_equal(_np(d[k]), v, err_msg=k)
    del graph
