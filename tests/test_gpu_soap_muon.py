"""SOAP-Muon parity: the CUDA path through the C ABI against the fp64
oracle and its bf16-emulation mode, from the same seeded warm state."""
import numpy as np
import pytest

import workloads as wl
from gates import basis_gate, ns_gate, rel
from gpu_env import context
from oracle import muon as omuon
from oracle import soap_muon as osm

pytestmark = pytest.mark.gpu

HP = dict(lr=0.02, weight_decay=0.01, momentum=0.95, beta2=0.95, shampoo_beta=0.9, eps=1e-8)


@pytest.fixture(scope="module")
def ctx():
    return context()


def _cuda(a):
    import torch
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _np(t):
    return None if t is None else t.detach().cpu().numpy().astype(np.float64)


def warm_state(m, n, left, right, steps, tag):
    """fp64 oracle steps from zero state; float32 state + the next gradient."""
    st = wl.SpikeStream(tag, "warm", m * 1000 + n, m, n, wl.CFG4_MINI)
    S = dict(W=st.W.astype(np.float64), B=np.zeros((m, n)), V=np.zeros((m, n)),
             L=np.zeros((m, m)) if left else None, QL=np.eye(m) if left else None,
             R=np.zeros((n, n)) if right else None, QR=np.eye(n) if right else None)
    for t in range(1, steps + 1):
        out = osm.soap_muon_step(S["W"], st.next(), S["B"], S["V"], S["L"], S["QL"], S["R"], S["QR"],
                                 t=t, **HP)
        S = {k: out[k] for k in S}
    return {k: (None if v is None else v.astype(np.float32)) for k, v in S.items()}, st.next(), steps + 1


def run_gpu(ctx, states, grads, t, flags=None, **kw):
    import torch
    ds = []
    for S, G in zip(states, grads):
        d = {k: _cuda(v) for k, v in S.items()}
        d["G"] = _cuda(G)
        ds.append(d)
    ctx.soap_muon_step(ds, t, nonfinite=flags, **{**HP, **kw})
    torch.cuda.synchronize()
    assert ctx.device_status() == 0
    return [{k: _np(v) for k, v in d.items() if k != "G"} for d in ds]


def check(S, G, t, out, **kw):
    hp = {**HP, **kw}
    args = (S["W"], G, S["B"], S["V"], S["L"], S["QL"], S["R"], S["QR"])
    ref = osm.soap_muon_step(*args, t=t, **hp)
    emu = osm.soap_muon_step(*args, t=t, precision="bf16", **hp)
    res = {"B": rel(out["B"], ref["B"])}
    assert res["B"] <= 1e-6, res                                      # fp32 path
    for fac, q in (("L", "QL"), ("R", "QR")):
        if S[fac] is None:
            continue
        res[fac] = rel(out[fac], emu[fac])
        assert res[fac] <= 1e-4, res
        Q = out[q]
        sel, _ = basis_gate(Q, emu[fac], S[q])   # qr(L Q_old), column by column
        if sel.all():
            res[q] = rel(Q, emu[q])
            assert res[q] <= 5e-3, res
    res["V"] = rel(out["V"], emu["V"])
    assert res["V"] <= 1e-2, res
    m, n = G.shape
    s = omuon.shape_scale(m, n, hp.get("adjust_lr", "match_rms_adamw"))
    decay = np.float64(np.float32(1 - hp["lr"] * hp["weight_decay"]))
    O_gpu = (decay * S["W"].astype(np.float64) - out["W"]) / (hp["lr"] * s)
    res["gate"] = ns_gate(ref["P"], O_gpu, ref["O"], emu["O"])
    return res


@pytest.mark.parametrize("m,n,left,right", [
    (256, 256, True, True),      # two-sided, square
    (128, 384, True, True),      # two-sided, wide (NS on the fused small-matrix kernel)
    (256, 896, True, False),     # right side identity
    (160, 96, False, True),      # left side identity, tall
    (64, 128, False, False),     # both identity: Adam-normalised momentum into NS
])
def test_warm_step_parity(ctx, m, n, left, right):
    S, G, t = warm_state(m, n, left, right, 6, "soap-muon")
    out = run_gpu(ctx, [S], [G], t)[0]
    check(S, G, t, out)


def test_batch_of_mixed_groups_and_options(ctx):
    """Several groups in one call (two shapes, one-sided and two-sided), with
    Nesterov off and the 'original' scale."""
    kw = dict(nesterov=False, adjust_lr="original")
    cases = [(256, 256, True, True), (256, 256, True, True), (192, 512, True, False)]
    states, grads, ts = [], [], []
    for i, (m, n, l, r) in enumerate(cases):
        S, G, t = warm_state(m, n, l, r, 4, f"soap-muon-mix{i}")
        states.append(S); grads.append(G); ts.append(t)
    import torch
    flags = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    outs = run_gpu(ctx, states, grads, ts[0], flags=flags, **kw)
    assert (flags.cpu().numpy() == 0).all()
    for S, G, out in zip(states, grads, outs):
        check(S, G, ts[0], out, **kw)


def test_stale_basis_keeps_q(ctx):
    S, G, t = warm_state(256, 256, True, True, 4, "soap-muon-stale")
    out = run_gpu(ctx, [S], [G], t, refresh=False)[0]
    np.testing.assert_array_equal(out["QL"], S["QL"])
    np.testing.assert_array_equal(out["QR"], S["QR"])


def test_cold_start_from_zero_state(ctx):
    """Step 1: identity bases for the preconditioning (the stored Q = I), then
    the first refresh of square two-sided factors (nearly singular: its last
    basis vectors are gated only for orthonormality)."""
    import torch
    m = n = 256
    st = wl.SpikeStream("soap-muon-cold", "x", 0, m, n, wl.CFG4_MINI)
    S = dict(W=st.W, B=np.zeros((m, n), np.float32), V=np.zeros((m, n), np.float32),
             L=np.zeros((m, m), np.float32), QL=np.eye(m, dtype=np.float32),
             R=np.zeros((n, n), np.float32), QR=np.eye(n, dtype=np.float32))
    G = st.next()
    flags = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    out = run_gpu(ctx, [S], [G], 1, flags=flags)[0]
    assert int(flags.item()) == 0
    res = check(S, G, 1, out)
    assert res["gate"]["k"] > 0
