"""Gradients of the chunked scan (swimba_ssd_scan_bwd) against the oracle's adjoint recurrence, through the
C ABI.  The streams are the oracle layer's own, rounded to the stream dtype the GPU reads; the oracle then
differentiates exactly those values.  Shapes: the tiny fp32 layer, bf16 layers with N = 128 (one head per
group, two groups of two, G = 1 with k = 3, P = 128), ragged sequence tails (64-token sub-chunks), an initial
state, and upstream gradients scaled by 2^-110 and 2^100."""
import numpy as np
import pytest
import torch

from oracle import swimba_oracle as O
from parameter_space_moe_b200 import configs, inputs, swimba

from .parity import f64, rel, stream_torch_dtype

pytestmark = pytest.mark.gpu

CASES = [
    configs.TINY_F32,
    configs.TINY_F32.with_(name="bwd_f32_ragged_G1", seqlen=203, nheads=4, headdim=32, ngroups=1, seed=121),
    configs.BASE.with_(name="bwd_bf16_ragged", batch=2, seqlen=333, d_model=128, nheads=2, n_experts=4, chunk=128,
                       seed=122),
    configs.BASE.with_(name="bwd_bf16_G2", batch=1, seqlen=256, d_model=128, nheads=4, ngroups=2, n_experts=4,
                       chunk=128, seed=123),
    configs.BASE.with_(name="bwd_bf16_G1_k3", batch=1, seqlen=190, d_model=128, nheads=3, ngroups=1, n_experts=5,
                       top_k=3, chunk=64, seed=124),
    configs.BASE.with_(name="bwd_bf16_P128", batch=1, seqlen=200, d_model=128, nheads=2, headdim=128, n_experts=4,
                       chunk=128, seed=125),
]
# fp32 arithmetic on the same inputs: norm-wise bounds (measured 2e-7 .. 4e-7 for the stream and state
# gradients).  d dt and dA sum many terms of both signs (the log-decay gradient is a difference of score-tile
# row and column sums) and measure up to 2.1e-6, so they are held to 2e-5.
TOL = dict(dBpi=1e-5, dXs=1e-5, dCt=1e-5, dinit=1e-5, ddt=2e-5, dA=2e-5)


@pytest.mark.parametrize("with_init", [False, True], ids=["zero_init", "init"])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_scan_gradients_match_oracle(w, with_init):
    _check(w, with_init)


@pytest.mark.parametrize("scale", [2.0 ** -110, 2.0 ** 100], ids=["dy_2^-110", "dy_2^100"])
def test_scan_gradients_extreme_dy_scale(scale):
    """Every gradient is linear in dy; the tensor-core adjoint sources scale dy by a power of two before
    splitting it into fp16 halves, which must hold for upstream gradients far outside fp16's range."""
    _check(CASES[2], True, scale)


def _check(w, with_init, dy_scale=1.0):
    inp = inputs.make_inputs(w)
    ref = O.layer_fwd(f64(inp["X"]), f64(inp["W_r"]), f64(inp["W_dt"]), f64(inp["b_dt"]), f64(inp["A"]),
                      f64(inp["W_exp"]), w.nheads, w.headdim, w.dstate, w.G, w.top_k)
    sdt = stream_torch_dtype(w)
    Bpi, Xs, Cpi = (torch.from_numpy(ref[k]).to(sdt) for k in ("Bpi", "Xs", "Cpi"))
    dt = torch.from_numpy(ref["dt"]).float()
    A = inp["A"]
    rng = np.random.default_rng(w.seed)
    dy = torch.from_numpy((rng.standard_normal((w.M, w.nheads, w.headdim)) * dy_scale).astype(np.float32))
    init = (torch.from_numpy(rng.standard_normal((w.batch, w.nheads, w.dstate, w.headdim)).astype(np.float32))
            if with_init else None)
    d = swimba.dims_of(w)
    dev = {k: v.cuda() for k, v in dict(Bpi=Bpi, Xs=Xs, Cpi=Cpi, dt=dt, A=A, dy=dy).items()}
    out = dict(dBpi=torch.full((w.M, w.top_k, w.G, w.dstate), float("nan"), device="cuda"),
               dXs=torch.full((w.M, w.top_k, w.nheads, w.headdim), float("nan"), device="cuda"),
               dCt=torch.full((w.M, w.G, w.dstate), float("nan"), device="cuda"),
               ddt=torch.full((w.M, w.nheads), float("nan"), device="cuda"),
               dA=torch.full((w.nheads,), float("nan"), device="cuda"),
               dinit=torch.full((w.batch, w.nheads, w.dstate, w.headdim), float("nan"), device="cuda"))
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")
    swimba.ssd_scan_bwd(d, dev["Bpi"], dev["Xs"], dev["Cpi"], dev["dt"], dev["A"],
                        None if init is None else init.cuda(), dev["dy"], out["dBpi"], out["dXs"], out["dCt"],
                        out["ddt"], out["dA"], out["dinit"], ws)
    assert swimba.check_device_status() == 0
    got = {k: v.cpu().double().numpy() for k, v in out.items()}
    # the oracle on exactly the values the GPU read, one sequence at a time
    Bq, Xq, Cq = (t.double().numpy() for t in (Bpi, Xs, Cpi))
    Ct = Cq.sum(1)
    dtq, Aq, dyq = dt.double().numpy(), f64(A), dy.double().numpy()
    want = {k: [] for k in TOL}
    for b in range(w.batch):
        r = slice(b * w.seqlen, (b + 1) * w.seqlen)
        o = O.scan_backward(Bq[r], Xq[r], Ct[r], dtq[r], Aq, dyq[r], None if init is None else init[b].double().numpy())
        for k in TOL:
            want[k].append(o[k])
    want = {k: (np.sum(v, axis=0) if k == "dA" else np.stack(v) if k == "dinit" else np.concatenate(v))
            for k, v in want.items()}
    for k, tol in TOL.items():
        assert np.isfinite(got[k]).all(), k
        e = rel(got[k].reshape(want[k].shape), want[k])
        print(f"{w.name} {k}: rel err {e:.2e}")
        assert e <= tol, (k, e)


def test_scan_gradients_base_size():
    """The base layer's sizes (B4 T2048 H24 P64 N128 k2), the launch bench.py times, on seeded streams of the
    layer's scale; every gradient of two (sequence, head) rows against the oracle (heads are independent when
    G = H, so the oracle runs on those heads alone)."""
    w = configs.BASE
    g = torch.Generator().manual_seed(131)
    M, k, H, P, N = w.M, w.top_k, w.nheads, w.headdim, w.dstate
    Bpi = (0.5 * torch.randn(M, k, H, N, generator=g)).half()
    Xs = torch.randn(M, k, H, P, generator=g).half()
    Cpi = (0.5 * torch.randn(M, k, H, N, generator=g)).half()
    dt = (1e-3 + 0.099 * torch.rand(M, H, generator=g)).float()
    A = inputs.make_inputs(w, with_x=False)["A"]
    dy = torch.randn(M, H, P, generator=g)
    d = swimba.dims_of(w)
    outs = [torch.empty(M, k, H, N, device="cuda"), torch.empty(M, k, H, P, device="cuda"),
            torch.empty(M, H, N, device="cuda"), torch.empty(M, H, device="cuda"), torch.empty(H, device="cuda")]
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")
    swimba.ssd_scan_bwd(d, Bpi.cuda(), Xs.cuda(), Cpi.cuda(), dt.cuda(), A.cuda(), None, dy.cuda(), *outs, None, ws)
    assert swimba.check_device_status() == 0
    dBpi, dXs, dCt, ddt, _ = (o.cpu().double().numpy() for o in outs)
    for b, h in ((1, 0), (3, 13)):
        r = slice(b * w.seqlen, (b + 1) * w.seqlen)
        sl = lambda t: t[r].double().numpy()
        o = O.scan_backward(sl(Bpi)[:, :, h:h + 1], sl(Xs)[:, :, h:h + 1], sl(Cpi)[:, :, h:h + 1].sum(1),
                            sl(dt)[:, h:h + 1], f64(A)[h:h + 1], sl(dy)[:, h:h + 1])
        for name, got, want in (("dBpi", dBpi[r][:, :, h:h + 1], o["dBpi"]), ("dXs", dXs[r][:, :, h:h + 1], o["dXs"]),
                                ("dCt", dCt[r][:, h:h + 1], o["dCt"]), ("ddt", ddt[r][:, h:h + 1], o["ddt"])):
            e = rel(got, want)
            print(f"base b{b} h{h} {name}: rel err {e:.2e}")
            assert e <= TOL[name], (name, e)
