"""The expert-mixed diagonal transition (swimba_weights.A_exp) against the fp64 oracle, through the C ABI.

With A_exp the transition of token t and head h is A~ = sum_j pi_tj A_exp[K_tj][h], a convex combination of
the active experts' values (Swimba notes, limitations and outlook).  Checked: the layer (fp32 CUDA-core path
and the bf16 tensor-core path, a ragged tail, k = 3), the decode step against the layer, equal expert rows
against the shared-A layer, and the stability flag for a non-negative A~."""
import numpy as np
import pytest
import torch

from oracle import swimba_oracle as O
from parameter_space_moe_b200 import configs, inputs, swimba

from .parity import check_topk, f64, out_dtype, rel, state_tol_of, to_np, tol_of

pytestmark = pytest.mark.gpu

CASES = [
    configs.TINY_F32.with_(name="mixedA_f32", seed=111),
    configs.BASE.with_(name="mixedA_bf16_ragged_k3", batch=2, seqlen=333, d_model=256, nheads=4, n_experts=6,
                       top_k=3, chunk=128, seed=112),
    configs.BASE.with_(name="mixedA_bf16_B2_T1024", batch=2, seqlen=1024, d_model=256, nheads=8, seed=113),
]


def _weights(inp, A_exp="A_exp"):
    t = [inp[k].cuda() for k in ("W_r", "W_dt", "b_dt", "A", "W_exp")]
    return swimba.WeightSet(*t, A_exp=None if A_exp is None else inp[A_exp].cuda())


def _layer(w, inp, W):
    d = swimba.dims_of(w)
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")
    y = torch.empty(w.M, w.nheads * w.headdim, dtype=out_dtype(w), device="cuda")
    fin = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, device="cuda")
    idx = torch.empty(w.M, w.top_k, dtype=torch.int32, device="cuda")
    swimba.layer_fwd(d, inp["X"].cuda().reshape(w.M, -1), W, None, y, fin, idx, None, ws)
    return y, fin, idx


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_layer_with_mixed_A(w):
    inp = inputs.make_inputs(w)
    y, fin, idx = _layer(w, inp, _weights(inp))
    assert swimba.check_device_status() == 0
    X = f64(inp["X"])
    g = O.router_logits(X.reshape(w.M, -1), f64(inp["W_r"]))
    fl, forced = check_topk(to_np(idx), g, w.top_k)
    ref = O.layer_fwd(X, f64(inp["W_r"]), f64(inp["W_dt"]), f64(inp["b_dt"]), None, f64(inp["W_exp"]), w.nheads,
                      w.headdim, w.dstate, w.G, w.top_k,
                      forced_idx=forced.reshape(w.batch, w.seqlen, w.top_k) if fl.any() else None,
                      A_exp=f64(inp["A_exp"]))
    ey = rel(to_np(y).reshape(ref["y"].shape), ref["y"])
    ef = rel(to_np(fin), ref["final"])
    print(f"{w.name}: mixed-A layer rel err y {ey:.3e} final {ef:.3e}")
    assert ey <= tol_of(w)
    assert ef <= state_tol_of(w)
    # the mixed transition differs from the shared one on these inputs (the check above is not vacuous)
    shared = O.layer_fwd(X, f64(inp["W_r"]), f64(inp["W_dt"]), f64(inp["b_dt"]), f64(inp["A"]), f64(inp["W_exp"]),
                         w.nheads, w.headdim, w.dstate, w.G, w.top_k)
    assert rel(shared["y"], ref["y"]) > 10 * tol_of(w)


@pytest.mark.parametrize("w", [CASES[0], CASES[1].with_(name="mixedA_dec_bf16", batch=3, seqlen=20)],
                         ids=lambda w: w.name)
def test_steps_equal_layer_with_mixed_A(w):
    inp = inputs.make_inputs(w)
    W = _weights(inp)
    y, fin, _ = _layer(w, inp, W)
    d1 = swimba.dims_of(w, seqlen=1)
    ws1 = torch.empty(swimba.workspace_size(d1), dtype=torch.uint8, device="cuda")
    state = torch.zeros(w.batch, w.nheads, w.dstate, w.headdim, device="cuda")
    X = inp["X"].cuda()
    ys = []
    for t in range(w.seqlen):
        yt = torch.empty(w.batch, w.nheads * w.headdim, dtype=out_dtype(w), device="cuda")
        swimba.step(d1, X[:, t].contiguous(), W, state, yt, None, ws1)
        ys.append(yt)
    assert swimba.check_device_status() == 0
    ystep = torch.stack(ys, 1).reshape(y.shape)
    assert rel(to_np(ystep), to_np(y)) < tol_of(w)
    assert rel(to_np(state), to_np(fin)) < state_tol_of(w)


def test_equal_expert_rows_give_the_shared_layer():
    w = CASES[0]
    inp = inputs.make_inputs(w)
    inp["A_same"] = inp["A"].repeat(w.n_experts, 1).contiguous()
    y_mixed, fin_mixed, _ = _layer(w, inp, _weights(inp, "A_same"))
    y_shared, fin_shared, _ = _layer(w, inp, _weights(inp, None))
    assert swimba.check_device_status() == 0
    # the weights of a token sum to 1 up to fp32 rounding, so A~ = A to about one ulp
    assert rel(to_np(y_mixed), to_np(y_shared)) < 1e-6
    assert rel(to_np(fin_mixed), to_np(fin_shared)) < 1e-6


def test_non_negative_mixed_A_is_flagged():
    """A~ >= 0 is not a contraction: the layer still runs (small positive values keep it finite here) and
    the status word reports SWIMBA_ERR_UNSTABLE."""
    w = CASES[0].with_(name="mixedA_unstable", seqlen=64)
    inp = inputs.make_inputs(w)
    inp["A_pos"] = torch.full((w.n_experts, w.nheads), 0.01)
    y, fin, _ = _layer(w, inp, _weights(inp, "A_pos"))
    assert swimba.check_device_status() == 8
    assert torch.isfinite(fin).all()
    # the flag is sticky until read, then clear
    assert swimba.check_device_status() == 0
