"""Recurrent decode (swimba_step) against the oracle: T steps reproduce the layer's forward pass, and
the 256-sequence decode workload (state from a 512-token prefill) matches on sampled heads."""
import numpy as np
import pytest
import torch

from oracle import swimba_oracle as O
from parameter_space_moe_b200 import configs, inputs, swimba

from .parity import (TOL_STATE_BF16, check_topk, device_weights, f64, head_slice, oracle_heads_blocked, out_dtype, rel,
                     to_np)

pytestmark = pytest.mark.gpu


def _step(w, d, W, X, state, ws):
    y = torch.empty(w.batch, w.nheads * w.headdim, dtype=out_dtype(w), device="cuda")
    idx = torch.empty(w.batch, w.top_k, dtype=torch.int32, device="cuda")
    swimba.step(d, X, W, state, y, idx, ws)
    return y, idx


@pytest.mark.parametrize("w", [configs.TINY_F32.with_(batch=3, seqlen=40, seed=41),
                               configs.BASE.with_(name="dec_bf16", batch=4, seqlen=24, d_model=256, nheads=4,
                                                  seed=42)], ids=lambda w: w.name)
def test_steps_equal_layer_fwd(w):
    inp = inputs.make_inputs(w)
    W = device_weights(inp)
    d = swimba.dims_of(w)
    X = inp["X"].cuda()
    y = torch.empty(w.M, w.nheads * w.headdim, dtype=out_dtype(w), device="cuda")
    fin = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, device="cuda")
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")
    swimba.layer_fwd(d, X.reshape(w.M, -1), W, None, y, fin, None, None, ws)
    d1 = swimba.dims_of(w, seqlen=1)
    ws1 = torch.empty(swimba.workspace_size(d1), dtype=torch.uint8, device="cuda")
    state = torch.zeros(w.batch, w.nheads, w.dstate, w.headdim, device="cuda")
    ys = []
    for t in range(w.seqlen):
        yt, _ = _step(w, d1, W, X[:, t].contiguous(), state, ws1)
        ys.append(yt)
    assert swimba.check_device_status() == 0
    ystep = torch.stack(ys, 1).reshape(y.shape)
    tol = 1e-5 if w.dtype == "f32" else 2e-3
    assert rel(to_np(ystep), to_np(y)) < tol
    assert rel(to_np(state), to_np(fin)) < (1e-5 if w.dtype == "f32" else 1e-3)


def test_decode_workload():
    """256 sequences x one token, H64 N128 P64 E16 k2 D2048, state from a 512-token GPU prefill.

    Prefill: every head of 4 sampled sequences against the oracle (near-tied router decisions replayed
    with the GPU's own indices, so the comparison always runs).  Step: every head of all 256 sequences,
    starting from the GPU's prefill state."""
    w = configs.DECODE
    inp = inputs.make_inputs(w)
    W = device_weights(inp)
    dp = swimba.dims_of(w, seqlen=w.prefill)
    Xp = inp["X"].cuda()
    M = w.batch * w.prefill
    yp = torch.empty(M, w.nheads * w.headdim, dtype=torch.bfloat16, device="cuda")
    state = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, device="cuda")
    idxp = torch.empty(M, w.top_k, dtype=torch.int32, device="cuda")
    ws = torch.empty(swimba.workspace_size(dp), dtype=torch.uint8, device="cuda")
    swimba.layer_fwd(dp, Xp.reshape(M, -1), W, None, yp, state, idxp, None, ws)
    assert swimba.check_device_status() == 0
    del ws
    heads = list(range(w.nheads))
    # prefill parity on 4 sampled sequences, all heads (rows are independent)
    seqs = [0, 85, 170, 255]
    Xs = f64(inp["X"][seqs])
    wsub = w.with_(batch=len(seqs), seqlen=w.prefill)
    g = O.router_logits(Xs.reshape(-1, w.d_model), f64(inp["W_r"]))
    gpu_idx = to_np(idxp).reshape(w.batch, w.prefill, w.top_k)[seqs].reshape(-1, w.top_k)
    fl, forced = check_topk(gpu_idx, g, w.top_k)
    ref = oracle_heads_blocked(inp, wsub, Xs, heads,
                               forced.reshape(len(seqs), w.prefill, w.top_k) if fl.any() else None)
    st_gpu = to_np(state)
    ypg = to_np(yp).reshape(w.batch, w.prefill, w.nheads, w.headdim)[seqs]
    assert rel(ypg, ref["y"]) < 2e-3
    assert rel(st_gpu[seqs], ref["final"]) < 2e-3
    del yp
    # the step on all 256 sequences and all heads, starting from the GPU state
    d1 = swimba.dims_of(w, seqlen=1)
    ws1 = torch.empty(swimba.workspace_size(d1), dtype=torch.uint8, device="cuda")
    y, idx = _step(w, d1, W, inp["X_step"].cuda(), state, ws1)
    assert swimba.check_device_status() == 0
    Xt = f64(inp["X_step"])
    g1 = O.router_logits(Xt, f64(inp["W_r"]))
    fl, forced = check_topk(to_np(idx), g1, w.top_k)
    yg = to_np(y).reshape(w.batch, w.nheads, w.headdim)
    new_gpu = to_np(state)
    for h0 in range(0, w.nheads, 16):
        hb = list(range(h0, h0 + 16))
        s = head_slice(inp, w, hb)
        yr, new, _ = O.step(Xt, s["W_r"], s["W_dt"], s["b_dt"], s["A"], s["W_exp"], s["H"], w.headdim, w.dstate,
                            s["G"], w.top_k, st_gpu[:, hb], forced_idx=forced if fl.any() else None)
        assert rel(yg[:, hb], yr) < 2e-3
        # the new state carries the fp16 rounding of the step's injection streams: the bf16 layers' state bar
        assert rel(new_gpu[:, hb], new) < TOL_STATE_BF16
