"""Whole-layer parity of swimba_layer_fwd against the fp64 oracle, plus the layer's properties on the
GPU: chunk-size invariance, state hand-off, determinism, ragged and degenerate shapes."""
import numpy as np
import pytest
import torch

from oracle import swimba_oracle as O
from parameter_space_moe_b200 import configs, inputs, swimba

from .parity import (check_topk, device_weights, f64, oracle_heads, oracle_heads_blocked, out_dtype, rel, to_np,
                     tol_of)

pytestmark = pytest.mark.gpu


def run_layer(w, inp, X=None, init=None, W=None, d=None):
    d = d or swimba.dims_of(w)
    X = inp["X"] if X is None else X
    W = W or device_weights(inp)
    Bsz, T = X.shape[0], X.shape[1]
    y = torch.empty(Bsz * T, w.nheads * w.headdim, dtype=out_dtype(w), device="cuda")
    fin = torch.empty(Bsz, w.nheads, w.dstate, w.headdim, device="cuda")
    idx = torch.empty(Bsz * T, w.top_k, dtype=torch.int32, device="cuda")
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")
    swimba.layer_fwd(d, X.cuda().reshape(Bsz * T, -1), W, None if init is None else init.cuda(), y, fin, idx, None, ws)
    assert swimba.check_device_status() == 0
    return y, fin, idx


def full_parity(w, inp=None):
    inp = inp or inputs.make_inputs(w)
    y, fin, idx = run_layer(w, inp)
    X = f64(inp["X"])
    g = O.router_logits(X.reshape(w.M, -1), f64(inp["W_r"]))
    fl, forced = check_topk(to_np(idx), g, w.top_k)
    ref = O.layer_fwd(X, f64(inp["W_r"]), f64(inp["W_dt"]), f64(inp["b_dt"]), f64(inp["A"]), f64(inp["W_exp"]),
                      w.nheads, w.headdim, w.dstate, w.G, w.top_k,
                      forced_idx=forced.reshape(w.batch, w.seqlen, w.top_k) if fl.any() else None)
    ey = rel(to_np(y), ref["y"].reshape(w.M, -1))
    ef = rel(to_np(fin), ref["final"])
    return ey, ef, int(fl.sum())


TINY_VARIANTS = [
    configs.TINY_F32,
    configs.TINY_F32.with_(name="tiny_ragged", seqlen=203, seed=11),             # T % Q != 0
    configs.TINY_F32.with_(name="tiny_short", seqlen=37, seed=12),               # T < Q
    configs.TINY_F32.with_(name="tiny_one_token", seqlen=1, batch=3, seed=13),  # T = 1
    configs.TINY_F32.with_(name="tiny_E1k1", n_experts=1, top_k=1, seed=14),    # plain single SSM
    configs.TINY_F32.with_(name="tiny_k4", n_experts=8, top_k=4, seed=15),
    configs.TINY_F32.with_(name="tiny_G1", nheads=4, headdim=32, ngroups=1, seed=16),
    configs.TINY_F32.with_(name="tiny_maxdims", nheads=2, headdim=128, dstate=128, chunk=256, seqlen=300, seed=17),
    configs.TINY_F32.with_(name="tiny_E64", n_experts=64, top_k=8, seed=18),
]


@pytest.mark.parametrize("w", TINY_VARIANTS, ids=lambda w: w.name)
def test_layer_fp32(w):
    ey, ef, nfl = full_parity(w)
    assert ey <= 1e-5 and ef <= 1e-5, (ey, ef, nfl)


BF16_VARIANTS = [
    configs.BASE.with_(name="bf16_small", batch=2, seqlen=520, d_model=256, nheads=4, n_experts=8, seed=21),
    configs.BASE.with_(name="bf16_P128_N64", batch=1, seqlen=300, d_model=128, nheads=2, headdim=128, dstate=64,
                       chunk=64, seed=22),
    configs.BASE.with_(name="bf16_G2", batch=1, seqlen=400, d_model=256, nheads=4, ngroups=2, chunk=128, seed=23),
    # B and C shared by all 8 heads (G = 1), ragged, k = 3
    configs.BASE.with_(name="bf16_H8_G1_k3", batch=2, seqlen=777, d_model=256, nheads=8, ngroups=1, n_experts=6,
                       top_k=3, chunk=128, seed=26),
    # CTA-pair expert GEMM (>= 1536 rows per expert on average); the second has a ragged last column tile
    configs.BASE.with_(name="bf16_pair_gemm", batch=2, seqlen=1600, d_model=256, nheads=4, n_experts=2, seed=24),
    configs.BASE.with_(name="bf16_pair_ragged_cols", batch=3, seqlen=3100, d_model=192, nheads=3, dstate=64,
                       ngroups=1, n_experts=3, top_k=1, chunk=128, seed=25),
]


@pytest.mark.parametrize("w", BF16_VARIANTS, ids=lambda w: w.name)
def test_layer_bf16_small(w):
    ey, ef, nfl = full_parity(w)
    assert ey <= 2e-3 and ef <= 2e-3, (ey, ef, nfl)


@pytest.mark.parametrize("G", [6, 1])
def test_layer_base_groups(G):
    """Base sizes with B and C shared by groups of heads (G = H/4 and G = 1).  Every head of two of the four
    sequences against the oracle."""
    w = {6: configs.BASE_G6, 1: configs.BASE_G1}[G]
    inp = inputs.make_inputs(w)
    y, fin, idx = run_layer(w, inp)
    X = f64(inp["X"])
    g = O.router_logits(X.reshape(w.M, -1), f64(inp["W_r"]))
    fl, forced = check_topk(to_np(idx), g, w.top_k)
    fr = forced.reshape(w.batch, w.seqlen, w.top_k) if fl.any() else None
    seqs = [0, 2]
    ws = w.with_(batch=len(seqs))
    ref = oracle_heads_blocked(inp, ws, X[seqs], list(range(w.nheads)), None if fr is None else fr[seqs],
                               block=max(16 // (w.nheads // G), 1) * (w.nheads // G))
    ya = to_np(y).reshape(w.batch, w.seqlen, w.nheads, w.headdim)[seqs]
    ey, ef = rel(ya, ref["y"]), rel(to_np(fin)[seqs], ref["final"])
    print(f"base G={G}: rel err y {ey:.3e} final {ef:.3e}")
    assert ey <= 2e-3 and ef <= 2e-3


def test_layer_base_full():
    """The headline workload (B4 T2048 D768 H24 P64 N128 E8 k2 Q256), every output checked."""
    ey, ef, nfl = full_parity(configs.BASE)
    print(f"base layer: rel err y {ey:.3e} final {ef:.3e}, flagged tokens {nfl}")
    assert ey <= 2e-3 and ef <= 2e-3


@pytest.mark.parametrize("E", configs.ESWEEP_E)
def test_layer_esweep_sampled(E):
    """Expert-count sweep: full-size launch, outputs of sampled heads checked against the oracle."""
    w = configs.esweep(E)
    inp = inputs.make_inputs(w)
    y, fin, idx = run_layer(w, inp)
    X = f64(inp["X"])
    g = O.router_logits(X.reshape(w.M, -1), f64(inp["W_r"]))
    fl, forced = check_topk(to_np(idx), g, w.top_k)
    heads = [0, 13, 23]
    fr = forced.reshape(w.batch, w.seqlen, w.top_k) if fl.any() else None
    ref = oracle_heads(inp, w, X, heads, fr)
    yg = to_np(y).reshape(w.batch, w.seqlen, w.nheads, w.headdim)[:, :, heads]
    assert rel(yg, ref["y"]) <= 2e-3
    assert rel(to_np(fin)[:, heads], ref["final"]) <= 2e-3
    # every head of two of the four sequences (sequences are independent)
    seqs = [1, 3]
    ws = w.with_(batch=len(seqs))
    refa = oracle_heads_blocked(inp, ws, X[seqs], list(range(w.nheads)), None if fr is None else fr[seqs])
    ya = to_np(y).reshape(w.batch, w.seqlen, w.nheads, w.headdim)[seqs]
    assert rel(ya, refa["y"]) <= 2e-3
    assert rel(to_np(fin)[seqs], refa["final"]) <= 2e-3


def test_chunk_size_invariance():
    w = configs.BASE.with_(batch=1, seqlen=1000, seed=31)
    inp = inputs.make_inputs(w)
    outs = [run_layer(w.with_(chunk=q), inp) for q in (64, 128, 256)]
    for y, fin, idx in outs[1:]:
        assert torch.equal(idx, outs[0][2])
        assert rel(to_np(y), to_np(outs[0][0])) < 2e-3
        assert rel(to_np(fin), to_np(outs[0][1])) < 1e-3


def test_state_handoff():
    w = configs.BASE.with_(batch=2, seqlen=700, d_model=256, nheads=4, seed=32)
    inp = inputs.make_inputs(w)
    y, fin, _ = run_layer(w, inp)
    X = inp["X"]
    w1 = w.with_(seqlen=300)
    w2 = w.with_(seqlen=400)
    y1, f1, _ = run_layer(w1, inp, X=X[:, :300].contiguous())
    y2, f2, _ = run_layer(w2, inp, X=X[:, 300:].contiguous(), init=f1)
    ycat = torch.cat([y1.view(2, 300, -1), y2.view(2, 400, -1)], 1).reshape(y.shape)
    assert rel(to_np(ycat), to_np(y)) < 1e-3
    assert rel(to_np(f2), to_np(fin)) < 1e-3


def test_determinism():
    w = configs.BASE.with_(batch=2, seqlen=512, seed=33)
    inp = inputs.make_inputs(w)
    a = run_layer(w, inp)
    b = run_layer(w, inp)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("with_final", [True, False], ids=["time_segments", "sequence_groups"])
@pytest.mark.parametrize("chunks", [1, 2, 3, 5])
def test_host_pipeline_matches_device_call(chunks, with_final):
    """swimba_layer_fwd_host (host X in, host y out, per-group copies overlapping compute) gives exactly the
    device-resident call's y and final states: every row's arithmetic is independent of the grouping.  With a
    final state the groups are sub-chunk-aligned time segments of all five sequences, chained through it;
    without one they are groups of whole sequences."""
    w = configs.BASE.with_(batch=5, seqlen=300, d_model=256, nheads=4, seed=35)
    inp = inputs.make_inputs(w)
    y, fin, _ = run_layer(w, inp)
    d = swimba.dims_of(w)
    W = device_weights(inp)
    Xh = inp["X"].reshape(w.M, -1).contiguous().pin_memory()
    yh = torch.empty(w.M, w.nheads * w.headdim, dtype=torch.bfloat16).pin_memory()
    Xd = torch.empty(w.M, w.d_model, dtype=torch.bfloat16, device="cuda")
    yd = torch.empty_like(yh, device="cuda")
    fh = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, device="cuda") if with_final else None
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")
    swimba.layer_fwd_host(d, Xh, W, None, yh, fh, Xd, yd, ws, chunks=chunks)
    torch.cuda.synchronize()
    assert swimba.check_device_status() == 0
    assert torch.equal(yh, y.cpu())
    if with_final:
        assert torch.equal(fh, fin)


@pytest.mark.parametrize("chunks", [2, 4])
def test_host_pipeline_time_segments(chunks):
    """One sequence is split into sub-chunk-aligned time segments chained through the final state; the
    result is the one-call result bit for bit (the decays restart at every 128-token sub-chunk and the
    state passes through fp32 unchanged)."""
    w = configs.BASE.with_(batch=1, seqlen=1000, d_model=256, nheads=4, seed=36)
    inp = inputs.make_inputs(w)
    y, fin, _ = run_layer(w, inp)
    d = swimba.dims_of(w)
    W = device_weights(inp)
    Xh = inp["X"].reshape(w.M, -1).contiguous().pin_memory()
    yh = torch.empty(w.M, w.nheads * w.headdim, dtype=torch.bfloat16).pin_memory()
    Xd = torch.empty(w.M, w.d_model, dtype=torch.bfloat16, device="cuda")
    yd = torch.empty_like(yh, device="cuda")
    fh = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, device="cuda")
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")
    swimba.layer_fwd_host(d, Xh, W, None, yh, fh, Xd, yd, ws, chunks=chunks)
    torch.cuda.synchronize()
    assert swimba.check_device_status() == 0
    assert torch.equal(yh, y.cpu())
    assert torch.equal(fh, fin)


def test_range_flag_on_fp16_overflow():
    """Inputs whose projections exceed the fp16 stream range raise SWIMBA_ERR_RANGE (no fault)."""
    w = configs.BASE.with_(batch=1, seqlen=64, d_model=128, nheads=2, seed=34)
    inp = inputs.make_inputs(w)
    inp["X"] = (inp["X"].float() * 3e4).to(torch.bfloat16)
    d = swimba.dims_of(w)
    W = device_weights(inp)
    y = torch.empty(w.M, w.nheads * w.headdim, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")
    swimba.layer_fwd(d, inp["X"].cuda().reshape(w.M, -1), W, None, y, None, None, None, ws)
    assert swimba.check_device_status() == 6
    assert swimba.check_device_status() == 0      # the flag was cleared by the read
