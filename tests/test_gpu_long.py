"""Long-sequence layer (B1 T32768 D2048 H64 E16 k2 Q256): full-size launch, sampled heads checked
against the oracle's token-by-token recurrence over all 32768 tokens."""
import numpy as np
import pytest
import torch

from oracle import swimba_oracle as O
from parameter_space_moe_b200 import configs, inputs

from .parity import check_topk, f64, oracle_heads, oracle_heads_blocked, rel, to_np
from .test_gpu_layer import run_layer

pytestmark = pytest.mark.gpu


def test_layer_long_sampled():
    w = configs.LONG
    inp = inputs.make_inputs(w)
    y, fin, idx = run_layer(w, inp)
    X = f64(inp["X"])
    g = O.router_logits(X.reshape(w.M, -1), f64(inp["W_r"]))
    fl, forced = check_topk(to_np(idx), g, w.top_k)
    heads = [5, 40]
    ref = oracle_heads(inp, w, X, heads, forced.reshape(1, w.seqlen, w.top_k) if fl.any() else None)
    yg = to_np(y).reshape(1, w.seqlen, w.nheads, w.headdim)[:, :, heads]
    print(f"long layer: flagged {int(fl.sum())}, rel err y {rel(yg, ref['y']):.3e}")
    assert rel(yg, ref["y"]) <= 2e-3
    assert rel(to_np(fin)[:, heads], ref["final"]) <= 2e-3
    # every head over the first 4096 tokens (outputs there depend on no later token)
    Tp = 4096
    allh = list(range(w.nheads))
    refp = oracle_heads_blocked(inp, w.with_(seqlen=Tp), X[:, :Tp], allh,
                                forced.reshape(1, w.seqlen, w.top_k)[:, :Tp] if fl.any() else None)
    ygp = to_np(y).reshape(1, w.seqlen, w.nheads, w.headdim)[:, :Tp]
    print(f"long layer, all heads, first {Tp} tokens: rel err y {rel(ygp, refp['y']):.3e}")
    assert rel(ygp, refp["y"]) <= 2e-3
