"""Parity of the output projection (swimba_out_proj) against the fp64 oracle, through the C ABI.

The projection reads y as the layer writes it ([M][H*P], dtype) and W_out [D][H*P].  Shapes cover several
128-row (one-CTA kernel) and 256-row (CTA-pair kernel) tiles and 256-column tiles with ragged tails, a K
that is not a multiple of the 64-wide K step, a single row, the fp32 CUDA-core kernel, the full base
workload, and the layer and projection chained."""
import numpy as np
import pytest
import torch

from oracle import swimba_oracle as O
from parameter_space_moe_b200 import configs, inputs, swimba

from .parity import check_topk, device_weights, f64, out_dtype, rel, to_np, tol_of

pytestmark = pytest.mark.gpu

CASES = [
    configs.TINY_F32,
    configs.TINY_F32.with_(name="f32_ragged", batch=3, seqlen=111, d_model=72, nheads=3, headdim=16, seed=101),
    # 333 rows (3 row tiles, ragged), K = 48 (one partial K step), D = 320 (a full and a partial column tile)
    configs.BASE.with_(name="bf16_ragged_K48_D320", batch=3, seqlen=111, d_model=320, nheads=3, headdim=16,
                       seed=102),
    # the CTA-pair kernel (from 1024 rows) on ragged sizes: 1500 rows (6 pair tiles, the last partial), K = 48,
    # D = 320
    configs.BASE.with_(name="bf16_pair_ragged_K48_D320", batch=3, seqlen=500, d_model=320, nheads=3, headdim=16,
                       seed=106),
    # one row; K = 320 (five K steps); D = 192 (less than one column tile)
    configs.BASE.with_(name="bf16_one_row", batch=1, seqlen=1, d_model=192, nheads=5, headdim=64, seed=103),
    # more tiles than SMs: 4000 x 1536 with K = 1536 (32 row tiles x 6 column tiles)
    configs.BASE.with_(name="bf16_wide", batch=1, seqlen=4000, d_model=1536, seed=104),
    configs.BASE,
]


def _y(w, seed):
    """Seeded y of the layer's output shape and scale (unit normal), in the layer's dtype."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn(w.M, w.nheads * w.headdim, generator=g).to(out_dtype(w))


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_out_proj_matches_oracle(w):
    inp = inputs.make_inputs(w, with_x=False)
    y = _y(w, w.seed + 1)
    out = torch.full((w.M, w.d_model), float("nan"), dtype=out_dtype(w), device="cuda")
    swimba.out_proj(swimba.dims_of(w), y.cuda(), inp["W_out"].cuda(), out)
    assert swimba.check_device_status() == 0
    ref = O.out_proj(f64(y), f64(inp["W_out"]))
    got = to_np(out)
    assert np.isfinite(got).all()
    e = rel(got, ref)
    print(f"{w.name}: out_proj rel err {e:.3e}")
    assert e <= tol_of(w)
    # every element, not only the norm: an fp32 sum of K products (error at most K 2^-24 sum|y||W|) rounded
    # once to bf16 (unit roundoff 2^-8)
    if w.dtype == "bf16":
        K = w.nheads * w.headdim
        acc = 1.01 * K * 2.0 ** -24 * (np.abs(f64(y)) @ np.abs(f64(inp["W_out"])).T)
        assert (np.abs(got - ref) <= 2.0 ** -8 * (np.abs(ref) + acc) + acc).all()


@pytest.mark.parametrize("w", [configs.TINY_F32,
                               configs.BASE.with_(name="bf16_chain", batch=2, seqlen=320, d_model=128, nheads=4,
                                                  n_experts=6, top_k=3, chunk=128, seed=105)],
                         ids=lambda w: w.name)
def test_layer_then_out_proj(w):
    """The layer and its output projection chained on the GPU, against the oracle's layer and projection."""
    inp = inputs.make_inputs(w)
    d = swimba.dims_of(w)
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")
    y = torch.empty(w.M, w.nheads * w.headdim, dtype=out_dtype(w), device="cuda")
    idx = torch.empty(w.M, w.top_k, dtype=torch.int32, device="cuda")
    X = inp["X"].cuda().reshape(w.M, w.d_model)
    swimba.layer_fwd(d, X, device_weights(inp), None, y, None, idx, None, ws)
    out = torch.empty(w.M, w.d_model, dtype=out_dtype(w), device="cuda")
    swimba.out_proj(d, y, inp["W_out"].cuda(), out)
    assert swimba.check_device_status() == 0
    g = O.router_logits(f64(inp["X"]).reshape(w.M, -1), f64(inp["W_r"]))
    fl, forced = check_topk(to_np(idx), g, w.top_k)
    ref = O.layer_fwd(f64(inp["X"]), f64(inp["W_r"]), f64(inp["W_dt"]), f64(inp["b_dt"]), f64(inp["A"]),
                      f64(inp["W_exp"]), w.nheads, w.headdim, w.dstate, w.G, w.top_k,
                      forced_idx=forced.reshape(w.batch, w.seqlen, w.top_k) if fl.any() else None)
    yg = to_np(y)
    ref_out = O.out_proj(ref["y"].reshape(w.M, -1), f64(inp["W_out"]))
    e_y = rel(yg, ref["y"].reshape(w.M, -1))
    e_proj = rel(to_np(out), O.out_proj(yg, f64(inp["W_out"])))
    e = rel(to_np(out), ref_out)
    print(f"{w.name}: layer y rel err {e_y:.3e}, projection of the GPU's y {e_proj:.3e}, chained {e:.3e}")
    # each step within its own bar; the chained result carries both roundings to the output dtype (y, then
    # out: about 1.7e-3 each in bf16), so it is held to the sum of the two bars
    assert e_y <= tol_of(w) and e_proj <= tol_of(w)
    assert e <= 2 * tol_of(w)
