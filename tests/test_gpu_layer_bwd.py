"""Gradients of the whole layer (swimba_layer_bwd) against the oracle's stage-by-stage reverse mode, through
the C ABI.  The active set the GPU's router chose is replayed in the oracle on near-tied tokens (as in the
forward tests); the upstream gradient dy is seeded.  Shapes: the tiny fp32 layer (CUDA-core forward), bf16
tensor-core layers (N = 128) with G = H and G < H, k = 3 with a ragged tail, W_e not a multiple of 64, experts
that receive no rows, and an initial state."""
import numpy as np
import pytest
import torch

from oracle import swimba_oracle as O
from parameter_space_moe_b200 import configs, inputs, swimba

from .parity import check_topk, device_weights, f64, out_dtype, rel

pytestmark = pytest.mark.gpu

CASES = [
    configs.TINY_F32.with_(name="lbwd_f32", seqlen=200, seed=141),
    configs.BASE.with_(name="lbwd_bf16", batch=2, seqlen=256, d_model=128, nheads=2, n_experts=4, chunk=128,
                       seed=142),
    configs.BASE.with_(name="lbwd_bf16_G1_k3_ragged", batch=1, seqlen=333, d_model=192, nheads=4, ngroups=1,
                       n_experts=6, top_k=3, chunk=128, seed=143),
    # W_e = 3*16 + 2*3*32 = 240, not a multiple of the tensor-core products' 64-wide K blocks
    configs.BASE.with_(name="lbwd_bf16_We240", batch=1, seqlen=300, d_model=128, nheads=3, headdim=16, dstate=32,
                       n_experts=5, chunk=64, seed=144),
    # 40 (token, slot) rows over 64 experts: most experts receive no rows and their weight gradient is 0
    configs.BASE.with_(name="lbwd_bf16_empty_experts", batch=1, seqlen=40, d_model=64, nheads=2, headdim=16,
                       dstate=16, n_experts=64, top_k=1, chunk=64, seed=145),
]
NAMES = ("dX", "dW_r", "dW_dt", "db_dt", "dA", "dW_exp", "dinit")


def _tol(w, name):
    # fp32 layers: fp32 arithmetic throughout (measured 2.6e-7 .. 9.3e-7): the layer's 1e-5 bar.  bf16 layers:
    # the forward's mixed streams are fp16 (the values the GPU differentiates), so every gradient carries that
    # rounding (measured 1.1e-4 .. 4.1e-4): the layer's own 2e-3 bar
    return 1e-5 if w.dtype == "f32" else 2e-3


# the base layer's widths (D 768, H24 P64 N128, W_e 7680, E8 k2) over 512 tokens: the tensor-core expert
# products at their full K and N extents (the oracle needs about 25 s; the full base workload takes minutes)
BASE_WIDTH = configs.BASE.with_(name="lbwd_bf16_base_width", batch=1, seqlen=512, seed=146)


@pytest.mark.parametrize("with_init", [False, True], ids=["zero_init", "init"])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_layer_gradients_match_oracle(w, with_init):
    _check(w, with_init)


def test_layer_gradients_base_width():
    _check(BASE_WIDTH, False)


def _check(w, with_init):
    inp = inputs.make_inputs(w)
    d = swimba.dims_of(w)
    W = device_weights(inp)
    X = inp["X"].cuda().reshape(w.M, w.d_model)
    rng = np.random.default_rng(w.seed)
    dy = torch.from_numpy(rng.standard_normal((w.M, w.nheads, w.headdim)).astype(np.float32))
    init = (torch.from_numpy(rng.standard_normal((w.batch, w.nheads, w.dstate, w.headdim)).astype(np.float32))
            if with_init else None)
    # the GPU's routing (the backward recomputes the same one)
    ws = torch.empty(swimba.layer_bwd_workspace_size(d), dtype=torch.uint8, device="cuda")
    y = torch.empty(w.M, w.nheads * w.headdim, dtype=out_dtype(w), device="cuda")
    idx = torch.empty(w.M, w.top_k, dtype=torch.int32, device="cuda")
    swimba.layer_fwd(d, X, W, None, y, None, idx, None, ws)
    out = dict(dX=torch.full((w.M, w.d_model), float("nan"), device="cuda"),
               dW_r=torch.full((w.n_experts, w.d_model), float("nan"), device="cuda"),
               dW_dt=torch.full((w.nheads, w.d_model), float("nan"), device="cuda"),
               db_dt=torch.full((w.nheads,), float("nan"), device="cuda"),
               dA=torch.full((w.nheads,), float("nan"), device="cuda"),
               dW_exp=torch.full((w.n_experts, w.W_e, w.d_model), float("nan"), device="cuda"),
               dinit=torch.full((w.batch, w.nheads, w.dstate, w.headdim), float("nan"), device="cuda"))
    swimba.layer_bwd(d, X, W, None if init is None else init.cuda(), dy.cuda(), out["dX"], out["dW_r"],
                     out["dW_dt"], out["db_dt"], out["dA"], out["dW_exp"], out["dinit"], ws)
    assert swimba.check_device_status() == 0
    if w.name.endswith("empty_experts"):
        assert len(np.unique(idx.cpu().numpy())) < w.n_experts
    Xf = f64(inp["X"])
    g = O.router_logits(Xf.reshape(w.M, -1), f64(inp["W_r"]))
    fl, forced = check_topk(idx.cpu().numpy(), g, w.top_k)
    ref = O.layer_bwd(Xf, f64(inp["W_r"]), f64(inp["W_dt"]), f64(inp["b_dt"]), f64(inp["A"]), f64(inp["W_exp"]),
                      w.nheads, w.headdim, w.dstate, w.G, w.top_k, dy.double().numpy().reshape(w.batch, w.seqlen,
                                                                                               w.nheads, w.headdim),
                      None if init is None else init.double().numpy(),
                      forced.reshape(w.batch, w.seqlen, w.top_k) if fl.any() else None)
    for name in NAMES:
        got = out[name].cpu().double().numpy()
        assert np.isfinite(got).all(), name
        e = rel(got.reshape(ref[name].shape), ref[name])
        print(f"{w.name} {name}: rel err {e:.2e}")
        assert e <= _tol(w, name), (name, e)
