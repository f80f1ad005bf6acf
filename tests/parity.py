"""Helpers shared by the parity tests: device upload of the seeded inputs, the near-tie policy for
top-k indices, norm-wise errors, and the oracle restricted to sampled heads.

Near-tie policy.  The kernels take the top-k decision on fp32 logits accumulated in their own order;
the oracle takes it on its fp64 logits rounded to fp32.  A token is *flagged* when its oracle gap
between the k-th and (k+1)-th largest logit is below DELTA; there either choice is a correct top-k of
logits within DELTA, so the test checks the GPU's choice is such a set and replays it in the oracle.
Every unflagged token must match bit for bit.
"""
import numpy as np
import torch

from oracle import swimba_oracle as O
from parameter_space_moe_b200 import inputs as I
from parameter_space_moe_b200 import swimba

DELTA = 1e-4
TOL_F32 = 1e-5      # norm-wise relative error, all-fp32 layer
TOL_BF16 = 2e-3     # norm-wise relative error, bf16 in/out with fp32 state
# SSM states (fp32) of bf16 layers: the tensor-core scan feeds the end-state product with the
# decay-scaled values rounded once to fp16 (~3e-4 relative per element), so states are held to 1e-3.
TOL_STATE_BF16 = 1e-3

f64 = I.to_f64


def tol_of(w):
    return TOL_F32 if w.dtype == "f32" else TOL_BF16


def state_tol_of(w):
    return TOL_F32 if w.dtype == "f32" else TOL_STATE_BF16


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to_np(t):
    return t.detach().cpu().double().numpy() if t.dtype != torch.int32 else t.detach().cpu().numpy()


def device_weights(inp, dev="cuda"):
    return swimba.WeightSet(*(inp[k].to(dev) for k in ("W_r", "W_dt", "b_dt", "A", "W_exp")))


def out_dtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def stream_torch_dtype(w):
    return torch.float16 if w.dtype == "bf16" else torch.float32


def flagged(g, k, delta=DELTA):
    """Rows whose k-th and (k+1)-th largest logits are within delta."""
    E = g.shape[1]
    if k >= E:
        return np.zeros(g.shape[0], dtype=bool)
    s = -np.sort(-g, axis=1)
    return (s[:, k - 1] - s[:, k]) < delta


def check_topk(gpu_idx, g, k, delta=DELTA):
    """Bit-exact on unflagged rows; on flagged rows the GPU set must be a top-k of a logit vector
    within delta.  Returns (flag mask, forced index array for the oracle replay)."""
    gpu_idx = np.asarray(gpu_idx).reshape(-1, k).astype(np.int64)
    want = O.topk_select(g.astype(np.float32), k)
    fl = flagged(g, k, delta)
    bad = np.nonzero((gpu_idx != want).any(axis=1) & ~fl)[0]
    assert bad.size == 0, f"{bad.size} unflagged tokens differ, first {bad[:5]}"
    forced = -np.ones_like(gpu_idx)
    for t in np.nonzero(fl)[0]:
        sel = gpu_idx[t]
        assert len(set(sel.tolist())) == k
        rest = np.setdiff1d(np.arange(g.shape[1]), sel)
        assert g[t, sel].min() >= g[t, rest].max() - delta
        forced[t] = sel
    return fl, forced


def head_slice(inp, w, heads):
    """Weights of the layer restricted to the given heads (the layer is separable per head once the
    routing is fixed: routing depends only on W_r).  Returns f64 arrays for the oracle with H'=len(heads)
    and G' = number of distinct groups, and the group map."""
    H, P, N, G = w.nheads, w.headdim, w.dstate, w.G
    hpg = H // G
    groups = sorted({h // hpg for h in heads})
    whole = list(heads) == sorted(heads) and all(sum(1 for h in heads if h // hpg == g) == hpg for g in groups)
    assert len(groups) == len(heads) or G == H or whole, "sample one head per group, or whole groups in order"
    W = inp["W_exp"]
    xcols = np.concatenate([np.arange(h * P, (h + 1) * P) for h in heads])
    bcols = np.concatenate([H * P + np.arange(g * N, (g + 1) * N) for g in groups])
    ccols = bcols + G * N
    cols = torch.from_numpy(np.concatenate([xcols, bcols, ccols]))
    return dict(W_r=f64(inp["W_r"]), W_dt=f64(inp["W_dt"][list(heads)]), b_dt=f64(inp["b_dt"][list(heads)]),
                A=f64(inp["A"][list(heads)]), W_exp=f64(W.index_select(1, cols)), H=len(heads), G=len(groups))


def oracle_heads(inp, w, X, heads, forced=None, init=None):
    """Oracle layer output for the sampled heads only: y [B,T,len(heads),P], final [B,len,N,P]."""
    s = head_slice(inp, w, heads)
    return O.layer_fwd(X, s["W_r"], s["W_dt"], s["b_dt"], s["A"], s["W_exp"], s["H"], w.headdim, w.dstate,
                       s["G"], w.top_k, init=init, forced_idx=forced)


def oracle_heads_blocked(inp, w, X, heads, forced=None, init=None, block=16):
    """oracle_heads over many heads, a block of heads at a time (bounded fp64 weight copies): y
    [B,T,len(heads),P], final [B,len(heads),N,P].  init, when given, is [B,len(heads),N,P]."""
    ys, fins = [], []
    for i in range(0, len(heads), block):
        hb = heads[i:i + block]
        r = oracle_heads(inp, w, X, hb, forced, None if init is None else init[:, i:i + block])
        ys.append(r["y"])
        fins.append(r["final"])
    return dict(y=np.concatenate(ys, axis=2), final=np.concatenate(fins, axis=1))
