"""Seeded synthetic inputs for a Swimba layer.

This module only draws random numbers; it holds none of the layer's arithmetic.
It is shared by the CUDA path's tests and benchmark and by the oracle's tests so
that both sides see exactly the same values.

Recipe (one numpy PCG64 stream per workload seed, tensors drawn in this order):
  X     ~ N(0, 1)                         [B, T, D]
  W_r   ~ N(0, 1/D)                       [E, D]     router
  W_dt  ~ N(0, 0.01/D)                    [H, D]     dt projection (small, so dt stays near dt0)
  dt0   ~ U[1e-3, 0.1]                    [H]
  b_dt  = softplus^-1(dt0)                [H]        so that softplus(0*X + b_dt) = dt0
  A     = -exp(U[log 1, log 16])          [H]        negative, shared by all experts
  W_exp ~ N(0, 1/D)                       [E, W_e, D] rows ordered [x: H*P | B: G*N | C: G*N]
  (decode workloads then draw X_step ~ N(0,1) [B, D]; X above is the prefill, [B, prefill, D])
  W_out ~ N(0, 1/(H*P))                   [D, H*P]   output projection (drawn after the layer's own
                                                     tensors, so those are the same with or without it)
  A_exp = -exp(U[log 1, log 16])          [E, H]     per-expert transitions for the expert-mixed A~
                                                     (drawn last; fp32)
In bf16 workloads X, W_r, W_dt, W_exp and W_out are rounded to bf16 (round to nearest even) once, here;
b_dt and A stay fp32.  Both sides then read the same rounded values.
"""
import math

import numpy as np
import torch

from .configs import BF16, Workload


def _normal(rng, shape, std):
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def _store(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(torch.bfloat16) if dtype == BF16 else t.to(torch.float32)


def make_inputs(w: Workload, with_x=True):
    """Return a dict of CPU torch tensors in storage dtype (bf16 or fp32; b_dt, A fp32)."""
    rng = np.random.Generator(np.random.PCG64(w.seed))
    D, H, E = w.d_model, w.nheads, w.n_experts
    T = w.prefill if w.prefill else w.seqlen
    out = {}
    x = _normal(rng, (w.batch, T, D), 1.0)
    out["X"] = _store(x, w.dtype) if with_x else None
    del x
    out["W_r"] = _store(_normal(rng, (E, D), 1.0 / math.sqrt(D)), w.dtype)
    out["W_dt"] = _store(_normal(rng, (H, D), math.sqrt(0.01 / D)), w.dtype)
    dt0 = rng.uniform(1e-3, 0.1, size=H)
    out["dt0"] = torch.from_numpy(dt0.astype(np.float32))
    # inverse softplus: log(exp(dt0) - 1) written stably
    out["b_dt"] = torch.from_numpy((dt0 + np.log(-np.expm1(-dt0))).astype(np.float32))
    out["A"] = torch.from_numpy((-np.exp(rng.uniform(0.0, math.log(16.0), size=H))).astype(np.float32))
    out["W_exp"] = _store(_normal(rng, (E, w.W_e, D), 1.0 / math.sqrt(D)), w.dtype)
    if w.prefill:
        out["X_step"] = _store(_normal(rng, (w.batch, D), 1.0), w.dtype)
    HP = H * w.headdim
    out["W_out"] = _store(_normal(rng, (D, HP), 1.0 / math.sqrt(HP)), w.dtype)
    out["A_exp"] = torch.from_numpy((-np.exp(rng.uniform(0.0, math.log(16.0), size=(E, H)))).astype(np.float32))
    return out


def to_f64(t):
    """Exact widening of a stored tensor to a float64 numpy array."""
    return t.double().numpy()
