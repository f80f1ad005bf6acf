"""The pins are strong enough: each plausible mistake, planted in the oracle (on the CPU, by replacing one
of its functions for the duration of a test), makes at least one pin of tests/test_oracle_pins.py fail.

Mistakes planted: no renormalisation over the winners, ties broken toward the higher expert index, the
dt clamp dropped, every slot projected with its first slot's expert, B and C swapped in the stream
split, C~ summed without the router weights, the injection added before the decay, the decay's sign
flipped, the chunked form's causal mask shifted by one, the chunk-state decay taken from the chunk
start instead of its end, the separated-E design advancing only the active experts, the output
projection applied with its matrix transposed, the expert-mixed transition summed without the router
weights or taken from the first active expert alone, the scan's adjoint recurrence without its decay or
with the decay gradient taken one state late, and the layer backward passing the Bpi gradient on without its
router weight or the softmax gradient without its renormalisation term."""
import numpy as np
import pytest

from oracle import swimba_oracle as O

from . import test_oracle_pins as pins


def _topk_weights_not_renormalised(g, idx):
    sel = np.take_along_axis(g, idx, axis=-1)
    m = g.max(axis=-1, keepdims=True)
    return np.exp(sel - m) / np.exp(g - m).sum(axis=-1, keepdims=True)


def _topk_select_ties_high(g, k):
    g = np.asarray(g)
    rev = g[..., ::-1]
    order = np.argsort(-rev, axis=-1, kind="stable")
    return (g.shape[-1] - 1 - order[..., :k]).astype(np.int64)


def _dt_unclamped(X, W_dt, b_dt, dt_min=1e-3, dt_max=0.1):
    return O.softplus(X @ W_dt.T + b_dt)


def _expert_proj_first_slot(X, W_exp, idx):
    M, k = idx.shape
    z = np.zeros((M, k, W_exp.shape[1]))
    for m in range(M):
        for j in range(k):
            z[m, j] = W_exp[idx[m, 0]] @ X[m]
    return z


def _split_swapped(z, H, P, G, N):
    x, B, C = ORIG["split_streams"](z, H, P, G, N)
    return x, C, B


def _mix_unweighted_c(z, w, H, P, G, N):
    x, B, C = O.split_streams(z, H, P, G, N)
    Bpi = w[:, :, None, None] * B
    Cpi = w[:, :, None, None] * C
    return Bpi, x, C.sum(axis=1), Cpi


def _scan_inject_then_decay(Bpi, Xs, Ct, dt, A, init=None, stats=None):
    T, k, H, P = Xs.shape
    G, N = Bpi.shape[2], Bpi.shape[3]
    g = O.group_of(H, G)
    h = np.zeros((H, N, P)) if init is None else np.array(init, dtype=np.float64)
    y = np.zeros((T, H, P))
    for t in range(T):
        a = np.exp(dt[t] * A)
        U = np.einsum("jhn,jhp->hnp", Bpi[t][:, g], Xs[t])
        h = a[:, None, None] * (h + U)
        O._count_update(stats)
        y[t] = np.einsum("hn,hnp->hp", Ct[t][g], h)
    return y, h


def _scan_decay_sign(Bpi, Xs, Ct, dt, A, init=None, stats=None):
    return ORIG["scan_sequential"](Bpi, Xs, Ct, dt, -A, init, stats)


def _dense_skips_inactive_experts(xE, BE, CE, pi_dense, dt, A):
    # the separated-E design advancing only the experts active on a token (k trajectories, not E); its
    # output is unchanged under static routing, so only the trajectory count can catch it
    T, E, H, P = xE.shape
    G, N = BE.shape[2], BE.shape[3]
    g = O.group_of(H, G)
    h = np.zeros((E, H, N, P))
    hs = np.zeros((T, E, H, N, P))
    y = np.zeros((T, H, P))
    stats = {}
    for t in range(T):
        a = np.exp(dt[t] * A)
        for e in range(E):
            if pi_dense[t, e] == 0:
                continue
            h[e] = a[:, None, None] * h[e] + np.einsum("hn,hp->hnp", BE[t, e][g], xE[t, e])
            O._count_update(stats)
            y[t] += pi_dense[t, e] * np.einsum("hn,hnp->hp", CE[t, e][g], h[e])
        hs[t] = h
    return y, hs, stats.get("updates", 0) // max(T, 1)


def _chunked_strict_mask(Bpi, Xs, Ct, dt, A, Q, init=None):
    # the intra-chunk sum over s < t instead of s <= t
    T, k, H, P = Xs.shape
    G, N = Bpi.shape[2], Bpi.shape[3]
    g = O.group_of(H, G)
    nc = (T + Q - 1) // Q
    Hc = np.zeros((H, N, P)) if init is None else np.array(init, dtype=np.float64)
    Hs = np.zeros((nc, H, N, P))
    y = np.zeros((T, H, P))
    for c in range(nc):
        t0, t1 = c * Q, min(T, (c + 1) * Q)
        cs = np.cumsum(dt[t0:t1] * A, axis=0)
        Cg, Bg, Xc = Ct[t0:t1][:, g], Bpi[t0:t1][:, :, g], Xs[t0:t1]
        L = t1 - t0
        Hs[c] = Hc
        scores = np.einsum("thn,sjhn->tsjh", Cg, Bg)
        seg = cs[:, None, :] - cs[None, :, :]
        causal = np.tril(np.ones((L, L), dtype=bool), k=-1)
        decay = np.where(causal[:, :, None], np.exp(np.where(causal[:, :, None], seg, 0.0)), 0.0)
        y[t0:t1] = np.einsum("tsh,tsjh,sjhp->thp", decay, scores, Xc)
        y[t0:t1] += np.exp(cs)[:, :, None] * np.einsum("thn,hnp->thp", Cg, Hc)
        wend = np.exp(cs[-1][None, :] - cs)
        Hc = np.exp(cs[-1])[:, None, None] * Hc + np.einsum("sh,sjhn,sjhp->hnp", wend, Bg, Xc)
    return y, Hs, Hc


def _chunked_state_decay_from_start(Bpi, Xs, Ct, dt, A, Q, init=None):
    # the chunk state weighted by exp(cs_s) (decay from the chunk start) instead of exp(cs_end - cs_s)
    T, k, H, P = Xs.shape
    G, N = Bpi.shape[2], Bpi.shape[3]
    g = O.group_of(H, G)
    nc = (T + Q - 1) // Q
    Hc = np.zeros((H, N, P)) if init is None else np.array(init, dtype=np.float64)
    Hs = np.zeros((nc, H, N, P))
    y = np.zeros((T, H, P))
    for c in range(nc):
        t0, t1 = c * Q, min(T, (c + 1) * Q)
        cs = np.cumsum(dt[t0:t1] * A, axis=0)
        Cg, Bg, Xc = Ct[t0:t1][:, g], Bpi[t0:t1][:, :, g], Xs[t0:t1]
        L = t1 - t0
        Hs[c] = Hc
        scores = np.einsum("thn,sjhn->tsjh", Cg, Bg)
        seg = cs[:, None, :] - cs[None, :, :]
        causal = np.tril(np.ones((L, L), dtype=bool))
        decay = np.where(causal[:, :, None], np.exp(np.where(causal[:, :, None], seg, 0.0)), 0.0)
        y[t0:t1] = np.einsum("tsh,tsjh,sjhp->thp", decay, scores, Xc)
        y[t0:t1] += np.exp(cs)[:, :, None] * np.einsum("thn,hnp->thp", Cg, Hc)
        wstart = np.exp(cs)
        Hc = np.exp(cs[-1])[:, None, None] * Hc + np.einsum("sh,sjhn,sjhp->hnp", wstart, Bg, Xc)
    return y, Hs, Hc


def _mixed_A_unweighted(idx, w, A_exp):
    # the active experts' A summed without the router weights
    return np.asarray(A_exp)[idx].sum(axis=1)


def _mixed_A_first_slot(idx, w, A_exp):
    # the transition of the first active expert alone
    return np.asarray(A_exp)[idx[:, 0]]


def _backward_mutant(Bpi, Xs, Ct, dt, A, dy, init=None, decay_adjoint=True, h_shift=0):
    # the adjoint recurrence with one planted change: no decay between adjoint steps, or the log-decay
    # gradient taken against h_t instead of h_{t-1}
    T, k, H, P = Xs.shape
    G, N = Bpi.shape[2], Bpi.shape[3]
    g = O.group_of(H, G)
    a = np.exp(O.log_decay(dt, A) * np.ones((T, H)))
    hs = np.zeros((T + 1, H, N, P))
    if init is not None:
        hs[0] = init
    for t in range(T):
        hs[t + 1] = a[t][:, None, None] * hs[t] + np.einsum("jhn,jhp->hnp", Bpi[t][:, g], Xs[t])
    out = {n: np.zeros(v.shape) for n, v in (("dBpi", Bpi), ("dXs", Xs), ("dCt", Ct))}
    gdA = np.zeros((T, H))
    lam = np.zeros((H, N, P))
    for t in range(T - 1, -1, -1):
        if t + 1 < T and decay_adjoint:
            lam = a[t + 1][:, None, None] * lam
        lam = lam + np.einsum("hn,hp->hnp", Ct[t][g], dy[t])
        for gi in range(G):
            heads = np.nonzero(g == gi)[0]
            out["dBpi"][t, :, gi] = np.einsum("hnp,jhp->jn", lam[heads], Xs[t][:, heads])
            out["dCt"][t, gi] = np.einsum("hnp,hp->n", hs[t + 1][heads], dy[t][heads])
        out["dXs"][t] = np.einsum("hnp,jhn->jhp", lam, Bpi[t][:, g])
        gdA[t] = a[t] * np.einsum("hnp,hnp->h", lam, hs[t + h_shift])
    out["ddt"] = gdA * (np.ones((T, H)) * np.asarray(A))
    out["dA"] = (gdA * dt).sum(axis=0) if np.ndim(A) == 1 else gdA * dt
    out["dinit"] = a[0][:, None, None] * lam
    return out


def _backward_no_adjoint_decay(Bpi, Xs, Ct, dt, A, dy, init=None):
    return _backward_mutant(Bpi, Xs, Ct, dt, A, dy, init, decay_adjoint=False)


def _backward_decay_gradient_off_by_one(Bpi, Xs, Ct, dt, A, dy, init=None):
    return _backward_mutant(Bpi, Xs, Ct, dt, A, dy, init, h_shift=1)


def _mix_bwd_unweighted_B(dBpi, dXs, dCt, w, Bz, Cz):
    # the Bpi gradient passed on to the projection without its router weight
    dz, dw = ORIG["mix_bwd"](dBpi, dXs, dCt, w, Bz, Cz)
    M, k = w.shape
    HP = dXs.shape[2] * dXs.shape[3]
    GN = dBpi.shape[2] * dBpi.shape[3]
    dz = dz.copy()
    dz[:, :, HP:HP + GN] = dBpi.reshape(M, k, GN)
    return dz, dw


def _mix_bwd_no_readout_term(dBpi, dXs, dCt, w, Bz, Cz):
    # the router weight's gradient without the readout's term <C_j, dC~>
    dz, _ = ORIG["mix_bwd"](dBpi, dXs, dCt, w, Bz, Cz)
    return dz, np.einsum("mjgn,mjgn->mj", Bz, dBpi)


def _mix_bwd_unweighted_C(dBpi, dXs, dCt, w, Bz, Cz):
    # the C~ gradient passed on to every slot's C without its router weight
    dz, dw = ORIG["mix_bwd"](dBpi, dXs, dCt, w, Bz, Cz)
    M, k = w.shape
    HP = dXs.shape[2] * dXs.shape[3]
    GN = dBpi.shape[2] * dBpi.shape[3]
    dz = dz.copy()
    dz[:, :, HP + GN:] = np.broadcast_to(dCt.reshape(M, 1, GN), (M, k, GN))
    return dz, dw


def _router_bwd_not_renormalised(w, dw):
    # the softmax gradient without the renormalisation term
    return w * dw


def _out_proj_transposed(y, W_out):
    # the projection matrix applied transposed (shapes permitting: D == H*P)
    return np.asarray(y) @ np.asarray(W_out)


ORIG = {name: getattr(O, name) for name in
        ("topk_weights", "topk_select", "dt_proj", "expert_proj", "split_streams", "mix", "scan_sequential",
         "scan_chunked", "scan_separated_dense", "out_proj", "mixed_A", "scan_backward", "mix_bwd", "router_bwd")}

# every pin, called with the parameters its decorator gives
ALL_PINS = [
    pins.test_topk_matches_bruteforce_sort_with_ties, pins.test_topk_is_a_maximal_set,
    pins.test_topk_weights_are_renormalised_softmax, pins.test_thm35_sigmoid_worked_example,
    pins.test_dt_recipe_and_clamp, pins.test_expert_proj_matches_elementwise_dot_products,
    pins.test_split_streams_layout, pins.test_group_map, pins.test_polynomial_degree_three_single_expert,
    pins.test_single_expert_reduces_to_plain_ssm_streams, pins.test_identical_experts_equal_unrouted_ssm,
    pins.test_geometric_closed_form_one_injection, lambda: pins.test_sequential_equals_bruteforce_semiseparable(2),
    pins.test_groups_equal_replicated_heads, lambda: pins.test_chunked_equals_sequential(70, 16),
    pins.test_thm33_bibo_bound, pins.test_thm34_static_routing_equivalence_and_counts,
    pins.test_thm34_dynamic_routing_bound, pins.test_layer_fwd_state_handoff, pins.test_steps_equal_layer_fwd,
    pins.test_forced_routing_replays_given_indices, pins.test_out_proj_matches_elementwise_dot_products,
    pins.test_out_proj_identity_and_selection, pins.test_mixed_A_is_the_router_weighted_mean,
    pins.test_mixed_A_with_equal_experts_is_the_shared_layer, pins.test_mixed_A_decay_closed_form,
    pins.test_mixed_A_steps_equal_layer_fwd, pins.test_chunked_with_per_token_A_equals_sequential,
    lambda: pins.test_scan_backward_matches_finite_differences(2), pins.test_scan_backward_per_token_transition,
    pins.test_layer_backward_matches_finite_differences,
]

MUTATIONS = {
    "weights_not_renormalised": ("topk_weights", _topk_weights_not_renormalised),
    "ties_to_higher_index": ("topk_select", _topk_select_ties_high),
    "dt_clamp_dropped": ("dt_proj", _dt_unclamped),
    "slots_use_first_expert": ("expert_proj", _expert_proj_first_slot),
    "B_and_C_swapped": ("split_streams", _split_swapped),
    "C_tilde_without_weights": ("mix", _mix_unweighted_c),
    "inject_before_decay": ("scan_sequential", _scan_inject_then_decay),
    "decay_sign_flipped": ("scan_sequential", _scan_decay_sign),
    "causal_mask_shifted": ("scan_chunked", _chunked_strict_mask),
    "chunk_state_decay_from_start": ("scan_chunked", _chunked_state_decay_from_start),
    "dense_skips_inactive_experts": ("scan_separated_dense", _dense_skips_inactive_experts),
    "out_proj_transposed": ("out_proj", _out_proj_transposed),
    "mixed_A_without_weights": ("mixed_A", _mixed_A_unweighted),
    "mixed_A_first_slot_only": ("mixed_A", _mixed_A_first_slot),
    "adjoint_without_decay": ("scan_backward", _backward_no_adjoint_decay),
    "decay_gradient_off_by_one": ("scan_backward", _backward_decay_gradient_off_by_one),
    "mix_gradient_without_router_weight": ("mix_bwd", _mix_bwd_unweighted_B),
    "router_weight_gradient_without_readout_term": ("mix_bwd", _mix_bwd_no_readout_term),
    "readout_gradient_without_router_weight": ("mix_bwd", _mix_bwd_unweighted_C),
    "router_gradient_not_renormalised": ("router_bwd", _router_bwd_not_renormalised),
}


def test_unmutated_oracle_passes_every_pin():
    for pin in ALL_PINS:
        pin()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for pin in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except Exception as e:  # an assertion, or an error a wrong shape or value leads to
            caught.append(getattr(pin, "__name__", "pin"))
    assert caught, f"no pin caught the planted mistake {name}"
