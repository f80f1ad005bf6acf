"""Pins of the fp64 oracle against what the Swimba pages and plain mathematics fix.

Each test checks the oracle against something other than itself: a closed form, a brute-force
enumeration, a theorem's bound or equality case, a worked example printed on the pages, or an
invariant that a dropped term, a wrong sign or index or a transposed operand would break.
"""
import itertools
import math
import os

import numpy as np
import pytest

from oracle import swimba_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")
rng0 = np.random.default_rng(1234)


def _rand_streams(rng, T, k, H, P, G, N, scale=1.0):
    Bpi = rng.standard_normal((T, k, G, N)) * scale
    Xs = rng.standard_normal((T, k, H, P)) * scale
    Ct = rng.standard_normal((T, G, N)) * scale
    dt = rng.uniform(1e-3, 0.1, size=(T, H))
    A = -np.exp(rng.uniform(0, math.log(16), size=H))
    return Bpi, Xs, Ct, dt, A


def _small_layer(rng, B=2, T=12, D=16, H=4, P=8, N=4, G=None, E=4, k=2):
    G = G or H
    W_e = H * P + 2 * G * N
    X = rng.standard_normal((B, T, D))
    W_r = rng.standard_normal((E, D)) / math.sqrt(D)
    W_dt = rng.standard_normal((H, D)) * math.sqrt(0.01 / D)
    dt0 = rng.uniform(1e-3, 0.1, size=H)
    b_dt = dt0 + np.log(-np.expm1(-dt0))
    A = -np.exp(rng.uniform(0, math.log(16), size=H))
    W_exp = rng.standard_normal((E, W_e, D)) / math.sqrt(D)
    return dict(X=X, W_r=W_r, W_dt=W_dt, b_dt=b_dt, A=A, W_exp=W_exp, H=H, P=P, N=N, G=G, k=k)


def _fwd(L, **kw):
    args = dict(L)
    args.update(kw)
    return O.layer_fwd(args["X"], args["W_r"], args["W_dt"], args["b_dt"], args["A"], args["W_exp"],
                       args["H"], args["P"], args["N"], args["G"], args["k"],
                       init=args.get("init"), forced_idx=args.get("forced_idx"))


# ----------------------------------------------------------------------------- router

def test_topk_matches_bruteforce_sort_with_ties():
    rng = np.random.default_rng(1)
    for E, k in ((5, 1), (5, 2), (7, 3), (8, 8)):
        g = rng.integers(-3, 4, size=(64, E)).astype(np.float64)   # many exact ties
        got = O.topk_select(g, k)
        for t in range(g.shape[0]):
            # textbook: sort the (value, index) pairs, largest value first, lower index first on ties
            want = [e for _, e in sorted(((-g[t, e], e) for e in range(E)))][:k]
            assert list(got[t]) == want


def test_topk_is_a_maximal_set():
    rng = np.random.default_rng(2)
    g = rng.standard_normal((200, 6))
    idx = O.topk_select(g, 2)
    for t in range(200):
        best = max(itertools.combinations(range(6), 2), key=lambda s: g[t, list(s)].sum())
        assert set(idx[t]) == set(best)
        assert g[t, idx[t][0]] >= g[t, idx[t][1]]


def test_topk_weights_are_renormalised_softmax():
    rng = np.random.default_rng(3)
    g = rng.standard_normal((50, 8)) * 3
    idx = O.topk_select(g, 2)
    w = O.topk_weights(g, idx)
    full = np.exp(g) / np.exp(g).sum(axis=1, keepdims=True)       # softmax over all E
    sel = np.take_along_axis(full, idx, axis=1)
    np.testing.assert_allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-14)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-15)
    assert np.all(w[:, 0] >= w[:, 1])
    w1 = O.topk_weights(g, O.topk_select(g, 1))
    assert np.all(w1 == 1.0)


def test_thm35_sigmoid_worked_example():
    """Theorem 3.5: two experts, logits (0, x): expert 1's weight is sigma(x)."""
    rows = [l.split() for l in open(os.path.join(GOLD, "thm35_sigmoid.txt")) if not l.startswith("#")]
    for xs, sig in rows:
        x, sig = float(xs), float(sig)
        X = np.array([[x]])
        W_r = np.array([[0.0], [1.0]])                              # g = (0, x)
        g = O.router_logits(X, W_r)
        idx = O.topk_select(g, 2)
        w = O.topk_weights(g, idx)
        w_e1 = w[0][list(idx[0]).index(1)]
        assert abs(w_e1 - sig) < 1e-15


def test_dt_recipe_and_clamp():
    dt0 = np.array([1e-3, 0.01, 0.05, 0.1])
    b = dt0 + np.log(-np.expm1(-dt0))
    X = np.zeros((3, 5))
    dt = O.dt_proj(X, np.zeros((4, 5)), b)
    np.testing.assert_allclose(dt, np.broadcast_to(dt0, (3, 4)), rtol=1e-12)
    big = O.dt_proj(np.ones((1, 1)), np.array([[50.0], [-50.0]]), np.zeros(2))
    assert big[0, 0] == 0.1 and big[0, 1] == 1e-3
    # softplus against its definition at moderate arguments
    v = np.linspace(-5, 5, 11)
    np.testing.assert_allclose(O.softplus(v), np.log1p(np.exp(v)), rtol=1e-14)


# ----------------------------------------------------------------------------- projections / mixing

def test_expert_proj_matches_elementwise_dot_products():
    rng = np.random.default_rng(4)
    M, D, E, k, W = 9, 6, 3, 2, 5
    X = rng.standard_normal((M, D))
    W_exp = rng.standard_normal((E, W, D))
    idx = np.array([rng.permutation(E)[:k] for _ in range(M)])
    z = O.expert_proj(X, W_exp, idx)
    for t in range(M):
        for j in range(k):
            for c in range(W):
                assert abs(z[t, j, c] - sum(W_exp[idx[t, j], c, d] * X[t, d] for d in range(D))) < 1e-12


# ----------------------------------------------------------------------------- scan gradients

def _loss(Bpi, Xs, Ct, dt, A, dy, init):
    y, _ = O.scan_sequential(Bpi, Xs, Ct, dt, A, init)
    return float((dy * y).sum())


@pytest.mark.parametrize("G", [2, 1])
def test_scan_backward_matches_finite_differences(G):
    # every gradient of L = sum <dy, y> against central differences of the forward recurrence, entry by entry
    rng = np.random.default_rng(13 + G)
    T, k, H, P, N = 6, 2, 2, 3, 2
    Bpi, Xs, Ct, dt, A = _rand_streams(rng, T, k, H, P, G, N)
    dy = rng.standard_normal((T, H, P))
    init = rng.standard_normal((H, N, P))
    got = O.scan_backward(Bpi, Xs, Ct, dt, A, dy, init)
    args = dict(Bpi=Bpi, Xs=Xs, Ct=Ct, dt=dt, A=A, init=init)
    names = dict(Bpi="dBpi", Xs="dXs", Ct="dCt", dt="ddt", A="dA", init="dinit")
    eps = 1e-6
    for name, arr in args.items():
        num = np.zeros(arr.shape)
        for idx in np.ndindex(arr.shape):
            hi = {n: v.copy() for n, v in args.items()}
            lo = {n: v.copy() for n, v in args.items()}
            hi[name][idx] += eps
            lo[name][idx] -= eps
            num[idx] = (_loss(dy=dy, **hi) - _loss(dy=dy, **lo)) / (2 * eps)
        np.testing.assert_allclose(got[names[name]], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_layer_backward_matches_finite_differences():
    # every gradient of L = sum <dy, y> for a tiny layer against central differences of layer_fwd, entry by
    # entry; the inputs keep every token's top-k gap and every dt well away from the clamp bounds, so small
    # perturbations change neither the active set nor the clamp
    rng = np.random.default_rng(21)
    L = _small_layer(rng, B=2, T=5, D=6, H=2, P=3, N=2, G=1, E=3, k=2)
    L["b_dt"] = np.log(np.expm1(rng.uniform(0.02, 0.08, size=2)))
    H, P, N, G, k = L["H"], L["P"], L["N"], L["G"], L["k"]
    init = rng.standard_normal((2, H, N, P))
    dy = rng.standard_normal((2, 5, H, P))
    g = L["X"].reshape(-1, 6) @ L["W_r"].T
    srt = -np.sort(-g, axis=1)
    assert (srt[:, k - 1] - srt[:, k]).min() > 1e-3
    got = O.layer_bwd(L["X"], L["W_r"], L["W_dt"], L["b_dt"], L["A"], L["W_exp"], H, P, N, G, k, dy, init)

    def loss(X=L["X"], W_r=L["W_r"], W_dt=L["W_dt"], b_dt=L["b_dt"], A=L["A"], W_exp=L["W_exp"], init=init):
        y = O.layer_fwd(X, W_r, W_dt, b_dt, A, W_exp, H, P, N, G, k, init=init)["y"]
        return float((dy * y).sum())

    args = dict(X=L["X"], W_r=L["W_r"], W_dt=L["W_dt"], b_dt=L["b_dt"], A=L["A"], W_exp=L["W_exp"], init=init)
    names = dict(X="dX", W_r="dW_r", W_dt="dW_dt", b_dt="db_dt", A="dA", W_exp="dW_exp", init="dinit")
    eps = 1e-6
    for name, arr in args.items():
        num = np.zeros(arr.shape)
        for ix in np.ndindex(arr.shape):
            hi, lo = arr.copy(), arr.copy()
            hi[ix] += eps
            lo[ix] -= eps
            num[ix] = (loss(**{name: hi}) - loss(**{name: lo})) / (2 * eps)
        np.testing.assert_allclose(got[names[name]], num, rtol=1e-5, atol=1e-7, err_msg=name)


def test_scan_backward_per_token_transition():
    # with a [T,H] transition the dA gradient is per token; central differences on each entry
    rng = np.random.default_rng(17)
    T, k, H, P, N = 5, 1, 2, 2, 3
    Bpi, Xs, Ct, dt, _ = _rand_streams(rng, T, k, H, P, 2, N)
    At = -np.exp(rng.uniform(0, math.log(16), size=(T, H)))
    dy = rng.standard_normal((T, H, P))
    got = O.scan_backward(Bpi, Xs, Ct, dt, At, dy)
    eps = 1e-6
    for idx in np.ndindex(At.shape):
        hi, lo = At.copy(), At.copy()
        hi[idx] += eps
        lo[idx] -= eps
        num = (_loss(Bpi, Xs, Ct, dt, hi, dy, None) - _loss(Bpi, Xs, Ct, dt, lo, dy, None)) / (2 * eps)
        assert abs(got["dA"][idx] - num) <= 1e-6 * max(1.0, abs(num))


# ----------------------------------------------------------------------------- expert-mixed transition

def test_mixed_A_is_the_router_weighted_mean():
    # A~[t,h] = sum_j pi_tj A_exp[K_tj, h], written out term by term
    rng = np.random.default_rng(8)
    M, k, E, H = 6, 3, 5, 4
    idx = np.array([rng.permutation(E)[:k] for _ in range(M)])
    w = rng.dirichlet(np.ones(k), size=M)
    A_exp = -np.exp(rng.uniform(0, math.log(16), size=(E, H)))
    At = O.mixed_A(idx, w, A_exp)
    for t in range(M):
        for h in range(H):
            assert abs(At[t, h] - sum(w[t, j] * A_exp[idx[t, j], h] for j in range(k))) < 1e-12
    # a convex combination of negative values: strictly between the most and least negative expert values
    assert (At < 0).all()
    assert (At >= A_exp.min(axis=0) - 1e-12).all() and (At <= A_exp.max(axis=0) + 1e-12).all()


def test_mixed_A_with_equal_experts_is_the_shared_layer():
    # every expert carrying the same A row reduces the mixed transition to the shared one (the weights sum to 1)
    L = _small_layer(np.random.default_rng(9), E=4, k=2)
    E = L["W_exp"].shape[0]
    ref = _fwd(L)
    mixed = O.layer_fwd(L["X"], L["W_r"], L["W_dt"], L["b_dt"], None, L["W_exp"], L["H"], L["P"], L["N"], L["G"],
                        L["k"], A_exp=np.tile(L["A"], (E, 1)))
    np.testing.assert_allclose(mixed["y"], ref["y"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(mixed["final"], ref["final"], rtol=1e-11, atol=1e-12)


def test_mixed_A_decay_closed_form():
    # a carried state with no injection (the B rows of every expert are zero) decays by
    # prod_t exp(dt_t (pi_t0 A_e0 + pi_t1 A_e1)), read out by C~; checked against that product
    rng = np.random.default_rng(10)
    L = _small_layer(rng, B=1, T=5, E=3, k=2)
    H, P, N, G = L["H"], L["P"], L["N"], L["G"]
    L["W_exp"][:, H * P:H * P + G * N] = 0.0
    E = L["W_exp"].shape[0]
    A_exp = -np.exp(rng.uniform(0, math.log(16), size=(E, H)))
    init = rng.standard_normal((1, H, N, P))
    out = O.layer_fwd(L["X"], L["W_r"], L["W_dt"], L["b_dt"], None, L["W_exp"], H, P, N, G, L["k"], init=init,
                      A_exp=A_exp)
    g = L["X"][0] @ L["W_r"].T
    dt = np.clip(np.log1p(np.exp(L["X"][0] @ L["W_dt"].T + L["b_dt"])), 1e-3, 0.1)
    decay = np.ones(H)
    for t in range(5):
        top = np.argsort(-g[t].astype(np.float32), kind="stable")[:2]
        e0, e1 = top
        p1 = 1.0 / (1.0 + np.exp(g[t, e0] - g[t, e1]))
        decay = decay * np.exp(dt[t] * ((1 - p1) * A_exp[e0] + p1 * A_exp[e1]))
    np.testing.assert_allclose(out["final"][0], decay[:, None, None] * init[0], rtol=1e-12)
    gh = O.group_of(H, G)
    Ct = out["Ct"][4]
    np.testing.assert_allclose(out["y"][0, 4], np.einsum("hn,hnp->hp", Ct[gh], decay[:, None, None] * init[0]),
                               rtol=1e-10, atol=1e-12)


def test_mixed_A_steps_equal_layer_fwd():
    rng = np.random.default_rng(11)
    L = _small_layer(rng, B=2, T=6, E=4, k=2)
    A_exp = -np.exp(rng.uniform(0, math.log(16), size=(4, L["H"])))
    full = O.layer_fwd(L["X"], L["W_r"], L["W_dt"], L["b_dt"], None, L["W_exp"], L["H"], L["P"], L["N"], L["G"],
                       L["k"], A_exp=A_exp)
    state = np.zeros((2, L["H"], L["N"], L["P"]))
    for t in range(6):
        y, state, _ = O.step(L["X"][:, t], L["W_r"], L["W_dt"], L["b_dt"], None, L["W_exp"], L["H"], L["P"], L["N"],
                             L["G"], L["k"], state, A_exp=A_exp)
        np.testing.assert_allclose(y, full["y"][:, t], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(state, full["final"], rtol=1e-11, atol=1e-12)


def test_chunked_with_per_token_A_equals_sequential():
    rng = np.random.default_rng(12)
    Bpi, Xs, Ct, dt, A = _rand_streams(rng, 37, 2, 3, 4, 3, 5)
    At = -np.exp(rng.uniform(0, math.log(16), size=(37, 3)))
    ys, hs = O.scan_sequential(Bpi, Xs, Ct, dt, At)
    yc, Hs, hc = O.scan_chunked(Bpi, Xs, Ct, dt, At, 16)
    np.testing.assert_allclose(yc, ys, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(hc, hs, rtol=1e-10, atol=1e-12)
    yb = O.scan_bruteforce(Bpi, Xs, Ct, dt, At)
    np.testing.assert_allclose(yb, ys, rtol=1e-10, atol=1e-12)


def test_out_proj_matches_elementwise_dot_products():
    # out[m][d] = sum_c y[m][c] W_out[d][c], written out term by term; a transposed W_out fails the shapes
    # (D != H*P) and, for a square W_out, the values
    rng = np.random.default_rng(5)
    for M, HP, D in ((7, 6, 5), (4, 5, 5)):
        y = rng.standard_normal((M, HP))
        W_out = rng.standard_normal((D, HP))
        out = O.out_proj(y, W_out)
        assert out.shape == (M, D)
        for m in range(M):
            for d in range(D):
                assert abs(out[m, d] - sum(y[m, c] * W_out[d, c] for c in range(HP))) < 1e-12


def test_out_proj_identity_and_selection():
    # W_out = I returns y; a row-selection W_out returns the selected columns of y, in W_out's row order
    rng = np.random.default_rng(6)
    y = rng.standard_normal((3, 2, 8))
    np.testing.assert_array_equal(O.out_proj(y, np.eye(8)), y)
    sel = [5, 0, 7]
    W_out = np.zeros((3, 8))
    W_out[np.arange(3), sel] = 1.0
    np.testing.assert_array_equal(O.out_proj(y, W_out), y[..., sel])


def test_split_streams_layout():
    H, P, G, N = 2, 3, 1, 2
    z = np.arange(H * P + 2 * G * N, dtype=float)
    x, B, C = O.split_streams(z, H, P, G, N)
    assert x.tolist() == [[0, 1, 2], [3, 4, 5]]
    assert B.tolist() == [[6, 7]]
    assert C.tolist() == [[8, 9]]


def test_group_map():
    assert O.group_of(4, 2).tolist() == [0, 0, 1, 1]
    assert O.group_of(4, 1).tolist() == [0, 0, 0, 0]
    assert O.group_of(3, 3).tolist() == [0, 1, 2]


def test_polynomial_degree_three_single_expert():
    """Theorem 3.5's remark: with one expert, T = 1, A = 0, N = P = 1 the output is a polynomial of
    degree 3 in X; the layer is homogeneous of degree 3 (B, C and x are each linear in X)."""
    rng = np.random.default_rng(5)
    L = _small_layer(rng, B=1, T=1, D=5, H=1, P=1, N=1, E=1, k=1)
    L["A"] = np.zeros(1)
    y1 = _fwd(L)["y"]
    for lam in (2.0, -0.5, 3.0):
        yl = _fwd(L, X=lam * L["X"])["y"]
        np.testing.assert_allclose(yl, lam ** 3 * y1, rtol=1e-12)
    # and it equals (C.X)(B.X)(x.X) directly
    w = L["W_exp"][0]
    Xv = L["X"][0, 0]
    assert abs(y1[0, 0, 0, 0] - (w[0] @ Xv) * (w[1] @ Xv) * (w[2] @ Xv)) < 1e-12


def test_single_expert_reduces_to_plain_ssm_streams():
    """(a) E = 1, k = 1: pi = 1, the mixed streams are the expert's own B, x, C."""
    rng = np.random.default_rng(6)
    L = _small_layer(rng, E=1, k=1)
    out = _fwd(L)
    assert np.all(out["w"] == 1.0) and np.all(out["idx"] == 0)
    x, B, C = O.split_streams(out["z"], L["H"], L["P"], L["G"], L["N"])
    assert np.array_equal(out["Bpi"], B) and np.array_equal(out["Xs"], x)
    assert np.array_equal(out["Ct"], C[:, 0])


def test_identical_experts_equal_unrouted_ssm():
    """(b) all experts identical: the output equals the unrouted single SSM whatever the routing,
    because the renormalised weights sum to one."""
    rng = np.random.default_rng(7)
    L = _small_layer(rng, E=1, k=1)
    ref = _fwd(L)
    for E, k in ((4, 2), (6, 3), (5, 1)):
        LE = dict(L, W_exp=np.repeat(L["W_exp"], E, axis=0), k=k,
                  W_r=rng.standard_normal((E, L["X"].shape[2])))
        out = _fwd(LE)
        assert len(np.unique(out["idx"])) > 1 or E == 1
        np.testing.assert_allclose(out["y"], ref["y"], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(out["final"], ref["final"], rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------- the recurrence

def test_geometric_closed_form_one_injection():
    """Constant transition a, one injection at s = 0, constant readout: y_t = a^t (C . B_0) x_0,
    and a carried state alone decays as y_t = a^(t+1) C^T h_init."""
    T, H, P, N = 10, 1, 3, 4
    rng = np.random.default_rng(8)
    Bpi = np.zeros((T, 1, H, N)); Xs = np.zeros((T, 1, H, P))
    Bpi[0, 0, 0] = rng.standard_normal(N); Xs[0, 0, 0] = rng.standard_normal(P)
    c = rng.standard_normal(N)
    Ct = np.broadcast_to(c, (T, H, N)).copy()
    dt = np.full((T, H), 0.05); A = np.array([-3.0]); a = math.exp(-0.15)
    y, hT = O.scan_sequential(Bpi, Xs, Ct, dt, A)
    for t in range(T):
        np.testing.assert_allclose(y[t, 0], a ** t * (c @ Bpi[0, 0, 0]) * Xs[0, 0, 0], rtol=1e-13)
    np.testing.assert_allclose(hT[0], a ** (T - 1) * np.outer(Bpi[0, 0, 0], Xs[0, 0, 0]), rtol=1e-13)
    h0 = rng.standard_normal((H, N, P))
    y0, _ = O.scan_sequential(np.zeros_like(Bpi), np.zeros_like(Xs), Ct, dt, A, init=h0)
    for t in range(T):
        np.testing.assert_allclose(y0[t, 0], a ** (t + 1) * (c @ h0[0]), rtol=1e-13)


@pytest.mark.parametrize("G", [4, 2, 1])
def test_sequential_equals_bruteforce_semiseparable(G):
    """(c) the token-by-token recurrence equals the materialised semiseparable product."""
    rng = np.random.default_rng(9 + G)
    T, k, H, P, N = 13, 2, 4, 3, 5
    Bpi, Xs, Ct, dt, A = _rand_streams(rng, T, k, H, P, G, N)
    init = rng.standard_normal((H, N, P))
    y, _ = O.scan_sequential(Bpi, Xs, Ct, dt, A, init)
    yb = O.scan_bruteforce(Bpi, Xs, Ct, dt, A, init)
    np.testing.assert_allclose(y, yb, rtol=1e-12, atol=1e-12)


def test_groups_equal_replicated_heads():
    """G < H shares B and C across the heads of a group: identical to G = H with the group's streams
    copied to each of its heads (pins the head -> group index)."""
    rng = np.random.default_rng(10)
    T, k, H, P, N, G = 9, 2, 6, 3, 4, 2
    Bpi, Xs, Ct, dt, A = _rand_streams(rng, T, k, H, P, G, N)
    y, hT = O.scan_sequential(Bpi, Xs, Ct, dt, A)
    rep = np.repeat(np.arange(G), H // G)
    y2, hT2 = O.scan_sequential(Bpi[:, :, rep], Xs, Ct[:, rep], dt, A)
    np.testing.assert_array_equal(y, y2)
    np.testing.assert_array_equal(hT, hT2)


@pytest.mark.parametrize("T,Q", [(64, 16), (70, 16), (5, 16), (33, 8)])
def test_chunked_equals_sequential(T, Q):
    rng = np.random.default_rng(T * 100 + Q)
    k, H, P, N, G = 2, 3, 4, 5, 3
    Bpi, Xs, Ct, dt, A = _rand_streams(rng, T, k, H, P, G, N)
    init = rng.standard_normal((H, N, P))
    y, hT = O.scan_sequential(Bpi, Xs, Ct, dt, A, init)
    yc, Hs, hc = O.scan_chunked(Bpi, Xs, Ct, dt, A, Q, init)
    np.testing.assert_allclose(yc, y, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(hc, hT, rtol=1e-11, atol=1e-12)
    for c in range(Hs.shape[0]):
        if c == 0:
            np.testing.assert_array_equal(Hs[0], init)
        else:
            _, hprev = O.scan_sequential(Bpi[:c * Q], Xs[:c * Q], Ct[:c * Q], dt[:c * Q], A, init)
            np.testing.assert_allclose(Hs[c], hprev, rtol=1e-11, atol=1e-12)


def test_thm33_bibo_bound():
    """(d) Theorem 3.3: with h_0 = 0 and a_t <= rho < 1, ||h_t|| <= (1 - rho^t)/(1 - rho) max ||U~||
    and ||y_t|| <= max ||C~|| times that bound; equality for a constant injection and transition."""
    rng = np.random.default_rng(11)
    T, k, H, P, N = 40, 2, 3, 4, 6
    Bpi, Xs, Ct, dt, A = _rand_streams(rng, T, k, H, P, H, N)
    U = np.einsum("tjhn,tjhp->thnp", Bpi, Xs)
    Unorm = np.linalg.norm(U.reshape(T, H, -1), axis=2).max(axis=0)      # per head
    Cnorm = np.linalg.norm(Ct, axis=2).max(axis=0)
    rho = np.exp(dt * A).max(axis=0)
    for t in range(1, T + 1):
        y, h = O.scan_sequential(Bpi[:t], Xs[:t], Ct[:t], dt[:t], A)
        bound = (1 - rho ** t) / (1 - rho) * Unorm
        hn = np.linalg.norm(h.reshape(H, -1), axis=1)
        assert np.all(hn <= bound * (1 + 1e-12))
        assert np.all(np.linalg.norm(y[t - 1], axis=1) <= Cnorm * bound * (1 + 1e-12))
    # equality case: same positive injection every step, constant a
    u = np.abs(rng.standard_normal((1, 1, 1, N))); xv = np.abs(rng.standard_normal((1, 1, 1, P)))
    Bc = np.repeat(u, T, 0); Xc = np.repeat(xv, T, 0)
    dtc = np.full((T, 1), 0.04); Ac = np.array([-2.0]); a = math.exp(-0.08)
    _, h = O.scan_sequential(Bc, Xc, np.zeros((T, 1, N)), dtc, Ac)
    np.testing.assert_allclose(np.linalg.norm(h), (1 - a ** T) / (1 - a) * np.linalg.norm(np.outer(u, xv)),
                               rtol=1e-12)


def _dense_streams(rng, T, E, H, P, G, N):
    xE = rng.standard_normal((T, E, H, P))
    BE = rng.standard_normal((T, E, G, N))
    CE = rng.standard_normal((T, E, G, N))
    return xE, BE, CE


def test_thm34_static_routing_equivalence_and_counts():
    """(e) Theorem 3.4: with static routing and equal readouts the separated designs and the mixed
    layer coincide; the mixed layer runs 1 recurrence, separated-k runs k, separated-E runs E
    (trajectory counts of the efficiency table)."""
    rng = np.random.default_rng(12)
    T, E, k, H, P, N = 20, 4, 2, 2, 3, 4
    xE, BE, CE = _dense_streams(rng, T, E, H, P, H, N)
    CE[:] = CE[:, :1]                                                     # equal readouts
    K = np.array([2, 0]); pi = np.array([0.7, 0.3])                       # static routing
    dt = rng.uniform(1e-3, 0.1, size=(T, H)); A = -np.exp(rng.uniform(0, 2, size=H))
    pi_dense = np.zeros((T, E)); pi_dense[:, K] = pi
    y_sepE, _, nE = O.scan_separated_dense(xE, BE, CE, pi_dense, dt, A)
    Bk, Xk, Ck = BE[:, K], xE[:, K], CE[:, K]
    Bpi = pi[None, :, None, None] * Bk
    Cpi = pi[None, :, None, None] * Ck
    mixed_stats = {}
    y_mix, _ = O.scan_sequential(Bpi, Xk, Cpi.sum(1), dt, A, stats=mixed_stats)
    y_sepk, _, nk = O.scan_separated_k(Bk, Xk, Cpi, dt, A)
    # separated-E keeps all E experts running but reads out only the active ones: with the inactive
    # experts' contribution weighted 0 it matches as well
    np.testing.assert_allclose(y_sepk, y_mix, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y_sepE, y_mix, rtol=1e-12, atol=1e-12)
    rows = [l.split() for l in open(os.path.join(GOLD, "efficiency_table_trajectories.txt"))
            if not l.startswith("#")]
    counts = {r[0]: int(r[3]) for r in rows}
    # the counts are state updates the oracle actually performed, divided by T
    assert mixed_stats["updates"] == T * counts["mixed"]
    _, _, n1 = O.scan_separated_k(Bk[:, :1], Xk[:, :1], Cpi[:, :1], dt, A)
    assert n1 == counts["separated_k"]
    _, _, n4 = O.scan_separated_dense(xE, BE, CE, pi_dense, dt, A)
    assert n4 == counts["separated_E"] == E and nk == k
    # the mixed layer's count does not grow with k (one trajectory whatever the number of slots)
    s1, s2 = {}, {}
    O.scan_sequential(Bpi[:, :1], Xk[:, :1], Cpi[:, :1].sum(1), dt, A, stats=s1)
    O.scan_sequential(Bpi, Xk, Cpi.sum(1), dt, A, stats=s2)
    assert s1["updates"] == s2["updates"] == T


def test_thm34_dynamic_routing_bound():
    """Theorem 3.4 under dynamic routing: ||Y_sep - Y_mix|| <= sum_e pi_te ||C^(e)|| ||h^(e) - h||."""
    rng = np.random.default_rng(13)
    T, E, k, H, P, N = 25, 4, 2, 1, 3, 4
    xE, BE, CE = _dense_streams(rng, T, E, H, P, H, N)
    g = rng.standard_normal((T, E))
    idx = O.topk_select(g, k); w = O.topk_weights(g, idx)
    pi_dense = np.zeros((T, E))
    np.put_along_axis(pi_dense, idx, w, axis=1)
    dt = rng.uniform(1e-3, 0.1, size=(T, H)); A = np.array([-1.5])
    y_sep, hs, _ = O.scan_separated_dense(xE, BE, CE, pi_dense, dt, A)
    Bk = np.take_along_axis(BE, idx[:, :, None, None], 1)
    Xk = np.take_along_axis(xE, idx[:, :, None, None], 1)
    Ck = np.take_along_axis(CE, idx[:, :, None, None], 1)
    Bpi = w[:, :, None, None] * Bk
    Ct = (w[:, :, None, None] * Ck).sum(1)
    for t in range(1, T + 1):
        y_mix, h = O.scan_sequential(Bpi[:t], Xk[:t], Ct[:t], dt[:t], A)
        lhs = np.linalg.norm(y_sep[t - 1, 0] - y_mix[t - 1, 0])
        rhs = sum(pi_dense[t - 1, e] * np.linalg.norm(CE[t - 1, e, 0]) *
                  np.linalg.norm(hs[t - 1, e, 0] - h[0], 2) for e in range(E))
        assert lhs <= rhs * (1 + 1e-12) + 1e-13


# ----------------------------------------------------------------------------- the layer and decode

def test_layer_fwd_state_handoff():
    rng = np.random.default_rng(14)
    L = _small_layer(rng, T=10)
    full = _fwd(L)
    a = _fwd(L, X=L["X"][:, :6])
    b = _fwd(L, X=L["X"][:, 6:], init=a["final"])
    np.testing.assert_allclose(np.concatenate([a["y"], b["y"]], 1), full["y"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b["final"], full["final"], rtol=1e-12, atol=1e-13)


def test_steps_equal_layer_fwd():
    """T decode steps from a zero state reproduce the layer's forward pass."""
    rng = np.random.default_rng(15)
    L = _small_layer(rng, T=7, G=2)
    full = _fwd(L)
    Bsz, T = L["X"].shape[:2]
    state = np.zeros((Bsz, L["H"], L["N"], L["P"]))
    for t in range(T):
        y, state, idx = O.step(L["X"][:, t], L["W_r"], L["W_dt"], L["b_dt"], L["A"], L["W_exp"],
                               L["H"], L["P"], L["N"], L["G"], L["k"], state)
        np.testing.assert_allclose(y, full["y"][:, t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(state, full["final"], rtol=1e-12, atol=1e-13)


def test_forced_routing_replays_given_indices():
    rng = np.random.default_rng(16)
    L = _small_layer(rng, B=1, T=5, E=4, k=2)
    base = _fwd(L)
    forced = -np.ones((1, 5, 2), dtype=np.int64)
    forced[0, 3] = [3, 1]
    out = _fwd(L, forced_idx=forced)
    assert list(out["idx"][3]) == [3, 1]
    np.testing.assert_array_equal(out["idx"][[0, 1, 2, 4]], base["idx"][[0, 1, 2, 4]])
    np.testing.assert_allclose(out["y"][0, :3], base["y"][0, :3], rtol=1e-12, atol=1e-14)
