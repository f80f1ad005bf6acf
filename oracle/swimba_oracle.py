"""Swimba layer oracle: a plain, slow, fp64 CPU restatement of what the layer computes.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the CUDA library and imports nothing
from it; its inputs are plain numpy arrays.

Sources (all describe arXiv 2603.06938, "Swimba: Switch Mamba Model Scales State Space Models"):
  [notes]  papernotes.org NeurIPS 2026 notes on Swimba, Method ("overall framework", its flowchart,
           key design 1 with the two display equations, key design 2 with Theorems 3.3/3.4,
           key design 3 with Theorem 3.5) and the efficiency table.
  [gist]   gist.science English summary, Technical Summary section 2 "Methodology",
           "Architecture Details" and "Theoretical Guarantees".
Where the pages leave a step open the reading used here is stated beside the step.

Notation: tokens t, batch row b, heads h (group g(h) = h // (H // G)), experts e, slots j < k.
Shapes: X [B,T,D]; W_r [E,D]; W_dt [H,D]; b_dt [H]; A [H]; W_exp [E, H*P + 2*G*N, D].
Everything is computed in float64.
"""
import numpy as np


# ----------------------------------------------------------------------------- router

def softplus(v):
    """log(1 + e^v), evaluated without overflow."""
    return np.logaddexp(0.0, v)


def router_logits(X, W_r):
    """g_t = W_r X_t: the token router R(X_t) of [notes] Method, flowchart node "token router".

    Reading: a linear router without bias, temperature 1.
    """
    return X @ W_r.T


def dt_proj(X, W_dt, b_dt, dt_min=1e-3, dt_max=0.1):
    """dt_{t,h} = clamp(softplus(W_dt[h] . X_t + b_dt[h]), dt_min, dt_max).

    The pages fix A as shared by all experts ([notes] key design 2; [gist] Architecture Details);
    the step size dt that discretises it comes from one shared (non-expert) projection, so the
    transition a_t = exp(dt_t A_h) is shared by every expert while staying input-dependent.
    """
    return np.clip(softplus(X @ W_dt.T + b_dt), dt_min, dt_max)


def topk_select(g, k):
    """Active set K_t of [notes] key design 1 ("usually top-k sparse"): the indices of the k
    largest entries of each row of g, largest first, equal values ordered by lower expert index.

    The caller passes g in the precision the decision is taken in (the kernels take it on
    fp32 logits; pass g.astype(np.float32) for a like-for-like decision).
    """
    g = np.asarray(g)
    # a stable sort of -g keeps equal values in index order, i.e. ties go to the lower index
    order = np.argsort(-g, axis=-1, kind="stable")
    return order[..., :k].astype(np.int64)


def topk_weights(g, idx):
    """pi_{t,j} = softmax(g_t) restricted to K_t and renormalised over the k winners
    ([notes] key design 1: pi_t = softmax(g_t); renormalisation over K_t is the reading used).
    Equal to exp(g_{K_j}) / sum_j' exp(g_{K_j'})."""
    sel = np.take_along_axis(g, idx, axis=-1)
    m = sel.max(axis=-1, keepdims=True)
    ex = np.exp(sel - m)
    return ex / ex.sum(axis=-1, keepdims=True)


def router(X, W_r, W_dt, b_dt, k, decision_dtype=np.float32, forced_idx=None):
    """Router stage on flattened tokens X [M, D]: returns (g, dt, topk_idx, topk_w).

    forced_idx (optional [M,k]) replaces the active set on rows where it is >= 0; the tests use it
    to replay the kernel's choice on near-tied tokens, where either choice is a correct top-k.
    """
    g = router_logits(X, W_r)
    dt = dt_proj(X, W_dt, b_dt)
    idx = topk_select(g.astype(decision_dtype), k)
    if forced_idx is not None:
        rows = forced_idx[:, 0] >= 0
        idx[rows] = forced_idx[rows]
    w = topk_weights(g, idx)
    return g, dt, idx, w


# ----------------------------------------------------------------------------- experts and mixing

def split_streams(z, H, P, G, N):
    """Split one expert projection z [..., H*P + 2*G*N] into the candidate streams
    (x [...,H,P], B [...,G,N], C [...,G,N]) of [notes] key design 1.

    Reading of the stream shapes: B and C are N-vectors and x a P-vector per head (the notes'
    "B in R^{N x P}" cannot give a P-vector readout); G groups, G = H meaning every head has its own.
    """
    HP, GN = H * P, G * N
    x = z[..., :HP].reshape(z.shape[:-1] + (H, P))
    B = z[..., HP:HP + GN].reshape(z.shape[:-1] + (G, N))
    C = z[..., HP + GN:HP + 2 * GN].reshape(z.shape[:-1] + (G, N))
    return x, B, C


def expert_proj(X, W_exp, idx):
    """Candidate streams of the active experts: z[t, j] = W_exp[K_tj] X_t  ([notes] key design 1:
    every expert applies its own linear projection to the same X_t).  X [M,D] -> z [M,k,W_e]."""
    M, k = idx.shape
    z = np.zeros((M, k, W_exp.shape[1]))
    for e in range(W_exp.shape[0]):
        rows, slots = np.nonzero(idx == e)
        if rows.size:
            z[rows, slots] = X[rows] @ W_exp[e].T
    return z


def mix(z, w, H, P, G, N):
    """Parameter-space mixing ([notes] key design 1, first display equation; [gist] Parameter Mixing):
      U~_t = sum_j pi_tj B_t^(j) x_t^(j)T   kept factored as (Bpi = pi B, Xs = x) per slot,
      C~_t = sum_j pi_tj C_t^(j).
    Returns Bpi [M,k,G,N], Xs [M,k,H,P], Ct [M,G,N] and the per-slot pi C [M,k,G,N]."""
    x, B, C = split_streams(z, H, P, G, N)
    Bpi = w[:, :, None, None] * B
    Cpi = w[:, :, None, None] * C
    return Bpi, x, Cpi.sum(axis=1), Cpi


def mixed_A(idx, w, A_exp):
    """Expert-mixed diagonal transition ([notes] limitations and outlook: parameter-space mixing carried over
    to the diagonal of the transition A, with Lyapunov stability kept):
        A~_t,h = sum_j pi_tj A^(K_tj)_h,        a_t = exp(dt_t A~_t)  for every head.
    Reading: one A^(e) per expert and head (Mamba-2's scalar-per-head diagonal), mixed with the same router
    weights as B and C; dt stays the one shared projection.  Every A^(e) < 0 makes A~_t a convex combination
    of negative values, so 0 < a_t < 1: the transition stays a contraction and the recurrence is still one
    trajectory.  idx [M,k], w [M,k], A_exp [E,H]; returns A~ [M,H]."""
    return np.einsum("mj,mjh->mh", w, np.asarray(A_exp)[idx])


# ----------------------------------------------------------------------------- the single recurrence

def group_of(H, G):
    return np.arange(H) // (H // G)


def _count_update(stats):
    """Counts one state update of one trajectory (all heads at once) when a stats dict is passed."""
    if stats is not None:
        stats["updates"] = stats.get("updates", 0) + 1


def log_decay(dt, A):
    """dt_t A_h per token and head, [T,H]: A is the shared [H] vector, or a per-token [T,H] array (the
    expert-mixed A~ of mixed_A)."""
    return np.asarray(dt) * np.asarray(A)


def scan_sequential(Bpi, Xs, Ct, dt, A, init=None, stats=None):
    """The single-trajectory recurrence, token by token ([notes] key design 1, second display
    equation; [gist] "h_t = A h_{t-1} + sum pi B X"):
        h_t = a_t h_{t-1} + sum_j Bpi_tj (x) Xs_tj,     y_t = C~_t^T h_t,     a_t = exp(dt_t A_h).
    Reading: no dt factor on the injection (the pages' equation has none).

    One batch row: Bpi [T,k,G,N], Xs [T,k,H,P], Ct [T,G,N], dt [T,H], A [H] (or [T,H], see log_decay),
    init [H,N,P] or None.
    Returns y [T,H,P] and the final state [H,N,P].  stats (optional dict): "updates" is increased by one
    for every state update, so a T-token call adds T (one trajectory).
    """
    T, k, H, P = Xs.shape
    G, N = Bpi.shape[2], Bpi.shape[3]
    g = group_of(H, G)
    h = np.zeros((H, N, P)) if init is None else np.array(init, dtype=np.float64)
    y = np.zeros((T, H, P))
    dA = log_decay(dt, A)
    for t in range(T):
        a = np.exp(dA[t])                                               # [H]
        U = np.einsum("jhn,jhp->hnp", Bpi[t][:, g], Xs[t])              # rank-k injection per head
        h = a[:, None, None] * h + U
        _count_update(stats)
        y[t] = np.einsum("hn,hnp->hp", Ct[t][g], h)
    return y, h


def scan_backward(Bpi, Xs, Ct, dt, A, dy, init=None):
    """Gradients of L = sum_t <dy_t, y_t> for one batch row of scan_sequential, by the adjoint recurrence
    run backwards in time (reverse-mode differentiation of [notes] key design 1's second display equation):
        lam_t    = dL/dh_t = C~_t (x) dy_t + a_{t+1} lam_{t+1}          (lam = 0 after the last token)
        dBpi_tj  = lam_t Xs_tj          dXs_tj = lam_t^T Bpi_tj          dC~_t = h_t dy_t
        g_t      = a_t <lam_t, h_{t-1}>  (the gradient of the log-decay dA_t = dt_t A)
        d dt_t   = g_t A_h,   dA_h = sum_t g_t dt_t,   d init = a_0 lam_0 (with h_{-1} = init).
    With G < H groups the B and C~ gradients sum over the heads of a group.  A may be [H] or [T,H] (then dA
    is [T,H], the gradient of each token's transition).
    Returns a dict: dBpi [T,k,G,N], dXs [T,k,H,P], dCt [T,G,N], ddt [T,H], dA, dinit [H,N,P]."""
    T, k, H, P = Xs.shape
    G, N = Bpi.shape[2], Bpi.shape[3]
    g = group_of(H, G)
    dAt = log_decay(dt, A) * np.ones((T, H))
    a = np.exp(dAt)                                                    # [T,H]
    hs = np.zeros((T + 1, H, N, P))                                    # hs[t + 1] = h_t, hs[0] = init
    if init is not None:
        hs[0] = init
    for t in range(T):
        U = np.einsum("jhn,jhp->hnp", Bpi[t][:, g], Xs[t])
        hs[t + 1] = a[t][:, None, None] * hs[t] + U
    dBpi = np.zeros(Bpi.shape)
    dXs = np.zeros(Xs.shape)
    dCt = np.zeros(Ct.shape)
    gdA = np.zeros((T, H))
    lam = np.zeros((H, N, P))
    for t in range(T - 1, -1, -1):
        if t + 1 < T:
            lam = a[t + 1][:, None, None] * lam
        lam = lam + np.einsum("hn,hp->hnp", Ct[t][g], dy[t])
        for gi in range(G):
            heads = np.nonzero(g == gi)[0]
            dBpi[t, :, gi] = np.einsum("hnp,jhp->jn", lam[heads], Xs[t][:, heads])
            dCt[t, gi] = np.einsum("hnp,hp->n", hs[t + 1][heads], dy[t][heads])
        dXs[t] = np.einsum("hnp,jhn->jhp", lam, Bpi[t][:, g])
        gdA[t] = a[t] * np.einsum("hnp,hnp->h", lam, hs[t])
    ddt = gdA * (np.ones((T, H)) * np.asarray(A))
    dA = (gdA * dt).sum(axis=0) if np.ndim(A) == 1 else gdA * dt
    dinit = a[0][:, None, None] * lam
    return dict(dBpi=dBpi, dXs=dXs, dCt=dCt, ddt=ddt, dA=dA, dinit=dinit)


def scan_bruteforce(Bpi, Xs, Ct, dt, A, init=None):
    """The same layer as one materialised semiseparable matrix product (quadratic in T):
        y_t = sum_{s<=t} (prod_{r=s+1..t} a_r) sum_j (C~_t . Bpi_sj) Xs_sj  +  (prod_{r<=t} a_r) C~_t^T h_init.
    Structure preservation ([notes] key design 1, Theorem 3.1): the mixed layer is one selective SSM,
    whose input-output map is this lower-triangular matrix.  For tiny T only."""
    T, k, H, P = Xs.shape
    g = group_of(H, G=Bpi.shape[2])
    dA = log_decay(dt, A)                                              # [T,H]
    y = np.zeros((T, H, P))
    for t in range(T):
        for s in range(t + 1):
            decay = np.exp(dA[s + 1:t + 1].sum(axis=0))                # [H]
            for j in range(k):
                score = np.einsum("hn,hn->h", Ct[t][g], Bpi[s, j][g])   # C~_t . Bpi_sj
                y[t] += (decay * score)[:, None] * Xs[s, j]
        if init is not None:
            decay0 = np.exp(dA[:t + 1].sum(axis=0))
            y[t] += decay0[:, None] * np.einsum("hn,hnp->hp", Ct[t][g], init)
    return y


def scan_chunked(Bpi, Xs, Ct, dt, A, Q, init=None):
    """The same recurrence solved chunk by chunk, the SSD decomposition the pages reuse
    ([notes] overall framework: Mamba-2's chunked SSD algorithm, reused unchanged):
      cs_t   = sum of dt*A from the chunk start to t (inclusive)
      y_t    = sum_{s in chunk, s<=t} exp(cs_t - cs_s) sum_j (C~_t . Bpi_sj) Xs_sj      (intra-chunk)
             + exp(cs_t) C~_t^T H_c                                                     (carried state)
      S_c    = sum_{s in chunk} exp(cs_end - cs_s) sum_j Bpi_sj (x) Xs_sj               (chunk state)
      H_{c+1}= exp(cs_end) H_c + S_c,   H_0 = init or 0.
    Returns y [T,H,P], chunk-start states Hs [nc,H,N,P] (Hs[c] = H_c) and the final state."""
    T, k, H, P = Xs.shape
    G, N = Bpi.shape[2], Bpi.shape[3]
    g = group_of(H, G)
    nc = (T + Q - 1) // Q
    dA = log_decay(dt, A) * np.ones((T, H))
    Hc = np.zeros((H, N, P)) if init is None else np.array(init, dtype=np.float64)
    Hs = np.zeros((nc, H, N, P))
    y = np.zeros((T, H, P))
    for c in range(nc):
        t0, t1 = c * Q, min(T, (c + 1) * Q)
        cs = np.cumsum(dA[t0:t1], axis=0)                              # [L,H]
        Cg = Ct[t0:t1][:, g]                                           # [L,H,N]
        Bg = Bpi[t0:t1][:, :, g]                                       # [L,k,H,N]
        Xc = Xs[t0:t1]                                                 # [L,k,H,P]
        L = t1 - t0
        Hs[c] = Hc
        scores = np.einsum("thn,sjhn->tsjh", Cg, Bg)                   # [L,L,k,H]
        seg = cs[:, None, :] - cs[None, :, :]                          # [L,L,H] = cs_t - cs_s
        causal = np.tril(np.ones((L, L), dtype=bool))
        decay = np.where(causal[:, :, None], np.exp(np.where(causal[:, :, None], seg, 0.0)), 0.0)
        y[t0:t1] = np.einsum("tsh,tsjh,sjhp->thp", decay, scores, Xc)
        y[t0:t1] += np.exp(cs)[:, :, None] * np.einsum("thn,hnp->thp", Cg, Hc)
        wend = np.exp(cs[-1][None, :] - cs)                            # [L,H]
        S = np.einsum("sh,sjhn,sjhp->hnp", wend, Bg, Xc)
        Hc = np.exp(cs[-1])[:, None, None] * Hc + S
    return y, Hs, Hc


# ----------------------------------------------------------------------------- the separated contrast designs

def scan_separated_k(B, Xs, Cpi, dt, A, init=None):
    """"k scans": one trajectory per active slot j, driven by that slot's own (unscaled) injection
    B^(K_j) x^(K_j)T, read out with pi_j C^(K_j):
        h^(j)_t = a_t h^(j)_{t-1} + B_tj (x) Xs_tj,    y_t = sum_j (pi_tj C_tj)^T h^(j)_t.
    This is the separated-trajectory design of [notes] key design 1 restricted to the active slots;
    it runs k recurrences where the mixed layer runs one.  B [T,k,G,N], Cpi [T,k,G,N], init [k,H,N,P].
    Returns y [T,H,P], the k final states [k,H,N,P] and the number of trajectories it ran, counted as
    state updates per token."""
    T, k, H, P = Xs.shape
    G, N = B.shape[2], B.shape[3]
    g = group_of(H, G)
    h = np.zeros((k, H, N, P)) if init is None else np.array(init, dtype=np.float64)
    y = np.zeros((T, H, P))
    stats = {}
    for t in range(T):
        a = np.exp(dt[t] * A)
        for j in range(k):
            h[j] = a[:, None, None] * h[j] + np.einsum("hn,hp->hnp", B[t, j][g], Xs[t, j])
            _count_update(stats)
            y[t] += np.einsum("hn,hnp->hp", Cpi[t, j][g], h[j])
    return y, h, stats.get("updates", 0) // max(T, 1)


def scan_separated_dense(xE, BE, CE, pi_dense, dt, A):
    """MoE over separated SSMs ([notes] key design 1, the O(T E C_step) design; Theorem 3.4):
    every expert e keeps its own state h^(e), driven on every token by its own B^(e) x^(e)T, and the
    output is y_t = sum_e pi_te C^(e)_t^T h^(e)_t (pi_te = 0 off the active set).
    xE [T,E,H,P], BE/CE [T,E,G,N], pi_dense [T,E].  Returns y, the states [T,E,H,N,P] and the number
    of trajectories it ran, counted as state updates per token."""
    T, E, H, P = xE.shape
    G, N = BE.shape[2], BE.shape[3]
    g = group_of(H, G)
    h = np.zeros((E, H, N, P))
    hs = np.zeros((T, E, H, N, P))
    y = np.zeros((T, H, P))
    stats = {}
    for t in range(T):
        a = np.exp(dt[t] * A)
        for e in range(E):
            h[e] = a[:, None, None] * h[e] + np.einsum("hn,hp->hnp", BE[t, e][g], xE[t, e])
            _count_update(stats)
            y[t] += pi_dense[t, e] * np.einsum("hn,hnp->hp", CE[t, e][g], h[e])
        hs[t] = h
    return y, hs, stats.get("updates", 0) // max(T, 1)


# ----------------------------------------------------------------------------- the layer

def layer_fwd(X, W_r, W_dt, b_dt, A, W_exp, H, P, N, G, k, init=None, forced_idx=None,
              decision_dtype=np.float32, A_exp=None):
    """Forward pass of one Swimba token-mixer layer ([notes] Method flowchart: router -> expert
    projections -> parameter-space mixing -> one recurrence with the shared transition -> readout).

    X [B,T,D]; init [B,H,N,P] or None; forced_idx [B,T,k] or None (see router); A_exp [E,H] or None:
    with it the transition is the expert-mixed A~ of mixed_A (A is then not used).
    Returns a dict: y [B,T,H,P], final [B,H,N,P] and the stage values (g, dt, idx, w, z, Bpi, Xs,
    Ct, Cpi, At = the [M,H] or [H] transition used) flattened over tokens (row = b*T + t)."""
    Bsz, T, D = X.shape
    Xf = X.reshape(Bsz * T, D)
    fidx = None if forced_idx is None else forced_idx.reshape(Bsz * T, k)
    g, dt, idx, w = router(Xf, W_r, W_dt, b_dt, k, decision_dtype, fidx)
    z = expert_proj(Xf, W_exp, idx)
    Bpi, Xs, Ct, Cpi = mix(z, w, H, P, G, N)
    At = A if A_exp is None else mixed_A(idx, w, A_exp)
    y = np.zeros((Bsz, T, H, P))
    final = np.zeros((Bsz, H, N, P))
    for b in range(Bsz):
        r = slice(b * T, (b + 1) * T)
        y[b], final[b] = scan_sequential(Bpi[r], Xs[r], Ct[r], dt[r], At if A_exp is None else At[r],
                                         None if init is None else init[b])
    return dict(y=y, final=final, g=g, dt=dt, idx=idx, w=w, z=z, Bpi=Bpi, Xs=Xs, Ct=Ct, Cpi=Cpi, At=At)


def mix_bwd(dBpi, dXs, dCt, w, Bz, Cz):
    """Reverse of mix: the gradient of each slot's projection z = [x | B | C] and of its router weight, from the
    gradients of the mixed streams (Bpi = pi B, Xs = x, C~ = sum_j pi_j C_j):
        dz_j = [dXs_j | pi_j dBpi_j | pi_j dC~],    dpi_j = <B_j, dBpi_j> + <C_j, dC~>.
    dBpi [M,k,G,N], dXs [M,k,H,P], dCt [M,G,N], w [M,k], Bz/Cz [M,k,G,N]; returns dz [M,k,W_e], dpi [M,k]."""
    M, k = w.shape
    dz = np.concatenate([dXs.reshape(M, k, -1), (w[:, :, None, None] * dBpi).reshape(M, k, -1),
                         (w[:, :, None, None] * dCt[:, None]).reshape(M, k, -1)], axis=-1)
    dw = np.einsum("mjgn,mjgn->mj", Bz, dBpi) + np.einsum("mjgn,mgn->mj", Cz, dCt)
    return dz, dw


def router_bwd(w, dw):
    """Reverse of the renormalised softmax over the winners: with pi_j = e^{g_j} / sum_i e^{g_i} over K_t,
    dg_j = pi_j (dpi_j - sum_i pi_i dpi_i)  (the losers get no gradient)."""
    return w * (dw - (w * dw).sum(axis=1, keepdims=True))


def layer_bwd(X, W_r, W_dt, b_dt, A, W_exp, H, P, N, G, k, dy, init=None, forced_idx=None,
              decision_dtype=np.float32):
    """Gradients of L = sum <dy, y> for the layer of layer_fwd, with respect to X, every weight and the
    initial state, by reverse-mode differentiation of each stage in turn (the notes train the model: loss
    function / training strategy).  The active set K_t is held fixed (a top-k choice has no gradient); the dt
    clamp passes the gradient only strictly inside [1e-3, 0.1].
        scan   -> scan_backward: dBpi, dXs, dC~, d dt, dA, d init
        mix    -> dz = [dXs_j | pi_j dBpi_j | pi_j dC~] per slot;  dpi_j = <B_j, dBpi_j> + <C_j, dC~>
        router -> dg_j = pi_j (dpi_j - sum_i pi_i dpi_i) on the winners (softmax renormalised over K_t);
                  du = d dt * sigmoid(u) on the unclamped tokens, u = W_dt X + b
        linear -> dW_exp[e] = sum over (t, j) routed to e of dz_tj (x) X_t;  dX_t = sum_j W_exp[K_tj]^T dz_tj
                  + W_r^T dg_t + W_dt^T du_t;  dW_r = dg^T X;  dW_dt = du^T X;  db_dt = sum_t du_t.
    dy [B,T,H,P]; returns a dict with dX [B,T,D], dW_r, dW_dt, db_dt, dA, dW_exp, dinit [B,H,N,P]."""
    Bsz, T, D = X.shape
    M = Bsz * T
    Xf = X.reshape(M, D)
    fidx = None if forced_idx is None else forced_idx.reshape(M, k)
    g, dt, idx, w = router(Xf, W_r, W_dt, b_dt, k, decision_dtype, fidx)
    z = expert_proj(Xf, W_exp, idx)
    Bpi, Xs, Ct, Cpi = mix(z, w, H, P, G, N)
    x, Bz, Cz = split_streams(z, H, P, G, N)
    dyf = dy.reshape(M, H, P)
    dBpi = np.zeros(Bpi.shape); dXs = np.zeros(Xs.shape); dCt = np.zeros(Ct.shape); ddt = np.zeros(dt.shape)
    dA = np.zeros(np.shape(A)); dinit = np.zeros((Bsz, H, N, P))
    for b in range(Bsz):
        r = slice(b * T, (b + 1) * T)
        o = scan_backward(Bpi[r], Xs[r], Ct[r], dt[r], A, dyf[r], None if init is None else init[b])
        dBpi[r], dXs[r], dCt[r], ddt[r] = o["dBpi"], o["dXs"], o["dCt"], o["ddt"]
        dA = dA + o["dA"]
        dinit[b] = o["dinit"]
    dz, dw = mix_bwd(dBpi, dXs, dCt, w, Bz, Cz)
    dg_sel = router_bwd(w, dw)
    dg = np.zeros(g.shape)
    np.put_along_axis(dg, idx, dg_sel, axis=1)
    u = Xf @ W_dt.T + b_dt
    sp = softplus(u)
    du = ddt * (1.0 / (1.0 + np.exp(-u))) * ((sp > 1e-3) & (sp < 0.1))
    # linear maps
    dW_exp = np.zeros(W_exp.shape)
    dX = Xf * 0.0
    for m in range(M):
        for j in range(k):
            e = idx[m, j]
            dW_exp[e] += np.outer(dz[m, j], Xf[m])
            dX[m] += W_exp[e].T @ dz[m, j]
    dX += dg @ W_r + du @ W_dt
    return dict(dX=dX.reshape(Bsz, T, D), dW_r=dg.T @ Xf, dW_dt=du.T @ Xf, db_dt=du.sum(axis=0), dA=dA,
                dW_exp=dW_exp, dinit=dinit)


def out_proj(y, W_out):
    """out_t = W_out y_t: the one output projection that follows the shared recurrence's readout
    ([gist] Architecture Details).  There is one recurrence, so one projection, shared by all experts.

    y [..., H*P] with the heads flattened head-major (y[..., h*P + p]), W_out [D, H*P]; returns [..., D].
    Reading: a plain linear map without bias, applied to y as the readout returns it; the pages name no
    gate, normalisation or skip term before it, so none is applied.
    """
    return np.asarray(y) @ np.asarray(W_out).T


def step(Xt, W_r, W_dt, b_dt, A, W_exp, H, P, N, G, k, state, forced_idx=None, decision_dtype=np.float32,
         A_exp=None):
    """One recurrent decode step per sequence: the layer applied to a single new token X_t [B,D]
    with the cached state [B,H,N,P] (the recurrence of [notes] key design 1 advanced by one token);
    A_exp [E,H] or None as in layer_fwd.  Returns (y [B,H,P], new state [B,H,N,P], idx)."""
    g, dt, idx, w = router(Xt, W_r, W_dt, b_dt, k, decision_dtype, forced_idx)
    z = expert_proj(Xt, W_exp, idx)
    Bpi, Xs, Ct, _ = mix(z, w, H, P, G, N)
    gh = group_of(H, G)
    a = np.exp(log_decay(dt, A if A_exp is None else mixed_A(idx, w, A_exp)))   # [B,H]
    U = np.einsum("bjhn,bjhp->bhnp", Bpi[:, :, gh], Xs)
    new = a[:, :, None, None] * state + U
    y = np.einsum("bhn,bhnp->bhp", Ct[:, gh], new)
    return y, new, idx
