"""Stage-by-stage parity of the CUDA path against the fp64 oracle, through the C ABI.

Each stage runs on the GPU alone, fed with the same seeded inputs as the oracle: router (bit-exact
top-k outside near ties), dispatch (bit-exact stable sort), expert projection, mixing and the chunked
scan (the latter fed with the oracle's own streams rounded to the stream dtype)."""
import numpy as np
import pytest
import torch

from oracle import swimba_oracle as O
from parameter_space_moe_b200 import configs, inputs, swimba

from .parity import (check_topk, device_weights, f64, out_dtype, rel, state_tol_of, stream_torch_dtype, to_np,
                     tol_of)

pytestmark = pytest.mark.gpu

SMALL_BF16 = configs.BASE.with_(name="small_bf16", batch=2, seqlen=320, d_model=128, nheads=4, dstate=32,
                                n_experts=6, top_k=3, chunk=128, seed=77)
SMALL_G = configs.BASE.with_(name="small_groups", batch=2, seqlen=200, d_model=192, nheads=4, headdim=32,
                             dstate=64, ngroups=2, n_experts=4, top_k=2, chunk=64, seed=78)
# tensor-core scan shapes (N = 128): P = 128, three slots, shared groups, ragged T
TC_P128 = configs.BASE.with_(name="tc_P128_k3_G2", batch=2, seqlen=333, d_model=128, nheads=4, headdim=128,
                             dstate=128, ngroups=2, n_experts=5, top_k=3, chunk=128, seed=79)
TC_Q64 = configs.BASE.with_(name="tc_Q64_ragged", batch=3, seqlen=201, d_model=128, nheads=2, n_experts=4,
                            chunk=64, seed=80)
# enough rows per expert (>= 1536 on average) for the CTA-pair expert GEMM, ragged expert tails
PAIR_GEMM = configs.BASE.with_(name="pair_gemm_E2", batch=2, seqlen=1600, d_model=256, nheads=4, n_experts=2,
                               chunk=128, seed=86)
STAGE_CFGS = [configs.TINY_F32, SMALL_BF16, SMALL_G, TC_P128, TC_Q64, PAIR_GEMM, configs.BASE]
# tensor-core scan (P = 64, N = 128): one key slot, a single partial sub-chunk, one head whose 16 sub-chunks chain
# through the hand-off, more (sequence, head) rows than SMs; and long hand-off chains (32 or more 128-token
# sub-chunks per sequence): two key slots with a ragged tail, one key slot, a single head whose 40 sub-chunks
# all chain, and more head rows than SMs
SCAN_K1 = configs.BASE.with_(name="scan_k1_ragged", batch=2, seqlen=333, d_model=128, nheads=3, n_experts=3, top_k=1,
                             chunk=128, seed=88)
SCAN_SHORT = configs.BASE.with_(name="scan_one_partial_sub_chunk", batch=3, seqlen=50, d_model=128, nheads=2,
                                n_experts=4, chunk=128, seed=89)
SCAN_CHAIN = configs.BASE.with_(name="scan_one_head_16_sub_chunks", batch=1, seqlen=2000, d_model=128, nheads=1,
                                n_experts=4, chunk=256, seed=90)
SCAN_WIDE = configs.BASE.with_(name="scan_200_heads", batch=2, seqlen=300, d_model=128, nheads=100, n_experts=2,
                               chunk=256, seed=91)
LONGCHAIN_K2 = configs.BASE.with_(name="longchain_k2_ragged", batch=2, seqlen=4500, d_model=128, nheads=2,
                                  n_experts=4, chunk=256, seed=92)
LONGCHAIN_K1 = configs.BASE.with_(name="longchain_k1", batch=1, seqlen=4200, d_model=128, nheads=3, n_experts=3,
                                  top_k=1, chunk=128, seed=93)
LONGCHAIN_ONE_HEAD = configs.BASE.with_(name="longchain_one_head_40_sub_chunks", batch=1, seqlen=5100, d_model=128,
                                        nheads=1, n_experts=4, chunk=256, seed=94)
LONGCHAIN_WIDE = configs.BASE.with_(name="longchain_160_heads", batch=2, seqlen=4100, d_model=128, nheads=80,
                                    n_experts=2, chunk=256, seed=95)
# B and C shared by groups of heads: G = H / 4 with a ragged tail, G = 1 over 6 heads with k = 3, G = H / 2 on a
# long hand-off chain, and 400 (sequence, head) rows in 200 groups
SCAN_G4 = configs.BASE.with_(name="scan_H8_G2_ragged", batch=2, seqlen=333, d_model=128, nheads=8, ngroups=2,
                             n_experts=4, chunk=128, seed=96)
SCAN_G1_K3 = configs.BASE.with_(name="scan_H6_G1_k3", batch=1, seqlen=700, d_model=128, nheads=6, ngroups=1,
                                n_experts=5, top_k=3, chunk=256, seed=97)
LONGCHAIN_G = configs.BASE.with_(name="longchain_H4_G2", batch=1, seqlen=4300, d_model=128, nheads=4, ngroups=2,
                                 n_experts=4, chunk=256, seed=98)
SCAN_G_WIDE = configs.BASE.with_(name="scan_400_heads_G100", batch=2, seqlen=300, d_model=128, nheads=200,
                                 ngroups=100, n_experts=2, chunk=256, seed=99)
SCAN_GROUPED = [SCAN_G4, SCAN_G1_K3, LONGCHAIN_G, SCAN_G_WIDE]
SCAN_CFGS = STAGE_CFGS + [SCAN_K1, SCAN_SHORT, SCAN_CHAIN, SCAN_WIDE, LONGCHAIN_K2, LONGCHAIN_K1, LONGCHAIN_ONE_HEAD,
                          LONGCHAIN_WIDE] + SCAN_GROUPED
_cache = {}


def _setup(w):
    if w.name in _cache:
        return _cache[w.name]
    inp = inputs.make_inputs(w)
    Xf = f64(inp["X"]).reshape(w.M, w.d_model)
    ref = O.layer_fwd(f64(inp["X"]), f64(inp["W_r"]), f64(inp["W_dt"]), f64(inp["b_dt"]), f64(inp["A"]),
                      f64(inp["W_exp"]), w.nheads, w.headdim, w.dstate, w.G, w.top_k)
    dev = {"X": inp["X"].cuda().reshape(w.M, w.d_model), "W": device_weights(inp)}
    _cache[w.name] = (inp, Xf, ref, dev)
    return _cache[w.name]


def _ws(d):
    return torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")


# Router shapes at the edges of the tensor-core router: one partial 128-token tile, E = 64 with k = 8,
# the widest logit row it takes (ceil8(E) + H = 128 columns), one column past it (the CUDA-core router
# takes over), an odd number of 64-wide K blocks (no K split) and a K split over 4 CTAs on a ragged tail.
ROUTER_EDGES = [
    configs.BASE.with_(name="r_one_partial_tile", batch=1, seqlen=50, d_model=256, nheads=8, n_experts=64,
                       top_k=8, seed=81),
    configs.BASE.with_(name="r_row128", batch=3, seqlen=300, d_model=512, nheads=64, n_experts=64, top_k=4,
                       seed=82),
    configs.BASE.with_(name="r_row129_fallback", batch=3, seqlen=300, d_model=512, nheads=66, n_experts=63,
                       top_k=2, seed=83),
    configs.BASE.with_(name="r_odd_kblocks", batch=2, seqlen=777, d_model=320, nheads=12, n_experts=12, top_k=3,
                       seed=84),
    configs.BASE.with_(name="r_ksplit4_ragged", batch=5, seqlen=1001, d_model=1024, nheads=16, n_experts=32,
                       top_k=2, seed=85),
]


@pytest.mark.parametrize("w", ROUTER_EDGES, ids=lambda w: w.name)
def test_router_edges(w):
    inp = inputs.make_inputs(w)
    g, dt_ref, _, _ = O.router(f64(inp["X"]).reshape(w.M, w.d_model), f64(inp["W_r"]), f64(inp["W_dt"]),
                               f64(inp["b_dt"]), w.top_k)
    d = swimba.dims_of(w)
    W = device_weights(inp)
    X = inp["X"].cuda().reshape(w.M, w.d_model)
    idx = torch.empty(w.M, w.top_k, dtype=torch.int32, device="cuda")
    wts = torch.empty(w.M, w.top_k, device="cuda")
    dt = torch.empty(w.M, w.nheads, device="cuda")
    swimba.router_topk(d, X, W, idx, wts, dt)
    torch.cuda.synchronize()
    assert swimba.check_device_status() == 0
    fl, forced = check_topk(to_np(idx), g, w.top_k)
    _, _, _, w_ref = O.router(f64(inp["X"]).reshape(w.M, w.d_model), f64(inp["W_r"]), f64(inp["W_dt"]),
                              f64(inp["b_dt"]), w.top_k, forced_idx=forced)
    np.testing.assert_allclose(to_np(wts), w_ref, rtol=2e-5, atol=1e-6)
    np.testing.assert_allclose(to_np(dt), dt_ref, rtol=2e-5)


@pytest.mark.parametrize("w", STAGE_CFGS, ids=lambda w: w.name)
def test_router(w):
    inp, Xf, ref, dev = _setup(w)
    d = swimba.dims_of(w)
    idx = torch.empty(w.M, w.top_k, dtype=torch.int32, device="cuda")
    wts = torch.empty(w.M, w.top_k, device="cuda")
    dt = torch.empty(w.M, w.nheads, device="cuda")
    swimba.router_topk(d, dev["X"], dev["W"], idx, wts, dt)
    torch.cuda.synchronize()
    fl, forced = check_topk(to_np(idx), ref["g"], w.top_k)
    ok = ~fl
    np.testing.assert_allclose(to_np(wts)[ok], ref["w"][ok], rtol=2e-5, atol=1e-6)
    np.testing.assert_allclose(to_np(wts).sum(1), 1.0, rtol=1e-6)
    np.testing.assert_allclose(to_np(dt), ref["dt"], rtol=2e-5)


@pytest.mark.parametrize("w", STAGE_CFGS, ids=lambda w: w.name)
def test_dispatch_is_stable_sort(w):
    inp, Xf, ref, dev = _setup(w)
    d = swimba.dims_of(w)
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    off = torch.empty(w.n_experts + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(w.M * w.top_k, dtype=torch.int32, device="cuda")
    swimba.dispatch(d, idx, off, perm, _ws(d))
    torch.cuda.synchronize()
    flat = ref["idx"].reshape(-1)
    np.testing.assert_array_equal(to_np(perm), np.argsort(flat, kind="stable"))
    np.testing.assert_array_equal(to_np(off), np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=w.n_experts))]))


def test_dispatch_skips_out_of_range_indices():
    """Caller-given indices outside [0, E) are left out of the sort and reported as SWIMBA_ERR_INDEX; the
    valid pairs are still sorted stably (the kernels index no table with the bad values)."""
    w = configs.BASE.with_(batch=1, seqlen=3000, n_experts=8, top_k=2)
    rng = np.random.default_rng(5)
    idx_np = np.stack([rng.permutation(w.n_experts)[:w.top_k] for _ in range(w.M)]).astype(np.int32)
    bad = rng.choice(w.M * w.top_k, size=37, replace=False)
    flat = idx_np.reshape(-1)
    flat[bad[:20]] = 99
    flat[bad[20:]] = -3
    d = swimba.dims_of(w)
    off = torch.empty(w.n_experts + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((w.M * w.top_k,), -7, dtype=torch.int32, device="cuda")
    swimba.dispatch(d, torch.from_numpy(idx_np).cuda(), off, perm, _ws(d))
    assert swimba.check_device_status() == 7
    assert swimba.check_device_status() == 0
    ok = (flat >= 0) & (flat < w.n_experts)
    want = np.nonzero(ok)[0][np.argsort(flat[ok], kind="stable")]
    n = int(ok.sum())
    np.testing.assert_array_equal(to_np(off), np.concatenate([[0], np.cumsum(np.bincount(flat[ok], minlength=8))]))
    np.testing.assert_array_equal(to_np(perm)[:n], want)
    assert (to_np(perm)[n:] == -7).all()


@pytest.mark.parametrize("w", STAGE_CFGS, ids=lambda w: w.name)
def test_expert_proj_and_mix(w):
    inp, Xf, ref, dev = _setup(w)
    d = swimba.dims_of(w)
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    Z = torch.empty(w.M, w.top_k, w.W_e, device="cuda")
    ws = _ws(d)
    swimba.expert_proj(d, dev["X"], dev["W"], idx, Z, ws)
    torch.cuda.synchronize()
    assert rel(to_np(Z), ref["z"]) < 1e-5
    sdt = stream_torch_dtype(w)
    wts = torch.from_numpy(ref["w"].astype(np.float32)).cuda()
    Bpi = torch.empty(w.M, w.top_k, w.G, w.dstate, dtype=sdt, device="cuda")
    Xs = torch.empty(w.M, w.top_k, w.nheads, w.headdim, dtype=sdt, device="cuda")
    Cpi = torch.empty_like(Bpi)
    swimba.mix(d, Z, wts, 0, Bpi, Xs, Cpi)
    assert swimba.check_device_status() == 0
    tol = 1e-6 if w.dtype == "f32" else 6e-4     # fp16 streams keep 11 significant bits
    assert rel(to_np(Bpi), ref["Bpi"]) < tol
    assert rel(to_np(Xs), ref["Xs"]) < tol
    assert rel(to_np(Cpi), ref["Cpi"]) < tol
    swimba.mix(d, Z, wts, swimba.MIX_UNSCALED_B, Bpi, Xs, Cpi)
    torch.cuda.synchronize()
    _, B, _ = O.split_streams(ref["z"], w.nheads, w.headdim, w.G, w.dstate)
    assert rel(to_np(Bpi), B) < tol


def _oracle_streams_on_device(w, ref):
    sdt = stream_torch_dtype(w)
    Bpi = torch.from_numpy(ref["Bpi"]).to(sdt)
    Xs = torch.from_numpy(ref["Xs"]).to(sdt)
    Cpi = torch.from_numpy(ref["Cpi"]).to(sdt)
    dt = torch.from_numpy(ref["dt"]).float()
    return Bpi, Xs, Cpi, dt


@pytest.mark.parametrize("w", SCAN_CFGS, ids=lambda w: w.name)
@pytest.mark.parametrize("with_init", [False, True])
def test_ssd_scan(w, with_init):
    inp, Xf, ref, dev = _setup(w)
    if w.name == configs.BASE.name and with_init:
        pytest.skip("covered by the small configs")
    d = swimba.dims_of(w)
    Bpi, Xs, Cpi, dt = _oracle_streams_on_device(w, ref)
    A = inp["A"]
    rng = np.random.default_rng(5)
    init = rng.standard_normal((w.batch, w.nheads, w.dstate, w.headdim)).astype(np.float32) if with_init else None
    y = torch.empty(w.M, w.nheads * w.headdim, dtype=out_dtype(w), device="cuda")
    fin = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, device="cuda")
    nc = -(-w.seqlen // w.chunk)
    cst = torch.empty(w.batch, w.nheads, nc, w.dstate, w.headdim, device="cuda")
    swimba.ssd_scan(d, Bpi.cuda(), Xs.cuda(), Cpi.cuda(), dt.cuda(), A.cuda(),
                    None if init is None else torch.from_numpy(init).cuda(), y, fin, cst, _ws(d))
    torch.cuda.synchronize()
    # the oracle on exactly the streams the GPU read
    Bq, Xq, Cq = (t.double().numpy() for t in (Bpi, Xs, Cpi))
    dtq = dt.double().numpy()
    Ct = Cq.sum(1)
    for b in range(w.batch):
        r = slice(b * w.seqlen, (b + 1) * w.seqlen)
        yc, Hs, hT = O.scan_chunked(Bq[r], Xq[r], Ct[r], dtq[r], f64(A), w.chunk,
                                    None if init is None else init[b].astype(np.float64))
        tol = tol_of(w)
        assert rel(to_np(y)[r].reshape(yc.shape), yc) < tol
        assert rel(to_np(fin)[b], hT) < state_tol_of(w)
        assert rel(to_np(cst)[b].transpose(1, 0, 2, 3), Hs) < state_tol_of(w)


@pytest.mark.parametrize("w", [configs.TINY_F32, TC_P128, TC_Q64, LONGCHAIN_K2, SCAN_G4, SCAN_G1_K3],
                         ids=lambda w: w.name)
def test_separated_scan(w):
    """The separated design ("k scans"): k trajectories with unscaled injections, pi-scaled readouts."""
    inp, Xf, ref, dev = _setup(w)
    d = swimba.dims_of(w)
    sdt = stream_torch_dtype(w)
    _, B, _ = O.split_streams(ref["z"], w.nheads, w.headdim, w.G, w.dstate)
    Bq = torch.from_numpy(B).to(sdt)
    Xq = torch.from_numpy(ref["Xs"]).to(sdt)
    Cq = torch.from_numpy(ref["Cpi"]).to(sdt)
    dt = torch.from_numpy(ref["dt"]).float()
    y = torch.empty(w.M, w.nheads * w.headdim, dtype=out_dtype(w), device="cuda")
    fin = torch.empty(w.top_k, w.batch, w.nheads, w.dstate, w.headdim, device="cuda")
    swimba.separated_scan(d, Bq.cuda(), Xq.cuda(), Cq.cuda(), dt.cuda(), inp["A"].cuda(), None, y, fin, _ws(d))
    assert swimba.check_device_status() == 0
    Bd, Xd, Cd, dtd = (t.double().numpy() for t in (Bq, Xq, Cq, dt))
    for b in range(w.batch):
        r = slice(b * w.seqlen, (b + 1) * w.seqlen)
        ys, hs, nrec = O.scan_separated_k(Bd[r], Xd[r], Cd[r], dtd[r], f64(inp["A"]))
        assert nrec == w.top_k
        assert rel(to_np(y)[r].reshape(ys.shape), ys) < tol_of(w)
        assert rel(to_np(fin)[:, b], hs) < state_tol_of(w)


@pytest.mark.parametrize("seqlen,groups", [(512, 0), (4200, 0), (512, 1)], ids=["T512", "T4200", "T512_G1"])
def test_scan_lost_predecessor_times_out_without_fault(seqlen, groups):
    """Failure detection: the first sub-chunk of every head is made to go missing, so the successors'
    flag waits can never succeed.  They give up after their bounded wait, the status word reports
    SWIMBA_ERR_TIMEOUT (no fault, no hang), and the context stays usable: the normal scan that follows
    is correct."""
    import time
    w = configs.BASE.with_(name=f"lost_chunk_T{seqlen}_G{groups}", batch=1, seqlen=seqlen, d_model=128, nheads=2,
                           ngroups=groups, seed=87)
    inp, Xf, ref, dev = _setup(w)
    d = swimba.dims_of(w)
    Bpi, Xs, Cpi, dt = (t.cuda() for t in _oracle_streams_on_device(w, ref))
    A = inp["A"].cuda()
    y = torch.empty(w.M, w.nheads * w.headdim, dtype=out_dtype(w), device="cuda")
    ws = _ws(d)
    assert swimba.check_device_status() == 0
    t0 = time.time()
    swimba.debug_scan_lost_first_chunk(d, Bpi, Xs, Cpi, dt, A, y, ws)
    assert swimba.check_device_status() == 5          # SWIMBA_ERR_TIMEOUT, read and cleared
    assert time.time() - t0 < 30.0
    assert swimba.check_device_status() == 0
    swimba.ssd_scan(d, Bpi, Xs, Cpi, dt, A, None, y, None, None, ws)
    torch.cuda.synchronize()
    assert swimba.check_device_status() == 0
    Bq, Xq, Cq = (t.double().cpu().numpy() for t in (Bpi, Xs, Cpi))
    yc, _, _ = O.scan_chunked(Bq, Xq, Cq.sum(1), dt.double().cpu().numpy(), f64(inp["A"]), w.chunk, None)
    assert rel(to_np(y).reshape(yc.shape), yc) < tol_of(w)
