"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry point that
include/swimba.h declares, sizes workspaces, and rejects invalid or unsupported arguments before
launching anything."""
import ctypes
import os
import re

import pytest

from parameter_space_moe_b200 import configs, swimba

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "swimba.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(swimba_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    try:
        return swimba.lib()
    except OSError:
        import __graft_entry__
        __graft_entry__.build()
        return swimba.lib()


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(swimba.EXPORTS)


def test_status_strings(L):
    for code, name in swimba.STATUS.items():
        assert swimba.status_string(code) == name


def test_workspace_size_and_stream_dtype(L):
    for w in configs.ALL.values():
        d = swimba.dims_of(w)
        assert swimba.workspace_size(d) > 0
        assert swimba.stream_dtype(d) == (swimba.F16 if w.dtype == "bf16" else swimba.F32)
    big = swimba.workspace_size(swimba.dims_of(configs.BASE))
    small = swimba.workspace_size(swimba.dims_of(configs.BASE, seqlen=256))
    assert big > small


BAD_DIMS = [
    dict(headdim=48), dict(dstate=256), dict(chunk=32), dict(chunk=512), dict(top_k=9, n_experts=16),
    dict(n_experts=65), dict(d_model=100),
]
INVALID_DIMS = [dict(batch=0), dict(seqlen=-1), dict(top_k=5, n_experts=4), dict(ngroups=5), dict(dtype=7)]


@pytest.mark.parametrize("kw", BAD_DIMS)
def test_unsupported_shapes(L, kw):
    base = dict(batch=1, seqlen=64, d_model=128, nheads=2, headdim=64, dstate=16, ngroups=2, n_experts=4, top_k=2,
                chunk=64, dtype=swimba.BF16)
    base.update(kw)
    d = swimba.dims(**base)
    assert swimba.workspace_size(d) == 0
    fake = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: validation fails first
    w = swimba.Weights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    rc = L.swimba_layer_fwd(ctypes.byref(d), fake, ctypes.byref(w), None, fake, None, None, None, fake, 1 << 40, None)
    assert rc == 2


@pytest.mark.parametrize("kw", INVALID_DIMS)
def test_invalid_dims(L, kw):
    base = dict(batch=1, seqlen=64, d_model=128, nheads=2, headdim=64, dstate=16, ngroups=2, n_experts=4, top_k=2,
                chunk=64, dtype=swimba.BF16)
    base.update(kw)
    d = swimba.dims(**base)
    assert swimba.workspace_size(d) == 0
    fake = ctypes.c_void_p(1 << 20)
    w = swimba.Weights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    rc = L.swimba_router_topk(ctypes.byref(d), fake, ctypes.byref(w), fake, fake, fake, None)
    assert rc == 1
    # both dispatch entry points give the same code for the same invalid dims
    assert L.swimba_dispatch(ctypes.byref(d), fake, fake, fake, fake, 1 << 40, None) == 1
    assert L.swimba_dispatch_noalloc(ctypes.byref(d), fake, fake, fake, None) == 1
    assert L.swimba_out_proj(ctypes.byref(d), fake, fake, fake, None) == 1


@pytest.mark.parametrize("kw", BAD_DIMS)
def test_dispatch_entry_points_agree_on_unsupported_dims(L, kw):
    base = dict(batch=1, seqlen=64, d_model=128, nheads=2, headdim=64, dstate=16, ngroups=2, n_experts=4, top_k=2,
                chunk=64, dtype=swimba.BF16)
    base.update(kw)
    d = swimba.dims(**base)
    fake = ctypes.c_void_p(1 << 20)
    assert L.swimba_dispatch(ctypes.byref(d), fake, fake, fake, fake, 1 << 40, None) == 2
    assert L.swimba_dispatch_noalloc(ctypes.byref(d), fake, fake, fake, None) == 2
    assert L.swimba_out_proj(ctypes.byref(d), fake, fake, fake, None) == 2
    assert L.swimba_ssd_scan_bwd(ctypes.byref(d), fake, fake, fake, fake, fake, None, fake, fake, fake, fake, fake,
                                 fake, None, fake, 1 << 40, None) == 2


def test_null_misaligned_and_workspace_errors(L):
    d = swimba.dims_of(configs.TINY_F32)
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    w = swimba.Weights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    need = swimba.workspace_size(d)
    args = lambda X, ws, n: (ctypes.byref(d), X, ctypes.byref(w), None, fake, None, None, None, ws, n, None)
    assert L.swimba_layer_fwd(*args(None, fake, need)) == 1           # null X
    assert L.swimba_layer_fwd(*args(odd, fake, need)) == 1            # misaligned X
    assert L.swimba_layer_fwd(*args(fake, None, need)) == 4           # no workspace
    assert L.swimba_layer_fwd(*args(fake, fake, need - 1)) == 4       # workspace too small
    assert L.swimba_layer_fwd(*args(fake, odd, need)) == 4            # misaligned workspace
    # A may be left out only when the expert-mixed A_exp is given
    wnoA = swimba.Weights(1 << 20, 1 << 20, 1 << 20, None, 1 << 20)
    assert L.swimba_layer_fwd(ctypes.byref(d), fake, ctypes.byref(wnoA), None, fake, None, None, None, fake, need,
                              None) == 1
    wnull = swimba.Weights(1 << 20, None, 1 << 20, 1 << 20, 1 << 20)
    assert L.swimba_layer_fwd(ctypes.byref(d), fake, ctypes.byref(wnull), None, fake, None, None, None, fake, need,
                              None) == 1
    assert L.swimba_layer_fwd(None, fake, ctypes.byref(w), None, fake, None, None, None, fake, need, None) == 1
    # decode needs seqlen == 1
    assert L.swimba_step(ctypes.byref(d), fake, ctypes.byref(w), fake, fake, None, fake, need, None) == 1
    # mix rejects unknown flags
    assert L.swimba_mix(ctypes.byref(d), fake, fake, 8, fake, fake, fake, None) == 1
    # scan gradients: null and misaligned pointers, workspace too small
    bwd = lambda dy, ws=fake, n=need: L.swimba_ssd_scan_bwd(ctypes.byref(d), fake, fake, fake, fake, fake, None, dy,
                                                         fake, fake, fake, fake, fake, None, ws, n, None)
    assert bwd(None) == 1
    assert bwd(odd) == 1
    assert bwd(fake, n=need - 1) == 4
    # layer gradients: null pointers, a workspace sized for the forward only, the mixed transition
    nb = swimba.layer_bwd_workspace_size(d)
    assert nb > need
    lbwd = lambda wts, dy, n: L.swimba_layer_bwd(ctypes.byref(d), fake, ctypes.byref(wts), None, dy, fake, fake,
                                                 fake, fake, fake, fake, None, fake, n, None)
    assert lbwd(w, None, nb) == 1
    assert lbwd(w, fake, need) == 4
    wmix = swimba.Weights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    assert lbwd(wmix, fake, nb) == 2
    # output projection: every pointer non-null and 16-byte aligned
    assert L.swimba_out_proj(ctypes.byref(d), None, fake, fake, None) == 1
    assert L.swimba_out_proj(ctypes.byref(d), fake, odd, fake, None) == 1
    assert L.swimba_out_proj(ctypes.byref(d), fake, fake, None, None) == 1
    assert L.swimba_out_proj(None, fake, fake, fake, None) == 1


@pytest.mark.parametrize("w", [configs.BASE, configs.BASE.with_(name="ws_We240", nheads=3, headdim=16, dstate=32,
                                                                n_experts=5)], ids=lambda w: w.name)
def test_layer_bwd_workspace_holds_the_tensor_core_operands(w):
    """A bf16 layer's gradient workspace holds, besides the forward's workspace and the fp32 gradient buffers,
    the tensor-core expert products' operands: dz as bf16 hi and lo over expert-padded rows
    (Rp = M*k + 64 E rows rounded up to 128, 2 Wp columns with Wp = W_e rounded up to 64) and the X rows in
    the same padded order."""
    d = swimba.dims_of(w)
    Mk = w.M * w.top_k
    Rp = -(-(Mk + 64 * w.n_experts) // 128) * 128
    Wp = -(-w.W_e // 64) * 64
    fp32_bufs = Mk * (w.W_e + w.G * w.dstate + w.nheads * w.headdim + w.d_model) * 4
    operands = Rp * 2 * Wp * 2 + Rp * w.d_model * 2 + Rp * 4 + Mk * 4
    assert swimba.layer_bwd_workspace_size(d) >= swimba.workspace_size(d) + fp32_bufs + operands


def test_host_pipeline_and_debug_hook_validation(L):
    """swimba_layer_fwd_host and the failure-detection hook reject bad arguments before any CUDA call."""
    d = swimba.dims_of(configs.BASE.with_(batch=2, seqlen=512, d_model=128, nheads=2))
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    w = swimba.Weights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    need = swimba.workspace_size(d)
    host = lambda Xh, yh, Xd, yd, chunks, ws=fake, n=need: L.swimba_layer_fwd_host(
        ctypes.byref(d), Xh, ctypes.byref(w), None, yh, None, Xd, yd, ws, n, chunks, None)
    assert host(None, fake, fake, fake, 2) == 1        # no host input
    assert host(fake, None, fake, fake, 2) == 1        # no host output
    assert host(fake, fake, odd, fake, 2) == 1         # misaligned device staging
    assert host(fake, fake, fake, None, 2) == 1        # no device staging for y
    assert host(fake, fake, fake, fake, 0) == 1        # at least one group
    assert host(fake, fake, fake, fake, 2, n=need - 1) == 4   # workspace too small
    hook = lambda dims, Bpi=fake: L.swimba_debug_scan_lost_first_chunk(
        ctypes.byref(dims), Bpi, fake, fake, fake, fake, fake, fake, swimba.workspace_size(dims), None)
    assert hook(swimba.dims_of(configs.TINY_F32)) == 2                      # not a tensor-core scan shape
    assert hook(swimba.dims_of(configs.BASE.with_(batch=1, seqlen=128))) == 2   # one sub-chunk: nothing to lose
    assert hook(d, Bpi=None) == 1
