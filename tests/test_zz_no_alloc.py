"""swimba_dispatch_noalloc: the dispatch entry point for callers that cannot allocate device memory (hosts
that pass an operator only its inputs and outputs, runtimes that forbid allocations after start-up).  Its
results must equal swimba_dispatch's on two calls in a row (the second call must not see the first one's
leftovers in the shared scratch array), and shapes beyond its fixed scratch must be refused."""
import numpy as np
import pytest
import torch

from parameter_space_moe_b200 import configs, swimba

pytestmark = pytest.mark.gpu


def _idx(w, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(np.stack([rng.permutation(w.n_experts)[:w.top_k] for _ in range(w.M)]).astype(np.int32)).cuda()


def _check_same(w, seed):
    d = swimba.dims_of(w)
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device="cuda")
    idx = _idx(w, seed)
    off_ref = torch.empty(w.n_experts + 1, dtype=torch.int32, device="cuda")
    perm_ref = torch.empty(w.M * w.top_k, dtype=torch.int32, device="cuda")
    swimba.dispatch(d, idx, off_ref, perm_ref, ws)
    off = torch.full_like(off_ref, -1)
    perm = torch.full_like(perm_ref, -1)
    swimba.dispatch_noalloc(d, idx, off, perm)
    torch.cuda.synchronize()
    assert swimba.check_device_status() == 0
    assert torch.equal(off, off_ref)
    assert torch.equal(perm, perm_ref)


@pytest.mark.parametrize("w", [configs.BASE, configs.TINY_F32.with_(n_experts=64, top_k=8, seqlen=777)],
                         ids=lambda w: w.name)
def test_noalloc_dispatch_matches_workspace_dispatch(w):
    for seed in (1, 2):                                  # two calls in a row, different routings
        _check_same(w, seed)


def test_noalloc_dispatch_after_a_larger_call():
    """A large call (64 experts, k = 8) leaves more tile counts and schedule rows in the shared array than a
    smaller call that follows it (fewer tokens, 8 experts) writes; the smaller call must not read them."""
    big = configs.TINY_F32.with_(batch=3, seqlen=2000, n_experts=64, top_k=8)
    small = configs.TINY_F32.with_(batch=1, seqlen=300, n_experts=8, top_k=2)
    _check_same(big, 3)
    _check_same(small, 4)
    _check_same(big, 5)


def test_noalloc_dispatch_rejects_shapes_beyond_its_scratch():
    w = configs.TINY_F32.with_(batch=4096, seqlen=2048, n_experts=64, top_k=2)
    d = swimba.dims_of(w)
    fake = torch.empty(16, dtype=torch.int32, device="cuda")   # never touched: the call fails before launching
    with pytest.raises(swimba.SwimbaError) as e:
        swimba.dispatch_noalloc(d, fake, fake, fake)
    assert e.value.code == 4
