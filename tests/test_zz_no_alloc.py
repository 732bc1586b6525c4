"""moe_permute_noalloc — the dispatch entry point for callers that cannot
allocate device memory at the call site (a plugin whose host framework owns
the device-memory budget, a loop that must not call cudaMalloc) — must give
exactly what moe_permute gives with a caller-provided workspace, call after
call, although every call reuses the library's one scratch array.

Kept in its own file, collected last, and independent of the other tests so
it also runs alone in a fresh process. Needs a B200.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_58_b200 import _lib as L
from mixture_experts_layer_58_b200 import synth
from oracle import moe_oracle as om

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    L.load()


def _case(T, d, n_routed, top_k, seed):
    cfg = synth.CONFIGS["tiny"].replace(T=T, d=d, n_routed=n_routed, top_k=top_k, seed=seed)
    u, e, b = synth.tokens(cfg), synth.centroids(cfg), synth.bias(cfg)
    r = om.route(u, e, b, top_k, 1.0)
    return (u.cuda(), torch.from_numpy(r.idx.astype(np.int32)).cuda(),
            torch.from_numpy(r.counts.astype(np.int32)).cuda())


def _outputs(T, d, n_routed, top_k):
    dev = "cuda"
    return (torch.full((T * top_k, d), 7.0, dtype=torch.bfloat16, device=dev),
            torch.full((n_routed + 1,), -9, dtype=torch.int32, device=dev),
            torch.full((T, top_k), -9, dtype=torch.int32, device=dev),
            torch.full((T * top_k,), -9, dtype=torch.int32, device=dev))


def _with_workspace(u, idx, counts, T, d, n, k):
    x, off, pos, src = _outputs(T, d, n, k)
    wsb = L.moe_permute_workspace_size(T, n)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    L.moe_permute(u, idx, counts, T, d, n, k, x, off, pos, src, ws, wsb)
    return x, off, pos, src


def _no_alloc(u, idx, counts, T, d, n, k):
    x, off, pos, src = _outputs(T, d, n, k)
    L.moe_permute_noalloc(u, idx, counts, T, d, n, k, x, off, pos, src)
    return x, off, pos, src


def _same(a, b):
    for ta, tb in zip(a, b):
        assert torch.equal(ta, tb)


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # a large case, then a smaller one with other shapes, then the large one
    # again: the second and third calls find the previous call's histograms
    # in the shared scratch array
    big = (4096, 512, 64, 6)
    small = (300, 256, 16, 4)
    inputs = {big: _case(*big, seed=3), small: _case(*small, seed=4)}
    want = {s: _with_workspace(*inputs[s], *s) for s in (big, small)}
    got1 = _no_alloc(*inputs[big], *big)
    got2 = _no_alloc(*inputs[small], *small)
    got3 = _no_alloc(*inputs[big], *big)
    torch.cuda.synchronize()
    _same(got1, want[big])
    _same(got2, want[small])
    _same(got3, want[big])
    # the shared outputs are the oracle's dispatch order
    d = om.dispatch(inputs[small][1].cpu().numpy(), small[2])
    assert np.array_equal(got2[2].cpu().numpy(), d.pos)
    assert L.moe_get_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    T, d, n, k = 40000, 256, 256, 8       # ceil(40000/128) * 256 = 80128 > 65536
    u = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    counts = torch.zeros(n, dtype=torch.int32, device="cuda")
    x, off, pos, src = _outputs(T, d, n, k)
    with pytest.raises(L.MoEError) as ei:
        L.moe_permute_noalloc(u, idx, counts, T, d, n, k, x, off, pos, src)
    assert ei.value.status == L.MOE_ERR_UNSUPPORTED_SHAPE
    torch.cuda.synchronize()
    assert int(off[0]) == -9          # nothing was launched


def _random_routing(T, n, k, seed):
    g = torch.Generator().manual_seed(seed)
    idx = torch.argsort(torch.rand(T, n, generator=g), dim=1)[:, :k].to(torch.int32)
    counts = torch.bincount(idx.flatten().long(), minlength=n).to(torch.int32)
    u = torch.randn(T, 256, generator=g).bfloat16()
    return u.cuda(), idx.cuda(), counts.cuda()


def test_noalloc_at_its_largest_accepted_size():
    # ceil(32768/128) * 256 = 65536 histogram entries: exactly the scratch
    # array, every entry of it used; one token more is refused
    T, d, n, k = 32768, 256, 256, 8
    u, idx, counts = _random_routing(T, n, k, seed=5)
    want = _with_workspace(u, idx, counts, T, d, n, k)
    got = _no_alloc(u, idx, counts, T, d, n, k)
    torch.cuda.synchronize()
    _same(got, want)
    T1 = T + 1
    u1 = torch.zeros((T1, d), dtype=torch.bfloat16, device="cuda")
    idx1 = torch.zeros((T1, k), dtype=torch.int32, device="cuda")
    x, off, pos, src = _outputs(T1, d, n, k)
    with pytest.raises(L.MoEError) as ei:
        L.moe_permute_noalloc(u1, idx1, counts, T1, d, n, k, x, off, pos, src)
    assert ei.value.status == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_get_device_status() == 0
