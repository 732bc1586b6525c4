"""The IPC helpers behind the peer-memory expert-parallel layer, across two
processes on one GPU: the parent takes the handle of a tensor that starts
inside a larger allocation (non-zero offset), a spawned child maps it and
reads its rows with the library's own row-gather kernel, then unmaps it.
Neither process waits on a kernel of the other. Needs a B200."""
import multiprocessing as mp

import pytest
import torch

from mixture_experts_layer_58_b200 import _lib as L

pytestmark = pytest.mark.gpu


def _child(handle, offset, n, d, q):
    import torch
    from mixture_experts_layer_58_b200 import _lib as L
    try:
        torch.cuda.set_device(0)
        L.load()
        base = L.moe_ipc_open_handle(handle)
        idx = torch.arange(n, dtype=torch.int32, device="cuda")
        dst = torch.empty(n, d, dtype=torch.bfloat16, device="cuda")
        L.moe_gather_rows(base + offset, n, idx, n, d, dst)
        torch.cuda.synchronize()
        # a numpy array pickles by value (a torch CPU tensor would be shared
        # through a file descriptor that dies with this process)
        q.put(("ok", dst.float().cpu().numpy()))
        L.moe_ipc_close_handle(base)
    except Exception as exc:  # noqa: BLE001 - reported to the parent
        q.put(("error", repr(exc)))


def test_ipc_handle_maps_a_tensor_in_another_process(cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    L.load()
    d = 256
    whole = torch.randn(1000, d, generator=torch.Generator().manual_seed(3)).bfloat16().cuda()
    x = whole[100:]                              # starts 51200 bytes into the tensor
    handle, offset = L.moe_ipc_get_handle(x)
    assert len(handle) == 64 and offset >= 100 * d * 2 and offset % 16 == 0
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_child, args=(handle, offset, x.shape[0], d, q))
    p.start()
    try:
        status, got = q.get(timeout=240)
    finally:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert status == "ok", got
    assert torch.equal(torch.from_numpy(got), x.float().cpu())
