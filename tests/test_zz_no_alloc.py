"""moe_fused_router_topk_noalloc against moe_fused_router_topk (GPU only).

The allocation-free entry point serves callers that may not allocate device
memory when they route (engines that reserve all device memory at start-up,
plugin hosts without an allocator).  It takes its scratch from a fixed array
inside the library instead of a caller workspace, so it must give the same
result as the workspace entry point - on repeated calls too, since the array
keeps the previous call's contents.  Collected last so that a failure here
does not hide the other tests; it passes alone or after them.
"""
import ctypes

import pytest
import torch

import moe_expert_routing_token_b200 as moe
from moe_expert_routing_token_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _call_noalloc(lib, h, w, b, M, K, out_w, out_ids, logits):
    return lib.moe_fused_router_topk_noalloc(
        h.data_ptr(), w.data_ptr(), 0, b.data_ptr(), M, K, 256, 8, 1, 8, 4, 2.5,
        out_w.data_ptr(), out_ids.data_ptr(), logits.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M", [64, 1, 128])
def test_noalloc_matches_workspace_entry_point_twice(M):
    lib = moe.lib()
    d = inputs.make("fused", M, seed=4242 + M)
    h, w, b = d["hidden"].to(DEV), d["weight"].to(DEV), d["bias"].to(DEV)
    K = h.shape[1]
    assert moe.fused_router_workspace_size(M, K, 256) > 0  # the scratch-using path
    ref_w, ref_ids, ref_logits = moe.fused_router_topk(h, w, b, 8, True, 8, 4, 2.5, return_logits=True)
    for _ in range(2):  # the shared array keeps the previous call's contents
        out_w = torch.full((M, 8), -1.0, device=DEV)
        out_ids = torch.full((M, 8), -1, dtype=torch.int32, device=DEV)
        logits = torch.full((M, 256), float("nan"), device=DEV)
        st = _call_noalloc(lib, h, w, b, M, K, out_w, out_ids, logits)
        assert st == 0, lib.moe_last_error().decode()
        torch.cuda.synchronize()
        assert torch.equal(out_ids, ref_ids)
        assert torch.allclose(out_w, ref_w, rtol=2e-3, atol=0.0)
        assert torch.allclose(logits, ref_logits, rtol=0.0, atol=1e-5)


def test_noalloc_serves_the_largest_decode_workspace():
    """M = 128 with K = 9216 once needed more scratch than the built-in
    2 MiB; the decode path caps its partial logits at 2 MiB, so the call runs
    and matches the workspace entry point."""
    lib = moe.lib()
    M, K = 128, 9216
    need = moe.fused_router_workspace_size(M, K, 256)
    assert 0 < need <= (2 << 20)
    g = torch.Generator().manual_seed(9216)
    h = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    w = (torch.randn(K, 256, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    b = (torch.randn(256, generator=g) * 0.05).to(DEV)
    ref_w, ref_ids, ref_logits = moe.fused_router_topk(h, w, b, 8, True, 8, 4, 2.5, return_logits=True)
    out_w = torch.empty(M, 8, device=DEV)
    out_ids = torch.empty(M, 8, dtype=torch.int32, device=DEV)
    logits = torch.empty(M, 256, device=DEV)
    st = _call_noalloc(lib, h, w, b, M, K, out_w, out_ids, logits)
    assert st == 0, lib.moe_last_error().decode()
    torch.cuda.synchronize()
    assert torch.equal(out_ids, ref_ids)
    assert torch.equal(logits, ref_logits)
    assert torch.allclose(out_w, ref_w, rtol=2e-3, atol=0.0)
