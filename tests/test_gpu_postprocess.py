"""Shared-expert slot fill and ascending-id order on routing results, against
the oracle, through the C ABI (GPU only)."""
import numpy as np
import pytest
import torch

import moe_expert_routing_token_b200 as moe
import oracle
from moe_expert_routing_token_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _routed(M, k, seed):
    """A DeepSeek-V3 style result: 8 routed experts + one slot for the shared expert."""
    d = inputs.make("biased", M, seed=seed)
    w, ids = moe.biased_grouped_topk(d["logits"].to(DEV), d["bias"].to(DEV), k, True, 8, 4, 2.5)
    return w, ids


@pytest.mark.parametrize("M,k", [(1, 9), (1000, 9), (16384, 9), (333, 1), (257, 32)])
@pytest.mark.parametrize("rsf", [2.5, None])
def test_fill_shared_expert_slot(M, k, rsf):
    if k == 32:
        g = torch.Generator().manual_seed(M)
        w = torch.rand(M, k, generator=g).to(DEV)
        ids = torch.randint(0, 256, (M, k), generator=g, dtype=torch.int32).to(DEV)
    else:
        w, ids = _routed(M, k, seed=M + k)
    num_shared = 3
    pick = torch.randint(0, num_shared, (M,), generator=torch.Generator().manual_seed(7),
                         dtype=torch.int32).to(DEV)
    w0, ids0 = w.cpu().numpy(), ids.cpu().numpy()
    moe.fill_shared_expert_slot(w, ids, 256, num_shared, pick, rsf)
    torch.cuda.synchronize()
    w_ref, ids_ref = oracle.fill_shared_slot(w0, ids0, 256, num_shared, pick.cpu().numpy(), rsf)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    got = w.cpu().numpy().astype(np.float64)
    assert np.array_equal(got[:, :-1], w0[:, :-1].astype(np.float64))       # other slots untouched
    # the kernel sums the k-1 positive fp32 weights in order and divides once:
    # at most (k-2) + 1 roundings of 2^-24 relative to the sum
    assert np.allclose(got[:, -1], w_ref[:, -1], rtol=max(k - 1, 1) * 2.0**-24, atol=0.0)


@pytest.mark.parametrize("M,k", [(1, 8), (5000, 8), (16384, 9), (700, 1), (129, 32)])
def test_sort_topk_by_id(M, k):
    g = torch.Generator().manual_seed(M * 3 + k)
    if k in (8, 9):
        w, ids = _routed(M, k, seed=M)
    else:
        w = torch.rand(M, k, generator=g).to(DEV)
        ids = torch.randint(0, 16, (M, k), generator=g, dtype=torch.int32).to(DEV)   # repeated ids
    w0, ids0 = w.cpu().numpy(), ids.cpu().numpy()
    moe.sort_topk_by_id(w, ids)
    torch.cuda.synchronize()
    w_ref, ids_ref = oracle.sort_by_id(w0, ids0)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.array_equal(w.cpu().numpy().astype(np.float64), w_ref)       # a permutation: exact


def test_fill_then_sort_composes():
    w, ids = _routed(4096, 9, seed=5)
    pick = torch.zeros(4096, dtype=torch.int32, device=DEV)
    moe.fill_shared_expert_slot(w, ids, 256, 1, pick, 2.5)
    moe.sort_topk_by_id(w, ids)
    torch.cuda.synchronize()
    ids_h = ids.cpu().numpy()
    assert np.all(np.diff(ids_h, axis=1) >= 0) and np.all(ids_h[:, -1] == 256)


@pytest.mark.parametrize("M,k,num_shared,seed,offset", [
    (1, 9, 1, 0, 0),
    (1000, 9, 3, 2025, 0),
    (16384, 9, 2, 7, 123456789),
    (4097, 9, 5, 2**63 + 11, 2**64 - 100),   # the counter carries into its second word
    (257, 32, 7, 99, 5),
])
@pytest.mark.parametrize("rsf", [2.5, None])
def test_fill_shared_expert_slot_philox(M, k, num_shared, seed, offset, rsf):
    """The library's seeded draw: the shared experts bit-exact with the
    oracle's Philox4x64-10 picks; the weights as for the explicit draw."""
    if k == 32:
        g = torch.Generator().manual_seed(M)
        w = torch.rand(M, k, generator=g).to(DEV)
        ids = torch.randint(0, 256, (M, k), generator=g, dtype=torch.int32).to(DEV)
    else:
        w, ids = _routed(M, k, seed=M + k)
    w0, ids0 = w.cpu().numpy(), ids.cpu().numpy()
    moe.fill_shared_expert_slot_philox(w, ids, 256, num_shared, seed, offset, rsf)
    torch.cuda.synchronize()
    pick = oracle.shared_pick_philox(M, num_shared, seed, offset)
    w_ref, ids_ref = oracle.fill_shared_slot(w0, ids0, 256, num_shared, pick, rsf)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    got = w.cpu().numpy().astype(np.float64)
    assert np.array_equal(got[:, :-1], w0[:, :-1].astype(np.float64))
    assert np.allclose(got[:, -1], w_ref[:, -1], rtol=max(k - 1, 1) * 2.0**-24, atol=0.0)


def test_philox_draws_advance_with_offset():
    """Consecutive calls with offset advanced by M give the draws of one call
    over 2M rows; the same (seed, offset) repeats them."""
    M = 3000
    w, ids = _routed(2 * M, 9, seed=1)
    a_w, a_ids = w[:M].clone(), ids[:M].clone()
    b_w, b_ids = w[M:].clone(), ids[M:].clone()
    moe.fill_shared_expert_slot_philox(w, ids, 256, 4, 31, 1000, 2.5)
    moe.fill_shared_expert_slot_philox(a_w, a_ids, 256, 4, 31, 1000, 2.5)
    moe.fill_shared_expert_slot_philox(b_w, b_ids, 256, 4, 31, 1000 + M, 2.5)
    torch.cuda.synchronize()
    assert torch.equal(ids[:M], a_ids) and torch.equal(ids[M:], b_ids)
    c_w, c_ids = w[:M].clone(), ids[:M].clone()
    moe.fill_shared_expert_slot_philox(c_w, c_ids, 256, 4, 31, 1000, 2.5)
    torch.cuda.synchronize()
    assert torch.equal(c_ids, a_ids)
