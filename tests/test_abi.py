"""The C-ABI library loads, exports every declared symbol and validates its
arguments on the host (CPU only: no compute call needs a GPU here)."""
import ctypes
import os
import re

import pytest

import moe_expert_routing_token_b200 as moe
from moe_expert_routing_token_b200 import routing

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_routing.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return moe.lib()


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ("moe_topk_softmax", "moe_grouped_topk", "moe_biased_grouped_topk",
              "moe_fused_router_topk", "moe_fused_router_workspace_size"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in routing.SIGNATURES, f"binding lacks {name}"


def test_version_and_status_strings(lib):
    assert lib.moe_abi_version() == 5
    assert lib.moe_status_string(0) == b"MOE_OK"
    assert lib.moe_status_string(1) == b"MOE_ERR_INVALID_ARG"
    assert lib.moe_status_string(2) == b"MOE_ERR_UNSUPPORTED"
    assert lib.moe_status_string(3) == b"MOE_ERR_CUDA"


# Host-side validation returns before any CUDA call, so it runs without a GPU.
P = 4096  # a non-null dummy address; never dereferenced on these paths


@pytest.mark.parametrize("args,status,needle", [
    # moe_grouped_topk(logits, dtype, M, E, topk, renorm, G, TG, rsf, w, ids, stream)
    ((P, 0, 4, 8, 2, 1, 3, 1, 1.0, P, P, None), 1, "does not divide"),
    ((P, 0, 4, 8, 2, 1, 4, 5, 1.0, P, P, None), 1, "topk_group"),
    ((P, 0, 4, 8, 2, 1, 4, 0, 1.0, P, P, None), 1, "topk_group"),
    ((P, 0, 4, 8, 5, 1, 4, 2, 1.0, P, P, None), 1, "topk=5"),
    ((P, 0, 4, 8, 0, 1, 4, 2, 1.0, P, P, None), 1, "topk=0"),
    ((P, 7, 4, 8, 2, 1, 4, 2, 1.0, P, P, None), 1, "dtype"),
    ((P, 0, -1, 8, 2, 1, 4, 2, 1.0, P, P, None), 1, "M=-1"),
    ((P, 0, 4, 0, 2, 1, 1, 1, 1.0, P, P, None), 1, "E=0"),
    ((P, 0, 4, 8, 2, 1, 4, 2, float("nan"), P, P, None), 1, "scaling"),
    ((None, 0, 4, 8, 2, 1, 4, 2, 1.0, P, P, None), 1, "null"),
    ((P, 0, 4, 8, 2, 1, 4, 2, 1.0, None, P, None), 1, "null"),
    ((P + 2, 0, 4, 8, 2, 1, 4, 2, 1.0, P, P, None), 1, "aligned"),
    ((P, 0, 4, 2048, 2, 1, 1, 1, 1.0, P, P, None), 2, "E=2048"),
    ((P, 0, 4, 64, 33, 1, 1, 1, 1.0, P, P, None), 2, "topk=33"),
])
def test_grouped_topk_validation(lib, args, status, needle):
    assert lib.moe_grouped_topk(*args) == status
    assert needle in lib.moe_last_error().decode()


def test_empty_batch_is_ok_without_launch(lib):
    assert lib.moe_topk_softmax(None, 0, 0, 8, 2, 1, None, None, None) == 0
    assert lib.moe_biased_grouped_topk(None, 1, None, 0, 256, 8, 1, 8, 4, 2.5, None, None, None) == 0


def test_softcap_validation(lib):
    # moe_grouped_topk_softcap(logits, dtype, M, E, topk, renorm, G, TG, rsf, softcap, w, ids, stream)
    for c in (float("nan"), float("inf"), -float("inf")):
        for M in (4, 0):                                  # rejected even for an empty batch
            assert lib.moe_grouped_topk_softcap(P, 0, M, 8, 2, 1, 4, 2, 1.0, c, P, P, None) == 1
            assert b"softcap" in lib.moe_last_error()
    assert lib.moe_grouped_topk_softcap(None, 0, 0, 8, 2, 1, 4, 2, 1.0, 30.0, None, None, None) == 0


def test_biased_validation(lib):
    # bias pointer not 4-byte aligned
    assert lib.moe_biased_grouped_topk(P, 1, P + 1, 4, 256, 8, 1, 8, 4, 2.5, P, P, None) == 1
    assert lib.moe_biased_grouped_topk(P, 1, None, 4, 256, 8, 1, 8, 9, 2.5, P, P, None) == 1


def test_fused_router_workspace_query(lib):
    assert lib.moe_fused_router_workspace_size(-1, 7168, 256) == ctypes.c_size_t(-1).value
    n = lib.moe_fused_router_workspace_size(64, 7168, 256)
    assert n != ctypes.c_size_t(-1).value


def test_fused_router_rejects_huge_batches(lib):
    # (hidden, W, layout, bias, M, K, E, topk, renorm, G, TG, rsf, w, ids, logits_out, ws, ws_bytes, stream)
    assert lib.moe_fused_router_topk(P, P, 0, None, 1 << 31, 7168, 256, 8, 1, 8, 4, 2.5, P, P, None,
                                     None, 0, None) == 2
    assert b"2^31" in lib.moe_last_error()


def test_top1_router_validation(lib):
    # (hidden, W, layout, M, K, E, softcap, w, ids, logits_out, stream)
    assert lib.moe_fused_router_top1(P, P, 1, -1, 64, 8, 0.0, P, P, None, None) == 1      # M < 0
    assert lib.moe_fused_router_top1(P, P, 1, 4, 0, 8, 0.0, P, P, None, None) == 1        # K < 1
    assert lib.moe_fused_router_top1(P, P, 2, 4, 64, 8, 0.0, P, P, None, None) == 1       # layout
    assert lib.moe_fused_router_top1(P, P, 1, 4, 64, 8, float("nan"), P, P, None, None) == 1
    assert b"softcap" in lib.moe_last_error()
    # E > 8 only on the tensor-core kernel: (E, K) layout, K % 64 == 0, E <= 256
    assert lib.moe_fused_router_top1(P, P, 0, 4, 64, 9, 0.0, P, P, None, None) == 2       # (K, E) layout
    assert b"tensor-core" in lib.moe_last_error()
    assert lib.moe_fused_router_top1(P, P, 1, 4, 72, 9, 0.0, P, P, None, None) == 2       # K % 64
    assert lib.moe_fused_router_top1(P, P, 1, 4, 64, 257, 0.0, P, P, None, None) == 2     # E > 256
    assert lib.moe_fused_router_top1(P, P, 1, 4, 60, 8, 0.0, P, P, None, None) == 2       # K % 8
    assert lib.moe_fused_router_top1(None, P, 1, 4, 64, 8, 0.0, P, P, None, None) == 1    # null
    assert lib.moe_fused_router_top1(P + 8, P, 1, 4, 64, 8, 0.0, P, P, None, None) == 1   # 16-B alignment
    assert b"aligned" in lib.moe_last_error()
    assert lib.moe_fused_router_top1(None, None, 0, 0, 64, 8, 30.0, None, None, None, None) == 0  # empty


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(4, 8)
    with pytest.raises(ValueError):
        moe.topk_softmax(x, 2, True)


def test_expert_permutation_validation(lib):
    ws = lib.moe_expert_permutation_workspace_size(16384, 8, 256)
    assert ws == 128 * 256 * 4                       # one int32 per (1024-pair tile, expert)
    assert lib.moe_expert_permutation_workspace_size(10, 8, 2048) == ctypes.c_size_t(-1).value
    # (ids, weights, M, k, E, counts, offsets, gather, scatter, gate, workspace, bytes, stream)
    assert lib.moe_expert_permutation(P, None, 4, 0, 16, P, P, P, P, None, P, 4096, None) == 1   # k < 1
    assert lib.moe_expert_permutation(P, None, 4, 2, 2048, P, P, P, P, None, P, 4096, None) == 2  # E > 1024
    assert b"E=2048" in lib.moe_last_error()
    assert lib.moe_expert_permutation(P, P, 4, 2, 16, P, P, P, P, None, P, 4096, None) == 1     # gate missing
    assert lib.moe_expert_permutation(P, None, 4, 2, 16, P, P, P, P, None, P, 3, None) == 1     # workspace short
    assert b"workspace" in lib.moe_last_error()
    assert lib.moe_expert_permutation(P, None, 4, 2, 16, None, P, P, P, None, P, 4096, None) == 1  # no counts
    # M*k at or beyond 2^31, including products that overflow int64
    for M, k in ((1 << 28, 8), (1 << 40, 8), (1 << 62, 32)):
        assert lib.moe_expert_permutation_workspace_size(M, k, 256) == ctypes.c_size_t(-1).value
        assert lib.moe_expert_permutation(P, None, M, k, 256, P, P, P, P, None, P, 1 << 40, None) == 2
        assert b"2^31" in lib.moe_last_error()


def test_postprocess_validation(lib):
    # (weights, ids, M, k, E, num_shared, pick, rsf, stream)
    assert lib.moe_fill_shared_expert_slot(P, P, 4, 0, 256, 1, P, 2.5, None) == 1       # k < 1
    assert lib.moe_fill_shared_expert_slot(P, P, 4, 33, 256, 1, P, 2.5, None) == 2      # k > 32
    assert lib.moe_fill_shared_expert_slot(P, P, 4, 9, 256, 0, P, 2.5, None) == 1       # no shared expert
    assert lib.moe_fill_shared_expert_slot(P, P, 4, 9, 256, 1, None, 2.5, None) == 1    # no picks
    assert lib.moe_fill_shared_expert_slot(P, P, 4, 9, 256, 1, P, float("nan"), None) == 1
    assert lib.moe_fill_shared_expert_slot(P, P, 0, 9, 256, 1, None, 2.5, None) == 0    # empty: no launch
    # (weights, ids, M, k, E, num_shared, seed, offset, rsf, stream)
    assert lib.moe_fill_shared_expert_slot_philox(P, P, 4, 0, 256, 1, 7, 0, 2.5, None) == 1     # k < 1
    assert lib.moe_fill_shared_expert_slot_philox(P, P, 4, 33, 256, 1, 7, 0, 2.5, None) == 2    # k > 32
    assert lib.moe_fill_shared_expert_slot_philox(P, P, 4, 9, 256, 0, 7, 0, 2.5, None) == 1     # no shared expert
    assert lib.moe_fill_shared_expert_slot_philox(P, P, 4, 9, 256, 1, 7, 0, float("nan"), None) == 1
    assert lib.moe_fill_shared_expert_slot_philox(None, P, 4, 9, 256, 1, 7, 0, 2.5, None) == 1  # null weights
    assert lib.moe_fill_shared_expert_slot_philox(P, P, 0, 9, 256, 1, 7, 0, 2.5, None) == 0     # empty: no launch
    assert lib.moe_sort_topk_by_id(P, None, 4, 8, None) == 1
    assert lib.moe_sort_topk_by_id(P, P, 4, 40, None) == 2
    assert lib.moe_sort_topk_by_id(P, P, 0, 8, None) == 0
