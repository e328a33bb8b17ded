"""The Python binding rejects operands spread over several GPUs before it
touches the library (CPU only: duck-typed stand-ins for CUDA tensors)."""
import math

import pytest
import torch

import moe_expert_routing_token_b200 as moe


class FakeCuda:
    """Enough of a CUDA tensor for the binding's checks; its memory is never
    read, so data_ptr() fails the test if a call gets that far."""

    is_cuda = True

    def __init__(self, shape, dtype, device):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device(device)

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return True

    def numel(self):
        return math.prod(self.shape)

    def element_size(self):
        return torch.empty((), dtype=self.dtype).element_size()

    def data_ptr(self):
        raise AssertionError("the binding must reject these operands before passing pointers")


def test_fused_router_weight_on_another_gpu():
    h = FakeCuda((64, 7168), torch.bfloat16, "cuda:0")
    w = FakeCuda((7168, 256), torch.bfloat16, "cuda:1")
    with pytest.raises(ValueError, match="router_weight is on cuda:1"):
        moe.fused_router_topk(h, w, None, 8, True, 8, 4, 2.5)


def test_fused_router_workspace_on_another_gpu():
    h = FakeCuda((64, 7168), torch.bfloat16, "cuda:0")
    w = FakeCuda((7168, 256), torch.bfloat16, "cuda:0")
    ws = FakeCuda((1 << 20,), torch.uint8, "cuda:1")
    with pytest.raises(ValueError, match="workspace is on cuda:1"):
        moe.fused_router_topk(h, w, None, 8, True, 8, 4, 2.5, workspace=ws)


def test_bias_on_another_gpu():
    x = FakeCuda((16, 256), torch.bfloat16, "cuda:0")
    b = FakeCuda((256,), torch.float32, "cuda:1")
    with pytest.raises(ValueError, match="correction_bias"):
        moe.biased_grouped_topk(x, b, 8, True, 8, 4, 2.5)


def test_permutation_operands_on_two_gpus():
    ids = FakeCuda((16, 8), torch.int32, "cuda:0")
    with pytest.raises(ValueError, match="topk_weights is on cuda:1"):
        moe.expert_permutation(ids, 256, topk_weights=FakeCuda((16, 8), torch.float32, "cuda:1"))
    with pytest.raises(ValueError, match="workspace is on cuda:2"):
        moe.expert_permutation(ids, 256, workspace=FakeCuda((4096,), torch.uint8, "cuda:2"))


def test_postprocess_operands_on_two_gpus():
    w = FakeCuda((16, 9), torch.float32, "cuda:1")
    ids = FakeCuda((16, 9), torch.int32, "cuda:0")
    with pytest.raises(ValueError, match="topk_weights is on cuda:1"):
        moe.sort_topk_by_id(w, ids)
    w0 = FakeCuda((16, 9), torch.float32, "cuda:0")
    pick = FakeCuda((16,), torch.int32, "cuda:1")
    with pytest.raises(ValueError, match="shared_pick is on cuda:1"):
        moe.fill_shared_expert_slot(w0, ids, 256, 1, pick, 2.5)
