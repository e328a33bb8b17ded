"""moe_expert_permutation (expert-sorted token permutation) against the oracle,
bit-exact, through the C ABI (GPU only)."""
import numpy as np
import pytest
import torch

import moe_expert_routing_token_b200 as moe
import oracle
from moe_expert_routing_token_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _check(ids, E, w=None, workspace=None):
    counts, offsets, gather, scatter, gate = moe.expert_permutation(
        ids.to(DEV), E, None if w is None else w.to(DEV), workspace=workspace)
    torch.cuda.synchronize()
    ref = oracle.expert_permutation(ids, E, w)
    nv = int(ref.offsets[-1])
    assert np.array_equal(counts.cpu().numpy(), ref.counts)
    assert np.array_equal(offsets.cpu().numpy(), ref.offsets)
    assert np.array_equal(gather.cpu().numpy()[:nv], ref.gather[:nv])
    assert np.array_equal(scatter.cpu().numpy(), ref.scatter)
    if w is not None:
        assert np.array_equal(gate.cpu().numpy()[:nv], ref.gate[:nv].astype(np.float32))
    return counts, offsets, gather, scatter, gate


def _random_ids(M, k, E, seed, distinct=True):
    g = torch.Generator().manual_seed(seed)
    if distinct and k <= E:
        return torch.argsort(torch.rand(M, E, generator=g), dim=1)[:, :k].to(torch.int32).contiguous()
    return torch.randint(0, E, (M, k), generator=g, dtype=torch.int32)


@pytest.mark.parametrize("M,k,E", [(1, 1, 8), (7, 2, 16), (1000, 6, 160), (5000, 8, 256), (2049, 3, 33),
                                   (3000, 8, 1024), (128, 8, 256), (129, 8, 256)])
@pytest.mark.parametrize("with_weights", [True, False])
def test_random_ids(M, k, E, with_weights):
    ids = _random_ids(M, k, E, seed=M * 7 + k)
    w = torch.rand(M, k, generator=torch.Generator().manual_seed(M)) if with_weights else None
    _check(ids, E, w)


@pytest.mark.parametrize("M,k,E", [(65536, 8, 256),    # 512 tiles of 1024 pairs: the two-launch path
                                   (65537, 8, 256),    # 513 tiles: count, scan, scatter
                                   (40000, 16, 64)])   # 625 tiles, few experts
def test_tile_count_paths(M, k, E):
    _check(_random_ids(M, k, E, seed=M + k), E, torch.rand(M, k, generator=torch.Generator().manual_seed(k)))


def test_repeated_ids_and_one_hot_expert():
    _check(_random_ids(777, 5, 12, seed=3, distinct=False), 12)
    _check(torch.full((513, 4), 3, dtype=torch.int32), 8, torch.rand(513, 4))


def test_routed_ids_at_benchmark_size():
    d = inputs.make("sigmoid", 16384)
    w, ids = moe.biased_grouped_topk(d["logits"].to(DEV), d["bias"].to(DEV), 8, True, 1, 1, 1.0)
    torch.cuda.synchronize()
    _check(ids.cpu(), 256, w.cpu())


def test_ids_outside_the_expert_range_are_skipped():
    ids = _random_ids(300, 4, 64, seed=5, distinct=False)
    ids[::7, 1] = -1
    ids[::11, 2] = 64
    ids[5, 0] = 1 << 30
    _, offsets, _, scatter, _ = _check(ids, 64)
    assert int(offsets[-1]) < 300 * 4
    assert bool((scatter.cpu().view(300, 4)[::7, 1] == -1).all())


def test_empty_batch():
    counts, offsets, gather, scatter, gate = moe.expert_permutation(
        torch.empty(0, 8, dtype=torch.int32, device=DEV), 256)
    torch.cuda.synchronize()
    assert int(counts.abs().sum()) == 0 and int(offsets.abs().sum()) == 0 and gather.numel() == 0


def test_deterministic_with_reused_workspace():
    ids = _random_ids(9000, 8, 256, seed=11)
    need = moe.expert_permutation_workspace_size(9000, 8, 256)
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device=DEV)   # no initial contents needed
    a = _check(ids, 256, workspace=ws)
    b = _check(ids, 256, workspace=ws)
    for x, y in zip(a[:4], b[:4]):
        assert torch.equal(x, y)


def test_workspace_not_16_byte_aligned():
    """A workspace that 16-byte loads cannot read takes the three-launch path;
    the result is the same."""
    ids = _random_ids(3000, 8, 256, seed=12)
    need = moe.expert_permutation_workspace_size(3000, 8, 256)
    buf = torch.full((need + 16,), 0xCD, dtype=torch.uint8, device=DEV)
    a = _check(ids, 256, workspace=buf[4:4 + need])
    b = _check(ids, 256)
    for x, y in zip(a[:4], b[:4]):
        assert torch.equal(x, y)
