"""Parity of the direct routing kernel (E = 256, k <= 8, batches above 3072
rows; fp32 E = 160 above 4096 rows) against the oracle, element by element
(GPU only).

Batches of more than 3072 rows with E = 256 and every group kept, or eight
groups, take the direct kernel: eight lanes per row, a threshold from block
maxima, candidates ranked by counting.  The cases cover its key modes
(approximate sigmoid keys, exact grouped keys, raw logits), k = 8 and the
sorted k-th path for k < 8, fp32 and bf16 logits, a ragged last octet, and
the three ways a row is ranked:

* the straight-line path (every row of the warp has at most 16 candidates);
* the general list path (some row has 17..32 candidates);
* the whole-warp path (more than 32 candidates, or all keys equal).
"""
import pytest
import torch

from moe_expert_routing_token_b200 import inputs
from tests.test_gpu_routing import check, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

# (op, G, TG, k, renorm, rsf, bias)
SHAPES = [
    ("sigmoid", 1, 1, 8, True, 1.0, True),    # approximate keys (the benchmark shape)
    ("sigmoid", 1, 1, 6, False, 2.5, True),   # approximate keys, k < 8, no renormalisation
    ("sigmoid", 1, 1, 8, True, 1.0, False),   # raw logits order the sigmoid scores
    ("sigmoid", 8, 4, 8, True, 2.5, True),    # grouped, exact keys (DeepSeek-V3)
    ("sigmoid", 8, 2, 3, True, 1.0, True),    # grouped, two groups kept, k = 3
    ("sigmoid", 8, 8, 4, True, 1.0, True),    # every group kept: approximate keys, k = 4
    ("softmax", 1, 1, 8, True, 1.0, False),   # raw logits
    ("softmax", 1, 1, 5, False, 1.0, False),  # raw logits, the full softmax denominator
    ("softmax", 8, 3, 6, True, 1.0, False),   # grouped softmax
]


@pytest.mark.parametrize("op,G,TG,k,renorm,rsf,use_bias", SHAPES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("M", [3073, 4099, 9001])
def test_direct_shapes(op, G, TG, k, renorm, rsf, use_bias, dtype, M):
    x = inputs.random_logits(M, 256, 2.0, dtype, seed=M + 13 * G + k)
    bias = inputs.random_bias(256, 0.05, seed=G + k) if use_bias else None
    check(op, x, bias, k, renorm, G, TG, rsf)


def _crowded_rows(M, n_close, dtype, seed, every=1):
    """N(0, 2^2) logits; in every `every`-th row, n_close experts drawn from
    [6.5, 8.5], whose sigmoids lie within 1.5e-3 of one another, so that all
    of them fall inside the candidate band."""
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(M, 256, generator=gen) * 2.0
    rows = torch.arange(0, M, every)
    idx = torch.stack([torch.randperm(256, generator=gen)[:n_close] for _ in range(len(rows))])
    vals = 6.5 + 2.0 * torch.rand(len(rows), n_close, generator=gen)
    x[rows] = x[rows].scatter(1, idx, vals)
    return x.to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("n_close,every", [(24, 1), (24, 7), (40, 5)])
@pytest.mark.parametrize("G,TG", [(1, 1), (8, 4)])
def test_crowded_rows(dtype, n_close, every, G, TG):
    """17..32 candidates take the general list path, more than 32 the
    whole-warp path; with `every` > 1 those rows share warps with rows on
    the straight-line path."""
    M = 6000
    x = _crowded_rows(M, n_close, dtype, seed=n_close * 10 + every + G, every=every)
    bias = inputs.random_bias(256, 2e-5, seed=3)
    check("sigmoid", x, bias, 8, True, G, TG, 1.0)


@pytest.mark.parametrize("op,G,TG,k", [("sigmoid", 1, 1, 8), ("sigmoid", 8, 4, 8), ("softmax", 1, 1, 6)])
def test_equal_rows_pick_lowest_indices(op, G, TG, k):
    """Rows of equal logits among ordinary rows: the lowest admissible
    indices win, exactly as in the oracle."""
    import numpy as np
    M = 5003
    x = inputs.random_logits(M, 256, 2.0, torch.bfloat16, seed=11)
    x[::9] = 0.0
    w, ids = run_gpu(op, x, None, k, True, G, TG, 1.0)
    orc = run_oracle(op, x, None, k, True, G, TG, 1.0)
    assert np.array_equal(ids[::9], orc.ids[::9])
    check(op, x, None, k, True, G, TG, 1.0)


# fp32 E = 160, eight groups of 20 (one lane each when grouped)
SHAPES_160 = [
    ("softmax", 8, 3, 6, False, 1.0, False),  # grouped softmax, the full denominator (DeepSeek-V2)
    ("softmax", 1, 1, 6, True, 1.0, False),   # raw logits
    ("sigmoid", 8, 4, 8, True, 2.5, True),    # grouped, exact keys
    ("sigmoid", 1, 1, 4, True, 1.0, True),    # approximate keys, k = 4
]


@pytest.mark.parametrize("op,G,TG,k,renorm,rsf,use_bias", SHAPES_160)
@pytest.mark.parametrize("M", [5003, 9001])
def test_e160_fp32_shapes(op, G, TG, k, renorm, rsf, use_bias, M):
    x = inputs.random_logits(M, 160, 1.5, torch.float32, seed=M + 7 * G + k)
    bias = inputs.random_bias(160, 0.05, seed=G + k + 1) if use_bias else None
    check(op, x, bias, k, renorm, G, TG, rsf)


@pytest.mark.parametrize("n_close,every", [(20, 1), (40, 3)])
@pytest.mark.parametrize("op,G,TG,k", [("softmax", 8, 3, 6), ("sigmoid", 1, 1, 8)])
def test_e160_crowded_rows(n_close, every, op, G, TG, k):
    """fp32 E = 160 rows with 20 or 40 experts close together: the general
    list path and the whole-warp path of the 20-experts-per-lane form."""
    M, E = 6007, 160
    gen = torch.Generator().manual_seed(n_close + every + G)
    x = torch.randn(M, E, generator=gen) * 1.5
    rows = torch.arange(0, M, every)
    idx = torch.stack([torch.randperm(E, generator=gen)[:n_close] for _ in range(len(rows))])
    vals = 6.5 + 2.0 * torch.rand(len(rows), n_close, generator=gen)
    x[rows] = x[rows].scatter(1, idx, vals)
    bias = inputs.random_bias(E, 2e-5, seed=4) if op == "sigmoid" else None
    check(op, x, bias, k, True, G, TG, 1.0)
