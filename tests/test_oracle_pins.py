"""The CPU oracle agrees with hand-worked closed forms, brute force over
subsets, library routines and its own stated invariants (CPU only)."""
import numpy as np
import pytest
from scipy.special import expit, softmax

import oracle
from moe_expert_routing_token_b200 import inputs
from tests import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(lib, check):
    fails = check(lib)
    assert not fails, "\n".join(fails[:20])


def _invariants(r, x_scores, bias, G, TG, k, renorm, rsf):
    M, E = x_scores.shape
    S = E // G
    s = x_scores + (0.0 if bias is None else bias[None, :])
    for i in range(M):
        ids = r.ids[i]
        assert len(set(ids.tolist())) == k, "ids unique"
        assert ids.min() >= 0 and ids.max() < E
        # kept groups: the TG best by group score, ties to the lower index
        order = sorted(range(G), key=lambda g: (-r.group_scores[i, g], g))
        kept = set(order[:TG])
        assert all(int(e) // S in kept for e in ids), "ids confined to kept groups"
        # descending selection score
        assert all(s[i, ids[j]] >= s[i, ids[j + 1]] for j in range(k - 1))
        w = r.weights[i]
        if renorm:
            assert abs(w.sum() - rsf) <= 1e-12 * max(1.0, rsf)
        else:
            assert np.allclose(w, rsf * x_scores[i, ids], rtol=1e-14)


@pytest.mark.parametrize("name", ["softmax", "sigmoid", "biased", "grouped"])
def test_invariants_on_workloads(lib, name):
    d = inputs.make(name, 64)
    sp = d["spec"]
    x = oracle.as_f64(d["logits"])
    if name in ("softmax", "grouped"):
        r = oracle.grouped_topk(x, sp.topk, sp.renormalize, sp.num_expert_group, sp.topk_group,
                                sp.routed_scaling_factor, lib=lib)
        scores = softmax(x, axis=1)
        bias = None
    else:
        bias = oracle.as_f64(d["bias"])
        r = oracle.biased_grouped_topk(x, bias, sp.topk, sp.renormalize, sp.num_expert_group,
                                       sp.topk_group, sp.routed_scaling_factor, lib=lib)
        scores = expit(x)
    _invariants(r, scores, bias, sp.num_expert_group, sp.topk_group, sp.topk, sp.renormalize,
                sp.routed_scaling_factor)


def test_single_group_equals_plain_sigmoid_topk(lib):
    """num_expert_group=1, topk_group=1 (the aiter call) is plain sigmoid +
    bias top-k: checked against a stable sort of scipy's expit + bias."""
    d = inputs.make("sigmoid", 256)
    x = oracle.as_f64(d["logits"])
    b = oracle.as_f64(d["bias"])
    r = oracle.biased_grouped_topk(x, b, 8, True, 1, 1, lib=lib)
    s = expit(x) + b[None, :]
    ids = np.argsort(-s, axis=1, kind="stable")[:, :8]
    assert np.array_equal(r.ids, ids)


def test_rejects_bad_arguments(lib):
    x = np.zeros((2, 8))
    with pytest.raises(ValueError):
        oracle.grouped_topk(x, 2, True, 3, 1, lib=lib)      # 3 does not divide 8
    with pytest.raises(ValueError):
        oracle.grouped_topk(x, 2, True, 4, 5, lib=lib)      # topk_group > groups
    with pytest.raises(ValueError):
        oracle.grouped_topk(x, 5, True, 4, 2, lib=lib)      # k > admissible experts


def test_empty_batch(lib):
    r = oracle.topk_softmax(np.zeros((0, 8)), 2, True, lib=lib)
    assert r.ids.shape == (0, 2)
