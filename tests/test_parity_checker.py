"""The parity checker itself (CPU): planted mistakes are caught, legitimate
alternatives at near ties are accepted."""
import numpy as np
import torch

import oracle
from oracle import parity

E, G, TG, K = 256, 8, 4, 8
S = E // G


def _route(x):
    return oracle.biased_grouped_topk(x, torch.zeros(E), K, True, G, TG, 2.5)


def _weights(orc, ids):
    pw = np.take_along_axis(orc.scores, ids, axis=1)
    return pw / pw.sum(axis=1, keepdims=True) * 2.5


def _check(orc, ids):
    return parity.compare(_weights(orc, ids), ids, orc, E=E, G=G, TG=TG, k=K, renorm=True, rsf=2.5,
                          fp32_logits=True)


def _logits(seed, M=32):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(M, E, generator=g) * 2.0).to(torch.float64)


def test_oracle_answer_passes():
    orc = _route(_logits(1))
    assert _check(orc, orc.ids.astype(np.int64)).ok()


def test_swapped_order_in_a_clear_row_fails():
    orc = _route(_logits(2))
    ids = orc.ids.astype(np.int64).copy()
    r = int(np.nonzero((orc.margins[:, 0] > 1e-5) & (orc.margins[:, 1] > 1e-5) & (orc.margins[:, 2] > 1e-5))[0][0])
    ids[r, [0, 1]] = ids[r, [1, 0]]
    assert not _check(orc, ids).ok()


def test_wrong_expert_in_a_clear_row_fails():
    orc = _route(_logits(3))
    ids = orc.ids.astype(np.int64).copy()
    r = int(np.nonzero((orc.margins[:, 0] > 1e-5) & (orc.margins[:, 1] > 1e-5))[0][0])
    g = ids[r, K - 1] // S
    spare = [e for e in range(g * S, (g + 1) * S) if e not in ids[r]]
    ids[r, K - 1] = spare[0]
    assert not _check(orc, ids).ok()


def _tied_groups_row():
    """One row where each group's score is set by two equal top experts and
    groups 3 and 5 tie exactly for the last kept place."""
    x = torch.full((1, E), -5.0, dtype=torch.float64)
    top = [3.0, 2.9, 2.8, 2.7, 1.0, 2.7, 1.2, 1.1]
    for gi, v in enumerate(top):
        x[0, gi * S + 7] = v
        x[0, gi * S + 19] = v
    return x


def test_other_group_at_an_exact_group_tie_passes():
    x = _tied_groups_row()
    orc = _route(x)
    assert orc.margins[0, 1] == 0.0
    # the same routing with the tie broken the other way
    x2 = x.clone()
    x2[0, 3 * S:4 * S] -= 1e-6
    alt = _route(x2).ids.astype(np.int64)
    assert set((alt[0] // S).tolist()) != set((orc.ids[0] // S).tolist())
    assert _check(orc, alt).ok()


def test_worse_expert_of_a_kept_group_at_a_group_tie_fails():
    x = _tied_groups_row()
    orc = _route(x)
    x2 = x.clone()
    x2[0, 3 * S:4 * S] -= 1e-6
    alt = _route(x2).ids.astype(np.int64)
    # replace the weakest pick by an expert of the same group that scores lower
    g = alt[0, K - 1] // S
    s = orc.sel[0]
    lower = [e for e in range(g * S, (g + 1) * S) if e not in alt[0] and s[e] < s[alt[0, K - 1]] - 1e-3]
    bad = alt.copy()
    bad[0, K - 1] = lower[0]
    assert not _check(orc, bad).ok()


def test_expert_of_a_clearly_dropped_group_fails():
    orc = _route(_logits(5))
    ids = orc.ids.astype(np.int64).copy()
    r = 0
    worst = int(np.argmin(orc.group_scores[r]))
    ids[r, K - 1] = worst * S
    assert not _check(orc, ids).ok()


def test_weight_error_fails():
    orc = _route(_logits(6))
    ids = orc.ids.astype(np.int64)
    w = _weights(orc, ids)
    w[3, 2] += 1e-5
    rep = parity.compare(w, ids, orc, E=E, G=G, TG=TG, k=K, renorm=True, rsf=2.5, fp32_logits=True)
    assert not rep.ok()
