"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each check takes an oracle library handle and returns a list of failure
strings (empty = pass), so the same checks can be run against the real
oracle (tests/test_oracle_pins.py) and against deliberately broken copies of
its source (tests/test_oracle_mutants.py), proving that a plausible slip in
the oracle would be caught.

Pins used:
* golden hand-worked cases (tests/golden/*.json, closed forms, each cited);
* brute force: the kept groups are the topk_group-subset with the largest
  total group score, and the picks are the k-subset of admissible experts
  with the largest total selection score (unique for distinct values);
* library cross-checks for the ungrouped cases: scipy's softmax / expit and a
  stable numpy argsort reproduce the scores, ids and weights;
* the router projection against numpy's float64 matmul and a hand case;
* the expert permutation against a hand case, and against numpy's stable
  argsort, bincount and cumsum on random and routed ids (plus its inverse-
  permutation and stability invariants);
* softcapping against the closed form tanh(ln(a) / 2) = (a - 1) / (a + 1), its
  saturation at +-c and the identity at c = 0;
* the fused router's top-1 form against hand cases whose weight is the
  logistic function of the logit gap, and against numpy's arg-max and the
  page's 1 / sum exp(l - max l) on random rows.
"""
from __future__ import annotations

import glob
import itertools
import json
import math
import os

import numpy as np
from scipy.special import expit, softmax

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _logits_from(case):
    if case["logits_from"] == "ln(u)":
        return np.log(np.asarray(case["u"], dtype=np.float64))[None, :]
    if case["logits_from"] == "logit(p)":
        p = np.asarray(case["p"], dtype=np.float64)
        return np.log(p / (1.0 - p))[None, :]
    raise ValueError(case["logits_from"])


def _run_case(case, lib):
    x = _logits_from(case)
    op = case["op"]
    if op == "topk_softmax":
        return oracle.topk_softmax(x, case["topk"], case["renormalize"], lib=lib)
    if op == "grouped_topk":
        return oracle.grouped_topk(x, case["topk"], case["renormalize"], case["num_expert_group"],
                                   case["topk_group"], case["routed_scaling_factor"], lib=lib)
    if op == "biased_grouped_topk":
        return oracle.biased_grouped_topk(x, np.asarray(case["bias"], np.float64), case["topk"],
                                          case["renormalize"], case["num_expert_group"],
                                          case["topk_group"], case["routed_scaling_factor"],
                                          lib=lib)
    raise ValueError(op)


def check_golden(lib) -> list[str]:
    fails = []
    for path in sorted(glob.glob(os.path.join(GOLDEN, "*_e8.json"))):
        doc = json.load(open(path))
        for n, case in enumerate(doc["cases"]):
            try:
                r = _run_case(case, lib)
            except Exception as exc:  # a broken oracle may reject valid args
                fails.append(f"{os.path.basename(path)}[{n}]: raised {exc!r}")
                continue
            if r.ids[0].tolist() != case["ids"]:
                fails.append(f"{os.path.basename(path)}[{n}]: ids {r.ids[0].tolist()} != {case['ids']}")
            if not np.allclose(r.weights[0], case["weights"], rtol=0, atol=1e-12):
                fails.append(f"{os.path.basename(path)}[{n}]: weights {r.weights[0]} != {case['weights']}")
    return fails


def check_router_golden(lib) -> list[str]:
    doc = json.load(open(os.path.join(GOLDEN, "router_logits_small.json")))
    h = np.asarray(doc["hidden"], np.float64)
    w = np.asarray(doc["weight_ke"], np.float64)
    fails = []
    got = oracle.router_logits(h, w, weight_layout=0, lib=lib)
    if not np.array_equal(got, np.asarray(doc["logits"])):
        fails.append(f"router (K,E) hand case: {got.tolist()}")
    got_t = oracle.router_logits(h, np.ascontiguousarray(w.T), weight_layout=1, lib=lib)
    if not np.array_equal(got_t, np.asarray(doc["logits"])):
        fails.append(f"router (E,K) hand case: {got_t.tolist()}")
    return fails


def check_router_numpy(lib, seed=7) -> list[str]:
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((5, 37))
    w = rng.standard_normal((37, 11))
    ref = h @ w
    fails = []
    for layout, wt in ((0, w), (1, np.ascontiguousarray(w.T))):
        got = oracle.router_logits(h, wt, weight_layout=layout, lib=lib)
        if not np.allclose(got, ref, rtol=1e-12, atol=1e-12):
            fails.append(f"router layout {layout}: max err {np.abs(got - ref).max()}")
    return fails


# --------------------------------------------------------------------------
# brute force over subsets
# --------------------------------------------------------------------------
def _brute(s, G, TG, k, group_kind):
    """Independent formulation: best TG-subset of groups by total group score,
    then the best k-subset of their experts by total selection score."""
    E = len(s)
    S = E // G
    gs = []
    for g in range(G):
        vals = sorted(s[g * S:(g + 1) * S], reverse=True)
        gs.append(vals[0] if group_kind == oracle.GROUP_MAX else sum(vals[:2]))
    best_groups = max(itertools.combinations(range(G), TG), key=lambda c: sum(gs[g] for g in c))
    adm = [e for e in range(E) if e // S in best_groups]
    best = max(itertools.combinations(adm, k), key=lambda c: sum(s[e] for e in c))
    return set(best_groups), set(best)


def check_brute(lib, trials=150, seed=11) -> list[str]:
    rng = np.random.default_rng(seed)
    fails = []
    shapes = [(8, 1, 1, 2), (8, 4, 2, 3), (8, 2, 1, 4), (12, 3, 2, 5), (12, 4, 3, 4),
              (12, 6, 2, 3), (10, 5, 4, 6), (9, 3, 1, 3), (6, 6, 3, 3), (12, 12, 5, 5)]
    for t in range(trials):
        E, G, TG, k = shapes[t % len(shapes)]
        x = rng.standard_normal((1, E)) * 2.0
        kind = t % 3
        if kind == 0:   # softmax, group max
            r = oracle.grouped_topk(x, k, True, G, TG, lib=lib)
            p = softmax(x[0])
            s = p
            gk = oracle.GROUP_MAX
        else:           # sigmoid + bias, sum of top-2
            b = rng.standard_normal(E) * (0.3 if kind == 1 else 0.0)
            r = oracle.biased_grouped_topk(x, b, k, True, G, TG, lib=lib)
            p = expit(x[0])
            s = p + b
            gk = oracle.GROUP_TOP2_SUM
        _, picks = _brute(list(s), G, TG, k, gk)
        got = r.ids[0].tolist()
        if set(got) != picks:
            fails.append(f"brute t={t} E={E} G={G} TG={TG} k={k}: {sorted(got)} != {sorted(picks)}")
            continue
        if any(s[got[j]] < s[got[j + 1]] for j in range(k - 1)):
            fails.append(f"brute t={t}: ids not in descending score order")
        w = p[got]
        w = w / w.sum()
        if not np.allclose(r.weights[0], w, rtol=1e-12, atol=1e-15):
            fails.append(f"brute t={t}: weights {r.weights[0]} != {w}")
    return fails


# --------------------------------------------------------------------------
# library cross-checks (ungrouped cases reduce to a stable sort)
# --------------------------------------------------------------------------
def _stable_topk(s, k):
    # stable sort on -s: equal scores keep ascending index order
    return np.argsort(-s, kind="stable")[:k]


def check_library(lib, seed=5) -> list[str]:
    rng = np.random.default_rng(seed)
    fails = []
    # softmax top-k, E=64, with and without renormalise
    x = rng.standard_normal((40, 64)) * 1.5
    for renorm in (False, True):
        r = oracle.topk_softmax(x, 6, renorm, lib=lib)
        for i in range(x.shape[0]):
            p = softmax(x[i])
            ids = _stable_topk(p, 6)
            w = p[ids] / (p[ids].sum() if renorm else 1.0)
            if r.ids[i].tolist() != ids.tolist():
                fails.append(f"softmax row {i}: ids {r.ids[i]} != {ids}")
                break
            if not np.allclose(r.weights[i], w, rtol=1e-12, atol=1e-15):
                fails.append(f"softmax row {i}: weights")
                break
    # sigmoid + bias, one group (the aiter form), scaled
    x = rng.standard_normal((40, 96)) * 2.0
    b = rng.standard_normal(96) * 0.05
    r = oracle.biased_grouped_topk(x, b, 8, True, 1, 1, 2.5, lib=lib)
    for i in range(x.shape[0]):
        p = expit(x[i])
        ids = _stable_topk(p + b, 8)
        w = 2.5 * p[ids] / p[ids].sum()
        if r.ids[i].tolist() != ids.tolist():
            fails.append(f"sigmoid row {i}: ids {r.ids[i]} != {ids}")
            break
        if not np.allclose(r.weights[i], w, rtol=1e-12, atol=1e-15):
            fails.append(f"sigmoid row {i}: weights")
            break
    # no bias, no renormalise: weights are the plain sigmoid scores
    r = oracle.biased_grouped_topk(x, None, 5, False, 1, 1, lib=lib)
    for i in range(x.shape[0]):
        p = expit(x[i])
        ids = _stable_topk(p, 5)
        if r.ids[i].tolist() != ids.tolist() or not np.allclose(r.weights[i], p[ids], rtol=1e-12):
            fails.append(f"plain sigmoid row {i}")
            break
    # grouping with every group kept (TG == G) equals the ungrouped result
    x = rng.standard_normal((20, 32))
    a = oracle.grouped_topk(x, 4, True, 8, 8, lib=lib)
    c = oracle.topk_softmax(x, 4, True, lib=lib)
    if not (np.array_equal(a.ids, c.ids) and np.allclose(a.weights, c.weights, rtol=1e-14)):
        fails.append("TG == G differs from ungrouped")
    # margins: the expert margin is the gap between the k-th and (k+1)-th score
    r = oracle.biased_grouped_topk(x, None, 4, True, 1, 1, lib=lib)
    for i in range(x.shape[0]):
        srt = np.sort(expit(x[i]))[::-1]
        if not math.isclose(r.margins[i, 0], srt[3] - srt[4], rel_tol=1e-12, abs_tol=1e-15):
            fails.append(f"margin row {i}")
            break
    return fails


def check_permutation_golden(lib) -> list[str]:
    """Hand-worked cases: a plain one, and one whose ids include a shared-expert
    slot (id E, the routing page's §6) and a masked pair (id -1).  Only the
    first offsets[E] entries of gather and gate are defined."""
    fails = []
    for name in ("expert_permutation_small.json", "expert_permutation_out_of_range.json"):
        doc = json.load(open(os.path.join(GOLDEN, name)))
        p = oracle.expert_permutation(np.asarray(doc["topk_ids"], np.int32), doc["num_experts"],
                                      np.asarray(doc["topk_weights"], np.float64), lib=lib)
        placed = int(p.offsets[-1])
        got = {"counts": p.counts.tolist(), "offsets": p.offsets.tolist(), "gather": p.gather[:placed].tolist(),
               "scatter": p.scatter.tolist(), "gate": p.gate[:placed].tolist()}
        for key, val in got.items():
            if val != doc[key]:
                fails.append(f"permutation hand case {name}: {key} {val} != {doc[key]}")
    return fails


def check_permutation_after_shared_slot(lib, seed=29) -> list[str]:
    """The routing page's §6 writes the shared expert's id E + j into the last
    slot; a permutation over the E routed experts then places exactly the
    other k - 1 slots of every row, in the order it gives them without the
    shared slot (pair indices mapped from (token, slot) over k - 1 to k)."""
    rng = np.random.default_rng(seed)
    fails = []
    M, k, E, n_shared = 50, 4, 12, 2
    x = rng.normal(0, 2, size=(M, E))
    r = oracle.topk_softmax(x, k, True, lib=lib)
    w_sh, ids_sh = oracle.fill_shared_slot(r.weights, r.ids, E, n_shared, rng.integers(0, n_shared, M), 2.0,
                                           lib=lib)
    full = oracle.expert_permutation(ids_sh, E, w_sh, lib=lib)
    part = oracle.expert_permutation(ids_sh[:, : k - 1], E, w_sh[:, : k - 1], lib=lib)
    to_full = (part.gather[: int(part.offsets[-1])] // (k - 1)) * k + part.gather[: int(part.offsets[-1])] % (k - 1)
    if not np.array_equal(full.counts, part.counts) or not np.array_equal(full.offsets, part.offsets):
        fails.append("shared slot: counts or offsets include the shared expert's pairs")
    if not np.array_equal(full.gather[: int(full.offsets[-1])], to_full):
        fails.append("shared slot: placed pairs differ from the permutation without that slot")
    if not np.all(full.scatter.reshape(M, k)[:, k - 1] == -1):
        fails.append("shared slot: a shared-expert pair has a position")
    return fails


def check_permutation_numpy(lib, seed=13) -> list[str]:
    """numpy's stable argsort / bincount / cumsum define the same permutation."""
    rng = np.random.default_rng(seed)
    fails = []
    cases = [(rng.integers(0, 16, size=(37, 3)), 16), (rng.integers(0, 3, size=(50, 2)), 8),
             (np.zeros((9, 4), np.int64), 5), (rng.integers(0, 256, size=(300, 8)), 256)]
    # ids produced by routing (distinct within a row)
    x = rng.normal(0, 2, size=(120, 64))
    cases.append((oracle.topk_softmax(x, 6, True, lib=lib).ids, 64))
    for n, (ids, E) in enumerate(cases):
        ids = np.asarray(ids, np.int32)
        w = rng.random(ids.shape)
        p = oracle.expert_permutation(ids, E, w, lib=lib)
        flat = ids.reshape(-1)
        order = np.argsort(flat, kind="stable")
        counts = np.bincount(flat, minlength=E)
        if not np.array_equal(p.gather, order):
            fails.append(f"permutation case {n}: gather differs from stable argsort")
        if not np.array_equal(p.counts, counts):
            fails.append(f"permutation case {n}: counts differ from bincount")
        if not np.array_equal(p.offsets, np.concatenate([[0], np.cumsum(counts)])):
            fails.append(f"permutation case {n}: offsets differ from cumsum")
        if not np.array_equal(p.gather[p.scatter], np.arange(flat.size)):
            fails.append(f"permutation case {n}: scatter is not the inverse of gather")
        if not np.array_equal(p.gate, w.reshape(-1)[order]):
            fails.append(f"permutation case {n}: gate is not the sorted weights")
    # ids outside [0, E) are skipped: the valid pairs keep their stable order
    ids = rng.integers(-3, 12, size=(40, 3)).astype(np.int32)
    p = oracle.expert_permutation(ids, 10, lib=lib)
    flat = ids.reshape(-1)
    ok = (flat >= 0) & (flat < 10)
    order = np.nonzero(ok)[0][np.argsort(flat[ok], kind="stable")]
    if not np.array_equal(p.gather[: ok.sum()], order) or p.offsets[-1] != ok.sum():
        fails.append("permutation with invalid ids: valid pairs misplaced")
    if not np.all(p.scatter[~ok] == -1) or not np.array_equal(p.scatter[order], np.arange(ok.sum())):
        fails.append("permutation with invalid ids: scatter wrong")
    return fails


def check_postprocess(lib) -> list[str]:
    """Shared-expert slot and ascending-id order: hand cases and invariants."""
    doc = json.load(open(os.path.join(GOLDEN, "postprocess_small.json")))
    fails = []
    sh = doc["shared"]
    w, ids = oracle.fill_shared_slot(np.asarray(sh["weights"]), np.asarray(sh["ids"]), sh["num_experts"],
                                     sh["num_shared"], np.asarray(sh["pick"]), sh["routed_scaling_factor"], lib=lib)
    if ids.tolist() != sh["out_ids"] or not np.allclose(w, sh["out_weights"], rtol=0, atol=1e-15):
        fails.append(f"shared slot hand case: {ids.tolist()} {w.tolist()}")
    w, ids = oracle.fill_shared_slot(np.asarray(sh["weights"]), np.asarray(sh["ids"]), sh["num_experts"],
                                     sh["num_shared"], np.asarray(sh["pick"]), None, lib=lib)
    if ids.tolist() != sh["out_ids"] or w.tolist() != sh["out_weights_no_scale"]:
        fails.append("shared slot without a scaling factor changed the weight")
    so = doc["sort"]
    w, ids = oracle.sort_by_id(np.asarray(so["weights"]), np.asarray(so["ids"]), lib=lib)
    if ids.tolist() != so["out_ids"] or w.tolist() != so["out_weights"]:
        fails.append(f"ascending-id hand case: {ids.tolist()} {w.tolist()}")
    # invariants on random rows: a stable sort by id is numpy's stable argsort
    rng = np.random.default_rng(17)
    ids0 = rng.integers(0, 6, size=(64, 7)).astype(np.int32)
    w0 = rng.random((64, 7))
    w, ids = oracle.sort_by_id(w0, ids0, lib=lib)
    order = np.argsort(ids0, axis=1, kind="stable")
    if not np.array_equal(ids, np.take_along_axis(ids0, order, 1)) or \
            not np.array_equal(w, np.take_along_axis(w0, order, 1)):
        fails.append("ascending-id order differs from a stable argsort")
    return fails


def check_softcap(lib) -> list[str]:
    """c * tanh(x / c) at points where tanh has a closed form: x = (c / 2) ln a
    gives c (a - 1) / (a + 1).  Also saturation and the c = 0 identity."""
    fails = []
    for c in (0.5, 1.0, 4.0, 30.0):
        a = np.array([1.0 / 1024, 0.25, 1.0 / 3, 1.0, 1.5, 3.0, 7.0, 1e6])
        x = (c / 2.0) * np.log(a)
        want = c * (a - 1.0) / (a + 1.0)
        got = oracle.softcap_logits(x, c, lib=lib)
        if not np.allclose(got, want, rtol=1e-14, atol=1e-15 * c):
            fails.append(f"softcap c={c}: {got.tolist()} != {want.tolist()}")
        big = oracle.softcap_logits(np.array([60.0 * c, -60.0 * c]), c, lib=lib)
        if not np.allclose(big, [c, -c], rtol=1e-15, atol=0):
            fails.append(f"softcap c={c} does not saturate at +-c: {big.tolist()}")
    x = np.random.default_rng(3).standard_normal(50) * 20
    if not np.array_equal(oracle.softcap_logits(x, 0.0, lib=lib), x):
        fails.append("softcap with c = 0 changed the logits")
    if not np.array_equal(oracle.softcap_logits(x, -4.0, lib=lib), oracle.softcap_logits(x, 4.0, lib=lib)):
        fails.append("softcap with -c differs from c")
    return fails


def check_fused_top1(lib) -> list[str]:
    """Hand cases (tests/golden/fused_top1_small.json) and random rows."""
    doc = json.load(open(os.path.join(GOLDEN, "fused_top1_small.json")))
    fails = []
    for case in doc["cases"]:
        if "hidden" in case:
            h = np.asarray(case["hidden"], np.float64)
        else:
            h = 2.0 * np.log(np.asarray(case["a"], np.float64))
        w = np.asarray(case["weight_ke"], np.float64)
        r, capped = oracle.fused_router_top1(h, w, case["softcap"], lib=lib)
        want_w = [1.0 / (1.0 + math.exp(-d)) for d in case["gap"]]
        if r.ids[:, 0].tolist() != case["ids"]:
            fails.append(f"fused top-1 {case['name']}: ids {r.ids[:, 0].tolist()} != {case['ids']}")
        if not np.allclose(r.weights[:, 0], want_w, rtol=0, atol=1e-12):
            fails.append(f"fused top-1 {case['name']}: weights {r.weights[:, 0].tolist()} != {want_w}")
        if "capped" in case and not np.allclose(capped, case["capped"], rtol=0, atol=1e-12):
            fails.append(f"fused top-1 {case['name']}: capped logits {capped.tolist()}")
    # random rows: arg-max (first of equals) and the page's invsumexp weight
    rng = np.random.default_rng(29)
    h = rng.standard_normal((40, 24))
    wt = rng.standard_normal((24, 8)) * 0.5
    for c in (0.0, 2.0, 30.0):
        r, capped = oracle.fused_router_top1(h, wt, c, lib=lib)
        l = h @ wt
        if not np.array_equal(r.ids[:, 0], np.argmax(l, axis=1)):
            fails.append(f"fused top-1 c={c}: arg-max differs from numpy's")
        inv = 1.0 / np.sum(np.exp(capped - capped.max(axis=1, keepdims=True)), axis=1)
        if not np.allclose(r.weights[:, 0], inv, rtol=1e-13, atol=0):
            fails.append(f"fused top-1 c={c}: weight is not 1 / sum exp(l - max l)")
        r_t, _ = oracle.fused_router_top1(h, np.ascontiguousarray(wt.T), c, weight_layout=1, lib=lib)
        if not np.array_equal(r_t.ids, r.ids) or not np.allclose(r_t.weights, r.weights, rtol=1e-14, atol=0):
            fails.append(f"fused top-1 c={c}: (E, K) weight layout differs from (K, E)")
    return fails


def check_philox(lib) -> list[str]:
    """The seeded shared-expert draw: Philox4x64-10 against numpy's
    implementation of the same generator (numpy advances its counter once
    before the first block, so numpy at counter c gives the block at c + 1),
    the pick mapping floor(u n / 2^64) against its closed form for n = 2^j
    (the top j bits of u), the counter carry past 2^64, and the range."""
    fails = []
    for c0, k0, k1 in [(0, 0, 0), (41, 123456789, 987654321), (2**40 + 3, 2**63 + 5, 17)]:
        got = oracle.philox4x64([c0 + 1, 0, 0, 0], [k0, k1], lib=lib)
        ref = np.random.Philox(counter=np.array([c0, 0, 0, 0], np.uint64),
                               key=np.array([k0, k1], np.uint64)).random_raw(4)
        if not np.array_equal(got, ref.astype(np.uint64)):
            fails.append(f"philox4x64 counter {c0 + 1} key ({k0}, {k1}) differs from numpy's Philox")
    # the draw is word 0 of the block at counter offset + i, key (seed, 0)
    seed, offset, M = 20250, 7, 64
    raw = np.array([oracle.philox4x64([offset + i, 0, 0, 0], [seed, 0], lib=lib)[0] for i in range(M)],
                   dtype=np.uint64)
    for j in (0, 1, 3, 5):
        pick = oracle.shared_pick_philox(M, 2 ** j, seed, offset, lib=lib)
        expect = (raw >> np.uint64(64 - j)).astype(np.int64) if j else np.zeros(M, np.int64)
        if not np.array_equal(pick.astype(np.int64), expect):
            fails.append(f"shared pick with n = 2^{j} is not the top {j} bits of the Philox word")
    # counter carry: offset + i passes 2^64 into word 1
    top = 2**64 - 2
    pick = oracle.shared_pick_philox(4, 2**5, seed, top, lib=lib)
    words = [oracle.philox4x64([(top + i) % 2**64, (top + i) >> 64, 0, 0], [seed, 0], lib=lib)[0] for i in range(4)]
    if pick.tolist() != [int(w) >> 59 for w in words]:
        fails.append("shared pick: the counter does not carry into its second word past 2^64")
    # range and a loose uniformity check for a non-power-of-two count
    pick = oracle.shared_pick_philox(30000, 3, 99, 0, lib=lib)
    counts = np.bincount(pick, minlength=3)
    if pick.min() < 0 or pick.max() > 2 or np.any(np.abs(counts - 10000) > 600):
        fails.append(f"shared pick over 3 values: counts {counts.tolist()}")
    return fails


ALL_CHECKS = (check_golden, check_router_golden, check_router_numpy, check_brute, check_library,
              check_permutation_golden, check_permutation_after_shared_slot, check_permutation_numpy,
              check_postprocess, check_philox, check_softcap,
              check_fused_top1)


def run_all(lib) -> list[str]:
    fails = []
    for chk in ALL_CHECKS:
        try:
            fails += chk(lib)
        except Exception as exc:
            fails.append(f"{chk.__name__} raised {exc!r}")
    return fails
