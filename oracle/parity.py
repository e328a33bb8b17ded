"""Element-by-element comparison of the CUDA routing outputs with the oracle
(test infrastructure, like the rest of this package).

Rules (the tolerance and near-tie margin are the ones the routing spec fixes;
all margins are measured by the oracle in double precision):

* A row is *clear* when its expert margin s_(k) - s_(k+1) over the admissible
  experts and its group margin gs_(TG) - gs_(TG+1) both exceed ``eps`` (1e-5).
  Clear rows need ids bit-exact with the oracle, order included.  If two of
  the *selected* experts are themselves within ``eps`` of each other, the
  order inside that run is free but the id set must still match exactly.
* Other rows are *near-tie* rows: counted, and accepted when the ids are
  unique, every id lies in a group scoring >= gs_(TG) - eps, and the choice
  is a top-k within eps inside the groups kept:
  - group margin clear (the GPU keeps the oracle's groups): every chosen
    expert scores >= s_(k) - eps and every oracle pick the GPU left out
    scores <= s_(k) + eps;
  - group margin within eps (another set of groups is as valid): the GPU's
    groups plus the clearly kept ones (gs > gs_(TG) + eps) number at most
    TG, and no expert of those groups that the GPU left out scores more than
    eps above the GPU's weakest pick.
* Weights are compared per slot against the oracle's unbiased score of the
  expert the GPU chose, renormalised over the GPU's chosen set and scaled:
  |dw| <= 1e-6 for fp32 logits, |dw| <= 2e-3 |w| for bf16 logits (a 1e-30
  absolute floor covers sigmoid scores that underflow in fp32).
"""
from __future__ import annotations

import dataclasses

import numpy as np

EPS = 1e-5
ABS_TOL_F32 = 1e-6
REL_TOL_BF16 = 2e-3


@dataclasses.dataclass
class Report:
    rows: int = 0
    clear: int = 0
    near_tie: int = 0
    order_ties: int = 0
    max_weight_err: float = 0.0
    failures: list = dataclasses.field(default_factory=list)

    def ok(self) -> bool:
        return not self.failures

    def summary(self) -> str:
        head = (f"rows={self.rows} clear={self.clear} near_tie={self.near_tie} "
                f"order_ties={self.order_ties} max_weight_err={self.max_weight_err:.3g}")
        return head + ("" if self.ok() else "\n  " + "\n  ".join(self.failures[:12]))


def compare(w_gpu, ids_gpu, orc, *, E: int, G: int, TG: int, k: int, renorm: bool, rsf: float,
            fp32_logits: bool, rows=None, eps: float = EPS, w_rtol: float | None = None) -> Report:
    """Compare GPU outputs (numpy or CPU tensors) with an oracle Routing.

    ``rows``: optional index array - the GPU rows that the oracle rows
    correspond to (for sampled comparisons at full size)."""
    w_gpu = np.asarray(w_gpu, dtype=np.float64)
    ids_gpu = np.asarray(ids_gpu, dtype=np.int64)
    if rows is not None:
        w_gpu = w_gpu[rows]
        ids_gpu = ids_gpu[rows]
    M = orc.ids.shape[0]
    rep = Report(rows=M)
    if M == 0:
        return rep
    S = E // G
    ids_o = orc.ids.astype(np.int64)
    s = orc.sel
    p = orc.scores
    gs = orc.group_scores
    d_exp, d_grp, gap = orc.margins[:, 0], orc.margins[:, 1], orc.margins[:, 2]

    if ids_gpu.min() < 0 or ids_gpu.max() >= E:
        bad = np.argwhere((ids_gpu < 0) | (ids_gpu >= E))[0][0]
        rep.failures.append(f"row {bad}: id out of range {ids_gpu[bad].tolist()}")
        return rep

    clear = (d_exp > eps) & (d_grp > eps)
    rep.clear = int(clear.sum())
    rep.near_tie = M - rep.clear
    strict = clear & (gap > eps)
    rep.order_ties = int((clear & ~strict).sum())

    mism = np.nonzero(strict & np.any(ids_gpu != ids_o, axis=1))[0]
    for r in mism[:8]:
        rep.failures.append(f"row {r} (clear, margin {d_exp[r]:.3g}/{d_grp[r]:.3g}): "
                            f"gpu {ids_gpu[r].tolist()} != oracle {ids_o[r].tolist()}")
    if len(mism) > 8:
        rep.failures.append(f"... {len(mism)} clear rows differ in total")

    for r in np.nonzero(clear & ~strict)[0]:
        if sorted(ids_gpu[r].tolist()) != sorted(ids_o[r].tolist()):
            rep.failures.append(f"row {r} (order tie): id set {sorted(ids_gpu[r].tolist())} != "
                                f"{sorted(ids_o[r].tolist())}")
        elif any(s[r, ids_gpu[r, j]] < s[r, ids_gpu[r, j + 1]] - eps for j in range(k - 1)):
            rep.failures.append(f"row {r} (order tie): gpu order not descending")

    for r in np.nonzero(~clear)[0]:
        ids = ids_gpu[r]
        if len(set(ids.tolist())) != k:
            rep.failures.append(f"row {r} (near tie): duplicate ids {ids.tolist()}")
            continue
        gs_tg = np.sort(gs[r])[::-1][TG - 1]
        if np.any(gs[r, ids // S] < gs_tg - eps):
            rep.failures.append(f"row {r} (near tie): id in a dropped group {ids.tolist()}")
        if d_grp[r] > eps:
            s_k = s[r, ids_o[r, k - 1]]
            if np.any(s[r, ids] < s_k - eps):
                rep.failures.append(f"row {r} (near tie): chose an expert below s_(k) - eps")
            omitted = np.setdiff1d(ids_o[r], ids)
            if omitted.size and np.any(s[r, omitted] > s_k + eps):
                rep.failures.append(f"row {r} (near tie): left out an expert above s_(k) + eps")
        else:
            kept = set((ids // S).tolist()) | set(np.nonzero(gs[r] > gs_tg + eps)[0].tolist())
            if len(kept) > TG:
                rep.failures.append(f"row {r} (group near tie): {len(kept)} groups kept > {TG}")
            members = np.concatenate([np.arange(g * S, (g + 1) * S) for g in sorted(kept)])
            others = np.setdiff1d(members, ids)
            if others.size and np.any(s[r, others] > s[r, ids].min() + eps):
                rep.failures.append(f"row {r} (group near tie): left out a better expert of a kept group")

    # weights for the GPU's choice
    pw = np.take_along_axis(p, ids_gpu, axis=1)
    if renorm:
        pw = pw / pw.sum(axis=1, keepdims=True)
    expect = pw * rsf
    err = np.abs(w_gpu - expect)
    rep.max_weight_err = float(err.max())
    if w_rtol is not None:  # a tolerance the caller derives for its arithmetic
        bad = err > w_rtol * np.abs(expect) + 1e-30
    elif fp32_logits:
        bad = err > ABS_TOL_F32
    else:
        bad = err > REL_TOL_BF16 * np.abs(expect) + 1e-30
    for r in np.nonzero(bad.any(axis=1))[0][:6]:
        rep.failures.append(f"row {r}: weights {w_gpu[r].tolist()} vs {expect[r].tolist()}")
    # the oracle's own weights agree with the formula on rows where the sets match
    same = np.all(ids_gpu == ids_o, axis=1)
    if same.any() and not np.allclose(orc.weights[same], expect[same], rtol=1e-12, atol=1e-15):
        rep.failures.append("oracle weights disagree with the renormalise/scale formula")
    return rep
