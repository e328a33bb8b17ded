"""Fused router (router projection on tcgen05 + biased grouped top-k) against
the CPU oracle (GPU only).

Three checks per case:
* the fp32 logits the kernel routed (debug output) against the oracle's
  double-precision projection, within the fp32-accumulation bound below;
* the routing of those logits against the oracle fed the same logits
  (isolates the routing step: the usual bit-exact / near-tie rules);
* the routing against the oracle's own end-to-end result (double GEMM), with
  the near-tie margin widened by the logits error bound.
"""
import numpy as np
import pytest
import torch

import moe_expert_routing_token_b200 as moe
import oracle
from moe_expert_routing_token_b200 import inputs
from oracle import parity

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

# fp32 accumulation of K bf16 products: |error| <= c * u * sum_k |h_k w_k|
# with u = 2^-24; c = 64 leaves a wide margin over the sqrt(K)-scaled typical
# error while still catching any dropped or duplicated k-block (which would
# move a logit by ~sum_{64 k} |h w| >> this bound).
LOGIT_REL = 64 * 2.0 ** -24


def _draw(M, K, E=256, seed=0):
    g = torch.Generator().manual_seed(seed)
    h = (torch.randn(M, K, generator=g) * 1.0).to(torch.bfloat16)
    w = (torch.randn(K, E, generator=g) * 0.02).to(torch.bfloat16)
    b = torch.randn(E, generator=g) * 0.05
    return h, w, b


def _run(h, w_ke, bias, layout, k=8, renorm=True, G=8, TG=4, rsf=2.5):
    hd = h.to(DEV)
    wd = (w_ke if layout == "ke" else w_ke.t().contiguous()).to(DEV)
    bd = None if bias is None else bias.to(DEV)
    out = moe.fused_router_topk(hd, wd, bd, k, renorm, G, TG, rsf, weight_layout=layout,
                                return_logits=True)
    torch.cuda.synchronize()
    return [t.cpu() for t in out]


def _check(h, w_ke, bias, layout, rows=None, **kw):
    k, renorm, G, TG, rsf = (kw.get("k", 8), kw.get("renorm", True), kw.get("G", 8),
                             kw.get("TG", 4), kw.get("rsf", 2.5))
    w_gpu, ids_gpu, logits_gpu = _run(h, w_ke, bias, layout, k, renorm, G, TG, rsf)
    sel = slice(None) if rows is None else rows
    hs = h[sel]
    ref = oracle.router_logits(hs, w_ke, weight_layout=0)
    absum = np.abs(oracle.as_f64(hs)) @ np.abs(oracle.as_f64(w_ke))
    err = np.abs(logits_gpu[sel].double().numpy() - ref)
    assert np.all(err <= LOGIT_REL * absum + 1e-30), f"logits max err {err.max():.3g}"
    # routing step alone: oracle on the GPU's logits
    orc_same = oracle.biased_grouped_topk(logits_gpu[sel].double().numpy(), bias, k, renorm, G, TG, rsf)
    rep = parity.compare(w_gpu[sel].numpy(), ids_gpu[sel].numpy(), orc_same, E=256, G=G, TG=TG, k=k,
                         renorm=renorm, rsf=rsf, fp32_logits=False)
    assert rep.ok(), "routing of kernel logits: " + rep.summary()
    # end to end against the double-precision projection; a logit error e moves
    # a sigmoid score by <= e/4, so widen the near-tie margin accordingly
    orc = oracle.biased_grouped_topk(ref, bias, k, renorm, G, TG, rsf)
    eps = parity.EPS + 2 * 0.25 * float(err.max())
    rep2 = parity.compare(w_gpu[sel].numpy(), ids_gpu[sel].numpy(), orc, E=256, G=G, TG=TG, k=k,
                          renorm=renorm, rsf=rsf, fp32_logits=False, eps=eps)
    assert rep2.ok(), "end to end: " + rep2.summary()
    return rep2


@pytest.mark.parametrize("layout", ["ke", "ek"])
def test_small_tile(layout):
    h, w, b = _draw(128, 128, seed=1)
    _check(h, w, b, layout)


@pytest.mark.parametrize("layout", ["ke", "ek"])
@pytest.mark.parametrize("M,K", [(256, 7168), (64, 7168), (1, 7168), (300, 1024), (129, 576),
                                 (200, 64), (1000, 2048)])
def test_shapes(layout, M, K):
    h, w, b = _draw(M, K, seed=M + K)
    _check(h, w, b, layout)


@pytest.mark.parametrize("use_bias", [True, False])
@pytest.mark.parametrize("G,TG,k,renorm,rsf", [(8, 4, 8, True, 2.5), (1, 1, 8, True, 1.0),
                                               (4, 2, 6, False, 1.0), (8, 8, 16, True, 1.0)])
def test_routing_variants(use_bias, G, TG, k, renorm, rsf):
    h, w, b = _draw(192, 1024, seed=7)
    _check(h, w, b if use_bias else None, "ke", k=k, renorm=renorm, G=G, TG=TG, rsf=rsf)


@pytest.mark.parametrize("M", [8192, 64])
def test_workload_full_size(M):
    """The fused workload at its quoted sizes, in the launch configuration
    the benchmark uses; the double-precision oracle checks sampled rows."""
    d = inputs.make("fused", M)
    sp = d["spec"]
    rng = np.random.default_rng(M)
    rows = np.sort(rng.choice(M, size=min(M, 192), replace=False))
    rep = _check(d["hidden"], d["weight"], d["bias"], "ke", rows=rows, k=sp.topk,
                 renorm=sp.renormalize, G=sp.num_expert_group, TG=sp.topk_group,
                 rsf=sp.routed_scaling_factor)
    assert rep.near_tie <= max(3, len(rows) // 50), rep.summary()
    # the routing step on every row: the oracle fed the kernel's own logits
    w_gpu, ids_gpu, logits_gpu = _run(d["hidden"], d["weight"], d["bias"], "ke", sp.topk, sp.renormalize,
                                      sp.num_expert_group, sp.topk_group, sp.routed_scaling_factor)
    orc = oracle.biased_grouped_topk(logits_gpu.double().numpy(), d["bias"], sp.topk, sp.renormalize,
                                     sp.num_expert_group, sp.topk_group, sp.routed_scaling_factor)
    rep_all = parity.compare(w_gpu.numpy(), ids_gpu.numpy(), orc, E=256, G=sp.num_expert_group,
                             TG=sp.topk_group, k=sp.topk, renorm=sp.renormalize, rsf=sp.routed_scaling_factor,
                             fp32_logits=False)
    assert rep_all.ok() and rep_all.rows == M, "routing of kernel logits, all rows: " + rep_all.summary()


def test_without_logits_output_matches():
    h, w, b = _draw(512, 2048, seed=3)
    hd, wd, bd = h.to(DEV), w.to(DEV), b.to(DEV)
    w1, i1, _ = moe.fused_router_topk(hd, wd, bd, 8, True, 8, 4, 2.5, return_logits=True)
    w2, i2 = moe.fused_router_topk(hd, wd, bd, 8, True, 8, 4, 2.5)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2) and torch.equal(w1, w2)


def test_deterministic_across_calls():
    h, w, b = _draw(1024, 4096, seed=4)
    hd, wd, bd = h.to(DEV), w.to(DEV), b.to(DEV)
    a = moe.fused_router_topk(hd, wd, bd, 8, True, 8, 4, 2.5, return_logits=True)
    c = moe.fused_router_topk(hd, wd, bd, 8, True, 8, 4, 2.5, return_logits=True)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, c))


@pytest.mark.parametrize("M", [1, 7, 64, 128])
def test_decode_path_reuses_its_workspace(M):
    """Single-tile batches spread K over CTAs whose partial logits meet in
    the workspace: any initial contents, and back-to-back calls on one
    workspace give identical results (the partials are added in a fixed
    order)."""
    K = 7168
    need = moe.fused_router_workspace_size(M, K, 256)
    assert 0 < need <= (2 << 20) and need % (M * 256 * 4) == 0
    h, w, b = _draw(M, K, seed=11 + M)
    hd, wd, bd = h.to(DEV), w.to(DEV), b.to(DEV)
    ws = torch.full((need,), 0x7F, dtype=torch.uint8, device=DEV)   # no initial contents needed
    outs = [moe.fused_router_topk(hd, wd, bd, 8, True, 8, 4, 2.5, return_logits=True, workspace=ws)
            for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert all(torch.equal(x, y) for x, y in zip(outs[0], o))
    _check(h, w, b, "ke")


@pytest.mark.parametrize("M,K,layout,G,TG", [(64, 1024, "ek", 8, 4),    # 16 k-blocks: the smallest K on this path
                                              (33, 4160, "ke", 4, 2),    # 65 k-blocks, ragged split
                                              (128, 16384, "ek", 1, 1),  # partials capped at 2 MiB
                                              (2, 7168, "ke", 8, 8)])    # every group kept
def test_decode_path_shapes(M, K, layout, G, TG):
    h, w, b = _draw(M, K, seed=M + K)
    assert moe.fused_router_workspace_size(M, K, 256) > 0
    _check(h, w, b, layout, G=G, TG=TG)


def test_wide_split_needs_workspace():
    h = torch.zeros(64, 7168, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(7168, 256, dtype=torch.bfloat16, device=DEV)
    weights = torch.empty(64, 8, device=DEV)
    ids = torch.empty(64, 8, dtype=torch.int32, device=DEV)
    L = moe.lib()
    st = L.moe_fused_router_topk(h.data_ptr(), w.data_ptr(), 0, None, 64, 7168, 256, 8, 1, 8, 4, 2.5,
                                 weights.data_ptr(), ids.data_ptr(), None, None, 0,
                                 torch.cuda.current_stream().cuda_stream)
    assert st == 1 and b"workspace" in L.moe_last_error()


def test_invalid_arguments():
    h = torch.zeros(4, 100, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(100, 256, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(NotImplementedError):     # K not a multiple of 64
        moe.fused_router_topk(h, w, None, 8, True, 8, 4)
    h = torch.zeros(4, 128, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(128, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(NotImplementedError):     # E != 256
        moe.fused_router_topk(h, w, None, 8, True, 8, 4)
    w = torch.zeros(128, 256, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):              # topk_group > groups
        moe.fused_router_topk(h, w, None, 8, True, 8, 9)


def test_no_watchdog_trips_fused():
    torch.cuda.synchronize()
    assert moe.watchdog_trips() == 0
