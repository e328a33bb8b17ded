"""The fused top-1 router (projection, softcapping, top-1 with the softmax
weight 1 / sum exp(cap(l) - cap(l_max))), on both its kernels (tensor cores
for (E, K) weights with K % 64 == 0, CUDA cores for the (K, E) layout or
other K, E <= 8) against the CPU oracle, through the C ABI (GPU only).

Three checks per case:
* the kernel's raw fp32 logits (debug output) against the oracle's double
  projection, within the fp32 summation bound below;
* the top-1 of those logits against the oracle fed the same logits (softcap
  and weight in double): clear rows need the same id, near-tie rows a valid
  one; weights within 2e-5 relative;
* against the oracle's end-to-end result (double projection), with the
  near-tie margin and the weight tolerance widened by the logits' error.
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

# Weight tolerance on the kernel's own logits: the capped logit carries
# tanhf's error (a few ulp of c), the exponent difference twice that, and the
# base-2 exponential, the E-term sum and the division add a few ulp each:
# below 1.4e-5 relative at c = 30.
W_RTOL = 2e-5


def _logit_rel(K: int) -> float:
    """fp32 summation bound for one logit, as a multiple of sum_k |h_k w_k|:
    each thread chains the FMAs of its ceil(K / 1024) chunks of 8 values,
    then 5 shuffle levels and 3 cross-warp additions (products of bf16 values
    are exact in fp32); 16 extra roundings of margin."""
    per_thread = -(-K // 1024) * 8
    return (per_thread + 5 + 3 + 16) * 2.0 ** -24


def _draw(M, K, E, seed):
    g = torch.Generator().manual_seed(seed)
    h = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w_ek = (torch.randn(E, K, generator=g) * 0.02).to(torch.bfloat16)
    return h, w_ek


def _run(h, w_ek, layout, c):
    wd = (w_ek if layout == "ek" else w_ek.t().contiguous()).to(DEV)
    w, ids, logits = moe.fused_router_top1(h.to(DEV), wd, c, weight_layout=layout, return_logits=True)
    torch.cuda.synchronize()
    return w.cpu(), ids.cpu(), logits.cpu()


# Tensor-core kernel: fp32 accumulation of K bf16 products in TMEM, then the
# split-K partials added in rank order: |error| <= c * u * sum_k |h_k w_k|
# with u = 2^-24; c = 64 is far above the typical sqrt(K)-scaled error and far
# below the effect of a dropped or repeated 64-wide k-block.
TC_LOGIT_REL = 64 * 2.0 ** -24


def _uses_tc(M, K, E, layout):
    """The library's dispatch: tensor cores for (E, K) weights, K % 64 == 0."""
    return K % 64 == 0 and layout == "ek" and E <= 256


def _check(h, w_ek, layout, c):
    M, K = h.shape
    E = w_ek.shape[0]
    w_gpu, ids_gpu, logits_gpu = _run(h, w_ek, layout, c)
    assert w_gpu.shape == (M, 1) and ids_gpu.shape == (M, 1)
    ref = oracle.router_logits(h, w_ek, weight_layout=1)
    absum = np.abs(oracle.as_f64(h)) @ np.abs(oracle.as_f64(w_ek)).T
    err = np.abs(logits_gpu.double().numpy() - ref)
    rel = TC_LOGIT_REL if _uses_tc(M, K, E, layout) else _logit_rel(K)
    assert np.all(err <= rel * absum + 1e-30), f"logits max err {err.max():.3g}"
    # the top-1 step alone: the oracle on the kernel's logits
    orc_same = oracle.topk_softmax(oracle.softcap_logits(logits_gpu, c), 1, False)
    rep = parity.compare(w_gpu.numpy(), ids_gpu.numpy(), orc_same, E=E, G=1, TG=1, k=1, renorm=False, rsf=1.0,
                         fp32_logits=True, w_rtol=W_RTOL)
    assert rep.ok(), "top-1 of kernel logits: " + rep.summary()
    # end to end: a logit error e moves each softmax probability by at most
    # e / 2 (the cap's slope is <= 1) and its logarithm by at most 2 e
    orc, _ = oracle.fused_router_top1(h, w_ek, c, weight_layout=1)
    e = float(err.max())
    rep2 = parity.compare(w_gpu.numpy(), ids_gpu.numpy(), orc, E=E, G=1, TG=1, k=1, renorm=False, rsf=1.0,
                          fp32_logits=True, eps=parity.EPS + 2 * e, w_rtol=W_RTOL + 4 * e)
    assert rep2.ok(), "end to end: " + rep2.summary()
    return rep2


@pytest.mark.parametrize("M,K,E,layout,c", [
    (1, 64, 8, "ek", 0.0),         # one row, 8 of 128 threads carry a chunk
    (7, 7168, 8, "ek", 30.0),      # a ragged 4-row tile
    (64, 4096, 8, "ke", 0.0),
    (511, 2048, 4, "ek", 30.0),    # below the page's 512-token switch
    (512, 2048, 2, "ke", 2.0),     # at it (here the same kernel)
    (3000, 7168, 8, "ek", 30.0),   # more tiles than resident blocks
    (2049, 1032, 3, "ke", 5.0),    # 129 chunks: one thread takes two
    (100, 512, 1, "ek", 0.0),      # one expert: id 0, weight 1
    (7, 7176, 8, "ek", 30.0),      # K % 64 != 0: the CUDA-core kernel on (E, K) weights
    (300, 1000, 5, "ek", 5.0),     # likewise, 125 chunks
])
def test_top1_router(M, K, E, layout, c):
    h, w = _draw(M, K, E, seed=M + K + E)
    _check(h, w, layout, c)


def test_bench_workload_full_size():
    """The configuration bench.py times: the seeded top1 workload, M = 8192,
    hidden 7168, the (E, K) weight, softcap 30; every row against the oracle."""
    d = inputs.make("top1", 8192)
    sp = d["spec"]
    rep = _check(d["hidden"], d["weight"], "ek", sp.softcap)
    assert rep.near_tie <= 8192 // 200, rep.summary()


@pytest.mark.parametrize("E", [5, 6, 7])
@pytest.mark.parametrize("layout", ["ek", "ke"])
def test_every_expert_count(E, layout):
    h, w = _draw(777, 2048, E, seed=E)
    _check(h, w, layout, 10.0)


def test_zero_rows_and_equal_logits():
    """A zero hidden row gives equal logits: expert 0, weight 1/E.  Two
    identical weight rows give two equal largest logits: the lower index."""
    M, K, E = 256, 1024, 8
    g = torch.Generator().manual_seed(4)
    h = torch.randn(M, K, generator=g).abs().to(torch.bfloat16)
    h[::3] = 0
    w = torch.zeros(E, K)
    v = torch.rand(K, generator=g) * 0.05
    w[2] = v
    w[5] = v
    w = w.to(torch.bfloat16)
    for layout in ("ek", "ke"):
        wt, ids, logits = _run(h, w, layout, 30.0)
        zero = np.arange(M) % 3 == 0
        assert np.all(ids.numpy()[zero, 0] == 0)
        assert np.allclose(wt.numpy()[zero, 0], 1.0 / E, rtol=1e-6, atol=0)
        # equal weight rows give equal logits (the tensor-core kernel is only
        # required to pick the lower index where they came out equal)
        same = (logits[:, 2] == logits[:, 5]).numpy()
        if not _uses_tc(M, K, E, layout):
            assert same.all()
        assert np.all(ids.numpy()[~zero & same, 0] == 2)
        assert np.all(np.isin(ids.numpy()[~zero, 0], [2, 5]))
        _check(h, w, layout, 30.0)


def test_saturated_softcap_ties():
    """With c = 1, logits 20 and 25 both cap to exactly 1 (tanh saturates in
    fp32 and in double), so the capped row has two equal largest values.  The
    kernel picks on the raw logits (expert 1), the oracle takes the lower
    index among equal capped values (expert 0): both are in the tie set, the
    row must count as a near tie and pass, and the weight, which depends only
    on the capped values, is the same for either choice."""
    M, K, E = 4, 8, 4
    h = torch.zeros(M, K)
    h[:, 0] = 1.0
    w = torch.zeros(E, K)
    w[0, 0], w[1, 0], w[2, 0], w[3, 0] = 20.0, 25.0, -3.0, 0.5  # exact in bf16
    h, w = h.to(torch.bfloat16), w.to(torch.bfloat16)
    for layout in ("ek", "ke"):
        rep = _check(h, w, layout, 1.0)
        assert rep.near_tie == M and rep.clear == 0, rep.summary()
        wt, ids, _ = _run(h, w, layout, 1.0)
        assert np.all(np.isin(ids.numpy()[:, 0], [0, 1]))
        expect = 1.0 / (2.0 + np.exp(np.tanh(-3.0) - 1.0) + np.exp(np.tanh(0.5) - 1.0))
        assert np.allclose(wt.numpy()[:, 0], expect, rtol=W_RTOL, atol=0)


def test_empty_batch():
    h = torch.empty(0, 512, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(8, 512, dtype=torch.bfloat16, device=DEV)
    wt, ids = moe.fused_router_top1(h, w, 30.0)
    assert wt.shape == (0, 1) and ids.shape == (0, 1)


def test_unsupported_shapes_raise():
    h = torch.zeros(4, 512, dtype=torch.bfloat16, device=DEV)
    # E > 8 needs the tensor-core kernel: (E, K) weights, K % 64 == 0, E <= 256
    with pytest.raises(NotImplementedError, match="tensor-core"):
        moe.fused_router_top1(h, torch.zeros(512, 16, dtype=torch.bfloat16, device=DEV), weight_layout="ke")
    with pytest.raises(NotImplementedError, match="tensor-core"):
        moe.fused_router_top1(h, torch.zeros(257, 512, dtype=torch.bfloat16, device=DEV))
    with pytest.raises(NotImplementedError, match="tensor-core"):
        moe.fused_router_top1(torch.zeros(4, 520, dtype=torch.bfloat16, device=DEV),
                              torch.zeros(16, 520, dtype=torch.bfloat16, device=DEV))
    with pytest.raises(NotImplementedError, match="multiple of 8"):
        moe.fused_router_top1(torch.zeros(4, 500, dtype=torch.bfloat16, device=DEV),
                              torch.zeros(8, 500, dtype=torch.bfloat16, device=DEV))


# ---------------------------------------------------------------- tensor-core kernel

@pytest.mark.parametrize("M,K,E,c", [
    (1, 64, 9, 0.0),          # one k-block, one row, no split
    (64, 7168, 16, 30.0),     # decode batch: split 16, 7 k-blocks each
    (64, 7168, 256, 30.0),    # E = 256, split 16
    (127, 1024, 17, 5.0),     # NP = 32 with E = 17: 15 zero-filled weight rows
    (129, 2048, 40, 0.0),     # two tiles, the second with one row
    (1000, 2112, 64, 30.0),   # split 8 over 33 k-blocks: the last CTA has none
    (1000, 832, 100, 2.0),    # 13 k-blocks, split 2 (7 + 6)
    (4096, 7168, 128, 30.0),  # split 4
    (5000, 1024, 160, 30.0),  # ragged last tile, split 2
    (20000, 512, 12, 30.0),   # 157 tiles: no split
    (512, 2048, 8, 30.0),     # E <= 8 at the page's batch-size switch
    (700, 256, 255, 0.0),     # NP = 256 with one zero-filled row, K = 4 k-blocks
])
def test_top1_tensor_core(M, K, E, c):
    assert _uses_tc(M, K, E, "ek")
    h, w = _draw(M, K, E, seed=3 * M + K + E)
    _check(h, w, "ek", c)


def test_top1_tensor_core_equal_experts():
    """Zero rows give E equal logits (expert 0, weight 1/E); two identical
    weight rows give equal largest logits, settled to the lower index."""
    M, K, E = 1500, 1024, 48
    g = torch.Generator().manual_seed(11)
    h = torch.randn(M, K, generator=g).abs().to(torch.bfloat16)
    h[::5] = 0
    w = torch.zeros(E, K)
    v = torch.rand(K, generator=g) * 0.05
    w[7] = v
    w[30] = v
    w = w.to(torch.bfloat16)
    wt, ids, logits = _run(h, w, "ek", 30.0)
    zero = np.arange(M) % 5 == 0
    assert np.all(ids.numpy()[zero, 0] == 0)
    assert np.allclose(wt.numpy()[zero, 0], 1.0 / E, rtol=W_RTOL, atol=0)
    same = (logits[:, 7] == logits[:, 30]).numpy() & ~zero
    assert np.all(ids.numpy()[same, 0] == 7)
    assert np.all(np.isin(ids.numpy()[~zero, 0], [7, 30]))
    _check(h, w, "ek", 30.0)


def test_top1_tensor_core_full_size_e256():
    """A (8192, 7168) batch against 256 experts: every row against the oracle."""
    h, w = _draw(8192, 7168, 256, seed=99)
    rep = _check(h, w, "ek", 30.0)
    assert rep.near_tie <= 8192 // 100, rep.summary()


def test_top1_tensor_core_no_watchdog_trips():
    import ctypes
    n = ctypes.c_uint(0)
    h, w = _draw(300, 1024, 32, seed=5)
    _run(h, w, "ek", 0.0)
    assert moe.lib().moe_watchdog_trips(ctypes.byref(n)) == 0
    assert n.value == 0
