"""CUDA routing kernels against the CPU oracle (GPU only).

Every call goes through the C ABI (via the thin binding).  Covers the four
routing workloads at their quoted token counts (the full sizes, in the same
launch configuration the benchmark times), ragged and tiny batches, dtype
variants, every kernel family (segment / small-E / generic), massive ties,
saturated logits, out-of-bounds canaries and CUDA-graph replay.
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


def run_gpu(op, x, bias, k, renorm, G, TG, rsf):
    xd = x.to(DEV)
    if op == "softmax":
        if G == 1 and TG == 1 and rsf == 1.0:
            w, ids = moe.topk_softmax(xd, k, renorm)
        else:
            w, ids = moe.grouped_topk(xd, k, renorm, G, TG, rsf)
    else:
        bd = None if bias is None else bias.to(DEV)
        w, ids = moe.biased_grouped_topk(xd, bd, k, renorm, G, TG, rsf)
    torch.cuda.synchronize()
    return w.cpu().numpy(), ids.cpu().numpy()


def run_oracle(op, x, bias, k, renorm, G, TG, rsf):
    if op == "softmax":
        return oracle.grouped_topk(x, k, renorm, G, TG, rsf)
    return oracle.biased_grouped_topk(x, bias, k, renorm, G, TG, rsf)


def check(op, x, bias, k, renorm, G, TG, rsf):
    w, ids = run_gpu(op, x, bias, k, renorm, G, TG, rsf)
    orc = run_oracle(op, x, bias, k, renorm, G, TG, rsf)
    rep = parity.compare(w, ids, orc, E=x.shape[1], G=G, TG=TG, k=k, renorm=renorm, rsf=rsf,
                         fp32_logits=(x.dtype == torch.float32))
    assert rep.ok(), rep.summary()
    return rep


def _spec_args(name):
    sp = inputs.SPECS[name]
    op = "softmax" if name in ("softmax", "grouped") else "sigmoid"
    return op, sp.topk, sp.renormalize, sp.num_expert_group, sp.topk_group, sp.routed_scaling_factor


@pytest.mark.parametrize("name,M", [(n, m) for n in ("softmax", "sigmoid", "biased", "grouped")
                                    for m in inputs.SIZES[n]])
def test_workloads_full_size(name, M):
    d = inputs.make(name, M)
    op, k, renorm, G, TG, rsf = _spec_args(name)
    rep = check(op, d["logits"], d["bias"], k, renorm, G, TG, rsf)
    # near ties must stay rare on these draws
    assert rep.near_tie <= max(3, M // 200), rep.summary()


@pytest.mark.parametrize("name", ["softmax", "sigmoid", "biased", "grouped"])
@pytest.mark.parametrize("M", [1, 2, 3, 5, 17, 31, 33, 63, 129, 1000, 4099])
def test_ragged_batches(name, M):
    d = inputs.make(name, M, seed=77 + M)
    op, k, renorm, G, TG, rsf = _spec_args(name)
    check(op, d["logits"], d["bias"], k, renorm, G, TG, rsf)


@pytest.mark.parametrize("name", ["softmax", "sigmoid", "biased", "grouped"])
@pytest.mark.parametrize("M", [777, 2777])
def test_other_dtype(name, M):
    """bf16 for the fp32 workloads and fp32 for the bf16 ones (direct-load and
    TMA-staged paths)."""
    d = inputs.make(name, M, seed=5)
    x = d["logits"]
    x = x.to(torch.bfloat16) if x.dtype == torch.float32 else x.to(torch.float32)
    op, k, renorm, G, TG, rsf = _spec_args(name)
    check(op, x, d["bias"], k, renorm, G, TG, rsf)


# (op, E, G, TG, k, renorm, rsf, bias) across the kernel families (M = 531 takes the
# warp-per-row kernel for E = 160 and 256 with G dividing 32)
SHAPES = [
    ("sigmoid", 256, 8, 4, 8, True, 2.5, True),    # segment, DeepSeek-V3
    ("sigmoid", 256, 4, 2, 6, False, 1.0, True),   # segment, 2 lanes per group
    ("sigmoid", 256, 2, 1, 7, True, 1.0, True),    # segment, odd k
    ("sigmoid", 256, 1, 1, 1, True, 1.0, False),   # segment, no bias, k=1
    ("sigmoid", 256, 8, 8, 32, True, 1.0, True),   # segment, k=32, all groups kept
    ("softmax", 256, 8, 4, 8, True, 1.0, False),   # segment, softmax on 256
    ("softmax", 160, 8, 3, 6, True, 2.0, False),   # segment, renormalised
    ("softmax", 160, 1, 1, 4, False, 1.0, False),  # segment, E=160 ungrouped
    ("sigmoid", 160, 8, 2, 4, True, 1.0, True),    # segment, sigmoid on 160
    ("softmax", 8, 1, 1, 2, True, 1.0, False),     # small
    ("softmax", 16, 4, 2, 3, False, 1.0, False),   # small, grouped
    ("sigmoid", 32, 4, 2, 5, True, 1.5, True),     # small, biased
    ("sigmoid", 8, 2, 1, 4, True, 1.0, True),      # small, k = admissible
    ("softmax", 64, 8, 3, 5, True, 1.0, False),    # generic
    ("sigmoid", 128, 16, 4, 8, True, 2.5, True),   # generic
    ("sigmoid", 384, 8, 4, 8, True, 2.5, True),    # generic
    ("softmax", 1024, 32, 8, 16, False, 1.0, False),  # generic, large
    ("sigmoid", 256, 16, 4, 8, True, 2.5, True),   # generic (lanes would straddle groups)
    ("sigmoid", 72, 9, 3, 6, True, 1.0, True),     # generic, odd group count
    ("sigmoid", 256, 32, 8, 8, True, 2.5, True),   # one lane per group (warp-per-row kernel)
    ("softmax", 160, 16, 4, 6, True, 1.0, False),  # two lanes per group of 10
    ("sigmoid", 160, 32, 6, 8, False, 1.0, True),  # groups of 5 experts, one lane each
]


@pytest.mark.parametrize("op,E,G,TG,k,renorm,rsf,use_bias", SHAPES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("M", [531, 1500])
def test_kernel_families(op, E, G, TG, k, renorm, rsf, use_bias, dtype, M):
    x = inputs.random_logits(M, E, 2.0, dtype, seed=E * 31 + G * 7 + k)
    bias = inputs.random_bias(E, 0.05, seed=E + 1) if use_bias else None
    check(op, x, bias, k, renorm, G, TG, rsf)


@pytest.mark.parametrize("op,E,G,TG,k", [("sigmoid", 256, 8, 4, 8), ("sigmoid", 256, 1, 1, 8),
                                         ("softmax", 160, 8, 3, 6), ("softmax", 8, 1, 1, 2),
                                         ("sigmoid", 64, 4, 2, 4)])
def test_all_equal_logits_pick_lowest_indices(op, E, G, TG, k):
    """Massive ties (exact-fallback path): the lowest indices win, exactly."""
    x = torch.zeros(70, E, dtype=torch.bfloat16)
    w, ids = run_gpu(op, x, None, k, True, G, TG, 1.0)
    orc = run_oracle(op, x, None, k, True, G, TG, 1.0)
    assert np.array_equal(ids, orc.ids)
    assert np.allclose(w, 1.0 / k, rtol=1e-6)


def test_some_rows_tied_some_not():
    """A warp that mixes tied and clear rows takes the exact path for all."""
    d = inputs.make("biased", 64, seed=3)
    x = d["logits"].clone()
    x[5] = 0
    x[6, :64] = 1.0
    op, k, renorm, G, TG, rsf = _spec_args("biased")
    check(op, x, None, k, renorm, G, TG, rsf)


@pytest.mark.parametrize("scale", [20.0, 60.0, 120.0])
def test_saturated_logits(scale):
    """Large logits saturate the sigmoid; ties among saturated scores are
    near ties and must still be valid choices."""
    x = inputs.random_logits(300, 256, scale, torch.float32, seed=int(scale))
    bias = inputs.random_bias(256, 0.05, seed=9)
    check("sigmoid", x, bias, 8, True, 8, 4, 2.5)
    check("softmax", x, None, 8, True, 8, 4, 1.0)


def test_outputs_have_no_out_of_bounds_writes():
    M, k = 1000, 8
    d = inputs.make("biased", M)
    x = d["logits"].to(DEV)
    b = d["bias"].to(DEV)
    pad = 4096
    wbuf = torch.full((M * k + 2 * pad,), 12345.0, device=DEV)
    ibuf = torch.full((M * k + 2 * pad,), -777, dtype=torch.int32, device=DEV)
    w = wbuf[pad:pad + M * k].view(M, k)
    ids = ibuf[pad:pad + M * k].view(M, k)
    moe.biased_grouped_topk(x, b, k, True, 8, 4, 2.5, out=(w, ids))
    torch.cuda.synchronize()
    assert torch.all(wbuf[:pad] == 12345.0) and torch.all(wbuf[pad + M * k:] == 12345.0)
    assert torch.all(ibuf[:pad] == -777) and torch.all(ibuf[pad + M * k:] == -777)
    assert torch.all((ids >= 0) & (ids < 256))


@pytest.mark.parametrize("M", [1, 16, 64])
def test_cuda_graph_replay_matches_eager(M):
    d = inputs.make("sigmoid", M)
    x = d["logits"].to(DEV)
    b = d["bias"].to(DEV)
    w0, i0 = moe.biased_grouped_topk(x, b, 8, True, 1, 1)
    w = torch.empty_like(w0)
    ids = torch.empty_like(i0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        moe.biased_grouped_topk(x, b, 8, True, 1, 1, out=(w, ids))  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.biased_grouped_topk(x, b, 8, True, 1, 1, out=(w, ids))
    w.zero_()
    ids.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(ids, i0) and torch.equal(w, w0)


def test_invalid_arguments_raise_before_launch():
    x = torch.zeros(4, 256, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        moe.biased_grouped_topk(x, None, 8, True, 3, 1)      # 3 does not divide 256
    with pytest.raises(ValueError):
        moe.grouped_topk(x, 8, True, 8, 0)
    with pytest.raises(NotImplementedError):
        moe.topk_softmax(x, 33, True)


def test_empty_batch():
    x = torch.zeros(0, 256, dtype=torch.bfloat16, device=DEV)
    w, ids = moe.biased_grouped_topk(x, None, 8, True, 8, 4)
    assert w.shape == (0, 8) and ids.shape == (0, 8)


def test_no_watchdog_trips():
    """No kernel gave up on a barrier wait during the tests above."""
    torch.cuda.synchronize()
    assert moe.watchdog_trips() == 0


@pytest.mark.parametrize("M,E,G,TG,k", [(2048, 256, 1, 1, 8),    # streaming kernel (approximate keys)
                                        (2048, 256, 8, 4, 8),    # streaming kernel (exact keys)
                                        (2048, 256, 8, 8, 16),   # staged kernel (k > 8)
                                        (500, 256, 8, 4, 8),     # segment kernel
                                        (600, 32, 4, 2, 5),      # small-E kernel
                                        (700, 128, 16, 4, 8)])   # generic kernel
def test_aiter_bias_cast_variant(M, E, G, TG, k):
    """moe_biased_grouped_topk_aiter rounds the fp32 bias to the bf16 logits'
    dtype first: it must match the oracle on the rounded bias, and biases in
    [0.25, 0.5] (rounding error up to ~5e-4, above the key gaps near the top)
    make it differ from the fp32-bias call on clear rows."""
    g = torch.Generator().manual_seed(E * 13 + k)
    x = (torch.randn(M, E, generator=g) * 0.5).to(torch.bfloat16)
    bias = 0.25 + 0.25 * torch.rand(E, generator=g)
    xd, bd = x.to(DEV), bias.to(DEV)
    w, ids = moe.biased_grouped_topk(xd, bd, k, True, G, TG, 2.5, bias_as_logits_dtype=True)
    w2, ids2 = moe.biased_grouped_topk(xd, bd, k, True, G, TG, 2.5)
    torch.cuda.synchronize()
    b16 = bias.to(torch.bfloat16).to(torch.float32)
    orc = run_oracle("sigmoid", x, b16, k, True, G, TG, 2.5)
    rep = parity.compare(w.cpu().numpy(), ids.cpu().numpy(), orc, E=E, G=G, TG=TG, k=k, renorm=True, rsf=2.5,
                         fp32_logits=False)
    assert rep.ok(), rep.summary()
    assert not torch.equal(ids, ids2), "rounding the bias changed no routing decision"


def test_aiter_variant_is_the_plain_call_for_fp32_logits():
    d = inputs.make("grouped", 3000)
    x = d["logits"].to(DEV)
    bias = inputs.random_bias(160, 0.05, seed=3).to(DEV)
    a = moe.biased_grouped_topk(x, bias, 6, True, 8, 3, 1.0, bias_as_logits_dtype=True)
    b = moe.biased_grouped_topk(x, bias, 6, True, 8, 3, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[0], b[0])


@pytest.mark.parametrize("M,E,G,TG,k,renorm", [(2048, 256, 1, 1, 8, True),    # streaming kernel
                                               (2048, 160, 8, 3, 6, False),   # streaming, full denominators
                                               (2048, 256, 8, 8, 16, True),   # staged kernel (k > 8)
                                               (500, 256, 8, 4, 8, False),    # segment kernel
                                               (600, 8, 1, 1, 1, False),      # small-E: top-1 = 1 / sum exp
                                               (700, 64, 8, 3, 5, True)])     # generic kernel
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_softcapped_softmax(M, E, G, TG, k, renorm, dtype):
    """moe_grouped_topk_softcap: the oracle's softmax routing of the oracle's
    capped logits 30 * tanh(x / 30) (computed in double).  Weight tolerance for fp32
    logits: tanhf's ~2 ulp, times c, plus roundings, gives ~4e-7 * c on each
    capped logit and, through exp and the sum, below 1.4e-5 relative; 2e-5."""
    c = 30.0
    x = inputs.random_logits(M, E, 20.0, dtype, seed=E + k + M)
    w, ids = moe.grouped_topk(x.to(DEV), k, renorm, G, TG, 1.5, softcap=c)
    torch.cuda.synchronize()
    xc = oracle.softcap_logits(x, c)
    orc = oracle.grouped_topk(xc, k, renorm, G, TG, 1.5)
    rep = parity.compare(w.cpu().numpy(), ids.cpu().numpy(), orc, E=E, G=G, TG=TG, k=k, renorm=renorm, rsf=1.5,
                         fp32_logits=(dtype == torch.float32),
                         w_rtol=2e-5 if dtype == torch.float32 else None)
    assert rep.ok(), rep.summary()


@pytest.mark.parametrize("E,k", [(8, 2), (256, 8)])
def test_softcap_saturated_ties(E, k):
    """c = 1 and logits far into tanh's saturation: 20, 25 and 30 (and, at
    E = 256, a block of 24 logits in [20, 40]) all cap to exactly 1.  The kernels select
    on the raw logits, the oracle on the capped values with ties to the lower
    index; the rows must count as near ties and pass."""
    M = 64
    x = inputs.random_logits(M, E, 1.0, torch.float32, seed=E)
    x[:, 1] = 20.0
    x[:, 3] = 25.0
    x[:, 5] = 30.0  # k + 1 saturated values at E = 8: the k-th pick is tied
    if E == 256:
        x[:, 100:124] = torch.linspace(20.0, 40.0, 24)
    w, ids = moe.grouped_topk(x.to(DEV), k, True, 1, 1, 1.0, softcap=1.0)
    torch.cuda.synchronize()
    orc = oracle.grouped_topk(oracle.softcap_logits(x, 1.0), k, True, 1, 1, 1.0)
    rep = parity.compare(w.cpu().numpy(), ids.cpu().numpy(), orc, E=E, G=1, TG=1, k=k, renorm=True, rsf=1.0,
                         fp32_logits=True, w_rtol=2e-5)
    assert rep.ok(), rep.summary()
    assert rep.near_tie == M, rep.summary()


def test_softcap_zero_is_the_plain_call():
    x = inputs.random_logits(3000, 256, 3.0, torch.bfloat16, seed=8).to(DEV)
    a = moe.grouped_topk(x, 8, True, 8, 4, 1.0)
    b = torch.empty_like(a[0]), torch.empty_like(a[1])
    st = moe.lib().moe_grouped_topk_softcap(x.data_ptr(), 1, 3000, 256, 8, 1, 8, 4, 1.0, 0.0, b[0].data_ptr(),
                                            b[1].data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0 and torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
