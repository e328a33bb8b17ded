"""The two-phase routing kernel's key bounds, and parity where they matter (GPU only).

The streaming kernel for E = 160/256, k <= 8 selects candidates in phase 1
with keys that may differ from the exact phase-2 keys by at most eps, and
widens its threshold by 2 eps.  Two bounds feed eps:

* the hardware tanh (``tanh.approx.f32``) used for the approximate sigmoid
  key 0.5 tanh(x/2) + 0.5 + bias: its error must stay below the constant
  ``kTanhApproxErr`` in the kernel header.  Checked for every bf16 value and
  a dense fp32 sweep against tanh in double;
* the paired-reciprocal sigmoid of the exact phase 1 against the single
  sigmoid of phase 2: below ``kPairKeyErr``.

The parity tests then build rows whose exact keys sit 1e-5..5e-5 apart, far
closer than the approximate keys' error, so that only a correct band plus
the exact phase-2 ranking can return the oracle's experts.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

from moe_expert_routing_token_b200 import inputs
from tests.test_gpu_routing import check

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(HERE, "..", "moe_expert_routing_token_b200", "csrc", "routing_common.cuh")


def _header_constant(name):
    src = open(HEADER).read()
    m = re.search(rf"constexpr float {name} = 1\.0f / (\d+)\.0f;", src)
    assert m, f"{name} not found in the kernel header"
    return 1.0 / float(m.group(1))


@pytest.fixture(scope="module")
def bounds_lib(tmp_path_factory):
    out = tmp_path_factory.mktemp("score_bounds") / "libscore_bounds.so"
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-shared",
                    "-Xcompiler", "-fPIC", os.path.join(HERE, "cuda", "score_bounds.cu"), "-o", str(out)],
                   check=True)
    lib = ctypes.CDLL(str(out))
    lib.score_bounds.restype = ctypes.c_int
    lib.score_bounds.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    return lib


def _errors(lib, x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    et = np.zeros(x.size, np.float64)
    ep = np.zeros(x.size, np.float64)
    rc = lib.score_bounds(x.ctypes.data, x.size, et.ctypes.data, ep.ctypes.data)
    assert rc == 0
    return et, ep


def _all_bf16_values():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    x = bits.view(np.float32)
    return x[np.isfinite(x)]


def test_tanh_bound_every_bf16_input(bounds_lib):
    bound = _header_constant("kTanhApproxErr")
    et, _ = _errors(bounds_lib, _all_bf16_values())
    assert et.max() <= bound, f"tanh.approx error {et.max():.3e} above the kernel's bound {bound:.3e}"


def test_tanh_bound_fp32_sweep(bounds_lib):
    bound = _header_constant("kTanhApproxErr")
    rng = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-40.0, 40.0, 1 << 21, dtype=np.float32),
        rng.normal(0.0, 3.0, 1 << 21).astype(np.float32),
        (rng.standard_normal(1 << 20) * 10.0 ** rng.uniform(-8, 3, 1 << 20)).astype(np.float32),
        np.array([0.0, -0.0, 1e-38, -1e-38, 3e38, -3e38, np.inf, -np.inf], np.float32),
    ])
    et, _ = _errors(bounds_lib, x)
    assert et.max() <= bound, f"tanh.approx error {et.max():.3e} above the kernel's bound {bound:.3e}"


def test_pair_sigmoid_bound(bounds_lib):
    bound = _header_constant("kPairKeyErr")
    rng = np.random.default_rng(8)
    xb = _all_bf16_values()
    xb = xb[: xb.size - (xb.size % 2)]
    xf = rng.normal(0.0, 6.0, 1 << 21).astype(np.float32)
    for x in (xb, rng.permutation(xb), xf):
        _, ep = _errors(bounds_lib, x)
        assert ep.max() <= bound, f"pair/single sigmoid gap {ep.max():.3e} above {bound:.3e}"


def _close_key_rows(M, E, n_close, dtype, seed):
    """N(0, 2^2) logits with n_close experts per row drawn from [6.5, 8.5]:
    their sigmoids differ by 1e-5..5e-5 between neighbouring bf16 values,
    while the approximate keys err by up to ~2.5e-4."""
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(M, E, generator=gen) * 2.0
    idx = torch.stack([torch.randperm(E, generator=gen)[:n_close] for _ in range(M)])
    vals = 6.5 + 2.0 * torch.rand(M, n_close, generator=gen)
    x.scatter_(1, idx, vals)
    return x.to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("G,TG", [(1, 1), (8, 4), (8, 8)])
@pytest.mark.parametrize("bias_std", [0.0, 2e-5])
def test_close_keys_beyond_the_approximation(dtype, G, TG, bias_std):
    M, E, k = 2048, 256, 8   # the warp-per-row kernel (larger batches below)
    x = _close_key_rows(M, E, 24, dtype, seed=G * 10 + TG)
    bias = inputs.random_bias(E, bias_std, seed=5) if bias_std else torch.zeros(E)
    check("sigmoid", x, bias, k, True, G, TG, 2.5)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_close_keys_e160(dtype):
    M, E = 2048, 160
    x = _close_key_rows(M, E, 18, dtype, seed=31)
    bias = inputs.random_bias(E, 2e-5, seed=6)
    check("sigmoid", x, bias, 6, True, 8, 3, 1.0)
    check("sigmoid", x, bias, 6, False, 1, 1, 1.0)


def test_inputs_written_by_the_previous_kernel():
    """The streaming kernel starts while the previous kernel in the stream may
    still run (programmatic dependent launch) and must read its inputs only
    after that kernel has finished: rewrite the logits in place right before
    each call and compare with a fresh call on the final data."""
    import moe_expert_routing_token_b200 as moe
    M, E, k = 16384, 256, 8
    dev = "cuda:0"
    pool = [inputs.random_logits(M, E, 2.0, torch.bfloat16, seed=100 + i).to(dev) for i in range(4)]
    bias = inputs.random_bias(E, 0.05, seed=9).to(dev)
    x = torch.empty_like(pool[0])
    outs = []
    for rep in range(3):
        for i in range(4):
            x.copy_(pool[i])                     # a torch kernel writes the input ...
            w, ids = moe.biased_grouped_topk(x, bias, k, True, 1, 1, 1.0)  # ... read at once
            outs.append((i, w, ids))
    torch.cuda.synchronize()
    for i, w, ids in outs:
        w_ref, ids_ref = moe.biased_grouped_topk(pool[i].clone(), bias, k, True, 1, 1, 1.0)
        torch.cuda.synchronize()
        assert torch.equal(ids, ids_ref) and torch.equal(w, w_ref)


# The sizes and shapes that reach the two-phase streaming kernel: E = 256
# above 65536 rows, fp32 E = 160 above 16384 rows, bf16 E = 160 and E = 256
# with groups dropped out of 2 or 4 above 4096 rows.
STREAM_CASES = [
    ("sigmoid", 256, 1, 1, 8, True, 1.0, True, torch.bfloat16, 65603),
    ("sigmoid", 256, 8, 4, 8, True, 2.5, True, torch.bfloat16, 65603),
    ("softmax", 160, 8, 3, 6, False, 1.0, False, torch.float32, 16411),
    ("softmax", 160, 8, 3, 6, False, 1.0, False, torch.bfloat16, 5003),
    ("sigmoid", 256, 4, 2, 6, True, 1.0, True, torch.bfloat16, 5003),
    ("sigmoid", 256, 2, 1, 7, True, 1.0, True, torch.float32, 5003),
]


@pytest.mark.parametrize("op,E,G,TG,k,renorm,rsf,use_bias,dtype,M", STREAM_CASES)
def test_streaming_kernel_sizes(op, E, G, TG, k, renorm, rsf, use_bias, dtype, M):
    x = inputs.random_logits(M, E, 2.0, dtype, seed=M + E + G)
    bias = inputs.random_bias(E, 0.05, seed=E + G) if use_bias else None
    check(op, x, bias, k, renorm, G, TG, rsf)


@pytest.mark.parametrize("G,TG", [(1, 1), (8, 4)])
def test_close_keys_streaming_sizes(G, TG):
    """Rows of close keys (as above) in a batch the streaming kernel takes."""
    M, E, k = 65603, 256, 8
    x = _close_key_rows(M, E, 24, torch.bfloat16, seed=G * 10 + TG + 1)
    bias = inputs.random_bias(E, 2e-5, seed=5)
    check("sigmoid", x, bias, k, True, G, TG, 2.5)
