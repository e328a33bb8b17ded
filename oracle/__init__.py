"""CPU oracle for MoE token-to-expert routing (test infrastructure only).

This package is the slow, plain reference that the CUDA library is checked
against.  Only the tests, the smoke check and the CPU-baseline leg of the
benchmark may import it; the product package never does.  It shares no code
with the CUDA path: the arithmetic lives in ``moe_routing_oracle.c`` (plain C,
double precision, one row at a time) and this module only compiles it with
gcc and marshals numpy arrays into it.

Operations (each a restatement of the SGLang MoE routing page,
"[SGLang] MoE 라우팅: 토큰에서 전문가로의 배분 알고리즘"):

* :func:`topk_softmax`        - §2 softmax top-k (optional renormalise)
* :func:`grouped_topk`        - §3 grouped top-k, group score = max
* :func:`biased_grouped_topk` - §4 sigmoid + correction_bias, group score =
  sum of the top-2 biased scores; with num_expert_group = topk_group = 1 it is
  the sigmoid top-k of the aiter page ("SGLang MoE 라우팅 최적화: AMD GPU에서
  aiter.biased_grouped_topk 활용", 코드 분석)
* :func:`router_logits`       - §5 router projection, exact products summed
  in double
* :func:`fused_router_topk`   - §5 projection followed by §4 routing
* :func:`softcap_logits`      - §5 softcapping, c * tanh(logits / c)
* :func:`fused_router_top1`   - §5 projection, softcapping and softmax top-1
  (weight = 1 / sum_e exp(l_e - max l), the page's invsumexp)
* :func:`philox4x64`, :func:`shared_pick_philox` - the §6 shared-expert draw
  from a seed (Philox4x64-10 of Salmon et al., SC'11)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_routing_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

SOFTMAX, SIGMOID = 0, 1
GROUP_MAX, GROUP_TOP2_SUM = 0, 1

_DBL = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_U64 = ctypes.POINTER(ctypes.c_uint64)


def compile_oracle(src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the C oracle into a shared library with gcc (IEEE double, no
    fast-math, no FMA contraction).  Returns the library path."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _bind(path: str):
    lib = ctypes.CDLL(path)
    lib.oracle_route.restype = ctypes.c_int
    lib.oracle_route.argtypes = [
        _DBL, ctypes.c_int64, ctypes.c_int, ctypes.c_int, _DBL, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
        _I32, _DBL, _DBL, _DBL, _DBL, _DBL]
    lib.oracle_router_logits.restype = ctypes.c_int
    lib.oracle_router_logits.argtypes = [
        _DBL, _DBL, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, _DBL]
    lib.oracle_softcap.restype = ctypes.c_int
    lib.oracle_softcap.argtypes = [_DBL, ctypes.c_int64, ctypes.c_double, _DBL]
    lib.oracle_fill_shared_slot.restype = ctypes.c_int
    lib.oracle_fill_shared_slot.argtypes = [_DBL, _I32, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            _I32, ctypes.c_double]
    lib.oracle_philox4x64.restype = None
    lib.oracle_philox4x64.argtypes = [_U64, _U64, _U64]
    lib.oracle_shared_pick_philox.restype = ctypes.c_int
    lib.oracle_shared_pick_philox.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64, _I32]
    lib.oracle_sort_by_id.restype = ctypes.c_int
    lib.oracle_sort_by_id.argtypes = [_DBL, _I32, ctypes.c_int64, ctypes.c_int]
    lib.oracle_expert_permutation.restype = ctypes.c_int
    lib.oracle_expert_permutation.argtypes = [
        _I32, _DBL, ctypes.c_int64, ctypes.c_int, ctypes.c_int, _I32, _I32, _I32, _I32, _DBL]
    return lib


def load(path: str | None = None):
    """Load (compiling first if needed) the oracle library."""
    global _lib
    if path is not None:
        return _bind(path)
    with _lock:
        if _lib is None:
            if (not os.path.exists(_LIB_PATH)
                    or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
                compile_oracle()
            _lib = _bind(_LIB_PATH)
    return _lib


def as_f64(a) -> np.ndarray:
    """Exact conversion of stored input values (numpy, or a CPU torch tensor of
    any float dtype including bfloat16) to a C-contiguous float64 array."""
    if hasattr(a, "detach"):
        import torch  # local: only needed when handed a tensor
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, ty):
    return None if a is None else a.ctypes.data_as(ty)


class Routing:
    """Result of one oracle call (all numpy)."""

    def __init__(self, ids, weights, scores, sel, gsc, margins):
        self.ids = ids          # (M, k) int32
        self.weights = weights  # (M, k) float64
        self.scores = scores    # (M, E) float64 unbiased scores
        self.sel = sel          # (M, E) float64 selection scores
        self.group_scores = gsc  # (M, G) float64
        self.margins = margins  # (M, 3) float64: expert, group, selected-gap


def route(logits, *, scoring: int, bias=None, num_expert_group: int = 1,
          topk_group: int = 1, group_kind: int = GROUP_MAX, topk: int,
          renormalize: bool, routed_scaling_factor: float = 1.0,
          lib=None) -> Routing:
    x = as_f64(logits)
    if x.ndim != 2:
        raise ValueError("logits must be 2-D (M, E)")
    M, E = x.shape
    b = None if bias is None else as_f64(bias).reshape(E)
    G = int(num_expert_group)
    ids = np.zeros((M, topk), dtype=np.int32)
    w = np.zeros((M, topk), dtype=np.float64)
    scores = np.zeros((M, E), dtype=np.float64)
    sel = np.zeros((M, E), dtype=np.float64)
    gsc = np.zeros((M, G), dtype=np.float64)
    mg = np.zeros((M, 3), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_route(_ptr(x, _DBL), M, E, scoring, _ptr(b, _DBL), G,
                          int(topk_group), group_kind, int(topk), int(bool(renormalize)),
                          float(routed_scaling_factor), _ptr(ids, _I32), _ptr(w, _DBL),
                          _ptr(scores, _DBL), _ptr(sel, _DBL), _ptr(gsc, _DBL), _ptr(mg, _DBL))
    if rc == 1:
        raise ValueError("oracle_route: invalid arguments")
    if rc != 0:
        raise MemoryError("oracle_route: out of memory")
    return Routing(ids, w, scores, sel, gsc, mg)


def topk_softmax(logits, topk: int, renormalize: bool, lib=None) -> Routing:
    return route(logits, scoring=SOFTMAX, topk=topk, renormalize=renormalize,
                 group_kind=GROUP_MAX, lib=lib)


def grouped_topk(logits, topk: int, renormalize: bool, num_expert_group: int,
                 topk_group: int, routed_scaling_factor: float = 1.0, lib=None) -> Routing:
    return route(logits, scoring=SOFTMAX, topk=topk, renormalize=renormalize,
                 num_expert_group=num_expert_group, topk_group=topk_group,
                 group_kind=GROUP_MAX, routed_scaling_factor=routed_scaling_factor,
                 lib=lib)


def biased_grouped_topk(logits, correction_bias, topk: int, renormalize: bool,
                        num_expert_group: int, topk_group: int,
                        routed_scaling_factor: float = 1.0, lib=None) -> Routing:
    return route(logits, scoring=SIGMOID, bias=correction_bias, topk=topk,
                 renormalize=renormalize, num_expert_group=num_expert_group,
                 topk_group=topk_group, group_kind=GROUP_TOP2_SUM,
                 routed_scaling_factor=routed_scaling_factor, lib=lib)


def router_logits(hidden_states, router_weight, *, weight_layout: int = 0,
                  lib=None) -> np.ndarray:
    """logits = hidden_states x W.  weight_layout 0: W is (K, E); 1: W is (E, K)."""
    h = as_f64(hidden_states)
    w = as_f64(router_weight)
    M, K = h.shape
    E = w.shape[1] if weight_layout == 0 else w.shape[0]
    if (weight_layout == 0 and w.shape[0] != K) or (weight_layout == 1 and w.shape[1] != K):
        raise ValueError("router_weight shape does not match hidden_states")
    out = np.zeros((M, E), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_router_logits(_ptr(h, _DBL), _ptr(w, _DBL), M, K, E, int(weight_layout),
                                  _ptr(out, _DBL))
    if rc != 0:
        raise ValueError("oracle_router_logits: invalid arguments")
    return out


def fused_router_topk(hidden_states, router_weight, correction_bias, topk: int,
                      renormalize: bool, num_expert_group: int, topk_group: int,
                      routed_scaling_factor: float = 1.0, weight_layout: int = 0,
                      lib=None):
    """Projection then biased grouped top-k.  Returns (Routing, logits)."""
    logits = router_logits(hidden_states, router_weight, weight_layout=weight_layout, lib=lib)
    r = biased_grouped_topk(logits, correction_bias, topk, renormalize, num_expert_group,
                            topk_group, routed_scaling_factor, lib=lib)
    return r, logits


def softcap_logits(logits, softcap: float, lib=None) -> np.ndarray:
    """c * tanh(logits / c) elementwise (oracle_softcap); c == 0 returns a copy."""
    x = as_f64(logits)
    out = np.empty_like(x)
    lib = lib or load()
    if lib.oracle_softcap(_ptr(x, _DBL), x.size, float(softcap), _ptr(out, _DBL)) != 0:
        raise ValueError("oracle_softcap: invalid arguments")
    return out


def fused_router_top1(hidden_states, router_weight, softcap: float = 0.0, weight_layout: int = 0,
                      lib=None):
    """The fused router's top-1 form: projection, softcapping (c == 0: none),
    then softmax top-1 without renormalisation, so the weight is the softmax
    probability of the arg-max, 1 / sum_e exp(l_e - max l).  Returns
    (Routing, capped logits)."""
    logits = router_logits(hidden_states, router_weight, weight_layout=weight_layout, lib=lib)
    capped = softcap_logits(logits, softcap, lib=lib)
    return topk_softmax(capped, 1, False, lib=lib), capped


class Permutation:
    """Expert-sorted token permutation (all numpy): counts (E,), offsets (E+1,),
    gather (M*k,), scatter (M*k,), gate (M*k,) float64 or None."""

    def __init__(self, counts, offsets, gather, scatter, gate):
        self.counts, self.offsets, self.gather, self.scatter, self.gate = counts, offsets, gather, scatter, gate


def expert_permutation(topk_ids, num_experts: int, topk_weights=None, lib=None) -> Permutation:
    """Stable counting sort of the (token, slot) pairs of topk_ids (M, k) by
    expert id (oracle_expert_permutation); pairs with an id outside [0, E) are
    skipped (scatter -1, gather holds offsets[E] entries)."""
    if hasattr(topk_ids, "detach"):
        topk_ids = topk_ids.detach().cpu().numpy()
    ids = np.ascontiguousarray(np.asarray(topk_ids, dtype=np.int32))
    if ids.ndim != 2:
        raise ValueError("topk_ids must be (M, k)")
    M, k = ids.shape
    n = M * k
    w = None if topk_weights is None else as_f64(topk_weights).reshape(-1)
    counts = np.zeros(num_experts, np.int32)
    offsets = np.zeros(num_experts + 1, np.int32)
    gather = np.zeros(n, np.int32)
    scatter = np.zeros(n, np.int32)
    gate = None if w is None else np.zeros(n, np.float64)
    lib = lib or load()
    rc = lib.oracle_expert_permutation(_ptr(ids, _I32), _ptr(w, _DBL), M, k, int(num_experts),
                                       _ptr(counts, _I32), _ptr(offsets, _I32), _ptr(gather, _I32),
                                       _ptr(scatter, _I32), _ptr(gate, _DBL))
    if rc != 0:
        raise ValueError("oracle_expert_permutation: invalid arguments")
    return Permutation(counts, offsets, gather, scatter, gate)


def philox4x64(counter, key, lib=None) -> np.ndarray:
    """Philox4x64-10 (oracle_philox4x64): four uint64 outputs of one block for
    a counter of four words and a key of two."""
    c = np.ascontiguousarray(np.asarray(counter, dtype=np.uint64))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint64))
    if c.shape != (4,) or k.shape != (2,):
        raise ValueError("counter has 4 words, key has 2")
    out = np.zeros(4, np.uint64)
    (lib or load()).oracle_philox4x64(_ptr(c, _U64), _ptr(k, _U64), _ptr(out, _U64))
    return out


def shared_pick_philox(M: int, num_shared: int, seed: int, offset: int = 0, lib=None) -> np.ndarray:
    """The seeded shared-expert draw (oracle_shared_pick_philox): int32 (M,)
    values in [0, num_shared)."""
    pick = np.zeros(max(0, int(M)), np.int32)
    rc = (lib or load()).oracle_shared_pick_philox(int(M), int(num_shared), int(seed) & (2**64 - 1),
                                                  int(offset) & (2**64 - 1), _ptr(pick, _I32))
    if rc != 0:
        raise ValueError("oracle_shared_pick_philox: invalid arguments")
    return pick


def fill_shared_slot(topk_weights, topk_ids, num_experts: int, num_shared: int, picks,
                     routed_scaling_factor=None, lib=None):
    """[R] §6 on a routing result: last slot -> shared expert E + pick, weight
    -> sum of the other weights / routed_scaling_factor (unchanged if None).
    Returns new (weights float64, ids int32) arrays."""
    w = as_f64(topk_weights).copy()
    ids = np.ascontiguousarray(np.asarray(topk_ids if not hasattr(topk_ids, "detach") else topk_ids.cpu().numpy(),
                                          dtype=np.int32)).copy()
    pk = np.ascontiguousarray(np.asarray(picks if not hasattr(picks, "detach") else picks.cpu().numpy(),
                                         dtype=np.int32))
    M, k = ids.shape
    rsf = 0.0 if routed_scaling_factor is None else float(routed_scaling_factor)
    lib = lib or load()
    rc = lib.oracle_fill_shared_slot(_ptr(w, _DBL), _ptr(ids, _I32), M, k, int(num_experts), int(num_shared),
                                     _ptr(pk, _I32), rsf)
    if rc != 0:
        raise ValueError("oracle_fill_shared_slot: invalid arguments")
    return w, ids


def sort_by_id(topk_weights, topk_ids, lib=None):
    """Each row's (weight, id) pairs in ascending id, stable.  Returns new arrays."""
    w = as_f64(topk_weights).copy()
    ids = np.ascontiguousarray(np.asarray(topk_ids if not hasattr(topk_ids, "detach") else topk_ids.cpu().numpy(),
                                          dtype=np.int32)).copy()
    M, k = ids.shape
    lib = lib or load()
    if lib.oracle_sort_by_id(_ptr(w, _DBL), _ptr(ids, _I32), M, k) != 0:
        raise ValueError("oracle_sort_by_id: invalid arguments")
    return w, ids
