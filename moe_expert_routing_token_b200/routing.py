"""Thin Python binding of libmoe_routing (argument marshalling only).

Every function here checks tensor placement, dtype and layout, allocates the
outputs the way SGLang's ``fused_topk`` does (``torch.empty`` of (M, k) fp32
weights and int32 ids), and calls the matching C entry point of
``include/moe_routing.h`` with raw device pointers and the current CUDA
stream.  All routing arithmetic runs in the library's CUDA kernels; there is
no CPU or PyTorch fallback - if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libmoe_routing.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA = 0, 1, 2, 3
MOE_DTYPE_F32, MOE_DTYPE_BF16 = 0, 1
MOE_WEIGHT_K_BY_E, MOE_WEIGHT_E_BY_K = 0, 1

_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_f32 = ctypes.c_float
_sz = ctypes.c_size_t

SIGNATURES = {
    "moe_abi_version": (ctypes.c_int, []),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_watchdog_trips": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint)]),
    "moe_topk_softmax": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_grouped_topk": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i32, _i32, _i32, _i32, _i32, _f32,
                                        _vp, _vp, _vp]),
    "moe_biased_grouped_topk": (ctypes.c_int, [_vp, ctypes.c_int, _vp, _i64, _i32, _i32, _i32, _i32,
                                               _i32, _f32, _vp, _vp, _vp]),
    "moe_biased_grouped_topk_aiter": (ctypes.c_int, [_vp, ctypes.c_int, _vp, _i64, _i32, _i32, _i32, _i32,
                                               _i32, _f32, _vp, _vp, _vp]),
    "moe_grouped_topk_softcap": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i32, _i32, _i32, _i32, _i32, _f32,
                                                _f32, _vp, _vp, _vp]),
    "moe_fused_router_workspace_size": (_sz, [_i64, _i32, _i32]),
    "moe_fused_router_topk": (ctypes.c_int, [_vp, _vp, ctypes.c_int, _vp, _i64, _i32, _i32, _i32, _i32,
                                             _i32, _i32, _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_fused_router_topk_noalloc": (ctypes.c_int, [_vp, _vp, ctypes.c_int, _vp, _i64, _i32, _i32, _i32,
                                                     _i32, _i32, _i32, _f32, _vp, _vp, _vp, _vp]),
    "moe_fused_router_top1": (ctypes.c_int, [_vp, _vp, ctypes.c_int, _i64, _i32, _i32, _f32, _vp, _vp, _vp,
                                             _vp]),
    "moe_expert_permutation_workspace_size": (_sz, [_i64, _i32, _i32]),
    "moe_fill_shared_expert_slot": (ctypes.c_int, [_vp, _vp, _i64, _i32, _i32, _i32, _vp, _f32, _vp]),
    "moe_fill_shared_expert_slot_philox": (ctypes.c_int, [_vp, _vp, _i64, _i32, _i32, _i32, ctypes.c_uint64,
                                                           ctypes.c_uint64, _f32, _vp]),
    "moe_sort_topk_by_id": (ctypes.c_int, [_vp, _vp, _i64, _i32, _vp]),
    "moe_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint64, _vp, _vp]),
    "moe_expert_permutation": (ctypes.c_int, [_vp, _vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                              _vp]),
}


class RoutingError(RuntimeError):
    """A CUDA-side failure reported by libmoe_routing."""


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libmoe_routing.so not found at {LIB_PATH}; build it with "
                    "`python -m moe_expert_routing_token_b200.build`")
            handle = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def _check(status: int, what: str) -> None:
    if status == MOE_OK:
        return
    msg = lib().moe_last_error().decode()
    if status == MOE_ERR_INVALID_ARG:
        raise ValueError(f"{what}: {msg}")
    if status == MOE_ERR_UNSUPPORTED:
        raise NotImplementedError(f"{what}: {msg}")
    raise RoutingError(f"{what}: {msg}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MOE_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return MOE_DTYPE_BF16
    raise ValueError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _cuda_2d(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 2 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 2-D tensor")


def _bias_ptr(bias, E: int, device) -> int | None:
    if bias is None:
        return None
    if not bias.is_cuda or bias.device != device or bias.dtype != torch.float32:
        raise ValueError("correction_bias must be a float32 CUDA tensor on the logits' device")
    if bias.numel() != E or not bias.is_contiguous():
        raise ValueError("correction_bias must be a contiguous (E,) tensor")
    return bias.data_ptr()


def _outputs(M: int, topk: int, device, out):
    if out is not None:
        w, ids = out
        if (w.shape != (M, topk) or w.dtype != torch.float32 or ids.shape != (M, topk)
                or ids.dtype != torch.int32 or not w.is_contiguous() or not ids.is_contiguous()
                or w.device != device or ids.device != device):
            raise ValueError("out must be ((M, topk) float32, (M, topk) int32) contiguous on the device")
        return w, ids
    return (torch.empty(M, topk, dtype=torch.float32, device=device),
            torch.empty(M, topk, dtype=torch.int32, device=device))


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _on(device):
    """Make the operands' device current for the call: the library sizes
    grids, sets kernel attributes and launches on the current device."""
    return torch.cuda.device(device)


def _same_device(device, **tensors) -> None:
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, not on {device} with the other operands")


def topk_softmax(gating_output: torch.Tensor, topk: int, renormalize: bool, out=None):
    """Softmax top-k of each row.  Returns (topk_weights fp32, topk_ids int32)."""
    _cuda_2d(gating_output, "gating_output")
    M, E = gating_output.shape
    w, ids = _outputs(M, topk, gating_output.device, out)
    with _on(gating_output.device):
        st = lib().moe_topk_softmax(gating_output.data_ptr(), _dtype_code(gating_output), M, E, topk,
                                    int(bool(renormalize)), w.data_ptr(), ids.data_ptr(),
                                    _stream(gating_output.device))
    _check(st, "moe_topk_softmax")
    return w, ids


def grouped_topk(gating_output: torch.Tensor, topk: int, renormalize: bool, num_expert_group: int,
                 topk_group: int, routed_scaling_factor: float = 1.0, out=None, softcap: float = 0.0):
    """Softmax grouped top-k (group score = max).  Returns (weights, ids).
    softcap != 0: weights from the softmax of softcap * tanh(logits / softcap)
    (moe_grouped_topk_softcap)."""
    _cuda_2d(gating_output, "gating_output")
    M, E = gating_output.shape
    w, ids = _outputs(M, topk, gating_output.device, out)
    if softcap:
        with _on(gating_output.device):
            st = lib().moe_grouped_topk_softcap(gating_output.data_ptr(), _dtype_code(gating_output), M, E,
                                                topk, int(bool(renormalize)), num_expert_group, topk_group,
                                                float(routed_scaling_factor), float(softcap), w.data_ptr(),
                                                ids.data_ptr(), _stream(gating_output.device))
        _check(st, "moe_grouped_topk_softcap")
        return w, ids
    with _on(gating_output.device):
        st = lib().moe_grouped_topk(gating_output.data_ptr(), _dtype_code(gating_output), M, E, topk,
                                    int(bool(renormalize)), num_expert_group, topk_group,
                                    float(routed_scaling_factor), w.data_ptr(), ids.data_ptr(),
                                    _stream(gating_output.device))
    _check(st, "moe_grouped_topk")
    return w, ids


def biased_grouped_topk(gating_output: torch.Tensor, correction_bias, topk: int,
                        renormalize: bool, num_expert_group: int = 1, topk_group: int = 1,
                        routed_scaling_factor: float = 1.0, out=None, bias_as_logits_dtype: bool = False):
    """Sigmoid + correction_bias grouped top-k (group score = sum of top-2).
    With num_expert_group = topk_group = 1 it is the sigmoid top-k.
    bias_as_logits_dtype: the aiter variant (moe_biased_grouped_topk_aiter),
    the bias rounded to bf16 logits' dtype before it is added."""
    _cuda_2d(gating_output, "gating_output")
    M, E = gating_output.shape
    bp = _bias_ptr(correction_bias, E, gating_output.device)
    w, ids = _outputs(M, topk, gating_output.device, out)
    fn = lib().moe_biased_grouped_topk_aiter if bias_as_logits_dtype else lib().moe_biased_grouped_topk
    with _on(gating_output.device):
        st = fn(gating_output.data_ptr(), _dtype_code(gating_output), bp, M, E,
                topk, int(bool(renormalize)), num_expert_group, topk_group,
                float(routed_scaling_factor), w.data_ptr(), ids.data_ptr(),
                _stream(gating_output.device))
    _check(st, "moe_biased_grouped_topk")
    return w, ids


def watchdog_trips() -> int:
    """Times a library kernel gave up on a barrier wait (0 in normal use)."""
    n = ctypes.c_uint(0)
    _check(lib().moe_watchdog_trips(ctypes.byref(n)), "moe_watchdog_trips")
    return n.value


def fused_router_workspace_size(M: int, K: int, E: int) -> int:
    n = lib().moe_fused_router_workspace_size(M, K, E)
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("moe_fused_router_workspace_size: invalid sizes")
    return n


def fused_router_topk(hidden_states: torch.Tensor, router_weight: torch.Tensor, correction_bias,
                      topk: int, renormalize: bool, num_expert_group: int, topk_group: int,
                      routed_scaling_factor: float = 1.0, weight_layout: str = "ke",
                      return_logits: bool = False, workspace: torch.Tensor | None = None, out=None):
    """Router projection on the tensor cores fused with biased grouped top-k.

    ``weight_layout`` "ke": router_weight is (K, E); "ek": (E, K).  Returns
    (weights, ids) or (weights, ids, logits fp32) with ``return_logits``.
    """
    _cuda_2d(hidden_states, "hidden_states")
    _cuda_2d(router_weight, "router_weight")
    if hidden_states.dtype != torch.bfloat16 or router_weight.dtype != torch.bfloat16:
        raise ValueError("hidden_states and router_weight must be bfloat16")
    M, K = hidden_states.shape
    if weight_layout == "ke":
        layout, (Kw, E) = MOE_WEIGHT_K_BY_E, router_weight.shape
    elif weight_layout == "ek":
        layout, (E, Kw) = MOE_WEIGHT_E_BY_K, router_weight.shape
    else:
        raise ValueError("weight_layout must be 'ke' or 'ek'")
    if Kw != K:
        raise ValueError("router_weight does not match hidden_states' hidden size")
    dev = hidden_states.device
    _same_device(dev, router_weight=router_weight, workspace=workspace)
    bp = _bias_ptr(correction_bias, E, dev)
    w, ids = _outputs(M, topk, dev, out)
    logits = torch.empty(M, E, dtype=torch.float32, device=dev) if return_logits else None
    need = fused_router_workspace_size(M, K, E)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        # the workspace must start zeroed; the library leaves it zeroed again
        workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    wsp = workspace.data_ptr() if (need and workspace is not None) else None
    with _on(dev):
        st = lib().moe_fused_router_topk(hidden_states.data_ptr(), router_weight.data_ptr(), layout, bp, M,
                                         K, E, topk, int(bool(renormalize)), num_expert_group, topk_group,
                                         float(routed_scaling_factor), w.data_ptr(), ids.data_ptr(),
                                         None if logits is None else logits.data_ptr(), wsp,
                                         need if wsp else 0, _stream(dev))
    _check(st, "moe_fused_router_topk")
    return (w, ids, logits) if return_logits else (w, ids)


def fused_router_top1(hidden_states: torch.Tensor, router_weight: torch.Tensor, softcap: float = 0.0,
                      weight_layout: str = "ek", return_logits: bool = False, out=None):
    """Router projection, softcapping and top-1 (moe_fused_router_top1): the
    tensor-core kernel for the "ek" layout with K % 64 == 0 and E <= 256,
    else the CUDA-core kernel (E <= 8).  ``weight_layout`` "ek":
    router_weight is (E, K); "ke": (K, E).  Returns (weights (M, 1) fp32,
    ids (M, 1) int32) or, with ``return_logits``, also the raw fp32 logits
    (M, E)."""
    _cuda_2d(hidden_states, "hidden_states")
    _cuda_2d(router_weight, "router_weight")
    if hidden_states.dtype != torch.bfloat16 or router_weight.dtype != torch.bfloat16:
        raise ValueError("hidden_states and router_weight must be bfloat16")
    M, K = hidden_states.shape
    if weight_layout == "ek":
        layout, (E, Kw) = MOE_WEIGHT_E_BY_K, router_weight.shape
    elif weight_layout == "ke":
        layout, (Kw, E) = MOE_WEIGHT_K_BY_E, router_weight.shape
    else:
        raise ValueError("weight_layout must be 'ek' or 'ke'")
    if Kw != K:
        raise ValueError("router_weight does not match hidden_states' hidden size")
    dev = hidden_states.device
    _same_device(dev, router_weight=router_weight)
    w, ids = _outputs(M, 1, dev, out)
    logits = torch.empty(M, E, dtype=torch.float32, device=dev) if return_logits else None
    with _on(dev):
        st = lib().moe_fused_router_top1(hidden_states.data_ptr(), router_weight.data_ptr(), layout, M, K, E,
                                         float(softcap), w.data_ptr(), ids.data_ptr(),
                                         None if logits is None else logits.data_ptr(), _stream(dev))
    _check(st, "moe_fused_router_top1")
    return (w, ids, logits) if return_logits else (w, ids)


def expert_permutation_workspace_size(M: int, k: int, E: int) -> int:
    n = lib().moe_expert_permutation_workspace_size(int(M), int(k), int(E))
    if n == ctypes.c_size_t(-1).value:
        raise ValueError(f"expert_permutation_workspace_size: bad sizes M={M} k={k} E={E}")
    return n


def expert_permutation(topk_ids: torch.Tensor, num_experts: int, topk_weights=None, workspace=None):
    """Expert-sorted permutation of a routing result (see
    moe_expert_permutation in include/moe_routing.h).  Returns
    (expert_counts, expert_offsets, gather_indx, scatter_indx, gate_scal);
    gate_scal is None when topk_weights is None."""
    _cuda_2d(topk_ids, "topk_ids")
    if topk_ids.dtype != torch.int32:
        raise ValueError("topk_ids must be int32")
    M, k = topk_ids.shape
    dev = topk_ids.device
    n = M * k
    if topk_weights is not None:
        _cuda_2d(topk_weights, "topk_weights")
        if topk_weights.dtype != torch.float32 or tuple(topk_weights.shape) != (M, k):
            raise ValueError("topk_weights must be fp32 with the shape of topk_ids")
    _same_device(dev, topk_weights=topk_weights, workspace=workspace)
    need = expert_permutation_workspace_size(M, k, num_experts)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    counts = torch.empty(num_experts, dtype=torch.int32, device=dev)
    offsets = torch.empty(num_experts + 1, dtype=torch.int32, device=dev)
    gather = torch.empty(n, dtype=torch.int32, device=dev)
    scatter = torch.empty(n, dtype=torch.int32, device=dev)
    gate = None if topk_weights is None else torch.empty(n, dtype=torch.float32, device=dev)
    with _on(dev):
        st = lib().moe_expert_permutation(
            topk_ids.data_ptr(), None if topk_weights is None else topk_weights.data_ptr(), M, k,
            int(num_experts), counts.data_ptr(), offsets.data_ptr(), gather.data_ptr(), scatter.data_ptr(),
            None if gate is None else gate.data_ptr(), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), _stream(dev))
    _check(st, "moe_expert_permutation")
    return counts, offsets, gather, scatter, gate


def _result_pair(topk_weights: torch.Tensor, topk_ids: torch.Tensor):
    _cuda_2d(topk_weights, "topk_weights")
    _cuda_2d(topk_ids, "topk_ids")
    if topk_weights.dtype != torch.float32 or topk_ids.dtype != torch.int32 or \
            topk_weights.shape != topk_ids.shape:
        raise ValueError("topk_weights must be fp32 and topk_ids int32 of the same (M, k) shape")
    _same_device(topk_ids.device, topk_weights=topk_weights)
    return topk_ids.shape


def fill_shared_expert_slot(topk_weights: torch.Tensor, topk_ids: torch.Tensor, num_experts: int,
                            num_shared: int, shared_pick: torch.Tensor, routed_scaling_factor=None):
    """In place: the last slot of each row -> shared expert num_experts +
    shared_pick[row]; its weight -> sum of the other weights /
    routed_scaling_factor (unchanged when it is None)."""
    M, k = _result_pair(topk_weights, topk_ids)
    if not shared_pick.is_cuda or shared_pick.dtype != torch.int32 or shared_pick.numel() != M or \
            not shared_pick.is_contiguous():
        raise ValueError("shared_pick must be a contiguous CUDA int32 tensor of M values")
    _same_device(topk_ids.device, shared_pick=shared_pick)
    rsf = 0.0 if routed_scaling_factor is None else float(routed_scaling_factor)
    if routed_scaling_factor is not None and rsf == 0.0:
        raise ValueError("routed_scaling_factor 0 is reserved for None")
    with _on(topk_ids.device):
        st = lib().moe_fill_shared_expert_slot(topk_weights.data_ptr(), topk_ids.data_ptr(), M, k,
                                               int(num_experts), int(num_shared), shared_pick.data_ptr(), rsf,
                                               _stream(topk_ids.device))
    _check(st, "moe_fill_shared_expert_slot")
    return topk_weights, topk_ids


def fill_shared_expert_slot_philox(topk_weights: torch.Tensor, topk_ids: torch.Tensor, num_experts: int,
                                   num_shared: int, seed: int, offset: int = 0, routed_scaling_factor=None):
    """As fill_shared_expert_slot, with the shared expert of row i drawn by
    the library: Philox4x64-10 at counter offset + i under key (seed, 0)."""
    M, k = _result_pair(topk_weights, topk_ids)
    rsf = 0.0 if routed_scaling_factor is None else float(routed_scaling_factor)
    if routed_scaling_factor is not None and rsf == 0.0:
        raise ValueError("routed_scaling_factor 0 is reserved for None")
    with _on(topk_ids.device):
        st = lib().moe_fill_shared_expert_slot_philox(topk_weights.data_ptr(), topk_ids.data_ptr(), M, k,
                                                      int(num_experts), int(num_shared), int(seed) & (2**64 - 1),
                                                      int(offset) & (2**64 - 1), rsf, _stream(topk_ids.device))
    _check(st, "moe_fill_shared_expert_slot_philox")
    return topk_weights, topk_ids


def sort_topk_by_id(topk_weights: torch.Tensor, topk_ids: torch.Tensor):
    """In place: each row's (weight, id) pairs in ascending id (stable)."""
    M, k = _result_pair(topk_weights, topk_ids)
    with _on(topk_ids.device):
        st = lib().moe_sort_topk_by_id(topk_weights.data_ptr(), topk_ids.data_ptr(), M, k,
                                       _stream(topk_ids.device))
    _check(st, "moe_sort_topk_by_id")
    return topk_weights, topk_ids
