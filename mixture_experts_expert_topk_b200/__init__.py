"""B200 (sm_100a) fused Mixture-of-Experts layer forward.

Thin Python binding over the C ABI of ``libmoe_b200.so`` (``include/moe_b200.h``).
Every step of the layer runs in the library's CUDA kernels; this module only
marshals torch tensors into pointers and sizes, allocates outputs and workspaces
with torch, and passes ``torch.cuda.current_stream()``.

    import mixture_experts_expert_topk_b200 as moe
    prob = moe.make_problem(T, H, E, topk, I, renormalize=True, activation="swiglu")
    w13p, w2p = moe.prepare_weights(prob, w13, w2, I_in)
    out = moe.moe_forward(hidden, router_logits, w13p, w2p, topk, True, "swiglu")
"""
from __future__ import annotations

import ctypes
from typing import Dict, Optional, Tuple

import torch

from . import _capi
from ._capi import (MOE_ACT_GELU_TANH, MOE_ACT_RELU2, MOE_ACT_SWIGLU, MOE_ACT_SWIGLUOAI, MOE_DTYPE_BF16, MOE_DTYPE_FP8_BLOCK128,
                    MOE_DTYPE_FP8_PER_TENSOR, MOE_DTYPE_MXFP8, MOE_DTYPE_NVFP4,
                    MOE_FLAG_PDL, MoeError, Problem, check, lib)

__all__ = [
    "MoeError", "Problem", "make_problem", "padded_intermediate", "workspace_layout",
    "workspace_size", "new_workspace", "prepare_weights", "quantize_weights_fp8",
    "quantize_weights_fp8_per_tensor", "quantize_weights_mxfp8", "quantize_weights_nvfp4", "moe_forward",
    "moe_forward_host", "stage_route", "stage_align", "stage_quant_act", "stage_gemm1",
    "stage_gemm2", "stage_combine", "device_status", "read_workspace", "lib", "check",
]

_ACT = {"swiglu": MOE_ACT_SWIGLU, "silu": MOE_ACT_SWIGLU, "relu2": MOE_ACT_RELU2,
        "gelu_tanh": MOE_ACT_GELU_TANH, "gelu": MOE_ACT_GELU_TANH,
        "swigluoai": MOE_ACT_SWIGLUOAI, "swigluoai_uninterleave": MOE_ACT_SWIGLUOAI,
        MOE_ACT_SWIGLU: MOE_ACT_SWIGLU, MOE_ACT_RELU2: MOE_ACT_RELU2, MOE_ACT_GELU_TANH: MOE_ACT_GELU_TANH,
        MOE_ACT_SWIGLUOAI: MOE_ACT_SWIGLUOAI}


def _act(a) -> int:
    if a not in _ACT:
        raise ValueError(f"unknown activation_type {a!r}")
    return _ACT[a]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def make_problem(T: int, H: int, num_routed: int, topk: int, intermediate: int, *,
                 renormalize: bool = True, activation="swiglu", num_shared: int = 0,
                 fp8=False, pdl: bool = True, block_m: int = 0, input_scale: float = 0.0,
                 activation_scale: float = 0.0) -> Problem:
    """Problem description; ``intermediate`` must already be padded. ``fp8``: False (bf16),
    True or "block128" (e4m3, 128x128 weight blocks, 1x128 activation groups), or
    "per_tensor" (e4m3, one scale per expert matrix and the static ``input_scale`` /
    ``activation_scale``), or "mxfp8" (e4m3 with an E8M0 scale per 32 values of K on both
    GEMM inputs), or "nvfp4" (E2M1 with an E4M3 scale per 16 values of K, tensor scales:
    per expert matrix for the weights, ``input_scale`` / ``activation_scale`` for the GEMM
    inputs)."""
    if fp8 == "per_tensor":
        wdtype = MOE_DTYPE_FP8_PER_TENSOR
    elif fp8 == "mxfp8":
        wdtype = MOE_DTYPE_MXFP8
    elif fp8 == "nvfp4":
        wdtype = MOE_DTYPE_NVFP4
    elif fp8 in (True, "block128"):
        wdtype = MOE_DTYPE_FP8_BLOCK128
    elif fp8 is False or fp8 is None:
        wdtype = MOE_DTYPE_BF16
    else:
        raise ValueError(f"fp8 must be False, True/'block128', 'per_tensor', 'mxfp8' or 'nvfp4', got {fp8!r}")
    return Problem(num_tokens=T, hidden=H, num_routed=num_routed, num_shared=num_shared,
                   intermediate=intermediate, topk=topk, renormalize=int(bool(renormalize)),
                   activation=_act(activation), wdtype=wdtype, block_m=block_m,
                   flags=MOE_FLAG_PDL if pdl else 0, input_scale=float(input_scale),
                   activation_scale=float(activation_scale))


def padded_intermediate(intermediate: int, activation="swiglu", fp8=False) -> int:
    wd = MOE_DTYPE_NVFP4 if fp8 == "nvfp4" else (MOE_DTYPE_FP8_BLOCK128 if fp8 else MOE_DTYPE_BF16)
    v = lib().moe_padded_intermediate(intermediate, _act(activation), wd)  # every 8-bit format pads to 128
    if v < 0:
        raise ValueError("invalid intermediate size or activation")
    return v


def workspace_layout(prob: Problem) -> Dict[str, int]:
    lay = _capi.Layout()
    check(lib().moe_workspace_layout(ctypes.byref(prob), ctypes.byref(lay)), "moe_workspace_layout")
    return {name: getattr(lay, name) for name, _ in _capi.Layout._fields_}


def workspace_size(prob: Problem) -> int:
    n = lib().moe_workspace_size(ctypes.byref(prob))
    if n == 0:
        check(lib().moe_check_problem(ctypes.byref(prob)), "moe_workspace_size")
    return n


def new_workspace(prob: Problem, device=None) -> torch.Tensor:
    """A uint8 CUDA tensor of moe_workspace_size bytes (256-byte aligned by torch)."""
    return torch.empty(workspace_size(prob), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


def prepare_weights(prob: Problem, w13: torch.Tensor, w2: torch.Tensor, intermediate_in: int,
                    stream=None, w13_scale: Optional[torch.Tensor] = None,
                    w2_scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Load-time padding + gate/up interleave (bf16, or e4m3 codes as uint8), in the layout
    the problem's GEMMs read: row-major [E, N1, H] / [E, H, I] for 128-row tiles, else the
    tiled layout (1-D tensors; ``.moe_intermediate`` records I for :func:`moe_forward`).
    MXFP8 problems also take the uint8 scale bytes ``w13_scale`` [E, N1, H/32] and
    ``w2_scale`` [E, H, I/32]; the prepared tensors then carry them (``.moe_mxfp8``)."""
    if prob.wdtype == MOE_DTYPE_MXFP8:
        return _prepare_weights_mxfp8(prob, w13, w2, w13_scale, w2_scale, stream)
    if prob.wdtype == MOE_DTYPE_NVFP4:
        return _prepare_weights_nvfp4(prob, w13, w2, w13_scale, w2_scale, stream)
    fp8 = prob.wdtype in (MOE_DTYPE_FP8_BLOCK128, MOE_DTYPE_FP8_PER_TENSOR)
    dt = torch.uint8 if fp8 else torch.bfloat16
    _dev(w13, "w13", dt)
    _dev(w2, "w2", dt)
    E = prob.num_routed + prob.num_shared
    I = prob.intermediate
    N1 = I if prob.activation == MOE_ACT_RELU2 else 2 * I
    elt = 1 if fp8 else 2
    n13 = lib().moe_prepared_weights_bytes(ctypes.byref(prob), 0)
    n2 = lib().moe_prepared_weights_bytes(ctypes.byref(prob), 1)
    if n13 == 0 or n2 == 0:
        check(lib().moe_check_problem(ctypes.byref(prob)), "moe_prepared_weights_bytes")
    if workspace_layout(prob)["block_m"] == 16:
        w13p = torch.empty(n13 // elt, dtype=dt, device=w13.device)
        w2p = torch.empty(n2 // elt, dtype=dt, device=w2.device)
    else:
        w13p = torch.empty((E, N1, prob.hidden), dtype=dt, device=w13.device)
        w2p = torch.empty((E, prob.hidden, I), dtype=dt, device=w2.device)
    check(lib().moe_prepare_weights(ctypes.byref(prob), intermediate_in, _ptr(w13), _ptr(w2),
                                    _ptr(w13p), _ptr(w2p), _stream(stream)), "moe_prepare_weights")
    w13p.moe_intermediate = I
    w2p.moe_intermediate = I
    return w13p, w2p


def _prepare_weights_mxfp8(prob, w13, w2, w13_scale, w2_scale, stream):
    for t, n in ((w13, "w13"), (w2, "w2"), (w13_scale, "w13_scale"), (w2_scale, "w2_scale")):
        if t is None:
            raise ValueError(f"MXFP8 preparation needs {n}")
        _dev(t, n, torch.uint8)
    n13 = lib().moe_prepared_weights_bytes(ctypes.byref(prob), 0)
    n2 = lib().moe_prepared_weights_bytes(ctypes.byref(prob), 1)
    if n13 == 0 or n2 == 0:
        check(lib().moe_check_problem(ctypes.byref(prob)), "moe_prepared_weights_bytes")
    w13p = torch.empty(n13, dtype=torch.uint8, device=w13.device)
    w2p = torch.empty(n2, dtype=torch.uint8, device=w2.device)
    check(lib().moe_prepare_weights_mxfp8(ctypes.byref(prob), _ptr(w13), _ptr(w13_scale), _ptr(w2),
                                          _ptr(w2_scale), _ptr(w13p), _ptr(w2p), _stream(stream)),
          "moe_prepare_weights_mxfp8")
    for t in (w13p, w2p):
        t.moe_intermediate = prob.intermediate
        t.moe_mxfp8 = True
    return w13p, w2p


def _prepare_weights_nvfp4(prob, w13, w2, w13_scale, w2_scale, stream):
    for t, n in ((w13, "w13"), (w2, "w2"), (w13_scale, "w13_scale"), (w2_scale, "w2_scale")):
        if t is None:
            raise ValueError(f"NVFP4 preparation needs {n} (packed codes and E4M3 block scales)")
        _dev(t, n, torch.uint8)
    n13 = lib().moe_prepared_weights_bytes(ctypes.byref(prob), 0)
    n2 = lib().moe_prepared_weights_bytes(ctypes.byref(prob), 1)
    if n13 == 0 or n2 == 0:
        check(lib().moe_check_problem(ctypes.byref(prob)), "moe_prepared_weights_bytes")
    w13p = torch.empty(n13, dtype=torch.uint8, device=w13.device)
    w2p = torch.empty(n2, dtype=torch.uint8, device=w2.device)
    check(lib().moe_prepare_weights_nvfp4(ctypes.byref(prob), _ptr(w13), _ptr(w13_scale), _ptr(w2),
                                          _ptr(w2_scale), _ptr(w13p), _ptr(w2p), _stream(stream)),
          "moe_prepare_weights_nvfp4")
    for t in (w13p, w2p):
        t.moe_intermediate = prob.intermediate
        t.moe_nvfp4 = True
    return w13p, w2p


def quantize_weights_nvfp4(w: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """NVFP4 quantisation of bf16 [..., rows, cols] weights along each row: (packed E2M1
    codes uint8 [..., rows, cols/2], E4M3 block scales uint8 [..., rows, cols/16], tensor
    scales fp32 [...] = amax / (6 * 448) per matrix)."""
    _dev(w, "w", torch.bfloat16)
    rows, cols = w.shape[-2], w.shape[-1]
    mats = w.numel() // (rows * cols)
    codes = torch.empty(tuple(w.shape[:-1]) + (cols // 2,), dtype=torch.uint8, device=w.device)
    scales = torch.empty(tuple(w.shape[:-1]) + (cols // 16,), dtype=torch.uint8, device=w.device)
    g = torch.empty(tuple(w.shape[:-2]), dtype=torch.float32, device=w.device)
    check(lib().moe_quantize_weights_nvfp4(_ptr(w), mats, rows, cols, _ptr(codes), _ptr(scales), _ptr(g),
                                           _stream(stream)), "moe_quantize_weights_nvfp4")
    return codes, scales, g


def quantize_weights_mxfp8(w: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MXFP8 quantisation of bf16 [..., rows, cols] weights along each row: (codes uint8
    [..., rows, cols], E8M0 scale bytes uint8 [..., rows, cols/32])."""
    _dev(w, "w", torch.bfloat16)
    rows, cols = w.shape[-2], w.shape[-1]
    mats = w.numel() // (rows * cols)
    codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    scales = torch.empty(tuple(w.shape[:-1]) + (cols // 32,), dtype=torch.uint8, device=w.device)
    check(lib().moe_quantize_weights_mxfp8(_ptr(w), mats, rows, cols, _ptr(codes), _ptr(scales),
                                           _stream(stream)), "moe_quantize_weights_mxfp8")
    return codes, scales


def quantize_weights_fp8_per_tensor(w: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-matrix e4m3 quantisation of bf16 [..., rows, cols] weights: (codes uint8, scales
    fp32 [...]) with scale = amax / 448 per matrix."""
    _dev(w, "w", torch.bfloat16)
    rows, cols = w.shape[-2], w.shape[-1]
    mats = w.numel() // (rows * cols)
    codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    scales = torch.empty(tuple(w.shape[:-2]), dtype=torch.float32, device=w.device)
    check(lib().moe_quantize_weights_fp8_per_tensor(_ptr(w), mats, rows, cols, _ptr(codes), _ptr(scales),
                                                    _stream(stream)), "moe_quantize_weights_fp8_per_tensor")
    return codes, scales


def quantize_weights_fp8(w: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-128x128-block e4m3 quantisation of bf16 [..., rows, cols] weights."""
    _dev(w, "w", torch.bfloat16)
    rows, cols = w.shape[-2], w.shape[-1]
    mats = w.numel() // (rows * cols)
    codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    scales = torch.empty(tuple(w.shape[:-2]) + (rows // 128, cols // 128), dtype=torch.float32,
                         device=w.device)
    check(lib().moe_quantize_weights_fp8(_ptr(w), mats, rows, cols, _ptr(codes), _ptr(scales),
                                         _stream(stream)), "moe_quantize_weights_fp8")
    return codes, scales


def _problem_from(hidden, router_logits, w2, topk, renormalize, activation_type, num_shared,
                  fp8, pdl, input_scale=0.0, activation_scale=0.0) -> Problem:
    T, H = hidden.shape
    E_r = router_logits.shape[1]
    I = getattr(w2, "moe_intermediate", None)
    if I is None:
        if w2.dim() != 3:
            raise ValueError("w2 must come from prepare_weights (or be [E, H, I] row-major)")
        I = w2.shape[2]
    return make_problem(T, H, E_r, topk, I, renormalize=renormalize,
                        activation=activation_type, num_shared=num_shared, fp8=fp8, pdl=pdl,
                        input_scale=input_scale, activation_scale=activation_scale)


_WS_CACHE: Dict[tuple, torch.Tensor] = {}


def _workspace_for(prob: Problem, device, stream=None) -> torch.Tensor:
    """The cached workspace of calls that pass none: one per device, stream and problem
    shape apart from the token count, grown to the largest token count seen (a workspace
    sized for more tokens serves fewer), so a caller whose batch size changes from call to
    call reuses one buffer. Calls on different streams get different workspaces."""
    s = stream if stream is not None else torch.cuda.current_stream(device)
    key = (str(device), s.cuda_stream, prob.hidden, prob.num_routed, prob.num_shared, prob.intermediate,
           prob.topk, prob.activation, prob.wdtype, prob.block_m)
    ws = _WS_CACHE.get(key)
    if ws is None or ws.numel() < workspace_size(prob):
        ws = new_workspace(prob, device)
        _WS_CACHE[key] = ws
    return ws


def moe_forward(hidden: torch.Tensor, router_logits: torch.Tensor, w13: torch.Tensor,
                w2: torch.Tensor, topk: int, renormalize: bool, activation_type,
                w13_scale: Optional[torch.Tensor] = None, w2_scale: Optional[torch.Tensor] = None,
                num_shared: int = 0, *, workspace: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, pdl: bool = True, stream=None,
                input_scale: Optional[float] = None, activation_scale: Optional[float] = None) -> torch.Tensor:
    """Fused MoE layer forward on the current CUDA stream.

    ``hidden`` bf16 [T,H]; ``router_logits`` fp32 [T,E_r]; ``w13``/``w2`` prepared by
    :func:`prepare_weights` (bf16, or uint8 e4m3 codes with fp32 block scales
    ``w13_scale`` [E, N1/128, H/128] and ``w2_scale`` [E, H/128, I/128]; with
    ``input_scale`` and ``activation_scale`` given, per-tensor FP8 with ``w13_scale`` and
    ``w2_scale`` fp32 [E]). Returns bf16 [T,H].
    """
    per_tensor = input_scale is not None or activation_scale is not None
    if getattr(w13, "moe_mxfp8", False):
        fp8 = "mxfp8"  # scales inside the prepared weights
    elif getattr(w13, "moe_nvfp4", False):
        fp8 = "nvfp4"  # block scales inside the prepared weights; w13_scale / w2_scale: tensor scales
    else:
        fp8 = "per_tensor" if per_tensor else w13_scale is not None
    _dev(hidden, "hidden", torch.bfloat16)
    _dev(router_logits, "router_logits", torch.float32)
    _dev(w13, "w13")
    _dev(w2, "w2")
    prob = _problem_from(hidden, router_logits, w2, topk, renormalize, activation_type,
                         num_shared, fp8, pdl, input_scale or 0.0, activation_scale or 0.0)
    if workspace is None:
        workspace = _workspace_for(prob, hidden.device, stream)
    if out is None:
        out = torch.empty_like(hidden)
    check(lib().moe_forward(ctypes.byref(prob), _ptr(hidden), _ptr(router_logits), _ptr(w13),
                            _ptr(w2), _ptr(w13_scale), _ptr(w2_scale), _ptr(out),
                            _ptr(workspace), workspace.numel(), _stream(stream)), "moe_forward")
    return out


def moe_forward_routed(hidden: torch.Tensor, topk_ids: torch.Tensor, topk_weights: torch.Tensor,
                       w13: torch.Tensor, w2: torch.Tensor, num_routed: int, activation_type,
                       w13_scale: Optional[torch.Tensor] = None, w2_scale: Optional[torch.Tensor] = None,
                       num_shared: int = 0, *, workspace: Optional[torch.Tensor] = None,
                       out: Optional[torch.Tensor] = None, pdl: bool = True, stream=None) -> torch.Tensor:
    """The forward with caller-supplied routing: ``topk_ids`` int32 [T, topk] in
    [0, num_routed), ``topk_weights`` fp32 [T, topk] (used as given); the rest as
    :func:`moe_forward`. Out-of-range ids are dropped and reported by
    :func:`device_status`."""
    fp8 = ("mxfp8" if getattr(w13, "moe_mxfp8", False) else
           ("nvfp4" if getattr(w13, "moe_nvfp4", False) else w13_scale is not None))
    _dev(hidden, "hidden", torch.bfloat16)
    _dev(topk_ids, "topk_ids", torch.int32)
    _dev(topk_weights, "topk_weights", torch.float32)
    _dev(w13, "w13")
    _dev(w2, "w2")
    T, H = hidden.shape
    topk = topk_ids.shape[1]
    if topk_ids.shape != (T, topk) or topk_weights.shape != (T, topk):
        raise ValueError("topk_ids and topk_weights must both be [T, topk]")
    I = getattr(w2, "moe_intermediate", None)
    if I is None:
        if w2.dim() != 3:
            raise ValueError("w2 must come from prepare_weights (or be [E, H, I] row-major)")
        I = w2.shape[2]
    prob = make_problem(T, H, num_routed, topk, I, renormalize=False, activation=activation_type,
                        num_shared=num_shared, fp8=fp8, pdl=pdl)
    if workspace is None:
        workspace = _workspace_for(prob, hidden.device, stream)
    if out is None:
        out = torch.empty_like(hidden)
    check(lib().moe_forward_routed(ctypes.byref(prob), _ptr(hidden), _ptr(topk_ids), _ptr(topk_weights),
                                   _ptr(w13), _ptr(w2), _ptr(w13_scale), _ptr(w2_scale), _ptr(out),
                                   _ptr(workspace), workspace.numel(), _stream(stream)), "moe_forward_routed")
    return out


def moe_forward_host(prob: Problem, hidden_host: torch.Tensor, logits_host: torch.Tensor,
                     w13: torch.Tensor, w2: torch.Tensor, out_host: torch.Tensor,
                     workspace: torch.Tensor, w13_scale=None, w2_scale=None, stream=None) -> None:
    """The forward on HOST tensors (pinned for asynchronous copies); blocks until done."""
    for t, n in ((hidden_host, "hidden"), (logits_host, "logits"), (out_host, "out")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous CPU tensor")
    check(lib().moe_forward_host(ctypes.byref(prob), _ptr(hidden_host), _ptr(logits_host),
                                 _ptr(w13), _ptr(w2), _ptr(w13_scale), _ptr(w2_scale),
                                 _ptr(out_host), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "moe_forward_host")


# ---- the five steps, for tests and per-kernel timing -----------------------------------

def stage_route(prob, router_logits, workspace, stream=None):
    check(lib().moe_stage_route(ctypes.byref(prob), _ptr(router_logits), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "moe_stage_route")


def stage_align(prob, workspace, stream=None):
    check(lib().moe_stage_align(ctypes.byref(prob), _ptr(workspace), workspace.numel(),
                                _stream(stream)), "moe_stage_align")


def stage_quant_act(prob, hidden, workspace, stream=None):
    check(lib().moe_stage_quant_act(ctypes.byref(prob), _ptr(hidden), _ptr(workspace),
                                    workspace.numel(), _stream(stream)), "moe_stage_quant_act")


def stage_permute(prob, hidden, workspace, stream=None):
    check(lib().moe_stage_permute(ctypes.byref(prob), _ptr(hidden), _ptr(workspace),
                                  workspace.numel(), _stream(stream)), "moe_stage_permute")


def stage_gemm1(prob, hidden, w13, workspace, w13_scale=None, stream=None):
    check(lib().moe_stage_gemm1(ctypes.byref(prob), _ptr(hidden), _ptr(w13), _ptr(w13_scale),
                                _ptr(workspace), workspace.numel(), _stream(stream)),
          "moe_stage_gemm1")


def stage_gemm2(prob, w2, workspace, w2_scale=None, stream=None):
    check(lib().moe_stage_gemm2(ctypes.byref(prob), _ptr(w2), _ptr(w2_scale), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "moe_stage_gemm2")


def stage_combine(prob, out, workspace, stream=None):
    check(lib().moe_stage_combine(ctypes.byref(prob), _ptr(out), _ptr(workspace),
                                  workspace.numel(), _stream(stream)), "moe_stage_combine")


def device_status(workspace: torch.Tensor, stream=None) -> Tuple[int, int]:
    """(status, raw word) of the workspace's device status; synchronises the stream."""
    detail = ctypes.c_int32(0)
    st = lib().moe_get_device_status(_ptr(workspace), _stream(stream), ctypes.byref(detail))
    return st, detail.value


def read_workspace(prob: Problem, workspace: torch.Tensor) -> Dict[str, torch.Tensor]:
    """Views of the intermediates inside a workspace (device tensors, no copy)."""
    L = workspace_layout(prob)
    T, kk = prob.num_tokens, prob.topk + prob.num_shared
    P = T * kk
    E = prob.num_routed + prob.num_shared
    rows = L["max_rows"]
    fp8 = prob.wdtype == MOE_DTYPE_FP8_BLOCK128
    I, H = prob.intermediate, prob.hidden

    def view(off, n, dtype):
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        return workspace[off:off + nbytes].view(dtype)

    out = {
        "status": view(L["status"], 1, torch.int32),
        "num_blocks": view(L["num_blocks"], 2, torch.int32),
        "topk_ids": view(L["topk_ids"], P, torch.int32).view(T, kk),
        "topk_w": view(L["topk_w"], P, torch.float32).view(T, kk),
        "sorted_pair_ids": view(L["sorted_pair_ids"], rows, torch.int32),
        "expert_offsets": view(L["expert_offsets"], E + 1, torch.int32),
        "block_expert": view(L["block_expert"], rows // L["block_m"], torch.int32),
        "pair_to_row": view(L["pair_to_row"], P, torch.int32),
    }
    if L["block_m"] == 16:
        # weighted GEMM2 rows as fp16 with a power-of-two exponent per 32 columns:
        # y = y16 * 2^y_exp
        out["y16"] = view(L["y"], rows * H, torch.float16).view(rows, H)
        out["y_exp"] = view(L["y"] + rows * H * 2, rows * (H // 32), torch.int8).view(rows, H // 32)
    else:
        out["y"] = view(L["y"], rows * H, torch.float32).view(rows, H)
    if prob.wdtype == MOE_DTYPE_MXFP8:
        # bf16 activation (64-column chunks), e4m3 codes of the hidden rows and of the
        # activation (128-column chunks), all in row-group order; the scale blocks raw
        act_cols = -(-I // 64) * 64
        out["act"] = view(L["act"], rows * act_cols, torch.bfloat16)
        out["xs"] = view(L["xs"], rows * H, torch.uint8)
        out["xs_scale"] = view(L["xs_scale"], rows // 16 * (H // 128) * 1024, torch.uint8)
        out["actq"] = view(L["actq"], rows * I, torch.uint8)
        out["act_scale"] = view(L["act_scale"], rows // 16 * (I // 128) * 1024, torch.uint8)
        out["group_info"] = view(L["group_info"], (rows // 16 + 1) * 2, torch.int32).view(-1, 2)
    elif fp8 and L["block_m"] == 16:
        # FP8 block-128 on the swapped-operand GEMMs: the bf16 activation (64-column
        # chunks), and the quantised hidden rows and activation with each K step's fp32 row
        # scales behind its codes (132 bytes per row per 128 columns); flat views
        act_cols = -(-I // 64) * 64
        out["act"] = view(L["act"], rows * act_cols, torch.bfloat16)
        out["xs"] = view(L["xs"], rows * (H // 128) * 132, torch.uint8)
        out["actq"] = view(L["actq"], rows * (I // 128) * 132, torch.uint8)
        out["group_info"] = view(L["group_info"], (rows // 16 + 1) * 2, torch.int32).view(-1, 2)
    elif prob.wdtype == MOE_DTYPE_NVFP4:
        # bf16 activation (64-column chunks); packed E2M1 codes of the hidden rows and of the
        # activation (128-byte chunks of 256 values) in row-group order; the scale blocks raw;
        # the per-token quantised hidden rows
        act_cols = -(-I // 64) * 64
        out["act"] = view(L["act"], rows * act_cols, torch.bfloat16)
        out["xq"] = view(L["xq"], T * H // 2, torch.uint8).view(T, H // 2)
        out["xq_scale"] = view(L["xq_scale"], T * H // 16, torch.uint8).view(T, H // 16)
        out["xs"] = view(L["xs"], rows * H // 2, torch.uint8)
        out["xs_scale"] = view(L["xs_scale"], rows // 16 * (H // 256) * 2048, torch.uint8)
        out["actq"] = view(L["actq"], rows * I // 2, torch.uint8)
        out["act_scale"] = view(L["act_scale"], rows // 16 * (I // 256) * 2048, torch.uint8)
        out["group_info"] = view(L["group_info"], (rows // 16 + 1) * 2, torch.int32).view(-1, 2)
    elif prob.wdtype == MOE_DTYPE_FP8_PER_TENSOR:
        # e4m3 codes in row-group order (128-column chunks per group, swizzled); flat views
        out["act"] = view(L["act"], rows * I, torch.uint8)
        out["xs"] = view(L["xs"], rows * H, torch.uint8)
        out["group_info"] = view(L["group_info"], (rows // 16 + 1) * 2, torch.int32).view(-1, 2)
    elif L["block_m"] == 16:
        # the swapped-operand GEMMs keep the activation and the permuted hidden rows in
        # row-group order (64-column chunks per group, swizzled); flat views
        act_cols = -(-I // 64) * 64
        out["act"] = view(L["act"], rows * act_cols, torch.bfloat16)
        out["xs"] = view(L["xs"], rows * H, torch.bfloat16)
        out["group_info"] = view(L["group_info"], (rows // 16 + 1) * 2, torch.int32).view(-1, 2)
    else:
        out["act"] = view(L["act"], rows * I, torch.bfloat16).view(rows, I)
    if fp8:
        out["xq"] = view(L["xq"], T * H, torch.uint8).view(T, H)
        out["xq_scale"] = view(L["xq_scale"], T * (H // 128), torch.float32).view(T, H // 128)
    if fp8 and L["block_m"] == 128:
        out["actq"] = view(L["actq"], rows * I, torch.uint8).view(rows, I)
        out["act_scale"] = view(L["act_scale"], rows * (I // 128), torch.float32).view(rows, I // 128)
    return out
