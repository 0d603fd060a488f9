"""Python binding of the NVFP4 routed-expert MoE library (libnvfp4moe.so, sm_100a).

Every function here has the name of a C entry point in ``include/nvfp4_moe.h`` and only
marshals arguments: it checks tensors, allocates outputs and workspaces with PyTorch,
passes raw device pointers and the current CUDA stream through ctypes, and turns a
negative status into an exception.  All arithmetic runs in the library's kernels; there is
no fallback.  If the shared library is missing, the first call raises (importing the
package alone does not, so the build script inside it stays importable).

Format (page "GLM-5-NVFP4-MTP", "Model Description"): 4-bit E2M1 values, one E4M3 scale per
16 consecutive elements, one fp32 global scale per tensor.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "PATH_AUTO", "PATH_GEMV", "PATH_GEMM", "NVFP4Error", "lib", "library_path",
    "nvfp4_quantize", "nvfp4_quantize_workspace_size", "nvfp4_dequantize", "nvfp4_cast_f32",
    "moe_nvfp4_route", "moe_nvfp4_workspace_size", "moe_nvfp4_forward",
    "moe_nvfp4_read_error_flag", "moe_nvfp4_forward_profiled", "alloc_moe_workspace",
    "moe_nvfp4_forward_static", "nvfp4_selftest_wait_timeout", "nvfp4_amax",
    "nvfp4_quantize_with_amax", "moe_nvfp4_ep_local_experts", "moe_nvfp4_forward_ep",
    "moe_nvfp4_ep_reduce", "EP_MAX_PARTS", "moe_nvfp4_router", "moe_nvfp4_forward_logits",
    "moe_nvfp4_shared_expert", "moe_nvfp4_layer", "moe_nvfp4_layer_workspace_size",
    "nvfp4_w4a4_prepare_scales", "moe_nvfp4_forward_w4a4", "moe_nvfp4_w4a4_workspace_size",
]

PATH_AUTO, PATH_GEMV, PATH_GEMM = 0, 1, 2
WORKSPACE_ZERO_BYTES = 512   # head of a workspace that must be zero before first use
EP_MAX_PARTS = 16            # partial outputs one moe_nvfp4_ep_reduce call sums
_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libnvfp4moe.so")


class NVFP4Error(RuntimeError):
    pass


def _load() -> ctypes.CDLL:
    if not os.path.exists(library_path):
        raise ImportError(
            f"{library_path} is missing: build it with "
            "`python -m bit_quantized_moe_nvfp4_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(library_path)
    P, I64, SZ, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
    sig = {
        "nvfp4_status_string": (ctypes.c_char_p, [I32]),
        "nvfp4_last_cuda_error": (ctypes.c_char_p, []),
        "nvfp4_quantize_workspace_size": (SZ, [I64, I64, I64]),
        "nvfp4_quantize": (I32, [P, I64, I64, I64, P, P, P, P, SZ, P]),
        "nvfp4_dequantize": (I32, [P, P, P, I64, I64, I64, P, P]),
        "nvfp4_cast_f32": (I32, [P, I64, P, P, P]),
        "moe_nvfp4_workspace_size": (SZ, [I64, I64, I64, I64, I64]),
        "moe_nvfp4_forward": (I32, [P, P, P, I64, I64, I64, I64, I64,
                                    P, P, P, P, P, P, P, P, SZ, P]),
        "moe_nvfp4_forward_path": (I32, [P, P, P, I64, I64, I64, I64, I64,
                                         P, P, P, P, P, P, P, P, SZ, I32, P]),
        "moe_nvfp4_forward_profiled": (I32, [P, P, P, I64, I64, I64, I64, I64,
                                             P, P, P, P, P, P, P, P, SZ, I32, P, P]),
        "moe_nvfp4_read_error_flag": (I32, [P, P, P]),
        "moe_nvfp4_route": (I32, [P, I64, I64, I64, P, P, P, P, P, P]),
        "moe_nvfp4_forward_static": (I32, [P, P, P, I64, I64, I64, I64, I64,
                                           P, P, P, P, P, P, P, P, P]),
        "nvfp4_selftest_wait_timeout": (I32, [P, I32, I64, P]),
        "nvfp4_amax": (I32, [P, I64, I64, I64, P, I32, P]),
        "nvfp4_quantize_with_amax": (I32, [P, I64, I64, I64, P, P, P, P, P]),
        "moe_nvfp4_ep_local_experts": (I64, [I64, I64, I64]),
        "moe_nvfp4_forward_ep": (I32, [P, P, P, I64, I64, I64, I64, I64, I64, I64,
                                       P, P, P, P, P, P, P, P, SZ, I32, P]),
        "moe_nvfp4_ep_reduce": (I32, [P, I64, I64, I64, P, P]),
        "moe_nvfp4_router": (I32, [P, I64, I64, I64, P, P, P]),
        "nvfp4_w4a4_prepare_scales": (I32, [P, I64, I64, I64, I64, P, P]),
        "moe_nvfp4_w4a4_workspace_size": (SZ, [I64, I64, I64, I64, I64]),
        "moe_nvfp4_forward_w4a4_profiled": (I32, [P, P, P, I64, I64, I64, I64, I64,
                                                  P, P, P, P, P, P, P, P, SZ, P, P]),
        "moe_nvfp4_forward_w4a4": (I32, [P, P, P, I64, I64, I64, I64, I64,
                                         P, P, P, P, P, P, P, P, SZ, P]),
        "moe_nvfp4_shared_workspace_size": (SZ, [I64, I64]),
        "moe_nvfp4_shared_expert": (I32, [P, I64, I64, I64, P, P, P, P, P, SZ, P]),
        "moe_nvfp4_layer_workspace_size": (SZ, [I64, I64, I64, I64, I64, I64]),
        "moe_nvfp4_layer": (I32, [P, P, I64, I64, I64, I64, I64, P, P, P, P, P, P, P, P, I64,
                                  P, P, P, P, SZ, I32, P]),
        "moe_nvfp4_forward_logits": (I32, [P, P, I64, I64, I64, I64, I64,
                                           P, P, P, P, P, P, P, P, P, P, SZ, I32, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


_LIB = None


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    if name == "lib":
        return _lib()
    raise AttributeError(name)


def _check(status: int) -> None:
    lib = _lib()
    if status != 0:
        msg = lib.nvfp4_status_string(status).decode()
        if status == -4:
            msg += " -- " + lib.nvfp4_last_cuda_error().decode()
        raise NVFP4Error(msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or not t.is_cuda \
            or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA tensor of {dtype}")


# ------------------------------------------------------------------------------ codec
def nvfp4_quantize_workspace_size(n_tensors: int, rows: int, cols: int) -> int:
    return int(_lib().nvfp4_quantize_workspace_size(n_tensors, rows, cols))


def nvfp4_quantize(x: torch.Tensor, packed=None, scales=None, global_scale=None,
                   workspace=None):
    """bf16 [n, rows, cols] (or [rows, cols]) -> (packed u8 [..., cols/2],
    scales u8 (E4M3 codes) [..., cols/16], global_scale fp32 [n])."""
    _need(x, torch.bfloat16, "x")
    squeeze = x.dim() == 2
    x3 = x.unsqueeze(0) if squeeze else x
    n, rows, cols = x3.shape
    dev = x.device
    if packed is None:
        packed = torch.empty((n, rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((n, rows, cols // 16), dtype=torch.uint8, device=dev)
    if global_scale is None:
        global_scale = torch.empty((n,), dtype=torch.float32, device=dev)
    ws_bytes = nvfp4_quantize_workspace_size(n, rows, cols)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    _check(_lib().nvfp4_quantize(_ptr(x3), n, rows, cols, _ptr(packed), _ptr(scales),
                              _ptr(global_scale), _ptr(workspace), workspace.numel(),
                              _stream(dev)))
    if squeeze:
        return packed[0], scales[0], global_scale
    return packed, scales, global_scale


def nvfp4_amax(x: torch.Tensor, out=None, merge: bool = False) -> torch.Tensor:
    """Per-tensor max |x| of bf16 [n, rows, cols] (or [rows, cols]) -> fp32 [n].  With
    merge=True, `out` holds the amax of earlier calibration passes and becomes the
    element-wise max of it and this pass's."""
    _need(x, torch.bfloat16, "x")
    x3 = x.unsqueeze(0) if x.dim() == 2 else x
    n, rows, cols = x3.shape
    if out is None:
        if merge:
            raise ValueError("merge=True needs the running amax in `out`")
        out = torch.empty((n,), dtype=torch.float32, device=x.device)
    _need(out, torch.float32, "out")
    _check(_lib().nvfp4_amax(_ptr(x3), n, rows, cols, _ptr(out), int(bool(merge)),
                             _stream(x.device)))
    return out


def nvfp4_quantize_with_amax(x: torch.Tensor, amax: torch.Tensor, packed=None, scales=None,
                             global_scale=None):
    """nvfp4_quantize with the per-tensor amax given (a calibrated one): g = amax / 2688.
    -> (packed, scales, global_scale) as nvfp4_quantize."""
    _need(x, torch.bfloat16, "x")
    _need(amax, torch.float32, "amax")
    squeeze = x.dim() == 2
    x3 = x.unsqueeze(0) if squeeze else x
    n, rows, cols = x3.shape
    dev = x.device
    if packed is None:
        packed = torch.empty((n, rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((n, rows, cols // 16), dtype=torch.uint8, device=dev)
    if global_scale is None:
        global_scale = torch.empty((n,), dtype=torch.float32, device=dev)
    _check(_lib().nvfp4_quantize_with_amax(_ptr(x3), n, rows, cols, _ptr(amax), _ptr(packed),
                                           _ptr(scales), _ptr(global_scale), _stream(dev)))
    if squeeze:
        return packed[0], scales[0], global_scale
    return packed, scales, global_scale


def nvfp4_dequantize(packed: torch.Tensor, scales: torch.Tensor, global_scale: torch.Tensor,
                     out=None) -> torch.Tensor:
    """Inverse of nvfp4_quantize up to rounding: bf16( fp32(e2m1 * e4m3) * g )."""
    _need(packed, torch.uint8, "packed")
    _need(scales, torch.uint8, "scales")
    _need(global_scale, torch.float32, "global_scale")
    squeeze = packed.dim() == 2
    p3 = packed.unsqueeze(0) if squeeze else packed
    n, rows, half = p3.shape
    cols = half * 2
    if out is None:
        out = torch.empty((n, rows, cols), dtype=torch.bfloat16, device=packed.device)
    _check(_lib().nvfp4_dequantize(_ptr(p3), _ptr(scales), _ptr(global_scale), n, rows, cols,
                                _ptr(out), _stream(packed.device)))
    return out[0] if squeeze else out


def nvfp4_cast_f32(v: torch.Tensor):
    """fp32 values -> (E4M3 codes u8, E2M1 codes u8), as the quantizer rounds them."""
    _need(v, torch.float32, "v")
    e4 = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    e2 = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _check(_lib().nvfp4_cast_f32(_ptr(v), v.numel(), _ptr(e4), _ptr(e2), _stream(v.device)))
    return e4, e2


# ------------------------------------------------------------------------------ MoE
def moe_nvfp4_workspace_size(T: int, H: int, I: int, E: int, K: int) -> int:
    return int(_lib().moe_nvfp4_workspace_size(T, H, I, E, K))


def alloc_moe_workspace(T, H, I, E, K, device="cuda") -> torch.Tensor:
    """Workspace for moe_nvfp4_forward: its head (error flag and work counters) zeroed."""
    ws = torch.empty((moe_nvfp4_workspace_size(T, H, I, E, K),), dtype=torch.uint8,
                     device=device)
    ws[:WORKSPACE_ZERO_BYTES].zero_()
    return ws


def moe_nvfp4_route(topk_ids: torch.Tensor, E: int):
    """int32 [T, K] -> (counts [E], offsets [E+1], perm [T*K], inv [T*K], flag [1])."""
    _need(topk_ids, torch.int32, "topk_ids")
    T, K = topk_ids.shape
    dev = topk_ids.device
    counts = torch.empty((E,), dtype=torch.int32, device=dev)
    offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    perm = torch.full((T * K,), -1, dtype=torch.int32, device=dev)
    inv = torch.empty((T * K,), dtype=torch.int32, device=dev)
    flag = torch.zeros((1,), dtype=torch.int32, device=dev)
    _check(_lib().moe_nvfp4_route(_ptr(topk_ids), T, K, E, _ptr(counts), _ptr(offsets),
                               _ptr(perm), _ptr(inv), _ptr(flag), _stream(dev)))
    return counts, offsets, perm, inv, flag


def moe_nvfp4_forward(x, topk_ids, topk_w, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn,
                      out=None, workspace=None, path: int = PATH_AUTO) -> torch.Tensor:
    """Routed-expert MoE MLP from NVFP4 weights (see include/nvfp4_moe.h).

    x bf16 [T,H]; topk_ids int32 [T,K]; topk_w fp32 [T,K]; w_gu u8 [E,2I,H/2];
    s_gu u8 [E,2I,H/16]; g_gu fp32 [E]; w_dn u8 [E,H,I/2]; s_dn u8 [E,H,I/16];
    g_dn fp32 [E].  Returns out bf16 [T,H]."""
    _need(x, torch.bfloat16, "x")
    _need(topk_ids, torch.int32, "topk_ids")
    _need(topk_w, torch.float32, "topk_w")
    for t, n in ((w_gu, "w_gu"), (s_gu, "s_gu"), (w_dn, "w_dn"), (s_dn, "s_dn")):
        _need(t, torch.uint8, n)
    _need(g_gu, torch.float32, "g_gu")
    _need(g_dn, torch.float32, "g_dn")
    T, H = x.shape
    K = topk_ids.shape[1]
    E, twoI, _ = w_gu.shape
    I = twoI // 2
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = alloc_moe_workspace(T, H, I, E, K, x.device)
    _check(_lib().moe_nvfp4_forward_path(
        _ptr(x), _ptr(topk_ids), _ptr(topk_w), T, H, I, E, K, _ptr(w_gu), _ptr(s_gu),
        _ptr(g_gu), _ptr(w_dn), _ptr(s_dn), _ptr(g_dn), _ptr(out), _ptr(workspace),
        workspace.numel(), int(path), _stream(x.device)))
    return out


def moe_nvfp4_router(logits: torch.Tensor, K: int, ids=None, w=None):
    """Top-K experts and renormalised softmax weights from fp32 logits [T, E] (see
    include/nvfp4_moe.h).  Returns (ids int32 [T, K], w fp32 [T, K])."""
    _need(logits, torch.float32, "logits")
    T, E = logits.shape
    if ids is None:
        ids = torch.empty((T, K), dtype=torch.int32, device=logits.device)
    if w is None:
        w = torch.empty((T, K), dtype=torch.float32, device=logits.device)
    _need(ids, torch.int32, "ids")
    _need(w, torch.float32, "w")
    _check(_lib().moe_nvfp4_router(_ptr(logits), T, E, K, _ptr(ids), _ptr(w),
                                   _stream(logits.device)))
    return ids, w


def moe_nvfp4_forward_logits(x, router_logits, K: int, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn,
                             out=None, ids_out=None, w_out=None, workspace=None,
                             path: int = PATH_AUTO) -> torch.Tensor:
    """The router on fp32 logits [T, E], then the layer on its decisions, in one call.
    ids_out / w_out (optional, [T, K]) receive the router's decisions."""
    _need(x, torch.bfloat16, "x")
    _need(router_logits, torch.float32, "router_logits")
    for t, n in ((w_gu, "w_gu"), (s_gu, "s_gu"), (w_dn, "w_dn"), (s_dn, "s_dn")):
        _need(t, torch.uint8, n)
    _need(g_gu, torch.float32, "g_gu")
    _need(g_dn, torch.float32, "g_dn")
    if ids_out is not None:
        _need(ids_out, torch.int32, "ids_out")
    if w_out is not None:
        _need(w_out, torch.float32, "w_out")
    T, H = x.shape
    E, twoI, _ = w_gu.shape
    I = twoI // 2
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = alloc_moe_workspace(T, H, I, E, K, x.device)
    _check(_lib().moe_nvfp4_forward_logits(
        _ptr(x), _ptr(router_logits), T, H, I, E, K, _ptr(w_gu), _ptr(s_gu), _ptr(g_gu),
        _ptr(w_dn), _ptr(s_dn), _ptr(g_dn), _ptr(out), _ptr(ids_out), _ptr(w_out),
        _ptr(workspace), workspace.numel(), int(path), _stream(x.device)))
    return out


def moe_nvfp4_shared_expert(x, w_gu, w_dn, routed=None, out=None, workspace=None):
    """The BF16 shared expert (see include/nvfp4_moe.h): out = bf16(routed + W_dn .
    bf16(silu(W_g x) * W_u x)) per token.  x bf16 [T,H]; w_gu bf16 [2Is,H]; w_dn bf16
    [H,Is]; routed fp32 [T,H] or None.  Returns out bf16 [T,H]."""
    _need(x, torch.bfloat16, "x")
    _need(w_gu, torch.bfloat16, "w_gu")
    _need(w_dn, torch.bfloat16, "w_dn")
    if routed is not None:
        _need(routed, torch.float32, "routed")
    T, H = x.shape
    Is = w_gu.shape[0] // 2
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        n = int(_lib().moe_nvfp4_shared_workspace_size(T, Is))
        workspace = torch.empty((max(n, 16),), dtype=torch.uint8, device=x.device)
    _check(_lib().moe_nvfp4_shared_expert(_ptr(x), T, H, Is, _ptr(w_gu), _ptr(w_dn),
                                          _ptr(routed), _ptr(out), _ptr(workspace),
                                          workspace.numel(), _stream(x.device)))
    return out


def moe_nvfp4_layer_workspace_size(T, H, I, E, K, Is) -> int:
    return int(_lib().moe_nvfp4_layer_workspace_size(T, H, I, E, K, Is))


def moe_nvfp4_layer(x, router_logits, K: int, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn,
                    shared_gu, shared_dn, out=None, ids_out=None, w_out=None, workspace=None,
                    path: int = PATH_AUTO) -> torch.Tensor:
    """The whole MoE layer in one call: router on the logits, the routed NVFP4 experts,
    and the BF16 shared expert added before the single rounding to bf16."""
    _need(x, torch.bfloat16, "x")
    _need(router_logits, torch.float32, "router_logits")
    for t, n in ((w_gu, "w_gu"), (s_gu, "s_gu"), (w_dn, "w_dn"), (s_dn, "s_dn")):
        _need(t, torch.uint8, n)
    _need(g_gu, torch.float32, "g_gu")
    _need(g_dn, torch.float32, "g_dn")
    _need(shared_gu, torch.bfloat16, "shared_gu")
    _need(shared_dn, torch.bfloat16, "shared_dn")
    T, H = x.shape
    E, twoI, _ = w_gu.shape
    I, Is = twoI // 2, shared_gu.shape[0] // 2
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty((moe_nvfp4_layer_workspace_size(T, H, I, E, K, Is),),
                                dtype=torch.uint8, device=x.device)
        workspace[:WORKSPACE_ZERO_BYTES].zero_()
    _check(_lib().moe_nvfp4_layer(
        _ptr(x), _ptr(router_logits), T, H, I, E, K, _ptr(w_gu), _ptr(s_gu), _ptr(g_gu),
        _ptr(w_dn), _ptr(s_dn), _ptr(g_dn), _ptr(shared_gu), _ptr(shared_dn), Is, _ptr(out),
        _ptr(ids_out), _ptr(w_out), _ptr(workspace), workspace.numel(), int(path),
        _stream(x.device)))
    return out


def nvfp4_w4a4_prepare_scales(scales: torch.Tensor, gate_rows: int = 0, out=None):
    """A weight's E4M3 scales [n, rows, cols/16] rearranged into the block-scaled tensor
    cores' layout (see include/nvfp4_moe.h); gate_rows = I for a fused gate/up weight."""
    _need(scales, torch.uint8, "scales")
    n, rows, c16 = scales.shape
    if out is None:
        out = torch.empty_like(scales)
    _need(out, torch.uint8, "out")
    _check(_lib().nvfp4_w4a4_prepare_scales(_ptr(scales), n, rows, c16 * 16, int(gate_rows),
                                            _ptr(out), _stream(scales.device)))
    return out


def moe_nvfp4_w4a4_workspace_size(T, H, I, E, K) -> int:
    return int(_lib().moe_nvfp4_w4a4_workspace_size(T, H, I, E, K))


def moe_nvfp4_forward_w4a4(x, topk_ids, topk_w, w_gu, sf_gu, g_gu, w_dn, sf_dn, g_dn,
                           out=None, workspace=None) -> torch.Tensor:
    """The routed layer on the FP4 tensor cores with NVFP4 activations (W4A4); sf_gu / sf_dn
    are the prepared scales.  Returns out bf16 [T, H]."""
    _need(x, torch.bfloat16, "x")
    _need(topk_ids, torch.int32, "topk_ids")
    _need(topk_w, torch.float32, "topk_w")
    for t, n in ((w_gu, "w_gu"), (sf_gu, "sf_gu"), (w_dn, "w_dn"), (sf_dn, "sf_dn")):
        _need(t, torch.uint8, n)
    _need(g_gu, torch.float32, "g_gu")
    _need(g_dn, torch.float32, "g_dn")
    T, H = x.shape
    K = topk_ids.shape[1]
    E, twoI, _ = w_gu.shape
    I = twoI // 2
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty((moe_nvfp4_w4a4_workspace_size(T, H, I, E, K),),
                                dtype=torch.uint8, device=x.device)
        workspace[:WORKSPACE_ZERO_BYTES].zero_()
    _check(_lib().moe_nvfp4_forward_w4a4(
        _ptr(x), _ptr(topk_ids), _ptr(topk_w), T, H, I, E, K, _ptr(w_gu), _ptr(sf_gu),
        _ptr(g_gu), _ptr(w_dn), _ptr(sf_dn), _ptr(g_dn), _ptr(out), _ptr(workspace),
        workspace.numel(), _stream(x.device)))
    return out


def moe_nvfp4_forward_w4a4_profiled(x, topk_ids, topk_w, w_gu, sf_gu, g_gu, w_dn, sf_dn, g_dn,
                                    out, workspace, stage_events):
    """moe_nvfp4_forward_w4a4 with five torch.cuda.Event recorded between its stages."""
    T, H = x.shape
    K = topk_ids.shape[1]
    E, twoI, _ = w_gu.shape
    arr = (ctypes.c_void_p * 5)(*[ctypes.c_void_p(e.cuda_event) for e in stage_events])
    _check(_lib().moe_nvfp4_forward_w4a4_profiled(
        _ptr(x), _ptr(topk_ids), _ptr(topk_w), T, H, twoI // 2, E, K, _ptr(w_gu), _ptr(sf_gu),
        _ptr(g_gu), _ptr(w_dn), _ptr(sf_dn), _ptr(g_dn), _ptr(out), _ptr(workspace),
        workspace.numel(), arr, _stream(x.device)))
    return out


def moe_nvfp4_ep_local_experts(E: int, ep_size: int, ep_rank: int) -> int:
    """Experts rank ep_rank of ep_size owns (those e < E with e % ep_size == ep_rank)."""
    return int(_lib().moe_nvfp4_ep_local_experts(E, ep_size, ep_rank))


def moe_nvfp4_forward_ep(x, topk_ids, topk_w, E: int, ep_size: int, ep_rank: int,
                         w_gu, s_gu, g_gu, w_dn, s_dn, g_dn, out=None, workspace=None,
                         path: int = PATH_AUTO) -> torch.Tensor:
    """This rank's experts only (expert-parallel forward; see include/nvfp4_moe.h).

    topk_ids hold global ids in [0, E); the weight tensors hold this rank's experts,
    local index l = expert l * ep_size + ep_rank.  Returns the fp32 partial [T,H]."""
    _need(x, torch.bfloat16, "x")
    _need(topk_ids, torch.int32, "topk_ids")
    _need(topk_w, torch.float32, "topk_w")
    for t, n in ((w_gu, "w_gu"), (s_gu, "s_gu"), (w_dn, "w_dn"), (s_dn, "s_dn")):
        _need(t, torch.uint8, n)
    _need(g_gu, torch.float32, "g_gu")
    _need(g_dn, torch.float32, "g_dn")
    T, H = x.shape
    K = topk_ids.shape[1]
    E_loc, twoI, _ = w_gu.shape
    if E_loc != moe_nvfp4_ep_local_experts(E, ep_size, ep_rank):
        raise ValueError(f"w_gu holds {E_loc} experts; rank {ep_rank} of {ep_size} owns "
                         f"{moe_nvfp4_ep_local_experts(E, ep_size, ep_rank)} of {E}")
    I = twoI // 2
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32, device=x.device)
    _need(out, torch.float32, "out")
    if workspace is None:
        workspace = alloc_moe_workspace(T, H, I, E_loc, K, x.device)
    _check(_lib().moe_nvfp4_forward_ep(
        _ptr(x), _ptr(topk_ids), _ptr(topk_w), T, H, I, E, K, ep_size, ep_rank, _ptr(w_gu),
        _ptr(s_gu), _ptr(g_gu), _ptr(w_dn), _ptr(s_dn), _ptr(g_dn), _ptr(out),
        _ptr(workspace), workspace.numel(), int(path), _stream(x.device)))
    return out


def moe_nvfp4_ep_reduce(partials, out=None) -> torch.Tensor:
    """bf16(partials[0] + partials[1] + ...) in fp32, in list order.  partials: fp32
    [rows, cols] CUDA tensors (this device's, or peer memory it can read)."""
    partials = list(partials)
    if not partials:
        raise ValueError("partials: at least one tensor")
    for j, p in enumerate(partials):
        _need(p, torch.float32, f"partials[{j}]")
        if p.shape != partials[0].shape or p.dim() != 2:
            raise ValueError("partials: fp32 tensors of one [rows, cols] shape")
    rows, cols = partials[0].shape
    dev = partials[0].device
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
    _need(out, torch.bfloat16, "out")
    arr = (ctypes.c_void_p * len(partials))(*[p.data_ptr() for p in partials])
    _check(_lib().moe_nvfp4_ep_reduce(arr, len(partials), rows, cols, _ptr(out),
                                      _stream(dev)))
    return out


def moe_nvfp4_forward_profiled(x, topk_ids, topk_w, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn,
                               out, workspace, stage_events, path: int = PATH_AUTO):
    """moe_nvfp4_forward with five torch.cuda.Event (enable_timing=True) recorded around
    the stages: before route, after route, after gate/up, after down, after combine."""
    T, H = x.shape
    K = topk_ids.shape[1]
    E, twoI, _ = w_gu.shape
    evs = [ctypes.c_void_p(e.cuda_event) for e in stage_events]
    arr = (ctypes.c_void_p * 5)(*evs)
    _check(_lib().moe_nvfp4_forward_profiled(
        _ptr(x), _ptr(topk_ids), _ptr(topk_w), T, H, twoI // 2, E, K, _ptr(w_gu), _ptr(s_gu),
        _ptr(g_gu), _ptr(w_dn), _ptr(s_dn), _ptr(g_dn), _ptr(out), _ptr(workspace),
        workspace.numel(), int(path), arr, _stream(x.device)))
    return out


def moe_nvfp4_forward_static(x, topk_ids, topk_w, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn,
                             out=None, error_flag=None) -> torch.Tensor:
    """The small-batch forward with the library's fixed scratch instead of a workspace
    (see include/nvfp4_moe.h).  error_flag: optional int32 [1] device tensor that
    receives the error bits.  Returns out bf16 [T,H]."""
    _need(x, torch.bfloat16, "x")
    _need(topk_ids, torch.int32, "topk_ids")
    _need(topk_w, torch.float32, "topk_w")
    for t, n in ((w_gu, "w_gu"), (s_gu, "s_gu"), (w_dn, "w_dn"), (s_dn, "s_dn")):
        _need(t, torch.uint8, n)
    _need(g_gu, torch.float32, "g_gu")
    _need(g_dn, torch.float32, "g_dn")
    if error_flag is not None:
        _need(error_flag, torch.int32, "error_flag")
    T, H = x.shape
    K = topk_ids.shape[1]
    E, twoI, _ = w_gu.shape
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    _check(_lib().moe_nvfp4_forward_static(
        _ptr(x), _ptr(topk_ids), _ptr(topk_w), T, H, twoI // 2, E, K, _ptr(w_gu), _ptr(s_gu),
        _ptr(g_gu), _ptr(w_dn), _ptr(s_dn), _ptr(g_dn), _ptr(out),
        _ptr(error_flag) if error_flag is not None else None, _stream(x.device)))
    return out


def nvfp4_selftest_wait_timeout(flag: torch.Tensor, kind: int, limit_ns: int) -> None:
    """Test hook: one kernel waits for something nothing completes (kind 0: an mbarrier
    phase, 1: bulk-copy bytes, 2: a global counter) with a limit of limit_ns; the wait
    runs out and bit 1 is ORed into flag's first int32 (device tensor, e.g. a forward
    workspace)."""
    if not isinstance(flag, torch.Tensor) or not flag.is_cuda:
        raise ValueError("flag: expected a CUDA tensor")
    _check(_lib().nvfp4_selftest_wait_timeout(_ptr(flag), int(kind), int(limit_ns),
                                              _stream(flag.device)))


def moe_nvfp4_read_error_flag(workspace: torch.Tensor) -> int:
    """Error bits of the last forward on this workspace (1 = id out of range,
    2 = a device wait gave up).  Synchronises the current stream."""
    flag = ctypes.c_int32(0)
    _check(_lib().moe_nvfp4_read_error_flag(_ptr(workspace), ctypes.byref(flag),
                                         _stream(workspace.device)))
    return int(flag.value)
