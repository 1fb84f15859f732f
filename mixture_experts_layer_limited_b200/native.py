"""ctypes binding of libmoe's C ABI (include/moe.h), one function per entry.

Argument marshalling only: torch tensors are passed as raw device pointers on
torch's current CUDA stream; every step of the layer runs in libmoe's kernels.
The library is loaded on first use; a missing library is an error, never a
fallback.
"""
import ctypes
import os
from typing import Optional

import torch

from .build import lib_path

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_ALIGNMENT = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_CHECK = 5
MOE_ERR_DEVICE_TIMEOUT = 6
MOE_DEVSTAT_BAD_EXPERT_ID = 0x1
MOE_DEVSTAT_TIMEOUT = 0x2
MOE_F32, MOE_BF16, MOE_E4M3 = 0, 1, 2
MOE_SOFTMAX, MOE_SIGMOID = 0, 1

EXPORTED = [
    "moe_route", "moe_gate_logits", "moe_permute_workspace_size", "moe_permute", "moe_permute_static_ws",
    "moe_grouped_swiglu",
    "moe_gate_up_swiglu", "moe_gate_up_swiglu_gather", "moe_down_proj",
    "moe_gate_up_swiglu_with_shared", "moe_down_proj_with_shared", "moe_down_proj_combine",
    "moe_swiglu_ffn_sync_size", "moe_swiglu_ffn_with_shared", "moe_tile_ffn_weights",
    "moe_combine", "moe_bias_update", "moe_aux_loss_workspace_size", "moe_aux_loss",
    "moe_quantize_blocks", "moe_quantize_rows",
    "moe_read_device_status", "moe_last_cuda_error", "moe_status_string", "moe_abi_version",
    "moe_set_wait_limit_ns", "moe_wait_limit_ns",
]


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        super().__init__(f"{fn} failed: status {status} ({detail})")


class RouteParams(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
                ("scoring", ctypes.c_int32), ("norm_topk_prob", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("dev_status", ctypes.c_void_p)]


class FFNWeights(ctypes.Structure):
    _fields_ = [("w13", ctypes.c_void_p), ("w2", ctypes.c_void_p),
                ("w13_scale", ctypes.c_void_p), ("w2_scale", ctypes.c_void_p),
                ("dtype", ctypes.c_int32), ("groups", ctypes.c_int32), ("I", ctypes.c_int32),
                ("tiled", ctypes.c_int32)]


_LIB = None
_P = ctypes.c_void_p
_I = ctypes.c_int32


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Loads libmoe.so (once). Raises if it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = path or lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"libmoe not built: {path} is missing "
                           "(run python -m mixture_experts_layer_limited_b200.build)")
    lib = ctypes.CDLL(path)
    sig = {
        "moe_route": [ctypes.POINTER(RouteParams), _P, _P, _P, _P, _P, _P, _P, _P],
        "moe_gate_logits": [_I, _I, _I, _P, _P, _P, _P, _P],
        "moe_permute_workspace_size": [_I, _I, _I, ctypes.POINTER(ctypes.c_size_t)],
        "moe_permute": [_I, _I, _I, _I, _P, _P, _P, _I, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P,
                        ctypes.c_size_t, _P, _P],
        "moe_permute_static_ws": [_I, _I, _I, _I, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P],
        "moe_grouped_swiglu": [_I, _I, ctypes.POINTER(FFNWeights), _P, _P, _P, _P, _P, _P, _P, _P, _P],
        "moe_gate_up_swiglu": [_I, _I, ctypes.POINTER(FFNWeights), _P, _P, _P, _P, _P, _P, _P],
        "moe_down_proj": [_I, _I, ctypes.POINTER(FFNWeights), _P, _P, _P, _P, _P, _P, _P],
        "moe_gate_up_swiglu_gather": [_I, _I, ctypes.POINTER(FFNWeights), _P, _I, _P, _P, _P, _P, _P],
        "moe_gate_up_swiglu_with_shared": [_I, _I, ctypes.POINTER(FFNWeights), _P, _P, _P, _P, _P,
                                           _I, ctypes.POINTER(FFNWeights), _P, _P, _P, _P, _P, _P],
        "moe_down_proj_with_shared": [_I, _I, ctypes.POINTER(FFNWeights), _P, _P, _P, _P, _P,
                                      _I, ctypes.POINTER(FFNWeights), _P, _P, _P, _P, _P],
        "moe_swiglu_ffn_sync_size": [_I, _I, _I, ctypes.POINTER(ctypes.c_size_t)],
        "moe_tile_ffn_weights": [_I, ctypes.POINTER(FFNWeights), _P, _P, _P],
        "moe_swiglu_ffn_with_shared": [_I, _I, ctypes.POINTER(FFNWeights), _P, _P, _P, _P, _P,
                                       _I, ctypes.POINTER(FFNWeights), _P, _P, _P, _P, ctypes.c_size_t,
                                       _P, _P],
        "moe_down_proj_combine": [_I, _I, _I, ctypes.POINTER(FFNWeights), _P, _P, _P, _P,
                                  ctypes.POINTER(FFNWeights), _P, _P, _P, _P, _P],
        "moe_combine": [_I, _I, _I, _P, _P, _P, _P, _P, _P],
        "moe_bias_update": [_I, _I, _I, _P, _P, ctypes.c_float, _P, _P],
        "moe_aux_loss_workspace_size": [_I, _I, _I, ctypes.POINTER(ctypes.c_size_t)],
        "moe_aux_loss": [_I, _I, _I, _I, _I, _P, _P, ctypes.c_float, _P, _P, ctypes.c_size_t, _P, _P],
        "moe_quantize_blocks": [_I, _I, _I, _P, _P, _P, _P],
        "moe_quantize_rows": [_I, _I, _P, _P, _P, _P],
        "moe_read_device_status": [_P, ctypes.POINTER(ctypes.c_int32), _P],
        "moe_last_cuda_error": [],
        "moe_status_string": [_I],
        "moe_abi_version": [],
        "moe_set_wait_limit_ns": [ctypes.c_uint64],
        "moe_wait_limit_ns": [],
    }
    restype = {"moe_status_string": ctypes.c_char_p, "moe_wait_limit_ns": ctypes.c_uint64}
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = restype.get(name, ctypes.c_int32)
    _LIB = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmoe takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, status: int):
    if status != MOE_OK:
        lib = load_library()
        detail = lib.moe_status_string(status).decode()
        if status == MOE_ERR_CUDA:
            detail += f", cuda error {lib.moe_last_cuda_error()}"
        raise MoEError(fn, status, detail)


# ---------------------------------------------------------------- the ABI
def moe_route(T, H, E, k, n_group, topk_group, scoring, norm_topk_prob, routed_scaling_factor,
              x, gate_w, sel_bias, logits, topk_ids, topk_w, expert_counts, dev_status=None,
              stream=None):
    p = RouteParams(T, H, E, k, n_group, topk_group, scoring, int(bool(norm_topk_prob)),
                    float(routed_scaling_factor), _ptr(dev_status))
    _check("moe_route", load_library().moe_route(
        ctypes.byref(p), _ptr(x), _ptr(gate_w), _ptr(sel_bias), _ptr(logits), _ptr(topk_ids),
        _ptr(topk_w), _ptr(expert_counts), _stream(stream)))


def moe_gate_logits(T, H, E, x, gate_w, logits, dev_status=None, stream=None):
    _check("moe_gate_logits", load_library().moe_gate_logits(
        T, H, E, _ptr(x), _ptr(gate_w), _ptr(logits), _ptr(dev_status), _stream(stream)))


def moe_permute_workspace_size(T, k, E) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_permute_workspace_size",
           load_library().moe_permute_workspace_size(T, k, E, ctypes.byref(n)))
    return n.value


def moe_permute(T, k, E, H, topk_ids, topk_w, x, x_dtype, x_scale, x_perm, x_perm_scale,
                expert_offsets, src_token, slot_to_row, row_w, workspace, dev_status=None, stream=None,
                perm_dtype=None, x_q=None, x_q_scale=None):
    """perm_dtype defaults to x_dtype (a copy); MOE_E4M3 with bf16 x quantises
    the rows per 1x128 tile on the way (x_q / x_q_scale: the token's own codes)."""
    ws_bytes = workspace.numel() * workspace.element_size()
    pdt = x_dtype if perm_dtype is None else perm_dtype
    _check("moe_permute", load_library().moe_permute(
        T, k, E, H, _ptr(topk_ids), _ptr(topk_w), _ptr(x), x_dtype, _ptr(x_scale), _ptr(x_perm), pdt,
        _ptr(x_perm_scale), _ptr(x_q), _ptr(x_q_scale), _ptr(expert_offsets), _ptr(src_token),
        _ptr(slot_to_row), _ptr(row_w), _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream)))


def moe_grouped_swiglu(rows, H, w13, w2, dtype, groups, I, a, offsets, row_w, h_ws, out,
                       w13_scale=None, w2_scale=None, a_scale=None, h_scale_ws=None,
                       dev_status=None, stream=None, tiled=False):
    w = FFNWeights(_ptr(w13), _ptr(w2), _ptr(w13_scale), _ptr(w2_scale), dtype, groups, I)
    w.tiled = int(tiled)
    _check("moe_grouped_swiglu", load_library().moe_grouped_swiglu(
        rows, H, ctypes.byref(w), _ptr(a), _ptr(a_scale), _ptr(offsets), _ptr(row_w), _ptr(h_ws),
        _ptr(h_scale_ws), _ptr(out), _ptr(dev_status), _stream(stream)))


def moe_gate_up_swiglu(rows, H, w13, dtype, groups, I, a, offsets, h_ws, w13_scale=None,
                       a_scale=None, h_scale_ws=None, dev_status=None, stream=None, tiled=False):
    w = FFNWeights(_ptr(w13), None, _ptr(w13_scale), None, dtype, groups, I)
    w.tiled = int(tiled)
    _check("moe_gate_up_swiglu", load_library().moe_gate_up_swiglu(
        rows, H, ctypes.byref(w), _ptr(a), _ptr(a_scale), _ptr(offsets), _ptr(h_ws),
        _ptr(h_scale_ws), _ptr(dev_status), _stream(stream)))


def moe_gate_up_swiglu_gather(rows, H, w13, groups, I, x, T, src_token, offsets, h_ws,
                              dev_status=None, stream=None, tiled=False):
    w = FFNWeights(_ptr(w13), None, None, None, MOE_BF16, groups, I)
    w.tiled = int(tiled)
    _check("moe_gate_up_swiglu_gather", load_library().moe_gate_up_swiglu_gather(
        rows, H, ctypes.byref(w), _ptr(x), T, _ptr(src_token), _ptr(offsets), _ptr(h_ws),
        _ptr(dev_status), _stream(stream)))


def moe_down_proj(rows, H, w2, dtype, groups, I, h, offsets, row_w, out, w2_scale=None,
                  h_scale=None, dev_status=None, stream=None, tiled=False):
    w = FFNWeights(None, _ptr(w2), None, _ptr(w2_scale), dtype, groups, I)
    w.tiled = int(tiled)
    _check("moe_down_proj", load_library().moe_down_proj(
        rows, H, ctypes.byref(w), _ptr(h), _ptr(h_scale), _ptr(offsets), _ptr(row_w), _ptr(out),
        _ptr(dev_status), _stream(stream)))


def moe_gate_up_swiglu_with_shared(rows, H, w13, dtype, groups, I, a, offsets, h_ws,
                                   sh_rows, sw13, I_s, sh_a, sh_h_ws, w13_scale=None, a_scale=None,
                                   h_scale_ws=None, sw13_scale=None, sh_a_scale=None, sh_h_scale_ws=None,
                                   dev_status=None, stream=None, tiled=False):
    w = FFNWeights(_ptr(w13), None, _ptr(w13_scale), None, dtype, groups, I)
    w.tiled = int(tiled)
    sw = FFNWeights(_ptr(sw13), None, _ptr(sw13_scale), None, dtype, 1, I_s)
    sw.tiled = int(tiled)
    _check("moe_gate_up_swiglu_with_shared", load_library().moe_gate_up_swiglu_with_shared(
        rows, H, ctypes.byref(w), _ptr(a), _ptr(a_scale), _ptr(offsets), _ptr(h_ws), _ptr(h_scale_ws),
        sh_rows, ctypes.byref(sw), _ptr(sh_a), _ptr(sh_a_scale), _ptr(sh_h_ws), _ptr(sh_h_scale_ws),
        _ptr(dev_status), _stream(stream)))


def moe_down_proj_with_shared(rows, H, w2, dtype, groups, I, h, offsets, row_w, out,
                              sh_rows, sw2, I_s, sh_h, sh_out, w2_scale=None, h_scale=None,
                              sw2_scale=None, sh_h_scale=None, dev_status=None, stream=None, tiled=False):
    w = FFNWeights(None, _ptr(w2), None, _ptr(w2_scale), dtype, groups, I)
    w.tiled = int(tiled)
    sw = FFNWeights(None, _ptr(sw2), None, _ptr(sw2_scale), dtype, 1, I_s)
    sw.tiled = int(tiled)
    _check("moe_down_proj_with_shared", load_library().moe_down_proj_with_shared(
        rows, H, ctypes.byref(w), _ptr(h), _ptr(h_scale), _ptr(offsets), _ptr(row_w), _ptr(out),
        sh_rows, ctypes.byref(sw), _ptr(sh_h), _ptr(sh_h_scale), _ptr(sh_out),
        _ptr(dev_status), _stream(stream)))


def moe_swiglu_ffn_sync_size(rows, groups, sh_rows):
    n = ctypes.c_size_t(0)
    _check("moe_swiglu_ffn_sync_size", load_library().moe_swiglu_ffn_sync_size(rows, groups, sh_rows,
                                                                               ctypes.byref(n)))
    return n.value


def moe_swiglu_ffn_with_shared(rows, H, w13, w2, groups, I, a, offsets, row_w, h_ws, out,
                               sh_rows, sw13, sw2, I_s, sh_a, sh_h_ws, sh_out, sync_ws,
                               dev_status=None, stream=None, tiled=False):
    w = FFNWeights(_ptr(w13), _ptr(w2), None, None, MOE_BF16, groups, I)
    w.tiled = int(tiled)
    sw = FFNWeights(_ptr(sw13), _ptr(sw2), None, None, MOE_BF16, 1, I_s)
    sw.tiled = int(tiled)
    _check("moe_swiglu_ffn_with_shared", load_library().moe_swiglu_ffn_with_shared(
        rows, H, ctypes.byref(w), _ptr(a), _ptr(offsets), _ptr(row_w), _ptr(h_ws), _ptr(out),
        sh_rows, ctypes.byref(sw), _ptr(sh_a), _ptr(sh_h_ws), _ptr(sh_out),
        _ptr(sync_ws), sync_ws.numel() * sync_ws.element_size(), _ptr(dev_status), _stream(stream)))


def moe_tile_ffn_weights(H, w13, w2, groups, I, w13_t, w2_t, stream=None):
    """bf16 w13 [groups, 2I, H] / w2 [groups, H, I] -> the tiled copies w13_t /
    w2_t (same sizes; either pair may be None)."""
    for src, dst, n in ((w13, w13_t, groups * 2 * I * H), (w2, w2_t, groups * H * I)):
        if dst is not None and (src.numel() != n or dst.numel() != n):
            raise ValueError(f"moe_tile_ffn_weights: expected {n} elements, got {src.numel()} / {dst.numel()}")
    w = FFNWeights(_ptr(w13), _ptr(w2), None, None, MOE_BF16, groups, I)
    _check("moe_tile_ffn_weights", load_library().moe_tile_ffn_weights(
        H, ctypes.byref(w), _ptr(w13_t), _ptr(w2_t), _stream(stream)))


def moe_down_proj_combine(rows, T, H, w2, groups, I, h, offsets, row_w, src_token, sw2, I_s, sh_h,
                          acc_ws, y, dev_status=None, stream=None, tiled=False):
    w = FFNWeights(None, _ptr(w2), None, None, MOE_BF16, groups, I)
    w.tiled = int(tiled)
    sw = FFNWeights(None, _ptr(sw2), None, None, MOE_BF16, 1, I_s) if sw2 is not None else None
    if sw is not None:
        sw.tiled = int(tiled)
    _check("moe_down_proj_combine", load_library().moe_down_proj_combine(
        rows, T, H, ctypes.byref(w), _ptr(h), _ptr(offsets), _ptr(row_w), _ptr(src_token),
        ctypes.byref(sw) if sw is not None else None, _ptr(sh_h), _ptr(acc_ws), _ptr(y),
        _ptr(dev_status), _stream(stream)))


def moe_combine(T, k, H, expert_out, slot_to_row, topk_w, shared_out, y, stream=None):
    _check("moe_combine", load_library().moe_combine(
        T, k, H, _ptr(expert_out), _ptr(slot_to_row), _ptr(topk_w), _ptr(shared_out), _ptr(y),
        _stream(stream)))


def moe_bias_update(E, T, k, expert_counts, bias, gamma, load_cv=None, stream=None):
    _check("moe_bias_update", load_library().moe_bias_update(
        E, T, k, _ptr(expert_counts), _ptr(bias), float(gamma), _ptr(load_cv), _stream(stream)))


def moe_aux_loss_workspace_size(T, E, seq_len) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_aux_loss_workspace_size",
           load_library().moe_aux_loss_workspace_size(T, E, seq_len, ctypes.byref(n)))
    return n.value


def moe_aux_loss(T, E, k, seq_len, scoring, logits, topk_ids, alpha, aux_out, workspace,
                 dev_status=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("moe_aux_loss", load_library().moe_aux_loss(
        T, E, k, seq_len, scoring, _ptr(logits), _ptr(topk_ids), float(alpha), _ptr(aux_out),
        _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream)))


def moe_quantize_blocks(batch, N, K, w, q, scale, stream=None):
    _check("moe_quantize_blocks", load_library().moe_quantize_blocks(
        batch, N, K, _ptr(w), _ptr(q), _ptr(scale), _stream(stream)))


def moe_quantize_rows(M, K, a, q, scale, stream=None):
    _check("moe_quantize_rows", load_library().moe_quantize_rows(
        M, K, _ptr(a), _ptr(q), _ptr(scale), _stream(stream)))


def moe_read_device_status(dev_status, stream=None) -> int:
    """Synchronises the stream and returns the raw device status word."""
    out = ctypes.c_int32(0)
    st = load_library().moe_read_device_status(_ptr(dev_status), ctypes.byref(out), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_DEVICE_CHECK, MOE_ERR_DEVICE_TIMEOUT):
        _check("moe_read_device_status", st)
    return out.value


def moe_set_wait_limit_ns(ns: int):
    """Limit of every bounded device-side wait for later launches (0: the
    default, 2 s). A debugging knob; process-wide."""
    _check("moe_set_wait_limit_ns", load_library().moe_set_wait_limit_ns(int(ns)))


def moe_wait_limit_ns() -> int:
    return int(load_library().moe_wait_limit_ns())
