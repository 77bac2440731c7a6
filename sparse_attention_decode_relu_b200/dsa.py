"""Thin Python binding of libdsa.so (C ABI in include/dsa_decode.h).

The functions carry the C names and do argument marshalling only: torch
tensors become ``dsa_tensor_t`` descriptors, the current CUDA stream is passed
through, and a non-OK status raises ``DsaError``.  Every step of the path runs
in the CUDA library; there is no other implementation to fall back to, and a
missing library is an error.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import numpy as np
import torch

from . import build as _build

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE = 0, 1, 2, 3, 4
BF16, FP8_E4M3, F32, I32 = 0, 1, 2, 3
WS_CTRL_BYTES = 263168   # DSA_WS_CTRL_BYTES: leading workspace bytes that must be zero before first use
WS_WORDS_ZERO_AFTER_CALL = [0, 32] + list(range(96, 104)) + list(range(128, 136)) + list(range(160, 168)) + [192]   # int32 words a call leaves at 0

_lock = threading.Lock()
_lib = None


class DsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"dsa status {status}: {message}")
        self.status = status


class dsa_tensor_t(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4), ("scale", ctypes.c_void_p)]


def library_path() -> str:
    return _build.LIB


def lib():
    """Load libdsa.so (building it in-tree first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            if _build.stale():
                _build.build()
            if not os.path.exists(_build.LIB):
                raise RuntimeError("libdsa.so is missing and could not be built")
            L = ctypes.CDLL(_build.LIB)
            P, T = ctypes.c_void_p, ctypes.POINTER(dsa_tensor_t)
            st = ctypes.c_int32
            L.dsa_workspace_bytes.restype = ctypes.c_size_t
            L.dsa_workspace_bytes.argtypes = [ctypes.c_int32, ctypes.c_int64, ctypes.c_int32]
            L.dsa_decode.restype = st
            L.dsa_decode.argtypes = [T, T, T, T, T, P, ctypes.c_int32, T, T, P]
            L.dsa_decode_ws.restype = st
            L.dsa_decode_ws.argtypes = [T, T, T, T, T, P, ctypes.c_int32, T, T, P, P, ctypes.c_size_t]
            L.dsa_decode_sink_ws.restype = st
            L.dsa_decode_sink_ws.argtypes = [T, T, T, T, T, P, ctypes.c_int32, P, T, T, P, P, ctypes.c_size_t]
            L.dsa_decode_devpos_ws.restype = st
            L.dsa_decode_devpos_ws.argtypes = [T, T, T, T, T, P, ctypes.c_int32, P, T, T, P, P, ctypes.c_size_t]
            L.dsa_set_short_context_bypass.restype = None
            L.dsa_set_short_context_bypass.argtypes = [ctypes.c_int32]
            L.dsa_swa_decode.restype = st
            L.dsa_swa_decode.argtypes = [T, T, P, ctypes.c_int32, P, T, P, P, ctypes.c_size_t]
            L.dsa_index_scores.restype = st
            L.dsa_index_scores.argtypes = [T, T, T, P, P, ctypes.c_int64, P]
            L.dsa_topk_from_scores.restype = st
            L.dsa_topk_from_scores.argtypes = [P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int32,
                                               P, ctypes.c_int64, P, P, ctypes.c_size_t]
            L.dsa_topk_from_scores_noalloc.restype = st
            L.dsa_topk_from_scores_noalloc.argtypes = [P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, P,
                                                       ctypes.c_int32, P, ctypes.c_int64, P]
            L.dsa_sparse_attn.restype = st
            L.dsa_sparse_attn.argtypes = [T, T, T, P, P, T, P, P, ctypes.c_size_t]
            L.dsa_device_status.restype = st
            L.dsa_device_status.argtypes = [P]
            L.dsa_status_str.restype = ctypes.c_char_p
            L.dsa_status_str.argtypes = [st]
            L.dsa_last_error.restype = ctypes.c_char_p
            L.dsa_launch_count.restype = ctypes.c_uint64
            L.dsa_debug_fail_next_barriers.restype = st
            L.dsa_debug_fail_next_barriers.argtypes = [ctypes.c_int64]
            L.dsa_set_step_trace.restype = None
            L.dsa_set_step_trace.argtypes = [P]
            L.dsa_step_grid.restype = ctypes.c_int32
            L.dsa_step_grid.argtypes = [ctypes.c_int32]
            L.dsa_set_stage_events.restype = None
            L.dsa_set_stage_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]
            _lib = L
    return _lib


_DTYPES = {torch.bfloat16: BF16, torch.float8_e4m3fn: FP8_E4M3, torch.uint8: FP8_E4M3, torch.float32: F32,
           torch.int32: I32}


def _desc(t: torch.Tensor, scale: Optional[torch.Tensor] = None) -> dsa_tensor_t:
    if t is None:
        raise ValueError("tensor argument is None")
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if t.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {t.dtype}")
    if t.dim() > 4:
        raise ValueError("at most 4 dimensions")
    d = dsa_tensor_t()
    d.data = t.data_ptr()
    d.dtype = _DTYPES[t.dtype]
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    if scale is not None:
        if not scale.is_cuda or scale.dtype != torch.float32 or not scale.is_contiguous():
            raise ValueError("k_scale must be a contiguous float32 CUDA tensor")
        d.scale = scale.data_ptr()
    return d


def _pos(pos) -> ctypes.Array:
    a = np.ascontiguousarray(torch.as_tensor(pos).cpu().numpy() if isinstance(pos, torch.Tensor) else pos,
                             dtype=np.int32).reshape(-1)
    return (ctypes.c_int32 * len(a))(*a.tolist())


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int):
    if status != OK:
        L = lib()
        raise DsaError(status, (L.dsa_last_error() or b"").decode() or L.dsa_status_str(status).decode())


def dsa_workspace_bytes(T: int, L: int, topk: int) -> int:
    return int(lib().dsa_workspace_bytes(T, L, topk))


def dsa_decode(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, out, sel_idx, stream=None, *, k_scale=None):
    a = [_desc(q), _desc(q_idx), _desc(w_idx), _desc(k_idx_cache, k_scale), _desc(kv_cache)]
    o = [_desc(out), _desc(sel_idx)]
    _check(lib().dsa_decode(*[ctypes.byref(x) for x in a], _pos(pos), int(topk), ctypes.byref(o[0]),
                            ctypes.byref(o[1]), _stream(stream)))


def _sink_ptr(sink):
    if sink is None:
        return None
    if not sink.is_cuda or sink.dtype != torch.float32 or sink.numel() != 64 or not sink.is_contiguous():
        raise ValueError("sink must be a contiguous float32 CUDA tensor of 64 logits")
    return sink.data_ptr()


def dsa_decode_ws(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, out, sel_idx, workspace, stream=None, *,
                  k_scale=None, sink=None):
    """dsa_decode_ws, or dsa_decode_sink_ws when a sink is given."""
    a = [_desc(q), _desc(q_idx), _desc(w_idx), _desc(k_idx_cache, k_scale), _desc(kv_cache)]
    o = [_desc(out), _desc(sel_idx)]
    ws = (workspace.data_ptr(), workspace.numel() * workspace.element_size())
    if sink is None:
        _check(lib().dsa_decode_ws(*[ctypes.byref(x) for x in a], _pos(pos), int(topk), ctypes.byref(o[0]),
                                   ctypes.byref(o[1]), _stream(stream), *ws))
    else:
        _check(lib().dsa_decode_sink_ws(*[ctypes.byref(x) for x in a], _pos(pos), int(topk), _sink_ptr(sink),
                                        ctypes.byref(o[0]), ctypes.byref(o[1]), _stream(stream), *ws))


def dsa_decode_sink_ws(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, sink, out, sel_idx, workspace,
                       stream=None, *, k_scale=None):
    dsa_decode_ws(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, out, sel_idx, workspace, stream,
                  k_scale=k_scale, sink=sink)


def dsa_decode_devpos_ws(q, q_idx, w_idx, k_idx_cache, kv_cache, pos_device, topk, out, sel_idx, workspace,
                         stream=None, *, k_scale=None, sink=None):
    """The step with query positions read from pos_device (int32 CUDA tensor [T]) at launch."""
    if not pos_device.is_cuda or pos_device.dtype != torch.int32 or pos_device.numel() != q.shape[0]:
        raise ValueError("pos_device must be an int32 CUDA tensor with one position per query")
    a = [_desc(q), _desc(q_idx), _desc(w_idx), _desc(k_idx_cache, k_scale), _desc(kv_cache)]
    o = [_desc(out), _desc(sel_idx)]
    _check(lib().dsa_decode_devpos_ws(*[ctypes.byref(x) for x in a], pos_device.data_ptr(), int(topk),
                                      _sink_ptr(sink), ctypes.byref(o[0]), ctypes.byref(o[1]), _stream(stream),
                                      workspace.data_ptr(), workspace.numel() * workspace.element_size()))


def dsa_set_short_context_bypass(enable: bool):
    lib().dsa_set_short_context_bypass(1 if enable else 0)


def dsa_swa_decode(q, kv_cache, pos, window, out, workspace, stream=None, *, sink=None):
    _check(lib().dsa_swa_decode(ctypes.byref(_desc(q)), ctypes.byref(_desc(kv_cache)), _pos(pos), int(window),
                                _sink_ptr(sink), ctypes.byref(_desc(out)), _stream(stream), workspace.data_ptr(),
                                workspace.numel() * workspace.element_size()))


def dsa_index_scores(q_idx, w_idx, k_idx_cache, pos, scores, stream=None, *, k_scale=None):
    a = [_desc(q_idx), _desc(w_idx), _desc(k_idx_cache, k_scale)]
    if scores.dtype != torch.float32 or scores.dim() != 2 or scores.stride(1) != 1:
        raise ValueError("scores must be float32 [T][ld] with unit inner stride")
    _check(lib().dsa_index_scores(*[ctypes.byref(x) for x in a], _pos(pos), scores.data_ptr(), scores.stride(0),
                                  _stream(stream)))


def dsa_topk_from_scores(scores, L, pos, topk, sel_idx, workspace, stream=None):
    if scores.dtype != torch.float32 or scores.dim() != 2 or scores.stride(1) != 1:
        raise ValueError("scores must be float32 [T][ld] with unit inner stride")
    if sel_idx.dtype != torch.int32 or sel_idx.stride(1) != 1:
        raise ValueError("sel_idx must be int32 [T][>= topk] with unit inner stride")
    _check(lib().dsa_topk_from_scores(scores.data_ptr(), scores.shape[0], int(L), scores.stride(0), _pos(pos),
                                      int(topk), sel_idx.data_ptr(), sel_idx.stride(0), _stream(stream),
                                      workspace.data_ptr(), workspace.numel() * workspace.element_size()))


def dsa_topk_from_scores_noalloc(scores, L, pos, topk, sel_idx, stream=None):
    """dsa_topk_from_scores with the library's static scratch instead of a
    workspace (T <= 8, L <= 262144; concurrent calls on the GPU race)."""
    if scores.dtype != torch.float32 or scores.dim() != 2 or scores.stride(1) != 1:
        raise ValueError("scores must be float32 [T][ld] with unit inner stride")
    if sel_idx.dtype != torch.int32 or sel_idx.stride(1) != 1:
        raise ValueError("sel_idx must be int32 [T][>= topk] with unit inner stride")
    _check(lib().dsa_topk_from_scores_noalloc(scores.data_ptr(), scores.shape[0], int(L), scores.stride(0),
                                              _pos(pos), int(topk), sel_idx.data_ptr(), sel_idx.stride(0),
                                              _stream(stream)))


def dsa_sparse_attn(q, kv_cache, sel_idx, pos, out, workspace, stream=None, *, sink=None):
    d = [_desc(q), _desc(kv_cache), _desc(sel_idx)]
    o = _desc(out)
    _check(lib().dsa_sparse_attn(*[ctypes.byref(x) for x in d], _pos(pos), _sink_ptr(sink), ctypes.byref(o),
                                 _stream(stream),
                                 workspace.data_ptr(), workspace.numel() * workspace.element_size()))


def dsa_device_status(stream=None):
    _check(lib().dsa_device_status(_stream(stream)))


def dsa_debug_fail_next_barriers(limit_cycles: int):
    """Test hook: the next step launch from this thread waits at every grid
    barrier for a block that never comes, giving up after limit_cycles."""
    _check(lib().dsa_debug_fail_next_barriers(int(limit_cycles)))


def dsa_launch_count() -> int:
    return int(lib().dsa_launch_count())


def dsa_set_step_trace(buf: Optional[torch.Tensor]):
    """Record per-block phase-boundary timestamps into buf (int64 CUDA tensor of
    dsa_step_grid(...) * 32 entries) on the following calls; None disables."""
    lib().dsa_set_step_trace(None if buf is None else buf.data_ptr())


def dsa_step_grid(fp8_keys: bool = False) -> int:
    return int(lib().dsa_step_grid(1 if fp8_keys else 0))


def dsa_set_stage_events(events: Optional[Sequence[torch.cuda.Event]]):
    if not events:
        lib().dsa_set_stage_events(None, 0)
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    lib().dsa_set_stage_events(arr, len(events))


# ------------------------------------------------------------------ conveniences
def workspace(T: int, L: int, topk: int, device=None) -> torch.Tensor:
    n = dsa_workspace_bytes(T, L, topk)
    if n == 0:
        raise DsaError(ERR_INVALID_ARG, "invalid sizes for a workspace")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    ws[:WS_CTRL_BYTES].zero_()   # the control region starts at zero; every call leaves it ready for the next
    return ws


def decode(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk=2048, *, k_scale=None, ws=None, stream=None):
    """Allocate out / sel_idx (and a workspace unless given) and run the step."""
    T = q.shape[0]
    out = torch.empty((T, 64, 128), dtype=torch.bfloat16, device=q.device)
    sel = torch.empty((T, topk), dtype=torch.int32, device=q.device)
    if ws is None:
        dsa_decode(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, out, sel, stream, k_scale=k_scale)
    else:
        dsa_decode_ws(q, q_idx, w_idx, k_idx_cache, kv_cache, pos, topk, out, sel, ws, stream, k_scale=k_scale)
    return out, sel


def to_device(w, device="cuda", with_kv=True):
    """Move a synthetic workload's numpy arrays to the device as the library expects them."""
    def bits(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dt).to(device)

    d = {
        "q": bits(w.q, torch.bfloat16),
        "q_idx": bits(w.q_idx, torch.bfloat16),
        "w_idx": torch.from_numpy(w.w_idx).to(device),
        "kv": bits(w.kv, torch.bfloat16) if with_kv else None,
        "pos": w.pos.copy(),
    }
    if w.key_dtype == "bf16":
        d["k_idx"] = bits(w.k_idx, torch.bfloat16)
    else:
        d["k_idx"] = torch.from_numpy(np.ascontiguousarray(w.k_idx)).view(torch.float8_e4m3fn).to(device)
    d["k_scale"] = None if w.k_scale is None else torch.from_numpy(w.k_scale).to(device)
    return d
