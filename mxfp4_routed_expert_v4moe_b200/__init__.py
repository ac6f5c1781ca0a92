"""Python binding of libv4moe (routed MoE FFN layer of DeepSeek-V4-Flash, B200).

Argument marshalling only: every step of the layer runs in the CUDA kernels
of ``libv4moe.so`` (built in-tree by ``build.py``). The functions keep the C
names and argument order of ``include/v4moe.h``; pointer arguments accept a
torch tensor (its ``data_ptr()``), an int address or None, and ``stream``
defaults to the current torch CUDA stream. Each returns the C status code;
``check`` turns a non-zero code into a ``V4moeError``.

There is no CPU fallback: if the library is missing, loading it raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libv4moe.so")

V4MOE_OK = 0
V4MOE_ERR_INVALID_ARG = 1
V4MOE_ERR_WORKSPACE = 2
V4MOE_ERR_UNSUPPORTED_DEVICE = 3
V4MOE_ERR_LAUNCH = 4
V4MOE_ERR_DATA = 5
V4MOE_ERR_TIMEOUT = 6

EXPORTED = ("v4moe_workspace_bytes", "v4moe_route", "v4moe_permute", "v4moe_forward",
            "v4moe_read_device_status", "v4moe_clear_device_status", "v4moe_status_string",
            "v4moe_profile_enable", "v4moe_profile_reset", "v4moe_profile_read",
            "v4moe_launch_count", "v4moe_permute_static", "v4moe_layer",
            "v4moe_linear_w8a16_workspace_bytes", "v4moe_linear_w8a16",
            "v4moe_linear_w8a16_grouped_workspace_bytes", "v4moe_linear_w8a16_grouped")


class V4moeError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


class v4moe_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("shared_inter", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("routed_scale", ctypes.c_float), ("swiglu_limit", ctypes.c_float)]


class v4moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w13_codes", "w13_scales", "w2_codes", "w2_scales",
                                               "sh_w13", "sh_w13_scale", "sh_w2", "sh_w2_scale")]


_lib = None
_lock = threading.Lock()


def load(path: str | None = None):
    """Load libv4moe.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            p = path or LIB_PATH
            if not os.path.exists(p):
                raise RuntimeError(f"{p} is missing: build it with "
                                   "`python -m mxfp4_routed_expert_v4moe_b200.build`")
            L = ctypes.CDLL(p)
            P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
            cfgp = ctypes.POINTER(v4moe_config)
            L.v4moe_workspace_bytes.argtypes = [cfgp, i32]
            L.v4moe_workspace_bytes.restype = sz
            L.v4moe_route.argtypes = [cfgp, i32, P, P, P, P, P, P, P, P, sz, P]
            L.v4moe_route.restype = i32
            L.v4moe_permute.argtypes = [cfgp, i32, P, P, P, P, P, P, sz, P]
            L.v4moe_permute.restype = i32
            L.v4moe_permute_static.argtypes = [cfgp, i32, P, P, P, P, P, P]
            L.v4moe_permute_static.restype = i32
            L.v4moe_forward.argtypes = [cfgp, i32, P, P, P, P, P, P, ctypes.POINTER(v4moe_weights),
                                        P, P, sz, P]
            L.v4moe_forward.restype = i32
            L.v4moe_layer.argtypes = [cfgp, i32, P, P, P, P, P, ctypes.POINTER(v4moe_weights), P, P, P, P,
                                      P, P, P, P, sz, P]
            L.v4moe_layer.restype = i32
            L.v4moe_linear_w8a16_workspace_bytes.argtypes = [i32, i32, i32]
            L.v4moe_linear_w8a16_workspace_bytes.restype = sz
            L.v4moe_linear_w8a16.argtypes = [i32, i32, i32, P, P, P, P, P, sz, P]
            L.v4moe_linear_w8a16.restype = i32
            L.v4moe_linear_w8a16_grouped_workspace_bytes.argtypes = [i32, i32, i32, i32]
            L.v4moe_linear_w8a16_grouped_workspace_bytes.restype = sz
            L.v4moe_linear_w8a16_grouped.argtypes = [i32, i32, i32, i32, P, P, P, P, P, sz, P]
            L.v4moe_linear_w8a16_grouped.restype = i32
            L.v4moe_read_device_status.argtypes = [P, P]
            L.v4moe_read_device_status.restype = i32
            L.v4moe_clear_device_status.argtypes = [P, P]
            L.v4moe_clear_device_status.restype = i32
            L.v4moe_status_string.argtypes = [i32]
            L.v4moe_status_string.restype = ctypes.c_char_p
            L.v4moe_profile_enable.argtypes = [i32]
            L.v4moe_profile_enable.restype = i32
            L.v4moe_profile_reset.argtypes = []
            L.v4moe_profile_reset.restype = i32
            L.v4moe_profile_read.argtypes = [ctypes.c_char_p, i32, P, P, i32, P]
            L.v4moe_profile_read.restype = i32
            L.v4moe_launch_count.argtypes = []
            L.v4moe_launch_count.restype = ctypes.c_uint64
            _lib = L
    return _lib


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def make_config(H, I, E, k, Is, vocab=129280, routed_scale=1.5, swiglu_limit=10.0) -> v4moe_config:
    return v4moe_config(H, I, E, k, Is, vocab, routed_scale, swiglu_limit)


def make_weights(w13_codes, w13_scales, w2_codes, w2_scales, sh_w13=None, sh_w13_scale=None,
                 sh_w2=None, sh_w2_scale=None) -> v4moe_weights:
    return v4moe_weights(*[_ptr(t) for t in (w13_codes, w13_scales, w2_codes, w2_scales, sh_w13,
                                             sh_w13_scale, sh_w2, sh_w2_scale)])


def status_string(code: int) -> str:
    return load().v4moe_status_string(code).decode()


def check(code: int, where: str = "v4moe"):
    if code != V4MOE_OK:
        raise V4moeError(code, where)
    return code


# ---- same names as the C ABI -------------------------------------------------

def v4moe_workspace_bytes(cfg: v4moe_config, T: int) -> int:
    return load().v4moe_workspace_bytes(ctypes.byref(cfg), T)


def v4moe_route(cfg, T, x, gate, bias, token_ids, tid2eid, topk_ids, topk_w, ws, ws_bytes,
                stream=None) -> int:
    return load().v4moe_route(ctypes.byref(cfg), T, _ptr(x), _ptr(gate), _ptr(bias), _ptr(token_ids),
                              _ptr(tid2eid), _ptr(topk_ids), _ptr(topk_w), _ptr(ws), ws_bytes,
                              _stream(stream))


def v4moe_permute(cfg, T, topk_ids, counts, offsets, sorted_slot, slot_pos, ws, ws_bytes,
                  stream=None) -> int:
    return load().v4moe_permute(ctypes.byref(cfg), T, _ptr(topk_ids), _ptr(counts), _ptr(offsets),
                                _ptr(sorted_slot), _ptr(slot_pos), _ptr(ws), ws_bytes,
                                _stream(stream))


def v4moe_permute_static(cfg, T, topk_ids, counts, offsets, sorted_slot, slot_pos,
                         stream=None) -> int:
    """v4moe_permute for callers that cannot allocate: no workspace argument;
    scratch lives in a fixed array inside the library (see include/v4moe.h)."""
    return load().v4moe_permute_static(ctypes.byref(cfg), T, _ptr(topk_ids), _ptr(counts),
                                       _ptr(offsets), _ptr(sorted_slot), _ptr(slot_pos),
                                       _stream(stream))


def v4moe_forward(cfg, T, x, topk_ids, topk_w, offsets, sorted_slot, slot_pos, weights, out, ws,
                  ws_bytes, stream=None) -> int:
    return load().v4moe_forward(ctypes.byref(cfg), T, _ptr(x), _ptr(topk_ids), _ptr(topk_w),
                                _ptr(offsets), _ptr(sorted_slot), _ptr(slot_pos),
                                ctypes.byref(weights), _ptr(out), _ptr(ws), ws_bytes,
                                _stream(stream))


def v4moe_layer(cfg, T, x, gate, bias, token_ids, tid2eid, weights, topk_ids, topk_w, counts,
                offsets, sorted_slot, slot_pos, out, ws, ws_bytes, stream=None) -> int:
    return load().v4moe_layer(ctypes.byref(cfg), T, _ptr(x), _ptr(gate), _ptr(bias), _ptr(token_ids),
                              _ptr(tid2eid), ctypes.byref(weights), _ptr(topk_ids), _ptr(topk_w),
                              _ptr(counts), _ptr(offsets), _ptr(sorted_slot), _ptr(slot_pos),
                              _ptr(out), _ptr(ws), ws_bytes, _stream(stream))


def v4moe_linear_w8a16_workspace_bytes(T: int, N: int, K: int) -> int:
    return load().v4moe_linear_w8a16_workspace_bytes(T, N, K)


def v4moe_linear_w8a16(T, N, K, x, q, scale, out, ws, ws_bytes, stream=None) -> int:
    return load().v4moe_linear_w8a16(T, N, K, _ptr(x), _ptr(q), _ptr(scale), _ptr(out), _ptr(ws), ws_bytes,
                                     _stream(stream))


def v4moe_linear_w8a16_grouped_workspace_bytes(T: int, G: int, N: int, K: int) -> int:
    return load().v4moe_linear_w8a16_grouped_workspace_bytes(T, G, N, K)


def v4moe_linear_w8a16_grouped(T, G, N, K, x, q, scale, out, ws, ws_bytes, stream=None) -> int:
    return load().v4moe_linear_w8a16_grouped(T, G, N, K, _ptr(x), _ptr(q), _ptr(scale), _ptr(out), _ptr(ws),
                                             ws_bytes, _stream(stream))


def v4moe_read_device_status(ws, stream=None) -> int:
    return load().v4moe_read_device_status(_ptr(ws), _stream(stream))


def v4moe_clear_device_status(ws, stream=None) -> int:
    return load().v4moe_clear_device_status(_ptr(ws), _stream(stream))


def v4moe_status_string(code: int) -> str:
    return status_string(code)


def v4moe_profile_enable(on: bool) -> int:
    return load().v4moe_profile_enable(1 if on else 0)


def v4moe_profile_reset() -> int:
    return load().v4moe_profile_reset()


def v4moe_profile_read(max_entries: int = 64, name_len: int = 64):
    """-> {kernel name: (total_ms, launches)} for the launches timed since the last reset."""
    names = ctypes.create_string_buffer(max_entries * name_len)
    ms = (ctypes.c_float * max_entries)()
    cnt = (ctypes.c_int32 * max_entries)()
    n = ctypes.c_int32(0)
    check(load().v4moe_profile_read(names, name_len, ctypes.addressof(ms), ctypes.addressof(cnt),
                                    max_entries, ctypes.addressof(n)), "v4moe_profile_read")
    out = {}
    for i in range(min(n.value, max_entries)):
        nm = names.raw[i * name_len:(i + 1) * name_len].split(b"\0", 1)[0].decode()
        out[nm] = (float(ms[i]), int(cnt[i]))
    return out


def v4moe_launch_count() -> int:
    return int(load().v4moe_launch_count())


from .layer import MoELayer  # noqa: E402  (convenience wrapper over the calls above)
