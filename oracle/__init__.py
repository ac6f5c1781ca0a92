"""CPU oracle of the routed MoE FFN layer (fp64, single-threaded C++).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers. The CUDA library never
imports or links this package, and this package never imports the CUDA one.

``v4moe_oracle.cpp`` holds the arithmetic and the citations of the passages
each function follows. This module only marshals numpy arrays into it. The
helpers that evaluate many tokens split the token list over Python threads:
each thread runs the unchanged single-threaded oracle on its share (ctypes
releases the GIL), which changes nothing in what is computed.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "v4moe_oracle.cpp")
_LIB = os.path.join(_HERE, "libv4moe_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile libv4moe_oracle.so in-tree (g++ -O2, no fast-math) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off", "-Wno-free-nonheap-object",
                               _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


class OrcLayer(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("I", ctypes.c_int32), ("Is", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("pad_", ctypes.c_int32),
                ("routed_scale", ctypes.c_double), ("swiglu_limit", ctypes.c_double),
                ("x", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("token_ids", ctypes.c_void_p), ("tid2eid", ctypes.c_void_p),
                ("w13_codes", ctypes.c_void_p), ("w13_scales", ctypes.c_void_p),
                ("w2_codes", ctypes.c_void_p), ("w2_scales", ctypes.c_void_p),
                ("sh13", ctypes.c_void_p), ("sh13_scale", ctypes.c_void_p),
                ("sh2", ctypes.c_void_p), ("sh2_scale", ctypes.c_void_p)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            P, i32, d = ctypes.c_void_p, ctypes.c_int32, ctypes.c_double
            L.orc_linear_w8a16.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
            L.orc_linear_w8a16.restype = None
            L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
            L.orc_bf16_to_double.restype = d
            L.orc_e2m1.argtypes = [ctypes.c_int]
            L.orc_e2m1.restype = d
            L.orc_e8m0.argtypes = [ctypes.c_int]
            L.orc_e8m0.restype = d
            L.orc_mxfp4_at.argtypes = [P, P, ctypes.c_int64]
            L.orc_mxfp4_at.restype = d
            L.orc_sqrt_softplus.argtypes = [d]
            L.orc_sqrt_softplus.restype = d
            L.orc_silu.argtypes = [d]
            L.orc_silu.restype = d
            L.orc_clamped_swiglu.argtypes = [d, d, d]
            L.orc_clamped_swiglu.restype = d
            L.orc_route.argtypes = [ctypes.POINTER(OrcLayer), P, P, P, P]
            L.orc_route.restype = ctypes.c_int
            L.orc_permute.argtypes = [i32, i32, i32, P, P, P, P, P]
            L.orc_permute.restype = ctypes.c_int
            L.orc_moe_tokens.argtypes = [ctypes.POINTER(OrcLayer), i32, P, P, P, P, P, P]
            L.orc_moe_tokens.restype = ctypes.c_int
            L.orc_moe_dense.argtypes = [ctypes.POINTER(OrcLayer), P, P, P]
            L.orc_moe_dense.restype = ctypes.c_int
            _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "arrays passed to the oracle must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


# scalar helpers ---------------------------------------------------------------

def e2m1(code: int) -> float:
    return lib().orc_e2m1(code)


def e8m0(e: int) -> float:
    return lib().orc_e8m0(e)


def bf16_to_double(b: int) -> float:
    return lib().orc_bf16_to_double(b)


def mxfp4_at(codes_row: np.ndarray, scales_row: np.ndarray, k: int) -> float:
    return lib().orc_mxfp4_at(_p(codes_row), _p(scales_row), k)


def sqrt_softplus(z: float) -> float:
    return lib().orc_sqrt_softplus(z)


def silu(v: float) -> float:
    return lib().orc_silu(v)


def clamped_swiglu(g: float, u: float, limit: float = 10.0) -> float:
    return lib().orc_clamped_swiglu(g, u, limit)


# layer-level ------------------------------------------------------------------

class Layer:
    """Holds references to numpy inputs and the ctypes struct pointing at them."""

    def __init__(self, li):
        wl = li.wl
        self.li = li
        self._keep = [li.x, li.gate, li.bias, li.token_ids, li.tid2eid, li.w13_codes,
                      li.w13_scales, li.w2_codes, li.w2_scales, li.sh13, li.sh13_scale, li.sh2,
                      li.sh2_scale]
        s = OrcLayer()
        s.T, s.H, s.E, s.k, s.I, s.Is = wl.T, wl.H, wl.E, wl.k, wl.I, wl.Is
        s.vocab = wl.vocab if li.tid2eid is None else li.tid2eid.shape[0]
        s.routed_scale, s.swiglu_limit = wl.routed_scale, wl.swiglu_limit
        for name in ("x", "gate", "bias", "token_ids", "tid2eid", "w13_codes", "w13_scales",
                     "w2_codes", "w2_scales", "sh13", "sh13_scale", "sh2", "sh2_scale"):
            setattr(s, name, _p(getattr(li, name)))
        if li.bias is not None and li.token_ids is not None:
            raise ValueError("give either a bias (learned routing) or token ids (hash routing)")
        self.s = s

    def route(self, want_scores: bool = False):
        """-> ids [T,k] int32, w [T,k] float64, margin [T] float64, scores [T,E] or None."""
        T, k, E = self.s.T, self.s.k, self.s.E
        ids = np.zeros((T, k), np.int32)
        w = np.zeros((T, k), np.float64)
        margin = np.zeros(T, np.float64)
        scores = np.zeros((T, E), np.float64) if want_scores else None
        rc = lib().orc_route(ctypes.byref(self.s), _p(ids), _p(w), _p(margin), _p(scores))
        if rc:
            raise ValueError("out-of-range token id or tid2eid entry")
        return ids, w, margin, scores

    def moe_tokens(self, tokens, ids, w, threads: int = 1, want_h: bool = False):
        """Layer output (fp64) for the listed tokens, given routing ids/w for all T tokens."""
        tokens = np.ascontiguousarray(tokens, np.int32)
        ids = np.ascontiguousarray(ids, np.int32)
        w = np.ascontiguousarray(w, np.float64)
        n, H, k, I, Is = len(tokens), self.s.H, self.s.k, self.s.I, self.s.Is
        out = np.zeros((n, H), np.float64)
        h = np.zeros((n, k, I), np.float64) if want_h else None
        hs = np.zeros((n, max(Is, 1)), np.float64) if want_h else None

        def run(a, b):
            rc = lib().orc_moe_tokens(
                ctypes.byref(self.s), b - a, _p(tokens[a:b]), _p(ids), _p(w),
                ctypes.c_void_p(out.ctypes.data + a * H * 8),
                None if h is None else ctypes.c_void_p(h.ctypes.data + a * k * I * 8),
                None if hs is None else ctypes.c_void_p(hs.ctypes.data + a * hs.shape[1] * 8))
            if rc:
                raise ValueError("out-of-range token or expert id")

        threads = max(1, min(threads, n))
        if threads == 1:
            run(0, n)
        else:
            bounds = [int(b) for b in np.linspace(0, n, threads + 1).round()]
            with ThreadPoolExecutor(threads) as ex:
                list(ex.map(lambda i: run(bounds[i], bounds[i + 1]), range(threads)))
        if want_h:
            return out, h, hs
        return out

    def moe_dense(self, ids, w):
        ids = np.ascontiguousarray(ids, np.int32)
        w = np.ascontiguousarray(w, np.float64)
        out = np.zeros((self.s.T, self.s.H), np.float64)
        rc = lib().orc_moe_dense(ctypes.byref(self.s), _p(ids), _p(w), _p(out))
        if rc:
            raise ValueError("out-of-range expert id")
        return out


def permute(ids: np.ndarray, E: int):
    """-> counts [E], offsets [E+1], sorted_slot [T*k], slot_pos [T*k] (int32)."""
    ids = np.ascontiguousarray(ids, np.int32)
    T, k = ids.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    sorted_slot = np.zeros(T * k, np.int32)
    slot_pos = np.zeros(T * k, np.int32)
    rc = lib().orc_permute(T, k, E, _p(ids), _p(counts), _p(offsets), _p(sorted_slot), _p(slot_pos))
    if rc:
        raise ValueError("out-of-range expert id")
    return counts, offsets, sorted_slot, slot_pos


def linear_w8a16(x_bf16: np.ndarray, q: np.ndarray, scale: np.ndarray, rows=None) -> np.ndarray:
    """W8A16 linear (config group linears_w8a16): out[t, n] = sum_k x[t, k] q[n, k]
    scale[n] in fp64. x_bf16: [T, K] uint16 bf16 bit patterns; q: [N, K] int8;
    scale: [N] fp32. rows: optional token subset (the rows of out returned)."""
    x = np.ascontiguousarray(x_bf16 if rows is None else x_bf16[np.asarray(rows)], np.uint16)
    q = np.ascontiguousarray(q, np.int8)
    scale = np.ascontiguousarray(scale, np.float32)
    T, K = x.shape
    N = q.shape[0]
    out = np.zeros((T, N), np.float64)
    lib().orc_linear_w8a16(T, N, K, _p(x), _p(q), _p(scale), _p(out))
    return out


def linear_w8a16_grouped(x_bf16: np.ndarray, q: np.ndarray, scale: np.ndarray, G: int, rows=None) -> np.ndarray:
    """The W8A16 linear in G independent groups (the config's wo_a: o_groups
    groups of heads, each with its own block of rows of one int8 matrix):
    out[t, g N + n] = sum_k x[t, g K + k] q[g N + n, k] scale[g N + n].
    x_bf16: [T, G K]; q: [G N, K]; scale: [G N]. Each group is the plain linear
    on its slice of columns and rows."""
    T, GK = x_bf16.shape
    GN, K = q.shape
    assert GK == G * K and GN % G == 0
    N = GN // G
    parts = [linear_w8a16(x_bf16[:, g * K:(g + 1) * K], q[g * N:(g + 1) * N], scale[g * N:(g + 1) * N], rows=rows)
             for g in range(G)]
    return np.concatenate(parts, axis=1)
