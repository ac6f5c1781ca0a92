"""Seeded synthetic inputs for the routed MoE layer (shared by the oracle side
and the CUDA side of every test and of the benchmark).

The module draws random tensors and stores them in the layer's storage formats
(bf16 activations, MXFP4 expert weights with E8M0 block scales, int8 per-channel
shared-expert weights, Zipf token ids, a token-id -> expert table). It holds no
routing, decoding or GEMM arithmetic; all of that lives separately in the oracle
and in the CUDA library. The heavy lifting is in ``v4moe_inputs.cpp`` (built
in-tree with g++ on first use).

Workloads are the five synthetic MoE-layer shapes of the DeepSeek-V4-Flash
routed expert FFN (model constants from the model's ``config.json``:
hidden_size 4096, moe_intermediate_size 2048, n_routed_experts 256,
num_experts_per_tok 6, n_shared_experts 1, vocab_size 129280).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "v4moe_inputs.cpp")
_LIB = os.path.join(_HERE, "libv4moe_inputs.so")
_lock = threading.Lock()
_lib = None

# Tensor tags of the Philox streams (key = (seed, tag)).
TAG_X, TAG_GATE, TAG_BIAS, TAG_W13, TAG_W2, TAG_SH13, TAG_SH2, TAG_TOKID, TAG_TID2EID = range(1, 10)


def build(force: bool = False) -> str:
    """Compile libv4moe_inputs.so in-tree if it is missing or older than its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["g++", "-O3", "-std=c++17", "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            u64, u32, i64, i32, f32, f64 = (ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64,
                                            ctypes.c_int32, ctypes.c_float, ctypes.c_double)
            P = ctypes.c_void_p
            L.v4in_philox4x32_10.argtypes = [u32] * 6 + [P]
            L.v4in_normal_f32.argtypes = [u64, u32, u64, u64, f32, f32, P, ctypes.c_int]
            L.v4in_normal_bf16.argtypes = [u64, u32, u64, u64, f32, f32, P, ctypes.c_int]
            L.v4in_f32_to_bf16.argtypes = [P, u64, P]
            L.v4in_quantize_mxfp4.argtypes = [P, i64, i64, P, P, ctypes.c_int]
            L.v4in_quantize_mxfp4.restype = ctypes.c_int
            L.v4in_mxfp4_normal.argtypes = [u64, u32, i64, i64, i64, f32, P, P, ctypes.c_int]
            L.v4in_mxfp4_normal.restype = ctypes.c_int
            L.v4in_quantize_int8.argtypes = [P, i64, i64, P, P, ctypes.c_int]
            L.v4in_int8_normal.argtypes = [u64, u32, i64, i64, f32, P, P, ctypes.c_int]
            L.v4in_zipf_ids.argtypes = [u64, u32, i64, i64, f64, P, ctypes.c_int]
            L.v4in_zipf_ids.restype = ctypes.c_int
            L.v4in_tid2eid.argtypes = [u64, u32, i64, i32, i32, P, ctypes.c_int]
            L.v4in_tid2eid.restype = ctypes.c_int
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


# ----------------------------------------------------------------------------- primitives

def philox4x32_10(counter, key):
    out = np.zeros(4, np.uint32)
    lib().v4in_philox4x32_10(*[int(c) for c in counter], *[int(k) for k in key], _p(out))
    return out


def normal_f32(seed, tag, n, mean=0.0, std=1.0, first=0, threads=0):
    out = np.empty(int(n), np.float32)
    lib().v4in_normal_f32(seed, tag, first, int(n), mean, std, _p(out), threads)
    return out


def normal_bf16(seed, tag, n, mean=0.0, std=1.0, first=0, threads=0):
    """bf16 bit patterns (uint16) of N(mean, std) draws rounded to nearest even."""
    out = np.empty(int(n), np.uint16)
    lib().v4in_normal_bf16(seed, tag, first, int(n), mean, std, _p(out), threads)
    return out


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().v4in_f32_to_bf16(_p(x), x.size, _p(out))
    return out


def quantize_mxfp4(w: np.ndarray, threads=0):
    """MXFP4-quantise fp32 rows [..., K] -> (codes [..., K/2] u8, scales [..., K/32] u8)."""
    w = np.ascontiguousarray(w, np.float32)
    K = w.shape[-1]
    rows = w.size // K
    codes = np.empty(w.shape[:-1] + (K // 2,), np.uint8)
    scales = np.empty(w.shape[:-1] + (K // 32,), np.uint8)
    rc = lib().v4in_quantize_mxfp4(_p(w), rows, K, _p(codes), _p(scales), threads)
    if rc:
        raise ValueError("K must be a multiple of 32")
    return codes, scales


def mxfp4_normal(seed, tag, rows, K, std, row0=0, threads=0):
    codes = np.empty((rows, K // 2), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    rc = lib().v4in_mxfp4_normal(seed, tag, row0, rows, K, std, _p(codes), _p(scales), threads)
    if rc:
        raise ValueError("K must be a multiple of 32")
    return codes, scales


def quantize_int8(w: np.ndarray, threads=0):
    w = np.ascontiguousarray(w, np.float32)
    rows, K = w.shape
    q = np.empty((rows, K), np.int8)
    s = np.empty(rows, np.float32)
    lib().v4in_quantize_int8(_p(w), rows, K, _p(q), _p(s), threads)
    return q, s


def int8_normal(seed, tag, rows, K, std, threads=0):
    q = np.empty((rows, K), np.int8)
    s = np.empty(rows, np.float32)
    lib().v4in_int8_normal(seed, tag, rows, K, std, _p(q), _p(s), threads)
    return q, s


def zipf_ids(seed, tag, n, vocab, s, threads=0):
    out = np.empty(int(n), np.int32)
    rc = lib().v4in_zipf_ids(seed, tag, int(n), int(vocab), float(s), _p(out), threads)
    if rc:
        raise ValueError("vocab must be positive")
    return out


def tid2eid(seed, tag, vocab, k, E, threads=0):
    out = np.empty((int(vocab), int(k)), np.int32)
    rc = lib().v4in_tid2eid(seed, tag, int(vocab), int(k), int(E), _p(out), threads)
    if rc:
        raise ValueError("need 0 < k <= E")
    return out


# ----------------------------------------------------------------------------- workloads

@dataclass(frozen=True)
class Workload:
    """One synthetic MoE-layer configuration (shapes, routing mode, generator recipe)."""
    name: str
    T: int
    H: int = 4096
    E: int = 256
    k: int = 6
    I: int = 2048
    Is: int = 2048              # shared-expert intermediate size (0 = no shared expert)
    routing: str = "learned"    # "learned" (sqrt-softplus, biased top-k) or "hash" (tid2eid)
    bias_std: float = 0.01
    vocab: int = 129280
    zipf_s: float = 1.1
    w_std: float = 0.02
    gate_std: float = 0.02
    x_std: float = 1.0
    routed_scale: float = 1.5
    swiglu_limit: float = 10.0
    seed: int = 0
    notes: str = ""

    def with_T(self, T: int) -> "Workload":
        d = dict(self.__dict__)
        d["T"] = T
        return Workload(**d)

    def replace(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny": Workload("tiny", T=32, H=512, E=16, I=256, Is=256,
                     notes="tiny MoE layer, all experts hit"),
    "decode_b1": Workload("decode_b1", T=1,
                          notes="full-size layer, decode batch 1: ~6 experts + shared streamed"),
    "decode_b64": Workload("decode_b64", T=64, bias_std=0.5,
                           notes="full-size layer, decode batch 64; bias N(0,0.5) spreads load"),
    "prefill_4096": Workload("prefill_4096", T=4096,
                             notes="full-size layer, prefill 4096 tokens, near-uniform load"),
    "hash_16384": Workload("hash_16384", T=16384, routing="hash", bias_std=0.0,
                           notes="hash-routed layer, Zipf(1.1) token ids, skewed expert load"),
    # Smaller cases of the same kernels for profiler captures (64 experts keep
    # the weights under 1 GB; per-expert token counts match the full cases).
    "decode_b1_e64": Workload("decode_b1_e64", T=1, E=64,
                              notes="decode batch 1 with 64 experts (profiling size)"),
    "decode_b64_e64": Workload("decode_b64_e64", T=64, E=64, bias_std=0.5,
                               notes="decode batch 64 with 64 experts (profiling size)"),
    "prefill_1024_e64": Workload("prefill_1024_e64", T=1024, E=64,
                                 notes="prefill, ~96 tokens per expert, 64 experts (profiling size)"),
}
WORKLOAD_ORDER = ["tiny", "decode_b1", "decode_b64", "prefill_4096", "hash_16384"]


@dataclass
class LayerInputs:
    wl: Workload
    x: np.ndarray            # [T, H] uint16 (bf16 bits)
    gate: np.ndarray         # [E, H] uint16 (bf16 bits)
    bias: np.ndarray | None  # [E] float32 (learned routing)
    token_ids: np.ndarray | None  # [T] int32 (hash routing)
    tid2eid: np.ndarray | None    # [vocab, k] int32 (hash routing)
    w13_codes: np.ndarray    # [E, 2I, H/2] uint8
    w13_scales: np.ndarray   # [E, 2I, H/32] uint8
    w2_codes: np.ndarray     # [E, H, I/2] uint8
    w2_scales: np.ndarray    # [E, H, I/32] uint8
    sh13: np.ndarray | None        # [2Is, H] int8
    sh13_scale: np.ndarray | None  # [2Is] float32
    sh2: np.ndarray | None         # [H, Is] int8
    sh2_scale: np.ndarray | None   # [H] float32
    extra: dict = field(default_factory=dict)


def make_weights(wl: Workload, threads=0):
    """Expert and shared weights + gate for a workload (independent of T)."""
    E, H, I, Is, s = wl.E, wl.H, wl.I, wl.Is, wl.seed
    gate = normal_bf16(s, TAG_GATE, E * H, 0.0, wl.gate_std, threads=threads).reshape(E, H)
    c13, s13 = mxfp4_normal(s, TAG_W13, E * 2 * I, H, wl.w_std, threads=threads)
    c2, s2 = mxfp4_normal(s, TAG_W2, E * H, I, wl.w_std, threads=threads)
    w = dict(gate=gate,
             w13_codes=c13.reshape(E, 2 * I, H // 2), w13_scales=s13.reshape(E, 2 * I, H // 32),
             w2_codes=c2.reshape(E, H, I // 2), w2_scales=s2.reshape(E, H, I // 32))
    if Is > 0:
        q13, sc13 = int8_normal(s, TAG_SH13, 2 * Is, H, wl.w_std, threads=threads)
        q2, sc2 = int8_normal(s, TAG_SH2, H, Is, wl.w_std, threads=threads)
        w.update(sh13=q13, sh13_scale=sc13, sh2=q2, sh2_scale=sc2)
    else:
        w.update(sh13=None, sh13_scale=None, sh2=None, sh2_scale=None)
    return w


def make_activations(wl: Workload, threads=0):
    """Per-batch inputs: x and (learned) bias or (hash) token ids + table."""
    s = wl.seed
    x = normal_bf16(s, TAG_X, wl.T * wl.H, 0.0, wl.x_std, threads=threads).reshape(wl.T, wl.H)
    a = dict(x=x, bias=None, token_ids=None, tid2eid=None)
    if wl.routing == "learned":
        a["bias"] = normal_f32(s, TAG_BIAS, wl.E, 0.0, wl.bias_std, threads=threads)
    elif wl.routing == "hash":
        a["token_ids"] = zipf_ids(s, TAG_TOKID, wl.T, wl.vocab, wl.zipf_s, threads=threads)
        a["tid2eid"] = tid2eid(s, TAG_TID2EID, wl.vocab, wl.k, wl.E, threads=threads)
    else:
        raise ValueError(wl.routing)
    return a


def make_layer_inputs(wl: Workload, weights: dict | None = None, threads=0) -> LayerInputs:
    w = weights if weights is not None else make_weights(wl, threads)
    a = make_activations(wl, threads)
    return LayerInputs(wl=wl, x=a["x"], gate=w["gate"], bias=a["bias"], token_ids=a["token_ids"],
                       tid2eid=a["tid2eid"], w13_codes=w["w13_codes"], w13_scales=w["w13_scales"],
                       w2_codes=w["w2_codes"], w2_scales=w["w2_scales"], sh13=w["sh13"],
                       sh13_scale=w["sh13_scale"], sh2=w["sh2"], sh2_scale=w["sh2_scale"])
