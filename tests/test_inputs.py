"""Pins of the seeded input generator (CPU only)."""
import math

import numpy as np
import pytest

import inputs as IN
from conftest import read_golden


def _e2m1_table():
    return np.array([float(v) for _, v in read_golden("ocp_mx_e2m1_table.txt")])


def _decode_np(codes, scales):
    """Decode packed MXFP4 with the OCP table from the golden file (numpy)."""
    tab = _e2m1_table()
    lo = codes & 0xF
    hi = codes >> 4
    c = np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * 2,))
    v = tab[c]
    s = np.repeat(np.ldexp(1.0, scales.astype(np.int64) - 127), 32, axis=-1)
    return v * s


def test_philox_known_answers():
    # Known-answer vectors published with Random123 (Salmon et al., SC'11) for
    # philox4x32 with 10 rounds.
    kat = [
        ([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
        ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2, [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
        ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
         [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
    ]
    for ctr, key, want in kat:
        assert list(IN.philox4x32_10(ctr, key)) == want


def test_streams_independent_of_thread_count():
    a = IN.normal_f32(3, 7, 100_003, threads=1)
    b = IN.normal_f32(3, 7, 100_003, threads=5)
    assert np.array_equal(a, b)
    # an offset window is the same elements
    c = IN.normal_f32(3, 7, 1000, first=50_001, threads=3)
    assert np.array_equal(a[50_001:51_001], c)
    ca, sa = IN.mxfp4_normal(0, 4, 33, 256, 0.02, threads=1)
    cb, sb = IN.mxfp4_normal(0, 4, 33, 256, 0.02, threads=8)
    assert np.array_equal(ca, cb) and np.array_equal(sa, sb)
    # rows generated from an offset row0 equal the same rows of a full draw
    cc, sc = IN.mxfp4_normal(0, 4, 10, 256, 0.02, row0=7)
    assert np.array_equal(ca[7:17], cc) and np.array_equal(sa[7:17], sc)


def test_normal_moments():
    z = IN.normal_f32(0, 1, 2_000_000, mean=0.5, std=2.0)
    assert abs(z.mean() - 0.5) < 0.01
    assert abs(z.std() - 2.0) < 0.01
    # fourth standardized moment of a normal is 3
    k4 = np.mean(((z - z.mean()) / z.std()) ** 4)
    assert abs(k4 - 3.0) < 0.05


def test_bf16_rounding_is_rne():
    x = IN.normal_f32(1, 2, 10000)
    got = IN.f32_to_bf16(x)
    u = x.view(np.uint32).astype(np.uint64)
    lower = (u >> 16) & 0xFFFF
    rem = u & 0xFFFF
    up = (rem > 0x8000) | ((rem == 0x8000) & ((lower & 1) == 1))
    want = (lower + up).astype(np.uint16)
    assert np.array_equal(got, want)
    # ties: 1 + 2^-8 is halfway between bf16 1.0 and 1.0078125 -> even (1.0)
    t = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], np.float32)
    assert list(IN.f32_to_bf16(t)) == [0x3F80, 0x3F82]


def test_mxfp4_representable_round_trip():
    tab = _e2m1_table()
    rng = np.random.default_rng(0)
    rows = []
    exps = []
    for r in range(64):
        X = int(rng.integers(-20, 10))
        codes = rng.integers(0, 16, 32)
        codes[0] = 7  # amax = 6 * 2^X makes the shared exponent exactly X
        rows.append(tab[codes] * 2.0 ** X)
        exps.append(X)
    w = np.array(rows, np.float32)
    c, s = IN.quantize_mxfp4(w)
    assert list(s[:, 0].astype(int) - 127) == exps
    assert np.array_equal(_decode_np(c, s), w.astype(np.float64))


def test_mxfp4_ties_and_saturation():
    # Scale forced to 2^0 by amax in [4, 8): X = floor(log2 amax) - 2 = 0.
    def q(vals):
        v = np.zeros(32, np.float32)
        v[: len(vals)] = vals
        v[31] = 4.0
        c, s = IN.quantize_mxfp4(v[None, :])
        assert s[0, 0] == 127
        return list(_decode_np(c, s)[0, : len(vals)])

    # ties go to the even code
    assert q([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    assert q([-0.25, -0.75, -2.5, -5.0]) == [-0.0, -1.0, -2.0, -4.0]
    # non-ties go to the nearest value
    assert q([0.26, 0.74, 1.26, 2.51, 4.99, 5.01]) == [0.5, 0.5, 1.5, 3.0, 4.0, 6.0]
    # amax 7.9 -> X = 0, 7.9 saturates to 6
    v = np.zeros((1, 32), np.float32)
    v[0, 0] = 7.9
    c, s = IN.quantize_mxfp4(v)
    assert s[0, 0] == 127 and _decode_np(c, s)[0, 0] == 6.0
    # all-zero block: scale byte 0, all codes 0
    c, s = IN.quantize_mxfp4(np.zeros((1, 64), np.float32))
    assert s.tolist() == [[0, 0]] and not c.any()


def test_mxfp4_nibble_order():
    v = np.zeros((1, 32), np.float32)
    v[0, 0] = 1.0   # code 2 in the low nibble of byte 0
    v[0, 1] = -6.0  # code 15 in the high nibble of byte 0
    v[0, 2] = 4.0   # sets X = 0
    c, s = IN.quantize_mxfp4(v)
    assert s[0, 0] == 127
    assert c[0, 0] == (2 | (15 << 4))
    assert c[0, 1] == 6


def test_mxfp4_generated_equals_quantized_draw():
    # the fused draw+quantise path equals quantising the fp32 draw of the same stream
    c, s = IN.mxfp4_normal(0, 4, 64, 512, 0.02)
    w = IN.normal_f32(0, 4, 64 * 512, std=0.02).reshape(64, 512)
    c2, s2 = IN.quantize_mxfp4(w)
    assert np.array_equal(c, c2) and np.array_equal(s, s2)
    # error bound: block values scaled by 2^-X lie in [-8, 8), E2M1 gaps are at
    # most 2 (4 -> 6) and saturation above 6 costs < 2, so |w - deq| < 2 * 2^X
    X = np.repeat(s.astype(np.int64) - 127, 32, axis=1)
    err = np.abs(_decode_np(c, s) - w)
    assert np.all(err < 2.0 * np.ldexp(1.0, X))
    assert np.mean(err / np.ldexp(1.0, X)) < 0.3


def test_int8_quantizer():
    # power-of-two scale: amax = 127 * 2^-7 -> scale = 2^-7 exactly
    w = (np.append(np.arange(-127, 128), 0)[None, :].astype(np.float32) * 2.0 ** -7).astype(np.float32)
    q, s = IN.quantize_int8(w)
    assert s[0] == np.float32(2.0 ** -7)
    assert np.array_equal(q[0].astype(np.float32) * s[0], w[0])
    # rounding: 0.5 steps round to even, values clamp to +-127
    w2 = np.array([[127.0, 0.5, 1.5, -2.5, -127.0] + [0.0] * 3], np.float32)
    q2, s2 = IN.quantize_int8(w2)
    assert s2[0] == 1.0 and q2[0, :5].tolist() == [127, 0, 2, -2, -127]
    qz, sz = IN.quantize_int8(np.zeros((2, 8), np.float32))
    assert sz.tolist() == [1.0, 1.0] and not qz.any()
    # generated rows: |w - q*s| <= s/2 (re-draw the same stream in fp32)
    q3, s3 = IN.int8_normal(0, 6, 4, 64, 0.02)
    w3 = IN.normal_f32(0, 6, 4 * 64, std=0.02).reshape(4, 64)
    err = np.abs(q3.astype(np.float64) * s3[:, None] - w3)
    assert np.all(err <= s3[:, None] * 0.5 * (1 + 1e-6))
    assert np.all(np.abs(q3).max(axis=1) == 127)


def test_zipf_token_ids():
    V, s, n = 129280, 1.1, 200_000
    ids = IN.zipf_ids(0, 8, n, V, s)
    assert ids.min() >= 0 and ids.max() < V
    Hn = sum(r ** -s for r in range(1, V + 1))
    counts = np.bincount(ids, minlength=V)
    for r in (1, 2, 10):
        p = r ** -s / Hn
        sd = math.sqrt(n * p * (1 - p))
        assert abs(counts[r - 1] - n * p) < 5 * sd
    # determinism under threads
    assert np.array_equal(ids[:1000], IN.zipf_ids(0, 8, 1000, V, s, threads=1))


def test_tid2eid_rows_distinct():
    t = IN.tid2eid(0, 9, 5000, 6, 256)
    assert t.min() >= 0 and t.max() < 256
    assert all(len(set(r)) == 6 for r in t.tolist())
    # roughly uniform over experts
    cnt = np.bincount(t.ravel(), minlength=256)
    assert cnt.min() > 0.6 * cnt.mean() and cnt.max() < 1.4 * cnt.mean()
    assert np.array_equal(t, IN.tid2eid(0, 9, 5000, 6, 256, threads=1))
    with pytest.raises(ValueError):
        IN.tid2eid(0, 9, 10, 7, 6)


def test_workloads_match_page_constants():
    consts = {k: v for k, v in read_golden("v4_flash_moe_constants.txt")}
    for name in ("decode_b1", "decode_b64", "prefill_4096", "hash_16384"):
        wl = IN.WORKLOADS[name]
        assert wl.H == int(consts["hidden_size"])
        assert wl.I == int(consts["moe_intermediate_size"])
        assert wl.Is == int(consts["moe_intermediate_size"])  # one shared expert of the same size
        assert wl.E == int(consts["n_routed_experts"])
        assert wl.k == int(consts["num_experts_per_tok"])
        assert wl.routed_scale == float(consts["routed_scaling_factor"])
        assert wl.swiglu_limit == float(consts["swiglu_limit"])
        assert wl.vocab == int(consts["vocab_size"])
    assert IN.WORKLOADS["hash_16384"].routing == "hash"
