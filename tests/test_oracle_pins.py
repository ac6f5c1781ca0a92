"""Pins of the CPU oracle against what the pages and the mathematics fix (CPU only).

Each test names what it pins. Values come from the OCP MX table
(tests/golden/ocp_mx_e2m1_table.txt), hand arithmetic
(tests/golden/mx_hand_blocks.txt), closed forms, invariants, library primitives
on special cases, or brute force on tiny shapes.
"""
import math

import numpy as np
import pytest

import inputs as IN
import oracle as O
from conftest import read_golden


def table():
    return np.array([float(v) for _, v in read_golden("ocp_mx_e2m1_table.txt")])


def bf16(x):
    return IN.f32_to_bf16(np.asarray(x, np.float32))


def bf16_val(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)


def tiny_inputs(T=4, H=64, E=8, k=2, I=32, Is=32, seed=0, routing="learned", bias_std=0.3):
    wl = IN.Workload("t", T=T, H=H, E=E, k=k, I=I, Is=Is, routing=routing, bias_std=bias_std,
                     vocab=97, seed=seed)
    return IN.make_layer_inputs(wl)


def with_fields(li, **kw):
    d = dict(li.__dict__)
    d.update(kw)
    return IN.LayerInputs(**d)


# ----------------------------------------------------------------------------- formats

def test_e2m1_matches_ocp_table():
    tab = table()
    got = np.array([O.e2m1(c) for c in range(16)])
    assert np.array_equal(got, tab)
    assert all(math.copysign(1, O.e2m1(c)) == math.copysign(1, tab[c]) for c in range(16))


def test_e8m0_exhaustive():
    for e in range(255):
        assert O.e8m0(e) == 2.0 ** (e - 127)
    assert math.isnan(O.e8m0(255))


def test_mxfp4_decode_exhaustive_codes_by_exponents():
    tab = table()
    for e in range(0, 255, 1):
        scales = np.array([e, 255 - e if 255 - e < 255 else 0], np.uint8)
        for c in range(16):
            other = (c * 7 + 3) & 15
            codes = np.zeros(32, np.uint8)
            codes[0] = c | (other << 4)        # k=0 low nibble, k=1 high nibble
            codes[16] = other | (c << 4)       # k=32 (second group) low, k=33 high
            assert O.mxfp4_at(codes, scales, 0) == tab[c] * 2.0 ** (e - 127)
            assert O.mxfp4_at(codes, scales, 1) == tab[other] * 2.0 ** (e - 127)
            assert O.mxfp4_at(codes, scales, 33) == tab[c] * 2.0 ** (int(scales[1]) - 127)


def test_hand_built_blocks():
    for row in read_golden("mx_hand_blocks.txt"):
        e, want, codes = int(row[0]), float(row[1]), [int(c) for c in row[2:]]
        assert len(codes) == 32
        packed = np.array([codes[2 * i] | (codes[2 * i + 1] << 4) for i in range(16)], np.uint8)
        sc = np.array([e], np.uint8)
        got = sum(O.mxfp4_at(packed, sc, k) * 1.0 for k in range(32))
        assert got == want


def test_bf16_to_double_exact():
    for bits, val in [(0x3F80, 1.0), (0xBF80, -1.0), (0x4049, 3.140625), (0x0001, 2.0 ** -133),
                      (0x7F7F, 3.3895313892515355e38), (0x0000, 0.0)]:
        assert O.bf16_to_double(bits) == val


# ----------------------------------------------------------------------------- scoring / clamp

def test_sqrt_softplus_closed_forms():
    assert O.sqrt_softplus(0.0) == pytest.approx(0.8325546111576977, rel=0, abs=1e-16)
    assert O.sqrt_softplus(0.0) == pytest.approx(math.sqrt(math.log(2.0)), rel=1e-15)
    # large z: softplus(z) = z + log1p(e^-z) -> sqrt(z) (1 + e^-z / (2z))
    for z in (40.0, 100.0, 700.0):
        assert O.sqrt_softplus(z) == pytest.approx(math.sqrt(z), rel=1e-15)
    # very negative z: softplus(z) ~ e^z (1 - e^z/2) -> sqrt ~ e^(z/2)
    for z in (-30.0, -100.0, -700.0):
        assert O.sqrt_softplus(z) == pytest.approx(math.exp(z / 2), rel=1e-12)
    zs = np.linspace(-50, 50, 2001)
    v = np.array([O.sqrt_softplus(z) for z in zs])
    assert np.all(v > 0) and np.all(np.diff(v) > 0)


def test_silu_identity():
    # silu(x) - silu(-x) = x (since sigma(x) + sigma(-x) = 1); silu(0) = 0
    for x in (0.0, 0.3, 1.0, 7.5, 10.0, 50.0):
        assert O.silu(x) - O.silu(-x) == pytest.approx(x, rel=1e-15, abs=1e-15)
    assert O.silu(0.0) == 0.0
    assert O.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)


def test_clamp_sides():
    grid = [-50.0, -10.0, 0.0, 10.0, 50.0]
    L = 10.0
    for g in grid:
        for u in grid:
            v = O.clamped_swiglu(g, u, L)
            # up is clamped on both sides
            assert v == O.clamped_swiglu(g, max(-L, min(L, u)), L)
            # gate is clamped from above only
            if g > L:
                assert v == O.clamped_swiglu(L, u, L)
    # gate has no lower clamp: g = -50 is not treated as -10
    assert O.clamped_swiglu(-50.0, 1.0, L) != O.clamped_swiglu(-10.0, 1.0, L)
    assert O.clamped_swiglu(-50.0, 1.0, L) == pytest.approx(-50.0 / (1.0 + math.exp(50.0)), rel=1e-14)
    assert O.clamped_swiglu(50.0, 50.0, L) == pytest.approx(10.0 * 10.0 / (1.0 + math.exp(-10.0)), rel=1e-15)
    assert O.clamped_swiglu(3.0, -50.0, L) == pytest.approx(-10.0 * 3.0 / (1.0 + math.exp(-3.0)), rel=1e-15)


# ----------------------------------------------------------------------------- routing

def _onehot_router(logits, bias, k=6, scale=1.5):
    """x = e_0 and gate[:, 0] = logits makes z_e = logits[e] exactly."""
    E = len(logits)
    H = 32
    li = tiny_inputs(T=1, H=H, E=E, k=k, I=32, Is=0)
    x = np.zeros((1, H), np.uint16)
    x[0, 0] = 0x3F80  # 1.0
    gate = np.zeros((E, H), np.uint16)
    gate[:, 0] = bf16(logits)
    li = with_fields(li, x=x, gate=gate, bias=np.asarray(bias, np.float32))
    return O.Layer(li), bf16_val(gate[:, 0])


def test_bias_selects_but_does_not_weight():
    E = 16
    logits = np.linspace(2.0, -2.0, E)  # descending: unbiased top-6 = {0..5}
    lay, z = _onehot_router(logits, np.zeros(E))
    ids, w, margin, s = lay.route(want_scores=True)
    assert ids[0].tolist() == [0, 1, 2, 3, 4, 5]
    bias = np.zeros(E, np.float32)
    bias[6:12] = 100.0
    lay2, z2 = _onehot_router(logits, bias)
    ids2, w2, _, s2 = lay2.route(want_scores=True)
    assert ids2[0].tolist() == [6, 7, 8, 9, 10, 11]
    # weights come from the unbiased scores at the selected ids
    sel = np.array([O.sqrt_softplus(v) for v in z2[6:12]])
    assert np.allclose(w2[0], 1.5 * sel / sel.sum(), rtol=1e-15, atol=0)
    assert np.allclose(s2[0], [O.sqrt_softplus(v) for v in z2], rtol=0, atol=0)


def test_tie_breaks_to_lower_index_and_ascending_output():
    E = 12
    logits = np.full(E, -1.0)
    logits[[9, 1, 7, 3, 11]] = 1.0   # five clear winners
    logits[[4, 8]] = 0.5            # tie for the 6th place between 4 and 8
    lay, _ = _onehot_router(logits, np.zeros(E))
    ids, w, margin, _ = lay.route()
    assert ids[0].tolist() == [1, 3, 4, 7, 9, 11]
    assert margin[0] == 0.0


def test_weights_sum_and_positivity():
    li = tiny_inputs(T=64, H=128, E=32, k=6, I=32, Is=0, bias_std=0.5)
    ids, w, margin, _ = O.Layer(li).route()
    sums = w.sum(axis=1)
    assert np.all(np.abs(sums - 1.5) <= 4 * np.spacing(1.5))
    assert np.all(w > 0)
    assert np.all(np.diff(ids, axis=1) > 0)   # ascending, distinct


def test_topk_matches_full_sort():
    li = tiny_inputs(T=200, H=96, E=40, k=6, I=32, Is=0, bias_std=0.2, seed=3)
    ids, w, margin, scores = O.Layer(li).route(want_scores=True)
    b = scores + li.bias.astype(np.float64)[None, :]
    for t in range(li.wl.T):
        order = np.lexsort((np.arange(40), -b[t]))   # by b descending, then index ascending
        assert sorted(order[:6].tolist()) == ids[t].tolist()
        assert margin[t] == b[t, order[5]] - b[t, order[6]]


def test_scores_are_fp64_gate_gemv():
    li = tiny_inputs(T=5, H=64, E=8, k=2, I=32, Is=0)
    _, _, _, scores = O.Layer(li).route(want_scores=True)
    z = bf16_val(li.x) @ bf16_val(li.gate).T       # exact products, fp64 sums (library matmul)
    sp = np.logaddexp(0.0, z)                       # softplus via a library routine
    assert np.allclose(scores, np.sqrt(sp), rtol=1e-13, atol=0)


def test_hash_routing_ids_are_table_rows():
    li = tiny_inputs(T=50, H=64, E=16, k=6, I=32, Is=0, routing="hash")
    ids, w, margin, scores = O.Layer(li).route(want_scores=True)
    assert np.array_equal(ids, li.tid2eid[li.token_ids])
    sel = np.take_along_axis(scores, ids, axis=1)
    assert np.allclose(w, 1.5 * sel / sel.sum(axis=1, keepdims=True), rtol=1e-15, atol=0)
    assert np.all(np.isinf(margin))
    bad = with_fields(li, token_ids=np.full(50, 97, np.int32))
    with pytest.raises(ValueError):
        O.Layer(bad).route()


# ----------------------------------------------------------------------------- permutation

def test_permutation_is_stable_counting_sort():
    rng = np.random.default_rng(1)
    ids = rng.integers(0, 20, (37, 6)).astype(np.int32)
    ids[:, 0] = 3   # a hot expert
    counts, offsets, sorted_slot, slot_pos = O.permute(ids, 20)
    flat = ids.ravel()
    assert np.array_equal(counts, np.bincount(flat, minlength=20))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    assert np.array_equal(sorted_slot, np.argsort(flat, kind="stable"))
    assert np.array_equal(slot_pos[sorted_slot], np.arange(flat.size))
    with pytest.raises(ValueError):
        O.permute(np.array([[0, 20]], np.int32), 20)
    # empty input
    c, o, s, p = O.permute(np.zeros((0, 6), np.int32), 5)
    assert not c.any() and not o.any() and s.size == 0


# ----------------------------------------------------------------------------- layer

def _np_expert(li, e, x):
    """One routed expert in numpy with the golden OCP table (independent decode)."""
    tab = table()
    H, I = li.wl.H, li.wl.I

    def deq(codes, scales):
        lo, hi = codes & 15, codes >> 4
        c = np.stack([lo, hi], -1).reshape(codes.shape[0], -1)
        return tab[c] * np.repeat(np.ldexp(1.0, scales.astype(np.int64) - 127), 32, axis=1)

    W13 = deq(li.w13_codes[e], li.w13_scales[e])
    W2 = deq(li.w2_codes[e], li.w2_scales[e])
    gu = W13 @ x
    g, u = gu[:I], gu[I:]
    L = li.wl.swiglu_limit
    gc = np.minimum(g, L)
    h = gc / (1.0 + np.exp(-gc)) * np.clip(u, -L, L)
    return W2 @ h, h


def test_single_expert_matches_numpy_dequant_gemv():
    li = tiny_inputs(T=3, H=64, E=4, k=1, I=64, Is=0)
    lay = O.Layer(li)
    ids = np.array([[2], [0], [3]], np.int32)
    w = np.ones((3, 1))
    out, h, _ = lay.moe_tokens(np.arange(3), ids, w, want_h=True)
    for t in range(3):
        y, hh = _np_expert(li, ids[t, 0], bf16_val(li.x[t]))
        assert np.allclose(out[t], y, rtol=1e-12, atol=1e-14)
        assert np.allclose(h[t, 0], hh, rtol=1e-12, atol=1e-14)


def test_gate_and_up_halves_of_w13():
    # Gate rows that give g >= 10 and up rows that give u = 1 make h = silu(10);
    # swapping the halves would give silu(1) * 10 instead.
    H, I = 32, 32
    li = tiny_inputs(T=1, H=H, E=1, k=1, I=I, Is=0)
    x = np.zeros((1, H), np.uint16)
    x[0, :] = 0x3F80
    codes = np.zeros((1, 2 * I, H // 2), np.uint8)
    scales = np.full((1, 2 * I, 1), 127, np.uint8)
    codes[0, :I, :] = 0x77       # gate rows: every element 6.0 -> g = 192
    codes[0, I:, 0] = 0x02       # up rows: one element 1.0 -> u = 1
    w2c = np.zeros((1, H, I // 2), np.uint8)
    w2c[0, :, 0] = 0x02          # y_m = h_0
    w2s = np.full((1, H, 1), 127, np.uint8)
    li = with_fields(li, x=x, w13_codes=codes, w13_scales=scales, w2_codes=w2c, w2_scales=w2s)
    out = O.Layer(li).moe_tokens([0], np.zeros((1, 1), np.int32), np.ones((1, 1)))
    assert np.allclose(out[0], 10.0 / (1.0 + math.exp(-10.0)), rtol=1e-15)


@pytest.mark.parametrize("k", [2, 4, 6])
def test_sparse_oracle_matches_dense_brute_force(k):
    li = tiny_inputs(T=5, H=64, E=8, k=k, I=32, Is=32, seed=k)
    lay = O.Layer(li)
    ids, w, _, _ = lay.route()
    sparse = lay.moe_tokens(np.arange(5), ids, w)
    dense = lay.moe_dense(ids, w)
    assert np.allclose(sparse, dense, rtol=1e-12, atol=1e-14 * np.abs(dense).max())


def test_routing_off_gives_shared_expert_alone():
    li = tiny_inputs(T=4, H=64, E=8, k=6, I=32, Is=64)
    lay = O.Layer(li)
    ids, _, _, _ = lay.route()
    out = lay.moe_tokens(np.arange(4), ids, np.zeros((4, 6)))
    # shared expert as plain int8 GEMMs in numpy
    x = bf16_val(li.x)
    W13 = li.sh13.astype(np.float64) * li.sh13_scale.astype(np.float64)[:, None]
    W2 = li.sh2.astype(np.float64) * li.sh2_scale.astype(np.float64)[:, None]
    gu = x @ W13.T
    g, u = gu[:, :64], gu[:, 64:]
    gc = np.minimum(g, 10.0)
    h = gc / (1.0 + np.exp(-gc)) * np.clip(u, -10.0, 10.0)
    assert np.allclose(out, h @ W2.T, rtol=1e-12, atol=1e-14)
    # without a shared expert and with zero weights the output is exactly zero
    li0 = tiny_inputs(T=4, H=64, E=8, k=6, I=32, Is=0)
    lay0 = O.Layer(li0)
    ids0, _, _, _ = lay0.route()
    assert not lay0.moe_tokens(np.arange(4), ids0, np.zeros((4, 6))).any()


def test_output_is_linear_in_routing_weights():
    li = tiny_inputs(T=3, H=64, E=8, k=3, I=32, Is=0)
    lay = O.Layer(li)
    ids, w, _, _ = lay.route()
    a = lay.moe_tokens(np.arange(3), ids, w)
    b = lay.moe_tokens(np.arange(3), ids, 2.0 * w)
    assert np.allclose(b, 2.0 * a, rtol=1e-14, atol=0)


def test_threaded_token_split_changes_nothing():
    li = tiny_inputs(T=7, H=64, E=8, k=3, I=32, Is=32)
    lay = O.Layer(li)
    ids, w, _, _ = lay.route()
    a = lay.moe_tokens(np.arange(7), ids, w, threads=1)
    b = lay.moe_tokens(np.arange(7), ids, w, threads=3)
    assert np.array_equal(a, b)
    a2, h2, hs2 = lay.moe_tokens(np.array([6, 1]), ids, w, threads=2, want_h=True)
    assert np.array_equal(a2, a[[6, 1]])


# ----------------------------------------------------------------------------- W8A16 linear

def test_linear_w8a16_hand_case():
    # x = [1, 2], q = [[1, 2], [3, -4]], scale = [0.5, 2]: (1 + 4) * 0.5 and (3 - 8) * 2
    x = np.array([[0x3F80, 0x4000]], np.uint16)
    q = np.array([[1, 2], [3, -4]], np.int8)
    s = np.array([0.5, 2.0], np.float32)
    assert O.linear_w8a16(x, q, s).tolist() == [[2.5, -10.0]]


def test_linear_w8a16_scaled_identity_is_exact():
    # q = c * I with scale 2^-3: out = x * c / 8 exactly (powers of two, small c)
    K = 64
    x = bf16(np.linspace(-3.0, 3.0, 2 * K).reshape(2, K))
    for c in (-127, -3, 1, 5, 127):
        q = (np.eye(K) * c).astype(np.int8)
        s = np.full(K, 0.125, np.float32)
        assert np.array_equal(O.linear_w8a16(x, q, s), bf16_val(x) * c * 0.125)


def test_linear_w8a16_matches_numpy_and_row_subset():
    rng = np.random.default_rng(3)
    T, N, K = 5, 40, 96
    x = bf16(rng.standard_normal((T, K)))
    q = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    s = (rng.random(N) * 0.01).astype(np.float32)
    ref = bf16_val(x) @ (q.astype(np.float64) * s.astype(np.float64)[:, None]).T
    got = O.linear_w8a16(x, q, s)
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-15)
    assert np.array_equal(O.linear_w8a16(x, q, s, rows=[4, 1]), got[[4, 1]])


def test_linear_w8a16_grouped_is_block_diagonal():
    # G groups on their own column and row slices == one linear whose weight is
    # block-diagonal (zeros between groups): checks which x columns and which
    # weight rows each group takes
    rng = np.random.default_rng(5)
    T, G, N, K = 3, 3, 4, 8
    x = bf16(rng.standard_normal((T, G * K)))
    q = rng.integers(-127, 128, size=(G * N, K)).astype(np.int8)
    s = (rng.random(G * N) * 0.01 + 0.001).astype(np.float32)
    bd = np.zeros((G * N, G * K), np.int8)
    for g in range(G):
        bd[g * N:(g + 1) * N, g * K:(g + 1) * K] = q[g * N:(g + 1) * N]
    got = O.linear_w8a16_grouped(x, q, s, G)
    assert got.shape == (T, G * N)
    assert np.allclose(got, O.linear_w8a16(x, bd, s), rtol=1e-14, atol=0)
    ref = np.concatenate([bf16_val(x)[:, g * K:(g + 1) * K] @ (q[g * N:(g + 1) * N].astype(np.float64)
                          * s[g * N:(g + 1) * N, None].astype(np.float64)).T for g in range(G)], axis=1)
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-15)
    assert np.array_equal(O.linear_w8a16_grouped(x, q, s, G, rows=[2]), got[[2]])
