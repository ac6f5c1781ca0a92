"""GPU parity on what N(0,1) inputs never reach: the SwiGLU clamp engaged on
every dispatch path, exact ties at the top-k boundary, and activations and
weights whose magnitudes spread widely inside one 32-element block. The
oracle and the tolerances are those of the other parity tests (rel-L2 5e-3,
max-abs 1e-2 * max|ref|)."""
import numpy as np
import pytest

import inputs as IN
import oracle as O
from conftest import read_golden
from parity_util import assert_close, bf16_to_f64, host_threads, run_parity, upload_activations

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _layer(li):
    from mxfp4_routed_expert_v4moe_b200 import MoELayer
    return MoELayer.from_host(li)


def _with(li, **kw):
    d = dict(li.__dict__)
    d.update(kw)
    return IN.LayerInputs(**d)


def _bf16_vals(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)


def _clamp_fractions(li, ids):
    """Fractions of (token, expert, channel) with g > L, g < -L, |u| > L, from a
    numpy dequantisation with the OCP table (independent of both sides)."""
    tab = np.array([float(v) for _, v in read_golden("ocp_mx_e2m1_table.txt")])
    I, L = li.wl.I, li.wl.swiglu_limit
    x = _bf16_vals(li.x)
    hi = lo = up = n = 0
    for e in np.unique(ids):
        c, s = li.w13_codes[e], li.w13_scales[e]
        q = np.stack([c & 15, c >> 4], -1).reshape(c.shape[0], -1)
        W = tab[q] * np.repeat(np.ldexp(1.0, s.astype(np.int64) - 127), 32, axis=1)
        toks = np.nonzero((ids == e).any(axis=1))[0]
        gu = x[toks] @ W.T
        g, u = gu[:, :I], gu[:, I:]
        hi += (g > L).sum()
        lo += (g < -L).sum()
        up += (np.abs(u) > L).sum()
        n += g.size
    return hi / n, lo / n, up / n


# (name, T, H, E, I, Is): the routed GEMM and shared-expert kernel each case reaches
CLAMP_CASES = [
    ("decode", 5, 1024, 32, 512, 512),        # decode kernels (T <= 8)
    ("mx_tile32", 40, 1024, 32, 512, 512),    # weight-major block-scaled, 32-slot tiles; shared on the f16 dequant GEMM
    ("mx_tile128", 128, 1024, 32, 512, 512),  # weight-major, 128-slot tiles (experts average 24 slots)
    ("mxt_sh", 600, 1024, 32, 512, 512),      # token-major block-scaled; shared expert's f16 GEMM with the combine
    ("mx128_sh", 512, 1024, 128, 512, 512),   # weight-major 128-slot tiles with the shared f16 GEMM
    ("tc_dequant", 50, 256, 16, 256, 256),    # H % 512 != 0: routed experts on the dequantising f16 GEMM
]


@pytest.mark.parametrize("name,T,H,E,I,Is", CLAMP_CASES, ids=[c[0] for c in CLAMP_CASES])
def test_swiglu_clamp_engaged(name, T, H, E, I, Is):
    # w_std sets std(g) = std(u) ~ sqrt(H) * w_std ~ 13: a large share of the
    # gate values lie above L and below -L (no lower clamp on the gate), and
    # of the up values beyond +-L.
    w_std = 13.0 / np.sqrt(H)
    wl = IN.Workload(f"clamp_{name}", T=T, H=H, E=E, I=I, Is=Is, w_std=w_std, bias_std=0.05, seed=21)
    li = IN.make_layer_inputs(wl)
    ids_o, _, _, _ = O.Layer(li).route()
    hi, lo, up = _clamp_fractions(li, ids_o)
    assert hi > 0.1 and lo > 0.1 and up > 0.2, (hi, lo, up)
    run_parity(li, _layer(li))


def _tie_inputs(T, E, H=512, seed=3, I=256):
    """Gate rows one-hot (value 1) so that z_e = x[t, col(e)] exactly; experts 4
    and 8 read the same column, so their scores (and, with a zero bias, their
    biased scores) tie exactly in fp32 and in fp64. Every token has five
    clear winners above that pair and everything else below it."""
    wl = IN.Workload("ties", T=T, H=H, E=E, I=I, Is=256, bias_std=0.0, seed=seed)
    li = IN.make_layer_inputs(wl)
    col = np.arange(E)
    col[8] = 4
    gate = np.zeros((E, H), np.uint16)
    gate[np.arange(E), col] = 0x3F80          # bf16 1.0
    rng = np.random.default_rng(seed)
    x = li.x.copy()
    others = np.array([e for e in range(E) if e not in (4, 8)])
    for t in range(T):
        win = rng.choice(others, size=5, replace=False)
        v = np.full(E, 0.0, np.float32)
        v[others] = -1.0 - rng.permutation(len(others)).astype(np.float32) / 64.0
        v[win] = 2.0 + np.arange(5, dtype=np.float32) / 8.0
        v[4] = 1.0
        vals = IN.f32_to_bf16(v)
        x[t, :E] = 0
        for e in range(E):
            if e != 8:
                x[t, col[e]] = vals[e]
    return _with(li, gate=gate, x=x, bias=np.zeros(E, np.float32))


# I = 512 puts batches of at most 8 tokens on the decode kernels, whose router
# selects inside the whole-layer call (E = 300: more experts than its warps,
# and more than 256 per token)
@pytest.mark.parametrize("T,E,I", [(5, 16, 256), (40, 16, 256), (3, 300, 256), (5, 16, 512), (3, 300, 512)])
def test_exact_tie_goes_to_lower_expert_id(T, E, I):
    """An exact tie at the 6th place: the lower id (4) is chosen on the GPU,
    by the standalone router and inside the whole-layer call, on every
    token (no near-tie exclusion here)."""
    li = _tie_inputs(T, E, I=I)
    lay = O.Layer(li)
    ids_o, w_o, margin, _ = lay.route()
    assert (margin == 0.0).all()
    assert (ids_o == 4).any(axis=1).all() and not (ids_o == 8).any()
    layer = _layer(li)
    x, bias, _, _ = upload_activations(li)
    ids_r, w_r = layer.route(x, bias)
    out = layer(x, bias)
    torch.cuda.synchronize()
    ids_l = layer.buffers(T)["topk_ids"].cpu().numpy()
    assert np.array_equal(ids_r.cpu().numpy(), ids_o)
    assert np.array_equal(ids_l, ids_o)
    assert_close(w_r.cpu().numpy().astype(np.float64), w_o, "tie topk_w")
    ref = lay.moe_tokens(np.arange(T), ids_o, w_o.astype(np.float32).astype(np.float64), threads=host_threads())
    assert_close(bf16_to_f64(out), ref, "tie out")


def _spread_weights(wl, seed):
    """Routed MXFP4 weights whose 32-element groups span 2^0 .. 2^-20 within a
    row (widely spread E8M0 exponents), and int8 shared rows scaled by 2^0 ..
    2^-20 (per-row scales); drawn from the seeded generator, then quantised."""
    rng = np.random.default_rng(seed)
    E, H, I, Is = wl.E, wl.H, wl.I, wl.Is

    def mx(rows, K, tag):
        w = IN.normal_f32(wl.seed, tag, rows * K, 0.0, wl.w_std).reshape(rows, K // 32, 32)
        w *= np.ldexp(1.0, -rng.integers(0, 21, size=(rows, K // 32, 1))).astype(np.float32)
        return IN.quantize_mxfp4(w.reshape(rows, K))

    c13, s13 = mx(E * 2 * I, H, IN.TAG_W13)
    c2, s2 = mx(E * H, I, IN.TAG_W2)
    sh = IN.normal_f32(wl.seed, IN.TAG_SH13, 2 * Is * H, 0.0, wl.w_std).reshape(2 * Is, H)
    sh *= np.ldexp(1.0, -rng.integers(0, 21, size=(2 * Is, 1))).astype(np.float32)
    q13, sc13 = IN.quantize_int8(sh)
    sh2 = IN.normal_f32(wl.seed, IN.TAG_SH2, H * Is, 0.0, wl.w_std).reshape(H, Is)
    sh2 *= np.ldexp(1.0, -rng.integers(0, 21, size=(H, 1))).astype(np.float32)
    q2, sc2 = IN.quantize_int8(sh2)
    return dict(w13_codes=c13.reshape(E, 2 * I, H // 2), w13_scales=s13.reshape(E, 2 * I, H // 32),
                w2_codes=c2.reshape(E, H, I // 2), w2_scales=s2.reshape(E, H, I // 32),
                sh13=q13, sh13_scale=sc13, sh2=q2, sh2_scale=sc2)


@pytest.mark.parametrize("T", [4, 40, 600])
def test_wide_dynamic_range_in_blocks(T):
    """x elements spread over 2^0 .. 2^-16 of their block's largest magnitude
    (inside the exactness bound of the two E4M3 activation planes, 2^-14,
    and beyond it), one token at 2^12 and one at 2^-4 overall; expert weights
    with widely spread group exponents. Decode (T = 4), weight-major (40) and
    token-major (600) paths; every token within the bar on its own."""
    wl = IN.Workload("spread", T=T, H=1024, E=32, I=512, Is=512, bias_std=0.05, seed=17)
    li = IN.make_layer_inputs(wl)
    rng = np.random.default_rng(5)
    x = _bf16_vals(li.x).reshape(T, -1, 32)
    x *= np.ldexp(1.0, -rng.integers(0, 17, size=x.shape))
    x[:, :, 0] = np.where(np.abs(x[:, :, 0]) < 1.0, 2.0, x[:, :, 0])   # a block maximum near 2
    x = x.reshape(T, -1)
    x[0] *= 2.0 ** 12
    x[T - 1] *= 2.0 ** -4
    li = _with(li, x=IN.f32_to_bf16(x.astype(np.float32)), **_spread_weights(wl, 9))
    run_parity(li, _layer(li), per_token=np.ones(T, bool))
