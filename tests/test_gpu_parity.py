"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs. Integer outputs bit-exact (learned-routing tokens whose
6th-vs-7th biased-score margin is below 1e-4 are counted and left out of the id
comparison); float outputs within rel-L2 5e-3 and max-abs 1e-2 * max|ref|."""
import numpy as np
import pytest

import inputs as IN
import oracle as O
from parity_util import assert_close, bf16_to_f64, host_threads, run_parity, upload_activations

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _layer(li):
    from mxfp4_routed_expert_v4moe_b200 import MoELayer
    return MoELayer.from_host(li)


@pytest.fixture(scope="module")
def full_weights():
    """Full-size weights (identical for every full-size workload, seed 0)."""
    return IN.make_weights(IN.WORKLOADS["decode_b1"])


def test_tiny_layer_all_tokens():
    li = IN.make_layer_inputs(IN.WORKLOADS["tiny"])
    rep = {}
    run_parity(li, _layer(li), report=rep)
    print("tiny", rep)


@pytest.mark.parametrize("T", [1, 7, 37, 300])
def test_ragged_token_counts_multi_tile(T):
    wl = IN.Workload("mid", T=T, H=1024, E=32, I=512, Is=256, bias_std=0.05, seed=11)
    li = IN.make_layer_inputs(wl)
    run_parity(li, _layer(li))


@pytest.mark.parametrize("T,routing", [(600, "learned"), (1100, "hash")])
def test_prefill_sized_ragged(T, routing):
    """Token-major block-scaled tiles with the shared expert on its own f16
    GEMM (the combine in its epilogue); ragged last token tiles."""
    if routing == "hash":
        wl = IN.Workload("pre_hash", T=T, H=512, E=16, I=512, Is=256, routing="hash", vocab=3000, seed=9)
    else:
        wl = IN.Workload("pre_mid", T=T, H=1024, E=32, I=512, Is=512, bias_std=0.05, seed=13)
    li = IN.make_layer_inputs(wl)
    run_parity(li, _layer(li))


@pytest.mark.parametrize("T", [5, 200])
def test_hash_routing_small(T):
    wl = IN.Workload("hash_small", T=T, H=512, E=16, I=256, Is=256, routing="hash", vocab=1000,
                     seed=5)
    li = IN.make_layer_inputs(wl)
    run_parity(li, _layer(li))


@pytest.mark.parametrize("T", [1, 5, 8])
def test_decode_hash_routing(T):
    """Hash routing on the decode kernels (at most 8 tokens, K a power of two
    from 512): the router's leader reads the token ids and the table."""
    wl = IN.Workload("dec_hash", T=T, H=1024, E=32, I=512, Is=256, routing="hash", vocab=1000, seed=23)
    li = IN.make_layer_inputs(wl)
    run_parity(li, _layer(li))


@pytest.mark.parametrize("T", [2, 8])
def test_decode_more_experts_than_router_warps(T):
    """E = 320: the decode router's warps score a second row each, and the
    selection holds 10 scores per lane."""
    wl = IN.Workload("dec_e320", T=T, H=1024, E=320, I=512, Is=256, bias_std=0.05, seed=29)
    li = IN.make_layer_inputs(wl)
    run_parity(li, _layer(li))


@pytest.mark.parametrize("T", [3, 50])
def test_no_shared_expert_and_k1(T):
    wl = IN.Workload("noshared", T=T, H=256, E=8, k=1, I=128, Is=0, seed=2)
    li = IN.make_layer_inputs(wl)
    run_parity(li, _layer(li))


def test_all_tokens_on_one_expert_set():
    wl = IN.Workload("skew", T=129, H=512, E=16, I=256, Is=256, seed=4)
    li = IN.make_layer_inputs(wl)
    layer = _layer(li)
    ids = np.tile(np.array([[2, 3, 5, 7, 11, 13]], np.int32), (wl.T, 1))
    w = np.full((wl.T, 6), 0.25, np.float32)
    x, *_ = upload_activations(li)
    ids_d = torch.from_numpy(ids).cuda()
    _, offsets, ss, sp = layer.permute(ids_d)
    out = layer.forward(x, ids_d, torch.from_numpy(w).cuda(), offsets, ss, sp)
    torch.cuda.synchronize()
    ref = O.Layer(li).moe_tokens(np.arange(wl.T), ids, w.astype(np.float64), threads=host_threads())
    assert_close(bf16_to_f64(out), ref, "skew")


def test_empty_batch():
    wl = IN.Workload("empty", T=0, H=512, E=16, I=256, Is=256)
    li = IN.make_layer_inputs(wl.with_T(4))
    layer = _layer(li)
    x = torch.empty((0, 512), dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros(16, device="cuda")
    out = layer(x, bias)
    torch.cuda.synchronize()
    assert out.shape == (0, 512)
    assert not layer.buffers(0)["offsets"].any().item()


def test_bad_ids_flagged_not_faulting():
    import mxfp4_routed_expert_v4moe_b200 as V
    wl = IN.Workload("bad", T=16, H=512, E=16, I=256, Is=256)
    li = IN.make_layer_inputs(wl)
    layer = _layer(li)
    ws = layer.workspace(16)
    assert V.v4moe_clear_device_status(ws) == 0
    assert V.v4moe_read_device_status(ws) == V.V4MOE_OK
    ids = np.zeros((16, 6), np.int32)
    ids[:, :] = np.arange(6)
    ids[3, 2] = 16      # out of range
    ids[5, 0] = -1      # negative
    layer.permute(torch.from_numpy(ids).cuda())
    assert V.v4moe_read_device_status(ws) == V.V4MOE_ERR_DATA
    V.v4moe_clear_device_status(ws)
    assert V.v4moe_read_device_status(ws) == V.V4MOE_OK
    # hash routing with a token id beyond the table
    wlh = IN.Workload("badh", T=16, H=512, E=16, I=256, Is=256, routing="hash", vocab=50)
    lih = IN.make_layer_inputs(wlh)
    layh = _layer(lih)
    x, _, tok, tab = upload_activations(lih)
    tok[4] = 50
    ids_g, w_g = layh.route(x, None, tok, tab)
    assert V.v4moe_read_device_status(layh.workspace(16)) == V.V4MOE_ERR_DATA
    assert float(w_g[4].abs().sum().item()) == 0.0


@pytest.mark.parametrize("name,n_tok", [("decode_b1", None), ("decode_b64", None),
                                        ("prefill_1024", 256), ("prefill_4096", 256),
                                        ("hash_16384", 256)])
def test_full_size_workloads(name, n_tok, full_weights):
    """The five workloads at full size, plus a 1024-token prefill chunk whose
    experts average 24 slots (the weight-major block-scaled GEMM with 128-slot
    token tiles, and the shared expert's f16 GEMM). Float outputs on 256
    sampled tokens for the large batches, always including tokens of the
    hottest expert."""
    wl = IN.WORKLOADS[name] if name in IN.WORKLOADS else IN.WORKLOADS["prefill_4096"].replace(name=name, T=1024)
    li = IN.make_layer_inputs(wl, weights=full_weights)
    rep = {}
    run_parity(li, _layer(li), n_float_tokens=n_tok, report=rep)
    print(name, rep)
