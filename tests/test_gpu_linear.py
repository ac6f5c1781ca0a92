"""GPU parity of the W8A16 linear (config group linears_w8a16: int8 weights,
symmetric, one scale per output channel, bf16 activations) against the fp64
oracle, through the C ABI. Shapes: the attention projections as read from the
config (fused_wqa_wkv: q_lora_rank + head_dim outputs from hidden_size; wq_b:
num_attention_heads * head_dim from q_lora_rank; wo_b: hidden_size from
o_groups * o_lora_rank; the indexer's wq_b: index_n_heads * index_head_dim from
q_lora_rank) and ragged small cases. Tolerance: the layer's float bar."""
import numpy as np
import pytest

import inputs as IN
import oracle as O
from parity_util import assert_close, bf16_to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _run(T, N, K, seed, rows=None, G=1):
    import mxfp4_routed_expert_v4moe_b200 as V
    x_bits = IN.normal_bf16(seed, 1, T * G * K).reshape(T, G * K)
    q, s = IN.int8_normal(seed, 2, G * N, K, 0.02)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    qd = torch.from_numpy(q).cuda()
    sd = torch.from_numpy(s).cuda()
    out = torch.full((T, G * N), float("nan"), dtype=torch.bfloat16, device="cuda")
    if G == 1:
        nbytes = V.v4moe_linear_w8a16_workspace_bytes(T, N, K)
        ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        rc = V.v4moe_linear_w8a16(T, N, K, x, qd, sd, out, ws, nbytes)
    else:
        nbytes = V.v4moe_linear_w8a16_grouped_workspace_bytes(T, G, N, K)
        ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        rc = V.v4moe_linear_w8a16_grouped(T, G, N, K, x, qd, sd, out, ws, nbytes)
    assert rc == V.V4MOE_OK, V.status_string(rc)
    assert V.v4moe_read_device_status(ws) == V.V4MOE_OK
    got = bf16_to_f64(out)
    rows = np.arange(T) if rows is None else np.asarray(rows)
    if G == 1:
        ref = O.linear_w8a16(x_bits, q, s, rows=rows)
    else:
        ref = O.linear_w8a16_grouped(x_bits, q, s, G, rows=rows)
    assert np.isfinite(got).all()
    return got[rows], ref


@pytest.mark.parametrize("T,N,K", [(1, 64, 128), (37, 96, 128), (300, 512, 256), (130, 1536, 4096)])
def test_linear_small_and_ragged(T, N, K):
    got, ref = _run(T, N, K, seed=7)
    assert_close(got, ref, f"linear T={T} N={N} K={K}")


@pytest.mark.parametrize("name,N,K", [("wq_b", 64 * 512, 1024), ("wo_b", 4096, 8 * 1024),
                                      ("indexer_wq_b", 64 * 128, 1024)])
def test_linear_attention_projection_shapes(name, N, K):
    T = 257
    rows = [0, 1, 128, 129, 255, 256]  # both token tiles and the ragged tail
    got, ref = _run(T, N, K, seed=11, rows=rows)
    assert_close(got, ref, name)


def test_linear_tokens_outnumber_channels():
    # more tokens than channels (token tiles walked inside a weight block's
    # row of tiles) and exactly one wave of 256-row tiles with a ragged tail
    T, N, K = 4700, 1024, 192
    rows = [0, 127, 128, 2047, 4607, 4608, 4699]
    got, ref = _run(T, N, K, seed=13, rows=rows)
    assert_close(got, ref, "tokens > channels")


@pytest.mark.parametrize("T,G,N,K", [(70, 3, 96, 128), (129, 2, 288, 192)])
def test_linear_grouped_small(T, G, N, K):
    got, ref = _run(T, N, K, seed=17, G=G)
    assert_close(got, ref, f"grouped T={T} G={G} N={N} K={K}")


def test_linear_grouped_wo_a_shape():
    # wo_a: o_groups = 8 groups, o_lora_rank = 1024 outputs from the group's
    # 8 heads x head_dim 512 = 4096 inputs
    T = 257
    rows = [0, 1, 128, 129, 255, 256]
    got, ref = _run(T, 1024, 4096, seed=19, rows=rows, G=8)
    assert_close(got, ref, "wo_a")


def test_linear_empty_batch():
    import mxfp4_routed_expert_v4moe_b200 as V
    ws = torch.zeros(V.v4moe_linear_w8a16_workspace_bytes(0, 64, 128), dtype=torch.uint8, device="cuda")
    q = torch.zeros((64, 128), dtype=torch.int8, device="cuda")
    s = torch.ones(64, device="cuda")
    assert V.v4moe_linear_w8a16(0, 64, 128, None, q, s, None, ws, ws.numel()) == V.V4MOE_OK
