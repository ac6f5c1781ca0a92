"""Failure detection on the GPU without a fault: device-side waits are
bounded. Word 1 of the workspace's status block, when non-zero, makes the
decode expert kernel wait on a barrier that nothing arrives at, capped at that
many polls; the wait gives up, the kernel sets the timeout bit of the status
word and returns, and the context stays usable. Clearing the status block
disarms it."""
import numpy as np
import pytest

import inputs as IN
import oracle as O
from parity_util import assert_close, bf16_to_f64, host_threads, upload_activations

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def test_router_wait_gives_up_then_the_next_call_is_exact():
    import mxfp4_routed_expert_v4moe_b200 as V
    from mxfp4_routed_expert_v4moe_b200 import MoELayer
    wl = IN.Workload("timeout", T=2, H=1024, E=32, I=512, Is=512, seed=3)
    li = IN.make_layer_inputs(wl)
    layer = MoELayer.from_host(li)
    x, bias, _, _ = upload_activations(li)
    ws = layer.workspace(wl.T)
    assert V.v4moe_clear_device_status(ws) == V.V4MOE_OK
    ws[:256].view(torch.int32)[1] = 2000   # arm: a wait that can never be met
    layer(x, bias)
    assert V.v4moe_read_device_status(ws) == V.V4MOE_ERR_TIMEOUT
    # the context is intact and the counters were reset: clear and run again
    assert V.v4moe_clear_device_status(ws) == V.V4MOE_OK
    for _ in range(2):
        out = layer(x, bias)
        assert V.v4moe_read_device_status(ws) == V.V4MOE_OK
    ids = layer.buffers(wl.T)["topk_ids"].cpu().numpy()
    w = layer.buffers(wl.T)["topk_w"].cpu().numpy().astype(np.float64)
    ref = O.Layer(li).moe_tokens(np.arange(wl.T), ids, w, threads=host_threads())
    assert_close(bf16_to_f64(out), ref, "after timeout")
