"""Expert parallelism: the dispatch / combine plumbing (host side) on two gloo
ranks. Each rank holds half the tokens and half the routed experts; rows go to
their expert's owner and come back for the combine. The result must equal
the single-process layer: exactly with a stand-in expert function, and to
fp64 rounding with the oracle's experts (the oracle reads the rows each rank
actually received)."""
import os
import socket

import numpy as np
import pytest

import inputs as IN

torch = pytest.importorskip("torch")


def _ep():
    from mxfp4_routed_expert_v4moe_b200 import ep
    return ep


# ----------------------------------------------------------------- the plan

def test_dispatch_plan_orders_slots_by_owner_then_expert_stably():
    ep = _ep()
    ids = np.array([[5, 1, 14], [1, 9, 5], [12, 3, 1], [5, 14, 0]], np.int32)
    plan = ep.dispatch_plan(ids, E=16, world=2)
    flat = ids.reshape(-1)
    owner = flat // 8
    assert plan.send_counts.tolist() == [int((owner == 0).sum()), int((owner == 1).sum())]
    o, e = owner[plan.send_order], flat[plan.send_order]
    keys = list(zip(o, e, plan.send_order))
    assert keys == sorted(keys)                      # (owner, expert, home slot)
    assert sorted(plan.send_order.tolist()) == list(range(flat.size))
    assert np.array_equal(plan.send_experts, e)


def test_owner_blocks_and_bad_ids():
    ep = _ep()
    assert ep.experts_per_rank(256, 8) == 32
    assert ep.experts_per_rank(10, 4) == 3            # ceil: the last rank owns fewer
    assert ep.owner_of(np.array([0, 2, 3, 9]), 10, 4).tolist() == [0, 0, 1, 3]
    with pytest.raises(ValueError):
        ep.owner_of(np.array([10]), 10, 4)
    with pytest.raises(ValueError):
        ep.owner_of(np.array([-1]), 10, 4)


def test_recv_expert_order_groups_by_expert_in_arrival_order():
    ep = _ep()
    e = np.array([9, 8, 9, 10, 8, 8])
    order = ep.recv_expert_order(e)
    assert order.tolist() == [1, 4, 5, 0, 2, 3]


# ----------------------------------------------------------------- two ranks

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WL = IN.Workload("ep", T=24, H=256, E=16, I=128, Is=128, bias_std=0.05, seed=31)


def _bf16_vals(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import oracle as O
    from mxfp4_routed_expert_v4moe_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        li = IN.make_layer_inputs(WL)
        ids, w, _, _ = O.Layer(li).route()
        T = WL.T
        home = np.arange(rank * T // world, (rank + 1) * T // world)
        x = torch.as_tensor(_bf16_vals(li.x[home]))
        res = {}

        # stand-in experts: exact arithmetic in fp64
        def fake_expert(e, rows):
            return rows * (e + 1) + e

        out = ep.ep_moe(x, ids[home], w[home], WL.E, fake_expert, lambda r: 0.5 * r)
        ref = 0.5 * x
        for j in range(WL.k):
            ref = ref + torch.as_tensor(w[home, j:j + 1]) * (x * (torch.as_tensor(ids[home, j:j + 1]) + 1)
                                                              + torch.as_tensor(ids[home, j:j + 1]).double())
        res["fake_equal"] = bool(torch.equal(out, ref))

        # the oracle's experts on the rows this rank received
        def oracle_rows(rows, k, Is):
            bits = IN.f32_to_bf16(rows.numpy().astype(np.float32)).reshape(rows.shape)
            wl = WL.replace(T=rows.shape[0], k=k, Is=Is)
            d = dict(li.__dict__)
            d.update(wl=wl, x=np.ascontiguousarray(bits), bias=li.bias[:WL.E])
            return O.Layer(IN.LayerInputs(**d))

        def oracle_expert(e, rows):
            n = rows.shape[0]
            lay = oracle_rows(rows, 1, 0)
            y = lay.moe_tokens(np.arange(n), np.full((n, 1), e, np.int32), np.ones((n, 1)))
            return torch.as_tensor(y)

        def oracle_shared(rows):
            n = rows.shape[0]
            lay = oracle_rows(rows, WL.k, WL.Is)
            return torch.as_tensor(lay.moe_tokens(np.arange(n), np.zeros((n, WL.k), np.int32),
                                                  np.zeros((n, WL.k))))

        out = ep.ep_moe(x, ids[home], w[home], WL.E, oracle_expert, oracle_shared).numpy()
        full = O.Layer(li).moe_tokens(home, ids, w)
        res["oracle_rel"] = float(np.linalg.norm(out - full) / np.linalg.norm(full))
        res["oracle_maxabs"] = float(np.abs(out - full).max() / np.abs(full).max())
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_ep_dispatch_combine_two_gloo_ranks_match_the_single_process_layer():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = dict(q.get(timeout=300) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    for r in (0, 1):
        assert res[r]["fake_equal"], r
        assert res[r]["oracle_rel"] < 1e-12 and res[r]["oracle_maxabs"] < 1e-12, res[r]
