"""Expert parallelism: the index plumbing of the token dispatch and combine.

With experts partitioned over the ranks of a group (rank r owns the
contiguous block of routed experts [r * E_r, (r + 1) * E_r), E_r =
ceil(E / world)), each token stays on its home rank for the router, the shared
expert and the output; each of its k slots (token t, choice j, slot s = t k +
j) travels to the owner of its expert and comes back as that expert's output
row. The layer's output is unchanged ("Checked in its code" rows "Mixture of
experts" and "Shared expert": out[t] = shared(x[t]) + sum_j w[t, j] *
FFN_{ids[t, j]}(x[t])); only where each product is computed moves.

This module fixes the orders every implementation of the exchange must agree
on, and runs the exchange with ``torch.distributed.all_to_all_single`` (any
backend; the tests use two gloo ranks on the CPU):

* send order: a rank's slots sorted stably by (owner rank, expert), so each
  destination receives one contiguous run, grouped by expert, and within an
  expert in home-slot order;
* receive order: source rank ascending, each source's run as sent; an owner
  processes its experts' rows in (expert, source rank, home slot) order
  (``recv_expert_order``);
* combine order: the returned rows land in slot order on the home rank, and
  out[t] adds the shared term, then w[t, j] * y[t, j] for j = 0 .. k - 1.

The fused device form (dispatch written by the router's permutation kernel
straight into the owner's receive buffer, combine written by the down
projection's epilogue into the home rank's slot rows, over NVLink peer
stores with a flag per source rank) keeps these orders; the library does not
contain it yet. Remote rows are to be stored into the receiving GPU's own
memory before any kernel reads them: no tensor-memory copy with cluster
multicast and no library GEMM is given another GPU's memory.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def experts_per_rank(E: int, world: int) -> int:
    if E <= 0 or world <= 0:
        raise ValueError("E and world must be positive")
    return (E + world - 1) // world


def owner_of(ids: np.ndarray, E: int, world: int) -> np.ndarray:
    """Owning rank of each expert id (contiguous blocks of experts_per_rank)."""
    ids = np.asarray(ids)
    if ids.size and (ids.min() < 0 or ids.max() >= E):
        raise ValueError("expert id out of range")
    return ids // experts_per_rank(E, world)


@dataclass
class DispatchPlan:
    """One rank's side of the exchange for its T home tokens."""
    send_order: np.ndarray   # [T k] home slots in send order
    send_counts: np.ndarray  # [world] slots sent to each rank
    send_experts: np.ndarray  # [T k] expert of each slot in send order


def dispatch_plan(topk_ids: np.ndarray, E: int, world: int) -> DispatchPlan:
    """Slots sorted stably by (owner, expert); counts per destination."""
    ids = np.asarray(topk_ids, np.int64).reshape(-1)
    owner = owner_of(ids, E, world)
    order = np.lexsort((np.arange(ids.size), ids, owner))  # last key sorts first
    counts = np.bincount(owner, minlength=world).astype(np.int64)
    return DispatchPlan(order.astype(np.int64), counts, ids[order])


def recv_expert_order(recv_experts: np.ndarray) -> np.ndarray:
    """Order in which an owner processes its received rows: by expert, then
    in arrival order (source rank ascending, each source's home-slot order)."""
    e = np.asarray(recv_experts, np.int64)
    return np.lexsort((np.arange(e.size), e)).astype(np.int64)


def _a2a(dist, group, send, send_counts, recv_counts):
    import torch
    recv = torch.empty((int(sum(recv_counts)),) + tuple(send.shape[1:]), dtype=send.dtype)
    dist.all_to_all_single(recv, send.contiguous(), [int(c) for c in recv_counts],
                           [int(c) for c in send_counts], group=group)
    return recv


def ep_moe(x, topk_ids, topk_w, E, expert_fn, shared_fn, group=None):
    """out [T, H] for this rank's T tokens with experts partitioned over the
    group: dispatch (counts, then rows and their expert ids), the owned
    experts' rows (expert_fn(e, rows) -> rows, one call per expert in
    ascending id), the rows sent back, and the combine in the fixed order.
    x, the returned rows and out are float torch tensors on the CPU."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    ids = np.asarray(topk_ids)
    T, k = ids.shape
    w = torch.as_tensor(np.asarray(topk_w), dtype=x.dtype)
    plan = dispatch_plan(ids, E, world)
    # counts first (every rank learns how many rows it receives from each)
    send_counts = torch.as_tensor(plan.send_counts, dtype=torch.int64)
    recv_counts = torch.empty(world, dtype=torch.int64)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    rc = recv_counts.tolist()
    sc = plan.send_counts.tolist()
    # rows (a slot's token row) and their expert ids
    rows = x[torch.as_tensor(plan.send_order // k)]
    recv_rows = _a2a(dist, group, rows, sc, rc)
    recv_e = _a2a(dist, group, torch.as_tensor(plan.send_experts), sc, rc).numpy()
    e_lo = rank * experts_per_rank(E, world)
    if recv_e.size and (recv_e.min() < e_lo or recv_e.max() >= e_lo + experts_per_rank(E, world)):
        raise RuntimeError("received a row of an expert this rank does not own")
    # the owned experts, in ascending id; results back in arrival order
    y_recv = torch.empty_like(recv_rows)
    order = recv_expert_order(recv_e)
    for e in np.unique(recv_e):
        sel = order[recv_e[order] == e]
        idx = torch.as_tensor(sel)
        y_recv[idx] = expert_fn(int(e), recv_rows[idx])
    # back to the home ranks (the reverse exchange), into slot order
    y_send = _a2a(dist, group, y_recv, rc, sc)
    y_slot = torch.empty((T * k,) + tuple(x.shape[1:]), dtype=x.dtype)
    y_slot[torch.as_tensor(plan.send_order)] = y_send
    y_slot = y_slot.reshape(T, k, *x.shape[1:])
    out = shared_fn(x).clone()
    for j in range(k):
        out += w[:, j:j + 1] * y_slot[:, j]
    return out
