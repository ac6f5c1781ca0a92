"""Helpers shared by the GPU parity tests: upload, run the C-ABI steps, compare
with the oracle. Tolerances are the layer's stated acceptance bar."""
from __future__ import annotations

import os

import numpy as np

REL_L2_TOL = 5e-3          # relative L2 error of float outputs
MAX_ABS_FRAC_TOL = 1e-2    # max abs error <= 1e-2 * max |ref|
NEAR_TIE = 1e-4            # learned routing: 6th-vs-7th biased-score margin


def host_threads():
    return max(1, min(32, os.cpu_count() or 1))


def bf16_to_f64(t):
    """torch bf16 tensor (any device) -> float64 numpy."""
    import torch
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def float_errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = got - ref
    rel_l2 = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    return rel_l2, max_abs, scale


def assert_close(got, ref, what=""):
    rel_l2, max_abs, scale = float_errors(got, ref)
    assert rel_l2 <= REL_L2_TOL, f"{what}: rel-L2 {rel_l2:.3e} > {REL_L2_TOL}"
    assert max_abs <= MAX_ABS_FRAC_TOL * scale, \
        f"{what}: max-abs {max_abs:.3e} > {MAX_ABS_FRAC_TOL} * {scale:.3e}"
    return rel_l2, max_abs


def sample_tokens(T, ids, n, seed=0):
    """Deterministic token subset that always includes tokens of the hottest expert."""
    if n >= T:
        return np.arange(T, dtype=np.int32)
    rng = np.random.default_rng(seed)
    hot = np.bincount(ids.ravel(), minlength=1).argmax()
    hot_tokens = np.nonzero((ids == hot).any(axis=1))[0]
    pick = set(hot_tokens[: max(1, n // 8)].tolist())
    pick.update([0, T - 1])
    rest = rng.permutation(T)
    for t in rest:
        if len(pick) >= n:
            break
        pick.add(int(t))
    return np.array(sorted(pick), dtype=np.int32)


def upload_activations(li, device="cuda"):
    import torch
    x = torch.from_numpy(li.x).view(torch.bfloat16).to(device)
    bias = None if li.bias is None else torch.from_numpy(li.bias).to(device)
    tok = None if li.token_ids is None else torch.from_numpy(li.token_ids).to(device)
    tab = None if li.tid2eid is None else torch.from_numpy(li.tid2eid).to(device)
    return x, bias, tok, tab


def run_parity(li, layer, n_float_tokens=None, report=None, per_token=None):
    """Route, permute and forward through the C ABI (each step on the oracle's
    inputs), then the whole-layer call; every result against the oracle."""
    import torch

    import oracle as O
    import mxfp4_routed_expert_v4moe_b200 as V
    wl = li.wl
    T = wl.T
    lay = O.Layer(li)
    x, bias, tok, tab = upload_activations(li)
    # --- routing -------------------------------------------------------------
    ids_o, w_o, margin, _ = lay.route()
    ids_g, w_g = layer.route(x, bias, tok, tab)
    torch.cuda.synchronize()
    ids_g = ids_g.cpu().numpy()
    w_g = w_g.cpu().numpy().astype(np.float64)
    near = margin < NEAR_TIE
    ok = ~near
    assert np.array_equal(ids_g[ok], ids_o[ok]), "router ids differ on non-tie tokens"
    if ok.any():
        assert_close(w_g[ok], w_o[ok], "topk_w")
    # --- permutation on the oracle's ids (bit-exact) ---------------------------
    ids_dev = torch.from_numpy(ids_o).cuda()
    counts, offsets, sorted_slot, slot_pos = layer.permute(ids_dev)
    c_o, off_o, ss_o, sp_o = O.permute(ids_o, wl.E)
    torch.cuda.synchronize()
    assert np.array_equal(counts.cpu().numpy(), c_o)
    assert np.array_equal(offsets.cpu().numpy(), off_o)
    S = T * wl.k
    assert np.array_equal(sorted_slot.cpu().numpy()[:S], ss_o)
    assert np.array_equal(slot_pos.cpu().numpy()[:S], sp_o)
    # --- forward on the oracle's routing ---------------------------------------
    w32 = w_o.astype(np.float32)
    w_dev = torch.from_numpy(w32).cuda()
    out = layer.forward(x, ids_dev, w_dev, offsets, sorted_slot, slot_pos)
    torch.cuda.synchronize()
    got = bf16_to_f64(out)
    toks = sample_tokens(T, ids_o, n_float_tokens or T)
    ref = lay.moe_tokens(toks, ids_o, w32.astype(np.float64), threads=host_threads())
    rel, mabs = assert_close(got[toks], ref, f"{wl.name} out")
    if per_token is not None:   # the bar on each listed token's row alone
        for i, t in enumerate(toks):
            if per_token[t]:
                assert_close(got[t], ref[i], f"{wl.name} out, token {t}")
    # --- end to end (GPU routing) on tokens whose routing is unambiguous ------
    out2 = layer(x, bias, tok, tab)
    torch.cuda.synchronize()
    got2 = bf16_to_f64(out2)
    e2e = toks[ok[toks]]
    if e2e.size:
        assert_close(got2[e2e], ref[ok[toks]], f"{wl.name} end-to-end")
    # routing outputs of the whole-layer call (small batches route inside the
    # fused decode kernel): ids / weights as the oracle's, permutation exact
    assert V.v4moe_read_device_status(layer.workspace(T)) == V.V4MOE_OK
    b = layer.buffers(T)
    ids_l = b["topk_ids"].cpu().numpy()
    w_l = b["topk_w"].cpu().numpy().astype(np.float64)
    assert np.array_equal(ids_l[ok], ids_o[ok]), "whole-layer ids differ on non-tie tokens"
    if ok.any():
        assert_close(w_l[ok], w_o[ok], "whole-layer topk_w")
    c_l, off_l, ss_l, sp_l = O.permute(ids_l, wl.E)
    assert np.array_equal(b["counts"].cpu().numpy(), c_l)
    assert np.array_equal(b["offsets"].cpu().numpy(), off_l)
    assert np.array_equal(b["sorted_slot"].cpu().numpy()[:S], ss_l)
    assert np.array_equal(b["slot_pos"].cpu().numpy()[:S], sp_l)
    if report is not None:
        report.update(near_ties=int(near.sum()), rel_l2=rel, max_abs=mabs, tokens=len(toks))
    return got, ref


