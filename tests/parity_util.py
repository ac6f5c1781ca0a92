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
