"""v4moe_permute_static: the permutation for callers that cannot allocate
device memory (their runtime planned all device memory up front, or they must
not reach an allocator). Its scratch is a fixed array inside the library; it
must give exactly what v4moe_permute gives with a caller workspace, call after
call, since every call reuses the same array."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _ids(T, k, E, seed):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    ids[: T // 3, 0] = 5  # a hot expert
    return ids.reshape(T, k)


def _run(V, cfg, ids, static):
    T, k = ids.shape
    E = cfg.n_experts
    d = torch.from_numpy(np.ascontiguousarray(ids)).cuda()
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    ss = torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda")
    sp = torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda")
    if static:
        rc = V.v4moe_permute_static(cfg, T, d, counts, offsets, ss, sp)
    else:
        nbytes = V.v4moe_workspace_bytes(cfg, T)
        ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        rc = V.v4moe_permute(cfg, T, d, counts, offsets, ss, sp, ws, nbytes)
    assert rc == V.V4MOE_OK, V.status_string(rc)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (counts, offsets, ss, sp)]


def test_static_scratch_permute_matches_workspace_permute_call_after_call():
    import mxfp4_routed_expert_v4moe_b200 as V
    cfg = V.make_config(4096, 2048, 256, 6, 2048)
    bad = _ids(300, 6, 256, 3)
    bad[17, 2] = 256      # out of range: skipped by both entry points
    bad[40, 0] = -3
    # Both multi-chunk calls use the shared chunk tables with different chunk
    # counts (27, then 15), so stale contents from one call would show in the
    # next; then the single-CTA path, an empty batch, and bad ids.
    for ids in (_ids(9000, 6, 256, 1), _ids(5000, 6, 256, 2), _ids(37, 6, 256, 4),
                np.zeros((0, 6), np.int32), bad, _ids(9000, 6, 256, 5)):
        want = _run(V, cfg, ids, static=False)
        got = _run(V, cfg, ids, static=True)
        for a, b in zip(got, want):
            assert np.array_equal(a, b)
    # sizes beyond the fixed array, and configs v4moe_permute refuses, are
    # refused before any launch
    assert V.v4moe_permute_static(cfg, 65536 // 6 + 1, 16, 16, 16, 16, 16) == V.V4MOE_ERR_INVALID_ARG
    odd = V.make_config(4096, 2048 + 64, 256, 6, 2048)   # inter not a multiple of 128
    assert V.v4moe_permute_static(odd, 4, 16, 16, 16, 16, 16) == V.V4MOE_ERR_INVALID_ARG
