"""lsh_sort_noalloc: the sort for callers that cannot provide a workspace
(a host framework that owns all device memory, or a loop that cannot afford
cudaMalloc's implicit synchronisation). It uses the library's own 16 MiB
scratch array instead of caller memory.

The GPU test calls it through the C ABI twice in a row, on two different
problems, and checks each permutation against lsh_sort with a caller
workspace (bit-exact, the bar of every integer result here). This file is
collected last so that a run stopping at the first failure has already run
every other test."""
import ctypes

import numpy as np
import pytest

from efficient_transformer_lsh_b200 import _lib


def _problem(B, H, L, n_buckets, n_rounds):
    return _lib.make_problem(B, H, L, 64, n_buckets, n_rounds, 64, True, 0.125, "bf16")


def test_too_large_problem_is_rejected_before_launch():
    # 8 heads x 4 rounds x 2^20 positions with 8192 buckets needs 32 MiB of
    # sort scratch (per-block bucket counts)
    p = _problem(1, 8, 1 << 20, 8192, 4)
    assert _lib.lsh_sort_workspace_size(p) > _lib.SORT_NOALLOC_SCRATCH_BYTES
    FAKE = 1 << 20
    assert _lib.lib().lsh_sort_noalloc(ctypes.byref(p), FAKE, FAKE, None) == 3  # LSH_ERR_WORKSPACE
    bad = _lib.lsh_problem(1, 1, 128, 64, 15, 1, 64, 1, 0.125, 1)              # odd bucket count
    assert _lib.lib().lsh_sort_noalloc(ctypes.byref(bad), FAKE, FAKE, None) == 1


@pytest.mark.gpu
def test_sort_noalloc_matches_sort_two_calls():
    import torch
    dev = torch.device("cuda")
    rng = np.random.default_rng(7)
    # different problems back to back: each reuses the scratch that still
    # holds the previous one's counters; the last has more than 8192 buckets,
    # so it takes the other sort path, which must clear its counters itself
    shapes = [(1, 8, 65536, 1024, 4), (2, 3, 12288 + 64, 192, 5), (1, 2, 65536, 16384, 1)]
    for B, H, L, nb, nr in shapes:
        p = _problem(B, H, L, nb, nr)
        assert _lib.lsh_sort_workspace_size(p) <= _lib.SORT_NOALLOC_SCRATCH_BYTES
        bucket = torch.from_numpy(rng.integers(0, nb, size=(B, H, nr, L), dtype=np.int32)).to(dev)
        perm_ref = torch.empty_like(bucket)
        perm_na = torch.full_like(bucket, -1)
        ws_bytes = _lib.lsh_sort_workspace_size(p)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        _lib.lsh_sort(p, bucket, perm_ref, ws, ws_bytes)
        _lib.lsh_sort_noalloc(p, bucket, perm_na)
        torch.cuda.synchronize()
        assert _lib.lsh_device_status() == 0
        assert torch.equal(perm_na, perm_ref)
        # and it is the stable sort by bucket
        a = perm_na.reshape(-1, L).cpu().numpy()
        k = bucket.reshape(-1, L).cpu().numpy()
        for s in range(0, a.shape[0], max(1, a.shape[0] // 4)):
            assert np.array_equal(a[s], np.argsort(k[s], kind="stable"))
