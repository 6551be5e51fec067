"""moe_dispatch_noalloc: the permutation for callers that cannot provide device
scratch memory (for example a plugin host that hands a kernel only its
tensors, or a capped memory pool that is full).  Its scratch is a fixed array
inside the library, shared by every call.

Checked through the C ABI against moe_dispatch (the workspace entry point) on
two calls in a row with different sizes, so that contents left in the shared
array by the first call cannot leak into the second.  The permutation is
integer work: the comparison is exact.  This file runs last in the suite
(a failure here leaves every other test already run) and also alone."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

lm = pytest.importorskip("sigmoid_top_routing_latentmoe_b200")


def _ids(N, k, R, seed):
    rng = np.random.default_rng(seed)
    return np.argsort(rng.random((N, R)), axis=1)[:, :k].astype(np.int32)


def _outputs(N, k, R):
    return (torch.empty(R, dtype=torch.int32, device="cuda"),
            torch.empty(R + 1, dtype=torch.int32, device="cuda"),
            torch.empty(N * k, dtype=torch.int32, device="cuda"),
            torch.empty(N, k, dtype=torch.int32, device="cuda"))


def _both(N, k, R, seed):
    ids = torch.from_numpy(_ids(N, k, R, seed)).cuda()
    dims = lm.make_dims(N, 64, 32, R, k, 0, 64, 64)
    ref = _outputs(N, k, R)
    ws = lm.alloc_workspace(dims)
    lm.moe_dispatch(dims, ids, *ref, ws)
    got = _outputs(N, k, R)
    for t in got:
        t.fill_(-1)
    lm.moe_dispatch_noalloc(dims, ids, *got)
    torch.cuda.synchronize()
    return ref, got


def test_noalloc_matches_workspace_dispatch_twice():
    # first call: a large histogram area; second: smaller sizes, different R
    for (N, k, R, seed) in [(8192, 16, 896, 1), (1000, 2, 16, 2)]:
        ref, got = _both(N, k, R, seed)
        for a, b in zip(ref, got):
            assert torch.equal(a, b)


def test_noalloc_rejects_sizes_beyond_its_array():
    d = lm.make_dims(4_000_000, 64, 32, 4096, 8, 0, 64, 64)   # ~31 MB of histograms
    st = lm._lib.moe_dispatch_noalloc(ctypes.byref(d), None, None, None, None, None, None)
    assert st == lm.EUNSUPPORTED
    assert "fixed array" in lm._lib.lmoe_last_error().decode()


def test_noalloc_out_of_range_id_is_dropped_with_inv_pair_minus_one():
    """A pair whose id is outside [0, R) takes no sorted slot: counts and offsets
    cover the valid pairs only, its inv_pair entry is -1, and the valid pairs
    are permuted as if it were absent (bit for bit against a stable argsort)."""
    N, k, R = 300, 2, 16
    ids_np = _ids(N, k, R, 3)
    ids_np[17, 1] = R + 5                      # one out-of-range id
    flat = ids_np.reshape(-1)
    valid = (flat >= 0) & (flat < R)
    counts_ref = np.bincount(flat[valid], minlength=R).astype(np.int32)
    offsets_ref = np.concatenate([[0], np.cumsum(counts_ref)]).astype(np.int32)
    order = np.flatnonzero(valid)[np.argsort(flat[valid], kind="stable")]
    inv_ref = np.full(N * k, -1, dtype=np.int32)
    inv_ref[order] = np.arange(order.size, dtype=np.int32)
    perm_ref = (order // k).astype(np.int32)

    ids = torch.from_numpy(ids_np).cuda()
    dims = lm.make_dims(N, 64, 32, R, k, 0, 64, 64)
    got = _outputs(N, k, R)
    for t in got:
        t.fill_(-7)
    lm.moe_dispatch_noalloc(dims, ids, *got)
    torch.cuda.synchronize()
    counts, offsets, perm, inv = (t.cpu().numpy() for t in got)
    np.testing.assert_array_equal(counts, counts_ref)
    np.testing.assert_array_equal(offsets, offsets_ref)
    np.testing.assert_array_equal(inv.reshape(-1), inv_ref)
    np.testing.assert_array_equal(perm[:order.size], perm_ref)
