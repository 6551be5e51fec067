"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/latent_moe.h declares, sizes workspaces, and rejects
bad arguments before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            names += re.findall(r"^LMOE_API\s+[\w\s\*]+?\b(\w+)\(", text, flags=re.M)
    return names


@pytest.fixture(scope="module")
def lm():
    import sigmoid_top_routing_latentmoe_b200 as lm
    return lm


def test_library_exports_every_declared_symbol(lm):
    names = _declared_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lm._lib, n), n
    for n in ("moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "latent_moe_forward"):
        assert n in names


def test_workspace_size_and_validation(lm):
    import torch
    d = lm.make_dims(4096, 768, 384, 16, 2, 2, 768, 1536)
    n = lm.workspace_size(d)
    assert n > 4096 * 2 * 768 * 2          # at least the permuted rows
    assert lm.workspace_size(d, host=True) > n
    bad = lm.make_dims(4096, 768, 384, 16, 17, 2, 768, 1536)   # top_k > n_routed
    with pytest.raises(lm.LmoeError):
        lm.workspace_size(bad)
    bad = lm.make_dims(4096, 770, 384, 16, 2, 2, 768, 1536)    # d not a multiple of 8
    assert lm._lib.lmoe_workspace_size(ctypes.byref(bad)) == 0
    bad = lm.make_dims(4096, 768, 384, 16, 2, 2, 768, 1536, router=2)   # no such routing rule
    assert lm._lib.lmoe_workspace_size(ctypes.byref(bad)) == 0
    ok = lm.make_dims(4096, 768, 384, 16, 2, 2, 768, 1536, router=lm.ROUTER_SOFTMAX_TOPK)
    assert lm.workspace_size(ok) == n
    out_ws = 1 << 20                                # never dereferenced: checks fail first
    st = lm._lib.moe_router_losses(ctypes.byref(d), None, 0, None, None, out_ws, 0, None)
    assert st == lm.EINVAL
    # argument errors are reported before anything touches a device
    st = lm._lib.moe_dispatch(ctypes.byref(d), None, None, None, None, None, None, 0, None)
    assert st == lm.EINVAL
    assert "NULL" in lm._lib.lmoe_last_error().decode()
    st = lm._lib.latent_moe_forward(None, None, None, None, None, None, None, None, 0, None)
    assert st == lm.EINVAL
    assert lm.status_string(lm.ETIMEOUT) == "LMOE_ETIMEOUT"


def test_misaligned_and_short_workspace_rejected(lm):
    d = lm.make_dims(8, 64, 32, 4, 2, 1, 64, 64)
    fake = 1 << 20                                   # never dereferenced: checks fail first
    w = lm.Weights(*([fake] * 11))
    st = lm._lib.latent_moe_forward(ctypes.byref(d), ctypes.byref(w), fake, fake, None, None,
                                    None, fake + 8, 10 ** 9, None)
    assert st == lm.EINVAL                           # ws not 256-byte aligned
    st = lm._lib.latent_moe_forward(ctypes.byref(d), ctypes.byref(w), fake, fake, None, None,
                                    None, fake, 16, None)
    assert st == lm.EWORKSPACE
    st = lm._lib.latent_moe_forward(ctypes.byref(d), ctypes.byref(w), fake + 4, fake, None, None,
                                    None, fake, 10 ** 9, None)
    assert st == lm.EINVAL                           # x misaligned


def test_forward_plan(lm):
    """lmoe_forward_plan: the launch plan the forward takes, decided on the host."""
    import torch
    on = lambda dims: {k for k, v in lm.forward_plan(dims).items() if v}
    halfb = lm.make_dims(4096, 768, 384, 16, 2, 2, 768, 1536)
    mid = lm.make_dims(16384, 2048, 1024, 64, 8, 1, 1024, 4096)
    k3 = lm.make_dims(8192, 7168, 3584, 896, 16, 1, 512, 2048)
    assert on(halfb) == {"combine_fused", "rows_in_scatter", "counts_in_xpass"}
    assert on(mid) == {"gemm1_pairs"}     # GEMM2 on single CTAs
    assert on(k3) == {"gemm1_pairs", "gemm2_pairs", "gemm1_wide"}
    # the x-pass counts the pairs per expert for R <= 32 when each chunk of the
    # counting sort is whole rows of 32 tokens and the rows are few enough
    assert "counts_in_xpass" in on(lm.make_dims(16384, 768, 384, 16, 2, 2, 768, 1536))
    assert "counts_in_xpass" not in on(lm.make_dims(16416, 768, 384, 16, 2, 2, 768, 1536))
    assert "counts_in_xpass" not in on(lm.make_dims(4096, 768, 384, 16, 3, 2, 768, 1536))
    assert "counts_in_xpass" in on(lm.make_dims(4096, 768, 384, 32, 8, 2, 768, 1536))
    assert "counts_in_xpass" not in on(lm.make_dims(4096, 768, 384, 33, 2, 2, 768, 1536))
    # the scatter copies the sorted z rows only from 4096 pairs on (and up to 16 MiB)
    assert on(lm.make_dims(128, 256, 128, 16, 2, 2, 256, 512, dtype=torch.float32)) == set()
    assert "rows_in_scatter" in on(lm.make_dims(2048, 768, 384, 16, 2, 2, 768, 1536))
    assert "rows_in_scatter" not in on(lm.make_dims(2047, 768, 384, 16, 2, 2, 768, 1536))
    flags = ctypes.c_int32(0)
    assert lm._lib.lmoe_forward_plan(ctypes.byref(halfb), None) == lm.EINVAL
    bad = lm.make_dims(4096, 770, 384, 16, 2, 2, 768, 1536)
    assert lm._lib.lmoe_forward_plan(ctypes.byref(bad), ctypes.byref(flags)) == lm.EINVAL
