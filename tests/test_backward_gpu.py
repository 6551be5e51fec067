"""GPU parity of the layer's backward (latent_moe_backward, through the C ABI)
against the fp64 oracle backward on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import synth
from harness import device_inputs, host, ldims, odims, oracle_weights, prepare, rel_err

pytestmark = pytest.mark.gpu

lm = pytest.importorskip("sigmoid_top_routing_latentmoe_b200")

W = synth.WORKLOADS
# fp32 recomputation and sums against fp64, relative to each gradient's largest entry
GRAD_TOL = 1e-4

PAIRS = [("dx", "x"), ("dw_down", "w_down"), ("dw_router", "w_router"), ("dw_up", "w_up"),
         ("drms_weight", "rms_weight"), ("dw_g", "w_g"), ("dw_u", "w_u"), ("dw_o", "w_o"),
         ("dws_g", "ws_g"), ("dws_u", "ws_u"), ("dws_o", "ws_o")]


def _grads(wl):
    N, d, L, R, F, S, G = (wl.n_tokens, wl.d, wl.latent, wl.n_routed, wl.ff_routed, wl.n_shared,
                           wl.ff_shared)
    shapes = {"dx": (N, d), "dw_down": (L, d), "dw_router": (R, d), "dw_up": (d, L),
              "drms_weight": (L,), "dw_g": (R, F, L), "dw_u": (R, F, L), "dw_o": (R, L, F)}
    if S:
        shapes.update(dws_g=(S, G, d), dws_u=(S, G, d), dws_o=(S, d, G))
    return {n: torch.full(s, float("nan"), dtype=torch.float32, device="cuda")
            for n, s in shapes.items()}


def _run(wl, dev, dy):
    dims = ldims(wl)
    ws = lm.alloc_backward_workspace(dims)
    g = _grads(wl)
    lm.latent_moe_backward(dims, dev, dev["x"], dy, g, ws)
    torch.cuda.synchronize()
    assert lm.get_device_status(ws) == lm.OK
    return g


# The last two token counts make the weight-gradient contractions (K = tokens)
# run as K slices with a shorter last slice, in the fp32 and the bf16 kernels.
CASES = [("toy_fp32", 128, 0), ("halfb_uniform", 64, 0), ("halfb_skewed", 48, 0),
         ("halfb_uniform", 40, 1), ("mid", 16, 0), ("toy_fp32", 1000, 0), ("halfb_uniform", 300, 0)]


@pytest.mark.parametrize("name,n,router", CASES)
def test_backward_parity(name, n, router):
    wl = W[name].with_tokens(n).replace(router=router)
    inp = prepare(wl)
    dev = device_inputs(inp)
    dy_np = synth.normal(1, "dy", (n, wl.d), 1.0, dtype="bf16" if wl.dtype == "bf16" else "f32")
    dy = device_inputs({"x": dy_np})["x"]
    g = _run(wl, dev, dy)
    ref = oracle.backward(odims(wl), oracle_weights(inp), synth.to_f32(inp["x"]),
                          synth.to_f32(dy_np))
    for gname, oname in PAIRS:
        if gname not in g:
            continue
        got = host(g[gname]).astype(np.float64)
        assert np.isfinite(got).all(), gname
        assert rel_err(got, ref[oname]) <= GRAD_TOL, (gname, rel_err(got, ref[oname]))
    # experts no token selected: exactly 0
    ids, _, _, _ = oracle.route(odims(wl), synth.to_f32(inp["x"]), synth.to_f32(inp["w_router"]),
                                inp["expert_bias"])
    unused = sorted(set(range(wl.n_routed)) - set(ids.reshape(-1).tolist()))
    for e in unused:
        for gname in ("dw_g", "dw_u", "dw_o", "dw_router"):
            assert (host(g[gname])[e] == 0).all(), (gname, e)


def test_backward_is_deterministic_and_unselected_experts_are_zero():
    wl = W["halfb_skewed"].with_tokens(96)   # skewed routing leaves experts unselected
    inp = prepare(wl)
    dev = device_inputs(inp)
    dy = device_inputs({"x": synth.normal(2, "dy", (96, wl.d), 1.0)})["x"]
    g1 = _run(wl, dev, dy)
    g2 = _run(wl, dev, dy)
    for n in g1:
        assert torch.equal(g1[n], g2[n]), n
    counts = np.bincount(oracle.route(odims(wl), synth.to_f32(inp["x"]),
                                      synth.to_f32(inp["w_router"]),
                                      inp["expert_bias"])[0].reshape(-1), minlength=wl.n_routed)
    assert (counts == 0).any()
    for e in np.nonzero(counts == 0)[0]:
        assert (host(g1["dw_o"])[e] == 0).all() and (host(g1["dw_g"])[e] == 0).all()
