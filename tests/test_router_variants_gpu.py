"""GPU parity of the routing rule switch (the pages' earlier router: top-k of the
raw logits, softmax weights) and of the router balancing losses, through the C
ABI against the CPU oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from harness import device_inputs, host, ldims, odims, oracle_weights, prepare, rel_err, y_tol

pytestmark = pytest.mark.gpu

lm = pytest.importorskip("sigmoid_top_routing_latentmoe_b200")

W = synth.WORKLOADS
LOSS_RTOL = 1e-4   # fp32 logits of bf16 inputs against the fp64 oracle
# Softmax weights move by p_i (dl_i - sum_j p_j dl_j) for logit errors dl, and
# fp32 logits accumulated over d <= 7168 bf16 products carry |dl| of order
# 1e-5; the K3 weights s_i / sum s see dl only through s(1 - s) <= 1/4.  So the
# softmax weights get 1e-5 (the largest difference seen, at mid: 1.02e-6).
SOFTMAX_P_TOL = 1e-5


def _forward(wl, dev):
    dims = ldims(wl)
    ws = lm.alloc_workspace(dims)
    N = wl.n_tokens
    y = torch.empty(N, wl.d, dtype=dev["x"].dtype, device="cuda")
    ids = torch.empty(N, wl.top_k, dtype=torch.int32, device="cuda")
    probs = torch.empty(N, wl.top_k, dtype=torch.float32, device="cuda")
    lm.latent_moe_forward(dims, dev, dev["x"], y, ws, ids, probs)
    torch.cuda.synchronize()
    assert lm.get_device_status(ws) == lm.OK
    return dims, ws, y, ids, probs


# (workload, tokens): R <= 32 routes in the x-pass epilogue (bf16) or the
# warp-per-token GEMV (fp32, standalone); R > 32 through logits + top-k kernel
CASES = [("toy_fp32", 128), ("halfb_uniform", 300), ("mid", 136), ("k3_width", 24)]


@pytest.mark.parametrize("name,n", CASES)
def test_route_softmax_topk(name, n):
    wl = W[name].with_tokens(n).replace(router=1)
    inp = prepare(wl)
    dev = device_inputs(inp)
    dims = ldims(wl)
    ws = lm.alloc_workspace(dims)
    ids = torch.empty(n, wl.top_k, dtype=torch.int32, device="cuda")
    probs = torch.empty(n, wl.top_k, dtype=torch.float32, device="cuda")
    lm.moe_route(dims, dev["x"], dev["w_router"], dev["expert_bias"], ids, probs, ws)
    torch.cuda.synchronize()
    r_ids, r_probs, _, _ = oracle.route(odims(wl), synth.to_f32(inp["x"]),
                                        synth.to_f32(inp["w_router"]), inp["expert_bias"])
    np.testing.assert_array_equal(host(ids), r_ids)
    np.testing.assert_allclose(host(probs), r_probs, atol=SOFTMAX_P_TOL, rtol=0)


@pytest.mark.parametrize("name,n", CASES)
def test_forward_softmax_topk(name, n):
    wl = W[name].with_tokens(n).replace(router=1)
    inp = prepare(wl)
    dev = device_inputs(inp)
    _, _, y, ids, probs = _forward(wl, dev)
    ref = oracle.forward(odims(wl), oracle_weights(inp), synth.to_f32(inp["x"]))
    np.testing.assert_array_equal(host(ids), ref["ids"])
    np.testing.assert_allclose(host(probs), ref["probs"], atol=SOFTMAX_P_TOL, rtol=0)
    assert rel_err(host(y), ref["y"]) <= y_tol(wl)


def _check_losses(got, ref, R):
    assert got[0] == pytest.approx(ref["aux"], rel=LOSS_RTOL)
    assert got[1] == pytest.approx(ref["z"], rel=LOSS_RTOL)
    np.testing.assert_allclose(got[2:2 + R], ref["frac"], rtol=1e-6, atol=0)
    np.testing.assert_allclose(got[2 + R:], ref["prob_mean"], rtol=LOSS_RTOL, atol=0)


@pytest.mark.parametrize("name,n,router", [("toy_fp32", 128, 0), ("halfb_uniform", 300, 0),
                                           ("halfb_skewed", 520, 0), ("mid", 136, 0),
                                           ("halfb_uniform", 300, 1), ("k3_width", 24, 0)])
def test_router_losses_after_forward(name, n, router):
    """The losses from the logits the forward leaves in its workspace."""
    wl = W[name].with_tokens(n).replace(router=router)
    inp = prepare(wl)
    dev = device_inputs(inp)
    dims, ws, _, ids, _ = _forward(wl, dev)
    out = torch.empty(2 + 2 * wl.n_routed, dtype=torch.float32, device="cuda")
    lm.moe_router_losses(dims, ids, out, ws)
    torch.cuda.synchronize()
    assert lm.get_device_status(ws) == lm.OK
    ref = oracle.router_losses(odims(wl), synth.to_f32(inp["x"]), synth.to_f32(inp["w_router"]),
                               host(ids))
    _check_losses(host(out).astype(np.float64), ref, wl.n_routed)


def test_router_losses_collapsed_case_of_the_pages():
    """The pages' collapse test on the GPU: router rows 0 := 1, 1 := 0.5, x = 1
    (all exact in bf16); aux = R (sigma(32) + sigma(16)) / 2 > 1.2 and z > 0."""
    n, d, R, k = 64, 32, 8, 2
    wl = synth.Workload("collapsed", n, d, 16, R, k, 24, 1, 24, "bf16")
    dims = ldims(wl)
    ws = lm.alloc_workspace(dims)
    x = torch.ones(n, d, dtype=torch.bfloat16, device="cuda")
    w_r = torch.zeros(R, d, dtype=torch.bfloat16, device="cuda")
    w_r[0], w_r[1] = 1.0, 0.5
    ids = torch.empty(n, k, dtype=torch.int32, device="cuda")
    probs = torch.empty(n, k, dtype=torch.float32, device="cuda")
    lm.moe_route(dims, x, w_r, None, ids, probs, ws)
    out = torch.empty(2 + 2 * R, dtype=torch.float32, device="cuda")
    lm.moe_router_losses(dims, ids, out, ws)
    torch.cuda.synchronize()
    got = host(out).astype(np.float64)
    assert (host(ids) == np.array([0, 1], np.int32)).all()
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))
    assert got[0] == pytest.approx(R * (sig(32.0) + sig(16.0)) / 2.0, rel=1e-6)
    assert got[1] == pytest.approx((32.0 + math.log1p(math.exp(-16.0))) ** 2, rel=1e-6)
    assert got[0] > 1.2 and got[1] > 0.0


def test_router_losses_from_given_logits():
    """Logits passed in explicitly (row stride ld > R) give the oracle's losses of
    the same logits."""
    rng = np.random.default_rng(9)
    n, R, k, ld = 777, 24, 3, 40
    wl = synth.Workload("given", n, 64, 32, R, k, 64, 0, 64, "bf16")
    dims = ldims(wl)
    ws = lm.alloc_workspace(dims)
    x = rng.standard_normal((n, 64)).astype(np.float32)
    w_r = (rng.standard_normal((R, 64)) * 0.3).astype(np.float32)
    ids_np, _, _, _ = oracle.route(odims(wl), x, w_r)
    logits = np.zeros((n, ld), np.float32)
    logits[:, :R] = (x.astype(np.float64) @ w_r.astype(np.float64).T).astype(np.float32)
    out = torch.empty(2 + 2 * R, dtype=torch.float32, device="cuda")
    lm.moe_router_losses(dims, torch.from_numpy(ids_np).cuda(), out, ws,
                         logits=torch.from_numpy(logits).cuda(), ld=ld)
    torch.cuda.synchronize()
    ref = oracle.router_losses(odims(wl), x, w_r, ids_np)
    _check_losses(host(out).astype(np.float64), ref, R)
