"""GPU parity: the CUDA library, called through its C ABI, against the CPU
oracle on the same seeded inputs.

Routing ids, counts, offsets and the permutation must match bit for bit;
routing weights within 1e-6; y within 2e-2 * max|y_ref| for bf16 inputs and
1e-5 * max|y_ref| in fp32.  Small cases run the oracle on every token; the
full-size workloads (the launch configuration the benchmark times) compare
sampled tokens and check the permutation's defining properties on all pairs.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from harness import (P_ABS_TOL, check_permutation_properties, device_inputs, host, ldims, odims,
                     oracle_weights, prepare, rel_err, round_act, to_device, y_tol)

pytestmark = pytest.mark.gpu

lm = pytest.importorskip("sigmoid_top_routing_latentmoe_b200")

W = synth.WORKLOADS


def _run_forward(wl, dev, ws=None):
    dims = ldims(wl)
    if ws is None:
        ws = lm.alloc_workspace(dims)
    N = wl.n_tokens
    y = torch.empty(N, wl.d, dtype=dev["x"].dtype, device="cuda")
    ids = torch.empty(N, wl.top_k, dtype=torch.int32, device="cuda")
    probs = torch.empty(N, wl.top_k, dtype=torch.float32, device="cuda")
    counts = torch.empty(wl.n_routed, dtype=torch.int32, device="cuda")
    lm.latent_moe_forward(dims, dev, dev["x"], y, ws, ids, probs, counts)
    torch.cuda.synchronize()
    assert lm.get_device_status(ws) == lm.OK
    return y, ids, probs, counts, ws


def _compare_forward(wl, inp, y, ids, probs, rows=None):
    x = synth.to_f32(inp["x"])
    rows = np.arange(wl.n_tokens) if rows is None else np.asarray(rows)
    ref = oracle.forward(odims(wl, len(rows)), oracle_weights(inp), x[rows])
    np.testing.assert_array_equal(host(ids)[rows], ref["ids"])
    np.testing.assert_allclose(host(probs)[rows], ref["probs"], atol=P_ABS_TOL, rtol=0)
    err = rel_err(host(y)[rows], ref["y"])
    assert err <= y_tol(wl), f"{wl.name}: max|dy|/max|y| = {err:.3e}"
    return err, ref


# ------------------------------------------------------------ whole layer

SMALL_CASES = [
    ("toy_fp32", 128),            # the full toy workload
    ("halfb_uniform", 300),       # ragged tail: 300*2 pairs over 16 experts
    ("halfb_skewed", 520),
    ("mid", 136),
    ("k3_width", 40),             # 640 pairs over 896 experts: most experts empty
    ("halfb_skewed", 1200),       # routed GEMMs on CTA pairs: 0 to ~900 rows per expert
    ("mid", 520),                 # CTA pairs, ~65 rows per expert (second CTA's rows empty)
]


@pytest.mark.parametrize("name,n", SMALL_CASES)
def test_forward_parity_small(name, n):
    wl = W[name].with_tokens(n)
    inp = prepare(wl)
    dev = device_inputs(inp)
    y, ids, probs, counts, _ = _run_forward(wl, dev)
    _compare_forward(wl, inp, y, ids, probs)
    np.testing.assert_array_equal(host(counts), np.bincount(host(ids).reshape(-1),
                                                            minlength=wl.n_routed))


@pytest.mark.parametrize("name,sample", [("halfb_uniform", None), ("halfb_skewed", None),
                                         ("mid", 192), ("k3_width", 48), ("k3_decode", None)])
def test_forward_parity_full_size(name, sample):
    """The benchmark's workloads at full size.  Where the oracle cannot run every
    token in seconds, a fixed sample of tokens is compared (the margin is enforced
    on those rows) and routing is checked through its properties on all tokens."""
    wl = W[name]
    rows = None if sample is None else np.linspace(0, wl.n_tokens - 1, sample).astype(np.int64)
    inp = prepare(wl, margin_rows=rows)
    dev = device_inputs(inp)
    y, ids, probs, counts, ws = _run_forward(wl, dev)
    _compare_forward(wl, inp, y, ids, probs, rows)
    h_ids = host(ids)
    assert ((h_ids >= 0) & (h_ids < wl.n_routed)).all()
    assert (np.sort(h_ids, axis=1)[:, 1:] != np.sort(h_ids, axis=1)[:, :-1]).all()
    np.testing.assert_allclose(host(probs).sum(1), 1.0, atol=1e-5)
    np.testing.assert_array_equal(host(counts), np.bincount(h_ids.reshape(-1), minlength=wl.n_routed))
    # the permutation the forward built (in its workspace), on every pair
    v = lm.workspace_views(ldims(wl), ws)
    check_permutation_properties(h_ids, host(counts), host(v["offsets"]), host(v["perm"]),
                                 host(v["inv"]), wl.n_routed)
    # deterministic: a second run is bit-identical
    y2, ids2, _, _, _ = _run_forward(wl, dev, ws)
    assert torch.equal(y, y2) and torch.equal(ids, ids2)


# ---------------------------------------------------------- entry points

ROUTE_CASES = [("halfb_uniform", 333, {}), ("mid", 200, {}), ("k3_width", 64, {}),
               ("toy_fp32", 128, {}),
               # many experts: threshold + candidate sort, k up to its limit of 32
               ("mid", 150, dict(n_routed=100, top_k=32)),
               ("mid", 150, dict(n_routed=300, top_k=5)),
               ("mid", 150, dict(n_routed=2000, top_k=24)),
               ("k3_width", 96, dict(router=1))]


@pytest.mark.parametrize("name,n,over", ROUTE_CASES)
def test_route_parity(name, n, over):
    wl = W[name].with_tokens(n).replace(**over)
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
    # the softmax over the selected logits passes the logits' rounding through
    # undamped (the K3 rule's sigmoid damps it by s(1 - s) <= 1/4): 1e-5 there
    np.testing.assert_allclose(host(probs), r_probs, atol=P_ABS_TOL if wl.router == 0 else 1e-5,
                               rtol=0)


@pytest.mark.parametrize("R,k", [(896, 16), (128, 32)])
def test_route_all_keys_equal(R, k):
    """A zero router gives every expert the same key: more candidates than the
    candidate sort takes, so the k-round selection decides; ties go to the lower
    expert index (ids 0..k-1) and p = 1/k."""
    N = 40
    dims = lm.make_dims(N, 256, 128, R, k, 0, 64, 64)
    ws = lm.alloc_workspace(dims)
    x = torch.randn(N, 256, device="cuda").to(torch.bfloat16)
    w_r = torch.zeros(R, 256, device="cuda", dtype=torch.bfloat16)
    ids = torch.empty(N, k, dtype=torch.int32, device="cuda")
    probs = torch.empty(N, k, dtype=torch.float32, device="cuda")
    lm.moe_route(dims, x, w_r, None, ids, probs, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(ids), np.tile(np.arange(k, dtype=np.int32), (N, 1)))
    np.testing.assert_allclose(host(probs), 1.0 / k, rtol=0, atol=P_ABS_TOL)


def _random_ids(N, k, R, seed, skew=False):
    rng = np.random.default_rng(seed)
    if skew:   # every token picks the same k experts: one segment per expert holds all N
        return np.tile(rng.permutation(R)[:k].astype(np.int32), (N, 1))
    keys = rng.random((N, R))
    return np.argsort(keys, axis=1)[:, :k].astype(np.int32)


@pytest.mark.parametrize("N,k,R,skew", [(4096, 2, 16, False), (1000, 8, 64, False),
                                        (8192, 16, 896, False), (777, 3, 5, True),
                                        (1, 2, 4, False), (5000, 4, 4, False),
                                        (70000, 2, 16, False)])
def test_dispatch_parity_bit_exact(N, k, R, skew):
    ids_np = _random_ids(N, k, R, seed=N + k, skew=skew)
    counts_r, offsets_r, perm_r, inv_r = oracle.permute(ids_np, R)
    dims = lm.make_dims(N, 64, 32, R, k, 0, 64, 64)
    ws = lm.alloc_workspace(dims)
    ids = to_device(ids_np, "")
    counts = torch.empty(R, dtype=torch.int32, device="cuda")
    offsets = torch.empty(R + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(N * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(N, k, dtype=torch.int32, device="cuda")
    lm.moe_dispatch(dims, ids, counts, offsets, perm, inv, ws)
    torch.cuda.synchronize()
    assert lm.get_device_status(ws) == lm.OK
    np.testing.assert_array_equal(host(counts), counts_r)
    np.testing.assert_array_equal(host(offsets), offsets_r)
    np.testing.assert_array_equal(host(perm), perm_r)
    np.testing.assert_array_equal(host(inv), inv_r)
    check_permutation_properties(ids_np, host(counts), host(offsets), host(perm), host(inv), R)


def test_dispatch_flags_out_of_range_ids():
    ids_np = _random_ids(64, 2, 8, seed=3)
    ids_np[5, 1] = 8                       # out of range: reported, its pair dropped
    dims = lm.make_dims(64, 64, 32, 8, 2, 0, 64, 64)
    ws = lm.alloc_workspace(dims)
    counts = torch.empty(8, dtype=torch.int32, device="cuda")
    offsets = torch.empty(9, dtype=torch.int32, device="cuda")
    perm = torch.full((128,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((64, 2), -7, dtype=torch.int32, device="cuda")
    lm.moe_dispatch(dims, to_device(ids_np, ""), counts, offsets, perm, inv, ws)
    assert lm.get_device_status(ws) == lm.EDEVICE
    assert host(counts).sum() == 127 and host(inv)[5, 1] == -1   # dropped: no sorted slot
    assert lm.get_device_status(ws) == lm.OK   # reading clears the word


@pytest.mark.parametrize("name,n", [("halfb_uniform", 257), ("halfb_skewed", 300), ("mid", 96),
                                    ("toy_fp32", 128),
                                    # >= 64 pairs per expert: routed GEMMs on CTA pairs over
                                    # 256-row tiles (tails of <= 128 rows, and experts over 256)
                                    ("halfb_uniform", 700), ("halfb_skewed", 1500), ("mid", 600)])
def test_expert_ffn_and_combine_parity(name, n):
    """moe_expert_ffn on the oracle's z and permutation vs the oracle's SiTU per
    pair; moe_combine on the oracle's expert outputs vs RMSNorm of the p-weighted sum."""
    wl = W[name].with_tokens(n)
    inp = prepare(wl)
    ow = oracle_weights(inp)
    ref = oracle.forward(odims(wl), ow, synth.to_f32(inp["x"]), want=("z", "routed", "u", "uhat"))
    counts, offsets, perm, inv = oracle.permute(ref["ids"], wl.n_routed)
    z = round_act(ref["z"], wl)
    # expected expert outputs in sorted-pair order, from the rounded z the GPU sees
    P = n * wl.top_k
    exp_eo = np.empty((P, wl.latent))
    for t in range(n):
        for i in range(wl.top_k):
            e = ref["ids"][t, i]
            exp_eo[inv[t, i]] = oracle.situ(ow["w_g"][e], ow["w_u"][e], ow["w_o"][e], z[t],
                                            wl.beta1, wl.beta2)[0]
    dims = ldims(wl)
    ws = lm.alloc_workspace(dims)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    zd = torch.from_numpy(z).to("cuda", dt)
    eo = torch.empty(P, wl.latent, dtype=dt, device="cuda")
    dev = device_inputs({k: inp[k] for k in ("w_g", "w_u", "w_o", "rms_weight")})
    lm.moe_expert_ffn(dims, zd, to_device(perm, ""), to_device(offsets, ""), dev["w_g"],
                      dev["w_u"], dev["w_o"], eo, ws)
    torch.cuda.synchronize()
    tol = 2e-2 if wl.dtype == "bf16" else 1e-5
    assert rel_err(host(eo), exp_eo) <= tol
    # combine: inputs are the oracle's expert outputs rounded to the activation dtype
    eo_in = round_act(exp_eo, wl)
    u_exp = np.zeros((n, wl.latent))
    for t in range(n):
        for i in range(wl.top_k):
            u_exp[t] += ref["probs"][t, i] * eo_in[inv[t, i]].astype(np.float64)
    uhat_exp = oracle.rmsnorm(u_exp, inp["rms_weight"], wl.rms_eps)
    out = torch.empty(n, wl.latent, dtype=dt, device="cuda")
    lm.moe_combine(dims, torch.from_numpy(eo_in).to("cuda", dt), to_device(inv, ""),
                   torch.from_numpy(ref["probs"].astype(np.float32)).cuda(), dev["rms_weight"],
                   out)
    torch.cuda.synchronize()
    tol_c = 1e-2 if wl.dtype == "bf16" else 1e-5
    assert rel_err(host(out), uhat_exp) <= tol_c


# ------------------------------------------------------------- edge cases

EDGE = [
    # (label, workload overrides)
    ("one_token", dict(n_tokens=1)),
    ("top1", dict(top_k=1)),
    ("k_equals_R", dict(n_routed=8, top_k=8)),
    ("pages_toy_dff96", dict(ff_routed=96, ff_shared=96)),
    ("no_shared", dict(n_shared=0)),
    ("ragged_1000", dict(n_tokens=1000)),
    # widths that are multiples of 8 but not of 64: ragged K blocks, masked columns
    ("odd_widths", dict(d=200, latent=104, ff_routed=72, ff_shared=136)),
]


@pytest.mark.parametrize("label,over", EDGE, ids=[e[0] for e in EDGE])
@pytest.mark.parametrize("base", ["halfb_uniform", "toy_fp32"])
def test_forward_edge_cases(label, over, base):
    wl = W[base].with_tokens(200).replace(**over)
    inp = prepare(wl)
    y, ids, probs, counts, _ = _run_forward(wl, device_inputs(inp))
    _compare_forward(wl, inp, y, ids, probs)


def test_forward_saturated_situ():
    """Expert weights of std 1: SiTU gates and ups run deep into saturation (the
    router keeps std 0.02 so that its top-k stays well separated)."""
    from oracle.conditioning import enforce_topk_margin
    wl = W["halfb_uniform"].with_tokens(160).replace(w_std=1.0)
    inp = synth.make_inputs(wl)
    inp["w_router"] = synth.normal(0, "w_router", (wl.n_routed, wl.d), 0.02)
    enforce_topk_margin(wl, inp)
    y, ids, probs, _, _ = _run_forward(wl, device_inputs(inp))
    _compare_forward(wl, inp, y, ids, probs)


@pytest.mark.parametrize("name,n", [("halfb_uniform", 300), ("mid", 136), ("k3_width", 24)])
def test_forward_intermediates(name, n):
    """Each stage of the forward against the oracle: z, router logits, shared
    hidden units, RMSNorm(u), then y."""
    wl = W[name].with_tokens(n)
    inp = prepare(wl)
    dev = device_inputs(inp)
    y, ids, probs, _, ws = _run_forward(wl, dev)
    v = lm.workspace_views(ldims(wl), ws)
    ow = oracle_weights(inp)
    x = synth.to_f32(inp["x"]).astype(np.float64)
    ref = oracle.forward(odims(wl), ow, synth.to_f32(inp["x"]), want=("z", "uhat"))
    assert rel_err(host(v["z"]), ref["z"]) <= 1e-2, "z"
    if wl.n_routed > 32:   # up to 32 experts the x-pass routes in its epilogue, no logits
        logits = x @ ow["w_router"].astype(np.float64).T
        assert rel_err(host(v["logits"]), logits) <= 1e-5, "router logits"
    if wl.n_shared:
        hs = np.empty((n, wl.n_shared * wl.ff_shared))
        for t in range(n):
            for j in range(wl.n_shared):
                hs[t, j * wl.ff_shared:(j + 1) * wl.ff_shared] = oracle.situ(
                    ow["ws_g"][j], ow["ws_u"][j], ow["ws_o"][j], x[t], wl.beta1, wl.beta2)[1]
        assert rel_err(host(v["hsh"]), hs) <= 2e-2, "shared hidden"
    assert rel_err(host(v["uhat"]), ref["uhat"]) <= 2e-2, "uhat"
    _compare_forward(wl, inp, y, ids, probs)


def test_forward_zero_tokens():
    wl = W["halfb_uniform"].with_tokens(0)
    inp = synth.make_inputs(wl)
    dev = device_inputs(inp)
    dims = ldims(wl)
    ws = lm.alloc_workspace(dims)
    counts = torch.full((wl.n_routed,), 9, dtype=torch.int32, device="cuda")
    lm.latent_moe_forward(dims, dev, dev["x"], dev["x"], ws, None, None, counts)
    assert (host(counts) == 0).all()


def test_unselected_expert_leaves_y_bitwise():
    wl = W["halfb_uniform"].with_tokens(256)
    inp = prepare(wl)
    inp["expert_bias"][3] = -10.0          # expert 3 is never selected
    dev = device_inputs(inp)
    y0, ids0, _, _, ws = _run_forward(wl, dev)
    assert not (host(ids0) == 3).any()
    for name in ("w_g", "w_u", "w_o"):
        dev[name][3] = 7.0
    y1, _, _, _, _ = _run_forward(wl, dev, ws)
    assert torch.equal(y0, y1)


def test_host_entry_point_matches_device():
    wl = W["halfb_uniform"].with_tokens(512)
    inp = prepare(wl)
    dev = device_inputs(inp)
    y, _, _, _, _ = _run_forward(wl, dev)
    dims = ldims(wl)
    ws = lm.alloc_workspace(dims, host=True)
    x_h = dev["x"].cpu().pin_memory()
    y_h = torch.empty_like(x_h).pin_memory()
    lm.latent_moe_forward_host(dims, dev, x_h, y_h, ws)
    assert torch.equal(y_h, y.cpu())


@pytest.mark.parametrize("name,n,chunks", [("halfb_uniform", 1000, "3"), ("mid", 700, "2"),
                                           ("halfb_skewed", 4096, "8")])
def test_host_entry_point_in_chunks(name, n, chunks, monkeypatch):
    """latent_moe_forward_host pipelining the tokens in several chunks (x in on
    one copy stream, each chunk's forward, y out on another, uneven last
    chunk): y against the oracle on sampled rows and against one device-side
    forward over all tokens (the chunks may tile the GEMMs differently, so
    within rounding)."""
    monkeypatch.setenv("LMOE_HOST_CHUNKS", chunks)
    wl = W[name].with_tokens(n)
    inp = prepare(wl)
    dev = device_inputs(inp)
    y, ids, probs, _, _ = _run_forward(wl, dev)
    dims = ldims(wl)
    ws = lm.alloc_workspace(dims, host=True)
    x_h = dev["x"].cpu().pin_memory()
    y_h = torch.empty_like(x_h).pin_memory()
    lm.latent_moe_forward_host(dims, dev, x_h, y_h, ws)
    assert lm.get_device_status(ws) == lm.OK
    assert rel_err(host(y_h), host(y)) <= 1e-2
    rows = np.arange(0, n, max(1, n // 64))
    ref = oracle.forward(odims(wl, len(rows)), oracle_weights(inp),
                         synth.to_f32(inp["x"])[rows])
    assert rel_err(host(y_h)[rows], ref["y"]) <= y_tol(wl)


def test_capped_wait_reports_timeout():
    dims = lm.make_dims(8, 64, 32, 4, 2, 1, 64, 64)
    ws = lm.alloc_workspace(dims)
    lm.selftest_capped_wait(ws, 50)
    assert lm.get_device_status(ws) == lm.ETIMEOUT
    # the context is still usable afterwards
    t = torch.ones(4, device="cuda") * 2
    assert float(t.sum()) == 8.0


# ------------------------------------------------ device-side consistency check

def _dispatch(N, k, R, seed, skew=False):
    dims = lm.make_dims(N, 64, 32, R, k, 0, 64, 64)
    ws = lm.alloc_workspace(dims)
    ids = torch.from_numpy(_random_ids(N, k, R, seed=seed, skew=skew)).cuda()
    counts = torch.empty(R, dtype=torch.int32, device="cuda")
    offsets = torch.empty(R + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(N * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(N * k, dtype=torch.int32, device="cuda")
    lm.moe_dispatch(dims, ids, counts, offsets, perm, inv, ws)
    return dims, ws, ids, counts, offsets, perm, inv


@pytest.mark.parametrize("N,k,R,skew", [(300, 2, 16, False), (4096, 2, 16, True),
                                        (1000, 16, 896, False), (1, 1, 4, False)])
def test_check_dispatch_accepts_the_permutation(N, k, R, skew):
    dims, ws, ids, counts, offsets, perm, inv = _dispatch(N, k, R, seed=N + R, skew=skew)
    lm.check_dispatch(dims, ids, counts, offsets, perm, inv, ws)
    torch.cuda.synchronize()
    assert lm.get_device_status(ws) == lm.OK


def test_check_dispatch_flags_corruptions():
    """Each corruption (in-range values only) sets EDEVICE: two pairs swapped
    across experts, a wrong token in perm_token, a count moved between experts,
    two pairs on one slot."""
    N, k, R = 512, 2, 16
    dims, ws, ids, counts, offsets, perm, inv = _dispatch(N, k, R, seed=5)
    h_ids = host(ids).reshape(-1)
    a = 0
    b = int(np.nonzero(h_ids != h_ids[0])[0][0])

    def flagged(**bad):
        lm.workspace_init(ws)
        args = dict(ids=ids, counts=counts, offsets=offsets, perm=perm, inv=inv)
        args.update(bad)
        lm.check_dispatch(dims, args["ids"], args["counts"], args["offsets"], args["perm"],
                          args["inv"], ws)
        torch.cuda.synchronize()
        return lm.get_device_status(ws) == lm.EDEVICE

    assert not flagged()
    inv2 = inv.clone()
    inv2[a], inv2[b] = inv[b], inv[a]
    assert flagged(inv=inv2)
    perm2 = perm.clone()
    perm2[0] = (perm[0] + 1) % N
    assert flagged(perm=perm2)
    counts2 = counts.clone()
    counts2[0] += 1
    counts2[1] -= 1
    assert flagged(counts=counts2)
    inv3 = inv.clone()
    inv3[1] = inv[0]
    assert flagged(inv=inv3)


@pytest.mark.parametrize("name,n", [("halfb_uniform", 700), ("mid", 300)])
def test_fused_combine_matches_combine_entry_point(name, n):
    """For l <= 1024 the forward's final GEMM computes RMSNorm(u) itself (the
    combine fused into its epilogue warps).  Its rows must equal moe_combine on
    the same expert outputs bit for bit, and every launch must leave the
    synchronisation area after the workspace header zeroed for the next one."""
    wl = W[name].with_tokens(n)
    assert lm.forward_plan(ldims(wl))["combine_fused"]
    inp = prepare(wl)
    dev = device_inputs(inp)
    y, ids, probs, counts, ws = _run_forward(wl, dev)
    dims = ldims(wl)
    v = lm.workspace_views(dims, ws)
    u2 = torch.empty_like(v["uhat"])
    lm.moe_combine(dims, v["eo"], v["inv"], probs, dev["rms_weight"], u2)
    torch.cuda.synchronize()
    assert torch.equal(u2, v["uhat"])
    sync = ws[256:256 + 4096].view(torch.int32)
    assert int(sync.abs().sum().item()) == 0
    y2, _, _, _, _ = _run_forward(wl, dev, ws)
    assert torch.equal(y, y2)


@pytest.mark.parametrize("name,n,mode", [("k3_width", 320, None), ("halfb_uniform", 300, "1"),
                                         ("mid", 136, "1"), ("halfb_uniform", 4096, "1"),
                                         # one row tile split many ways: 1 K block per pair
                                         ("halfb_uniform", 1, "1"), ("k3_width", 3, "1")])
def test_stream_k_final_gemm(name, n, mode, monkeypatch):
    """Stream-K final GEMM: the CTA pairs share the tiles x K-blocks iterations
    and a tile split between pairs is summed in fp32 in a fixed order.  At the
    K3 width with 320 tokens (14 tiles of 256 x 512) it is the default;
    LMOE_STREAM_K=1 forces it, here also together with the fused combine.
    y against the oracle on sampled rows, bitwise repeatable, within bf16
    rounding of the whole-tile schedule (LMOE_STREAM_K=0) and not equal to it
    everywhere (the split path ran), with the flags left zeroed."""
    wl = W[name].with_tokens(n)
    inp = prepare(wl)
    dev = device_inputs(inp)
    if mode is not None:
        monkeypatch.setenv("LMOE_STREAM_K", mode)
    y, ids, probs, _, ws = _run_forward(wl, dev)
    _compare_forward(wl, inp, y, ids, probs, rows=np.arange(0, n, max(1, n // 128)))
    sync = ws[256:256 + 4096].view(torch.int32)
    assert int(sync.abs().sum().item()) == 0
    y2, _, _, _, _ = _run_forward(wl, dev, ws)
    assert torch.equal(y, y2)
    monkeypatch.setenv("LMOE_STREAM_K", "0")
    y0, _, _, _, _ = _run_forward(wl, dev, ws)
    assert rel_err(host(y), host(y0)) <= 1e-2
    if n >= 100:   # enough outputs that some bf16 rounding must differ
        assert not torch.equal(y, y0)


def test_routed_gemms_on_different_tile_heights():
    """Experts over 256 pairs with l >= 1024: routed GEMM1 on CTA pairs over
    256-row tiles, GEMM2 on single CTAs over its own 128-row tile list.
    moe_expert_ffn on the oracle's z and permutation, sampled sorted rows
    against the oracle's SiTU expert (bf16 tolerance of the forward)."""
    wl = W["mid"].with_tokens(2200)          # 17600 pairs over 64 experts: ~275 each
    plan = lm.forward_plan(ldims(wl))
    assert plan["gemm1_pairs"] and not plan["gemm2_pairs"]
    inp = prepare(wl)
    ow = oracle_weights(inp)
    ref = oracle.forward(odims(wl), ow, synth.to_f32(inp["x"]), want=("z",))
    counts, offsets, perm, inv = oracle.permute(ref["ids"], wl.n_routed)
    assert counts.mean() > 256
    z = round_act(ref["z"], wl)
    P = wl.n_tokens * wl.top_k
    dims = ldims(wl)
    ws = lm.alloc_workspace(dims)
    dev = device_inputs({k: inp[k] for k in ("w_g", "w_u", "w_o")})
    eo = torch.empty(P, wl.latent, dtype=torch.bfloat16, device="cuda")
    lm.moe_expert_ffn(dims, torch.from_numpy(z).to("cuda", torch.bfloat16), to_device(perm, ""),
                      to_device(offsets, ""), dev["w_g"], dev["w_u"], dev["w_o"], eo, ws)
    torch.cuda.synchronize()
    assert lm.get_device_status(ws) == lm.OK
    # every expert's first and last rows (tile edges of both heights) and a stride
    rows = np.unique(np.concatenate([offsets[:-1], offsets[1:] - 1, np.arange(0, P, 41)]))
    rows = rows[(rows >= 0) & (rows < P)]
    expert = np.searchsorted(offsets, rows, side="right") - 1
    exp_eo = np.stack([oracle.situ(ow["w_g"][e], ow["w_u"][e], ow["w_o"][e], z[perm[r]],
                                   wl.beta1, wl.beta2)[0] for r, e in zip(rows, expert)])
    assert rel_err(host(eo)[rows], exp_eo) <= 2e-2


@pytest.mark.parametrize("name,n,colscan", [("halfb_uniform", 4096, False), ("mid", 2200, False),
                                            ("k3_width", 320, True)])
def test_forward_launches_follow_the_plan(name, n, colscan):
    """The launches of one forward are the ones lmoe_forward_plan reports: the
    x-pass, top-k for R > 32, histogram unless the x-pass counted the pairs (+
    column scan for a large count matrix) + scatter, GEMM2's own tile list
    when the two routed GEMMs use different tile heights, the gather unless the
    scatter copies the rows, the two routed GEMMs, the combine unless it is
    fused, and the final GEMM."""
    wl = W[name].with_tokens(n)
    plan = lm.forward_plan(ldims(wl))
    assert plan["counts_in_xpass"] == (name == "halfb_uniform")
    expected = (1 + (wl.n_routed > 32) + (not plan["counts_in_xpass"]) + 1 + colscan
                + (plan["gemm1_pairs"] != plan["gemm2_pairs"]) + (not plan["rows_in_scatter"])
                + 2 + (not plan["combine_fused"]) + 1)
    inp = prepare(wl)
    dev = device_inputs(inp)
    _run_forward(wl, dev)          # first call: one-time setup outside the count
    lm.launch_count(reset=True)
    _run_forward(wl, dev)
    assert lm.launch_count() == expected, (plan, expected)


def test_wide_routed_gemm_parity():
    """Routed experts at the K3 latent width (l = 3584) with 64..256 rows per
    expert: CTA pairs and 256 x 512 tiles of 256 hidden units for GEMM1.
    moe_expert_ffn on the oracle's z and permutation, every 8th sorted row
    against the oracle's SiTU expert (bf16 tolerance of the forward)."""
    wl = W["k3_width"].with_tokens(512).replace(n_routed=16, top_k=4)
    inp = prepare(wl)
    ow = oracle_weights(inp)
    ref = oracle.forward(odims(wl), ow, synth.to_f32(inp["x"]), want=("z",))
    counts, offsets, perm, inv = oracle.permute(ref["ids"], wl.n_routed)
    assert (counts >= 64).all() and (counts <= 256).all()
    z = round_act(ref["z"], wl)
    P = wl.n_tokens * wl.top_k
    dims = ldims(wl)
    ws = lm.alloc_workspace(dims)
    dev = device_inputs({k: inp[k] for k in ("w_g", "w_u", "w_o")})
    eo = torch.empty(P, wl.latent, dtype=torch.bfloat16, device="cuda")
    lm.moe_expert_ffn(dims, torch.from_numpy(z).to("cuda", torch.bfloat16), to_device(perm, ""),
                      to_device(offsets, ""), dev["w_g"], dev["w_u"], dev["w_o"], eo, ws)
    torch.cuda.synchronize()
    assert lm.get_device_status(ws) == lm.OK
    rows = np.arange(0, P, 8)
    expert = np.searchsorted(offsets, rows, side="right") - 1
    exp_eo = np.stack([oracle.situ(ow["w_g"][e], ow["w_u"][e], ow["w_o"][e], z[perm[r]],
                                   wl.beta1, wl.beta2)[0] for r, e in zip(rows, expert)])
    assert rel_err(host(eo)[rows], exp_eo) <= 2e-2


@pytest.mark.parametrize("n,over", [(4096, {}), (1000, {}), (1, {}),
                                    (777, dict(top_k=8, n_routed=32)),
                                    (5000, dict(top_k=1)),
                                    (16384, dict(top_k=4, n_routed=8))])
def test_counts_in_xpass_match_the_histogram(n, over, monkeypatch):
    """Routing in the x-pass's epilogue (R <= 32): the expert counts of every 32
    tokens written there replace the dispatch's histogram kernel.  The forward
    is bit-identical with the histogram kernel (LMOE_XPASS_COUNTS=0): ids,
    counts, the permutation and y; ragged token counts (partial 32-token rows,
    a partial last chunk), k = 1, 2, 4, 8 (1, 4, 8 or 32 count rows per chunk
    of the counting sort)."""
    wl = W["halfb_uniform"].with_tokens(n).replace(**over)
    dims = ldims(wl)
    assert lm.forward_plan(dims)["counts_in_xpass"]
    inp = prepare(wl)
    dev = device_inputs(inp)
    monkeypatch.delenv("LMOE_XPASS_COUNTS", raising=False)
    y, ids, probs, counts, ws = _run_forward(wl, dev)
    v = lm.workspace_views(dims, ws)
    got = [host(v[k]).copy() for k in ("offsets", "perm", "inv")]
    monkeypatch.setenv("LMOE_XPASS_COUNTS", "0")
    assert not lm.forward_plan(dims)["counts_in_xpass"]
    y0, ids0, probs0, counts0, ws0 = _run_forward(wl, dev)
    v0 = lm.workspace_views(dims, ws0)
    assert torch.equal(ids, ids0) and torch.equal(counts, counts0)
    for a, b in zip(got, [host(v0[k]) for k in ("offsets", "perm", "inv")]):
        np.testing.assert_array_equal(a, b)
    assert torch.equal(y, y0)
    h_ids = host(ids)
    check_permutation_properties(h_ids, host(counts), got[0], got[1], got[2], wl.n_routed)
    rows = np.unique(np.linspace(0, n - 1, min(n, 64)).astype(np.int64))
    _compare_forward(wl, inp, y, ids, probs, rows)
