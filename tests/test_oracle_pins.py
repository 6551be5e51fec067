"""Pins of the CPU oracle against what the K3 pages and mathematics fix.

Each test ties one part of the oracle to something other than the oracle
itself: brute force on tiny inputs, a library routine for a special case, a
closed form, an invariant the pages state, or a worked case the pages' own
tests assert.  The set is chosen so that a dropped term, a wrong sign, a
wrong index or a transposed operand in the oracle fails at least one test.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth
from oracle.conditioning import enforce_topk_margin, topk_gap

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sig(v):
    return 1.0 / (1.0 + math.exp(-v))


def _rand_inputs(dims: oracle.Dims, seed=1, w_std=0.3, x_std=1.0, bias_std=0.0):
    rng = np.random.default_rng(seed)
    d, L, R, F, S, G = dims.d, dims.latent, dims.n_routed, dims.ff_routed, dims.n_shared, dims.ff_shared
    f = lambda *shape: (rng.standard_normal(shape) * w_std).astype(np.float32)
    w = dict(w_down=f(L, d), w_router=f(R, d), w_up=f(d, L),
             rms_weight=(1.0 + 0.1 * rng.standard_normal(L)).astype(np.float32),
             expert_bias=(rng.standard_normal(R) * bias_std).astype(np.float32),
             w_g=f(R, F, L), w_u=f(R, F, L), w_o=f(R, L, F),
             ws_g=f(S, G, d), ws_u=f(S, G, d), ws_o=f(S, d, G))
    x = (rng.standard_normal((dims.n_tokens, d)) * x_std).astype(np.float32)
    return x, w


SMALL = oracle.Dims(n_tokens=12, d=32, latent=16, n_routed=8, top_k=2, n_shared=1,
                    ff_routed=24, ff_shared=24)


# ---------------------------------------------------------------- routing

@pytest.mark.parametrize("R,k", [(6, 1), (6, 2), (7, 3), (8, 4), (9, 2), (10, 5), (6, 6)])
def test_topk_is_the_max_sum_subset_by_brute_force(R, k):
    """TopK(s+b, k) selects the k largest keys: among all C(R,k) subsets the
    selected one has the largest key sum, and slots are in descending key order."""
    dims = oracle.Dims(40, 12, 6, R, k, 1, 4, 4)
    rng = np.random.default_rng(R * 100 + k)
    x = rng.standard_normal((40, 12)).astype(np.float32)
    w_r = rng.standard_normal((R, 12)).astype(np.float32)
    b = (0.3 * rng.standard_normal(R)).astype(np.float32)
    ids, probs, keys, scores = oracle.route(dims, x, w_r, b)
    for t in range(40):
        best = max(itertools.combinations(range(R), k), key=lambda c: sum(keys[t, list(c)]))
        assert set(ids[t]) == set(best)
        assert all(keys[t, ids[t, i]] >= keys[t, ids[t, i + 1]] for i in range(k - 1))
        # against a library sort: stable argsort of -key (ties to the lower index)
        assert list(ids[t]) == list(np.argsort(-keys[t], kind="stable")[:k])
        # the keys are s + b with s = sigmoid(W_r x) computed independently here
        l = w_r.astype(np.float64) @ x[t].astype(np.float64)
        np.testing.assert_allclose(scores[t], 1.0 / (1.0 + np.exp(-l)), rtol=1e-13)
        np.testing.assert_allclose(keys[t], scores[t] + b.astype(np.float64), rtol=1e-13)
    if k == R:
        assert all(sorted(row) == list(range(R)) for row in ids)


def test_topk_tie_goes_to_lower_index():
    dims = oracle.Dims(1, 4, 2, 5, 2, 1, 2, 2)
    x = np.zeros((1, 4), np.float32)          # every logit 0, every score 0.5
    w_r = np.ones((5, 4), np.float32)
    ids, probs, _, _ = oracle.route(dims, x, w_r, np.zeros(5, np.float32))
    assert list(ids[0]) == [0, 1]
    np.testing.assert_array_equal(probs[0], [0.5, 0.5])


def test_collapsed_router_worked_case():
    """The pages' collapsed-router case: router rows 0 := 1, 1 := 0.5, others 0, x = 1."""
    with open(os.path.join(GOLDEN, "collapsed_router.json")) as f:
        g = json.load(f)
    d, R, k = g["hidden_size"], g["n_routed"], g["top_k"]
    n = int(np.prod(g["x_shape"][:-1]))
    dims = oracle.Dims(n, d, g["latent_size"], R, k, g["n_shared"], g["d_ff"], g["d_ff"])
    w_r = np.zeros((R, d), np.float32)
    for row, val in g["router_rows"].items():
        w_r[int(row)] = val
    x = np.full((n, d), g["x_value"], np.float32)
    ids, probs, _, _ = oracle.route(dims, x, w_r)
    assert set(ids.reshape(-1).tolist()) == set(g["expected_selected"])
    assert all(list(r) == [0, 1] for r in ids)           # key order: sigma(32) > sigma(16)
    s0, s1 = _sig(32.0), _sig(16.0)
    for r in probs:
        assert r[0] == pytest.approx(s0 / (s0 + s1), rel=1e-15)
        assert r[1] == pytest.approx(s1 / (s0 + s1), rel=1e-15)


def test_probs_sum_to_one_and_bias_only_selects():
    """p_i = s_i / sum_T s_j sums to 1; b changes which experts are chosen but not p."""
    dims = oracle.Dims(64, 24, 12, 10, 3, 1, 8, 8)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((64, 24)).astype(np.float32)
    w_r = (0.5 * rng.standard_normal((10, 24))).astype(np.float32)
    b = (0.2 * rng.standard_normal(10)).astype(np.float32)
    ids, probs, keys, scores = oracle.route(dims, x, w_r, b)
    np.testing.assert_allclose(probs.sum(1), 1.0, atol=4e-16)
    # p is the selected raw scores renormalised (not the biased keys)
    sel = np.take_along_axis(scores, ids, 1)
    np.testing.assert_allclose(probs, sel / sel.sum(1, keepdims=True), rtol=1e-15)
    # shifting every bias by the same amount keeps T, hence p bit for bit
    ids2, probs2, _, _ = oracle.route(dims, x, w_r, b + np.float32(0.25))
    np.testing.assert_array_equal(ids, ids2)
    np.testing.assert_array_equal(probs, probs2)
    # a bias that pushes expert 0 to the top changes T, and p still uses s
    b3 = b.copy(); b3[0] = 10.0
    ids3, probs3, _, scores3 = oracle.route(dims, x, w_r, b3)
    assert (ids3[:, 0] == 0).all()
    sel3 = np.take_along_axis(scores3, ids3, 1)
    np.testing.assert_allclose(probs3, sel3 / sel3.sum(1, keepdims=True), rtol=1e-15)


def test_probs_clamp_when_scores_vanish():
    """The denominator is clamped at 1e-9: with every logit near -40 the sum of
    the selected scores is ~4e-18, so p = s / 1e-9 (far below 1)."""
    dims = oracle.Dims(1, 2, 2, 4, 2, 1, 2, 2)
    x = np.array([[1.0, 0.0]], np.float32)
    w_r = np.array([[-40.0, 0], [-41.0, 0], [-42.0, 0], [-43.0, 0]], np.float32)
    ids, probs, _, _ = oracle.route(dims, x, w_r)
    assert list(ids[0]) == [0, 1]
    assert probs[0, 0] == pytest.approx(_sig(-40.0) / 1e-9, rel=1e-12)
    assert probs[0, 1] == pytest.approx(_sig(-41.0) / 1e-9, rel=1e-12)


# ------------------------------------------------------------ permutation

@pytest.mark.parametrize("N,k,R,mode", [(50, 2, 8, "random"), (64, 1, 5, "random"),
                                        (33, 4, 4, "all"), (40, 3, 16, "skewed"),
                                        (1, 2, 3, "random"), (0, 2, 4, "random")])
def test_permutation_is_the_stable_argsort(N, k, R, mode):
    """counts/offsets/perm are bincount, cumsum - counts and a stable argsort of
    the token-major expert ids (the pages' dispatch), here numpy's routines."""
    rng = np.random.default_rng(N * 7 + k)
    if mode == "all":
        ids = np.tile(np.arange(k, dtype=np.int32), (N, 1))
    else:
        p = np.ones(R) if mode == "random" else np.r_[np.full(3, 30.0), np.ones(R - 3)]
        rows = [rng.choice(R, size=k, replace=False, p=p / p.sum()) for _ in range(N)]
        ids = np.array(rows, dtype=np.int32).reshape(N, k)
    counts, offsets, perm_token, inv_pair = oracle.permute(ids, R)
    eid = ids.reshape(-1)
    order = np.argsort(eid, kind="stable")
    np.testing.assert_array_equal(counts, np.bincount(eid, minlength=R))
    np.testing.assert_array_equal(offsets[:-1], np.cumsum(counts) - counts)
    assert offsets[-1] == N * k
    np.testing.assert_array_equal(perm_token, order // k)
    inv = np.empty(N * k, np.int64); inv[order] = np.arange(N * k)
    np.testing.assert_array_equal(inv_pair.reshape(-1), inv)


# ------------------------------------------------------------------ SiTU

def test_situ_hidden_bounded_by_beta1_beta2():
    """|gate * up| <= beta1 * beta2 = 100 for any input (property table)."""
    rng = np.random.default_rng(3)
    w_g = rng.standard_normal((64, 8)).astype(np.float32)
    w_u = rng.standard_normal((64, 8)).astype(np.float32)
    w_o = rng.standard_normal((8, 64)).astype(np.float32)
    for scale in (1e-3, 1.0, 10.0, 1e2, 1e3, 1e4):
        v = rng.standard_normal(8) * scale
        _, h = oracle.situ(w_g, w_u, w_o, v)
        assert np.abs(h).max() <= 100.0
    _, h = oracle.situ(w_g, w_u, w_o, np.full(8, 1e4))
    assert np.abs(h).max() > 99.0      # the bound is reached in saturation


def test_situ_small_input_limit_is_swiglu():
    """Near the origin beta*tanh(v/beta) ~ v, so SiTU ~ W_o(silu(W_g v) * (W_u v))
    with relative error O((v/beta)^2) (property table)."""
    rng = np.random.default_rng(4)
    dim, ff = 16, 40
    w_g = rng.standard_normal((ff, dim)).astype(np.float32)
    w_u = rng.standard_normal((ff, dim)).astype(np.float32)
    w_o = rng.standard_normal((dim, ff)).astype(np.float32)
    v = rng.standard_normal(dim) * 0.01          # |a|, |c| ~ 0.04
    out, _ = oracle.situ(w_g, w_u, w_o, v)
    a = w_g.astype(np.float64) @ v
    c = w_u.astype(np.float64) @ v
    swiglu = w_o.astype(np.float64) @ (a / (1.0 + np.exp(-a)) * c)
    err = np.abs(out - swiglu).max() / np.abs(swiglu).max()
    assert err < 5e-4, err
    # and the gap closes like (v/beta)^2: ten times smaller input, ~100x smaller error
    out2, _ = oracle.situ(w_g, w_u, w_o, v * 0.1)
    a2, c2 = a * 0.1, c * 0.1
    sw2 = w_o.astype(np.float64) @ (a2 / (1.0 + np.exp(-a2)) * c2)
    err2 = np.abs(out2 - sw2).max() / np.abs(sw2).max()
    assert err2 < err / 30


def test_situ_saturation_levels():
    """Far from the origin: gate -> beta1 (a -> +inf), gate -> 0 (a -> -inf),
    up -> +-beta2; the caps are beta1 = 4 on the gate and beta2 = 25 on up."""
    one = np.ones((1, 1), np.float32)

    def hidden(a, c):
        _, h = oracle.situ(np.array([[a]], np.float32), np.array([[c]], np.float32), one, [1.0])
        return h[0]

    assert hidden(1e4, 1e4) == pytest.approx(100.0, rel=1e-12)
    assert hidden(1e4, -1e4) == pytest.approx(-100.0, rel=1e-12)
    assert abs(hidden(-1e3, 1e4)) < 1e-100
    # gate cap alone: up in its linear range (c tiny) => hidden / c -> beta1
    c = 2.0 ** -20                               # exact in float32
    assert hidden(1e4, c) / c == pytest.approx(4.0, rel=1e-9)
    # up cap alone: gate at a = 1 is 4 tanh(1/4) sigmoid(1); hidden / gate -> beta2
    gate1 = 4.0 * math.tanh(0.25) * _sig(1.0)
    assert hidden(1.0, 1e4) / gate1 == pytest.approx(25.0, rel=1e-12)
    # near zero: gate ~ a * sigmoid(a) with sigmoid(0) = 1/2, up ~ c
    assert hidden(c, c) == pytest.approx(0.5 * c * c, rel=1e-5)


def test_situ_output_uses_w_o_as_out_by_ff():
    """W_o is [dim_in, ff] (nn.Linear(ff, dim_in)): with one-hot rows the output
    picks single hidden units."""
    rng = np.random.default_rng(5)
    dim, ff = 3, 5
    w_g = rng.standard_normal((ff, dim)).astype(np.float32)
    w_u = rng.standard_normal((ff, dim)).astype(np.float32)
    w_o = np.zeros((dim, ff), np.float32)
    w_o[0, 4] = 1.0; w_o[1, 2] = 2.0; w_o[2, 0] = -1.0
    out, h = oracle.situ(w_g, w_u, w_o, rng.standard_normal(dim))
    np.testing.assert_allclose(out, [h[4], 2 * h[2], -h[0]], rtol=1e-15)


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_constant_vector_and_scale_invariance():
    c, eps = 0.37, 1e-6
    w = np.linspace(0.5, 1.5, 16).astype(np.float32)
    out = oracle.rmsnorm(np.full((1, 16), c), w, eps)
    np.testing.assert_allclose(out[0], w.astype(np.float64) * c / math.sqrt(c * c + eps), rtol=1e-14)
    rng = np.random.default_rng(6)
    u = rng.standard_normal((4, 16))
    a = oracle.rmsnorm(u, w, eps)
    b = oracle.rmsnorm(u * 1000.0, w, eps)
    np.testing.assert_allclose(a, b, rtol=1e-6)
    # unit RMS rows are left as they are (up to eps) with w = 1
    v = u / np.sqrt((u * u).mean(1, keepdims=True))
    np.testing.assert_allclose(oracle.rmsnorm(v, np.ones(16, np.float32), 0.0), v, rtol=1e-14)


# ----------------------------------------------------------- whole layer

def test_dense_equals_sparse():
    """The pages' identity: sparse dispatch == all-experts evaluation + gather."""
    x, w = _rand_inputs(SMALL, seed=11, bias_std=0.2)
    out = oracle.forward(SMALL, w, x, want=("u",))
    y_dense, u_dense = oracle.forward_dense(SMALL, w, x)
    np.testing.assert_allclose(out["u"], u_dense, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(out["y"], y_dense, rtol=1e-13, atol=1e-15)


def test_routed_sum_is_probability_weighted_expert_outputs():
    """u_t = sum_i p_i E_{ids_i}(z_t) with E from the SiTU function on z = W_down x."""
    x, w = _rand_inputs(SMALL, seed=12)
    out = oracle.forward(SMALL, w, x, want=("u", "z", "routed", "uhat", "shared"))
    # routing inside the forward reads the full-width x, not z
    ids_r, probs_r, _, _ = oracle.route(SMALL, x, w["w_router"], w["expert_bias"])
    np.testing.assert_array_equal(out["ids"], ids_r)
    np.testing.assert_array_equal(out["probs"], probs_r)
    np.testing.assert_allclose(out["z"], x.astype(np.float64) @ w["w_down"].astype(np.float64).T,
                               rtol=1e-12, atol=1e-14)
    for t in range(SMALL.n_tokens):
        acc = np.zeros(SMALL.latent)
        for i in range(SMALL.top_k):
            e = out["ids"][t, i]
            eo, _ = oracle.situ(w["w_g"][e], w["w_u"][e], w["w_o"][e], out["z"][t])
            np.testing.assert_allclose(out["routed"][t, i], eo, rtol=1e-13)
            acc += out["probs"][t, i] * eo
        np.testing.assert_allclose(out["u"][t], acc, rtol=1e-13, atol=1e-16)
    # y = shared + W_up uhat, uhat = RMSNorm(u), with W_up stored [d, l]
    np.testing.assert_allclose(out["uhat"], oracle.rmsnorm(out["u"], w["rms_weight"]), rtol=1e-14)
    up = out["uhat"] @ w["w_up"].astype(np.float64).T
    np.testing.assert_allclose(out["y"], out["shared"] + up, rtol=1e-12, atol=1e-14)


def test_unselected_experts_contribute_nothing():
    """Perturbing the weights of an expert no token selects leaves y bit for bit."""
    x, w = _rand_inputs(SMALL, seed=13)
    w["expert_bias"] = np.zeros(SMALL.n_routed, np.float32)
    w["expert_bias"][5] = -10.0                  # expert 5 can never be in T
    y0 = oracle.forward(SMALL, w, x)
    assert not (y0["ids"] == 5).any()
    w2 = dict(w)
    for name in ("w_g", "w_u", "w_o"):
        w2[name] = w[name].copy()
        w2[name][5] = 123.0
    y1 = oracle.forward(SMALL, w2, x)
    np.testing.assert_array_equal(y0["y"], y1["y"])
    # ...while perturbing a selected expert does change y
    e = int(y0["ids"][0, 0])
    w3 = dict(w); w3["w_o"] = w["w_o"].copy(); w3["w_o"][e] *= 2.0
    assert not np.array_equal(oracle.forward(SMALL, w3, x)["y"], y0["y"])


def test_shared_only_when_routed_or_up_is_zero():
    """W_up = 0 => y = s_sh;  routed W_o = 0 => u = 0 => uhat = 0 => y = s_sh;
    and s_sh is the plain sum of the shared SiTU experts on x."""
    dims = oracle.Dims(6, 32, 16, 8, 2, 3, 24, 20)
    x, w = _rand_inputs(dims, seed=14)
    sh = np.zeros((6, 32))
    for t in range(6):
        for j in range(3):
            sh[t] += oracle.situ(w["ws_g"][j], w["ws_u"][j], w["ws_o"][j], x[t])[0]
    wa = dict(w); wa["w_up"] = np.zeros_like(w["w_up"])
    np.testing.assert_allclose(oracle.forward(dims, wa, x)["y"], sh, rtol=1e-13, atol=1e-16)
    wb = dict(w); wb["w_o"] = np.zeros_like(w["w_o"])
    ob = oracle.forward(dims, wb, x, want=("uhat",))
    assert (ob["uhat"] == 0).all()
    np.testing.assert_allclose(ob["y"], sh, rtol=1e-13, atol=1e-16)


def test_shared_experts_equal_one_concatenated_expert():
    """sum_j SiTU_j(x) equals one SiTU whose hidden units are the concatenation."""
    dims = oracle.Dims(5, 32, 16, 8, 2, 3, 24, 20)
    x, w = _rand_inputs(dims, seed=15)
    o = oracle.forward(dims, w, x, want=("shared",))
    g = w["ws_g"].reshape(60, 32)
    u = w["ws_u"].reshape(60, 32)
    wo = np.concatenate(list(w["ws_o"]), axis=1)   # [d, S*G]
    for t in range(5):
        np.testing.assert_allclose(o["shared"][t], oracle.situ(g, u, wo, x[t])[0], rtol=1e-12,
                                   atol=1e-15)


def test_tokens_are_independent():
    """Permuting the token rows of x permutes the rows of y, ids and p."""
    x, w = _rand_inputs(SMALL, seed=16)
    perm = np.random.default_rng(0).permutation(SMALL.n_tokens)
    a = oracle.forward(SMALL, w, x)
    b = oracle.forward(SMALL, w, x[perm])
    np.testing.assert_array_equal(a["y"][perm], b["y"])
    np.testing.assert_array_equal(a["ids"][perm], b["ids"])


def test_top1_routing_uses_weight_one():
    """k = 1 => p = 1 exactly and u = E_{id}(z)."""
    dims = oracle.Dims(7, 32, 16, 8, 1, 1, 24, 24)
    x, w = _rand_inputs(dims, seed=17)
    o = oracle.forward(dims, w, x, want=("u", "routed"))
    assert (o["probs"] == 1.0).all()
    np.testing.assert_array_equal(o["u"], o["routed"][:, 0, :])


# ---------------------------------------------------- inputs and margins

def test_generator_statistics_and_determinism():
    a = synth.normal(0, "w_g", (1 << 16,), 0.02, dtype="f32")
    b = synth.normal(0, "w_g", (1 << 16,), 0.02, dtype="f32")
    np.testing.assert_array_equal(a, b)
    assert abs(a.mean()) < 3e-4 and abs(a.std() - 0.02) < 3e-4
    # any slice can be drawn on its own
    np.testing.assert_array_equal(synth.normal(0, "w_g", (100,), 0.02, dtype="f32", offset=500),
                                  a[500:600])
    # bf16 is the round-to-nearest-even of the same float draws
    hb = synth.normal(0, "w_g", (1 << 16,), 0.02, dtype="bf16")
    f = synth.to_f32(hb)
    assert np.abs(f - a).max() <= np.abs(a).max() * 2.0 ** -8
    assert not np.array_equal(synth.normal(1, "w_g", (64,), dtype="f32"), a[:64])


def test_skewed_workload_offsets_experts_0_to_3():
    wl = synth.WORKLOADS["halfb_skewed"].with_tokens(256)
    inp = synth.make_inputs(wl)
    x = synth.to_f32(inp["x"]); wr = synth.to_f32(inp["w_router"])
    assert (x[:, -1] == 1.0).all() and (wr[:4, -1] == 2.0).all()
    dims = oracle.Dims(256, wl.d, wl.latent, wl.n_routed, wl.top_k, wl.n_shared, wl.ff_routed,
                       wl.ff_shared)
    ids, _, _, scores = oracle.route(dims, x, wr, inp["expert_bias"])
    # the constant channel adds exactly +2.0 to logits 0-3: sigma(2) ~ 0.88 vs sigma(0) = 0.5
    logit = np.log(scores / (1.0 - scores))
    x0 = x.copy(); x0[:, -1] = 0.0
    base = x0.astype(np.float64) @ wr.astype(np.float64).T
    np.testing.assert_allclose(logit[:, :4] - base[:, :4], 2.0, atol=1e-9)
    np.testing.assert_allclose(logit[:, 4:] - base[:, 4:],
                               np.broadcast_to(wr[4:, -1].astype(np.float64), (256, 12)), atol=1e-9)
    load = np.bincount(ids.reshape(-1), minlength=16)
    assert load.max() > 8 * max(load.min(), 1)     # strongly uneven expert loads


def test_margin_conditioning_reaches_the_margin():
    wl = synth.WORKLOADS["halfb_uniform"].with_tokens(512)
    inp = synth.make_inputs(wl)
    stats = enforce_topk_margin(wl, inp, margin=1e-3)   # a wide margin forces redraws
    assert stats["redrawn"] > 0
    dims = oracle.Dims(512, wl.d, wl.latent, wl.n_routed, wl.top_k, wl.n_shared, wl.ff_routed,
                       wl.ff_shared)
    _, _, keys, _ = oracle.route(dims, synth.to_f32(inp["x"]), synth.to_f32(inp["w_router"]),
                                 inp["expert_bias"])
    assert topk_gap(keys, wl.top_k).min() >= 1e-3


# ------------------------------------------------- earlier router (softmax over top-k)

def _prior(dims: oracle.Dims) -> oracle.Dims:
    return oracle.Dims(dims.n_tokens, dims.d, dims.latent, dims.n_routed, dims.top_k,
                       dims.n_shared, dims.ff_routed, dims.ff_shared, router=1)


@pytest.mark.parametrize("R,k", [(6, 1), (6, 2), (8, 3), (9, 4), (7, 7)])
def test_prior_router_selects_the_largest_logits(R, k):
    """router = 1: T = TopK(l, k) on the raw logits, bias ignored; brute force over
    all C(R,k) subsets and numpy's stable argsort of -l."""
    dims = _prior(oracle.Dims(30, 10, 6, R, k, 1, 4, 4))
    rng = np.random.default_rng(7 * R + k)
    x = rng.standard_normal((30, 10)).astype(np.float32)
    w_r = rng.standard_normal((R, 10)).astype(np.float32)
    b = (5.0 * rng.standard_normal(R)).astype(np.float32)   # large, and must not matter
    ids, probs, keys, _ = oracle.route(dims, x, w_r, b)
    ids0, probs0, _, _ = oracle.route(dims, x, w_r, None)
    np.testing.assert_array_equal(ids, ids0)
    np.testing.assert_array_equal(probs, probs0)
    for t in range(30):
        l = w_r.astype(np.float64) @ x[t].astype(np.float64)
        np.testing.assert_allclose(keys[t], l, rtol=1e-13)
        best = max(itertools.combinations(range(R), k), key=lambda c: sum(l[list(c)]))
        assert set(ids[t]) == set(best)
        assert list(ids[t]) == list(np.argsort(-l, kind="stable")[:k])


def test_prior_router_weights():
    """Softmax over the selected logits: Σp = 1, p decreasing with the slot, k = 1
    gives 1, and for k = 2 the first weight is the logistic of the logit gap."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((50, 16)).astype(np.float32)
    w_r = rng.standard_normal((8, 16)).astype(np.float32)
    for k in (1, 2, 4):
        dims = _prior(oracle.Dims(50, 16, 8, 8, k, 1, 4, 4))
        ids, probs, keys, _ = oracle.route(dims, x, w_r)
        np.testing.assert_allclose(probs.sum(1), 1.0, rtol=0, atol=1e-15)
        assert (np.diff(probs, axis=1) <= 0).all()
        if k == 1:
            np.testing.assert_array_equal(probs, 1.0)
        if k == 2:
            gap = keys[np.arange(50), ids[:, 0]] - keys[np.arange(50), ids[:, 1]]
            np.testing.assert_allclose(probs[:, 0], 1.0 / (1.0 + np.exp(-gap)), rtol=1e-13)


def test_prior_router_is_shift_invariant():
    """Adding one constant to every logit (a constant input channel whose router
    column is the constant) changes neither the selection nor the weights."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((40, 12)).astype(np.float32)
    w_r = rng.standard_normal((8, 12)).astype(np.float32)
    x[:, -1] = 1.0
    w_r[:, -1] = 0.0
    dims = _prior(oracle.Dims(40, 12, 6, 8, 3, 1, 4, 4))
    ids0, p0, _, _ = oracle.route(dims, x, w_r)
    w_r[:, -1] = 7.5
    ids1, p1, _, _ = oracle.route(dims, x, w_r)
    np.testing.assert_array_equal(ids0, ids1)
    np.testing.assert_allclose(p0, p1, rtol=1e-12)


# ------------------------------------------------------------ router balancing losses

def test_router_losses_with_zero_router():
    """W_r = 0: every logit is 0, every score 1/2, so prob_mean = 1/2, aux = R/2
    (frac sums to 1) and z = (ln R)^2."""
    for R, k in ((8, 2), (16, 4), (5, 5)):
        dims = oracle.Dims(20, 10, 6, R, k, 1, 4, 4)
        x = np.random.default_rng(R).standard_normal((20, 10)).astype(np.float32)
        w_r = np.zeros((R, 10), np.float32)
        ids, _, _, _ = oracle.route(dims, x, w_r)
        out = oracle.router_losses(dims, x, w_r, ids)
        np.testing.assert_allclose(out["prob_mean"], 0.5, rtol=1e-15)
        assert out["frac"].sum() == pytest.approx(1.0, rel=1e-15)
        assert out["aux"] == pytest.approx(R / 2.0, rel=1e-14)
        assert out["z"] == pytest.approx(math.log(R) ** 2, rel=1e-13)


def test_router_losses_collapsed_case_of_the_pages():
    """The pages' collapse test: router rows 0 := 1, 1 := 0.5, x = 1.  Every token
    picks {0, 1}, so frac = (1/2, 1/2, 0...), logits (32, 16, 0 x 6):
    aux = R (sigma(32) + sigma(16)) / 2, z = (32 + ln(1 + e^-16 + 6 e^-32))^2.
    The page asserts aux > 1.2, aux above the random-router value, and z > 0."""
    with open(os.path.join(GOLDEN, "collapsed_router_losses.json")) as f:
        g = json.load(f)
    d, R, k = g["hidden_size"], g["n_routed"], g["top_k"]
    n = int(np.prod(g["x_shape"][:-1]))
    dims = oracle.Dims(n, d, 16, R, k, 1, 24, 24)
    w_r = np.zeros((R, d), np.float32)
    for row, val in g["router_rows"].items():
        w_r[int(row)] = val
    x = np.full((n, d), g["x_value"], np.float32)
    ids, _, _, _ = oracle.route(dims, x, w_r)
    out = oracle.router_losses(dims, x, w_r, ids)
    np.testing.assert_allclose(out["frac"], [0.5, 0.5] + [0.0] * (R - 2), rtol=0, atol=0)
    assert out["aux"] == pytest.approx(R * (_sig(32.0) + _sig(16.0)) / 2.0, rel=1e-14)
    assert out["z"] == pytest.approx((32.0 + math.log1p(math.exp(-16.0) + 6 * math.exp(-32.0))) ** 2,
                                     rel=1e-14)
    assert out["aux"] > g["asserted"]["aux_collapsed_greater_than"]
    assert out["z"] > g["asserted"]["z_greater_than"]
    rng = np.random.default_rng(0)
    xs = rng.standard_normal((n, d)).astype(np.float32)
    ws = (rng.standard_normal((R, d)) / math.sqrt(d)).astype(np.float32)
    ids_s, _, _, _ = oracle.route(dims, xs, ws)
    assert out["aux"] > oracle.router_losses(dims, xs, ws, ids_s)["aux"]


def test_router_losses_frac_is_the_routing_histogram_and_token_order_free():
    """frac = counts / (N k) from the permutation's counts; aux and z do not depend
    on the token order; aux <= R * max prob_mean."""
    dims = oracle.Dims(64, 24, 12, 12, 3, 1, 8, 8)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((64, 24)).astype(np.float32)
    w_r = (rng.standard_normal((12, 24)) * 0.4).astype(np.float32)
    ids, _, _, _ = oracle.route(dims, x, w_r)
    out = oracle.router_losses(dims, x, w_r, ids)
    counts, _, _, _ = oracle.permute(ids, 12)
    np.testing.assert_allclose(out["frac"], counts / (64 * 3), rtol=1e-15)
    perm = rng.permutation(64)
    out2 = oracle.router_losses(dims, x[perm], w_r, ids[perm])
    assert out2["aux"] == pytest.approx(out["aux"], rel=1e-13)
    assert out2["z"] == pytest.approx(out["z"], rel=1e-13)
    assert out["aux"] <= 12 * out["prob_mean"].max() + 1e-12
    assert ((out["prob_mean"] > 0) & (out["prob_mean"] < 1)).all()


# ------------------------------------------------------------------ backward

def _grid(rng, shape, scale, step=2.0 ** -8):
    """Values on a coarse binary grid, so that +-2^-17 perturbations are exact in float32."""
    return (np.round(rng.standard_normal(shape) * scale / step) * step).astype(np.float32)


def _fd_case(router=0, S=1, clamp=False, seed=0):
    dims = oracle.Dims(5, 16, 8, 6, 2, S, 12, 10, router=router)
    rng = np.random.default_rng(seed)
    d, L, R, F, G = dims.d, dims.latent, dims.n_routed, dims.ff_routed, dims.ff_shared
    Sx = max(S, 1)
    w = dict(w_down=_grid(rng, (L, d), 0.3), w_router=_grid(rng, (R, d), 0.5),
             w_up=_grid(rng, (d, L), 0.3), rms_weight=(1.0 + _grid(rng, (L,), 0.2)),
             expert_bias=_grid(rng, (R,), 0.1), w_g=_grid(rng, (R, F, L), 0.4),
             w_u=_grid(rng, (R, F, L), 0.4), w_o=_grid(rng, (R, L, F), 0.3),
             ws_g=_grid(rng, (Sx, G, d), 0.3), ws_u=_grid(rng, (Sx, G, d), 0.3),
             ws_o=_grid(rng, (Sx, d, G), 0.3))
    x = _grid(rng, (dims.n_tokens, d), 1.0)
    if clamp:   # every logit near -30: the selected scores sum below 1e-9
        x[:, -1] = 1.0
        w["w_router"][:, -1] = -30.0
    dy = _grid(rng, (dims.n_tokens, d), 1.0)
    return dims, w, x, dy


def _loss(dims, w, x, dy):
    y = oracle.forward(dims, w, x)["y"]
    return float((dy.astype(np.float64) * y).sum())


@pytest.mark.parametrize("router,S,clamp", [(0, 1, False), (1, 2, False), (0, 0, False),
                                            (0, 1, True)])
def test_backward_matches_central_differences(router, S, clamp):
    """Every gradient of <dy, y> against central differences of the forward
    (h = 2^-17, exact in float32 on the inputs' grid, truncation error ~h^2;
    routing unchanged by the perturbations).  Covers x, and sampled entries of every weight; the
    K3 router (plain and with its 1e-9 clamp active) and the softmax router."""
    dims, w, x, dy = _fd_case(router, S, clamp, seed=router * 10 + S + 3 * clamp)
    ids0 = oracle.route(dims, x, w["w_router"], w["expert_bias"])[0]
    g = oracle.backward(dims, w, x, dy)
    h = 2.0 ** -17
    rng = np.random.default_rng(42)

    def fd(perturb):
        plus, minus = perturb(h), perturb(-h)
        return (_loss(dims, *plus, dy) - _loss(dims, *minus, dy)) / (2 * h)

    checked = 0
    # x: every entry
    for t in range(dims.n_tokens):
        for i in range(dims.d):
            def px(eps, t=t, i=i):
                xx = x.copy()
                xx[t, i] += np.float32(eps)
                assert (oracle.route(dims, xx, w["w_router"], w["expert_bias"])[0] == ids0).all()
                return w, xx
            got, want = g["x"][t, i], fd(px)
            assert got == pytest.approx(want, rel=1e-6, abs=1e-8), ("x", t, i)
            checked += 1
    names = ["w_down", "w_router", "w_up", "rms_weight", "w_g", "w_u", "w_o"]
    if S:
        names += ["ws_g", "ws_u", "ws_o"]
    for name in names:
        arr = w[name]
        picks = [tuple(rng.integers(0, n) for n in arr.shape) for _ in range(6)]
        if name in ("w_g", "w_u", "w_o"):   # entries of a selected expert too
            e = int(ids0[0, 0])
            picks += [(e,) + tuple(rng.integers(0, n) for n in arr.shape[1:]) for _ in range(4)]
        for idx in picks:
            def pw(eps, name=name, idx=idx):
                ww = dict(w)
                ww[name] = w[name].copy()
                ww[name][idx] += np.float32(eps)
                return ww, x
            got, want = g[name][idx], fd(pw)
            assert got == pytest.approx(want, rel=1e-6, abs=1e-8), (name, idx)
            checked += 1
    assert checked > dims.n_tokens * dims.d


def test_backward_unselected_experts_get_exactly_zero():
    """The pages' test_moe_unselected_experts_have_zero_grad: experts no token
    selects get gradients that are exactly 0; a selected one gets nonzero ones."""
    dims, w, x, dy = _fd_case(seed=7)
    ids = oracle.route(dims, x, w["w_router"], w["expert_bias"])[0]
    g = oracle.backward(dims, w, x, dy)
    used = set(ids.reshape(-1).tolist())
    for e in range(dims.n_routed):
        for name in ("w_g", "w_u", "w_o"):
            if e in used:
                assert np.abs(g[name][e]).sum() > 0
            else:
                assert (g[name][e] == 0).all()
        if e not in used:
            assert (g["w_router"][e] == 0).all()   # through p only: unselected rows get none


def test_backward_with_zero_up_projection():
    """W_up = 0 cuts the routed path: every routed, router, RMSNorm and W_down
    gradient is 0, dW_up = dy^T RMSNorm(u), and dx is the shared experts' alone."""
    dims, w, x, dy = _fd_case(seed=9)
    w["w_up"] = np.zeros_like(w["w_up"])
    g = oracle.backward(dims, w, x, dy)
    for name in ("w_g", "w_u", "w_o", "w_router", "w_down", "rms_weight"):
        assert (g[name] == 0).all(), name
    uhat = oracle.forward(dims, w, x, want=("uhat",))["uhat"]
    np.testing.assert_allclose(g["w_up"], dy.astype(np.float64).T @ uhat, rtol=1e-12, atol=1e-14)
    w2 = dict(w)
    w2["w_g"] = np.zeros_like(w["w_g"])
    w2["w_down"] = np.zeros_like(w["w_down"])
    np.testing.assert_allclose(oracle.backward(dims, w2, x, dy)["x"], g["x"], rtol=1e-13, atol=1e-15)
