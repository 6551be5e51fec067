"""Helpers shared by the GPU parity tests: inputs from ``synth``, their device
copies, and the oracle's view of the same bytes."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
from oracle.conditioning import enforce_topk_margin

MARGIN = 1e-4          # routing margin of the parity inputs (see oracle.conditioning)
Y_REL_TOL_BF16 = 2e-2  # max|y_gpu - y_ref| <= tol * max|y_ref|
Y_REL_TOL_F32 = 1e-5
P_ABS_TOL = 1e-6       # routing weights


def odims(wl: synth.Workload, n=None) -> oracle.Dims:
    return oracle.Dims(wl.n_tokens if n is None else n, wl.d, wl.latent, wl.n_routed, wl.top_k,
                       wl.n_shared, wl.ff_routed, wl.ff_shared, wl.beta1, wl.beta2, wl.rms_eps,
                       wl.router)


def ldims(wl: synth.Workload, n=None):
    import sigmoid_top_routing_latentmoe_b200 as lm
    return lm.make_dims(wl.n_tokens if n is None else n, wl.d, wl.latent, wl.n_routed, wl.top_k,
                        wl.n_shared, wl.ff_routed, wl.ff_shared, wl.beta1, wl.beta2, wl.rms_eps,
                        torch.bfloat16 if wl.dtype == "bf16" else torch.float32, wl.router)


def prepare(wl: synth.Workload, seed: int = 0, margin_rows=None, margin: float = MARGIN) -> dict:
    """Inputs with the routing margin enforced on all rows (or on ``margin_rows``)."""
    inp = synth.make_inputs(wl, seed)
    enforce_topk_margin(wl, inp, seed, margin=margin, rows=margin_rows)
    return inp


def to_device(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(device)
    if a.dtype == np.float32:
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)
    if a.dtype == np.int32:
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)
    raise TypeError(a.dtype)


def device_inputs(inp: dict, device="cuda") -> dict:
    return {k: to_device(v, "", device) for k, v in inp.items()}


def oracle_weights(inp: dict) -> dict:
    return {k: synth.to_f32(inp[k]) for k in synth.WEIGHT_NAMES}


def act_dtype(wl: synth.Workload):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def round_act(a: np.ndarray, wl: synth.Workload) -> np.ndarray:
    """Rounds float values to the workload's activation dtype (as float32)."""
    a = np.asarray(a, np.float32)
    return synth.to_f32(synth.to_bf16(a)) if wl.dtype == "bf16" else a


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    return float(np.abs(np.asarray(got, np.float64) - ref).max() / max(scale, 1e-300))


def y_tol(wl: synth.Workload) -> float:
    return Y_REL_TOL_BF16 if wl.dtype == "bf16" else Y_REL_TOL_F32


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def check_permutation_properties(ids: np.ndarray, counts, offsets, perm_token, inv_pair, R: int):
    """What the stable expert-major permutation must satisfy at any size."""
    N, k = ids.shape
    P = N * k
    eid = ids.reshape(-1)
    assert counts.sum() == P
    np.testing.assert_array_equal(counts, np.bincount(eid, minlength=R))
    assert offsets[0] == 0 and offsets[-1] == P
    np.testing.assert_array_equal(np.diff(offsets), counts)
    inv = inv_pair.reshape(-1).astype(np.int64)
    # a bijection between pairs and sorted slots, consistent with perm_token
    assert np.array_equal(np.sort(inv), np.arange(P))
    np.testing.assert_array_equal(perm_token[inv], np.arange(P) // k)
    # slot of pair p lies in its expert's segment, tokens ascending inside it
    assert (inv >= offsets[eid]).all() and (inv < offsets[eid + 1]).all()
    seg_expert = np.repeat(np.arange(R), counts)
    d = np.diff(perm_token.astype(np.int64))
    same = seg_expert[1:] == seg_expert[:-1]
    assert (d[same] > 0).all()
