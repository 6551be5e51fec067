"""Routing-margin conditioning of synthetic inputs -- test infrastructure.

Top-k selection is a discrete decision taken from floating-point keys s + b.
The CUDA path forms the router logits in fp32 from bf16 operands; the oracle
forms them in double.  The two orders of summation differ by far less than
1e-4 in a key, so when every token has a gap of at least ``margin`` between
its k-th and (k+1)-th largest key, both sides must select the same experts,
and routing ids, counts, offsets and the permutation can be compared bit for
bit.  The slot order is a floating-point decision too (descending key), so
the selected keys must also stay ``order_margin`` (1e-5) apart from one
another.  This module finds the tokens under either margin (with the oracle's
router) and replaces their x rows by independent redraws from ``synth`` until
none is left.  It changes inputs only; it computes nothing the tests compare.
"""
from __future__ import annotations

import numpy as np

import synth

from . import Dims, route


def topk_gap(keys: np.ndarray, k: int) -> np.ndarray:
    """Per-row gap between the k-th and (k+1)-th largest key (inf when k == R)."""
    R = keys.shape[1]
    if k >= R:
        return np.full(keys.shape[0], np.inf)
    part = -np.partition(-keys, (k - 1, k), axis=1)
    return part[:, k - 1] - part[:, k]


def order_gap(keys: np.ndarray, k: int) -> np.ndarray:
    """Per-row smallest gap between consecutive keys among the k largest (inf if k == 1)."""
    if k <= 1:
        return np.full(keys.shape[0], np.inf)
    top = -np.sort(-keys, axis=1)[:, :k]
    return (top[:, :-1] - top[:, 1:]).min(axis=1)


def enforce_topk_margin(wl: synth.Workload, inputs: dict, seed: int = 0, margin: float = 1e-4,
                        rows=None, max_rounds: int = 200, order_margin: float = 1e-5) -> dict:
    """Redraws, in place, the x rows (all tokens, or ``rows``) whose gap between
    the k-th and (k+1)-th key is below ``margin`` (it decides the selected set),
    or whose selected keys come closer than ``order_margin`` to one another (it
    decides the slot order).  Returns {'redrawn': rows_redrawn, 'rounds': r}."""
    x = inputs["x"]
    w_r = synth.to_f32(inputs["w_router"])
    b = inputs["expert_bias"]
    todo = np.arange(wl.n_tokens) if rows is None else np.unique(np.asarray(rows, np.int64))
    redrawn = 0
    for rnd in range(1, max_rounds + 1):
        if len(todo) == 0:
            return {"redrawn": redrawn, "rounds": rnd - 1}
        xf = synth.to_f32(x[todo])
        dims = Dims(len(todo), wl.d, wl.latent, wl.n_routed, wl.top_k, wl.n_shared,
                    wl.ff_routed, wl.ff_shared, router=wl.router)
        _, _, keys, _ = route(dims, xf, w_r, b)
        bad = todo[(topk_gap(keys, wl.top_k) < margin) |
                   (order_gap(keys, wl.top_k) < order_margin)]
        if len(bad) == 0:
            return {"redrawn": redrawn, "rounds": rnd - 1}
        x[bad] = synth.make_x_rows(wl, seed, bad, redraw_round=rnd)
        redrawn += len(bad)
        todo = bad
    raise RuntimeError(f"top-k margin not reached after {max_rounds} redraw rounds")
