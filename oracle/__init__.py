"""LatentMoE forward oracle -- test infrastructure, not part of the product.

A ctypes binding over ``latent_moe_oracle.c``: a plain, slow, double-precision
CPU restatement of the LatentMoE feed-forward layer (K3 notes sec-07, "SiTU-GLU
与 Stable LatentMoE"; kda/layers/latent_moe.py in the K3 compare view).  Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import it.  It shares no code with the CUDA library.

Every function takes float32 numpy arrays (bf16 inputs widened exactly) and
returns float64 results, int32 for ids and permutation arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "latent_moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE arithmetic, OpenMP over tokens)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


class _Dims(ctypes.Structure):
    _fields_ = [
        ("n_tokens", ctypes.c_int64),
        ("d", ctypes.c_int32),
        ("latent", ctypes.c_int32),
        ("n_routed", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("n_shared", ctypes.c_int32),
        ("ff_routed", ctypes.c_int32),
        ("ff_shared", ctypes.c_int32),
        ("beta1", ctypes.c_double),
        ("beta2", ctypes.c_double),
        ("rms_eps", ctypes.c_double),
        ("router", ctypes.c_int32),
    ]


_P = ctypes.c_void_p


class _Weights(ctypes.Structure):
    _fields_ = [(name, _P) for name in (
        "w_down", "w_router", "w_up", "rms_weight", "expert_bias",
        "w_g", "w_u", "w_o", "ws_g", "ws_u", "ws_o")]


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.orc_situ.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_double, ctypes.c_double,
                                  _P, _P, _P, _P, _P, _P]
        _lib.orc_route.argtypes = [ctypes.POINTER(_Dims), _P, _P, _P, _P, _P, _P, _P]
        _lib.orc_permute.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                     _P, _P, _P, _P, _P]
        _lib.orc_forward.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Weights), _P, _P,
                                     _P, _P, _P, _P, _P, _P, _P]
        _lib.orc_forward_dense.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Weights),
                                           _P, _P, _P]
        _lib.orc_rmsnorm_rows.argtypes = [ctypes.c_int64, ctypes.c_int32, _P, _P,
                                          ctypes.c_double, _P]
        _lib.orc_router_losses.argtypes = [ctypes.POINTER(_Dims), _P, _P, _P, _P]
        _lib.orc_backward.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Weights), _P, _P] + [_P] * 11
        for f in ("orc_situ", "orc_route", "orc_permute", "orc_forward", "orc_forward_dense",
                  "orc_rmsnorm_rows", "orc_router_losses", "orc_backward"):
            getattr(_lib, f).restype = None
    return _lib


@dataclass(frozen=True)
class Dims:
    """LatentMoE layer sizes (the pages' LatentMoE constructor, with B*T flattened to N)."""
    n_tokens: int
    d: int
    latent: int
    n_routed: int
    top_k: int
    n_shared: int
    ff_routed: int
    ff_shared: int
    beta1: float = 4.0
    beta2: float = 25.0
    rms_eps: float = 1e-6
    router: int = 0          # 0: K3 sigmoid routing; 1: softmax over the top-k logits

    def _c(self) -> _Dims:
        return _Dims(self.n_tokens, self.d, self.latent, self.n_routed, self.top_k,
                     self.n_shared, self.ff_routed, self.ff_shared,
                     self.beta1, self.beta2, self.rms_eps, self.router)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data


_WEIGHT_NAMES = ("w_down", "w_router", "w_up", "rms_weight", "expert_bias",
                 "w_g", "w_u", "w_o", "ws_g", "ws_u", "ws_o")


def _weights(w: dict):
    keep = {}
    for name in _WEIGHT_NAMES:
        v = w.get(name)
        keep[name] = None if v is None else _f32(v)
    cw = _Weights(*[_ptr(keep[n]) for n in _WEIGHT_NAMES])
    return cw, keep


def situ(w_g, w_u, w_o, v, beta1=4.0, beta2=25.0):
    """One SiTU-GLU expert on one vector; returns (out, hidden = gate*up)."""
    w_g, w_u, w_o = _f32(w_g), _f32(w_u), _f32(w_o)
    ff, dim_in = w_g.shape
    assert w_u.shape == (ff, dim_in) and w_o.shape == (dim_in, ff)
    v = np.ascontiguousarray(v, dtype=np.float64).reshape(dim_in)
    out = np.empty(dim_in, np.float64)
    hidden = np.empty(ff, np.float64)
    _load().orc_situ(dim_in, ff, beta1, beta2, _ptr(w_g), _ptr(w_u), _ptr(w_o), _ptr(v),
                     _ptr(out), _ptr(hidden))
    return out, hidden


def route(dims: Dims, x, w_router, expert_bias=None):
    """Routing for all tokens (K3 sigmoid, or dims.router == 1: softmax over the
    top-k logits): returns ids [N,k] int32, probs [N,k], keys [N,R] (the
    selection keys), scores [N,R] (sigmoid of the logits)."""
    x, w_router = _f32(x), _f32(w_router)
    b = None if expert_bias is None else _f32(expert_bias)
    N, k, R = dims.n_tokens, dims.top_k, dims.n_routed
    assert x.shape == (N, dims.d) and w_router.shape == (R, dims.d)
    ids = np.empty((N, k), np.int32)
    probs = np.empty((N, k), np.float64)
    keys = np.empty((N, R), np.float64)
    scores = np.empty((N, R), np.float64)
    c = dims._c()
    _load().orc_route(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(b), _ptr(ids), _ptr(probs),
                      _ptr(keys), _ptr(scores))
    return ids, probs, keys, scores


def router_losses(dims: Dims, x, w_router, ids):
    """Balancing losses before their coefficients: {'aux', 'z', 'frac' [R], 'prob_mean' [R]}."""
    x, w_router = _f32(x), _f32(w_router)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    R = dims.n_routed
    assert x.shape == (dims.n_tokens, dims.d) and ids.shape == (dims.n_tokens, dims.top_k)
    out = np.empty(2 + 2 * R, np.float64)
    c = dims._c()
    _load().orc_router_losses(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(ids), _ptr(out))
    return {"aux": float(out[0]), "z": float(out[1]), "frac": out[2:2 + R].copy(),
            "prob_mean": out[2 + R:].copy()}


GRAD_NAMES = ("x", "w_down", "w_router", "w_up", "rms_weight", "w_g", "w_u", "w_o",
              "ws_g", "ws_u", "ws_o")


def backward(dims: Dims, weights: dict, x, dy):
    """Gradients of <dy, y> (y the layer's output) with respect to x and every
    weight except expert_bias (which only selects): {name: float64 array}."""
    cw, keep = _weights(weights)
    x = _f32(x)
    dy = _f32(dy)
    N, d, L, R, F, S, G = (dims.n_tokens, dims.d, dims.latent, dims.n_routed, dims.ff_routed,
                           dims.n_shared, dims.ff_shared)
    assert x.shape == (N, d) and dy.shape == (N, d)
    shapes = {"x": (N, d), "w_down": (L, d), "w_router": (R, d), "w_up": (d, L),
              "rms_weight": (L,), "w_g": (R, F, L), "w_u": (R, F, L), "w_o": (R, L, F),
              "ws_g": (max(S, 1), G, d), "ws_u": (max(S, 1), G, d), "ws_o": (max(S, 1), d, G)}
    out = {n: np.zeros(shapes[n], np.float64) for n in GRAD_NAMES}
    c = dims._c()
    _load().orc_backward(ctypes.byref(c), ctypes.byref(cw), _ptr(x), _ptr(dy),
                         *[_ptr(out[n]) for n in GRAD_NAMES])
    if S == 0:
        for n in ("ws_g", "ws_u", "ws_o"):
            out[n] = out[n][:0]
    return out


def permute(ids, n_routed: int):
    """Stable expert-major permutation of the token-expert pairs.

    Returns counts [R], offsets [R+1], perm_token [N*k], inv_pair [N,k] (int32)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    N, k = ids.shape
    counts = np.empty(n_routed, np.int32)
    offsets = np.empty(n_routed + 1, np.int32)
    perm_token = np.empty(N * k, np.int32)
    inv_pair = np.empty((N, k), np.int32)
    _load().orc_permute(N, k, n_routed, _ptr(ids), _ptr(counts), _ptr(offsets), _ptr(perm_token),
                        _ptr(inv_pair))
    return counts, offsets, perm_token, inv_pair


def forward(dims: Dims, weights: dict, x, want=()):
    """Token-wise LatentMoE forward.  Returns a dict with y, ids, probs and any of
    'z', 'u', 'uhat', 'shared', 'routed' listed in ``want``."""
    x = _f32(x)
    N, d, L, k = dims.n_tokens, dims.d, dims.latent, dims.top_k
    assert x.shape == (N, d)
    cw, keep = _weights(weights)
    out = {"y": np.empty((N, d), np.float64), "ids": np.empty((N, k), np.int32),
           "probs": np.empty((N, k), np.float64)}
    shapes = {"z": (N, L), "u": (N, L), "uhat": (N, L), "shared": (N, d), "routed": (N, k, L)}
    for name in want:
        out[name] = np.empty(shapes[name], np.float64)
    c = dims._c()
    _load().orc_forward(ctypes.byref(c), ctypes.byref(cw), _ptr(x), _ptr(out["y"]),
                        _ptr(out["ids"]), _ptr(out["probs"]), _ptr(out.get("z")),
                        _ptr(out.get("u")), _ptr(out.get("uhat")), _ptr(out.get("shared")),
                        _ptr(out.get("routed")))
    del keep
    return out


def forward_dense(dims: Dims, weights: dict, x):
    """Dense all-experts evaluation (the pages' _dense_moe_forward); returns (y, u)."""
    x = _f32(x)
    N, d, L = dims.n_tokens, dims.d, dims.latent
    cw, keep = _weights(weights)
    y = np.empty((N, d), np.float64)
    u = np.empty((N, L), np.float64)
    c = dims._c()
    _load().orc_forward_dense(ctypes.byref(c), ctypes.byref(cw), _ptr(x), _ptr(y), _ptr(u))
    del keep
    return y, u


def rmsnorm(u, w, eps=1e-6):
    """RMSNorm of each row of u (float64) with weight w."""
    u = np.ascontiguousarray(u, dtype=np.float64)
    N, n = u.shape
    w = _f32(w)
    out = np.empty_like(u)
    _load().orc_rmsnorm_rows(N, n, _ptr(u), _ptr(w), eps, _ptr(out))
    return out
