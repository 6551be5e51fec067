"""Seeded synthetic inputs for the LatentMoE layer (random draws only).

This package holds no step of the layer's arithmetic.  It draws the layer input
x and every weight from a counter-based generator (``synth.c``) so that the CUDA
library's tests and benchmark and the CPU oracle see the same bytes, and it
states the five workload shapes the library is measured and tested on.

Workloads (sizes, dtypes and value distributions):

=============  =====  ====  ====  ========  ====  =======  =====  ===============================
name           N      d     l     R / k     F     S / G    dtype  values
=============  =====  ====  ====  ========  ====  =======  =====  ===============================
toy_fp32       128    256   128   16 / 2    256   2 / 512  f32    b = 0
halfb_uniform  4096   768   384   16 / 2    768   2 / 1536 bf16   b = 0
halfb_skewed   4096   768   384   16 / 2    768   2 / 1536 bf16   +2 logit offset e0-3, b~U(-.5,.5)
mid            16384  2048  1024  64 / 8    1024  1 / 4096 bf16   b ~ N(0, 0.01^2)
k3_width       8192   7168  3584  896 / 16  512   1 / 2048 bf16   b = 0
=============  =====  ====  ====  ========  ====  =======  =====  ===============================

Everywhere: x ~ N(0, 1); every weight matrix ~ N(0, 0.02^2); RMSNorm weight 1,
eps 1e-6; beta1 = 4, beta2 = 25.  The skewed workload realises its +2.0 logit
offset for experts 0-3 through a constant input channel: x[:, d-1] = 1 and
W_r[0:4, d-1] = 2, so those four logits carry an exact +2.0 term.

bf16 tensors are returned as raw ``uint16`` arrays (use :func:`to_f32`), fp32
ones as ``float32``.  The expert bias and the RMSNorm weight are always fp32.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None
_P = ctypes.c_void_p


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        u64, i64, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
        for f in ("synth_normal_f32", "synth_normal_bf16", "synth_uniform_f32"):
            getattr(_lib, f).argtypes = [u64, u64, i64, i64, dbl, dbl, _P]
            getattr(_lib, f).restype = None
        _lib.synth_bf16_to_f32.argtypes = [i64, _P, _P]
        _lib.synth_f32_to_bf16.argtypes = [i64, _P, _P]
    return _lib


def tag_id(tag: str) -> int:
    """64-bit FNV-1a hash of a tensor's name: the stream id of that tensor."""
    h = 0xCBF29CE484222325
    for byte in tag.encode():
        h ^= byte
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def normal(seed: int, tag: str, shape, std: float = 1.0, mean: float = 0.0,
           dtype: str = "bf16", offset: int = 0) -> np.ndarray:
    """Draws ``mean + std * N(0,1)`` for counters offset .. offset+size-1."""
    n = int(np.prod(shape))
    if dtype == "bf16":
        out = np.empty(shape, np.uint16)
        _load().synth_normal_bf16(seed, tag_id(tag), offset, n, mean, std, out.ctypes.data)
    elif dtype == "f32":
        out = np.empty(shape, np.float32)
        _load().synth_normal_f32(seed, tag_id(tag), offset, n, mean, std, out.ctypes.data)
    else:
        raise ValueError(dtype)
    return out


def uniform(seed: int, tag: str, shape, lo: float, hi: float, offset: int = 0) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(shape, np.float32)
    _load().synth_uniform_f32(seed, tag_id(tag), offset, n, lo, hi, out.ctypes.data)
    return out


def to_f32(a: np.ndarray) -> np.ndarray:
    """bf16 (raw uint16) -> float32 exactly; float32 passes through."""
    if a.dtype == np.float32:
        return a
    assert a.dtype == np.uint16
    a = np.ascontiguousarray(a)
    out = np.empty(a.shape, np.float32)
    _load().synth_bf16_to_f32(a.size, a.ctypes.data, out.ctypes.data)
    return out


def to_bf16(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 (raw uint16), round to nearest even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, np.uint16)
    _load().synth_f32_to_bf16(a.size, a.ctypes.data, out.ctypes.data)
    return out


@dataclass(frozen=True)
class Workload:
    name: str
    n_tokens: int
    d: int
    latent: int
    n_routed: int
    top_k: int
    ff_routed: int
    n_shared: int
    ff_shared: int
    dtype: str                    # "bf16" or "f32"
    bias: tuple = ("zero",)       # ("zero",) | ("uniform", lo, hi) | ("normal", std)
    skew_experts: int = 0         # experts 0..skew_experts-1 get the +2.0 logit offset
    x_std: float = 1.0
    w_std: float = 0.02
    beta1: float = 4.0
    beta2: float = 25.0
    rms_eps: float = 1e-6
    router: int = 0               # 0: K3 sigmoid routing; 1: softmax over the top-k logits
    extra: dict = field(default_factory=dict, compare=False)

    def with_tokens(self, n: int) -> "Workload":
        return Workload(self.name, n, self.d, self.latent, self.n_routed, self.top_k,
                        self.ff_routed, self.n_shared, self.ff_shared, self.dtype, self.bias,
                        self.skew_experts, self.x_std, self.w_std, self.beta1, self.beta2,
                        self.rms_eps, self.router)

    def replace(self, **kw) -> "Workload":
        fields = dict(name=self.name, n_tokens=self.n_tokens, d=self.d, latent=self.latent,
                      n_routed=self.n_routed, top_k=self.top_k, ff_routed=self.ff_routed,
                      n_shared=self.n_shared, ff_shared=self.ff_shared, dtype=self.dtype,
                      bias=self.bias, skew_experts=self.skew_experts, x_std=self.x_std,
                      w_std=self.w_std, beta1=self.beta1, beta2=self.beta2, rms_eps=self.rms_eps,
                      router=self.router)
        fields.update(kw)
        return Workload(**fields)

    # Algorithmic work of one forward over all N tokens (only the k selected experts).
    def flops(self) -> float:
        d, L, R, k, F, S, G = (self.d, self.latent, self.n_routed, self.top_k, self.ff_routed,
                               self.n_shared, self.ff_shared)
        per_tok = 2 * d * L + 2 * d * R + 6 * k * L * F + 6 * S * d * G + 2 * L * d
        return float(per_tok) * self.n_tokens

    def compulsory_bytes(self, experts_used=None) -> float:
        """Every weight once + x + y (intermediates are implementation traffic).
        experts_used: how many routed experts the routing selected at least once
        (default all R); only their weights must be read."""
        es = 2 if self.dtype == "bf16" else 4
        d, L, R, F, S, G = (self.d, self.latent, self.n_routed, self.ff_routed, self.n_shared,
                            self.ff_shared)
        used = R if experts_used is None else experts_used
        weights = (L * d + R * d + d * L + 3 * used * F * L + 3 * S * G * d) * es + (L + R) * 4
        return float(weights + 2 * self.n_tokens * d * es)


WORKLOADS = {
    "toy_fp32": Workload("toy_fp32", 128, 256, 128, 16, 2, 256, 2, 512, "f32"),
    "halfb_uniform": Workload("halfb_uniform", 4096, 768, 384, 16, 2, 768, 2, 1536, "bf16"),
    "halfb_skewed": Workload("halfb_skewed", 4096, 768, 384, 16, 2, 768, 2, 1536, "bf16",
                             bias=("uniform", -0.5, 0.5), skew_experts=4),
    "mid": Workload("mid", 16384, 2048, 1024, 64, 8, 1024, 1, 4096, "bf16",
                    bias=("normal", 0.01)),
    "k3_width": Workload("k3_width", 8192, 7168, 3584, 896, 16, 512, 1, 2048, "bf16"),
    # a decode-sized step of the K3-width layer: 64 tokens, ~1.1 pairs per expert,
    # about 610 of the 896 experts selected: streaming their weights dominates
    "k3_decode": Workload("k3_decode", 64, 7168, 3584, 896, 16, 512, 1, 2048, "bf16"),
}


def make_x_rows(wl: Workload, seed: int, rows, redraw_round: int = 0) -> np.ndarray:
    """x rows for the given token indices.  Redraw 0 is the base draw; redraw r > 0
    is an independent draw of the same rows (stream "x.redraw.<r>")."""
    rows = np.asarray(rows, dtype=np.int64)
    tag = "x" if redraw_round == 0 else f"x.redraw.{redraw_round}"
    out = np.empty((len(rows), wl.d), np.uint16 if wl.dtype == "bf16" else np.float32)
    # consecutive runs are drawn in one call
    i = 0
    while i < len(rows):
        j = i
        while j + 1 < len(rows) and rows[j + 1] == rows[j] + 1:
            j += 1
        out[i:j + 1] = normal(seed, tag, (j - i + 1, wl.d), wl.x_std, dtype=wl.dtype,
                              offset=int(rows[i]) * wl.d)
        i = j + 1
    if wl.skew_experts:
        out[:, wl.d - 1] = _one(wl.dtype)
    return out


def _one(dtype):
    return np.uint16(0x3F80) if dtype == "bf16" else np.float32(1.0)


def make_inputs(wl: Workload, seed: int = 0, with_x: bool = True) -> dict:
    """All inputs of one workload: x [N,d] and the weights in nn.Linear layout."""
    dt, s = wl.dtype, wl.w_std
    d, L, R, F, S, G = wl.d, wl.latent, wl.n_routed, wl.ff_routed, wl.n_shared, wl.ff_shared
    inp = {}
    if with_x:
        inp["x"] = make_x_rows(wl, seed, np.arange(wl.n_tokens))
    inp["w_down"] = normal(seed, "w_down", (L, d), s, dtype=dt)
    w_r = normal(seed, "w_router", (R, d), s, dtype=dt)
    if wl.skew_experts:
        w_r[:wl.skew_experts, d - 1] = np.uint16(0x4000) if dt == "bf16" else np.float32(2.0)
    inp["w_router"] = w_r
    inp["w_up"] = normal(seed, "w_up", (d, L), s, dtype=dt)
    inp["rms_weight"] = np.ones(L, np.float32)
    kind = wl.bias[0]
    if kind == "zero":
        inp["expert_bias"] = np.zeros(R, np.float32)
    elif kind == "uniform":
        inp["expert_bias"] = uniform(seed, "expert_bias", (R,), wl.bias[1], wl.bias[2])
    elif kind == "normal":
        inp["expert_bias"] = normal(seed, "expert_bias", (R,), wl.bias[1], dtype="f32")
    else:
        raise ValueError(kind)
    inp["w_g"] = normal(seed, "w_g", (R, F, L), s, dtype=dt)
    inp["w_u"] = normal(seed, "w_u", (R, F, L), s, dtype=dt)
    inp["w_o"] = normal(seed, "w_o", (R, L, F), s, dtype=dt)
    inp["ws_g"] = normal(seed, "ws_g", (S, G, d), s, dtype=dt)
    inp["ws_u"] = normal(seed, "ws_u", (S, G, d), s, dtype=dt)
    inp["ws_o"] = normal(seed, "ws_o", (S, d, G), s, dtype=dt)
    return inp


WEIGHT_NAMES = ("w_down", "w_router", "w_up", "rms_weight", "expert_bias",
                "w_g", "w_u", "w_o", "ws_g", "ws_u", "ws_o")
