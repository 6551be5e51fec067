"""Python binding of liblatent_moe.so, the B200 LatentMoE forward library.

Argument marshalling only: every function here passes torch tensors' device
pointers to the C ABI of the same name (include/latent_moe.h) and raises
:class:`LmoeError` on a non-OK status.  All work runs in the library's CUDA
kernels; there is no Python or CPU fallback.  If the shared library is
missing, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblatent_moe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python sigmoid_top_routing_latentmoe_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

OK, EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA, EDEVICE, ETIMEOUT = range(7)
F32, BF16 = 0, 1


class LmoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = _lib.lmoe_status_string(status).decode()
        msg = _lib.lmoe_last_error().decode()
        super().__init__(f"{where}: {name}: {msg}")


class Dims(ctypes.Structure):
    """lmoe_dims."""
    _fields_ = [("n_tokens", ctypes.c_int64), ("d", ctypes.c_int32), ("latent", ctypes.c_int32),
                ("n_routed", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("ff_routed", ctypes.c_int32),
                ("ff_shared", ctypes.c_int32), ("beta1", ctypes.c_float),
                ("beta2", ctypes.c_float), ("rms_eps", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("router", ctypes.c_int32)]


_P = ctypes.c_void_p
WEIGHT_NAMES = ("w_down", "w_router", "w_up", "rms_weight", "expert_bias",
                "w_g", "w_u", "w_o", "ws_g", "ws_u", "ws_o")


class Weights(ctypes.Structure):
    """lmoe_weights."""
    _fields_ = [(n, _P) for n in WEIGHT_NAMES]


GRAD_NAMES = ("dx", "dw_down", "dw_router", "dw_up", "drms_weight", "dw_g", "dw_u", "dw_o",
              "dws_g", "dws_u", "dws_o")


class Grads(ctypes.Structure):
    """lmoe_grads."""
    _fields_ = [(n, _P) for n in GRAD_NAMES]


_S = ctypes.c_int
_DP = ctypes.POINTER(Dims)
_sigs = {
    "lmoe_workspace_size": (ctypes.c_size_t, [_DP]),
    "lmoe_workspace_size_host": (ctypes.c_size_t, [_DP]),
    "moe_route": (_S, [_DP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_dispatch": (_S, [_DP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_dispatch_noalloc": (_S, [_DP, _P, _P, _P, _P, _P, _P]),
    "moe_expert_ffn": (_S, [_DP, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_combine": (_S, [_DP, _P, _P, _P, _P, _P, _P]),
    "moe_router_losses": (_S, [_DP, _P, ctypes.c_int64, _P, _P, _P, ctypes.c_size_t, _P]),
    "lmoe_backward_workspace_size": (ctypes.c_size_t, [_DP]),
    "lmoe_check_dispatch": (_S, [_DP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "latent_moe_backward": (_S, [_DP, ctypes.POINTER(Weights), _P, _P, ctypes.POINTER(Grads), _P,
                                 ctypes.c_size_t, _P]),
    "latent_moe_forward": (_S, [_DP, ctypes.POINTER(Weights), _P, _P, _P, _P, _P, _P,
                                ctypes.c_size_t, _P]),
    "latent_moe_forward_host": (_S, [_DP, ctypes.POINTER(Weights), _P, _P, _P, ctypes.c_size_t,
                                     _P]),
    "lmoe_workspace_init": (_S, [_P, ctypes.c_size_t, _P]),
    "lmoe_get_device_status": (_S, [_P, _P]),
    "lmoe_selftest_capped_wait": (_S, [_P, ctypes.c_size_t, ctypes.c_int32, _P]),
    "lmoe_status_string": (ctypes.c_char_p, [_S]),
    "lmoe_last_error": (ctypes.c_char_p, []),
    "lmoe_launch_count": (ctypes.c_uint64, [ctypes.c_int32]),
    "lmoe_profile_enable": (_S, [ctypes.c_char_p]),
    "lmoe_workspace_layout": (_S, [_DP, ctypes.POINTER(ctypes.c_size_t), ctypes.c_int32]),
    "lmoe_forward_plan": (_S, [_DP, ctypes.POINTER(ctypes.c_int32)]),
    "lmoe_profile_read": (_S, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]),
    "lmoe_profile_read_tag": (_S, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double),
                                   ctypes.POINTER(ctypes.c_int64)]),
    "lmoe_profile_peek_tag": (_S, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double),
                                   ctypes.POINTER(ctypes.c_int64)]),
}
for _name, (_res, _args) in _sigs.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


ROUTER_K3, ROUTER_SOFTMAX_TOPK = 0, 1


def make_dims(n_tokens, d, latent, n_routed, top_k, n_shared, ff_routed, ff_shared,
              beta1=4.0, beta2=25.0, rms_eps=1e-6, dtype=torch.bfloat16,
              router=ROUTER_K3) -> Dims:
    code = {torch.bfloat16: BF16, torch.float32: F32}[dtype]
    return Dims(n_tokens, d, latent, n_routed, top_k, n_shared, ff_routed, ff_shared,
                beta1, beta2, rms_eps, code, router)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return _P(torch.cuda.current_stream().cuda_stream)
    return _P(stream.cuda_stream if hasattr(stream, "cuda_stream") else stream)


def _check(status, where):
    if status != OK:
        raise LmoeError(status, where)


def workspace_size(dims: Dims, host: bool = False) -> int:
    n = (_lib.lmoe_workspace_size_host if host else _lib.lmoe_workspace_size)(ctypes.byref(dims))
    if n == 0:
        raise LmoeError(EINVAL, "workspace_size")
    return n


def alloc_workspace(dims: Dims, device="cuda", host: bool = False, stream=None) -> torch.Tensor:
    """A byte tensor of the required size (256-byte aligned), header zeroed."""
    n = workspace_size(dims, host)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + n]
    workspace_init(ws, stream)
    return ws


def workspace_views(dims: Dims, ws: torch.Tensor) -> dict:
    """Views of the forward's intermediates inside ``ws`` (for inspection)."""
    off = (ctypes.c_size_t * 11)()
    _check(_lib.lmoe_workspace_layout(ctypes.byref(dims), off, 11), "lmoe_workspace_layout")
    act = torch.bfloat16 if dims.dtype == BF16 else torch.float32
    es = 2 if dims.dtype == BF16 else 4
    N, L, k, F = dims.n_tokens, dims.latent, dims.top_k, dims.ff_routed
    SG = dims.n_shared * dims.ff_shared

    def view(o, rows, cols, dt, size):
        return ws[o:o + rows * cols * size].view(dt).view(rows, cols)

    return {"z": view(off[0], N, L, act, es),
            "logits": view(off[1], N, off[7], torch.float32, 4)[:, :dims.n_routed],
            "hsh": view(off[2], N, SG, act, es), "uhat": view(off[3], N, L, act, es),
            "eo": view(off[4], N * k, L, act, es), "h": view(off[5], N * k, F, act, es),
            "zp": view(off[6], N * k, L, act, es),
            "offsets": view(off[8], 1, dims.n_routed + 1, torch.int32, 4)[0],
            "perm": view(off[9], 1, N * k, torch.int32, 4)[0],
            "inv": view(off[10], N, k, torch.int32, 4)}


PLAN_BITS = {"combine_fused": 1, "xpass_wide": 2, "gemm1_pairs": 4, "gemm2_pairs": 8,
             "gemm1_wide": 16, "rows_in_scatter": 32, "counts_in_xpass": 64}


def forward_plan(dims: Dims) -> dict:
    """The launch plan of latent_moe_forward for ``dims`` (lmoe_forward_plan)."""
    f = ctypes.c_int32(0)
    _check(_lib.lmoe_forward_plan(ctypes.byref(dims), ctypes.byref(f)), "lmoe_forward_plan")
    return {name: bool(f.value & bit) for name, bit in PLAN_BITS.items()}


def workspace_init(ws: torch.Tensor, stream=None):
    _check(_lib.lmoe_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "lmoe_workspace_init")


def weights_struct(w: dict) -> Weights:
    return Weights(*[_ptr(w.get(n)) for n in WEIGHT_NAMES])


def moe_route(dims, x, w_router, expert_bias, ids, probs, ws, stream=None):
    _check(_lib.moe_route(ctypes.byref(dims), _ptr(x), _ptr(w_router), _ptr(expert_bias),
                          _ptr(ids), _ptr(probs), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_route")


def moe_dispatch(dims, ids, counts, offsets, perm_token, inv_pair, ws, stream=None):
    _check(_lib.moe_dispatch(ctypes.byref(dims), _ptr(ids), _ptr(counts), _ptr(offsets),
                             _ptr(perm_token), _ptr(inv_pair), _ptr(ws), ws.numel(),
                             _stream(stream)), "moe_dispatch")


def check_dispatch(dims, ids, counts, offsets, perm_token, inv_pair, ws, stream=None):
    """Device-side consistency check of a permutation; a violation sets EDEVICE
    in the workspace status word (lmoe_get_device_status)."""
    _check(_lib.lmoe_check_dispatch(ctypes.byref(dims), _ptr(ids), _ptr(counts), _ptr(offsets),
                                    _ptr(perm_token), _ptr(inv_pair), _ptr(ws), ws.numel(),
                                    _stream(stream)), "lmoe_check_dispatch")


def moe_dispatch_noalloc(dims, ids, counts, offsets, perm_token, inv_pair, stream=None):
    """moe_dispatch for callers that cannot provide a workspace (the library's
    fixed device scratch array is used; calls must not overlap on the GPU)."""
    _check(_lib.moe_dispatch_noalloc(ctypes.byref(dims), _ptr(ids), _ptr(counts), _ptr(offsets),
                                     _ptr(perm_token), _ptr(inv_pair), _stream(stream)),
           "moe_dispatch_noalloc")


def moe_expert_ffn(dims, z, perm_token, offsets, w_g, w_u, w_o, expert_out, ws, stream=None):
    _check(_lib.moe_expert_ffn(ctypes.byref(dims), _ptr(z), _ptr(perm_token), _ptr(offsets),
                               _ptr(w_g), _ptr(w_u), _ptr(w_o), _ptr(expert_out), _ptr(ws),
                               ws.numel(), _stream(stream)), "moe_expert_ffn")


def moe_combine(dims, expert_out, inv_pair, probs, rms_weight, u_normed, stream=None):
    _check(_lib.moe_combine(ctypes.byref(dims), _ptr(expert_out), _ptr(inv_pair), _ptr(probs),
                            _ptr(rms_weight), _ptr(u_normed), _stream(stream)), "moe_combine")


def moe_router_losses(dims, ids, out, ws, logits=None, ld=0, stream=None):
    """out [2 + 2R] fp32 <- aux, z, frac[R], prob_mean[R] (logits=None: those left
    in ``ws`` by the last moe_route / latent_moe_forward)."""
    _check(_lib.moe_router_losses(ctypes.byref(dims), _ptr(logits), ld, _ptr(ids), _ptr(out),
                                  _ptr(ws), ws.numel(), _stream(stream)), "moe_router_losses")


def latent_moe_forward(dims, weights, x, y, ws, ids_out=None, probs_out=None, counts_out=None,
                       stream=None):
    ws_struct = weights if isinstance(weights, Weights) else weights_struct(weights)
    _check(_lib.latent_moe_forward(ctypes.byref(dims), ctypes.byref(ws_struct), _ptr(x), _ptr(y),
                                   _ptr(ids_out), _ptr(probs_out), _ptr(counts_out), _ptr(ws),
                                   ws.numel(), _stream(stream)), "latent_moe_forward")


def alloc_backward_workspace(dims: Dims, device="cuda") -> torch.Tensor:
    """A 256-byte aligned byte tensor of lmoe_backward_workspace_size(dims)."""
    n = _lib.lmoe_backward_workspace_size(ctypes.byref(dims))
    if n == 0:
        raise LmoeError("lmoe_backward_workspace_size: " + _lib.lmoe_last_error().decode())
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def latent_moe_backward(dims, weights, x, dy, grads: dict, ws, stream=None):
    """grads: {name in GRAD_NAMES: fp32 tensor} (dws_* may be absent when S = 0)."""
    act = torch.bfloat16 if dims.dtype == BF16 else torch.float32
    for name, t in (("x", x), ("dy", dy)):
        if t.dtype != act or t.numel() != dims.n_tokens * dims.d or not t.is_contiguous():
            raise LmoeError(f"{name}: expected a contiguous {act} tensor of {dims.n_tokens}x{dims.d}")
    N, d, L, R, F, S, G = (dims.n_tokens, dims.d, dims.latent, dims.n_routed, dims.ff_routed,
                           dims.n_shared, dims.ff_shared)
    sizes = {"dx": N * d, "dw_down": L * d, "dw_router": R * d, "dw_up": d * L,
             "drms_weight": L, "dw_g": R * F * L, "dw_u": R * F * L, "dw_o": R * L * F,
             "dws_g": S * G * d, "dws_u": S * G * d, "dws_o": S * d * G}
    for name, n in sizes.items():
        t = grads.get(name)
        if n and (t is None or t.dtype != torch.float32 or t.numel() != n or not t.is_contiguous()):
            raise LmoeError(f"grads[{name}]: expected a contiguous float32 tensor of {n} elements")
    ws_struct = weights if isinstance(weights, Weights) else weights_struct(weights)
    g = Grads(*[_ptr(grads.get(n)) for n in GRAD_NAMES])
    _check(_lib.latent_moe_backward(ctypes.byref(dims), ctypes.byref(ws_struct), _ptr(x), _ptr(dy),
                                    ctypes.byref(g), _ptr(ws), ws.numel(), _stream(stream)),
           "latent_moe_backward")


def latent_moe_forward_host(dims, weights, x_host, y_host, ws, stream=None):
    ws_struct = weights if isinstance(weights, Weights) else weights_struct(weights)
    _check(_lib.latent_moe_forward_host(ctypes.byref(dims), ctypes.byref(ws_struct),
                                        _ptr(x_host), _ptr(y_host), _ptr(ws), ws.numel(),
                                        _stream(stream)), "latent_moe_forward_host")


def get_device_status(ws, stream=None) -> int:
    """Waits for the stream; returns (and clears) the workspace status code."""
    return _lib.lmoe_get_device_status(_ptr(ws), _stream(stream))


def selftest_capped_wait(ws, cap_ms: int, stream=None):
    _check(_lib.lmoe_selftest_capped_wait(_ptr(ws), ws.numel(), cap_ms, _stream(stream)),
           "lmoe_selftest_capped_wait")


def launch_count(reset: bool = False) -> int:
    return _lib.lmoe_launch_count(1 if reset else 0)


def profile_enable(tags):
    """Brackets every launch of the kernels in ``tags`` ("a,b", "*" or None: off)."""
    _check(_lib.lmoe_profile_enable(None if tags is None else tags.encode()), "lmoe_profile_enable")


def profile_read(tag=None):
    """(summed device ms, launches) of the bracketed kernel ``tag`` (None: all)
    since the last read."""
    ms, n = ctypes.c_double(), ctypes.c_int64()
    _check(_lib.lmoe_profile_read_tag(None if tag is None else tag.encode(), ctypes.byref(ms),
                                      ctypes.byref(n)), "lmoe_profile_read_tag")
    return ms.value, n.value


def profile_peek(tag=None):
    """(summed device ms, launches) of the bracketed kernel ``tag``, keeping the
    events (for launches inside a CUDA graph, re-recorded on every replay)."""
    ms, n = ctypes.c_double(), ctypes.c_int64()
    _check(_lib.lmoe_profile_peek_tag(None if tag is None else tag.encode(), ctypes.byref(ms),
                                      ctypes.byref(n)), "lmoe_profile_peek_tag")
    return ms.value, n.value


def status_string(code: int) -> str:
    return _lib.lmoe_status_string(code).decode()
