"""Grok-1 mixture-of-experts feed-forward layer on NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libmoe_b200.so``, whose C ABI is declared in
``include/moe.h``.  Each function here has the name of its C entry point and
only marshals arguments: tensors become device (or host) pointers, the stream
becomes a ``cudaStream_t``.  Every step of the layer runs in the library's
CUDA kernels; there is no CPU or PyTorch fallback, and importing this package
fails loudly if the library has not been built.

Functions return the library's integer status (``MOE_OK`` = 0); ``check`` turns
a non-zero status into ``MoEError``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_EINVAL = -1
MOE_EUNSUPPORTED = -2
MOE_ENOMEM = -3
MOE_ECUDA = -4
MOE_ETIMEOUT = -5
MOE_ENODEV = -6
MOE_ERANGE = -7
MOE_MAX_TOKENS = 262144
MOE_LAYOUT_IN_OUT = 0
MOE_LAYOUT_PACKED = 1
MOE_NOALLOC_MAX_TOKENS = 65536

KERNEL_NAMES = ("router", "dispatch", "gather", "up_proj", "down_proj", "combine", "prenorm", "route_small")

# every symbol include/moe.h declares
EXPORTS = (
    "moe_strerror", "moe_version", "moe_create", "moe_destroy", "moe_set_router_bias", "moe_set_padding_mask",
    "moe_set_scale_block",
    "moe_forward", "moe_forward_host", "moe_block_forward", "moe_get_routing", "moe_get_block_input",
    "moe_sync_status", "moe_set_timeout", "moe_set_profiling", "moe_get_kernel_times", "moe_plan",
    "moe_set_weight_layout", "moe_pack_weight", "moe_route_noalloc",
    "moe_ep_dispatch", "moe_ep_experts", "moe_ep_combine", "moe_set_cta_pairs", "moe_pack_weight_n",
    "moe_set_host_overlap", "moe_host_wait",
)


class MoEError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {moe_strerror(code)} ({code})" if what else f"{moe_strerror(code)} ({code})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python mixture_experts_softmax_b200/build.py` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    sig = {
        "moe_strerror": (ctypes.c_char_p, [I]),
        "moe_version": (I, []),
        "moe_create": (I, [I, I, I, I, ctypes.POINTER(P)]),
        "moe_destroy": (I, [P]),
        "moe_set_router_bias": (I, [P, P]),
        "moe_set_padding_mask": (I, [P, P]),
        "moe_set_scale_block": (I, [P, I]),
        "moe_forward": (I, [P, I, P, P, P, P, P, P, P, P, P, P]),
        "moe_forward_host": (I, [P, I, P, P, P, P, P, P, P, P, P, P]),
        "moe_block_forward": (I, [P, I, P, P, P, F, P, P, P, P, P, P, P, P]),
        "moe_get_routing": (I, [P, P, P, P, P, P]),
        "moe_get_block_input": (I, [P, P, P]),
        "moe_sync_status": (I, [P, P]),
        "moe_set_timeout": (I, [P, ctypes.c_longlong]),
        "moe_set_profiling": (I, [P, I]),
        "moe_get_kernel_times": (I, [P, P, P, I]),
        "moe_plan": (I, [P, I, ctypes.POINTER(I), ctypes.POINTER(I)]),
        "moe_set_weight_layout": (I, [P, I]),
        "moe_pack_weight": (I, [P, P, P, I, P]),
        "moe_pack_weight_n": (I, [P, P, P, I, I, P]),
        "moe_route_noalloc": (I, [I, I, P, P, P, P, P, P, P, P]),
        "moe_ep_dispatch": (I, [P, I, P, P, P, P, P]),
        "moe_ep_experts": (I, [P, I, I, P, P, P, P, P, P, P, P, P, P]),
        "moe_ep_combine": (I, [P, I, P, P, P]),
        "moe_set_cta_pairs": (I, [P, I]),
        "moe_set_host_overlap": (I, [P, I]),
        "moe_host_wait": (I, [P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def _ptr(t) -> Optional[int]:
    """torch tensor / int / None -> raw address."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    raise TypeError(f"cannot pass {type(t).__name__} as a pointer")


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def check(rc: int, what: str = "") -> None:
    if rc != MOE_OK:
        raise MoEError(rc, what)


def moe_strerror(code: int) -> str:
    return _lib.moe_strerror(int(code)).decode()


def moe_version() -> int:
    return _lib.moe_version()


def moe_create(d: int, ffn: int, E: int = 8, k: int = 2) -> Tuple[int, Optional[int]]:
    h = ctypes.c_void_p()
    rc = _lib.moe_create(d, ffn, E, k, ctypes.byref(h))
    return rc, h.value


def moe_destroy(h) -> int:
    return _lib.moe_destroy(h)


def moe_set_router_bias(h, bias) -> int:
    return _lib.moe_set_router_bias(h, _ptr(bias))


def moe_set_padding_mask(h, mask) -> int:
    """mask: device uint8 [T] (0 = padding token) or None; kept, not copied."""
    return _lib.moe_set_padding_mask(h, _ptr(mask))


def moe_set_scale_block(h, kb: int) -> int:
    """0: per-output-channel scales; 128: per block of 128 input rows ([E, in/128, out])."""
    return _lib.moe_set_scale_block(h, int(kb))


def moe_forward(h, T, x, router_w, w_lin, s_lin, w_v, s_v, w_1, s_1, out, stream=None) -> int:
    return _lib.moe_forward(h, int(T), _ptr(x), _ptr(router_w), _ptr(w_lin), _ptr(s_lin), _ptr(w_v),
                            _ptr(s_v), _ptr(w_1), _ptr(s_1), _ptr(out), _stream(stream))


def moe_forward_host(h, T, x_host, router_w, w_lin, s_lin, w_v, s_v, w_1, s_1, out_host, stream=None) -> int:
    return _lib.moe_forward_host(h, int(T), _ptr(x_host), _ptr(router_w), _ptr(w_lin), _ptr(s_lin),
                                 _ptr(w_v), _ptr(s_v), _ptr(w_1), _ptr(s_1), _ptr(out_host), _stream(stream))


def moe_block_forward(h, T, h_io, g_pre, g_post, eps, router_w, w_lin, s_lin, w_v, s_v, w_1, s_1,
                      stream=None) -> int:
    return _lib.moe_block_forward(h, int(T), _ptr(h_io), _ptr(g_pre), _ptr(g_post), float(eps),
                                  _ptr(router_w), _ptr(w_lin), _ptr(s_lin), _ptr(w_v), _ptr(s_v),
                                  _ptr(w_1), _ptr(s_1), _stream(stream))


def moe_get_routing(h, idx=None, gate=None, offsets=None, perm=None, stream=None) -> int:
    return _lib.moe_get_routing(h, _ptr(idx), _ptr(gate), _ptr(offsets), _ptr(perm), _stream(stream))


def moe_get_block_input(h, u, stream=None) -> int:
    """u: device bf16 [T, d] receiving the last moe_block_forward's MoE input."""
    return _lib.moe_get_block_input(h, _ptr(u), _stream(stream))


def moe_sync_status(h, stream=None) -> int:
    return _lib.moe_sync_status(h, _stream(stream))


def moe_set_timeout(h, ns: int) -> int:
    return _lib.moe_set_timeout(h, int(ns))


def moe_set_profiling(h, on: bool) -> int:
    return _lib.moe_set_profiling(h, 1 if on else 0)


def moe_get_kernel_times(h):
    """-> (status, {kernel name: (total ms, launches)}) since the previous call."""
    n = len(KERNEL_NAMES)
    ms = (ctypes.c_float * n)()
    cnt = (ctypes.c_int * n)()
    rc = _lib.moe_get_kernel_times(h, ms, cnt, n)
    return rc, {KERNEL_NAMES[i]: (ms[i], cnt[i]) for i in range(n)}


MOE_PAIRS_OFF = 0          # one CTA per GEMM tile
MOE_PAIRS_LARGE_DOWN = 1   # CTA pairs for the down-projection of 128-route plans (the default)
MOE_PAIRS_LARGE = 2        # CTA pairs for both GEMMs of 128-route plans
MOE_PAIRS_ALL = 3          # CTA pairs also for small batches (32-route plans)


def moe_set_cta_pairs(h, mode: int) -> int:
    """GEMMs on CTA pairs: one of the MOE_PAIRS_* modes (MOE_PAIRS_LARGE_DOWN by default)."""
    return _lib.moe_set_cta_pairs(h, int(mode))


def moe_set_host_overlap(h, on: int) -> int:
    return _lib.moe_set_host_overlap(h, int(on))


def moe_host_wait(h, stream=None) -> int:
    return _lib.moe_host_wait(h, _stream(stream))


def moe_set_weight_layout(h, layout: int) -> int:
    return _lib.moe_set_weight_layout(h, int(layout))


def moe_pack_weight(h, w, w_packed, which: int, stream=None) -> int:
    return _lib.moe_pack_weight(h, _ptr(w), _ptr(w_packed), int(which), _stream(stream))


def moe_pack_weight_n(h, w, w_packed, which: int, n_experts: int, stream=None) -> int:
    return _lib.moe_pack_weight_n(h, _ptr(w), _ptr(w_packed), int(which), int(n_experts), _stream(stream))


def pack_layer(h, layer: dict, stream=None) -> dict:
    """A copy of `layer` with its three int8 weights rewritten to MOE_LAYOUT_PACKED
    (new device buffers; scales and router weight shared with `layer`).  The weights may
    hold fewer experts than the handle (an expert-parallel rank's share)."""
    import torch
    out = dict(layer)
    for key, which in (("wl", 0), ("wv", 0), ("w1", 1)):
        w = layer[key]
        E, a, b = w.shape
        p = torch.empty((E, b, a), dtype=torch.int8, device=w.device)
        check(moe_pack_weight_n(h, w, p, which, E, stream), "moe_pack_weight_n")
        out[key] = p
    return out


def moe_route_noalloc(T, d, x, router_w, bias, idx, gate, offsets, perm, stream=None) -> int:
    return _lib.moe_route_noalloc(int(T), int(d), _ptr(x), _ptr(router_w), _ptr(bias), _ptr(idx), _ptr(gate),
                                  _ptr(offsets), _ptr(perm), _stream(stream))


def moe_ep_dispatch(h, T, x, router_w, send_rows, send_counts, stream=None) -> int:
    return _lib.moe_ep_dispatch(h, int(T), _ptr(x), _ptr(router_w), _ptr(send_rows), _ptr(send_counts),
                                _stream(stream))


def moe_ep_experts(h, n_src, E_local, recv_counts, recv_rows, w_lin, s_lin, w_v, s_v, w_1, s_1, y_rows,
                   stream=None) -> int:
    """recv_counts: HOST int32 [n_src, E_local] (a CPU tensor or a sequence of ints)."""
    import torch
    rc = torch.as_tensor(recv_counts, dtype=torch.int32).contiguous()
    if rc.device.type != "cpu":
        raise ValueError("recv_counts must be on the host")
    return _lib.moe_ep_experts(h, int(n_src), int(E_local), rc.data_ptr(), _ptr(recv_rows), _ptr(w_lin),
                               _ptr(s_lin), _ptr(w_v), _ptr(s_v), _ptr(w_1), _ptr(s_1), _ptr(y_rows),
                               _stream(stream))


def moe_ep_combine(h, T, y_back, out, stream=None) -> int:
    return _lib.moe_ep_combine(h, int(T), _ptr(y_back), _ptr(out), _stream(stream))


def moe_plan(h, T: int):
    """-> (status, routes per GEMM tile, K-splits of the down-projection) for T tokens."""
    bn, sp = ctypes.c_int(), ctypes.c_int()
    rc = _lib.moe_plan(h, int(T), ctypes.byref(bn), ctypes.byref(sp))
    return rc, bn.value, sp.value


def layer_args(layer: dict):
    """The weight arguments of moe_forward, in order, from a dict with keys
    router_w, wl, sl, wv, sv, w1, s1."""
    return (layer["router_w"], layer["wl"], layer["sl"], layer["wv"], layer["sv"], layer["w1"], layer["s1"])


class MoELayer:
    """Owns one handle; raises MoEError on any non-zero status."""

    def __init__(self, d: int, ffn: int, E: int = 8, k: int = 2):
        rc, self.h = moe_create(d, ffn, E, k)
        check(rc, "moe_create")
        self.d, self.ffn, self.E, self.k = d, ffn, E, k

    def close(self):
        if self.h:
            moe_destroy(self.h)
            self.h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass

    def forward(self, x, layer: dict, out, stream=None):
        check(moe_forward(self.h, x.shape[0], x, *layer_args(layer), out, stream), "moe_forward")
        return out

    def block_forward(self, h_io, g_pre, g_post, eps, layer: dict, stream=None):
        check(moe_block_forward(self.h, h_io.shape[0], h_io, g_pre, g_post, eps, *layer_args(layer), stream),
              "moe_block_forward")
        return h_io

    def sync(self, stream=None):
        check(moe_sync_status(self.h, stream), "moe_sync_status")
