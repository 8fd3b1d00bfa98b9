"""fp64 CPU oracle of the Grok-1 MoE feed-forward layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package.  The product (``mixture_experts_softmax_b200``)
never imports it, and it never imports the product: the two share no code.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64); this module only
marshals arrays into it and composes the stacked-block workload from its calls.
Passages followed are cited in ``moe_oracle.c``.

Parity status of each function (what pins it is in ``tests/test_oracle_pins.py``):

* ``route``        pinned: brute force over all expert pairs, closed-form gates, tie rule.
* ``dispatch``     pinned: brute-force stable grouping.
* ``expert_ffn``   pinned: numpy float64 dense gated FFN (library matmul).
* ``forward``      pinned: forced-expert and closed-form-gate reductions, permutation
                   invariance, zero input, linearity in the output scale.
* ``rmsnorm``      pinned: unit-RMS property, scale invariance, the closed form of a
                   constant row (which fixes where eps enters).
* ``block_chain``  pinned: power-of-two scalings that the pre-norm, the post-norm, the
                   gains and the residual add each fix exactly.
* ``round_bf16``   pinned: torch's fp32 -> bf16 round-to-nearest-even.
* ``gelu``         tanh form pinned against torch's tanh-approximate GELU (and by its
                   odd-part identity); the erf form against math.erf.  Choosing the
                   tanh form is a reading of the pages (they say "gelu" only); the two
                   forms differ by < 1e-3.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")

# -O3 vectorises the plain loops; -ffp-contract=off keeps every multiply and add a
# separately rounded IEEE operation (no fused multiply-add), as written.
CFLAGS = ["-O3", "-march=x86-64-v3", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
          "-shared", "-pthread", "-fvisibility=hidden", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the oracle's C library in place (gcc)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", *CFLAGS, "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.moe_oracle_round_bf16.restype = ctypes.c_double
        L.moe_oracle_round_bf16.argtypes = [ctypes.c_double]
        L.moe_oracle_round_bf16_array.restype = None
        L.moe_oracle_round_bf16_array.argtypes = [ctypes.c_long, P, P]
        L.moe_oracle_gelu.restype = ctypes.c_double
        L.moe_oracle_gelu.argtypes = [ctypes.c_double, i]
        L.moe_oracle_ffn_size.restype = ctypes.c_long
        L.moe_oracle_ffn_size.argtypes = [ctypes.c_long, ctypes.c_double]
        L.moe_oracle_route.restype = i
        L.moe_oracle_route.argtypes = [i, i, i, P, P, P, P, P, P, P]
        L.moe_oracle_dispatch.restype = i
        L.moe_oracle_dispatch.argtypes = [i, i, P, P, P, P]
        L.moe_oracle_expert_ffn.restype = i
        L.moe_oracle_expert_ffn.argtypes = [i, i, P, P, P, P, P, P, P, P, P, i, i, i]
        L.moe_oracle_forward.restype = i
        L.moe_oracle_forward.argtypes = [i, i, i, i, P, P, P, P, P, P, P, P, P, P, i, P, P, P, P, P, i, i, i]
        L.moe_oracle_rmsnorm.restype = i
        L.moe_oracle_rmsnorm.argtypes = [i, i, P, P, ctypes.c_double, P]
        _lib = L
    return _lib


# ---- array marshalling -------------------------------------------------------

def _np(a, dtype=None):
    """torch tensor or array -> C-contiguous numpy array (bf16 as raw uint16 bits)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach()
            if a.device.type != "cpu":
                a = a.cpu()
            if a.dtype == torch.bfloat16:
                a = a.contiguous().view(torch.int16).numpy().view(np.uint16)
            else:
                a = a.contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if dtype is not None and a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 raw bits (uint16) -> float64 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """fp64 values that are exactly bf16-representable -> raw uint16 bits."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    if not np.array_equal(f.astype(np.float64), np.asarray(v, dtype=np.float64)):
        raise ValueError("values are not bf16-representable")
    bits = f.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("values are not bf16-representable")
    return (bits >> 16).astype(np.uint16)


# ---- scalar helpers ----------------------------------------------------------

def ffn_size(emb: int, widening: float) -> int:
    return int(lib().moe_oracle_ffn_size(int(emb), float(widening)))


def gelu(a: float, kind: int = 0) -> float:
    return float(lib().moe_oracle_gelu(float(a), int(kind)))


def round_bf16(v) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), kept as fp64."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.empty_like(v)
    lib().moe_oracle_round_bf16_array(v.size, _p(v), _p(out))
    return out


# ---- the layer ---------------------------------------------------------------

def route(x, router_w, bias=None) -> Dict[str, np.ndarray]:
    """fp32 logits, fp64 softmax, top-2 on every token of x (bf16 [T,d])."""
    xb = _np(x, np.uint16)
    rw = _np(router_w, np.float32)
    T, d = xb.shape
    E = rw.shape[1]
    b = None if bias is None else _np(bias, np.float32)
    logits = np.zeros((T, E), np.float32)
    probs = np.zeros((T, E), np.float64)
    idx = np.zeros((T, 2), np.int32)
    gate = np.zeros((T, 2), np.float64)
    _check(lib().moe_oracle_route(T, d, E, _p(xb), _p(rw), _p(b), _p(logits), _p(probs), _p(idx),
                                  _p(gate)), "route")
    return dict(logits=logits, probs=probs, idx=idx, gate=gate)


def dispatch(idx, E: int):
    """counts [E], offsets [E+1], perm [2T] (route id 2t+j), grouped by expert, stable in t.

    Expert id -1 (a padding token's route) is not dispatched; perm entries from offsets[E]
    on are then unused (0)."""
    ia = _np(idx, np.int32)
    T = ia.shape[0]
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(2 * T, np.int32)
    _check(lib().moe_oracle_dispatch(T, E, _p(ia), _p(counts), _p(offsets), _p(perm)), "dispatch")
    return counts, offsets, perm


def check_layer(layer, d: Optional[int] = None) -> tuple:
    """Shapes of one layer in the [E, in, out] orientation -> (E, d, F, kb); raises ValueError
    when the tensors do not fit together (for example a layer whose weights were transposed
    to another layout, or scales of another matrix)."""
    shp = {k: tuple(layer[k].shape) for k in ("router_w", "wl", "sl", "wv", "sv", "w1", "s1")}
    if len(shp["wl"]) != 3:
        raise ValueError(f"wl must be [E, d, F], got {shp['wl']}")
    E, dd, F = shp["wl"]
    if d is not None and dd != d:
        raise ValueError(f"wl is [E, {dd}, F] but the tokens have width {d} (weights in another layout?)")
    if shp["wv"] != (E, dd, F):
        raise ValueError(f"wv must be {(E, dd, F)}, got {shp['wv']}")
    if shp["w1"] != (E, F, dd):
        raise ValueError(f"w1 must be {(E, F, dd)}, got {shp['w1']}")
    if shp["router_w"] != (dd, E):
        raise ValueError(f"router_w must be {(dd, E)}, got {shp['router_w']}")
    if len(shp["sl"]) == 2:
        kb = 0
        want = {"sl": (E, F), "sv": (E, F), "s1": (E, dd)}
    else:
        if len(shp["sl"]) != 3 or shp["sl"][1] == 0 or dd % shp["sl"][1]:
            raise ValueError(f"sl must be [E, F] or [E, d/kb, F], got {shp['sl']}")
        kb = dd // shp["sl"][1]
        if F % kb:
            raise ValueError(f"scale block {kb} does not divide F = {F}")
        want = {"sl": (E, dd // kb, F), "sv": (E, dd // kb, F), "s1": (E, F // kb, dd)}
    for k, v in want.items():
        if shp[k] != v:
            raise ValueError(f"{k} must be {v}, got {shp[k]}")
    return E, dd, F, kb


def scale_block(layer) -> int:
    """Block of inputs sharing a scale: 0 when the scales are per output channel ([E, out]),
    else in / (number of scale rows) for per-block scales ([E, in/kb, out])."""
    sl, wl = layer["sl"], layer["wl"]
    return 0 if len(sl.shape) == 2 else wl.shape[1] // sl.shape[1]


def expert_ffn(xt: np.ndarray, layer, e: int, nthreads: int = 0, gelu_kind: int = 0,
               return_h: bool = False):
    """One expert's gated-GELU FFN on one fp64 token row."""
    xt = np.ascontiguousarray(xt, dtype=np.float64)
    check_layer(layer, xt.shape[0])
    wl, sl = _np(layer["wl"], np.int8), _np(layer["sl"], np.uint16)
    wv, sv = _np(layer["wv"], np.int8), _np(layer["sv"], np.uint16)
    w1, s1 = _np(layer["w1"], np.int8), _np(layer["s1"], np.uint16)
    E, d, F = wl.shape
    y = np.zeros(d, np.float64)
    h = np.zeros(F, np.float64)
    _check(lib().moe_oracle_expert_ffn(d, F, _p(xt), _p(wl[e]), _p(np.ascontiguousarray(sl[e])), _p(wv[e]),
                                       _p(np.ascontiguousarray(sv[e])), _p(w1[e]), _p(np.ascontiguousarray(s1[e])),
                                       _p(h), _p(y), nthreads, gelu_kind, scale_block(layer)),
           "expert_ffn")
    return (y, h) if return_h else y


def forward(layer, x, bias=None, tokens: Optional[Sequence[int]] = None, forced_idx=None,
            nthreads: int = 0, gelu_kind: int = 0, mask=None):
    """The MoE layer on the selected tokens: returns (out fp64 [n,d], idx [n,2], gate [n,2]).

    ``mask`` (bool/uint8 [T], optional): tokens with mask 0 are padding, routed nowhere
    (out row 0, experts -1, gates 0)."""
    xb = _np(x, np.uint16)
    T, d = xb.shape
    check_layer(layer, d)
    rw = _np(layer["router_w"], np.float32)
    wl, sl = _np(layer["wl"], np.int8), _np(layer["sl"], np.uint16)
    wv, sv = _np(layer["wv"], np.int8), _np(layer["sv"], np.uint16)
    w1, s1 = _np(layer["w1"], np.int8), _np(layer["s1"], np.uint16)
    E, _, F = wl.shape
    b = None if bias is None else _np(bias, np.float32)
    tk = None if tokens is None else np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
    n = T if tk is None else len(tk)
    fi = None if forced_idx is None else np.ascontiguousarray(np.asarray(forced_idx, dtype=np.int32))
    if fi is not None and fi.shape != (n, 2):
        raise ValueError("forced_idx must be [n_sel, 2]")
    mk = None if mask is None else np.ascontiguousarray(_np(mask).astype(np.uint8).reshape(-1))
    if mk is not None and mk.shape[0] != T:
        raise ValueError("mask must have one entry per token")
    out = np.zeros((n, d), np.float64)
    idx = np.zeros((n, 2), np.int32)
    gate = np.zeros((n, 2), np.float64)
    _check(lib().moe_oracle_forward(T, d, F, E, _p(xb), _p(rw), _p(b), _p(wl), _p(sl), _p(wv),
                                    _p(sv), _p(w1), _p(s1), _p(tk), n, _p(fi), _p(mk), _p(out), _p(idx),
                                    _p(gate), nthreads, gelu_kind, scale_block(layer)), "forward")
    return out, idx, gate


def rmsnorm(z, gamma=None, eps: float = 1e-5) -> np.ndarray:
    z = np.ascontiguousarray(np.asarray(z, dtype=np.float64))
    T, d = z.shape
    g = None if gamma is None else _np(gamma, np.uint16)
    out = np.zeros_like(z)
    _check(lib().moe_oracle_rmsnorm(T, d, _p(z), _p(g), float(eps), _p(out)), "rmsnorm")
    return out


def near_ties(probs: np.ndarray, thresh: float = 1e-6) -> np.ndarray:
    """Tokens whose top-3 sorted probabilities have a gap below ``thresh``.

    For such tokens either selection is a correct top-2, so routing and dispatch
    are not compared bit-exactly there."""
    s = -np.sort(-np.asarray(probs, dtype=np.float64), axis=1)
    g01 = s[:, 0] - s[:, 1]
    g12 = s[:, 1] - s[:, 2] if s.shape[1] > 2 else np.full(s.shape[0], np.inf)
    return (g01 < thresh) | (g12 < thresh)


def block_chain(layers: List[dict], gammas: List[dict], h, eps: float = 1e-5,
                tokens: Optional[Sequence[int]] = None, forced: Optional[List[Optional[np.ndarray]]] = None,
                nthreads: int = 0, gelu_kind: int = 0, mask=None):
    """Stacked residual MoE blocks on the selected token rows of h (bf16 [T,d]).

    Per block b:  u = bf16( RMSNorm(h; g_pre) )        (the MoE layer's bf16 input)
                  y = MoE_b(u)                          (fp64)
                  h = bf16( h + RMSNorm(y; g_post) )    (bf16 residual stream)
    Returns a list of per-block dicts: h_in (fp64 values of bf16), u_exact (RMSNorm(h; g_pre)
    before its bf16 rounding), u, idx, gate, probs, y, delta (RMSNorm(y; g_post), the fp64
    value added to the residual stream before its bf16 rounding) and h_out.
    ``forced[b]`` (optional [n,2]) names the experts to use in block b.
    ``mask`` (optional [T]) marks padding tokens (0): their MoE output is 0, so their row of
    the residual stream passes through unchanged.
    """
    hb = _np(h, np.uint16)
    T, d = hb.shape
    rows = list(range(T)) if tokens is None else [int(t) for t in tokens]
    cur = bf16_bits_to_f64(hb[rows])
    mk = None if mask is None else np.asarray(_np(mask)).astype(np.uint8).reshape(-1)[rows]
    res = []
    for b, (layer, gm) in enumerate(zip(layers, gammas)):
        u_exact = rmsnorm(cur, gm["pre"], eps)
        u = round_bf16(u_exact)
        ub = f64_to_bf16_bits(u)
        r = route(ub, layer["router_w"])
        fb = None if forced is None else forced[b]
        y, idx, gate = forward(layer, ub, tokens=None, forced_idx=fb, nthreads=nthreads,
                               gelu_kind=gelu_kind, mask=mk)
        delta = rmsnorm(y, gm["post"], eps)
        nxt = round_bf16(cur + delta)
        res.append(dict(h_in=cur, u_exact=u_exact, u=u, idx=idx, gate=gate, probs=r["probs"], y=y,
                        delta=delta, h_out=nxt))
        cur = nxt
    return res
