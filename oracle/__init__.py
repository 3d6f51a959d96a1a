"""CPU oracle of the decode step -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``oracle.c`` (plain C, double
precision, OpenMP over output rows) with numpy marshalling.  It shares no code
with the CUDA path and never imports it.

What is computed, and where the pages leave a step open, is stated in the
header of ``oracle.c``.  Every function is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants and library routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Callable, Dict, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboracle.so")
SOURCES = ("oracle.c",)


def build(verbose: bool = False) -> None:
    cmd = ["gcc", "-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared",
           os.path.join(_HERE, "oracle.c"), "-o", LIB_PATH, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)


class _Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("hidden", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int),
                ("vocab", ctypes.c_int), ("rms_eps", ctypes.c_double),
                ("rope_theta", ctypes.c_double), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("expert_ffn", ctypes.c_int),
                ("moe_renorm", ctypes.c_int)]


# int provider(layer, expert, which, dst, user): 0 once dst is filled, nonzero on failure
PROVIDER = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                            ctypes.c_void_p)

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        stale = (not os.path.exists(LIB_PATH) or
                 any(os.path.getmtime(os.path.join(_HERE, s)) > os.path.getmtime(LIB_PATH)
                     for s in SOURCES))
        if stale:
            build()
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.oc_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oc_bf16_to_double.restype = f64
        L.oc_bf16_round.argtypes = [f64]
        L.oc_bf16_round.restype = ctypes.c_uint16
        L.oc_silu.argtypes = [f64]
        L.oc_silu.restype = f64
        L.oc_rmsnorm.argtypes = [vp, vp, i32, f64, vp]
        L.oc_rope.argtypes = [vp, i32, i32, f64]
        L.oc_gemv.argtypes = [vp, i32, i32, vp, vp]
        L.oc_attention.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
        L.oc_argmax.argtypes = [vp, i32]
        L.oc_argmax.restype = i32
        L.oc_swiglu_ffn.argtypes = [vp, vp, vp, i32, i32, vp, vp]
        L.oc_moe_route.argtypes = [vp, i32, i32, vp, i32, i32, vp, vp, vp, vp]
        L.oc_decode_step.argtypes = [ctypes.POINTER(_Config), vp, vp, vp, i32, i32, i32, vp, vp,
                                     PROVIDER, vp, vp, vp, vp]
        L.oc_decode_step.restype = i32
        L.oc_forward_nocache.argtypes = [ctypes.POINTER(_Config), vp, vp, i32, vp, PROVIDER, vp]
        L.oc_forward_nocache.restype = i32
        L.oc_num_threads.restype = i32
        for f in (L.oc_rmsnorm, L.oc_rope, L.oc_gemv, L.oc_attention, L.oc_swiglu_ffn,
                  L.oc_moe_route):
            f.restype = None
        _lib = L
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 operands are passed as uint16 bit patterns"
    return a


# ----------------------------------------------------------------------------- primitives

def bf16_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_round(x: float) -> int:
    return int(lib().oc_bf16_round(float(x)))


def bf16_round_array(x) -> np.ndarray:
    f = lib().oc_bf16_round
    flat = np.asarray(x, dtype=np.float64).ravel()
    return np.array([f(float(v)) for v in flat], dtype=np.uint16).reshape(np.shape(x))


def silu(z: float) -> float:
    return float(lib().oc_silu(float(z)))


def rmsnorm(x, g_bits, eps: float) -> np.ndarray:
    x = _f64(x)
    g = _u16(g_bits)
    out = np.empty_like(x)
    lib().oc_rmsnorm(x.ctypes.data, g.ctypes.data, x.size, eps, out.ctypes.data)
    return out


def rope(v, pos: int, theta: float) -> np.ndarray:
    out = _f64(v).copy()
    lib().oc_rope(out.ctypes.data, out.size, pos, theta)
    return out


def gemv(W_bits, x) -> np.ndarray:
    W = _u16(W_bits)
    x = _f64(x)
    rows, cols = W.shape
    assert x.size == cols
    y = np.empty(rows, dtype=np.float64)
    lib().oc_gemv(W.ctypes.data, rows, cols, x.ctypes.data, y.ctypes.data)
    return y


def attention(q, K_bits, V_bits, n_q: int, n_kv: int, d: int) -> np.ndarray:
    """q [n_q*d]; K, V bf16 [n_tok][n_kv][d] -> o [n_q][d]."""
    q = _f64(q)
    K, V = _u16(K_bits), _u16(V_bits)
    n_tok = K.size // (n_kv * d)
    o = np.empty((n_q, d), dtype=np.float64)
    lib().oc_attention(q.ctypes.data, K.ctypes.data, V.ctypes.data, n_tok, n_q, n_kv, d,
                       o.ctypes.data)
    return o


def argmax(v) -> int:
    v = _f64(v)
    return int(lib().oc_argmax(v.ctypes.data, v.size))


def swiglu_ffn(wg_bits, wu_bits, wd_bits, h) -> np.ndarray:
    wg, wu, wd = _u16(wg_bits), _u16(wu_bits), _u16(wd_bits)
    F, H = wg.shape
    h = _f64(h)
    y = np.empty(H, dtype=np.float64)
    lib().oc_swiglu_ffn(wg.ctypes.data, wu.ctypes.data, wd.ctypes.data, H, F, h.ctypes.data,
                        y.ctypes.data)
    return y


def moe_route(w_router_bits, h, top_k: int, renorm: bool, override: Optional[Sequence[int]] = None):
    """Returns (selected experts, their weights, softmax probabilities)."""
    W = _u16(w_router_bits)
    E, H = W.shape
    h = _f64(h)
    sel = np.empty(top_k, dtype=np.int32)
    wts = np.empty(top_k, dtype=np.float64)
    probs = np.empty(E, dtype=np.float64)
    ov = None if override is None else np.ascontiguousarray(override, dtype=np.int32)
    lib().oc_moe_route(W.ctypes.data, E, H, h.ctypes.data, top_k, int(renorm),
                       None if ov is None else ov.ctypes.data, sel.ctypes.data, wts.ctypes.data,
                       probs.ctypes.data)
    return sel, wts, probs


def num_threads() -> int:
    return int(lib().oc_num_threads())


# ----------------------------------------------------------------------------- model

class Model:
    """Oracle model over host bf16 weights (dict name -> uint16 array, the names of
    ``synthetic.tensor_specs``) with its own position-major KV cache per layer.

    ``expert_provider(layer, expert, which) -> uint16 array`` may replace the
    held expert matrices for models too large for host memory (which: 0 gate,
    1 up, 2 down).
    """

    def __init__(self, cfg, weights: Dict[str, np.ndarray], ctx_cap: int,
                 names: Sequence[str], expert_provider: Optional[Callable] = None):
        self.cfg = cfg
        self.ctx_cap = ctx_cap
        self._keep: List[np.ndarray] = []
        ptrs = []
        for n in names:
            a = weights.get(n)
            if a is None:
                ptrs.append(None)
            else:
                a = _u16(a)
                self._keep.append(a)
                ptrs.append(a.ctypes.data)
        self._wptrs = (ctypes.c_void_p * len(ptrs))(*ptrs)
        c = _Config()
        c.n_layers, c.hidden, c.n_q_heads = cfg.n_layers, cfg.hidden, cfg.n_q_heads
        c.n_kv_heads, c.head_dim, c.ffn, c.vocab = cfg.n_kv_heads, cfg.head_dim, cfg.ffn, cfg.vocab
        c.rms_eps, c.rope_theta = cfg.rms_eps, cfg.rope_theta
        c.n_experts, c.top_k, c.expert_ffn, c.moe_renorm = (cfg.n_experts, cfg.top_k,
                                                           cfg.expert_ffn, cfg.moe_renorm)
        self._c = c
        kv_shape = (ctx_cap, cfg.n_kv_heads, cfg.head_dim)
        self.k = [np.zeros(kv_shape, dtype=np.uint16) for _ in range(cfg.n_layers)]
        self.v = [np.zeros(kv_shape, dtype=np.uint16) for _ in range(cfg.n_layers)]
        self._prov_error: Optional[BaseException] = None
        self._kp = (ctypes.c_void_p * cfg.n_layers)(*[a.ctypes.data for a in self.k])
        self._vp = (ctypes.c_void_p * cfg.n_layers)(*[a.ctypes.data for a in self.v])
        if expert_provider is not None:
            Fe, H = cfg.expert_ffn, cfg.hidden

            def _prov(layer, expert, which, dst, user):
                # an exception cannot cross the C frames: it is kept, the oracle is told
                # to stop, and the calling method raises it
                n = Fe * H
                try:
                    arr = np.ascontiguousarray(expert_provider(layer, expert, which), dtype=np.uint16)
                    if arr.size != n:
                        raise ValueError(f"expert provider returned {arr.size} elements for layer {layer}, "
                                         f"expert {expert}, matrix {which}; expected {n}")
                    ctypes.memmove(dst, arr.ctypes.data, 2 * n)
                    return 0
                except BaseException as exc:       # noqa: BLE001 - re-raised by the caller
                    if self._prov_error is None:
                        self._prov_error = exc
                    return 1

            self._prov = PROVIDER(_prov)
        else:
            self._prov = PROVIDER()

    def decode_step(self, token: int, pos: int, want_hidden: bool = False,
                    moe_override: Optional[np.ndarray] = None):
        """Runs one step; returns dict(logits, hidden?, moe_sel?, moe_wts?)."""
        cfg = self.cfg
        logits = np.empty(cfg.vocab, dtype=np.float64)
        hidden = np.empty((2 * cfg.n_layers + 1, cfg.hidden)) if want_hidden else None
        sel = wts = ov = None
        if cfg.is_moe:
            sel = np.empty((cfg.n_layers, cfg.top_k), dtype=np.int32)
            wts = np.empty((cfg.n_layers, cfg.top_k), dtype=np.float64)
            if moe_override is not None:
                ov = np.ascontiguousarray(moe_override, dtype=np.int32)
        rc = lib().oc_decode_step(ctypes.byref(self._c), self._wptrs, self._kp, self._vp,
                                  self.ctx_cap, int(token), int(pos), logits.ctypes.data,
                                  None if hidden is None else hidden.ctypes.data, self._prov, None,
                                  None if ov is None else ov.ctypes.data,
                                  None if sel is None else sel.ctypes.data,
                                  None if wts is None else wts.ctypes.data)
        self._raise_on(rc, "decode_step")
        out = {"logits": logits}
        if hidden is not None:
            out["hidden"] = hidden
        if sel is not None:
            out["moe_sel"], out["moe_wts"] = sel, wts
        return out

    def forward_nocache(self, tokens: Sequence[int]) -> np.ndarray:
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        T = toks.size
        logits = np.empty((T, self.cfg.vocab), dtype=np.float64)
        rc = lib().oc_forward_nocache(ctypes.byref(self._c), self._wptrs, toks.ctypes.data, T,
                                      logits.ctypes.data, self._prov, None)
        self._raise_on(rc, "forward_nocache")
        return logits

    def _raise_on(self, rc: int, what: str) -> None:
        err, self._prov_error = self._prov_error, None
        if rc == -2:
            raise RuntimeError(f"oracle {what}: the expert provider failed") from err
        if rc != 0:
            raise ValueError(f"oracle {what}: bad argument")
