"""fp64 CPU oracle for batch-1 Llama/Mixtral decode (ctypes wrapper of oracle.c).

TEST INFRASTRUCTURE ONLY.  Only `tests/`, the smoke check and the benchmark's
CPU-baseline leg may import this package; the product library never does, and
this package imports nothing from the product.  Inputs come from the seeded
generator (`synth`), which holds none of the decode arithmetic.

Every function follows the plain decoder definition written out in oracle.c
(epic-kernel README, "3B model support" and "Mixtral 8x7B MoE for batch-1
inference"; Hyperkernel teardown, "What a megakernel buys").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

_P = ctypes.c_void_p
_D = ctypes.c_double
_I = ctypes.c_int


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "oracle.c")
    hdr = os.path.join(_HERE, "oracle.h")
    newest = max(os.path.getmtime(src), os.path.getmtime(hdr))
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < newest:
        # -ffp-contract=off: every product and sum is a separately rounded double op.
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", "-o", _SO, src,
                               "-lm"])
    return _SO


class Shape(ctypes.Structure):
    _fields_ = [("n_layers", _I), ("hidden", _I), ("n_heads", _I), ("n_kv_heads", _I), ("head_dim", _I),
                ("ffn", _I), ("vocab", _I), ("n_experts", _I), ("top_k", _I), ("max_seq", _I),
                ("rms_eps", _D), ("rope_theta", _D)]


class Weights(ctypes.Structure):
    _fields_ = [("embed", _P), ("lm_head", _P), ("final_norm", _P)] + [
        (n, ctypes.POINTER(_P)) for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up",
                                          "w_down", "router")]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_double.restype = _D
        L.orc_bf16_from_double.argtypes = [_D]
        L.orc_bf16_from_double.restype = ctypes.c_uint16
        L.orc_rmsnorm.argtypes = [_P, _P, _I, _D, _P]
        L.orc_gemv.argtypes = [_P, _I, _I, _P, _P]
        L.orc_rope.argtypes = [_P, _I, _I, _I, _D]
        L.orc_softmax.argtypes = [_P, _I, _P]
        L.orc_attend.argtypes = [_P, _P, _P, _I, _I, _P]
        L.orc_silu.argtypes = [_D]
        L.orc_silu.restype = _D
        L.orc_topk.argtypes = [_P, _I, _I, _P, _P]
        L.orc_argmax.argtypes = [_P, _I]
        L.orc_argmax.restype = _I
        L.orc_decode_step.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), _P, _P, _I, _I, _P, _P, _P,
                                      _P]
        L.orc_decode_step.restype = _I
        L.orc_num_threads.restype = _I
        L.orc_predict_experts.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), _I, _P, _P]
        L.orc_predict_experts.restype = _I
        _lib = L
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16
    return a


# ---- building blocks --------------------------------------------------------

def bf16_to_double(b: int) -> float:
    return lib().orc_bf16_to_double(int(b))


def bf16_from_double(v: float) -> int:
    return int(lib().orc_bf16_from_double(float(v)))


def rmsnorm(x, w_bf16, eps: float) -> np.ndarray:
    x = _f64(x)
    w = _u16(w_bf16)
    out = np.empty_like(x)
    lib().orc_rmsnorm(x.ctypes.data, w.ctypes.data, x.size, eps, out.ctypes.data)
    return out


def gemv(W_bf16, x) -> np.ndarray:
    W = _u16(W_bf16)
    x = _f64(x)
    rows, cols = W.shape
    assert x.size == cols
    y = np.empty(rows, dtype=np.float64)
    lib().orc_gemv(W.ctypes.data, rows, cols, x.ctypes.data, y.ctypes.data)
    return y


def rope(v, n_heads: int, head_dim: int, pos: int, theta: float) -> np.ndarray:
    out = _f64(v).copy()
    lib().orc_rope(out.ctypes.data, n_heads, head_dim, pos, theta)
    return out


def softmax(s) -> np.ndarray:
    s = _f64(s)
    p = np.empty_like(s)
    lib().orc_softmax(s.ctypes.data, s.size, p.ctypes.data)
    return p


def attend(q, K_bf16, V_bf16) -> np.ndarray:
    q = _f64(q)
    K = _u16(K_bf16)
    V = _u16(V_bf16)
    n, d = K.shape
    out = np.empty(d, dtype=np.float64)
    lib().orc_attend(q.ctypes.data, K.ctypes.data, V.ctypes.data, n, d, out.ctypes.data)
    return out


def silu(z: float) -> float:
    return lib().orc_silu(float(z))


def topk(r, k: int):
    r = _f64(r)
    idx = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    lib().orc_topk(r.ctypes.data, r.size, k, idx.ctypes.data, w.ctypes.data)
    return idx, w


def argmax(v) -> int:
    v = _f64(v)
    return int(lib().orc_argmax(v.ctypes.data, v.size))


def num_threads() -> int:
    return int(lib().orc_num_threads())


# ---- whole decode step ------------------------------------------------------

class Model:
    """Binds a synth-made weight dict (bf16 numpy arrays) to the oracle ABI.

    `cache` is the oracle's own (K, V) bf16 cache pair; decode steps append to
    it in place."""

    def __init__(self, cfg, weights: dict, kcache: np.ndarray, vcache: np.ndarray):
        self.cfg = cfg
        self.w = weights
        self.k = kcache
        self.v = vcache
        assert kcache.dtype == np.uint16 and kcache.flags.c_contiguous
        self.shape = Shape(cfg.n_layers, cfg.hidden, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.ffn,
                           cfg.vocab, cfg.n_experts, cfg.top_k, kcache.shape[2], cfg.rms_eps, cfg.rope_theta)
        L = cfg.n_layers
        self._keep = []

        def arr(items):
            a = (_P * max(1, len(items)))(*[it.ctypes.data for it in items])
            self._keep.append(a)
            return ctypes.cast(a, ctypes.POINTER(_P))

        layers = weights["layers"]
        kw = {}
        for name in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm"):
            kw[name] = arr([layers[l][name] for l in range(L)])
        if cfg.n_experts:
            for name in ("w_gate", "w_up", "w_down"):
                kw[name] = arr([layers[l][name][e] for l in range(L) for e in range(cfg.n_experts)])
            kw["router"] = arr([layers[l]["router"] for l in range(L)])
        else:
            for name in ("w_gate", "w_up", "w_down"):
                kw[name] = arr([layers[l][name] for l in range(L)])
            kw["router"] = ctypes.cast(None, ctypes.POINTER(_P))
        self.weights = Weights(weights["embed"].ctypes.data, weights["lm_head"].ctypes.data,
                               weights["final_norm"].ctypes.data, **kw)

    def step(self, token: int, pos: int, want_hidden: bool = True) -> dict:
        cfg = self.cfg
        logits = np.empty(cfg.vocab, dtype=np.float64)
        hidden = np.empty((cfg.n_layers + 1, cfg.hidden), dtype=np.float64) if want_hidden else None
        K = max(cfg.top_k, 1)
        ridx = np.full((cfg.n_layers, K), -1, dtype=np.int32)
        rw = np.zeros((cfg.n_layers, K), dtype=np.float64)
        nxt = lib().orc_decode_step(ctypes.byref(self.shape), ctypes.byref(self.weights), self.k.ctypes.data,
                                    self.v.ctypes.data, int(token), int(pos), logits.ctypes.data,
                                    hidden.ctypes.data if hidden is not None else None,
                                    ridx.ctypes.data if cfg.n_experts else None,
                                    rw.ctypes.data if cfg.n_experts else None)
        if nxt < 0:
            raise ValueError(f"oracle rejected token={token} pos={pos}")
        pred = None
        if cfg.n_experts and hidden is not None:
            pred = np.stack([self.predicted_experts(hidden[l], l) for l in range(cfg.n_layers)]) \
                if cfg.n_layers else np.zeros((0, K), dtype=np.int32)
        return {"logits": logits, "hidden": hidden, "next": nxt, "router_idx": ridx, "router_w": rw,
                "pred_idx": pred}

    def predicted_experts(self, x, layer: int) -> np.ndarray:
        """Speculative expert prediction of `layer` from the residual x entering it (orc_predict_experts)."""
        x = _f64(x)
        idx = np.empty(self.cfg.top_k, dtype=np.int32)
        if lib().orc_predict_experts(ctypes.byref(self.shape), ctypes.byref(self.weights), int(layer),
                                     x.ctypes.data, idx.ctypes.data) != 0:
            raise ValueError(f"oracle rejected the prediction of layer {layer}")
        return idx
