"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

Holds no decoder arithmetic: it only draws bf16 bit patterns (numpy uint16
arrays) and token ids.  `libsynth.so` is built from `synth.c` by `build()`.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import configs
from .configs import ModelConfig

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _SO, src, "-lm"])
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        L.synth_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_char_p,
                                        ctypes.c_float]
        L.synth_const_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_float]
        L.synth_tokens.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_char_p,
                                   ctypes.c_int32]
        L.synth_kv_prefill.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 5 + [ctypes.c_uint64, ctypes.c_char_p,
                                                                               ctypes.c_float]
        L.synth_f32_to_bf16.argtypes = [ctypes.c_float]
        L.synth_f32_to_bf16.restype = ctypes.c_uint16
        L.synth_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_char_p]
        L.synth_stream_key.restype = ctypes.c_uint64
        _lib = L
    return _lib


def normal_bf16(shape, seed: int, name: str, sigma: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    lib().synth_normal_bf16(out.ctypes.data, out.size, seed, name.encode(), sigma)
    return out


def const_bf16(shape, value: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    lib().synth_const_bf16(out.ctypes.data, out.size, value)
    return out


def tokens(n: int, seed: int, name: str, vocab: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    lib().synth_tokens(out.ctypes.data, n, seed, name.encode(), vocab)
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (a bit shift)."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (vectorised)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def make_model(cfg: ModelConfig) -> dict:
    """All weights of `cfg` as bf16 bit patterns, [out, in] row-major.

    Stream names fix the draws independently of creation order:
    "embed", "lm_head", "final_norm" (constant), "layers.<l>.<w>" for w in
    wq, wk, wv, wo, w_gate, w_up, w_down, router, and
    "layers.<l>.experts.<e>.<w>" for expert weights.
    """
    s, sd = cfg.seed, cfg.weight_sigma
    H, d, F = cfg.hidden, cfg.head_dim, cfg.ffn
    m = {"embed": normal_bf16((cfg.vocab, H), s, "embed", sd)}
    m["lm_head"] = m["embed"] if cfg.tied else normal_bf16((cfg.vocab, H), s, "lm_head", sd)
    m["final_norm"] = const_bf16((H,), 1.0)
    layers = []
    for l in range(cfg.n_layers):
        p = f"layers.{l}."
        L = {
            "attn_norm": const_bf16((H,), 1.0),
            "wq": normal_bf16((cfg.n_heads * d, H), s, p + "wq", sd),
            "wk": normal_bf16((cfg.n_kv_heads * d, H), s, p + "wk", sd),
            "wv": normal_bf16((cfg.n_kv_heads * d, H), s, p + "wv", sd),
            "wo": normal_bf16((H, cfg.n_heads * d), s, p + "wo", sd),
            "ffn_norm": const_bf16((H,), 1.0),
        }
        if cfg.n_experts:
            L["router"] = normal_bf16((cfg.n_experts, H), s, p + "router", cfg.router_sigma)
            L["w_gate"] = [normal_bf16((F, H), s, p + f"experts.{e}.w_gate", sd) for e in range(cfg.n_experts)]
            L["w_up"] = [normal_bf16((F, H), s, p + f"experts.{e}.w_up", sd) for e in range(cfg.n_experts)]
            L["w_down"] = [normal_bf16((H, F), s, p + f"experts.{e}.w_down", sd) for e in range(cfg.n_experts)]
        else:
            L["w_gate"] = normal_bf16((F, H), s, p + "w_gate", sd)
            L["w_up"] = normal_bf16((F, H), s, p + "w_up", sd)
            L["w_down"] = normal_bf16((H, F), s, p + "w_down", sd)
        layers.append(L)
    m["layers"] = layers
    return m


def make_kv_cache(cfg: ModelConfig, max_seq: int | None = None, stream: str = ""):
    """(K, V) bf16 caches [L][nkv][max_seq][d]; positions < cfg.prefill hold
    N(0, kv_sigma^2) draws (taken as already rotated), the rest zero.  `stream`
    names an independent draw (the caches of the sequences of a batch)."""
    ms = cfg.max_seq if max_seq is None else max_seq
    shape = (cfg.n_layers, cfg.n_kv_heads, ms, cfg.head_dim)
    out = []
    for prefix in ("kcache" + stream, "vcache" + stream):
        c = np.empty(shape, dtype=np.uint16)
        lib().synth_kv_prefill(c.ctypes.data, cfg.n_layers, cfg.n_kv_heads, ms, cfg.head_dim, cfg.prefill,
                               cfg.seed, prefix.encode(), cfg.kv_sigma)
        out.append(c)
    return out[0], out[1]


def prompt_tokens(cfg: ModelConfig, stream: str = "") -> np.ndarray:
    """Random prompt (tiny model: 16 tokens) or, for pre-filled caches, the one
    random token fed at the first decode position.  `stream` names an
    independent draw (the prompts of the sequences of a batch)."""
    n = cfg.prompt_len if cfg.prompt_len else 1
    return tokens(n, cfg.seed, "prompt" + stream, cfg.vocab)


__all__ = ["configs", "ModelConfig", "build", "normal_bf16", "const_bf16", "tokens", "bf16_to_f32", "f32_to_bf16",
           "make_model", "make_kv_cache", "prompt_tokens"]
