"""ctypes binding of libmk.so (include/mk.h): argument marshalling only.

Every step of the decode path runs in the library's CUDA kernels; PyTorch is
used here only to own device memory and streams.  There is no CPU fallback: if
libmk.so cannot be loaded, `load()` raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmk.so")

MK_OK = 0
ERRORS = {
    -1: "MK_ERR_INVALID_ARG", -2: "MK_ERR_CUDA", -3: "MK_ERR_NOT_RESIDENT", -4: "MK_ERR_TIMEOUT",
    -5: "MK_ERR_BAD_INSTR", -6: "MK_ERR_SCHEDULE", -7: "MK_ERR_STOPPED", -8: "MK_ERR_NO_SCHEDULE",
    -9: "MK_ERR_CAPACITY", -10: "MK_ERR_UNSUPPORTED",
}
CODES = {v: k for k, v in ERRORS.items()}
MODE_MEGAKERNEL, MODE_MULTI_KERNEL, MODE_MULTI_KERNEL_GRAPH = 0, 1, 2
FAULT_NONE, FAULT_UNREACHABLE_WAIT, FAULT_BAD_OPCODE, FAULT_PRESET_STOP = 0, 1, 2, 3
INSTR_WORDS = 16

_I, _F, _P = ctypes.c_int, ctypes.c_float, ctypes.c_void_p


class MkConfig(ctypes.Structure):
    _fields_ = [("n_layers", _I), ("hidden", _I), ("n_q_heads", _I), ("n_kv_heads", _I), ("head_dim", _I),
                ("ffn", _I), ("vocab", _I), ("n_experts", _I), ("top_k", _I), ("rms_eps", _F), ("rope_theta", _F),
                ("max_seq", _I), ("tied_embeddings", _I)]


class MkWeights(ctypes.Structure):
    _fields_ = [("embed", _P), ("lm_head", _P), ("final_norm", _P)] + [
        (n, ctypes.POINTER(_P)) for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up",
                                          "w_down", "router")] + [("k_cache", _P), ("v_cache", _P)]


class MkOptions(ctypes.Structure):
    _fields_ = [("ring_stages", _I), ("stage_bytes", _I), ("rows_per_instr", _I), ("kv_splits", _I),
                ("l2_prefetch", _I), ("trace", _I), ("snapshots", _I), ("spin_limit_ns", ctypes.c_ulonglong),
                ("mode", _I), ("n_sm", _I), ("prefetch_ahead", _I), ("prefetch_max_bytes", _I),
                ("attn_sm_ffn_permille", _I), ("serve_idle_ns", ctypes.c_ulonglong), ("general_kernel", _I),
                ("split_ffn", _I), ("l2_head_start", _I), ("sm_speed", ctypes.c_void_p), ("n_sm_speed", _I),
                ("spec_experts", _I), ("batch", _I), ("attn_merge", _I),
                ("ffn_early_stages", _I)]


class MkStatus(ctypes.Structure):
    _fields_ = [("code", _I), ("sm", _I), ("instr", _I), ("opcode", _I), ("counter", _I),
                ("observed", ctypes.c_uint), ("expected", ctypes.c_uint), ("cuda_error", _I)]

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k, _ in self._fields_}


# Every exported entry point of include/mk.h, with its ctypes signature.
SIGNATURES = {
    "mk_default_options": (None, [ctypes.POINTER(MkOptions)]),
    "mk_create": (_I, [ctypes.POINTER(MkConfig), ctypes.POINTER(MkWeights), ctypes.POINTER(MkOptions), _P,
                       ctypes.POINTER(_P)]),
    "mk_build_schedule": (_I, [_P]),
    "mk_get_schedule": (_I, [_P, _P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(_I),
                             ctypes.POINTER(_I)]),
    "mk_decode_step": (_I, [_P, ctypes.c_int32, ctypes.c_int32, _P, _P]),
    "mk_decode_step_batch": (_I, [_P, _P, _P, _P, _P]),
    "mk_get_hidden": (_I, [_P, _I, _P]),
    "mk_get_router": (_I, [_P, _I, _P, _P]),
    "mk_get_predicted_experts": (_I, [_P, _I, _P]),
    "mk_get_counters": (_I, [_P, _P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)]),
    "mk_get_counter_increments": (_I, [_P, _P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)]),
    "mk_get_status": (_I, [_P, ctypes.POINTER(MkStatus)]),
    "mk_get_trace": (_I, [_P, _P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)]),
    "mk_reset": (_I, [_P]),
    "mk_inject_fault": (_I, [_P, _I, _I]),
    "mk_last_step_ns": (_I, [_P, ctypes.POINTER(ctypes.c_double)]),
    "mk_strerror": (ctypes.c_char_p, [_I]),
    "mk_destroy": (None, [_P]),
    "mk_plan": (_I, [ctypes.POINTER(MkConfig), ctypes.POINTER(MkOptions), _I, _P, ctypes.c_size_t,
                     ctypes.POINTER(_I), _P, _P, ctypes.c_size_t, ctypes.POINTER(_I)]),
    "mk_simulate": (_I, [_P, _I, _I, _P, _P, _I, _I, ctypes.c_uint64, ctypes.POINTER(ctypes.c_longlong)]),
    "mk_serve_start": (_I, [_P, _P]),
    "mk_serve_step": (_I, [_P, ctypes.c_int32, ctypes.c_int32, _P]),
    "mk_serve_stop": (_I, [_P]),
    "mk_attention_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I]),
    "mk_attention_decode": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, ctypes.c_size_t, _P]),
    "mk_attention_decode_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]),
}
NOALLOC_SCRATCH_BYTES = 1 << 20  # MK_ATTENTION_NOALLOC_SCRATCH_BYTES

_lib = None


def load(path: str | None = None):
    """Load libmk.so (built in-tree by `build()`); raises if it is missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libmk.so not found at {p}: run decode_persistent_block_b200.build() first "
                           "(there is no fallback path)")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


class MkError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        self.name = ERRORS.get(code, str(code))
        msg = load().mk_strerror(code).decode()
        super().__init__(f"{where}: {self.name} ({msg})" if where else f"{self.name} ({msg})")


def check(rc: int, where: str = ""):
    if rc != MK_OK:
        raise MkError(rc, where)


def make_config(cfg) -> MkConfig:
    """From any object with the model-shape attributes (n_layers, hidden,
    n_heads, n_kv_heads, head_dim, ffn, vocab, n_experts, top_k, rms_eps,
    rope_theta, max_seq, tied)."""
    g = (lambda k, d=0: cfg[k] if k in cfg else d) if isinstance(cfg, dict) else (lambda k, d=0: getattr(cfg, k, d))
    return MkConfig(g("n_layers"), g("hidden"), g("n_heads"), g("n_kv_heads"), g("head_dim"), g("ffn"),
                    g("vocab"), g("n_experts", 0), g("top_k", 0), g("rms_eps", 1e-5), g("rope_theta", 10000.0),
                    g("max_seq"), int(bool(g("tied", False))))


def make_options(**kw) -> MkOptions:
    """mk_options with the library defaults, then the given fields.  `sm_speed`
    takes a sequence of per-block speeds; the returned struct keeps the array
    alive (the library copies it when it reads the options)."""
    o = MkOptions()
    load().mk_default_options(ctypes.byref(o))
    for k, v in kw.items():
        if not hasattr(o, k):
            raise KeyError(f"unknown option {k}")
        if k == "sm_speed":
            if v is None:
                continue
            arr = np.ascontiguousarray(v, dtype=np.float32)
            o._sm_speed = arr
            o.sm_speed = arr.ctypes.data
            o.n_sm_speed = int(arr.size)
            continue
        setattr(o, k, v)
    return o


def plan(cfg, n_sm: int, **options):
    """Host-only schedule planning: (words [n_sm, max_instr, 16] int32, n_instr [n_sm], ctr_inc [n_counters])."""
    lib = load()
    c = make_config(cfg)
    o = make_options(**options)
    max_instr, n_ctr = _I(0), _I(0)
    rc = lib.mk_plan(ctypes.byref(c), ctypes.byref(o), n_sm, None, 0, ctypes.byref(max_instr), None, None, 0,
                     ctypes.byref(n_ctr))
    if rc not in (MK_OK, CODES["MK_ERR_CAPACITY"]):
        check(rc, "mk_plan")
    words = np.zeros((n_sm, max_instr.value, INSTR_WORDS), dtype=np.int32)
    n_instr = np.zeros(n_sm, dtype=np.int32)
    inc = np.zeros(n_ctr.value, dtype=np.uint32)
    check(lib.mk_plan(ctypes.byref(c), ctypes.byref(o), n_sm, words.ctypes.data, words.size, ctypes.byref(max_instr),
                      n_instr.ctypes.data, inc.ctypes.data, inc.size, ctypes.byref(n_ctr)), "mk_plan")
    return words, n_instr, inc


def simulate(words: np.ndarray, n_instr: np.ndarray, ctr_inc: np.ndarray, steps: int = 1, seed: int = 0):
    """Run a planned schedule on the host under a seeded random interleaving.
    Returns (status code, instructions executed)."""
    words = np.ascontiguousarray(words, dtype=np.int32)
    n_instr = np.ascontiguousarray(n_instr, dtype=np.int32)
    ctr_inc = np.ascontiguousarray(ctr_inc, dtype=np.uint32)
    done = ctypes.c_longlong(0)
    rc = load().mk_simulate(words.ctypes.data, words.shape[0], words.shape[1], n_instr.ctypes.data,
                            ctr_inc.ctypes.data, ctr_inc.size, steps, seed, ctypes.byref(done))
    return rc, done.value


def _ptr(t) -> int:
    return int(t.data_ptr())


class Decoder:
    """A handle bound to device-resident weights and KV caches.

    weights: dict with "embed", "lm_head", "final_norm" and "layers" (list of
    dicts with attn_norm, wq, wk, wv, wo, ffn_norm, w_gate, w_up, w_down and,
    for MoE, router plus per-expert lists for w_gate/w_up/w_down), each a CUDA
    tensor holding bf16 bits (any 2-byte dtype).  kcache/vcache: CUDA tensors
    [L, n_kv, max_seq, d] of bf16 bits ([batch, L, n_kv, max_seq, d] with the
    option batch > 1).  The tensors must stay alive as long as the decoder.
    `stream`: a torch.cuda.Stream or None (current stream)."""

    def __init__(self, cfg, weights: dict, kcache, vcache, stream=None, build_schedule: bool = True, **options):
        import torch
        self.lib = load()
        self.cfg = cfg
        self._keep = [weights, kcache, vcache]
        self.config = make_config(cfg)
        self.config.max_seq = int(kcache.shape[-2])
        nb = max(1, int(options.get("batch", 1) or 1))
        if (kcache.dim() == 5) != (nb > 1) or (nb > 1 and kcache.shape[0] != nb):
            raise ValueError(f"KV cache shape {tuple(kcache.shape)} does not match batch={nb}")
        self.batch = nb
        L = self.config.n_layers
        E = self.config.n_experts
        layers = weights["layers"]

        def arr(ptrs):
            a = (_P * max(1, len(ptrs)))(*ptrs)
            self._keep.append(a)
            return ctypes.cast(a, ctypes.POINTER(_P))

        kw = {n: arr([_ptr(layers[l][n]) for l in range(L)])
              for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm")}
        if E:
            for n in ("w_gate", "w_up", "w_down"):
                kw[n] = arr([_ptr(layers[l][n][e]) for l in range(L) for e in range(E)])
            kw["router"] = arr([_ptr(layers[l]["router"]) for l in range(L)])
        else:
            for n in ("w_gate", "w_up", "w_down"):
                kw[n] = arr([_ptr(layers[l][n]) for l in range(L)])
            kw["router"] = ctypes.cast(None, ctypes.POINTER(_P))
        self.weights = MkWeights(_ptr(weights["embed"]), _ptr(weights["lm_head"]), _ptr(weights["final_norm"]),
                                 k_cache=_ptr(kcache), v_cache=_ptr(vcache), **kw)
        self.options = make_options(**options)
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        h = _P()
        check(self.lib.mk_create(ctypes.byref(self.config), ctypes.byref(self.weights), ctypes.byref(self.options),
                                 ctypes.c_void_p(self.stream.cuda_stream), ctypes.byref(h)), "mk_create")
        self.h = h
        if build_schedule:
            self.build_schedule()

    # -- lifecycle ------------------------------------------------------------------
    def build_schedule(self):
        check(self.lib.mk_build_schedule(self.h), "mk_build_schedule")

    def close(self):
        if getattr(self, "h", None):
            self.lib.mk_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()

    # -- launch-once serving ---------------------------------------------------------
    def serve_start(self, logits=None):
        """Launch the resident grid; logits: optional CUDA fp32 tensor [vocab]."""
        check(self.lib.mk_serve_start(self.h, _ptr(logits) if logits is not None else None), "mk_serve_start")

    def serve_step(self, token: int, pos: int) -> int:
        """Run one step on the resident grid; returns the next token."""
        out = ctypes.c_int32(-1)
        check(self.lib.mk_serve_step(self.h, int(token), int(pos), ctypes.byref(out)), "mk_serve_step")
        return int(out.value)

    def serve_stop(self):
        check(self.lib.mk_serve_stop(self.h), "mk_serve_stop")

    # -- the step -------------------------------------------------------------------
    def step(self, token: int, pos: int, logits=None, sync: bool = True):
        """One decode step.  token < 0 feeds the previous step's on-device argmax.
        With sync=True returns the next token (int); else only enqueues."""
        out = ctypes.c_int32(-1)
        rc = self.lib.mk_decode_step(self.h, int(token), int(pos), _ptr(logits) if logits is not None else None,
                                     ctypes.byref(out) if sync else None)
        check(rc, "mk_decode_step")
        return out.value if sync else None

    def step_rc(self, token: int, pos: int, logits=None, sync: bool = True) -> int:
        out = ctypes.c_int32(-1)
        return self.lib.mk_decode_step(self.h, int(token), int(pos), _ptr(logits) if logits is not None else None,
                                       ctypes.byref(out) if sync else None)

    def step_batch(self, tokens, pos, logits=None, sync: bool = True):
        """One decode step of every sequence of the batch: tokens and pos are sequences of `batch`
        ints (token < 0: that sequence's previous argmax).  logits: optional CUDA fp32 tensor
        [batch, vocab].  With sync=True returns the next tokens (int32 array); else only enqueues."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        ps = np.ascontiguousarray(pos, dtype=np.int32)
        if t.size != self.batch or ps.size != self.batch:
            raise ValueError(f"expected {self.batch} tokens and positions")
        out = np.full(self.batch, -1, dtype=np.int32)
        rc = self.lib.mk_decode_step_batch(self.h, t.ctypes.data, ps.ctypes.data,
                                           _ptr(logits) if logits is not None else None,
                                           out.ctypes.data if sync else None)
        check(rc, "mk_decode_step_batch")
        return out if sync else None

    # -- debug getters ------------------------------------------------------------------
    def hidden(self, layer: int) -> np.ndarray:
        """Residual stream after `layer`: [hidden], or [batch, hidden] with batch > 1."""
        out = np.empty((self.batch, self.config.hidden), dtype=np.float32)
        check(self.lib.mk_get_hidden(self.h, layer, out.ctypes.data), "mk_get_hidden")
        return out[0] if self.batch == 1 else out

    def hidden_all(self) -> np.ndarray:
        return np.stack([self.hidden(l) for l in range(self.config.n_layers + 1)])

    def predicted_experts(self, layer: int) -> np.ndarray:
        """The experts predicted for `layer` in the last step (options.spec_experts = 1)."""
        idx = np.empty(self.config.top_k, dtype=np.int32)
        check(self.lib.mk_get_predicted_experts(self.h, layer, idx.ctypes.data), "mk_get_predicted_experts")
        return idx

    def router(self, layer: int):
        k = self.config.top_k
        idx = np.empty(k, dtype=np.int32)
        w = np.empty(k, dtype=np.float32)
        check(self.lib.mk_get_router(self.h, layer, idx.ctypes.data, w.ctypes.data), "mk_get_router")
        return idx, w

    def counters(self) -> np.ndarray:
        n = ctypes.c_size_t(0)
        check(self.lib.mk_get_counters(self.h, None, 0, ctypes.byref(n)), "mk_get_counters")
        out = np.empty(n.value, dtype=np.uint32)
        check(self.lib.mk_get_counters(self.h, out.ctypes.data, out.size, ctypes.byref(n)), "mk_get_counters")
        return out

    def counter_increments(self) -> np.ndarray:
        n = ctypes.c_size_t(0)
        check(self.lib.mk_get_counter_increments(self.h, None, 0, ctypes.byref(n)), "mk_get_counter_increments")
        out = np.empty(n.value, dtype=np.uint32)
        check(self.lib.mk_get_counter_increments(self.h, out.ctypes.data, out.size, ctypes.byref(n)),
              "mk_get_counter_increments")
        return out

    def schedule(self) -> np.ndarray:
        n, nsm, mi = ctypes.c_size_t(0), _I(0), _I(0)
        check(self.lib.mk_get_schedule(self.h, None, 0, ctypes.byref(n), ctypes.byref(nsm), ctypes.byref(mi)),
              "mk_get_schedule")
        out = np.empty((nsm.value, mi.value, INSTR_WORDS), dtype=np.int32)
        check(self.lib.mk_get_schedule(self.h, out.ctypes.data, out.size, ctypes.byref(n), ctypes.byref(nsm),
                                       ctypes.byref(mi)), "mk_get_schedule")
        return out

    def status(self) -> dict:
        st = MkStatus()
        check(self.lib.mk_get_status(self.h, ctypes.byref(st)), "mk_get_status")
        return st.as_dict()

    def trace(self) -> np.ndarray:
        n = ctypes.c_size_t(0)
        check(self.lib.mk_get_trace(self.h, None, 0, ctypes.byref(n)), "mk_get_trace")
        out = np.empty(n.value, dtype=np.uint64)
        check(self.lib.mk_get_trace(self.h, out.ctypes.data, out.size, ctypes.byref(n)), "mk_get_trace")
        return out

    def reset(self):
        check(self.lib.mk_reset(self.h), "mk_reset")

    def inject_fault(self, kind: int, arg: int = 0):
        check(self.lib.mk_inject_fault(self.h, kind, arg), "mk_inject_fault")

    def last_step_ns(self) -> float:
        ns = ctypes.c_double(0)
        check(self.lib.mk_last_step_ns(self.h, ctypes.byref(ns)), "mk_last_step_ns")
        return ns.value


def attention_decode(q, kcache, vcache, n_pos: int, splits: int, out, workspace=None, stream=None):
    """mk_attention_decode on torch CUDA tensors: q [nq, d] fp32, kcache/vcache
    [nkv, max_seq, d] bf16 bits, out [nq, d] fp32.  Allocates the workspace
    with torch when none is given."""
    import torch
    lib = load()
    nq, d = int(q.shape[0]), int(q.shape[1])
    nkv, max_seq = int(kcache.shape[0]), int(kcache.shape[1])
    need = lib.mk_attention_workspace_bytes(nq, d, splits)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    s = stream if stream is not None else torch.cuda.current_stream()
    check(lib.mk_attention_decode(_ptr(q), _ptr(kcache), _ptr(vcache), nq, nkv, d, n_pos, max_seq, splits, _ptr(out),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  ctypes.c_void_p(s.cuda_stream)), "mk_attention_decode")
    return out


def attention_decode_noalloc(q, kcache, vcache, n_pos: int, splits: int, out, stream=None):
    """mk_attention_decode_noalloc on torch CUDA tensors (same layout as
    attention_decode); the library uses its own fixed device scratch, so
    nothing is allocated for the call."""
    import torch
    lib = load()
    nq, d = int(q.shape[0]), int(q.shape[1])
    nkv, max_seq = int(kcache.shape[0]), int(kcache.shape[1])
    s = stream if stream is not None else torch.cuda.current_stream()
    check(lib.mk_attention_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), nq, nkv, d, n_pos, max_seq, splits,
                                          _ptr(out), ctypes.c_void_p(s.cuda_stream)), "mk_attention_decode_noalloc")
    return out


def to_device(model: dict, device="cuda"):
    """Copy a dict of bf16-bit numpy arrays (the layout Decoder expects) to the
    device as int16 tensors (same bits).  Tied heads stay one tensor."""
    import torch
    memo = {}

    def up(a):
        if isinstance(a, list):
            return [up(x) for x in a]
        key = id(a)
        if key not in memo:
            memo[key] = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device)
        return memo[key]

    out = {k: up(v) for k, v in model.items() if k != "layers"}
    out["layers"] = [{k: up(v) for k, v in L.items()} for L in model["layers"]]
    return out
