"""Workload recipes for the batch-1 decode path (shapes, distributions, seeds).

These are synthetic random-init models with the shapes of the public models the
epic-kernel README targets ("3B model support": Llama 3.2 1B/3B; "Mixtral 8x7B
MoE for batch-1 inference").  No trained weights are involved: every weight is a
bf16 N(0, weight_sigma^2) draw (router: N(0, router_sigma^2)), every RMSNorm
weight is 1.0, and the pre-filled KV cache holds bf16 N(0, 1) keys and values
that are taken as already rotated.  Readings where the workload text is silent
(theta for the 3B and Mixtral shapes, eps beyond the tiny model, untied heads)
are the plain Llama/Mixtral values and are listed with the design notes.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    name: str
    n_layers: int
    hidden: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    n_experts: int = 0          # 0 = dense SiLU-gated FFN
    top_k: int = 0
    rms_eps: float = 1e-5
    rope_theta: float = 500000.0
    tied: bool = False
    seed: int = 0
    weight_sigma: float = 0.02
    router_sigma: float = 0.1
    kv_sigma: float = 1.0
    prefill: int = 0            # cache positions filled with random K/V before decoding
    prompt_len: int = 0         # random prompt tokens decoded one by one from pos 0
    steps: int = 0              # greedy decode steps after the prompt / prefill

    @property
    def max_seq(self) -> int:
        return self.prefill + self.prompt_len + self.steps

    @property
    def qkv_rows(self) -> int:
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim

    def with_(self, **kw) -> "ModelConfig":
        return dataclasses.replace(self, **kw)

    def weight_bytes_per_token(self) -> int:
        """Bytes of weights one decode step must read once (bf16): all GEMV
        matrices, norm vectors, one embedding row, the LM head, and for MoE only
        the router plus the top-k selected experts."""
        H, d, F = self.hidden, self.head_dim, self.ffn
        per_layer = self.qkv_rows * H + H * self.n_heads * d + 2 * H  # qkv, o, two norms
        if self.n_experts:
            per_layer += self.n_experts * H + self.top_k * 3 * F * H
        else:
            per_layer += 3 * F * H
        total = self.n_layers * per_layer + H + self.vocab * H + H  # + embed row, lm head, final norm
        return 2 * total

    def kv_bytes_per_token(self, pos: int) -> int:
        """KV bytes one step at position `pos` moves: read of positions 0..pos-1
        and the append write at pos (the new position itself is read from the
        freshly computed projection)."""
        per_pos = self.n_layers * 2 * self.n_kv_heads * self.head_dim * 2
        return per_pos * pos + per_pos


TINY = ModelConfig(name="tiny", n_layers=2, hidden=256, n_heads=4, n_kv_heads=2, head_dim=64, ffn=768,
                   vocab=4096, rms_eps=1e-5, rope_theta=10000.0, prompt_len=16, steps=8)

LLAMA_1B = ModelConfig(name="llama1b", n_layers=16, hidden=2048, n_heads=32, n_kv_heads=8, head_dim=64,
                       ffn=8192, vocab=128256, tied=True, rope_theta=500000.0, prefill=1024, steps=128)

LLAMA_3B = ModelConfig(name="llama3b", n_layers=28, hidden=3072, n_heads=24, n_kv_heads=8, head_dim=128,
                       ffn=8192, vocab=128256, rope_theta=500000.0, prefill=2048, steps=128)

SWEEP_PREFILLS = (128, 512, 2048, 8192, 16384)


def llama1b_sweep(prefill: int) -> ModelConfig:
    return LLAMA_1B.with_(name=f"llama1b_kv{prefill}", prefill=prefill, steps=64)


MIXTRAL_8L = ModelConfig(name="mixtral8l", n_layers=8, hidden=4096, n_heads=32, n_kv_heads=8, head_dim=128,
                         ffn=14336, vocab=32000, n_experts=8, top_k=2, rope_theta=1000000.0,
                         prefill=1024, steps=64)

# Beyond the sweep: long-context decode, the 1B shape with the cache pre-filled
# to 32768 and 65536 positions (attention becomes a large share of the bytes).
LONG_PREFILLS = (32768, 65536)

ALL = {c.name: c for c in (TINY, LLAMA_1B, LLAMA_3B, MIXTRAL_8L)}
for _p in SWEEP_PREFILLS + LONG_PREFILLS:
    ALL[f"llama1b_kv{_p}"] = llama1b_sweep(_p)


def get(name: str) -> ModelConfig:
    return ALL[name]
