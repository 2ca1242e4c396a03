"""Second, independent CPU restatement of the decode step in fp32 (torch CPU ops).

TEST INFRASTRUCTURE ONLY.  It exists to measure the fp32-vs-fp64 noise floor
(the Hyperkernel teardown, "Which claims the repo backs", weighs agreement
with an independent implementation against that implementation's own noise
floor) and to cross-check the C oracle: it is written from the same plain decoder definition with torch
tensor ops, sharing no code with oracle.c.
"""
from __future__ import annotations

import numpy as np
import torch


def _bf(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).float()


class Fp32Model:
    def __init__(self, cfg, weights: dict, kcache: np.ndarray, vcache: np.ndarray):
        self.cfg = cfg
        self.embed = _bf(weights["embed"])
        self.lm_head = _bf(weights["lm_head"])
        self.final_norm = _bf(weights["final_norm"])
        self.layers = []
        for L in weights["layers"]:
            d = {k: _bf(L[k]) for k in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm")}
            if cfg.n_experts:
                d["router"] = _bf(L["router"])
                for k in ("w_gate", "w_up", "w_down"):
                    d[k] = [_bf(t) for t in L[k]]
            else:
                for k in ("w_gate", "w_up", "w_down"):
                    d[k] = _bf(L[k])
            self.layers.append(d)
        # bf16 caches kept as bf16 tensors (appends round to bf16).
        self.k = torch.from_numpy(kcache.view(np.int16).copy()).view(torch.bfloat16)
        self.v = torch.from_numpy(vcache.view(np.int16).copy()).view(torch.bfloat16)

    def _norm(self, x, w):
        return x * torch.rsqrt(x.pow(2).mean() + self.cfg.rms_eps) * w

    def _rope(self, t, pos):
        d = self.cfg.head_dim
        half = d // 2
        inv = self.cfg.rope_theta ** (-torch.arange(half, dtype=torch.float64) * 2.0 / d)
        ang = (pos * inv)
        c = torch.cos(ang).float()
        s = torch.sin(ang).float()
        a, b = t[..., :half], t[..., half:]
        return torch.cat([a * c - b * s, b * c + a * s], dim=-1)

    def _ffn(self, xn, wg, wu, wd):
        g = wg @ xn
        u = wu @ xn
        return wd @ (torch.nn.functional.silu(g) * u)

    @torch.no_grad()
    def step(self, token: int, pos: int) -> dict:
        cfg = self.cfg
        nq, nkv, d = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
        x = self.embed[token].clone()
        hidden = [x.clone()]
        for l, W in enumerate(self.layers):
            xn = self._norm(x, W["attn_norm"])
            q = self._rope((W["wq"] @ xn).view(nq, d), pos)
            k = self._rope((W["wk"] @ xn).view(nkv, d), pos)
            v = (W["wv"] @ xn).view(nkv, d)
            self.k[l, :, pos] = k.to(torch.bfloat16)
            self.v[l, :, pos] = v.to(torch.bfloat16)
            K = self.k[l, :, : pos + 1].float()             # [nkv, n, d]
            V = self.v[l, :, : pos + 1].float()
            rep = nq // nkv
            Kq = K.repeat_interleave(rep, dim=0)            # [nq, n, d]
            Vq = V.repeat_interleave(rep, dim=0)
            sc = torch.einsum("hd,hnd->hn", q, Kq) / (d ** 0.5)
            p = torch.softmax(sc, dim=-1)
            att = torch.einsum("hn,hnd->hd", p, Vq).reshape(-1)
            x = x + W["wo"] @ att
            xn = self._norm(x, W["ffn_norm"])
            if cfg.n_experts:
                r = W["router"] @ xn
                top = torch.topk(r, cfg.top_k)
                wts = torch.softmax(top.values, dim=-1)
                acc = torch.zeros_like(x)
                for t in range(cfg.top_k):
                    e = int(top.indices[t])
                    acc += wts[t] * self._ffn(xn, W["w_gate"][e], W["w_up"][e], W["w_down"][e])
                x = x + acc
            else:
                x = x + self._ffn(xn, W["w_gate"], W["w_up"], W["w_down"])
            hidden.append(x.clone())
        logits = self.lm_head @ self._norm(x, self.final_norm)
        return {"logits": logits.double().numpy(), "hidden": torch.stack(hidden).double().numpy(),
                "next": int(torch.argmax(logits))}
