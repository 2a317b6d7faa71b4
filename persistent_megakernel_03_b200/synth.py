"""Seeded synthetic models and prompts.

This module is the one piece of Python shared by the CPU oracle's tests and
the CUDA path.  It holds no model arithmetic: it only draws random numbers and
describes shapes.  Both sides always receive the same bytes.

Shapes are the decoder families the MPK pages and the Qwen2.5 slides discuss
(de.news.hada.io/topic?id=21563 "Der zentrale Wert von MPK": 39-token prompt,
512 generated tokens; speakerdeck "LLM高速化勉強会資料" slide 8: Qwen2.5-0.5B).

Weights: every matrix and bias is drawn i.i.d. N(0, 0.02) in fp32 and rounded
to bf16 (round-to-nearest-even, torch's ``.to(torch.bfloat16)``); norm weights
are 1.  Tensors are drawn in a fixed order from one generator: embed, then per
layer wq, wk, wv, [bq, bk, bv], wo, w_gate, w_up, w_down, then lm_head (when
untied).  On CPU the generator is ``torch.Generator('cpu')``; a model that is
made directly on a CUDA device draws from ``torch.Generator('cuda')`` with the
same seed (different bytes, same distribution: the CPU stream would take
minutes for the 8B shape).  Whoever compares two implementations copies one
set of bytes to both.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch


@dataclass(frozen=True)
class ModelConfig:
    name: str
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float
    rope_theta: float
    qkv_bias: bool = False
    tied_embeddings: bool = False

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def n_params(self) -> int:
        h, f = self.hidden, self.ffn
        per_layer = (2 * h                       # two norms
                     + (self.q_dim + 2 * self.kv_dim) * h
                     + (self.q_dim + 2 * self.kv_dim if self.qkv_bias else 0)
                     + h * self.q_dim + 3 * f * h)
        emb = self.vocab * h
        return emb + self.n_layers * per_layer + h + (0 if self.tied_embeddings else emb)

    def with_layers(self, n: int) -> "ModelConfig":
        return dataclasses.replace(self, n_layers=n, name=f"{self.name}-{n}l")


# The three decoder shapes.  RMSNorm eps: the tiny shape states 1e-6; the Qwen
# and Llama shapes use their named models' own values (1e-6 and 1e-5).
TINY = ModelConfig("tiny", n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2,
                   head_dim=64, ffn=768, vocab=4096, rms_eps=1e-6, rope_theta=10000.0)
QWEN05B = ModelConfig("qwen2.5-0.5b-shape", n_layers=24, hidden=896, n_q_heads=14,
                      n_kv_heads=2, head_dim=64, ffn=4864, vocab=151936, rms_eps=1e-6,
                      rope_theta=1e6, qkv_bias=True, tied_embeddings=True)
LLAMA8B = ModelConfig("llama-3-8b-shape", n_layers=32, hidden=4096, n_q_heads=32,
                      n_kv_heads=8, head_dim=128, ffn=14336, vocab=128256, rms_eps=1e-5,
                      rope_theta=500000.0)

MODELS = {m.name: m for m in (TINY, QWEN05B, LLAMA8B)}


@dataclass(frozen=True)
class Workload:
    """One decode workload: a model, prompt lengths and decode steps."""
    name: str
    model: ModelConfig
    prompt_lens: tuple          # one entry per request
    decode_steps: int

    @property
    def n_req(self) -> int:
        return len(self.prompt_lens)

    @property
    def max_seq(self) -> int:
        return max(self.prompt_lens) + self.decode_steps


def packed_batch_lengths(n_req: int = 8, lo: int = 32, hi: int = 2048, seed: int = 2) -> tuple:
    g = torch.Generator("cpu").manual_seed(seed)
    return tuple(int(v) for v in torch.randint(lo, hi + 1, (n_req,), generator=g))


WORKLOADS = {
    "tiny": Workload("tiny", TINY, (16,), 16),
    "qwen05b": Workload("qwen05b", QWEN05B, (39,), 512),
    "llama8b": Workload("llama8b", LLAMA8B, (39,), 512),
    "llama8b-32k": Workload("llama8b-32k", LLAMA8B, (32768,), 256),
    "llama8b-batch8": Workload("llama8b-batch8", LLAMA8B, packed_batch_lengths(), 256),
}


LAYER_KEYS = ("attn_norm", "wq", "wk", "wv", "bq", "bk", "bv", "wo",
              "ffn_norm", "w_gate", "w_up", "w_down")


def weight_shapes(cfg: ModelConfig) -> List[tuple]:
    """(name, shape) in generation order; norm weights are listed last."""
    h, f = cfg.hidden, cfg.ffn
    out = [("embed", (cfg.vocab, h))]
    for l in range(cfg.n_layers):
        p = f"layers.{l}."
        out += [(p + "wq", (cfg.q_dim, h)), (p + "wk", (cfg.kv_dim, h)),
                (p + "wv", (cfg.kv_dim, h))]
        if cfg.qkv_bias:
            out += [(p + "bq", (cfg.q_dim,)), (p + "bk", (cfg.kv_dim,)),
                    (p + "bv", (cfg.kv_dim,))]
        out += [(p + "wo", (h, cfg.q_dim)), (p + "w_gate", (f, h)),
                (p + "w_up", (f, h)), (p + "w_down", (h, f))]
    if not cfg.tied_embeddings:
        out.append(("lm_head", (cfg.vocab, h)))
    return out


def make_model(cfg: ModelConfig, seed: int = 0, device: str = "cpu",
               std: float = 0.02) -> Dict[str, torch.Tensor]:
    """Random-init bf16 weights of ``cfg`` (see module docstring)."""
    dev = torch.device(device)
    g = torch.Generator(dev.type if dev.type == "cuda" else "cpu")
    g.manual_seed(seed)
    w: Dict[str, torch.Tensor] = {}
    for name, shape in weight_shapes(cfg):
        t = torch.empty(shape, dtype=torch.float32, device=dev)
        t.normal_(0.0, std, generator=g)
        w[name] = t.to(torch.bfloat16)
        del t
    ones = lambda: torch.ones(cfg.hidden, dtype=torch.bfloat16, device=dev)
    for l in range(cfg.n_layers):
        w[f"layers.{l}.attn_norm"] = ones()
        w[f"layers.{l}.ffn_norm"] = ones()
    w["final_norm"] = ones()
    return w


def make_prompt(n: int, vocab: int, seed: int = 1) -> torch.Tensor:
    """Uniform random token ids in [0, vocab), int32, on CPU."""
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randint(0, vocab, (n,), generator=g, dtype=torch.int64).to(torch.int32)


def make_packed_prompts(lens, vocab: int, seed: int = 1):
    """Requests packed as one flat token sequence plus offsets (n_req + 1)."""
    total = int(sum(lens))
    toks = make_prompt(total, vocab, seed)
    offs = [0]
    for n in lens:
        offs.append(offs[-1] + int(n))
    return toks, torch.tensor(offs, dtype=torch.int32)


def layer_tensor(w: Dict[str, torch.Tensor], l: int, key: str) -> Optional[torch.Tensor]:
    return w.get(f"layers.{l}.{key}")
