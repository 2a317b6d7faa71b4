"""Algorithmic bytes of one decode step (the HBM roofline's numerator).

Decode is bound by memory bandwidth: every weight is read once per generated
token ("Crear desde cero un motor de inferencia ..." §1.2; "LLMs in einen
MegaKernel kompilieren ...", "Der zentrale Wert von MPK": 16 GB of weights at
1.6 TB/s bound a token at 10 ms).  The bytes one step must move are:

  weights  every bf16 matrix once (fused QKV, O, gate/up, down, LM head),
           the norm vectors, the QKV biases, and one embedding row per request
           (the whole table is the LM head when embeddings are tied);
  KV read  (pos + 1) keys and values per layer and KV head, bf16, per request;
  KV write one key and one value per layer and KV head, bf16, per request;
  outputs  the next ids (4 bytes per request), plus fp32 logits when asked.

Activations (a few KB per layer, L2-resident) are not counted.
"""
from __future__ import annotations


def weight_bytes(m, wbytes: int = 2) -> int:
    """wbytes: bytes per matrix weight -- 2 for bf16, 1 for fp8 (plus one fp32
    scale per matrix row); norms and biases stay bf16."""
    h, f, qd, kvd = m.hidden, m.ffn, m.q_dim, m.kv_dim
    mat = m.n_layers * ((qd + 2 * kvd) * h + h * qd + 2 * f * h + h * f) + m.vocab * h
    rows = m.n_layers * ((qd + 2 * kvd) + h + 2 * f + h) + m.vocab
    vec = m.n_layers * (2 * h + ((qd + 2 * kvd) if m.qkv_bias else 0)) + h   # norms, biases
    return wbytes * mat + 2 * vec + (4 * rows if wbytes == 1 else 0)


def kv_read_bytes(m, pos: int) -> int:
    return (pos + 1) * 2 * m.n_layers * m.kv_dim * 2


def kv_write_bytes(m) -> int:
    return 2 * m.n_layers * m.kv_dim * 2


def step_bytes(m, positions, want_logits: bool = False, wbytes: int = 2) -> int:
    """Bytes one decode step moves for requests at `positions`."""
    n = len(positions)
    b = weight_bytes(m, wbytes)
    b += n * (0 if m.tied_embeddings else m.hidden * 2)   # embedding rows
    if m.tied_embeddings:
        b += 0                                             # rows come from the LM-head read
    for p in positions:
        b += kv_read_bytes(m, p) + kv_write_bytes(m)
    b += 4 * n + (4 * m.vocab * n if want_logits else 0)
    return b


def step_flops(m, positions) -> int:
    """2 flops per weight per request plus the attention dot products."""
    n = len(positions)
    h, f, qd, kvd = m.hidden, m.ffn, m.q_dim, m.kv_dim
    mat = m.n_layers * ((qd + 2 * kvd) * h + h * qd + 3 * f * h) + m.vocab * h
    att = sum(4 * m.n_layers * m.n_q_heads * m.head_dim * (p + 1) for p in positions)
    return 2 * mat * n + att


def bound_ms(bytes_per_token: float, bandwidth_bytes_per_s: float) -> float:
    return 1e3 * bytes_per_token / bandwidth_bytes_per_s
