"""Per-stage parity at the edge positions, in every execution mode.

A one-layer model makes every stage of the step observable: after a decode
step at position p the library's last-layer vectors are read back (rotated
queries, attention output, SwiGLU activation, residual stream, and the K/V
cache), and each is compared with the oracle's function for that stage
applied to the same inputs the library's stage had:

  q     = RoPE(Wq rmsnorm(E[token]) (+ bq), p)            per query head
  attn  = softmax(q K^T / sqrt(d)) V over the cache rows 0..p   (GQA groups)
  act   = silu(Wg rmsnorm(x1)) * (Wu rmsnorm(x1)),  x1 = E[token] + Wo attn
  x     = x1 + Wd act

Positions: 0 (a single key), both sides of every key-split boundary the
attention tasks can have (a split holds one ring chunk of keys: 64 keys at
head_dim 128, 128 at head_dim 64; beyond S chunks the splits grow), and
max_seq - 1.  Differences are fp32 reassociation only, so the bars are tight
(relative L2 <= 2e-5 for the GEMV stages, 1e-5 for attention).
"""
import numpy as np
import pytest
import torch

import oracle
from persistent_megakernel_03_b200 import binding, synth

pytestmark = pytest.mark.gpu

GEMV_REL = 2e-5
ATTN_REL = 1e-5


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / max(np.linalg.norm(b), 1e-30))


def _stage_check(model, w, dec, tok, p):
    d, G = model.head_dim, model.group
    H, F, qd = model.hidden, model.ffn, model.q_dim
    q = torch.empty(qd, device="cuda")
    att = torch.empty(qd, device="cuda")
    act = torch.empty(F, device="cuda")
    x = torch.empty(H, device="cuda")
    dec.copy_activation(binding.ACT_Q, q)
    dec.copy_activation(binding.ACT_ATTN, att)
    dec.copy_activation(binding.ACT_FFN, act)
    dec.copy_activation(binding.ACT_X, x)
    K, V = [], []
    for g in range(model.n_kv_heads):
        for which, dst in ((0, K), (1, V)):
            buf = torch.empty(p + 1, d, dtype=torch.bfloat16, device="cuda")
            dec.copy_kv(0, 0, g, which, p + 1, buf)
            dst.append(buf)
    torch.cuda.synchronize()
    q, att, act, x = (t.cpu().numpy() for t in (q, att, act, x))
    K = [k.float().cpu().numpy() for k in K]
    V = [v.float().cpu().numpy() for v in V]
    L = lambda key: w[f"layers.0.{key}"]
    # QKV + bias + RoPE (and the newest cache row)
    x0 = w["embed"][tok].float().numpy()
    xn = oracle.rmsnorm(x0, L("attn_norm"), model.rms_eps)
    proj = {}
    for key, bkey in (("wq", "bq"), ("wk", "bk"), ("wv", "bv")):
        y = oracle.gemv(L(key), xn)
        if model.qkv_bias:
            y = y + L(bkey).float().numpy()
        proj[key] = y.astype(np.float32)
    q_want = np.concatenate([oracle.rope(proj["wq"][h * d:(h + 1) * d], p, model.rope_theta)
                             for h in range(model.n_q_heads)])
    assert _rel(q, q_want) <= GEMV_REL, ("q", p, _rel(q, q_want))
    for g in range(model.n_kv_heads):
        k_want = oracle.rope(proj["wk"][g * d:(g + 1) * d], p, model.rope_theta)
        k_want = torch.from_numpy(k_want).to(torch.bfloat16).float().numpy()
        v_want = torch.from_numpy(proj["wv"][g * d:(g + 1) * d]).to(torch.bfloat16).float().numpy()
        # the newest row: equal, or one bf16 step apart where the fp32 value sat
        # next to a rounding boundary
        assert np.allclose(K[g][p], k_want, rtol=2**-7, atol=1e-6), ("k row", p, g)
        assert np.allclose(V[g][p], v_want, rtol=2**-7, atol=1e-6), ("v row", p, g)
    # attention over the library's own cache and queries
    att_want = np.concatenate([oracle.attend(q[h * d:(h + 1) * d], K[h // G], V[h // G])
                               for h in range(model.n_q_heads)])
    assert _rel(att, att_want) <= ATTN_REL, ("attn", p, _rel(att, att_want))
    # O projection + residual, RMSNorm, gate/up + SwiGLU on the library's attn
    x1 = (x0 + oracle.gemv(L("wo"), att)).astype(np.float32)
    xn2 = oracle.rmsnorm(x1, L("ffn_norm"), model.rms_eps)
    gte, up = oracle.gemv(L("w_gate"), xn2), oracle.gemv(L("w_up"), xn2)
    act_want = np.array([oracle.silu(float(a)) for a in gte], np.float32) * up
    assert _rel(act, act_want) <= GEMV_REL, ("act", p, _rel(act, act_want))
    # down + residual on the library's act
    x_want = x1 + oracle.gemv(L("w_down"), act)
    assert _rel(x, x_want) <= GEMV_REL, ("x", p, _rel(x, x_want))


def _edge_positions(model, max_seq, splits):
    kpc = 16384 // (model.head_dim * 2)          # keys per ring chunk
    ps = {0, max_seq - 1}
    for b in (kpc, 2 * kpc, splits * kpc):       # one, two and S chunks of keys
        ps.update({b - 1, b})
    return sorted(p for p in ps if p < max_seq)


CASES = [
    (synth.LLAMA8B.with_layers(1), 1300),
    (synth.QWEN05B.with_layers(1), 2400),
]


@pytest.mark.parametrize("mode", [binding.MODE_MEGAKERNEL, binding.MODE_PER_OP,
                                  binding.MODE_PER_OP_GRAPH], ids=["mk", "per_op", "graph"])
@pytest.mark.parametrize("model,max_seq", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_each_stage_at_edge_positions(cuda_ok, model, max_seq, mode):
    w = synth.make_model(model, 11, device="cuda")
    # non-unit norm weights: a stage that applies the wrong norm must show
    g = torch.Generator("cuda").manual_seed(12)
    for key in ("layers.0.attn_norm", "layers.0.ffn_norm", "final_norm"):
        w[key] = (1 + 0.25 * torch.randn(model.hidden, generator=g, device="cuda")).to(torch.bfloat16)
    w_cpu = {k: v.cpu() for k, v in w.items()}
    dec = binding.Decoder(model, w, max_seq, mode=mode)
    splits = binding.Plan(model, max_seq, torch.cuda.get_device_properties(0).multi_processor_count
                          ).info.attn_splits
    prompt = synth.make_prompt(max_seq, model.vocab, seed=13).to(torch.int32).cuda()
    ids = torch.empty(1, dtype=torch.int32, device="cuda")
    tok = torch.empty(1, dtype=torch.int32, device="cuda")
    for p in _edge_positions(model, max_seq, splits):
        if p > 0:
            dec.prefill(prompt[:p], [0, p], None, ids)   # cache rows 0..p-1
        t = int(prompt[p].item())
        tok.fill_(t)
        dec.decode(tok, [p], None, ids)
        assert dec.status() == 0, dec.last_error()
        _stage_check(model, w_cpu, dec, t, p)
