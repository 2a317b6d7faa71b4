"""Decode after a 32768-token prompt (the long-context workload) against the oracle.

A full-length oracle prefill takes far too long on host cores, so the long
context is checked with what holds at any length, on a model of the
Llama-3-8B shape's widths cut to two layers:

* layer 0's cached K and V at a position depend on that position's token
  alone (RMSNorm, the K/V projections, RoPE at that position), so the oracle
  computes sampled rows directly from the embedding (the prompt runs through
  the tensor-core prefill, whose sums round differently: entries agree to a
  bf16 step of the row's scale);
* the oracle takes the GPU's cache for positions [0, P-1) as its own state,
  recomputes the last prompt position and decodes teacher-forced steps after
  it; logits, residual stream and greedy ids must meet the usual acceptance
  bar against the GPU's prefill output and decode steps.

The prompt is filled by the library's prefill, the attention runs with the
automatic split count (about 18 splits of ~1820 keys per KV head here).
"""
import numpy as np
import pytest
import torch

import oracle
from persistent_megakernel_03_b200 import binding, synth
from parity_util import OracleTrace, assert_within, compare

pytestmark = pytest.mark.gpu

P = 32768
STEPS = 4


@pytest.fixture(scope="module")
def long_ctx(cuda_ok):
    cfg = synth.LLAMA8B.with_layers(2)
    w = synth.make_model(cfg, 0, device="cuda")
    w_cpu = {k: v.cpu() for k, v in w.items()}
    max_seq = P + STEPS + 1
    dec = binding.Decoder(cfg, w, max_seq)
    del w
    prompt = synth.make_prompt(P, cfg.vocab, seed=1)
    logits = torch.empty(cfg.vocab, device="cuda")
    ids = torch.empty(1, dtype=torch.int32, device="cuda")
    hidden = torch.empty(cfg.hidden, device="cuda")
    dec.prefill(prompt.to(torch.int32).cuda(), [0, P], logits, ids)
    dec.copy_hidden(hidden)
    torch.cuda.synchronize()
    assert dec.status() == 0, dec.last_error()
    first = (logits.cpu().numpy().copy(), hidden.cpu().numpy().copy(), int(ids.item()))
    return cfg, w_cpu, dec, prompt.tolist(), first


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def test_layer0_cache_rows_at_sampled_positions(long_ctx):
    cfg, w, dec, prompt, _ = long_ctx
    d = cfg.head_dim
    positions = [0, 1, 255, 256, 4097, 17000, 32000, P - 1]
    buf = torch.empty((P, d), dtype=torch.bfloat16, device="cuda")
    for g in range(cfg.n_kv_heads):
        for which, name in ((0, "wk"), (1, "wv")):
            dec.copy_kv(0, 0, g, which, P, buf)
            torch.cuda.synchronize()
            got = buf.float().cpu().numpy()
            Wg = w[f"layers.0.{name}"][g * d:(g + 1) * d]
            for p in positions:
                x = w["embed"][prompt[p]].float().numpy()
                xn = oracle.rmsnorm(x, w["layers.0.attn_norm"], cfg.rms_eps)
                v = oracle.gemv(Wg, xn)
                if which == 0:
                    v = oracle.rope(v, p, cfg.rope_theta)
                want = _bf16(v)
                diff = np.abs(got[p] - want)
                # one bf16 step of the value, floored at the row's rms: the
                # prefill's tensor-core sums round differently from the
                # oracle's sequential fp32 sums, which moves entries near a
                # rounding boundary (and tiny entries) by a step
                rms = float(np.sqrt(np.mean(want * want)))
                step = np.maximum(np.abs(want), rms) * 2.0 ** -7
                assert np.mean(diff == 0) > 0.9, (g, which, p)
                assert np.all(diff <= step * 1.01), (g, which, p)


def test_decode_after_long_prompt_matches_oracle(long_ctx):
    cfg, w, dec, prompt, first = long_ctx
    d = cfg.head_dim
    om = oracle.OracleModel(cfg, w)
    st = om.new_state(P + STEPS + 1)
    buf = torch.empty((P - 1, d), dtype=torch.bfloat16, device="cuda")
    for l in range(cfg.n_layers):
        for g in range(cfg.n_kv_heads):
            for which in (0, 1):
                dec.copy_kv(0, l, g, which, P - 1, buf)
                torch.cuda.synchronize()
                st.set_kv(l, g, which, buf.float().cpu().numpy())
    tr = OracleTrace(prompt=prompt, feed=[])
    nid, lg, hid = om.decode(st, prompt[-1], P - 1)
    tr.logits.append(lg), tr.hidden.append(hid), tr.ids.append(nid)
    for s in range(STEPS):
        tr.feed.append(tr.ids[-1])
        nid, lg, hid = om.decode(st, tr.feed[-1], P + s)
        tr.logits.append(lg), tr.hidden.append(hid), tr.ids.append(nid)
    gl, gh, gi = [first[0]], [first[1]], [first[2]]
    logits = torch.empty(cfg.vocab, device="cuda")
    ids = torch.empty(1, dtype=torch.int32, device="cuda")
    hidden = torch.empty(cfg.hidden, device="cuda")
    tok = torch.empty(1, dtype=torch.int32, device="cuda")
    for s, t in enumerate(tr.feed):
        tok.fill_(int(t))
        dec.decode(tok, [P + s], logits, ids)
        dec.copy_hidden(hidden)
        torch.cuda.synchronize()
        gl.append(logits.cpu().numpy().copy())
        gh.append(hidden.cpu().numpy().copy())
        gi.append(int(ids.item()))
    assert dec.status() == 0, dec.last_error()
    assert_within(compare(tr, gl, gh, gi))
