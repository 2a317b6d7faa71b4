"""Parity at the benchmark's own shapes, against the oracle's own prefill.

- the whole 32-layer Llama-3-8B-shaped model the benchmark times: 39-token
  prompt, then teacher-forced decode steps ("LLMs in einen MegaKernel
  kompilieren ...", "Der zentrale Wert von MPK": a 39-token prompt);
- a prompt longer than one 2048-position block of the tensor-core prefill
  at Llama widths: the oracle runs the whole prompt itself (orc_prefill, one
  decode step per position), so every cache row of every layer past the
  block boundary meets an independent value;
- the eight requests of the batched workload, with its prompt lengths
  (uniform in [32, 2048], packed with offsets: "LLM高速化勉強会資料" slides
  14-16), at Llama widths.

Acceptance (bf16 weights, fp32 accumulation): logits max-abs <= 3e-2,
residual-stream relative L2 <= 1e-2, the greedy id where the oracle's
top-1/top-2 margin >= 0.1; cache rows within a relative L2 of 2e-3 per head
(the tensor cores' accumulation order; the decode bar applies after it).
"""
import numpy as np
import pytest
import torch

from persistent_megakernel_03_b200 import binding, synth
from parity_util import assert_within, compare, oracle_trace, run_gpu
from test_gpu_batch import _run_batch

pytestmark = pytest.mark.gpu

CACHE_REL_L2 = 2e-3


def test_llama8b_full_depth(cuda_ok):
    model = synth.LLAMA8B
    w = synth.make_model(model, 0, device="cuda")
    w_cpu = {k: v.cpu() for k, v in w.items()}
    prompt = synth.make_prompt(39, model.vocab).tolist()
    steps = 4
    tr, _, _ = oracle_trace(model, w_cpu, prompt, steps, 600)
    dec = binding.Decoder(model, w, 600)
    del w
    gl, gh, gi = run_gpu(dec, model, tr)
    reports = compare(tr, gl, gh, gi)
    assert_within(reports)
    dec.close()


def _cache_rel(dec, st, layer, g, which, n, positions):
    got = torch.empty(n, st.model.cfg.head_dim, dtype=torch.bfloat16, device="cuda")
    dec.copy_kv(0, layer, g, which, n, got)
    torch.cuda.synchronize()
    got = got.float().cpu().numpy()[positions]
    want = st.kv(layer, g, which, n)[positions]
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


def test_llama_width_prefill_past_one_block_against_the_oracles_prefill(cuda_ok):
    model = synth.LLAMA8B.with_layers(2)
    w = synth.make_model(model, 3, device="cuda")
    w_cpu = {k: v.cpu() for k, v in w.items()}
    P, steps = 2100, 3
    prompt = synth.make_prompt(P, model.vocab, seed=5).tolist()
    tr, om, st = oracle_trace(model, w_cpu, prompt, steps, P + steps)
    dec = binding.Decoder(model, w, P + steps)
    gl, gh, gi = run_gpu(dec, model, tr)
    assert_within(compare(tr, gl, gh, gi))
    # every layer's cache inside the first block, across its end and past it
    for positions in (np.arange(0, 64), np.arange(2040, 2056), np.arange(2056, P)):
        for layer in range(model.n_layers):
            for g in (0, model.n_kv_heads - 1):
                for which in (0, 1):
                    rel = _cache_rel(dec, st, layer, g, which, P, positions)
                    assert rel <= CACHE_REL_L2, (layer, g, which, positions[0], rel)


def test_llama_width_eight_requests_of_the_batched_workload(cuda_ok):
    model = synth.LLAMA8B.with_layers(2)
    lens = list(synth.packed_batch_lengths())
    w = synth.make_model(model, 4)
    _run_batch(model, w, lens, 3, max(lens) + 3)
