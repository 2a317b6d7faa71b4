"""The tensor-core prefill against the decode-step prefill and the oracle.

mk_prefill runs positions 0..len-2 of each prompt as whole-sequence
operators (tcgen05 GEMMs on bf16 weights and the fp32 activations split into
three bf16 parts, causal attention over the cache on the tensor cores; by
default all of it one persistent kernel per block) and the last position as a
decode step.  The cache it leaves must be the decode-step prefill's up to the
tensor cores' accumulation rounding: per cache head a relative L2 difference
of a few 1e-4 (bf16 entries equal or a step or two apart), and what follows
must match the oracle at the usual bar.  Prompt lengths cover several 128-token GEMM tiles
with a ragged tail, a block boundary (2048 positions) and single-token
prompts (nothing for the GEMM path).
"""
import numpy as np
import pytest
import torch

from persistent_megakernel_03_b200 import binding, synth
from parity_util import assert_within, compare, oracle_trace, run_gpu

pytestmark = pytest.mark.gpu


def _cache(dec, model, lens):
    d = model.head_dim
    out = []
    for r, n in enumerate(lens):
        buf = torch.empty((n, d), dtype=torch.bfloat16, device="cuda")
        for l in range(model.n_layers):
            for g in range(model.n_kv_heads):
                for which in (0, 1):
                    dec.copy_kv(r, l, g, which, n, buf)
                    torch.cuda.synchronize()
                    out.append(buf.float().cpu().numpy().copy())
    return out


def _prefill(model, w, lens, steps_mode):
    toks, offs = synth.make_packed_prompts(lens, model.vocab, seed=11)
    dec = binding.Decoder(model, w, max(lens) + 2, max_batch=len(lens), prefill_steps=steps_mode)
    logits = torch.empty(len(lens), model.vocab, device="cuda")
    ids = torch.empty(len(lens), dtype=torch.int32, device="cuda")
    dec.prefill(toks.to(torch.int32).cuda(), offs.tolist(), logits, ids)
    torch.cuda.synchronize()
    assert dec.status() == 0, dec.last_error()
    return dec, logits.cpu().numpy(), ids.cpu().numpy()


@pytest.mark.parametrize("model,lens", [
    (synth.TINY, [300, 1, 129, 2100]),
    (synth.QWEN05B.with_layers(2), [200, 77]),
    (synth.LLAMA8B.with_layers(2), [260, 5]),
], ids=["tiny", "qwen-2l", "llama-2l"])
def test_tensor_core_prefill_matches_step_prefill(cuda_ok, model, lens):
    w = {k: v.cuda() for k, v in synth.make_model(model, 4).items()}
    a, la, ia = _prefill(model, w, lens, 0)
    b, lb, ib = _prefill(model, w, lens, 1)
    ca, cb = _cache(a, model, lens), _cache(b, model, lens)
    far = total = 0
    for x, y in zip(ca, cb):
        diff = np.abs(x - y)
        rms = float(np.sqrt(np.mean(y * y)))
        step = np.maximum(np.abs(y), rms) * 2.0 ** -7   # one bf16 step (floor: the head's rms)
        assert np.linalg.norm(x - y) <= 2e-3 * np.linalg.norm(y)
        assert diff.max() <= 0.02 * np.abs(y).max()     # no row or column gone astray
        far += int(np.sum(diff > step * 1.01))
        total += diff.size
    assert far / total < 0.01, far / total
    np.testing.assert_allclose(la, lb, atol=5e-3, rtol=0)


def test_tensor_core_prefill_then_decode_matches_oracle(cuda_ok):
    model = synth.LLAMA8B.with_layers(2)
    w = synth.make_model(model, 6)
    prompt = synth.make_prompt(333, model.vocab, seed=8).tolist()
    tr, _, _ = oracle_trace(model, w, prompt, 4, 340)
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, 340)
    gl, gh, gi = run_gpu(dec, model, tr)
    assert_within(compare(tr, gl, gh, gi))


@pytest.mark.parametrize("model,lens", [
    (synth.TINY, [300, 1, 129, 2100]),
    (synth.QWEN05B.with_layers(2), [200, 77, 130]),
    (synth.LLAMA8B.with_layers(2), [260, 5, 64, 129]),
], ids=["tiny", "qwen-2l", "llama-2l"])
def test_tensor_core_attention_matches_cuda_core_attention(cuda_ok, model, lens):
    # the prefill's attention on the tensor cores (queries and probabilities as
    # two bf16 parts, fp32 accumulation) against the fp32 CUDA-core attention:
    # the caches they leave differ by the accumulation order only
    w = {k: v.cuda() for k, v in synth.make_model(model, 5).items()}
    a, la, _ = _prefill_opt(model, w, lens, prefill_per_operator=1, prefill_attention=0)
    b, lb, _ = _prefill_opt(model, w, lens, prefill_per_operator=1, prefill_attention=1)
    for x, y in zip(_cache(a, model, lens), _cache(b, model, lens)):
        assert np.linalg.norm(x - y) <= 2e-3 * np.linalg.norm(y)
        assert np.abs(x - y).max() <= 0.02 * np.abs(y).max()
    np.testing.assert_allclose(la, lb, atol=5e-3, rtol=0)


def _prefill_opt(model, w, lens, **kw):
    toks, offs = synth.make_packed_prompts(lens, model.vocab, seed=11)
    dec = binding.Decoder(model, w, max(lens) + 2, max_batch=len(lens), **kw)
    logits = torch.empty(len(lens), model.vocab, device="cuda")
    ids = torch.empty(len(lens), dtype=torch.int32, device="cuda")
    dec.prefill(toks.to(torch.int32).cuda(), offs.tolist(), logits, ids)
    torch.cuda.synchronize()
    assert dec.status() == 0, dec.last_error()
    return dec, logits.cpu().numpy(), ids.cpu().numpy()
