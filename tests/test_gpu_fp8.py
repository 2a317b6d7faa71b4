"""fp8 (e4m3, per-row power-of-two scales) decode weights against the oracle.

The library is given the raw bf16 model with mk_options.weight_format = 1
and quantizes it on the device; the oracle runs the model its own rule
(orc_quantize_fp8_rows) makes from the same raw weights, in fp32.  The decode
GEMVs stream the fp8 codes; the tensor-core prefill and the batched step use
the same values."""
import pytest
import torch

import oracle
from persistent_megakernel_03_b200 import binding, synth
from parity_util import assert_within, compare, oracle_trace, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("model,P,steps", [
    (synth.TINY, 16, 12),
    (synth.LLAMA8B.with_layers(2), 39, 6),
    (synth.QWEN05B.with_layers(2), 39, 6),
], ids=["tiny", "llama-2l", "qwen-2l"])
def test_fp8_from_raw_bf16_matches_oracle(cuda_ok, model, P, steps):
    raw = synth.make_model(model, 5)
    prompt = synth.make_prompt(P, model.vocab, seed=6).tolist()
    tr, _, _ = oracle_trace(model, oracle.quantize_fp8_model(model, raw), prompt, steps, P + steps)
    dec = binding.Decoder(model, {k: v.cuda() for k, v in raw.items()}, P + steps, weight_format=1)
    gl, gh, gi = run_gpu(dec, model, tr)
    assert_within(compare(tr, gl, gh, gi))


def test_fp8_multistep_loop_equals_single_steps(cuda_ok):
    model = synth.TINY
    w = synth.make_model(model, 1)
    prompt = torch.tensor(synth.make_prompt(16, model.vocab).tolist(), dtype=torch.int32, device="cuda")
    outs = []
    for loop in (False, True):
        dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, 32, weight_format=1)
        ids = torch.empty(1, dtype=torch.int32, device="cuda")
        dec.prefill(prompt, [0, 16], None, ids)
        seq = torch.empty(10, dtype=torch.int32, device="cuda")
        if loop:
            dec.decode_steps(ids, 16, 10, seq)
        else:
            nxt = torch.empty(1, dtype=torch.int32, device="cuda")
            for s in range(10):
                dec.decode(ids, [16 + s], None, nxt)
                seq[s] = nxt[0]
                ids.copy_(nxt)
        torch.cuda.synchronize()
        assert dec.status() == 0, dec.last_error()
        outs.append(seq.tolist())
    assert outs[0] == outs[1]
