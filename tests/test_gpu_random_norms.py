"""The CUDA paths against the oracle with non-unit RMSNorm weights.

The synthetic models' norm weights are all 1, which would hide a step that
applies the wrong norm's weights (a layer's attention or FFN norm, the final
norm).  Here every norm weight is 1 + 0.25 N(0, 1): the tensor-core prefill,
the persistent decode step and the batched step must still meet the
acceptance bar under teacher forcing.
"""
import pytest

from persistent_megakernel_03_b200 import binding, synth
from parity_util import assert_within, compare, oracle_trace, run_gpu
from test_gpu_batch import _run_batch
from test_oracle_pins import _random_norms

pytestmark = pytest.mark.gpu

MODELS = [synth.TINY, synth.QWEN05B.with_layers(2), synth.LLAMA8B.with_layers(2)]


@pytest.mark.parametrize("model", MODELS, ids=lambda m: m.name)
def test_prefill_and_decode_with_random_norms(model, cuda_ok):
    w = _random_norms(synth.make_model(model, 0), 11)
    prompt = synth.make_prompt(39, model.vocab).tolist()
    steps = 6
    max_seq = len(prompt) + steps
    tr, _, _ = oracle_trace(model, w, prompt, steps, max_seq)
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, max_seq)
    assert_within(compare(tr, *run_gpu(dec, model, tr)))


@pytest.mark.parametrize("model", [synth.TINY, synth.LLAMA8B.with_layers(2)],
                         ids=lambda m: m.name)
def test_batched_step_with_random_norms(model, cuda_ok):
    w = _random_norms(synth.make_model(model, 0), 12)
    _run_batch(model, w, [40, 71, 23], 3, 80)
