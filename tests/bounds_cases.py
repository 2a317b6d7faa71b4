"""Decode cases run against the debug-bounds build of the library (loaded
through MK_LIBRARY by tests/test_gpu_debug_bounds.py, in a process of its
own): every task checks the indices of its accesses, and a violation would
end the run with MK_ERR_BOUNDS.  Each case also meets the oracle."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import torch  # noqa: E402

import oracle  # noqa: E402
from persistent_megakernel_03_b200 import binding, synth  # noqa: E402
from parity_util import assert_within, compare, oracle_trace, run_gpu  # noqa: E402
from test_gpu_batch import _run_batch  # noqa: E402
from test_gpu_paged import _run as _run_paged  # noqa: E402


def single(model, w, P, steps, **kw):
    prompt = synth.make_prompt(P, model.vocab, seed=40).tolist()
    tr, _, _ = oracle_trace(model, w, prompt, steps, P + steps)
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, P + steps, **kw)
    gl, gh, gi = run_gpu(dec, model, tr)
    assert_within(compare(tr, gl, gh, gi))
    assert dec.status() == 0, dec.last_error()
    dec.close()


def main():
    assert binding.lib().mk_build_flags() & 1, "not the debug-bounds build"
    tiny = synth.TINY
    w = synth.make_model(tiny, 41)
    for mode in (binding.MODE_MEGAKERNEL, binding.MODE_PER_OP, binding.MODE_PER_OP_GRAPH):
        single(tiny, w, 300, 6, mode=mode)            # several key splits, merges
    single(tiny, w, 1, 4)                              # a single-key context
    _run_batch(tiny, w, [5, 17, 90, 1], 4, 100)       # the batched step
    _run_paged(tiny, w, [130, 5, 64], 4, 140, [2, 0, 1])   # shuffled pages
    raw = synth.make_model(tiny, 42)                   # fp8 weights from raw bf16
    prompt = synth.make_prompt(40, tiny.vocab, seed=43).tolist()
    tr, _, _ = oracle_trace(tiny, oracle.quantize_fp8_model(tiny, raw), prompt, 4, 44)
    dec = binding.Decoder(tiny, {k: v.cuda() for k, v in raw.items()}, 44, weight_format=1)
    assert_within(compare(tr, *run_gpu(dec, tiny, tr)))
    dec.close()
    llama = synth.LLAMA8B.with_layers(2)
    single(llama, synth.make_model(llama, 44), 70, 3)  # Llama widths, split boundary at 64
    print("bounds cases ok")


if __name__ == "__main__":
    main()
