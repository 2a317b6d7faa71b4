"""Several requests per step (the 8-request workload's shape) against the oracle.

Requests of different prompt lengths are packed as one flat token sequence
with offsets, prefilled together, then decoded together for a few steps with
the oracle's tokens fed to every request (teacher forcing).  The oracle runs
each request on its own cache; every request's logits, residual stream and
greedy id must meet the acceptance bar at every step, and no request may see
another's keys.
"""
import numpy as np
import pytest
import torch

from persistent_megakernel_03_b200 import binding, synth
from parity_util import assert_within, compare, oracle_trace

pytestmark = pytest.mark.gpu


def _run_batch(model, w, lens, steps, max_seq, seed=1, **kw):
    toks, offs = synth.make_packed_prompts(lens, model.vocab, seed=seed)
    prompts = [toks[offs[r]:offs[r + 1]].tolist() for r in range(len(lens))]
    traces = [oracle_trace(model, w, p, steps, max_seq)[0] for p in prompts]
    n = len(lens)
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, max_seq, max_batch=n, **kw)
    V, H = model.vocab, model.hidden
    logits = torch.empty(n, V, device="cuda")
    ids = torch.empty(n, dtype=torch.int32, device="cuda")
    hidden = torch.empty(n, H, device="cuda")
    dec.prefill(toks.to(torch.int32).cuda(), offs.tolist(), logits, ids)
    dec.copy_hidden(hidden, n)
    torch.cuda.synchronize()
    got = [([logits[r].cpu().numpy().copy()], [hidden[r].cpu().numpy().copy()], [int(ids[r])])
           for r in range(n)]
    tok = torch.empty(n, dtype=torch.int32, device="cuda")
    for s in range(steps):
        tok.copy_(torch.tensor([tr.feed[s] for tr in traces], dtype=torch.int32))
        dec.decode(tok, [lens[r] + s for r in range(n)], logits, ids)
        dec.copy_hidden(hidden, n)
        torch.cuda.synchronize()
        for r in range(n):
            got[r][0].append(logits[r].cpu().numpy().copy())
            got[r][1].append(hidden[r].cpu().numpy().copy())
            got[r][2].append(int(ids[r]))
    assert dec.status() == 0, dec.last_error()
    for r in range(n):
        assert_within(compare(traces[r], *got[r]))
    return dec


@pytest.mark.parametrize("sequential", [0, 1], ids=["batched", "sequential"])
def test_tiny_eight_requests(cuda_ok, sequential):
    # batched: one step streams each weight matrix once (tensor-core GEMMs over
    # the requests); sequential: the requests run through the megakernel in turn
    w = synth.make_model(synth.TINY, 7)
    _run_batch(synth.TINY, w, [5, 17, 9, 30, 1, 12, 23, 8], 6, 40, batch_sequential=sequential)


def test_tiny_long_contexts_batched(cuda_ok):
    # contexts past 256 keys: several attention splits per request and KV head
    w = synth.make_model(synth.TINY, 9)
    _run_batch(synth.TINY, w, [700, 40, 333, 1024], 4, 1030)


def test_tiny_eight_requests_per_op_graph(cuda_ok):
    w = synth.make_model(synth.TINY, 7)
    _run_batch(synth.TINY, w, [5, 17, 9, 30, 1, 12, 23, 8], 4, 40,
               mode=binding.MODE_PER_OP_GRAPH)


def test_fewer_requests_than_the_batch(cuda_ok):
    # a context made for 8 requests decodes 3 of them
    model = synth.TINY
    w = synth.make_model(model, 8)
    lens = [11, 3, 20]
    toks, offs = synth.make_packed_prompts(lens, model.vocab, seed=3)
    traces = [oracle_trace(model, w, toks[offs[r]:offs[r + 1]].tolist(), 3, 32)[0]
              for r in range(3)]
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, 32, max_batch=8)
    ids = torch.empty(3, dtype=torch.int32, device="cuda")
    dec.prefill(toks.to(torch.int32).cuda(), offs.tolist(), None, ids)
    tok = torch.empty(3, dtype=torch.int32, device="cuda")
    for s in range(3):
        tok.copy_(torch.tensor([tr.feed[s] for tr in traces], dtype=torch.int32))
        dec.decode(tok, [lens[r] + s for r in range(3)], None, ids)
        torch.cuda.synchronize()
        for r in range(3):
            if traces[r].logits[s + 1] is not None:
                lg = traces[r].logits[s + 1]
                top2 = np.partition(lg, -2)[-2:]
                if top2[1] - top2[0] >= 0.1:
                    assert int(ids[r]) == traces[r].ids[s + 1]
    assert dec.status() == 0


@pytest.mark.parametrize("model", [synth.QWEN05B.with_layers(2), synth.LLAMA8B.with_layers(2)],
                         ids=lambda m: m.name)
def test_wide_shapes_three_requests(model, cuda_ok):
    w = synth.make_model(model, 2)
    _run_batch(model, w, [39, 7, 300], 3, 310)
