"""The device-resident decode loop (mk_decode_steps): n greedy steps in one
persistent launch, each step's argmax feeding the next step's embedding.

It must give exactly what n calls of mk_decode_step give (same task bodies,
same order of every sum), and its last logits must meet the oracle bar when
the oracle is fed the same ids."""
import numpy as np
import pytest
import torch

import oracle
from persistent_megakernel_03_b200 import binding, synth
from parity_util import LOGITS_ATOL

pytestmark = pytest.mark.gpu


def _prefilled(model, w, prompt, max_seq):
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, max_seq)
    ids = torch.empty(1, dtype=torch.int32, device="cuda")
    dec.prefill(torch.tensor(prompt, dtype=torch.int32, device="cuda"), [0, len(prompt)], None, ids)
    torch.cuda.synchronize()
    return dec, ids


@pytest.mark.parametrize("model,P,n", [
    (synth.TINY, 16, 12),
    (synth.LLAMA8B.with_layers(2), 39, 8),
    (synth.QWEN05B.with_layers(2), 39, 8),
], ids=["tiny", "llama-2l", "qwen-2l"])
def test_loop_equals_single_steps(cuda_ok, model, P, n):
    w = synth.make_model(model, 3)
    prompt = synth.make_prompt(P, model.vocab, seed=4).tolist()
    V = model.vocab
    # n single launches
    a, ids_a = _prefilled(model, w, prompt, P + n + 1)
    single, lg_a = [], torch.empty(V, device="cuda")
    tok = ids_a.clone()
    nxt = torch.empty(1, dtype=torch.int32, device="cuda")
    for s in range(n):
        a.decode(tok, [P + s], lg_a if s == n - 1 else None, nxt)
        torch.cuda.synchronize()
        single.append(int(nxt.item()))
        tok.copy_(nxt)
    # one launch of n steps
    b, ids_b = _prefilled(model, w, prompt, P + n + 1)
    seq = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    lg_b = torch.empty(V, device="cuda")
    b.decode_steps(ids_b, P, n, seq, lg_b)
    torch.cuda.synchronize()
    assert b.status() == 0, b.last_error()
    assert seq.tolist() == single
    assert torch.equal(lg_a, lg_b)
    # the oracle, fed the same ids, agrees on the last logits
    om = oracle.OracleModel(model, w)
    st = om.new_state(P + n + 1)
    for p, t in enumerate(prompt):
        first, _, _ = om.decode(st, t, p, want_logits=False)
    feed = [int(ids_b.item())] + single[:-1]
    for s, t in enumerate(feed):
        _, lg, _ = om.decode(st, t, P + s, want_logits=(s == n - 1))
    assert float(np.abs(lg_b.cpu().numpy() - lg).max()) <= LOGITS_ATOL


def test_loop_rejects_positions_past_the_cache(cuda_ok):
    model = synth.TINY
    w = synth.make_model(model, 0)
    dec, ids = _prefilled(model, w, synth.make_prompt(8, model.vocab).tolist(), 12)
    seq = torch.empty(8, dtype=torch.int32, device="cuda")
    with pytest.raises(binding.MkError) as e:
        dec.decode_steps(ids, 8, 8, seq)
    assert e.value.code == -5
