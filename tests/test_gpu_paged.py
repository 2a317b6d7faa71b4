"""Paged KV cache and continuous batching against the oracle.

With mk_options.kv_page_tokens the cache is a pool of pages of that many
positions, assigned to a request slot through a block table
("LLM高速化勉強会資料" slides 15-17: PagedAttention; requests joining and
leaving a running batch).  The oracle keeps its own contiguous cache per
request: pages are only storage, so every request must still meet the
acceptance bar under teacher forcing.  Page tables here are shuffled, so
consecutive positions of a request sit in scattered, non-monotonic pages.
"""
import numpy as np
import pytest
import torch

from persistent_megakernel_03_b200 import binding, synth
from parity_util import assert_within, compare, oracle_trace

pytestmark = pytest.mark.gpu

PAGE = 64


def _shuffled_tables(dec, slots, n_pages_each, seed):
    pool = dec.kv_free_pages()
    perm = np.random.default_rng(seed).permutation(pool).tolist()
    for i, s in enumerate(slots):
        dec.kv_set_pages(s, perm[i * n_pages_each:(i + 1) * n_pages_each])


def _run(model, w, lens, steps, max_seq, slots, **kw):
    """Prefill every request into its slot (shuffled pages), then decode all
    of them together, teacher-forced; each request against its own oracle run."""
    n = len(lens)
    toks, offs = synth.make_packed_prompts(lens, model.vocab, seed=21)
    prompts = [toks[offs[r]:offs[r + 1]].tolist() for r in range(n)]
    traces = [oracle_trace(model, w, p, steps, max_seq)[0] for p in prompts]
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, max_seq,
                          max_batch=max(slots) + 1, kv_page_tokens=PAGE, **kw)
    _shuffled_tables(dec, slots, (max_seq + PAGE - 1) // PAGE, seed=22)
    V, H = model.vocab, model.hidden
    logits = torch.empty(n, V, device="cuda")
    ids = torch.empty(n, dtype=torch.int32, device="cuda")
    hidden = torch.empty(n, H, device="cuda")
    dec.prefill_slots(toks.to(torch.int32).cuda(), offs.tolist(), slots, logits, ids)
    dec.copy_hidden(hidden, n)
    torch.cuda.synchronize()
    got = [([logits[r].cpu().numpy().copy()], [hidden[r].cpu().numpy().copy()], [int(ids[r])])
           for r in range(n)]
    tok = torch.empty(n, dtype=torch.int32, device="cuda")
    for s in range(steps):
        tok.copy_(torch.tensor([tr.feed[s] for tr in traces], dtype=torch.int32))
        dec.decode_slots(tok, [lens[r] + s for r in range(n)], slots, logits, ids)
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


@pytest.mark.parametrize("mode", [binding.MODE_MEGAKERNEL, binding.MODE_PER_OP_GRAPH],
                         ids=["mk", "graph"])
def test_tiny_one_request_shuffled_pages(cuda_ok, mode):
    # 300 positions over 5 pages, split boundaries inside and across pages
    w = synth.make_model(synth.TINY, 31)
    _run(synth.TINY, w, [290], 8, 300, [0], mode=mode)


def test_tiny_batched_requests_shuffled_pages(cuda_ok):
    w = synth.make_model(synth.TINY, 32)
    _run(synth.TINY, w, [5, 130, 64, 257, 1, 70], 5, 300, [3, 0, 5, 1, 7, 2])


@pytest.mark.parametrize("n_req", [1, 3], ids=["one", "three"])
def test_llama_width_shuffled_pages(cuda_ok, n_req):
    model = synth.LLAMA8B.with_layers(2)
    w = synth.make_model(model, 33)
    lens = [300, 39, 129][:n_req]
    _run(model, w, lens, 3, 320, [2, 0, 1][:n_req])


def test_qwen_width_shuffled_pages(cuda_ok):
    model = synth.QWEN05B.with_layers(2)
    w = synth.make_model(model, 34)
    _run(model, w, [200, 65], 3, 260, [1, 0])


def test_continuous_batching_requests_join_and_leave(cuda_ok):
    """A starts alone; B joins (batched with A); A leaves and releases its
    pages; C joins in A's slot, on the pages A returned.  Every request is
    compared with the oracle running it alone."""
    model = synth.TINY
    w = synth.make_model(model, 35)
    max_seq = 200
    P = {"A": 70, "B": 33, "C": 90}
    toks, offs = synth.make_packed_prompts(list(P.values()), model.vocab, seed=36)
    prompt = {k: toks[offs[i]:offs[i + 1]] for i, k in enumerate(P)}
    tr = {k: oracle_trace(model, w, prompt[k].tolist(), 12, max_seq)[0] for k in P}
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, max_seq, max_batch=4,
                          kv_page_tokens=PAGE, kv_pool_pages=8)
    slot = {"A": 2, "B": 0, "C": 2}
    step = {k: 0 for k in P}                     # decode steps taken
    got = {k: [] for k in P}
    V = model.vocab

    def join(k):
        lg = torch.empty(1, V, device="cuda")
        dec.prefill_slots(prompt[k].to(torch.int32).cuda(), [0, P[k]], [slot[k]], lg, None)
        torch.cuda.synchronize()
        got[k].append(lg[0].cpu().numpy().copy())

    def decode(active):
        n = len(active)
        tok = torch.tensor([tr[k].feed[step[k]] for k in active], dtype=torch.int32).cuda()
        lg = torch.empty(n, V, device="cuda")
        dec.decode_slots(tok, [P[k] + step[k] for k in active], [slot[k] for k in active], lg, None)
        torch.cuda.synchronize()
        for r, k in enumerate(active):
            got[k].append(lg[r].cpu().numpy().copy())
            step[k] += 1

    join("A")
    for _ in range(3):
        decode(["A"])
    join("B")
    for _ in range(4):
        decode(["B", "A"])
    free_before = dec.kv_free_pages()
    dec.kv_release(slot["A"])                    # A finished: its pages go back
    assert dec.kv_free_pages() == free_before + 2    # 77 positions on 64-position pages
    join("C")                                    # C takes A's slot (and free pages)
    for _ in range(5):
        decode(["C", "B"])
    assert dec.status() == 0, dec.last_error()
    for k in P:
        for s, lg in enumerate(got[k]):
            err = float(np.abs(lg - tr[k].logits[s]).max())
            assert err <= 3e-2, (k, s, err)


def test_pool_exhaustion_is_reported_before_launch(cuda_ok):
    model = synth.TINY
    w = synth.make_model(model, 37)
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, 256, max_batch=2,
                          kv_page_tokens=PAGE, kv_pool_pages=3)
    toks = synth.make_prompt(130, model.vocab).to(torch.int32).cuda()
    dec.prefill_slots(toks, [0, 130], [0])       # 3 pages
    assert dec.kv_free_pages() == 0
    with pytest.raises(binding.MkError, match="OOM"):
        dec.prefill_slots(toks[:10], [0, 10], [1])
    assert dec.status() == 0                     # refused before any launch
    dec.kv_release(0)
    assert dec.kv_free_pages() == 3
    dec.prefill_slots(toks[:10], [0, 10], [1])
    assert dec.status() == 0 and dec.kv_pages(1)[0] >= 0
