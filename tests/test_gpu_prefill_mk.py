"""The prefill as one persistent kernel (the default tensor-core prefill).

Every operator of every layer of a block of prompt positions is a task of one
launch ("LLMs in einen MegaKernel kompilieren ...", "Part 1. Compiler":
operators refined into SM-sized tasks linked by events per data tile); the
arithmetic is the per-operator tensor-core prefill's (three bf16 parts of the
fp32 activation, three tensor-memory accumulators), so the cache it leaves
must equal that path's up to the order of the fp32 additions, and what
follows must match the oracle at the decode bar.  Cases: several 128-position
tiles with ragged tails, single-token prompts (no prefill positions), a
2048-position block boundary, several requests per block (attention runs cut
at request boundaries), a QKV bias (the Qwen shape), paged KV slots.
"""
import numpy as np
import pytest
import torch

from persistent_megakernel_03_b200 import binding, synth
from parity_util import assert_within, compare, oracle_trace, run_gpu
from test_gpu_batch import _run_batch
from test_gpu_prefill import _cache

pytestmark = pytest.mark.gpu

CACHE_REL_L2 = 2e-3


def _prefill(model, w, lens, **kw):
    toks, offs = synth.make_packed_prompts(lens, model.vocab, seed=11)
    dec = binding.Decoder(model, w, max(lens) + 2, max_batch=len(lens), **kw)
    logits = torch.empty(len(lens), model.vocab, device="cuda")
    ids = torch.empty(len(lens), dtype=torch.int32, device="cuda")
    dec.prefill(toks.to(torch.int32).cuda(), offs.tolist(), logits, ids)
    torch.cuda.synchronize()
    assert dec.status() == 0, dec.last_error()
    return dec, logits.cpu().numpy(), ids.cpu().numpy()


@pytest.mark.parametrize("model,lens", [
    (synth.TINY, [300, 1, 129, 2100]),
    (synth.QWEN05B.with_layers(2), [200, 77, 1]),
    (synth.LLAMA8B.with_layers(2), [260, 5]),
], ids=["tiny", "qwen-2l", "llama-2l"])
def test_persistent_prefill_matches_per_operator_prefill(cuda_ok, model, lens):
    w = {k: v.cuda() for k, v in synth.make_model(model, 4).items()}
    a, la, _ = _prefill(model, w, lens)
    b, lb, _ = _prefill(model, w, lens, prefill_per_operator=1)
    for x, y in zip(_cache(a, model, lens), _cache(b, model, lens)):
        assert np.linalg.norm(x - y) <= CACHE_REL_L2 * np.linalg.norm(y)
        assert np.abs(x - y).max() <= 0.02 * np.abs(y).max()
    np.testing.assert_allclose(la, lb, atol=5e-3, rtol=0)


def test_persistent_prefill_then_decode_matches_oracle(cuda_ok):
    model = synth.QWEN05B.with_layers(2)
    w = synth.make_model(model, 6)
    prompt = synth.make_prompt(333, model.vocab, seed=8).tolist()
    tr, _, _ = oracle_trace(model, w, prompt, 4, 340)
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, 340)
    gl, gh, gi = run_gpu(dec, model, tr)
    assert_within(compare(tr, gl, gh, gi))


def test_persistent_prefill_past_one_block_against_the_oracles_prefill(cuda_ok):
    model = synth.LLAMA8B.with_layers(2)
    w = synth.make_model(model, 3, device="cuda")
    w_cpu = {k: v.cpu() for k, v in w.items()}
    P, steps = 2100, 3
    prompt = synth.make_prompt(P, model.vocab, seed=5).tolist()
    tr, om, st = oracle_trace(model, w_cpu, prompt, steps, P + steps)
    dec = binding.Decoder(model, w, P + steps)
    gl, gh, gi = run_gpu(dec, model, tr)
    assert_within(compare(tr, gl, gh, gi))
    for positions in (np.arange(0, 130), np.arange(2040, 2056), np.arange(2056, P)):
        for layer in range(model.n_layers):
            for g in (0, model.n_kv_heads - 1):
                for which in (0, 1):
                    got = torch.empty(P, model.head_dim, dtype=torch.bfloat16, device="cuda")
                    dec.copy_kv(0, layer, g, which, P, got)
                    torch.cuda.synchronize()
                    got = got.float().cpu().numpy()[positions]
                    want = st.kv(layer, g, which, P)[positions]
                    rel = float(np.linalg.norm(got - want) / np.linalg.norm(want))
                    assert rel <= CACHE_REL_L2, (layer, g, which, positions[0], rel)


def test_persistent_prefill_several_requests_paged(cuda_ok):
    # eight requests in one block (attention runs end at request boundaries and
    # at 128-position tiles), the cache in 64-position pages
    w = synth.make_model(synth.TINY, 7)
    _run_batch(synth.TINY, w, [5, 170, 9, 300, 1, 129, 23, 64], 4, 310,
               kv_page_tokens=64)


def test_persistent_prefill_eight_requests_at_llama_widths(cuda_ok):
    model = synth.LLAMA8B.with_layers(2)
    w = synth.make_model(model, 4)
    _run_batch(model, w, [40, 700, 129, 1, 256, 333, 90, 517], 3, 705)


def test_prefill_timeline_records_every_task_in_dependency_order(cuda_ok):
    # mk_set_prefill_trace: one record per task of the first block, the
    # timestamps of a task in order, every tile and layer present, sixteen
    # elementwise tasks per tile and stage, attention after its keys' RoPE
    model = synth.LLAMA8B.with_layers(2)
    w = {k: v.cuda() for k, v in synth.make_model(model, 2).items()}
    P = 300
    dec = binding.Decoder(model, w, P + 2)
    tr = torch.zeros(4 * 100000, dtype=torch.int64, device="cuda")
    dec.set_prefill_trace(tr)
    toks = synth.make_prompt(P, model.vocab, seed=3).to(torch.int32).cuda()
    dec.prefill(toks, [0, P], None, None)
    torch.cuda.synchronize()
    assert dec.status() == 0, dec.last_error()
    dec.set_prefill_trace(None)
    a = tr.view(-1, 4).cpu().numpy().astype(np.uint64)
    a = a[a[:, 2] != 0]
    assert len(a) > 0
    assert np.all(a[:, 0] <= a[:, 1]) and np.all(a[:, 1] <= a[:, 2])
    d = a[:, 3]
    kind = (d >> 16) & 15
    layer = (d >> 24) & 255
    tile = (d >> 32) & 0xFFFF
    cta = d & 0xFFFF
    assert int(cta.max()) < torch.cuda.get_device_properties(0).multi_processor_count
    n_tiles = (P + 127) // 128  # every position, the last one included
    assert set(int(t) for t in tile) == set(range(n_tiles))
    # the layers, then the LM head (layer index n_layers) of the last position's tile
    assert set(int(x) for x in layer) == set(range(model.n_layers + 1))
    lm = (kind == 1) & (layer == model.n_layers)
    assert int(np.sum(lm)) == (model.vocab + 127) // 128
    assert set(int(t) for t in tile[lm]) == {(P - 1) // 128}
    # per layer: 16 tasks per tile for each elementwise stage present
    for l in range(model.n_layers):
        for k, stages in ((2, 1), (4, 1), (5, 1), (6, 1)):
            assert int(np.sum((kind == k) & (layer == l))) == 16 * n_tiles * stages
    # an attention task of tile n starts only after every RoPE task of tiles
    # <= n has started (it waits for their completion signals)
    for l in range(model.n_layers):
        rope_start = {n: a[(kind == 2) & (layer == l) & (tile == n), 1].max() for n in range(n_tiles)}
        for n in range(n_tiles):
            att = a[(kind == 3) & (layer == l) & (tile == n)]
            assert len(att) > 0
            assert att[:, 1].min() >= max(rope_start[m] for m in range(n + 1))


@pytest.mark.parametrize("P,folded", [(129, False), (130, True), (39, True)])
def test_last_position_folds_only_into_room_in_the_final_tile(cuda_ok, P, folded):
    # a prompt whose other positions fill the final 128-position tile exactly
    # (P - 1 = 128) leaves its last position to the decode step: no LM-head
    # tasks in the kernel; one more position (or a short prompt) folds it in.
    # Either way the greedy id and logits are the per-operator path's.
    model = synth.LLAMA8B.with_layers(2)
    w = {k: v.cuda() for k, v in synth.make_model(model, 2).items()}
    toks = synth.make_prompt(P, model.vocab, seed=9).to(torch.int32).cuda()
    dec = binding.Decoder(model, w, P + 2)
    tr = torch.zeros(4 * 60000, dtype=torch.int64, device="cuda")
    dec.set_prefill_trace(tr)
    lg = torch.empty(1, model.vocab, device="cuda")
    ids = torch.empty(1, dtype=torch.int32, device="cuda")
    dec.prefill(toks, [0, P], lg, ids)
    torch.cuda.synchronize()
    assert dec.status() == 0, dec.last_error()
    a = tr.view(-1, 4).cpu().numpy().astype(np.uint64)
    a = a[a[:, 2] != 0]
    layer = (a[:, 3] >> 24) & 255
    kind = (a[:, 3] >> 16) & 15
    assert bool(np.any((kind == 1) & (layer == model.n_layers))) == folded
    ref = binding.Decoder(model, w, P + 2, prefill_per_operator=1)
    lg2 = torch.empty(1, model.vocab, device="cuda")
    ids2 = torch.empty(1, dtype=torch.int32, device="cuda")
    ref.prefill(toks, [0, P], lg2, ids2)
    torch.cuda.synchronize()
    np.testing.assert_allclose(lg.cpu().numpy(), lg2.cpu().numpy(), atol=5e-3, rtol=0)
    l0 = lg2.cpu().numpy()[0]
    top = np.sort(l0)[-2:]
    if top[1] - top[0] >= 0.1:
        assert int(ids[0]) == int(ids2[0])
