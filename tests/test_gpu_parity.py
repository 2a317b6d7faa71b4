"""CUDA path vs the oracle, element by element, through the C-ABI."""
import numpy as np
import pytest
import torch

from persistent_megakernel_03_b200 import binding, synth
from parity_util import assert_within, compare, oracle_trace, run_gpu

pytestmark = pytest.mark.gpu

MODES = [binding.MODE_MEGAKERNEL, binding.MODE_PER_OP, binding.MODE_PER_OP_GRAPH]


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.TINY
    w = synth.make_model(cfg, 0)
    prompt = synth.make_prompt(16, cfg.vocab).tolist()
    tr, _, _ = oracle_trace(cfg, w, prompt, 16, 32)
    return cfg, w, tr


@pytest.mark.parametrize("mode", MODES, ids=["megakernel", "per_op", "per_op_graph"])
def test_tiny_teacher_forced(tiny, cuda_ok, mode):
    cfg, w, tr = tiny
    dec = binding.Decoder(cfg, {k: v.cuda() for k, v in w.items()}, 32, mode=mode)
    gl, gh, gi = run_gpu(dec, cfg, tr)
    assert_within(compare(tr, gl, gh, gi))


def test_megakernel_equals_per_op_bitwise(tiny, cuda_ok):
    cfg, w, tr = tiny
    wg = {k: v.cuda() for k, v in w.items()}
    outs = []
    for mode in MODES:
        dec = binding.Decoder(cfg, wg, 32, mode=mode)
        outs.append(run_gpu(dec, cfg, tr))
        dec.close()
    for o in outs[1:]:
        for a, b in zip(outs[0][0], o[0]):
            assert np.array_equal(a, b)


def test_tiny_kv_cache_matches_oracle(tiny, cuda_ok):
    # every position through the decode step (fp32 sums like the oracle's);
    # the tensor-core prefill's cache is checked in test_gpu_prefill.py
    cfg, w, tr = tiny
    dec = binding.Decoder(cfg, {k: v.cuda() for k, v in w.items()}, 32, prefill_steps=1)
    run_gpu(dec, cfg, tr)
    _, om, st = oracle_trace(cfg, w, tr.prompt, 16, 32)
    n = 32
    buf = torch.empty((n, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
    for l in range(cfg.n_layers):
        for g in range(cfg.n_kv_heads):
            for which in (0, 1):
                dec.copy_kv(0, l, g, which, n, buf)
                torch.cuda.synchronize()
                got = buf.float().cpu().numpy()
                want = st.kv(l, g, which, n)
                # bf16 values: equal, or one bf16 step apart where the fp32
                # inputs straddled a rounding boundary
                diff = np.abs(got - want)
                step = np.abs(want) * 2.0 ** -7 + 1e-30
                assert np.mean(diff == 0) > 0.98
                assert np.all(diff <= step * 1.01 + 1e-6)


@pytest.mark.parametrize("splits", [1, 3, 7, 40])
def test_tiny_attention_split_counts(tiny, cuda_ok, splits):
    cfg, w, tr = tiny
    dec = binding.Decoder(cfg, {k: v.cuda() for k, v in w.items()}, 32, attn_splits=splits)
    gl, gh, gi = run_gpu(dec, cfg, tr)
    assert_within(compare(tr, gl, gh, gi))


@pytest.fixture(scope="module")
def tiny_long():
    # 300-token prompt: the context spans several ring chunks of keys, so the
    # attention runs on several splits whose partials are merged
    cfg = synth.TINY
    w = synth.make_model(cfg, 5)
    prompt = synth.make_prompt(300, cfg.vocab, seed=6).tolist()
    tr, _, _ = oracle_trace(cfg, w, prompt, 6, 320)
    return cfg, w, tr


@pytest.mark.parametrize("splits", [1, 2, 3, 7])
def test_tiny_merged_splits(tiny_long, cuda_ok, splits):
    cfg, w, tr = tiny_long
    dec = binding.Decoder(cfg, {k: v.cuda() for k, v in w.items()}, 320, attn_splits=splits)
    gl, gh, gi = run_gpu(dec, cfg, tr)
    assert_within(compare(tr, gl, gh, gi))


@pytest.mark.parametrize("ctas", [1, 5, 64])
def test_tiny_fewer_ctas(tiny, cuda_ok, ctas):
    cfg, w, tr = tiny
    dec = binding.Decoder(cfg, {k: v.cuda() for k, v in w.items()}, 32, num_ctas=ctas)
    gl, gh, gi = run_gpu(dec, cfg, tr)
    assert_within(compare(tr, gl, gh, gi))


def test_last_position_and_single_token_prompt(cuda_ok):
    cfg = synth.TINY
    w = synth.make_model(cfg, 3)
    prompt = synth.make_prompt(1, cfg.vocab, seed=5).tolist()
    max_seq = 9
    tr, _, _ = oracle_trace(cfg, w, prompt, max_seq - 1, max_seq)
    dec = binding.Decoder(cfg, {k: v.cuda() for k, v in w.items()}, max_seq)
    gl, gh, gi = run_gpu(dec, cfg, tr)
    assert_within(compare(tr, gl, gh, gi))
    tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(binding.MkError) as e:
        dec.decode(tok, [max_seq])
    assert e.value.code == -5


def test_determinism_over_repeats(tiny, cuda_ok):
    cfg, w, tr = tiny
    wg = {k: v.cuda() for k, v in w.items()}
    first = None
    for _ in range(5):
        dec = binding.Decoder(cfg, wg, 32)
        out = run_gpu(dec, cfg, tr)
        dec.close()
        if first is None:
            first = out
        else:
            assert all(np.array_equal(a, b) for a, b in zip(first[0], out[0]))


def test_host_entry_point_matches_device_path(tiny, cuda_ok):
    cfg, w, tr = tiny
    wg = {k: v.cuda() for k, v in w.items()}
    a = binding.Decoder(cfg, wg, 32)
    gl, gh, gi = run_gpu(a, cfg, tr)
    b = binding.Decoder(cfg, wg, 32)
    toks = torch.tensor(tr.prompt, dtype=torch.int32, device="cuda")
    b.prefill(toks, [0, len(tr.prompt)])
    host_ids = [b.decode_host([t], [len(tr.prompt) + s])[0] for s, t in enumerate(tr.feed)]
    assert host_ids == gi[1:]


def test_token_out_of_range_is_reported_not_faulted(tiny, cuda_ok):
    cfg, w, tr = tiny
    dec = binding.Decoder(cfg, {k: v.cuda() for k, v in w.items()}, 32)
    tok = torch.tensor([cfg.vocab + 5], dtype=torch.int32, device="cuda")
    dec.decode(tok, [0])
    assert dec.status() == -8
    with pytest.raises(binding.MkError):
        dec.decode(tok, [1])


def test_host_token_out_of_range_is_rejected_before_launch(tiny, cuda_ok):
    cfg, w, tr = tiny
    dec = binding.Decoder(cfg, {k: v.cuda() for k, v in w.items()}, 32)
    for bad in (cfg.vocab, -1):
        with pytest.raises(binding.MkError, match="TOKEN_RANGE"):
            dec.decode_host([bad], [0])
    assert dec.status() == 0  # an argument error does not poison the context
    out = dec.decode_host([0], [0])
    assert 0 <= out[0] < cfg.vocab and dec.status() == 0


WIDE = [
    synth.QWEN05B.with_layers(2),
    synth.LLAMA8B.with_layers(2),
]


@pytest.mark.parametrize("model", WIDE, ids=lambda m: m.name)
def test_wide_shapes_two_layers(model, cuda_ok):
    w = synth.make_model(model, 0)
    prompt = synth.make_prompt(39, model.vocab).tolist()
    steps = 8
    tr, _, _ = oracle_trace(model, w, prompt, steps, 39 + steps)
    dec = binding.Decoder(model, {k: v.cuda() for k, v in w.items()}, 39 + steps)
    gl, gh, gi = run_gpu(dec, model, tr)
    assert_within(compare(tr, gl, gh, gi))


def test_qwen05b_full_depth(cuda_ok):
    model = synth.QWEN05B
    w = synth.make_model(model, 0, device="cuda")
    w_cpu = {k: v.cpu() for k, v in w.items()}
    prompt = synth.make_prompt(39, model.vocab).tolist()
    steps = 6
    tr, _, _ = oracle_trace(model, w_cpu, prompt, steps, 600)
    dec = binding.Decoder(model, w, 600)
    gl, gh, gi = run_gpu(dec, model, tr)
    assert_within(compare(tr, gl, gh, gi))
