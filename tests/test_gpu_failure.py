"""Failure detection on the GPU without a fault: a task's event wait is made
unreachable from the host (mk_inject_stall), the megakernel's bounded waits
must end the launch with MK_ERR_TIMEOUT, mk_status must report it and poison
the context, and the CUDA context must stay usable for a new decoder."""
import time

import pytest
import torch

from persistent_megakernel_03_b200 import binding, synth

pytestmark = pytest.mark.gpu

MK_ERR_INVALID_ARG, MK_ERR_TIMEOUT, MK_ERR_NOT_RESIDENT = -1, -4, -6
TIMEOUT_MS = 100


def _prefilled(cfg, w, prompt):
    dec = binding.Decoder(cfg, w, 32, timeout_ms=TIMEOUT_MS)
    toks = torch.tensor(prompt, dtype=torch.int32, device="cuda")
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    dec.prefill(toks, [0, len(prompt)], None, ids)
    assert dec.status() == 0, dec.last_error()
    return dec, ids


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.TINY
    w = {k: v.cuda() for k, v in synth.make_model(cfg, 0).items()}
    return cfg, w, synth.make_prompt(8, cfg.vocab).tolist()


def _healthy_afterwards(cfg, w, prompt, ids_before):
    # a new context on the same device decodes as before the stall
    torch.cuda.synchronize()
    dec, ids = _prefilled(cfg, w, prompt)
    assert int(ids[0]) == int(ids_before[0])
    dec.decode(ids, [len(prompt)])
    assert dec.status() == 0, dec.last_error()
    dec.close()


def test_stalled_event_times_out_and_poisons(tiny, cuda_ok):
    cfg, w, prompt = tiny
    dec, ids = _prefilled(cfg, w, prompt)
    ids_before = ids.clone()
    dec.inject_stall(-1)
    t0 = time.monotonic()
    dec.decode(ids, [len(prompt)])
    assert dec.status() == MK_ERR_TIMEOUT
    elapsed = time.monotonic() - t0
    assert "timed out" in dec.last_error()
    assert elapsed < 5.0  # the limit is 100 ms per wait
    with pytest.raises(binding.MkError):  # poisoned
        dec.decode(ids, [len(prompt) + 1])
    dec.close()
    _healthy_afterwards(cfg, w, prompt, ids_before)


def test_stall_inside_the_device_loop_times_out(tiny, cuda_ok):
    cfg, w, prompt = tiny
    dec, ids = _prefilled(cfg, w, prompt)
    ids_before = ids.clone()
    # a task of the last layer: the loop's first step runs up to it
    n_tasks = len(dec_plan_tasks(cfg))
    dec.inject_stall(n_tasks - 1)
    seq = torch.zeros(4, dtype=torch.int32, device="cuda")
    dec.decode_steps(ids, len(prompt), 4, seq)
    assert dec.status() == MK_ERR_TIMEOUT
    dec.close()
    _healthy_afterwards(cfg, w, prompt, ids_before)


def test_bad_stall_index_is_an_argument_error(tiny, cuda_ok):
    cfg, w, prompt = tiny
    dec, ids = _prefilled(cfg, w, prompt)
    with pytest.raises(binding.MkError) as e:
        dec.inject_stall(10 ** 7)
    assert "INVALID_ARG" in str(e.value)
    # nothing was changed: the context still decodes
    dec.decode(ids, [len(prompt)])
    assert dec.status() == 0, dec.last_error()
    dec.close()


def dec_plan_tasks(cfg):
    """The task table of a context with the default options on this device
    (the same plan mk_create builds)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return binding.Plan(cfg, 32, sms).tasks()


@pytest.mark.parametrize("task", [-1, 0, 500])
def test_stalled_prefill_task_times_out_and_poisons(cuda_ok, task):
    # the persistent prefill: one task of the first block's graph can never
    # see its event; every CTA's bounded wait must end the launch, the call
    # must return MK_ERR_TIMEOUT within the limit, and the device must stay
    # usable.  Task -1 is the last waiting task (layer L-1), task 0 the first
    # elementwise task (no wait: refused), 500 a GEMM tile of layer 0.
    cfg = synth.LLAMA8B.with_layers(2)
    w = {k: v.cuda() for k, v in synth.make_model(cfg, 1).items()}
    prompt = synth.make_prompt(300, cfg.vocab, seed=4)
    toks = prompt.to(torch.int32).cuda()
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = binding.Decoder(cfg, w, 310, timeout_ms=TIMEOUT_MS)
    ref.prefill(toks, [0, 300], None, ids)
    assert ref.status() == 0, ref.last_error()
    want = int(ids[0])
    ref.close()
    dec = binding.Decoder(cfg, w, 310, timeout_ms=TIMEOUT_MS)
    dec.inject_prefill_stall(task)
    t0 = time.monotonic()
    with pytest.raises(binding.MkError) as err:
        dec.prefill(toks, [0, 300], None, ids)
    elapsed = time.monotonic() - t0
    if task == 0:
        assert err.value.code == MK_ERR_INVALID_ARG or "no such task" in str(err.value)
    else:
        assert err.value.code == MK_ERR_TIMEOUT, str(err.value)
        assert "timed out" in str(err.value)
        assert elapsed < 5.0  # 2 x 100 ms per wait
    with pytest.raises(binding.MkError):  # poisoned
        dec.prefill(toks, [0, 300], None, ids)
    dec.close()
    torch.cuda.synchronize()
    again = binding.Decoder(cfg, w, 310, timeout_ms=TIMEOUT_MS)
    ids.zero_()
    again.prefill(toks, [0, 300], None, ids)
    assert again.status() == 0, again.last_error()
    assert int(ids[0]) == want
    again.close()


def test_more_ctas_than_can_be_co_resident_is_refused_before_any_launch(tiny, cuda_ok):
    # the persistent kernel needs every CTA resident at once: a request for
    # more CTAs than the device holds is refused by mk_create (no launch), and
    # the device stays usable
    cfg, w, prompt = tiny
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    with pytest.raises(binding.MkError) as e:
        binding.Decoder(cfg, w, 32, num_ctas=4 * sms)
    assert e.value.code == MK_ERR_NOT_RESIDENT
    assert "co-resident" in str(e.value)
    dec, ids = _prefilled(cfg, w, prompt)
    dec.decode(ids, [len(prompt)])
    assert dec.status() == 0, dec.last_error()
    dec.close()
