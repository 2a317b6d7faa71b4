"""The bytes-per-step model behind the bench's roofline."""
import os

import pytest

from persistent_megakernel_03_b200 import roofline, synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_pages_bandwidth_bound_example():
    # "LLMs in einen MegaKernel kompilieren ...": 16 GB at 1.6 TB/s -> 10 ms.
    with open(os.path.join(GOLDEN, "bandwidth_bound.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    for gb, tbps, ms in rows:
        assert roofline.bound_ms(float(gb) * 1e9, float(tbps) * 1e12) == pytest.approx(float(ms))


def test_llama8b_weight_bytes():
    # every bf16 parameter except the 128,255 embedding rows a step does not read
    m = synth.LLAMA8B
    assert roofline.weight_bytes(m) + m.hidden * 2 == 15_009_857_536
    assert roofline.weight_bytes(m) + m.vocab * m.hidden * 2 == 2 * m.n_params()


def test_qwen_tied_weight_bytes_equal_all_parameters():
    m = synth.QWEN05B
    assert roofline.weight_bytes(m) == 2 * m.n_params() == 988_065_536


def test_kv_bytes_per_token_and_long_context():
    m = synth.LLAMA8B
    assert roofline.kv_write_bytes(m) == 131_072
    # 32768 cached positions of K and V: exactly 4 GiB
    assert roofline.kv_read_bytes(m, 32767) == 4 * 2**30


def test_step_bytes_mean_of_the_39_plus_512_workload():
    m = synth.LLAMA8B
    mean = sum(roofline.step_bytes(m, [p]) for p in range(39, 39 + 512)) / 512
    assert mean == pytest.approx(15.05e9, rel=2e-3)
