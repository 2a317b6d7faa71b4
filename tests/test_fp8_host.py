"""The fp8 weight rule of the oracle (orc_quantize_fp8_rows): every weight of
a row becomes e4m3(w / 2^k) * 2^k, k the smallest integer with
max|row| <= 448 * 2^k ("LLM高速化勉強会資料" slide 33: fewer bits per
parameter with block-wise scaling; here a block is one row).  Pinned against
the e4m3 format's definition (hand-worked grid points, ties and subnormals)
and against torch's own float8_e4m3fn conversion, an independent
implementation of the same rounding."""
import numpy as np
import torch

import oracle
from persistent_megakernel_03_b200 import roofline, synth


def test_hand_worked_grid_points_ties_and_subnormals():
    # one row, max 448 -> k = 0, so the values are the e4m3 grid itself:
    #   0.1 lies in [2^-4, 2^-3), spacing 2^-7: 0.1 / 2^-7 = 12.8 -> 13 -> 0.1015625
    #   17 lies in [16, 32), spacing 2: 8.5 is a tie -> even 8 -> 16
    #   19: 9.5 is a tie -> even 10 -> 20
    #   3 * 2^-9 is a subnormal, kept exactly
    #   2^-10 is half the smallest subnormal: a tie between 0 and 2^-9 -> 0
    #   -1.5 * 2^-9: a tie between 1 and 2 steps -> 2 steps = -2^-8
    row = [448, 1, 0.1, -17, 19, 3 * 2**-9, 2**-10, -1.5 * 2**-9]
    q, k = oracle.quantize_fp8_rows(torch.tensor([row], dtype=torch.bfloat16))
    want = [448, 1, 0.1015625, -16, 20, 3 * 2**-9, 0, -2**-8]
    assert k.tolist() == [0]
    assert q.float()[0].tolist() == want
    # max 900: k = 2 (448 * 2 = 896 < 900 <= 1792); 900 / 4 = 225 in [128, 256),
    # spacing 16: 14.06 -> 14 -> 224 * 4 = 896; a row of zeros keeps k = 0
    q, k = oracle.quantize_fp8_rows(torch.tensor([[900, 3, 0.5, -0.25], [0, 0, 0, 0]],
                                                 dtype=torch.bfloat16))
    assert k.tolist() == [2, 0]
    assert q.float().tolist() == [[896, 3, 0.5, -0.25], [0, 0, 0, 0]]


def _random_rows():
    g = torch.Generator("cpu").manual_seed(0)
    w = (torch.randn(64, 96, generator=g) * 0.02).to(torch.bfloat16)
    w[3] = 0                                    # a row of zeros
    w[5, 7] = 3.0                               # a row with a large entry
    w[9] *= 2.0**-20                            # tiny values: deep negative exponents
    return w


def test_rows_equal_torch_e4m3_conversion_at_the_smallest_power_of_two_scale():
    w = _random_rows()
    q, k = oracle.quantize_fp8_rows(w)
    s = torch.exp2(torch.from_numpy(k).double()).unsqueeze(1)
    mx = w.double().abs().amax(dim=1)
    nz = mx > 0
    # the scale: smallest power of two that fits the row's maximum
    assert torch.all(mx[nz] <= 448 * s[nz, 0]) and torch.all(mx[nz] > 224 * s[nz, 0])
    # torch's own RNE conversion to float8_e4m3fn of w / 2^k, back times 2^k
    want = ((w.double() / s).float().to(torch.float8_e4m3fn).double() * s).to(torch.bfloat16)
    assert torch.equal(q, want)
    codes = q.double() / s
    assert torch.equal(codes.float().to(torch.float8_e4m3fn).double(), codes)   # exact e4m3
    assert codes.abs().max() <= 448
    assert torch.all(q[3] == 0)


def test_quantization_is_a_fixed_point_and_close():
    w = synth.make_model(synth.TINY, 0)
    q = oracle.quantize_fp8_model(synth.TINY, w)
    for key in ("layers.0.wq", "layers.1.w_down", "lm_head"):
        assert torch.equal(oracle.quantize_fp8_rows(q[key])[0], q[key])
        rel = (q[key].float() - w[key].float()).norm() / w[key].float().norm()
        assert rel < 0.04                        # e4m3: 3 significand bits
    assert torch.equal(q["embed"], w["embed"])   # untied: the embedding stays bf16
    assert torch.equal(q["layers.0.attn_norm"], w["layers.0.attn_norm"])
    qt = oracle.quantize_fp8_model(synth.QWEN05B.with_layers(1), synth.make_model(
        synth.QWEN05B.with_layers(1), 0))
    assert torch.equal(oracle.quantize_fp8_rows(qt["embed"])[0], qt["embed"])  # tied: quantized


def test_fp8_weight_bytes_halve_the_matrices():
    m = synth.LLAMA8B
    b16, b8 = roofline.weight_bytes(m, 2), roofline.weight_bytes(m, 1)
    rows = m.n_layers * (m.q_dim + 2 * m.kv_dim + m.hidden + 2 * m.ffn + m.hidden) + m.vocab
    vec = 2 * (m.n_layers * 2 * m.hidden + m.hidden)
    assert b16 - vec == 2 * (b8 - vec - 4 * rows)
