"""Host side of the fp8 weight option: the row quantization that defines the
fp8 model (every weight e4m3 code * 2^k, one k per row) -- the weights both
the oracle and the fp8 decode path use."""
import torch

from persistent_megakernel_03_b200 import roofline, synth


def test_quantized_rows_are_e4m3_codes_times_a_row_power_of_two():
    g = torch.Generator("cpu").manual_seed(0)
    w = (torch.randn(64, 96, generator=g) * 0.02).to(torch.bfloat16)
    w[3] = 0                                    # a row of zeros
    w[5, 7] = 3.0                               # a row with a large entry
    q = synth.quantize_fp8_rows(w)
    k = synth.fp8_row_scale_exponents(q.float())
    s = torch.exp2(k).unsqueeze(1)
    codes = q.float() / s
    assert torch.equal(codes.to(torch.float8_e4m3fn).float(), codes)   # exact e4m3 values
    assert codes.abs().max() <= 448
    assert torch.all(q[3] == 0)
    # the scale is the smallest power of two that fits the row's maximum
    mx = q.float().abs().amax(dim=1)
    nz = mx > 0
    assert torch.all(mx[nz] / torch.exp2(k[nz]) > 224)


def test_quantization_is_a_fixed_point_and_close():
    w = synth.make_model(synth.TINY, 0)
    q = synth.quantize_fp8_model(synth.TINY, w)
    for key in ("layers.0.wq", "layers.1.w_down", "lm_head"):
        assert torch.equal(synth.quantize_fp8_rows(q[key]), q[key])
        rel = (q[key].float() - w[key].float()).norm() / w[key].float().norm()
        assert rel < 0.04                        # e4m3: 3 significand bits
    assert torch.equal(q["embed"], w["embed"])   # untied: the embedding stays bf16
    assert torch.equal(q["layers.0.attn_norm"], w["layers.0.attn_norm"])


def test_fp8_weight_bytes_halve_the_matrices():
    m = synth.LLAMA8B
    b16, b8 = roofline.weight_bytes(m, 2), roofline.weight_bytes(m, 1)
    rows = m.n_layers * (m.q_dim + 2 * m.kv_dim + m.hidden + 2 * m.ffn + m.hidden) + m.vocab
    vec = 2 * (m.n_layers * 2 * m.hidden + m.hidden)
    assert b16 - vec == 2 * (b8 - vec - 4 * rows)
