"""Plant plausible mistakes in copies of the oracle's C source (on the CPU)
and check that the pins catch every one of them.  The unmodified source is
the control and must pass."""
import math

import numpy as np
import pytest
import torch

import oracle
from persistent_megakernel_03_b200 import synth

MUTATIONS = {
    "rope_sign": ("v[i] = a * c - b * s;", "v[i] = a * c + b * s;"),
    "rope_exponent": ("pow(theta, -2.0 * (double)i / (double)head_dim)",
                      "pow(theta, -1.0 * (double)i / (double)head_dim)"),
    "gqa_mapping": ("int kvh = h / G;", "int kvh = h % hkv;"),
    "ffn_residual_dropped": ("x[i] = x[i] + d[i];", "x[i] = d[i];"),
    "attn_scale": ("1.0f / sqrtf((float)head_dim);", "1.0f / (float)head_dim;"),
    "rms_mean": ("ss / (float)n + eps", "ss + eps"),
    "silu_sign": ("z / (1.0f + expf(-z))", "z / (1.0f + expf(z))"),
    "argmax_ties": ("if (v[i] > v[best]) best = i;", "if (v[i] >= v[best]) best = i;"),
    "combine_no_rescale": ("float c = expf(ms[b] - m);", "float c = 1.0f;"),
    "gate_up_swapped": ("g[i] = orc_silu(g[i]) * u[i];", "g[i] = orc_silu(u[i]) * g[i];"),
    "kv_store_position": ("kv_store(s, kv_index(c, s->max_seq, l, h, 0, pos)",
                          "kv_store(s, kv_index(c, s->max_seq, l, h, 0, pos ? pos - 1 : 0)"),
    "oproj_residual_dropped": ("for (int i = 0; i < H; ++i) x[i] = x[i] + tmp[i];",
                               "for (int i = 0; i < H; ++i) x[i] = tmp[i];"),
    "bias_dropped": ("y[i] = y[i] + bf16_to_f32(b[i]);", "y[i] = y[i];"),
    "ffn_norm_uses_attn_norm": ("orc_rmsnorm(x, L->ffn_norm, c->hidden, c->rms_eps, xn);",
                                "orc_rmsnorm(x, L->attn_norm, c->hidden, c->rms_eps, xn);"),
    "final_norm_uses_a_layer_norm": (
        "orc_rmsnorm(x, m->final_norm, c->hidden, c->rms_eps, xn);",
        "orc_rmsnorm(x, m->layers[c->n_layers - 1].ffn_norm, c->hidden, c->rms_eps, xn);"),
    "lm_head_always_tied": ("m->lm_head = lm_head ? lm_head : embed;", "m->lm_head = embed;"),
    "eps_outside_sqrt": ("float r = 1.0f / sqrtf(ss / (float)n + eps);",
                         "float r = 1.0f / (sqrtf(ss / (float)n) + eps);"),
    "rope_pairs_adjacent": ("float a = v[i], b = v[i + half];\n    v[i] = a * c - b * s;\n"
                            "    v[i + half] = a * s + b * c;",
                            "float a = v[2 * i], b = v[2 * i + 1];\n    v[2 * i] = a * c - b * s;\n"
                            "    v[2 * i + 1] = a * s + b * c;"),
    "v_stored_as_k": ("kv_store(s, kv_index(c, s->max_seq, l, h, 0, pos), k + (size_t)h * d, d);",
                      "kv_store(s, kv_index(c, s->max_seq, l, h, 0, pos), v + (size_t)h * d, d);"),
    "embedding_row": ("const uint16_t* e = m->embed + (size_t)token * H;",
                      "const uint16_t* e = m->embed + (size_t)(token ^ 1) * H;"),
}

QWEN_MINI = synth.ModelConfig("qwen-mini", n_layers=2, hidden=128, n_q_heads=6, n_kv_heads=2,
                              head_dim=32, ffn=256, vocab=512, rms_eps=1e-6, rope_theta=1e6,
                              qkv_bias=True, tied_embeddings=True)


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _pins_pass(L, hf_refs) -> bool:
    rng = np.random.default_rng(7)
    # RoPE closed form (d = 4)
    for vec, want in (([1, 0, 0, 0], [math.cos(3), 0, math.sin(3), 0]),
                      ([0, 1, 0, 0], [0, math.cos(3 * 1e4 ** -0.5), 0, math.sin(3 * 1e4 ** -0.5)])):
        v = _f32(vec)
        L.orc_rope(v, 4, 3, 1e4)
        if not np.allclose(v, want, atol=1e-6):
            return False
    # attention: dominant key, split == direct
    d = 64
    q = _f32(rng.standard_normal(d) * 0.3)
    K = _f32(rng.standard_normal((40, d)))
    V = _f32(rng.standard_normal((40, d)))
    o1, o2 = np.empty(d, np.float32), np.empty(d, np.float32)
    L.orc_attend(q, K, V, 40, d, o1)
    L.orc_attend_split(q, K, V, 40, d, 5, o2)
    w = np.exp(K.astype(np.float64) @ q.astype(np.float64) / math.sqrt(d))
    bf = (w / w.sum()) @ V.astype(np.float64)
    if not (np.allclose(o1, bf, rtol=1e-5, atol=2e-6) and np.allclose(o2, bf, rtol=1e-5, atol=2e-6)):
        return False
    # argmax ties, silu identity
    if L.orc_argmax(_f32([1, 3, 3, 2]), 4) != 1:
        return False
    if abs(L.orc_silu(2.0) - L.orc_silu(-2.0) - 2.0) > 1e-6:
        return False
    # rmsnorm unit RMS
    x = _f32(rng.standard_normal(256) * 0.02)
    y = np.empty_like(x)
    ones = torch.ones(256, dtype=torch.bfloat16)
    L.orc_rmsnorm(x, ones.data_ptr(), 256, 1e-6, y)
    if abs(math.sqrt(float(np.mean(y.astype(np.float64) ** 2))) - 1) > 2e-3:
        return False
    # whole decoder: cached decode == full recompute, and the library witness
    for cfg, w, toks, ref in hf_refs:
        m = oracle.OracleModel(cfg, w, kv_bf16=False, _lib=L)
        lf, _ = m.forward_full(toks)
        st = m.new_state(len(toks))
        for p, t in enumerate(toks):
            _, lg, _ = m.decode(st, int(t), p)
            if not np.allclose(lg, lf[p], rtol=1e-5, atol=1e-5):
                return False
        if np.abs(lf - ref).max() > 2e-5 * max(1.0, float(np.abs(ref).max())):
            return False
    return True


@pytest.fixture(scope="module")
def hf_refs():
    from test_oracle_pins import _hf_model, _random_norms
    refs = []
    for cfg in (synth.TINY, QWEN_MINI):
        w = _random_norms(synth.make_model(cfg, 0), 5)
        toks = synth.make_prompt(10, cfg.vocab).numpy()
        with torch.no_grad():
            ref = _hf_model(cfg, w)(torch.from_numpy(toks.astype(np.int64))[None]).logits[0]
        refs.append((cfg, w, toks, ref.double().numpy()))
    return refs


@pytest.fixture(scope="module")
def variant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("oracle_variants"))


def test_control_source_passes(hf_refs, variant_dir):
    so = oracle.compile_variant(oracle.source_text(), variant_dir, "control")
    assert _pins_pass(oracle.load_variant(so), hf_refs)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, hf_refs, variant_dir):
    src = oracle.source_text()
    old, new = MUTATIONS[name]
    assert old in src, f"mutation anchor for {name} not found"
    so = oracle.compile_variant(src.replace(old, new), variant_dir, f"mut_{name}")
    assert not _pins_pass(oracle.load_variant(so), hf_refs), f"pins missed {name}"


# Mistakes in the fp8 weight rule (orc_quantize_fp8_rows).
FP8_MUTATIONS = {
    "fp8_truncates": ("double r = rint(a / step) * step;", "double r = floor(a / step) * step;"),
    "fp8_no_subnormal_floor": ("if (e < -6) e = -6;", "if (e < -60) e = -60;"),
    "fp8_scale_one_too_small": ("while (mx <= ldexp(448.0, k - 1)) --k;",
                                "while (mx <= ldexp(448.0, k)) --k;"),
    "fp8_sign_dropped": ("ldexp(v < 0 ? -q : q, k)", "ldexp(q, k)"),
    "fp8_four_significand_bits": ("double step = ldexp(1.0, e - 3);",
                                  "double step = ldexp(1.0, e - 4);"),
}


def _fp8_pins_pass(L) -> bool:
    def q(rows):
        w = torch.tensor(rows, dtype=torch.bfloat16)
        out = torch.empty_like(w)
        k = np.empty(w.shape[0], dtype=np.int32)
        L.orc_quantize_fp8_rows(w.data_ptr(), w.shape[0], w.shape[1], out.data_ptr(), k)
        return out, k
    out, k = q([[448, 1, 0.1, -17, 19, 3 * 2**-9, 2**-10, -1.5 * 2**-9]])
    if out.float()[0].tolist() != [448, 1, 0.1015625, -16, 20, 3 * 2**-9, 0, -2**-8]:
        return False
    g = torch.Generator("cpu").manual_seed(0)
    w = (torch.randn(16, 64, generator=g) * 0.02).to(torch.bfloat16)
    out = torch.empty_like(w)
    k = np.empty(16, dtype=np.int32)
    L.orc_quantize_fp8_rows(w.data_ptr(), 16, 64, out.data_ptr(), k)
    s = torch.exp2(torch.from_numpy(k).double()).unsqueeze(1)
    want = ((w.double() / s).float().to(torch.float8_e4m3fn).double() * s).to(torch.bfloat16)
    mx = w.double().abs().amax(dim=1)
    return bool(torch.equal(out, want) and torch.all(mx <= 448 * s[:, 0]) and
                torch.all(mx > 224 * s[:, 0]))


def test_fp8_control_passes(variant_dir):
    so = oracle.compile_variant(oracle.source_text(), variant_dir, "control_fp8")
    assert _fp8_pins_pass(oracle.load_variant(so))


@pytest.mark.parametrize("name", sorted(FP8_MUTATIONS))
def test_planted_fp8_mistake_is_caught(name, variant_dir):
    src = oracle.source_text()
    old, new = FP8_MUTATIONS[name]
    assert old in src, f"mutation anchor for {name} not found"
    so = oracle.compile_variant(src.replace(old, new), variant_dir, f"mut_{name}")
    assert not _fp8_pins_pass(oracle.load_variant(so)), f"pins missed {name}"
