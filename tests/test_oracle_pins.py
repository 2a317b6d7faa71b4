"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here re-types the oracle's formulas: every check is a printed worked
example, a closed form, an invariant, a special case that reduces to a library
routine, or an independent library implementation of the same decoder
(Hugging Face transformers' Llama and Qwen2 models in fp32).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from persistent_megakernel_03_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [list(map(float, ln.split())) for ln in f if ln.strip() and not ln.startswith("#")]


# ------------------------------------------------------- closed forms

def test_kv_cache_size_worked_example():
    # "LLM高速化勉強会資料" slide 10: the printed example is 192 GiB.
    for b, L, S, hd, h, by, gib in _rows("kv_cache_size.txt"):
        assert oracle.kv_cache_bytes(b, L, S, hd, h, by) == gib * 2**30


def test_kv_cache_size_long_context_shape():
    # 32 layers x 32768 positions x 8 KV heads x 128 dims, bf16, one request.
    assert oracle.kv_cache_bytes(1, 32, 32768, 128, 8, 2) == 4 * 2**30
    # per token per layer of the Llama-3-8B shape: 2 * 8 * 128 * 2 bytes
    assert oracle.kv_cache_bytes(1, 1, 1, 128, 8, 2) == 4096


def test_bf16_round_matches_torch():
    xs = np.concatenate([RNG.standard_normal(4000).astype(np.float32) * 10,
                         np.array([1.0 + 2**-8, 1.0 + 3 * 2**-8, -1.0 - 2**-8, 0.0, -0.0,
                                   1e-40, 3.0e38], dtype=np.float32)])
    want = torch.from_numpy(xs).to(torch.bfloat16).float().numpy()
    got = np.array([oracle.bf16_round(float(x)) for x in xs], dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


# ------------------------------------------------------------ softmax

def test_softmax_rows_sum_to_one_and_shift_invariant():
    for n in (1, 2, 7, 128, 4097):
        s = RNG.standard_normal(n).astype(np.float32) * 5
        p = oracle.softmax(s)
        assert abs(float(p.astype(np.float64).sum()) - 1.0) <= 1e-6 * max(1, math.log2(n))
        assert np.all(p >= 0)
        p2 = oracle.softmax(s + 1000.0)          # max subtraction: no overflow
        np.testing.assert_allclose(p2, p, rtol=1e-4, atol=1e-7)


def test_softmax_two_point_closed_form():
    for a, b in [(0.0, 0.0), (1.0, -2.0), (30.0, -30.0), (-5.5, 2.25)]:
        p = oracle.softmax([a, b])
        assert p[0] == pytest.approx(1.0 / (1.0 + math.exp(b - a)), rel=1e-6, abs=1e-30)


def test_softmax_uniform():
    p = oracle.softmax(np.full(10, 3.7, np.float32))
    np.testing.assert_allclose(p, 0.1, rtol=1e-6)


# --------------------------------------------------------------- RoPE

def test_rope_identity_at_position_zero():
    v = RNG.standard_normal(128).astype(np.float32)
    assert np.array_equal(oracle.rope(v, 0, 500000.0), v)


def test_rope_preserves_norm():
    for d, theta in ((64, 1e4), (128, 5e5), (64, 1e6)):
        v = RNG.standard_normal(d).astype(np.float32)
        for p in (1, 17, 551, 32767):
            r = oracle.rope(v, p, theta)
            assert np.linalg.norm(r.astype(np.float64)) == pytest.approx(
                np.linalg.norm(v.astype(np.float64)), rel=1e-6)


def test_rope_closed_form_rotate_half_pairs():
    # d = 4: pair (0, 2) turns by pos * theta^0, pair (1, 3) by pos * theta^(-1/2).
    theta, pos = 10000.0, 3
    e0 = oracle.rope([1, 0, 0, 0], pos, theta)
    np.testing.assert_allclose(e0, [math.cos(3), 0, math.sin(3), 0], atol=1e-7)
    e1 = oracle.rope([0, 1, 0, 0], pos, theta)
    a = pos * theta ** -0.5
    np.testing.assert_allclose(e1, [0, math.cos(a), 0, math.sin(a)], atol=1e-7)
    e2 = oracle.rope([0, 0, 1, 0], pos, theta)
    np.testing.assert_allclose(e2, [-math.sin(3), 0, math.cos(3), 0], atol=1e-7)


def test_rope_scores_depend_on_relative_position_only():
    d, theta = 128, 500000.0
    q = RNG.standard_normal(d).astype(np.float32)
    k = RNG.standard_normal(d).astype(np.float32)
    ref = float(np.dot(oracle.rope(q, 7, theta).astype(np.float64),
                       oracle.rope(k, 0, theta).astype(np.float64)))
    for m in (10, 300, 2000):
        got = float(np.dot(oracle.rope(q, m + 7, theta).astype(np.float64),
                           oracle.rope(k, m, theta).astype(np.float64)))
        assert got == pytest.approx(ref, rel=2e-4, abs=2e-4)


# ---------------------------------------------------------- attention

def test_single_key_returns_v():
    q = RNG.standard_normal(64).astype(np.float32)
    K = RNG.standard_normal((1, 64)).astype(np.float32)
    V = RNG.standard_normal((1, 64)).astype(np.float32)
    assert np.array_equal(oracle.attend(q, K, V), V[0])
    assert np.array_equal(oracle.attend_split(q, K, V, 1), V[0])


def test_equal_scores_give_mean_of_v():
    q = np.zeros(64, np.float32)
    K = RNG.standard_normal((37, 64)).astype(np.float32)
    V = RNG.standard_normal((37, 64)).astype(np.float32)
    np.testing.assert_allclose(oracle.attend(q, K, V), V.astype(np.float64).mean(0),
                               rtol=1e-5, atol=1e-6)


def test_dominant_key_selects_its_value():
    d = 64
    K = np.zeros((5, d), np.float32)
    K[3, 0] = 1000.0
    q = np.zeros(d, np.float32)
    q[0] = 8.0
    V = RNG.standard_normal((5, d)).astype(np.float32)
    np.testing.assert_allclose(oracle.attend(q, K, V), V[3], rtol=1e-6)


def test_attention_is_permutation_invariant_over_keys():
    q = RNG.standard_normal(128).astype(np.float32)
    K = RNG.standard_normal((50, 128)).astype(np.float32)
    V = RNG.standard_normal((50, 128)).astype(np.float32)
    perm = RNG.permutation(50)
    np.testing.assert_allclose(oracle.attend(q, K[perm], V[perm]), oracle.attend(q, K, V),
                               rtol=1e-5, atol=1e-6)


def _brute_force_attention_f64(q, K, V):
    """Tiny-input brute force: enumerate exp(score) weights in fp64."""
    d = K.shape[1]
    w = [math.exp(float(np.dot(q.astype(np.float64), K[j].astype(np.float64))) / math.sqrt(d))
         for j in range(K.shape[0])]
    tot = sum(w)
    return sum(w[j] / tot * V[j].astype(np.float64) for j in range(K.shape[0]))


@pytest.mark.parametrize("n,splits", [(1, 1), (5, 2), (64, 4), (301, 7), (1000, 18), (9, 16)])
def test_split_combine_equals_direct_softmax(n, splits):
    # Online softmax is exact up to rounding ("Hạt nhân là gì ...").
    d = 128
    q = (RNG.standard_normal(d) * 0.3).astype(np.float32)
    K = RNG.standard_normal((n, d)).astype(np.float32)
    V = RNG.standard_normal((n, d)).astype(np.float32)
    direct = oracle.attend(q, K, V)
    split = oracle.attend_split(q, K, V, splits)
    np.testing.assert_allclose(split, direct, rtol=2e-5, atol=2e-6)
    bf = _brute_force_attention_f64(q, K, V)
    np.testing.assert_allclose(direct, bf, rtol=1e-5, atol=2e-6)
    np.testing.assert_allclose(split, bf, rtol=1e-5, atol=2e-6)


# ------------------------------------------------------ norm / gemv / misc

def test_rmsnorm_unit_rms_and_scale_invariance():
    for n in (256, 896, 4096):
        x = (RNG.standard_normal(n) * 0.02).astype(np.float32)
        w = torch.ones(n, dtype=torch.bfloat16)
        y = oracle.rmsnorm(x, w, 1e-6)
        assert math.sqrt(float(np.mean(y.astype(np.float64) ** 2))) == pytest.approx(1.0, rel=2e-3)
        np.testing.assert_allclose(oracle.rmsnorm(x * 8.0, w, 0.0), oracle.rmsnorm(x, w, 0.0),
                                   rtol=1e-6)
        w2 = torch.full((n,), 2.0, dtype=torch.bfloat16)
        np.testing.assert_allclose(oracle.rmsnorm(x, w2, 1e-6), 2 * y, rtol=1e-7)


def test_rmsnorm_against_torch_library():
    x = RNG.standard_normal(4096).astype(np.float32)
    w = (torch.randn(4096) * 0.1 + 1).to(torch.bfloat16)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x).double(), (4096,),
                                       w.double(), eps=1e-5).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(x, w, 1e-5), ref, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("rows,cols", [(1, 1), (3, 256), (129, 896), (64, 4864), (17, 14336)])
def test_gemv_against_numpy_fp64(rows, cols):
    W = (torch.randn(rows, cols) * 0.02).to(torch.bfloat16)
    x = RNG.standard_normal(cols).astype(np.float32)
    ref = W.double().numpy() @ x.astype(np.float64)
    got = oracle.gemv(W, x)
    bound = 2 * cols * 2**-24 * (np.abs(W.double().numpy()) @ np.abs(x.astype(np.float64)))
    assert np.all(np.abs(got - ref) <= bound + 1e-30)


def test_argmax_lowest_index_on_ties():
    assert oracle.argmax([1, 3, 3, 2]) == 1
    assert oracle.argmax([5, 5, 5]) == 0
    assert oracle.argmax([-1, -2, -0.5, -0.5]) == 2
    v = RNG.standard_normal(128256).astype(np.float32)
    assert oracle.argmax(v) == int(np.argmax(v))


def test_silu_identities():
    assert oracle.silu(0.0) == 0.0
    for z in (0.1, 1.0, 3.0, 7.5):
        assert oracle.silu(z) - oracle.silu(-z) == pytest.approx(z, rel=1e-6)
        assert oracle.silu(z) == pytest.approx(float(torch.nn.functional.silu(
            torch.tensor(z, dtype=torch.float64))), rel=1e-6)
    assert oracle.silu(40.0) == pytest.approx(40.0, rel=1e-7)


# ---------------------------------------------------------- whole decoder

SMALL_QWEN = synth.ModelConfig("qwen-width-2l", n_layers=2, hidden=896, n_q_heads=14,
                               n_kv_heads=2, head_dim=64, ffn=4864, vocab=2048, rms_eps=1e-6,
                               rope_theta=1e6, qkv_bias=True, tied_embeddings=True)
SMALL_LLAMA = synth.ModelConfig("llama-width-1l", n_layers=1, hidden=4096, n_q_heads=32,
                                n_kv_heads=8, head_dim=128, ffn=14336, vocab=1024,
                                rms_eps=1e-5, rope_theta=500000.0)


@pytest.fixture(scope="module")
def tiny():
    return synth.TINY, synth.make_model(synth.TINY, 0)


def test_cached_decode_equals_full_recompute_tiny(tiny):
    cfg, w = tiny
    m = oracle.OracleModel(cfg, w)
    toks = synth.make_prompt(24, cfg.vocab).numpy()
    st = m.new_state(32)
    steps = [m.decode(st, int(t), p) for p, t in enumerate(toks)]
    lf, hf = m.forward_full(toks)
    for p, (nid, lg, hid) in enumerate(steps):
        assert np.array_equal(lg, lf[p]) and np.array_equal(hid, hf[p])
        assert nid == int(np.argmax(lf[p]))


@pytest.mark.parametrize("cfg", [SMALL_QWEN, SMALL_LLAMA], ids=lambda c: c.name)
def test_cached_decode_equals_full_recompute_wide(cfg):
    w = synth.make_model(cfg, 0)
    m = oracle.OracleModel(cfg, w)
    toks = synth.make_prompt(5, cfg.vocab).numpy()
    st = m.new_state(8)
    lf, hf = m.forward_full(toks)
    for p, t in enumerate(toks):
        nid, lg, hid = m.decode(st, int(t), p)
        np.testing.assert_allclose(lg, lf[p], rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(hid, hf[p], rtol=1e-5, atol=1e-5)


def test_prefill_equals_full_recompute_and_sequential_steps(tiny):
    # the prompt-only entry point: the last position's logits and hidden as
    # the uncached forward gives them, and a cache identical to the one of
    # the same positions run as decode steps
    cfg, w = tiny
    m = oracle.OracleModel(cfg, w)
    toks = synth.make_prompt(20, cfg.vocab, seed=3).numpy()
    a = m.new_state(24)
    nid, lg, hid = m.prefill(a, toks)
    lf, hf = m.forward_full(toks)
    assert np.array_equal(lg, lf[-1]) and np.array_equal(hid, hf[-1])
    assert nid == int(np.argmax(lf[-1]))
    b = m.new_state(24)
    for p, t in enumerate(toks):
        m.decode(b, int(t), p)
    for l in range(cfg.n_layers):
        for which in (0, 1):
            assert np.array_equal(a.kv(l, 1, which, 20), b.kv(l, 1, which, 20))
    with pytest.raises(ValueError):
        m.prefill(m.new_state(8), toks)          # longer than the state


def test_cache_holds_rotated_bf16_keys(tiny):
    cfg, w = tiny
    m = oracle.OracleModel(cfg, w)
    st = m.new_state(8)
    toks = synth.make_prompt(3, cfg.vocab).numpy()
    for p, t in enumerate(toks):
        m.decode(st, int(t), p)
    K = st.kv(0, 1, 0, 3)
    assert np.all(K == torch.from_numpy(K).to(torch.bfloat16).float().numpy())
    # position 0 of layer 0 is exactly rope(Wk rmsnorm(E[t0]), 0) rounded to bf16
    x = w["embed"][int(toks[0])].float().numpy()
    xn = oracle.rmsnorm(x, w["layers.0.attn_norm"], cfg.rms_eps)
    k = oracle.gemv(w["layers.0.wk"], xn)[64:128]
    assert np.array_equal(K[0], torch.from_numpy(k).to(torch.bfloat16).float().numpy())


def test_decode_continues_identically_from_a_copied_cache(tiny):
    # the long-context checks hand the oracle a cache it did not build: a
    # state whose cache was written through set_kv must decode exactly like
    # the state that built it
    cfg, w = tiny
    m = oracle.OracleModel(cfg, w)
    toks = synth.make_prompt(12, cfg.vocab, seed=4).numpy()
    a = m.new_state(16)
    for p, t in enumerate(toks[:-1]):
        m.decode(a, int(t), p)
    b = m.new_state(16)
    n = len(toks) - 1
    for l in range(cfg.n_layers):
        for g in range(cfg.n_kv_heads):
            for which in (0, 1):
                b.set_kv(l, g, which, a.kv(l, g, which, n))
    ra = m.decode(a, int(toks[-1]), n)
    rb = m.decode(b, int(toks[-1]), n)
    assert ra[0] == rb[0]
    assert np.array_equal(ra[1], rb[1]) and np.array_equal(ra[2], rb[2])
    # and a cache that differs in one key changes the result
    c = m.new_state(16)
    for l in range(cfg.n_layers):
        for g in range(cfg.n_kv_heads):
            for which in (0, 1):
                kv = a.kv(l, g, which, n)
                if (l, g, which) == (1, 0, 0):
                    kv[3] = -kv[3]
                c.set_kv(l, g, which, kv)
    rc = m.decode(c, int(toks[-1]), n)
    assert not np.array_equal(ra[1], rc[1])


def _hf_model(cfg, w):
    transformers = pytest.importorskip("transformers")
    common = dict(hidden_size=cfg.hidden, intermediate_size=cfg.ffn,
                  num_hidden_layers=cfg.n_layers, num_attention_heads=cfg.n_q_heads,
                  num_key_value_heads=cfg.n_kv_heads, head_dim=cfg.head_dim,
                  vocab_size=cfg.vocab, rms_norm_eps=cfg.rms_eps,
                  tie_word_embeddings=cfg.tied_embeddings, max_position_embeddings=4096)
    if cfg.qkv_bias:
        hc = transformers.Qwen2Config(rope_theta=cfg.rope_theta, **common)
        model = transformers.Qwen2ForCausalLM(hc)
    else:
        hc = transformers.LlamaConfig(rope_theta=cfg.rope_theta, attention_bias=False,
                                      mlp_bias=False, **common)
        model = transformers.LlamaForCausalLM(hc)
    sd = {"model.embed_tokens.weight": w["embed"], "model.norm.weight": w["final_norm"]}
    names = {"wq": "self_attn.q_proj.weight", "wk": "self_attn.k_proj.weight",
             "wv": "self_attn.v_proj.weight", "wo": "self_attn.o_proj.weight",
             "bq": "self_attn.q_proj.bias", "bk": "self_attn.k_proj.bias",
             "bv": "self_attn.v_proj.bias", "w_gate": "mlp.gate_proj.weight",
             "w_up": "mlp.up_proj.weight", "w_down": "mlp.down_proj.weight",
             "attn_norm": "input_layernorm.weight", "ffn_norm": "post_attention_layernorm.weight"}
    for l in range(cfg.n_layers):
        for k, hf in names.items():
            t = w.get(f"layers.{l}.{k}")
            if t is not None:
                sd[f"model.layers.{l}.{hf}"] = t
    sd["lm_head.weight"] = w["embed"] if cfg.tied_embeddings else w["lm_head"]
    sd = {k: v.float() for k, v in sd.items()}
    model = model.float().eval()
    missing, unexpected = model.load_state_dict(sd, strict=False)
    assert not unexpected and all("rotary" in k for k in missing), (missing, unexpected)
    return model


def _random_norms(w, seed: int):
    """The same weights with every RMSNorm weight drawn as 1 + 0.25 N(0, 1)
    (bf16): the synthetic models' unit norms hide which norm a step applies."""
    g = torch.Generator("cpu").manual_seed(seed)
    out = dict(w)
    for k, t in w.items():
        if k.endswith("norm"):
            out[k] = (1.0 + 0.25 * torch.randn(t.shape, generator=g)).to(torch.bfloat16)
    return out


@pytest.mark.parametrize("norms", ["unit", "random"])
@pytest.mark.parametrize("cfg", [synth.TINY, SMALL_QWEN], ids=lambda c: c.name)
def test_forward_matches_transformers_library(cfg, norms):
    """An independent implementation of the same decoder (Llama / Qwen2 in
    transformers, fp32, no KV rounding) must give the oracle's logits, also
    with non-unit norm weights."""
    torch.manual_seed(0)
    w = synth.make_model(cfg, 0)
    if norms == "random":
        w = _random_norms(w, 3)
    hf = _hf_model(cfg, w)
    toks = synth.make_prompt(12, cfg.vocab).numpy()
    with torch.no_grad():
        out = hf(torch.from_numpy(toks.astype(np.int64))[None], output_hidden_states=True)
    ref = out.logits[0].double().numpy()
    m = oracle.OracleModel(cfg, w, kv_bf16=False)
    lf, hf_hidden = m.forward_full(toks)
    scale = float(np.abs(ref).max())
    assert np.abs(lf - ref).max() <= 2e-5 * max(scale, 1.0)
    st = m.new_state(16)
    for p, t in enumerate(toks):
        nid, lg, _ = m.decode(st, int(t), p)
        assert np.abs(lg - ref[p]).max() <= 2e-5 * max(scale, 1.0)


def test_bf16_kv_rounding_stays_inside_parity_tolerance(tiny):
    cfg, w = tiny
    toks = synth.make_prompt(16, cfg.vocab).numpy()
    a, _ = oracle.OracleModel(cfg, w, kv_bf16=True).forward_full(toks)
    b, _ = oracle.OracleModel(cfg, w, kv_bf16=False).forward_full(toks)
    d = np.abs(a - b).max()
    assert 0 < d < 3e-2
