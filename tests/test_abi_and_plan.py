"""Host-side checks of libmk: the C-ABI exports and the task-graph builder.

No GPU: the library is loaded, but only its host-only entry points are called.
"""
import os
import random
import re
import subprocess

import pytest

from persistent_megakernel_03_b200 import binding, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
QKV, ATTN, OPROJ, GATEUP, DOWN, LMHEAD = range(6)


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(mk_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    L = binding.lib()
    names = declared_functions()
    assert len(names) >= 15, names
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert getattr(L, n) is not None
    assert set(binding.EXPORTS) <= set(names)


def test_create_rejects_bad_config_without_gpu():
    import ctypes as C
    L = binding.lib()
    bad = synth.ModelConfig("bad", 2, 256, 4, 2, 96, 768, 4096, 1e-6, 1e4)
    cfg = binding.make_config(bad, 32)
    h = C.c_void_p()
    w = binding.Weights()
    assert L.mk_create(C.byref(cfg), C.byref(w), None, None, C.byref(h)) == -1
    assert b"head_dim" in L.mk_last_error(None)


def _fake_weights(model, **override):
    """Weight structs whose pointers are 16-byte-aligned addresses that are
    never dereferenced: mk_create checks them before any CUDA call."""
    import ctypes as C
    layers = (binding.LayerWeights * model.n_layers)()
    addr = 0x100000
    for l in range(model.n_layers):
        for k in binding.LAYER_FIELDS:
            setattr(layers[l], k, addr)
            addr += 0x1000
    for (l, k), v in override.get("layer", {}).items():
        setattr(layers[l], k, v)
    w = binding.Weights(override.get("embed", 0x10000), layers, override.get("final_norm", 0x20000),
                        override.get("lm_head", 0x30000))
    return w, layers


@pytest.mark.parametrize("case,want_rc,want_msg", [
    ("no embedding", -1, b"missing weight pointer"),
    ("no final norm", -1, b"missing weight pointer"),
    ("no LM head, untied", -1, b"missing weight pointer"),
    ("null down projection", -1, b"16-byte aligned"),
    ("misaligned O projection", -1, b"16-byte aligned"),
    ("bias flag without a bias", -1, b"bias pointer is null"),
    ("three query heads per KV head", -9, b"query heads per KV head"),
])
def test_create_rejects_weights_and_shapes_before_any_launch(case, want_rc, want_msg):
    # argument errors come back before mk_create touches the device, so these
    # run without a GPU
    import ctypes as C
    import dataclasses
    L = binding.lib()
    model = dataclasses.replace(synth.TINY, tied_embeddings=False)
    override = {
        "no embedding": {"embed": None},
        "no final norm": {"final_norm": None},
        "no LM head, untied": {"lm_head": None},
        "null down projection": {"layer": {(1, "w_down"): None}},
        "misaligned O projection": {"layer": {(0, "wo"): 0x100008}},
    }.get(case, {})
    if case == "bias flag without a bias":
        model = dataclasses.replace(model, qkv_bias=True)
        override = {"layer": {(1, "bk"): None}}
    if case == "three query heads per KV head":
        model = dataclasses.replace(model, n_q_heads=6, n_kv_heads=2)
    w, keep = _fake_weights(model, **override)
    cfg = binding.make_config(model, 32)
    h = C.c_void_p()
    assert L.mk_create(C.byref(cfg), C.byref(w), None, None, C.byref(h)) == want_rc
    assert want_msg in L.mk_last_error(None)
    assert not h.value


def test_null_context_calls_are_argument_errors_without_gpu():
    L = binding.lib()
    assert L.mk_inject_stall(None, -1) == -1
    assert L.mk_status(None) == -1
    assert L.mk_set_mode(None, 0) == -1


@pytest.mark.parametrize("model,bad", [
    (synth.TINY, dict(head_dim=96)),
    (synth.TINY, dict(n_kv_heads=3)),
    (synth.TINY, dict(hidden=250)),
    (synth.LLAMA8B, dict(ffn=20000)),
])
def test_plan_rejects_invalid_shapes(model, bad):
    import dataclasses
    m = dataclasses.replace(model, **bad)
    with pytest.raises(binding.MkError):
        binding.Plan(m, 64, 148)


def _simulate(plan, model, max_batch, rng):
    """Run the per-CTA queues in a random interleaving under the event rules
    and check every read happens after its producer wrote."""
    tasks = plan.tasks()
    counts = plan.event_counts()
    P = plan.info.num_ctas
    S = plan.info.attn_splits
    queues = [plan.queue(c) for c in range(P)]
    head = [0] * P
    ev = [0] * len(counts)
    L, nkv = model.n_layers, model.n_kv_heads
    G = model.n_q_heads // nkv
    d = model.head_dim
    per_group = (G + 2) * d
    qkv_rows = (model.n_q_heads + 2 * nkv) * d
    written = {}      # (kind, layer) -> set of rows
    done_kind = {}    # (kind, layer) -> count of finished tasks
    tickets = {}
    total = {}
    for t in tasks:
        total[(t["kind"], t["layer"])] = total.get((t["kind"], t["layer"]), 0) + 1
    finished = 0
    while finished < len(tasks):
        ready = [c for c in range(P) if head[c] < len(queues[c]) and
                 (tasks[queues[c][head[c]]]["wait_event"] < 0 or
                  ev[tasks[queues[c][head[c]]]["wait_event"]] >=
                  tasks[queues[c][head[c]]]["wait_count"])]
        assert ready, "deadlock: no CTA can run its next task"
        c = rng.choice(ready)
        t = tasks[queues[c][head[c]]]
        head[c] += 1
        k, l = t["kind"], t["layer"]
        # reads must see complete producers
        if k == QKV and l > 0:
            assert done_kind.get((DOWN, l - 1), 0) == total[(DOWN, l - 1)]
        if k == ATTN:
            rows = set(range(t["row0"] * per_group, (t["row0"] + 1) * per_group))
            assert rows <= written.get((QKV, l), set())
        if k == OPROJ:
            # every split of every (slot, group) wrote its partial ...
            assert done_kind.get((ATTN, l), 0) == total[(ATTN, l)] == max_batch * nkv * S
            # ... and every QKV(l) task read x before OPROJ(l) overwrites it
            assert done_kind.get((QKV, l), 0) == total[(QKV, l)]
        if k == GATEUP:
            assert len(written.get((OPROJ, l), ())) == model.hidden
        if k == DOWN:
            assert len(written.get((GATEUP, l), ())) == 2 * model.ffn
            assert done_kind.get((GATEUP, l), 0) == total[(GATEUP, l)]
        if k == LMHEAD:
            assert len(written.get((DOWN, L - 1), ())) == model.hidden
        # effects
        if k != ATTN:
            rs = written.setdefault((k, l), set())
            assert not (rs & set(range(t["row0"], t["row1"]))), "row written twice"
            rs.update(range(t["row0"], t["row1"]))
        else:
            key = (t["req"], l, t["row0"], t["row1"])
            assert key not in tickets, "split computed twice"
            tickets[key] = 1
        for e in range(t["signal_event0"], t["signal_event0"] + t["n_signal"]):
            ev[e] += 1
        done_kind[(k, l)] = done_kind.get((k, l), 0) + 1
        finished += 1
    assert ev == counts
    assert len(written[(QKV, 0)]) == qkv_rows
    return tasks


@pytest.mark.parametrize("model,max_seq,P", [
    (synth.TINY, 32, 148), (synth.TINY, 32, 7), (synth.TINY, 32, 1),
    (synth.QWEN05B.with_layers(3), 600, 148), (synth.LLAMA8B.with_layers(2), 600, 148),
    (synth.LLAMA8B.with_layers(2), 33024, 148), (synth.LLAMA8B.with_layers(2), 600, 132),
])
def test_plan_is_deadlock_free_and_hazard_free(model, max_seq, P):
    plan = binding.Plan(model, max_seq, P)
    for seed in range(3):
        tasks = _simulate(plan, model, 1, random.Random(seed))
    # thresholds are the full per-step counts of their events
    counts = plan.event_counts()
    for t in tasks:
        if t["wait_event"] >= 0:
            assert t["wait_count"] == counts[t["wait_event"]] > 0


@pytest.mark.parametrize("model", [synth.TINY, synth.QWEN05B, synth.LLAMA8B],
                         ids=lambda m: m.name)
def test_plan_rows_partition_and_fit(model):
    P = 148
    plan = binding.Plan(model, 1024, P)
    tasks = plan.tasks()
    H, F, V = model.hidden, model.ffn, model.vocab
    qd = model.n_q_heads * model.head_dim
    rows = {QKV: (model.n_q_heads + 2 * model.n_kv_heads) * model.head_dim,
            OPROJ: H, GATEUP: 2 * F, DOWN: H, LMHEAD: V}
    K = {QKV: H, OPROJ: qd, GATEUP: H, DOWN: F, LMHEAD: H}
    for kind in (QKV, OPROJ, GATEUP, DOWN, LMHEAD):
        layers = [model.n_layers - 1] if kind == LMHEAD else range(model.n_layers)
        for l in layers:
            ts = sorted((t for t in tasks if t["kind"] == kind and t["layer"] == l),
                        key=lambda t: t["row0"])
            assert ts[0]["row0"] == 0 and ts[-1]["row1"] == rows[kind]
            for a, b in zip(ts, ts[1:]):
                assert a["row1"] == b["row0"]
            tpr = 32
            while tpr < K[kind] // 8 and tpr < 512:
                tpr *= 2
            cap = min(1024, 20480 // (4 * (tpr // 32)))
            assert all(0 < t["row1"] - t["row0"] <= cap for t in ts)
            if kind in (QKV, GATEUP):
                assert all(t["row0"] % 2 == 0 and t["row1"] % 2 == 0 for t in ts)
            # one CTA's share stays within one row range of the stage
            assert len({t["cta"] for t in ts}) == min(P, len({t["cta"] for t in ts}))
    info = plan.info
    wb = model.n_layers * (rows[QKV] * H + H * qd + 2 * F * H + H * F) * 2 + V * H * 2
    assert info.weight_bytes_per_step == wb


def test_llama8b_weight_bytes_match_the_shape():
    # bf16 matrices of the Llama-3-8B shape: 32 x 218,103,808 + 128,256 x 4,096 elements.
    plan = binding.Plan(synth.LLAMA8B, 600, 148)
    assert plan.info.weight_bytes_per_step == 15_009_316_864


@pytest.mark.parametrize("model", [synth.TINY, synth.QWEN05B, synth.LLAMA8B],
                         ids=lambda m: m.name)
def test_qkv_packing_is_a_bijection_with_rope_pairs_adjacent(model):
    d, nq, nkv = model.head_dim, model.n_q_heads, model.n_kv_heads
    G = nq // nkv
    n = (nq + 2 * nkv) * d
    seen = set()
    for r in range(n):
        w, h, dim = binding.qkv_row_source(model, r)
        seen.add((w, h, dim))
        g = r // ((G + 2) * d)
        assert (h // G if w == 0 else h) == g
        if w < 2 and r % 2 == 1:
            w0, h0, d0 = binding.qkv_row_source(model, r - 1)
            assert (w0, h0) == (w, h) and dim == d0 + d // 2
    want = {(0, h, i) for h in range(nq) for i in range(d)} | \
           {(w, h, i) for w in (1, 2) for h in range(nkv) for i in range(d)}
    assert seen == want
