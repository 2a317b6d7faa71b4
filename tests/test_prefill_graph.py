"""The persistent prefill's layout and task graph, on the host (no GPU).

mk_prefill_layout returns the order in which a call's prompt positions go
through the kernel (every position but each prompt's last, then the last
positions that fit the final block's last 128-position tile) and the
attention runs of each block; mk_prefill_graph returns the graph one block
gets: its tasks
(kind, layer, 128-position tile, a, b, wait event, wait count, signalled
events) and the per-CTA queues.  The kernel runs each CTA's queue in order,
a task starting once its event reached its wait count ("LLMs in einen
MegaKernel kompilieren ...", "Ereignisbasierte Ausführung").  These tests run
the queues in a simulator -- CTAs advancing in random interleavings -- and
check that every graph finishes (no CTA waits for a task queued behind it),
that every wait count is exactly what its event finally receives (a lower
count would let a task start before its inputs are complete), and the
dependency structure the kernel relies on.
"""
import random

import pytest

from persistent_megakernel_03_b200 import binding, synth

KIND_NORM, KIND_GEMM, KIND_ROPE, KIND_ATTN, KIND_RES1, KIND_SWIGLU, KIND_RES2 = range(7)
MAT_QKV, MAT_O, MAT_GU, MAT_DN, MAT_LM = range(5)
TILE = 128


def _block(lens, max_tokens=2048, block=0):
    """Block `block` of a call with these prompt lengths, as the library lays
    it out (mk_prefill_layout): (positions T, attention runs, request per
    position or -1)."""
    offs = [0]
    for n in lens:
        offs.append(offs[-1] + n)
    positions, runs, _ = binding.prefill_layout(offs, list(range(len(lens))), max_tokens)
    b0 = block * max_tokens
    blk = positions[b0:b0 + max_tokens]
    tiles = [r[1:] for r in runs if r[0] == block]
    return len(blk), tiles, [p[3] for p in blk]


def _simulate(rows, qoff, queue, n_events, rng):
    events = [0] * n_events
    waiters = {}
    ptr = [qoff[c] for c in range(len(qoff) - 1)]
    end = qoff[1:]
    done_order = []
    while True:
        ready = [c for c in range(len(ptr)) if ptr[c] < end[c] and
                 (rows[queue[ptr[c]]][5] < 0 or events[rows[queue[ptr[c]]][5]] >= rows[queue[ptr[c]]][6])]
        if not ready:
            break
        c = rng.choice(ready)
        ti = queue[ptr[c]]
        ptr[c] += 1
        kind, layer, n, a, b, wev, wcnt, sig0, nsig = rows[ti]
        if wev >= 0:
            waiters.setdefault(wev, set()).add(wcnt)
        for e in range(sig0, sig0 + nsig):
            events[e] += 1
        done_order.append(ti)
    stuck = [c for c in range(len(ptr)) if ptr[c] < end[c]]
    return events, waiters, done_order, stuck


CASES = [
    ("one prompt", [300]),
    ("tile-aligned prompt", [129]),
    ("eight requests", [5, 170, 9, 300, 1, 129, 23, 64]),
    ("many short", [2, 3, 4, 5, 6, 7, 8, 9]),
]


@pytest.mark.parametrize("name,lens", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("num_ctas", [1, 7, 148])
def test_graph_finishes_and_every_wait_count_is_exact(name, lens, num_ctas):
    model = synth.TINY
    T, tiles, lm = _block(lens)
    rows, qoff, queue, n_events = binding.prefill_graph(model, T, tiles, lm, num_ctas)
    assert sorted(queue) == list(range(len(rows)))          # every task queued once
    for c in range(num_ctas):                               # queues keep the graph's order
        q = queue[qoff[c]:qoff[c + 1]]
        assert q == sorted(q)
    for seed in range(3):
        events, waiters, order, stuck = _simulate(rows, qoff, queue, n_events, random.Random(seed))
        assert not stuck, f"CTAs {stuck[:5]} never finish"
        for e, counts in waiters.items():
            assert counts == {events[e]}, (e, counts, events[e])


def test_dependencies_follow_the_tiles():
    model = synth.TINY
    lens = [5, 170, 9, 300, 1, 129, 23, 64]
    T, tiles, lm = _block(lens)
    rows, qoff, queue, n_events = binding.prefill_graph(model, T, tiles, lm, 148)
    n_tiles = (T + TILE - 1) // TILE
    producers = {}
    for i, r in enumerate(rows):
        for e in range(r[7], r[7] + r[8]):
            producers.setdefault(e, []).append(i)
    L = model.n_layers
    for i, (kind, layer, n, a, b, wev, wcnt, sig0, nsig) in enumerate(rows):
        deps = [rows[j] for j in producers.get(wev, [])] if wev >= 0 else []
        if kind == KIND_GEMM and a == MAT_QKV:
            # the attention norms of its own tile only (layer 0: the embedding tasks)
            assert all(d[2] == n for d in deps) and len(deps) == 16
            assert all(d[0] == (KIND_NORM if layer == 0 else KIND_RES2) for d in deps)
        if kind == KIND_ATTN:
            # the RoPE of every tile up to its own, and nothing else
            assert all(d[0] == KIND_ROPE and d[1] == layer for d in deps)
            assert {d[2] for d in deps} == set(range(n + 1))
        if kind == KIND_GEMM and a == MAT_O:
            assert all(d[0] == KIND_ATTN and d[2] == n and d[1] == layer for d in deps)
        if kind == KIND_GEMM and a == MAT_LM:
            # only tiles holding a prompt's last position, after the last layer's norms
            assert layer == L
            assert any(lm[t] >= 0 for t in range(n * TILE, min(T, (n + 1) * TILE)))
            assert all(d[0] == KIND_RES2 and d[1] == L - 1 and d[2] == n for d in deps)
    # every elementwise stage: 16 eight-position tasks per tile and layer
    for kind in (KIND_ROPE, KIND_RES1, KIND_SWIGLU, KIND_RES2):
        for l in range(L):
            assert sum(1 for r in rows if r[0] == kind and r[1] == l) == 16 * n_tiles
    # attention: one task per run and query head
    assert sum(1 for r in rows if r[0] == KIND_ATTN and r[1] == 0) == len(tiles) * model.n_q_heads
    assert sum(1 for r in rows if r[0] == KIND_GEMM and r[3] == MAT_LM) == \
        (model.vocab + 127) // 128 * len({t // TILE for t in range(T) if lm[t] >= 0})


def test_no_lm_head_without_a_folded_position():
    model = synth.TINY
    T, tiles, lm = _block([129, 257])     # 128 + 256 positions: no room in the final tile
    assert all(v < 0 for v in lm)
    rows, _, _, _ = binding.prefill_graph(model, T, tiles, lm, 16)
    assert not any(r[0] == KIND_GEMM and r[3] == MAT_LM for r in rows)


def test_rejects_a_run_across_tiles():
    with pytest.raises(binding.MkError):
        binding.prefill_graph(synth.TINY, 200, [(100, 60, 0, 100)], [-1] * 200, 4)


def _random_call(rng):
    n_req = rng.randint(1, 8)
    lens = [rng.choice([1, 2, rng.randint(1, 40), rng.randint(100, 700), rng.randint(1000, 3000)])
            for _ in range(n_req)]
    slots = rng.sample(range(16), n_req)
    return lens, slots, rng.choice([2048, 2048, 1000, 302, 128])


@pytest.mark.parametrize("seed", range(40))
def test_layout_takes_every_position_once_and_folds_only_into_room(seed):
    rng = random.Random(seed)
    lens, slots, B = _random_call(rng)
    offs = [0]
    for n in lens:
        offs.append(offs[-1] + n)
    positions, runs, folded = binding.prefill_layout(offs, slots, B)
    # every position but each prompt's last, in request order
    body = [(offs[r] + p, slots[r], p, -1) for r in range(len(lens)) for p in range(lens[r] - 1)]
    N = len(body)
    assert positions[:N] == body
    # then last positions of prompts of two or more positions, in request order
    tail = positions[N:]
    eligible = [r for r in range(len(lens)) if lens[r] >= 2]
    assert [p[3] for p in tail] == eligible[:len(tail)]
    for tok, slot, pos, r in tail:
        assert (tok, slot, pos) == (offs[r + 1] - 1, slots[r], lens[r] - 1)
    assert folded == [r in {p[3] for p in tail} for r in range(len(lens))]
    if N == 0:
        assert not tail
        assert not runs
        return
    total = len(positions)
    # folding adds neither a block nor a 128-position tile, and stops only
    # when every eligible prompt is in or the final tile is full
    blocks = lambda n: (n + B - 1) // B
    assert blocks(total) == blocks(N)
    last_n, last_t = N - (blocks(N) - 1) * B, total - (blocks(N) - 1) * B
    assert (last_t + 127) // 128 == (last_n + 127) // 128
    assert len(tail) == len(eligible) or last_t % 128 == 0 or last_t == B
    # attention runs: cover each block in order, one request and consecutive
    # positions inside one 128-position tile, a new run only where the tile or
    # the request changes
    for b in range(blocks(total)):
        T = min(B, total - b * B)
        rs = [r for r in runs if r[0] == b]
        t = 0
        for k, (_, first, count, slot, p0) in enumerate(rs):
            assert first == t and count >= 1
            assert first // 128 == (first + count - 1) // 128
            for i in range(count):
                _, s_, p_, _ = positions[b * B + first + i]
                assert (s_, p_) == (slot, p0 + i)
            if k > 0:
                prev = rs[k - 1]
                assert first % 128 == 0 or prev[3] != slot
            t += count
        assert t == T


@pytest.mark.parametrize("seed", range(6))
def test_graphs_of_random_calls_finish(seed):
    # layout and graph together, as mk_prefill launches them: every block of a
    # random call, 148 CTAs
    rng = random.Random(100 + seed)
    lens, _, B = _random_call(rng)
    n_blocks = (sum(max(n - 1, 0) for n in lens) + B - 1) // B
    for block in range(n_blocks):
        T, tiles, lm = _block(lens, B, block)
        rows, qoff, queue, n_events = binding.prefill_graph(synth.TINY, T, tiles, lm, 148)
        events, waiters, order, stuck = _simulate(rows, qoff, queue, n_events, rng)
        assert not stuck
        for e, counts in waiters.items():
            assert counts == {events[e]}


def test_layout_rejects_decreasing_offsets():
    with pytest.raises(binding.MkError):
        binding.prefill_layout([0, 10, 5], [0, 1], 2048)


def test_graph_rejects_an_invalid_shape():
    import dataclasses
    bad = dataclasses.replace(synth.TINY, head_dim=96)
    with pytest.raises(binding.MkError):
        binding.prefill_graph(bad, 10, [(0, 10, 0, 0)], [-1] * 10, 4)
