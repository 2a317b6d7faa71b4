"""Decode-step benchmark: one JSON line per run.

Workload: Llama-3-8B-shaped decoder (32 layers, hidden 4096, 32 q / 8 KV
heads, head_dim 128, SwiGLU 14336, vocab 128256), bf16 random-init weights
N(0, 0.02), batch 1, 39-token random prompt, then greedy decoding.  A "step"
is one decode step: one token through the whole model (one persistent
kernel launch).  W untimed warm-up steps, then exactly K timed steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

--impl reference times the CPU oracle (the only reference this method has)
on the host's cores on a bounded sample of the same workload.
Multi-GPU (under torchrun): independent replicas, one request per GPU, no
collective on the data path; time = max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode ms/token (batch 1, Llama-3-8B-shape) & achieved HBM GB/s vs 8 TB/s peak"
NOMINAL_HBM = 8000.0   # GB/s, the metric's denominator
SHORT_PROMPT = 39      # the 39-token prompt, 512 greedy steps workload
LONG_PROMPT = 32768    # the long-context workload: 32768-token prompt, 256 steps
LONG_STEPS = 256


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus, backend: str = "nccl"):
    """Rank, world size and local rank from the launcher's environment; with
    more than one rank, a process group (NCCL on the GPUs; gloo for the CPU
    tests of this host logic) with a short timeout."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def per_token_ms(total_ms_max: float, steps: int, world: int) -> float:
    """Whole-job ms per token of N independent replicas: every rank decodes
    `steps` tokens, the job ends with the slowest rank (max over ranks)."""
    return total_ms_max / (steps * world)


def run_reference(args):
    """The oracle as it stands, timed on the host's cores on the megakernel
    arm's workload (same metric, unit and config): W untimed and K timed
    steps, a step decoding one token of every request at the positions the
    megakernel arm decodes.  So that any K finishes within the time budget
    (MK_REF_BUDGET_S, default 120 s), a step may run the oracle on the model's
    first Ls layers (with its final norm and LM head); each request's time
    then scales to the whole model by the ratio of the two decode steps'
    algorithmic bytes (the oracle's GEMVs stream its weights from host
    memory).  The cache positions before the first decoded one hold random
    values: the timing does not depend on them."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    from persistent_megakernel_03_b200 import roofline, synth
    spec = workload_spec(args)
    model, lens, n, W, K = spec.model, spec.lens, spec.n, spec.W, spec.K
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = synth.make_model(model, 0, device=dev)
    w_cpu = {k: v.cpu() for k, v in w.items()}
    del w
    budget = float(os.environ.get("MK_REF_BUDGET_S", "120"))
    rng = np.random.default_rng(0)

    def states(m):
        om = oracle.OracleModel(m, w_cpu)
        sts = []
        for r in range(n):
            st = om.new_state(lens[r] + W + K + 1)
            fill = rng.standard_normal((lens[r], m.head_dim), dtype=np.float32)
            for l in range(m.n_layers):
                for g in range(m.n_kv_heads):
                    for which in (0, 1):
                        st.set_kv(l, g, which, fill)
            sts.append(st)
        return om, sts

    def step(om, sts, j):
        """One step (positions lens[r] + j); per-request seconds."""
        out = []
        for r in range(n):
            t0 = time.perf_counter()
            om.decode(sts[r], 1, lens[r] + j, want_logits=False)
            out.append(time.perf_counter() - t0)
        return out

    def nbytes(m, p):
        return roofline.step_bytes(m, [p])

    # the depth Ls whose W + K steps fit the budget, from a one-layer probe
    m1 = model.with_layers(1)
    om, sts = states(m1)
    step(om, sts, 0)
    t1 = sum(step(om, sts, 1))
    del om, sts
    per_step_full = t1 * nbytes(model, lens[0]) / nbytes(m1, lens[0])
    Ls = model.n_layers
    while Ls > 1 and (W + K) * per_step_full * nbytes(model.with_layers(Ls), lens[0]) / \
            nbytes(model, lens[0]) > budget:
        Ls -= 1
    m_run = model if Ls == model.n_layers else model.with_layers(Ls)
    om, sts = states(m_run)
    scaled = []
    for j in range(W + K):
        per_req = step(om, sts, j)
        if j >= W:
            scaled.append(sum(t * nbytes(model, lens[r] + j) / nbytes(m_run, lens[r] + j)
                              for r, t in enumerate(per_req)))
    cores = oracle.num_threads()
    ms = 1e3 * sum(scaled) / len(scaled)
    depth = (f"all {model.n_layers} layers" if Ls == model.n_layers else
             f"the first {Ls} of {model.n_layers} layers with the final norm and LM head, "
             f"scaled to the whole model by the algorithmic bytes")
    sample = (f"{K} oracle steps ({W} untimed before them) of the {spec.shape_cap} model "
              f"at the megakernel arm's positions, {depth}; fp32 with bf16 weights widened "
              f"on the fly, {cores} OpenMP threads"
              + (f"; one decode per request, {n} requests per step" if n > 1 else ""))
    line = {
        "impl": "reference", "metric": spec.metric, "value": ms, "unit": spec.unit,
        "n_gpus": args.gpus, "steps": K, "warmup": W, "ms_per_step": ms,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": spec.workload, "sample": "bounded oracle sample"},
        "cpu_baseline": {"value": ms, "unit": spec.unit, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": ms, "unit": spec.unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def load_traffic(workload):
    """DRAM traffic per launch from the committed ncu summary, when it was
    taken on the current kernel sources and scaled to this workload."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "megakernel_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for name in ("step_kernel.cuh", "step_bf16_d128.cu", "mk_internal.h", "ptx.cuh",
                 "attn_math.cuh"):
        with open(os.path.join(ROOT, "persistent_megakernel_03_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    if rec.get("source_sha256") != h.hexdigest() or rec.get("workload") != workload:
        return None
    return rec.get("traffic_bytes_per_launch_full")


def workload_spec(args):
    """The model, prompt lengths, step counts, metric, unit and workload
    description of one workload, as both arms report it."""
    from types import SimpleNamespace

    from persistent_megakernel_03_b200 import synth
    qwen = args.workload == "qwen05b"
    model = synth.QWEN05B if qwen else synth.LLAMA8B
    shape = "qwen2.5-0.5b-shape" if qwen else "llama-3-8b-shape"
    shape_cap = "Qwen2.5-0.5B-shape" if qwen else "Llama-3-8B-shape"
    if args.layers:
        model = model.with_layers(args.layers)
    W, K = args.warmup, args.steps
    if args.workload == "llama8b-32k":
        lens = [LONG_PROMPT]
    elif args.workload == "llama8b-batch8":
        lens = list(synth.packed_batch_lengths())
    else:
        lens = [SHORT_PROMPT]
    n = len(lens)
    if args.workload in ("llama8b-32k", "llama8b-batch8") and W + K > LONG_STEPS:
        K = LONG_STEPS - W   # these workloads decode 256 steps after their prompts
    if n == 1:
        workload = (f"{shape} decode, batch 1, {lens[0]}-token random prompt, "
                    f"greedy decode steps {lens[0] + W}..{lens[0] + W + K - 1} timed")
        unit = "ms/token"
        metric = METRIC if model.name.startswith("llama") else (
            f"decode ms/token (batch 1, {shape_cap}) & achieved HBM GB/s vs 8 TB/s peak")
    else:
        workload = (f"llama-3-8b-shape decode, {n} requests per step, random prompts of "
                    f"{lens} tokens packed with offsets, greedy decode steps {W}..{W + K - 1} "
                    "after each prompt timed; one batched step per token (tcgen05 GEMMs over "
                    "the requests' columns, each weight matrix streamed once; CUDA graph)")
        unit, metric = "ms/step", f"decode ms/step ({n} requests, Llama-3-8B-shape)"
    return SimpleNamespace(name=args.workload, model=model, shape=shape, shape_cap=shape_cap,
                           lens=lens, n=n, W=W, K=K, workload=workload, unit=unit,
                           metric=metric)


# The other workloads the default run measures next to the headline one, each
# as a sub-record of the same JSON line: (workload, weights).
SUB_WORKLOADS = (("qwen05b", "bf16"), ("llama8b-batch8", "bf16"), ("llama8b-32k", "bf16"),
                 ("llama8b", "fp8"))


def oracle_steps(model, w_cpu, lens, first_step: int, n_steps: int, budget_s: float):
    """The oracle's decode step timed on host cores at the positions the GPU
    arm times (lens[r] + first_step + j for request r), one decode per request
    per step; the cache rows before hold random values (the timing does not
    depend on them).  Stops early once budget_s of steps ran (at least 2).
    Returns per-step seconds (summed over requests) and the thread count."""
    import numpy as np

    import oracle
    om = oracle.OracleModel(model, w_cpu)
    rng = np.random.default_rng(0)
    states = []
    for n0 in lens:
        p0 = n0 + first_step
        st = om.new_state(p0 + n_steps + 1)
        fill = rng.standard_normal((p0, model.head_dim), dtype=np.float32)
        for l in range(model.n_layers):
            for g in range(model.n_kv_heads):
                for which in (0, 1):
                    st.set_kv(l, g, which, fill)
        states.append((st, p0))
    times = []
    t_all = time.perf_counter()
    for j in range(n_steps):
        t0 = time.perf_counter()
        for st, p0 in states:
            om.decode(st, 1, p0 + j, want_logits=False)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_all > budget_s and len(times) >= 2:
            break
    return times, oracle.num_threads()


def measure(spec, w, fp8: bool, world: int, local: int, *, full: bool, w_cpu=None,
            cpu_budget_s: float = 25.0, trace_path=None, l2_prefetch: int = 0,
            layers_flag: int = 0, prefill_per_operator: int = 0) -> dict:
    """One workload on one decoder: W untimed and K device-timed decode steps
    (CUDA events on the launching stream, barrier + synchronize around them,
    max over ranks), the same steps end to end through the host entry point,
    the per-operator CUDA-graph baseline, clocks during the timed region and,
    with w_cpu, the oracle on host cores at the same positions.  full adds the
    per-operator baseline, the device-resident loop, the read probe and the
    optional per-task trace."""
    import numpy as np
    import torch

    from persistent_megakernel_03_b200 import binding, roofline, synth
    model, lens, n, W, K = spec.model, spec.lens, spec.n, spec.W, spec.K
    max_seq = max(lens) + W + K + 1
    wbytes = 1 if fp8 else 2
    stream = torch.cuda.current_stream()
    dec = binding.Decoder(model, w, max_seq, max_batch=n, stream=stream,
                          prefill_per_operator=prefill_per_operator,
                          l2_prefetch=l2_prefetch, weight_format=1 if fp8 else 0)
    torch.cuda.empty_cache()
    if n == 1:
        prompt, offs = synth.make_prompt(lens[0], model.vocab), [0, lens[0]]
    else:
        prompt, offs = synth.make_packed_prompts(lens, model.vocab)
        offs = offs.tolist()
    prompt = prompt.to(torch.int32).cuda()
    ids = [torch.zeros(n, dtype=torch.int32, device="cuda") for _ in range(2)]
    first_id, prefill_ms = [], []

    def prefill():
        # Decode steps write the cache only at positions past each prompt, so
        # after the first prefill the prompts' cache stays valid: later
        # "prefills" only restore the first generated ids.
        if not first_id:
            # twice: the first call includes one-time setup (scratch, tensor
            # maps, module loading); the second rewrites the same cache rows
            for _ in range(2):
                pe0 = torch.cuda.Event(enable_timing=True)
                pe1 = torch.cuda.Event(enable_timing=True)
                pe0.record(stream)
                dec.prefill(prompt, offs, None, ids[0])
                pe1.record(stream)
                torch.cuda.synchronize()
                prefill_ms.append(pe0.elapsed_time(pe1))
            first_id.append(ids[0].clone())
        else:
            ids[0].copy_(first_id[0])

    def positions(step):
        return [lens[r] + step for r in range(n)]

    def run_steps(first_step, count, evs=None):
        for k in range(count):
            dec.decode(ids[k % 2], positions(first_step + k), None, ids[(k + 1) % 2])
            if evs is not None:
                evs[k + 1].record(stream)

    def check():
        rc = dec.status()
        if rc != 0:
            raise RuntimeError(f"device status {rc}: {dec.last_error()}")

    # ---- device-timed region (megakernel, or the batched step for n > 1)
    prefill()
    run_steps(0, W)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    torch.cuda.synchronize()
    barrier(world)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        evs[0].record(stream)
        run_steps(W, K, evs)
        torch.cuda.synchronize()
    barrier(world)
    check()
    per_step = [evs[k].elapsed_time(evs[k + 1]) for k in range(K)]
    total_ms = max_over_ranks(evs[0].elapsed_time(evs[K]), world)
    value = per_token_ms(total_ms, K, world)
    bytes_mean = sum(roofline.step_bytes(model, positions(W + k), wbytes=wbytes)
                     for k in range(K)) / K
    achieved = bytes_mean / ((sum(per_step) / K) * 1e-3) / 1e9
    peak, peak_src = measured_peaks()
    rec = {
        "workload": spec.workload, "metric": spec.metric, "unit": spec.unit, "value": value,
        "steps": K, "warmup": W, "ms_per_step": total_ms / K,
        "weights": "fp8 e4m3, one power-of-two scale per row" if fp8 else "bf16",
        "tok_per_s": 1e3 * n / value,
        "step_ms": {"median": statistics.median(per_step),
                    "p10": float(np.percentile(per_step, 10)),
                    "p90": float(np.percentile(per_step, 90))},
        "achieved_gbs": achieved, "frac_of_8tbs": achieved / NOMINAL_HBM,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_src,
                     "traffic": (load_traffic(spec.name)
                                 if n == 1 and not fp8 and not layers_flag else None),
                     "bytes_per_launch": bytes_mean},
        "clocks": clk.summary(),
        "prefill": {"ms": prefill_ms[1], "first_call_ms": prefill_ms[0],
                    "positions": int(sum(lens)),
                    "positions_per_s": float(sum(lens)) / (prefill_ms[1] * 1e-3),
                    "path": ("one persistent kernel per block of <= 2048 positions (tcgen05 GEMM "
                             "and attention tasks), each prompt's last position with its LM head "
                             "and greedy id inside the kernel when its tile has room; ms: a second "
                             "call, first_call_ms: the first, setup included")},
        # one persistent launch per step; the batched step's graph holds an
        # embedding kernel, 7 kernels per layer and 3 for the LM head and argmax
        "gpu_launches": K if n == 1 else K * (7 * model.n_layers + 4),
    }
    if n > 1:
        rec["roofline"]["bytes_note"] = ("algorithmic bytes: weights once per step plus every "
                                         "request's KV")

    # ---- the device-resident loop: the same K steps in one persistent launch
    if full and n == 1 and world == 1:
        prefill()
        run_steps(0, W)
        seq = torch.empty(K, dtype=torch.int32, device="cuda")
        le = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        torch.cuda.synchronize()
        le[0].record(stream)
        dec.decode_steps(ids[W % 2], lens[0] + W, K, seq)
        le[1].record(stream)
        torch.cuda.synchronize()
        check()
        rec["device_loop"] = {"ms_per_token": le[0].elapsed_time(le[1]) / K,
                              "steps_per_launch": K}

    # ---- read-stream probe: practical read ceiling on this GPU
    if full:
        probe_buf = torch.empty(4 * 2**30, dtype=torch.uint8, device="cuda")
        sink = torch.zeros(1, dtype=torch.int64, device="cuda")
        for _ in range(3):
            binding.read_probe(probe_buf, sink)
        pe = [torch.cuda.Event(enable_timing=True) for _ in range(11)]
        pe[0].record(stream)
        for i in range(10):
            binding.read_probe(probe_buf, sink)
            pe[i + 1].record(stream)
        torch.cuda.synchronize()
        probe_gbs = max(probe_buf.numel() / (pe[i].elapsed_time(pe[i + 1]) * 1e-3) / 1e9
                        for i in range(10))
        del probe_buf
        rec["read_probe_gbs"] = probe_gbs
        rec["frac_of_read_probe"] = achieved / probe_gbs

    # ---- baselines: the same task bodies, one launch per operator (requests in turn)
    baselines = {}
    nb = min(K, 64 if full else 16)
    modes = (("per_op", binding.MODE_PER_OP), ("per_op_graph", binding.MODE_PER_OP_GRAPH))
    for name, mode in (modes if full else modes[1:]):
        dec.set_mode(mode)
        prefill()
        run_steps(0, min(W, 4))
        bev = [torch.cuda.Event(enable_timing=True) for _ in range(nb + 1)]
        torch.cuda.synchronize()
        bev[0].record(stream)
        run_steps(min(W, 4), nb, bev)
        torch.cuda.synchronize()
        steps_ms = [bev[k].elapsed_time(bev[k + 1]) for k in range(nb)]
        baselines[name] = {"ms_per_token": statistics.median(steps_ms) / n, "steps": nb,
                           "launches_per_step": n * (5 * model.n_layers + 1)}
    dec.set_mode(binding.MODE_MEGAKERNEL)
    check()
    rec["baselines"] = baselines

    # ---- end to end through the host entry point (tokens in, ids out, per step)
    prefill()
    torch.cuda.synchronize()
    toks = [int(v) for v in ids[0].tolist()]
    for k in range(W):
        toks = dec.decode_host(toks, positions(k))
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for k in range(K):
        toks = dec.decode_host(toks, positions(W + k))
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world) / (K * world)
    rec["e2e"] = {"value": e2e_ms, "unit": spec.unit,
                  "h2d_bytes_per_step": 4 * n, "d2h_bytes_per_step": 4 * n,
                  "api": "mk_decode_step_host (pinned host buffers, one sync per step)"}

    if trace_path and n == 1:
        # a few more steps with the per-task timeline on (not part of the timing)
        from persistent_megakernel_03_b200 import trace as mktrace
        plan = binding.Plan(model, max_seq, dec_num_ctas())
        tbuf = torch.zeros((plan.info.n_tasks, 8), dtype=torch.int64, device="cuda")
        prefill()
        run_steps(0, W)
        dec.set_trace(tbuf)
        run_steps(W, 1)
        torch.cuda.synchronize()
        dec.set_trace(None)
        rows = tbuf.cpu().numpy().astype("uint64").tolist()
        summary = mktrace.summarize(rows, plan.tasks())
        with open(trace_path, "w") as f:
            json.dump(summary, f, indent=1)
        rec["trace"] = {k: summary[k] for k in ("step_us", "mean_cta_busy_frac")}
    dec.close()
    del dec
    torch.cuda.empty_cache()

    # ---- the oracle on the host's cores at the same positions
    if w_cpu is not None:
        times, cores = oracle_steps(model, w_cpu, lens, W, 3, cpu_budget_s)
        timed = times[1:] if len(times) > 1 else times
        cms = 1e3 * sum(timed) / len(timed)
        j0 = W + len(times) - len(timed)
        pos_txt = (f"{lens[0] + j0}..{lens[0] + W + len(times) - 1}" if n == 1 else
                   f"prompt length + {j0}..{W + len(times) - 1} for each of the {n} requests")
        rec["cpu_baseline"] = {
            "value": cms, "unit": spec.unit, "cores": cores, "kind": "oracle",
            "sample": f"{len(timed)} oracle decode steps of the same {spec.shape_cap} model "
                      f"at positions {pos_txt} (the GPU arm's first timed positions; cache "
                      "rows before them hold random values, the timing does not depend on "
                      "them), fp32 with bf16 weights widened on the fly"
                      + (" (for the fp8 workload the bf16 weights before quantization: the "
                         "oracle's time does not depend on the values)" if fp8 else "")
                      + (f"; one decode per request, {n} requests per step" if n > 1 else "")}
    return rec


def run_mk(args):
    import torch

    from persistent_megakernel_03_b200 import roofline, synth

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    spec = workload_spec(args)
    model = spec.model
    fp8 = args.weights == "fp8"
    w = synth.make_model(model, 0, device="cuda")
    cpu = world == 1 and rank == 0 and not args.no_cpu_baseline
    w_cpu = {k: v.cpu() for k, v in w.items()} if cpu else None
    rec = measure(spec, w, fp8, world, local, full=True, w_cpu=w_cpu, trace_path=args.trace,
                  l2_prefetch=args.l2_prefetch, layers_flag=args.layers,
                  prefill_per_operator=1 if args.prefill_per_operator else 0)
    line = {
        "metric": spec.metric, "value": rec["value"], "unit": spec.unit, "n_gpus": world,
        "steps": spec.K, "warmup": spec.W, "ms_per_step": rec["ms_per_step"],
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "weights": rec["weights"], "data": "synthetic",
        "config": {"workload": spec.workload,
                   "l2": (f"inputs larger than L2 ({roofline.weight_bytes(model, 1 if fp8 else 2) / 1e9:.2f} "
                          "GB of weights streamed per step)"),
                   "parallelism": f"replicas x{world}"},
    }
    for k, v in rec.items():
        if k not in ("workload", "metric", "unit", "value", "steps", "warmup", "ms_per_step",
                     "weights"):
            line[k] = v
    if args.layers:
        line["config"]["workload"] += f" [profiling case: {args.layers} layers]"
    if args.l2_prefetch:
        line["config"]["l2_prefetch_chunks"] = args.l2_prefetch
    if args.prefill_per_operator:
        line["config"]["prefill"] = "one launch per operator (profiling aid)"
    # ---- the other workloads, each a sub-record (1 GPU only; not with --layers)
    if (world == 1 and not args.no_workloads and not args.layers and args.workload == "llama8b"
            and not fp8):
        subs = {}
        k_sub = max(16, min(args.steps, 64))
        for wl, wts in SUB_WORKLOADS:
            sargs = argparse.Namespace(workload=wl, layers=0, steps=k_sub, warmup=args.warmup)
            sspec = workload_spec(sargs)
            if sspec.model is model:
                sw, sw_cpu = w, w_cpu
            else:
                sw = synth.make_model(sspec.model, 0, device="cuda")
                sw_cpu = {k: v.cpu() for k, v in sw.items()} if cpu else None
            key = wl + ("-fp8" if wts == "fp8" else "")
            subs[key] = measure(sspec, sw, wts == "fp8", world, local, full=False,
                                w_cpu=sw_cpu, cpu_budget_s=12.0)
            if sw is not w:
                del sw, sw_cpu
            torch.cuda.empty_cache()
        line["workloads"] = subs
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def dec_num_ctas() -> int:
    import torch
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=504)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="mk", choices=["mk", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="only the selected workload (no sub-records of the other ones)")
    ap.add_argument("--trace", default=None, help="write a per-task timeline summary here")
    ap.add_argument("--l2-prefetch", type=int, default=0,
                    help="ring chunks prefetched into L2 beyond the ring (0: library default)")
    ap.add_argument("--workload", default="llama8b",
                    choices=["llama8b", "llama8b-32k", "llama8b-batch8", "qwen05b"],
                    help="llama8b: 39-token prompt (default); llama8b-32k: 32768-token "
                         "prompt; llama8b-batch8: 8 requests with prompts of U[32, 2048] "
                         "tokens (these two decode at most 256 steps); qwen05b: the "
                         "Qwen2.5-0.5B shape, 39-token prompt")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "fp8"],
                    help="fp8: the row-quantized e4m3 model through the fp8 decode path "
                         "(not the headline configuration)")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling aid: a shallower model of the same widths (not a bench line)")
    ap.add_argument("--prefill-per-operator", action="store_true",
                    help="profiling aid: the prefill as one launch per operator (its kernels "
                         "become launches of their own), not the persistent prefill kernel")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_mk(args)


if __name__ == "__main__":
    main()
