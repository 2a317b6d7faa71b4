"""ctypes binding of libmk (include/mk.h): argument marshalling only.

Every step of the decode path runs in libmk's CUDA kernels; this module only
converts Python / torch arguments to the C-ABI's plain pointers and sizes.
torch provides device memory and streams.  When libmk.so cannot be loaded the
binding raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, List, Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
# MK_LIBRARY selects another build of the library (A/B comparisons of builds).
LIB_PATH = os.environ.get("MK_LIBRARY") or os.path.join(HERE, "libmk.so")

MK_OK = 0
ERRORS = {-1: "MK_ERR_INVALID_ARG", -2: "MK_ERR_OOM", -3: "MK_ERR_CUDA", -4: "MK_ERR_TIMEOUT",
          -5: "MK_ERR_POS_RANGE", -6: "MK_ERR_NOT_RESIDENT", -7: "MK_ERR_POISONED",
          -8: "MK_ERR_TOKEN_RANGE", -9: "MK_ERR_UNSUPPORTED", -10: "MK_ERR_BOUNDS"}
MODE_MEGAKERNEL, MODE_PER_OP, MODE_PER_OP_GRAPH = 0, 1, 2
ACT_Q, ACT_ATTN, ACT_FFN, ACT_X = 0, 1, 2, 3
TASK_KINDS = ("QKV", "ATTN", "OPROJ", "GATEUP", "DOWN", "LMHEAD")

EXPORTS = ("mk_create", "mk_prefill", "mk_decode_step", "mk_decode_steps", "mk_decode_step_host",
           "mk_copy_hidden", "mk_copy_activation", "mk_prefill_slots", "mk_decode_step_slots",
           "mk_kv_release", "mk_kv_set_pages", "mk_kv_get_pages", "mk_kv_free_pages",
           "mk_build_flags",
           "mk_kv_pointer", "mk_copy_kv", "mk_set_mode", "mk_status", "mk_last_error",
           "mk_destroy", "mk_plan_build", "mk_plan_get_info", "mk_plan_get_tasks",
           "mk_plan_get_queue", "mk_plan_get_event_counts", "mk_plan_destroy",
           "mk_qkv_row_source", "mk_read_probe", "mk_set_trace", "mk_set_prefill_trace", "mk_inject_prefill_stall", "mk_prefill_graph",
           "mk_prefill_layout",
           "mk_attention_workspace_bytes", "mk_attention_decode",
           "mk_attention_decode_noalloc", "mk_inject_stall")


class MkError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


class Config(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("hidden", C.c_int), ("n_q_heads", C.c_int),
                ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
                ("vocab", C.c_int), ("rms_eps", C.c_float), ("rope_theta", C.c_double),
                ("qkv_bias", C.c_int), ("tied_embeddings", C.c_int), ("max_seq", C.c_int),
                ("max_batch", C.c_int)]


LAYER_FIELDS = ("attn_norm", "wq", "wk", "wv", "bq", "bk", "bv", "wo", "ffn_norm", "w_gate",
                "w_up", "w_down")


class LayerWeights(C.Structure):
    _fields_ = [(k, C.c_void_p) for k in LAYER_FIELDS]


class Weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("layers", C.POINTER(LayerWeights)),
                ("final_norm", C.c_void_p), ("lm_head", C.c_void_p)]


class Options(C.Structure):
    _fields_ = [("num_ctas", C.c_int), ("attn_splits", C.c_int), ("timeout_ms", C.c_int),
                ("mode", C.c_int), ("l2_prefetch", C.c_int), ("weight_format", C.c_int),
                ("batch_sequential", C.c_int), ("prefill_steps", C.c_int),
                ("kv_page_tokens", C.c_int), ("kv_pool_pages", C.c_int),
                ("prefill_per_operator", C.c_int), ("prefill_attention", C.c_int)]


class PlanInfo(C.Structure):
    _fields_ = [("num_ctas", C.c_int), ("n_tasks", C.c_int), ("n_events", C.c_int),
                ("n_stages", C.c_int), ("attn_splits", C.c_int), ("n_lm_tasks", C.c_int),
                ("ring_slots", C.c_int), ("slot_bytes", C.c_int), ("smem_bytes", C.c_int),
                ("threads_per_cta", C.c_int), ("weight_bytes_per_step", C.c_longlong)]


class PlanTask(C.Structure):
    _fields_ = [("kind", C.c_int), ("layer", C.c_int), ("row0", C.c_int), ("row1", C.c_int),
                ("req", C.c_int), ("wait_event", C.c_int), ("wait_count", C.c_int),
                ("signal_event0", C.c_int), ("n_signal", C.c_int), ("cta", C.c_int),
                ("stage", C.c_int)]


_lib = None


def lib(build_if_missing: bool = True):
    """Loads libmk.so (building it with nvcc when absent); raises on failure."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH) and build_if_missing and not os.environ.get("MK_LIBRARY"):
        from . import build as _build
        _build.build()
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmk.so not found at {LIB_PATH}; run the package build")
    L = C.CDLL(LIB_PATH)
    vp, ip, i = C.c_void_p, C.POINTER(C.c_int32), C.c_int
    L.mk_create.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.POINTER(Options), vp,
                            C.POINTER(vp)]
    L.mk_prefill.argtypes = [vp, vp, ip, i, vp, vp]
    L.mk_decode_step.argtypes = [vp, vp, ip, i, vp, vp]
    L.mk_decode_step_host.argtypes = [vp, ip, ip, i, ip]
    L.mk_decode_steps.argtypes = [vp, vp, i, i, vp, vp]
    L.mk_copy_hidden.argtypes = [vp, vp, i]
    L.mk_copy_activation.argtypes = [vp, i, vp, i]
    L.mk_prefill_slots.argtypes = [vp, vp, ip, ip, i, vp, vp]
    L.mk_decode_step_slots.argtypes = [vp, vp, ip, ip, i, vp, vp]
    L.mk_kv_release.argtypes = [vp, i]
    L.mk_kv_set_pages.argtypes = [vp, i, ip, i]
    L.mk_kv_get_pages.argtypes = [vp, i, ip, i]
    L.mk_kv_free_pages.argtypes = [vp]
    L.mk_build_flags.argtypes = []
    L.mk_build_flags.restype = i
    L.mk_kv_pointer.argtypes = [vp, i, i, i, i, C.POINTER(vp)]
    L.mk_copy_kv.argtypes = [vp, i, i, i, i, i, vp]
    L.mk_set_mode.argtypes = [vp, i]
    L.mk_status.argtypes = [vp]
    L.mk_last_error.argtypes = [vp]
    L.mk_last_error.restype = C.c_char_p
    L.mk_destroy.argtypes = [vp]
    L.mk_destroy.restype = None
    L.mk_inject_stall.argtypes = [vp, i]
    L.mk_inject_prefill_stall.argtypes = [vp, i]
    L.mk_prefill_graph.argtypes = [vp, i, vp, i, vp, i, vp, i, vp, vp, i, vp, vp]
    L.mk_prefill_layout.argtypes = [vp, vp, i, i, vp, i, vp, i, vp, vp, vp]
    L.mk_plan_build.argtypes = [C.POINTER(Config), C.POINTER(Options), i, C.POINTER(vp)]
    L.mk_plan_get_info.argtypes = [vp, C.POINTER(PlanInfo)]
    L.mk_plan_get_tasks.argtypes = [vp, C.POINTER(PlanTask), i]
    L.mk_plan_get_queue.argtypes = [vp, i, ip, i]
    L.mk_plan_get_event_counts.argtypes = [vp, ip, i]
    L.mk_plan_destroy.argtypes = [vp]
    L.mk_plan_destroy.restype = None
    L.mk_qkv_row_source.argtypes = [C.POINTER(Config), i, ip, ip, ip]
    L.mk_read_probe.argtypes = [vp, C.c_size_t, vp, vp]
    L.mk_set_trace.argtypes = [vp, vp]
    L.mk_set_prefill_trace.argtypes = [vp, vp, C.c_int]
    L.mk_attention_workspace_bytes.argtypes = [i, i, i]
    L.mk_attention_workspace_bytes.restype = C.c_size_t
    L.mk_attention_decode.argtypes = [vp, vp, vp, i, i, i, i, vp, vp, vp]
    L.mk_attention_decode_noalloc.argtypes = [vp, vp, vp, i, i, i, i, vp, vp]
    _lib = L
    return L


def make_config(model, max_seq: int, max_batch: int = 1) -> Config:
    return Config(model.n_layers, model.hidden, model.n_q_heads, model.n_kv_heads,
                  model.head_dim, model.ffn, model.vocab, float(model.rms_eps),
                  float(model.rope_theta), int(bool(model.qkv_bias)),
                  int(bool(model.tied_embeddings)), int(max_seq), int(max_batch))


def _ints(vals: Sequence[int]):
    return (C.c_int32 * len(vals))(*[int(v) for v in vals])


def _check(rc: int, h=None):
    if rc != MK_OK:
        msg = lib().mk_last_error(h).decode(errors="replace")
        raise MkError(rc, msg)


# ------------------------------------------------------------------ plan

def prefill_layout(offsets, slots, max_tokens: int):
    """How mk_prefill lays out a call's positions for the persistent prefill
    (host only, see mk_prefill_layout): (positions as rows of (token index,
    slot, position, request or -1), attention runs as rows of (block, first
    block position, count, slot, first position), folded flag per request)."""
    L = lib()
    n_req = len(offsets) - 1
    off_c = (C.c_int32 * len(offsets))(*[int(v) for v in offsets])
    sl_c = (C.c_int32 * n_req)(*[int(v) for v in slots])
    n_pos, n_runs = C.c_int(0), C.c_int(0)
    rc = L.mk_prefill_layout(off_c, sl_c, n_req, max_tokens, None, 0, None, 0, C.byref(n_pos),
                             C.byref(n_runs), None)
    if rc != MK_OK:
        raise MkError(rc, "mk_prefill_layout rejected the call")
    pos_c = (C.c_int32 * (4 * n_pos.value))()
    runs_c = (C.c_int32 * (5 * n_runs.value))()
    fold_c = (C.c_int32 * n_req)()
    _check(L.mk_prefill_layout(off_c, sl_c, n_req, max_tokens, pos_c, n_pos.value, runs_c,
                               n_runs.value, C.byref(n_pos), C.byref(n_runs), fold_c))
    positions = [tuple(pos_c[4 * t:4 * t + 4]) for t in range(n_pos.value)]
    runs = [tuple(runs_c[5 * i:5 * i + 5]) for i in range(n_runs.value)]
    return positions, runs, [bool(v) for v in fold_c]


def prefill_graph(model, T: int, tiles, lm_req, num_ctas: int):
    """The persistent prefill's task graph of one block (host only, see
    mk_prefill_graph): (tasks as rows of 9 ints, queue offsets, queues, number
    of events)."""
    L = lib()
    cfg = make_config(model, max(T, 1), 1)
    flat = [int(v) for t in tiles for v in t]
    tiles_c = (C.c_int32 * len(flat))(*flat)
    lm_c = (C.c_int32 * T)(*[int(v) for v in lm_req])
    n_tasks, n_events = C.c_int(0), C.c_int(0)
    rc = L.mk_prefill_graph(C.byref(cfg), T, tiles_c, len(tiles), lm_c, num_ctas, None, 0, None,
                            None, 0, C.byref(n_tasks), C.byref(n_events))
    if rc != MK_OK:
        raise MkError(rc, "mk_prefill_graph rejected the block")
    n = n_tasks.value
    tasks = (C.c_int32 * (9 * n))()
    qoff = (C.c_int32 * (num_ctas + 1))()
    queue = (C.c_int32 * n)()
    _check(L.mk_prefill_graph(C.byref(cfg), T, tiles_c, len(tiles), lm_c, num_ctas, tasks, n, qoff,
                              queue, n, C.byref(n_tasks), C.byref(n_events)))
    rows = [list(tasks[9 * i:9 * i + 9]) for i in range(n)]
    return rows, list(qoff), list(queue), n_events.value


class Plan:
    """The task graph mk_create would build (host only)."""

    def __init__(self, model, max_seq: int, num_ctas: int, max_batch: int = 1,
                 attn_splits: int = 0, weight_format: int = 0):
        L = lib()
        self.h = C.c_void_p()
        cfg = make_config(model, max_seq, max_batch)
        opt = Options(num_ctas, attn_splits, 0, 0, 0, weight_format, 0, 0, 0, 0, 0, 0)
        rc = L.mk_plan_build(C.byref(cfg), C.byref(opt), int(num_ctas), C.byref(self.h))
        if rc != MK_OK:
            raise MkError(rc, "mk_plan_build rejected the configuration")
        self.info = PlanInfo()
        _check(L.mk_plan_get_info(self.h, C.byref(self.info)))

    def tasks(self) -> List[dict]:
        n = self.info.n_tasks
        arr = (PlanTask * n)()
        got = lib().mk_plan_get_tasks(self.h, arr, n)
        assert got == n
        return [{f: getattr(t, f) for f, _ in PlanTask._fields_} for t in arr]

    def queue(self, cta: int) -> List[int]:
        n = lib().mk_plan_get_queue(self.h, cta, None, 0)
        buf = (C.c_int32 * max(n, 1))()
        lib().mk_plan_get_queue(self.h, cta, buf, n)
        return list(buf[:n])

    def event_counts(self) -> List[int]:
        n = lib().mk_plan_get_event_counts(self.h, None, 0)
        buf = (C.c_int32 * max(n, 1))()
        lib().mk_plan_get_event_counts(self.h, buf, n)
        return list(buf[:n])

    def __del__(self):
        if getattr(self, "h", None):
            lib().mk_plan_destroy(self.h)
            self.h = None


def qkv_row_source(model, r: int):
    cfg = make_config(model, 1)
    w, h, d = C.c_int32(), C.c_int32(), C.c_int32()
    _check(lib().mk_qkv_row_source(C.byref(cfg), int(r), C.byref(w), C.byref(h), C.byref(d)))
    return w.value, h.value, d.value


# ---------------------------------------------------------------- decoder

class Decoder:
    """One libmk context.  ``weights`` maps the synthetic generator's names to
    CUDA bf16 tensors; mk_create copies them, so they may be dropped after."""

    def __init__(self, model, weights: Dict[str, "torch.Tensor"], max_seq: int,
                 max_batch: int = 1, num_ctas: int = 0, attn_splits: int = 0,
                 timeout_ms: int = 0, mode: int = MODE_MEGAKERNEL, stream=None,
                 l2_prefetch: int = 0, prefill_steps: int = 0, batch_sequential: int = 0,
                 weight_format: int = 0, kv_page_tokens: int = 0, kv_pool_pages: int = 0,
                 prefill_per_operator: int = 0, prefill_attention: int = 0):
        import torch
        L = lib()
        self.model = model
        self.max_seq = max_seq
        self.max_batch = max_batch
        self.stream = stream if stream is not None else torch.cuda.current_stream()

        def ptr(name):
            t = weights.get(name)
            if t is None:
                return None
            assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), name
            return t.data_ptr()

        layers = (LayerWeights * model.n_layers)()
        for l in range(model.n_layers):
            for k in LAYER_FIELDS:
                setattr(layers[l], k, ptr(f"layers.{l}.{k}"))
        w = Weights(ptr("embed"), layers, ptr("final_norm"),
                    None if model.tied_embeddings else ptr("lm_head"))
        cfg = make_config(model, max_seq, max_batch)
        opt = Options(num_ctas, attn_splits, timeout_ms, mode, l2_prefetch, weight_format,
                      batch_sequential, prefill_steps, kv_page_tokens, kv_pool_pages,
                      prefill_per_operator, prefill_attention)
        self.h = C.c_void_p()
        rc = L.mk_create(C.byref(cfg), C.byref(w), C.byref(opt), self.stream.cuda_stream,
                         C.byref(self.h))
        if rc != MK_OK:
            msg = L.mk_last_error(None).decode(errors="replace")
            self.h = None
            raise MkError(rc, msg)

    def close(self):
        if getattr(self, "h", None):
            lib().mk_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown: the library may be gone already
            pass

    def set_mode(self, mode: int):
        _check(lib().mk_set_mode(self.h, int(mode)), self.h)

    def prefill(self, tokens_dev, offsets: Sequence[int], logits_dev=None, next_ids_dev=None):
        n_req = len(offsets) - 1
        _check(lib().mk_prefill(self.h, tokens_dev.data_ptr(), _ints(offsets), n_req,
                                None if logits_dev is None else logits_dev.data_ptr(),
                                None if next_ids_dev is None else next_ids_dev.data_ptr()),
               self.h)

    def decode(self, tokens_dev, pos: Sequence[int], logits_dev=None, next_ids_dev=None):
        _check(lib().mk_decode_step(self.h, tokens_dev.data_ptr(), _ints(pos), len(pos),
                                    None if logits_dev is None else logits_dev.data_ptr(),
                                    None if next_ids_dev is None else next_ids_dev.data_ptr()),
               self.h)

    def prefill_slots(self, tokens_dev, offsets: Sequence[int], slots: Sequence[int],
                      logits_dev=None, next_ids_dev=None):
        """mk_prefill with request r on KV-cache slot slots[r]."""
        _check(lib().mk_prefill_slots(self.h, tokens_dev.data_ptr(), _ints(offsets), _ints(slots),
                                      len(slots),
                                      None if logits_dev is None else logits_dev.data_ptr(),
                                      None if next_ids_dev is None else next_ids_dev.data_ptr()),
               self.h)

    def decode_slots(self, tokens_dev, pos: Sequence[int], slots: Sequence[int], logits_dev=None,
                     next_ids_dev=None):
        """mk_decode_step with request r on KV-cache slot slots[r]."""
        _check(lib().mk_decode_step_slots(self.h, tokens_dev.data_ptr(), _ints(pos), _ints(slots),
                                          len(pos),
                                          None if logits_dev is None else logits_dev.data_ptr(),
                                          None if next_ids_dev is None else next_ids_dev.data_ptr()),
               self.h)

    def kv_release(self, slot: int):
        _check(lib().mk_kv_release(self.h, int(slot)), self.h)

    def kv_set_pages(self, slot: int, pages: Sequence[int]):
        _check(lib().mk_kv_set_pages(self.h, int(slot), _ints(pages), len(pages)), self.h)

    def kv_pages(self, slot: int) -> List[int]:
        n = lib().mk_kv_get_pages(self.h, int(slot), None, 0)
        _check(min(n, 0), self.h)
        out = (C.c_int32 * max(n, 1))()
        lib().mk_kv_get_pages(self.h, int(slot), out, n)
        return list(out)[:n]

    def kv_free_pages(self) -> int:
        n = lib().mk_kv_free_pages(self.h)
        _check(min(n, 0), self.h)
        return int(n)

    def decode_steps(self, token_dev, pos0: int, n_steps: int, ids_dev, last_logits_dev=None):
        """n_steps greedy steps in one persistent launch; ids_dev[s] gets step s's id."""
        _check(lib().mk_decode_steps(self.h, token_dev.data_ptr(), int(pos0), int(n_steps),
                                     ids_dev.data_ptr(),
                                     None if last_logits_dev is None else last_logits_dev.data_ptr()),
               self.h)

    def decode_host(self, tokens: Sequence[int], pos: Sequence[int]) -> List[int]:
        out = (C.c_int32 * len(tokens))()
        _check(lib().mk_decode_step_host(self.h, _ints(tokens), _ints(pos), len(tokens), out),
               self.h)
        return list(out)

    def copy_hidden(self, dst_dev, n_req: int = 1):
        _check(lib().mk_copy_hidden(self.h, dst_dev.data_ptr(), int(n_req)), self.h)

    def copy_activation(self, which: int, dst_dev):
        """The last single-request step's ACT_Q / ACT_ATTN / ACT_FFN / ACT_X vector
        (see mk_copy_activation) into the fp32 CUDA tensor ``dst_dev``."""
        _check(lib().mk_copy_activation(self.h, int(which), dst_dev.data_ptr(),
                                        int(dst_dev.numel())), self.h)

    def copy_kv(self, req: int, layer: int, kv_head: int, which: int, n: int, dst_dev):
        _check(lib().mk_copy_kv(self.h, req, layer, kv_head, which, n, dst_dev.data_ptr()),
               self.h)

    def set_trace(self, trace_dev=None):
        """Per-task timeline of later megakernel steps into ``trace_dev``
        (int64 CUDA tensor, 8 words per task); None turns it off."""
        _check(lib().mk_set_trace(self.h, None if trace_dev is None else trace_dev.data_ptr()),
               self.h)

    def set_prefill_trace(self, trace_dev=None):
        """Per-task timeline of the persistent prefill's first block into
        ``trace_dev`` (int64 CUDA tensor, 4 words per task); None turns it off."""
        cap = 0 if trace_dev is None else trace_dev.numel() // 4
        _check(lib().mk_set_prefill_trace(self.h, None if trace_dev is None else trace_dev.data_ptr(),
                                          cap), self.h)

    def status(self) -> int:
        return int(lib().mk_status(self.h))

    def inject_stall(self, task: int = -1):
        """Makes one task's event wait unreachable (failure-detection test hook):
        the next megakernel step ends with MK_ERR_TIMEOUT after timeout_ms."""
        _check(lib().mk_inject_stall(self.h, int(task)), self.h)

    def inject_prefill_stall(self, task: int = -1):
        """The same for the persistent prefill: the next prefill call ends with
        MK_ERR_TIMEOUT after 2 x timeout_ms."""
        _check(lib().mk_inject_prefill_stall(self.h, int(task)), self.h)

    def last_error(self) -> str:
        return lib().mk_last_error(self.h).decode(errors="replace")


def read_probe(src_dev, sink_dev, stream=None):
    """Enqueues one read-only pass over ``src_dev`` (a contiguous CUDA tensor)."""
    import torch
    st = stream if stream is not None else torch.cuda.current_stream()
    nbytes = src_dev.numel() * src_dev.element_size()
    _check(lib().mk_read_probe(src_dev.data_ptr(), nbytes, sink_dev.data_ptr(), st.cuda_stream))


def attention_workspace_bytes(n_q_per_kv: int, head_dim: int, splits: int) -> int:
    return int(lib().mk_attention_workspace_bytes(n_q_per_kv, head_dim, splits))


def attention_decode(q_dev, k_dev, v_dev, n_keys: int, splits: int, workspace_dev, out_dev,
                     stream=None):
    """Split-KV decode attention for one KV head (see mk_attention_decode)."""
    import torch
    st = stream if stream is not None else torch.cuda.current_stream()
    G, d = q_dev.shape
    _check(lib().mk_attention_decode(q_dev.data_ptr(), k_dev.data_ptr(), v_dev.data_ptr(),
                                     int(n_keys), int(G), int(d), int(splits),
                                     workspace_dev.data_ptr(), out_dev.data_ptr(), st.cuda_stream))


def attention_decode_noalloc(q_dev, k_dev, v_dev, n_keys: int, splits: int, out_dev,
                             stream=None):
    """mk_attention_decode with the library's static scratch instead of a
    caller workspace (see mk_attention_decode_noalloc)."""
    import torch
    st = stream if stream is not None else torch.cuda.current_stream()
    G, d = q_dev.shape
    _check(lib().mk_attention_decode_noalloc(q_dev.data_ptr(), k_dev.data_ptr(),
                                             v_dev.data_ptr(), int(n_keys), int(G), int(d),
                                             int(splits), out_dev.data_ptr(), st.cuda_stream))
