"""ctypes wrapper of the C oracle (oracle.c).  TEST INFRASTRUCTURE ONLY.

Builds ``liboracle.so`` next to this file with gcc (-O2 -fopenmp
-ffp-contract=off) on first use.  Arrays cross the boundary as numpy fp32 or
as CPU bf16 torch tensors (their raw 16-bit patterns); the model keeps a
reference to every weight tensor it was given.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_lock = threading.Lock()
_lib = None

_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile liboracle.so if it is missing or older than its sources."""
    with _lock:
        fresh = (os.path.exists(_SO) and
                 os.path.getmtime(_SO) >= max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
        if force or not fresh:
            tmp = _SO + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                   "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
            subprocess.run(cmd, check=True, cwd=_HERE)
            os.replace(tmp, _SO)
    return _SO


class _Config(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("hidden", C.c_int), ("n_q_heads", C.c_int),
                ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
                ("vocab", C.c_int), ("rms_eps", C.c_float), ("rope_theta", C.c_double),
                ("qkv_bias", C.c_int), ("kv_bf16", C.c_int)]


_LAYER_FIELDS = ("attn_norm", "wq", "wk", "wv", "bq", "bk", "bv", "wo",
                 "ffn_norm", "w_gate", "w_up", "w_down")


class _Layer(C.Structure):
    _fields_ = [(k, C.c_void_p) for k in _LAYER_FIELDS]


def _bind(L):
    """Declare the C signatures on a loaded liboracle (or a test variant)."""
    L.orc_bf16_round.argtypes = [C.c_float]
    L.orc_bf16_round.restype = C.c_float
    L.orc_rmsnorm.argtypes = [_f32p, C.c_void_p, C.c_int, C.c_float, _f32p]
    L.orc_gemv.argtypes = [C.c_void_p, _f32p, C.c_int, C.c_int, _f32p]
    L.orc_rope.argtypes = [_f32p, C.c_int, C.c_int, C.c_double]
    L.orc_softmax.argtypes = [_f32p, C.c_int, _f32p]
    L.orc_attend.argtypes = [_f32p, _f32p, _f32p, C.c_int, C.c_int, _f32p]
    L.orc_attend_split.argtypes = [_f32p, _f32p, _f32p, C.c_int, C.c_int, C.c_int, _f32p]
    L.orc_silu.argtypes = [C.c_float]
    L.orc_silu.restype = C.c_float
    L.orc_argmax.argtypes = [_f32p, C.c_int]
    L.orc_argmax.restype = C.c_int
    L.orc_kv_cache_bytes.argtypes = [C.c_double] * 6
    L.orc_kv_cache_bytes.restype = C.c_double
    L.orc_create.argtypes = [C.POINTER(_Config), C.c_void_p, C.POINTER(_Layer),
                             C.c_void_p, C.c_void_p]
    L.orc_create.restype = C.c_void_p
    L.orc_destroy.argtypes = [C.c_void_p]
    L.orc_state_create.argtypes = [C.c_void_p, C.c_int]
    L.orc_state_create.restype = C.c_void_p
    L.orc_state_destroy.argtypes = [C.c_void_p]
    L.orc_state_set_kv.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, _f32p]
    L.orc_decode.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p,
                             C.c_void_p]
    L.orc_decode.restype = C.c_int
    L.orc_state_kv.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, _f32p]
    L.orc_state_kv.restype = C.c_int
    L.orc_forward_full.argtypes = [C.c_void_p, _i32p, C.c_int, C.c_void_p, C.c_void_p]
    L.orc_forward_full.restype = C.c_int
    L.orc_num_threads.restype = C.c_int
    L.orc_quantize_fp8_rows.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_void_p, _i32p]
    L.orc_prefill.argtypes = [C.c_void_p, C.c_void_p, _i32p, C.c_int, C.c_void_p, C.c_void_p]
    L.orc_prefill.restype = C.c_int
    return L


def load_variant(path: str):
    """Load another build of oracle.c (tests compile deliberately broken
    copies to show that the pins catch them)."""
    return _bind(C.CDLL(path))


def compile_variant(src_text: str, out_dir: str, name: str) -> str:
    """Compile oracle.c text (possibly edited) into out_dir/name.so."""
    import shutil
    src = os.path.join(out_dir, name + ".c")
    shutil.copy(_HDR, os.path.join(out_dir, "oracle.h"))
    with open(src, "w") as f:
        f.write(src_text)
    so = os.path.join(out_dir, name + ".so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                    "-ffp-contract=off", "-fno-fast-math", "-o", so, src, "-lm"],
                   check=True, cwd=out_dir)
    return so


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(C.CDLL(_SO))
    return _lib


# --------------------------------------------------------------- helpers

def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _bf16_ptr(t):
    """Raw pointer of a contiguous CPU bf16 torch tensor (kept alive by caller)."""
    import torch
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu" and t.is_contiguous()
    return t.data_ptr()


def bf16_round(x: float) -> float:
    return float(lib().orc_bf16_round(float(x)))


def rmsnorm(x, w_bf16, eps: float) -> np.ndarray:
    x = _f32(x)
    y = np.empty_like(x)
    lib().orc_rmsnorm(x, _bf16_ptr(w_bf16), x.size, float(eps), y)
    return y


def gemv(W_bf16, x) -> np.ndarray:
    rows, cols = W_bf16.shape
    x = _f32(x)
    assert x.size == cols
    y = np.empty(rows, dtype=np.float32)
    lib().orc_gemv(_bf16_ptr(W_bf16), x, rows, cols, y)
    return y


def rope(v, pos: int, theta: float) -> np.ndarray:
    v = _f32(v).copy()
    lib().orc_rope(v, v.size, int(pos), float(theta))
    return v


def softmax(s) -> np.ndarray:
    s = _f32(s)
    p = np.empty_like(s)
    lib().orc_softmax(s, s.size, p)
    return p


def attend(q, K, V) -> np.ndarray:
    q, K, V = _f32(q), _f32(K), _f32(V)
    n, d = K.shape
    out = np.empty(d, dtype=np.float32)
    lib().orc_attend(q, K, V, n, d, out)
    return out


def attend_split(q, K, V, n_splits: int) -> np.ndarray:
    q, K, V = _f32(q), _f32(K), _f32(V)
    n, d = K.shape
    out = np.empty(d, dtype=np.float32)
    lib().orc_attend_split(q, K, V, n, d, int(n_splits), out)
    return out


def silu(z: float) -> float:
    return float(lib().orc_silu(float(z)))


def argmax(v) -> int:
    v = _f32(v)
    return int(lib().orc_argmax(v, v.size))


def kv_cache_bytes(batch, layers, seq, head_dim, kv_heads, bytes_per_elem) -> float:
    return float(lib().orc_kv_cache_bytes(batch, layers, seq, head_dim, kv_heads,
                                          bytes_per_elem))


def num_threads() -> int:
    return int(lib().orc_num_threads())


def quantize_fp8_rows(W_bf16):
    """fp8 row quantization of a bf16 [rows, cols] CPU tensor: returns (the
    values e4m3(w / 2^k) * 2^k as bf16, the row exponents k as int32 numpy)."""
    import torch
    W = W_bf16.detach().to("cpu").contiguous()
    assert W.dtype == torch.bfloat16 and W.dim() == 2
    rows, cols = W.shape
    out = torch.empty_like(W)
    exps = np.empty(rows, dtype=np.int32)
    lib().orc_quantize_fp8_rows(W.data_ptr(), rows, cols, out.data_ptr(), exps)
    return out, exps


def quantize_fp8_model(cfg, weights):
    """The model the fp8 decode path computes: every matrix a decode GEMV
    streams (q, k, v, o, gate, up, down and the LM head -- the embedding when
    tied) row-quantized by quantize_fp8_rows; norms, biases and an untied
    embedding unchanged.  CPU bf16 tensors."""
    out = {k: v.detach().to("cpu") for k, v in weights.items()}
    for l in range(cfg.n_layers):
        for key in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down"):
            out[f"layers.{l}.{key}"] = quantize_fp8_rows(out[f"layers.{l}.{key}"])[0]
    head = "embed" if cfg.tied_embeddings else "lm_head"
    out[head] = quantize_fp8_rows(out[head])[0]
    return out


# ----------------------------------------------------------------- model

class OracleModel:
    """The whole decoder on CPU.  ``cfg`` is any object with the decoder's
    shape attributes (n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn,
    vocab, rms_eps, rope_theta, qkv_bias, tied_embeddings); ``weights`` maps
    the synthetic generator's names to bf16 tensors (moved to CPU here)."""

    def __init__(self, cfg, weights, kv_bf16: bool = True, _lib=None):
        import torch
        L = _lib or lib()
        self._L = L
        self.cfg = cfg
        self._keep = {}

        def host(name):
            t = weights.get(name)
            if t is None:
                return None
            t = t.detach().to("cpu").contiguous()
            assert t.dtype == torch.bfloat16
            self._keep[name] = t
            return t.data_ptr()

        c = _Config(cfg.n_layers, cfg.hidden, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim,
                    cfg.ffn, cfg.vocab, float(cfg.rms_eps), float(cfg.rope_theta),
                    int(bool(cfg.qkv_bias)), int(bool(kv_bf16)))
        layers = (_Layer * cfg.n_layers)()
        for l in range(cfg.n_layers):
            for k in _LAYER_FIELDS:
                setattr(layers[l], k, host(f"layers.{l}.{k}"))
        embed = host("embed")
        final = host("final_norm")
        lm = None if cfg.tied_embeddings else host("lm_head")
        self._cfg_struct, self._layers = c, layers
        self.h = L.orc_create(C.byref(c), embed, layers, final, lm)
        if not self.h:
            raise ValueError("orc_create rejected the configuration")

    def __del__(self):
        if getattr(self, "h", None):
            self._L.orc_destroy(self.h)
            self.h = None

    def new_state(self, max_seq: int) -> "OracleState":
        return OracleState(self, max_seq)

    def decode(self, state: "OracleState", token: int, pos: int, want_logits: bool = True):
        """One decode step; returns (next_id, logits or None, hidden)."""
        logits = np.empty(self.cfg.vocab, dtype=np.float32) if want_logits else None
        hidden = np.empty(self.cfg.hidden, dtype=np.float32)
        nid = self._L.orc_decode(self.h, state.h, int(token), int(pos),
                               logits.ctypes.data if want_logits else None,
                               hidden.ctypes.data)
        if nid < 0:
            raise ValueError("orc_decode rejected its arguments")
        return nid, logits, hidden

    def prefill(self, state: "OracleState", tokens, want_logits: bool = True):
        """The prompt at positions 0..n-1 into an empty state (n decode steps,
        the LM head at the last only); returns (next_id, logits or None, hidden)."""
        tokens = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        logits = np.empty(self.cfg.vocab, dtype=np.float32) if want_logits else None
        hidden = np.empty(self.cfg.hidden, dtype=np.float32)
        nid = self._L.orc_prefill(self.h, state.h, tokens, tokens.size,
                                  logits.ctypes.data if want_logits else None,
                                  hidden.ctypes.data)
        if nid < 0:
            raise ValueError("orc_prefill rejected its arguments")
        return nid, logits, hidden

    def forward_full(self, tokens):
        tokens = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        n = tokens.size
        logits = np.empty((n, self.cfg.vocab), dtype=np.float32)
        hidden = np.empty((n, self.cfg.hidden), dtype=np.float32)
        rc = self._L.orc_forward_full(self.h, tokens, n, logits.ctypes.data, hidden.ctypes.data)
        if rc != 0:
            raise ValueError("orc_forward_full rejected its arguments")
        return logits, hidden


class OracleState:
    """KV cache of one request."""

    def __init__(self, model: OracleModel, max_seq: int):
        self.model = model
        self.max_seq = max_seq
        self._L = model._L
        self.h = self._L.orc_state_create(model.h, int(max_seq))
        if not self.h:
            raise MemoryError("orc_state_create failed")

    def __del__(self):
        if getattr(self, "h", None):
            self._L.orc_state_destroy(self.h)
            self.h = None

    def kv(self, layer: int, kv_head: int, which: int, n: int) -> np.ndarray:
        d = self.model.cfg.head_dim
        out = np.empty(n * d, dtype=np.float32)
        rc = self._L.orc_state_kv(self.h, layer, kv_head, which, n, out)
        if rc != 0:
            raise ValueError("bad kv query")
        return out.reshape(n, d)

    def set_kv(self, layer: int, kv_head: int, which: int, values) -> None:
        """Writes positions [0, len(values)) of one cache head (K: which 0, V: 1)."""
        v = np.ascontiguousarray(np.asarray(values, dtype=np.float32))
        n = v.shape[0]
        rc = self._L.orc_state_set_kv(self.h, layer, kv_head, which, n, v.reshape(-1))
        if rc != 0:
            raise ValueError("bad kv write")
