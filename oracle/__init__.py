"""Float64 CPU oracle of the Gemma 4 attention layer (ctypes wrapper).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this package.  It shares no code
with the CUDA library (``attention_prologue_b200``) and never imports it.

The arithmetic lives in ``g4attn_oracle.c`` (plain C, float64, one explicit
loop per query row); this module only marshals arrays.  Each wrapper names
the page passage its C function follows.

Inputs may be torch CPU tensors (bf16 or fp32) or numpy float32 arrays; bf16
values are passed as their raw bits and widened exactly inside the oracle.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "g4attn_oracle.c")
_LIB = os.path.join(_HERE, "libg4attn_oracle.so")

BF16, FP32, FP64 = 0, 1, 2
SLIDING, GLOBAL, BIDIRECTIONAL = 0, 1, 2
ROPE_ZEROPAD, ROPE_PREFIX = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math: IEEE float64 throughout)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


class _Layer(ctypes.Structure):
    _fields_ = [("layer_type", ctypes.c_int), ("window", ctypes.c_int),
                ("rotary_fraction", ctypes.c_double), ("rope_theta", ctypes.c_double),
                ("k_eq_v", ctypes.c_int), ("num_heads", ctypes.c_int),
                ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("softmax_scale", ctypes.c_double), ("rms_eps", ctypes.c_double),
                ("rope_mode", ctypes.c_int), ("window_plus_one", ctypes.c_int),
                ("logit_softcap", ctypes.c_double)]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_double
        LP = ctypes.POINTER(_Layer)
        lib.or_rms_normalize.argtypes = [P, I, D, P, P]
        lib.or_rope.argtypes = [P, I, L, LP]
        lib.or_rotated_pairs.argtypes = [LP]
        lib.or_rotated_pairs.restype = I
        lib.or_interval.argtypes = [LP, P, I, I, P, P]
        lib.or_prologue_q.argtypes = [LP, P, L, I, P, I, L, P]
        lib.or_prologue_kv.argtypes = [LP, P, P, L, I, P, I, L, P, P]
        lib.or_prefill_kv.argtypes = [LP, I, I, P, P, P, I, I, P, P, I]
        lib.or_prefill_kv_at.argtypes = [LP, I, I, I, P, P, P, I, I, P, P, I]
        lib.or_prefill_rows.argtypes = [LP, I, I, P, P, I, I, P, P, P, P, I, P, I]
        lib.or_prefill_chunk_rows.argtypes = [LP, I, I, I, P, P, I, I, P, P, P, P, I, P, I]
        lib.or_prefill_chunk_rows_masked.argtypes = [LP, I, I, I, P, P, I, I, P, P, P, P, P, I,
                                                     P, I]
        lib.or_decode.argtypes = [LP, LP, P, P, I, I, P, P, I, I, I, P, P, P, P, P, I, P, I, P,
                                  I]
        lib.or_attend_rows.argtypes = [LP, I, I, I, P, P, P, P, P, P, I, P, I]
        lib.or_prologue_q_all.argtypes = [LP, I, I, I, P, P, I, I, P]
        lib.or_decode.restype = I
        lib.or_partial.argtypes = [P, P, P, L, I, I, I, D, P, P, P]
        lib.or_combine.argtypes = [I, P, P, P, I, P]
        _lib = lib
    return _lib


@dataclass
class Layer:
    """One attention layer as the pages state it ("Gemma 4" Keras docs,
    ``Gemma4Model`` argument table; "What changed from Gemma 3")."""
    layer_type: int = SLIDING
    window: int = 0
    rotary_fraction: float = 1.0
    rope_theta: float = 1e4
    k_eq_v: bool = False
    num_heads: int = 1
    num_kv_heads: int = 1
    head_dim: int = 64
    softmax_scale: float = 1.0
    rms_eps: float = 1e-6
    rope_mode: int = ROPE_ZEROPAD
    window_plus_one: bool = False
    logit_softcap: float = 0.0  # 0: none; else s <- cap * tanh(s / cap)

    def _c(self) -> _Layer:
        return _Layer(int(self.layer_type), int(self.window), float(self.rotary_fraction),
                      float(self.rope_theta), int(bool(self.k_eq_v)), int(self.num_heads),
                      int(self.num_kv_heads), int(self.head_dim), float(self.softmax_scale),
                      float(self.rms_eps), int(self.rope_mode), int(bool(self.window_plus_one)),
                      float(self.logit_softcap))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _raw(x):
    """(contiguous array holding the input bits, dtype code)."""
    if x is None:
        return None, FP32
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().contiguous().cpu()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), FP32
            if x.dtype == torch.float64:
                return x.numpy(), FP64
            raise TypeError(f"oracle input dtype {x.dtype} not supported")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, FP32
    if x.dtype == np.float64:
        return x, FP64
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle input dtype {x.dtype} not supported")


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _i32(a):
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.int32))


# --- single-vector steps -------------------------------------------------

def rms_normalize(x, eps: float, w=None) -> np.ndarray:
    """RMSNorm over one head, weight used as is ("What changed": plain-weight
    RMSNorm; "Attention Backend Notes": x_normed * weight).  w=None is the
    weightless V-norm."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = None if w is None else np.ascontiguousarray(w, dtype=np.float64)
    y = np.empty_like(x)
    _load().or_rms_normalize(_p(x), x.size, eps, _p(w), _p(y))
    return y


def rope(x, pos: int, layer: Layer) -> np.ndarray:
    """RoPE of one head at integer position ("Dual RoPE configurations":
    2x2 rotation per two-dimensional subspace; "What changed": zero-pad
    partial rope)."""
    y = np.array(x, dtype=np.float64, copy=True)
    c = layer._c()
    _load().or_rope(_p(y), y.size, int(pos), ctypes.byref(c))
    return y


def rotated_pairs(layer: Layer) -> int:
    c = layer._c()
    return _load().or_rotated_pairs(ctypes.byref(c))


def interval(layer: Layer, ids, T: int, i: int) -> tuple[int, int]:
    """Keys row i may see, [lo, hi] ("Sliding-window attention", "Global
    attention layers"; image blocks: "What changed", NaViT bullet)."""
    ids = _i32(ids)
    lo, hi = ctypes.c_int(), ctypes.c_int()
    c = layer._c()
    _load().or_interval(ctypes.byref(c), _p(ids), T, i, ctypes.byref(lo), ctypes.byref(hi))
    return lo.value, hi.value


def prologue_q(layer: Layer, q_vec, wq, pos: int) -> np.ndarray:
    q, dt = _raw(q_vec)
    w, wdt = _raw(wq)
    out = np.empty(layer.head_dim, np.float64)
    c = layer._c()
    _load().or_prologue_q(ctypes.byref(c), _p(q), 0, dt, _p(w), wdt, int(pos), _p(out))
    return out


def prologue_kv(layer: Layer, k_vec, v_vec, wk, pos: int):
    k, dt = _raw(k_vec)
    v, _ = _raw(v_vec)
    w, wdt = _raw(wk)
    ko = np.empty(layer.head_dim, np.float64)
    vo = np.empty(layer.head_dim, np.float64)
    c = layer._c()
    _load().or_prologue_kv(ctypes.byref(c), _p(k), _p(v), 0, dt, _p(w), wdt, int(pos),
                           _p(ko), _p(vo))
    return ko, vo


# --- whole-layer entry points --------------------------------------------

def prefill_kv(layer: Layer, k_raw, v_raw, wk, nthreads: int | None = None, p0: int = 0):
    """Post-prologue K and V of every token, float64 [B, T, Hkv, d]; the
    tokens sit at positions p0 .. p0 + T - 1 (RoPE)."""
    k, dt = _raw(k_raw)
    v, _ = _raw(v_raw)
    w, wdt = _raw(wk)
    B, T, Hkv, d = k_raw.shape
    kh = np.empty((B, T, Hkv, d), np.float64)
    vh = np.empty((B, T, Hkv, d), np.float64)
    c = layer._c()
    _load().or_prefill_kv_at(ctypes.byref(c), B, T, int(p0), _p(k),
                             _p(v) if v is not None else None, _p(w), dt, wdt, _p(kh), _p(vh),
                             nthreads or default_threads())
    return kh, vh


def prefill_rows(layer: Layer, q_raw, wq, khat, vhat, block_ids=None, rows=None,
                 nthreads: int | None = None, attention_mask=None) -> np.ndarray:
    """Attention output of the given query rows, float64 [B, n_rows, Hq, d].
    attention_mask [B, T] (1 = keep, 0 = padding) drops padding keys; a row
    left without keys outputs 0."""
    if attention_mask is not None:
        return prefill_chunk_rows(layer, q_raw, wq, khat, vhat, 0, block_ids, rows, nthreads,
                                  attention_mask)
    q, dt = _raw(q_raw)
    w, wdt = _raw(wq)
    B, T, Hq, d = q_raw.shape
    ids = _i32(block_ids)
    rows_a = _i32(rows)
    n_rows = T if rows_a is None else rows_a.size
    out = np.empty((B, n_rows, Hq, d), np.float64)
    khat = np.ascontiguousarray(khat, np.float64)
    vhat = np.ascontiguousarray(vhat, np.float64)
    c = layer._c()
    _load().or_prefill_rows(ctypes.byref(c), B, T, _p(q), _p(w), dt, wdt, _p(ids), _p(khat),
                            _p(vhat), _p(rows_a), n_rows, _p(out), nthreads or default_threads())
    return out


def prefill(layer: Layer, q_raw, k_raw, v_raw, wq, wk, block_ids=None, rows=None,
            nthreads: int | None = None, attention_mask=None) -> np.ndarray:
    """Prologue + masked softmax attention of a whole prompt."""
    kh, vh = prefill_kv(layer, k_raw, v_raw, wk, nthreads)
    return prefill_rows(layer, q_raw, wq, kh, vh, block_ids, rows, nthreads, attention_mask)


def prefill_chunk_rows(layer: Layer, q_raw, wq, khat, vhat, p0: int, block_ids=None, rows=None,
                       nthreads: int | None = None, attention_mask=None) -> np.ndarray:
    """Cached (chunked) prefill ("gemma4-pt-claude" README, "Tests": the
    cached path reproduces the uncached forward pass, image spans included).
    q_raw [B, T, Hq, d] holds the chunk's queries at positions p0 .. p0+T-1;
    khat/vhat [B, p0 + T, Hkv, d] the post-prologue keys and values of every
    position up to the chunk's last; block_ids [B, p0 + T] or None.  Each
    row attends over the interval of its position in a prompt of p0 + T
    tokens; attention_mask [B, p0 + T] (1 = keep, 0 = padding) drops padding
    keys.  Returns float64 [B, n_rows, Hq, d]."""
    q, dt = _raw(q_raw)
    w, wdt = _raw(wq)
    B, T, Hq, d = q_raw.shape
    if khat.shape[1] != p0 + T or vhat.shape[1] != p0 + T:
        raise ValueError("khat/vhat must hold positions 0 .. p0 + T - 1")
    ids = _i32(block_ids)
    if ids is not None and ids.shape != (B, p0 + T):
        raise ValueError("block_ids must be [B, p0 + T]")
    rows_a = _i32(rows)
    n_rows = T if rows_a is None else rows_a.size
    out = np.empty((B, n_rows, Hq, d), np.float64)
    khat = np.ascontiguousarray(khat, np.float64)
    vhat = np.ascontiguousarray(vhat, np.float64)
    keep = None
    if attention_mask is not None:
        keep = np.ascontiguousarray(np.asarray(attention_mask) != 0, np.uint8)
        if keep.shape != (B, p0 + T):
            raise ValueError("attention_mask must be [B, p0 + T]")
    c = layer._c()
    _load().or_prefill_chunk_rows_masked(ctypes.byref(c), B, T, int(p0), _p(q), _p(w), dt, wdt,
                                         _p(ids), _p(keep), _p(khat), _p(vhat), _p(rows_a),
                                         n_rows, _p(out), nthreads or default_threads())
    return out


def prologue_q_all(layer: Layer, q_raw, wq, p0: int = 0) -> np.ndarray:
    """Post-prologue queries of every token, float64 [B, T, Hq, d], the
    tokens at positions p0 .. p0 + T - 1 ("What changed": plain-weight
    RMSNorm, zero-pad partial rope)."""
    q, dt = _raw(q_raw)
    w, wdt = _raw(wq)
    B, T, Hq, d = q_raw.shape
    out = np.empty((B, T, Hq, d), np.float64)
    c = layer._c()
    _load().or_prologue_q_all(ctypes.byref(c), B, T, int(p0), _p(q), _p(w), dt, wdt, _p(out))
    return out


def _f64(x) -> np.ndarray:
    """The exact values of a bf16 / fp32 / fp64 tensor or array as float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, np.float64)


def qkv_prologue(layer: Layer, x, w_qkv, wq, wk=None, p0: int = 0, with_kv: bool = True):
    """The projection in front of the layer, then its prologue ("Gemma 4"
    overview blog, "Shared KV Cache": the key and value projections produce
    the K/V a layer stores; "Gemma 4" Keras docs, "What changed from Gemma 3":
    the prologue).  raw = x W^T is one float64 matmul of the exact input
    values (a library primitive standing for the projection; the products of
    bf16 values are exact in float64), split by rows of W into the num_heads
    query heads, then (with_kv) the num_kv_heads key heads and, unless k_eq_v,
    the num_kv_heads value heads; then prologue_q_all and prefill_kv at
    positions p0 .. p0 + T - 1.

    x [B, T, hidden], w_qkv [n_heads * d, hidden].  Returns float64
    (q_hat [B, T, Hq, d], k_hat, v_hat [B, T, Hkv, d]); k_hat, v_hat are None
    without KV heads."""
    X = _f64(x)
    Wm = _f64(w_qkv)
    B, T, _ = X.shape
    Hq, Hkv, d = layer.num_heads, layer.num_kv_heads, layer.head_dim
    n_heads = Hq + ((Hkv if layer.k_eq_v else 2 * Hkv) if with_kv else 0)
    if Wm.shape[0] != n_heads * d or Wm.shape[1] != X.shape[2]:
        raise ValueError("w_qkv must be [n_heads * d, hidden]")
    raw = X @ Wm.T
    qh = prologue_q_all(layer, np.ascontiguousarray(raw[..., :Hq * d].reshape(B, T, Hq, d)),
                        wq, p0)
    if not with_kv:
        return qh, None, None
    k_raw = np.ascontiguousarray(raw[..., Hq * d:(Hq + Hkv) * d].reshape(B, T, Hkv, d))
    v_raw = None if layer.k_eq_v else np.ascontiguousarray(
        raw[..., (Hq + Hkv) * d:(Hq + 2 * Hkv) * d].reshape(B, T, Hkv, d))
    kh, vh = prefill_kv(layer, k_raw, v_raw, wk, p0=p0)
    return qh, kh, vh


def attend_rows(layer: Layer, qhat, khat, vhat, p0: int = 0, block_ids=None, rows=None,
                nthreads: int | None = None, attention_mask=None) -> np.ndarray:
    """The attention of prefill_chunk_rows from given post-prologue queries
    qhat [B, T, Hq, d] (float64), keys/values khat/vhat [B, p0 + T, Hkv, d]:
    the same intervals, padding, soft-cap and softmax.  For modelling a
    storage format of the post-prologue vectors (round them, then attend).
    Returns float64 [B, n_rows, Hq, d]."""
    qhat = np.ascontiguousarray(qhat, np.float64)
    B, T, Hq, d = qhat.shape
    khat = np.ascontiguousarray(khat, np.float64)
    vhat = np.ascontiguousarray(vhat, np.float64)
    if khat.shape[1] != p0 + T or vhat.shape[1] != p0 + T:
        raise ValueError("khat/vhat must hold positions 0 .. p0 + T - 1")
    ids = _i32(block_ids)
    rows_a = _i32(rows)
    n_rows = T if rows_a is None else rows_a.size
    keep = None
    if attention_mask is not None:
        keep = np.ascontiguousarray(np.asarray(attention_mask) != 0, np.uint8)
    out = np.empty((B, n_rows, Hq, d), np.float64)
    c = layer._c()
    _load().or_attend_rows(ctypes.byref(c), B, T, int(p0), _p(qhat), _p(ids), _p(keep),
                           _p(khat), _p(vhat), _p(rows_a), n_rows, _p(out),
                           nthreads or default_threads())
    return out


def prefill_chunk(layer: Layer, q_raw, k_raw, v_raw, wq, wk, khat_cache, vhat_cache,
                  block_ids=None, rows=None, nthreads: int | None = None):
    """A chunk of T tokens after p0 = khat_cache.shape[1] cached ones: the
    key/value prologue of the chunk at positions p0 .. p0+T-1, appended to
    the cached keys/values, then chunked attention.  Returns (out,
    khat, vhat) with khat/vhat [B, p0 + T, Hkv, d]."""
    p0 = khat_cache.shape[1]
    kh, vh = prefill_kv(layer, k_raw, v_raw, wk, nthreads, p0=p0)
    khat = np.concatenate([khat_cache, kh], axis=1)
    vhat = np.concatenate([vhat_cache, vh], axis=1)
    out = prefill_chunk_rows(layer, q_raw, wq, khat, vhat, p0, block_ids, rows, nthreads)
    return out, khat, vhat


def decode(layer_q: Layer, q_raw, wq, cache_k, cache_v, capacity: int, rolling: bool, lens,
           k_new=None, v_new=None, wk=None, layer_kv: Layer | None = None, seqs=None,
           nthreads: int | None = None, attention_mask=None) -> np.ndarray:
    """One decode step ("Gemma4ConditionalGenerate": decoding over the
    per-layer KV cache; "KV Cache": rolling sliding caches; "Shared KV
    Cache": a later layer reads an earlier layer's K/V).

    cache_k/cache_v [B, Hkv, C, d] hold positions 0..lens[b]-1.  With k_new the
    new token is appended at position lens[b]; without it (KV-shared layer) the
    cache already holds it at lens[b]-1.  attention_mask [B, mask_len] (1 = keep,
    0 = padding) drops the padding keys among positions 0..mask_len-1; later
    positions are kept.  Returns float64 [n_seqs, Hq, d].  A bidirectional
    (vision-tower) layer has no decode step."""
    if BIDIRECTIONAL in (layer_q.layer_type, (layer_kv or layer_q).layer_type):
        raise ValueError("a bidirectional layer has no decode step")
    q, dt = _raw(q_raw)
    w, wdt = _raw(wq)
    ck, cdt = _raw(cache_k)
    cv, _ = _raw(cache_v)
    kn, _ = _raw(k_new)
    vn, _ = _raw(v_new)
    wkk, _ = _raw(wk)
    lens = _i32(lens)
    seqs_a = _i32(seqs)
    B = lens.size
    n = B if seqs_a is None else seqs_a.size
    out = np.empty((n, layer_q.num_heads, layer_q.head_dim), np.float64)
    keep, mask_len = None, 0
    if attention_mask is not None:
        keep = np.ascontiguousarray(np.asarray(attention_mask) != 0, np.uint8)
        if keep.ndim != 2 or keep.shape[0] != B:
            raise ValueError("attention_mask must be [B, mask_len]")
        mask_len = keep.shape[1]
    lq = layer_q._c()
    lkv = (layer_kv or layer_q)._c()
    rc = _load().or_decode(ctypes.byref(lq), ctypes.byref(lkv), _p(q), _p(w), dt, wdt, _p(ck),
                           _p(cv), cdt, int(capacity), int(bool(rolling)), _p(lens), _p(kn),
                           _p(vn), _p(wkk), _p(keep), int(mask_len), _p(seqs_a), n, _p(out),
                           nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle decode: a key the query needs is not in the cache")
    return out


def partial(q, kk, vv, lo: int, hi: int, scale: float):
    """Split-KV partial (m, l, o_tilde) of one query over keys lo..hi."""
    q = np.ascontiguousarray(q, np.float64)
    kk = np.ascontiguousarray(kk, np.float64)
    vv = np.ascontiguousarray(vv, np.float64)
    d = q.size
    m, l = ctypes.c_double(), ctypes.c_double()
    ot = np.empty(d, np.float64)
    _load().or_partial(_p(q), _p(kk), _p(vv), d, lo, hi, d, scale, ctypes.byref(m),
                       ctypes.byref(l), _p(ot))
    return m.value, l.value, ot


def combine(m, l, o_tilde) -> np.ndarray:
    """Log-sum-exp merge of split-KV partials."""
    m = np.ascontiguousarray(m, np.float64)
    l = np.ascontiguousarray(l, np.float64)
    o_tilde = np.ascontiguousarray(o_tilde, np.float64)
    n, d = o_tilde.shape
    o = np.empty(d, np.float64)
    _load().or_combine(n, _p(m), _p(l), _p(o_tilde), d, _p(o))
    return o
