"""Python binding of libg4attn.so (the C ABI in include/g4attn.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory (tensors, workspace) and the stream.
There is no fallback: if the library is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libg4attn.so")

G4ATTN_OK, G4ATTN_EINVAL, G4ATTN_EUNSUPPORTED, G4ATTN_ECACHE_OVERFLOW = 0, 1, 2, 3
G4ATTN_ECUDA, G4ATTN_EDEVICE, G4ATTN_EWORKSPACE, G4ATTN_ECACHE_EMPTY = 4, 5, 6, 7
G4ATTN_SLIDING, G4ATTN_GLOBAL, G4ATTN_BIDIRECTIONAL = 0, 1, 2
G4ATTN_BF16, G4ATTN_FP32 = 0, 1

EXPORTED = ("g4attn_prefill_workspace_size", "g4attn_decode_workspace_size", "g4attn_prefill",
            "g4attn_prefill_chunk_workspace_size", "g4attn_prefill_chunk",
            "g4attn_qkv_prologue", "g4attn_attend_workspace_size", "g4attn_attend",
            "g4attn_cache_append", "g4attn_decode", "g4attn_decode_noalloc",
            "g4attn_get_device_status", "g4attn_time_next_attention", "g4attn_launch_count",
            "g4attn_status_string")


class G4AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {g4attn_status_string(status)} (status {status})")


class LayerDesc(ctypes.Structure):
    """g4attn_layer_desc."""
    _fields_ = [("layer_type", ctypes.c_int), ("window", ctypes.c_int),
                ("rotary_fraction", ctypes.c_float), ("rope_theta", ctypes.c_double),
                ("k_eq_v", ctypes.c_int), ("num_heads", ctypes.c_int),
                ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("dtype", ctypes.c_int), ("logit_softcap", ctypes.c_float)]


class _CCache(ctypes.Structure):
    """g4attn_cache."""
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("len", ctypes.c_void_p),
                ("capacity", ctypes.c_int), ("rolling", ctypes.c_int), ("batch", ctypes.c_int),
                ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("dtype", ctypes.c_int), ("key_mask", ctypes.c_void_p),
                ("mask_len", ctypes.c_int), ("k_norm_w", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is not built: run `python -m attention_prologue_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        DP, CP = ctypes.POINTER(LayerDesc), ctypes.POINTER(_CCache)
        L.g4attn_prefill_workspace_size.argtypes = [DP, I, I]
        L.g4attn_prefill_workspace_size.restype = S
        L.g4attn_decode_workspace_size.argtypes = [DP, CP]
        L.g4attn_decode_workspace_size.restype = S
        L.g4attn_prefill.argtypes = [DP, I, I, P, P, P, P, P, P, P, CP, P, P, S, P]
        L.g4attn_prefill.restype = I
        L.g4attn_prefill_chunk_workspace_size.argtypes = [DP, I, I, I]
        L.g4attn_prefill_chunk_workspace_size.restype = S
        L.g4attn_prefill_chunk.argtypes = [DP, I, I, I, P, P, P, P, P, P, P, CP, P, P, S, P]
        L.g4attn_prefill_chunk.restype = I
        L.g4attn_qkv_prologue.argtypes = [DP, I, I, I, P, I, P, P, P, P, CP, P]
        L.g4attn_qkv_prologue.restype = I
        L.g4attn_attend_workspace_size.argtypes = [DP, I, I, I]
        L.g4attn_attend_workspace_size.restype = ctypes.c_size_t
        L.g4attn_attend.argtypes = [DP, I, I, I, P, P, P, CP, P, P, S, P]
        L.g4attn_cache_append.argtypes = [DP, CP, P, P, P, P]
        L.g4attn_cache_append.restype = I
        L.g4attn_decode.argtypes = [DP, CP, P, P, P, P, S, P]
        L.g4attn_decode.restype = I
        L.g4attn_decode_noalloc.argtypes = [DP, CP, P, P, P, P]
        L.g4attn_decode_noalloc.restype = I
        L.g4attn_get_device_status.argtypes = [P]
        L.g4attn_get_device_status.restype = I
        L.g4attn_time_next_attention.argtypes = [P, P]
        L.g4attn_time_next_attention.restype = None
        L.g4attn_launch_count.argtypes = []
        L.g4attn_launch_count.restype = ctypes.c_uint64
        L.g4attn_status_string.argtypes = [I]
        L.g4attn_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return G4ATTN_BF16
    if dt == torch.float32:
        return G4ATTN_FP32
    raise ValueError(f"unsupported dtype {dt}")


def make_desc(layer_type: int, num_heads: int, num_kv_heads: int, head_dim: int, *,
              window: int = 0, rotary_fraction: float = 1.0, rope_theta: float = 1e4,
              k_eq_v: bool = False, softmax_scale: float | None = None, rms_eps: float = 1e-6,
              dtype: torch.dtype = torch.bfloat16, logit_softcap: float = 0.0) -> LayerDesc:
    scale = head_dim ** -0.5 if softmax_scale is None else softmax_scale
    return LayerDesc(int(layer_type), int(window), float(rotary_fraction), float(rope_theta),
                     int(bool(k_eq_v)), int(num_heads), int(num_kv_heads), int(head_dim),
                     float(scale), float(rms_eps), _dtype_code(dtype), float(logit_softcap))


def _ptr(t: torch.Tensor | None, name: str, device: torch.device | None = None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def cache_bytes(batch: int, num_kv_heads: int, capacity: int, head_dim: int,
                dtype: torch.dtype = torch.bfloat16) -> int:
    """Device bytes of one layer's cache: K and V stored separately, each
    [batch, num_kv_heads, capacity, head_dim] (len[] not counted)."""
    es = torch.empty((), dtype=dtype).element_size()
    return 2 * batch * num_kv_heads * capacity * head_dim * es


@dataclass
class KVCache:
    """A layer's KV cache in device memory owned by torch.  key_mask (uint8
    [batch, mask_len], optional) marks the padding positions of the prompt it
    holds (0 = padding); later positions are kept.  v = None: a single-tensor
    cache of a K=V layer (k holds V = RMSNorm(k_raw); k_norm_w, the owning
    layer's key-norm weight, rebuilds K on read)."""
    k: torch.Tensor
    v: torch.Tensor | None
    len: torch.Tensor
    rolling: bool = False
    key_mask: torch.Tensor | None = None
    k_norm_w: torch.Tensor | None = None

    @classmethod
    def allocate(cls, batch: int, num_kv_heads: int, capacity: int, head_dim: int, *,
                 rolling: bool = False, dtype: torch.dtype = torch.bfloat16,
                 device="cuda", single: bool = False,
                 k_norm_w: torch.Tensor | None = None) -> "KVCache":
        shape = (batch, num_kv_heads, capacity, head_dim)
        return cls(torch.empty(shape, dtype=dtype, device=device),
                   None if single else torch.empty(shape, dtype=dtype, device=device),
                   torch.zeros(batch, dtype=torch.int32, device=device), rolling,
                   k_norm_w=k_norm_w)

    @property
    def capacity(self) -> int:
        return self.k.shape[2]

    def c(self) -> _CCache:
        B, Hkv, C, d = self.k.shape
        if self.v is not None and (self.v.shape != self.k.shape or self.v.dtype != self.k.dtype):
            raise ValueError("cache k and v differ in shape or dtype")
        if self.len.dtype != torch.int32 or self.len.numel() != B:
            raise ValueError("cache len must be int32 [batch]")
        km, mlen = None, 0
        if self.key_mask is not None:
            if self.key_mask.dtype != torch.uint8 or self.key_mask.dim() != 2 \
                    or self.key_mask.shape[0] != B:
                raise ValueError("cache key_mask must be uint8 [batch, mask_len]")
            km, mlen = _ptr(self.key_mask, "cache.key_mask"), self.key_mask.shape[1]
        return _CCache(_ptr(self.k, "cache.k"), _ptr(self.v, "cache.v"),
                       _ptr(self.len, "cache.len"), C, int(self.rolling), B, Hkv, d,
                       _dtype_code(self.k.dtype), km, mlen,
                       _ptr(self.k_norm_w, "cache.k_norm_w"))


def _check(rc: int, where: str):
    if rc != G4ATTN_OK:
        raise G4AttnError(rc, where)


def g4attn_prefill_workspace_size(desc: LayerDesc, B: int, T: int) -> int:
    return int(lib().g4attn_prefill_workspace_size(ctypes.byref(desc), B, T))


def g4attn_decode_workspace_size(desc: LayerDesc, cache: KVCache) -> int:
    cc = cache.c()
    return int(lib().g4attn_decode_workspace_size(ctypes.byref(desc), ctypes.byref(cc)))


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _mask(m: torch.Tensor | None, shape, name: str):
    if m is None:
        return None
    if m.dtype != torch.uint8 or tuple(m.shape) != tuple(shape):
        raise ValueError(f"{name} must be uint8 {list(shape)}")
    return m


def g4attn_prefill(desc: LayerDesc, q_raw: torch.Tensor, k_raw: torch.Tensor | None,
                   v_raw: torch.Tensor | None, q_norm_w: torch.Tensor,
                   k_norm_w: torch.Tensor | None, image_block_ids: torch.Tensor | None = None,
                   cache: KVCache | None = None, out: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None, stream=None,
                   attention_mask: torch.Tensor | None = None) -> torch.Tensor:
    """Prefill of q_raw [B, T, Hq, d] (see g4attn_prefill in g4attn.h);
    attention_mask uint8 [B, T], 0 = padding key."""
    B, T = q_raw.shape[0], q_raw.shape[1]
    dev = q_raw.device
    if out is None:
        out = torch.empty_like(q_raw)
    if workspace is None:
        workspace = _workspace(g4attn_prefill_workspace_size(desc, B, T), dev)
    if image_block_ids is not None and image_block_ids.dtype != torch.int32:
        raise ValueError("image_block_ids must be int32")
    am = _mask(attention_mask, (B, T), "attention_mask")
    cc = cache.c() if cache is not None else None
    rc = lib().g4attn_prefill(
        ctypes.byref(desc), B, T, _ptr(q_raw, "q_raw", dev), _ptr(k_raw, "k_raw", dev),
        _ptr(v_raw, "v_raw", dev), _ptr(q_norm_w, "q_norm_w", dev),
        _ptr(k_norm_w, "k_norm_w", dev), _ptr(image_block_ids, "image_block_ids", dev),
        _ptr(am, "attention_mask", dev),
        ctypes.byref(cc) if cc is not None else None, _ptr(out, "out", dev),
        _ptr(workspace, "workspace", dev), workspace.numel(), _stream(stream))
    _check(rc, "g4attn_prefill")
    return out


def g4attn_prefill_chunk_workspace_size(desc: LayerDesc, B: int, T: int, p0: int) -> int:
    return int(lib().g4attn_prefill_chunk_workspace_size(ctypes.byref(desc), B, T, p0))


def g4attn_prefill_chunk(desc: LayerDesc, p0: int, q_raw: torch.Tensor,
                         k_raw: torch.Tensor | None, v_raw: torch.Tensor | None,
                         q_norm_w: torch.Tensor, k_norm_w: torch.Tensor | None,
                         image_block_ids: torch.Tensor | None, cache: KVCache,
                         out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                         stream=None, attention_mask: torch.Tensor | None = None) -> torch.Tensor:
    """Cached prefill of a chunk q_raw [B, T, Hq, d] at positions p0 .. p0+T-1
    (see g4attn_prefill_chunk in g4attn.h); image_block_ids and
    attention_mask (uint8, 0 = padding key) [B, p0 + T]."""
    B, T = q_raw.shape[0], q_raw.shape[1]
    dev = q_raw.device
    if out is None:
        out = torch.empty_like(q_raw)
    if workspace is None:
        workspace = _workspace(g4attn_prefill_chunk_workspace_size(desc, B, T, p0), dev)
    if image_block_ids is not None and image_block_ids.dtype != torch.int32:
        raise ValueError("image_block_ids must be int32")
    am = _mask(attention_mask, (B, p0 + T), "attention_mask")
    cc = cache.c()
    rc = lib().g4attn_prefill_chunk(
        ctypes.byref(desc), B, T, p0, _ptr(q_raw, "q_raw", dev), _ptr(k_raw, "k_raw", dev),
        _ptr(v_raw, "v_raw", dev), _ptr(q_norm_w, "q_norm_w", dev),
        _ptr(k_norm_w, "k_norm_w", dev), _ptr(image_block_ids, "image_block_ids", dev),
        _ptr(am, "attention_mask", dev), ctypes.byref(cc), _ptr(out, "out", dev), _ptr(workspace, "workspace", dev),
        workspace.numel(), _stream(stream))
    _check(rc, "g4attn_prefill_chunk")
    return out


def g4attn_qkv_prologue(desc: LayerDesc, p0: int, x: torch.Tensor, w_qkv: torch.Tensor,
                        q_norm_w: torch.Tensor, k_norm_w: torch.Tensor | None,
                        cache: KVCache | None, q_hat: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """QKV projection of x [B, T, hidden] by w_qkv [n_heads * d, hidden] with
    the prologue in its epilogue (see g4attn_qkv_prologue in g4attn.h):
    returns q_hat [B, T, Hq, d]; K/V go to `cache` at positions p0 .. p0+T-1."""
    B, T, hidden = x.shape
    dev = x.device
    if q_hat is None:
        q_hat = torch.empty(B, T, desc.num_heads, desc.head_dim, dtype=x.dtype, device=dev)
    cc = cache.c() if cache is not None else None
    rc = lib().g4attn_qkv_prologue(
        ctypes.byref(desc), B, T, p0, _ptr(x, "x", dev), hidden, _ptr(w_qkv, "w_qkv", dev),
        _ptr(q_norm_w, "q_norm_w", dev), _ptr(k_norm_w, "k_norm_w", dev),
        _ptr(q_hat, "q_hat", dev), ctypes.byref(cc) if cc is not None else None,
        _stream(stream))
    _check(rc, "g4attn_qkv_prologue")
    return q_hat


def g4attn_attend_workspace_size(desc: LayerDesc, B: int, T: int, p0: int) -> int:
    return int(lib().g4attn_attend_workspace_size(ctypes.byref(desc), B, T, p0))


def g4attn_attend(desc: LayerDesc, p0: int, q_hat: torch.Tensor, cache: KVCache,
                  image_block_ids: torch.Tensor | None = None,
                  attention_mask: torch.Tensor | None = None, out: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Attention of post-prologue queries q_hat [B, T, Hq, d] at positions
    p0 .. p0+T-1 over the cache's positions 0 .. p0+T-1 (see g4attn_attend in
    g4attn.h); image_block_ids and attention_mask [B, p0 + T]."""
    B, T = q_hat.shape[0], q_hat.shape[1]
    dev = q_hat.device
    if out is None:
        out = torch.empty_like(q_hat)
    if workspace is None:
        workspace = _workspace(g4attn_attend_workspace_size(desc, B, T, p0), dev)
    if image_block_ids is not None and image_block_ids.dtype != torch.int32:
        raise ValueError("image_block_ids must be int32")
    am = _mask(attention_mask, (B, p0 + T), "attention_mask")
    cc = cache.c()
    rc = lib().g4attn_attend(
        ctypes.byref(desc), B, T, p0, _ptr(q_hat, "q_hat", dev),
        _ptr(image_block_ids, "image_block_ids", dev), _ptr(am, "attention_mask", dev),
        ctypes.byref(cc), _ptr(out, "out", dev), _ptr(workspace, "workspace", dev),
        workspace.numel(), _stream(stream))
    _check(rc, "g4attn_attend")
    return out


def g4attn_cache_append(desc: LayerDesc, cache: KVCache, k_raw: torch.Tensor,
                        v_raw: torch.Tensor | None, k_norm_w: torch.Tensor, stream=None) -> None:
    cc = cache.c()
    dev = cache.k.device
    rc = lib().g4attn_cache_append(ctypes.byref(desc), ctypes.byref(cc), _ptr(k_raw, "k_raw", dev),
                                   _ptr(v_raw, "v_raw", dev), _ptr(k_norm_w, "k_norm_w", dev),
                                   _stream(stream))
    _check(rc, "g4attn_cache_append")


def g4attn_decode(desc: LayerDesc, cache: KVCache, q_raw: torch.Tensor, q_norm_w: torch.Tensor,
                  out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """Decode of q_raw [B, 1, Hq, d] over `cache` (see g4attn_decode in g4attn.h)."""
    cc = cache.c()
    dev = cache.k.device
    if out is None:
        out = torch.empty_like(q_raw)
    if workspace is None:
        workspace = _workspace(g4attn_decode_workspace_size(desc, cache), dev)
    rc = lib().g4attn_decode(ctypes.byref(desc), ctypes.byref(cc), _ptr(q_raw, "q_raw", dev),
                             _ptr(q_norm_w, "q_norm_w", dev), _ptr(out, "out", dev),
                             _ptr(workspace, "workspace", dev), workspace.numel(), _stream(stream))
    _check(rc, "g4attn_decode")
    return out


def g4attn_decode_noalloc(desc: LayerDesc, cache: KVCache, q_raw: torch.Tensor,
                          q_norm_w: torch.Tensor, out: torch.Tensor | None = None,
                          stream=None) -> torch.Tensor:
    """g4attn_decode without a workspace: the split-KV partials live in the
    library's fixed 16 MiB device array (see g4attn_decode_noalloc in
    g4attn.h).  For callers that cannot hand the library device memory per
    call.  Calls that overlap on the GPU race on that array."""
    cc = cache.c()
    dev = cache.k.device
    if out is None:
        out = torch.empty_like(q_raw)
    rc = lib().g4attn_decode_noalloc(ctypes.byref(desc), ctypes.byref(cc),
                                     _ptr(q_raw, "q_raw", dev), _ptr(q_norm_w, "q_norm_w", dev),
                                     _ptr(out, "out", dev), _stream(stream))
    _check(rc, "g4attn_decode_noalloc")
    return out


def g4attn_get_device_status(stream=None) -> int:
    return int(lib().g4attn_get_device_status(_stream(stream)))


def g4attn_time_next_attention(start: torch.cuda.Event | None, stop: torch.cuda.Event | None):
    """Record `start`/`stop` around the attention kernel of the next call.
    The events must have been recorded once (torch creates them lazily)."""
    def h(e):
        return None if e is None else ctypes.c_void_p(e.cuda_event)
    lib().g4attn_time_next_attention(h(start), h(stop))


def g4attn_launch_count() -> int:
    return int(lib().g4attn_launch_count())


def g4attn_status_string(status: int) -> str:
    return lib().g4attn_status_string(int(status)).decode()
