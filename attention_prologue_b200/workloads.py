"""Seeded synthetic inputs shaped like the Gemma 4 variants' attention layers.

This module only draws random tensors and lays out shapes; it holds none of
the layer's arithmetic.  Both the CUDA path and the CPU oracle consume what it
produces.  Shapes follow the variant table of the "gemma4-pt-claude" README
("Supported Models": heads / KV heads per variant), the window sizes of the
"Gemma 4" overview blog ("Window sizes by model family": 512 on E2B/E4B,
1024 on 31B / 26B-A4B), the K=V global layers at global_head_dim 512 of the
Keras docs ("What changed from Gemma 3") and the image token budgets of the
overview blog ("Image token budgets": 70/140/280/560/1120).  No dataset is
involved: every value is drawn from a seeded generator.

Draw order for a prefill workload: q, k, v (skipped with K=V), w_q, w_k, then
the image block positions (numpy PCG64 with the same seed).  Decode
workloads draw the sequence lengths first (numpy), then per layer the new
token's q, k, v, the weights, then the cache contents sequence by sequence.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

SLIDING, GLOBAL, BIDIRECTIONAL = 0, 1, 2


@dataclass(frozen=True)
class LayerShape:
    """One attention layer: the fields of the Keras ``Gemma4Model`` table."""
    layer_type: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    window: int = 0
    rotary_fraction: float = 1.0
    rope_theta: float = 1e4
    k_eq_v: bool = False
    softmax_scale: float | None = None  # None: 1/sqrt(head_dim)
    rms_eps: float = 1e-6
    logit_softcap: float = 0.0          # 0: none

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim) if self.softmax_scale is None else self.softmax_scale


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    layer: LayerShape
    B: int
    T: int
    dtype: torch.dtype = torch.bfloat16
    n_blocks: int = 0          # image blocks per sequence (sliding layers)
    block_len: int = 0         # tokens per image block
    weights: str = "one_plus"  # "one_plus": 1 + N(0, 0.1); "normal": N(0, 1)


def sliding(num_heads, num_kv_heads, head_dim, window, **kw) -> LayerShape:
    return LayerShape(SLIDING, num_heads, num_kv_heads, head_dim, window=window,
                      rotary_fraction=1.0, rope_theta=1e4, **kw)


def global_(num_heads, num_kv_heads, head_dim, k_eq_v=True, **kw) -> LayerShape:
    return LayerShape(GLOBAL, num_heads, num_kv_heads, head_dim, rotary_fraction=0.25,
                      rope_theta=1e6, k_eq_v=k_eq_v, **kw)


def bidirectional(num_heads, num_kv_heads, head_dim, **kw) -> LayerShape:
    """The vision tower's attention: every patch sees every patch of its image
    ("gemma4-pt-claude" README, "Key architectural features"), softmax scale
    1.0 ("Attention Backend Notes")."""
    kw.setdefault("softmax_scale", 1.0)
    kw.setdefault("rotary_fraction", 1.0)
    kw.setdefault("rope_theta", 1e4)
    return LayerShape(BIDIRECTIONAL, num_heads, num_kv_heads, head_dim, **kw)


# -- the five workloads ------------------------------------------------------

# tiny fp32 check: one sliding layer and one K=V global layer
TINY_SLIDING = PrefillWorkload("tiny-fp32-sliding", sliding(2, 1, 64, 16), 1, 64,
                               torch.float32, weights="normal")
TINY_GLOBAL = PrefillWorkload("tiny-fp32-global", global_(2, 1, 64), 1, 64, torch.float32,
                              weights="normal")
# E2B-shaped sliding layer: 8 query heads on 1 KV head, d 256, window 512
E2B_SLIDING = PrefillWorkload("e2b-sliding-prefill", sliding(8, 1, 256, 512), 1, 8192)
# 12B-shaped sliding layer with 4 image blocks of 280 tokens per sequence
G12B_SLIDING_MM = PrefillWorkload("12b-sliding-multimodal-prefill", sliding(16, 8, 256, 1024),
                                  2, 16384, n_blocks=4, block_len=280)
# 31B-shaped K=V global layer: 32 query heads on 4 KV heads, d 512
G31B_GLOBAL = PrefillWorkload("31b-global-prefill", global_(32, 4, 512), 1, 32768)

# Vision-tower-shaped bidirectional attention: images of up to 2520 patches
# (the image processor's 280 soft tokens times its 3x3 pooling, Keras docs
# "Gemma4ImageProcessor"), 16 heads of 64 dims (the pages give no tower
# dimensions: a reading), scale 1.0
VISION_BIDIR = PrefillWorkload("vision-bidirectional", bidirectional(16, 16, 64), 8, 2520)

PREFILL_WORKLOADS = {w.name: w for w in
                     (TINY_SLIDING, TINY_GLOBAL, E2B_SLIDING, G12B_SLIDING_MM, G31B_GLOBAL)}


@dataclass(frozen=True)
class DecodeWorkload:
    """26B-A4B-shaped decode step: a sliding layer on a rolling cache, a K=V
    global layer, and a third layer that reads the global layer's cache."""
    name: str = "26b-a4b-decode"
    batch: int = 64
    len_lo: int = 4096
    len_hi: int = 131072
    sliding: LayerShape = field(default_factory=lambda: sliding(16, 8, 256, 1024))
    global_: LayerShape = field(default_factory=lambda: global_(16, 2, 512))
    dtype: torch.dtype = torch.bfloat16

    @property
    def sliding_capacity(self) -> int:
        return self.sliding.window

    @property
    def global_capacity(self) -> int:
        return self.len_hi + 1


A4B_DECODE = DecodeWorkload()


def scaled_down(w: PrefillWorkload, T: int, B: int | None = None, **layer_kw) -> PrefillWorkload:
    """Same layer shape with fewer tokens (parity cases the oracle finishes)."""
    lay = replace(w.layer, **layer_kw) if layer_kw else w.layer
    return replace(w, name=f"{w.name}-T{T}", T=T, B=B or w.B, layer=lay)


# -- draws -------------------------------------------------------------------

def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn(shape, g, device, dtype):
    """N(0,1) drawn in fp32 then rounded to dtype (chunked to bound memory)."""
    out = torch.empty(shape, device=device, dtype=dtype)
    flat = out.view(-1)
    step = 1 << 26
    for s in range(0, flat.numel(), step):
        n = min(step, flat.numel() - s)
        flat[s:s + n] = torch.randn(n, generator=g, device=device, dtype=torch.float32).to(dtype)
    return out


def norm_weight(d, g, device, dtype, kind):
    x = torch.randn(d, generator=g, device=device, dtype=torch.float32)
    if kind == "one_plus":
        x = 1.0 + 0.1 * x
    return x.to(dtype)


def block_starts(T: int, n_blocks: int, block_len: int, rng: np.random.Generator,
                 gap: int = 2) -> list[int]:
    """Sorted, non-overlapping block starts with at least `gap` text tokens
    between blocks (room for the image start/end markers)."""
    if n_blocks == 0:
        return []
    slack = T - n_blocks * (block_len + gap)
    if slack < 0:
        raise ValueError("blocks do not fit")
    u = np.sort(rng.integers(0, slack + 1, size=n_blocks))
    return [int(u[i]) + i * (block_len + gap) for i in range(n_blocks)]


def make_block_ids(B: int, T: int, n_blocks: int, block_len: int, seed: int) -> torch.Tensor | None:
    """int32 [B, T]: block index inside each image block, -1 on text."""
    if n_blocks == 0:
        return None
    rng = np.random.Generator(np.random.PCG64(seed))
    ids = np.full((B, T), -1, np.int32)
    for b in range(B):
        for i, s in enumerate(block_starts(T, n_blocks, block_len, rng)):
            ids[b, s:s + block_len] = i
    return torch.from_numpy(ids)


def prefill_inputs(w: PrefillWorkload, device="cpu", seed: int = 0) -> dict:
    """q_raw, k_raw, v_raw (None with K=V), w_q, w_k, image_block_ids."""
    L = w.layer
    g = _gen(device, seed)
    q = randn((w.B, w.T, L.num_heads, L.head_dim), g, device, w.dtype)
    k = randn((w.B, w.T, L.num_kv_heads, L.head_dim), g, device, w.dtype)
    v = None if L.k_eq_v else randn((w.B, w.T, L.num_kv_heads, L.head_dim), g, device, w.dtype)
    wq = norm_weight(L.head_dim, g, device, w.dtype, w.weights)
    wk = norm_weight(L.head_dim, g, device, w.dtype, w.weights)
    ids = make_block_ids(w.B, w.T, w.n_blocks, w.block_len, seed) if L.layer_type == SLIDING else None
    if ids is not None:
        ids = ids.to(device)
    return dict(q_raw=q, k_raw=k, v_raw=v, q_norm_w=wq, k_norm_w=wk, image_block_ids=ids)


# hidden size of the layer's input per variant ("gemma4-pt-claude" README,
# "Supported Models": E2B 1536, 12B 3840, 31B 5376)
HIDDEN = {"e2b-sliding-prefill": 1536, "12b-sliding-multimodal-prefill": 3840,
          "31b-global-prefill": 5376}


def projection_inputs(L: LayerShape, B: int, T: int, hidden: int, device="cpu", seed: int = 0,
                      with_kv: bool = True) -> dict:
    """Input of the QKV projection: x [B, T, hidden] ~ N(0, 1) and w_qkv
    [n_heads * d, hidden] ~ N(0, 1/hidden) (raw projections of unit
    variance; rows: the query heads, then the key heads, then the value heads
    unless K=V), and the norm weights; drawn in that order."""
    g = _gen(device, seed)
    n_heads = L.num_heads + ((L.num_kv_heads if L.k_eq_v else 2 * L.num_kv_heads)
                             if with_kv else 0)
    x = randn((B, T, hidden), g, device, torch.bfloat16)
    w = (randn((n_heads * L.head_dim, hidden), g, device, torch.float32) *
         hidden ** -0.5).to(torch.bfloat16)
    wq = norm_weight(L.head_dim, g, device, torch.bfloat16, "one_plus")
    wk = norm_weight(L.head_dim, g, device, torch.bfloat16, "one_plus") if with_kv else None
    return dict(x=x, w_qkv=w, q_norm_w=wq, k_norm_w=wk)


def vision_inputs(w: PrefillWorkload, device="cpu", seed: int = 0) -> dict:
    """Post-prologue inputs of a bidirectional layer (the tower applies its
    own 2-D rotary before attention): q_hat [B, T, Hq, d], k_hat and v_hat
    [B, Hkv, T, d], all N(0, 1) (unit RMS, like RMS-normalised vectors), and a
    padding mask [B, T] (uint8): image b has n_b valid patches, n_b uniform
    in [T/4, T] (numpy PCG64 with the seed), the rest is padding."""
    L = w.layer
    g = _gen(device, seed)
    q = randn((w.B, w.T, L.num_heads, L.head_dim), g, device, w.dtype)
    k = randn((w.B, L.num_kv_heads, w.T, L.head_dim), g, device, w.dtype)
    v = randn((w.B, L.num_kv_heads, w.T, L.head_dim), g, device, w.dtype)
    rng = np.random.Generator(np.random.PCG64(seed))
    n = rng.integers(w.T // 4, w.T, size=w.B, endpoint=True)
    keep = (np.arange(w.T)[None, :] < n[:, None]).astype(np.uint8)
    return dict(q_hat=q, k_hat=k, v_hat=v, attention_mask=torch.from_numpy(keep).to(device),
                valid=n.astype(np.int64))


def decode_lengths(w: DecodeWorkload, seed: int = 0) -> np.ndarray:
    """Tokens already in each sequence's cache, uniform in [len_lo, len_hi]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(w.len_lo, w.len_hi, size=w.batch, endpoint=True).astype(np.int32)


def decode_token_inputs(L: LayerShape, batch: int, g, device, dtype, with_kv=True) -> dict:
    """The new token's raw q (and k, v) and the layer's norm weights."""
    q = randn((batch, 1, L.num_heads, L.head_dim), g, device, dtype)
    k = randn((batch, 1, L.num_kv_heads, L.head_dim), g, device, dtype) if with_kv else None
    v = (randn((batch, 1, L.num_kv_heads, L.head_dim), g, device, dtype)
         if with_kv and not L.k_eq_v else None)
    wq = norm_weight(L.head_dim, g, device, dtype, "one_plus")
    wk = norm_weight(L.head_dim, g, device, dtype, "one_plus") if with_kv else None
    return dict(q_raw=q, k_raw=k, v_raw=v, q_norm_w=wq, k_norm_w=wk)


def fill_cache(cache_k: torch.Tensor, cache_v: torch.Tensor, lens, rolling: bool, g) -> None:
    """Post-prologue cache contents ~N(0,1) for positions 0..len[b]-1
    (a rolling cache: its whole ring).  Slots never written stay as they are."""
    B, Hkv, C, d = cache_k.shape
    for b in range(B):
        n = C if rolling else int(lens[b])
        for t in (cache_k, cache_v):
            t[b, :, :n] = randn((Hkv, n, d), g, t.device, t.dtype)
