"""GPU parity of the bidirectional (vision-tower) layer type and of
g4attn_attend (attention from post-prologue inputs) against the float64
oracle.

Bidirectional: every query sees every key of its sequence ("gemma4-pt-claude"
README, "Key architectural features": a ViT-style vision encoder with
bidirectional attention; "Attention Backend Notes": scale 1.0).  The
attention from given q_hat / K / V is the step after a prologue that is not
the library's (the tower's own 2-D rotary) or that ran in the QKV
projection's epilogue; its inputs are bf16, so the oracle reads exactly the
values the kernels read."""
import numpy as np
import pytest
import torch

import oracle
from attention_prologue_b200 import g4attn as G
from attention_prologue_b200 import workloads as W

from helpers import (bf16_round, check, check_beyond_output_rounding, desc_of, oracle_layer,
                     record)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cache_of(k_hat, v_hat, C=None):
    """A two-tensor cache whose slots 0..T-1 hold k_hat/v_hat [B, Hkv, T, d]."""
    B, Hkv, T, d = k_hat.shape
    cache = G.KVCache.allocate(B, Hkv, C or T, d, dtype=k_hat.dtype, device=DEV)
    cache.k[:, :, :T] = k_hat
    cache.v[:, :, :T] = v_hat
    cache.len.fill_(T)
    return cache


def _oracle_attend(L, q_hat, k_hat, v_hat, p0=0, ids=None, keep=None, rows=None):
    """oracle.attend_rows on the exact bf16 values; k/v [B, Hkv, Tk, d]."""
    kh = k_hat.double().cpu().numpy().transpose(0, 2, 1, 3)
    vh = v_hat.double().cpu().numpy().transpose(0, 2, 1, 3)
    return oracle.attend_rows(oracle_layer(L), q_hat.double().cpu().numpy(), kh, vh, p0,
                              None if ids is None else ids.cpu().numpy(), rows,
                              attention_mask=None if keep is None else keep.cpu().numpy())


def _p_bound(v_hat):
    return 2.0 ** -9 * float(v_hat.abs().max())


@pytest.mark.parametrize("shape", ["d64", "d128", "d256", "d512", "f32"])
def test_bidirectional_prefill_matches_the_oracle(shape):
    """The whole prefill (prologue with 1-D RoPE on the token index, then
    bidirectional attention) at 1/sqrt(d), with padding on sequence 0."""
    if shape == "d64":
        L, B, T, dt = W.bidirectional(16, 16, 64, softmax_scale=0.125), 2, 600, torch.bfloat16
    elif shape == "d128":
        L, B, T, dt = W.bidirectional(8, 2, 128, softmax_scale=128 ** -0.5), 2, 500, torch.bfloat16
    elif shape == "d256":
        L, B, T, dt = W.bidirectional(8, 1, 256, softmax_scale=0.0625), 1, 700, torch.bfloat16
    elif shape == "d512":
        L = W.bidirectional(8, 1, 512, softmax_scale=512 ** -0.5, k_eq_v=True,
                            rotary_fraction=0.25, rope_theta=1e6)
        B, T, dt = 1, 600, torch.bfloat16
    else:
        L, B, T, dt = W.bidirectional(2, 1, 64, softmax_scale=1.0), 1, 64, torch.float32
    w = W.PrefillWorkload(f"bidir-{shape}", L, B, T, dt, weights="normal" if dt == torch.float32
                          else "one_plus")
    inp = W.prefill_inputs(w, DEV, 51)
    keep = torch.ones(B, T, dtype=torch.uint8)
    keep[0, T - 90:] = 0  # an image with fewer patches than the budget
    keep[0, 7:19] = 0
    out = G.g4attn_prefill(desc_of(L, dt), inp["q_raw"], inp["k_raw"], inp["v_raw"],
                           inp["q_norm_w"], inp["k_norm_w"], attention_mask=keep.to(DEV))
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    cpu = {k: (v.cpu() if v is not None else None) for k, v in inp.items()}
    ref = oracle.prefill(oracle_layer(L), cpu["q_raw"], cpu["k_raw"], cpu["v_raw"],
                         cpu["q_norm_w"], cpu["k_norm_w"], attention_mask=keep.numpy())
    check(out, ref, dt, w.name)


def test_bidirectional_prefill_at_scale_one():
    """Scale 1.0 on tensor cores: compared with the oracle's attention of the
    bf16-stored post-prologue vectors (the storage the library keeps them in;
    at scale 1 that rounding alone moves outputs past the bar)."""
    L = W.bidirectional(16, 16, 64)
    w = W.PrefillWorkload("bidir-d64-scale1", L, 2, 800)
    inp = W.prefill_inputs(w, DEV, 52)
    out = G.g4attn_prefill(desc_of(L, w.dtype), inp["q_raw"], inp["k_raw"], inp["v_raw"],
                           inp["q_norm_w"], inp["k_norm_w"])
    torch.cuda.synchronize()
    cpu = {k: (v.cpu() if v is not None else None) for k, v in inp.items()}
    OL = oracle_layer(L)
    qh = bf16_round(oracle.prologue_q_all(OL, cpu["q_raw"], cpu["q_norm_w"]))
    kh, vh = oracle.prefill_kv(OL, cpu["k_raw"], cpu["v_raw"], cpu["k_norm_w"])
    kh, vh = bf16_round(kh), bf16_round(vh)
    ref = oracle.attend_rows(OL, qh, kh, vh, 0)
    check_beyond_output_rounding(out, ref, "bidirectional d64 scale 1 (bf16-stored)",
                                 p_bound=2.0 ** -9 * float(np.abs(vh).max()))


def test_vision_shape_attend_sampled_rows():
    """The vision-tower workload itself (8 images of up to 2520 patches, 16
    heads of 64, scale 1.0, per-image padding), through g4attn_attend, on
    sampled rows of every image (first, last, the last valid patch, padding
    rows and a stride)."""
    w = W.VISION_BIDIR
    inp = W.vision_inputs(w, DEV, 53)
    cache = _cache_of(inp["k_hat"], inp["v_hat"])
    d = desc_of(w.layer, w.dtype)
    out = G.g4attn_attend(d, 0, inp["q_hat"], cache, attention_mask=inp["attention_mask"])
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    T = w.T
    rows = sorted({0, 1, 127, 128, 1000, T - 1, *range(64, T, 311),
                   *[int(n) - 1 for n in inp["valid"]], *[int(n) for n in inp["valid"] if n < T]})
    ref = _oracle_attend(w.layer, inp["q_hat"], inp["k_hat"], inp["v_hat"],
                         keep=inp["attention_mask"], rows=rows)
    check_beyond_output_rounding(out[:, rows], ref, "vision attend (sampled rows)",
                                 p_bound=_p_bound(inp["v_hat"]))


@pytest.mark.parametrize("case", ["sliding_blocks_p0", "global_k_eq_v_p0", "bidir_d128",
                                  "sliding_pad_softcap"])
def test_attend_matches_the_oracle(case):
    """g4attn_attend over a cache at a position offset: image blocks seen up to
    the chunk's last position, padding, soft-cap; all rows."""
    g = torch.Generator(device=DEV)
    g.manual_seed(54)
    ids = keep = None
    if case == "sliding_blocks_p0":
        L, B, T, p0 = W.sliding(8, 2, 256, 128), 2, 300, 200
        ids = torch.full((B, p0 + T), -1, dtype=torch.int32)
        ids[:, 150:260] = 0  # a block cut by the chunk boundary
        ids[1, 400:420] = 1
        ids = ids.to(DEV)
    elif case == "global_k_eq_v_p0":
        L, B, T, p0 = W.global_(8, 1, 512), 1, 260, 400
    elif case == "bidir_d128":
        L, B, T, p0 = W.bidirectional(4, 4, 128), 2, 700, 0
    else:
        L, B, T, p0 = W.sliding(4, 1, 128, 64, logit_softcap=5.0), 2, 400, 100
        keep = (torch.rand(B, p0 + T, generator=torch.Generator().manual_seed(55)) > 0.25)
        keep = keep.to(torch.uint8).to(DEV)
    Hq, Hkv, hd = L.num_heads, L.num_kv_heads, L.head_dim
    q = W.randn((B, T, Hq, hd), g, DEV, torch.bfloat16)
    k = W.randn((B, Hkv, p0 + T, hd), g, DEV, torch.bfloat16)
    v = W.randn((B, Hkv, p0 + T, hd), g, DEV, torch.bfloat16)
    cache = _cache_of(k, v, C=p0 + T + 5)
    out = G.g4attn_attend(desc_of(L, torch.bfloat16), p0, q, cache, image_block_ids=ids,
                          attention_mask=keep)
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    ref = _oracle_attend(L, q, k, v, p0, ids, keep)
    check_beyond_output_rounding(out, ref, f"attend {case}", p_bound=_p_bound(v))
    record(out, ref, f"attend {case} (plain bar)")


def test_bidirectional_cached_prefill_chunks():
    """A bidirectional layer through g4attn_prefill then g4attn_prefill_chunk:
    the chunk's rows see every key up to the chunk's last position (the first
    chunk's rows saw only their own chunk); both against the oracle."""
    L = W.bidirectional(8, 2, 128, softmax_scale=128 ** -0.5)
    B, T, p0 = 2, 520, 300
    w = W.PrefillWorkload("bidir-chunks", L, B, T)
    inp = W.prefill_inputs(w, DEV, 56)
    d = desc_of(L, torch.bfloat16)
    cache = G.KVCache.allocate(B, 2, T, 128, device=DEV)
    sl = lambda t, a, b: t[:, a:b].contiguous()
    o0 = G.g4attn_prefill(d, sl(inp["q_raw"], 0, p0), sl(inp["k_raw"], 0, p0),
                          sl(inp["v_raw"], 0, p0), inp["q_norm_w"], inp["k_norm_w"], cache=cache)
    o1 = G.g4attn_prefill_chunk(d, p0, sl(inp["q_raw"], p0, T), sl(inp["k_raw"], p0, T),
                                sl(inp["v_raw"], p0, T), inp["q_norm_w"], inp["k_norm_w"], None,
                                cache)
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    cpu = {k: (v.cpu() if v is not None else None) for k, v in inp.items()}
    OL = oracle_layer(L)
    ref0 = oracle.prefill(OL, cpu["q_raw"][:, :p0], cpu["k_raw"][:, :p0], cpu["v_raw"][:, :p0],
                          cpu["q_norm_w"], cpu["k_norm_w"])
    kh, vh = oracle.prefill_kv(OL, cpu["k_raw"][:, :p0], cpu["v_raw"][:, :p0], cpu["k_norm_w"])
    ref1, _, _ = oracle.prefill_chunk(OL, cpu["q_raw"][:, p0:], cpu["k_raw"][:, p0:],
                                      cpu["v_raw"][:, p0:], cpu["q_norm_w"], cpu["k_norm_w"], kh, vh)
    check(o0, ref0, torch.bfloat16, "bidirectional first chunk")
    check(o1, ref1, torch.bfloat16, "bidirectional cached chunk")
