"""GPU parity of the padding mask and the attention-logit soft-cap against the
float64 oracle, on every kernel family: the tcgen05 prefill kernels (head_dim
128/256 and the head_dim-512 CTA pair), the CUDA-core fp32 prefill, the
cached-prefill chunk, and decode (tensor-core and CUDA-core split kernels).

Padding: "Gemma 4" Keras docs, "Gemma4ConditionalGenerate" arguments
(attention_mask (batch, seq), 1 = keep, 0 = padding).  Soft-cap:
"gemma4-pt-claude" README, "Attention Backend Notes" (attn_logits_soft_cap),
read as s -> c tanh(s / c) after the softmax scale.  A row left without any
key outputs 0."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from attention_prologue_b200 import g4attn as G
from attention_prologue_b200 import workloads as W

from helpers import check, desc_of, oracle_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


def padding(B, T, seed, left=(0,), holes=0.0, dead=None):
    """uint8 [B, T]: sequence b left-padded by left[b % len(left)] tokens,
    then random holes with probability `holes`; `dead` = (start, end) makes
    that span of sequence 0 padding too."""
    rng = np.random.default_rng(seed)
    keep = np.ones((B, T), np.uint8)
    for b in range(B):
        keep[b, :left[b % len(left)]] = 0
    if holes:
        keep &= (rng.random((B, T)) >= holes).astype(np.uint8)
    if dead:
        keep[0, dead[0]:dead[1]] = 0
    return torch.from_numpy(keep)


def run_prefill(w, seed, keep, dtype=None):
    inp = W.prefill_inputs(w, DEV, seed)
    d = desc_of(w.layer, w.dtype)
    out = G.g4attn_prefill(d, inp["q_raw"], inp["k_raw"], inp["v_raw"], inp["q_norm_w"],
                           inp["k_norm_w"], inp["image_block_ids"],
                           attention_mask=None if keep is None else keep.to(DEV))
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    cpu = {k: (v.cpu() if v is not None else None) for k, v in inp.items()}
    ids = cpu["image_block_ids"]
    ref = oracle.prefill(oracle_layer(w.layer), cpu["q_raw"], cpu["k_raw"], cpu["v_raw"],
                         cpu["q_norm_w"], cpu["k_norm_w"],
                         block_ids=None if ids is None else ids.numpy(),
                         attention_mask=None if keep is None else keep.numpy())
    check(out, ref, w.dtype, w.name)
    return out, ref


PREFILL = [
    # tcgen05, head_dim 256, GQA 8:1, window 64: left padding past the first
    # window (rows 0..99 of sequence 0 see no key) and holes
    (W.PrefillWorkload("pad-s256", W.sliding(8, 1, 256, 64), 2, 700), dict(left=(100, 3), holes=0.2)),
    # image blocks with padding inside and around them
    (W.PrefillWorkload("pad-s256-blocks", W.sliding(4, 2, 256, 96), 2, 900, n_blocks=2,
                       block_len=140), dict(left=(37, 0), holes=0.1)),
    (W.PrefillWorkload("pad-s128", W.sliding(4, 2, 128, 40), 2, 300), dict(left=(5,), holes=0.3)),
    # head_dim 512 pair, K=V, global: a dead span of 200 keys
    (W.PrefillWorkload("pad-g512", W.global_(8, 1, 512), 1, 800), dict(left=(64,), holes=0.15,
                                                                      dead=(300, 500))),
    (W.PrefillWorkload("pad-g256", W.global_(8, 2, 256), 2, 500), dict(left=(130, 0), holes=0.5)),
    # fp32 CUDA-core path
    (W.PrefillWorkload("pad-f32", W.sliding(2, 1, 64, 16), 1, 64, torch.float32, weights="normal"),
     dict(left=(20,), holes=0.3)),
]


@pytest.mark.parametrize("w,pad", PREFILL, ids=[p[0].name for p in PREFILL])
def test_prefill_with_padding(w, pad):
    keep = padding(w.B, w.T, 5, **pad)
    out, ref = run_prefill(w, 7, keep)
    # rows with no key left (sequence 0's first rows on the windowed layer)
    if w.name == "pad-s256":
        assert not out[0, :100].any()


@pytest.mark.parametrize("cap", [1.5, 30.0])
@pytest.mark.parametrize("shape", ["s256", "g512", "s128", "f32"])
def test_prefill_with_softcap(shape, cap):
    if shape == "s256":
        w = W.PrefillWorkload("cap-s256", W.sliding(8, 1, 256, 512, logit_softcap=cap), 1, 1000)
    elif shape == "g512":
        w = W.PrefillWorkload("cap-g512", W.global_(8, 1, 512, logit_softcap=cap), 1, 700)
    elif shape == "s128":
        w = W.PrefillWorkload("cap-s128", W.global_(4, 2, 128, k_eq_v=False, logit_softcap=cap),
                              2, 300)
    else:
        w = W.PrefillWorkload("cap-f32", W.global_(2, 1, 64, logit_softcap=cap), 1, 64,
                              torch.float32, weights="normal")
    # scale 1.0 with a tight cap: the cap decides most weights
    if cap < 5:
        w = replace(w, layer=replace(w.layer, softmax_scale=1.0 if w.dtype == torch.float32
                                     else w.layer.softmax_scale))
    run_prefill(w, 8, None)


def test_padding_and_softcap_together_at_scale_one_tiny_fp32():
    w = W.PrefillWorkload("pad-cap-f32", W.sliding(2, 1, 64, 16, softmax_scale=1.0,
                                                   logit_softcap=4.0), 2, 64, torch.float32,
                          weights="normal")
    run_prefill(w, 9, padding(2, 64, 6, left=(10, 0), holes=0.25))


def test_all_ones_mask_changes_nothing():
    w = W.PrefillWorkload("ones", W.sliding(8, 2, 256, 128), 1, 500)
    inp = W.prefill_inputs(w, DEV, 3)
    d = desc_of(w.layer, w.dtype)
    a = G.g4attn_prefill(d, inp["q_raw"], inp["k_raw"], inp["v_raw"], inp["q_norm_w"],
                         inp["k_norm_w"])
    b = G.g4attn_prefill(d, inp["q_raw"], inp["k_raw"], inp["v_raw"], inp["q_norm_w"],
                         inp["k_norm_w"],
                         attention_mask=torch.ones(1, 500, dtype=torch.uint8, device=DEV))
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# -- cached prefill chunk with padding ----------------------------------------

@pytest.mark.parametrize("hd,layer", [(256, "sliding"), (512, "global")])
def test_chunk_with_padding_and_softcap(hd, layer):
    L = (W.sliding(8, 2, hd, 200, logit_softcap=20.0) if layer == "sliding"
         else W.global_(8, 2, hd, logit_softcap=20.0))
    B, T, p0 = 2, 650, 400
    w = W.PrefillWorkload(f"chunk-pad-{layer}", L, B, T)
    inp = W.prefill_inputs(w, DEV, 12)
    keep = padding(B, T, 13, left=(150, 7), holes=0.2)
    d = desc_of(L, w.dtype)
    cache = G.KVCache.allocate(B, L.num_kv_heads, T, hd, device=DEV)
    sl0, sl1 = slice(0, p0), slice(p0, T)
    vv = (lambda s: None if inp["v_raw"] is None else inp["v_raw"][:, s].contiguous())
    o0 = G.g4attn_prefill(d, inp["q_raw"][:, sl0].contiguous(), inp["k_raw"][:, sl0].contiguous(),
                          vv(sl0), inp["q_norm_w"], inp["k_norm_w"], cache=cache,
                          attention_mask=keep[:, :p0].contiguous().to(DEV))
    o1 = G.g4attn_prefill_chunk(d, p0, inp["q_raw"][:, sl1].contiguous(),
                                inp["k_raw"][:, sl1].contiguous(), vv(sl1), inp["q_norm_w"],
                                inp["k_norm_w"], None, cache,
                                attention_mask=keep.contiguous().to(DEV))
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    cpu = {k: (v.cpu() if v is not None else None) for k, v in inp.items()}
    ref = oracle.prefill(oracle_layer(L), cpu["q_raw"], cpu["k_raw"], cpu["v_raw"],
                         cpu["q_norm_w"], cpu["k_norm_w"], attention_mask=keep.numpy())
    check(o0, ref[:, :p0], w.dtype, f"{w.name} first part")
    check(o1, ref[:, p0:], w.dtype, f"{w.name} chunk")


# -- decode with the cache's padding mask -------------------------------------

@pytest.mark.parametrize("case", ["global_d512", "sliding_rolling", "fp32_split", "softcap_d512"])
def test_decode_with_padding(case):
    lens = [5, 40, 300, 1000, 2500, 64, 700, 17]
    B = len(lens)
    dtype = torch.bfloat16
    rolling, cap = False, 2600
    if case == "global_d512":
        L = W.global_(16, 2, 512)
    elif case == "softcap_d512":
        L = W.global_(16, 2, 512, softmax_scale=1.0 / 8, logit_softcap=3.0)
    elif case == "sliding_rolling":
        L = W.sliding(8, 2, 256, 64)
        rolling, cap = True, 64
    else:
        L = W.global_(4, 1, 128, k_eq_v=False, logit_softcap=5.0)
        dtype = torch.float32
    g = torch.Generator(device=DEV)
    g.manual_seed(14)
    tok = W.decode_token_inputs(L, B, g, DEV, dtype)
    cache = G.KVCache.allocate(B, L.num_kv_heads, cap, L.head_dim, rolling=rolling, dtype=dtype,
                               device=DEV)
    W.fill_cache(cache.k, cache.v, lens, rolling, g)
    cache.len.copy_(torch.as_tensor(lens, dtype=torch.int32))
    # prompt padding over the first 1200 positions; sequence 0 (5 tokens)
    # has only padding before its new token
    keep = padding(B, 1200, 15, left=(5, 30, 0, 200), holes=0.2)
    cache.key_mask = keep.to(DEV)
    ck, cv = cache.k.cpu(), cache.v.cpu()
    d = desc_of(L, dtype)
    G.g4attn_cache_append(d, cache, tok["k_raw"], tok["v_raw"], tok["k_norm_w"])
    out = G.g4attn_decode(d, cache, tok["q_raw"], tok["q_norm_w"])
    out2 = G.g4attn_decode_noalloc(d, cache, tok["q_raw"], tok["q_norm_w"])
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    ref = oracle.decode(oracle_layer(L), tok["q_raw"].cpu(), tok["q_norm_w"].cpu(), ck, cv, cap,
                        rolling, lens, k_new=tok["k_raw"].cpu(),
                        v_new=None if tok["v_raw"] is None else tok["v_raw"].cpu(),
                        wk=tok["k_norm_w"].cpu(), attention_mask=keep.numpy())
    check(out[:, 0], ref, dtype, f"decode padding {case}")
    check(out2[:, 0], ref, dtype, f"decode_noalloc padding {case}")
