"""GPU parity of the single-tensor cache of K=V layers against the float64
oracle.  On a K=V layer ("Gemma 4" Keras docs, "What changed from Gemma 3")
V = RMSNorm(k_raw) and K = RoPE(V * w_k) derive from one raw vector, so the
cache can hold V alone and decode rebuilds K from it (half the bytes a decode
step reads).  The prompt's keys go in through g4attn_prefill (which writes V
alone into such a cache) and g4attn_cache_append; the oracle decodes from the
same raw inputs, so nothing it reads comes from the CUDA path."""
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


def _oracle_cache(kh, C):
    """[B, T, Hkv, d] post-prologue values -> an oracle cache [B, Hkv, C, d]."""
    B, T, Hkv, d = kh.shape
    c = np.zeros((B, Hkv, C, d))
    c[:, :, :T] = kh.transpose(0, 2, 1, 3)
    return c


@pytest.mark.parametrize("hd,heads", [(512, (16, 2)), (256, (8, 2)), (128, (8, 1))])
def test_single_cache_prefill_append_decode(hd, heads):
    """Prefill a prompt into a single-tensor cache, append one token, decode;
    and a KV-shared layer decoding from the same cache.  Per-sequence prompt
    lengths: after the prefill, len is cut back so sequences differ."""
    Hq, Hkv = heads
    L = W.global_(Hq, Hkv, hd)  # K=V, 25% rotated (for d 128 and 256 the
    B, T, C = 4, 700, 768     # rotated dims share 64-dim boxes with unrotated ones)
    w = W.PrefillWorkload(f"single-{hd}", L, B, T + 1)
    inp = W.prefill_inputs(w, DEV, 41)
    d = desc_of(L, torch.bfloat16)
    cache = G.KVCache.allocate(B, Hkv, C, hd, device=DEV, single=True, k_norm_w=inp["k_norm_w"])
    head_q = inp["q_raw"][:, :T].contiguous()
    head_k = inp["k_raw"][:, :T].contiguous()
    G.g4attn_prefill(d, head_q, head_k, None, inp["q_norm_w"], inp["k_norm_w"], cache=cache)
    lens = [T, 1, 333, 640]
    cache.len.copy_(torch.as_tensor(lens, dtype=torch.int32))
    # the new token of each sequence: the raw inputs at position T (any raw
    # vector will do; its position in the prompt is len[b])
    new_k = inp["k_raw"][:, T:].contiguous()
    new_q = inp["q_raw"][:, T:].contiguous()
    G.g4attn_cache_append(d, cache, new_k, None, inp["k_norm_w"])
    out = G.g4attn_decode(d, cache, new_q, inp["q_norm_w"])
    # a KV-shared layer: own queries and query-norm weight, the source's cache
    g = torch.Generator(device=DEV)
    g.manual_seed(42)
    Lx = replace(L, softmax_scale=0.05)
    xq = W.randn((B, 1, Hq, hd), g, DEV, torch.bfloat16)
    xw = W.norm_weight(hd, g, DEV, torch.bfloat16, "one_plus")
    outx = G.g4attn_decode(desc_of(Lx, torch.bfloat16), cache, xq, xw)
    outn = G.g4attn_decode_noalloc(d, cache, new_q, inp["q_norm_w"])
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    assert cache.len.tolist() == [n + 1 for n in lens]
    OL = oracle_layer(L)
    kh, vh = oracle.prefill_kv(OL, head_k.cpu(), None, inp["k_norm_w"].cpu())
    ck, cv = _oracle_cache(kh, C), _oracle_cache(vh, C)
    ref = oracle.decode(OL, new_q.cpu(), inp["q_norm_w"].cpu(), ck, cv, C, False, lens,
                        k_new=new_k.cpu(), wk=inp["k_norm_w"].cpu())
    check(out[:, 0], ref, torch.bfloat16, f"single-tensor decode d{hd}")
    check(outn[:, 0], ref, torch.bfloat16, f"single-tensor decode_noalloc d{hd}")
    # the shared layer reads the cache after the append: the new token's K/V
    # at position len[b] (the oracle's key prologue there)
    ck2, cv2 = ck.copy(), cv.copy()
    for b, n in enumerate(lens):
        for h in range(Hkv):
            kk, vv = oracle.prologue_kv(OL, new_k[b, 0, h].cpu(), None, inp["k_norm_w"].cpu(), n)
            ck2[b, h, n], cv2[b, h, n] = kk, vv
    refx = oracle.decode(oracle_layer(Lx), xq.cpu(), xw.cpu(), ck2, cv2, C, False,
                         [n + 1 for n in lens], layer_kv=OL)
    check(outx[:, 0], refx, torch.bfloat16, f"single-tensor KV-shared decode d{hd}")


def test_single_cache_with_padding_and_softcap():
    L = W.global_(16, 2, 512, logit_softcap=4.0, softmax_scale=1.0 / 8)
    B, T, C = 3, 500, 512
    w = W.PrefillWorkload("single-pad", L, B, T + 1)
    inp = W.prefill_inputs(w, DEV, 43)
    d = desc_of(L, torch.bfloat16)
    cache = G.KVCache.allocate(B, 2, C, 512, device=DEV, single=True, k_norm_w=inp["k_norm_w"])
    keep = np.ones((B, T), np.uint8)
    keep[0, :120] = 0
    keep[1] = (np.random.default_rng(44).random(T) > 0.3)
    cache.key_mask = torch.from_numpy(keep).to(DEV)
    G.g4attn_prefill(d, inp["q_raw"][:, :T].contiguous(), inp["k_raw"][:, :T].contiguous(), None,
                     inp["q_norm_w"], inp["k_norm_w"], cache=cache,
                     attention_mask=cache.key_mask)
    new_k = inp["k_raw"][:, T:].contiguous()
    new_q = inp["q_raw"][:, T:].contiguous()
    G.g4attn_cache_append(d, cache, new_k, None, inp["k_norm_w"])
    out = G.g4attn_decode(d, cache, new_q, inp["q_norm_w"])
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    OL = oracle_layer(L)
    kh, vh = oracle.prefill_kv(OL, inp["k_raw"][:, :T].cpu(), None, inp["k_norm_w"].cpu())
    ref = oracle.decode(OL, new_q.cpu(), inp["q_norm_w"].cpu(), _oracle_cache(kh, C),
                        _oracle_cache(vh, C), C, False, [T] * B, k_new=new_k.cpu(),
                        wk=inp["k_norm_w"].cpu(), attention_mask=keep)
    check(out[:, 0], ref, torch.bfloat16, "single-tensor decode, padding + soft-cap")


def test_single_cache_long_sequences_match_the_two_tensor_cache():
    """Long caches (several split-KV chunks, the 26B-A4B global layer's
    shape): the single-tensor decode equals the two-tensor one within the
    bf16 tolerance, and sampled sequences match the oracle."""
    L = W.global_(16, 2, 512)
    B, C = 8, 9000
    rng = np.random.default_rng(45)
    lens = rng.integers(4000, C - 1, size=B).astype(np.int32)
    g = torch.Generator(device=DEV)
    g.manual_seed(46)
    k_all = W.randn((B, C - 1, 2, 512), g, DEV, torch.bfloat16)
    q_all = W.randn((B, 1, 16, 512), g, DEV, torch.bfloat16)
    wq = W.norm_weight(512, g, DEV, torch.bfloat16, "one_plus")
    wk = W.norm_weight(512, g, DEV, torch.bfloat16, "one_plus")
    d = desc_of(L, torch.bfloat16)
    single = G.KVCache.allocate(B, 2, C, 512, device=DEV, single=True, k_norm_w=wk)
    both = G.KVCache.allocate(B, 2, C, 512, device=DEV)
    # the caches' contents: the key prologue of every position, written by
    # an append per position would be slow; a prefill of a short query does it
    qz = torch.zeros(B, C - 1, 16, 512, dtype=torch.bfloat16, device=DEV)
    for cache in (single, both):
        G.g4attn_prefill(d, qz, k_all, None, wq, wk, cache=cache)
        cache.len.copy_(torch.as_tensor(lens, dtype=torch.int32))
    new_k = W.randn((B, 1, 2, 512), g, DEV, torch.bfloat16)
    outs = []
    for cache in (single, both):
        G.g4attn_cache_append(d, cache, new_k, None, wk)
        outs.append(G.g4attn_decode(d, cache, q_all, wq))
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    err = (outs[0].float() - outs[1].float()).abs()
    assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3, err.max().item()
    seqs = [0, 5]
    OL = oracle_layer(L)
    sel = torch.as_tensor(seqs)
    kh, vh = oracle.prefill_kv(OL, k_all[sel].cpu(), None, wk.cpu())
    ref = oracle.decode(OL, q_all[sel].cpu(), wq.cpu(), _oracle_cache(kh, C),
                        _oracle_cache(vh, C), C, False, lens[seqs], k_new=new_k[sel].cpu(),
                        wk=wk.cpu())
    check(outs[0][sel, 0], ref, torch.bfloat16, "single-tensor decode, long caches")
