"""GPU parity of g4attn_cache_append + g4attn_decode (split-KV partials and
combine) against the float64 oracle, including rolling caches, KV sharing and
the full-size 26B-A4B-shaped decode step on sampled sequences."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from attention_prologue_b200 import g4attn as G
from attention_prologue_b200 import workloads as W

from helpers import check, desc_of, gpu_prefill, oracle_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


def make_layer_state(L, B, cap, rolling, lens, seed, dtype=torch.bfloat16):
    """Cache pre-filled with N(0,1) post-prologue values for positions
    0..len-1 (slot p % cap when rolling) plus the new token's raw inputs."""
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    tok = W.decode_token_inputs(L, B, g, DEV, dtype)
    cache = G.KVCache.allocate(B, L.num_kv_heads, cap, L.head_dim, rolling=rolling, dtype=dtype,
                               device=DEV)
    W.fill_cache(cache.k, cache.v, lens, rolling, g)
    cache.len.copy_(torch.as_tensor(lens, dtype=torch.int32))
    return tok, cache


def oracle_decode(L, tok, cache_k_pre, cache_v_pre, cap, rolling, lens, src_tok=None,
                  src_layer=None):
    """Oracle decode from the pre-append cache; the new token's K/V come from
    the raw inputs of the layer that owns the cache."""
    s = src_tok or tok
    return oracle.decode(oracle_layer(L), tok["q_raw"].cpu(), tok["q_norm_w"].cpu(),
                         cache_k_pre, cache_v_pre, cap, rolling, lens,
                         k_new=s["k_raw"].cpu(),
                         v_new=None if s["v_raw"] is None else s["v_raw"].cpu(),
                         wk=s["k_norm_w"].cpu(), layer_kv=oracle_layer(src_layer or L))


@pytest.mark.parametrize("case", ["sliding", "sliding_rolling", "global_kv", "global_gqa_fp32"])
def test_decode_small(case):
    lens = [0, 5, 16, 17, 40, 300, 1000, 2500]
    B = len(lens)
    dtype = torch.bfloat16
    if case.startswith("sliding"):
        L = W.sliding(8, 2, 256, 64)
        rolling = case == "sliding_rolling"
        cap = 64 if rolling else 2600
    elif case == "global_kv":
        L = W.global_(16, 2, 512)
        rolling, cap = False, 2600
    else:
        L = W.global_(4, 1, 128, k_eq_v=False)
        rolling, cap, dtype = False, 2600, torch.float32
    tok, cache = make_layer_state(L, B, cap, rolling, lens, seed=1, dtype=dtype)
    ck, cv = cache.k.cpu(), cache.v.cpu()
    d = desc_of(L, dtype)
    G.g4attn_cache_append(d, cache, tok["k_raw"], tok["v_raw"], tok["k_norm_w"])
    out = G.g4attn_decode(d, cache, tok["q_raw"], tok["q_norm_w"])
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    assert cache.len.tolist() == [n + 1 for n in lens]
    ref = oracle_decode(L, tok, ck, cv, cap, rolling, lens)
    check(out[:, 0], ref, dtype, case)


def test_append_writes_the_prologue_of_the_new_token():
    L = W.global_(4, 2, 512)
    lens = [3, 100]
    tok, cache = make_layer_state(L, 2, 128, False, lens, seed=2)
    d = desc_of(L, torch.bfloat16)
    G.g4attn_cache_append(d, cache, tok["k_raw"], tok["v_raw"], tok["k_norm_w"])
    torch.cuda.synchronize()
    OL = oracle_layer(L)
    for b, p in enumerate(lens):
        for h in range(2):
            kh, vh = oracle.prologue_kv(OL, tok["k_raw"][b, 0, h].cpu(), None,
                                        tok["k_norm_w"].cpu(), p)
            for got, ref in ((cache.k[b, h, p], kh), (cache.v[b, h, p], vh)):
                g = got.double().cpu().numpy()
                assert np.max(np.abs(g - ref) / (np.abs(ref) + 1e-3)) < 2 ** -8 + 1e-6


def test_kv_shared_decode_reads_the_source_cache():
    src = W.global_(16, 2, 512)
    shared = replace(src, softmax_scale=0.05)
    lens = [10, 700, 1500]
    tok, cache = make_layer_state(src, 3, 2048, False, lens, seed=3)
    ck, cv = cache.k.cpu(), cache.v.cpu()
    g = torch.Generator(device=DEV)
    g.manual_seed(4)
    stok = W.decode_token_inputs(shared, 3, g, DEV, torch.bfloat16, with_kv=False)
    G.g4attn_cache_append(desc_of(src, torch.bfloat16), cache, tok["k_raw"], None, tok["k_norm_w"])
    out = G.g4attn_decode(desc_of(shared, torch.bfloat16), cache, stok["q_raw"], stok["q_norm_w"])
    torch.cuda.synchronize()
    ref = oracle_decode(shared, stok, ck, cv, 2048, False, lens, src_tok=tok, src_layer=src)
    check(out[:, 0], ref, torch.bfloat16, "kv-shared")


@pytest.mark.parametrize("layer", ["sliding", "global"])
def test_decode_equals_last_prefill_row(layer):
    """Decode after a prefill of T tokens and one append equals row T of a
    prefill over T + 1 tokens (both on the GPU; "gemma4-pt-claude" README,
    tests: a cached decode reproduces the uncached forward)."""
    L = W.sliding(8, 1, 256, 128) if layer == "sliding" else W.global_(8, 1, 512)
    T = 300
    w = W.PrefillWorkload("p", L, 2, T + 1)
    inp = W.prefill_inputs(w, DEV, 12)
    full = gpu_prefill(w, inp)
    d = desc_of(L, torch.bfloat16)
    cap = 128 if layer == "sliding" else 512
    cache = G.KVCache.allocate(2, 1, cap, L.head_dim, rolling=layer == "sliding", device=DEV)
    head = {k: (v[:, :T].contiguous() if v is not None and v.dim() == 4 else v) for k, v in inp.items()}
    G.g4attn_prefill(d, head["q_raw"], head["k_raw"], head["v_raw"], inp["q_norm_w"],
                     inp["k_norm_w"], cache=cache)
    last = lambda x: None if x is None else x[:, T:T + 1].contiguous()
    G.g4attn_cache_append(d, cache, last(inp["k_raw"]), last(inp["v_raw"]), inp["k_norm_w"])
    out = G.g4attn_decode(d, cache, last(inp["q_raw"]), inp["q_norm_w"])
    torch.cuda.synchronize()
    diff = (out[:, 0].float() - full[:, T].float()).abs()
    assert diff.max().item() <= 2e-2 and diff.mean().item() <= 2e-3


def test_overflow_and_empty_cache_are_reported():
    L = W.global_(4, 1, 128)
    d = desc_of(L, torch.bfloat16)
    tok, cache = make_layer_state(L, 2, 8, False, [8, 3], seed=5)
    G.g4attn_cache_append(d, cache, tok["k_raw"], None, tok["k_norm_w"])
    assert G.g4attn_get_device_status() == G.G4ATTN_ECACHE_OVERFLOW
    assert cache.len.tolist() == [8, 4]  # full sequence untouched, the other appended
    assert G.g4attn_get_device_status() == G.G4ATTN_OK  # cleared by the read
    cache.len.zero_()
    out = G.g4attn_decode(d, cache, tok["q_raw"], tok["q_norm_w"])
    assert G.g4attn_get_device_status() == G.G4ATTN_ECACHE_EMPTY
    assert torch.count_nonzero(out).item() == 0


def test_full_size_decode_step_sampled():
    """The 26B-A4B-shaped step at its full size: sliding layer on a rolling
    1024-slot cache (all 64 sequences), K=V global layer and the KV-shared
    layer on sampled sequences."""
    w = W.A4B_DECODE
    lens = W.decode_lengths(w, 0)
    S, Gl = w.sliding, w.global_
    X = replace(Gl, softmax_scale=Gl.scale * 0.5)
    s_tok, s_cache = make_layer_state(S, w.batch, w.sliding_capacity, True, lens, seed=10)
    g_tok, g_cache = make_layer_state(Gl, w.batch, w.global_capacity, False, lens, seed=11)
    gx = torch.Generator(device=DEV)
    gx.manual_seed(12)
    x_tok = W.decode_token_inputs(X, w.batch, gx, DEV, torch.bfloat16, with_kv=False)
    seqs = [int(np.argmin(lens)), int(np.argmax(lens)), 7, 33]
    n_max = int(lens[seqs].max()) + 1
    g_k = g_cache.k[seqs, :, :n_max].cpu()
    g_v = g_cache.v[seqs, :, :n_max].cpu()
    s_k, s_v = s_cache.k.cpu(), s_cache.v.cpu()
    ds, dg, dx = (desc_of(L, torch.bfloat16) for L in (S, Gl, X))
    G.g4attn_cache_append(ds, s_cache, s_tok["k_raw"], s_tok["v_raw"], s_tok["k_norm_w"])
    s_out = G.g4attn_decode(ds, s_cache, s_tok["q_raw"], s_tok["q_norm_w"])
    G.g4attn_cache_append(dg, g_cache, g_tok["k_raw"], None, g_tok["k_norm_w"])
    g_out = G.g4attn_decode(dg, g_cache, g_tok["q_raw"], g_tok["q_norm_w"])
    x_out = G.g4attn_decode(dx, g_cache, x_tok["q_raw"], x_tok["q_norm_w"])
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    check(s_out[:, 0], oracle_decode(S, s_tok, s_k, s_v, w.sliding_capacity, True, lens),
          torch.bfloat16, "sliding")
    sub = lambda t: {k: (v[seqs] if v is not None and v.dim() == 4 else v) for k, v in t.items()}
    check(g_out[seqs, 0], oracle_decode(Gl, sub(g_tok), g_k, g_v, n_max, False, lens[seqs]),
          torch.bfloat16, "global")
    check(x_out[seqs, 0], oracle_decode(X, sub(x_tok), g_k, g_v, n_max, False, lens[seqs],
                                        src_tok=sub(g_tok), src_layer=Gl), torch.bfloat16,
          "kv-shared")


def test_long_chunks_repeated():
    """Caches longer than 4096 positions are split into 2048-key chunks
    (128 tiles per CTA, many laps of the K/V ring); run several times."""
    L = W.global_(16, 2, 512)
    lens = [4097, 6000, 8190, 5000, 7777, 4500, 8100, 6543]
    tok, cache = make_layer_state(L, len(lens), 8192, False, lens, seed=21)
    ck, cv = cache.k.cpu(), cache.v.cpu()
    d = desc_of(L, torch.bfloat16)
    G.g4attn_cache_append(d, cache, tok["k_raw"], None, tok["k_norm_w"])
    ref = oracle_decode(L, tok, ck, cv, 8192, False, lens)
    for _ in range(3):
        out = G.g4attn_decode(d, cache, tok["q_raw"], tok["q_norm_w"])
        torch.cuda.synchronize()
        assert G.g4attn_get_device_status() == G.G4ATTN_OK
        check(out[:, 0], ref, torch.bfloat16, "long chunks")
