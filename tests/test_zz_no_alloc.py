"""g4attn_decode_noalloc: decode for callers that cannot give the library
device memory per call (a runtime whose free device memory all belongs to
its KV-cache pool, a plugin host without an allocator).  Its split-KV partials
live in a fixed 16 MiB device array inside the library instead of a
caller-supplied workspace.

Checked through the C ABI against g4attn_decode (the entry point with a
workspace) on two calls in a row: the second call finds the first call's
leftovers in the shared array and must not depend on them.  This file is
collected last so that a run stopping at the first failure has already run
every other test."""
import numpy as np
import pytest
import torch

import oracle
from attention_prologue_b200 import g4attn as G
from attention_prologue_b200 import workloads as W

from helpers import BF16_MAX_ABS, BF16_MEAN_ABS, check, desc_of, oracle_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


def layer_state(L, B, cap, rolling, lens, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    tok = W.decode_token_inputs(L, B, g, DEV, torch.bfloat16)
    cache = G.KVCache.allocate(B, L.num_kv_heads, cap, L.head_dim, rolling=rolling, device=DEV)
    W.fill_cache(cache.k, cache.v, lens, rolling, g)
    cache.len.copy_(torch.as_tensor(lens, dtype=torch.int32))
    d = desc_of(L, torch.bfloat16)
    G.g4attn_cache_append(d, cache, tok["k_raw"], tok["v_raw"], tok["k_norm_w"])
    return d, tok, cache


def close(a, b):
    err = (a.float() - b.float()).abs()
    return err.max().item() <= BF16_MAX_ABS and err.mean().item() <= BF16_MEAN_ABS


def test_decode_noalloc_matches_decode_on_two_calls_in_a_row():
    rng = np.random.default_rng(21)
    # call 1: K=V global layer whose usual chunk count does not fit the fixed
    # array (64 sequences x 16 heads x 514 floats per chunk), so the keys are
    # cut into fewer, longer chunks
    Lg = W.global_(16, 2, 512)
    lens_g = rng.integers(1000, 32767, size=64).astype(np.int32)
    dg, tg, cg = layer_state(Lg, 64, 32768, False, lens_g, seed=1)
    # call 2: sliding layer on a rolling cache, where the usual plan fits
    Ls = W.sliding(16, 8, 256, 1024)
    lens_s = rng.integers(1, 5000, size=8).astype(np.int32)
    ds, ts, cs = layer_state(Ls, 8, 1024, True, lens_s, seed=2)

    ref_g = G.g4attn_decode(dg, cg, tg["q_raw"], tg["q_norm_w"])
    ref_s = G.g4attn_decode(ds, cs, ts["q_raw"], ts["q_norm_w"])
    out_g = G.g4attn_decode_noalloc(dg, cg, tg["q_raw"], tg["q_norm_w"])
    out_s = G.g4attn_decode_noalloc(ds, cs, ts["q_raw"], ts["q_norm_w"])
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    assert close(out_g, ref_g)
    assert close(out_s, ref_s)
    # the usual plan fits for the sliding layer: the same kernels, same chunks
    assert torch.equal(out_s, ref_s)


def test_decode_noalloc_rejects_a_batch_beyond_the_fixed_array():
    # one chunk of partials: 4096 x 16 x (512 + 2) x 4 bytes > 16 MiB
    L = W.global_(16, 2, 512)
    d = desc_of(L, torch.bfloat16)
    cache = G.KVCache.allocate(4096, 2, 8, 512, device=DEV)
    q = torch.zeros(4096, 1, 16, 512, dtype=torch.bfloat16, device=DEV)
    w = torch.ones(512, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(G.G4AttnError) as e:
        G.g4attn_decode_noalloc(d, cache, q, w)
    assert e.value.status == G.G4ATTN_EWORKSPACE


def oracle_rows(L, tok, k_pre, v_pre, cap, lens, seqs):
    """The float64 oracle's decode of the sampled sequences, from the cache
    contents before the append and the new token's raw inputs."""
    sel = torch.as_tensor(seqs)
    return oracle.decode(oracle_layer(L), tok["q_raw"].cpu()[sel], tok["q_norm_w"].cpu(),
                         k_pre, v_pre, cap, False, np.asarray(lens)[seqs],
                         k_new=tok["k_raw"].cpu()[sel],
                         v_new=None if tok["v_raw"] is None else tok["v_raw"].cpu()[sel],
                         wk=tok["k_norm_w"].cpu())


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_noalloc_reduced_chunk_plan_matches_the_oracle(dtype):
    """When the usual chunk count does not fit the fixed array the keys are
    cut into fewer, longer chunks: check that plan against the float64
    oracle on sampled sequences.  bf16: the K=V global layer of the 26B-A4B
    shape (64 sequences, 16 heads on 2 KV heads, 7 chunks of 4976 keys in
    place of 17 of 2048; tensor-core split kernel).  fp32: 64 query heads on
    one KV head, head_dim 64 (15 chunks of 2336 keys in place of 17; the
    CUDA-core split kernel)."""
    rng = np.random.default_rng(23)
    if dtype == torch.bfloat16:
        L, cap = W.global_(16, 2, 512), 32768
    else:
        L, cap = W.global_(64, 1, 64), 32768
    B = 64
    lens = rng.integers(1000, cap - 1, size=B).astype(np.int32)
    lens[:2] = (cap - 1, 1)  # the longest span the plan must cover, and a single key
    g = torch.Generator(device=DEV)
    g.manual_seed(24)
    tok = W.decode_token_inputs(L, B, g, DEV, dtype)
    cache = G.KVCache.allocate(B, L.num_kv_heads, cap, L.head_dim, dtype=dtype, device=DEV)
    W.fill_cache(cache.k, cache.v, lens, False, g)
    cache.len.copy_(torch.as_tensor(lens, dtype=torch.int32))
    seqs = [0, 1, 2, 17, 40, 63]
    sel = torch.as_tensor(seqs, device=DEV)
    k_pre, v_pre = cache.k[sel].cpu(), cache.v[sel].cpu()
    d = desc_of(L, dtype)
    G.g4attn_cache_append(d, cache, tok["k_raw"], tok["v_raw"], tok["k_norm_w"])
    out = G.g4attn_decode_noalloc(d, cache, tok["q_raw"], tok["q_norm_w"])
    again = G.g4attn_decode_noalloc(d, cache, tok["q_raw"], tok["q_norm_w"])
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    assert torch.equal(out, again)
    ref = oracle_rows(L, tok, k_pre, v_pre, cap, lens, seqs)
    check(out[sel, 0], ref, dtype, f"decode_noalloc reduced plan {dtype}")
