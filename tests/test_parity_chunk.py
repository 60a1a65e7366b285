"""GPU parity of g4attn_prefill_chunk (cached prefill: a chunk of a prompt
after the positions a layer's cache already holds) against the float64
oracle's chunked path ("gemma4-pt-claude" README, "Tests": the cached path
reproduces the uncached forward pass, image spans included).

Each case runs a prompt through the library in chunks cut between image
blocks (the first chunk with g4attn_prefill into the cache) and compares
every chunk's output with the oracle's rows of that chunk, and the cache's
keys/values with the oracle's."""
import numpy as np
import pytest
import torch

import oracle
from attention_prologue_b200 import g4attn as G
from attention_prologue_b200 import workloads as W

from helpers import check, desc_of, oracle_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_chunks(w, cuts, seed, cap=None, rolling=False, inp=None):
    if inp is None:
        inp = W.prefill_inputs(w, DEV, seed)
    d = desc_of(w.layer, w.dtype)
    B, T = w.B, w.T
    Hkv, hd = w.layer.num_kv_heads, w.layer.head_dim
    dt = torch.bfloat16 if w.dtype == torch.bfloat16 else torch.float32
    cache = G.KVCache.allocate(B, Hkv, cap or T, hd, rolling=rolling, device=DEV, dtype=dt)
    ids = inp["image_block_ids"]
    v = inp["v_raw"]
    outs = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        sl = slice(a, b)
        q = inp["q_raw"][:, sl].contiguous()
        k = inp["k_raw"][:, sl].contiguous()
        vv = None if v is None else v[:, sl].contiguous()
        if a == 0:
            o = G.g4attn_prefill(d, q, k, vv, inp["q_norm_w"], inp["k_norm_w"],
                                 None if ids is None else ids[:, :b].contiguous(), cache=cache)
        else:
            o = G.g4attn_prefill_chunk(d, a, q, k, vv, inp["q_norm_w"], inp["k_norm_w"],
                                       None if ids is None else ids[:, :b].contiguous(), cache)
        outs.append(o)
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    assert cache.len.tolist() == [T] * B
    cpu = {k: (x.cpu() if x is not None else None) for k, x in inp.items()}
    L = oracle_layer(w.layer)
    kh = np.zeros((B, 0, Hkv, hd))
    vh = np.zeros((B, 0, Hkv, hd))
    for (a, b), o in zip(zip(cuts[:-1], cuts[1:]), outs):
        sl = slice(a, b)
        ref, kh, vh = oracle.prefill_chunk(
            L, cpu["q_raw"][:, sl], cpu["k_raw"][:, sl],
            None if cpu["v_raw"] is None else cpu["v_raw"][:, sl], cpu["q_norm_w"],
            cpu["k_norm_w"], kh, vh,
            block_ids=None if cpu["image_block_ids"] is None else cpu["image_block_ids"][:, :b].numpy())
        check(o, ref, w.dtype, f"{w.name} chunk [{a}, {b})")
    return cache, kh, vh


@pytest.mark.parametrize("shape", ["sliding-d256-blocks", "global-d512-kv", "global-d128",
                                   "sliding-d64-gqa", "tiny-fp32"])
def test_chunked_prefill_matches_the_oracle(shape):
    inp = None
    if shape == "sliding-d256-blocks":
        w = W.PrefillWorkload("chunk-s256", W.sliding(8, 2, 256, 512), 2, 1500, n_blocks=2,
                              block_len=280)
        inp = W.prefill_inputs(w, DEV, 3)
        ids = inp["image_block_ids"].cpu().numpy()
        # cut where no block continues across (the oracle's reading of image
        # spans in a cached prefill), with windows reaching across the cuts
        free = [t for t in range(200, w.T - 200)
                if all(ids[b, t - 1] < 0 or ids[b, t] < 0 for b in range(w.B))]
        cuts = [0, free[len(free) // 3], free[2 * len(free) // 3], w.T]
    elif shape == "global-d512-kv":
        w = W.PrefillWorkload("chunk-g512", W.global_(8, 2, 512), 1, 700)
        cuts = [0, 129, 300, 700]
    elif shape == "global-d128":
        w = W.PrefillWorkload("chunk-g128", W.global_(8, 4, 128), 2, 520)
        cuts = [0, 1, 257, 520]
    elif shape == "sliding-d64-gqa":
        w = W.PrefillWorkload("chunk-s64", W.sliding(8, 2, 64, 96), 1, 400)
        cuts = [0, 150, 151, 400]
    else:  # the CUDA-core fp32 path
        w = W.PrefillWorkload("chunk-f32", W.sliding(2, 1, 64, 16), 1, 64, torch.float32)
        cuts = [0, 20, 64]
    run_chunks(w, cuts, seed=3, inp=inp)


def test_chunk_writes_the_cache_like_a_whole_prompt():
    w = W.PrefillWorkload("chunk-cache", W.sliding(8, 2, 256, 512), 1, 900)
    cache, kh, vh = run_chunks(w, [0, 333, 900], seed=5)
    for got, ref in ((cache.k, kh), (cache.v, vh)):
        g = got[:, :, :900].permute(0, 2, 1, 3).double().cpu().numpy()
        assert np.max(np.abs(g - ref) / (np.abs(ref) + 1e-3)) < 2 ** -8 + 1e-6
