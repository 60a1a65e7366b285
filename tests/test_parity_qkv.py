"""GPU parity of g4attn_qkv_prologue -- the QKV projection on tcgen05 tensor
cores with the prologue in its epilogue -- against the float64 oracle
(``oracle.qkv_prologue``: a float64 matmul of the exact inputs, then the
prologue).

The kernel keeps the raw projection in fp32 (TMEM) and rounds only its bf16
outputs, so an output element may differ from the exact value by half a bf16
ulp of that value plus the fp32 arithmetic before it (accumulation over the
hidden size, the RMS, the hardware sincos on a reduced angle): the bar is
|got - ref| - ulp(ref)/2 <= 2e-3 on values of magnitude <= ~5."""
import numpy as np
import pytest
import torch

import oracle
from attention_prologue_b200 import g4attn as G
from attention_prologue_b200 import workloads as W

from helpers import STATS, check, desc_of, oracle_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"
BAR = 2e-3


def check_vectors(got: torch.Tensor, ref: np.ndarray, what: str):
    g = got.detach().double().cpu().numpy()
    assert g.shape == ref.shape and np.all(np.isfinite(g)), what
    err = np.abs(g - ref)
    a = np.abs(ref)
    half_ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 8), 0.0)
    stats = dict(max_abs=float(err.max()), mean_abs=float(err.mean()),
                 rel=float(err.max() / max(a.max(), 1e-300)),
                 max_beyond_rounding=float((err - half_ulp).max()))
    STATS.append((what, stats))
    assert stats["max_beyond_rounding"] <= BAR, f"{what}: {stats}"


CASES = {
    # name: (layer, B, T, hidden, p0, cache kind)
    "e2b_like": (W.sliding(8, 1, 256, 512), 2, 300, 1536, 0, "two"),
    "global_k_eq_v_d512_ragged_hidden": (W.global_(8, 1, 512), 1, 260, 328, 100, "two"),
    "d128_rolling": (W.sliding(4, 2, 128, 64), 2, 300, 200, 0, "rolling"),
    "d64_bidirectional_queries_only": (W.bidirectional(4, 4, 64), 3, 130, 96, 0, None),
    "d512_single_tensor": (W.global_(8, 2, 512), 2, 140, 256, 7, "single"),
    "d256_global_separate_v": (W.global_(8, 2, 256, k_eq_v=False), 1, 390, 512, 0, "two"),
    # at most 128 tokens: the single-CTA kernel (M 128 MMAs) instead of CTA pairs
    "single_cta_d128_p0": (W.sliding(4, 2, 128, 64), 2, 50, 256, 10, "two"),
    "single_cta_d512_k_eq_v_128_tokens": (W.global_(8, 1, 512), 1, 128, 192, 0, "two"),
    "single_cta_d64_rolling": (W.sliding(2, 2, 64, 32), 1, 77, 64, 40, "rolling"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_qkv_prologue_matches_the_oracle(name):
    L, B, T, hidden, p0, kind = CASES[name]
    Hkv, d = L.num_kv_heads, L.head_dim
    inp = W.projection_inputs(L, B, T, hidden, DEV, 61, with_kv=kind is not None)
    desc = desc_of(L, torch.bfloat16)
    cache = None
    if kind == "two":
        cache = G.KVCache.allocate(B, Hkv, p0 + T + 3, d, device=DEV)
    elif kind == "rolling":
        cache = G.KVCache.allocate(B, Hkv, L.window, d, rolling=True, device=DEV)
    elif kind == "single":
        cache = G.KVCache.allocate(B, Hkv, p0 + T, d, device=DEV, single=True,
                                   k_norm_w=inp["k_norm_w"])
    if cache is not None:
        cache.k.fill_(7.0)  # slots the call must not touch keep this value
        if cache.v is not None:
            cache.v.fill_(7.0)
    q_hat = G.g4attn_qkv_prologue(desc, p0, inp["x"], inp["w_qkv"], inp["q_norm_w"],
                                  inp["k_norm_w"], cache)
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    qh, kh, vh = oracle.qkv_prologue(oracle_layer(L), inp["x"], inp["w_qkv"], inp["q_norm_w"],
                                     inp["k_norm_w"], p0, with_kv=kind is not None)
    check_vectors(q_hat, qh, f"qkv {name}: q_hat")
    if cache is None:
        return
    assert cache.len.tolist() == [p0 + T] * B
    if kind == "rolling":
        C = cache.capacity
        keep = np.arange(p0 + T - C, p0 + T)  # the last C positions, slot pos % C
        slots = keep % C
        check_vectors(cache.k[:, :, slots], kh[:, keep - p0].transpose(0, 2, 1, 3),
                      f"qkv {name}: K")
        check_vectors(cache.v[:, :, slots], vh[:, keep - p0].transpose(0, 2, 1, 3),
                      f"qkv {name}: V")
        return
    sl = slice(p0, p0 + T)
    if kind == "single":  # V alone, in k
        check_vectors(cache.k[:, :, sl], vh.transpose(0, 2, 1, 3), f"qkv {name}: V (single)")
        assert (cache.k[:, :, :p0] == 7.0).all()
        return
    check_vectors(cache.k[:, :, sl], kh.transpose(0, 2, 1, 3), f"qkv {name}: K")
    check_vectors(cache.v[:, :, sl], vh.transpose(0, 2, 1, 3), f"qkv {name}: V")
    assert (cache.k[:, :, :p0] == 7.0).all() and (cache.k[:, :, p0 + T:] == 7.0).all()


@pytest.mark.parametrize("shape", ["e2b", "31b"])
def test_qkv_prologue_at_the_variants_hidden_sizes(shape):
    """The E2B-shaped sliding layer at its full prompt (8192 tokens x hidden
    1536 -> 10 heads of 256) and the 31B-shaped K=V global layer (hidden
    5376 -> 36 heads of 512) on 384 tokens: every output against the oracle."""
    if shape == "e2b":
        L, B, T, hidden = W.E2B_SLIDING.layer, 1, 8192, W.HIDDEN["e2b-sliding-prefill"]
    else:
        L, B, T, hidden = W.G31B_GLOBAL.layer, 1, 384, W.HIDDEN["31b-global-prefill"]
    inp = W.projection_inputs(L, B, T, hidden, DEV, 62)
    cache = G.KVCache.allocate(B, L.num_kv_heads, T, L.head_dim, device=DEV)
    q_hat = G.g4attn_qkv_prologue(desc_of(L, torch.bfloat16), 0, inp["x"], inp["w_qkv"],
                                  inp["q_norm_w"], inp["k_norm_w"], cache)
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    qh, kh, vh = oracle.qkv_prologue(oracle_layer(L), inp["x"], inp["w_qkv"], inp["q_norm_w"],
                                     inp["k_norm_w"])
    check_vectors(q_hat, qh, f"qkv {shape}: q_hat")
    check_vectors(cache.k, kh.transpose(0, 2, 1, 3), f"qkv {shape}: K")
    check_vectors(cache.v, vh.transpose(0, 2, 1, 3), f"qkv {shape}: V")


def test_projection_then_attention_is_the_layer():
    """x -> g4attn_qkv_prologue -> g4attn_attend over two chunks (image
    blocks, the chunks cut between them) equals the oracle's projection,
    prologue and attention of the whole prompt."""
    L = W.sliding(8, 2, 256, 96)
    B, T, hidden, p0 = 2, 500, 640, 180
    inp = W.projection_inputs(L, B, T, hidden, DEV, 63)
    ids = torch.full((B, T), -1, dtype=torch.int32)
    ids[:, 200:330] = 0
    ids[1, 400:460] = 1
    ids = ids.to(DEV)
    desc = desc_of(L, torch.bfloat16)
    cache = G.KVCache.allocate(B, L.num_kv_heads, T, L.head_dim, device=DEV)
    outs = []
    for a, b in ((0, p0), (p0, T)):
        q_hat = G.g4attn_qkv_prologue(desc, a, inp["x"][:, a:b].contiguous(), inp["w_qkv"],
                                      inp["q_norm_w"], inp["k_norm_w"], cache)
        outs.append(G.g4attn_attend(desc, a, q_hat, cache,
                                    image_block_ids=ids[:, :b].contiguous()))
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    OL = oracle_layer(L)
    qh, kh, vh = oracle.qkv_prologue(OL, inp["x"], inp["w_qkv"], inp["q_norm_w"],
                                     inp["k_norm_w"])
    ref = oracle.attend_rows(OL, qh, kh, vh, 0, ids.cpu().numpy())
    out = torch.cat(outs, dim=1)
    check(out, ref, torch.bfloat16, "projection + attention over two chunks")
