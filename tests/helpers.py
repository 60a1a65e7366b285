"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the float64 oracle on the same seeded inputs, and compare them within the
stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from attention_prologue_b200 import g4attn as G
from attention_prologue_b200 import workloads as W

# Tolerances of the parity bar: bf16 outputs against the float64 oracle
# (max abs <= 2e-2 and mean abs <= 2e-3 per output tensor); the fp32 tiny
# configuration: max |gpu - oracle| / max |oracle| <= 1e-5 (norm-wise reading
# of a relative bound, since element-wise relative error blows up near 0).
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
FP32_REL = 1e-5

# every comparison's errors, printed at the end of the run (conftest.py)
STATS: list[tuple[str, dict]] = []


def desc_of(L: W.LayerShape, dtype: torch.dtype) -> G.LayerDesc:
    return G.make_desc(L.layer_type, L.num_heads, L.num_kv_heads, L.head_dim, window=L.window,
                       rotary_fraction=L.rotary_fraction, rope_theta=L.rope_theta,
                       k_eq_v=L.k_eq_v, softmax_scale=L.scale, rms_eps=L.rms_eps, dtype=dtype)


def oracle_layer(L: W.LayerShape) -> oracle.Layer:
    return oracle.Layer(layer_type=L.layer_type, window=L.window,
                        rotary_fraction=L.rotary_fraction, rope_theta=L.rope_theta,
                        k_eq_v=L.k_eq_v, num_heads=L.num_heads, num_kv_heads=L.num_kv_heads,
                        head_dim=L.head_dim, softmax_scale=L.scale, rms_eps=L.rms_eps)


def check(got: torch.Tensor, ref: np.ndarray, dtype: torch.dtype, what: str = "") -> dict:
    g = got.detach().double().cpu().numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    stats = dict(max_abs=float(err.max()), mean_abs=float(err.mean()),
                 rel=float(err.max() / max(np.abs(ref).max(), 1e-300)))
    STATS.append((what, stats))
    if dtype == torch.float32:
        assert stats["rel"] <= FP32_REL, f"{what}: {stats}"
    else:
        assert stats["max_abs"] <= BF16_MAX_ABS and stats["mean_abs"] <= BF16_MEAN_ABS, \
            f"{what}: {stats}"
    return stats


def sample_rows(T: int, n: int, tile: int = 128) -> list[int]:
    """First/last rows, rows at tile boundaries and evenly spaced rows."""
    rows = {0, 1, T // 2, T - 2, T - 1}
    for t in (tile, 2 * tile, T - tile):
        for r in (t - 1, t, t + 1):
            if 0 <= r < T:
                rows.add(r)
    rows.update(np.linspace(0, T - 1, max(n - len(rows), 2)).astype(int).tolist())
    return sorted(r for r in rows if 0 <= r < T)


def gpu_prefill(w: W.PrefillWorkload, inp: dict, cache: G.KVCache | None = None):
    d = desc_of(w.layer, w.dtype)
    out = G.g4attn_prefill(d, inp["q_raw"], inp["k_raw"], inp["v_raw"], inp["q_norm_w"],
                           inp["k_norm_w"], inp["image_block_ids"], cache=cache)
    torch.cuda.synchronize()
    assert G.g4attn_get_device_status() == G.G4ATTN_OK
    return out


def oracle_prefill(w: W.PrefillWorkload, inp: dict, rows=None) -> np.ndarray:
    cpu = {k: (v.cpu() if v is not None else None) for k, v in inp.items()}
    ids = cpu["image_block_ids"]
    return oracle.prefill(oracle_layer(w.layer), cpu["q_raw"], cpu["k_raw"], cpu["v_raw"],
                          cpu["q_norm_w"], cpu["k_norm_w"],
                          block_ids=None if ids is None else ids.numpy(), rows=rows)
