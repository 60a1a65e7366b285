"""Host-side checks of the C ABI: the library loads, exports every function
include/g4attn.h declares, and rejects bad arguments before touching the GPU.
No test here launches a kernel (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

from attention_prologue_b200 import g4attn as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first


def header_functions():
    src = open(os.path.join(ROOT, "include", "g4attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(g4attn_\w+)\s*\(", src)))


def test_library_exports_every_declared_function():
    lib = G.lib()
    declared = header_functions()
    assert set(declared) == set(G.EXPORTED)
    for name in declared:
        assert hasattr(lib, name), name


def test_binding_fails_loudly_without_the_library(monkeypatch):
    monkeypatch.setattr(G, "_lib", None)
    monkeypatch.setattr(G, "_LIB_PATH", "/nonexistent/libg4attn.so")
    with pytest.raises(RuntimeError):
        G.lib()


def desc(**kw):
    base = dict(layer_type=G.G4ATTN_SLIDING, num_heads=8, num_kv_heads=2, head_dim=256,
                window=512)
    base.update(kw)
    return G.make_desc(base.pop("layer_type"), base.pop("num_heads"), base.pop("num_kv_heads"),
                       base.pop("head_dim"), **base)


def prefill_rc(d, B=1, T=16, k=FAKE, v=FAKE, ids=None, cache=None, ws=FAKE, ws_bytes=1 << 40):
    return G.lib().g4attn_prefill(ctypes.byref(d), B, T, FAKE, k, v, FAKE, FAKE, ids, None,
                                  ctypes.byref(cache) if cache is not None else None, FAKE, ws,
                                  ws_bytes, None)


def ccache(d, B=1, C=64, rolling=0, **kw):
    c = G._CCache(FAKE, FAKE, FAKE, C, rolling, B, d.num_kv_heads, d.head_dim, d.dtype)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("bad", [
    dict(head_dim=0, softmax_scale=1.0), dict(head_dim=-64, softmax_scale=1.0),
    dict(head_dim=63), dict(num_heads=6, num_kv_heads=4),
    dict(num_kv_heads=0), dict(window=0),
    dict(rotary_fraction=0.3), dict(rotary_fraction=1.5), dict(rope_theta=-1.0),
    dict(rms_eps=-1.0), dict(softmax_scale=float("inf")), dict(softmax_scale=0.0),
    dict(softmax_scale=-0.5), dict(layer_type=3), dict(layer_type=-1), dict(logit_softcap=-1.0),
    dict(logit_softcap=float("inf")), dict(logit_softcap=float("nan")),
])
def test_bad_descriptors_are_rejected(bad):
    d = desc(**bad)
    assert prefill_rc(d) == G.G4ATTN_EINVAL
    assert G.lib().g4attn_prefill_workspace_size(ctypes.byref(d), 1, 16) == 0


@pytest.mark.parametrize("shape", [dict(head_dim=96), dict(head_dim=1024),
                                   dict(num_heads=64, num_kv_heads=64)])
def test_valid_layers_without_a_kernel_are_unsupported(shape):
    """Head sizes other than 64/128/256/512 and more than 32 KV heads are
    layers the pages allow but the library has no kernel for."""
    d = desc(**shape)
    assert prefill_rc(d) == G.G4ATTN_EUNSUPPORTED
    assert G.lib().g4attn_prefill_workspace_size(ctypes.byref(d), 1, 16) == 0
    c = ccache(d)
    assert G.lib().g4attn_decode_workspace_size(ctypes.byref(d), ctypes.byref(c)) == 0


def test_bad_dtype_code_is_rejected():
    d = desc()
    d.dtype = 7
    assert prefill_rc(d) == G.G4ATTN_EINVAL


def test_k_eq_v_and_value_pointer_must_agree():
    assert prefill_rc(desc(k_eq_v=True)) == G.G4ATTN_EINVAL  # v_raw given with K=V
    assert prefill_rc(desc(k_eq_v=False), v=None) == G.G4ATTN_EINVAL  # v_raw missing
    d = desc(layer_type=G.G4ATTN_GLOBAL, head_dim=512, rotary_fraction=0.25, k_eq_v=True)
    assert prefill_rc(d, v=None, ws=None, ws_bytes=0) == G.G4ATTN_EWORKSPACE


def test_kv_shared_prefill_needs_a_cache_holding_the_prompt():
    d = desc()
    assert prefill_rc(d, k=None, v=None) == G.G4ATTN_EINVAL  # no cache to read
    assert prefill_rc(d, k=None, v=None, cache=ccache(d, C=8, rolling=0), T=16) == \
        G.G4ATTN_ECACHE_OVERFLOW
    dr = desc(window=8)
    assert prefill_rc(dr, k=None, v=None, cache=ccache(dr, C=8, rolling=1), T=16) == \
        G.G4ATTN_EINVAL


def test_cache_checks():
    d = desc()
    assert prefill_rc(d, cache=ccache(d, C=8)) == G.G4ATTN_ECACHE_OVERFLOW  # T=16 > C
    assert prefill_rc(d, cache=ccache(d, B=2)) == G.G4ATTN_EINVAL  # batch mismatch
    assert prefill_rc(d, cache=ccache(d, head_dim=128)) == G.G4ATTN_EINVAL
    assert prefill_rc(d, cache=ccache(d, num_kv_heads=1)) == G.G4ATTN_EINVAL
    assert prefill_rc(d, cache=ccache(d, dtype=G.G4ATTN_FP32)) == G.G4ATTN_EINVAL
    assert prefill_rc(d, cache=ccache(d, C=256, rolling=1)) == G.G4ATTN_EINVAL  # C < window
    g = desc(layer_type=G.G4ATTN_GLOBAL, head_dim=512, rotary_fraction=0.25, k_eq_v=True)
    assert prefill_rc(g, v=None, cache=ccache(g, C=1024, rolling=1)) == G.G4ATTN_EINVAL
    c = ccache(d)
    c.k = None
    assert prefill_rc(d, cache=c) == G.G4ATTN_EINVAL


def test_append_and_decode_validation():
    lib = G.lib()
    d = desc()
    c = ccache(d, C=512)
    assert lib.g4attn_cache_append(ctypes.byref(d), None, FAKE, FAKE, FAKE, None) == G.G4ATTN_EINVAL
    assert lib.g4attn_cache_append(ctypes.byref(d), ctypes.byref(c), FAKE, None, FAKE, None) == \
        G.G4ATTN_EINVAL
    assert lib.g4attn_decode(ctypes.byref(d), ctypes.byref(c), FAKE, FAKE, FAKE, None, 0, None) == \
        G.G4ATTN_EWORKSPACE
    assert lib.g4attn_decode(ctypes.byref(d), ctypes.byref(c), None, FAKE, FAKE, FAKE, 1 << 30,
                             None) == G.G4ATTN_EINVAL
    # misaligned workspace
    assert lib.g4attn_decode(ctypes.byref(d), ctypes.byref(c), FAKE, FAKE, FAKE,
                             ctypes.c_void_p(0x10010), 1 << 30, None) == G.G4ATTN_EWORKSPACE


def test_empty_inputs_are_a_no_op():
    d = desc()
    assert prefill_rc(d, B=0) == G.G4ATTN_OK
    assert prefill_rc(d, T=0) == G.G4ATTN_OK
    assert prefill_rc(d, B=-1) == G.G4ATTN_EINVAL


def test_workspace_sizes():
    d = desc(num_heads=8, num_kv_heads=1, head_dim=256, window=512)
    B, T = 1, 8192
    ws = G.lib().g4attn_prefill_workspace_size(ctypes.byref(d), B, T)
    # q_hat + K/V scratch + two int32 interval arrays + the padding bits (one
    # 64-bit word per 64 keys) + each sequence's first and last kept position
    # (two int32), 256-aligned pieces
    bits = -(-(B * (T // 64) * 8) // 256) * 256
    span = -(-(B * 8) // 256) * 256
    assert ws == B * T * 8 * 256 * 2 + 2 * B * T * 1 * 256 * 2 + 2 * B * T * 4 + bits + span
    c = ccache(d, B=64, C=1024, rolling=1)
    dws = G.lib().g4attn_decode_workspace_size(ctypes.byref(d), ctypes.byref(c))
    assert dws > 0 and dws % 256 == 0


def test_status_strings():
    for code in range(8):
        assert G.g4attn_status_string(code) != "unknown status"
    assert G.g4attn_status_string(99) == "unknown status"


def test_cache_layout_reproduces_the_printed_kv_table():
    """The cache stores K and V separately (also on K=V global layers), bf16,
    [batch, kv_heads, capacity, head_dim]: the only layout that reproduces the
    KV-cache table of the "gemma4-pt-claude" README."""
    rows = [l.split() for l in open(os.path.join(ROOT, "tests", "golden", "kv_cache_table.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 2
    for (model, layers, skv, hd, gkv, ghd, pattern, window, ctx, full, windowed) in rows:
        layers, skv, hd, gkv, ghd, pattern, window, ctx = map(
            int, (layers, skv, hd, gkv, ghd, pattern, window, ctx))
        n_global = layers // pattern
        n_sliding = layers - n_global
        glob = n_global * G.cache_bytes(1, gkv, ctx, ghd, torch.bfloat16)
        full_b = n_sliding * G.cache_bytes(1, skv, ctx, hd, torch.bfloat16) + glob
        win_b = n_sliding * G.cache_bytes(1, skv, window, hd, torch.bfloat16) + glob
        assert round(full_b / 1e9, 1) == float(full), model
        assert round(win_b / 1e9, 1) == float(windowed), model


def chunk_rc(d, B=1, T=16, p0=32, k=FAKE, v=FAKE, cache=None, ws=FAKE, ws_bytes=1 << 40):
    return G.lib().g4attn_prefill_chunk(ctypes.byref(d), B, T, p0, FAKE, k, v, FAKE, FAKE, None,
                                        None,
                                        ctypes.byref(cache) if cache is not None else None, FAKE,
                                        ws, ws_bytes, None)


def test_chunked_prefill_validation():
    lib = G.lib()
    d = desc()
    assert chunk_rc(d) == G.G4ATTN_EINVAL  # a cached prefill needs its cache
    assert chunk_rc(d, p0=-1, cache=ccache(d, C=64)) == G.G4ATTN_EINVAL
    assert chunk_rc(d, p0=56, T=16, cache=ccache(d, C=64)) == G.G4ATTN_ECACHE_OVERFLOW
    dr = desc(window=8)
    assert chunk_rc(dr, p0=56, T=16, cache=ccache(dr, C=64, rolling=1)) == G.G4ATTN_EINVAL
    assert chunk_rc(d, k=None, v=None, p0=56, T=16, cache=ccache(d, C=64)) == G.G4ATTN_EINVAL
    assert chunk_rc(desc(k_eq_v=True), cache=ccache(d, C=64)) == G.G4ATTN_EINVAL
    assert chunk_rc(d, cache=ccache(d, C=64), ws=None, ws_bytes=0) == G.G4ATTN_EWORKSPACE
    assert chunk_rc(d, T=0, cache=ccache(d, C=64)) == G.G4ATTN_OK
    assert lib.g4attn_prefill_chunk_workspace_size(ctypes.byref(d), 1, 16, -1) == 0
    assert lib.g4attn_prefill_chunk_workspace_size(ctypes.byref(d), 2, 16, 48) >= \
        2 * 16 * 8 * 256 * 2 + 2 * 2 * 16 * 4


def test_cache_key_mask_length_is_checked():
    """A cache's padding mask needs a length >= 0 (decode reads it)."""
    d = desc()
    c = ccache(d, C=64)
    c.key_mask = FAKE
    c.mask_len = -1
    assert G.lib().g4attn_decode_workspace_size(ctypes.byref(d), ctypes.byref(c)) == 0
    assert G.lib().g4attn_decode(ctypes.byref(d), ctypes.byref(c), FAKE, FAKE, FAKE, FAKE,
                                 1 << 40, None) == G.G4ATTN_EINVAL
    c.mask_len = 0  # an empty mask: every position is kept
    assert G.lib().g4attn_decode_workspace_size(ctypes.byref(d), ctypes.byref(c)) > 0


def test_prefill_workspace_covers_the_padding_bits():
    """The workspace size covers the padding bits of the largest call (one
    64-bit word per 64 key positions and sequence)."""
    lib = G.lib()
    d = desc(layer_type=G.G4ATTN_GLOBAL)
    base = lib.g4attn_prefill_workspace_size(ctypes.byref(d), 2, 1000)
    q_hat = 2 * 1000 * 8 * 256 * 2
    kv = 2 * 2 * 1000 * 2 * 256 * 2
    assert base >= q_hat + kv + 2 * 16 * 8
    assert lib.g4attn_prefill_chunk_workspace_size(ctypes.byref(d), 2, 100, 900) >= \
        2 * 100 * 8 * 256 * 2 + 2 * 16 * 8


def test_single_tensor_cache_validation():
    """A single-tensor cache (v = NULL) is for K=V layers, non-rolling, with
    the owning layer's key-norm weight; readers without a kernel for it
    (prefill reading K from it, a chunk, fp32 decode, more than 8 query
    heads per KV head) say so with G4ATTN_EUNSUPPORTED."""
    lib = G.lib()
    g = desc(layer_type=G.G4ATTN_GLOBAL, head_dim=512, rotary_fraction=0.25, k_eq_v=True,
             num_heads=8, num_kv_heads=2)
    def single(d, **kw):
        c = ccache(d, C=64, **kw)
        c.v = None
        c.k_norm_w = FAKE
        return c
    c = single(g)
    assert lib.g4attn_decode_workspace_size(ctypes.byref(g), ctypes.byref(c)) > 0
    c.k_norm_w = None  # no weight to rebuild K with
    assert lib.g4attn_decode_workspace_size(ctypes.byref(g), ctypes.byref(c)) == 0
    s = desc(num_heads=8, num_kv_heads=2)  # not a K=V layer
    assert lib.g4attn_decode(ctypes.byref(s), ctypes.byref(single(s)), FAKE, FAKE, FAKE, FAKE,
                             1 << 40, None) == G.G4ATTN_EINVAL
    # readers without a kernel
    assert prefill_rc(g, k=None, v=None, cache=single(g)) == G.G4ATTN_EUNSUPPORTED
    assert chunk_rc(g, v=None, cache=single(g)) == G.G4ATTN_EUNSUPPORTED
    f32 = desc(layer_type=G.G4ATTN_GLOBAL, head_dim=512, rotary_fraction=0.25, k_eq_v=True,
               num_heads=8, num_kv_heads=2, dtype=torch.float32)
    assert lib.g4attn_decode(ctypes.byref(f32), ctypes.byref(single(f32)), FAKE, FAKE, FAKE,
                             FAKE, 1 << 40, None) == G.G4ATTN_EUNSUPPORTED
    wide = desc(layer_type=G.G4ATTN_GLOBAL, head_dim=512, rotary_fraction=0.25, k_eq_v=True,
                num_heads=32, num_kv_heads=2)
    assert lib.g4attn_decode_noalloc(ctypes.byref(wide), ctypes.byref(single(wide)), FAKE, FAKE,
                                     FAKE, None) == G.G4ATTN_EUNSUPPORTED


def attend_rc(d, B=1, T=16, p0=32, q=FAKE, cache=None, out=FAKE, ws=FAKE, ws_bytes=1 << 40):
    return G.lib().g4attn_attend(ctypes.byref(d), B, T, p0, q, None, None,
                                 ctypes.byref(cache) if cache is not None else None, out, ws,
                                 ws_bytes, None)


def test_attend_validation():
    """Attention from post-prologue queries reads a two-tensor cache that
    holds every position up to the call's last at slot = position."""
    lib = G.lib()
    d = desc()
    assert attend_rc(d) == G.G4ATTN_EINVAL  # no cache
    assert attend_rc(d, q=None, cache=ccache(d, C=64)) == G.G4ATTN_EINVAL
    assert attend_rc(d, out=None, cache=ccache(d, C=64)) == G.G4ATTN_EINVAL
    assert attend_rc(d, p0=56, T=16, cache=ccache(d, C=64)) == G.G4ATTN_EINVAL
    assert attend_rc(d, p0=-1, cache=ccache(d, C=64)) == G.G4ATTN_EINVAL
    assert attend_rc(d, B=2, cache=ccache(d, C=64)) == G.G4ATTN_EINVAL  # batch mismatch
    c = ccache(d, C=64)
    c.v = None  # a single-tensor cache holds no K to read
    assert attend_rc(d, cache=c) == G.G4ATTN_EINVAL  # ... and this layer is not K=V
    g = desc(layer_type=G.G4ATTN_GLOBAL, head_dim=512, rotary_fraction=0.25, k_eq_v=True,
             num_heads=8, num_kv_heads=2)
    c = ccache(g, C=64)
    c.v = None
    c.k_norm_w = FAKE
    assert attend_rc(g, cache=c) == G.G4ATTN_EUNSUPPORTED
    assert attend_rc(d, cache=ccache(d, C=64), ws=None, ws_bytes=0) == G.G4ATTN_EWORKSPACE
    assert attend_rc(d, T=0, cache=ccache(d, C=64)) == G.G4ATTN_OK
    assert lib.g4attn_attend_workspace_size(ctypes.byref(d), 1, 16, -1) == 0
    # no q_hat area: the row intervals and the padding bits only
    n = lib.g4attn_attend_workspace_size(ctypes.byref(d), 2, 100, 900)
    assert 2 * 2 * 100 * 4 + 2 * 16 * 8 <= n < 2 * 100 * 8 * 256 * 2


def test_bidirectional_layer_has_prefill_but_no_decode():
    """The vision-tower layer type: prefill and attend take it (the window is
    ignored), append and decode have no step for it."""
    lib = G.lib()
    d = desc(layer_type=G.G4ATTN_BIDIRECTIONAL, window=0, softmax_scale=1.0)
    assert prefill_rc(d, ws=None, ws_bytes=0) == G.G4ATTN_EWORKSPACE  # passes validation
    assert lib.g4attn_prefill_workspace_size(ctypes.byref(d), 1, 16) > 0
    assert attend_rc(d, cache=ccache(d, C=64), ws=None, ws_bytes=0) == G.G4ATTN_EWORKSPACE
    c = ccache(d, C=64)
    assert lib.g4attn_cache_append(ctypes.byref(d), ctypes.byref(c), FAKE, FAKE, FAKE,
                                   None) == G.G4ATTN_EUNSUPPORTED
    assert lib.g4attn_decode(ctypes.byref(d), ctypes.byref(c), FAKE, FAKE, FAKE, FAKE, 1 << 40,
                             None) == G.G4ATTN_EUNSUPPORTED
    assert lib.g4attn_decode_noalloc(ctypes.byref(d), ctypes.byref(c), FAKE, FAKE, FAKE,
                                     None) == G.G4ATTN_EUNSUPPORTED
    assert prefill_rc(d, cache=ccache(d, C=64, rolling=1)) == G.G4ATTN_EINVAL  # rolling: sliding only


def qkv_rc(d, B=1, T=16, p0=0, x=FAKE, hidden=64, w=FAKE, wk=FAKE, q=FAKE, cache=None):
    return G.lib().g4attn_qkv_prologue(ctypes.byref(d), B, T, p0, x, hidden, w, FAKE, wk, q,
                                       ctypes.byref(cache) if cache is not None else None, None)


def test_qkv_prologue_validation():
    """The fused projection checks its shapes and pointers before any launch:
    a hidden size whose rows are not 16-byte multiples, misaligned operands,
    a non-rolling cache too small for p0 + T, fp32 (no tensor-core kernel)."""
    d = desc()
    assert qkv_rc(d, x=None) == G.G4ATTN_EINVAL
    assert qkv_rc(d, w=None) == G.G4ATTN_EINVAL
    assert qkv_rc(d, q=None) == G.G4ATTN_EINVAL
    assert qkv_rc(d, hidden=4) == G.G4ATTN_EINVAL
    assert qkv_rc(d, hidden=100) == G.G4ATTN_EINVAL  # 200-byte rows
    assert qkv_rc(d, x=ctypes.c_void_p(0x10008)) == G.G4ATTN_EINVAL  # not 16-byte aligned
    assert qkv_rc(d, B=-1) == G.G4ATTN_EINVAL
    assert qkv_rc(d, p0=-3) == G.G4ATTN_EINVAL
    assert qkv_rc(desc(dtype=torch.float32)) == G.G4ATTN_EUNSUPPORTED
    assert qkv_rc(d, wk=None, cache=ccache(d, C=64)) == G.G4ATTN_EINVAL  # K needs w_k
    assert qkv_rc(d, p0=60, T=16, cache=ccache(d, C=64)) == G.G4ATTN_ECACHE_OVERFLOW
    assert qkv_rc(d, B=2, cache=ccache(d, C=64)) == G.G4ATTN_EINVAL  # batch mismatch
    assert qkv_rc(d, T=0, cache=ccache(d, C=64)) == G.G4ATTN_OK
    assert qkv_rc(d, T=0) == G.G4ATTN_OK  # queries only (a KV-shared layer)
