"""Pins of the float64 oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: each test checks it against a
closed form, an invariant the method must satisfy, a value a page prints, or
an independent dense formulation (complex-number RoPE, an explicit mask
matrix, numpy softmax) on tiny inputs.  CPU only.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import BIDIRECTIONAL, GLOBAL, ROPE_PREFIX, SLIDING, Layer

RNG = np.random.default_rng(1234)


def f32(*shape, rng=RNG):
    return rng.standard_normal(shape).astype(np.float32)


def sliding_layer(**kw):
    base = dict(layer_type=SLIDING, window=6, rotary_fraction=1.0, rope_theta=1e4,
                num_heads=4, num_kv_heads=2, head_dim=16, softmax_scale=0.25, rms_eps=1e-6)
    base.update(kw)
    return Layer(**base)


def global_layer(**kw):
    base = dict(layer_type=GLOBAL, rotary_fraction=0.25, rope_theta=1e6, k_eq_v=True,
                num_heads=4, num_kv_heads=1, head_dim=32, softmax_scale=1 / math.sqrt(32),
                rms_eps=1e-6)
    base.update(kw)
    return Layer(**base)


def inputs(L, B, T, rng=RNG, v=True):
    q = f32(B, T, L.num_heads, L.head_dim, rng=rng)
    k = f32(B, T, L.num_kv_heads, L.head_dim, rng=rng)
    vv = f32(B, T, L.num_kv_heads, L.head_dim, rng=rng) if (v and not L.k_eq_v) else None
    wq = f32(L.head_dim, rng=rng)
    wk = f32(L.head_dim, rng=rng)
    return q, k, vv, wq, wk


def ids_with_blocks(B, T, runs):
    ids = np.full((B, T), -1, np.int32)
    for b in range(B):
        for n, (s, e) in enumerate(runs):
            ids[b, s:e] = n
    return ids


# ---------------------------------------------------------------------------
# independent dense formulation (brute force on tiny inputs)

def dense_reference(L, q, k, v, wq, wk, ids, keep=None):
    """Whole-matrix float64 formulation: RoPE as complex multiplication, the
    mask as an explicit boolean matrix built from the set definition (window
    OR same image run, AND a kept key when a padding mask is given), softmax
    with numpy; a row with no allowed key is 0."""
    q, k = q.astype(np.float64), k.astype(np.float64)
    v = k if L.k_eq_v else v.astype(np.float64)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    half = d // 2
    R = int(round(L.rotary_fraction * d / 2))

    def rms(x, w):
        y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + L.rms_eps)
        return y if w is None else y * w.astype(np.float64)

    freq = np.zeros(half)
    freq[:R] = L.rope_theta ** (-2.0 * np.arange(R) / d)
    rot = np.exp(1j * np.arange(T)[:, None] * freq[None, :])  # [T, half]

    def rope(x):  # [B, T, H, d]
        z = (x[..., :half] + 1j * x[..., half:]) * rot[None, :, None, :]
        return np.concatenate([z.real, z.imag], axis=-1)

    qh = rope(rms(q, wq))
    kh = rope(rms(k, wk))
    vh = rms(v, None)
    g = Hq // Hkv
    kh = np.repeat(kh, g, axis=2)
    vh = np.repeat(vh, g, axis=2)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    out = np.empty((B, T, Hq, d))
    for b in range(B):
        if L.layer_type == GLOBAL:
            allowed = j <= i
        elif L.layer_type == BIDIRECTIONAL:
            allowed = np.ones((T, T), bool)
        else:
            allowed = (j <= i) & (i - j < L.window)
            if ids is not None:
                run = np.full(T, -1)
                r = -1
                for t in range(T):
                    if ids[b, t] >= 0:
                        if t == 0 or ids[b, t - 1] != ids[b, t]:
                            r += 1
                        run[t] = r
                same = (run[:, None] == run[None, :]) & (run[:, None] >= 0)
                allowed = allowed | same
        if keep is not None:
            allowed = allowed & (keep[b][None, :] != 0)
        s = np.einsum("ihd,jhd->hij", qh[b], kh[b]) * L.softmax_scale
        if L.logit_softcap > 0:
            s = L.logit_softcap * np.tanh(s / L.logit_softcap)
        s = np.where(allowed[None], s, -np.inf)
        m = s.max(axis=-1, keepdims=True)
        p = np.exp(s - np.where(np.isfinite(m), m, 0.0))  # a row with no key: all 0
        den = p.sum(axis=-1, keepdims=True)
        p = p / np.where(den > 0, den, 1.0)
        out[b] = np.einsum("hij,jhd->ihd", p, vh[b])
    return out


@pytest.mark.parametrize("case", ["sliding_blocks", "sliding_gqa_bf16", "global_kv", "global_gqa"])
def test_brute_force_dense(case):
    rng = np.random.default_rng(7)
    ids = None
    if case == "sliding_blocks":
        L = sliding_layer(window=6)
        T = 40
        ids = ids_with_blocks(2, T, [(5, 12), (20, 31), (33, 35)])  # block 11 > window 6
        q, k, v, wq, wk = inputs(L, 2, T, rng)
    elif case == "sliding_gqa_bf16":
        L = sliding_layer(window=9, num_heads=6, num_kv_heads=2, head_dim=8)
        T = 30
        q, k, v, wq, wk = inputs(L, 1, T, rng)
        # round to bf16 and feed the raw bits: the oracle widens them exactly
        tq, tk, tv, twq, twk = (torch.from_numpy(x).bfloat16() for x in (q, k, v, wq, wk))
        got = oracle.prefill(L, tq, tk, tv, twq, twk)
        ref = dense_reference(L, *(x.float().numpy() for x in (tq, tk, tv, twq, twk)), None)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
        return
    elif case == "global_kv":
        L = global_layer()
        T = 33
        ids = ids_with_blocks(1, T, [(4, 20)])  # ignored on global layers
        q, k, v, wq, wk = inputs(L, 1, T, rng)
    else:
        L = global_layer(k_eq_v=False, num_heads=8, num_kv_heads=2, head_dim=64)
        T = 25
        q, k, v, wq, wk = inputs(L, 1, T, rng)
    got = oracle.prefill(L, q, k, v, wq, wk, block_ids=ids)
    ref = dense_reference(L, q, k, v, wq, wk, ids)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# closed forms

@pytest.mark.parametrize("mk", [sliding_layer, global_layer])
def test_single_token_returns_its_value(mk):
    L = mk()
    q, k, v, wq, wk = inputs(L, 1, 1)
    out = oracle.prefill(L, q, k, v, wq, wk)
    _, vh = oracle.prefill_kv(L, k, v, wk)
    g = L.num_heads // L.num_kv_heads
    for h in range(L.num_heads):
        np.testing.assert_allclose(out[0, 0, h], vh[0, 0, h // g], rtol=0, atol=1e-15)


@pytest.mark.parametrize("mk", [sliding_layer, global_layer])
def test_zero_query_gives_mean_of_interval(mk):
    L = mk()
    T = 30
    q, k, v, wq, wk = inputs(L, 1, T)
    q[:] = 0.0  # RMSNorm(0) = 0 -> all scores 0 -> uniform weights
    ids = ids_with_blocks(1, T, [(10, 19)]) if L.layer_type == SLIDING else None
    out = oracle.prefill(L, q, k, v, wq, wk, block_ids=ids)
    _, vh = oracle.prefill_kv(L, k, v, wk)
    g = L.num_heads // L.num_kv_heads
    for i in range(T):
        if L.layer_type == GLOBAL:
            lo, hi = 0, i
        elif ids is not None and ids[0, i] >= 0:
            lo, hi = min(max(0, i - L.window + 1), 10), max(i, 18)
        else:
            lo, hi = max(0, i - L.window + 1), i
        for h in range(L.num_heads):
            np.testing.assert_allclose(out[0, i, h], vh[0, lo:hi + 1, h // g].mean(0),
                                       rtol=0, atol=1e-14)


def test_two_keys_is_a_sigmoid():
    """Row 1 over keys {0, 1}: o = sig(s1 - s0) v1 + sig(s0 - s1) v0 with
    s_j = scale * q_hat . k_hat_j -- pins the scale and the softmax form."""
    L = global_layer(k_eq_v=False, num_heads=1, num_kv_heads=1, softmax_scale=0.37)
    q, k, v, wq, wk = inputs(L, 1, 2)
    out = oracle.prefill(L, q, k, v, wq, wk)
    qh = oracle.prologue_q(L, q[0, 1, 0], wq, 1)
    k0, v0 = oracle.prologue_kv(L, k[0, 0, 0], v[0, 0, 0], wk, 0)
    k1, v1 = oracle.prologue_kv(L, k[0, 1, 0], v[0, 1, 0], wk, 1)
    s0, s1 = 0.37 * qh @ k0, 0.37 * qh @ k1
    sig = 1.0 / (1.0 + math.exp(-(s1 - s0)))
    np.testing.assert_allclose(out[0, 1, 0], sig * v1 + (1 - sig) * v0, rtol=0, atol=1e-14)


def test_equal_values_give_that_value():
    L = sliding_layer()
    T = 20
    q, k, v, wq, wk = inputs(L, 1, T)
    v[:] = v[:, :1]  # every position carries the same raw value vector
    out = oracle.prefill(L, q, k, v, wq, wk)
    vh = oracle.rms_normalize(v[0, 0, 0], L.rms_eps)
    vh1 = oracle.rms_normalize(v[0, 0, 1], L.rms_eps)
    np.testing.assert_allclose(out[0, :, :2], np.broadcast_to(vh, (T, 2, L.head_dim)), atol=1e-14)
    np.testing.assert_allclose(out[0, :, 2:], np.broadcast_to(vh1, (T, 2, L.head_dim)), atol=1e-14)


def test_gqa_grouping_is_consecutive():
    """KV head of query head h is h // g: give each KV head constant values."""
    L = sliding_layer(num_heads=6, num_kv_heads=3)
    T = 12
    q, k, v, wq, wk = inputs(L, 1, T)
    for kvh in range(3):
        v[0, :, kvh] = v[0, 0, kvh]
    out = oracle.prefill(L, q, k, v, wq, wk)
    for h in range(6):
        np.testing.assert_allclose(out[0, 5, h], oracle.rms_normalize(v[0, 0, h // 2], L.rms_eps),
                                   atol=1e-14)


# ---------------------------------------------------------------------------
# mask invariants, observed through the whole pipeline

@pytest.mark.parametrize("case", ["sliding", "sliding_blocks", "global"])
def test_mask_by_perturbation(case):
    """Changing the raw key/value of position j changes row i iff j is in I_i;
    outside I_i row i is bit-identical."""
    rng = np.random.default_rng(3)
    T = 28
    if case == "global":
        L = global_layer(k_eq_v=False)
        ids, expect = None, lambda i: (0, i)
    else:
        L = sliding_layer(window=5)
        ids = ids_with_blocks(1, T, [(8, 17)]) if case == "sliding_blocks" else None

        def expect(i):
            lo, hi = max(0, i - 4), i
            if ids is not None and 8 <= i < 17:
                lo, hi = min(lo, 8), 16
            return lo, hi
    q, k, v, wq, wk = inputs(L, 1, T, rng)
    rows = [0, 3, 4, 9, 12, 16, 17, 20, 27]
    base = oracle.prefill(L, q, k, v, wq, wk, block_ids=ids, rows=rows)
    for j in range(T):
        k2, v2 = k.copy(), v.copy()
        k2[0, j] += 1.0
        v2[0, j] -= 0.5
        pert = oracle.prefill(L, q, k2, v2, wq, wk, block_ids=ids, rows=rows)
        for r, i in enumerate(rows):
            lo, hi = expect(i)
            inside = lo <= j <= hi
            same = np.array_equal(pert[0, r], base[0, r])
            assert same != inside, (case, i, j)


def test_window_counts_and_block_union():
    L = sliding_layer(window=7)
    T = 50
    for i in range(T):
        lo, hi = oracle.interval(L, None, T, i)
        assert (lo, hi) == (max(0, i - 6), i)
        assert hi - lo + 1 == min(i + 1, 7)
    ids = ids_with_blocks(1, T, [(10, 30)])[0]  # block of 20 > window 7
    for i in range(T):
        lo, hi = oracle.interval(L, ids, T, i)
        if 10 <= i < 30:
            assert (lo, hi) == (min(max(0, i - 6), 10), 29)
        else:
            assert (lo, hi) == (max(0, i - 6), i)
    G = global_layer()
    for i in range(T):
        assert oracle.interval(G, ids, T, i) == (0, i)


def test_text_rows_ignore_block_ids_and_global_ignores_them():
    T = 36
    ids = ids_with_blocks(1, T, [(6, 14), (20, 33)])
    L = sliding_layer(window=8)
    q, k, v, wq, wk = inputs(L, 1, T)
    a = oracle.prefill(L, q, k, v, wq, wk, block_ids=ids)
    b = oracle.prefill(L, q, k, v, wq, wk, block_ids=None)
    text = ids[0] < 0
    assert np.array_equal(a[0, text], b[0, text])
    assert not np.allclose(a[0, ~text], b[0, ~text])
    G = global_layer()
    q, k, v, wq, wk = inputs(G, 1, T)
    assert np.array_equal(oracle.prefill(G, q, k, v, wq, wk, block_ids=ids),
                          oracle.prefill(G, q, k, v, wq, wk))


def test_adjacent_runs_with_distinct_ids_are_distinct_blocks():
    L = sliding_layer(window=3)
    T = 20
    ids = np.full((1, T), -1, np.int32)
    ids[0, 4:9] = 0
    ids[0, 9:15] = 1  # touches block 0 but is another block
    assert oracle.interval(L, ids[0], T, 9) == (min(7, 9), 14)
    assert oracle.interval(L, ids[0], T, 8) == (4, 8)


# ---------------------------------------------------------------------------
# RoPE

def test_rope_matches_the_printed_rotation_matrix():
    """Overview blog, "Dual RoPE configurations": each two-dimensional
    subspace is multiplied by [[cos, -sin], [sin, cos]].  With d = 2 the only
    pair has frequency theta^0 = 1, so the angle is the position."""
    L = Layer(layer_type=SLIDING, window=4, head_dim=2, rotary_fraction=1.0, rope_theta=1e4)
    x = np.array([0.3, -1.7])
    for p in (1, 2, 5, 1000):
        c, s = math.cos(p), math.sin(p)
        np.testing.assert_allclose(oracle.rope(x, p, L), [c * x[0] - s * x[1], s * x[0] + c * x[1]],
                                   rtol=0, atol=1e-15)


@pytest.mark.parametrize("mk", [sliding_layer, lambda: global_layer(head_dim=512)])
def test_rope_frequency_ladder(mk):
    """Rotating the unit vector of dim k by position 1 turns pair k by
    theta^(-2k/d) for k < R (RoFormer's frequencies) and by 0 for k >= R."""
    L = mk()
    d = L.head_dim
    R = oracle.rotated_pairs(L)
    assert R == round(L.rotary_fraction * d / 2)
    for k in range(d // 2):
        e = np.zeros(d)
        e[k] = 1.0
        y = oracle.rope(e, 1, L)
        ang = math.atan2(y[k + d // 2], y[k])
        want = L.rope_theta ** (-2.0 * k / d) if k < R else 0.0
        assert abs(ang - want) < 1e-15, (k, ang, want)


def test_rope_preserves_pair_norms_and_is_identity_at_zero():
    for L in (sliding_layer(head_dim=256), global_layer(head_dim=512)):
        x = RNG.standard_normal(L.head_dim)
        h = L.head_dim // 2
        assert np.array_equal(oracle.rope(x, 0, L), x)
        for p in (1, 77, 4095, 131072):
            y = oracle.rope(x, p, L)
            np.testing.assert_allclose(np.hypot(y[:h], y[h:]), np.hypot(x[:h], x[h:]),
                                       rtol=1e-13, atol=0)


def test_rope_scores_depend_only_on_offset():
    for L in (sliding_layer(head_dim=64), global_layer(head_dim=512)):
        q = RNG.standard_normal(L.head_dim)
        k = RNG.standard_normal(L.head_dim)
        for m, n in ((5, 2), (300, 17), (40000, 39000)):
            a = oracle.rope(q, m, L) @ oracle.rope(k, n, L)
            b = oracle.rope(q, m + 1000, L) @ oracle.rope(k, n + 1000, L)
            assert abs(a - b) < 1e-9 * max(1.0, abs(a))


def test_partial_rope_passes_75_percent_through_bit_exact():
    L = global_layer(head_dim=512)
    x = RNG.standard_normal(512)
    y = oracle.rope(x, 12345, L)
    rot = np.zeros(512, bool)
    rot[0:64] = True
    rot[256:320] = True
    assert np.array_equal(y[~rot], x[~rot])
    assert np.all(y[rot] != x[rot])


def test_prefix_reading_differs_and_coincides_at_full_rotation():
    """The alternative reading of partial RoPE (rotate the first 25% as its own
    head) is a different function; at rotary_fraction 1 both readings agree."""
    x = RNG.standard_normal(64)
    Lz = global_layer(head_dim=64)
    Lp = global_layer(head_dim=64, rope_mode=ROPE_PREFIX)
    assert not np.allclose(oracle.rope(x, 9, Lz), oracle.rope(x, 9, Lp))
    Fz = sliding_layer(head_dim=64)
    Fp = sliding_layer(head_dim=64, rope_mode=ROPE_PREFIX)
    assert np.array_equal(oracle.rope(x, 9, Fz), oracle.rope(x, 9, Fp))


# ---------------------------------------------------------------------------
# norms and K=V

def test_vnorm_is_weightless_with_eps_inside_the_root():
    eps = 0.5  # large eps makes its placement visible
    x = RNG.standard_normal(64)
    y = oracle.rms_normalize(x, eps)
    ms = np.mean(x * x)
    assert abs(math.sqrt(np.mean(y * y)) - math.sqrt(ms / (ms + eps))) < 1e-14
    y2 = oracle.rms_normalize(3.0 * x, 1e-6)
    np.testing.assert_allclose(y2, oracle.rms_normalize(x, 1e-6), rtol=1e-6)


def test_norm_weight_is_used_directly():
    """Plain-weight RMSNorm (no 1 + w): a zero weight zeroes the query and
    doubling the weight doubles it (exactly, before and after RoPE)."""
    L = sliding_layer(head_dim=32)
    q = RNG.standard_normal(32).astype(np.float32)
    w = RNG.standard_normal(32).astype(np.float32)
    assert np.array_equal(oracle.prologue_q(L, q, np.zeros(32, np.float32), 17), np.zeros(32))
    assert np.array_equal(oracle.prologue_q(L, q, 2 * w, 17), 2 * oracle.prologue_q(L, q, w, 17))


def test_k_eq_v_tying():
    L = global_layer(head_dim=512)
    k = RNG.standard_normal(512).astype(np.float32)
    ones = np.ones(512, np.float32)
    kh, vh = oracle.prologue_kv(L, k, None, ones, 0)
    assert np.array_equal(kh, vh)  # w_k = 1 and position 0: K and V coincide
    w = RNG.standard_normal(512).astype(np.float32)
    _, vh2 = oracle.prologue_kv(L, k, None, w, 9999)
    assert np.array_equal(vh, vh2)  # V does not depend on w_k or position
    kh2, _ = oracle.prologue_kv(L, k, None, w, 9999)
    assert not np.allclose(kh2, vh2)


# ---------------------------------------------------------------------------
# decode, rolling cache, KV sharing, split-KV combine

def _cache_from(kh, C, rolling):
    """fp64 cache [B, Hkv, C, d] holding exact post-prologue rows."""
    B, T, Hkv, d = kh.shape
    cache = np.zeros((B, Hkv, C, d))
    for p in range(T):
        slot = p % C if rolling else p
        cache[:, :, slot] = kh[:, p]
    return cache


@pytest.mark.parametrize("case", ["sliding", "sliding_rolling", "global_kv"])
def test_decode_equals_last_prefill_row(case):
    rng = np.random.default_rng(11)
    L = global_layer() if case == "global_kv" else sliding_layer(window=8)
    T = 37  # past the window
    q, k, v, wq, wk = inputs(L, 2, T + 1, rng)
    ref = oracle.prefill(L, q, k, v, wq, wk)[:, T]
    kh, vh = oracle.prefill_kv(L, k[:, :T], None if v is None else v[:, :T], wk)
    rolling = case == "sliding_rolling"
    C = L.window if rolling else 64
    out = oracle.decode(L, q[:, T:T + 1], wq, _cache_from(kh, C, rolling),
                        _cache_from(vh, C, rolling), C, rolling, [T, T],
                        k_new=k[:, T:T + 1], v_new=None if v is None else v[:, T:T + 1], wk=wk)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mk", [sliding_layer, global_layer])
def test_kv_shared_decode(mk):
    """A KV-shared layer computes only its own query and reads the source
    layer's cache, which already holds the new token (Shared KV Cache)."""
    rng = np.random.default_rng(5)
    L1 = mk()
    L2 = mk(softmax_scale=0.5)
    T = 30
    q1, k, v, wq1, wk = inputs(L1, 1, T + 1, rng)
    q2, _, _, wq2, _ = inputs(L2, 1, T + 1, rng)
    ref = oracle.prefill(L2, q2, k, v, wq2, wk)[:, T]
    kh, vh = oracle.prefill_kv(L1, k, v, wk)  # source cache after its append
    C = 40
    out = oracle.decode(L2, q2[:, T:T + 1], wq2, _cache_from(kh, C, False),
                        _cache_from(vh, C, False), C, False, [T + 1])
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_decode_rejects_keys_missing_from_the_cache():
    L = sliding_layer(window=8)
    q, k, v, wq, wk = inputs(L, 1, 20)
    kh, vh = oracle.prefill_kv(L, k, v, wk)
    C = 4  # ring smaller than the window
    with pytest.raises(ValueError):
        oracle.decode(L, q[:, 19:], wq, _cache_from(kh, C, True), _cache_from(vh, C, True), C, True,
                      [20])


def test_split_kv_combine_equals_unsplit():
    rng = np.random.default_rng(9)
    L = global_layer(k_eq_v=False, num_heads=1, num_kv_heads=1, head_dim=32)
    T = 50
    q, k, v, wq, wk = inputs(L, 1, T, rng)
    row = oracle.prefill(L, q, k, v, wq, wk, rows=[T - 1])[0, 0, 0]
    kh, vh = oracle.prefill_kv(L, k, v, wk)
    qh = oracle.prologue_q(L, q[0, T - 1, 0], wq, T - 1)
    kk, vv = kh[0, :, 0], vh[0, :, 0]
    ms, ls, os_ = [], [], []
    for lo, hi in ((0, 4), (5, 16), (17, 40), (41, 49)):
        m, l, ot = oracle.partial(qh, kk, vv, lo, hi, L.softmax_scale)
        ms.append(m)
        ls.append(l)
        os_.append(ot)
    np.testing.assert_allclose(oracle.combine(ms, ls, np.stack(os_)), row, rtol=0, atol=1e-12)
    m, l, ot = oracle.partial(qh, kk, vv, 0, T - 1, L.softmax_scale)
    np.testing.assert_allclose(ot / l, row, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# plumbing of the oracle itself

def test_row_sampling_and_threads_are_bit_exact():
    L = sliding_layer()
    T = 33
    ids = ids_with_blocks(2, T, [(3, 12)])
    q, k, v, wq, wk = inputs(L, 2, T)
    full = oracle.prefill(L, q, k, v, wq, wk, block_ids=ids, nthreads=1)
    rows = [0, 7, 32]
    part = oracle.prefill(L, q, k, v, wq, wk, block_ids=ids, rows=rows, nthreads=3)
    assert np.array_equal(part, full[:, rows])


def test_window_plus_one_reading_is_available():
    L = sliding_layer(window=5, window_plus_one=True)
    assert oracle.interval(L, None, 20, 10) == (5, 10)  # w + 1 keys


# ---------------------------------------------------------------------------
# cached (chunked) prefill: "gemma4-pt-claude" README, "Tests" -- the cached
# path reproduces the uncached forward pass, bidirectional image spans included

def _chunked(L, q, k, v, wq, wk, ids, cuts):
    """Run the prompt through the oracle's cached path in chunks [cuts[i], cuts[i+1])."""
    B, T = q.shape[:2]
    kh = np.zeros((B, 0, L.num_kv_heads, L.head_dim))
    vh = np.zeros((B, 0, L.num_kv_heads, L.head_dim))
    outs = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, kh, vh = oracle.prefill_chunk(L, q[:, a:b], k[:, a:b], None if v is None else v[:, a:b],
                                         wq, wk, kh, vh,
                                         block_ids=None if ids is None else ids[:, :b])
        outs.append(o)
    return np.concatenate(outs, axis=1), kh, vh


@pytest.mark.parametrize("case", ["sliding_blocks", "global_kv", "global_gqa"])
def test_chunked_prefill_reproduces_the_whole_prompt(case):
    rng = np.random.default_rng(11)
    ids = None
    if case == "sliding_blocks":
        L = sliding_layer(window=6)
        T = 40
        # cuts between blocks (a block cut in two cannot be reproduced: its
        # earlier rows would need later keys); windows reach across every cut
        ids = ids_with_blocks(2, T, [(5, 12), (20, 31), (33, 35)])
        cuts = [0, 13, 32, 40]
    elif case == "global_kv":
        L = global_layer()
        T = 33
        cuts = [0, 1, 17, 33]
    else:
        L = global_layer(k_eq_v=False, num_heads=8, num_kv_heads=2, head_dim=64)
        T = 25
        cuts = [0, 12, 25]
    q, k, v, wq, wk = inputs(L, ids.shape[0] if ids is not None else 1, T, rng)
    got, kh, vh = _chunked(L, q, k, v, wq, wk, ids, cuts)
    ref = dense_reference(L, q, k, v, wq, wk, ids)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # the keys/values accumulated chunk by chunk are those of the whole prompt
    # (the RoPE position of a chunk's token is its position in the prompt)
    kf, vf = oracle.prefill_kv(L, k, v, wk)
    np.testing.assert_array_equal(kh, kf)
    np.testing.assert_array_equal(vh, vf)


def test_chunk_sees_an_image_block_up_to_its_last_position():
    # A block that runs past the chunk's end is seen up to the chunk's last
    # position: the chunk's rows equal the rows of the prompt cut there.
    rng = np.random.default_rng(12)
    L = sliding_layer(window=4)
    T, cut = 30, 20
    ids = ids_with_blocks(1, T, [(14, 27)])
    q, k, v, wq, wk = inputs(L, 1, T, rng)
    kh, vh = oracle.prefill_kv(L, k[:, :10], v[:, :10], wk)
    got, _, _ = oracle.prefill_chunk(L, q[:, 10:cut], k[:, 10:cut], v[:, 10:cut], wq, wk, kh, vh,
                                     block_ids=ids[:, :cut])
    ref = dense_reference(L, q[:, :cut], k[:, :cut], v[:, :cut], wq, wk, ids[:, :cut])[:, 10:]
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # and they differ from the whole prompt's rows, which see the block's tail
    full = dense_reference(L, q, k, v, wq, wk, ids)[:, 10:cut]
    assert np.abs(got[:, 4:] - full[:, 4:]).max() > 1e-3


# ---------------------------------------------------------------------------
# logit soft-cap ("gemma4-pt-claude" README, "Attention Backend":
# attn_logits_soft_cap; reading s <- c * tanh(s / c))

def test_softcap_two_keys_is_a_sigmoid_of_capped_scores():
    L = global_layer(k_eq_v=False, num_heads=1, num_kv_heads=1, softmax_scale=0.37,
                     logit_softcap=0.8)
    q, k, v, wq, wk = inputs(L, 1, 2, rng=np.random.default_rng(21))
    out = oracle.prefill(L, q, k, v, wq, wk)
    qh = oracle.prologue_q(L, q[0, 1, 0], wq, 1)
    k0, v0 = oracle.prologue_kv(L, k[0, 0, 0], v[0, 0, 0], wk, 0)
    k1, v1 = oracle.prologue_kv(L, k[0, 1, 0], v[0, 1, 0], wk, 1)
    c0, c1 = (0.8 * math.tanh(0.37 * (qh @ kk) / 0.8) for kk in (k0, k1))
    sig = 1.0 / (1.0 + math.exp(-(c1 - c0)))
    np.testing.assert_allclose(out[0, 1, 0], sig * v1 + (1 - sig) * v0, rtol=0, atol=1e-14)


@pytest.mark.parametrize("mk", [sliding_layer, global_layer])
def test_softcap_vanishes_as_the_cap_grows(mk):
    rng = np.random.default_rng(22)
    L = mk()
    q, k, v, wq, wk = inputs(L, 1, 20, rng)
    plain = oracle.prefill(L, q, k, v, wq, wk)
    L.logit_softcap = 1e9  # c tanh(s / c) = s - s^3 / (3 c^2) + ...
    np.testing.assert_allclose(oracle.prefill(L, q, k, v, wq, wk), plain, rtol=0, atol=1e-12)


def test_softcap_bounds_every_weight():
    # |capped score| < c, so each of the n weights of a row lies in
    # (e^{-2c} / n, e^{2c} / n); one-hot values read the weights out
    L = global_layer(k_eq_v=False, num_heads=1, num_kv_heads=1, head_dim=32, softmax_scale=50.0,
                     logit_softcap=0.3)
    T = 24
    rng = np.random.default_rng(23)
    q, k, _, wq, wk = inputs(L, 1, T, rng)
    v = np.zeros((1, T, 1, 32), np.float32)
    for j in range(T):
        v[0, j, 0, j] = 1.0  # V-norm scales a one-hot row to e_j / sqrt(1/32 + eps)
    g = math.sqrt(1 / 32 + L.rms_eps)
    out = oracle.prefill(L, q, k, v, wq, wk)[0, :, 0] * g
    for i in range(T):
        w = out[i, :i + 1]
        n = i + 1
        assert abs(w.sum() - 1.0) < 1e-12
        assert w.min() > math.exp(-0.6) / n - 1e-15 and w.max() < math.exp(0.6) / n + 1e-15
    # without the cap the same scores (scale 50) are far from uniform
    L.logit_softcap = 0.0
    plain = oracle.prefill(L, q, k, v, wq, wk)[0, :, 0] * g
    assert plain[T - 1, :T].max() > 0.5


# ---------------------------------------------------------------------------
# padding ("Gemma4ConditionalGenerate" arguments: attention_mask, 1 = keep,
# 0 = padding): padding keys are never attended; a row left with no key is 0

@pytest.mark.parametrize("case", ["sliding_left_pad", "global_left_pad", "sliding_holes_softcap"])
def test_padding_mask_matches_the_dense_reference(case):
    rng = np.random.default_rng(31)
    ids = None
    if case == "sliding_left_pad":
        L = sliding_layer(window=6)
        T = 30
        ids = ids_with_blocks(2, T, [(12, 19)])
        keep = np.ones((2, T), np.int32)
        keep[0, :5] = 0  # sequence 0 left-padded by 5, sequence 1 not at all
    elif case == "global_left_pad":
        L = global_layer()
        T = 26
        keep = np.ones((1, T), np.int32)
        keep[0, :9] = 0
    else:
        L = sliding_layer(window=5, logit_softcap=2.0)
        T = 24
        keep = (rng.random((1, T)) > 0.3).astype(np.int32)
        keep[0, 10:16] = 0  # rows 10..15 (window 5) see no key at all
    B = keep.shape[0]
    q, k, v, wq, wk = inputs(L, B, T, rng)
    got = oracle.prefill(L, q, k, v, wq, wk, block_ids=ids, attention_mask=keep)
    ref = dense_reference(L, q, k, v, wq, wk, ids, keep)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    if case == "sliding_holes_softcap":
        assert not got[0, 14].any()  # a row with no key left is exactly 0


def test_all_ones_padding_mask_changes_nothing():
    rng = np.random.default_rng(32)
    L = sliding_layer(window=7)
    q, k, v, wq, wk = inputs(L, 2, 21, rng)
    plain = oracle.prefill(L, q, k, v, wq, wk)
    masked = oracle.prefill(L, q, k, v, wq, wk, attention_mask=np.ones((2, 21), np.int32))
    np.testing.assert_array_equal(masked, plain)


@pytest.mark.parametrize("case", ["sliding_left_pad", "global_holes_softcap", "rolling"])
def test_masked_decode_equals_last_row_of_the_masked_prefill(case):
    """Decode with the prompt's padding mask (positions past the mask are
    generated tokens, always kept) is the last row of the masked prefill over
    the prompt plus the new token."""
    rng = np.random.default_rng(41)
    T = 37  # cached positions; the new token sits at T
    if case == "global_holes_softcap":
        L = global_layer(logit_softcap=3.0)
    else:
        L = sliding_layer(window=12)
    B = 2
    q, k, v, wq, wk = inputs(L, B, T + 1, rng)
    keep = np.ones((B, T), np.int32)
    if case == "global_holes_softcap":
        keep[0] = (rng.random(T) > 0.4)
        keep[1, :20] = 0
    else:
        keep[0, :30] = 0  # left padding reaching into the last window
        keep[1, 26:29] = 0
    full = np.concatenate([keep, np.ones((B, 1), np.int32)], axis=1)
    ref = oracle.prefill(L, q, k, v, wq, wk, attention_mask=full)[:, T]
    kh, vh = oracle.prefill_kv(L, k[:, :T], None if v is None else v[:, :T], wk)
    rolling = case == "rolling"
    C = L.window if rolling else 64
    out = oracle.decode(L, q[:, T:T + 1], wq, _cache_from(kh, C, rolling),
                        _cache_from(vh, C, rolling), C, rolling, [T, T],
                        k_new=k[:, T:T + 1], v_new=None if v is None else v[:, T:T + 1], wk=wk,
                        attention_mask=keep)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # an all-ones mask is the unmasked decode, bit for bit
    plain = oracle.decode(L, q[:, T:T + 1], wq, _cache_from(kh, C, rolling),
                          _cache_from(vh, C, rolling), C, rolling, [T, T],
                          k_new=k[:, T:T + 1], v_new=None if v is None else v[:, T:T + 1], wk=wk)
    ones = oracle.decode(L, q[:, T:T + 1], wq, _cache_from(kh, C, rolling),
                         _cache_from(vh, C, rolling), C, rolling, [T, T],
                         k_new=k[:, T:T + 1], v_new=None if v is None else v[:, T:T + 1], wk=wk,
                         attention_mask=np.ones((B, T), np.int32))
    np.testing.assert_array_equal(ones, plain)


@pytest.mark.parametrize("case", ["sliding_blocks_mask_softcap", "global_chunk"])
def test_attend_rows_from_the_oracles_own_prologue_is_prefill(case):
    """Attention from given post-prologue vectors, fed the oracle's own
    q_hat / k_hat / v_hat, is the oracle's prefill bit for bit: the same
    intervals, padding, soft-cap and softmax (so it inherits every pin of
    the prefill path)."""
    rng = np.random.default_rng(51)
    if case == "sliding_blocks_mask_softcap":
        L = sliding_layer(window=6, logit_softcap=1.5, num_heads=4, num_kv_heads=2)
        T, p0 = 33, 0
        ids = ids_with_blocks(2, T, [(4, 15), (20, 24)])
        keep = (rng.random((2, T)) > 0.25).astype(np.int32)
    else:
        L = global_layer()
        T, p0 = 17, 20
        ids, keep = None, None
    B = 2
    q, k, v, wq, wk = inputs(L, B, p0 + T, rng)
    kh, vh = oracle.prefill_kv(L, k, v, wk)
    rows = [0, 3, T - 1]
    want = oracle.prefill_chunk_rows(L, q[:, p0:], wq, kh, vh, p0, block_ids=ids, rows=rows,
                                     attention_mask=keep)
    qh = oracle.prologue_q_all(L, q[:, p0:], wq, p0)
    got = oracle.attend_rows(L, qh, kh, vh, p0, block_ids=ids, rows=rows, attention_mask=keep)
    np.testing.assert_array_equal(got, want)
    # and each q_hat is the single-vector prologue at its position
    for t in (0, T - 1):
        np.testing.assert_array_equal(qh[1, t, 2 % L.num_heads],
                                      oracle.prologue_q(L, q[1, p0 + t, 2 % L.num_heads], wq,
                                                        p0 + t))


# ---------------------------------------------------------------------------
# the bidirectional (vision-tower) layer: every query sees every key of its
# sequence ("gemma4-pt-claude" README, "Key architectural features": a
# ViT-style encoder with bidirectional attention; "Attention Backend Notes":
# the tower's softmax scale is 1.0)

def bidirectional_layer(**kw):
    base = dict(layer_type=BIDIRECTIONAL, rotary_fraction=1.0, rope_theta=1e4, num_heads=4,
                num_kv_heads=4, head_dim=16, softmax_scale=1.0, rms_eps=1e-6)
    base.update(kw)
    return Layer(**base)


@pytest.mark.parametrize("pad", [False, True])
def test_bidirectional_matches_the_dense_reference(pad):
    rng = np.random.default_rng(31)
    L = bidirectional_layer(num_heads=6, num_kv_heads=2)
    B, T = 2, 29
    q, k, v, wq, wk = inputs(L, B, T, rng)
    keep = (rng.random((B, T)) > 0.3).astype(np.uint8) if pad else None
    got = oracle.prefill(L, q, k, v, wq, wk, attention_mask=keep)
    ref = dense_reference(L, q, k, v, wq, wk, None, keep)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_bidirectional_zero_query_gives_the_mean_of_every_value():
    """q = 0: uniform weights over all T keys, so every row -- the first one
    included -- is the mean of all normalised values (a causal row 0 would
    return v_0)."""
    L = bidirectional_layer()
    T = 17
    q, k, v, wq, wk = inputs(L, 1, T)
    got = oracle.prefill(L, np.zeros_like(q), k, v, wq, wk)
    _, vh = oracle.prefill_kv(L, k, v, wk)
    mean = vh[0].mean(axis=0)  # [Hkv, d]
    for i in range(T):
        np.testing.assert_allclose(got[0, i], mean, rtol=0, atol=1e-13)


def test_bidirectional_last_row_is_the_causal_last_row_and_block_ids_are_ignored():
    rng = np.random.default_rng(32)
    L = bidirectional_layer(rotary_fraction=0.25, rope_theta=1e6)
    T = 21
    q, k, v, wq, wk = inputs(L, 1, T, rng)
    bi = oracle.prefill(L, q, k, v, wq, wk)
    ca = oracle.prefill(global_layer(**{f: getattr(L, f) for f in (
        "rotary_fraction", "rope_theta", "k_eq_v", "num_heads", "num_kv_heads", "head_dim",
        "softmax_scale")}), q, k, v, wq, wk)
    assert np.array_equal(bi[0, T - 1], ca[0, T - 1])  # both see keys 0..T-1
    assert not np.allclose(bi[0, 0], ca[0, 0])
    ids = ids_with_blocks(1, T, [(3, 9)])
    assert np.array_equal(oracle.prefill(L, q, k, v, wq, wk, block_ids=ids), bi)


def test_bidirectional_rows_do_not_depend_on_the_key_order():
    """From given post-prologue vectors (no RoPE), a bidirectional row is a
    function of the key set: permuting the keys (K and V together) leaves
    every output unchanged."""
    rng = np.random.default_rng(33)
    L = bidirectional_layer(num_heads=4, num_kv_heads=2)
    B, T, d = 1, 19, L.head_dim
    qh = rng.standard_normal((B, T, 4, d))
    kh = rng.standard_normal((B, T, 2, d))
    vh = rng.standard_normal((B, T, 2, d))
    perm = rng.permutation(T)
    a = oracle.attend_rows(L, qh, kh, vh, 0)
    b = oracle.attend_rows(L, qh, kh[:, perm], vh[:, perm], 0)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_bidirectional_layer_has_no_decode():
    L = bidirectional_layer()
    with pytest.raises(ValueError):
        oracle.decode(L, np.zeros((1, 1, 4, 16), np.float32), np.ones(16, np.float32),
                      np.zeros((1, 4, 4, 16)), np.zeros((1, 4, 4, 16)), 4, False, [1])


# ---------------------------------------------------------------------------
# the QKV projection in front of the prologue

@pytest.mark.parametrize("mk", [sliding_layer, global_layer, bidirectional_layer])
def test_qkv_projection_by_a_permutation_is_the_prologue_of_permuted_inputs(mk):
    """W a (non-symmetric) permutation matrix: raw = x W^T picks coordinate
    perm[j] of x for output j, so the result is the prologue of those raw
    vectors, bit for bit.  A transposed W (x W picks perm^-1) or a wrong head
    order (Q rows, then K, then V) fails."""
    rng = np.random.default_rng(41)
    L = mk()
    Hq, Hkv, d = L.num_heads, L.num_kv_heads, L.head_dim
    n = Hq + (Hkv if L.k_eq_v else 2 * Hkv)
    B, T, hidden = 2, 9, n * d
    x = f32(B, T, hidden, rng=rng)
    perm = rng.permutation(hidden)
    Wm = np.zeros((hidden, hidden), np.float32)
    Wm[np.arange(hidden), perm] = 1.0
    wq, wk = f32(d, rng=rng), f32(d, rng=rng)
    qh, kh, vh = oracle.qkv_prologue(L, x, Wm, wq, wk, p0=5)
    raw = x[..., perm].astype(np.float64)
    q_raw = raw[..., :Hq * d].reshape(B, T, Hq, d)
    k_raw = raw[..., Hq * d:(Hq + Hkv) * d].reshape(B, T, Hkv, d)
    v_raw = None if L.k_eq_v else raw[..., (Hq + Hkv) * d:].reshape(B, T, Hkv, d)
    assert np.array_equal(qh, oracle.prologue_q_all(L, q_raw, wq, 5))
    k2, v2 = oracle.prefill_kv(L, k_raw, v_raw, wk, p0=5)
    assert np.array_equal(kh, k2) and np.array_equal(vh, v2)


def test_qkv_projection_is_scale_free_and_queries_only_without_kv():
    """RMSNorm removes a positive scale of x (eps = 0: exactly up to rounding);
    without KV heads W holds the query rows alone."""
    rng = np.random.default_rng(42)
    L = global_layer(rms_eps=0.0)
    Hq, d = L.num_heads, L.head_dim
    hidden = 48
    x = f32(1, 7, hidden, rng=rng)
    Wm = f32(Hq * d, hidden, rng=rng)
    wq = f32(d, rng=rng)
    a, k, v = oracle.qkv_prologue(L, x, Wm, wq, with_kv=False)
    assert k is None and v is None
    b, _, _ = oracle.qkv_prologue(L, 3.5 * x.astype(np.float64), Wm, wq, with_kv=False)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    with pytest.raises(ValueError):
        oracle.qkv_prologue(L, x, Wm, wq, f32(d, rng=rng))  # KV rows missing
