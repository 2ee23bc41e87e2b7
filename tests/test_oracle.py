"""Pins for the float64 oracle (CPU only).

Each check ties the oracle to something other than itself: closed forms of the
softmax, invariances the definition implies, a 50-digit brute force written in
the textbook exp(s)/sum(exp(s)) form (no max subtraction), torch's own CPU
float64 scaled_dot_product_attention, and values printed on the pages.  The
checks are chosen so that a dropped scale, a wrong sign, an off-by-one causal
mask, a transposed operand or a missing normalisation each fails at least one.
"""

import json
import math
import os

import mpmath
import numpy as np
import pytest
import torch

from oracle import (
    allowed_keys,
    attention,
    attention_batched,
    attention_rows,
    attention_tiled_online,
    online_softmax_step,
    resolve_scale,
    attention_paged,
    gather_paged_kv,
    merge_partials,
    band_mask,
    block_sparse_mask,
    attention_masked,
    attention_backward,
    attention_backward_batched,
    attention_backward_tiled,
)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def rnd(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


# ---------------------------------------------------------------- brute force
def brute(q, k, v, scale, causal):
    """50-digit brute force: p_ij = exp(s_ij) / sum_j' exp(s_ij'), no max shift."""
    mpmath.mp.dps = 50
    nq, d = q.shape
    nkv = k.shape[0]
    o = np.empty((nq, v.shape[1]))
    lse = np.empty(nq)
    for i in range(nq):
        js = range(nkv) if not causal else range(min(i + 1, nkv))
        s = {j: mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(q[i, c]) * mpmath.mpf(k[j, c]) for c in range(d))
             for j in js}
        ex = {j: mpmath.exp(s[j]) for j in js}
        z = mpmath.fsum(ex.values())
        for c in range(v.shape[1]):
            o[i, c] = float(mpmath.fsum(ex[j] * mpmath.mpf(v[j, c]) for j in js) / z)
        lse[i] = float(mpmath.log(z))
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nkv,d", [(1, 1, 1), (3, 5, 2), (5, 3, 4), (8, 8, 8), (7, 2, 3)])
def test_brute_force_tiny(nq, nkv, d, causal):
    q, k, v = rnd(nq, d), rnd(nkv, d), rnd(nkv, d)
    sc = 0.7
    o, lse = attention(q, k, v, scale=sc, causal=causal)
    ob, lb = brute(q, k, v, sc, causal)
    assert np.max(np.abs(o - ob)) <= 1e-13
    assert np.max(np.abs(lse - lb)) <= 1e-13


@pytest.mark.parametrize("kind", ["all_ones", "large_random", "alternating_extremes"])
def test_page1_regression_inputs_vs_brute(kind):
    """Page 1 section 数值安全的边界条件 lists three regression input families:
    all-ones, large random values and alternating extremes."""
    nq, nkv, d = 6, 7, 4
    if kind == "all_ones":
        q, k, v = np.ones((nq, d)), np.ones((nkv, d)), rnd(nkv, d)
    elif kind == "large_random":
        q, k, v = rnd(nq, d, scale=30), rnd(nkv, d, scale=30), rnd(nkv, d)
    else:
        sign = np.where(np.arange(nkv) % 2 == 0, 1.0, -1.0)[:, None]
        q = np.where(np.arange(nq)[:, None] % 2 == 0, 60.0, -60.0) * np.ones((nq, d))
        k = sign * 60.0 * np.ones((nkv, d))
        v = rnd(nkv, d)
    for causal in (False, True):
        o, lse = attention(q, k, v, scale=0.125, causal=causal)
        ob, lb = brute(q, k, v, 0.125, causal)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
        assert np.max(np.abs(o - ob)) <= 1e-12
        assert np.max(np.abs(lse - lb)) <= 1e-12 * max(1.0, np.max(np.abs(lb)))
    if kind == "all_ones":  # uniform weights: O is the plain mean of V
        o, _ = attention(q, k, v, scale=0.125)
        assert np.allclose(o, v.mean(axis=0)[None, :], atol=1e-14)


def test_worked_example_closed_form():
    """q = (1, 0), keys e1, e2, scale 1: weights e/(e+1) and 1/(e+1)."""
    q = np.array([[1.0, 0.0]])
    k = np.array([[1.0, 0.0], [0.0, 1.0]])
    v = np.array([[1.0, 2.0], [3.0, 4.0]])
    o, lse = attention(q, k, v, scale=1.0)
    e = math.e
    assert np.allclose(o[0], [(e + 3) / (e + 1), (2 * e + 4) / (e + 1)], atol=1e-15)
    assert abs(lse[0] - math.log(e + 1)) < 1e-15


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_visible_values(causal):
    nq, nkv, d = 37, 29, 16
    q, k, v = np.zeros((nq, d)), rnd(nkv, d), rnd(nkv, d)
    o, lse = attention(q, k, v, causal=causal)
    for i in range(nq):
        a = allowed_keys(i, nkv, causal)
        assert np.allclose(o[i], v[a].mean(axis=0), atol=1e-13)
        assert abs(lse[i] - math.log(len(a))) < 1e-13


def test_allowed_keys_is_top_left_triu():
    """Page 3 section 6.1: mask = triu(ones(Nq, Nkv), diagonal=1)."""
    for nq, nkv in [(5, 5), (3, 7), (7, 3)]:
        mask = torch.triu(torch.ones(nq, nkv), diagonal=1).bool().numpy()
        for i in range(nq):
            vis = np.zeros(nkv, bool)
            vis[allowed_keys(i, nkv, True)] = True
            assert np.array_equal(vis, ~mask[i])


@pytest.mark.parametrize("causal", [False, True])
def test_constant_value_rows_pass_through(causal):
    nq, nkv, d = 20, 33, 8
    c = rnd(d)
    q, k = rnd(nq, d, scale=3), rnd(nkv, d, scale=3)
    v = np.tile(c, (nkv, 1))
    o, _ = attention(q, k, v, causal=causal)
    assert np.allclose(o, c[None, :], atol=1e-13)


def test_causal_row0_and_single_key():
    nq, nkv, d = 9, 9, 5
    q, k, v = rnd(nq, d), rnd(nkv, d), rnd(nkv, d)
    sc = 0.31
    o, lse = attention(q, k, v, scale=sc, causal=True)
    assert np.allclose(o[0], v[0], atol=1e-15)
    assert abs(lse[0] - sc * q[0] @ k[0]) < 1e-14
    o1, lse1 = attention(q, k[:1], v[:1], scale=sc)
    assert np.allclose(o1, np.tile(v[0], (nq, 1)), atol=1e-15)
    assert np.allclose(lse1, sc * q @ k[0], atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(causal):
    nq, nkv, d = 15, 21, 6
    q, k, v = rnd(nq, d), rnd(nkv, d), rnd(nkv, d)
    c = rnd(d, scale=2)
    sc = 0.4
    o, lse = attention(q, k, v, scale=sc, causal=causal)
    o2, lse2 = attention(q, k + c[None, :], v, scale=sc, causal=causal)
    assert np.allclose(o, o2, atol=1e-12)
    assert np.allclose(lse2, lse + sc * (q @ c), atol=1e-12)


def test_permutation_invariance_noncausal():
    nq, nkv, d = 11, 17, 4
    q, k, v = rnd(nq, d), rnd(nkv, d), rnd(nkv, d)
    perm = RNG.permutation(nkv)
    o, lse = attention(q, k, v)
    o2, lse2 = attention(q, k[perm], v[perm])
    assert np.allclose(o, o2, atol=1e-13) and np.allclose(lse, lse2, atol=1e-13)


def test_scale_resolution():
    """Page 3 Config: softmax_scale = -1 means 1/sqrt(d)."""
    assert resolve_scale(None, 64) == 0.125
    assert resolve_scale(-1.0, 64) == 0.125
    assert resolve_scale(0.0, 16) == 0.25
    assert resolve_scale(float("nan"), 4) == 0.5
    assert resolve_scale(0.3, 4) == 0.3


# ---------------------------------------------------------------- tiled twin
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("br,bc", [(1, 1), (3, 16), (16, 3), (64, 128), (128, 64), (128, 128)])
def test_tiled_online_equals_naive(br, bc, causal):
    """Page 1 section 分块 Tiling 的计算骨架: the tiled result equals the global
    softmax exactly (up to rounding)."""
    nq, nkv, d = 150, 173, 8
    q, k, v = rnd(nq, d, scale=2), rnd(nkv, d, scale=2), rnd(nkv, d)
    o, lse = attention(q, k, v, causal=causal)
    o2, lse2 = attention_tiled_online(q, k, v, br, bc, causal=causal)
    assert np.max(np.abs(o - o2)) <= 1e-12
    assert np.max(np.abs(lse - lse2)) <= 1e-12


def test_online_step_matches_direct_sums():
    """Page 1 section 在线 Softmax: merging block statistics equals the direct sum."""
    x = rnd(300, scale=4)
    m, l = -math.inf, 0.0
    for c0 in range(0, 300, 37):
        m, l = online_softmax_step(m, l, x[c0:c0 + 37])
    assert abs(m - x.max()) == 0
    assert abs(l - np.exp(x - x.max()).sum()) <= 1e-12 * l


def test_golden_rescale_underflow():
    """Page 1 numerical-safety figure: a max jump of 100 rescales the previous
    sum by exp(-100) ~ 3.7e-44 (below float32's smallest normal ~1.2e-38); in
    float64 the merge is still exact."""
    g = json.load(open(os.path.join(GOLDEN, "page1_numerical_safety.json")))
    f = math.exp(-100.0)
    assert abs(f - g["exp_minus_100"]) <= g["exp_minus_100_rel_tol"] * g["exp_minus_100"]
    assert f < float(np.finfo(np.float32).tiny)
    assert abs(float(np.finfo(np.float32).tiny) - g["float32_min_normal"]) <= \
        g["float32_min_normal_rel_tol"] * g["float32_min_normal"]
    x1 = np.array([0.0, -1.0, -2.0])
    x2 = np.array([100.0, 99.0])
    m, l = online_softmax_step(-math.inf, 0.0, x1)
    m, l = online_softmax_step(m, l, x2)
    direct = np.exp(np.concatenate([x1, x2]) - 100.0).sum()
    assert m == 100.0 and abs(l - direct) <= 1e-15 * direct
    # the same jump inside the tiled attention: one key dominates by 100
    q = np.array([[1.0]])
    k = np.array([[0.0], [100.0]])
    v = np.array([[5.0], [7.0]])
    o, lse = attention_tiled_online(q, k, v, 1, 1, scale=1.0)
    assert abs(o[0, 0] - (5.0 * f + 7.0) / (1.0 + f)) <= 1e-15
    assert abs(lse[0] - (100.0 + math.log1p(f))) <= 1e-13


# ---------------------------------------------------------------- library cross-check
@pytest.mark.parametrize("causal", [False, True])
def test_torch_sdpa_float64_cross_check(causal):
    B, H, N, d = 2, 3, 97, 16
    q, k, v = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
    o, lse = attention_batched(q, k, v, causal=causal)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=causal).numpy()
    assert np.max(np.abs(o - ref)) <= 1e-12


def test_layouts_and_rows_agree():
    B, H, nq, nkv, d = 2, 3, 19, 23, 8
    q, k, v = rnd(B, H, nq, d), rnd(B, H, nkv, d), rnd(B, H, nkv, d)
    for causal in (False, True):
        o, lse = attention_batched(q, k, v, causal=causal, layout="BHND")
        o2, lse2 = attention_batched(q.transpose(0, 2, 1, 3), k.transpose(0, 2, 1, 3),
                                     v.transpose(0, 2, 1, 3), causal=causal, layout="BSND")
        assert np.array_equal(o, o2.transpose(0, 2, 1, 3)) and np.array_equal(lse, lse2)
        rows = [0, 5, 18]
        orow, lrow = attention_rows(q[1, 2, rows], k[1, 2], v[1, 2], rows, causal=causal)
        assert np.max(np.abs(orow - o[1, 2, rows])) <= 1e-13
        assert np.max(np.abs(lrow - lse[1, 2, rows])) <= 1e-13


def test_row_blocking_is_invisible():
    """Query rows beyond one internal row block give the same rows as alone."""
    import oracle.attention_ref as ar

    nq, nkv, d = 40, 31, 4
    q, k, v = rnd(nq, d), rnd(nkv, d), rnd(nkv, d)
    old = ar.ROW_BLOCK
    try:
        ar.ROW_BLOCK = 7
        o, lse = attention(q, k, v, causal=True)
    finally:
        ar.ROW_BLOCK = old
    o2, lse2 = attention(q, k, v, causal=True)
    assert np.max(np.abs(o - o2)) <= 1e-14 and np.max(np.abs(lse - lse2)) <= 1e-14


def test_row_offset_block_equals_full_rows():
    nq, nkv, d = 50, 60, 4
    q, k, v = rnd(nq, d), rnd(nkv, d), rnd(nkv, d)
    o, lse = attention(q, k, v, causal=True)
    o2, lse2 = attention(q[17:41], k, v, causal=True, row_offset=17)
    assert np.max(np.abs(o[17:41] - o2)) <= 1e-14 and np.max(np.abs(lse[17:41] - lse2)) <= 1e-14


def test_empty_and_invalid():
    o, lse = attention(np.zeros((0, 4)), rnd(3, 4), rnd(3, 4))
    assert o.shape == (0, 4) and lse.shape == (0,)
    with pytest.raises(ValueError):
        attention(rnd(2, 4), np.zeros((0, 4)), np.zeros((0, 4)))


# ---------------------------------------------------------------- grouped-query attention (K/V heads < query heads)
def test_gqa_grouping_is_contiguous_closed_form():
    """H = 6 query heads over Hkv = 3 K/V heads with a constant value row per
    K/V head: query heads 2g and 2g+1 must return that head's constant (a
    strided mapping h % Hkv, or a transposed group index, gives other values)."""
    B, H, hkv, nq, nkv, d = 1, 6, 3, 9, 11, 4
    q, k = rnd(B, H, nq, d), rnd(B, hkv, nkv, d)
    consts = np.array([1.5, -2.0, 7.25])
    v = np.broadcast_to(consts[None, :, None, None], (B, hkv, nkv, d)).copy()
    for causal in (False, True):
        o, _ = attention_batched(q, k, v, causal=causal)
        for h in range(H):
            assert np.max(np.abs(o[0, h] - consts[h // 2])) <= 1e-13, h


def test_mqa_zero_query_gives_mean_of_shared_values():
    """One K/V head shared by every query head (MQA) with Q = 0: each row is
    the uniform mean of the visible V rows and LSE = ln(#visible)."""
    B, H, n, d = 2, 5, 13, 6
    q, k, v = np.zeros((B, H, n, d)), rnd(B, 1, n, d), rnd(B, 1, n, d)
    for causal in (False, True):
        o, lse = attention_batched(q, k, v, causal=causal)
        for b in range(B):
            for i in range(n):
                cnt = i + 1 if causal else n
                assert np.max(np.abs(o[b, :, i] - v[b, 0, :cnt].mean(axis=0))) <= 1e-13
                assert np.max(np.abs(lse[b, :, i] - math.log(cnt))) <= 1e-13


@pytest.mark.parametrize("hkv", [1, 2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_torch_sdpa_float64_cross_check(hkv, causal):
    """Library cross-check: torch's scaled_dot_product_attention with
    enable_gqa (which repeats each K/V head over a contiguous block of query
    heads), float64 on the CPU; both layouts."""
    B, H, n, d = 2, 8, 37, 16
    q, k, v = rnd(B, H, n, d), rnd(B, hkv, n, d), rnd(B, hkv, n, d)
    o, _ = attention_batched(q, k, v, causal=causal)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=causal, enable_gqa=True).numpy()
    assert np.max(np.abs(o - ref)) <= 1e-12
    o2, _ = attention_batched(q.transpose(0, 2, 1, 3), k.transpose(0, 2, 1, 3), v.transpose(0, 2, 1, 3),
                              causal=causal, layout="BSND")
    assert np.array_equal(o, o2.transpose(0, 2, 1, 3))


def test_gqa_rejects_non_dividing_kv_heads():
    with pytest.raises(ValueError):
        attention_batched(rnd(1, 6, 4, 4), rnd(1, 4, 4, 4), rnd(1, 4, 4, 4))


# ---------------------------------------------------------------- paged K/V cache (gather through a block table)
def _scatter_into_cache(kv, bs, perm, n_phys):
    """Place the logical blocks of a contiguous [N, Hkv, d] sequence into the
    physical blocks perm[i] of a fresh cache, by an explicit loop; every other
    element of the cache (unused blocks, the tail of the last block) is NaN."""
    n, hkv, d = kv.shape
    cache = np.full((n_phys, bs, hkv, d), np.nan)
    for i in range(-(-n // bs)):
        rows = kv[i * bs:(i + 1) * bs]
        cache[perm[i], :rows.shape[0]] = rows
    return cache


def test_gather_identity_table_is_a_reshape():
    bs, nb, hkv, d = 16, 5, 2, 8
    k = rnd(nb * bs, hkv, d)
    cache = k.reshape(nb, bs, hkv, d)
    assert np.array_equal(gather_paged_kv(cache, np.arange(nb), nb * bs), k)
    assert np.array_equal(gather_paged_kv(cache, np.arange(nb), 37), k[:37])


@pytest.mark.parametrize("seq_len", [1, 16, 45, 80])
def test_gather_scattered_blocks_reads_only_its_rows(seq_len):
    rng = np.random.default_rng(seq_len)
    bs, hkv, d, n_phys = 16, 3, 4, 11
    k = rnd(seq_len, hkv, d)
    perm = rng.permutation(n_phys)
    cache = _scatter_into_cache(k, bs, perm, n_phys)
    table = np.concatenate([perm[:-(-seq_len // bs)], np.full(3, 10_000)])  # entries past the sequence are junk
    g = gather_paged_kv(cache, table, seq_len)
    assert np.all(np.isfinite(g)) and np.array_equal(g, k)


def test_gather_rejects_bad_tables():
    cache = rnd(4, 16, 1, 4)
    with pytest.raises(ValueError):
        gather_paged_kv(cache, np.array([0, 9]), 20)   # entry out of range
    with pytest.raises(ValueError):
        gather_paged_kv(cache, np.array([0]), 20)      # table too short


@pytest.mark.parametrize("layout", ["BHND", "BSND"])
@pytest.mark.parametrize("causal", [False, True])
def test_attention_paged_equals_contiguous(layout, causal):
    """Attention through a paged cache (a different block order per batch
    entry, NaN everywhere the table does not point) equals attention on the
    contiguous K/V, exactly."""
    rng = np.random.default_rng(7)
    B, H, hkv, n, d, bs = 2, 4, 2, 70, 8, 16
    k, v = rnd(B, n, hkv, d), rnd(B, n, hkv, d)
    nb = -(-n // bs)
    n_phys = B * nb + 3
    order = rng.permutation(n_phys)
    tables = np.stack([order[b * nb:(b + 1) * nb] for b in range(B)])
    kc = np.full((n_phys, bs, hkv, d), np.nan)
    vc = np.full((n_phys, bs, hkv, d), np.nan)
    for b in range(B):
        kc_b = _scatter_into_cache(k[b], bs, tables[b], n_phys)
        vc_b = _scatter_into_cache(v[b], bs, tables[b], n_phys)
        used = np.isfinite(kc_b)
        kc[used], vc[used] = kc_b[used], vc_b[used]
    q = rnd(B, H, n, d) if layout == "BHND" else rnd(B, n, H, d)
    kk, vv = (k, v) if layout == "BSND" else (k.transpose(0, 2, 1, 3), v.transpose(0, 2, 1, 3))
    o_ref, l_ref = attention_batched(q, kk, vv, causal=causal, layout=layout)
    o, lse = attention_paged(q, kc, vc, tables, n, causal=causal, layout=layout)
    assert np.all(np.isfinite(o)) and np.array_equal(o, o_ref) and np.array_equal(lse, l_ref)


# ---------------------------------------------------------------- split key sets: merging partial results
@pytest.mark.parametrize("causal", [False, True])
def test_merge_of_key_parts_equals_whole(causal):
    """Attention over the whole key set equals the merge of attention over
    disjoint key ranges (for causal rows, ranges they cannot see have
    LSE = -inf and weight 0)."""
    nq, nkv, d = 23, 41, 8
    q, k, v = rnd(nq, d), rnd(nkv, d), rnd(nkv, d)
    o, lse = attention(q, k, v, causal=causal)
    cuts = [0, 5, 17, 18, 41]
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        po, pl = np.zeros((nq, d)), np.full(nq, -np.inf)
        for i in range(nq):
            hi = min(b, i + 1) if causal else b
            if hi > a:
                ro, rl = attention(q[i:i + 1], k[a:hi], v[a:hi])
                po[i], pl[i] = ro[0], rl[0]
        parts_o.append(po)
        parts_l.append(pl)
    mo, ml = merge_partials(np.stack(parts_o), np.stack(parts_l))
    assert np.max(np.abs(mo - o)) <= 1e-13 and np.max(np.abs(ml - lse)) <= 1e-13


# ---------------------------------------------------------------- gradients (backward)
@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_finite_differences(causal):
    """Central differences of L = sum(O * W) + sum(LSE * u), through the forward
    oracle, against the gradient oracle, at every entry of Q, K and V."""
    nq, nkv, d = 5, 7, 4
    q, k, v = rnd(nq, d), rnd(nkv, d), rnd(nkv, d)
    w, u = rnd(nq, d), rnd(nq)

    def loss(qq, kk, vv):
        o, lse = attention(qq, kk, vv, causal=causal)
        return float(np.sum(o * w) + np.sum(lse * u))

    dq, dk, dv = attention_backward(q, k, v, w, causal=causal, dlse=u)
    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            lp = loss(q, k, v)
            x[idx] = old - h
            lm = loss(q, k, v)
            x[idx] = old
            assert abs((lp - lm) / (2 * h) - g[idx]) <= 1e-7, idx


@pytest.mark.parametrize("hkv", [4, 2, 1])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_torch_autograd_cross_check(hkv, causal):
    """Library cross-check: torch float64 scaled_dot_product_attention with
    autograd (grouped K/V heads included), both layouts."""
    B, H, n, d = 2, 4, 19, 8
    q, k, v, do = rnd(B, H, n, d), rnd(B, hkv, n, d), rnd(B, hkv, n, d), rnd(B, H, n, d)
    tq, tk, tv = (torch.from_numpy(x.copy()).requires_grad_(True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, enable_gqa=True)
    out.backward(torch.from_numpy(do))
    dq, dk, dv = attention_backward_batched(q, k, v, do, causal=causal)
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.max(np.abs(mine - ref.numpy())) <= 1e-10
    t = (0, 2, 1, 3)
    dq2, dk2, dv2 = attention_backward_batched(q.transpose(t), k.transpose(t), v.transpose(t), do.transpose(t),
                                               causal=causal, layout="BSND")
    assert np.array_equal(dq2.transpose(t), dq) and np.array_equal(dk2.transpose(t), dk)


@pytest.mark.parametrize("br,bc", [(1, 1), (3, 5), (16, 16), (64, 7)])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_tiled_recompute_equals_definition(br, bc, causal):
    """The page's recompute scheme (tiles rebuilt from the forward's LSE only)
    gives the definition's gradients, for any tile sizes."""
    nq, nkv, d = 29, 37, 8
    q, k, v, do = rnd(nq, d), rnd(nkv, d), rnd(nkv, d), rnd(nq, d)
    _, lse = attention(q, k, v, causal=causal)
    ref = attention_backward(q, k, v, do, causal=causal)
    got = attention_backward_tiled(q, k, v, do, lse, br, bc, causal=causal)
    for a, b in zip(got, ref):
        assert np.max(np.abs(a - b)) <= 1e-12


def test_backward_equal_keys_give_zero_query_gradient():
    """All keys equal: every row's scores are constant, the softmax does not
    depend on Q, so dQ = 0 (the rows of dS sum to zero)."""
    nq, nkv, d = 6, 9, 5
    q, v, do = rnd(nq, d), rnd(nkv, d), rnd(nq, d)
    k = np.tile(rnd(1, d), (nkv, 1))
    dq, _, dv = attention_backward(q, k, v, do)
    assert np.max(np.abs(dq)) <= 1e-13
    assert np.max(np.abs(dv - np.tile(do.sum(axis=0) / nkv, (nkv, 1)))) <= 1e-13  # uniform P = 1/Nkv: dV_j = sum_i dO_i / Nkv


# ---------------------------------------------------------------- band and block-sparse masks
def test_band_reduces_to_causal_and_full():
    """pre_tokens >= N, next_tokens = 0 (page 2's causal call) is the causal
    path; both >= N is unmasked attention."""
    n, d = 33, 8
    q, k, v = rnd(n, d), rnd(n, d), rnd(n, d)
    o_c, l_c = attention(q, k, v, causal=True)
    o_b, l_b = attention_masked(q, k, v, band_mask(n, n, n, 0))
    assert np.max(np.abs(o_b - o_c)) <= 1e-13 and np.max(np.abs(l_b - l_c)) <= 1e-13
    for i in range(n):  # the same visible sets as the causal reading
        assert np.array_equal(np.flatnonzero(band_mask(n, n, n, 0)[i]), allowed_keys(i, n, True))
    o_f, l_f = attention(q, k, v)
    o_b2, l_b2 = attention_masked(q, k, v, band_mask(n, n, n, n))
    assert np.max(np.abs(o_b2 - o_f)) <= 1e-13 and np.max(np.abs(l_b2 - l_f)) <= 1e-13


def test_band_of_width_one_is_the_diagonal():
    """pre = next = 0: every query sees only its own key: O_i = V_i and
    LSE_i = scale * q_i . k_i."""
    n, d = 7, 4
    q, k, v = rnd(n, d), rnd(n, d), rnd(n, d)
    o, lse = attention_masked(q, k, v, band_mask(n, n, 0, 0))
    assert np.max(np.abs(o - v)) <= 1e-14
    assert np.max(np.abs(lse - np.sum(q * k, axis=1) / math.sqrt(d))) <= 1e-13


@pytest.mark.parametrize("pre,nxt", [(3, 2), (0, 5), (10, 0), (1, 1)])
def test_band_torch_sdpa_cross_check(pre, nxt):
    """Library cross-check: torch float64 scaled_dot_product_attention with the
    band as an explicit boolean attn_mask."""
    n, d = 21, 8
    q, k, v = rnd(1, 1, n, d), rnd(1, 1, n, d), rnd(1, 1, n, d)
    mask = band_mask(n, n, pre, nxt)
    o, _ = attention_masked(q[0, 0], k[0, 0], v[0, 0], mask)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=torch.from_numpy(mask)).numpy()
    assert np.max(np.abs(o - ref[0, 0])) <= 1e-12


def test_block_sparse_mask_expands_tiles():
    """Each (query tile, key tile) entry covers exactly its rectangle, ragged
    last tiles included; an all-true block mask is unmasked attention."""
    nq, nkv, br, bc = 10, 13, 4, 5
    bm = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 0]], dtype=bool)
    m = block_sparse_mask(bm, br, bc, nq, nkv)
    for i in range(nq):
        for j in range(nkv):
            assert m[i, j] == bm[i // br, j // bc]
    q, k, v = rnd(nq, 4), rnd(nkv, 4), rnd(nkv, 4)
    o, lse = attention_masked(q, k, v, block_sparse_mask(np.ones((3, 3), bool), br, bc, nq, nkv))
    o2, l2 = attention(q, k, v)
    assert np.max(np.abs(o - o2)) <= 1e-13 and np.max(np.abs(lse - l2)) <= 1e-13
    with pytest.raises(ValueError):
        attention_masked(q, k, v, block_sparse_mask(np.zeros((3, 3), bool), br, bc, nq, nkv))

