"""Pins for the fp64 oracle against facts that do not come from the oracle itself.

Each test checks the oracle against a closed form, an invariant of the
definition, an independent brute-force formulation, or a value the pages print.
The last test plants plausible mistakes in a copy of the oracle's C source (on
the CPU) and checks that every one of them is caught by at least one pin.
"""
import contextlib
import ctypes
import json
import math
import os
import subprocess
import tempfile
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle
from oracle import brute

GOLDEN = Path(__file__).parent / "golden"


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mask", ["none", "causal", "patch"])
def test_equal_logits_give_mean_of_allowed_v(mask):
    """Q = 0 makes every score 0: O_i = mean of the allowed V rows, LSE_i = ln(#allowed)."""
    lens_q, lens_k = [5, 3], [5, 7]
    Hq, Hkv, D = 4, 2, 6
    q = np.zeros((sum(lens_q), Hq, D))
    k = rnd((sum(lens_k), Hkv, D), 1)
    v = rnd((sum(lens_k), Hkv, D), 2)
    patch = None
    if mask == "patch":
        patch = np.array([[0, 2], [1, 4], [2, 3], [0, 5], [3, 5], [0, 7], [2, 6], [6, 7]], np.int32)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu(lens_q), cu_seqlens_k=cu(lens_k),
                                num_heads_kv=Hkv, scale=0.3,
                                mask={"none": 0, "causal": 1, "patch": 2}[mask],
                                patch_kv_range=patch)
    cq, ck = cu(lens_q), cu(lens_k)
    for b in range(2):
        Lq, Lk = lens_q[b], lens_k[b]
        for i in range(Lq):
            r = cq[b] + i
            if mask == "none":
                keys = list(range(Lk))
            elif mask == "causal":
                keys = list(range(0, i + (Lk - Lq) + 1))
            else:
                keys = list(range(patch[r, 0], patch[r, 1]))
            for h in range(Hq):
                g = h // (Hq // Hkv)
                want = v[ck[b] + np.array(keys), g].mean(axis=0)
                np.testing.assert_allclose(o[r, h], want, rtol=0, atol=1e-14)
                assert lse[h, r] == pytest.approx(math.log(len(keys)), abs=1e-14)


def test_identical_keys_give_mean_and_shifted_lse():
    """All K rows equal to c: s_ij = scale q_i.c for every j, so O = mean(V), LSE = s + ln(Lk)."""
    Lk, Hq, D = 6, 2, 5
    q = rnd((3, Hq, D), 3)
    c = rnd((D,), 4)
    k = np.broadcast_to(c, (Lk, 1, D)).copy()
    v = rnd((Lk, 1, D), 5)
    scale = 0.7
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([3]), cu_seqlens_k=cu([Lk]),
                                num_heads_kv=1, scale=scale, mask=0)
    for i in range(3):
        for h in range(Hq):
            s = scale * float(q[i, h] @ c)
            np.testing.assert_allclose(o[i, h], v[:, 0].mean(axis=0), atol=1e-14)
            assert lse[h, i] == pytest.approx(s + math.log(Lk), abs=1e-13)


def test_single_allowed_key_returns_that_v_row():
    """A length-1 patch, or causal row 0, leaves one key: O = v_j exactly, LSE = s_ij."""
    Hq, Hkv, D = 2, 1, 8
    k = rnd((6, Hkv, D), 6)
    v = rnd((6, Hkv, D), 7)
    q = rnd((3, Hq, D), 8)
    patch = np.array([[4, 5], [0, 1], [2, 3]], np.int32)
    scale = 0.25
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([3]), cu_seqlens_k=cu([6]),
                                num_heads_kv=Hkv, scale=scale, mask=2, patch_kv_range=patch)
    for i in range(3):
        j = patch[i, 0]
        for h in range(Hq):
            np.testing.assert_array_equal(o[i, h], v[j, 0])
            assert lse[h, i] == pytest.approx(scale * float(q[i, h] @ k[j, 0]), rel=1e-15, abs=1e-15)
    # causal row 0 (Lq == Lk) sees key 0 only
    o2, lse2 = oracle.attn_varlen(q, k[:3], v[:3], cu_seqlens_q=cu([3]), cu_seqlens_k=cu([3]),
                                  num_heads_kv=Hkv, scale=scale, mask=1)
    np.testing.assert_array_equal(o2[0, 0], v[0, 0])
    assert lse2[0, 0] == pytest.approx(scale * float(q[0, 0] @ k[0, 0]), rel=1e-15)


def test_dominant_logit_gives_one_hot():
    """One key whose score exceeds all others by >= 50: O equals its V row to 1e-12."""
    D, Lk = 4, 9
    k = rnd((Lk, 1, D), 9) * 0.1
    star = 5
    k[star, 0] = np.array([60.0, 0.0, 0.0, 0.0])
    q = np.zeros((1, 1, D))
    q[0, 0, 0] = 1.0
    v = rnd((Lk, 1, D), 10)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([1]), cu_seqlens_k=cu([Lk]),
                                num_heads_kv=1, scale=1.0, mask=0)
    np.testing.assert_allclose(o[0, 0], v[star, 0], atol=1e-12, rtol=0)
    assert lse[0, 0] == pytest.approx(60.0, abs=1e-12)


def test_common_score_shift_moves_lse_only():
    """Adding c to every score (an extra dim: q=c/scale, k=1) leaves O unchanged and adds c to LSE.

    With c = 1000 a softmax without max subtraction overflows, so this pins the
    max-subtracted form as well.
    """
    D, Lk, scale, c = 6, 7, 0.5, 1000.0
    q = rnd((4, 2, D), 11)
    k = rnd((Lk, 1, D), 12)
    v = rnd((Lk, 1, D), 13)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([4]), cu_seqlens_k=cu([Lk]),
                                num_heads_kv=1, scale=scale, mask=1)
    q2 = np.concatenate([q, np.full((4, 2, 1), c / scale)], axis=2)
    k2 = np.concatenate([k, np.ones((Lk, 1, 1))], axis=2)
    v2 = np.concatenate([v, np.zeros((Lk, 1, 1))], axis=2)
    o2, lse2 = oracle.attn_varlen(q2, k2, v2, cu_seqlens_q=cu([4]), cu_seqlens_k=cu([Lk]),
                                  num_heads_kv=1, scale=scale, mask=1)
    np.testing.assert_allclose(o2[..., :D], o, atol=1e-11)
    np.testing.assert_allclose(lse2, lse + c, atol=1e-9, rtol=0)


def test_rows_without_keys_are_zero_and_minus_inf():
    """ROWS_GUARANTEED_SAFE=False: seqused_k = 0 or an empty patch gives O = 0, LSE = -inf."""
    D = 4
    q = rnd((3, 2, D), 14)
    k = rnd((5, 1, D), 15)
    v = rnd((5, 1, D), 16)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([1, 2]), cu_seqlens_k=cu([2, 3]),
                                seqused_k=np.array([0, 3], np.int32), num_heads_kv=1,
                                scale=0.5, mask=0)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[:, 0]))
    assert np.all(np.isfinite(lse[:, 1:]))
    patch = np.array([[2, 2], [0, 1], [1, 1]], np.int32)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([3]), cu_seqlens_k=cu([5]),
                                num_heads_kv=1, scale=0.5, mask=2, patch_kv_range=patch)
    assert np.all(o[[0, 2]] == 0) and np.all(np.isneginf(lse[:, [0, 2]]))
    np.testing.assert_array_equal(o[1, 0], v[0, 0])


# ----------------------------------------------------------------------------
# invariants
# ----------------------------------------------------------------------------

def test_paging_with_permuted_block_table_matches_contiguous():
    """K/V scattered over a shuffled page pool via a permuted block table == contiguous K/V, bit for bit."""
    rng = np.random.default_rng(17)
    lens = [37, 16, 1, 50]
    bs, Hkv, Hq, D = 16, 2, 4, 8
    total = sum(lens)
    q = rng.standard_normal((len(lens), Hq, D))
    k = rng.standard_normal((total, Hkv, D))
    v = rng.standard_normal((total, Hkv, D))
    npages = [(L + bs - 1) // bs for L in lens]
    pool_pages = sum(npages) + 7
    perm = rng.permutation(pool_pages)
    kp = rng.standard_normal((pool_pages, bs, Hkv, D))   # garbage everywhere else
    vp = rng.standard_normal((pool_pages, bs, Hkv, D))
    bt = np.zeros((len(lens), max(npages)), np.int32)
    pos, ck = 0, cu(lens)
    for b, L in enumerate(lens):
        for p in range(npages[b]):
            page = perm[pos]
            pos += 1
            bt[b, p] = page
            n = min(bs, L - p * bs)
            kp[page, :n] = k[ck[b] + p * bs: ck[b] + p * bs + n]
            vp[page, :n] = v[ck[b] + p * bs: ck[b] + p * bs + n]
    cq = np.arange(len(lens) + 1, dtype=np.int32)
    o1, l1 = oracle.attn_varlen(q, k, v, cu_seqlens_q=cq, cu_seqlens_k=ck, num_heads_kv=Hkv,
                                scale=0.3, mask=0)
    o2, l2 = oracle.attn_varlen(q, kp, vp, cu_seqlens_q=cq, seqused_k=np.array(lens, np.int32),
                                block_table=bt, block_size=bs, num_heads_kv=Hkv, scale=0.3, mask=0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("mask", [0, 1])
def test_gqa_equals_repeated_kv_heads(mask):
    """Hq/Hkv grouping == explicit repeat_interleave of the KV heads with Hkv = Hq, bit for bit."""
    lens = [9, 4]
    Hq, Hkv, D = 6, 2, 8
    q = rnd((sum(lens), Hq, D), 18)
    k = rnd((sum(lens), Hkv, D), 19)
    v = rnd((sum(lens), Hkv, D), 20)
    c = cu(lens)
    o1, l1 = oracle.attn_varlen(q, k, v, cu_seqlens_q=c, cu_seqlens_k=c, num_heads_kv=Hkv,
                                scale=0.4, mask=mask)
    kr = np.repeat(k, Hq // Hkv, axis=1)
    vr = np.repeat(v, Hq // Hkv, axis=1)
    o2, l2 = oracle.attn_varlen(q, kr, vr, cu_seqlens_q=c, cu_seqlens_k=c, num_heads_kv=Hq,
                                scale=0.4, mask=mask)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_causal_row_equals_unmasked_prefix():
    """With Lq == Lk, causal row i equals unmasked attention of query i over keys 0..i."""
    L, D = 7, 5
    q = rnd((L, 1, D), 21)
    k = rnd((L, 1, D), 22)
    v = rnd((L, 1, D), 23)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([L]), cu_seqlens_k=cu([L]),
                                num_heads_kv=1, scale=0.5, mask=1)
    for i in range(L):
        oi, li = oracle.attn_varlen(q[i:i + 1], k[:i + 1], v[:i + 1], cu_seqlens_q=cu([1]),
                                    cu_seqlens_k=cu([i + 1]), num_heads_kv=1, scale=0.5, mask=0)
        np.testing.assert_allclose(o[i], oi[0], atol=1e-14)
        assert lse[0, i] == pytest.approx(li[0, 0], abs=1e-14)


def test_split_kv_combine_reproduces_unsplit():
    """Partials over disjoint key ranges merged by the combine rule == the unsplit result."""
    Lk, D, Hq = 23, 6, 3
    q = rnd((1, Hq, D), 24)
    k = rnd((Lk, 1, D), 25)
    v = rnd((Lk, 1, D), 26)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([1]), cu_seqlens_k=cu([Lk]),
                                num_heads_kv=1, scale=0.6, mask=0)
    bounds = [0, 5, 5, 16, 23]             # includes an empty split
    op, lp = [], []
    for s in range(len(bounds) - 1):
        a, b = bounds[s], bounds[s + 1]
        oo, ll = oracle.attn_varlen(q, k[a:b], v[a:b], cu_seqlens_q=cu([1]),
                                    cu_seqlens_k=cu([b - a]), num_heads_kv=1, scale=0.6, mask=0)
        op.append(oo[0])
        lp.append(ll[:, 0])
    oc, lc = oracle.combine(np.stack(op), np.stack(lp))
    np.testing.assert_allclose(oc, o[0], atol=1e-14)
    np.testing.assert_allclose(lc, lse[:, 0], atol=1e-14)
    # every split empty -> O = 0, LSE = -inf
    oc, lc = oracle.combine(np.zeros((2, 1, D)), np.full((2, 1), -np.inf))
    assert np.all(oc == 0) and np.isneginf(lc[0])


# ----------------------------------------------------------------------------
# sliding window and softcap (the "local window on/off, softcap 0/50" options)
# ----------------------------------------------------------------------------

def test_window_zero_keeps_only_the_diagonal_key():
    """W = 0: row i sees only key i' = i + Lk - Lq, so O = v_i' exactly and LSE = s_ii'."""
    Lq, Lk, D = 5, 9, 4
    q, k, v = rnd((Lq, 2, D), 41), rnd((Lk, 1, D), 42), rnd((Lk, 1, D), 43)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([Lq]), cu_seqlens_k=cu([Lk]),
                                num_heads_kv=1, scale=0.4, mask=1, window_left=0)
    for i in range(Lq):
        d = i + Lk - Lq
        for h in range(2):
            np.testing.assert_array_equal(o[i, h], v[d, 0])
            assert lse[h, i] == pytest.approx(0.4 * float(np.dot(q[i, h], k[d, 0])), abs=1e-14)


@pytest.mark.parametrize("W", [1, 3, 6])
def test_window_equals_unmasked_attention_over_the_sliced_keys(W):
    """Row i with window W == unmasked attention of query i over keys max(0, i'-W) .. i'."""
    Lq, Lk, D = 6, 10, 5
    q, k, v = rnd((Lq, 1, D), 44), rnd((Lk, 1, D), 45), rnd((Lk, 1, D), 46)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([Lq]), cu_seqlens_k=cu([Lk]),
                                num_heads_kv=1, scale=0.5, mask=1, window_left=W)
    for i in range(Lq):
        d = i + Lk - Lq
        a = max(0, d - W)
        oi, li = oracle.attn_varlen(q[i:i + 1], k[a:d + 1], v[a:d + 1], cu_seqlens_q=cu([1]),
                                    cu_seqlens_k=cu([d + 1 - a]), num_heads_kv=1, scale=0.5,
                                    mask=0)
        np.testing.assert_allclose(o[i], oi[0], atol=1e-14, rtol=0)
        assert lse[0, i] == pytest.approx(li[0, 0], abs=1e-14)


def test_window_at_least_the_length_is_plain_causal():
    L, D = 7, 3
    q, k, v = rnd((L, 2, D), 47), rnd((L, 1, D), 48), rnd((L, 1, D), 49)
    kw = dict(cu_seqlens_q=cu([L]), cu_seqlens_k=cu([L]), num_heads_kv=1, scale=0.7, mask=1)
    o0, l0 = oracle.attn_varlen(q, k, v, **kw)
    o1, l1 = oracle.attn_varlen(q, k, v, window_left=L, **kw)
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(l0, l1)


def test_softcap_closed_form_two_keys():
    """Scaled scores c*atanh(1/2) and 0 become c/2 and 0 (tanh(ln(3)/2) = 1/2), so
    O = (e^(c/2) v1 + v2) / (e^(c/2) + 1) and LSE = ln(e^(c/2) + 1)."""
    c, scale = 3.0, 0.25
    q = np.ones((1, 1, 1))
    k = np.array([[[c * math.log(3.0) / 2 / scale]], [[0.0]]])
    v = np.array([[[2.0]], [[-5.0]]])
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([1]), cu_seqlens_k=cu([2]),
                                num_heads_kv=1, scale=scale, softcap=c)
    e = math.exp(c / 2)
    assert o[0, 0, 0] == pytest.approx((e * 2.0 - 5.0) / (e + 1), abs=1e-13)
    assert lse[0, 0] == pytest.approx(math.log(e + 1), abs=1e-13)


def test_softcap_limits():
    """A cap far below every score flattens the weights (O = mean of the allowed V,
    LSE = ln n); a cap far above them leaves the plain result."""
    L, D = 6, 4
    q, k, v = rnd((L, 1, D), 50) * 3, rnd((L, 1, D), 51) * 3, rnd((L, 1, D), 52)
    kw = dict(cu_seqlens_q=cu([L]), cu_seqlens_k=cu([L]), num_heads_kv=1, scale=0.9, mask=1)
    o, lse = oracle.attn_varlen(q, k, v, softcap=1e-9, **kw)
    for i in range(L):
        np.testing.assert_allclose(o[i, 0], v[:i + 1, 0].mean(axis=0), atol=1e-8, rtol=0)
        assert lse[0, i] == pytest.approx(math.log(i + 1), abs=1e-8)
    o0, l0 = oracle.attn_varlen(q, k, v, **kw)
    o1, l1 = oracle.attn_varlen(q, k, v, softcap=1e9, **kw)   # |s - c tanh(s/c)| <= |s|^3/(3c^2)
    np.testing.assert_allclose(o1, o0, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l1, l0, atol=1e-12, rtol=0)


def test_softcap_bounds_the_lse():
    """Capped logits lie in (-c, c), so ln n - c < LSE < ln n + c even for huge scores."""
    L, D, c = 9, 4, 2.0
    q, k, v = rnd((L, 1, D), 53), rnd((L, 1, D), 54), rnd((L, 1, D), 55)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([L]), cu_seqlens_k=cu([L]),
                                num_heads_kv=1, scale=1e3, mask=0, softcap=c)
    assert np.all(lse > math.log(L) - c) and np.all(lse < math.log(L) + c)
    assert np.all(np.isfinite(o))


def test_window_and_softcap_rejected_where_undefined():
    q = rnd((2, 1, 2), 56)
    with pytest.raises(ValueError):
        oracle.attn_varlen(q, q, q, cu_seqlens_q=cu([2]), cu_seqlens_k=cu([2]), num_heads_kv=1,
                           scale=1.0, mask=0, window_left=1)
    with pytest.raises(ValueError):
        oracle.attn_varlen(q, q, q, cu_seqlens_q=cu([2]), cu_seqlens_k=cu([2]), num_heads_kv=1,
                           scale=1.0, mask=1, softcap=-1.0)


# ----------------------------------------------------------------------------
# an independent implementation on tiny inputs
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("window,softcap", [(0, 0.0), (2, 0.0), (-1, 1.5), (3, 0.8)])
def test_brute_force_agrees_with_window_and_softcap(window, softcap, seed):
    rng = np.random.default_rng(200 + seed)
    Hq, Hkv, D = 2, 1, 3
    lens_q = [int(x) for x in rng.integers(1, 9, size=2)]
    lens_k = [max(lq, int(x)) for lq, x in zip(lens_q, rng.integers(1, 9, size=2))]
    cq, ck = cu(lens_q), cu(lens_k)
    q = rng.standard_normal((cq[-1], Hq, D)) * 2
    k = rng.standard_normal((ck[-1], Hkv, D)) * 2
    v = rng.standard_normal((ck[-1], Hkv, D))
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cq, cu_seqlens_k=ck, num_heads_kv=Hkv,
                                scale=0.6, mask=1, window_left=window, softcap=softcap)
    for b in range(2):
        ob, lb = brute.attention(q[cq[b]:cq[b + 1]].tolist(), k[ck[b]:ck[b + 1]].tolist(),
                                 v[ck[b]:ck[b + 1]].tolist(), 0.6, "causal", None, window,
                                 softcap)
        np.testing.assert_allclose(o[cq[b]:cq[b + 1]], np.array(ob), atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[:, cq[b]:cq[b + 1]], np.array(lb), atol=1e-12, rtol=0)


@pytest.mark.parametrize("mask", ["none", "causal", "patch"])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_enumeration_agrees(mask, seed):
    rng = np.random.default_rng(100 + seed)
    Hq, Hkv, D = 4, 2, 3
    lens_q = [int(x) for x in rng.integers(1, 9, size=2)]
    lens_k = [max(lq, int(x)) for lq, x in zip(lens_q, rng.integers(1, 9, size=2))]
    cq, ck = cu(lens_q), cu(lens_k)
    q = rng.standard_normal((cq[-1], Hq, D))
    k = rng.standard_normal((ck[-1], Hkv, D))
    v = rng.standard_normal((ck[-1], Hkv, D))
    patch = None
    if mask == "patch":
        patch = np.zeros((cq[-1], 2), np.int32)
        for b in range(2):
            for i in range(lens_q[b]):
                a = int(rng.integers(0, lens_k[b] + 1))
                patch[cq[b] + i] = (a, int(rng.integers(a, lens_k[b] + 1)))
    scale = 0.45
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cq, cu_seqlens_k=ck, num_heads_kv=Hkv,
                                scale=scale, mask={"none": 0, "causal": 1, "patch": 2}[mask],
                                patch_kv_range=patch)
    for b in range(2):
        qs = q[cq[b]:cq[b + 1]].tolist()
        ks = k[ck[b]:ck[b + 1]].tolist()
        vs = v[ck[b]:ck[b + 1]].tolist()
        pb = patch[cq[b]:cq[b + 1]].tolist() if patch is not None else None
        ob, lb = brute.attention(qs, ks, vs, scale, mask, pb)
        np.testing.assert_allclose(o[cq[b]:cq[b + 1]], np.array(ob), atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[:, cq[b]:cq[b + 1]], np.array(lb), atol=1e-12, rtol=0)


# ----------------------------------------------------------------------------
# values the pages print
# ----------------------------------------------------------------------------

def test_golden_default_scale_for_e256():
    """The BLT FlexAttention call on [2,1,128,256] tensors lowers with scale 0.0625 = 1/sqrt(256)."""
    g = json.loads((GOLDEN / "default_scale_e256.json").read_text())
    assert oracle.default_scale(g["head_dim"]) == g["scale"]
    B, H, L, E = g["shape_bhle"]
    q = rnd((B * 4, H, E), 27) * 0.1       # a short slice of the [2,1,128,256] shape
    k = rnd((B * 4, H, E), 28) * 0.1
    v = rnd((B * 4, H, E), 29)
    c = np.arange(B + 1, dtype=np.int32) * 4
    o1, l1 = oracle.attn_varlen(q, k, v, cu_seqlens_q=c, cu_seqlens_k=c, num_heads_kv=H,
                                scale=None, mask=0)
    o2, l2 = oracle.attn_varlen(q, k, v, cu_seqlens_q=c, cu_seqlens_k=c, num_heads_kv=H,
                                scale=g["scale"], mask=0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_golden_causal_predicate_4x4():
    """Causal rows see exactly the keys of the page's q_idx >= kv_idx grid (via Q = 0: LSE = ln #keys)."""
    g = json.loads((GOLDEN / "causal_mask_4x4.json").read_text())
    allowed = np.array(g["allowed"])
    L = g["q_len"]
    v = np.eye(L).reshape(L, 1, L)          # V row j = e_j: O_i reveals which keys were averaged
    q = np.zeros((L, 1, L))
    k = rnd((L, 1, L), 30)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu([L]), cu_seqlens_k=cu([g["kv_len"]]),
                                num_heads_kv=1, scale=1.0, mask=1)
    for i in range(L):
        n = allowed[i].sum()
        np.testing.assert_allclose(o[i, 0], allowed[i] / n, atol=1e-15)
        assert lse[0, i] == pytest.approx(math.log(n), abs=1e-15)


def test_dense_wrapper_layouts():
    """Dense [B,L,H,D] wrapper: O [B,L,H,D], LSE [B,H,L] match per-batch varlen calls."""
    B, L, H, D = 2, 5, 2, 4
    q, k, v = rnd((B, L, H, D), 31), rnd((B, L, H, D), 32), rnd((B, L, H, D), 33)
    o, lse = oracle.attn_dense(q, k, v, scale=0.5, causal=True)
    assert o.shape == (B, L, H, D) and lse.shape == (B, H, L)
    for b in range(B):
        ob, lb = oracle.attn_varlen(q[b], k[b], v[b], cu_seqlens_q=cu([L]), cu_seqlens_k=cu([L]),
                                    num_heads_kv=H, scale=0.5, mask=1)
        np.testing.assert_array_equal(o[b], ob)
        np.testing.assert_array_equal(lse[b], lb)


def test_decode_wrapper_matches_varlen():
    from attention_paged_kv_gqa_b200 import workloads
    w = workloads.paged_decode(B=3, Hq=4, Hkv=2, D=8, num_blocks=64, lmin=1, lmax=100, seed=5)
    t = w.tensors
    o, lse = oracle.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                t["seqused_k"], scale=0.3)
    assert o.shape == (3, 4, 8) and lse.shape == (3, 4)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))


# ----------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin above
# ----------------------------------------------------------------------------

MUTATIONS = {
    "gqa_head_index": ("const int g = h / group;", "const int g = h % Hkv;"),
    "causal_off_by_one": ("return j <= i + (Lk - Lq);", "return j < i + (Lk - Lq);"),
    "causal_top_left": ("return j <= i + (Lk - Lq);", "return j <= i;"),
    "no_max_subtraction": ("const double p = exp(s[j] - M);", "const double p = exp(s[j]);"),
    "no_normalisation": ("for (int d = 0; d < D; ++d) oi[d] /= Z;", ""),
    "scale_dropped": ("s[j] = scale * acc;", "s[j] = acc;"),
    "lse_without_max": ("*lse_i = M + log(Z);", "*lse_i = log(Z);"),
    "page_row_index": ("row = (long long)page * block_size + (j % block_size);",
                       "row = (long long)page * block_size + (j / block_size);"),
    "v_read_from_k": ("const double *vj = kv_row(v,", "const double *vj = kv_row(k,"),
    "patch_end_inclusive": ("return range_i[0] <= j && j < range_i[1];",
                            "return range_i[0] <= j && j <= range_i[1];"),
    "combine_weight": ("const double w = exp(lse_parts[(long long)s * N + n] - lse[n]);",
                       "const double w = exp(lse_parts[(long long)s * N + n] - M);"),
    "window_off_by_one": ("if (window_left >= 0 && j < i + (Lk - Lq) - window_left) return 0;",
                          "if (window_left >= 0 && j <= i + (Lk - Lq) - window_left) return 0;"),
    "window_ignored": ("if (window_left >= 0 && j < i + (Lk - Lq) - window_left) return 0;", ""),
    "window_top_left": ("if (window_left >= 0 && j < i + (Lk - Lq) - window_left) return 0;",
                        "if (window_left >= 0 && j < i - window_left) return 0;"),
    "softcap_ignored": ("if (softcap > 0.0) s[j] = softcap * tanh(s[j] / softcap);", ""),
    "softcap_no_outer_factor": ("if (softcap > 0.0) s[j] = softcap * tanh(s[j] / softcap);",
                                "if (softcap > 0.0) s[j] = tanh(s[j] / softcap);"),
    "softcap_no_inner_division": ("if (softcap > 0.0) s[j] = softcap * tanh(s[j] / softcap);",
                                  "if (softcap > 0.0) s[j] = softcap * tanh(s[j]);"),
    "softcap_before_scale": ("if (softcap > 0.0) s[j] = softcap * tanh(s[j] / softcap);",
                             "if (softcap > 0.0) s[j] = scale * softcap * tanh(acc / softcap);"),
}

PINS = [
    lambda: [test_equal_logits_give_mean_of_allowed_v(m) for m in ("none", "causal", "patch")],
    test_identical_keys_give_mean_and_shifted_lse,
    test_single_allowed_key_returns_that_v_row,
    test_dominant_logit_gives_one_hot,
    test_common_score_shift_moves_lse_only,
    test_rows_without_keys_are_zero_and_minus_inf,
    test_paging_with_permuted_block_table_matches_contiguous,
    lambda: [test_gqa_equals_repeated_kv_heads(m) for m in (0, 1)],
    test_causal_row_equals_unmasked_prefix,
    test_split_kv_combine_reproduces_unsplit,
    lambda: [test_brute_force_enumeration_agrees(m, s) for m in ("none", "causal", "patch")
             for s in (0, 1, 2)],
    test_golden_causal_predicate_4x4,
    test_window_zero_keeps_only_the_diagonal_key,
    lambda: [test_window_equals_unmasked_attention_over_the_sliced_keys(w) for w in (1, 3, 6)],
    test_window_at_least_the_length_is_plain_causal,
    test_softcap_closed_form_two_keys,
    test_softcap_limits,
    test_softcap_bounds_the_lse,
    lambda: [test_brute_force_agrees_with_window_and_softcap(w, c, s)
             for w, c in ((0, 0.0), (2, 0.0), (-1, 1.5), (3, 0.8)) for s in (0, 1, 2)],
]


@contextlib.contextmanager
def _mutated_oracle(src_text):
    with tempfile.TemporaryDirectory() as d:
        c = Path(d) / "m.c"
        so = Path(d) / "m.so"
        c.write_text(src_text)
        subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", str(c),
                        "-o", str(so), "-lm"], check=True)
        saved = oracle._lib
        lib = oracle.bind(ctypes.CDLL(str(so)))
        try:
            oracle._lib = lib
            yield
        finally:
            oracle._lib = saved


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    src = (Path(oracle.__file__).parent / "attn_oracle.c").read_text()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    with _mutated_oracle(src.replace(old, new)):
        caught = 0
        for pin in PINS:
            try:
                with np.errstate(all="ignore"):
                    pin()
            except (AssertionError, ValueError, FloatingPointError):
                caught += 1
        assert caught >= 1, "no pin caught the planted mistake " + name
