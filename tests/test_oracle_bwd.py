"""Pins for the fp64 backward oracle (CPU).

The gradients are checked against facts that do not come from the backward
code itself: central finite differences of the (separately pinned) forward
oracle, two translation invariances of unmasked attention (adding a vector
to every key leaves O unchanged, adding one to every value shifts O by it),
the grouped-query identity (a KV head's gradient is the sum over its query
heads), and the single-key case.  The last test plants mistakes in a copy of
the oracle's C source and checks that each is caught.
"""
import contextlib
import ctypes
import subprocess
import tempfile
from pathlib import Path

import numpy as np
import pytest

import oracle


def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def _data(lens_q, lens_k, Hq, Hkv, D, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((sum(lens_q), Hq, D))
    k = rng.standard_normal((sum(lens_k), Hkv, D))
    v = rng.standard_normal((sum(lens_k), Hkv, D))
    do = rng.standard_normal((sum(lens_q), Hq, D))
    return q, k, v, do


def _loss(q, k, v, do, cq, ck, Hkv, scale, mask, window):
    o, _ = oracle.attn_varlen(q, k, v, cu_seqlens_q=cq, cu_seqlens_k=ck, num_heads_kv=Hkv,
                              scale=scale, mask=mask, window_left=window, nthreads=1)
    return float(np.sum(do * o))


@pytest.mark.parametrize("mask,window", [(0, -1), (1, -1), (1, 2)])
def test_gradients_match_finite_differences(mask, window):
    """d/dx sum(dO * O(q, k, v)) by central differences (h = 1e-5) on tiny inputs."""
    lens_q, lens_k = [5, 3], [5, 4]
    Hq, Hkv, D, scale = 2, 1, 3, 0.7
    q, k, v, do = _data(lens_q, lens_k, Hq, Hkv, D, seed=mask * 10 + window + 1)
    cq, ck = _cu(lens_q), _cu(lens_k)
    dq, dk, dv = oracle.attn_bwd_varlen(q, k, v, do, cu_seqlens_q=cq, cu_seqlens_k=ck,
                                        num_heads_kv=Hkv, scale=scale, mask=mask,
                                        window_left=window, nthreads=1)
    h = 1e-5
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            saved = x[idx]
            x[idx] = saved + h
            lp = _loss(q, k, v, do, cq, ck, Hkv, scale, mask, window)
            x[idx] = saved - h
            lm = _loss(q, k, v, do, cq, ck, Hkv, scale, mask, window)
            x[idx] = saved
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, num, atol=2e-8, rtol=0)


def test_translation_invariances_unmasked():
    """No mask: k_j + c for all j leaves O unchanged, so sum_j dK_j = 0; v_j + c for all
    j adds c to O, so sum_j dV_j = sum over the group's query rows of dO."""
    lens = [6, 4]
    Hq, Hkv, D = 4, 2, 5
    q, k, v, do = _data(lens, lens, Hq, Hkv, D, seed=9)
    cq = _cu(lens)
    dq, dk, dv = oracle.attn_bwd_varlen(q, k, v, do, cu_seqlens_q=cq, cu_seqlens_k=cq,
                                        num_heads_kv=Hkv, scale=0.4, mask=0)
    for b in range(2):
        sl = slice(cq[b], cq[b + 1])
        for g in range(Hkv):
            np.testing.assert_allclose(dk[sl, g].sum(axis=0), 0.0, atol=1e-13)
            want = do[sl, 2 * g:2 * g + 2].sum(axis=(0, 1))
            np.testing.assert_allclose(dv[sl, g].sum(axis=0), want, atol=1e-13)


@pytest.mark.parametrize("mask", [0, 1])
def test_gqa_gradient_is_the_sum_over_the_group(mask):
    lens = [7, 3]
    Hq, Hkv, D = 4, 2, 3
    q, k, v, do = _data(lens, lens, Hq, Hkv, D, seed=11)
    cq = _cu(lens)
    dq, dk, dv = oracle.attn_bwd_varlen(q, k, v, do, cu_seqlens_q=cq, cu_seqlens_k=cq,
                                        num_heads_kv=Hkv, scale=0.5, mask=mask)
    kr, vr = np.repeat(k, Hq // Hkv, axis=1), np.repeat(v, Hq // Hkv, axis=1)
    dq_r, dk_r, dv_r = oracle.attn_bwd_varlen(q, kr, vr, do, cu_seqlens_q=cq, cu_seqlens_k=cq,
                                              num_heads_kv=Hq, scale=0.5, mask=mask)
    np.testing.assert_allclose(dq, dq_r, atol=1e-14)
    np.testing.assert_allclose(dk, dk_r.reshape(-1, Hkv, 2, D).sum(axis=2), atol=1e-14)
    np.testing.assert_allclose(dv, dv_r.reshape(-1, Hkv, 2, D).sum(axis=2), atol=1e-14)


def test_single_key():
    """One key: O = v for every row, so dQ = dK = 0 and dV = the sum of dO."""
    q, k, v, do = _data([4], [1], 2, 1, 3, seed=12)
    dq, dk, dv = oracle.attn_bwd_varlen(q, k, v, do, cu_seqlens_q=_cu([4]), cu_seqlens_k=_cu([1]),
                                        num_heads_kv=1, scale=0.8, mask=0)
    assert np.all(dq == 0) and np.allclose(dk, 0, atol=1e-15)
    np.testing.assert_allclose(dv[0, 0], do.sum(axis=(0, 1)), atol=1e-14)


PINS = [lambda: [test_gradients_match_finite_differences(m, w) for m, w in ((0, -1), (1, -1), (1, 2))],
        test_translation_invariances_unmasked,
        lambda: [test_gqa_gradient_is_the_sum_over_the_group(m) for m in (0, 1)],
        test_single_key]

MUTATIONS = {
    "dq_without_scale": ("dqi[d] += scale * ds * kj[d];", "dqi[d] += ds * kj[d];"),
    "dk_without_scale": ("dkj[d] += scale * ds * qi[d];", "dkj[d] += ds * qi[d];"),
    "ds_without_delta": ("const double ds = p[j] * (dp[j] - delta);", "const double ds = p[j] * dp[j];"),
    "dv_from_dp": ("dvj[d] += p[j] * doi[d];", "dvj[d] += dp[j] * doi[d];"),
    "delta_unweighted": ("delta += p[j] * dp[j];", "delta += dp[j];"),
    "unnormalised_p": ("const double lse = M + log(Z);", "const double lse = M;"),
    "dk_from_dq_row": ("dkj[d] += scale * ds * qi[d];", "dkj[d] += scale * ds * doi[d];"),
    "scores_without_scale": ("s[j] = acc * scale;", "s[j] = acc;"),
}


@contextlib.contextmanager
def _mutated(src_text):
    with tempfile.TemporaryDirectory() as d:
        c, so = Path(d) / "m.c", Path(d) / "m.so"
        c.write_text(src_text)
        subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", str(c), "-o",
                        str(so), "-lm"], check=True)
        saved = oracle._lib
        try:
            oracle._lib = oracle.bind(ctypes.CDLL(str(so)))
            yield
        finally:
            oracle._lib = saved


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    src = (Path(oracle.__file__).parent / "attn_oracle.c").read_text()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    with _mutated(src.replace(old, new)):
        caught = 0
        for pin in PINS:
            try:
                with np.errstate(all="ignore"):
                    pin()
            except (AssertionError, ValueError, FloatingPointError):
                caught += 1
        assert caught >= 1, "no pin caught the planted mistake " + name
