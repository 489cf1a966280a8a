"""Pins for the oracle's extra Qv score term (CPU).

The term comes from "Rope dim" (vllm-project flash-attention PR 172,
overview): a Qv GEMM adds qv . v to the score, and only_qv keeps that term
alone.  Pins that do not come from the oracle's own code:
  * the general score equals torch's scaled_dot_product_attention (fp64, CPU)
    run on the head-dimension concatenation [q | qv] . [k | v]^T with the
    values v (a library routine, with the causal mask given as numpy's tril);
  * qv = 0 reduces to the plain forward (pinned on its own elsewhere);
  * only_qv equals the plain forward with q := qv and k := v;
  * a planted mistake in a copy of the oracle's source fails one of them.
"""
import contextlib
import ctypes
import subprocess
import tempfile
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle


def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def _data(lens_q, lens_k, Hq, Hkv, D, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((sum(lens_q), Hq, D))
    qv = rng.standard_normal((sum(lens_q), Hq, D))
    k = rng.standard_normal((sum(lens_k), Hkv, D))
    v = rng.standard_normal((sum(lens_k), Hkv, D))
    return q, qv, k, v


def _sdpa_concat(q, qv, k, v, lens_q, lens_k, Hq, Hkv, scale, causal, only_qv):
    """torch SDPA per sequence on [q|qv], [k|v] (GQA by repeating KV heads)."""
    cq, ck = _cu(lens_q), _cu(lens_k)
    out = np.zeros_like(qv)
    lse = np.full((Hq, sum(lens_q)), -np.inf)
    for b in range(len(lens_q)):
        Lq, Lk = lens_q[b], lens_k[b]
        if Lq == 0:
            continue
        qq = qv[cq[b]:cq[b + 1]] if only_qv else np.concatenate([q[cq[b]:cq[b + 1]], qv[cq[b]:cq[b + 1]]], -1)
        kk = v[ck[b]:ck[b + 1]] if only_qv else np.concatenate([k[ck[b]:ck[b + 1]], v[ck[b]:ck[b + 1]]], -1)
        vv = v[ck[b]:ck[b + 1]]
        rep = Hq // Hkv
        Q = torch.from_numpy(qq).permute(1, 0, 2)
        K = torch.from_numpy(np.repeat(kk, rep, axis=1)).permute(1, 0, 2)
        V = torch.from_numpy(np.repeat(vv, rep, axis=1)).permute(1, 0, 2)
        m = None
        if causal:
            m = torch.from_numpy(np.tril(np.ones((Lq, Lk), dtype=bool), k=Lk - Lq))
        O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=m, scale=scale)
        out[cq[b]:cq[b + 1]] = O.permute(1, 0, 2).numpy()
        # LSE from torch's own logsumexp over the masked, scaled concatenated scores
        S = torch.einsum("hqd,hkd->hqk", Q, K) * scale
        if m is not None:
            S = S.masked_fill(~m, float("-inf"))
        lse[:, cq[b]:cq[b + 1]] = torch.logsumexp(S, dim=-1).numpy()
    return out, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("only_qv", [False, True])
def test_matches_sdpa_on_concatenated_head_dims(causal, only_qv):
    lens_q, lens_k = [5, 1, 7], [9, 4, 7]
    Hq, Hkv, D, scale = 4, 2, 6, 0.37
    q, qv, k, v = _data(lens_q, lens_k, Hq, Hkv, D, seed=3 + causal + 2 * only_qv)
    o, lse = oracle.attn_varlen_qv(q, qv, k, v, cu_seqlens_q=_cu(lens_q), cu_seqlens_k=_cu(lens_k),
                                   num_heads_kv=Hkv, scale=scale, mask=int(causal), only_qv=only_qv)
    o_ref, lse_ref = _sdpa_concat(q, qv, k, v, lens_q, lens_k, Hq, Hkv, scale, causal, only_qv)
    np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=0)


def _to_pages(x, lens, bs, num_blocks, seed):
    rng = np.random.default_rng(seed)
    mbps = max(1, max((n + bs - 1) // bs for n in lens))
    perm = rng.permutation(num_blocks)[:len(lens) * mbps].reshape(len(lens), mbps).astype(np.int32)
    store = rng.standard_normal((num_blocks, bs) + x.shape[1:])
    cu = _cu(lens)
    for b, n in enumerate(lens):
        for t in range(n):
            store[perm[b, t // bs], t % bs] = x[cu[b] + t]
    return store, perm


@pytest.mark.parametrize("only_qv", [False, True])
@pytest.mark.parametrize("mods", ["paged_window_softcap", "patch"])
def test_concatenated_head_dims_through_the_plain_forward(only_qv, mods):
    """[q|qv].[k|v]^T with values [v|0] through the (separately pinned) plain forward:
    the first D columns of its O and its LSE are the Qv forward's, for every mask,
    window, softcap and the paged store."""
    lens_q, lens_k = [7, 3, 12], [19, 3, 12]
    Hq, Hkv, D, scale, bs = 4, 2, 5, 0.45, 4
    q, qv, k, v = _data(lens_q, lens_k, Hq, Hkv, D, seed=31 + only_qv)
    cq, ck = _cu(lens_q), _cu(lens_k)
    qq = qv if only_qv else np.concatenate([q, qv], -1)
    kk = v if only_qv else np.concatenate([k, v], -1)
    vv = v if only_qv else np.concatenate([v, np.zeros_like(v)], -1)
    kw = dict(num_heads_kv=Hkv, scale=scale)
    if mods == "patch":
        rng = np.random.default_rng(5)
        pr = np.zeros((sum(lens_q), 2), np.int32)
        for b in range(3):
            for i in range(lens_q[b]):
                s0 = int(rng.integers(0, lens_k[b]))
                pr[cq[b] + i] = (s0, int(rng.integers(s0, lens_k[b] + 1)))
        kw.update(mask=2, patch_kv_range=pr)
        got = oracle.attn_varlen_qv(q, qv, k, v, cu_seqlens_q=cq, cu_seqlens_k=ck, only_qv=only_qv, **kw)
        ref = oracle.attn_varlen(qq, kk, vv, cu_seqlens_q=cq, cu_seqlens_k=ck, **kw)
    else:
        kw.update(mask=1, window_left=4, softcap=1.7)
        su = np.array(lens_k, np.int32)
        ks, bt = _to_pages(k, lens_k, bs, 24, 1)
        vs, _ = _to_pages(v, lens_k, bs, 24, 1)
        kks, _ = _to_pages(kk, lens_k, bs, 24, 1)
        vvs, _ = _to_pages(vv, lens_k, bs, 24, 1)
        got = oracle.attn_varlen_qv(q, qv, ks, vs, cu_seqlens_q=cq, block_table=bt, seqused_k=su,
                                    only_qv=only_qv, **kw)
        ref = oracle.attn_varlen(qq, kks, vvs, cu_seqlens_q=cq, block_table=bt, block_size=bs,
                                 seqused_k=su, **kw)
    np.testing.assert_allclose(got[0], ref[0][..., :D], atol=1e-13, rtol=0)
    np.testing.assert_allclose(got[1], ref[1], atol=1e-13, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_qv_is_the_plain_forward(causal):
    lens = [6, 3, 11]
    q, qv, k, v = _data(lens, lens, 4, 1, 5, seed=21)
    cu = _cu(lens)
    o, lse = oracle.attn_varlen_qv(q, np.zeros_like(qv), k, v, cu_seqlens_q=cu, cu_seqlens_k=cu,
                                   num_heads_kv=1, scale=0.5, mask=int(causal))
    o_ref, lse_ref = oracle.attn_varlen(q, k, v, cu_seqlens_q=cu, cu_seqlens_k=cu, num_heads_kv=1,
                                        scale=0.5, mask=int(causal))
    np.testing.assert_allclose(o, o_ref, atol=1e-13, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-13, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_only_qv_is_the_plain_forward_with_keys_equal_to_values(causal):
    lens_q, lens_k = [4, 9], [10, 9]
    q, qv, k, v = _data(lens_q, lens_k, 6, 2, 4, seed=22)
    cq, ck = _cu(lens_q), _cu(lens_k)
    o, lse = oracle.attn_varlen_qv(None, qv, None, v, cu_seqlens_q=cq, cu_seqlens_k=ck, num_heads_kv=2,
                                   scale=0.8, mask=int(causal), only_qv=True)
    o_ref, lse_ref = oracle.attn_varlen(qv, v, v, cu_seqlens_q=cq, cu_seqlens_k=ck, num_heads_kv=2,
                                        scale=0.8, mask=int(causal))
    np.testing.assert_allclose(o, o_ref, atol=1e-13, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-13, rtol=0)


def test_empty_rows_and_sequences():
    """A query with no allowed key (causal, Lk = 0) gives O = 0 and LSE = -inf."""
    q, qv, k, v = _data([3, 2], [0, 2], 2, 1, 4, seed=23)
    o, lse = oracle.attn_varlen_qv(q, qv, k, v, cu_seqlens_q=_cu([3, 2]), cu_seqlens_k=_cu([0, 2]),
                                   num_heads_kv=1, scale=1.0, mask=1)
    assert np.all(o[:3] == 0) and np.all(np.isneginf(lse[:, :3]))
    assert np.all(np.isfinite(lse[:, 3:]))


PINS = [lambda: [test_matches_sdpa_on_concatenated_head_dims(c, oq) for c in (False, True) for oq in (False, True)],
        lambda: [test_concatenated_head_dims_through_the_plain_forward(oq, m) for oq in (False, True)
                 for m in ("paged_window_softcap", "patch")],
        lambda: [test_zero_qv_is_the_plain_forward(c) for c in (False, True)],
        lambda: [test_only_qv_is_the_plain_forward_with_keys_equal_to_values(c) for c in (False, True)]]

_VROW = ("const double *v_j = kv_row(v, b, j, g, Hkv, D, block_table, max_blocks_per_seq,\n"
         "                                          block_size, cu_seqlens_k);\n"
         "                double qk = 0.0, qvv = 0.0;")
MUTATIONS = {
    "qk_term_dropped": ("srow[j] = scale * (qk + qvv);", "srow[j] = scale * qvv;"),
    "qv_term_dropped": ("srow[j] = scale * (qk + qvv);", "srow[j] = scale * qk;"),
    "qv_term_unscaled": ("srow[j] = scale * (qk + qvv);", "srow[j] = scale * qk + qvv;"),
    "query_in_place_of_qv": ("qvv += qvi[d] * v_j[d];", "qvv += (only_qv ? qvi : qi)[d] * v_j[d];"),
    "qv_against_the_wrong_kv_head": (_VROW, _VROW.replace("kv_row(v, b, j, g,", "kv_row(v, b, j, h % Hkv,")),
    "softcap_skipped": ("if (softcap > 0.0) srow[j] = softcap * tanh(srow[j] / softcap);", ""),
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
