"""Brute-force attention in pure Python scalars (test infrastructure only).

A second formulation, independent of ``attn_oracle.c``: for tiny inputs it
enumerates every (query, key) pair, applies the mask predicate by index, and
forms the softmax directly as exp(s_ij) / sum_j exp(s_ij) with ``math.fsum``
(no max subtraction, so keep |scores| small), with
LSE_i = ln(fsum_j exp(s_ij)).  Keys are read from per-sequence contiguous
lists; paging and head grouping are expressed here as plain Python indexing.

Definition followed: the FlexAttention forward with log-sum-exp output
("[FlexAttention] Enforce Q,K,V memory layouts for fp8 flex attention",
flex_attention docstring; "Cross Attention does not work on CPU and older
GPUs", OUTPUT_LOGSUMEXP), GQA as in the docstring's (B,Hq,L,E)/(B,Hkv,S,E)
shapes with query head h reading KV head h // (Hq/Hkv).
"""
from __future__ import annotations

import math


def _allowed(mask: str, i: int, j: int, Lq: int, Lk: int, rng, window) -> bool:
    if mask == "none":
        return True
    if mask == "causal":
        diag = i + (Lk - Lq)
        return j <= diag and (window < 0 or diag - j <= window)
    if mask == "patch":
        return rng[0] <= j < rng[1]
    raise ValueError(mask)


def attention(q, k, v, scale, mask="none", patch=None, window=-1, softcap=0.0):
    """One sequence.  q[i][h][d], k[j][g][d], v[j][g][d] as nested lists.

    window >= 0 (causal only) keeps the keys at most `window` positions
    before the row's diagonal; softcap > 0 replaces each scaled score s by
    softcap * tanh(s / softcap).

    Returns (o[i][h][d], lse[h][i]) as nested lists of Python floats.
    """
    Lq, Hq, D = len(q), len(q[0]), len(q[0][0])
    Lk = len(k)
    Hkv = len(k[0]) if Lk else 1
    group = Hq // Hkv
    o = [[[0.0] * D for _ in range(Hq)] for _ in range(Lq)]
    lse = [[0.0] * Lq for _ in range(Hq)]
    for h in range(Hq):
        g = h // group
        for i in range(Lq):
            keys = [j for j in range(Lk)
                    if _allowed(mask, i, j, Lq, Lk, patch[i] if patch else None, window)]
            if not keys:
                lse[h][i] = -math.inf
                continue
            e = {}
            for j in keys:
                s = scale * math.fsum(q[i][h][d] * k[j][g][d] for d in range(D))
                if softcap > 0:
                    s = softcap * math.tanh(s / softcap)
                e[j] = math.exp(s)
            z = math.fsum(e.values())
            for d in range(D):
                o[i][h][d] = math.fsum(e[j] / z * v[j][g][d] for j in keys)
            lse[h][i] = math.log(z)
    return o, lse
