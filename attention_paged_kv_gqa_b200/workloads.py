"""Seeded synthetic inputs for the attention forward workloads.

This module is shared by the CUDA path (bench, GPU tests) and by the fp64
oracle's tests.  It holds no attention arithmetic: it only draws random
numbers, builds sequence-length tables, page pools and block tables, and
quantises tensors to fp8 e4m3 (an input-preparation step of the fp8 workload).
It imports nothing else from this package.

Workloads (all on the CPU, reproducible from the seed):

* dense causal bf16      B=2,  Hq=Hkv=2,  L=128, D=64
* paged GQA decode bf16  B=32, Hq=32, Hkv=8, D=128, kv len ~ U[1, 8192],
                          16-token pages, 20000-page pool, permuted block table
* varlen paged prefill   16 sequences, q len = kv len ~ U[64, 4096], Hq=32,
                          Hkv=8, D=128, 16-token pages, causal
* patch cross-attention  B=4 x 8192 byte keys, patch lengths Geometric(0.22)
                          clipped to [1, 16], one query per patch, H=16, D=64
* fp8 dense causal       B=4, H=16, L=4096, D=128, per-tensor e4m3 + fp32 descale

Value distribution: every Q/K/V element is an independent N(0, 1) draw in
fp32 (torch.Generator), rounded to bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

FP8_E4M3_MAX = 448.0


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1_000_003 + int(stream))
    return g


def randn_bf16(shape, seed: int, stream: int, chunk_elems: int = 1 << 24) -> torch.Tensor:
    """N(0,1) fp32 draws rounded to bf16, generated in chunks to bound host memory."""
    g = _gen(seed, stream)
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.bfloat16)
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        out[s:e] = torch.randn(e - s, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return out.view(*shape)


def cu_from_lens(lens) -> torch.Tensor:
    lens = torch.as_tensor(lens, dtype=torch.int64)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lens, 0)
    return cu.to(torch.int32)


def uniform_lengths(n: int, lo: int, hi: int, seed: int, stream: int = 7) -> np.ndarray:
    """Integer lengths drawn uniformly from the inclusive range [lo, hi]."""
    rng = np.random.default_rng(int(seed) * 1_000_003 + stream)
    return rng.integers(lo, hi + 1, size=n).astype(np.int64)


def paged_block_table(lens, block_size: int, num_blocks: int, max_blocks_per_seq: int,
                      seed: int, stream: int = 11) -> torch.Tensor:
    """Block table over a randomly permuted page pool.

    Sequence b takes the next ceil(L_b / block_size) pages of one random
    permutation of the pool, in order; no page is shared.  Entries past a
    sequence's last page are 0 (never read for that sequence).
    """
    need = [(int(L) + block_size - 1) // block_size for L in lens]
    if sum(need) > num_blocks:
        raise ValueError("page pool too small for the requested lengths")
    perm = torch.randperm(num_blocks, generator=_gen(seed, stream)).to(torch.int32)
    bt = torch.zeros(len(lens), max_blocks_per_seq, dtype=torch.int32)
    pos = 0
    for b, n in enumerate(need):
        if n > max_blocks_per_seq:
            raise ValueError("sequence longer than max_blocks_per_seq pages")
        bt[b, :n] = perm[pos:pos + n]
        pos += n
    return bt


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor symmetric quantisation to float8_e4m3fn.

    scale = amax(|x|) / 448; x_q = e4m3(x / scale) with round-to-nearest-even
    (torch's cast), clamped to the finite e4m3 range; descale = scale (fp32).
    """
    xf = x.float()
    amax = float(xf.abs().max())
    scale = amax / FP8_E4M3_MAX if amax > 0 else 1.0
    q = (xf / scale).clamp_(-FP8_E4M3_MAX, FP8_E4M3_MAX).to(torch.float8_e4m3fn)
    return q, torch.tensor([scale], dtype=torch.float32)


@dataclass
class Workload:
    """A bundle of host tensors plus the scalar parameters that describe them."""
    name: str
    params: dict
    tensors: dict = field(default_factory=dict)


def dense(B=2, L=128, Hq=2, Hkv=2, D=64, causal=True, seed=0, Lk=None) -> Workload:
    """Dense [B, L, H, D] Q/K/V (bf16)."""
    Lk = L if Lk is None else Lk
    q = randn_bf16((B, L, Hq, D), seed, 1)
    k = randn_bf16((B, Lk, Hkv, D), seed, 2)
    v = randn_bf16((B, Lk, Hkv, D), seed, 3)
    return Workload("dense_causal_bf16" if causal else "dense_bf16",
                    dict(B=B, Lq=L, Lk=Lk, Hq=Hq, Hkv=Hkv, D=D, causal=causal,
                         scale=1.0 / math.sqrt(D), seed=seed),
                    dict(q=q, k=k, v=v))


def paged_decode(B=32, Hq=32, Hkv=8, D=128, block_size=16, num_blocks=20000,
                 lmin=1, lmax=8192, seed=0, lens=None) -> Workload:
    """One query token per sequence against a paged KV cache (bf16)."""
    lens = uniform_lengths(B, lmin, lmax, seed) if lens is None else np.asarray(lens, np.int64)
    mbps = (lmax + block_size - 1) // block_size
    bt = paged_block_table(lens, block_size, num_blocks, mbps, seed)
    k_cache = randn_bf16((num_blocks, block_size, Hkv, D), seed, 21)
    v_cache = randn_bf16((num_blocks, block_size, Hkv, D), seed, 22)
    q = randn_bf16((B, Hq, D), seed, 23)
    return Workload("paged_gqa_decode_bf16",
                    dict(B=B, Hq=Hq, Hkv=Hkv, D=D, block_size=block_size,
                         num_blocks=num_blocks, max_blocks_per_seq=mbps,
                         scale=1.0 / math.sqrt(D), seed=seed),
                    dict(q=q, k_cache=k_cache, v_cache=v_cache, block_table=bt,
                         seqused_k=torch.as_tensor(lens, dtype=torch.int32)))


def varlen_paged_prefill(nseq=16, lmin=64, lmax=4096, Hq=32, Hkv=8, D=128,
                         block_size=16, num_blocks=20000, seed=0, lens=None,
                         causal=True) -> Workload:
    """Packed varlen queries (q len = kv len) against a paged KV cache (bf16)."""
    lens = uniform_lengths(nseq, lmin, lmax, seed) if lens is None else np.asarray(lens, np.int64)
    mbps = (int(max(lmax, int(lens.max()))) + block_size - 1) // block_size
    bt = paged_block_table(lens, block_size, num_blocks, mbps, seed)
    total = int(lens.sum())
    q = randn_bf16((total, Hq, D), seed, 31)
    k_cache = randn_bf16((num_blocks, block_size, Hkv, D), seed, 32)
    v_cache = randn_bf16((num_blocks, block_size, Hkv, D), seed, 33)
    cu = cu_from_lens(lens)
    return Workload("varlen_paged_gqa_prefill_causal_bf16",
                    dict(B=nseq, Hq=Hq, Hkv=Hkv, D=D, block_size=block_size,
                         num_blocks=num_blocks, max_blocks_per_seq=mbps,
                         total_q=total, max_seqlen_q=int(lens.max()),
                         causal=causal, scale=1.0 / math.sqrt(D), seed=seed),
                    dict(q=q, k_cache=k_cache, v_cache=v_cache, block_table=bt,
                         cu_seqlens_q=cu, cu_seqlens_k=cu.clone(),
                         seqused_k=torch.as_tensor(lens, dtype=torch.int32)))


def patch_lengths(nbytes: int, p: float, max_len: int, rng: np.random.Generator) -> list:
    """Patch lengths ~ Geometric(p) (support >= 1) clipped to max_len, summing to nbytes.

    Lengths are appended until their sum reaches nbytes; the last one is cut so
    the sum is exactly nbytes (it stays >= 1).
    """
    out, total = [], 0
    while total < nbytes:
        n = int(min(rng.geometric(p), max_len))
        n = min(n, nbytes - total)
        out.append(n)
        total += n
    return out


def patch_cross(B=4, nbytes=8192, p=0.22, max_patch=16, H=16, D=64, seed=0) -> Workload:
    """Patch-to-byte cross-attention: query q (one per patch) sees only its patch's bytes."""
    rng = np.random.default_rng(int(seed) * 1_000_003 + 41)
    plens = [patch_lengths(nbytes, p, max_patch, rng) for _ in range(B)]
    nq = [len(x) for x in plens]
    total_q = int(sum(nq))
    ranges = torch.zeros(total_q, 2, dtype=torch.int32)
    r = 0
    for b in range(B):
        start = 0
        for n in plens[b]:
            ranges[r, 0] = start
            ranges[r, 1] = start + n
            start += n
            r += 1
    q = randn_bf16((total_q, H, D), seed, 42)
    k = randn_bf16((B * nbytes, H, D), seed, 43)
    v = randn_bf16((B * nbytes, H, D), seed, 44)
    return Workload("patch_cross_attention_bf16",
                    dict(B=B, Hq=H, Hkv=H, D=D, nbytes=nbytes, total_q=total_q,
                         total_k=B * nbytes, max_seqlen_q=max(nq),
                         scale=1.0 / math.sqrt(D), seed=seed),
                    dict(q=q, k=k, v=v, cu_seqlens_q=cu_from_lens(nq),
                         cu_seqlens_k=cu_from_lens([nbytes] * B),
                         patch_kv_range=ranges))


def fp8_dense_causal(B=4, H=16, L=4096, D=128, seed=0) -> Workload:
    """bf16 N(0,1) Q/K/V and their per-tensor e4m3 quantisations with fp32 descales."""
    w = dense(B=B, L=L, Hq=H, Hkv=H, D=D, causal=True, seed=seed)
    t = w.tensors
    for name in ("q", "k", "v"):
        t[name + "_fp8"], t["descale_" + name] = quantize_e4m3(t[name])
    w.name = "fp8_e4m3_dense_causal"
    return w


# The workloads by what they are, at their full sizes.
FULL_SIZE = {
    "dense_causal_bf16": lambda seed=0: dense(seed=seed),
    "paged_gqa_decode_bf16": lambda seed=0: paged_decode(seed=seed),
    "varlen_paged_gqa_prefill_causal_bf16": lambda seed=0: varlen_paged_prefill(seed=seed),
    "patch_cross_attention_bf16": lambda seed=0: patch_cross(seed=seed),
    "fp8_e4m3_dense_causal": lambda seed=0: fp8_dense_causal(seed=seed),
}
