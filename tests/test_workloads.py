"""Structure of the seeded synthetic inputs (lengths, page tables, patches, fp8)."""
import numpy as np
import torch

from attention_paged_kv_gqa_b200 import workloads as W


def test_uniform_lengths_inclusive_and_seeded():
    a = W.uniform_lengths(1000, 1, 8192, seed=0)
    b = W.uniform_lengths(1000, 1, 8192, seed=0)
    assert np.array_equal(a, b)
    assert a.min() >= 1 and a.max() <= 8192


def test_block_table_pages_distinct_and_in_pool():
    lens = [1, 16, 17, 300]
    bt = W.paged_block_table(lens, 16, 100, 20, seed=3)
    used = []
    for b, L in enumerate(lens):
        n = (L + 15) // 16
        used += bt[b, :n].tolist()
        assert torch.all(bt[b, n:] == 0)
    assert len(set(used)) == len(used)
    assert min(used) >= 0 and max(used) < 100


def test_patch_lengths_partition_bytes():
    w = W.patch_cross(B=3, nbytes=1000, H=2, D=8, seed=1)
    r = w.tensors["patch_kv_range"].numpy()
    cq = w.tensors["cu_seqlens_q"].numpy()
    for b in range(3):
        rb = r[cq[b]:cq[b + 1]]
        assert rb[0, 0] == 0 and rb[-1, 1] == 1000
        assert np.all(rb[1:, 0] == rb[:-1, 1])          # contiguous, in order
        lens = rb[:, 1] - rb[:, 0]
        assert lens.min() >= 1 and lens.max() <= 16


def test_fp8_quantisation_round_trip_bound():
    x = W.randn_bf16((64, 128), seed=0, stream=1)
    q, s = W.quantize_e4m3(x)
    assert q.dtype == torch.float8_e4m3fn
    back = q.float() * s
    # e4m3 keeps 3 mantissa bits: relative half-ulp 2^-4 for normal values
    err = (back - x.float()).abs()
    assert float((err - x.float().abs() * 2 ** -4 - 2 ** -9 * float(s)).max()) <= 1e-6
    assert float(q.float().abs().max()) <= 448.0


def test_varlen_prefill_shapes():
    w = W.varlen_paged_prefill(nseq=3, lmin=5, lmax=40, Hq=4, Hkv=2, D=8, num_blocks=32, seed=2)
    t = w.tensors
    assert t["q"].shape == (w.params["total_q"], 4, 8)
    assert int(t["cu_seqlens_q"][-1]) == w.params["total_q"]
    assert torch.equal(t["seqused_k"], (t["cu_seqlens_k"][1:] - t["cu_seqlens_k"][:-1]))
