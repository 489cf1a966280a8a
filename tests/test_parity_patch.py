"""Patch cross-attention through attn_fwd_patch: CUDA path vs the fp64 oracle.

The mask is the patch mask of the byte-latent model ("Cross Attention does not
work on CPU and older GPUs": one query per patch attending to its own patch's
bytes).  With max_interval <= 64 the CUDA-core kernel runs (one warp per query
and head, online softmax over 32-key chunks); above it the tiled tensor-core
kernel runs.  Tolerances as for the other bf16 paths: max |O err| <= 2e-2,
max |LSE err| <= 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from attention_paged_kv_gqa_b200 import binding as A
from attention_paged_kv_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_O, TOL_LSE = 2e-2, 1e-3
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert A.attn_check_device(0) == 0, "not a B200 or the kernel image does not load"
    torch.cuda.set_device(0)


def _cmp(o, lse, o_ref, lse_ref, what):
    o = o.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o)), what
    err = float(np.max(np.abs(o - o_ref)))
    assert err <= TOL_O, "%s: max|O err| %.3g" % (what, err)
    lse = lse.cpu().numpy().astype(np.float64)
    ninf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), ninf), what + ": -inf rows differ"
    if (~ninf).any():
        el = float(np.max(np.abs(lse[~ninf] - lse_ref[~ninf])))
        assert el <= TOL_LSE, "%s: max|LSE err| %.3g" % (what, el)


def _run(q, k, v, cq, ck, ranges, Hkv, max_interval, scale, max_seqlen_q):
    o, lse = A.attn_fwd_patch(q.to(DEV), k.to(DEV), v.to(DEV), cu_seqlens_q=cq.to(DEV),
                              cu_seqlens_k=ck.to(DEV), patch_kv_range=ranges.to(DEV),
                              max_seqlen_q=max_seqlen_q, max_interval=max_interval, scale=scale)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen(q, k, v, cu_seqlens_q=cq, cu_seqlens_k=ck, num_heads_kv=Hkv,
                                        scale=scale, mask=2, patch_kv_range=ranges)
    return o, lse, o_ref, lse_ref


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("max_interval", [16, 200])
def test_patch_cross_small(D, max_interval):
    w = W.patch_cross(B=2, nbytes=600, H=4, D=D, seed=D)
    t = w.tensors
    o, lse, o_ref, lse_ref = _run(t["q"], t["k"], t["v"], t["cu_seqlens_q"], t["cu_seqlens_k"],
                                  t["patch_kv_range"], 4, max_interval, w.params["scale"],
                                  w.params["max_seqlen_q"])
    _cmp(o, lse, o_ref, lse_ref, "patch D%d hint %d" % (D, max_interval))


@pytest.mark.parametrize("D", [64, 128])
def test_patch_gqa_ragged_intervals(D):
    """GQA, empty and one-key intervals, intervals past the sequence end (clamped), and
    intervals longer than one 32-key chunk (online softmax across chunks)."""
    rng = np.random.default_rng(7 + D)
    lens_q, lens_k = [9, 0, 14], [70, 5, 300]
    cq, ck = W.cu_from_lens(lens_q), W.cu_from_lens(lens_k)
    rows = []
    for b in range(3):
        for i in range(lens_q[b]):
            s0 = int(rng.integers(0, lens_k[b] + 1))
            n = int(rng.choice([0, 1, 2, 16, 33, 64]))
            rows.append((s0, s0 + n))          # may run past Lk: clamped
    ranges = torch.tensor(rows, dtype=torch.int32).reshape(-1, 2)
    Hq, Hkv = 8, 2
    q = W.randn_bf16((int(cq[-1]), Hq, D), 3, 1)
    k = W.randn_bf16((int(ck[-1]), Hkv, D), 3, 2)
    v = W.randn_bf16((int(ck[-1]), Hkv, D), 3, 3)
    o, lse, o_ref, lse_ref = _run(q, k, v, cq, ck, ranges, Hkv, 64, 0.2, max(lens_q))
    _cmp(o, lse, o_ref, lse_ref, "patch gqa D%d" % D)


def test_config_patch_cross_full_cuda_cores():
    """The bench's patch configuration at full size (B=4 x 8192 byte keys, Geometric(0.22)
    patches clipped to [1,16], H=16, D=64), every output, on the CUDA-core kernel."""
    w = W.FULL_SIZE["patch_cross_attention_bf16"]()
    t = w.tensors
    o, lse, o_ref, lse_ref = _run(t["q"], t["k"], t["v"], t["cu_seqlens_q"], t["cu_seqlens_k"],
                                  t["patch_kv_range"], 16, 16, w.params["scale"],
                                  w.params["max_seqlen_q"])
    _cmp(o, lse, o_ref, lse_ref, "patch full")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4), (8, 8), (16, 16)])
def test_patch_short_intervals_ragged(D, Hq, Hkv):
    """Intervals of at most 16 keys through attn_fwd_patch: GQA; empty, one-key and clipped
    intervals; starts out of order and overlapping; sequences with no queries or no keys."""
    rng = np.random.default_rng(100 + D + Hq)
    lens_q, lens_k = [0, 37, 5, 120, 1, 64, 9], [10, 100, 0, 700, 16, 90, 40]
    cq, ck = W.cu_from_lens(lens_q), W.cu_from_lens(lens_k)
    rows = []
    for b in range(len(lens_q)):
        for i in range(lens_q[b]):
            s0 = int(rng.integers(-3, lens_k[b] + 3))
            n = int(rng.choice([0, 1, 2, 7, 15, 16]))
            rows.append((s0, s0 + n))
    ranges = torch.tensor(rows, dtype=torch.int32).reshape(-1, 2)
    q = W.randn_bf16((int(cq[-1]), Hq, D), 5, 1)
    k = W.randn_bf16((int(ck[-1]), Hkv, D), 5, 2)
    v = W.randn_bf16((int(ck[-1]), Hkv, D), 5, 3)
    o, lse, o_ref, lse_ref = _run(q, k, v, cq, ck, ranges, Hkv, 16, 0.15, max(lens_q))
    _cmp(o, lse, o_ref, lse_ref, "patch short D%d Hq%d Hkv%d" % (D, Hq, Hkv))



@pytest.mark.parametrize("D", [64, 128])
def test_patch_equal_heads_long_intervals_and_many_sequences(D):
    """Hq == Hkv (the streaming kernel): intervals longer than the caller's max_interval
    (it chooses the kernel, never the result), overlapping and out-of-order intervals, and
    more sequences than fit the kernel's shared-memory sequence table."""
    rng = np.random.default_rng(300 + D)
    B = 300
    lens_q = rng.integers(0, 6, B)
    lens_k = rng.integers(0, 200, B)
    cq, ck = W.cu_from_lens(lens_q), W.cu_from_lens(lens_k)
    rows = []
    for b in range(B):
        for i in range(int(lens_q[b])):
            s0 = int(rng.integers(-3, int(lens_k[b]) + 3))
            n = int(rng.choice([0, 1, 5, 16, 40, 64, 65, 150]))
            rows.append((s0, s0 + n))
    ranges = torch.tensor(rows, dtype=torch.int32).reshape(-1, 2)
    Hq = 8
    q = W.randn_bf16((int(cq[-1]), Hq, D), 6, 1)
    k = W.randn_bf16((int(ck[-1]), Hq, D), 6, 2)
    v = W.randn_bf16((int(ck[-1]), Hq, D), 6, 3)
    o, lse, o_ref, lse_ref = _run(q, k, v, cq, ck, ranges, Hq, 16, 0.15, int(lens_q.max()))
    _cmp(o, lse, o_ref, lse_ref, "patch long/many D%d" % D)
