"""Attention backward: CUDA path vs the fp64 oracle, element by element.

The GPU backward is fed the GPU forward's O (bf16) and LSE (fp32), as a
training step would be; the oracle recomputes both exactly.  Tolerance,
derived from the arithmetic (no bound is stated for the backward):
P and dS are rounded to bf16 (relative 2^-9) as tensor-core operands with
fp32 accumulation, the outputs are bf16, and Delta = dO . O inherits the
bf16 rounding of O, so per gradient tensor
    max |g - g_ref| <= 2e-2 * max |g_ref| + 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from attention_paged_kv_gqa_b200 import binding as A
from attention_paged_kv_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
REL, ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert A.attn_check_device(0) == 0, "not a B200 or the kernel image does not load"
    torch.cuda.set_device(0)


def _check(got, ref, what):
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(g)), what + ": non-finite"
    tol = REL * float(np.max(np.abs(ref))) + ABS
    err = float(np.max(np.abs(g - ref))) if g.size else 0.0
    assert err <= tol, "%s: max err %.4g > %.4g" % (what, err, tol)


def _run(lens_q, lens_k, Hq, Hkv, D, causal, window=-1, seed=0, scale=None):
    cq = W.cu_from_lens(lens_q)
    ck = W.cu_from_lens(lens_k)
    q = W.randn_bf16((int(cq[-1]), Hq, D), seed, 41)
    k = W.randn_bf16((int(ck[-1]), Hkv, D), seed, 42)
    v = W.randn_bf16((int(ck[-1]), Hkv, D), seed, 43)
    do = W.randn_bf16((int(cq[-1]), Hq, D), seed, 44)
    scale = scale if scale is not None else 1.0 / D ** 0.5
    mask = A.MASK_CAUSAL if causal else A.MASK_NONE
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    cqd, ckd = cq.to(DEV), ck.to(DEV)
    o, lse = A.attn_fwd_varlen_paged(qd, kd, vd, cu_seqlens_q=cqd, cu_seqlens_k=ckd,
                                     max_seqlen_q=max(lens_q), mask=mask, scale=scale,
                                     window_left=window)
    dq, dk, dv = A.attn_bwd_varlen(qd, kd, vd, o, dod, lse, cu_seqlens_q=cqd, cu_seqlens_k=ckd,
                                   max_seqlen_q=max(lens_q), max_seqlen_k=max(lens_k), mask=mask,
                                   scale=scale, window_left=window)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    rq, rk, rv = oracle.attn_bwd_varlen(q, k, v, do, cu_seqlens_q=cq, cu_seqlens_k=ck,
                                        num_heads_kv=Hkv, scale=scale, mask=1 if causal else 0,
                                        window_left=window)
    _check(dq, rq, "dQ")
    _check(dk, rk, "dK")
    _check(dv, rv, "dV")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("L", [1, 100, 129, 300])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2)])
def test_bwd_dense_shapes(D, L, causal, Hq, Hkv):
    _run([L, L], [L, L], Hq, Hkv, D, causal, seed=L + D)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("window", [-1, 50])
def test_bwd_varlen_gqa(D, window):
    lens = [1, 16, 17, 129, 255, 64, 300]
    _run(lens, lens, 8, 2, D, True, window=window, seed=D + window)


def test_bwd_bottom_right_lq_lt_lk():
    _run([130, 5], [300, 200], 4, 1, 128, True, seed=3)


def test_bwd_unmasked_ragged_and_empty_sequences():
    _run([0, 33, 200], [7, 0, 150], 4, 4, 64, False, seed=4)


def test_bwd_longer_sequence_many_tiles():
    _run([1024], [1024], 8, 2, 128, True, seed=5)


def test_bwd_dense_wrapper_matches_varlen():
    """The dense-layout convenience gives the varlen call's result on the same data."""
    B, L, H, D = 2, 200, 4, 64
    q, k, v, do = (W.randn_bf16((B, L, H, D), 7, s).to(DEV) for s in (1, 2, 3, 4))
    o, lse = A.attn_fwd_dense(q, k, v, causal=True)
    dq, dk, dv = A.attn_bwd_dense(q, k, v, o, do, lse, causal=True)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attn_bwd_dense(q.cpu(), k.cpu(), v.cpu(), do.cpu(), scale=1 / 8, causal=True)
    _check(dq, rq, "dense dQ")
    _check(dk, rk, "dense dK")
    _check(dv, rv, "dense dV")


def test_bwd_config_varlen_causal_gqa_full():
    """The bench's backward workload at full size (16 sequences, L ~ U[64,4096], Hq=32, Hkv=8,
    D=128, causal): the GPU runs the whole batch; the oracle checks every gradient of the
    shortest sequence and of the fourth shortest (sequences are independent)."""
    wp = W.FULL_SIZE["varlen_paged_gqa_prefill_causal_bf16"]()
    lens = wp.tensors["seqused_k"].numpy().astype(np.int64)
    cu = W.cu_from_lens(lens)
    total, Hq, Hkv, D, scale = int(cu[-1]), 32, 8, 128, wp.params["scale"]
    q = W.randn_bf16((total, Hq, D), 0, 51)
    k = W.randn_bf16((total, Hkv, D), 0, 52)
    v = W.randn_bf16((total, Hkv, D), 0, 53)
    do = W.randn_bf16((total, Hq, D), 0, 54)
    qd, kd, vd, dod, cud = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV), cu.to(DEV)
    maxlen = int(lens.max())
    o, lse = A.attn_fwd_varlen_paged(qd, kd, vd, cu_seqlens_q=cud, cu_seqlens_k=cud, max_seqlen_q=maxlen,
                                     mask=A.MASK_CAUSAL, scale=scale)
    dq, dk, dv = A.attn_bwd_varlen(qd, kd, vd, o, dod, lse, cu_seqlens_q=cud, cu_seqlens_k=cud,
                                   max_seqlen_q=maxlen, max_seqlen_k=maxlen, mask=A.MASK_CAUSAL, scale=scale)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    order = np.argsort(lens)
    for b in (int(order[0]), int(order[3])):
        sl = slice(int(cu[b]), int(cu[b + 1]))
        c1 = np.array([0, lens[b]], np.int32)
        rq, rk, rv = oracle.attn_bwd_varlen(q[sl], k[sl], v[sl], do[sl], cu_seqlens_q=c1, cu_seqlens_k=c1,
                                            num_heads_kv=Hkv, scale=scale, mask=1)
        _check(dq[sl], rq, "dQ seq %d" % b)
        _check(dk[sl], rk, "dK seq %d" % b)
        _check(dv[sl], rv, "dV seq %d" % b)
