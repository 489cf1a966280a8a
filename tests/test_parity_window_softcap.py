"""Sliding window and softcap: CUDA path vs the fp64 oracle, element by element.

The two options are read from the "local window on/off" and "softcap 0/50"
columns of the parity matrix in "[CUDA] PagedAttention: add SM<80 fp16
fallback via memory-efficient attention" (Testing): a causal row keeps the
keys i' - W <= j <= i' (i' = i + Lk - Lq), and a softcap c maps each scaled
logit s to c * tanh(s / c).  The decode query is the newest cached token.

Tolerances (against fp64, after the kernel's bf16 output rounding), as for
the plain path: bf16 max |O err| <= 2e-2 and max |LSE err| <= 1e-3; fp8
max |O err| <= 6e-2.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_paged_kv_gqa_b200 import binding as A
from attention_paged_kv_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_O_BF16, TOL_LSE_BF16, TOL_O_FP8 = 2e-2, 1e-3, 6e-2
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert A.attn_check_device(0) == 0, "not a B200 or the kernel image does not load"
    torch.cuda.set_device(0)


def _cmp(o, lse, o_ref, lse_ref, tol_o, tol_lse, what=""):
    o = np.asarray(o.float().cpu().numpy(), np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), what + ": non-finite output"
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    assert err_o <= tol_o, "%s: max|O err| %.3g > %.3g" % (what, err_o, tol_o)
    if lse is not None:
        lse = np.asarray(lse.float().cpu().numpy(), np.float64)
        ninf = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse), ninf), what + ": -inf rows differ"
        if tol_lse is not None and (~ninf).any():
            err_l = float(np.max(np.abs(lse[~ninf] - lse_ref[~ninf])))
            assert err_l <= tol_lse, "%s: max|LSE err| %.3g > %.3g" % (what, err_l, tol_lse)


def _no_device_error():
    assert A.attn_device_error() == 0


def _scaled_bf16(x, f):
    """x * f rounded to bf16, so that both sides see the same (larger) logits."""
    return (x.float() * f).to(torch.bfloat16)


# ---------------------------------------------------------------------------- dense
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("L", [129, 700])
@pytest.mark.parametrize("window", [0, 5, 127, 128, 333])
def test_dense_sliding_window(D, L, window):
    w = W.dense(B=2, L=L, Hq=4, Hkv=2, D=D, causal=True, seed=L + window + D)
    t = w.tensors
    o, lse = A.attn_fwd_dense(t["q"].to(DEV), t["k"].to(DEV), t["v"].to(DEV), causal=True,
                              scale=w.params["scale"], window_left=window)
    torch.cuda.synchronize()
    _no_device_error()
    o_ref, lse_ref = oracle.attn_dense(t["q"], t["k"], t["v"], scale=w.params["scale"],
                                       causal=True, window_left=window)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "dense window %d" % window)


@pytest.mark.parametrize("window", [0, 64, 200])
def test_dense_sliding_window_bottom_right(window):
    """Lq < Lk: the window hangs off the bottom-right-aligned diagonal."""
    w = W.dense(B=2, L=130, Lk=500, Hq=2, Hkv=1, D=128, causal=True, seed=window + 1)
    t = w.tensors
    o, lse = A.attn_fwd_dense(t["q"].to(DEV), t["k"].to(DEV), t["v"].to(DEV), causal=True,
                              scale=w.params["scale"], window_left=window)
    o_ref, lse_ref = oracle.attn_dense(t["q"], t["k"], t["v"], scale=w.params["scale"],
                                       causal=True, window_left=window)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "bottom-right window")
    _no_device_error()


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("cap,window", [(2.0, -1), (50.0, -1), (2.0, 100)])
def test_dense_softcap(D, causal, cap, window):
    if window >= 0 and not causal:
        pytest.skip("a window needs the causal mask")
    w = W.dense(B=2, L=300, Hq=4, Hkv=2, D=D, causal=causal, seed=int(cap) + D)
    t = w.tensors
    q = _scaled_bf16(t["q"], 4.0)      # logits of several units, where the cap bites
    o, lse = A.attn_fwd_dense(q.to(DEV), t["k"].to(DEV), t["v"].to(DEV), causal=causal,
                              scale=w.params["scale"], softcap=cap, window_left=window)
    torch.cuda.synchronize()
    _no_device_error()
    o_ref, lse_ref = oracle.attn_dense(q, t["k"], t["v"], scale=w.params["scale"], causal=causal,
                                       softcap=cap, window_left=window)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "softcap %g" % cap)


def test_softcap_changes_the_result():
    """Guards against a cap that is silently ignored: at c = 2 the capped and the
    plain outputs differ by far more than the tolerance."""
    w = W.dense(B=1, L=200, Hq=2, Hkv=2, D=128, causal=True, seed=77)
    t = w.tensors
    q = _scaled_bf16(t["q"], 4.0).to(DEV)
    o1, _ = A.attn_fwd_dense(q, t["k"].to(DEV), t["v"].to(DEV), causal=True, softcap=2.0)
    o0, _ = A.attn_fwd_dense(q, t["k"].to(DEV), t["v"].to(DEV), causal=True)
    assert (o1.float() - o0.float()).abs().max().item() > 0.1


@pytest.mark.parametrize("D", [64, 128])
def test_fp8_sliding_window_and_softcap(D):
    """fp8 with a cap and/or a window.  N(0,1) inputs as in the fp8 workload, for
    which the fp8 tolerance is stated (logits up to about 4, so caps of 2 and 3
    still bite).  Lq < Lk gives every row at least 61 keys: over a handful of keys
    with flat weights the e4m3 rounding of P (2^-4 relative per weight) alone can
    exceed 6e-2, which is a property of e4m3 P, not of the cap or the window (the
    bf16 tests check those at a tight tolerance)."""
    w = W.dense(B=2, L=128, Lk=400, Hq=4, Hkv=2, D=D, causal=True, seed=5 + D)
    t = w.tensors
    qf, dq = W.quantize_e4m3(t["q"])
    kf, dk = W.quantize_e4m3(t["k"])
    vf, dv = W.quantize_e4m3(t["v"])
    for cap, window in ((2.0, -1), (0.0, 60), (3.0, 150)):
        o, lse = A.attn_fwd_dense(qf.to(DEV), kf.to(DEV), vf.to(DEV), causal=True,
                                  scale=w.params["scale"], softcap=cap, window_left=window,
                                  descale_q=dq.to(DEV), descale_k=dk.to(DEV),
                                  descale_v=dv.to(DEV))
        torch.cuda.synchronize()
        _no_device_error()
        o_ref, lse_ref = oracle.attn_dense(oracle.dequant_e4m3(qf, dq),
                                           oracle.dequant_e4m3(kf, dk),
                                           oracle.dequant_e4m3(vf, dv), scale=w.params["scale"],
                                           causal=True, softcap=cap, window_left=window)
        _cmp(o, lse, o_ref, lse_ref, TOL_O_FP8, None, "fp8 D%d cap %g window %d" % (D, cap, window))


# ---------------------------------------------------------------------------- varlen, paged
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("window,cap", [(0, 0.0), (50, 0.0), (200, 0.0), (-1, 5.0), (70, 5.0)])
def test_varlen_paged_window_softcap(D, window, cap):
    lens = [1, 16, 17, 129, 255, 64, 300]
    w = W.varlen_paged_prefill(nseq=len(lens), Hq=8, Hkv=2, D=D, num_blocks=200, lens=lens,
                               lmax=320, seed=D + window)
    t = w.tensors
    q = _scaled_bf16(t["q"], 3.0)
    o, lse = A.attn_fwd_varlen_paged(q.to(DEV), t["k_cache"].to(DEV), t["v_cache"].to(DEV),
                                     cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                                     max_seqlen_q=w.params["max_seqlen_q"],
                                     block_table=t["block_table"].to(DEV),
                                     seqused_k=t["seqused_k"].to(DEV), mask=A.MASK_CAUSAL,
                                     scale=w.params["scale"], window_left=window, softcap=cap)
    torch.cuda.synchronize()
    _no_device_error()
    o_ref, lse_ref = oracle.attn_varlen(q, t["k_cache"], t["v_cache"],
                                        cu_seqlens_q=t["cu_seqlens_q"], seqused_k=t["seqused_k"],
                                        block_table=t["block_table"], num_heads_kv=2,
                                        scale=w.params["scale"], mask=1, window_left=window,
                                        softcap=cap)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "varlen window %d cap %g" % (window, cap))


# ---------------------------------------------------------------------------- decode
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (16, 2)])
@pytest.mark.parametrize("splits", [0, 3])
@pytest.mark.parametrize("window,cap", [(0, 0.0), (15, 0.0), (16, 0.0), (17, 0.0), (100, 3.0),
                                        (-1, 3.0), (5000, 0.0)])
def test_decode_window_softcap(D, Hq, Hkv, splits, window, cap):
    lens = [0, 1, 15, 16, 17, 64, 65, 513, 1000, 2500]
    w = W.paged_decode(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, num_blocks=600, lmax=2560, lens=lens,
                       seed=D + Hq + window)
    t = w.tensors
    q = _scaled_bf16(t["q"], 3.0)
    o, lse = A.attn_decode_paged(q.to(DEV), t["k_cache"].to(DEV), t["v_cache"].to(DEV),
                                 t["block_table"].to(DEV), t["seqused_k"].to(DEV),
                                 scale=w.params["scale"], num_splits=splits, window_left=window,
                                 softcap=cap)
    torch.cuda.synchronize()
    _no_device_error()
    o_ref, lse_ref = oracle.attn_decode(q, t["k_cache"], t["v_cache"], t["block_table"],
                                        t["seqused_k"], scale=w.params["scale"],
                                        window_left=window, softcap=cap)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16,
         "decode window %d cap %g splits %d" % (window, cap, splits))
