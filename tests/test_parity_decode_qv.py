"""Paged decode with the extra Qv score term vs the fp64 oracle.

The logit of key j is scale * (q . k_j + qv . v_j) ("Rope dim", the Qv GEMM
beside the QK GEMM); the oracle is attn_varlen_qv with one query row per
sequence over the paged cache (pinned on the CPU in test_oracle_qv.py).
Tolerances as for the bf16 decode: max |O - O_ref| <= 2e-2, |LSE - LSE_ref| <= 1e-3.
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
    o = np.asarray(o.float().cpu().numpy(), np.float64)
    lse = np.asarray(lse.float().cpu().numpy(), np.float64)
    assert np.all(np.isfinite(o)), what + ": non-finite output"
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    assert err_o <= TOL_O, "%s: max|O err| %.3g" % (what, err_o)
    ninf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), ninf), what + ": -inf rows differ"
    assert np.all(o[ninf] == 0.0), what + ": empty rows not zero"
    if (~ninf).any():
        err_l = float(np.max(np.abs(lse[~ninf] - lse_ref[~ninf])))
        assert err_l <= TOL_LSE, "%s: max|LSE err| %.3g" % (what, err_l)


def _case(lens, Hq, Hkv, D, seed, window_left=-1, softcap=0.0, num_blocks=2000, lmax=3072):
    w = W.paged_decode(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, num_blocks=num_blocks, lmax=lmax,
                       lens=lens, seed=seed)
    t = w.tensors
    qv = W.randn_bf16((len(lens), Hq, D), seed, 31)
    o, lse = A.attn_decode_paged_qv(t["q"].to(DEV), qv.to(DEV), t["k_cache"].to(DEV),
                                    t["v_cache"].to(DEV), t["block_table"].to(DEV),
                                    t["seqused_k"].to(DEV), scale=w.params["scale"],
                                    window_left=window_left, softcap=softcap)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    B = len(lens)
    o_ref, lse_ref = oracle.attn_varlen_qv(
        t["q"], qv, t["k_cache"], t["v_cache"], cu_seqlens_q=np.arange(B + 1, dtype=np.int32),
        num_heads_kv=Hkv, scale=w.params["scale"], block_table=t["block_table"],
        seqused_k=t["seqused_k"], mask=oracle.MASK_CAUSAL if window_left >= 0 else oracle.MASK_NONE,
        window_left=window_left, softcap=softcap)
    return o, lse, o_ref, lse_ref.T


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 4), (4, 1), (16, 8), (16, 1), (8, 8)])
def test_decode_qv_many_sequences(D, Hq, Hkv):
    lens = [0, 1, 5, 16, 17, 31, 300, 0, 2048, 64, 65, 1000, 7, 129, 3000, 15] * 2
    o, lse, o_ref, lse_ref = _case(lens, Hq, Hkv, D, seed=3 * D + Hq + Hkv)
    _cmp(o, lse, o_ref, lse_ref, "decode qv D%d Hq%d Hkv%d" % (D, Hq, Hkv))


@pytest.mark.parametrize("window_left,softcap", [(0, 0.0), (37, 0.0), (-1, 30.0), (200, 15.0)])
def test_decode_qv_window_softcap(window_left, softcap):
    lens = [1, 2, 16, 17, 40, 255, 256, 1500, 0, 33]
    o, lse, o_ref, lse_ref = _case(lens, 16, 4, 128, seed=41 + window_left, window_left=window_left,
                                   softcap=softcap, num_blocks=400, lmax=1536)
    _cmp(o, lse, o_ref, lse_ref, "decode qv window %d softcap %g" % (window_left, softcap))


def test_decode_qv_zero_qv_is_the_plain_decode():
    """qv = 0 removes the extra term: the result equals attn_decode_paged's bit for bit."""
    lens = [3, 100, 700, 16]
    w = W.paged_decode(B=4, Hq=8, Hkv=2, D=128, num_blocks=200, lmax=1024, lens=lens, seed=5)
    t = {k: v.to(DEV) for k, v in w.tensors.items()}
    qv = torch.zeros_like(t["q"])
    o1, l1 = A.attn_decode_paged_qv(t["q"], qv, t["k_cache"], t["v_cache"], t["block_table"],
                                    t["seqused_k"], scale=w.params["scale"])
    o2, l2 = A.attn_decode_paged(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                 t["seqused_k"], scale=w.params["scale"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
