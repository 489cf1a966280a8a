"""The forward with the extra Qv score term vs the fp64 oracle, element by element.

"Rope dim" (vllm-project flash-attention PR 172, overview: HasQv) computes the
score from two GEMMs, s_ij = scale * (q_i . k_j + qv_i . v_j).  The kernel's HQ
instance issues the second score GEMM on the value tile (read K-major, like the
key tile), so each value tile feeds both that GEMM and P.V.  The oracle's
attn_varlen_qv is pinned on the CPU (tests/test_oracle_qv.py).

Tolerances as for the plain bf16 path: max |O err| <= 2e-2, max |LSE err| <= 1e-3.
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


def _cmp(o, lse, o_ref, lse_ref, what=""):
    o = np.asarray(o.float().cpu().numpy(), np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), what + ": non-finite output"
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    assert err_o <= TOL_O, "%s: max|O err| %.3g > %.3g" % (what, err_o, TOL_O)
    lse = np.asarray(lse.float().cpu().numpy(), np.float64)
    ninf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), ninf), what + ": -inf rows differ"
    if (~ninf).any():
        err_l = float(np.max(np.abs(lse[~ninf] - lse_ref[~ninf])))
        assert err_l <= TOL_LSE, "%s: max|LSE err| %.3g > %.3g" % (what, err_l, TOL_LSE)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4), (3, 1)])
def test_prefill_paged_qv(D, causal, Hq, Hkv):
    """Ragged lengths over several 128-key tiles (1, page edges, tile edges, 300+)."""
    lens = [1, 17, 129, 300, 64, 255, 513]
    w = W.varlen_paged_prefill(nseq=len(lens), Hq=Hq, Hkv=Hkv, D=D, num_blocks=300, lens=lens,
                               lmax=640, seed=2 * D + Hq + causal)
    t = w.tensors
    qv = W.randn_bf16(tuple(t["q"].shape), w.params["seed"], 41)
    mask = A.MASK_CAUSAL if causal else A.MASK_NONE
    o, lse = A.attn_fwd_varlen_paged_qv(t["q"].to(DEV), qv.to(DEV), t["k_cache"].to(DEV),
                                        t["v_cache"].to(DEV), cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                                        max_seqlen_q=w.params["max_seqlen_q"],
                                        block_table=t["block_table"].to(DEV),
                                        seqused_k=t["seqused_k"].to(DEV), mask=mask,
                                        scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_qv(t["q"], qv, t["k_cache"], t["v_cache"],
                                           cu_seqlens_q=t["cu_seqlens_q"], block_table=t["block_table"],
                                           seqused_k=t["seqused_k"], num_heads_kv=Hkv,
                                           scale=w.params["scale"], mask=int(mask))
    _cmp(o, lse, o_ref, lse_ref, "paged qv D%d Hq%d Hkv%d causal %d" % (D, Hq, Hkv, causal))


def test_prefill_packed_qv_lq_lt_lk():
    """Packed store, bottom-right causal with fewer queries than keys, an empty sequence."""
    lq, lk = [130, 0, 5, 77], [300, 9, 200, 77]
    Hq, Hkv, D = 4, 1, 128
    cq, ck = W.cu_from_lens(lq), W.cu_from_lens(lk)
    q = W.randn_bf16((int(cq[-1]), Hq, D), 4, 1)
    qv = W.randn_bf16((int(cq[-1]), Hq, D), 4, 2)
    k = W.randn_bf16((int(ck[-1]), Hkv, D), 4, 3)
    v = W.randn_bf16((int(ck[-1]), Hkv, D), 4, 4)
    o, lse = A.attn_fwd_varlen_paged_qv(q.to(DEV), qv.to(DEV), k.to(DEV), v.to(DEV),
                                        cu_seqlens_q=cq.to(DEV), cu_seqlens_k=ck.to(DEV),
                                        max_seqlen_q=max(lq), mask=A.MASK_CAUSAL, scale=0.1)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_qv(q, qv, k, v, cu_seqlens_q=cq, cu_seqlens_k=ck,
                                           num_heads_kv=Hkv, scale=0.1, mask=1)
    _cmp(o, lse, o_ref, lse_ref, "packed qv")


@pytest.mark.parametrize("window,softcap", [(100, 0.0), (-1, 30.0), (40, 20.0)])
def test_prefill_qv_window_softcap(window, softcap):
    lens = [33, 400, 129]
    w = W.varlen_paged_prefill(nseq=3, Hq=8, Hkv=2, D=128, num_blocks=100, lens=lens, lmax=512,
                               seed=window + 9)
    t = w.tensors
    qv = (W.randn_bf16(tuple(t["q"].shape), 9, 42).float() * 2).to(torch.bfloat16)
    o, lse = A.attn_fwd_varlen_paged_qv(t["q"].to(DEV), qv.to(DEV), t["k_cache"].to(DEV),
                                        t["v_cache"].to(DEV), cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                                        max_seqlen_q=w.params["max_seqlen_q"],
                                        block_table=t["block_table"].to(DEV),
                                        seqused_k=t["seqused_k"].to(DEV), mask=A.MASK_CAUSAL,
                                        scale=w.params["scale"], window_left=window, softcap=softcap)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_qv(t["q"], qv, t["k_cache"], t["v_cache"],
                                           cu_seqlens_q=t["cu_seqlens_q"], block_table=t["block_table"],
                                           seqused_k=t["seqused_k"], num_heads_kv=2,
                                           scale=w.params["scale"], mask=1, window_left=window,
                                           softcap=softcap)
    _cmp(o, lse, o_ref, lse_ref, "qv window/softcap")


def test_prefill_qv_patch_mask():
    w = W.patch_cross(B=2, nbytes=600, H=4, D=64, seed=6)
    t = w.tensors
    qv = W.randn_bf16(tuple(t["q"].shape), 6, 43)
    o, lse = A.attn_fwd_varlen_paged_qv(t["q"].to(DEV), qv.to(DEV), t["k"].to(DEV), t["v"].to(DEV),
                                        cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                                        cu_seqlens_k=t["cu_seqlens_k"].to(DEV),
                                        max_seqlen_q=w.params["max_seqlen_q"], mask=A.MASK_PATCH,
                                        patch_kv_range=t["patch_kv_range"].to(DEV),
                                        scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_qv(t["q"], qv, t["k"], t["v"], cu_seqlens_q=t["cu_seqlens_q"],
                                           cu_seqlens_k=t["cu_seqlens_k"], num_heads_kv=4,
                                           scale=w.params["scale"], mask=2,
                                           patch_kv_range=t["patch_kv_range"])
    _cmp(o, lse, o_ref, lse_ref, "qv patch")


def test_prefill_qv_zero_qv_is_the_plain_forward():
    """qv = 0 removes the extra term: the result equals attn_fwd_varlen_paged's bit for bit."""
    lens = [200, 5, 384]
    w = W.varlen_paged_prefill(nseq=3, Hq=8, Hkv=2, D=128, num_blocks=100, lens=lens, lmax=512,
                               seed=12)
    t = {k: v.to(DEV) for k, v in w.tensors.items()}
    kw = dict(cu_seqlens_q=t["cu_seqlens_q"], max_seqlen_q=w.params["max_seqlen_q"],
              block_table=t["block_table"], seqused_k=t["seqused_k"], mask=A.MASK_CAUSAL,
              scale=w.params["scale"])
    o1, l1 = A.attn_fwd_varlen_paged_qv(t["q"], torch.zeros_like(t["q"]), t["k_cache"],
                                        t["v_cache"], **kw)
    o2, l2 = A.attn_fwd_varlen_paged(t["q"], t["k_cache"], t["v_cache"], **kw)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
