"""fp8 e4m3 varlen forward (paged and packed K/V, causal, none and patch masks) vs the
fp64 oracle fed the dequantised values, at head_dim 64 and 128.

At head_dim 64 an e4m3 row is 64 bytes: the kernel's tiles then use the 64-byte
swizzle (TMA maps and tcgen05 descriptors), a layout of its own.  The fp8 operands
are per-tensor quantised ("[FlexAttention] Enforce Q,K,V memory layouts for fp8
flex attention": both GEMMs in the query dtype).  Tolerance max |O - O_ref| <= 6e-2.
"""
import numpy as np
import pytest
import torch

import oracle
from attention_paged_kv_gqa_b200 import binding as A
from attention_paged_kv_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_O_FP8 = 6e-2
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert A.attn_check_device(0) == 0, "not a B200 or the kernel image does not load"
    torch.cuda.set_device(0)


def _cmp(o, lse, o_ref, lse_ref, what):
    o = np.asarray(o.float().cpu().numpy(), np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), what + ": non-finite output"
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    assert err_o <= TOL_O_FP8, "%s: max|O err| %.3g" % (what, err_o)
    lse = np.asarray(lse.float().cpu().numpy(), np.float64)
    ninf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), ninf), what + ": -inf rows differ"
    assert np.all(o[np.moveaxis(ninf, 0, 1)] == 0.0), what + ": empty rows not zero"


def _q8(x):
    codes, ds = W.quantize_e4m3(x)
    return codes, ds, oracle.dequant_e4m3(codes, ds)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4), (3, 1)])
def test_fp8_varlen_paged(D, causal, Hq, Hkv):
    lens = [1, 17, 129, 300, 64, 255, 513]
    w = W.varlen_paged_prefill(nseq=len(lens), Hq=Hq, Hkv=Hkv, D=D, num_blocks=300, lens=lens,
                               lmax=640, seed=5 * D + Hq + causal)
    t = w.tensors
    q8, dq, qd = _q8(t["q"])
    k8, dk, kd = _q8(t["k_cache"])
    v8, dv, vd = _q8(t["v_cache"])
    mask = A.MASK_CAUSAL if causal else A.MASK_NONE
    o, lse = A.attn_fwd_varlen_paged(q8.to(DEV), k8.to(DEV), v8.to(DEV),
                                     cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                                     max_seqlen_q=w.params["max_seqlen_q"],
                                     block_table=t["block_table"].to(DEV),
                                     seqused_k=t["seqused_k"].to(DEV), mask=mask,
                                     scale=w.params["scale"], descale_q=dq.to(DEV),
                                     descale_k=dk.to(DEV), descale_v=dv.to(DEV))
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen(qd, kd, vd, cu_seqlens_q=t["cu_seqlens_q"],
                                        block_table=t["block_table"], seqused_k=t["seqused_k"],
                                        num_heads_kv=Hkv, scale=w.params["scale"], mask=int(mask))
    _cmp(o, lse, o_ref, lse_ref, "fp8 paged D%d Hq%d Hkv%d causal %d" % (D, Hq, Hkv, causal))


def test_fp8_packed_lq_lt_lk_d64():
    """Packed store, bottom-right causal with fewer queries than keys, an empty sequence."""
    lq, lk = [130, 0, 5, 77], [300, 9, 200, 77]
    Hq, Hkv, D = 4, 1, 64
    cq, ck = W.cu_from_lens(lq), W.cu_from_lens(lk)
    q8, dq, qd = _q8(W.randn_bf16((int(cq[-1]), Hq, D), 8, 1))
    k8, dk, kd = _q8(W.randn_bf16((int(ck[-1]), Hkv, D), 8, 2))
    v8, dv, vd = _q8(W.randn_bf16((int(ck[-1]), Hkv, D), 8, 3))
    o, lse = A.attn_fwd_varlen_paged(q8.to(DEV), k8.to(DEV), v8.to(DEV), cu_seqlens_q=cq.to(DEV),
                                     cu_seqlens_k=ck.to(DEV), max_seqlen_q=max(lq),
                                     mask=A.MASK_CAUSAL, scale=0.125, descale_q=dq.to(DEV),
                                     descale_k=dk.to(DEV), descale_v=dv.to(DEV))
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen(qd, kd, vd, cu_seqlens_q=cq, cu_seqlens_k=ck,
                                        num_heads_kv=Hkv, scale=0.125, mask=1)
    _cmp(o, lse, o_ref, lse_ref, "fp8 packed D64")


def test_fp8_patch_d64():
    """The patch mask with e4m3 operands at head_dim 64 (the tiled kernel)."""
    w = W.patch_cross(B=2, nbytes=600, H=4, D=64, seed=9)
    t = w.tensors
    q8, dq, qd = _q8(t["q"])
    k8, dk, kd = _q8(t["k"])
    v8, dv, vd = _q8(t["v"])
    o, lse = A.attn_fwd_patch(q8.to(DEV), k8.to(DEV), v8.to(DEV),
                              cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                              cu_seqlens_k=t["cu_seqlens_k"].to(DEV),
                              patch_kv_range=t["patch_kv_range"].to(DEV),
                              max_seqlen_q=w.params["max_seqlen_q"], max_interval=16,
                              scale=w.params["scale"], descale_q=dq.to(DEV), descale_k=dk.to(DEV),
                              descale_v=dv.to(DEV))
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen(qd, kd, vd, cu_seqlens_q=t["cu_seqlens_q"],
                                        cu_seqlens_k=t["cu_seqlens_k"], num_heads_kv=4,
                                        scale=w.params["scale"], mask=2,
                                        patch_kv_range=t["patch_kv_range"])
    _cmp(o, lse, o_ref, lse_ref, "fp8 patch D64")
