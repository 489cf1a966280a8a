"""The only_qv score path: CUDA path vs the fp64 oracle, element by element.

"Rope dim" (vllm-project flash-attention PR 172, overview) adds a mode that
skips the Q/K loads and the QK GEMM and builds the score from the Qv GEMM
alone: s_ij = scale * (qv_i . v_j).  The kernels read each value tile once
and use it for both GEMMs; the oracle computes the definition in fp64.

Tolerances as for the plain path (the arithmetic is the same: bf16 operands,
fp32 accumulation, bf16 output): max |O err| <= 2e-2, max |LSE err| <= 1e-3;
fp8 max |O err| <= 6e-2.
"""
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
    lse = np.asarray(lse.float().cpu().numpy(), np.float64)
    ninf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), ninf), what + ": -inf rows differ"
    if tol_lse is not None and (~ninf).any():
        err_l = float(np.max(np.abs(lse[~ninf] - lse_ref[~ninf])))
        assert err_l <= tol_lse, "%s: max|LSE err| %.3g > %.3g" % (what, err_l, tol_lse)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4)])
def test_prefill_paged_only_qv(D, causal, Hq, Hkv):
    lens = [1, 17, 129, 300, 64, 255]
    w = W.varlen_paged_prefill(nseq=len(lens), Hq=Hq, Hkv=Hkv, D=D, num_blocks=200, lens=lens,
                               lmax=512, seed=D + Hq + causal)
    t = w.tensors
    mask = A.MASK_CAUSAL if causal else A.MASK_NONE
    o, lse = A.attn_fwd_varlen_paged_only_qv(t["q"].to(DEV), t["v_cache"].to(DEV),
                                             cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                                             max_seqlen_q=w.params["max_seqlen_q"],
                                             block_table=t["block_table"].to(DEV),
                                             seqused_k=t["seqused_k"].to(DEV), mask=mask,
                                             scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_qv(None, t["q"], None, t["v_cache"],
                                           cu_seqlens_q=t["cu_seqlens_q"], block_table=t["block_table"],
                                           seqused_k=t["seqused_k"], num_heads_kv=Hkv,
                                           scale=w.params["scale"], mask=int(mask), only_qv=True)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "paged only_qv")


def test_prefill_packed_only_qv_lq_lt_lk():
    """Packed store, bottom-right causal with fewer queries than keys, an empty sequence."""
    lq, lk = [130, 0, 5, 77], [300, 9, 200, 77]
    Hq, Hkv, D = 4, 1, 128
    cq, ck = W.cu_from_lens(lq), W.cu_from_lens(lk)
    qv = W.randn_bf16((int(cq[-1]), Hq, D), 3, 1)
    v = W.randn_bf16((int(ck[-1]), Hkv, D), 3, 2)
    o, lse = A.attn_fwd_varlen_paged_only_qv(qv.to(DEV), v.to(DEV), cu_seqlens_q=cq.to(DEV),
                                             cu_seqlens_k=ck.to(DEV), max_seqlen_q=max(lq),
                                             mask=A.MASK_CAUSAL, scale=0.1)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_qv(None, qv, None, v, cu_seqlens_q=cq, cu_seqlens_k=ck,
                                           num_heads_kv=Hkv, scale=0.1, mask=1, only_qv=True)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "packed only_qv")


@pytest.mark.parametrize("window,softcap", [(100, 0.0), (-1, 30.0), (40, 20.0)])
def test_prefill_only_qv_window_softcap(window, softcap):
    lens = [33, 400, 129]
    w = W.varlen_paged_prefill(nseq=3, Hq=8, Hkv=2, D=128, num_blocks=100, lens=lens, lmax=512,
                               seed=window + 7)
    t = w.tensors
    # larger logits, so that the cap bites (x3 rounded to bf16 on both sides)
    qv = (t["q"].float() * 3).to(torch.bfloat16)
    o, lse = A.attn_fwd_varlen_paged_only_qv(qv.to(DEV), t["v_cache"].to(DEV),
                                             cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                                             max_seqlen_q=w.params["max_seqlen_q"],
                                             block_table=t["block_table"].to(DEV),
                                             seqused_k=t["seqused_k"].to(DEV), mask=A.MASK_CAUSAL,
                                             scale=w.params["scale"], window_left=window,
                                             softcap=softcap)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_qv(None, qv, None, t["v_cache"], cu_seqlens_q=t["cu_seqlens_q"],
                                           block_table=t["block_table"], seqused_k=t["seqused_k"],
                                           num_heads_kv=2, scale=w.params["scale"], mask=1,
                                           window_left=window, softcap=softcap, only_qv=True)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "only_qv window/softcap")


def test_prefill_only_qv_patch_mask():
    w = W.patch_cross(B=2, nbytes=600, H=4, D=64, seed=5)
    t = w.tensors
    o, lse = A.attn_fwd_varlen_paged_only_qv(t["q"].to(DEV), t["v"].to(DEV),
                                             cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                                             cu_seqlens_k=t["cu_seqlens_k"].to(DEV),
                                             max_seqlen_q=w.params["max_seqlen_q"], mask=A.MASK_PATCH,
                                             patch_kv_range=t["patch_kv_range"].to(DEV),
                                             scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_qv(None, t["q"], None, t["v"], cu_seqlens_q=t["cu_seqlens_q"],
                                           cu_seqlens_k=t["cu_seqlens_k"], num_heads_kv=4,
                                           scale=w.params["scale"], mask=2,
                                           patch_kv_range=t["patch_kv_range"], only_qv=True)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "only_qv patch")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_only_qv_fp8(causal, D):
    """e4m3 qv and v with per-tensor descales; the score uses descale_qv * descale_v."""
    lens = [128, 400]
    Hq, Hkv = 4, 2
    cu = W.cu_from_lens(lens)
    qv = W.randn_bf16((int(cu[-1]), Hq, D), 11, 1)
    v = W.randn_bf16((int(cu[-1]), Hkv, D), 11, 2)
    qf, dq = W.quantize_e4m3(qv)
    vf, dv = W.quantize_e4m3(v)
    o, lse = A.attn_fwd_varlen_paged_only_qv(qf.to(DEV), vf.to(DEV), cu_seqlens_q=cu.to(DEV),
                                             cu_seqlens_k=cu.to(DEV), max_seqlen_q=max(lens),
                                             mask=A.MASK_CAUSAL if causal else A.MASK_NONE,
                                             scale=1 / D ** 0.5, descale_qv=dq.to(DEV),
                                             descale_v=dv.to(DEV))
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_qv(None, oracle.dequant_e4m3(qf, dq), None,
                                           oracle.dequant_e4m3(vf, dv), cu_seqlens_q=cu, cu_seqlens_k=cu,
                                           num_heads_kv=Hkv, scale=1 / D ** 0.5, mask=int(causal),
                                           only_qv=True)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_FP8, None, "only_qv fp8")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("splits", [0, 1, 3])
@pytest.mark.parametrize("window", [-1, 50])
def test_decode_only_qv(D, splits, window):
    lens = [0, 1, 15, 16, 17, 100, 513, 1000]
    w = W.paged_decode(B=len(lens), Hq=32, Hkv=8, D=D, num_blocks=300, lmax=1024, lens=lens,
                       seed=D + splits)
    t = w.tensors
    o, lse = A.attn_decode_paged_only_qv(t["q"].to(DEV), t["v_cache"].to(DEV), t["block_table"].to(DEV),
                                         t["seqused_k"].to(DEV), scale=w.params["scale"],
                                         num_splits=splits, window_left=window)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    # the decode query is the newest cached token: causal, one row per sequence
    B = len(lens)
    su = t["seqused_k"]
    o_ref, lse_ref = oracle.attn_varlen_qv(None, t["q"], None, t["v_cache"],
                                           cu_seqlens_q=W.cu_from_lens([1] * B), block_table=t["block_table"],
                                           seqused_k=su, num_heads_kv=8, scale=w.params["scale"], mask=1,
                                           window_left=window, only_qv=True)
    # rows of empty sequences: the oracle has none (Lq 1, Lk 0 -> -inf), the kernel writes 0 / -inf
    _cmp(o, lse.T.contiguous(), o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "decode only_qv")


def test_decode_only_qv_equals_decode_with_keys_equal_to_values():
    """The fused path gives the plain decode's result on a cache whose keys are the values."""
    w = W.paged_decode(B=16, Hq=16, Hkv=4, D=128, num_blocks=2400, lmax=2048, seed=9)
    t = w.tensors
    q, v, bt, su = (t[n].to(DEV) for n in ("q", "v_cache", "block_table", "seqused_k"))
    o1, l1 = A.attn_decode_paged_only_qv(q, v, bt, su, scale=0.05)
    o2, l2 = A.attn_decode_paged(q, v, v, bt, su, scale=0.05)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _compact(v_cache, bt_row, n_keys):
    """The pages one sequence uses, as a small pool with its own (identity) block table."""
    n = (int(n_keys) + 15) // 16
    return v_cache[bt_row[:n].long()], torch.arange(n, dtype=torch.int32)[None]


def test_config_only_qv_decode_full():
    """only_qv paged decode at the bench's size: B=32, Hq=32, Hkv=8, D=128, L ~ U[1,8192],
    20000-page pool, automatic splits (sampled sequences)."""
    w = W.FULL_SIZE["paged_gqa_decode_bf16"]()
    t = w.tensors
    o, lse = A.attn_decode_paged_only_qv(t["q"].to(DEV), t["v_cache"].to(DEV), t["block_table"].to(DEV),
                                         t["seqused_k"].to(DEV), scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    lens = t["seqused_k"].numpy()
    sample = sorted(set([int(np.argmax(lens)), int(np.argmin(lens))] +
                        list(np.random.default_rng(2).choice(len(lens), 5, replace=False))))
    for b in sample:
        vc, bt = _compact(t["v_cache"], t["block_table"][b], lens[b])
        o_ref, lse_ref = oracle.attn_varlen_qv(None, t["q"][b:b + 1], None, vc, cu_seqlens_q=[0, 1],
                                               block_table=bt, seqused_k=[int(lens[b])], num_heads_kv=8,
                                               scale=w.params["scale"], mask=0, only_qv=True)
        _cmp(o[b:b + 1], lse[b:b + 1].T.contiguous(), o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16,
             "only_qv decode b%d" % b)


def test_config_only_qv_prefill_full():
    """only_qv varlen paged causal prefill at the bench's size (sampled rows: row i of a
    sequence is unmasked only_qv attention over its keys 0..i)."""
    w = W.FULL_SIZE["varlen_paged_gqa_prefill_causal_bf16"]()
    t = w.tensors
    o, lse = A.attn_fwd_varlen_paged_only_qv(t["q"].to(DEV), t["v_cache"].to(DEV),
                                             cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                                             max_seqlen_q=w.params["max_seqlen_q"],
                                             block_table=t["block_table"].to(DEV),
                                             seqused_k=t["seqused_k"].to(DEV), mask=A.MASK_CAUSAL,
                                             scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    cu = t["cu_seqlens_q"].numpy()
    rng = np.random.default_rng(3)
    for b in range(0, 16, 3):
        L = cu[b + 1] - cu[b]
        for i in sorted(set([0, L - 1, int(rng.integers(0, L)), min(128, L - 1)])):
            r = cu[b] + i
            vc, bt = _compact(t["v_cache"], t["block_table"][b], i + 1)
            o_ref, lse_ref = oracle.attn_varlen_qv(None, t["q"][r:r + 1], None, vc, cu_seqlens_q=[0, 1],
                                                   block_table=bt, seqused_k=[i + 1], num_heads_kv=8,
                                                   scale=w.params["scale"], mask=0, only_qv=True)
            assert np.max(np.abs(o[r] - o_ref[0])) <= TOL_O_BF16, (b, i)
            assert np.max(np.abs(lse[:, r] - lse_ref[:, 0])) <= TOL_LSE_BF16, (b, i)
