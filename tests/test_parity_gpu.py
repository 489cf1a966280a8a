"""CUDA path vs the fp64 oracle, element by element on the same seeded inputs.

Tolerances (against fp64, after the kernel's bf16 output rounding):
  bf16 inputs: max |O - O_ref| <= 2e-2, max |LSE - LSE_ref| <= 1e-3
  fp8 e4m3 inputs (oracle fed the same dequantised values): max |O - O_ref| <= 6e-2
Rows with no allowed key must give O == 0 and LSE == -inf exactly.
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
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    assert np.all(np.isfinite(o)), what + ": non-finite output"
    assert err_o <= tol_o, "%s: max|O err| %.3g > %.3g" % (what, err_o, tol_o)
    if lse is not None:
        lse = np.asarray(lse.float().cpu().numpy(), np.float64)
        ninf = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse), ninf), what + ": -inf rows differ"
        if tol_lse is not None and (~ninf).any():
            err_l = float(np.max(np.abs(lse[~ninf] - lse_ref[~ninf])))
            assert err_l <= tol_lse, "%s: max|LSE err| %.3g > %.3g" % (what, err_l, tol_lse)
    return err_o


def _no_device_error():
    assert A.attn_device_error() == 0


# ---------------------------------------------------------------------------- dense
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("L", [1, 15, 128, 129, 300])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (3, 1), (8, 2)])
def test_dense_bf16_small(D, L, causal, Hq, Hkv):
    w = W.dense(B=2, L=L, Hq=Hq, Hkv=Hkv, D=D, causal=causal, seed=L * 7 + D)
    t = w.tensors
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    o, lse = A.attn_fwd_dense(q, k, v, causal=causal, scale=w.params["scale"])
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_dense(t["q"], t["k"], t["v"], scale=w.params["scale"], causal=causal)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "dense D%d L%d" % (D, L))
    _no_device_error()


@pytest.mark.parametrize("Lq,Lk", [(5, 200), (130, 300), (64, 1)])
def test_dense_causal_bottom_right_lq_lt_lk(Lq, Lk):
    w = W.dense(B=2, L=Lq, Lk=Lk, Hq=2, Hkv=1, D=64, causal=True, seed=Lq + Lk)
    t = w.tensors
    o, lse = A.attn_fwd_dense(t["q"].to(DEV), t["k"].to(DEV), t["v"].to(DEV), causal=True,
                              scale=0.125)
    o_ref, lse_ref = oracle.attn_dense(t["q"], t["k"], t["v"], scale=0.125, causal=True)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "bottom-right")


def test_dense_causal_lq_gt_lk_has_empty_rows():
    """Lq > Lk with bottom-right alignment: the first Lq-Lk rows see no key -> O 0, LSE -inf."""
    w = W.dense(B=1, L=200, Lk=70, Hq=2, Hkv=2, D=64, causal=True, seed=3)
    t = w.tensors
    o, lse = A.attn_fwd_dense(t["q"].to(DEV), t["k"].to(DEV), t["v"].to(DEV), causal=True)
    o_ref, lse_ref = oracle.attn_dense(t["q"], t["k"], t["v"], scale=1 / 8, causal=True)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "empty rows")
    assert torch.all(o[:, :130] == 0)


def test_dense_strided_inputs():
    """Q/K/V given as views with non-packed strides (a [B, L, 3, H, D] qkv buffer)."""
    B, L, H, D = 2, 140, 2, 64
    qkv = W.randn_bf16((B, L, 3, H, D), seed=5, stream=1)
    q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    d = qkv.to(DEV)
    o, lse = A.attn_fwd_dense(d[:, :, 0], d[:, :, 1], d[:, :, 2], causal=True)
    o_ref, lse_ref = oracle.attn_dense(q, k, v, scale=1 / 8, causal=True)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "strided")


def test_default_scale_is_inverse_sqrt_d():
    w = W.dense(B=1, L=64, Hq=2, Hkv=2, D=128, causal=False, seed=9)
    t = w.tensors
    o1, l1 = A.attn_fwd_dense(t["q"].to(DEV), t["k"].to(DEV), t["v"].to(DEV), scale=None)
    o2, l2 = A.attn_fwd_dense(t["q"].to(DEV), t["k"].to(DEV), t["v"].to(DEV),
                              scale=1 / math.sqrt(128))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_config_dense_causal_full():
    """Dense causal bf16, B=2, Hq=Hkv=2, L=128, D=64 (full size, every output)."""
    w = W.FULL_SIZE["dense_causal_bf16"]()
    t = w.tensors
    o, lse = A.attn_fwd_dense(t["q"].to(DEV), t["k"].to(DEV), t["v"].to(DEV), causal=True,
                              scale=w.params["scale"])
    o_ref, lse_ref = oracle.attn_dense(t["q"], t["k"], t["v"], scale=w.params["scale"], causal=True)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "dense causal full")
    _no_device_error()


# ---------------------------------------------------------------------------- varlen / paged
def _run_varlen(w, mask, paged=True, patch=None):
    t = w.tensors
    kw = dict(cu_seqlens_q=t["cu_seqlens_q"].to(DEV), max_seqlen_q=w.params["max_seqlen_q"],
              mask=mask, scale=w.params["scale"])
    if paged:
        kw.update(block_table=t["block_table"].to(DEV), seqused_k=t["seqused_k"].to(DEV))
        kc, vc = t["k_cache"].to(DEV), t["v_cache"].to(DEV)
    else:
        kw.update(cu_seqlens_k=t["cu_seqlens_k"].to(DEV))
        kc, vc = t["k"].to(DEV), t["v"].to(DEV)
    if patch is not None:
        kw["patch_kv_range"] = patch.to(DEV)
    return A.attn_fwd_varlen_paged(t["q"].to(DEV), kc, vc, **kw)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4), (6, 2)])
@pytest.mark.parametrize("causal", [True, False])
def test_varlen_paged_small(D, Hq, Hkv, causal):
    lens = [1, 16, 17, 129, 255, 64, 300]
    w = W.varlen_paged_prefill(nseq=len(lens), Hq=Hq, Hkv=Hkv, D=D, num_blocks=200,
                               lens=lens, lmax=320, seed=D + Hq)
    t = w.tensors
    o, lse = _run_varlen(w, A.MASK_CAUSAL if causal else A.MASK_NONE)
    o_ref, lse_ref = oracle.attn_varlen(t["q"], t["k_cache"], t["v_cache"],
                                        cu_seqlens_q=t["cu_seqlens_q"], seqused_k=t["seqused_k"],
                                        block_table=t["block_table"], num_heads_kv=Hkv,
                                        scale=w.params["scale"], mask=1 if causal else 0)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "varlen paged")
    _no_device_error()


def test_varlen_packed_kv_and_empty_sequences():
    """Packed (non-paged) K/V, with a zero-length query sequence and a zero-length key sequence."""
    lq = [5, 0, 130, 7]
    lk = [5, 3, 130, 0]
    Hq, Hkv, D = 4, 2, 64
    cq, ck = W.cu_from_lens(lq), W.cu_from_lens(lk)
    q = W.randn_bf16((int(cq[-1]), Hq, D), 1, 1)
    k = W.randn_bf16((int(ck[-1]), Hkv, D), 1, 2)
    v = W.randn_bf16((int(ck[-1]), Hkv, D), 1, 3)
    o, lse = A.attn_fwd_varlen_paged(q.to(DEV), k.to(DEV), v.to(DEV), cu_seqlens_q=cq.to(DEV),
                                     cu_seqlens_k=ck.to(DEV), max_seqlen_q=130,
                                     mask=A.MASK_NONE, scale=0.125)
    o_ref, lse_ref = oracle.attn_varlen(q, k, v, cu_seqlens_q=cq, cu_seqlens_k=ck,
                                        num_heads_kv=Hkv, scale=0.125, mask=0)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "packed")
    assert torch.all(o[int(cq[3]):] == 0) and torch.all(torch.isneginf(lse[:, int(cq[3]):]))


def test_paged_tail_page_garbage_is_ignored():
    """Rows of the last page past the sequence end hold NaN: results must not change."""
    lens = [17, 40, 3]
    w = W.varlen_paged_prefill(nseq=3, Hq=4, Hkv=2, D=128, num_blocks=40, lens=lens, lmax=64,
                               seed=11)
    t = w.tensors
    bt = t["block_table"]
    for b, L in enumerate(lens):
        last = int(bt[b, (L - 1) // 16])
        t["k_cache"][last, L % 16 or 16:] = float("nan")
        t["v_cache"][last, L % 16 or 16:] = float("nan")
    o, lse = _run_varlen(w, A.MASK_CAUSAL)
    tc = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in t.items()}
    tc["k_cache"] = torch.nan_to_num(t["k_cache"], nan=0.0)
    tc["v_cache"] = torch.nan_to_num(t["v_cache"], nan=0.0)
    o_ref, lse_ref = oracle.attn_varlen(tc["q"], tc["k_cache"], tc["v_cache"],
                                        cu_seqlens_q=t["cu_seqlens_q"], seqused_k=t["seqused_k"],
                                        block_table=bt, num_heads_kv=2, scale=w.params["scale"],
                                        mask=1)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "nan tail")


def test_patch_small_with_empty_and_unit_intervals():
    w = W.patch_cross(B=2, nbytes=700, H=2, D=64, seed=4)
    t = w.tensors
    pr = t["patch_kv_range"].clone()
    pr[3] = torch.tensor([5, 5])        # empty interval -> O 0, LSE -inf
    pr[7] = torch.tensor([10, 11])      # single key -> that V row
    o, lse = _run_varlen(w, A.MASK_PATCH, paged=False, patch=pr)
    o_ref, lse_ref = oracle.attn_varlen(t["q"], t["k"], t["v"], cu_seqlens_q=t["cu_seqlens_q"],
                                        cu_seqlens_k=t["cu_seqlens_k"], num_heads_kv=2,
                                        scale=w.params["scale"], mask=2, patch_kv_range=pr)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "patch small")
    assert torch.all(o[3] == 0) and torch.all(torch.isneginf(lse[:, 3]))


# ---------------------------------------------------------------------------- decode
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 8), (16, 2), (16, 1)])
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_decode_small(D, Hq, Hkv, splits):
    lens = [1, 15, 16, 17, 1000, 64, 65, 513]
    w = W.paged_decode(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, num_blocks=200, lmax=1024, lens=lens,
                       seed=D + Hq + splits)
    t = w.tensors
    o, lse = A.attn_decode_paged(t["q"].to(DEV), t["k_cache"].to(DEV), t["v_cache"].to(DEV),
                                 t["block_table"].to(DEV), t["seqused_k"].to(DEV),
                                 scale=w.params["scale"], num_splits=splits)
    o_ref, lse_ref = oracle.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                        t["seqused_k"], scale=w.params["scale"])
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "decode")
    _no_device_error()


def test_decode_zero_length_sequence():
    lens = [0, 5, 0, 100]
    w = W.paged_decode(B=4, Hq=8, Hkv=2, D=128, num_blocks=20, lmax=128, lens=lens, seed=2)
    t = w.tensors
    for splits in (0, 1):
        o, lse = A.attn_decode_paged(t["q"].to(DEV), t["k_cache"].to(DEV), t["v_cache"].to(DEV),
                                     t["block_table"].to(DEV), t["seqused_k"].to(DEV),
                                     num_splits=splits)
        assert torch.all(o[0] == 0) and torch.all(o[2] == 0)
        assert torch.all(torch.isneginf(lse[0])) and torch.all(torch.isneginf(lse[2]))
        o_ref, lse_ref = oracle.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                            t["seqused_k"], scale=1 / math.sqrt(128))
        _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "decode zero")


# ---------------------------------------------------------------------------- full-size workloads
def _compact_pages(k_cache, v_cache, bt_row, n_keys):
    """The pages one sequence uses, as a small pool with its own (identity) block table."""
    n = (int(n_keys) + 15) // 16
    pages = bt_row[:n].long()
    bt = torch.arange(n, dtype=torch.int32)[None]
    return k_cache[pages], v_cache[pages], bt


def _prefix_rows_ref(q_rows, k_cache, v_cache, bt_row, n_keys, Hkv, scale):
    """Oracle for one causal query row i (Lq == Lk): unmasked attention over keys 0..i.

    The identity 'causal row i == unmasked attention over the prefix 0..i' is
    pinned by the oracle tests.
    """
    kc, vc, bt = _compact_pages(k_cache, v_cache, bt_row, n_keys)
    cq = np.array([0, 1], np.int32)
    o, lse = oracle.attn_varlen(q_rows[None], kc, vc, cu_seqlens_q=cq,
                                seqused_k=np.array([n_keys], np.int32),
                                block_table=bt, num_heads_kv=Hkv, scale=scale, mask=0)
    return o[0], lse[:, 0]


def test_config_paged_decode_full():
    """Paged GQA decode, B=32, Hq=32, Hkv=8, D=128, L ~ U[1,8192], 20000-page pool (auto splits)."""
    w = W.FULL_SIZE["paged_gqa_decode_bf16"]()
    t = w.tensors
    d = {k: v.to(DEV) for k, v in t.items()}
    o, lse = A.attn_decode_paged(d["q"], d["k_cache"], d["v_cache"], d["block_table"],
                                 d["seqused_k"], scale=w.params["scale"])
    torch.cuda.synchronize()
    _no_device_error()
    lens = t["seqused_k"].numpy()
    for b in range(len(lens)):                       # every sequence, element by element
        kc, vc, bt = _compact_pages(t["k_cache"], t["v_cache"], t["block_table"][b], lens[b])
        o_ref, lse_ref = oracle.attn_decode(t["q"][b:b + 1], kc, vc, bt, t["seqused_k"][b:b + 1],
                                            scale=w.params["scale"])
        _cmp(o[b:b + 1], lse[b:b + 1], o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "decode b%d" % b)


def test_config_varlen_paged_prefill_full():
    """Varlen paged GQA prefill, causal, 16 seqs, L ~ U[64,4096], Hq=32, Hkv=8, D=128: the
    longest sequence whole (every row, all 32 heads) and sampled rows of the others."""
    w = W.FULL_SIZE["varlen_paged_gqa_prefill_causal_bf16"]()
    t = w.tensors
    o, lse = _run_varlen(w, A.MASK_CAUSAL)
    torch.cuda.synchronize()
    _no_device_error()
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    cu = t["cu_seqlens_q"].numpy()
    lens = t["seqused_k"].numpy()
    bl = int(np.argmax(lens))
    L = int(lens[bl])
    kc, vc, bt = _compact_pages(t["k_cache"], t["v_cache"], t["block_table"][bl], L)
    o_ref, lse_ref = oracle.attn_varlen(t["q"][cu[bl]:cu[bl + 1]], kc, vc,
                                        cu_seqlens_q=np.array([0, L], np.int32),
                                        seqused_k=np.array([L], np.int32), block_table=bt,
                                        num_heads_kv=8, scale=w.params["scale"], mask=1)
    _cmp(torch.from_numpy(o[cu[bl]:cu[bl + 1]]), torch.from_numpy(lse[:, cu[bl]:cu[bl + 1]]),
         o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16,
         "varlen prefill, whole sequence %d (%d rows)" % (bl, L))
    rng = np.random.default_rng(1)
    for b in range(16):
        if b == bl:
            continue
        L = cu[b + 1] - cu[b]
        for i in sorted(set([0, L - 1, int(rng.integers(0, L)), min(127, L - 1), min(128, L - 1)])):
            r = cu[b] + i
            o_ref, lse_ref = _prefix_rows_ref(t["q"][r], t["k_cache"], t["v_cache"],
                                              t["block_table"][b], i + 1, 8, w.params["scale"])
            assert np.max(np.abs(o[r] - o_ref)) <= TOL_O_BF16, (b, i)
            assert np.max(np.abs(lse[:, r] - lse_ref)) <= TOL_LSE_BF16, (b, i)


def _patch_every_query_ref(t, scale):
    """The oracle for every query of the patch workload: query q attends exactly the bytes
    start_q <= j < end_q of its sequence, so with the keys of each patch as a sequence of
    its own (patches partition the bytes in order) it is unmasked attention over them."""
    cq = t["cu_seqlens_q"].numpy()
    r = t["patch_kv_range"].numpy().astype(np.int64)
    seq = np.repeat(np.arange(len(cq) - 1), np.diff(cq))
    starts = seq * 8192 + r[:, 0]
    ck = np.concatenate([starts, [starts[-1] + (r[-1, 1] - r[-1, 0])]]).astype(np.int32)
    assert np.all(np.diff(ck) == r[:, 1] - r[:, 0])
    return oracle.attn_varlen(t["q"], t["k"], t["v"],
                              cu_seqlens_q=np.arange(len(r) + 1, dtype=np.int32),
                              cu_seqlens_k=ck, num_heads_kv=16, scale=scale, mask=0)


def test_config_patch_cross_attention_full():
    """Patch cross-attention, B=4 x 8192 bytes, Geom(0.22) patches, H=16, D=64: every query
    (tiled kernel), and sampled queries against the oracle's patch mask itself."""
    w = W.FULL_SIZE["patch_cross_attention_bf16"]()
    t = w.tensors
    o, lse = _run_varlen(w, A.MASK_PATCH, paged=False, patch=t["patch_kv_range"])
    torch.cuda.synchronize()
    _no_device_error()
    o_all, lse_all = _patch_every_query_ref(t, w.params["scale"])
    _cmp(o, lse, o_all, lse_all, TOL_O_BF16, TOL_LSE_BF16, "patch, every query")
    cq = t["cu_seqlens_q"].numpy()
    rng = np.random.default_rng(2)
    for b in range(4):
        rows = np.unique(np.concatenate([[cq[b], cq[b + 1] - 1],
                                         rng.integers(cq[b], cq[b + 1], size=40)]))
        qs = t["q"][rows]
        k = t["k"][b * 8192:(b + 1) * 8192]
        v = t["v"][b * 8192:(b + 1) * 8192]
        o_ref, lse_ref = oracle.attn_varlen(qs, k, v, cu_seqlens_q=np.array([0, len(rows)], np.int32),
                                            cu_seqlens_k=np.array([0, 8192], np.int32),
                                            num_heads_kv=16, scale=w.params["scale"], mask=2,
                                            patch_kv_range=t["patch_kv_range"][rows])
        _cmp(o[rows], lse[:, rows], o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "patch b%d" % b)


def test_config_fp8_dense_causal_full():
    """fp8 e4m3 dense causal B=4, H=16, L=4096, D=128; plus the bf16 run on the same data."""
    w = W.FULL_SIZE["fp8_e4m3_dense_causal"]()
    t = w.tensors
    dq, dk, dv = (t["descale_" + n].to(DEV) for n in "qkv")
    o8, lse8 = A.attn_fwd_dense(t["q_fp8"].to(DEV), t["k_fp8"].to(DEV), t["v_fp8"].to(DEV),
                                causal=True, scale=w.params["scale"], descale_q=dq, descale_k=dk,
                                descale_v=dv)
    o16, lse16 = A.attn_fwd_dense(t["q"].to(DEV), t["k"].to(DEV), t["v"].to(DEV), causal=True,
                                  scale=w.params["scale"])
    torch.cuda.synchronize()
    _no_device_error()
    qd = oracle.dequant_e4m3(t["q_fp8"], t["descale_q"])
    kd = oracle.dequant_e4m3(t["k_fp8"], t["descale_k"])
    vd = oracle.dequant_e4m3(t["v_fp8"], t["descale_v"])
    rng = np.random.default_rng(3)
    o8, o16 = o8.float().cpu().numpy(), o16.float().cpu().numpy()
    lse8, lse16 = lse8.cpu().numpy(), lse16.cpu().numpy()
    # batch element 0 whole (4096 rows x 16 heads), in fp8 and in bf16
    for name, (qq, kk, vv), oo, ll, tol_o, tol_l in (
            ("fp8", (qd, kd, vd), o8, lse8, TOL_O_FP8, None),
            ("bf16", (t["q"], t["k"], t["v"]), o16, lse16, TOL_O_BF16, TOL_LSE_BF16)):
        ref_o, ref_l = oracle.attn_dense(qq[0:1], kk[0:1], vv[0:1], scale=w.params["scale"],
                                         causal=True)
        assert np.max(np.abs(oo[0] - ref_o[0])) <= tol_o, (name, "whole batch element 0")
        if tol_l is not None:
            assert np.max(np.abs(ll[0] - ref_l[0])) <= tol_l, (name, "whole batch element 0")
    for b in range(1, 4):
        for i in sorted(set([0, 1, 2, 127, 128, 4095, int(rng.integers(0, 4096))])):
            for name, (qq, kk, vv), oo, ll, tol_o, tol_l in (
                    ("fp8", (qd, kd, vd), o8, lse8, TOL_O_FP8, None),
                    ("bf16", (t["q"], t["k"], t["v"]), o16, lse16, TOL_O_BF16, TOL_LSE_BF16)):
                ref_o, ref_l = oracle.attn_varlen(
                    qq[b, i][None], kk[b, :i + 1], vv[b, :i + 1],
                    cu_seqlens_q=np.array([0, 1], np.int32),
                    cu_seqlens_k=np.array([0, i + 1], np.int32), num_heads_kv=16,
                    scale=w.params["scale"], mask=0)
                assert np.max(np.abs(oo[b, i] - ref_o[0])) <= tol_o, (name, b, i)
                if tol_l is not None:
                    assert np.max(np.abs(ll[b, :, i] - ref_l[:, 0])) <= tol_l, (name, b, i)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("L", [1, 100, 129, 300, 777])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (3, 1)])
def test_dense_fp8_small(L, causal, Hq, Hkv, D):
    """fp8 e4m3 dense attention over several 128-key tiles with a ragged tail, every
    output element against the oracle fed the dequantised values."""
    w = W.dense(B=2, L=L, Hq=Hq, Hkv=Hkv, D=D, causal=causal, seed=11 * L + Hq + D)
    t = w.tensors
    qf, dq = W.quantize_e4m3(t["q"])
    kf, dk = W.quantize_e4m3(t["k"])
    vf, dv = W.quantize_e4m3(t["v"])
    o, lse = A.attn_fwd_dense(qf.to(DEV), kf.to(DEV), vf.to(DEV), causal=causal,
                              scale=w.params["scale"], descale_q=dq.to(DEV), descale_k=dk.to(DEV),
                              descale_v=dv.to(DEV))
    torch.cuda.synchronize()
    _no_device_error()
    o_ref, lse_ref = oracle.attn_dense(oracle.dequant_e4m3(qf, dq), oracle.dequant_e4m3(kf, dk),
                                       oracle.dequant_e4m3(vf, dv), scale=w.params["scale"],
                                       causal=causal)
    _cmp(o, lse, o_ref, lse_ref, TOL_O_FP8, None, "fp8 dense D%d L%d" % (D, L))


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 4), (4, 1), (16, 8)])
@pytest.mark.parametrize("D", [64, 128])
def test_decode_page_stream_many_sequences(Hq, Hkv, D):
    """Automatic (page-stream) decode over many short and long sequences, including
    empty ones, so CTA shares start and end inside sequences."""
    lens = [0, 1, 5, 16, 17, 31, 300, 0, 2048, 64, 65, 1000, 7, 129, 3000, 15] * 3
    w = W.paged_decode(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, num_blocks=2000, lmax=3072, lens=lens,
                       seed=D + Hq + Hkv)
    t = w.tensors
    o, lse = A.attn_decode_paged(t["q"].to(DEV), t["k_cache"].to(DEV), t["v_cache"].to(DEV),
                                 t["block_table"].to(DEV), t["seqused_k"].to(DEV),
                                 scale=w.params["scale"])
    o_ref, lse_ref = oracle.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                        t["seqused_k"], scale=w.params["scale"])
    _cmp(o, lse, o_ref, lse_ref, TOL_O_BF16, TOL_LSE_BF16, "page-stream decode")
    _no_device_error()
