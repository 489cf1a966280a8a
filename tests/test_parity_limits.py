"""The CUDA path at the edges of its supported sizes, against the fp64 oracle.

  * the paged decode at its largest batch (4096 sequences, the on-device
    sequence table's limit), every output;
  * one very long decode sequence (65536 keys, 4096 pages) beside short ones;
  * more KV heads than the page-stream kernel's consumer warps (Hkv = 16: the
    per-head split kernel serves the automatic choice);
  * a prefill batch of 512 short sequences (many empty and single-row units);
  * one long causal prefill sequence (16384 tokens): whole rows at tile
    boundaries and the last rows, through the pinned prefix identity.
Tolerances as for the plain bf16 path: O <= 2e-2, LSE <= 1e-3.
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
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), what + ": non-finite output"
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    assert err_o <= TOL_O, "%s: max|O err| %.3g" % (what, err_o)
    ninf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), ninf), what + ": -inf rows differ"
    if (~ninf).any():
        err_l = float(np.max(np.abs(lse[~ninf] - lse_ref[~ninf])))
        assert err_l <= TOL_LSE, "%s: max|LSE err| %.3g" % (what, err_l)


def _decode_case(lens, Hq, Hkv, D, num_blocks, lmax, seed):
    w = W.paged_decode(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, num_blocks=num_blocks, lmax=lmax,
                       lens=lens, seed=seed)
    t = w.tensors
    o, lse = A.attn_decode_paged(t["q"].to(DEV), t["k_cache"].to(DEV), t["v_cache"].to(DEV),
                                 t["block_table"].to(DEV), t["seqused_k"].to(DEV),
                                 scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    o_ref, lse_ref = oracle.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                        t["seqused_k"], scale=w.params["scale"])
    return o, lse, o_ref, lse_ref


def test_decode_largest_batch():
    rng = np.random.default_rng(1)
    lens = rng.integers(0, 65, 4096).tolist()          # empty to four pages
    o, lse, o_ref, lse_ref = _decode_case(lens, 8, 2, 128, num_blocks=12000, lmax=64, seed=3)
    _cmp(o, lse, o_ref, lse_ref, "decode B=4096")


def test_decode_one_very_long_sequence():
    lens = [65536, 1, 300, 17]
    o, lse, o_ref, lse_ref = _decode_case(lens, 32, 8, 128, num_blocks=4200, lmax=65536, seed=4)
    _cmp(o, lse, o_ref, lse_ref, "decode 65536 keys")


@pytest.mark.parametrize("D", [64, 128])
def test_decode_more_kv_heads_than_consumer_warps(D):
    lens = [0, 1, 33, 700, 2048, 16]
    o, lse, o_ref, lse_ref = _decode_case(lens, 32, 16, D, num_blocks=400, lmax=2048, seed=5 + D)
    _cmp(o, lse, o_ref, lse_ref, "decode Hkv=16 D%d" % D)


def test_prefill_many_short_sequences():
    rng = np.random.default_rng(2)
    lens = rng.integers(0, 41, 512)
    lens[::7] = 0
    w = W.varlen_paged_prefill(nseq=len(lens), Hq=8, Hkv=2, D=64, num_blocks=3000, lens=lens,
                               lmax=64, seed=6)
    t = w.tensors
    for mask in (A.MASK_CAUSAL, A.MASK_NONE):
        o, lse = A.attn_fwd_varlen_paged(t["q"].to(DEV), t["k_cache"].to(DEV), t["v_cache"].to(DEV),
                                         cu_seqlens_q=t["cu_seqlens_q"].to(DEV),
                                         max_seqlen_q=max(int(lens.max()), 1),
                                         block_table=t["block_table"].to(DEV),
                                         seqused_k=t["seqused_k"].to(DEV), mask=mask,
                                         scale=w.params["scale"])
        torch.cuda.synchronize()
        assert A.attn_device_error() == 0
        o_ref, lse_ref = oracle.attn_varlen(t["q"], t["k_cache"], t["v_cache"],
                                            cu_seqlens_q=t["cu_seqlens_q"],
                                            block_table=t["block_table"], seqused_k=t["seqused_k"],
                                            num_heads_kv=2, scale=w.params["scale"], mask=int(mask))
        _cmp(o, lse, o_ref, lse_ref, "512 short sequences, mask %d" % mask)


def test_prefill_one_long_causal_sequence():
    L, Hq, Hkv, D = 16384, 8, 2, 128
    w = W.varlen_paged_prefill(nseq=1, Hq=Hq, Hkv=Hkv, D=D, num_blocks=1100, lens=[L], lmax=L,
                               seed=7)
    t = w.tensors
    o, lse = A.attn_fwd_varlen_paged(t["q"].to(DEV), t["k_cache"].to(DEV), t["v_cache"].to(DEV),
                                     cu_seqlens_q=t["cu_seqlens_q"].to(DEV), max_seqlen_q=L,
                                     block_table=t["block_table"].to(DEV),
                                     seqused_k=t["seqused_k"].to(DEV), mask=A.MASK_CAUSAL,
                                     scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    # causal row i == unmasked attention over keys 0..i (pinned on the CPU); rows at the
    # first, 128-boundary and last positions, each against the oracle over its prefix
    rows = [0, 1, 127, 128, 255, 256, 8191, 8192, 12345, L - 129, L - 128, L - 2, L - 1]
    for i in rows:
        n = i + 1
        npg = (n + 15) // 16
        pages = t["block_table"][0, :npg].long()
        bt = torch.arange(npg, dtype=torch.int32)[None]
        o_ref, lse_ref = oracle.attn_varlen(t["q"][i:i + 1], t["k_cache"][pages], t["v_cache"][pages],
                                            cu_seqlens_q=np.array([0, 1], np.int32),
                                            seqused_k=np.array([n], np.int32), block_table=bt,
                                            num_heads_kv=Hkv, scale=w.params["scale"], mask=0)
        _cmp(o[i:i + 1], lse[:, i:i + 1], o_ref, lse_ref, "long causal row %d" % i)
