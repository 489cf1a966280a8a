"""Failure detection without a GPU fault: a bounded wait that runs out.

Every mbarrier wait in the kernels is bounded; on expiry the kernel records a
code in the device error word, lets its copies land and returns, so a broken
protocol ends the kernel instead of hanging the GPU.  Here a test-only kernel
waits on a barrier that nothing arrives on, with a short limit: the call must
return, the stream must complete, the error word must name the wait (code
901, reported as ATTN_ERR_DEVICE_TIMEOUT and cleared by the read), and the
library must still compute correct results afterwards.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from attention_paged_kv_gqa_b200 import binding as A
from attention_paged_kv_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert A.attn_check_device(0) == 0
    torch.cuda.set_device(0)


def test_wait_runs_out_and_kernel_returns():
    assert A.attn_device_error() == 0            # nothing pending from earlier tests
    t0 = time.perf_counter()
    A.attn_selftest_wait_expiry(2_000_000)       # 2 ms
    torch.cuda.synchronize()                     # the kernel exits on its own
    elapsed = time.perf_counter() - t0
    code = ctypes.c_int(0)
    st = A.lib().attn_device_error(ctypes.byref(code), None)
    assert st == 7                               # ATTN_ERR_DEVICE_TIMEOUT
    assert code.value == 901
    assert elapsed < 5.0
    assert A.attn_device_error() == 0            # the read cleared the word


def test_status_of_an_out_of_range_limit():
    st = A.lib().attn_selftest_wait_expiry(-1, None)
    assert st == 1
    st = A.lib().attn_selftest_wait_expiry(20_000_000_000, None)
    assert st == 1


def test_library_still_correct_after_an_expired_wait():
    A.attn_selftest_wait_expiry(1_000_000)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 901
    w = W.dense(B=1, L=200, Hq=4, Hkv=2, D=64, seed=21)
    t = {k: v.cuda() for k, v in w.tensors.items()}
    o, lse = A.attn_fwd_dense(t["q"], t["k"], t["v"], causal=True, scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    ro, rl = oracle.attn_dense(w.tensors["q"], w.tensors["k"], w.tensors["v"],
                               scale=w.params["scale"], causal=True)
    assert float(np.abs(o.float().cpu().numpy() - ro).max()) <= 2e-2
    assert float(np.abs(lse.cpu().numpy() - rl).max()) <= 1e-3


def _bad_page_table(bt, lens):
    """A copy of the block table with one used entry per sequence pointing past the cache."""
    bad = bt.clone()
    for b, L in enumerate(lens):
        if L > 0:
            bad[b, (int(L) - 1) // 16] = 1 << 30
    return bad


def test_prefill_reports_block_table_entry_outside_the_cache():
    lens = [40, 200, 17]
    w = W.varlen_paged_prefill(nseq=3, Hq=4, Hkv=2, D=128, num_blocks=64, lens=lens, lmax=256,
                               seed=31)
    t = {k: v.cuda() for k, v in w.tensors.items()}
    bad = _bad_page_table(t["block_table"], lens)
    assert A.attn_device_error() == 0
    A.attn_fwd_varlen_paged(t["q"], t["k_cache"], t["v_cache"], cu_seqlens_q=t["cu_seqlens_q"],
                            max_seqlen_q=w.params["max_seqlen_q"], block_table=bad,
                            seqused_k=t["seqused_k"], mask=A.MASK_CAUSAL, scale=w.params["scale"])
    torch.cuda.synchronize()
    code = ctypes.c_int(0)
    assert A.lib().attn_device_error(ctypes.byref(code), None) == 9   # ATTN_ERR_DEVICE_RANGE
    assert code.value == 111
    # the data error stops nothing: the same call with a valid table is still correct
    o, lse = A.attn_fwd_varlen_paged(t["q"], t["k_cache"], t["v_cache"],
                                     cu_seqlens_q=t["cu_seqlens_q"],
                                     max_seqlen_q=w.params["max_seqlen_q"],
                                     block_table=t["block_table"], seqused_k=t["seqused_k"],
                                     mask=A.MASK_CAUSAL, scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    ro, rl = oracle.attn_varlen(w.tensors["q"], w.tensors["k_cache"], w.tensors["v_cache"],
                                cu_seqlens_q=w.tensors["cu_seqlens_q"],
                                seqused_k=w.tensors["seqused_k"],
                                block_table=w.tensors["block_table"], num_heads_kv=2,
                                scale=w.params["scale"], mask=1)
    assert float(np.abs(o.float().cpu().numpy() - ro).max()) <= 2e-2
    assert float(np.abs(lse.cpu().numpy() - rl).max()) <= 1e-3


@pytest.mark.parametrize("num_splits", [0, 3])
def test_decode_reports_block_table_entry_outside_the_cache(num_splits):
    lens = [1, 100, 700, 33]
    w = W.paged_decode(B=4, Hq=8, Hkv=2, D=128, num_blocks=128, lmax=800, lens=lens, seed=32)
    t = {k: v.cuda() for k, v in w.tensors.items()}
    bad = _bad_page_table(t["block_table"], lens)
    assert A.attn_device_error() == 0
    A.attn_decode_paged(t["q"], t["k_cache"], t["v_cache"], bad, t["seqused_k"],
                        scale=w.params["scale"], num_splits=num_splits)
    torch.cuda.synchronize()
    code = ctypes.c_int(0)
    assert A.lib().attn_device_error(ctypes.byref(code), None) == 9
    assert code.value == 411
