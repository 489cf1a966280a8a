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
