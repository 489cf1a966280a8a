"""The allocation-free paged decode entry point (attn_decode_paged_noalloc).

It serves callers that cannot allocate device memory while they run (a
plug-in inside a host program that owns all allocations, or a serving loop
whose memory is fixed at start-up and must never reach cudaMalloc), by taking
its split-KV scratch from a fixed array inside the library.  Its results must
equal those of attn_decode_paged with a caller-provided workspace and those of
the fp64 oracle, also on a second call that finds the previous call's data
left in that scratch.
"""
import ctypes

import oracle

import numpy as np
import pytest
import torch

from attention_paged_kv_gqa_b200 import binding as A
from attention_paged_kv_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_O, TOL_LSE = 2e-2, 1e-3
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert A.attn_check_device(0) == 0
    torch.cuda.set_device(0)


def _both(w):
    t = w.tensors
    args = [t[n].to(DEV) for n in ("q", "k_cache", "v_cache", "block_table", "seqused_k")]
    o_ref, l_ref = A.attn_decode_paged(*args, scale=w.params["scale"])
    o, l = A.attn_decode_paged_noalloc(*args, scale=w.params["scale"])
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    return o, l, o_ref, l_ref


def _close(o, l, o_ref, l_ref):
    assert float((o.float() - o_ref.float()).abs().max()) <= TOL_O
    fin = torch.isfinite(l_ref)
    assert torch.equal(torch.isneginf(l), torch.isneginf(l_ref))
    assert float((l[fin] - l_ref[fin]).abs().max()) <= TOL_LSE


def _oracle(w):
    t = w.tensors
    o, l = oracle.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                              t["seqused_k"], scale=w.params["scale"])
    return torch.from_numpy(o).to(DEV), torch.from_numpy(l).to(DEV)


def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row():
    first = W.paged_decode(B=32, Hq=32, Hkv=8, D=128, num_blocks=6000, lmin=1, lmax=2048, seed=11)
    second = W.paged_decode(B=20, Hq=16, Hkv=4, D=64, num_blocks=3000, lmin=1, lmax=1500,
                            lens=[0, 1, 17, 1500, 33, 0, 700, 16, 15, 999] * 2, seed=12)
    for w in (first, second):
        o, l, o_ref, l_ref = _both(w)
        _close(o, l, o_ref, l_ref)                  # against the workspace entry point
        _close(o, l, *_oracle(w))                   # and against the fp64 oracle


def test_noalloc_rejects_requests_beyond_its_scratch():
    """A batch whose partials exceed the fixed 8 MiB scratch is refused with its own status."""
    L = A.lib()
    p = ctypes.c_void_p(1 << 20)      # never dereferenced: the request is refused before launch
    st = L.attn_decode_paged_noalloc(p, p, p, p, 512, 20000, 16, p, 4000, 32, 8, 128,
                                     0.0, 0, p, None, None)
    assert st == 8
    assert "scratch" in A.status_string(st)
