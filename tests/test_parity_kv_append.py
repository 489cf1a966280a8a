"""Paged KV append: CUDA path vs the oracle.

The append is data movement, so the caches must match the oracle's scatter
bit for bit (bf16 values and e4m3 codes alike), and the new lengths exactly.
The decode-with-append call is compared with the fp64 oracle's decode over the
oracle-appended cache (bf16 tolerances: max |O err| <= 2e-2, max |LSE err|
<= 1e-3).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import kv_append as KA
from attention_paged_kv_gqa_b200 import binding as A
from attention_paged_kv_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_O_BF16, TOL_LSE_BF16 = 2e-2, 1e-3
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert A.attn_check_device(0) == 0, "not a B200 or the kernel image does not load"
    torch.cuda.set_device(0)


def _cache(num_blocks, Hkv, D, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(num_blocks, 16, Hkv, D, generator=g)
    return x.to(dtype)


def _rows(n, Hkv, D, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(n, Hkv, D, generator=g).to(dtype)


def _table(B, max_blocks, num_blocks, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randperm(num_blocks, generator=g)[:B * max_blocks].reshape(B, max_blocks).to(torch.int32)


def _bits(t):
    return t.view(torch.uint8) if t.dtype != torch.uint8 else t


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float8_e4m3fn])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hkv", [1, 8])
def test_kv_append_matches_oracle(dtype, D, Hkv):
    before = [0, 1, 15, 16, 17, 100, 255, 3]
    new = [3, 0, 1, 16, 40, 300, 1, 0]
    B, max_blocks, num_blocks = len(before), 40, 400
    kc = _cache(num_blocks, Hkv, D, dtype, 1)
    vc = _cache(num_blocks, Hkv, D, dtype, 2)
    kn = _rows(sum(new), Hkv, D, dtype, 3)
    vn = _rows(sum(new), Hkv, D, dtype, 4)
    bt = _table(B, max_blocks, num_blocks, 5)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(new)]), dtype=torch.int32)
    used = torch.tensor(before, dtype=torch.int32)
    k_ref, v_ref, u_ref = KA.kv_append_paged(kc, vc, kn, vn, bt, cu, used)
    kd, vd = kc.to(DEV), vc.to(DEV)
    out = A.attn_kv_append_paged(kn.to(DEV), vn.to(DEV), kd, vd, bt.to(DEV), used.to(DEV),
                                 cu_seqlens_new=cu.to(DEV))
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    assert torch.equal(_bits(kd.cpu()), _bits(k_ref)) and torch.equal(_bits(vd.cpu()), _bits(v_ref))
    assert torch.equal(out.cpu(), u_ref)


def test_kv_append_one_token_per_sequence():
    B, Hkv, D, num_blocks, max_blocks = 37, 8, 128, 800, 20
    before = list(range(0, 37 * 8, 8))            # lengths 0, 8, ..., 288 (some end pages)
    kc, vc = _cache(num_blocks, Hkv, D, torch.bfloat16, 6), _cache(num_blocks, Hkv, D, torch.bfloat16, 7)
    kn, vn = _rows(B, Hkv, D, torch.bfloat16, 8), _rows(B, Hkv, D, torch.bfloat16, 9)
    bt = _table(B, max_blocks, num_blocks, 10)
    used = torch.tensor(before, dtype=torch.int32)
    k_ref, v_ref, u_ref = KA.kv_append_paged(kc, vc, kn, vn, bt, torch.arange(B + 1, dtype=torch.int32),
                                             used)
    kd, vd = kc.to(DEV), vc.to(DEV)
    out = A.attn_kv_append_paged(kn.to(DEV), vn.to(DEV), kd, vd, bt.to(DEV), used.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(kd.cpu(), k_ref) and torch.equal(vd.cpu(), v_ref)
    assert torch.equal(out.cpu(), u_ref)


def test_kv_append_skips_positions_outside_the_table():
    """A sequence that runs past its block table and one whose page index is out of
    range: those tokens are not written (the kernel's bounds check), the device error
    word reports it, and every other token lands as in the oracle."""
    Hkv, D, num_blocks, max_blocks = 2, 64, 64, 3
    before, new = [40, 5, 10], [20, 4, 2]         # sequence 0 fits 8 of its 20 tokens
    kc, vc = _cache(num_blocks, Hkv, D, torch.bfloat16, 11), _cache(num_blocks, Hkv, D, torch.bfloat16, 12)
    kn, vn = _rows(sum(new), Hkv, D, torch.bfloat16, 13), _rows(sum(new), Hkv, D, torch.bfloat16, 14)
    bt = _table(3, max_blocks, num_blocks, 15)
    bt[2, 0] = num_blocks + 7                      # sequence 2 writes into a page that does not exist
    cu = torch.tensor(np.concatenate([[0], np.cumsum(new)]), dtype=torch.int32)
    used = torch.tensor(before, dtype=torch.int32)
    # expected: sequence 0 only up to position 47, sequence 1 whole, sequence 2 nothing
    keep = [8, 4, 0]
    idx = np.concatenate([np.arange(int(cu[b]), int(cu[b]) + keep[b]) for b in range(3)]).astype(np.int64)
    cu_keep = torch.tensor(np.concatenate([[0], np.cumsum(keep)]), dtype=torch.int32)
    bt_ok = bt.clone()
    bt_ok[2, 0] = 0
    k_ref, v_ref, _ = KA.kv_append_paged(kc, vc, kn[idx], vn[idx], bt_ok, cu_keep, used)
    kd, vd = kc.to(DEV), vc.to(DEV)
    A.attn_kv_append_paged(kn.to(DEV), vn.to(DEV), kd, vd, bt.to(DEV), used.to(DEV),
                           cu_seqlens_new=cu.to(DEV))
    torch.cuda.synchronize()
    assert A.attn_device_error() in (501, 502)
    assert torch.equal(kd.cpu(), k_ref) and torch.equal(vd.cpu(), v_ref)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("splits", [0, 3])
@pytest.mark.parametrize("window", [-1, 20])
def test_decode_with_append_matches_oracle(D, splits, window):
    lens = [0, 1, 15, 16, 17, 64, 513, 1000]
    # pages for one more token per sequence (the appended one); lengths before the append
    w = W.paged_decode(B=len(lens), Hq=32, Hkv=8, D=D, num_blocks=300, lmax=1024,
                       lens=[n + 1 for n in lens], seed=D + splits)
    t = w.tensors
    t["seqused_k"] = torch.tensor(lens, dtype=torch.int32)
    B, Hkv = len(lens), 8
    kn, vn = _rows(B, Hkv, D, torch.bfloat16, 16), _rows(B, Hkv, D, torch.bfloat16, 17)
    k_ref, v_ref, u_ref = KA.kv_append_paged(t["k_cache"], t["v_cache"], kn, vn, t["block_table"],
                                             torch.arange(B + 1, dtype=torch.int32), t["seqused_k"])
    kd, vd = t["k_cache"].to(DEV), t["v_cache"].to(DEV)
    o, lse, u_out = A.attn_decode_paged_append(t["q"].to(DEV), kn.to(DEV), vn.to(DEV), kd, vd,
                                               t["block_table"].to(DEV), t["seqused_k"].to(DEV),
                                               scale=w.params["scale"], num_splits=splits,
                                               window_left=window)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    assert torch.equal(kd.cpu(), k_ref) and torch.equal(vd.cpu(), v_ref)
    assert torch.equal(u_out.cpu(), u_ref)
    o_ref, lse_ref = oracle.attn_decode(t["q"], k_ref, v_ref, t["block_table"], u_ref,
                                        scale=w.params["scale"], window_left=window)
    o = o.float().cpu().numpy()
    assert np.max(np.abs(o - o_ref)) <= TOL_O_BF16
    assert np.max(np.abs(lse.cpu().numpy() - lse_ref)) <= TOL_LSE_BF16


def test_decode_with_append_repeated_steps():
    """Eight decode steps in a row, each appending one token and reading it back at once
    (the decode waits for the append on the device): the last step equals the oracle."""
    lens = [5, 16, 31, 200]
    B, Hq, Hkv, D = 4, 8, 2, 128
    w = W.paged_decode(B=B, Hq=Hq, Hkv=Hkv, D=D, num_blocks=100, lmax=256,
                       lens=[n + 8 for n in lens], seed=3)
    t = w.tensors
    t["seqused_k"] = torch.tensor(lens, dtype=torch.int32)
    kd, vd = t["k_cache"].to(DEV), t["v_cache"].to(DEV)
    bt = t["block_table"].to(DEV)
    used = t["seqused_k"].to(DEV)
    k_ref, v_ref, u_ref = t["k_cache"], t["v_cache"], t["seqused_k"]
    for step in range(8):
        kn, vn = _rows(B, Hkv, D, torch.bfloat16, 100 + step), _rows(B, Hkv, D, torch.bfloat16, 200 + step)
        q = _rows(B, Hq, D, torch.bfloat16, 300 + step)
        o, lse, used = A.attn_decode_paged_append(q.to(DEV), kn.to(DEV), vn.to(DEV), kd, vd, bt, used,
                                                  scale=0.1)
        k_ref, v_ref, u_ref = KA.kv_append_paged(k_ref, v_ref, kn, vn, t["block_table"],
                                                 torch.arange(B + 1, dtype=torch.int32), u_ref)
    torch.cuda.synchronize()
    assert torch.equal(used.cpu(), u_ref)
    o_ref, lse_ref = oracle.attn_decode(q, k_ref, v_ref, t["block_table"], u_ref, scale=0.1)
    assert np.max(np.abs(o.float().cpu().numpy() - o_ref)) <= TOL_O_BF16
    assert np.max(np.abs(lse.cpu().numpy() - lse_ref)) <= TOL_LSE_BF16
