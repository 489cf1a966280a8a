"""Pins for the paged KV append oracle (CPU).

The append is data movement, so its pins check where the new rows land
without restating the page arithmetic: attention over the appended paged
cache (through the separately pinned C oracle's block-table reads) must
equal attention over plainly concatenated packed K/V; two appends must equal
one; exactly the appended rows change.  The last test plants mistakes in a
copy of the oracle's source and checks that each is caught.
"""
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle
from oracle import kv_append as KA


def _setup(lens_new, Hkv=2, D=8, num_blocks=64, seed=0, max_blocks=12):
    g = torch.Generator().manual_seed(seed)
    B = len(lens_new)
    perm = torch.randperm(num_blocks, generator=g).to(torch.int32)
    bt = perm[:B * max_blocks].reshape(B, max_blocks).clone()
    kc = torch.randn(num_blocks, 16, Hkv, D, generator=g, dtype=torch.float64)
    vc = torch.randn(num_blocks, 16, Hkv, D, generator=g, dtype=torch.float64)
    tot = int(sum(lens_new))
    kn = torch.randn(tot, Hkv, D, generator=g, dtype=torch.float64)
    vn = torch.randn(tot, Hkv, D, generator=g, dtype=torch.float64)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens_new)]), dtype=torch.int32)
    return kc, vc, kn, vn, bt, cu


def _attend_paged(q, kc, vc, bt, used, Hkv):
    return oracle.attn_decode(q, kc, vc, bt, used, scale=0.3)


def _attend_packed(q, k_seqs, v_seqs, Hkv):
    """Attention of one query per sequence over the given packed K/V rows."""
    lens = [len(k) for k in k_seqs]
    ck = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    k = torch.cat(k_seqs) if sum(lens) else torch.zeros(0, Hkv, q.shape[2], dtype=torch.float64)
    v = torch.cat(v_seqs) if sum(lens) else torch.zeros(0, Hkv, q.shape[2], dtype=torch.float64)
    o, lse = oracle.attn_varlen(q, k, v, cu_seqlens_q=np.arange(len(lens) + 1, dtype=np.int32),
                                cu_seqlens_k=ck, num_heads_kv=Hkv, scale=0.3)
    return o, lse.T


def test_append_from_empty_then_again_equals_concatenation():
    """Append n1 tokens to empty sequences, then n2 more: attention over the cache
    equals attention over concat(first rows, second rows) read as packed K/V."""
    n1, n2 = [5, 16, 0, 33], [1, 17, 3, 0]
    Hkv, D = 2, 8
    kc, vc, kn1, vn1, bt, cu1 = _setup(n1, Hkv, D, seed=1)
    _, _, kn2, vn2, _, cu2 = _setup(n2, Hkv, D, seed=2)
    used0 = torch.zeros(4, dtype=torch.int32)
    kc1, vc1, used1 = KA.kv_append_paged(kc, vc, kn1, vn1, bt, cu1, used0)
    kc2, vc2, used2 = KA.kv_append_paged(kc1, vc1, kn2, vn2, bt, cu2, used1)
    assert used1.tolist() == n1 and used2.tolist() == [a + b for a, b in zip(n1, n2)]
    q = torch.randn(4, 4, D, generator=torch.Generator().manual_seed(3), dtype=torch.float64)
    ks = [torch.cat([kn1[cu1[b]:cu1[b + 1]], kn2[cu2[b]:cu2[b + 1]]]) for b in range(4)]
    vs = [torch.cat([vn1[cu1[b]:cu1[b + 1]], vn2[cu2[b]:cu2[b + 1]]]) for b in range(4)]
    o_p, l_p = _attend_paged(q, kc2, vc2, bt, used2, Hkv)
    o_c, l_c = _attend_packed(q, ks, vs, Hkv)
    np.testing.assert_array_equal(np.isneginf(l_p), np.isneginf(l_c))
    np.testing.assert_allclose(o_p, o_c, atol=1e-13, rtol=0)
    fin = ~np.isneginf(l_c)
    np.testing.assert_allclose(l_p[fin], l_c[fin], atol=1e-13, rtol=0)


def test_two_appends_equal_one():
    n1, n2 = [3, 20, 7], [14, 1, 9]
    kc, vc, kn1, vn1, bt, cu1 = _setup(n1, seed=4)
    _, _, kn2, vn2, _, cu2 = _setup(n2, seed=5)
    used = torch.tensor([2, 30, 16], dtype=torch.int32)
    a_k, a_v, a_u = KA.kv_append_paged(kc, vc, kn1, vn1, bt, cu1, used)
    a_k, a_v, a_u = KA.kv_append_paged(a_k, a_v, kn2, vn2, bt, cu2, a_u)
    kn = torch.cat([torch.cat([kn1[cu1[b]:cu1[b + 1]], kn2[cu2[b]:cu2[b + 1]]]) for b in range(3)])
    vn = torch.cat([torch.cat([vn1[cu1[b]:cu1[b + 1]], vn2[cu2[b]:cu2[b + 1]]]) for b in range(3)])
    cu = torch.tensor(np.concatenate([[0], np.cumsum(np.add(n1, n2))]), dtype=torch.int32)
    b_k, b_v, b_u = KA.kv_append_paged(kc, vc, kn, vn, bt, cu, used)
    assert torch.equal(a_k, b_k) and torch.equal(a_v, b_v) and torch.equal(a_u, b_u)


def test_exactly_the_appended_rows_change():
    """A sentinel-filled cache: after the append exactly total_new rows per head differ
    from the sentinel, and they hold the new rows (as a multiset)."""
    n = [4, 0, 19, 16]
    Hkv, D = 2, 4
    _, _, kn, vn, bt, cu = _setup(n, Hkv, D, seed=6)
    kc = torch.full((64, 16, Hkv, D), 7.0, dtype=torch.float64)
    vc = torch.full((64, 16, Hkv, D), -7.0, dtype=torch.float64)
    used = torch.tensor([1, 5, 12, 0], dtype=torch.int32)
    k2, v2, _ = KA.kv_append_paged(kc, vc, kn, vn, bt, cu, used)
    changed_k = (k2 != 7.0).any(dim=-1)          # [page, row, head]
    changed_v = (v2 != -7.0).any(dim=-1)
    assert int(changed_k.sum()) == sum(n) * Hkv and int(changed_v.sum()) == sum(n) * Hkv
    got = sorted(map(tuple, k2[changed_k].tolist()))
    want = sorted(map(tuple, kn.reshape(-1, D).tolist()))
    assert got == want


def test_no_new_tokens_changes_nothing():
    kc, vc, kn, vn, bt, cu = _setup([0, 0], seed=7)
    used = torch.tensor([5, 9], dtype=torch.int32)
    k2, v2, u2 = KA.kv_append_paged(kc, vc, kn, vn, bt, cu, used)
    assert torch.equal(k2, kc) and torch.equal(v2, vc) and torch.equal(u2, used)


def test_positions_beyond_the_block_table_are_rejected():
    kc, vc, kn, vn, bt, cu = _setup([3], seed=8, max_blocks=2)
    with pytest.raises(ValueError):
        KA.kv_append_paged(kc, vc, kn, vn, bt, cu, torch.tensor([30], dtype=torch.int32))


PINS = [test_append_from_empty_then_again_equals_concatenation, test_two_appends_equal_one,
        test_exactly_the_appended_rows_change, test_no_new_tokens_changes_nothing]

MUTATIONS = {
    "position_off_by_one": ("p = int(used[b]) + i", "p = int(used[b]) + i + 1"),
    "wrong_page": ("slot = p // block_size", "slot = p // block_size + 1"),
    "wrong_row": ("row = p % block_size", "row = (p + 1) % block_size"),
    "lengths_not_accumulated": ("after[b] = used[b] + n", "after[b] = n"),
    "v_from_k": ("vc[page, row] = v_new[cu[b] + i]", "vc[page, row] = k_new[cu[b] + i]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    src = Path(KA.__file__).read_text()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    ns = {}
    exec(compile(src.replace(old, new), "mutated_kv_append", "exec"), ns)
    monkeypatch.setattr(KA, "kv_append_paged", ns["kv_append_paged"])
    caught = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError, RuntimeError):
            caught += 1
    assert caught >= 1, "no pin caught the planted mistake " + name
