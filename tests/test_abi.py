"""The C-ABI library loads on a machine without a GPU, exports every declared
entry point, and rejects bad arguments before touching the device."""
import ctypes
import re
from pathlib import Path

import pytest

from attention_paged_kv_gqa_b200 import build as B
from attention_paged_kv_gqa_b200 import binding

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def L():
    B.build()
    return binding.lib()


def declared_entry_points():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        text = h.read_text()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for n in ("attn_fwd_dense", "attn_fwd_varlen_paged", "attn_decode_paged",
              "attn_decode_workspace_size", "attn_check_device", "attn_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in declared_entry_points():
        assert hasattr(L, n), n


def test_status_strings(L):
    for s in range(0, 10):
        assert binding.status_string(s)
    assert binding.status_string(0) == "ok"


def test_device_check_without_gpu_is_an_error_not_a_crash(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("has a GPU")
    assert L.attn_check_device(0) != 0


def _strides():
    return (ctypes.c_int64 * 3)(128 * 2 * 64, 2 * 64, 64)


def test_null_pointers_rejected_before_launch(L):
    st = L.attn_fwd_dense(None, None, None, None, None, 1, 128, 128, 2, 2, 64, _strides(),
                          _strides(), _strides(), 0.0, 1, -1, 0.0, 0, None, None, None, None)
    assert st == 1


def test_bad_group_and_head_dim(L):
    p = ctypes.c_void_p(1 << 20)
    st = L.attn_fwd_dense(p, p, p, p, None, 1, 128, 128, 3, 2, 64, _strides(), _strides(),
                          _strides(), 0.0, 1, -1, 0.0, 0, None, None, None, None)
    assert st == 1                     # Hq % Hkv != 0
    st = L.attn_fwd_dense(p, p, p, p, None, 1, 128, 128, 2, 2, 96, _strides(), _strides(),
                          _strides(), 0.0, 1, -1, 0.0, 0, None, None, None, None)
    assert st == 2                     # head_dim 96 unsupported


def test_misaligned_pointer_and_fp8_without_descale(L):
    p = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    st = L.attn_fwd_dense(bad, p, p, p, None, 1, 128, 128, 2, 2, 64, _strides(), _strides(),
                          _strides(), 0.0, 1, -1, 0.0, 0, None, None, None, None)
    assert st == 1
    s128 = (ctypes.c_int64 * 3)(128 * 2 * 128, 2 * 128, 128)
    st = L.attn_fwd_dense(p, p, p, p, None, 1, 128, 128, 2, 2, 128, s128, s128, s128, 0.0, 1, -1, 0.0,
                          1, None, None, None, None)
    assert st == 1


def test_paged_block_size_and_patch_requirements(L):
    p = ctypes.c_void_p(1 << 20)
    cu = ctypes.c_void_p(1 << 21)
    # block_size 32 -> unsupported
    st = L.attn_fwd_varlen_paged(p, p, p, p, 4, 100, 32, cu, None, cu, 1, 16, 0, 16, 2, 2, 64,
                                 0.0, 1, None, -1, 0.0, 0, None, None, None, p, None, None, 0,
                                 None)
    assert st == 2
    # patch mask without ranges -> invalid
    st = L.attn_fwd_varlen_paged(p, p, p, p, 4, 100, 16, cu, None, cu, 1, 16, 0, 16, 2, 2, 64,
                                 0.0, 2, None, -1, 0.0, 0, None, None, None, p, None, None, 0,
                                 None)
    assert st == 1


def test_decode_workspace_size_and_limits(L):
    n = L.attn_decode_workspace_size(32, 32, 8, 128, 512, 16, 0)
    assert n > 0 and n % 4 == 0
    assert L.attn_decode_workspace_size(0, 32, 8, 128, 512, 16, 0) == 0
    p = ctypes.c_void_p(1 << 20)
    # group of 32 query heads per KV head is beyond the decode kernel's 16 rows
    st = L.attn_decode_paged(p, p, p, p, 4, 100, 16, p, 1, 32, 1, 128, 0.0, -1, 0.0, 1, 0, None,
                             None, None, p, None, p, 1 << 20, None)
    assert st == 2


def test_window_and_softcap_rules(L):
    """A window needs the causal mask; a softcap must be finite and >= 0 (before any launch)."""
    p = ctypes.c_void_p(1 << 20)
    dense = lambda mask, w, c: L.attn_fwd_dense(p, p, p, p, None, 1, 128, 128, 2, 2, 64, _strides(),
                                                _strides(), _strides(), 0.0, mask, w, c, 0, None,
                                                None, None, None)
    assert dense(0, 16, 0.0) == 2                  # window without the causal mask
    assert dense(1, 16, -1.0) == 1                 # negative softcap
    assert dense(1, -1, float("nan")) == 1
    assert dense(1, -1, float("inf")) == 1
    cu = ctypes.c_void_p(1 << 21)
    st = L.attn_fwd_varlen_paged(p, p, p, p, 4, 100, 16, cu, None, cu, 1, 16, 0, 16, 2, 2, 64,
                                 0.0, 2, p, 8, 0.0, 0, None, None, None, p, None, None, 0, None)
    assert st == 2                                 # window with the patch mask
    st = L.attn_decode_paged(p, p, p, p, 4, 100, 16, p, 1, 8, 2, 128, 0.0, 5, -2.0, 0, 0, None,
                             None, None, p, None, p, 1 << 20, None)
    assert st == 1                                 # negative softcap in decode


def test_only_qv_entry_points_check_arguments(L):
    """The only_qv calls share the forward's and the decode's checks (no launch on a bad call)."""
    p = ctypes.c_void_p(1 << 20)
    cu = ctypes.c_void_p(1 << 21)
    # qv missing
    st = L.attn_fwd_varlen_paged_only_qv(None, p, p, 4, 100, 16, cu, None, cu, 1, 16, 0, 16, 2, 2,
                                         64, 0.0, 1, None, -1, 0.0, 0, None, None, p, None, None)
    assert st == 1
    # block_size 32 -> unsupported; fp8 without descales -> invalid
    st = L.attn_fwd_varlen_paged_only_qv(p, p, p, 4, 100, 32, cu, None, cu, 1, 16, 0, 16, 2, 2,
                                         64, 0.0, 1, None, -1, 0.0, 0, None, None, p, None, None)
    assert st == 2
    st = L.attn_fwd_varlen_paged_only_qv(p, p, p, 4, 100, 16, cu, None, cu, 1, 16, 0, 16, 2, 2,
                                         128, 0.0, 1, None, -1, 0.0, 1, None, None, p, None, None)
    assert st == 1
    # decode: group beyond 16 rows -> unsupported; missing seqused_k -> invalid
    st = L.attn_decode_paged_only_qv(p, p, p, 4, 100, 16, p, 1, 32, 1, 128, 0.0, -1, 0.0, 1, 0,
                                     p, None, p, 1 << 20, None)
    assert st == 2
    st = L.attn_decode_paged_only_qv(p, p, p, 4, 100, 16, None, 1, 8, 2, 128, 0.0, -1, 0.0, 1, 0,
                                     p, None, p, 1 << 20, None)
    assert st == 1


def test_patch_entry_point_checks_arguments(L):
    p = ctypes.c_void_p(1 << 20)
    # negative interval bound; missing ranges; head_dim 96
    st = L.attn_fwd_patch(p, p, p, p, p, p, 1, 16, 16, 16, 2, 2, 64, 0.0, -1, 0, None, None, None,
                          p, None, None)
    assert st == 1
    st = L.attn_fwd_patch(p, p, p, p, p, None, 1, 16, 16, 16, 2, 2, 64, 0.0, 16, 0, None, None, None,
                          p, None, None)
    assert st == 1
    st = L.attn_fwd_patch(p, p, p, p, p, p, 1, 16, 16, 16, 2, 2, 96, 0.0, 16, 0, None, None, None,
                          p, None, None)
    assert st == 2


def test_noalloc_decode_reports_bad_arguments_like_the_workspace_decode(L):
    """attn_decode_paged_noalloc gives the same status as attn_decode_paged for every bad call
    (also with B == 0), before it looks at its scratch or the device."""
    p = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    # (q, k, v, block_table, max_blocks, num_blocks, block_size, seqused_k, B, Hq, Hkv, D, dtype, o)
    good = [p, p, p, p, 4, 100, 16, p, 2, 8, 2, 128, 0, p]
    cases = {
        "null q": {0: None}, "null k": {1: None}, "null v": {2: None},
        "null block_table": {3: None}, "null seqused_k": {7: None}, "null o": {13: None},
        "null q, B 0": {0: None, 8: 0}, "null o, B 0": {13: None, 8: 0},
        "negative B": {8: -1}, "Hq not a multiple": {9: 6, 10: 4}, "Hkv 0": {10: 0},
        "max_blocks 0": {4: 0}, "num_blocks 0": {5: 0}, "dtype 7": {12: 7},
        "head_dim 96": {11: 96}, "head_dim 96, B 0": {11: 96, 8: 0},
        "block_size 32": {6: 32}, "group 32": {9: 32, 10: 1}, "B 5000": {8: 5000},
        "misaligned q": {0: odd}, "misaligned o": {13: odd},
    }
    for name, change in cases.items():
        a = list(good)
        for i, val in change.items():
            a[i] = val
        q, k, v, bt, mb, nb, bs, su, B_, Hq, Hkv, D, dt, o = a
        ws_status = L.attn_decode_paged(q, k, v, bt, mb, nb, bs, su, B_, Hq, Hkv, D, 0.0, -1, 0.0,
                                        0, dt, None, None, None, o, None, p, 1 << 24, None)
        na_status = L.attn_decode_paged_noalloc(q, k, v, bt, mb, nb, bs, su, B_, Hq, Hkv, D, 0.0,
                                                dt, o, None, None)
        assert ws_status != 0, name
        assert na_status == ws_status, name


def test_fp8_decode_argument_checks(L):
    """e4m3 decode: descales required (invalid without); head_dim 64 or 128, automatic split
    and the key store only (unsupported otherwise); the noalloc call takes bf16 only."""
    p = ctypes.c_void_p(1 << 20)

    def dec(D=128, splits=0, dq=p, dk=p, dv=p, Hq=8, Hkv=2, B=2):
        return L.attn_decode_paged(p, p, p, p, 4, 100, 16, p, B, Hq, Hkv, D, 0.0, -1, 0.0, splits,
                                   1, dq, dk, dv, p, None, p, 1 << 24, None)

    assert dec(dq=None) == 1 and dec(dk=None) == 1 and dec(dv=None) == 1
    assert dec(D=96) == 2
    assert dec(splits=3) == 2
    assert dec(Hq=32, Hkv=16) == 2          # more KV heads than consumer warps
    st = L.attn_decode_paged_only_qv(p, p, p, 4, 100, 16, p, 2, 8, 2, 128, 0.0, -1, 0.0, 0, 1,
                                     p, None, p, 1 << 24, None)
    assert st == 2
    st = L.attn_decode_paged_noalloc(p, p, p, p, 4, 100, 16, p, 2, 8, 2, 128, 0.0, 1, p, None, None)
    assert st == 2


def test_decode_qv_argument_checks(L):
    """Decode with the Qv term: qv required (invalid without); bf16 and the automatic split
    only (unsupported otherwise); a misaligned qv is invalid."""
    p = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)

    def dec(qv=p, D=128, splits=0, dtype=0, Hq=8, Hkv=2):
        return L.attn_decode_paged_qv(p, qv, p, p, p, 4, 100, 16, p, 2, Hq, Hkv, D, 0.0, -1, 0.0,
                                      splits, dtype, p, None, p, 1 << 24, None)

    assert dec(qv=None) == 1
    assert dec(qv=odd) == 1
    assert dec(D=96) == 2
    assert dec(splits=2) == 2
    assert dec(dtype=1) == 2
    assert dec(Hq=32, Hkv=16) == 2


def test_fwd_qv_argument_checks(L):
    """The forward with the Qv term: qv required; bf16 only; head_dim 64 / 128."""
    p = ctypes.c_void_p(1 << 20)
    cu = ctypes.c_void_p(1 << 21)

    def fwd(qv=p, D=128, dtype=0):
        return L.attn_fwd_varlen_paged_qv(p, qv, p, p, p, 4, 100, 16, cu, None, cu, 1, 16, 0, 16,
                                          2, 2, D, 0.0, 1, None, -1, 0.0, dtype, p, None, None)

    assert fwd(qv=None) == 1
    assert fwd(D=96) == 2
    assert fwd(dtype=1) == 2


def test_kv_append_argument_checks(L):
    """attn_kv_append_paged rejects bad calls on the host, before the device is touched."""
    p = ctypes.c_void_p(1 << 20)
    su_in, su_out = ctypes.c_void_p(1 << 21), ctypes.c_void_p(1 << 22)
    odd = ctypes.c_void_p((1 << 20) + 8)
    # (k_new, v_new, k_cache, v_cache, block_table, max_blocks, num_blocks, block_size,
    #  cu_seqlens_new, seqused_k, seqused_k_out, B, total_new, Hkv, D, dtype)
    good = [p, p, p, p, p, 4, 100, 16, None, su_in, su_out, 2, 2, 2, 128, 0]
    cases = {
        "null k_new": ({0: None}, 1), "null v_cache": ({3: None}, 1),
        "null block_table": ({4: None}, 1), "null seqused_k": ({9: None}, 1),
        "negative B": ({11: -1}, 1), "Hkv 0": ({13: 0}, 1), "max_blocks 0": ({5: 0}, 1),
        "num_blocks 0": ({6: 0}, 1), "dtype 7": ({15: 7}, 1),
        "one per sequence needs total_new == B": ({12: 3}, 1),
        "seqused_k_out aliases seqused_k": ({10: su_in}, 1),
        "block_size 32": ({7: 32}, 2),
        "row not a multiple of 16 bytes": ({14: 4}, 1),
        "misaligned k_new": ({0: odd}, 1), "misaligned k_cache": ({2: odd}, 1),
    }
    for name, (change, want) in cases.items():
        a = list(good)
        for i, val in change.items():
            a[i] = val
        assert L.attn_kv_append_paged(*a, None) == want, name


def test_decode_append_checks_the_decode_half_first(L):
    """attn_decode_paged_append validates the decode's arguments before the append could
    be launched, so a bad call leaves the cache untouched."""
    p = ctypes.c_void_p(1 << 20)
    su_in, su_out = ctypes.c_void_p(1 << 21), ctypes.c_void_p(1 << 22)
    odd = ctypes.c_void_p((1 << 20) + 8)
    # (q, k_new, v_new, k_cache, v_cache, block_table, max_blocks, num_blocks, block_size,
    #  seqused_k, seqused_k_out, B, Hq, Hkv, D, scale, window_left, softcap, num_splits, dtype,
    #  o, lse, workspace, workspace_bytes)
    good = [p, p, p, p, p, p, 4, 100, 16, su_in, su_out, 2, 8, 2, 128, 0.0, -1, 0.0, 0, 0,
            p, None, p, 1 << 24]
    cases = {
        "no seqused_k_out": ({10: None}, 1), "null q": ({0: None}, 1), "null o": ({20: None}, 1),
        "Hq not a multiple": ({12: 6, 13: 4}, 1), "dtype 7": ({19: 7}, 1),
        "fp8": ({19: 1}, 2), "head_dim 96": ({14: 96}, 2), "group 32": ({12: 32, 13: 1}, 2),
        "misaligned q": ({0: odd}, 1), "misaligned o": ({20: odd}, 1),
        "no workspace": ({22: None}, 1), "workspace too small": ({23: 16}, 5),
        "null k_new (the append half)": ({1: None}, 1),
    }
    for name, (change, want) in cases.items():
        a = list(good)
        for i, val in change.items():
            a[i] = val
        assert L.attn_decode_paged_append(*a, None) == want, name


def test_backward_argument_checks(L):
    p = ctypes.c_void_p(1 << 20)
    cu = ctypes.c_void_p(1 << 21)
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert L.attn_bwd_workspace_size(4, 10) >= 4 * 10 * 4
    assert L.attn_bwd_workspace_size(0, 10) == 0
    assert L.attn_bwd_workspace_size(4, -1) == 0
    # (q, k, v, o, dout, lse, dq, dk, dv, cu_q, cu_k, B, total_q, total_k, max_q, max_k,
    #  Hq, Hkv, D, scale, mask, window_left, workspace, workspace_bytes)
    good = [p, p, p, p, p, p, p, p, p, cu, cu, 1, 64, 64, 64, 64, 4, 2, 128, 0.0, 1, -1, p, 1 << 20]
    cases = {
        "null dout": ({4: None}, 1), "null lse": ({5: None}, 1), "null dv": ({8: None}, 1),
        "null cu_seqlens_k": ({10: None}, 1), "negative total_k": ({13: -1}, 1),
        "Hq not a multiple": ({16: 3}, 1), "mask 9": ({20: 9}, 1), "patch mask": ({20: 2}, 2),
        "window without causal": ({20: 0, 21: 8}, 2), "head_dim 96": ({18: 96}, 2),
        "misaligned dq": ({6: odd}, 1), "misaligned v": ({2: odd}, 1),
        "no workspace": ({22: None}, 1), "workspace too small": ({23: 64}, 5),
    }
    for name, (change, want) in cases.items():
        a = list(good)
        for i, val in change.items():
            a[i] = val
        assert L.attn_bwd_varlen(*a, None) == want, name
