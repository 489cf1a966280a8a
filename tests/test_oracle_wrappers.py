"""Pins for the oracle's Python wrappers (fp8 dequantisation, the decode window,
the dense backward layout) against facts that do not come from the wrappers.

* ``dequant_e4m3``: every finite e4m3 code is decoded here from the format's
  definition (sign, 4-bit exponent with bias 7, 3-bit mantissa, subnormals at
  exponent 0, no infinities; the ``float8_e4m3fn`` operands of "[FlexAttention]
  Enforce Q,K,V memory layouts for fp8 flex attention") and the real value is
  code x descale.  A quantise/dequantise round trip stays within e4m3's
  half-ulp.
* ``attn_decode`` with a window: the decode query is the newest of L cached
  tokens, so a window of W keys leaves keys L-1-W .. L-1; the wrapper must equal
  unmasked attention over exactly those keys (gathered through the block table
  here with plain indexing) and the brute-force enumeration.
* ``attn_bwd_dense``: equal to per-batch calls of the (finite-difference
  pinned) varlen backward, with Lq != Lk so that a swapped length is visible.

The last test plants plausible mistakes in a copy of the wrappers' source and
checks that each is caught by at least one of these pins.
"""
import math
import types
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from attention_paged_kv_gqa_b200 import workloads as W


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


# ----------------------------------------------------------------------------
# e4m3 dequantisation
# ----------------------------------------------------------------------------

def e4m3_value(code: int) -> float:
    """Real value of an e4m3fn byte from the format's definition (NaN codes excluded)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


FINITE_CODES = [c for c in range(256) if (c & 0x7F) != 0x7F]


def check_dequant_codes(orc):
    codes = torch.tensor(FINITE_CODES, dtype=torch.uint8).view(torch.float8_e4m3fn)
    for descale in (1.0, 0.375, 3.0e-3):
        got = orc.dequant_e4m3(codes, torch.tensor([descale], dtype=torch.float32))
        got = np.asarray(got, dtype=np.float64).reshape(-1)
        want = np.array([e4m3_value(c) for c in FINITE_CODES]) * float(np.float32(descale))
        np.testing.assert_array_equal(got, want)


def check_dequant_printed_points(orc):
    """Largest finite (448), smallest subnormal (2^-9), -1 and 0, times a descale of 0.5."""
    codes = torch.tensor([0x7E, 0x01, 0xB8, 0x00], dtype=torch.uint8).view(torch.float8_e4m3fn)
    got = np.asarray(orc.dequant_e4m3(codes, 0.5), dtype=np.float64).reshape(-1)
    np.testing.assert_array_equal(got, [224.0, 2.0 ** -10, -0.5, 0.0])


def check_dequant_round_trip(orc):
    """dequant(quantise(x)) is within half an e4m3 ulp of x (3 mantissa bits)."""
    x = W.randn_bf16((64, 128), seed=3, stream=9).to(torch.float64)
    q, s = W.quantize_e4m3(x)
    back = np.asarray(orc.dequant_e4m3(q, s), dtype=np.float64)
    sc = float(s[0])
    xa = x.numpy()
    # normal range: relative 2^-4; below 2^-6 (in code units) the subnormal step 2^-9 / 2
    bound = np.maximum(np.abs(xa) * 2.0 ** -4, sc * 2.0 ** -10) * (1 + 1e-12)
    assert np.all(np.abs(back - xa) <= bound)


def test_dequant_every_finite_code():
    check_dequant_codes(oracle)


def test_dequant_printed_points():
    check_dequant_printed_points(oracle)


def test_dequant_round_trip_within_half_ulp():
    check_dequant_round_trip(oracle)


# ----------------------------------------------------------------------------
# decode with a sliding window
# ----------------------------------------------------------------------------

DEC_LENS = [1, 15, 16, 17, 40, 100]


def _decode_case():
    w = W.paged_decode(B=len(DEC_LENS), Hq=4, Hkv=2, D=8, num_blocks=64, lmin=1, lmax=112,
                       seed=7, lens=DEC_LENS)
    return w.tensors


def _keys_of(t, b):
    """Sequence b's cached K and V rows in token order, read through its block table."""
    L = int(t["seqused_k"][b])
    rows_k, rows_v = [], []
    for j in range(L):
        page = int(t["block_table"][b, j // 16])
        rows_k.append(t["k_cache"][page, j % 16].double().numpy())
        rows_v.append(t["v_cache"][page, j % 16].double().numpy())
    return np.array(rows_k), np.array(rows_v)


def check_decode_window_slices(orc, windows=(0, 15, 16, 100)):
    t = _decode_case()
    q = t["q"].double().numpy()
    Hkv = t["k_cache"].shape[2]
    for Wl in windows:
        o, lse = orc.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                 t["seqused_k"], scale=0.4, window_left=Wl)
        for b, L in enumerate(DEC_LENS):
            k, v = _keys_of(t, b)
            first = max(0, L - 1 - Wl)
            ob, lb = oracle.attn_varlen(q[b:b + 1], k[first:], v[first:],
                                        cu_seqlens_q=cu([1]), cu_seqlens_k=cu([L - first]),
                                        num_heads_kv=Hkv, scale=0.4, mask=oracle.MASK_NONE)
            np.testing.assert_allclose(o[b], ob[0], rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[b], lb[:, 0], rtol=0, atol=1e-13)


def check_decode_window_brute(orc):
    t = _decode_case()
    q = t["q"].double().numpy()
    for Wl in (0, 5, 16):
        o, lse = orc.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                 t["seqused_k"], scale=0.4, window_left=Wl)
        for b in (0, 3, 4):
            k, v = _keys_of(t, b)
            bo, bl = brute.attention(q[b:b + 1].tolist(), k.tolist(), v.tolist(), 0.4,
                                     mask="causal", window=Wl)
            np.testing.assert_allclose(o[b], np.array(bo)[0], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b], np.array(bl)[:, 0], rtol=0, atol=1e-12)


def test_decode_window_equals_attention_over_the_window_keys():
    check_decode_window_slices(oracle)


def test_decode_window_agrees_with_brute_force():
    check_decode_window_brute(oracle)


def test_decode_window_covering_the_cache_is_the_plain_decode():
    t = _decode_case()
    o0, l0 = oracle.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                t["seqused_k"], scale=0.4)
    o1, l1 = oracle.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                t["seqused_k"], scale=0.4, window_left=max(DEC_LENS) - 1)
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(l0, l1)


# ----------------------------------------------------------------------------
# dense backward wrapper
# ----------------------------------------------------------------------------

def check_bwd_dense_layout(orc):
    B, Lq, Lk, Hq, Hkv, D = 2, 5, 7, 4, 2, 6
    q, k, v = rnd((B, Lq, Hq, D), 61), rnd((B, Lk, Hkv, D), 62), rnd((B, Lk, Hkv, D), 63)
    do = rnd((B, Lq, Hq, D), 64)
    for causal in (False, True):
        dq, dk, dv = orc.attn_bwd_dense(q, k, v, do, scale=0.45, causal=causal)
        assert dq.shape == (B, Lq, Hq, D) and dk.shape == (B, Lk, Hkv, D) and dv.shape == dk.shape
        for b in range(B):
            rq, rk, rv = oracle.attn_bwd_varlen(q[b], k[b], v[b], do[b], cu_seqlens_q=cu([Lq]),
                                                cu_seqlens_k=cu([Lk]), num_heads_kv=Hkv,
                                                scale=0.45, mask=1 if causal else 0)
            np.testing.assert_array_equal(dq[b], rq)
            np.testing.assert_array_equal(dk[b], rk)
            np.testing.assert_array_equal(dv[b], rv)


def test_bwd_dense_equals_per_batch_varlen():
    check_bwd_dense_layout(oracle)


# ----------------------------------------------------------------------------
# planted mistakes in the wrappers
# ----------------------------------------------------------------------------

WRAPPER_MUTATIONS = {
    "dequant_divides_by_descale": ("dequant_e4m3", "x_fp8.to(torch.float64) * float(",
                                   "x_fp8.to(torch.float64) / float("),
    "dequant_drops_descale": ("dequant_e4m3",
                              " * float(torch.as_tensor(descale).reshape(-1)[0])", ""),
    "dequant_reads_raw_bytes": ("dequant_e4m3", "x_fp8.to(torch.float64)",
                                "x_fp8.view(torch.uint8).to(torch.float64)"),
    "decode_window_dropped": ("attn_decode", "window_left=window_left, softcap",
                              "window_left=-1, softcap"),
    "decode_window_off_by_one": ("attn_decode", "window_left=window_left, softcap",
                                 "window_left=window_left + 1, softcap"),
    "decode_window_without_causal": ("attn_decode",
                                     "mask=MASK_CAUSAL if window_left >= 0 else MASK_NONE",
                                     "mask=MASK_NONE"),
    "bwd_dense_dq_transposed": ("attn_bwd_dense", "return dq.reshape(B, Lq, Hq, D),",
                                "return dq.reshape(B, Hq, Lq, D).transpose(0, 2, 1, 3),"),
    "bwd_dense_dk_transposed": ("attn_bwd_dense", "dk.reshape(B, Lk, Hkv, D),",
                                "dk.reshape(B, Hkv, Lk, D).transpose(0, 2, 1, 3),"),
    "bwd_dense_causal_ignored": ("attn_bwd_dense", "mask=MASK_CAUSAL if causal else MASK_NONE",
                                 "mask=MASK_NONE"),
    "bwd_dense_key_lengths_from_q": ("attn_bwd_dense",
                                     "ck = np.arange(B + 1, dtype=np.int32) * Lk",
                                     "ck = np.arange(B + 1, dtype=np.int32) * Lq"),
}

WRAPPER_PINS = [check_dequant_codes, check_dequant_printed_points, check_dequant_round_trip,
                check_decode_window_slices, check_decode_window_brute, check_bwd_dense_layout]


def mutated_oracle(func, old, new):
    """A copy of the oracle package module with one textual change inside `func`."""
    path = Path(oracle.__file__)
    src = path.read_text()
    start = src.index("\ndef " + func + "(")
    end = src.find("\ndef ", start + 1)
    end = len(src) if end < 0 else end
    seg = src[start:end]
    assert seg.count(old) == 1, "mutation anchor not unique in " + func
    mod = types.ModuleType("oracle_mutated")
    mod.__file__ = str(path)
    exec(compile(src[:start] + seg.replace(old, new) + src[end:], str(path), "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(WRAPPER_MUTATIONS))
def test_planted_wrapper_mistake_is_caught(name):
    func, old, new = WRAPPER_MUTATIONS[name]
    mod = mutated_oracle(func, old, new)
    caught = 0
    for pin in WRAPPER_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except (AssertionError, ValueError, RuntimeError, TypeError, FloatingPointError):
            caught += 1
    assert caught >= 1, "no pin caught the planted mistake " + name


def test_unmutated_copy_passes_every_pin():
    """The mutation harness itself: an identity change leaves every pin green."""
    mod = mutated_oracle("dequant_e4m3", "x_fp8.to(torch.float64)", "x_fp8.to(torch.float64)")
    for pin in WRAPPER_PINS:
        pin(mod)
