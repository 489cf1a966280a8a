"""Host-side arithmetic of bench.py on CPU: the algorithmic work and byte counts that
every roofline fraction divides by, checked against brute-force enumeration and hand
counts, the fraction arithmetic itself, and that the committed DRAM traffic figures
still belong to the kernel sources they were captured from."""
import numpy as np
import pytest
import torch

import bench


def _pairs_brute(L, window=None):
    n = 0
    for i in range(L):
        for j in range(L):
            if j <= i and (window is None or i - j <= window):
                n += 1
    return n


@pytest.mark.parametrize("lens", [[1], [5, 0, 7], [16, 17, 33], [128, 1, 64]])
def test_causal_flops_counts_allowed_pairs(lens):
    Hq, D = 3, 64
    want = 4 * D * Hq * sum(_pairs_brute(L) for L in lens)
    assert bench.causal_flops(lens, Hq, D) == want


@pytest.mark.parametrize("window", [0, 1, 5, 16, 200])
def test_window_causal_flops_counts_allowed_pairs(window):
    lens, Hq, D = [1, 7, 16, 40, 3], 2, 128
    want = 4 * D * Hq * sum(_pairs_brute(L, window) for L in lens)
    assert bench.window_causal_flops(lens, Hq, D, window) == want
    # a window at least as long as every sequence is the plain causal mask
    if window >= max(lens):
        assert bench.window_causal_flops(lens, Hq, D, window) == bench.causal_flops(lens, Hq, D)


def test_decode_bytes_hand_count():
    # 3 sequences of 1, 16 and 17 keys: 34 keys, 1 + 1 + 2 = 4 pages
    t = {"seqused_k": torch.tensor([1, 16, 17], dtype=torch.int32)}
    Hq, Hkv, D = 4, 2, 64
    kv = 34 * Hkv * D * 2 * 2           # K and V rows, bf16
    qo = 3 * Hq * D * 2 * 2             # q and O, bf16
    lse = 3 * Hq * 4
    bt = 4 * 4                          # used block-table entries
    seqused = 3 * 4
    assert bench.decode_bytes(t, Hq, Hkv, D) == kv + qo + lse + bt + seqused
    # e4m3: K, V and q one byte each, O stays bf16
    assert bench.decode_bytes_fp8(t, Hq, Hkv, D) == (34 * Hkv * D * 2 + 3 * Hq * D * (1 + 2)
                                                     + lse + bt + seqused)
    # a window covering every key changes nothing; window 0 keeps one key per sequence
    assert bench.window_decode_bytes(t, Hq, Hkv, D, 100) == bench.decode_bytes(t, Hq, Hkv, D)
    assert bench.window_decode_bytes(t, Hq, Hkv, D, 0) == (3 * Hkv * D * 2 * 2 + qo + lse
                                                          + 3 * 4 + seqused)


def test_patch_bytes_hand_count():
    P = dict(total_k=10, total_q=3, Hq=2, Hkv=2, D=64, B=2)
    want = (2 * 10 * 2 * 64 * 2       # every K and V row once
            + 2 * 3 * 2 * 64 * 2      # q and O
            + 3 * 2 * 4               # LSE
            + 3 * 8                   # the (start, end) range of each query
            + 2 * 3 * 4)              # both cu_seqlens arrays
    assert bench.patch_bytes(P) == want


def test_fractions_divide_by_the_named_peak():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "fp8_tflops": 3000.0}
    e = bench.entry(3000.0, "GB/s", 0.1, "hbm", peaks)
    assert e["frac"] == 0.5 and e["frac_spec"] == round(3000.0 / bench.SPEC_PEAKS["hbm_gbs"], 4)
    e = bench.entry(750.0, "TFLOP/s", 1.0, "tensor", peaks)
    assert e["frac"] == 0.5
    e = bench.entry(750.0, "TFLOP/s", 1.0, "tensor", peaks, dtype="fp8")
    assert e["frac"] == 0.25
    r = bench.roofline(1200.0, "TFLOP/s", "tensor", peaks, "measured", None, "k", dtype="fp8")
    assert r["peak"] == 3000.0 and r["frac"] == 0.4 and r["bound"] == "tensor"
    r = bench.roofline(4500.0, "GB/s", "hbm", peaks, "measured", 123, "k")
    assert r["peak"] == 6000.0 and r["frac"] == 0.75 and r["traffic"] == 123


@pytest.mark.parametrize("kind", ["decode", "decode_fp8", "prefill", "prefill_fp8"])
def test_committed_traffic_matches_current_kernel_sources(kind):
    """The DRAM traffic a bench line reports comes from an ncu capture of the kernel as
    committed; once the kernel's sources change, the figure no longer describes it."""
    assert bench.measured_traffic(kind) is not None, (
        "kernel sources changed since the traffic capture: %s" % bench.kernel_sources_sha(kind.split("_")[0]))
    assert bench.measured_traffic(kind) > 0


def test_traffic_lookup_rejects_other_sources(monkeypatch):
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "decode", {"bytes": 1, "sources": "0" * 16})
    assert bench.measured_traffic("decode") is None
