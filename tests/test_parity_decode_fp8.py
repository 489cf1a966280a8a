"""fp8 e4m3 paged decode vs the fp64 oracle.

The query and the cache hold e4m3 codes with per-tensor fp32 descales (real
value = code x descale), the layout of the fp8 path of "Enforce Q,K,V memory
layouts for fp8 flex attention" (per-tensor scaling), applied to the paged
decode of "[CUDA] PagedAttention: add SM<80 fp16 fallback via memory-efficient
attention".  The oracle is fed the dequantised values, so the only differences
are the kernel's rounding: P in f16 before P.V, fp32 accumulation, O rounded to
bf16.  Tolerances: max |O - O_ref| <= 6e-2 (the fp8 bound) and, because the
logits are exact products of the codes summed in fp32, max |LSE - LSE_ref| <= 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from attention_paged_kv_gqa_b200 import binding as A
from attention_paged_kv_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_O_FP8, TOL_LSE = 6e-2, 1e-3
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert A.attn_check_device(0) == 0, "not a B200 or the kernel image does not load"
    torch.cuda.set_device(0)


def _quantised(t, dequantise=True):
    """e4m3 codes and descales of q and the two caches (plus, by default, their
    dequantised values)."""
    out = {}
    for name in ("q", "k_cache", "v_cache"):
        codes, ds = W.quantize_e4m3(t[name])
        out[name] = codes
        out["descale_" + name] = ds
        if dequantise:
            out[name + "_deq"] = oracle.dequant_e4m3(codes, ds)
    return out


def _run(qz, t, **kw):
    dev = {k: v.to(DEV) for k, v in qz.items() if not k.endswith("_deq")}
    o, lse = A.attn_decode_paged(dev["q"], dev["k_cache"], dev["v_cache"],
                                 t["block_table"].to(DEV), t["seqused_k"].to(DEV),
                                 descale_q=dev["descale_q"], descale_k=dev["descale_k_cache"],
                                 descale_v=dev["descale_v_cache"], **kw)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    return o, lse


def _cmp(o, lse, o_ref, lse_ref, what):
    o = np.asarray(o.float().cpu().numpy(), np.float64)
    lse = np.asarray(lse.float().cpu().numpy(), np.float64)
    assert np.all(np.isfinite(o)), what + ": non-finite output"
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    assert err_o <= TOL_O_FP8, "%s: max|O err| %.3g" % (what, err_o)
    ninf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), ninf), what + ": -inf rows differ"
    assert np.all(o[ninf.reshape(o.shape[:2])] == 0.0), what + ": empty rows not zero"
    if (~ninf).any():
        err_l = float(np.max(np.abs(lse[~ninf] - lse_ref[~ninf])))
        assert err_l <= TOL_LSE, "%s: max|LSE err| %.3g" % (what, err_l)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 4), (4, 1), (16, 8), (16, 1), (8, 8)])
def test_decode_fp8_many_sequences(Hq, Hkv, D):
    """Empty, one-key, page-edge and long sequences, so CTA shares start and end
    inside sequences and pages end ragged.  At head_dim 64 an e4m3 row is 64 bytes
    (the 64-byte swizzle)."""
    lens = [0, 1, 5, 16, 17, 31, 300, 0, 2048, 64, 65, 1000, 7, 129, 3000, 15] * 3
    w = W.paged_decode(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, num_blocks=2000, lmax=3072, lens=lens,
                       seed=5 * Hq + Hkv + D)
    t = w.tensors
    qz = _quantised(t)
    o, lse = _run(qz, t, scale=w.params["scale"])
    o_ref, lse_ref = oracle.attn_decode(qz["q_deq"], qz["k_cache_deq"], qz["v_cache_deq"],
                                        t["block_table"], t["seqused_k"], scale=w.params["scale"])
    _cmp(o, lse, o_ref, lse_ref, "fp8 decode D%d Hq%d Hkv%d" % (D, Hq, Hkv))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("window_left,softcap", [(0, 0.0), (37, 0.0), (-1, 30.0), (200, 15.0)])
def test_decode_fp8_window_softcap(window_left, softcap, D):
    lens = [1, 2, 16, 17, 40, 255, 256, 1500, 0, 33]
    w = W.paged_decode(B=len(lens), Hq=16, Hkv=4, D=D, num_blocks=400, lmax=1536, lens=lens,
                       seed=71 + window_left + D)
    t = w.tensors
    qz = _quantised(t)
    o, lse = _run(qz, t, scale=w.params["scale"], window_left=window_left, softcap=softcap)
    o_ref, lse_ref = oracle.attn_decode(qz["q_deq"], qz["k_cache_deq"], qz["v_cache_deq"],
                                        t["block_table"], t["seqused_k"], scale=w.params["scale"],
                                        window_left=window_left, softcap=softcap)
    _cmp(o, lse, o_ref, lse_ref, "fp8 decode window %d softcap %g" % (window_left, softcap))


def test_decode_fp8_large_descales():
    """Codes near the e4m3 maximum with descales far from 1: the descales must be
    folded into the logit scale and the output exactly once."""
    lens = [500, 17, 1024, 3]
    w = W.paged_decode(B=len(lens), Hq=8, Hkv=2, D=128, num_blocks=200, lmax=1024, lens=lens,
                       seed=9)
    t = dict(w.tensors)
    t["q"] = (t["q"].float() * 0.05).bfloat16()
    t["k_cache"] = (t["k_cache"].float() * 3.0).bfloat16()
    t["v_cache"] = (t["v_cache"].float() * 40.0).bfloat16()
    qz = _quantised(t)
    o, lse = _run(qz, t, scale=w.params["scale"])
    o_ref, lse_ref = oracle.attn_decode(qz["q_deq"], qz["k_cache_deq"], qz["v_cache_deq"],
                                        t["block_table"], t["seqused_k"], scale=w.params["scale"])
    # O scales with the values (|v| up to ~200): compare relative to that range
    o_n = o.float() / 40.0
    _cmp(o_n, lse, o_ref / 40.0, lse_ref, "fp8 decode large descales")


def test_decode_fp8_full_size():
    """The paged GQA decode workload (B=32, Hq=32, Hkv=8, D=128, L ~ U[1, 8192], 20000-page
    pool) with q and the cache quantised to e4m3: every sequence against the oracle."""
    w = W.FULL_SIZE["paged_gqa_decode_bf16"]()
    t = w.tensors
    qz = _quantised(t, dequantise=False)
    o, lse = _run(qz, t, scale=w.params["scale"])
    lens = t["seqused_k"].numpy()
    q_deq = oracle.dequant_e4m3(qz["q"], qz["descale_q"])
    for b in range(len(lens)):
        n = (int(lens[b]) + 15) // 16
        pages = t["block_table"][b, :n].long()
        bt = torch.arange(n, dtype=torch.int32)[None]
        kc = oracle.dequant_e4m3(qz["k_cache"][pages], qz["descale_k_cache"])
        vc = oracle.dequant_e4m3(qz["v_cache"][pages], qz["descale_v_cache"])
        o_ref, lse_ref = oracle.attn_decode(q_deq[b:b + 1], kc, vc, bt, t["seqused_k"][b:b + 1],
                                            scale=w.params["scale"])
        _cmp(o[b:b + 1], lse[b:b + 1], o_ref, lse_ref, "fp8 decode b%d" % b)
