"""fp64 CPU oracle for the attention forward (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product path (the CUDA library and its
Python binding) never imports, links or calls it, and it imports nothing from
the product: it shares only the seeded input generators, which hold none of
the method's arithmetic.

The arithmetic lives in ``attn_oracle.c`` (plain fp64 loops, built here with
gcc); this module only converts tensors to fp64 arrays and back.  A second,
independent formulation for tiny inputs lives in ``brute.py``.

Every function follows the plain definition
    O = softmax(scale * Q K^T + mask) V,   LSE = ln sum_j exp(scale * q.k_j)
as given by the FlexAttention docstring and lowering arguments ("[FlexAttention]
Enforce Q,K,V memory layouts for fp8 flex attention", flex_attention
docstring; "Cross Attention does not work on CPU and older GPUs",
OUTPUT_LOGSUMEXP), with the paged/varlen/GQA addressing of "[CUDA]
PagedAttention: add SM<80 fp16 fallback via memory-efficient attention",
Implementation steps 2-3.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np
import torch

MASK_NONE, MASK_CAUSAL, MASK_PATCH = 0, 1, 2

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "attn_oracle.c"
_LIB_PATH = _HERE / "_build" / "libattn_oracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile the C oracle with gcc (-O2, OpenMP) into oracle/_build/."""
    _LIB_PATH.parent.mkdir(parents=True, exist_ok=True)
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(".so.tmp%d" % os.getpid())
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               str(_SRC), "-o", str(tmp), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def bind(lib):
    """Declares the C oracle's signatures on a loaded library handle."""
    P = ctypes.c_void_p
    I = ctypes.c_int
    D = ctypes.c_double
    lib.attn_oracle_fwd.restype = I
    lib.attn_oracle_fwd.argtypes = [P, P, P, P, I, I, P, P, P, I, I, I, I,
                                    D, I, P, I, D, P, P, I, I]
    lib.attn_oracle_combine.restype = None
    lib.attn_oracle_combine.argtypes = [P, P, I, I, I, P, P]
    lib.attn_oracle_fwd_qv.restype = I
    lib.attn_oracle_fwd_qv.argtypes = [P, P, P, P, P, I, I, P, P, P, I, I, I, I, D, I, P, I, D, I,
                                       P, P, I, I]
    lib.attn_oracle_bwd.restype = I
    lib.attn_oracle_bwd.argtypes = [P, P, P, P, P, P, I, I, I, I, D, I, I, P, P, P, I]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(ctypes.CDLL(str(build())))
    return _lib


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().to(torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _i32(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def dequant_e4m3(x_fp8: torch.Tensor, descale) -> torch.Tensor:
    """e4m3 codes -> fp64 values times the per-tensor descale (same values the GPU sees)."""
    return x_fp8.to(torch.float64) * float(torch.as_tensor(descale).reshape(-1)[0])


def default_scale(head_dim: int) -> float:
    """1/sqrt(E), the default softmax scale of the FlexAttention docstring."""
    return 1.0 / float(np.sqrt(head_dim))


def attn_varlen(q, k, v, *, cu_seqlens_q, num_heads_kv, scale, mask=MASK_NONE,
                cu_seqlens_k=None, seqused_k=None, block_table=None, block_size=16,
                patch_kv_range=None, window_left=-1, softcap=0.0, nthreads=None):
    """Varlen / paged attention forward in fp64.

    q [total_q, Hq, D]; k, v either [total_k, Hkv, D] (block_table None) or
    paged [num_blocks, block_size, Hkv, D].  Returns (O [total_q, Hq, D],
    LSE [Hq, total_q]) as fp64 numpy arrays.  window_left >= 0 (causal mask
    only) keeps the keys i' - window_left <= j <= i' of row i (i' = i + Lk -
    Lq); softcap > 0 maps each scaled score s to softcap * tanh(s / softcap).
    """
    lib = _load()
    qa, ka, va = _f64(q), _f64(k), _f64(v)
    total_q, Hq, D = qa.shape
    cq = _i32(cu_seqlens_q)
    ck = _i32(cu_seqlens_k)
    su = _i32(seqused_k)
    bt = _i32(block_table)
    pr = _i32(patch_kv_range)
    B = len(cq) - 1
    mbps = bt.shape[1] if bt is not None else 0
    o = np.zeros((total_q, Hq, D), np.float64)
    lse = np.zeros((Hq, total_q), np.float64)
    if scale is None or scale <= 0:
        scale = default_scale(D)
    rc = lib.attn_oracle_fwd(_ptr(qa), _ptr(ka), _ptr(va), _ptr(bt), mbps, int(block_size),
                             _ptr(cq), _ptr(ck), _ptr(su), B, Hq, int(num_heads_kv), D,
                             float(scale), int(mask), _ptr(pr), int(window_left),
                             float(softcap), _ptr(o), _ptr(lse),
                             total_q, int(nthreads or os.cpu_count() or 1))
    if rc != 0:
        raise ValueError("oracle rejected its arguments (rc=%d)" % rc)
    return o, lse


def attn_dense(q, k, v, *, scale, causal, window_left=-1, softcap=0.0, nthreads=None):
    """Dense [B, L, H, D] attention in fp64: returns O [B, Lq, Hq, D], LSE [B, Hq, Lq]."""
    qa, ka, va = _f64(q), _f64(k), _f64(v)
    B, Lq, Hq, D = qa.shape
    Lk, Hkv = ka.shape[1], ka.shape[2]
    cq = np.arange(B + 1, dtype=np.int32) * Lq
    ck = np.arange(B + 1, dtype=np.int32) * Lk
    o, lse = attn_varlen(qa.reshape(B * Lq, Hq, D), ka.reshape(B * Lk, Hkv, D),
                         va.reshape(B * Lk, Hkv, D), cu_seqlens_q=cq, cu_seqlens_k=ck,
                         num_heads_kv=Hkv, scale=scale,
                         mask=MASK_CAUSAL if causal else MASK_NONE, window_left=window_left,
                         softcap=softcap, nthreads=nthreads)
    return o.reshape(B, Lq, Hq, D), lse.reshape(Hq, B, Lq).transpose(1, 0, 2).copy()


def attn_decode(q, k_cache, v_cache, block_table, seqused_k, *, scale, block_size=16,
                window_left=-1, softcap=0.0, nthreads=None):
    """One query token per sequence against a paged cache: O [B, Hq, D], LSE [B, Hq].

    The query is the newest cached token, so with a sliding window it sees the
    keys Lk - 1 - window_left .. Lk - 1 (causal with Lq = 1 and the window).
    """
    qa = _f64(q)
    B, Hq, D = qa.shape
    Hkv = k_cache.shape[2]
    cq = np.arange(B + 1, dtype=np.int32)
    o, lse = attn_varlen(qa, k_cache, v_cache, cu_seqlens_q=cq, seqused_k=seqused_k,
                         block_table=block_table, block_size=block_size,
                         num_heads_kv=Hkv, scale=scale,
                         mask=MASK_CAUSAL if window_left >= 0 else MASK_NONE,
                         window_left=window_left, softcap=softcap, nthreads=nthreads)
    return o, lse.T.copy()


def combine(o_parts, lse_parts):
    """Merge split-KV partials: o_parts [S, N, D], lse_parts [S, N] -> (O [N, D], LSE [N])."""
    lib = _load()
    op, lp = _f64(o_parts), _f64(lse_parts)
    S, N, D = op.shape
    o = np.zeros((N, D), np.float64)
    lse = np.zeros(N, np.float64)
    lib.attn_oracle_combine(_ptr(op), _ptr(lp), S, N, D, _ptr(o), _ptr(lse))
    return o, lse


def attn_bwd_varlen(q, k, v, do, *, cu_seqlens_q, cu_seqlens_k, num_heads_kv, scale,
                    mask=MASK_NONE, window_left=-1, nthreads=None):
    """Gradients of the varlen forward in fp64: (dQ [total_q, Hq, D], dK, dV [total_k, Hkv, D]).

    q, do [total_q, Hq, D]; k, v [total_k, Hkv, D] (packed, no paging).  The
    forward's O and LSE are recomputed exactly from q, k, v.
    """
    lib = _load()
    qa, ka, va, da = _f64(q), _f64(k), _f64(v), _f64(do)
    total_q, Hq, D = qa.shape
    cq, ck = _i32(cu_seqlens_q), _i32(cu_seqlens_k)
    B = len(cq) - 1
    dq = np.zeros_like(qa)
    dk = np.zeros_like(ka)
    dv = np.zeros_like(va)
    if scale is None or scale <= 0:
        scale = default_scale(D)
    rc = lib.attn_oracle_bwd(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), _ptr(cq), _ptr(ck), B, Hq,
                             int(num_heads_kv), D, float(scale), int(mask), int(window_left),
                             _ptr(dq), _ptr(dk), _ptr(dv), int(nthreads or os.cpu_count() or 1))
    if rc != 0:
        raise ValueError("oracle rejected its arguments (rc=%d)" % rc)
    return dq, dk, dv


def attn_bwd_dense(q, k, v, do, *, scale, causal, window_left=-1, nthreads=None):
    """Dense [B, L, H, D] gradients in fp64: (dQ [B, Lq, Hq, D], dK, dV [B, Lk, Hkv, D])."""
    qa, ka, va, da = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Lq, Hq, D = qa.shape
    Lk, Hkv = ka.shape[1], ka.shape[2]
    cq = np.arange(B + 1, dtype=np.int32) * Lq
    ck = np.arange(B + 1, dtype=np.int32) * Lk
    dq, dk, dv = attn_bwd_varlen(qa.reshape(B * Lq, Hq, D), ka.reshape(B * Lk, Hkv, D),
                                 va.reshape(B * Lk, Hkv, D), da.reshape(B * Lq, Hq, D),
                                 cu_seqlens_q=cq, cu_seqlens_k=ck, num_heads_kv=Hkv, scale=scale,
                                 mask=MASK_CAUSAL if causal else MASK_NONE,
                                 window_left=window_left, nthreads=nthreads)
    return dq.reshape(B, Lq, Hq, D), dk.reshape(B, Lk, Hkv, D), dv.reshape(B, Lk, Hkv, D)


def attn_varlen_qv(q, qv, k, v, *, cu_seqlens_q, num_heads_kv, scale, cu_seqlens_k=None,
                   block_table=None, seqused_k=None, mask=MASK_NONE, patch_kv_range=None,
                   window_left=-1, softcap=0.0, only_qv=False, nthreads=None):
    """Forward with the extra Qv score term: s = scale * (q.k + qv.v) (only_qv: scale * qv.v).

    q, qv [total_q, Hq, D] (q and k may be None with only_qv); k, v packed
    [total_k, Hkv, D] addressed by cu_seqlens_k, or paged [num_blocks, bs, Hkv, D]
    through block_table.  Masks, window and softcap as attn_varlen.
    Returns (O [total_q, Hq, D], LSE [Hq, total_q]).
    """
    lib = _load()
    qva, va = _f64(qv), _f64(v)
    qa = None if only_qv else _f64(q)
    ka = None if only_qv else _f64(k)
    total_q, Hq, D = qva.shape
    cq = _i32(cu_seqlens_q)
    ck = None if cu_seqlens_k is None else _i32(cu_seqlens_k)
    bt = None if block_table is None else _i32(block_table)
    su = None if seqused_k is None else _i32(seqused_k)
    pr = None if patch_kv_range is None else _i32(patch_kv_range)
    B = len(cq) - 1
    mbps = 0 if bt is None else bt.shape[1]
    bs = 0 if bt is None else va.shape[1]
    o = np.zeros((total_q, Hq, D), np.float64)
    lse = np.zeros((Hq, total_q), np.float64)
    if scale is None or scale <= 0:
        scale = default_scale(D)
    rc = lib.attn_oracle_fwd_qv(_ptr(qa), _ptr(qva), _ptr(ka), _ptr(va), _ptr(bt), mbps, bs, _ptr(cq),
                                _ptr(ck), _ptr(su), B, Hq, int(num_heads_kv), D, float(scale),
                                int(mask), _ptr(pr), int(window_left), float(softcap),
                                int(bool(only_qv)), _ptr(o), _ptr(lse), total_q,
                                int(nthreads or os.cpu_count() or 1))
    if rc != 0:
        raise ValueError("oracle rejected its arguments (rc=%d)" % rc)
    return o, lse
