"""Python binding of libattn_b200.so (argument marshalling only).

Every function here has the name of the C entry point it calls (declared in
include/attn_b200.h).  It takes torch tensors, allocates the outputs with torch
when they are not given, passes raw device pointers, sizes and the current
CUDA stream, and raises ``AttnError`` on a non-OK status.  All arithmetic
happens in the CUDA kernels; there is no fallback: if the library is missing
or the device is not a B200, the call raises.
"""
from __future__ import annotations

import ctypes
import math
from pathlib import Path

import torch

_LIB_PATH = Path(__file__).resolve().parent / "libattn_b200.so"
_lib = None

MASK_NONE, MASK_CAUSAL, MASK_PATCH = 0, 1, 2
BF16, FP8_E4M3 = 0, 1


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, status_string(status), status))


def library_path() -> Path:
    return _LIB_PATH


def lib():
    """Loads the CUDA library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not _LIB_PATH.exists():
            raise RuntimeError("libattn_b200.so is not built; run "
                               "`python -m attention_paged_kv_gqa_b200.build`")
        L = ctypes.CDLL(str(_LIB_PATH))
        P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.attn_check_device.argtypes = [I]
        L.attn_check_device.restype = I
        L.attn_status_string.argtypes = [I]
        L.attn_status_string.restype = ctypes.c_char_p
        L.attn_device_error.argtypes = [ctypes.POINTER(I), P]
        L.attn_device_error.restype = I
        L.attn_selftest_wait_expiry.argtypes = [ctypes.c_longlong, P]
        L.attn_selftest_wait_expiry.restype = I
        L.attn_fwd_dense.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P, P, F, I, I, F, I,
                                     P, P, P, P]
        L.attn_fwd_dense.restype = I
        L.attn_fwd_varlen_paged.argtypes = [P, P, P, P, I, I, I, P, P, P, I, I, I, I, I, I, I,
                                            F, I, P, I, F, I, P, P, P, P, P, P, Z, P]
        L.attn_fwd_varlen_paged.restype = I
        L.attn_fwd_varlen_paged_only_qv.argtypes = [P, P, P, I, I, I, P, P, P, I, I, I, I, I, I, I,
                                                    F, I, P, I, F, I, P, P, P, P, P]
        L.attn_fwd_varlen_paged_only_qv.restype = I
        L.attn_decode_paged_only_qv.argtypes = [P, P, P, I, I, I, P, I, I, I, I, F, I, F, I, I, P, P,
                                                P, Z, P]
        L.attn_decode_paged_only_qv.restype = I
        L.attn_fwd_patch.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, I, P, P, P, P, P, P]
        L.attn_fwd_patch.restype = I
        L.attn_decode_workspace_size.argtypes = [I, I, I, I, I, I, I]
        L.attn_decode_workspace_size.restype = Z
        L.attn_decode_paged.argtypes = [P, P, P, P, I, I, I, P, I, I, I, I, F, I, F, I, I, P, P,
                                        P, P, P, P, Z, P]
        L.attn_decode_paged.restype = I
        L.attn_fwd_varlen_paged_qv.argtypes = [P, P, P, P, P, I, I, I, P, P, P, I, I, I, I, I, I,
                                               I, F, I, P, I, F, I, P, P, P]
        L.attn_fwd_varlen_paged_qv.restype = I
        L.attn_decode_paged_qv.argtypes = [P, P, P, P, P, I, I, I, P, I, I, I, I, F, I, F, I, I,
                                           P, P, P, Z, P]
        L.attn_decode_paged_qv.restype = I
        L.attn_decode_paged_noalloc.argtypes = [P, P, P, P, I, I, I, P, I, I, I, I, F, I, P, P, P]
        L.attn_decode_paged_noalloc.restype = I
        L.attn_kv_append_paged.argtypes = [P, P, P, P, P, I, I, I, P, P, P, I, I, I, I, I, P]
        L.attn_kv_append_paged.restype = I
        L.attn_decode_paged_append.argtypes = [P, P, P, P, P, P, I, I, I, P, P, I, I, I, I, F, I, F,
                                               I, I, P, P, P, Z, P]
        L.attn_decode_paged_append.restype = I
        L.attn_bwd_workspace_size.argtypes = [I, I]
        L.attn_bwd_workspace_size.restype = Z
        L.attn_bwd_varlen.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F,
                                      I, I, P, Z, P]
        L.attn_bwd_varlen.restype = I
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != 0:
        raise AttnError(status, where)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float8_e4m3fn:
        return FP8_E4M3
    raise TypeError("q/k/v must be bfloat16 or float8_e4m3fn, got %s" % t.dtype)


def _scale(scale):
    return 0.0 if scale is None else float(scale)


def _strides3(t: torch.Tensor):
    if t.stride(-1) != 1:
        raise ValueError("head_dim must be the contiguous dimension")
    return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))


def attn_check_device(device: int = 0) -> int:
    return lib().attn_check_device(int(device))


def attn_device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    st = lib().attn_device_error(ctypes.byref(code), _stream(stream))
    if st not in (0, 7, 9):
        _check(st, "attn_device_error")
    return code.value


def attn_selftest_wait_expiry(limit_ns: int, stream=None):
    """Launches the bounded-wait test kernel (a wait nothing satisfies, limited to limit_ns)."""
    _check(lib().attn_selftest_wait_expiry(int(limit_ns), _stream(stream)),
           "attn_selftest_wait_expiry")


def attn_fwd_dense(q, k, v, *, causal=False, scale=None, window_left=-1, softcap=0.0,
                   descale_q=None, descale_k=None, descale_v=None, out=None, lse=None,
                   return_lse=True, stream=None):
    """q [B, Lq, Hq, D], k/v [B, Lk, Hkv, D] -> (o [B, Lq, Hq, D] bf16, lse [B, Hq, Lq] fp32).

    window_left >= 0 (causal only): row i keeps keys i' - window_left .. i';
    softcap > 0: each logit s becomes softcap * tanh(s / softcap).
    """
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    if out is None:
        out = torch.empty((B, Lq, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    st = lib().attn_fwd_dense(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Lq, Lk, Hq, Hkv,
                              D, _strides3(q), _strides3(k), _strides3(v), _scale(scale),
                              MASK_CAUSAL if causal else MASK_NONE, int(window_left),
                              float(softcap), _dtype_code(q),
                              _ptr(descale_q), _ptr(descale_k), _ptr(descale_v), _stream(stream))
    _check(st, "attn_fwd_dense")
    return out, lse


def attn_fwd_varlen_paged(q, k_cache, v_cache, *, cu_seqlens_q, max_seqlen_q, block_table=None,
                          cu_seqlens_k=None, seqused_k=None, mask=MASK_NONE, scale=None,
                          patch_kv_range=None, window_left=-1, softcap=0.0, descale_q=None,
                          descale_k=None, descale_v=None, out=None, lse=None, return_lse=True,
                          stream=None):
    """q [total_q, Hq, D]; paged k/v [num_blocks, 16, Hkv, D] (or packed [total_k, Hkv, D]).

    Returns (o [total_q, Hq, D] bf16, lse [Hq, total_q] fp32).
    """
    total_q, Hq, D = q.shape
    B = cu_seqlens_q.numel() - 1
    if block_table is not None:
        num_blocks, block_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
        mbps, total_k = block_table.shape[1], 0
    else:
        num_blocks, block_size, mbps = 0, 0, 0
        total_k, Hkv = k_cache.shape[0], k_cache.shape[1]
    if out is None:
        out = torch.empty((total_q, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    st = lib().attn_fwd_varlen_paged(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), mbps, num_blocks, block_size,
        _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), _ptr(seqused_k), B, total_q, total_k,
        int(max_seqlen_q), Hq, Hkv, D, _scale(scale), int(mask), _ptr(patch_kv_range),
        int(window_left), float(softcap), _dtype_code(q), _ptr(descale_q), _ptr(descale_k), _ptr(descale_v), _ptr(out), _ptr(lse),
        None, 0, _stream(stream))
    _check(st, "attn_fwd_varlen_paged")
    return out, lse


def attn_fwd_varlen_paged_only_qv(qv, v_cache, *, cu_seqlens_q, max_seqlen_q, block_table=None,
                                  cu_seqlens_k=None, seqused_k=None, mask=MASK_NONE, scale=None,
                                  patch_kv_range=None, window_left=-1, softcap=0.0,
                                  descale_qv=None, descale_v=None, out=None, lse=None,
                                  return_lse=True, stream=None):
    """The only_qv score (scale * qv . v): qv [total_q, Hq, D]; v paged or packed as in
    attn_fwd_varlen_paged.  Returns (o [total_q, Hq, D] bf16, lse [Hq, total_q] fp32)."""
    total_q, Hq, D = qv.shape
    B = cu_seqlens_q.numel() - 1
    if block_table is not None:
        num_blocks, block_size, Hkv = v_cache.shape[0], v_cache.shape[1], v_cache.shape[2]
        mbps, total_k = block_table.shape[1], 0
    else:
        num_blocks, block_size, mbps = 0, 0, 0
        total_k, Hkv = v_cache.shape[0], v_cache.shape[1]
    if out is None:
        out = torch.empty((total_q, Hq, D), dtype=torch.bfloat16, device=qv.device)
    if lse is None and return_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=qv.device)
    st = lib().attn_fwd_varlen_paged_only_qv(
        _ptr(qv), _ptr(v_cache), _ptr(block_table), mbps, num_blocks, block_size,
        _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), _ptr(seqused_k), B, total_q, total_k,
        int(max_seqlen_q), Hq, Hkv, D, _scale(scale), int(mask), _ptr(patch_kv_range),
        int(window_left), float(softcap), _dtype_code(qv), _ptr(descale_qv), _ptr(descale_v),
        _ptr(out), _ptr(lse), _stream(stream))
    _check(st, "attn_fwd_varlen_paged_only_qv")
    return out, lse


def attn_fwd_varlen_paged_qv(q, qv, k_cache, v_cache, *, cu_seqlens_q, max_seqlen_q,
                             block_table=None, cu_seqlens_k=None, seqused_k=None, mask=MASK_NONE,
                             scale=None, patch_kv_range=None, window_left=-1, softcap=0.0,
                             out=None, lse=None, return_lse=True, stream=None):
    """The forward with the Qv score term, scale * (q.k + qv.v): q, qv [total_q, Hq, D] bf16;
    K/V paged or packed as in attn_fwd_varlen_paged.
    Returns (o [total_q, Hq, D] bf16, lse [Hq, total_q] fp32)."""
    total_q, Hq, D = q.shape
    B = cu_seqlens_q.numel() - 1
    if block_table is not None:
        num_blocks, block_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
        mbps, total_k = block_table.shape[1], 0
    else:
        num_blocks, block_size, mbps = 0, 0, 0
        total_k, Hkv = k_cache.shape[0], k_cache.shape[1]
    if out is None:
        out = torch.empty((total_q, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    st = lib().attn_fwd_varlen_paged_qv(
        _ptr(q), _ptr(qv), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), mbps, num_blocks,
        block_size, _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), _ptr(seqused_k), B, total_q, total_k,
        int(max_seqlen_q), Hq, Hkv, D, _scale(scale), int(mask), _ptr(patch_kv_range),
        int(window_left), float(softcap), _dtype_code(q), _ptr(out), _ptr(lse), _stream(stream))
    _check(st, "attn_fwd_varlen_paged_qv")
    return out, lse


def attn_fwd_patch(q, k, v, *, cu_seqlens_q, cu_seqlens_k, patch_kv_range, max_seqlen_q,
                   max_interval, scale=None, descale_q=None, descale_k=None, descale_v=None,
                   out=None, lse=None, return_lse=True, stream=None):
    """Patch cross-attention with intervals of at most max_interval keys (see the header):
    q [total_q, Hq, D], packed k/v [total_k, Hkv, D] -> (o, lse [Hq, total_q])."""
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty((total_q, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    st = lib().attn_fwd_patch(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                              _ptr(patch_kv_range), B, total_q, total_k, int(max_seqlen_q), Hq, Hkv, D,
                              _scale(scale), int(max_interval), _dtype_code(q), _ptr(descale_q),
                              _ptr(descale_k), _ptr(descale_v), _ptr(out), _ptr(lse), _stream(stream))
    _check(st, "attn_fwd_patch")
    return out, lse


def attn_decode_workspace_size(B, num_heads_q, num_heads_kv, head_dim, max_blocks_per_seq,
                               block_size=16, num_splits=0) -> int:
    return int(lib().attn_decode_workspace_size(B, num_heads_q, num_heads_kv, head_dim,
                                                max_blocks_per_seq, block_size, num_splits))


def attn_decode_paged(q, k_cache, v_cache, block_table, seqused_k, *, scale=None, num_splits=0,
                      window_left=-1, softcap=0.0, descale_q=None, descale_k=None,
                      descale_v=None, out=None, lse=None, workspace=None, return_lse=True,
                      stream=None):
    """q [B, Hq, D] against a paged cache -> (o [B, Hq, D] bf16, lse [B, Hq] fp32).

    The query is the newest cached token; window_left >= 0 keeps the keys
    L-1-window_left .. L-1; softcap > 0 caps the logits as in the prefill calls.
    With q and the cache in float8_e4m3fn, descale_q/k/v ([Hkv] fp32 each) are
    required (head_dim 128, automatic split).
    """
    B, Hq, D = q.shape
    num_blocks, block_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    mbps = block_table.shape[1]
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws_bytes = attn_decode_workspace_size(B, Hq, Hkv, D, mbps, block_size, num_splits)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    st = lib().attn_decode_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), mbps,
                                 num_blocks, block_size, _ptr(seqused_k), B, Hq, Hkv, D,
                                 _scale(scale), int(window_left), float(softcap), int(num_splits),
                                 _dtype_code(q), _ptr(descale_q), _ptr(descale_k), _ptr(descale_v),
                                 _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                                 _stream(stream))
    _check(st, "attn_decode_paged")
    return out, lse


def attn_decode_paged_qv(q, qv, k_cache, v_cache, block_table, seqused_k, *, scale=None,
                         num_splits=0, window_left=-1, softcap=0.0, out=None, lse=None,
                         workspace=None, return_lse=True, stream=None):
    """Paged decode whose logit adds the Qv term: scale * (q.k + qv.v).

    q, qv [B, Hq, D] bf16 -> (o [B, Hq, D] bf16, lse [B, Hq] fp32); arguments as
    attn_decode_paged.
    """
    B, Hq, D = q.shape
    num_blocks, block_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    mbps = block_table.shape[1]
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws_bytes = attn_decode_workspace_size(B, Hq, Hkv, D, mbps, block_size, num_splits)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    st = lib().attn_decode_paged_qv(_ptr(q), _ptr(qv), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(block_table), mbps, num_blocks, block_size,
                                    _ptr(seqused_k), B, Hq, Hkv, D, _scale(scale),
                                    int(window_left), float(softcap), int(num_splits),
                                    _dtype_code(q), _ptr(out), _ptr(lse), _ptr(workspace),
                                    workspace.numel(), _stream(stream))
    _check(st, "attn_decode_paged_qv")
    return out, lse


def attn_decode_paged_only_qv(qv, v_cache, block_table, seqused_k, *, scale=None, num_splits=0,
                              window_left=-1, softcap=0.0, out=None, lse=None, workspace=None,
                              return_lse=True, stream=None):
    """Paged decode with the only_qv score: qv [B, Hq, D] -> (o [B, Hq, D] bf16, lse [B, Hq])."""
    B, Hq, D = qv.shape
    num_blocks, block_size, Hkv = v_cache.shape[0], v_cache.shape[1], v_cache.shape[2]
    mbps = block_table.shape[1]
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=qv.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=qv.device)
    ws_bytes = attn_decode_workspace_size(B, Hq, Hkv, D, mbps, block_size, num_splits)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=qv.device)
    st = lib().attn_decode_paged_only_qv(_ptr(qv), _ptr(v_cache), _ptr(block_table), mbps,
                                         num_blocks, block_size, _ptr(seqused_k), B, Hq, Hkv, D,
                                         _scale(scale), int(window_left), float(softcap),
                                         int(num_splits), _dtype_code(qv), _ptr(out), _ptr(lse),
                                         _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "attn_decode_paged_only_qv")
    return out, lse


def attn_decode_paged_noalloc(q, k_cache, v_cache, block_table, seqused_k, *, scale=None,
                              out=None, lse=None, return_lse=True, stream=None):
    """attn_decode_paged whose split-KV scratch is the library's fixed device array.

    For callers that must not allocate device memory while they run: the C
    call allocates nothing (the outputs are allocated here only when not given).
    """
    B, Hq, D = q.shape
    num_blocks, block_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    st = lib().attn_decode_paged_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                         block_table.shape[1], num_blocks, block_size,
                                         _ptr(seqused_k), B, Hq, Hkv, D, _scale(scale),
                                         _dtype_code(q), _ptr(out), _ptr(lse), _stream(stream))
    _check(st, "attn_decode_paged_noalloc")
    return out, lse


def attn_kv_append_paged(k_new, v_new, k_cache, v_cache, block_table, seqused_k, *,
                         cu_seqlens_new=None, seqused_k_out=None, stream=None):
    """Writes new tokens' K/V ([total_new, Hkv, D]) into the paged cache in place.

    Sequence b's i-th new token goes to position seqused_k[b] + i.  Returns
    seqused_k_out (lengths after), allocated here when not given.
    cu_seqlens_new None means one new token per sequence.
    """
    total_new, Hkv, D = k_new.shape
    B = seqused_k.numel()
    num_blocks, block_size = k_cache.shape[0], k_cache.shape[1]
    if seqused_k_out is None:
        seqused_k_out = torch.empty_like(seqused_k)
    st = lib().attn_kv_append_paged(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(block_table), block_table.shape[1], num_blocks,
                                    block_size, _ptr(cu_seqlens_new), _ptr(seqused_k),
                                    _ptr(seqused_k_out), B, total_new, Hkv, D, _dtype_code(k_new),
                                    _stream(stream))
    _check(st, "attn_kv_append_paged")
    return seqused_k_out


def attn_decode_paged_append(q, k_new, v_new, k_cache, v_cache, block_table, seqused_k, *,
                             seqused_k_out=None, scale=None, num_splits=0, window_left=-1,
                             softcap=0.0, out=None, lse=None, workspace=None, return_lse=True,
                             stream=None):
    """Appends one token per sequence (k_new/v_new [B, Hkv, D]) to the paged cache, then
    decodes q [B, Hq, D] over the updated cache.  Returns (o, lse, seqused_k_out)."""
    B, Hq, D = q.shape
    num_blocks, block_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    mbps = block_table.shape[1]
    if seqused_k_out is None:
        seqused_k_out = torch.empty_like(seqused_k)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws_bytes = attn_decode_workspace_size(B, Hq, Hkv, D, mbps, block_size, num_splits)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    st = lib().attn_decode_paged_append(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), mbps,
        num_blocks, block_size, _ptr(seqused_k), _ptr(seqused_k_out), B, Hq, Hkv, D, _scale(scale),
        int(window_left), float(softcap), int(num_splits), _dtype_code(q), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "attn_decode_paged_append")
    return out, lse, seqused_k_out


def attn_bwd_varlen(q, k, v, o, dout, lse, *, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                    max_seqlen_k, mask=MASK_NONE, scale=None, window_left=-1, dq=None, dk=None,
                    dv=None, workspace=None, stream=None):
    """Gradients of the varlen forward: (dq [total_q, Hq, D], dk, dv [total_k, Hkv, D]).

    q, o, dout [total_q, Hq, D] bf16; k, v [total_k, Hkv, D] bf16; lse [Hq, total_q]
    fp32 from the forward.
    """
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.numel() - 1
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws_bytes = int(lib().attn_bwd_workspace_size(Hq, total_q))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    st = lib().attn_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                               _ptr(dk), _ptr(dv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B,
                               total_q, total_k, int(max_seqlen_q), int(max_seqlen_k), Hq, Hkv, D,
                               _scale(scale), int(mask), int(window_left), _ptr(workspace),
                               workspace.numel(), _stream(stream))
    _check(st, "attn_bwd_varlen")
    return dq, dk, dv


def attn_bwd_dense(q, k, v, o, dout, lse, *, causal=False, scale=None, window_left=-1,
                   stream=None):
    """Dense [B, L, H, D] convenience over attn_bwd_varlen (lse [B, Hq, Lq] from
    attn_fwd_dense).  Returns (dq, dk, dv) in the dense layouts."""
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    cq = torch.arange(B + 1, dtype=torch.int32, device=dev) * Lq
    ck = torch.arange(B + 1, dtype=torch.int32, device=dev) * Lk
    lse_v = lse.permute(1, 0, 2).reshape(Hq, B * Lq).contiguous()
    dq, dk, dv = attn_bwd_varlen(q.reshape(B * Lq, Hq, D), k.reshape(B * Lk, Hkv, D),
                                 v.reshape(B * Lk, Hkv, D), o.reshape(B * Lq, Hq, D),
                                 dout.reshape(B * Lq, Hq, D), lse_v, cu_seqlens_q=cq,
                                 cu_seqlens_k=ck, max_seqlen_q=Lq, max_seqlen_k=Lk,
                                 mask=MASK_CAUSAL if causal else MASK_NONE, scale=scale,
                                 window_left=window_left, stream=stream)
    return dq.reshape(B, Lq, Hq, D), dk.reshape(B, Lk, Hkv, D), dv.reshape(B, Lk, Hkv, D)
