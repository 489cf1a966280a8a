"""Paged KV append, written out plainly (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this module; the product path never does.

What it computes: the step that runs before paged attention and writes the
new tokens' keys and values into the paged cache (ReshapeAndCache in "[CUDA]
PagedAttention: add SM<80 fp16 fallback via memory-efficient attention",
Implementation step 1; the K_new / AppendKV path of "Rope dim").  Reading of
where a new token goes (the pages do not spell it out): sequence b holds
seqused_k[b] cached tokens before the call; its i-th new token (row
cu_seqlens_new[b] + i of k_new / v_new) becomes cache position
p = seqused_k[b] + i, stored at row p % block_size of page
block_table[b][p // block_size].  Afterwards the sequence holds
seqused_k[b] + n_b tokens.  Nothing else in the cache changes.
"""
from __future__ import annotations

import numpy as np
import torch


def _np(x):
    return x.detach().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)


def kv_append_paged(k_cache, v_cache, k_new, v_new, block_table, cu_seqlens_new, seqused_k,
                    block_size=16):
    """Returns (k_cache', v_cache', seqused_k') with the new tokens written in.

    k_cache, v_cache [num_blocks, block_size, Hkv, D] (any dtype, copied, not
    modified); k_new, v_new [total_new, Hkv, D] of the same dtype;
    block_table int32 [B, max_blocks_per_seq]; cu_seqlens_new int32 [B + 1];
    seqused_k int32 [B] (lengths before).  Raises ValueError when a new token
    would fall outside the sequence's block table or on a page index outside
    the cache.
    """
    kc = k_cache.clone()
    vc = v_cache.clone()
    bt = _np(block_table).astype(np.int64)
    cu = _np(cu_seqlens_new).astype(np.int64)
    used = _np(seqused_k).astype(np.int64)
    num_blocks = kc.shape[0]
    B = len(cu) - 1
    after = used.copy()
    for b in range(B):
        n = int(cu[b + 1] - cu[b])
        for i in range(n):
            p = int(used[b]) + i
            slot = p // block_size
            if slot >= bt.shape[1]:
                raise ValueError("sequence %d: position %d is beyond its block table" % (b, p))
            page = int(bt[b, slot])
            if not 0 <= page < num_blocks:
                raise ValueError("sequence %d: page index %d outside the cache" % (b, page))
            row = p % block_size
            kc[page, row] = k_new[cu[b] + i]
            vc[page, row] = v_new[cu[b] + i]
        after[b] = used[b] + n
    return kc, vc, torch.from_numpy(after.astype(np.int32))
