// append.cuh -- paged KV append: writes new tokens' keys and values into the
// paged cache through block_table (the ReshapeAndCache step of "[CUDA]
// PagedAttention: add SM<80 fp16 fallback via memory-efficient attention",
// Implementation step 1; the K_new / AppendKV path of "Rope dim").
//
// Sequence b holds seqused_k[b] cached tokens; its i-th new token (row
// cu_new[b] + i of k_new / v_new) becomes cache position p = seqused_k[b] + i,
// row p % 16 of page block_table[b][p / 16].  Pure data movement, HBM bound:
// one warp per new token copies the token's [Hkv][D] rows of K and of V
// (contiguous on both sides) in 16-byte pieces, so reads and writes coalesce.
// A position past the sequence's block table, or a page index outside the
// cache, is not written: the warp records an error code in the device error
// word instead (no out-of-bounds store on bad input).
#pragma once

#include "ptx.cuh"
#include "prefill.cuh"   // kPageRows

namespace attn {

constexpr int kAppendThreads = 256;
enum : int { kErrAppendSlot = 501, kErrAppendPage = 502 };

struct AppendArgs {
    const uint4* k_new;          // [total_new][Hkv][row_bytes / 16]
    const uint4* v_new;
    uint4* k_cache;              // [num_blocks][16][Hkv][row_bytes / 16]
    uint4* v_cache;
    const int* block_table;      // [B][max_blocks]
    int max_blocks, num_blocks;
    const int* cu_new;           // [B + 1], or null: one new token per sequence
    const int* seqused_k;        // [B] lengths before
    int* seqused_k_out;          // [B] lengths after, or null
    int B, total_new;
    int pieces_per_token;        // Hkv * head_dim * element bytes / 16
};

__global__ void __launch_bounds__(kAppendThreads) kv_append_kernel(const AppendArgs a) {
    // A decode launched after this grid as a programmatic dependent may be
    // scheduled now; it waits for this grid's completion before reading.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    const int P = a.pieces_per_token;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < a.total_new; t += warps) {
        // sequence of new token t: the largest b with cu_new[b] <= t (the
        // largest, so that empty sequences before it are passed over)
        int b = t, first = t;
        if (a.cu_new) {
            int lo = 0, hi = a.B;
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (__ldg(&a.cu_new[mid]) <= t) lo = mid; else hi = mid;
            }
            b = lo;
            first = __ldg(&a.cu_new[b]);
        }
        const int p = __ldg(&a.seqused_k[b]) + (t - first);
        const int slot = p >= 0 ? p / kPageRows : -1;
        if (slot < 0 || slot >= a.max_blocks) {
            if (lane == 0) record_data_error(kErrAppendSlot);
            continue;
        }
        const int page = __ldg(&a.block_table[(long long)b * a.max_blocks + slot]);
        if (page < 0 || page >= a.num_blocks) {
            if (lane == 0) record_data_error(kErrAppendPage);
            continue;
        }
        const uint4* __restrict__ ks = a.k_new + (long long)t * P;
        const uint4* __restrict__ vs = a.v_new + (long long)t * P;
        uint4* __restrict__ kd = a.k_cache + ((long long)page * kPageRows + p % kPageRows) * P;
        uint4* __restrict__ vd = a.v_cache + ((long long)page * kPageRows + p % kPageRows) * P;
        // all of a lane's loads of a group are in flight before its stores
        constexpr int U = 4;
        for (int i0 = lane; i0 < P; i0 += 32 * U) {
            uint4 kr[U], vr[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + 32 * u;
                if (i < P) {
                    kr[u] = __ldg(ks + i);
                    vr[u] = __ldg(vs + i);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + 32 * u;
                if (i < P) {
                    kd[i] = kr[u];
                    vd[i] = vr[u];
                }
            }
        }
    }
    if (a.seqused_k_out) {
        for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < a.B; b += gridDim.x * blockDim.x)
            a.seqused_k_out[b] = a.seqused_k[b] + (a.cu_new ? a.cu_new[b + 1] - a.cu_new[b] : 1);
    }
}

}  // namespace attn
