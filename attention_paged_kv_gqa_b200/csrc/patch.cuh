// patch.cuh -- patch-to-byte cross-attention with short key intervals, on the
// CUDA cores.
//
// Query i of sequence b attends to the keys [start_i, end_i) of its sequence
// only (the block / patch mask of the byte-latent model in "Cross Attention
// does not work on CPU and older GPUs": one query per patch, attending to its
// own patch's bytes).  When every interval is short -- the patches there are
// clipped to 16 bytes -- a query reads a handful of keys, and each key belongs
// to one query: the work is reading every K and V row once, about one flop per
// byte.  A 128 x 128 tensor-core score tile would compute two orders of
// magnitude more than the allowed pairs, so this path scores on the CUDA cores.
// patch_query_kernel (the common shapes): one warp per query and all its heads,
// each key row read whole.  patch_kernel (any shape): one warp per (query,
// head); lane j scores key start + c + j of a 32-key chunk (online softmax
// across chunks), then the lanes split D for O = sum_j p_j v_j.  Both take any
// interval length.  Same conventions as the
// prefill: O = softmax(scale q.k) V over the interval, LSE = ln sum exp(scale
// q.k); an empty interval gives O = 0 and LSE = -inf.
#pragma once

#include "prefill.cuh"

namespace attn {

struct PatchArgs {
    const __nv_bfloat16* q;    // [total_q][Hq][D]
    const __nv_bfloat16* k;    // [total_k][Hkv][D]
    const __nv_bfloat16* v;
    const int* cu_q;           // [B + 1]
    const int* cu_k;           // [B + 1]
    const int* range;          // [total_q][2] sequence-local [start, end)
    int B, Hq, Hkv, group;
    long long total_q;
    float scale;
    __nv_bfloat16* o;          // [total_q][Hq][D]
    float* lse;                // [Hq][total_q] or null
};

constexpr int kPatchWarps = 8;
constexpr int kPatchShortMax = 64;   // longest interval the caller may promise for this kernel

// 8 bf16 (one 16-byte piece) -> 8 floats
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
}

template <int D>
__global__ void __launch_bounds__(32 * kPatchWarps) patch_kernel(const PatchArgs a) {
    constexpr int PL = D / 32;                  // output columns per lane
    constexpr int NP = D / 8;                   // 16-byte pieces per row
    const int lane = threadIdx.x & 31;
    const long long n_items = a.total_q * a.Hq;
    const float sl2 = a.scale * kLog2e;
    for (long long item = (long long)blockIdx.x * kPatchWarps + (threadIdx.x >> 5); item < n_items;
         item += (long long)gridDim.x * kPatchWarps) {
        const long long i = item / a.Hq;        // packed query row
        const int h = (int)(item % a.Hq);
        const int g = h / a.group;
        // sequence of row i: the largest b with cu_q[b] <= i
        int lo = 0, hi = a.B;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(&a.cu_q[mid]) <= i) lo = mid; else hi = mid;
        }
        const int b = lo;
        const int kb = __ldg(&a.cu_k[b]);
        const int Lk = max(__ldg(&a.cu_k[b + 1]) - kb, 0);
        const int start = max(__ldg(&a.range[2 * i]), 0);
        const int end = min(__ldg(&a.range[2 * i + 1]), Lk);
        const __nv_bfloat16* qrow = a.q + (i * a.Hq + h) * D;
        float m = -INFINITY, l = 0.0f;
        float acc[PL];
#pragma unroll
        for (int e = 0; e < PL; ++e) acc[e] = 0.0f;
        for (int c0 = start; c0 < end; c0 += 32) {
            const int j = c0 + lane;
            float s = -INFINITY;
            if (j < end) {
                const uint4* kp = reinterpret_cast<const uint4*>(a.k + ((long long)(kb + j) * a.Hkv + g) * D);
                const uint4* qp = reinterpret_cast<const uint4*>(qrow);
                float dot = 0.0f;
#pragma unroll
                for (int pc = 0; pc < NP; ++pc) {
                    float kf[8], qf[8];
                    bf16x8_to_f32(__ldg(kp + pc), kf);
                    bf16x8_to_f32(__ldg(qp + pc), qf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) dot = fmaf(qf[e], kf[e], dot);
                }
                s = dot * sl2;
            }
            float cm = s;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
            const float m_new = fmaxf(m, cm);
            const float alpha = (m == -INFINITY) ? 0.0f : ex2(m - m_new);
            const float p = (j < end) ? ex2(s - m_new) : 0.0f;
            float ps = p;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
            l = l * alpha + ps;
#pragma unroll
            for (int e = 0; e < PL; ++e) acc[e] *= alpha;
            m = m_new;
            // O += p_j v_j: the lanes split D (PL consecutive columns each)
            const int nv = min(32, end - c0);
            for (int jj = 0; jj < nv; ++jj) {
                const float pj = __shfl_sync(0xffffffffu, p, jj);
                const __nv_bfloat16* vrow = a.v + ((long long)(kb + c0 + jj) * a.Hkv + g) * D + lane * PL;
#pragma unroll
                for (int e2 = 0; e2 < PL / 2; ++e2) {
                    const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(vrow) + e2);
                    acc[2 * e2] = fmaf(pj, __uint_as_float(u << 16), acc[2 * e2]);
                    acc[2 * e2 + 1] = fmaf(pj, __uint_as_float(u & 0xFFFF0000u), acc[2 * e2 + 1]);
                }
            }
        }
        const float inv = l > 0.0f ? 1.0f / l : 0.0f;
        __nv_bfloat16* orow = a.o + (i * a.Hq + h) * D + lane * PL;
        if constexpr (PL == 4) {
            uint2 u;
            u.x = pack_bf16(acc[0] * inv, acc[1] * inv);
            u.y = pack_bf16(acc[2] * inv, acc[3] * inv);
            *reinterpret_cast<uint2*>(orow) = u;
        } else {
            *reinterpret_cast<uint32_t*>(orow) = pack_bf16(acc[0] * inv, acc[1] * inv);
        }
        if (lane == 0 && a.lse) a.lse[(long long)h * a.total_q + i] = l > 0.0f ? (m + log2f(l)) * kLn2 : -INFINITY;
    }
}

// One warp per query, all Hq heads at once: LPH = 32 / Hq lanes per head, each
// holding DL = D / LPH consecutive columns of q, of the running O and of every key
// and value row it reads.  A key's K (or V) row of all heads is one contiguous
// Hkv * D * 2-byte piece, read whole by the warp.  For shapes with DL <= 32
// (Hq * D <= 1024); two blocks per SM.
template <int D, int HQ>
__global__ void __launch_bounds__(32 * kPatchWarps, 2) patch_query_kernel(const PatchArgs a) {
    constexpr int LPH = 32 / HQ;                // lanes per head
    constexpr int DL = D / LPH;                 // columns per lane
    constexpr int NU = DL / 8;                  // 16-byte pieces per lane and row
    static_assert(LPH >= 1 && DL % 8 == 0 && DL <= 32, "shape of the query-per-warp patch kernel");
    const int lane = threadIdx.x & 31;
    const int h = lane / LPH, part = lane % LPH;
    const int g = h / a.group;
    const float sl2 = a.scale * kLog2e;
    for (long long i = (long long)blockIdx.x * kPatchWarps + (threadIdx.x >> 5); i < a.total_q;
         i += (long long)gridDim.x * kPatchWarps) {
        int lo = 0, hi = a.B;                   // sequence of row i
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(&a.cu_q[mid]) <= i) lo = mid; else hi = mid;
        }
        const int kb = __ldg(&a.cu_k[lo]);
        const int Lk = max(__ldg(&a.cu_k[lo + 1]) - kb, 0);
        const int start = max(__ldg(&a.range[2 * i]), 0);
        const int end = min(__ldg(&a.range[2 * i + 1]), Lk);
        uint4 qr[NU];
        const uint4* qp = reinterpret_cast<const uint4*>(a.q + (i * a.Hq + h) * D + part * DL);
#pragma unroll
        for (int u = 0; u < NU; ++u) qr[u] = __ldg(qp + u);
        float m = -INFINITY, l = 0.0f;
        float acc[DL];
#pragma unroll
        for (int e = 0; e < DL; ++e) acc[e] = 0.0f;
        const long long row_stride = (long long)a.Hkv * D;         // elements between key rows
        const long long col0 = (long long)g * D + part * DL;       // this lane's columns
        for (int j = start; j < end; ++j) {
            uint4 kr[NU], vr[NU];
            const uint4* kp = reinterpret_cast<const uint4*>(a.k + (kb + j) * row_stride + col0);
            const uint4* vp = reinterpret_cast<const uint4*>(a.v + (kb + j) * row_stride + col0);
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                kr[u] = __ldg(kp + u);
                vr[u] = __ldg(vp + u);
            }
            float dot = 0.0f;
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                float kf[8], qf[8];
                bf16x8_to_f32(kr[u], kf);
                bf16x8_to_f32(qr[u], qf);
#pragma unroll
                for (int e = 0; e < 8; ++e) dot = fmaf(qf[e], kf[e], dot);
            }
#pragma unroll
            for (int off = 1; off < LPH; off <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            const float sc = dot * sl2;
            const float m_new = fmaxf(m, sc);
            const float alpha = (m == -INFINITY) ? 0.0f : ex2(m - m_new);
            const float p0 = ex2(sc - m_new);
            l = l * alpha + p0;
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                float v0[8];
                bf16x8_to_f32(vr[u], v0);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[8 * u + e] = fmaf(p0, v0[e], acc[8 * u + e] * alpha);
            }
            m = m_new;
        }
        const float inv = l > 0.0f ? 1.0f / l : 0.0f;
        uint4* op = reinterpret_cast<uint4*>(a.o + (i * a.Hq + h) * D + part * DL);
#pragma unroll
        for (int u = 0; u < NU; ++u) {
            uint4 w;
            w.x = pack_bf16(acc[8 * u + 0] * inv, acc[8 * u + 1] * inv);
            w.y = pack_bf16(acc[8 * u + 2] * inv, acc[8 * u + 3] * inv);
            w.z = pack_bf16(acc[8 * u + 4] * inv, acc[8 * u + 5] * inv);
            w.w = pack_bf16(acc[8 * u + 6] * inv, acc[8 * u + 7] * inv);
            op[u] = w;
        }
        if (part == 0 && a.lse) a.lse[(long long)h * a.total_q + i] = l > 0.0f ? (m + log2f(l)) * kLn2 : -INFINITY;
    }
}

}  // namespace attn
