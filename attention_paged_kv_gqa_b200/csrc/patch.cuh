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
    int total_k;               // rows of k / v
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

// ---------------------------------------------------------------------------
// patch_stream_kernel<D> (Hq == Hkv, heads in groups of HG = 256 / D: a 512-byte
// slice of every q, k, v and o row).  One CTA per (head group, contiguous range
// of the query list).  Its producer warp groups consecutive queries of one
// sequence into chunks (at most kPsQ queries whose key intervals together span
// at most kPsRows rows) and copies each chunk's q slices and the K and V slices
// of that span into a shared-memory stage with TMA (a head group's slices of
// contiguous rows of the packed layout, at most seven TMA boxes a chunk),
// kPsStages stages deep, so the whole CTA
// keeps tens of KB of reads in flight instead of one dependent row at a time.
// The consumer warps take a chunk's queries one per warp (LPH = 32 / HG lanes
// per head, 8 columns a lane, up to four keys a step) and read only shared memory.
// They form kPsTeams teams that take alternate chunks; chunk c uses stage
// c % kPsStages, so each stage serves one team, which waits for every phase of
// its barriers in turn (a parity wait cannot tell phases two apart).  Two CTAs
// share an SM, each with one team of 8 warps and 3 stages of 8 queries and 32
// rows (110 KB): on the patch workload that measured 4352 GB/s against 3930 for
// one CTA of 3 stages of 16 queries and 64 rows, in one A/B call; three CTAs of 2
// stages gave 4129, and two teams in one CTA were slower still.  A CTA's time
// follows its queries more than its bytes (a split of the query list for equal
// bytes measured 3355 against 4026), so the list is split by count.  A query
// whose own interval is longer than kPsRows is marked, and its consumer reads it
// from global memory, so any interval length is correct.
constexpr int kPsTeamWarps = 8;             // consumer warps of a team
constexpr int kPsTeams = 1;                 // teams take alternate chunks (two measured slower)
constexpr int kPsWarps = kPsTeams * kPsTeamWarps;
constexpr int kPsThreads = 32 * (kPsWarps + 1);
constexpr int kPsStages = 3;                // a multiple of kPsTeams: a stage serves one team only
constexpr int kPsQ = 8;                     // queries per chunk
constexpr int kPsRows = 32;                 // key rows per chunk
constexpr int kPsCtas = 2;                  // CTAs per SM (the grid is kPsCtas x the SM count)
constexpr int kPsSlice = 512;               // bytes of one head group's slice of a row
constexpr int kPsStageBytes = (kPsQ + 2 * kPsRows) * kPsSlice;
constexpr int kPsCuMax = 255;               // sequences whose cu_seqlens go to shared memory

enum : int { kErrPsFull = 701, kErrPsEmpty = 702, kErrPsDrain = 703 };

struct PatchStreamMeta {
    int i0;                   // first query of the chunk; -1: no more chunks
    int nq;
    int row0;                 // packed key row of the stage's first K / V row
    int pad;
    int rs[kPsQ], re[kPsQ];   // each query's rows in the stage; rs < 0: long, read from global
    int gs[kPsQ], ge[kPsQ];   // long queries: packed rows [gs, ge)
};

// Tensor maps of the streamed slices: q as [total_q rows][Hq * D], k and v as
// [total_k rows][Hkv * D], boxes of 256 elements (one head group's 512-byte
// slice) by kPsQ rows (q) or 8, 16, 32, 64 rows (k, v: a chunk's span, rounded up
// to 8 rows, is the sum of at most four of them).  No swizzle: the consumers read
// whole 512-byte rows, 16 bytes a lane.
struct PatchMaps {
    CUtensorMap q;
    CUtensorMap k[4];         // box heights 8, 16, 32, 64
    CUtensorMap v[4];
};

__host__ __device__ constexpr int patch_stream_smem_bytes() {
    return 128 + kPsStages * kPsStageBytes + kPsStages * (int)sizeof(PatchStreamMeta) + 2 * kPsStages * 8 +
           2 * (kPsCuMax + 1) * 4;
}
// kPsCtas CTAs fit the SM's 228 KB of shared memory, 1 KB of it reserved per CTA
static_assert(kPsCtas * (patch_stream_smem_bytes() + 1024) <= 228 * 1024, "CTAs per SM");

template <int D>
__global__ void __launch_bounds__(kPsThreads, kPsCtas)
    patch_stream_kernel(const __grid_constant__ PatchMaps maps, const PatchArgs a, int n_hg) {
    constexpr int HG = 256 / D;             // heads per 512-byte slice
    constexpr int LPH = 32 / HG;            // lanes per head
    static_assert(HG * D * 2 == kPsSlice && LPH * 8 == D, "slice layout");
    static_assert(kPsStages % kPsTeams == 0, "a stage serves one team");
    static_assert(kPsQ >= 8 && kPsRows % 8 == 0 && kPsRows <= 120, "groups of 8 queries; boxes of 8 to 64 rows");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    PatchStreamMeta* meta = reinterpret_cast<PatchStreamMeta*>(smem + kPsStages * kPsStageBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(meta + kPsStages);
    uint64_t* empty = full + kPsStages;
    auto sQ = [&](int st) { return smem + st * kPsStageBytes; };
    auto sK = [&](int st) { return smem + st * kPsStageBytes + kPsQ * kPsSlice; };
    auto sV = [&](int st) { return smem + st * kPsStageBytes + (kPsQ + kPsRows) * kPsSlice; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hg = (int)(blockIdx.x % n_hg);
    const long long n_rg = gridDim.x / n_hg;
    const long long per = (a.total_q + n_rg - 1) / n_rg;
    const long long q_begin = (long long)(blockIdx.x / n_hg) * per;
    const long long q_end = min(a.total_q, q_begin + per);
    const long long row_elems = (long long)a.Hq * D;          // Hq == Hkv
    const long long col_off = (long long)hg * HG * D;
    const int total_k = a.total_k;

    // cu_seqlens_q / _k in shared memory for batches of up to kPsCuMax sequences (the
    // producer's per-query sequence lookups); larger batches read them from global memory
    int* s_cuq = reinterpret_cast<int*>(empty + kPsStages);
    int* s_cuk = s_cuq + kPsCuMax + 1;
    const bool cu_in_smem = a.B <= kPsCuMax;
    if (cu_in_smem)
        for (int j = threadIdx.x; j <= a.B; j += blockDim.x) {
            s_cuq[j] = a.cu_q[j];
            s_cuk[j] = a.cu_k[j];
        }
    auto cu_q_of = [&](int j) { return cu_in_smem ? s_cuq[j] : __ldg(&a.cu_q[j]); };
    auto cu_k_of = [&](int j) { return cu_in_smem ? s_cuk[j] : __ldg(&a.cu_k[j]); };
    auto seq_of_query = [&](long long qi) {     // the largest b with cu_q[b] <= qi
        int lo = 0, hi = a.B;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (cu_q_of(mid) <= qi) lo = mid; else hi = mid;
        }
        return lo;
    };
    if (threadIdx.x == 0) {
        for (int i = 0; i < kPsStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kPsTeamWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kPsWarps) {
        // ---------------------------------------------------------------- producer
        int st = 0, issued = 0;
        uint32_t ph = 0;
        bool ok = true;
        // The next batch's intervals are loaded while this batch's chunks are issued.
        int2 rng_next = make_int2(0, 0);
        if (q_begin + lane < q_end)
            rng_next = make_int2(__ldg(&a.range[2 * (q_begin + lane)]), __ldg(&a.range[2 * (q_begin + lane) + 1]));
        for (long long i = q_begin; ok && i < q_end; i += 32) {
            const long long qi = i + lane;
            const int nb = (int)min(32LL, q_end - i);
            const int2 rng = rng_next;
            if (i + 32 + lane < q_end)
                rng_next = make_int2(__ldg(&a.range[2 * (i + 32 + lane)]), __ldg(&a.range[2 * (i + 32 + lane) + 1]));
            int bq = -1, kb = 0, s = 0, e = 0, lng = 0;
            if (qi < q_end) {
                bq = seq_of_query(qi);
                kb = cu_k_of(bq);
                const int Lk = max(min(cu_k_of(bq + 1), total_k) - kb, 0);
                s = max(rng.x, 0);
                e = min(rng.y, Lk);
                if (s >= e) s = e = 0;
                lng = e - s > kPsRows;
            }
            // Each group of 8 queries as one chunk when it can be (one sequence, no long
            // interval, a span of at most kPsRows rows): its bounds by segmented reductions
            // over the group's lanes.  Otherwise the chunks are grown one query at a time.
            int gbmin, gbmax, glo, ghi, glong;
            {
                const bool valid = lane < nb;
                const bool has = valid && !lng && s < e;
                gbmin = valid ? bq : 0x7fffffff;
                gbmax = valid ? bq : -0x7fffffff;
                glo = has ? kb + s : 0x7fffffff;
                ghi = has ? kb + e : -0x7fffffff;
                glong = valid && lng;
#pragma unroll
                for (int off = 1; off < 8; off <<= 1) {
                    gbmin = min(gbmin, __shfl_xor_sync(0xffffffffu, gbmin, off));
                    gbmax = max(gbmax, __shfl_xor_sync(0xffffffffu, gbmax, off));
                    glo = min(glo, __shfl_xor_sync(0xffffffffu, glo, off));
                    ghi = max(ghi, __shfl_xor_sync(0xffffffffu, ghi, off));
                    glong |= __shfl_xor_sync(0xffffffffu, glong, off);
                }
            }
            int c0 = 0;
            while (c0 < nb) {
                // chunk: queries c0 .. c1-1 of this batch (one sequence); every lane agrees
                int lo = 0x7fffffff, hi = -0x7fffffff, c1 = c0;
                const int fbmin = __shfl_sync(0xffffffffu, gbmin, c0);
                const int fbmax = __shfl_sync(0xffffffffu, gbmax, c0);
                const int flo = __shfl_sync(0xffffffffu, glo, c0);
                const int fhi = __shfl_sync(0xffffffffu, ghi, c0);
                const int flong = __shfl_sync(0xffffffffu, glong, c0);
                if ((c0 & 7) == 0 && fbmin == fbmax && !flong && (fhi < flo || fhi - flo <= kPsRows)) {
                    c1 = min(c0 + 8, nb);           // the whole group
                    if (fhi >= flo) {
                        lo = flo;
                        hi = fhi;
                    }
                } else {
                    // grown one query at a time
                    const int b0 = __shfl_sync(0xffffffffu, bq, c0);
                    while (c1 < nb && c1 - c0 < kPsQ) {
                        const int bj = __shfl_sync(0xffffffffu, bq, c1);
                        const int kj = __shfl_sync(0xffffffffu, kb, c1);
                        const int sj = __shfl_sync(0xffffffffu, s, c1);
                        const int ej = __shfl_sync(0xffffffffu, e, c1);
                        const int lj = __shfl_sync(0xffffffffu, lng, c1);
                        if (bj != b0) break;
                        if (!lj && sj < ej) {
                            const int nlo = min(lo, kj + sj), nhi = max(hi, kj + ej);
                            if (nhi - nlo > kPsRows) break;
                            lo = nlo;
                            hi = nhi;
                        }
                        ++c1;
                    }
                }
                const int nq = c1 - c0;
                const int nrows = hi > lo ? hi - lo : 0;
                const int nrows8 = (nrows + 7) & ~7;        // rows fetched (beyond hi: the next rows)
                if (nrows == 0) lo = 0;
                ok = mbar_wait(&empty[st], ph ^ 1u, kErrPsEmpty);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                // this lane's query of the chunk (lane < nq)
                const int src = min(c0 + lane, 31);
                const int kj = __shfl_sync(0xffffffffu, kb, src);
                const int sj = __shfl_sync(0xffffffffu, s, src);
                const int ej = __shfl_sync(0xffffffffu, e, src);
                const int lj = __shfl_sync(0xffffffffu, lng, src);
                PatchStreamMeta& m = meta[st];
                if (lane < nq) {
                    m.rs[lane] = lj ? -1 : (sj < ej ? kj + sj - lo : 0);
                    m.re[lane] = lj ? -1 : (sj < ej ? kj + ej - lo : 0);
                    m.gs[lane] = kj + sj;
                    m.ge[lane] = kj + ej;
                }
                if (lane == 0) {
                    m.i0 = (int)(i + c0);
                    m.nq = nq;
                    m.row0 = lo;
                }
                __syncwarp();
                if (lane == 0) {
                    // rows past the tensors' ends are filled with zeros by the copy
                    mbar_arrive_expect_tx(&full[st], (uint32_t)(kPsQ + 2 * nrows8) * kPsSlice);
                    tma_load_4d(&maps.q, &full[st], sQ(st), hg * 256, (int)(i + c0), 0, 0);
                    int r0 = 0;
#pragma unroll
                    for (int pc = 3; pc >= 0; --pc) {
                        const int h = 8 << pc;
                        if (nrows8 & h) {
                            tma_load_4d(&maps.k[pc], &full[st], sK(st) + r0 * kPsSlice, hg * 256, lo + r0, 0, 0);
                            tma_load_4d(&maps.v[pc], &full[st], sV(st) + r0 * kPsSlice, hg * 256, lo + r0, 0, 0);
                            r0 += h;
                        }
                    }
                }
                ++issued;
                if (++st == kPsStages) {
                    st = 0;
                    ph ^= 1u;
                }
                c0 = c1;
            }
        }
        // no more chunks: one stage per team whose meta says so, with no bytes
        int pushed = 0;
        for (int tm = 0; ok && tm < kPsTeams; ++tm) {
            ok = mbar_wait(&empty[st], ph ^ 1u, kErrPsEmpty);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (lane == 0) {
                meta[st].i0 = -1;
                meta[st].nq = 0;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[st]);
            ++pushed;
            if (++st == kPsStages) {
                st = 0;
                ph ^= 1u;
            }
        }
        // Let every copy this warp started land before the CTA can exit: wait for the
        // last chunk of each stage.  The stages of the no-more-chunks markers are
        // skipped: their barriers have moved on past those chunks, which had landed
        // before the markers' waits for the stages could end.
        if (lane == 0) {
            for (int k2 = 0; k2 < kPsStages && k2 < issued; ++k2) {
                bool marked = false;
                for (int d = 0; d < pushed; ++d) marked |= (issued + d) % kPsStages == k2;
                if (marked) continue;
                const int last = k2 + ((issued - 1 - k2) / kPsStages) * kPsStages;   // chunk index
                mbar_wait_drain(&full[k2], (uint32_t)((last / kPsStages) & 1), kErrPsDrain);
            }
        }
    } else {
        // ---------------------------------------------------------------- consumers
        // team `team` takes chunks team, team + kPsTeams, ...
        const int team = warp / kPsTeamWarps, tw = warp % kPsTeamWarps;
        const int hl = lane / LPH;                 // head within the group
        const float sl2 = a.scale * kLog2e;
        for (int ck = team;; ck += kPsTeams) {
            const int st = ck % kPsStages;
            const uint32_t ph = (uint32_t)((ck / kPsStages) & 1);
            bool ok = mbar_wait(&full[st], ph, kErrPsFull);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const PatchStreamMeta& m = meta[st];
            const int i0 = m.i0;
            if (i0 < 0) break;
            const int nq = m.nq;
            for (int t = tw; t < nq; t += kPsTeamWarps) {
                const long long qi = (long long)i0 + t;
                float qf[8];
                bf16x8_to_f32(*reinterpret_cast<const uint4*>(sQ(st) + t * kPsSlice + lane * 16), qf);
                float mrow = -INFINITY, l = 0.0f, acc[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
                auto step = [&](const uint4& kr, const uint4& vr) {
                    float kf[8];
                    bf16x8_to_f32(kr, kf);
                    float dot = 0.0f;
#pragma unroll
                    for (int c = 0; c < 8; ++c) dot = fmaf(qf[c], kf[c], dot);
#pragma unroll
                    for (int off = 1; off < LPH; off <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
                    const float sc = dot * sl2;
                    const float mn = fmaxf(mrow, sc);
                    const float alpha = (mrow == -INFINITY) ? 0.0f : ex2(mrow - mn);
                    const float p0 = ex2(sc - mn);
                    l = l * alpha + p0;
                    float vf[8];
                    bf16x8_to_f32(vr, vf);
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[c] = fmaf(p0, vf[c], acc[c] * alpha);
                    mrow = mn;
                };
                // two keys a step: their dot products and reductions interleave
                auto step2 = [&](const uint4& k0, const uint4& v0, const uint4& k1, const uint4& v1) {
                    float kf0[8], kf1[8];
                    bf16x8_to_f32(k0, kf0);
                    bf16x8_to_f32(k1, kf1);
                    float d0 = 0.0f, d1 = 0.0f;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        d0 = fmaf(qf[c], kf0[c], d0);
                        d1 = fmaf(qf[c], kf1[c], d1);
                    }
#pragma unroll
                    for (int off = 1; off < LPH; off <<= 1) {
                        d0 += __shfl_xor_sync(0xffffffffu, d0, off);
                        d1 += __shfl_xor_sync(0xffffffffu, d1, off);
                    }
                    const float s0 = d0 * sl2, s1 = d1 * sl2;
                    const float mn = fmaxf(mrow, fmaxf(s0, s1));
                    const float alpha = (mrow == -INFINITY) ? 0.0f : ex2(mrow - mn);
                    const float p0 = ex2(s0 - mn), p1 = ex2(s1 - mn);
                    l = l * alpha + (p0 + p1);
                    float vf0[8], vf1[8];
                    bf16x8_to_f32(v0, vf0);
                    bf16x8_to_f32(v1, vf1);
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[c] = fmaf(p1, vf1[c], fmaf(p0, vf0[c], acc[c] * alpha));
                    mrow = mn;
                };
                // four keys a step where four remain
                auto step4 = [&](int r) {
                    float d[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        float kf[8];
                        bf16x8_to_f32(*reinterpret_cast<const uint4*>(sK(st) + (r + u) * kPsSlice + lane * 16), kf);
                        d[u] = 0.0f;
#pragma unroll
                        for (int c = 0; c < 8; ++c) d[u] = fmaf(qf[c], kf[c], d[u]);
                    }
#pragma unroll
                    for (int off = 1; off < LPH; off <<= 1)
#pragma unroll
                        for (int u = 0; u < 4; ++u) d[u] += __shfl_xor_sync(0xffffffffu, d[u], off);
                    float sc[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) sc[u] = d[u] * sl2;
                    const float mn = fmaxf(mrow, fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3])));
                    const float alpha = (mrow == -INFINITY) ? 0.0f : ex2(mrow - mn);
                    float pr[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) pr[u] = ex2(sc[u] - mn);
                    l = l * alpha + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[c] *= alpha;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        float vf[8];
                        bf16x8_to_f32(*reinterpret_cast<const uint4*>(sV(st) + (r + u) * kPsSlice + lane * 16), vf);
#pragma unroll
                        for (int c = 0; c < 8; ++c) acc[c] = fmaf(pr[u], vf[c], acc[c]);
                    }
                    mrow = mn;
                };
                const int rs = m.rs[t], re = m.re[t];
                if (rs >= 0) {
                    int r = rs;
                    for (; r + 3 < re; r += 4) step4(r);
                    for (; r + 1 < re; r += 2)
                        step2(*reinterpret_cast<const uint4*>(sK(st) + r * kPsSlice + lane * 16),
                              *reinterpret_cast<const uint4*>(sV(st) + r * kPsSlice + lane * 16),
                              *reinterpret_cast<const uint4*>(sK(st) + (r + 1) * kPsSlice + lane * 16),
                              *reinterpret_cast<const uint4*>(sV(st) + (r + 1) * kPsSlice + lane * 16));
                    if (r < re)
                        step(*reinterpret_cast<const uint4*>(sK(st) + r * kPsSlice + lane * 16),
                             *reinterpret_cast<const uint4*>(sV(st) + r * kPsSlice + lane * 16));
                } else {
                    const int gs = m.gs[t], ge = m.ge[t];
                    for (int r = gs; r < ge; ++r) {
                        const long long off = (long long)r * row_elems + col_off + lane * 8;
                        step(__ldg(reinterpret_cast<const uint4*>(a.k + off)),
                             __ldg(reinterpret_cast<const uint4*>(a.v + off)));
                    }
                }
                const float inv = l > 0.0f ? 1.0f / l : 0.0f;
                uint4 w;
                w.x = pack_bf16(acc[0] * inv, acc[1] * inv);
                w.y = pack_bf16(acc[2] * inv, acc[3] * inv);
                w.z = pack_bf16(acc[4] * inv, acc[5] * inv);
                w.w = pack_bf16(acc[6] * inv, acc[7] * inv);
                *reinterpret_cast<uint4*>(a.o + qi * row_elems + col_off + lane * 8) = w;
                if (a.lse && (lane % LPH) == 0)
                    a.lse[(long long)(hg * HG + hl) * a.total_q + qi] = l > 0.0f ? (mrow + log2f(l)) * kLn2 : -INFINITY;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
    }
}

}  // namespace attn
