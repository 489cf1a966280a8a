// backward.cuh -- attention backward on sm_100a: dQ, dK, dV of the forward in
// prefill.cuh, for packed varlen batches (no paging), grouped-query heads and
// the none / causal (optionally windowed) masks.  The training path of the
// pages (BLT through the FlexAttention autograd; the FlashAttnVarlenFunc
// backward of "Rope dim").
//
// With P = exp(scale QK^T - LSE) (LSE from the forward) and
// Delta_i = dO_i . O_i:
//   dV = P^T dO,   dP = dO V^T,   dS = P (dP - Delta) scale,
//   dQ = dS K,     dK = dS^T Q    (dK, dV summed over a KV head's query heads).
//
// Three kernels, no atomics:
//   bwd_delta_kernel   Delta = rowsum(dO * O) in fp32.
//   bwd_dkdv_kernel    one CTA per (sequence, KV head, 128-key tile): K, V stay
//                      in shared memory; (query head, 128-query tile) items
//                      stream through a stage ring.  Per item the tensor core
//                      computes S^T = K Q^T and dP^T = V dO^T into TMEM (lanes
//                      = keys); the compute warpgroup turns them into P^T and
//                      dS^T (bf16, written back over S^T / dP^T); then
//                      dV += P^T dO and dK += dS^T Q accumulate in TMEM.
//   bwd_dq_kernel      one CTA per (sequence, head, 128-query tile): Q and dO
//                      stay; K/V tiles stream as in the forward.  S = Q K^T and
//                      dP = dO V^T into TMEM (lanes = queries), dS (bf16) over
//                      S, dQ += dS K.
// Operand layouts are those of the forward: every tile is a TMA 128-byte
// swizzled [rows][D] tile, read K-major for the score GEMMs and MN-major (as
// V is in the forward) for the accumulating ones.
#pragma once

#include "prefill.cuh"

namespace attn {

// Warps 0 .. 4 kBwdWG - 1: compute warpgroups (thread = TMEM lane; warpgroup h
// takes the 32-column blocks c4 = h, h + kBwdWG, .. of a 128-column score
// tile); then the TMA warp and the MMA warp.  A block's bf16 results (16
// columns) are written over the first half of the block itself, which its
// warpgroup has already read, so no warpgroup writes where another reads; the
// accumulating GEMMs read their A operand there.
constexpr int kBwdWG = 4;
constexpr int kBwdComputeThreads = 128 * kBwdWG;
constexpr int kBwdProducerWarp = 4 * kBwdWG;
constexpr int kBwdMmaWarp = 4 * kBwdWG + 1;
constexpr int kBwdThreads = kBwdComputeThreads + 64;

// TMEM column of the bf16 results of 32-column block c4 (0..3) of a score tile.
__device__ __forceinline__ uint32_t bwd_out_col(int c4) { return 32 * c4; }
// ... and of k-step kk (16 rows, 8 columns) of the accumulating GEMM's A operand.
__device__ __forceinline__ uint32_t bwd_a_col(int kk) { return 32 * (kk >> 1) + 8 * (kk & 1); }

enum : int {
    kErrBwdLoad = 601, kErrBwdMma = 602, kErrBwdCompute = 603, kErrBwdDrain = 604,
};

#ifndef ATTN_BWD_SEQ_MAJOR
#define ATTN_BWD_SEQ_MAJOR 1
#endif

// Sequence-major unit order for a varlen batch of at most 32 sequences: the
// sequences longest first (ties by index), each owning `my_units` consecutive
// units (lane s of every warp describes sequence s: its length and unit count;
// lanes >= B pass length -1 and 0 units).  The CTAs that run together then
// work on one sequence, whose operand tiles they share in L2.  Gives the
// sequence of unit `lin` and the unit's index inside it; false past the last
// unit.  Every warp computes the same answer.
__device__ __forceinline__ bool seq_major_unit(int lin, int B, int my_len, int my_units,
                                               int* seq_out, int* local_out) {
    const int lane = threadIdx.x & 31;
    int start = 0;
#pragma unroll 1
    for (int o = 0; o < B; ++o) {
        const int lo = __shfl_sync(0xffffffffu, my_len, o);
        const int no = __shfl_sync(0xffffffffu, my_units, o);
        start += (lo > my_len || (lo == my_len && o < lane)) ? no : 0;
    }
    const bool mine = lane < B && lin >= start && lin < start + my_units;
    const unsigned hit = __ballot_sync(0xffffffffu, mine);
    if (hit == 0u) return false;
    const int src = __ffs(hit) - 1;
    *seq_out = src;
    *local_out = lin - __shfl_sync(0xffffffffu, start, src);
    return true;
}

struct BwdArgs {
    int B, Hq, Hkv, group;
    int mask, window;          // window: causal only, < 0 none
    const int* cu_q;           // [B + 1]
    const int* cu_k;           // [B + 1]
    const float* lse;          // [Hq][total_q] natural log (the forward's)
    const float* delta;        // [Hq][total_q]
    float scale;
    __nv_bfloat16* dq;         // [total_q][Hq][D]
    __nv_bfloat16* dk;         // [total_k][Hkv][D]
    __nv_bfloat16* dv;
    int total_q;
    int nqt, nkt;              // query / key tiles of the longest sequence
};

template <int D>
struct BwdCfg {
    static constexpr int ROWB = D * 2;                 // bf16 row bytes
    static constexpr int NCHUNK = ROWB / 128;          // 128-byte swizzle columns per row
    static constexpr int TILE = 128 * ROWB;            // one [128][D] tile
    static constexpr int KSTEP = 16;
    static constexpr uint32_t IDESC_SS = instr_desc(1, 1, 0, 0, 128, 128);   // score GEMMs
    static constexpr uint32_t IDESC_TS = instr_desc(1, 1, 0, 1, 128, D);     // accumulating GEMMs
    // dK/dV kernel: K, V + NS stages of (Q, dO, LSE*log2e, Delta)
    static constexpr int STAGE_A = 2 * TILE + 2 * 128 * 4;
    static constexpr int NS_A = (2 * TILE + 3 * STAGE_A + 2048 <= 227 * 1024) ? 3 : 2;
    static constexpr int SMEM_A = 1024 + 2 * TILE + NS_A * STAGE_A + 1024;
    // dQ kernel: Q, dO + NS stages of (K, V)
    static constexpr int NS_B = (2 * TILE + 4 * 2 * TILE + 2048 <= 227 * 1024) ? 4
                                : (2 * TILE + 3 * 2 * TILE + 2048 <= 227 * 1024) ? 3 : 2;
    static constexpr int SMEM_B = 1024 + 2 * TILE + NS_B * 2 * TILE + 1024;
    static_assert(STAGE_A % 1024 == 0, "stages keep 1024-byte alignment");
};

// ---------------------------------------------------------------- Delta
// Delta[h][i] = sum_d dO[i][h][d] * O[i][h][d], one warp per (row, head).
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                        const __nv_bfloat16* __restrict__ dout,
                                                        float* __restrict__ delta, int total_q,
                                                        int Hq) {
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    const long long n = (long long)total_q * Hq;
    for (long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; w < n; w += warps) {
        const int i = (int)(w / Hq), h = (int)(w % Hq);
        const __nv_bfloat162* po = reinterpret_cast<const __nv_bfloat162*>(o + (w * D));
        const __nv_bfloat162* pd = reinterpret_cast<const __nv_bfloat162*>(dout + (w * D));
        float acc = 0.0f;
#pragma unroll
        for (int e = lane; e < D / 2; e += 32) {
            const float2 a = __bfloat1622float2(po[e]);
            const float2 b = __bfloat1622float2(pd[e]);
            acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) delta[(long long)h * total_q + i] = acc;
    }
}

// Row i's allowed keys under the mask: [lo, hi) (sequence-local).
__device__ __forceinline__ void bwd_row_keys(const BwdArgs& a, int i, int Lq, int Lk, int* lo,
                                             int* hi) {
    *lo = 0;
    *hi = Lk;
    if (a.mask == kMaskCausal) {
        *hi = min(Lk, i + (Lk - Lq) + 1);
        if (a.window >= 0) *lo = max(i + (Lk - Lq) - a.window, 0);
    }
}

// ---------------------------------------------------------------- dQ
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const BwdArgs a) {
    using C = BwdCfg<D>;
    constexpr int NS = C::NS_B;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem;
    uint8_t* sdO = sQ + C::TILE;
    uint8_t* sK = sdO + C::TILE;                  // [NS] key tiles
    uint8_t* sV = sK + NS * C::TILE;              // [NS] value tiles
    uint64_t* bars = reinterpret_cast<uint64_t*>(sV + NS * C::TILE);
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;                 // [NS]
    uint64_t* kv_empty = kv_full + NS;            // [NS]
    uint64_t* s_full = kv_empty + NS;
    uint64_t* p_full = s_full + 1;
    uint64_t* mma_done = p_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int qt, b, h;
    if (ATTN_BWD_SEQ_MAJOR && a.B <= 32) {
        // sequences longest first; in each, the query tile descending (causal tiles
        // with more key tiles first), all heads of a tile side by side
        const int len = lane < a.B ? a.cu_q[lane + 1] - a.cu_q[lane] : -1;
        const int nqb = lane < a.B ? (max(len, 0) + 127) / 128 : 0;
        int local;
        if (!seq_major_unit((int)blockIdx.x, a.B, len, nqb * a.Hq, &b, &local)) return;
        qt = __shfl_sync(0xffffffffu, nqb, b) - 1 - local / a.Hq;
        h = local % a.Hq;
    } else {
        // the query tile slowest and descending (causal units with more key tiles first)
        const int bh = a.B * a.Hq;
        qt = a.nqt - 1 - (int)(blockIdx.x / bh);
        b = (int)(blockIdx.x % bh) / a.Hq;
        h = (int)(blockIdx.x % bh) % a.Hq;
    }
    const int g = h / a.group;
    const int q_off = a.cu_q[b], Lq = a.cu_q[b + 1] - q_off;
    const int k_off = a.cu_k[b], Lk = max(a.cu_k[b + 1] - k_off, 0);
    const int q0 = qt * 128;
    if (q0 >= Lq) return;                         // uniform
    const int nk = (Lk + 127) / 128;
    int lo = 0, hi = nk;                          // key tiles some row of the tile can see
    if (a.mask == kMaskCausal) {
        const int maxkey = min(q0 + 128, Lq) - 1 + (Lk - Lq);
        hi = maxkey >= 0 ? min(nk, maxkey / 128 + 1) : 0;
        if (a.window >= 0) lo = max(q0 + (Lk - Lq) - a.window, 0) / 128;
        if (lo >= hi) lo = hi = 0;
    }
    const bool any_tiles = hi > lo;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < NS; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_full, kBwdComputeThreads);
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == kBwdMmaWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    // S is double-buffered (tile it in S[it & 1]); dP and the dQ accumulator are single
    const uint32_t tdP = tbase + 128, tdQ = tbase + 256;
    auto tSb = [&](int it) { return tbase + ((it & 1) ? 384u : 0u); };

    if (warp == kBwdProducerWarp) {
        // ---------------------------------------------------- TMA: Q, dO once; K/V tiles stream
        if (any_tiles && lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmdO);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            mbar_arrive_expect_tx(q_full, 2 * C::TILE);
#pragma unroll
            for (int c = 0; c < C::NCHUNK; ++c) {
                tma_load_4d(&tmQ, q_full, sQ + c * 128 * 128, c * 64, h, q_off + q0, 0);
                tma_load_4d(&tmdO, q_full, sdO + c * 128 * 128, c * 64, h, q_off + q0, 0);
            }
            const uint64_t pol = policy_evict_last();
            int issued = 0;
            for (int j = lo; j < hi; ++j) {
                const int it = j - lo, st = it % NS;
                if (!mbar_wait(&kv_empty[st], ((it / NS) & 1) ^ 1, kErrBwdLoad)) break;
                ++issued;
                mbar_arrive_expect_tx(&kv_full[st], 2 * C::TILE);
#pragma unroll
                for (int c = 0; c < C::NCHUNK; ++c) {
                    tma_load_4d_hint(&tmK, &kv_full[st], sK + st * C::TILE + c * 128 * 128, c * 64, g,
                                     k_off + j * 128, 0, pol);
                    tma_load_4d_hint(&tmV, &kv_full[st], sV + st * C::TILE + c * 128 * 128, c * 64, g,
                                     k_off + j * 128, 0, pol);
                }
            }
            // every copy started must land before the CTA can exit
            mbar_wait_drain(q_full, 0, kErrBwdDrain);
            for (int st = 0; st < NS && st < issued; ++st) {
                const int last = st + ((issued - 1 - st) / NS) * NS;
                mbar_wait_drain(&kv_full[st], (last / NS) & 1, kErrBwdDrain);
            }
        }
    } else if (warp == kBwdMmaWarp) {
        // ---------------------------------------------------- MMA issuer
        if (any_tiles && lane == 0) {
            const uint32_t sQa = smem_u32(sQ), sdOa = smem_u32(sdO), sKa = smem_u32(sK), sVa = smem_u32(sV);
            // Order per key tile it: S(it+1) into the other S buffer, then (once the compute
            // warps have turned S(it), dP(it) into dS(it)) dP(it+1), the signal for the next
            // compute, and dQ += dS(it) K(it) -- so dQ(it) runs beside the next tile's compute.
            auto issue_s = [&](int it, int st) {       // S = Q K^T (K-major, K = D)
#pragma unroll
                for (int kk = 0; kk < D / C::KSTEP; ++kk) {
                    const uint32_t cb = (kk * 32) / 128, off = (kk * 32) % 128;
                    const uint32_t ro = cb * 128 * 128 + off;
                    mma_f16_ss(tSb(it), smem_desc(sQa + ro, 16, 1024, 2),
                               smem_desc(sKa + st * C::TILE + ro, 16, 1024, 2), C::IDESC_SS, kk > 0);
                }
            };
            auto issue_dp = [&](int st) {              // dP = dO V^T
#pragma unroll
                for (int kk = 0; kk < D / C::KSTEP; ++kk) {
                    const uint32_t cb = (kk * 32) / 128, off = (kk * 32) % 128;
                    const uint32_t ro = cb * 128 * 128 + off;
                    mma_f16_ss(tdP, smem_desc(sdOa + ro, 16, 1024, 2),
                               smem_desc(sVa + st * C::TILE + ro, 16, 1024, 2), C::IDESC_SS, kk > 0);
                }
            };
            bool ok = mbar_wait(q_full, 0, kErrBwdMma);
            if (ok) ok = mbar_wait(&kv_full[0], 0, kErrBwdMma);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_dp(0);
                mma_commit(s_full);
            }
            for (int j = lo; ok && j < hi; ++j) {
                const int it = j - lo, st = it % NS, st1 = (it + 1) % NS;
                const bool next = j + 1 < hi;
                if (next) {
                    if (!(ok = mbar_wait(&kv_full[st1], ((it + 1) / NS) & 1, kErrBwdMma))) break;
                    tc_fence_after();
                    issue_s(it + 1, st1);
                }
                if (!(ok = mbar_wait(p_full, it & 1, kErrBwdMma))) break;
                tc_fence_after();
                if (next) {
                    issue_dp(st1);
                    mma_commit(s_full);
                }
                // dQ += dS K: A = dS (bf16 over S(it) in TMEM), B = the key tile read MN-major (K = keys)
#pragma unroll
                for (int kk = 0; kk < 128 / C::KSTEP; ++kk) {
                    const uint64_t db = smem_desc(sKa + st * C::TILE + kk * 2 * 1024, 128 * 128, 1024, 2);
                    mma_f16_ts(tdQ, tSb(it) + bwd_a_col(kk), db, C::IDESC_TS, (it > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&kv_empty[st]);
            }
            mma_commit(mma_done);
            mbar_wait_drain(mma_done, 0, kErrBwdMma);
        }
    } else {
        // ---------------------------------------------------- compute warpgroups: dS, then dQ out
        const int quad = warp & 3, hf = warp >> 2;   // TMEM lane quarter; warpgroup
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const int qi = q0 + r;
        const bool row_ok = qi < Lq;
        float lse2 = INFINITY, dlt = 0.0f;         // rows past the sequence: P = 0
        if (row_ok) {
            const float l = a.lse[(long long)h * a.total_q + q_off + qi];
            lse2 = (l == -INFINITY) ? INFINITY : l * kLog2e;
            dlt = a.delta[(long long)h * a.total_q + q_off + qi];
        }
        int klo, khi;
        bwd_row_keys(a, qi, Lq, Lk, &klo, &khi);
        const float sl2 = a.scale * kLog2e;
        bool ok = true;
        for (int j = lo; j < hi; ++j) {
            const int it = j - lo;
            ok = mbar_wait(s_full, it & 1, kErrBwdCompute);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const int kbase = j * 128;
            const bool partial = kbase < klo || kbase + 128 > khi;
#pragma unroll
            for (int cc = 0; cc < 4 / kBwdWG; ++cc) {
                const int c4 = hf + cc * kBwdWG;
                uint32_t us[32], ud[32];
                tmem_ld32(tSb(it) + lane_off + c4 * 32, us);
                tmem_ld32(tdP + lane_off + c4 * 32, ud);
                tmem_wait_ld();
                uint32_t pk[16];
                // two columns per packed f32x2 instruction
                const float2 sl2x2 = make_float2(sl2, sl2), nlse2 = make_float2(-lse2, -lse2);
                const float2 ndlt2 = make_float2(-dlt, -dlt), scale2 = make_float2(a.scale, a.scale);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float2 x = ffma2(make_float2(__uint_as_float(us[2 * c]), __uint_as_float(us[2 * c + 1])),
                                           sl2x2, nlse2);
                    float2 p = make_float2(ex2(x.x), ex2(x.y));
                    if (partial) {
                        const int kv = kbase + c4 * 32 + 2 * c;
                        if (kv < klo || kv >= khi) p.x = 0.0f;
                        if (kv + 1 < klo || kv + 1 >= khi) p.y = 0.0f;
                    }
                    const float2 dp = fadd2(make_float2(__uint_as_float(ud[2 * c]), __uint_as_float(ud[2 * c + 1])), ndlt2);
                    const float2 ds = fmul2(p, fmul2(dp, scale2));
                    pk[c] = pack_bf16(ds.x, ds.y);
                }
                // dS of block c4 -> columns this warpgroup has already read
                tmem_st16(tSb(it) + lane_off + bwd_out_col(c4), pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        bool have = false;
        if (ok && any_tiles) {
            const bool w = mbar_wait(mma_done, 0, kErrBwdCompute);
            have = __all_sync(0xffffffffu, w);
            tc_fence_after();
        }
        __nv_bfloat16* dst = a.dq + ((long long)(q_off + qi) * a.Hq + h) * D;
        __syncwarp();
        // warpgroup hf writes the 32-column blocks hf, hf + kBwdWG, .. of its rows' dQ
        if (have) {
#pragma unroll
            for (int c4 = hf; c4 < D / 32; c4 += kBwdWG) {
                uint32_t u[32];
                tmem_ld32(tdQ + lane_off + c4 * 32, u);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(u[8 * v4 + 0]), __uint_as_float(u[8 * v4 + 1]));
                        w.y = pack_bf16(__uint_as_float(u[8 * v4 + 2]), __uint_as_float(u[8 * v4 + 3]));
                        w.z = pack_bf16(__uint_as_float(u[8 * v4 + 4]), __uint_as_float(u[8 * v4 + 5]));
                        w.w = pack_bf16(__uint_as_float(u[8 * v4 + 6]), __uint_as_float(u[8 * v4 + 7]));
                        reinterpret_cast<uint4*>(dst + c4 * 32)[v4] = w;
                    }
                }
            }
        } else if (row_ok) {
            for (int c4 = hf; c4 < D / 32; c4 += kBwdWG)
                for (int v4 = 0; v4 < 4; ++v4)
                    reinterpret_cast<uint4*>(dst + c4 * 32)[v4] = make_uint4(0, 0, 0, 0);
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

// ---------------------------------------------------------------- dK, dV
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const BwdArgs a) {
    using C = BwdCfg<D>;
    constexpr int NS = C::NS_A;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sK = smem;
    uint8_t* sV = sK + C::TILE;
    uint8_t* stages = sV + C::TILE;               // [NS] x {Q tile, dO tile, LSE*log2e[128], Delta[128]}
    uint64_t* bars = reinterpret_cast<uint64_t*>(stages + NS * C::STAGE_A);
    uint64_t* kv_full = bars;
    uint64_t* st_full = bars + 1;                 // [NS]
    uint64_t* st_empty = st_full + NS;            // [NS]
    uint64_t* s_full = st_empty + NS;
    uint64_t* p_full = s_full + 1;
    uint64_t* mma_done = p_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    auto stQ = [&](int st) { return stages + st * C::STAGE_A; };
    auto stdO = [&](int st) { return stages + st * C::STAGE_A + C::TILE; };
    auto stL = [&](int st) { return reinterpret_cast<float*>(stages + st * C::STAGE_A + 2 * C::TILE); };
    auto stDl = [&](int st) { return stL(st) + 128; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int kt, b, g;
    if (ATTN_BWD_SEQ_MAJOR && a.B <= 32) {
        // sequences longest first; in each, the key tile ascending (causal key tiles
        // near the start see the most queries), all KV heads of a tile side by side
        const int len = lane < a.B ? a.cu_k[lane + 1] - a.cu_k[lane] : -1;
        const int nkb = lane < a.B ? (max(len, 0) + 127) / 128 : 0;
        int local;
        if (!seq_major_unit((int)blockIdx.x, a.B, len, nkb * a.Hkv, &b, &local)) return;
        kt = local / a.Hkv;
        g = local % a.Hkv;
    } else {
        // key tile slowest (ascending: causal key tiles near the start see the most queries)
        const int bg = a.B * a.Hkv;
        kt = (int)(blockIdx.x / bg);
        b = (int)(blockIdx.x % bg) / a.Hkv;
        g = (int)(blockIdx.x % bg) % a.Hkv;
    }
    const int q_off = a.cu_q[b], Lq = a.cu_q[b + 1] - q_off;
    const int k_off = a.cu_k[b], Lk = max(a.cu_k[b + 1] - k_off, 0);
    const int k0 = kt * 128;
    if (k0 >= Lk) return;                         // uniform
    const int dl = Lk - Lq;                       // diagonal offset (bottom-right aligned)
    const int nq = (max(Lq, 0) + 127) / 128;
    int qlo = 0, qhi = nq;                        // query tiles with a row that sees a key of the tile
    if (a.mask == kMaskCausal) {
        qlo = max(k0 - dl, 0) / 128;              // rows i >= k0 - dl
        if (a.window >= 0) {
            const int imax = k0 + 127 - dl + a.window;   // rows i <= imax
            qhi = imax >= 0 ? min(nq, imax / 128 + 1) : 0;
        }
        if (qlo >= qhi) qlo = qhi = 0;
    }
    const int nqr = qhi - qlo;
    const int n_items = a.group * nqr;            // (query head of the group, query tile)

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int i = 0; i < NS; ++i) {
            mbar_init(&st_full[i], 1);
            mbar_init(&st_empty[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_full, kBwdComputeThreads);
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == kBwdMmaWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tdV = tbase, tdK = tbase + D, tST = tbase + 2 * D, tdPT = tbase + 2 * D + 128;

    if (warp == kBwdProducerWarp) {
        // ---------------------------------------------------- K, V once; (Q, dO, LSE, Delta) per item
        if (n_items > 0) {
            if (lane == 0) {
                prefetch_tmap(&tmQ);
                prefetch_tmap(&tmdO);
                prefetch_tmap(&tmK);
                prefetch_tmap(&tmV);
                mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
#pragma unroll
                for (int c = 0; c < C::NCHUNK; ++c) {
                    tma_load_4d(&tmK, kv_full, sK + c * 128 * 128, c * 64, g, k_off + k0, 0);
                    tma_load_4d(&tmV, kv_full, sV + c * 128 * 128, c * 64, g, k_off + k0, 0);
                }
            }
            int issued = 0;
            for (int it = 0; it < n_items; ++it) {
                const int st = it % NS;
                const int h = g * a.group + it / nqr, qt = qlo + it % nqr;
                bool ok = mbar_wait(&st_empty[st], ((it / NS) & 1) ^ 1, kErrBwdLoad);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                // LSE (base 2) and Delta of the tile's 128 rows; rows past the sequence get
                // LSE = +inf (P = 0) and Delta = 0, as do rows the forward left without keys.
                float* sL = stL(st);
                float* sDl = stDl(st);
                for (int rr = lane; rr < 128; rr += 32) {
                    const int i = qt * 128 + rr;
                    float l2 = INFINITY, dd = 0.0f;
                    if (i < Lq) {
                        const float l = a.lse[(long long)h * a.total_q + q_off + i];
                        l2 = (l == -INFINITY) ? INFINITY : l * kLog2e;
                        dd = a.delta[(long long)h * a.total_q + q_off + i];
                    }
                    sL[rr] = l2;
                    sDl[rr] = dd;
                }
                __syncwarp();
                if (lane == 0) {
                    ++issued;
                    mbar_arrive_expect_tx(&st_full[st], 2 * C::TILE);
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c) {
                        tma_load_4d(&tmQ, &st_full[st], stQ(st) + c * 128 * 128, c * 64, h,
                                    q_off + qt * 128, 0);
                        tma_load_4d(&tmdO, &st_full[st], stdO(st) + c * 128 * 128, c * 64, h,
                                    q_off + qt * 128, 0);
                    }
                }
            }
            if (lane == 0) {
                mbar_wait_drain(kv_full, 0, kErrBwdDrain);
                for (int st = 0; st < NS && st < issued; ++st) {
                    const int last = st + ((issued - 1 - st) / NS) * NS;
                    mbar_wait_drain(&st_full[st], (last / NS) & 1, kErrBwdDrain);
                }
            }
        }
    } else if (warp == kBwdMmaWarp) {
        // ---------------------------------------------------- MMA issuer
        if (n_items > 0 && lane == 0) {
            const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
            bool ok = mbar_wait(kv_full, 0, kErrBwdMma);
            for (int it = 0; ok && it < n_items; ++it) {
                const int st = it % NS;
                if (!(ok = mbar_wait(&st_full[st], (it / NS) & 1, kErrBwdMma))) break;
                tc_fence_after();
                const uint32_t sQa = smem_u32(stQ(st)), sdOa = smem_u32(stdO(st));
                // S^T = K Q^T and dP^T = V dO^T (K-major, K = D; lanes = keys)
#pragma unroll
                for (int kk = 0; kk < D / C::KSTEP; ++kk) {
                    const uint32_t cb = (kk * 32) / 128, off = (kk * 32) % 128;
                    const uint32_t ro = cb * 128 * 128 + off;
                    mma_f16_ss(tST, smem_desc(sKa + ro, 16, 1024, 2), smem_desc(sQa + ro, 16, 1024, 2),
                               C::IDESC_SS, kk > 0);
                    mma_f16_ss(tdPT, smem_desc(sVa + ro, 16, 1024, 2), smem_desc(sdOa + ro, 16, 1024, 2),
                               C::IDESC_SS, kk > 0);
                }
                mma_commit(s_full);
                if (!(ok = mbar_wait(p_full, it & 1, kErrBwdMma))) break;
                tc_fence_after();
                // dV += P^T dO and dK += dS^T Q: A from TMEM (bf16 over S^T / dP^T),
                // B = the dO / Q tile read MN-major (K = query rows)
#pragma unroll
                for (int kk = 0; kk < 128 / C::KSTEP; ++kk) {
                    const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
                    mma_f16_ts(tdV, tST + bwd_a_col(kk), smem_desc(sdOa + kk * 2 * 1024, 128 * 128, 1024, 2),
                               C::IDESC_TS, acc);
                    mma_f16_ts(tdK, tdPT + bwd_a_col(kk), smem_desc(sQa + kk * 2 * 1024, 128 * 128, 1024, 2),
                               C::IDESC_TS, acc);
                }
                mma_commit(&st_empty[st]);
            }
            mma_commit(mma_done);
            mbar_wait_drain(mma_done, 0, kErrBwdMma);
        }
    } else {
        // ---------------------------------------------------- compute warpgroups (thread = key)
        const int quad = warp & 3, hf = warp >> 2;   // TMEM lane quarter; warpgroup
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const int j = k0 + r;
        const bool key_ok = j < Lk;
        const float sl2 = a.scale * kLog2e;
        bool ok = true;
        for (int it = 0; it < n_items; ++it) {
            const int st = it % NS;
            const int qt = qlo + it % nqr;
            // the stage's LSE / Delta were written by the producer's threads: acquire
            // them from the stage barrier (its phase cannot move on before this
            // item's P hand-over below releases the stage)
            ok = mbar_wait(&st_full[st], (it / NS) & 1, kErrBwdCompute);
            ok = ok && mbar_wait(s_full, it & 1, kErrBwdCompute);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const float* sL = stL(st);
            const float* sDl = stDl(st);
            const int ibase = qt * 128;
            // key j is allowed for row i iff (causal) j <= i + dl and (window) j >= i + dl - W;
            // a tile whose every (row, key) pair is allowed skips the per-element test
            // (rows past the sequence have LSE = +inf, so P = 0 there anyway)
            const bool causal = a.mask == kMaskCausal;
            bool all_ok = k0 + 128 <= Lk;
            if (causal) {
                all_ok = all_ok && k0 + 127 <= ibase + dl;
                if (a.window >= 0) all_ok = all_ok && k0 >= ibase + 127 + dl - a.window;
            }
#pragma unroll
            for (int cc = 0; cc < 4 / kBwdWG; ++cc) {
                const int c4 = hf + cc * kBwdWG;
                uint32_t us[32], ud[32];
                tmem_ld32(tST + lane_off + c4 * 32, us);
                tmem_ld32(tdPT + lane_off + c4 * 32, ud);
                tmem_wait_ld();
                uint32_t pp[8], dd[8];   // one half (8 words = 16 columns) of the block's results
                float4 lv, dv;   // 4 rows of LSE (base 2) and Delta, broadcast from shared memory
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    if ((c & 1) == 0) {
                        lv = reinterpret_cast<const float4*>(sL + c4 * 32)[c / 2];
                        dv = reinterpret_cast<const float4*>(sDl + c4 * 32)[c / 2];
                    }
                    // columns 2c, 2c+1 are rows with LSE / Delta at lanes (2c & 3), (2c & 3) + 1 of lv / dv
                    const float2 nl = (c & 1) ? make_float2(-lv.z, -lv.w) : make_float2(-lv.x, -lv.y);
                    const float2 nd = (c & 1) ? make_float2(-dv.z, -dv.w) : make_float2(-dv.x, -dv.y);
                    const float2 x = ffma2(make_float2(__uint_as_float(us[2 * c]), __uint_as_float(us[2 * c + 1])),
                                           make_float2(sl2, sl2), nl);
                    float2 p = make_float2(ex2(x.x), ex2(x.y));
                    if (!all_ok) {
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int i = ibase + c4 * 32 + 2 * c + e;
                            bool allowed = key_ok;
                            if (causal) {
                                allowed = allowed && j <= i + dl;
                                if (a.window >= 0) allowed = allowed && j >= i + dl - a.window;
                            }
                            if (!allowed) (e == 0 ? p.x : p.y) = 0.0f;
                        }
                    }
                    const float2 dp = fadd2(make_float2(__uint_as_float(ud[2 * c]), __uint_as_float(ud[2 * c + 1])), nd);
                    const float2 ds = fmul2(p, fmul2(dp, make_float2(a.scale, a.scale)));
                    pp[c & 7] = pack_bf16(p.x, p.y);
                    dd[c & 7] = pack_bf16(ds.x, ds.y);
                    if ((c & 7) == 7) {
                        // block c4, half c / 8 -> columns this warpgroup has already read
                        tmem_st8(tST + lane_off + bwd_out_col(c4) + (c & 8), pp);
                        tmem_st8(tdPT + lane_off + bwd_out_col(c4) + (c & 8), dd);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        bool have = false;
        if (ok && n_items > 0) {
            const bool w = mbar_wait(mma_done, 0, kErrBwdCompute);
            have = __all_sync(0xffffffffu, w);
            tc_fence_after();
        }
        __syncwarp();
        // the 2 D/32 output blocks (dV's, then dK's) go round the warpgroups
        for (int blk = hf; blk < 2 * (D / 32); blk += kBwdWG) {
            const int which = blk / (D / 32), c4 = blk % (D / 32);
            const uint32_t tacc = which == 0 ? tdV : tdK;
            __nv_bfloat16* dst = (which == 0 ? a.dv : a.dk) + ((long long)(k_off + j) * a.Hkv + g) * D;
            if (have) {
                {
                    uint32_t u[32];
                    tmem_ld32(tacc + lane_off + c4 * 32, u);
                    tmem_wait_ld();
                    if (key_ok) {
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4) {
                            uint4 w;
                            w.x = pack_bf16(__uint_as_float(u[8 * v4 + 0]), __uint_as_float(u[8 * v4 + 1]));
                            w.y = pack_bf16(__uint_as_float(u[8 * v4 + 2]), __uint_as_float(u[8 * v4 + 3]));
                            w.z = pack_bf16(__uint_as_float(u[8 * v4 + 4]), __uint_as_float(u[8 * v4 + 5]));
                            w.w = pack_bf16(__uint_as_float(u[8 * v4 + 6]), __uint_as_float(u[8 * v4 + 7]));
                            reinterpret_cast<uint4*>(dst + c4 * 32)[v4] = w;
                        }
                    }
                }
            } else if (key_ok) {
                for (int v4 = 0; v4 < 4; ++v4)
                    reinterpret_cast<uint4*>(dst + c4 * 32)[v4] = make_uint4(0, 0, 0, 0);
            }
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

}  // namespace attn
