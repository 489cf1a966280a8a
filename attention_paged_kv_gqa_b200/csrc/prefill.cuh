// prefill.cuh -- fused attention forward on sm_100a: TMA producer warp,
// tcgen05 MMA warp with S/O accumulators in TMEM, two softmax warpgroups.
//
// Computes, per query row, O = softmax(scale * q K^T + mask) V and
// LSE = ln sum exp(scale * q.k) (FlexAttention forward with OUTPUT_LOGSUMEXP;
// "Cross Attention does not work on CPU and older GPUs", lowering arguments),
// over dense or varlen batches, grouped-query heads, a KV cache read either
// packed or page by page through block_table ("[CUDA] PagedAttention: add
// SM<80 fp16 fallback via memory-efficient attention", Implementation step 2:
// here the pages are fetched straight into shared memory by TMA, with no
// gather-into-a-packed-buffer pass), causal and patch masks, bf16 or fp8 e4m3
// operands ("[FlexAttention] Enforce Q,K,V memory layouts for fp8 flex
// attention": both GEMMs in the query dtype).
//
// CTA = one work unit = two 128-row query sub-tiles that share every K/V tile:
//   * group size even: the same 128 query rows of two heads of one KV group;
//   * otherwise: two consecutive 128-row query tiles of one head.
// Warps 0-3 / 4-7: softmax warpgroups for sub-tile 0 / 1 (thread = query row =
// TMEM lane).  Warp 8: TMA producer.  Warp 9: TMEM allocator + MMA issuer.
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
// P (bf16, or e4m3 for fp8) overwrites the first columns of S and is the A
// operand of the P.V MMA straight from TMEM.  V is the B operand in its
// natural [key][d] layout as an MN-major shared-memory descriptor, so no
// transposing copy of V is ever made (for fp8 too).
#pragma once

#include "ptx.cuh"

namespace attn {

constexpr int kBM = 128;           // query rows per sub-tile
constexpr int kBN = 128;           // keys per KV tile
constexpr int kPrefillThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kPageRows = 16;      // paged KV: tokens per page
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8
constexpr float kLn2 = 0.69314718055994531f;
constexpr float kLog2e = 1.44269504088896341f;
enum : int { kMaskNone = 0, kMaskCausal = 1, kMaskPatch = 2 };


// Error codes recorded when a bounded wait gives up.
enum : int {
    kErrProdKEmpty = 101, kErrProdVEmpty = 102, kErrProdDrain = 103,
    kErrMmaQ = 201, kErrMmaK = 202, kErrMmaV = 203, kErrMmaP = 204, kErrMmaDone = 205,
    kErrSmS = 301, kErrSmV = 302, kErrSmO = 303,
    kErrDecFull = 401, kErrDecEmpty = 402,
    kErrSelftestWait = 901,
    kErrPageRange = 111, kErrDecPageRange = 411,   // a block_table entry outside the cache
};

struct PrefillArgs {
    int B, Hq, Hkv, group;
    int mask;
    int window;          // causal only: keys i' - window .. i' (i' = i + Lk - Lq); < 0: none
    float softcap;       // > 0: logit s -> softcap * tanh(s / softcap); 0: none
    int varlen;          // 1: rows addressed through cu_seqlens (batch coordinate 0)
    int paged;           // 1: K/V through block_table, 16-token pages
    int only_qv;         // 1: score = Qv . V (selects the OQ kernel instance)
    int Lq, Lk;          // dense sizes (varlen == 0)
    const int* cu_q;
    const int* cu_k;
    const int* seqused_k;
    const int* block_table;
    int max_blocks;
    int num_blocks;      // pages in the cache (paged): entries outside [0, num_blocks) are errors
    const int* patch;    // [total_q][2] sequence-local [start, end)
    float scale;         // softmax scale (natural units)
    const float* descale_q;
    const float* descale_k;
    const float* descale_v;
    __nv_bfloat16* o;
    float* lse;
    long long o_stride_row;   // elements between query rows of one head
    long long o_stride_b;     // dense: elements between batches
    long long lse_stride_h;
    long long lse_stride_b;
    int pair_heads;
    int NH;              // head units
    int NQ;              // query units per sequence (grid extent)
};

template <int D, bool FP8, bool HQ = false>
struct PrefillCfg {
    static constexpr int E = FP8 ? 1 : 2;              // bytes per element
    static constexpr int ROWB = D * E;                  // bytes per row
    // swizzle span: 128-byte columns, or one 64-byte column for 64-byte rows (fp8, D = 64)
    static constexpr int SW = ROWB >= 128 ? 128 : 64;
    static constexpr uint32_t SWZ = SW == 128 ? 2u : 4u;   // descriptor layout code
    static constexpr int NCHUNK = ROWB / SW;            // swizzle columns per row
    static constexpr int CHUNK_E = SW / E;              // elements per swizzle column
    static constexpr int QB = kBM * ROWB;
    static constexpr int KVB = kBN * ROWB;
    static constexpr int NS = (2 * QB + 4 * 2 * KVB + 2048 <= 227 * 1024) ? 4
                              : (2 * QB + 3 * 2 * KVB + 2048 <= 227 * 1024) ? 3 : 2;
    static constexpr int KSTEP = FP8 ? 32 : 16;         // K extent of one MMA (elements = 32 B)
    static constexpr int QK_STEPS = D / KSTEP;
    static constexpr int PV_STEPS = kBN / KSTEP;
    static constexpr uint32_t IDESC_QK = instr_desc(FP8 ? 0 : 1, FP8 ? 0 : 1, 0, 0, 128, kBN);
    static constexpr uint32_t IDESC_PV = instr_desc(FP8 ? 0 : 1, FP8 ? 0 : 1, 0, 1, 128, D);
    // HQ (the Qv score term): the Qv sub-tiles beside the Q sub-tiles, and the rings
    // as deep as the rest allows -- at D = 128 one key stage (a key tile is released
    // by its score GEMM, long before the next one is due) and two value stages (the
    // score GEMM of tile j + 1 reads V(j + 1) while P.V of tile j still reads V(j))
    static constexpr int QBUF = (HQ ? 4 : 2) * QB;
    static constexpr int NS_HQ = (4 * QB + 4 * 2 * KVB + 2048 <= 227 * 1024) ? 4
                                 : (4 * QB + 3 * 2 * KVB + 2048 <= 227 * 1024) ? 3
                                 : (4 * QB + 2 * 2 * KVB + 2048 <= 227 * 1024) ? 2 : 0;
    static constexpr int NSK = HQ ? (NS_HQ ? NS_HQ : 1) : NS;   // key stages
    static constexpr int NSV = HQ ? (NS_HQ ? NS_HQ : 2) : NS;   // value stages
    static constexpr int NBAR = 1 + 4 * NS + 2 + 2 + 2 + 1;
    static constexpr int SMEM_BYTES = 1024 /*align slack*/ + QBUF + (NSK + NSV) * KVB + 1024;
    static_assert(NSK <= NS && NSV <= NS, "barrier arrays are NS deep");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(ROWB % SW == 0, "rows must be whole swizzle columns");
    static_assert(NBAR * 8 + 64 <= 1024, "barrier area");
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// CAP: the score softcap is compiled in (a separate instance, so that the
// uncapped kernel carries none of its code).  HQ: the score adds the Qv term of
// the "Rope dim" forward (HasQv), q . k + q_v . v: a second score GEMM of the
// Qv sub-tile against the value tile (K-major, as the key tile), which must then
// have landed before the score GEMM; bf16.  OQ: the only_qv score, Qv . V --
// no key tiles are fetched, the value tile is the score GEMM's B operand, and
// the key stages and barriers deepen the value ring to 2 NS slots.  Both are
// template parameters because the single MMA-issuing thread's control path is
// on the critical path: runtime switches there cost measurable throughput.
template <int D, bool FP8, bool CAP, bool OQ, bool HQ>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQv,
                   const PrefillArgs a) {
    using C = PrefillCfg<D, FP8, HQ>;
    static_assert(!(HQ && (OQ || FP8)), "the Qv score term is a bf16 instance of its own");
    constexpr int NS = C::NS;       // barrier arrays
    constexpr int NSK = C::NSK;     // key ring
    constexpr int NSV = C::NSV;     // value stages

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem;
    uint8_t* sQv = sQ + 2 * C::QB;          // HQ only
    uint8_t* sK = sQ + C::QBUF;
    uint8_t* sV = sK + NSK * C::KVB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sV + NSV * C::KVB);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + NS;
    uint64_t* v_full = k_empty + NS;
    uint64_t* v_empty = v_full + NS;
    uint64_t* s_full = v_empty + NS;
    uint64_t* p_full = s_full + 2;
    uint64_t* o_final = p_full + 2;
    uint64_t* mma_done = o_final + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    // Value ring: the NS value stages, and with only_qv (no key tiles) the NS key
    // stages and their barriers too, so that 2 NS value tiles can be in flight.
    constexpr int vring = OQ ? 2 * NS : NSV;
    auto vslot_buf = [&](int st) { return st < NSV ? sV + st * C::KVB : sK + (st - NSV) * C::KVB; };
    auto vslot_full = [&](int st) { return st < NSV ? &v_full[st] : &k_full[st - NSV]; };
    auto vslot_empty = [&](int st) { return st < NSV ? &v_empty[st] : &k_empty[st - NSV]; };
    int* sched = reinterpret_cast<int*>(tmem_slot + 2);   // [t][0]=min start, [t][1]=max end

    // ------------------------------------------------------------ work unit (a1)
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Units are enumerated with the query-unit index slowest and descending, so
    // the causal units with the most KV tiles are launched first.
    const int bh = a.B * a.NH;
    const int lin = blockIdx.x;
    const int qu = a.NQ - 1 - lin / bh;
    const int b = (lin % bh) / a.NH;
    const int hu = (lin % bh) % a.NH;

    int q_off, Lq, k_off, Lk, bcoord;
    if (a.varlen) {
        q_off = a.cu_q[b];
        Lq = a.cu_q[b + 1] - q_off;
        k_off = a.cu_k ? a.cu_k[b] : 0;
        Lk = a.seqused_k ? a.seqused_k[b] : a.cu_k[b + 1] - a.cu_k[b];
        bcoord = 0;
    } else {
        q_off = 0;
        Lq = a.Lq;
        k_off = 0;
        Lk = a.Lk;
        bcoord = b;
    }
    Lk = max(Lk, 0);
    if (a.paged) Lk = min(Lk, a.max_blocks * kPageRows);   // keys past the block table are not addressable
    int head[2], q0[2];
    if (a.pair_heads) {
        head[0] = 2 * hu;
        head[1] = 2 * hu + 1;
        q0[0] = q0[1] = qu * kBM;
    } else {
        head[0] = head[1] = hu;
        q0[0] = (2 * qu) * kBM;
        q0[1] = (2 * qu + 1) * kBM;
    }
    const bool valid0 = q0[0] < Lq, valid1 = q0[1] < Lq;
    if (!valid0 && !valid1) return;   // uniform: nothing to do for this unit
    const int g = head[0] / a.group;
    const int nkt = (Lk + kBN - 1) / kBN;

    if (threadIdx.x == 0) {
        sched[0] = sched[2] = 0x7fffffff;
        sched[1] = sched[3] = -0x7fffffff;
    }
    __syncthreads();
    if (a.mask == kMaskPatch && warp < 8) {
        // Block-sparse tile range of each sub-tile from its rows' key intervals.
        const int t = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const int qi = (t ? q0[1] : q0[0]) + r;   // (a select: no dynamically indexed array)
        int s = 0x7fffffff, e = -0x7fffffff;
        if (qi < Lq) {
            const int rs = max(a.patch[2LL * (q_off + qi)], 0);
            const int re = min(a.patch[2LL * (q_off + qi) + 1], Lk);
            if (rs < re) { s = rs; e = re; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s = min(s, __shfl_xor_sync(0xffffffffu, s, o));
            e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
        }
        if (lane == 0) {
            atomicMin(&sched[2 * t], s);
            atomicMax(&sched[2 * t + 1], e);
        }
    }
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < NS; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], kBM);
            mbar_init(&o_final[t], 1);
        }
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    // KV tile range [lo_t, hi_t) per sub-tile (empty for an invalid sub-tile).
    int lo_t[2], hi_t[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        lo_t[t] = hi_t[t] = 0;
        if (!(t == 0 ? valid0 : valid1) || nkt == 0) continue;
        const int rows_end = min(q0[t] + kBM, Lq);
        if (a.mask == kMaskNone) {
            hi_t[t] = nkt;
        } else if (a.mask == kMaskCausal) {
            const int maxkey = rows_end - 1 + (Lk - Lq);
            if (maxkey >= 0) hi_t[t] = min(nkt, maxkey / kBN + 1);
            if (a.window >= 0 && hi_t[t] > 0) {
                // sliding window: the sub-tile's first row sees the earliest key
                lo_t[t] = max(q0[t] + (Lk - Lq) - a.window, 0) / kBN;
                if (lo_t[t] >= hi_t[t]) lo_t[t] = hi_t[t] = 0;
            }
        } else {
            const int s = sched[2 * t], e = sched[2 * t + 1];
            if (s < e) {
                lo_t[t] = s / kBN;
                hi_t[t] = min(nkt, (e + kBN - 1) / kBN);
            }
        }
    }
    int lo = 0x7fffffff, hi = 0;
#pragma unroll
    for (int t = 0; t < 2; ++t)
        if (hi_t[t] > lo_t[t]) {
            lo = min(lo, lo_t[t]);
            hi = max(hi, hi_t[t]);
        }
    const bool any_tiles = hi > lo;

    if (warp == kProducerWarp) {
        // -------------------------------------------------------- TMA producer (a2, a3)
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            if constexpr (HQ) prefetch_tmap(&tmQv);
        }
        int issued = 0;
        if (any_tiles) {
            if (lane == 0) {
                uint32_t qbytes = 0;
#pragma unroll
                for (int t = 0; t < 2; ++t)
                    if (hi_t[t] > lo_t[t]) qbytes += C::QB;
                mbar_arrive_expect_tx(q_full, HQ ? 2 * qbytes : qbytes);
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (hi_t[t] <= lo_t[t]) continue;
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c) {
                        tma_load_4d(&tmQ, q_full, sQ + t * C::QB + c * kBM * C::SW, c * C::CHUNK_E,
                                    head[t], q_off + q0[t], bcoord);
                        if constexpr (HQ)
                            tma_load_4d(&tmQv, q_full, sQv + t * C::QB + c * kBM * C::SW, c * C::CHUNK_E,
                                        head[t], q_off + q0[t], bcoord);
                    }
                }
            }
            const uint64_t pol = policy_evict_last();
            for (int j = lo; j < hi; ++j, ++issued) {
                const int it = j - lo;
                const int st = it % NSK;
                const uint32_t ph = (it / NSK) & 1;
                const int vst = it % vring;                 // value ring (2 NS deep with only_qv)
                const uint32_t vph = (it / vring) & 1;
                uint64_t* vfull = vslot_full(vst);
                uint8_t* vbuf = vslot_buf(vst);
                int page = -1;
                constexpr int PPT = kBN / kPageRows;   // pages per tile
                if (a.paged && lane < PPT) {
                    const int slot = j * PPT + lane;
                    if (slot * kPageRows < Lk && slot < a.max_blocks) {
                        page = a.block_table[(long long)b * a.max_blocks + slot];
                        if (page < 0 || page >= a.num_blocks) {
                            // outside the cache: reported, and a page inside it read instead
                            record_data_error(kErrPageRange);
                            page = 0;
                        }
                    }
                }
                int npv = 0;
#pragma unroll
                for (int p = 0; p < PPT; ++p) npv += (j * kBN + p * kPageRows < Lk) ? 1 : 0;
                const uint32_t bytes = a.paged ? npv * kPageRows * C::ROWB : C::KVB;

                bool ok = true;
                if constexpr (!OQ) {
                    ok = mbar_wait(&k_empty[st], ph ^ 1, kErrProdKEmpty);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    if (a.paged) {
                        // the tile's byte count first, then each page lane issues its own page's boxes
                        if (lane == 0) mbar_arrive_expect_tx(&k_full[st], bytes);
                        __syncwarp();
                        if (lane < PPT && j * kBN + lane * kPageRows < Lk) {
                            uint8_t* dst = sK + st * C::KVB + lane * kPageRows * C::SW;
#pragma unroll
                            for (int c = 0; c < C::NCHUNK; ++c)
                                tma_load_4d_hint(&tmK, &k_full[st], dst + c * kBN * C::SW, c * C::CHUNK_E, g,
                                                 page * kPageRows, 0, pol);
                        }
                    } else if (lane == 0) {
                        mbar_arrive_expect_tx(&k_full[st], bytes);
                        uint8_t* dst = sK + st * C::KVB;
#pragma unroll
                        for (int c = 0; c < C::NCHUNK; ++c)
                            tma_load_4d_hint(&tmK, &k_full[st], dst + c * kBN * C::SW,
                                             c * C::CHUNK_E, g, k_off + j * kBN, bcoord, pol);
                    }
                }
                ok = mbar_wait(vslot_empty(vst), vph ^ 1, kErrProdVEmpty);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) { if (!OQ) ++issued; break; }
                if (a.paged) {
                    // the tile's byte count first, then each page lane issues its own page's boxes
                    if (lane == 0) mbar_arrive_expect_tx(vfull, bytes);
                    __syncwarp();
                    if (lane < PPT && j * kBN + lane * kPageRows < Lk) {
                        uint8_t* dst = vbuf + lane * kPageRows * C::SW;
#pragma unroll
                        for (int c = 0; c < C::NCHUNK; ++c)
                            tma_load_4d_hint(&tmV, vfull, dst + c * kBN * C::SW, c * C::CHUNK_E, g,
                                             page * kPageRows, 0, pol);
                    }
                } else if (lane == 0) {
                    mbar_arrive_expect_tx(vfull, bytes);
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c)
                        tma_load_4d_hint(&tmV, vfull, vbuf + c * kBN * C::SW,
                                         c * C::CHUNK_E, g, k_off + j * kBN, bcoord, pol);
                }
            }
            // Let every copy this warp started land before the CTA can exit.
            if (lane == 0) {
                if constexpr (!OQ) {
                    for (int st = 0; st < NSK && st < issued; ++st) {
                        const int last = st + ((issued - 1 - st) / NSK) * NSK;
                        mbar_wait_drain(&k_full[st], (last / NSK) & 1, kErrProdDrain);
                    }
                }
                for (int st = 0; st < vring && st < issued; ++st) {
                    const int last = st + ((issued - 1 - st) / vring) * vring;
                    mbar_wait_drain(vslot_full(st), (last / vring) & 1, kErrProdDrain);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // -------------------------------------------------------- MMA issuer (a4, a6)
        if (any_tiles && lane == 0) {
            const uint32_t tS[2] = {tbase, tbase + 128};
            const uint32_t tO[2] = {tbase + 256, tbase + 256 + D};
            const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
            auto part = [&](int t, int j) { return lo_t[t] <= j && j < hi_t[t]; };
            // score GEMM: B operand at kb (the key tile; with only_qv the value tile, whose
            // slot is released by the P.V GEMM that reads it last)
            auto issue_s = [&](int t, uint32_t kb, uint32_t vb) {
#pragma unroll
                for (int kk = 0; kk < C::QK_STEPS; ++kk) {
                    // K-major, 8-row groups SW * 8 bytes apart; a K step of 32 bytes
                    // moves the start within the swizzle column
                    const uint32_t cb = (kk * 32) / C::SW, off = (kk * 32) % C::SW;
                    const uint32_t qa = sQa + t * C::QB + cb * kBM * C::SW + off;
                    const uint32_t ka = kb + cb * kBN * C::SW + off;
                    const uint64_t da = smem_desc(qa, 16, 8 * C::SW, C::SWZ);
                    const uint64_t db = smem_desc(ka, 16, 8 * C::SW, C::SWZ);
                    if constexpr (FP8) mma_f8_ss(tS[t], da, db, C::IDESC_QK, kk > 0);
                    else mma_f16_ss(tS[t], da, db, C::IDESC_QK, kk > 0);
                }
                if constexpr (HQ) {
                    // + Qv V^T: the value tile read K-major, exactly as the key tile
                    const uint32_t sQva = smem_u32(sQv);
#pragma unroll
                    for (int kk = 0; kk < C::QK_STEPS; ++kk) {
                        const uint32_t cb = (kk * 32) / C::SW, off = (kk * 32) % C::SW;
                        const uint64_t da = smem_desc(sQva + t * C::QB + cb * kBM * C::SW + off, 16, 8 * C::SW, C::SWZ);
                        const uint64_t db = smem_desc(vb + cb * kBN * C::SW + off, 16, 8 * C::SW, C::SWZ);
                        mma_f16_ss(tS[t], da, db, C::IDESC_QK, 1u);
                    }
                } else {
                    (void)vb;
                }
            };
            auto issue_pv = [&](int t, uint32_t vb, bool acc) {
#pragma unroll
                for (int kk = 0; kk < C::PV_STEPS; ++kk) {
                    // MN-major: swizzle columns of d kBN * SW bytes apart (LBO), 8-key
                    // groups 8 * SW bytes apart (SBO); a K step of KSTEP keys
                    const uint32_t va = vb + kk * (C::KSTEP / 8) * (8 * C::SW);
                    const uint64_t db = smem_desc(va, kBN * C::SW, 8 * C::SW, C::SWZ);
                    const uint32_t pa = tS[t] + kk * 8;
                    if constexpr (FP8) mma_f8_ts(tO[t], pa, db, C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
                    else mma_f16_ts(tO[t], pa, db, C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(q_full, 0, kErrMmaQ);
            bool started[2] = {false, false};
            int pcount[2] = {0, 0};
            if (ok) ok = mbar_wait(OQ ? vslot_full(0) : &k_full[0], 0, kErrMmaK);
            if (HQ && ok) ok = mbar_wait(vslot_full(0), 0, kErrMmaV);
            if (ok) {
                tc_fence_after();
                const uint32_t kb0 = OQ ? smem_u32(vslot_buf(0)) : sKa;
#pragma unroll
                for (int t = 0; t < 2; ++t)
                    if (part(t, lo)) {
                        issue_s(t, kb0, smem_u32(vslot_buf(0)));
                        mma_commit(&s_full[t]);
                    }
                if (!OQ) mma_commit(&k_empty[0]);
            }
            for (int j = lo; ok && j < hi; ++j) {
                const int it = j - lo;
                const int st1 = (it + 1) % NSK;
                const uint32_t ph1 = ((it + 1) / NSK) & 1;
                const int vst = it % vring, vst1 = (it + 1) % vring;
                const uint32_t vph = (it / vring) & 1, vph1 = ((it + 1) / vring) & 1;
                const bool next = j + 1 < hi;
                bool k1 = false;
                if (!(ok = mbar_wait(vslot_full(vst), vph, kErrMmaV))) break;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (part(t, j)) {
                        if (!(ok = mbar_wait(&p_full[t], pcount[t] & 1, kErrMmaP))) break;
                        ++pcount[t];
                        tc_fence_after();
                        issue_pv(t, smem_u32(vslot_buf(vst)), started[t]);
                        started[t] = true;
                        if (j == hi_t[t] - 1) mma_commit(&o_final[t]);
                    }
                    if (next && part(t, j + 1)) {
                        if (!k1) {
                            ok = OQ ? mbar_wait(vslot_full(vst1), vph1, kErrMmaK)
                                           : mbar_wait(&k_full[st1], ph1, kErrMmaK);
                            if (HQ && ok) ok = mbar_wait(vslot_full(vst1), vph1, kErrMmaV);
                            if (!ok) break;
                            tc_fence_after();
                            k1 = true;
                        }
                        issue_s(t, OQ ? smem_u32(vslot_buf(vst1)) : sKa + st1 * C::KVB,
                                smem_u32(vslot_buf(vst1)));
                        mma_commit(&s_full[t]);
                    }
                }
                if (!ok) break;
                mma_commit(vslot_empty(vst));
                if (next && !OQ) {
                    if (!k1 && !(ok = mbar_wait(&k_full[st1], ph1, kErrMmaK))) break;
                    mma_commit(&k_empty[st1]);
                }
            }
            // All MMAs this thread issued must finish before TMEM is released.
            mma_commit(mma_done);
            mbar_wait_drain(mma_done, 0, kErrMmaDone);
        }
    } else {
        // -------------------------------------------------------- softmax warpgroups (a5, a7)
        const int t = warp >> 2;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t tS = tbase + lane_off + t * 128;
        const uint32_t tO = tbase + lane_off + 256 + t * D;
        // This sub-tile's values as scalars (selects, so that the small per-sub-tile
        // arrays stay in registers instead of on the stack).
        const int lo_mine = t ? lo_t[1] : lo_t[0];
        const int hi_mine = t ? hi_t[1] : hi_t[0];
        const int qi = (t ? q0[1] : q0[0]) + r;
        const bool row_ok = (t == 0 ? valid0 : valid1) && qi < Lq;
        const int head_t = t ? head[1] : head[0];
        float sl2 = a.scale * kLog2e;
        float eff = a.scale;                 // logit = eff * (raw dot product)
        float out_scale = 1.0f;
        if constexpr (FP8) {
            sl2 *= __ldg(a.descale_q) * __ldg(a.descale_k);
            eff *= __ldg(a.descale_q) * __ldg(a.descale_k);
            out_scale = __ldg(a.descale_v);
        }
        const float cap_in = CAP ? eff / a.softcap : 0.0f;
        const float cap_out = CAP ? a.softcap / eff : 0.0f;
        // Allowed keys of this row: [klo, khi).
        int klo = 0, khi = Lk;
        if (a.mask == kMaskCausal) {
            khi = min(Lk, qi + (Lk - Lq) + 1);
            if (a.window >= 0) klo = max(qi + (Lk - Lq) - a.window, 0);
        }
        if (a.mask == kMaskPatch && row_ok) {
            klo = max(a.patch[2LL * (q_off + qi)], 0);
            khi = min(a.patch[2LL * (q_off + qi) + 1], Lk);
        }
        // Rows past the sequence end are computed like unmasked rows (their
        // inputs are finite: the next sequence's rows or TMA zero fill) and
        // never stored; masking them would only slow their warp down.
        if (!row_ok) { klo = 0; khi = Lk; }

        float m_run = -INFINITY, l_run = 0.0f;
        const int n_t = hi_mine - lo_mine;
        bool ok = true;
        for (int jj = 0; jj < n_t; ++jj) {
            const int j = lo_mine + jj;
            ok = mbar_wait(&s_full[t], jj & 1, kErrSmS);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            float s[kBN];
            {
                // All four column blocks in flight, one wait.
                uint32_t u[kBN];
#pragma unroll
                for (int c4 = 0; c4 < kBN / 32; ++c4)
                    tmem_ld32(tS + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c4 * 32]));
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < kBN; ++c) s[c] = __uint_as_float(u[c]);
            }
            if constexpr (CAP) {
                const float kin2 = cap_in * 2.88539008177792681f;   // 2 log2(e) k_in
#pragma unroll
                for (int c = 0; c < kBN; c += 2) {
                    const float2 v = softcap_raw2(make_float2(s[c], s[c + 1]), kin2, cap_out);
                    s[c] = v.x;
                    s[c + 1] = v.y;
                }
            }
            const int kbase = j * kBN;
            if (kbase < klo || kbase + kBN > khi) {
#pragma unroll
                for (int c = 0; c < kBN; ++c) {
                    const int kv = kbase + c;
                    s[c] = (kv >= klo && kv < khi) ? s[c] : -INFINITY;
                }
            }
            // Row max: 8 independent chains of three-input max.
            float mx;
            {
                float m8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) m8[i] = fmaxf(s[i], s[8 + i]);
#pragma unroll
                for (int c = 16; c < kBN; c += 16)
#pragma unroll
                    for (int i = 0; i < 8; ++i) m8[i] = fmax3(m8[i], s[c + i], s[c + 8 + i]);
                mx = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], fmax3(m8[5], m8[6], m8[7])));
            }
            const float m_new = fmaxf(m_run, mx * sl2);
            const bool want = m_new > m_run + kRescaleThreshold;
            float alpha = 1.0f;
            if (want) {
                alpha = ex2(m_run - m_new);
                l_run *= alpha;
                m_run = m_new;
            }
            const float mu = (m_run == -INFINITY) ? 0.0f : m_run;
            // x = s * sl2 - mu two lanes at a time (packed f32x2 FMA), and for fp8
            // without softcap the row sums too.
            const float2 sl2x2 = make_float2(sl2, sl2), nmu2 = make_float2(-mu, -mu);
            float2 sums2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
            __syncwarp();
            // P overwrites the first columns of S in TMEM, 32 keys at a time.
#pragma unroll
            for (int c4 = 0; c4 < kBN / 32; ++c4) {
                if constexpr (FP8) {
                    uint32_t pk[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float* sc = &s[c4 * 32 + 4 * c];
                        const float2 x01 = ffma2(make_float2(sc[0], sc[1]), sl2x2, nmu2);
                        const float2 x23 = ffma2(make_float2(sc[2], sc[3]), sl2x2, nmu2);
                        const float p0 = ex2(x01.x);
                        const float p1 = ex2(x01.y);
                        const float p2 = ex2(x23.x);
                        const float p3 = ex2(x23.y);
                        if constexpr (CAP) {   // (packed adds here cost registers with the softcap)
                            sums2[0].x += p0;
                            sums2[0].y += p1;
                            sums2[1].x += p2;
                            sums2[1].y += p3;
                        } else {
                            sums2[0] = fadd2(sums2[0], make_float2(p0, p1));
                            sums2[1] = fadd2(sums2[1], make_float2(p2, p3));
                        }
                        pk[c] = pack_e4m3x4(p0, p1, p2, p3);
                    }
                    tmem_st8(tS + c4 * 8, pk);
                } else {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float2 x = ffma2(make_float2(s[c4 * 32 + 2 * c], s[c4 * 32 + 2 * c + 1]), sl2x2, nmu2);
                        const float p0 = ex2(x.x);
                        const float p1 = ex2(x.y);
                        sums2[c & 1].x += p0;      // (packed adds here cost registers: spills)
                        sums2[c & 1].y += p1;
                        pk[c] = pack_bf16(p0, p1);
                    }
                    tmem_st16(tS + c4 * 16, pk);
                }
            }
            const float sum = (sums2[0].x + sums2[0].y) + (sums2[1].x + sums2[1].y);
            if (jj > 0 && __any_sync(0xffffffffu, want)) {
                // O holds the sum over earlier tiles (their P.V MMAs completed
                // before this tile's S was committed); rescale this row.  Rare
                // (only when the row max grows past the threshold), so the loop
                // stays rolled to keep register pressure down.
#pragma unroll 1
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t u[32];
                    tmem_ld32(tO + c4 * 32, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) u[c] = __float_as_uint(__uint_as_float(u[c]) * alpha);
                    tmem_st32(tO + c4 * 32, u);
                }
            }
            l_run += sum;
            // Keys past the end of the sequence in the final tile: V rows there
            // are not data of this sequence (stale stage contents, the unused
            // tail of the last page).  Zero them so 0 * V cannot be NaN.
            if (j == hi - 1 && (j + 1) * kBN > Lk) {
                const int zt = (lo_t[0] <= j && j < hi_t[0]) ? 0 : 1;
                if (zt == t) {
                    const int it = j - lo;
                    const int st = it % vring;
                    ok = mbar_wait(vslot_full(st), (it / vring) & 1, kErrSmV);
                    if (ok) {
                        const int first = Lk - j * kBN;
                        uint8_t* base = vslot_buf(st);
                        const int nrow = kBN - first;
                        constexpr int PPR = C::SW / 16;           // 16-byte pieces per column row
                        const int n16 = nrow * C::NCHUNK * PPR;
                        for (int i = r; i < n16; i += kBM) {
                            const int c = i / (nrow * PPR);
                            const int rem = i % (nrow * PPR);
                            const int row = first + rem / PPR;
                            const int piece = rem % PPR;
                            *reinterpret_cast<uint4*>(base + c * kBN * C::SW + row * C::SW + piece * 16) =
                                make_uint4(0, 0, 0, 0);
                        }
                        fence_proxy_async_smem();
                    }
                    ok = __all_sync(0xffffffffu, ok);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[t]);
            if (!ok) break;
        }
        // -------------------------------------------------------- epilogue (a7)
        bool have_o = false;
        if (ok && n_t > 0) {
            bool w = mbar_wait(&o_final[t], 0, kErrSmO);
            have_o = __all_sync(0xffffffffu, w);
            tc_fence_after();
        }
        const long long orow = a.o_stride_b * b + (long long)(q_off + qi) * a.o_stride_row +
                               (long long)head_t * D;
        const float inv = (l_run > 0.0f) ? out_scale / l_run : 0.0f;
        __syncwarp();
        if (have_o) {
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4) {
                uint32_t u[32];
                tmem_ld32(tO + c4 * 32, u);
                tmem_wait_ld();
                if (row_ok) {
                    uint4* dst = reinterpret_cast<uint4*>(a.o + orow + c4 * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(u[8 * v4 + 0]) * inv, __uint_as_float(u[8 * v4 + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(u[8 * v4 + 2]) * inv, __uint_as_float(u[8 * v4 + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(u[8 * v4 + 4]) * inv, __uint_as_float(u[8 * v4 + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(u[8 * v4 + 6]) * inv, __uint_as_float(u[8 * v4 + 7]) * inv);
                        dst[v4] = w;
                    }
                }
            }
        } else if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(a.o + orow);
            for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_uint4(0, 0, 0, 0);
        }
        if (row_ok && a.lse) {
            const float lse = (l_run > 0.0f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
            a.lse[a.lse_stride_b * b + a.lse_stride_h * head_t + q_off + qi] = lse;
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

}  // namespace attn
