// decode.cuh -- paged GQA decode on sm_100a: one query token per sequence,
// key range split across CTAs (split-KV), then an LSE-weighted combine.
//
// Two kernels, both HBM-bound (about 4 flop per byte of K/V at group size 4)
// and built around the memory path.  The page-stream kernel further below is
// the default (automatic split); the per-head split kernel here serves an
// explicit split count and the shapes the page stream does not take.  In the
// split kernel a producer warp fetches each 16-token
// page of K and V straight from the paged cache through block_table with TMA
// (128-byte swizzle, no gather pass), several stages deep; four consumer warps
// each own 16 keys of a 64-key stage and keep their own online-softmax state,
// merged once at the end.  The tiny per-stage contractions (G query heads x 16
// keys x D) run on the warp-level tensor-core MMA, which keeps the consumer
// warps far from being the bottleneck.
//
// The partial results of a split are (O_s normalised, LSE_s) in fp32; the
// combine kernel merges them as LSE = ln sum_s exp(LSE_s),
// O = sum_s exp(LSE_s - LSE) O_s.  Paging and the packed-free page walk follow
// "[CUDA] PagedAttention: add SM<80 fp16 fallback via memory-efficient
// attention" (Implementation; the fp32 accumulator buffer idea); seqused_k
// follows "Rope dim" (the varlen arguments).
#pragma once

#include "prefill.cuh"

namespace attn {

constexpr int kDecThreads = 160;      // warps 0-3 consumers, warp 4 producer
constexpr int kDecStageTok = 64;      // keys per stage (4 pages)
constexpr int kDecRows = 16;          // MMA rows = query heads of one KV group (padded)
constexpr int kDecMaxSeqs = 4096;     // sequences per call (on-device item table in smem)
constexpr int kMaxSplits = 256;       // partials merged per (sequence, head)
constexpr int kCombineRegs = 8;       // partials a combine thread merges from registers

struct DecodeArgs {
    int B, Hq, Hkv, group;
    const __nv_bfloat16* q;   // [B][Hq][D]
    const int* block_table;
    int max_blocks;
    int num_blocks;           // pages in the cache: entries outside [0, num_blocks) are errors
    const int* seqused_k;
    int tokens_per_split;     // multiple of kDecStageTok
    int num_splits;
    float scale;
    int window;               // sliding window: keys L-1-window .. L-1; < 0: none
    float softcap;            // > 0: logit s -> softcap * tanh(s / softcap)
    float* o_part;            // [splits][B][Hq][D]
    float* lse_part;          // [splits][B][Hq]
    __nv_bfloat16* o;         // [B][Hq][D]  (direct mode)
    float* lse;               // [B][Hq]     (direct mode, nullable)
    int direct;               // 1: single split, write the final result
    int nstages;              // stage ring depth (runtime: sized from G and B)
    int only_qv;              // 1: score = q . v (no K loads; the score reads the V rows)
};

template <int D>
struct DecodeCfg {
    static constexpr int ROWB = D * 2;
    static constexpr int NCHUNK = ROWB / 128;
    static constexpr int STAGE_K = kDecStageTok * ROWB;
    static constexpr int STAGE = 2 * STAGE_K;              // K then V
    static_assert(STAGE % 1024 == 0, "stages stay 1024-byte aligned for the 128-byte swizzle");
    // Shared memory after the stage ring, for group size G and B sequences:
    // merge area [4][G][D] f32 + m, l [4][16] f32; tables prefix [B+1] and
    // lengths [B] int32 (16-byte rounded); then 2*NS mbarriers.
    __host__ __device__ static constexpr int merge_bytes(int G) { return 4 * G * D * 4 + 2 * 4 * kDecRows * 4; }
    __host__ __device__ static constexpr int table_bytes(int B) { return ((2 * B + 1) * 4 + 15) / 16 * 16; }
    __host__ __device__ static constexpr int tail_bytes(int G, int B, int ns) {
        return merge_bytes(G) + table_bytes(B) + 2 * ns * 8;
    }
    // vonly: stages of V alone (the only_qv score reads no K)
    __host__ __device__ static constexpr int stage_bytes(bool vonly) { return vonly ? STAGE_K : STAGE; }
    __host__ __device__ static constexpr int smem_bytes(int G, int B, int ns, bool vonly = false) {
        return 1024 + ns * stage_bytes(vonly) + tail_bytes(G, B, ns);
    }
};

// Byte offset of element (row, col) of a [rows][D] bf16 tile stored as
// 128-byte swizzled columns of `rows` rows each (the TMA SWIZZLE_128B layout).
template <int D>
__device__ __forceinline__ uint32_t swz_off(int row, int col, int rows) {
    const int c = col >> 6;               // 64 bf16 per 128-byte column
    const int piece = (col & 63) >> 3;    // 16-byte piece
    return c * rows * 128 + row * 128 + ((piece ^ (row & 7)) << 4) + ((col & 7) << 1);
}

// The decode query is the newest of a sequence's L cached tokens, so a
// sliding window of W keys lets it see keys L-1-W .. L-1.  First such key,
// and the first key of the page holding it (where the key range streamed
// from the cache starts).  W < 0: no window.
__host__ __device__ __forceinline__ int win_first_key(int L, int W) {
    return (W >= 0 && L > 0) ? max(0, L - 1 - W) : 0;
}
__host__ __device__ __forceinline__ int win_first_page_key(int L, int W) {
    return win_first_key(L, W) / kPageRows * kPageRows;
}

// Work item -> (sequence, split, kv head) through the per-sequence split counts.
struct DecItem {
    int b, split, g, t_begin, t_end, k_first;
};

// Sequence of L keys -> ceil(L / tps) splits of nearly equal size (multiples
// of the stage), so the work items of one sequence are balanced.
__host__ __device__ __forceinline__ int dec_nsplit(int L, int tps) { return (L + tps - 1) / tps; }

__device__ __forceinline__ DecItem dec_item(int item, const int* prefix, int B, int Hkv, int tps,
                                            const int* lens, int window) {
    DecItem it;
    it.g = item % Hkv;
    const int r = item / Hkv;
    int lo = 0, hi = B;           // largest b with prefix[b] <= r
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= r) lo = mid; else hi = mid;
    }
    it.b = lo;
    it.split = r - prefix[lo];
    const int L = lens[lo];
    const int kb = win_first_page_key(L, window);   // page-aligned start of the streamed keys
    const int n = max(dec_nsplit(L - kb, tps), 1);
    int sz = (L - kb + n - 1) / n;
    sz = (sz + kDecStageTok - 1) / kDecStageTok * kDecStageTok;
    it.t_begin = kb + it.split * sz;
    it.t_end = min(L, it.t_begin + sz);
    it.k_first = win_first_key(L, window);
    return it;
}

// Persistent split-KV decode: one CTA per SM walks the work items
// blockIdx.x, blockIdx.x + gridDim.x, ...; the producer warp streams the pages
// of consecutive items through one stage ring without draining between them.
template <int D>
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const DecodeArgs a) {
    using C = DecodeCfg<D>;
    const int NS = a.nstages;
    const int G = a.group;
    // A stage is K then V (STAGE_K bytes each), or with only_qv V alone: stage st's
    // K and V sit at STAGE_K multiples kslot(st) and vslot(st).
    const int STG = C::stage_bytes(a.only_qv);
    auto kslot = [&](int st) { return a.only_qv ? st : 2 * st; };
    auto vslot = [&](int st) { return a.only_qv ? st : 2 * st + 1; };
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    float* mo = reinterpret_cast<float*>(smem + NS * STG);            // [4][G][D]
    float* mm = mo + 4 * G * D;                                        // [4][16]
    float* ml = mm + 4 * kDecRows;                                     // [4][16]
    int* prefix = reinterpret_cast<int*>(ml + 4 * kDecRows);           // [B+1] split-count prefix
    int* lenv = prefix + (a.B + 1);                                    // [B] keys per sequence
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * STG + C::merge_bytes(G) +
                                                 C::table_bytes(a.B));
    uint64_t* empty = full + NS;

    // Let the combine kernel launch now; it waits for this grid's results itself.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // Launched as a programmatic dependent of a KV append, wait for it before
    // reading the lengths or the cache (a no-op for an ordinary launch).
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tps = a.tokens_per_split;
    const int cap = a.max_blocks * kPageRows;
    // Split counts per sequence and their exclusive prefix sum (warp 0).
    if (warp == 0) {
        int run = 0;
        for (int base = 0; base < a.B; base += 32) {
            const int b = base + lane;
            int cnt = 0;
            if (b < a.B) {
                const int L = min(max(a.seqused_k[b], 0), cap);
                cnt = dec_nsplit(L - win_first_page_key(L, a.window), tps);
                if (a.direct && cnt == 0) cnt = 1;    // a zero-length row is still written
            }
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (b < a.B) prefix[b] = run + incl - cnt;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) prefix[a.B] = run;
    }
    for (int b = threadIdx.x; b < a.B; b += kDecThreads)
        lenv[b] = min(max(a.seqused_k[b], 0), cap);
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 4);
        }
        fence_mbar_init();
    }
    __syncthreads();
    const int total = prefix[a.B] * a.Hkv;

    if (warp == 4) {
        // ---------------------------------------------------- producer: page gather (a3)
        if (lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
        }
        const uint64_t pol = policy_evict_first();
        int ctr = 0;       // stages filled so far (ring position and phase)
        bool ok = true;
        for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
            const DecItem it = dec_item(item, prefix, a.B, a.Hkv, tps, lenv, a.window);
            const int nstage = (it.t_end > it.t_begin)
                                   ? (it.t_end - it.t_begin + kDecStageTok - 1) / kDecStageTok : 0;
            const int slot0 = it.t_begin / kPageRows;
            int window = -1, pg = 0;
            for (int s = 0; s < nstage; ++s, ++ctr) {
                const int st = ctr % NS;
                const uint32_t ph = (ctr / NS) & 1;
                const int sbase = slot0 + s * (kDecStageTok / kPageRows);
                const int w = (sbase - slot0) / 32;
                if (w != window) {
                    window = w;
                    const int slot = slot0 + w * 32 + lane;
                    pg = (slot * kPageRows < it.t_end && slot < a.max_blocks)
                             ? a.block_table[(long long)it.b * a.max_blocks + slot] : 0;
                    if (pg < 0 || pg >= a.num_blocks) {
                        record_data_error(kErrDecPageRange);   // outside the cache: reported, page 0 read
                        pg = 0;
                    }
                }
                int pages[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) pages[p] = __shfl_sync(0xffffffffu, pg, (sbase - slot0) % 32 + p);
                ok = mbar_wait(&empty[st], ph ^ 1, kErrDecEmpty);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                if (lane == 0) {
                    int npv = 0;
#pragma unroll
                    for (int p = 0; p < 4; ++p) npv += ((sbase + p) * kPageRows < it.t_end) ? 1 : 0;
                    mbar_arrive_expect_tx(&full[st], (a.only_qv ? 1 : 2) * npv * kPageRows * C::ROWB);
                    uint8_t* dk = smem + kslot(st) * C::STAGE_K;
                    uint8_t* dv = smem + vslot(st) * C::STAGE_K;
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        if ((sbase + p) * kPageRows >= it.t_end) continue;
#pragma unroll
                        for (int c = 0; c < C::NCHUNK; ++c) {
                            const int off = c * kDecStageTok * 128 + p * kPageRows * 128;
                            if (!a.only_qv)
                                tma_load_4d_hint(&tmK, &full[st], dk + off, c * 64, it.g,
                                                 pages[p] * kPageRows, 0, pol);
                            tma_load_4d_hint(&tmV, &full[st], dv + off, c * 64, it.g,
                                             pages[p] * kPageRows, 0, pol);
                        }
                    }
                }
            }
        }
        // Every copy started must land before the CTA exits.
        if (lane == 0) {
            for (int st = 0; st < NS && st < ctr; ++st) {
                const int last = st + ((ctr - 1 - st) / NS) * NS;
                mbar_wait_drain(&full[st], (last / NS) & 1, kErrDecFull);
            }
        }
    } else {
        // ---------------------------------------------------- consumers (a4-a6 for one token)
        const int gid = lane >> 2, t4 = lane & 3;
        const float sl2 = a.scale * kLog2e;
        const bool capped = a.softcap > 0.0f;
        const float cap_in = capped ? a.scale / a.softcap : 0.0f;
        const float cap_out = capped ? a.softcap / a.scale : 0.0f;
        int ctr = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total; item += gridDim.x) {
            const DecItem it = dec_item(item, prefix, a.B, a.Hkv, tps, lenv, a.window);
            const int nstage = (it.t_end > it.t_begin)
                                   ? (it.t_end - it.t_begin + kDecStageTok - 1) / kDecStageTok : 0;
            // Q fragments (rows = the G query heads of KV head g; rows >= G are zero).
            uint32_t qa[D / 16][4];
            {
                const __nv_bfloat16* qb = a.q + ((long long)it.b * a.Hq + (long long)it.g * G) * D;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int c0 = kk * 16 + 2 * t4;
                    auto ld = [&](int row, int col) -> uint32_t {
                        if (row >= G) return 0u;
                        return __ldg(reinterpret_cast<const unsigned int*>(qb + (long long)row * D + col));
                    };
                    qa[kk][0] = ld(gid, c0);
                    qa[kk][1] = ld(gid + 8, c0);
                    qa[kk][2] = ld(gid, c0 + 8);
                    qa[kk][3] = ld(gid + 8, c0 + 8);
                }
            }
            float o[D / 8][4];
#pragma unroll
            for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
            float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;   // rows gid, gid+8
            for (int s = 0; s < nstage; ++s, ++ctr) {
                const int st = ctr % NS;
                if (ok) {
                    ok = mbar_wait(&full[st], (ctr / NS) & 1, kErrDecFull);
                    ok = __all_sync(0xffffffffu, ok);
                }
                const int tok0 = it.t_begin + s * kDecStageTok + warp * 16;   // this warp's 16 keys
                uint8_t* sv = smem + vslot(st) * C::STAGE_K;
                uint8_t* sk = smem + kslot(st) * C::STAGE_K;
                const int lrow0 = warp * 16;
                if (ok && tok0 < it.t_end) {
                    if (tok0 + 16 > it.t_end) {
                        // Zero the V rows past the end of the sequence (not data of it).
                        for (int i = lane; i < 16 * (D / 8); i += 32) {
                            const int rr = i / (D / 8), cc = (i % (D / 8)) * 8;
                            if (tok0 + rr >= it.t_end)
                                *reinterpret_cast<uint4*>(sv + swz_off<D>(lrow0 + rr, cc, kDecStageTok)) =
                                    make_uint4(0, 0, 0, 0);
                        }
                        __syncwarp();
                    }
                    // S = Q K^T for 16 keys: two n-tiles of 8 keys.
                    float sc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
                    const uint32_t skb = smem_u32(sk);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const int mi = lane >> 3, ri = lane & 7;
                        const int row = lrow0 + (mi >> 1) * 8 + ri;
                        const int col = kk * 16 + (mi & 1) * 8;
                        uint32_t b0, b1, b2, b3;
                        ldmatrix_x4(skb + swz_off<D>(row, col, kDecStageTok), b0, b1, b2, b3);
                        mma_bf16_16816(sc[0], qa[kk], b0, b1);
                        mma_bf16_16816(sc[1], qa[kk], b2, b3);
                    }
                    if (capped) {
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) sc[nt][e] = softcap_raw(sc[nt][e], cap_in, cap_out);
                    }
                    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int kv = tok0 + nt * 8 + 2 * t4 + e;
                            if (kv >= it.t_end || kv < it.k_first) {
                                sc[nt][e] = -INFINITY;
                                sc[nt][2 + e] = -INFINITY;
                            }
                            mx0 = fmaxf(mx0, sc[nt][e]);
                            mx1 = fmaxf(mx1, sc[nt][2 + e]);
                        }
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                    const float mn0 = fmaxf(m0, mx0 * sl2), mn1 = fmaxf(m1, mx1 * sl2);
                    // m = -inf (nothing seen yet) -> alpha 0; both -inf -> 1
                    const float al0 = (mn0 == -INFINITY) ? 1.0f : ex2(m0 - mn0);
                    const float al1 = (mn1 == -INFINITY) ? 1.0f : ex2(m1 - mn1);
                    m0 = mn0;
                    m1 = mn1;
                    l0 *= al0;
                    l1 *= al1;
#pragma unroll
                    for (int i = 0; i < D / 8; ++i) {
                        o[i][0] *= al0;
                        o[i][1] *= al0;
                        o[i][2] *= al1;
                        o[i][3] *= al1;
                    }
                    const float mu0 = (m0 == -INFINITY) ? 0.0f : m0;
                    const float mu1 = (m1 == -INFINITY) ? 0.0f : m1;
                    float p[2][4];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        p[nt][0] = ex2(fmaf(sc[nt][0], sl2, -mu0));
                        p[nt][1] = ex2(fmaf(sc[nt][1], sl2, -mu0));
                        p[nt][2] = ex2(fmaf(sc[nt][2], sl2, -mu1));
                        p[nt][3] = ex2(fmaf(sc[nt][3], sl2, -mu1));
                        l0 += p[nt][0] + p[nt][1];
                        l1 += p[nt][2] + p[nt][3];
                    }
                    uint32_t pa[4];
                    pa[0] = pack_bf16(p[0][0], p[0][1]);
                    pa[1] = pack_bf16(p[0][2], p[0][3]);
                    pa[2] = pack_bf16(p[1][0], p[1][1]);
                    pa[3] = pack_bf16(p[1][2], p[1][3]);
                    const uint32_t svb = smem_u32(sv);
#pragma unroll
                    for (int nd = 0; nd < D / 8; nd += 2) {
                        const int mi = lane >> 3, ri = lane & 7;
                        const int row = lrow0 + (mi & 1) * 8 + ri;
                        const int col = nd * 8 + (mi >> 1) * 8;
                        uint32_t b0, b1, b2, b3;
                        ldmatrix_x4_trans(svb + swz_off<D>(row, col, kDecStageTok), b0, b1, b2, b3);
                        mma_bf16_16816(o[nd], pa, b0, b1);
                        mma_bf16_16816(o[nd + 1], pa, b2, b3);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }
            // row sums over the quad
            l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
            l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

            // ------------------------------------------------ merge the 4 warps (own smem area)
            asm volatile("bar.sync 1, 128;" ::: "memory");   // previous item's readers are done
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
                const int col = i * 8 + 2 * t4;
                if (gid < G) {
                    *reinterpret_cast<float2*>(&mo[(warp * G + gid) * D + col]) =
                        make_float2(o[i][0], o[i][1]);
                }
                if (gid + 8 < G) {
                    *reinterpret_cast<float2*>(&mo[(warp * G + gid + 8) * D + col]) =
                        make_float2(o[i][2], o[i][3]);
                }
            }
            if (t4 == 0) {
                mm[warp * kDecRows + gid] = m0;
                mm[warp * kDecRows + gid + 8] = m1;
                ml[warp * kDecRows + gid] = l0;
                ml[warp * kDecRows + gid + 8] = l1;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            for (int idx = threadIdx.x; idx < G * D; idx += 128) {
                const int row = idx / D, col = idx % D;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < 4; ++w) M = fmaxf(M, mm[w * kDecRows + row]);
                float acc = 0.0f, l = 0.0f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const float f = ex2(mm[w * kDecRows + row] - M);
                        acc += f * mo[(w * G + row) * D + col];
                        l += f * ml[w * kDecRows + row];
                    }
                }
                const int h = it.g * G + row;
                const float on = (l > 0.0f) ? acc / l : 0.0f;
                const float lse = (l > 0.0f) ? (M + log2f(l)) * kLn2 : -INFINITY;
                if (a.direct) {
                    a.o[((long long)it.b * a.Hq + h) * D + col] = __float2bfloat16_rn(on);
                    if (col == 0 && a.lse) a.lse[(long long)it.b * a.Hq + h] = lse;
                } else {
                    const long long base = ((long long)it.split * a.B + it.b) * a.Hq + h;
                    a.o_part[base * D + col] = on;
                    if (col == 0) a.lse_part[base] = lse;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Page-stream decode: the whole batch's pages, in sequence order, are cut into
// one contiguous, equal share per CTA (one CTA per SM).  Each page is fetched
// whole -- all KV heads of its 16 tokens, 16 * Hkv * D * 2 contiguous bytes --
// by two TMA boxes per tensor through a {d, token, head, page} view, which
// streams DRAM far faster than one head's 128-byte rows at a head-count stride.
// Consumer warp h owns KV head h (its G query heads) and keeps that head's
// online softmax; where a sequence ends or the CTA's share ends it writes the
// partial (O_s normalised, LSE_s) of (this CTA, that sequence) to slot
// CTA + sequence, so at most grid + B slots exist.  The combine kernel merges,
// for each sequence, the slots of the CTAs whose share covered it.
constexpr int kPgMaxWarps = 8;         // consumer warps (KV heads) of the page-stream kernel

struct DecodePagesArgs {
    int B, Hq, Hkv, group;
    const void* q;            // [B][Hq][D] bf16, or e4m3 (the FP8 instance)
    const void* qv;           // HQ instance: [B][Hq][D] bf16, the Qv operand of the score
    const float* descale_q;   // FP8: device fp32 scalars (real value = code x descale)
    const float* descale_k;
    const float* descale_v;
    const int* block_table;
    int max_blocks;
    int num_blocks;           // pages in the cache: entries outside [0, num_blocks) are errors
    const int* seqused_k;
    float scale;
    int window;               // sliding window: keys L-1-window .. L-1; < 0: none
    float softcap;            // > 0: logit s -> softcap * tanh(s / softcap)
    float* o_part;            // [grid + B][Hq][D]
    float* lse_part;          // [grid + B][Hq]
    int* meta;                // [B + 1] page prefix, then pages per CTA (written by CTA 0)
    int nstages;
    int only_qv;              // 1: score = q . v (no K loads; the score reads the V rows)
};

template <int D, bool FP8 = false>
struct DecodePagesCfg {
    static constexpr int E = FP8 ? 1 : 2;               // bytes per element
    static constexpr int ROWB = D * E;
    // swizzle span: 128-byte columns, or one 64-byte column for 64-byte rows (e4m3, D = 64)
    static constexpr int SW = ROWB >= 128 ? 128 : 64;
    static constexpr int NCHUNK = ROWB / SW;            // swizzle columns per row
    static constexpr int CHUNK_E = SW / E;              // elements per swizzle column
    // byte offset of 16-byte piece `piece` of row `row` inside one swizzle column
    __device__ static constexpr uint32_t swz(int row, int piece) {
        return SW == 128 ? row * 128 + ((piece ^ (row & 7)) << 4)
                         : row * 64 + ((piece ^ ((row >> 1) & 3)) << 4);
    }
    // stage = one page of K and V for all heads: 2 * 16 * Hkv * D * 2 bytes (half: V alone,
    // for the only_qv score)
    __host__ __device__ static constexpr int stage_bytes(int Hkv, bool vonly = false) {
        return (vonly ? 1 : 2) * kPageRows * Hkv * ROWB;
    }
    __host__ __device__ static constexpr int table_bytes(int B) { return ((2 * B + 2) * 4 + 15) / 16 * 16; }
    __host__ __device__ static constexpr int smem_bytes(int Hkv, int B, int ns, bool vonly = false) {
        return 1024 + ns * stage_bytes(Hkv, vonly) + table_bytes(B) + 2 * ns * 8;
    }
};

// FP8: the cache (and q) hold e4m3 codes with per-tensor descales.  Pages
// arrive half as large; the consumers turn the codes into f16 in registers
// (exact) and contract with the f16 warp MMA, the descales folded into the score
// scale and the output.  For Q.K^T the contraction index is permuted alike in
// q and k, so that each lane's non-transposed ldmatrix word (4 consecutive key
// bytes) is its B fragment; for P.V a transposed ldmatrix word holds 2 keys x 2
// columns, split by a byte permute into the fragments of two 8-column tiles
// (even and odd columns of a 16-column block).
// HQ: the score has the extra term q_v . v_j of the "Rope dim" forward (HasQv):
// logit = scale (q . k_j + q_v . v_j), the page's V rows serving as a second A
// operand of the score MMA (bf16 only).
template <int D, bool FP8, int NT, bool HQ>
__global__ void __launch_bounds__(32 * (kPgMaxWarps + 1), 1)
    decode_pages_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const DecodePagesArgs a) {
    using C = DecodePagesCfg<D, FP8>;
    static_assert(!(FP8 && HQ), "the Qv score term is bf16 only");
    const int NS = a.nstages;
    const int Hkv = a.Hkv, G = a.group;
    const int SB = C::stage_bytes(Hkv, a.only_qv);          // K and V of a page, or V alone
    const int VOFF = a.only_qv ? 0 : SB / 2;                 // V's offset inside a stage
    const int rows = kPageRows * Hkv;            // rows of one 128-byte column of a stage tensor
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    int* prefix = reinterpret_cast<int*>(smem + NS * SB);   // [B+1] pages before sequence b
    int* lenv = prefix + (a.B + 1);                          // [B] keys of sequence b
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * SB + C::table_bytes(a.B));
    uint64_t* empty = full + NS;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");   // after a KV append (see above)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cap = a.max_blocks * kPageRows;
    if (warp == 0) {
        int run = 0;
        for (int base = 0; base < a.B; base += 32) {
            const int b = base + lane;
            int cnt = 0;
            if (b < a.B) {
                const int L = min(max(a.seqused_k[b], 0), cap);
                lenv[b] = L;
                cnt = (L + kPageRows - 1) / kPageRows - win_first_page_key(L, a.window) / kPageRows;
            }
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (b < a.B) prefix[b] = run + incl - cnt;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) prefix[a.B] = run;
    }
    if (threadIdx.x == 32) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], Hkv);
        }
        fence_mbar_init();
    }
    __syncthreads();
    const int P = prefix[a.B];
    const int ppc = (P + gridDim.x - 1) / gridDim.x;
    const int p0 = min(P, blockIdx.x * ppc), p1 = min(P, p0 + ppc);
    if (blockIdx.x == 0) {
        for (int b = threadIdx.x; b <= a.B; b += blockDim.x) a.meta[b] = prefix[b];
        if (threadIdx.x == 0) a.meta[a.B + 1] = ppc;
    }
    // sequence containing global page g: largest b with prefix[b] <= g
    auto seq_of = [&](int g) {
        int lo = 0, hi = a.B;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (prefix[mid] <= g) lo = mid; else hi = mid;
        }
        return lo;
    };
    const int npages = p1 - p0;

    if (warp == Hkv) {
        // ------------------------------------------------------------ producer: whole pages (a3)
        if (lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
        }
        const uint64_t pol = policy_evict_first();
        int issued = 0;
        for (int base = 0; base < npages; base += 32) {
            // this lane's page of the next 32
            const int g = p0 + base + lane;
            int phys = 0;
            if (base + lane < npages) {
                const int b = seq_of(g);
                const int slot = g - prefix[b] + win_first_page_key(lenv[b], a.window) / kPageRows;
                phys = a.block_table[(long long)b * a.max_blocks + slot];
                if (phys < 0 || phys >= a.num_blocks) {
                    record_data_error(kErrDecPageRange);   // outside the cache: reported, page 0 read
                    phys = 0;
                }
            }
            const int cnt = min(32, npages - base);
            bool ok = true;
            for (int i = 0; i < cnt; ++i, ++issued) {
                const int page = __shfl_sync(0xffffffffu, phys, i);
                const int st = issued % NS;
                ok = mbar_wait(&empty[st], ((issued / NS) & 1) ^ 1, kErrDecEmpty);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[st], SB);
                    uint8_t* dk = smem + st * SB;
                    uint8_t* dv = dk + VOFF;
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c) {
                        if (!a.only_qv)
                            tma_load_4d_hint(&tmK, &full[st], dk + c * rows * C::SW, c * C::CHUNK_E, 0, 0,
                                             page, pol);
                        tma_load_4d_hint(&tmV, &full[st], dv + c * rows * C::SW, c * C::CHUNK_E, 0, 0, page,
                                         pol);
                    }
                }
            }
            if (!ok) break;
        }
        if (lane == 0) {
            for (int st = 0; st < NS && st < issued; ++st) {
                const int last = st + ((issued - 1 - st) / NS) * NS;
                mbar_wait_drain(&full[st], (last / NS) & 1, kErrDecFull);
            }
        }
    } else if (warp < Hkv) {
        // ------------------------------------------------------------ consumer warp = KV head
        // The page's 16 keys are the M side of both warp MMAs: S^T = K Q^T (16 keys x 8
        // query heads per n-tile; NT n-tiles cover the group), then O^T += V^T P^T (16
        // output columns x 8 heads).  Of n-tile nt a lane holds heads 8 nt + 2 t4 and
        // 8 nt + 2 t4 + 1 (t4 = lane % 4), for keys gid and gid + 8 (gid = lane / 4).
        const int h = warp;
        const int gid = lane >> 2, t4 = lane & 3;
        // logit = eff * (raw dot product); FP8: the raw dot product is of the codes
        float eff = a.scale, out_scale = 1.0f;
        if constexpr (FP8) {
            eff *= __ldg(a.descale_q) * __ldg(a.descale_k);
            out_scale = __ldg(a.descale_v);
        }
        const float sl2 = eff * kLog2e;
        const bool capped = a.softcap > 0.0f;
        const float cap_in = capped ? eff / a.softcap : 0.0f;
        const float cap_out = capped ? a.softcap / eff : 0.0f;
        constexpr int QW = FP8 ? D / 32 : D / 16;          // k-steps of the score MMA
        uint32_t qb[NT][QW][2];                             // B fragments of Q^T
        uint32_t qvb[HQ ? NT : 1][HQ ? QW : 1][2];          // HQ: B fragments of Qv^T
        float o[D / 16][NT][4];                             // O^T, one 16-column tile each
        float m[NT][2], l[NT][2];                           // l: this lane's keys only
        int b = -1, b_end = 0, L = 0, kb = 0, kf = 0;
        auto load_q = [&](int bb) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int head = nt * 8 + gid;
                const bool live = head < G;
                const long long row = (long long)bb * a.Hq + (long long)h * G + (live ? head : 0);
                if constexpr (FP8) {
                    // B (32 x 8 e4m3): word 0 = q[head][32 j + 4 t4 ..], word 1 = 16 columns on
                    const uint8_t* qr = static_cast<const uint8_t*>(a.q) + row * D;
#pragma unroll
                    for (int j = 0; j < QW; ++j) {
                        qb[nt][j][0] = live ? __ldg(reinterpret_cast<const unsigned int*>(qr + 32 * j + 4 * t4)) : 0u;
                        qb[nt][j][1] = live ? __ldg(reinterpret_cast<const unsigned int*>(qr + 32 * j + 16 + 4 * t4)) : 0u;
                    }
                } else {
                    // B (16 x 8 bf16): word 0 = q[head][16 kk + 2 t4 ..], word 1 = 8 columns on
                    const __nv_bfloat16* qr = static_cast<const __nv_bfloat16*>(a.q) + row * D;
#pragma unroll
                    for (int kk = 0; kk < QW; ++kk) {
                        qb[nt][kk][0] = live ? __ldg(reinterpret_cast<const unsigned int*>(qr + 16 * kk + 2 * t4)) : 0u;
                        qb[nt][kk][1] = live ? __ldg(reinterpret_cast<const unsigned int*>(qr + 16 * kk + 8 + 2 * t4)) : 0u;
                    }
                    if constexpr (HQ) {
                        const __nv_bfloat16* qvr = static_cast<const __nv_bfloat16*>(a.qv) + row * D;
#pragma unroll
                        for (int kk = 0; kk < QW; ++kk) {
                            qvb[nt][kk][0] = live ? __ldg(reinterpret_cast<const unsigned int*>(qvr + 16 * kk + 2 * t4)) : 0u;
                            qvb[nt][kk][1] = live ? __ldg(reinterpret_cast<const unsigned int*>(qvr + 16 * kk + 8 + 2 * t4)) : 0u;
                        }
                    }
                }
            }
        };
        auto reset = [&]() {
#pragma unroll
            for (int c = 0; c < D / 16; ++c)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) o[c][nt][0] = o[c][nt][1] = o[c][nt][2] = o[c][nt][3] = 0.0f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                m[nt][0] = m[nt][1] = -INFINITY;
                l[nt][0] = l[nt][1] = 0.0f;
            }
        };
        // write the partial of (this CTA, sequence b) for this head's G query heads
        auto flush_partial = [&]() {
            const long long slot = (long long)blockIdx.x + b;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float s = l[nt][e];
                    s += __shfl_xor_sync(0xffffffffu, s, 4);
                    s += __shfl_xor_sync(0xffffffffu, s, 8);
                    s += __shfl_xor_sync(0xffffffffu, s, 16);
                    const int head = nt * 8 + 2 * t4 + e;
                    if (head < G) {
                        const float inv = s > 0.0f ? out_scale / s : 0.0f;
                        float* rp = &a.o_part[(slot * a.Hq + h * G + head) * D];
#pragma unroll
                        for (int c = 0; c < D / 16; ++c) {
                            if constexpr (FP8) {
                                // tile rows gid / gid + 8 are columns 16 c + 2 gid and + 1
                                *reinterpret_cast<float2*>(rp + 16 * c + 2 * gid) =
                                    make_float2(o[c][nt][e] * inv, o[c][nt][2 + e] * inv);
                            } else {
                                rp[16 * c + gid] = o[c][nt][e] * inv;
                                rp[16 * c + 8 + gid] = o[c][nt][2 + e] * inv;
                            }
                        }
                        if (gid == 0)
                            a.lse_part[slot * a.Hq + h * G + head] =
                                s > 0.0f ? (m[nt][e] + log2f(s)) * kLn2 : -INFINITY;
                    }
                }
        };
        bool ok = true;
        for (int i = 0; i < npages; ++i) {
            const int g = p0 + i;
            if (g >= b_end) {                       // next sequence (skipping empty ones)
                if (b >= 0) flush_partial();
                b = seq_of(g);
                b_end = prefix[b + 1];
                L = lenv[b];
                kb = win_first_page_key(L, a.window);
                kf = win_first_key(L, a.window);
                load_q(b);
                reset();
            }
            const int st = i % NS;
            if (ok) {
                ok = mbar_wait(&full[st], (i / NS) & 1, kErrDecFull);
                ok = __all_sync(0xffffffffu, ok);
            }
            const int tok0 = kb + (g - prefix[b]) * kPageRows;     // first key of this page
            uint8_t* sv = smem + st * SB + VOFF;
            uint8_t* sk = a.only_qv ? sv : smem + st * SB;
            const int r0 = h * kPageRows;                      // this head's first row in the stage
            if (ok) {
                if (tok0 + kPageRows > L) {
                    // zero this head's V rows past the sequence end (not data of it): every
                    // 16-byte piece of those rows, in each 128-byte column of the stage
                    constexpr int PPR = C::ROWB / 16;             // pieces per row
                    constexpr int PPC = C::SW / 16;               // pieces per swizzle column row
                    for (int e = lane; e < kPageRows * PPR; e += 32) {
                        const int rr = e / PPR, pc = e % PPR;
                        if (tok0 + rr >= L)
                            *reinterpret_cast<uint4*>(sv + (pc / PPC) * rows * C::SW + (r0 + rr) * C::SW +
                                                      (pc % PPC) * 16) = make_uint4(0, 0, 0, 0);
                    }
                    __syncwarp();
                }
                const int mi = lane >> 3, ri = lane & 7;
                float sc[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.0f;
                const uint32_t skb = smem_u32(sk);
                if constexpr (FP8) {
                    // A (16 keys x 32 e4m3): one ldmatrix.x4 = keys 0-7 / 8-15 of the 16-byte
                    // pieces 2 j and 2 j + 1, which is the fragment as it stands
#pragma unroll
                    for (int j = 0; j < QW; ++j) {
                        const int row = r0 + (mi & 1) * 8 + ri;
                        const int piece = 2 * j + (mi >> 1);
                        uint32_t ka[4];
                        ldmatrix_x4(skb + C::swz(row, piece), ka[0], ka[1], ka[2], ka[3]);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_e4m3_16832(sc[nt], ka, qb[nt][j][0], qb[nt][j][1]);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < QW; ++kk) {
                        const int row = r0 + (mi & 1) * 8 + ri;
                        const int col = kk * 16 + (mi >> 1) * 8;
                        uint32_t ka[4];
                        ldmatrix_x4(skb + swz_off<D>(row, col, rows), ka[0], ka[1], ka[2], ka[3]);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sc[nt], ka, qb[nt][kk][0], qb[nt][kk][1]);
                    }
                    if constexpr (HQ) {
                        // + V Qv^T: the V rows as the A operand, read like the K rows
                        const uint32_t svs = smem_u32(sv);
#pragma unroll
                        for (int kk = 0; kk < QW; ++kk) {
                            const int row = r0 + (mi & 1) * 8 + ri;
                            const int col = kk * 16 + (mi >> 1) * 8;
                            uint32_t va[4];
                            ldmatrix_x4(svs + swz_off<D>(row, col, rows), va[0], va[1], va[2], va[3]);
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sc[nt], va, qvb[nt][kk][0], qvb[nt][kk][1]);
                        }
                    }
                }
                if (capped) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) sc[nt][e] = softcap_raw(sc[nt][e], cap_in, cap_out);
                }
                const int key0 = tok0 + gid, key1 = key0 + 8;
                const bool dead0 = key0 >= L || key0 < kf, dead1 = key1 >= L || key1 < kf;
                uint32_t pb[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (dead0) sc[nt][0] = sc[nt][1] = -INFINITY;
                    if (dead1) sc[nt][2] = sc[nt][3] = -INFINITY;
                    float p[4];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        // the max over the page's keys: this lane's two, then across gid
                        float mx = fmaxf(sc[nt][e], sc[nt][2 + e]);
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                        const float mn = fmaxf(m[nt][e], mx * sl2);
                        const float al = (mn == -INFINITY) ? 1.0f : ex2(m[nt][e] - mn);
                        m[nt][e] = mn;
#pragma unroll
                        for (int c = 0; c < D / 16; ++c) {
                            o[c][nt][e] *= al;
                            o[c][nt][2 + e] *= al;
                        }
                        const float mu = (mn == -INFINITY) ? 0.0f : mn;
                        p[e] = ex2(fmaf(sc[nt][e], sl2, -mu));
                        p[2 + e] = ex2(fmaf(sc[nt][2 + e], sl2, -mu));
                        l[nt][e] = l[nt][e] * al + p[e] + p[2 + e];
                    }
                    // P (keys x heads, this lane: keys gid / gid + 8, heads 2 t4, 2 t4 + 1)
                    // transposed in registers: B (16 keys x 8 heads) of the P.V MMA
                    if constexpr (FP8) {
                        pb[nt][0] = movmatrix_trans(pack_f16(p[0], p[1]));
                        pb[nt][1] = movmatrix_trans(pack_f16(p[2], p[3]));
                    } else {
                        pb[nt][0] = movmatrix_trans(pack_bf16(p[0], p[1]));
                        pb[nt][1] = movmatrix_trans(pack_bf16(p[2], p[3]));
                    }
                }
                const uint32_t svb = smem_u32(sv);
                if constexpr (FP8) {
                    // A (16 columns x 16 keys, f16): one ldmatrix.x4.trans = keys 0-7 / 8-15 of
                    // pieces cc and cc + 1; a lane's word holds v[2 t4][2 gid], v[2 t4][2 gid + 1],
                    // v[2 t4 + 1][2 gid], v[2 t4 + 1][2 gid + 1].  The byte permute pairs the
                    // keys of column 2 gid (tile row gid) and of column 2 gid + 1 (row gid + 8).
#pragma unroll
                    for (int cc = 0; cc < D / 16; cc += 2) {
                        const int row = r0 + (mi & 1) * 8 + ri;
                        const int piece = cc + (mi >> 1);
                        uint32_t w[4];
                        ldmatrix_x4_trans(svb + C::swz(row, piece), w[0], w[1], w[2], w[3]);
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const uint32_t lo = __byte_perm(w[2 * u], 0u, 0x3120u);       // keys 0..7
                            const uint32_t hi = __byte_perm(w[2 * u + 1], 0u, 0x3120u);   // keys 8..15
                            const uint32_t va[4] = {e4m3x2_to_f16x2(lo), e4m3x2_to_f16x2(lo >> 16),
                                                    e4m3x2_to_f16x2(hi), e4m3x2_to_f16x2(hi >> 16)};
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) mma_f16_16816(o[cc + u][nt], va, pb[nt][0], pb[nt][1]);
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < D / 16; ++c) {
                        const int row = r0 + (mi >> 1) * 8 + ri;
                        const int col = c * 16 + (mi & 1) * 8;
                        uint32_t va[4];
                        ldmatrix_x4_trans(svb + swz_off<D>(row, col, rows), va[0], va[1], va[2], va[3]);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[c][nt], va, pb[nt][0], pb[nt][1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        if (b >= 0) flush_partial();
    }
}

// Merge for the page-stream decode: for sequence b, the partials of CTAs
// c_first .. c_last sit in slots c + b.
template <int D>
__global__ void __launch_bounds__(D)
    decode_pages_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                                const int* __restrict__ meta, int B, int Hq,
                                __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
    __shared__ float w_s[kMaxSplits];
    __shared__ float lse_s;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int bh = blockIdx.x;
    const int b = bh / Hq, h = bh % Hq;
    const int d = threadIdx.x;
    const int ppc = max(meta[B + 1], 1);
    const int pb = meta[b], pe = meta[b + 1];
    const int c0 = pb / ppc, c1 = (pe - 1) / ppc;
    const int ns = (pe > pb) ? min(c1 - c0 + 1, kMaxSplits) : 0;
    if (ns <= kCombineRegs) {
        // Few partials (the common case): every thread loads all of their LSEs and
        // its own column of each O partial at once, and forms the weights itself,
        // so the merge costs one round trip to memory.
        float ls[kCombineRegs], ov[kCombineRegs];
#pragma unroll
        for (int s = 0; s < kCombineRegs; ++s) {
            const long long slot = (long long)(c0 + s + b) * Hq + h;
            ls[s] = s < ns ? lse_part[slot] : -INFINITY;
            ov[s] = s < ns ? o_part[slot * D + d] : 0.0f;
        }
        float M = -INFINITY;
#pragma unroll
        for (int s = 0; s < kCombineRegs; ++s) M = fmaxf(M, ls[s]);
        float W = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int s = 0; s < kCombineRegs; ++s) W += __expf(ls[s] - M);
        }
        const float out_lse = (M != -INFINITY && W > 0.0f) ? M + __logf(W) : -INFINITY;
        float acc = 0.0f;
        if (out_lse != -INFINITY) {
#pragma unroll
            for (int s = 0; s < kCombineRegs; ++s) acc += __expf(ls[s] - out_lse) * ov[s];
        }
        o[(long long)bh * D + d] = __float2bfloat16_rn(acc);
        if (lse && d == 0) lse[bh] = out_lse;
        return;
    }
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        float M = -INFINITY;
        for (int s = lane; s < ns; s += 32) M = fmaxf(M, lse_part[(long long)(c0 + s + b) * Hq + h]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float W = 0.0f;
        if (M != -INFINITY)
            for (int s = lane; s < ns; s += 32) W += __expf(lse_part[(long long)(c0 + s + b) * Hq + h] - M);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
        const float out_lse = (M != -INFINITY && W > 0.0f) ? M + __logf(W) : -INFINITY;
        for (int s = lane; s < ns; s += 32)
            w_s[s] = (out_lse == -INFINITY) ? 0.0f
                                            : __expf(lse_part[(long long)(c0 + s + b) * Hq + h] - out_lse);
        if (lane == 0) lse_s = out_lse;
    }
    __syncthreads();
    float acc = 0.0f;
#pragma unroll 4
    for (int s = 0; s < ns; ++s) acc += w_s[s] * o_part[((long long)(c0 + s + b) * Hq + h) * D + d];
    o[(long long)bh * D + d] = __float2bfloat16_rn(acc);
    if (lse && d == 0) lse[bh] = lse_s;
}

// Merge of the split partials (a9): one block per (sequence, query head).
// Warp 0 reads every split's LSE at once and turns them into weights
// w_s = exp(LSE_s - LSE) in shared memory; then each thread (one per d) sums
// w_s * O_s[d] with all of its loads in flight together.

template <int D>
__global__ void __launch_bounds__(D)
    decode_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                          const int* __restrict__ seqused_k, int B, int Hq, int num_splits,
                          int tokens_per_split, int max_tokens, int window,
                          __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
    __shared__ float w_s[kMaxSplits];
    __shared__ float lse_s;
    // Launched early (programmatic dependent launch): wait here for the split grid.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int bh = blockIdx.x;
    const int b = bh / Hq;
    const int d = threadIdx.x;
    const int L = min(max(seqused_k[b], 0), max_tokens);
    const int ns = min(num_splits, dec_nsplit(L - win_first_page_key(L, window), tokens_per_split));
    const long long stride = (long long)B * Hq;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        float M = -INFINITY;
        for (int s = lane; s < ns; s += 32) M = fmaxf(M, lse_part[s * stride + bh]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float W = 0.0f;
        if (M != -INFINITY)
            for (int s = lane; s < ns; s += 32) W += __expf(lse_part[s * stride + bh] - M);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
        const float out_lse = (M != -INFINITY && W > 0.0f) ? M + __logf(W) : -INFINITY;
        for (int s = lane; s < ns; s += 32)
            w_s[s] = (out_lse == -INFINITY) ? 0.0f : __expf(lse_part[s * stride + bh] - out_lse);
        if (lane == 0) lse_s = out_lse;
    }
    __syncthreads();
    float acc = 0.0f;
#pragma unroll 8
    for (int s = 0; s < ns; ++s) acc += w_s[s] * o_part[(s * stride + bh) * D + d];
    o[(long long)bh * D + d] = __float2bfloat16_rn(acc);
    if (lse && d == 0) lse[bh] = lse_s;
}

}  // namespace attn
