// attn_api.cu -- the C ABI of libattn_b200.so (declared in include/attn_b200.h):
// argument validation, the once-per-device architecture check, a cache of TMA
// descriptors, and the kernel launches on the caller's stream.
//
// Nothing here allocates device memory, synchronises the stream or reads
// device data on the host (the lesson of "[CUDA] PagedAttention: add SM<80
// fp16 fallback via memory-efficient attention", Scratch allocation: its
// fallback pays a per-call device-to-host sync to size buffers).  TMA
// descriptors are encoded once per (pointer, shape, stride, box) and reused,
// because host-side encoding is not free ("Rope dim", review comment: tens of
// microseconds of descriptor work per call on H200).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "attn_b200.h"
#include "decode.cuh"
#include "patch.cuh"
#include "prefill.cuh"
#include "append.cuh"
#include "backward.cuh"

using namespace attn;

namespace {

// ------------------------------------------------------------------ device check
constexpr int kMaxDevices = 64;
std::atomic<int> g_dev_status[kMaxDevices];   // 0 unknown, 1 ok, else attn_status_t + 100

attn_status_t check_device_uncached(int device) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    if (prop.major != 10 || prop.minor != 0) return ATTN_ERR_NO_KERNEL_IMAGE;
    int prev = -1;
    cudaGetDevice(&prev);
    if (prev != device) cudaSetDevice(device);
    cudaFuncAttributes fa;
    const cudaError_t e = cudaFuncGetAttributes(&fa, prefill_kernel<128, false, false, false, false>);
    if (prev != device && prev >= 0) cudaSetDevice(prev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_NO_KERNEL_IMAGE;
    }
    return ATTN_OK;
}

attn_status_t current_device_ok(int* dev_out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    if (dev_out) *dev_out = dev;
    if (dev < 0 || dev >= kMaxDevices) return check_device_uncached(dev);
    int s = g_dev_status[dev].load(std::memory_order_acquire);
    if (s == 0) {
        const attn_status_t r = check_device_uncached(dev);
        s = (r == ATTN_OK) ? 1 : 100 + static_cast<int>(r);
        g_dev_status[dev].store(s, std::memory_order_release);
    }
    return s == 1 ? ATTN_OK : static_cast<attn_status_t>(s - 100);
}

int sm_count(int dev) {
    static std::atomic<int> cache[kMaxDevices];
    if (dev >= 0 && dev < kMaxDevices) {
        int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        n = 148;
    }
    if (dev >= 0 && dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// ------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// A 4-d tiled map: dims {d, head, row, batch} (innermost first), strides in bytes
// for dims 1..3, box {box_d, 1, box_rows, 1}, 128-byte swizzle, zero fill.
struct MapKey {
    const void* ptr;
    int dtype;
    int device;
    uint64_t dims[4];
    uint64_t strides[3];
    uint32_t box[4];
    bool operator==(const MapKey& o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};

struct MapEntry {
    MapKey key;
    CUtensorMap map;
    bool used;
};

constexpr int kMapCache = 128;
MapEntry g_maps[kMapCache];
int g_map_next = 0;
std::mutex g_map_mu;

attn_status_t get_map(CUtensorMap* out, const void* ptr, int dtype, const uint64_t dims[4],
                      const uint64_t strides[3], const uint32_t box[4]) {
    MapKey k;
    std::memset(&k, 0, sizeof(k));
    k.ptr = ptr;
    k.dtype = dtype;
    cudaGetDevice(&k.device);
    std::memcpy(k.dims, dims, sizeof(k.dims));
    std::memcpy(k.strides, strides, sizeof(k.strides));
    std::memcpy(k.box, box, sizeof(k.box));
    std::lock_guard<std::mutex> lock(g_map_mu);
    for (int i = 0; i < kMapCache; ++i)
        if (g_maps[i].used && g_maps[i].key == k) {
            *out = g_maps[i].map;
            return ATTN_OK;
        }
    EncodeTiledFn enc = get_encoder();
    if (!enc) return ATTN_ERR_TMA_ENCODE;
    CUtensorMap m;
    const cuuint32_t estride[4] = {1, 1, 1, 1};
    // the swizzle span is the box's row: 128 bytes, or 64 (e4m3 rows of head_dim 64)
    // (rows wider than 128 bytes: no swizzle, for row-by-row reads of whole rows)
    const uint32_t row_bytes = box[0] * (dtype == ATTN_FP8_E4M3 ? 1u : 2u);
    const CUtensorMapSwizzle swz = row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                   : row_bytes <= 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
    const CUresult r = enc(&m,
                           dtype == ATTN_FP8_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                  : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                           4, const_cast<void*>(ptr), reinterpret_cast<const cuuint64_t*>(dims),
                           reinterpret_cast<const cuuint64_t*>(strides),
                           reinterpret_cast<const cuuint32_t*>(box), estride,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return ATTN_ERR_TMA_ENCODE;
    MapEntry& e = g_maps[g_map_next];
    g_map_next = (g_map_next + 1) % kMapCache;
    e.key = k;
    e.map = m;
    e.used = true;
    *out = m;
    return ATTN_OK;
}

// ------------------------------------------------------------------ validation helpers
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int elem_bytes(int dtype) { return dtype == ATTN_FP8_E4M3 ? 1 : 2; }

inline bool dtype_ok(int dtype) { return dtype == ATTN_BF16 || dtype == ATTN_FP8_E4M3; }

float resolve_scale(float s, int head_dim) {
    return (s > 0.0f && std::isfinite(s)) ? s : 1.0f / std::sqrt(static_cast<float>(head_dim));
}

template <typename K>
attn_status_t set_smem(K kernel, int bytes) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

attn_status_t launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Launches `kernel` on `st`; with `pdl` as a programmatic dependent of the
// kernel launched before it on the stream (the kernel must griddepcontrol.wait).
template <typename... KArgs, typename... Args>
attn_status_t launch_maybe_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t st, bool pdl, Args... args) {
    if (!pdl) {
        kernel<<<grid, block, smem, st>>>(args...);
        return launch_status();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

// ------------------------------------------------------------------ prefill dispatch
template <int D, bool FP8, bool CAP, bool OQ, bool HQ = false>
attn_status_t launch_prefill_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                               const CUtensorMap& mqv, const PrefillArgs& a, long long grid,
                               cudaStream_t stream) {
    using Cfg = PrefillCfg<D, FP8, HQ>;
    static std::atomic<uint64_t> attr_mask{0};   // one bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_mask.load() & bit)) {
        const attn_status_t s = set_smem(prefill_kernel<D, FP8, CAP, OQ, HQ>, Cfg::SMEM_BYTES);
        if (s != ATTN_OK) return s;
        attr_mask.fetch_or(bit);
    }
    prefill_kernel<D, FP8, CAP, OQ, HQ><<<static_cast<unsigned>(grid), kPrefillThreads, Cfg::SMEM_BYTES, stream>>>(
        mq, mk, mv, mqv, a);
    return launch_status();
}

attn_status_t launch_prefill(int D, int dtype, const CUtensorMap& mq, const CUtensorMap& mk,
                             const CUtensorMap& mv, const PrefillArgs& a, long long grid,
                             cudaStream_t stream, const CUtensorMap* mqv = nullptr) {
    if (grid <= 0) return ATTN_OK;
    if (grid >= (1LL << 31)) return ATTN_ERR_UNSUPPORTED;
    const bool cap = a.softcap > 0.0f;
    if (mqv) {
        // the Qv score term (bf16)
        if (dtype == ATTN_BF16 && D == 128)
            return cap ? launch_prefill_t<128, false, true, false, true>(mq, mk, mv, *mqv, a, grid, stream)
                       : launch_prefill_t<128, false, false, false, true>(mq, mk, mv, *mqv, a, grid, stream);
        if (dtype == ATTN_BF16 && D == 64)
            return cap ? launch_prefill_t<64, false, true, false, true>(mq, mk, mv, *mqv, a, grid, stream)
                       : launch_prefill_t<64, false, false, false, true>(mq, mk, mv, *mqv, a, grid, stream);
        return ATTN_ERR_UNSUPPORTED;
    }
    if (a.only_qv) {
        if (dtype == ATTN_BF16 && D == 128)
            return cap ? launch_prefill_t<128, false, true, true>(mq, mk, mv, mq, a, grid, stream)
                       : launch_prefill_t<128, false, false, true>(mq, mk, mv, mq, a, grid, stream);
        if (dtype == ATTN_BF16 && D == 64)
            return cap ? launch_prefill_t<64, false, true, true>(mq, mk, mv, mq, a, grid, stream)
                       : launch_prefill_t<64, false, false, true>(mq, mk, mv, mq, a, grid, stream);
        if (dtype == ATTN_FP8_E4M3 && D == 128)
            return cap ? launch_prefill_t<128, true, true, true>(mq, mk, mv, mq, a, grid, stream)
                       : launch_prefill_t<128, true, false, true>(mq, mk, mv, mq, a, grid, stream);
        if (dtype == ATTN_FP8_E4M3 && D == 64)
            return cap ? launch_prefill_t<64, true, true, true>(mq, mk, mv, mq, a, grid, stream)
                       : launch_prefill_t<64, true, false, true>(mq, mk, mv, mq, a, grid, stream);
        return ATTN_ERR_UNSUPPORTED;
    }
    if (dtype == ATTN_BF16 && D == 128)
        return cap ? launch_prefill_t<128, false, true, false>(mq, mk, mv, mq, a, grid, stream)
                   : launch_prefill_t<128, false, false, false>(mq, mk, mv, mq, a, grid, stream);
    if (dtype == ATTN_BF16 && D == 64)
        return cap ? launch_prefill_t<64, false, true, false>(mq, mk, mv, mq, a, grid, stream)
                   : launch_prefill_t<64, false, false, false>(mq, mk, mv, mq, a, grid, stream);
    if (dtype == ATTN_FP8_E4M3 && D == 128)
        return cap ? launch_prefill_t<128, true, true, false>(mq, mk, mv, mq, a, grid, stream)
                   : launch_prefill_t<128, true, false, false>(mq, mk, mv, mq, a, grid, stream);
    if (dtype == ATTN_FP8_E4M3 && D == 64)
        return cap ? launch_prefill_t<64, true, true, false>(mq, mk, mv, mq, a, grid, stream)
                   : launch_prefill_t<64, true, false, false>(mq, mk, mv, mq, a, grid, stream);
    return ATTN_ERR_UNSUPPORTED;
}

void unit_grid(PrefillArgs& a, int max_seqlen_q, long long* grid) {
    const int nqt = (max_seqlen_q + kBM - 1) / kBM;
    a.pair_heads = (a.group % 2 == 0) ? 1 : 0;
    a.NH = a.pair_heads ? a.Hq / 2 : a.Hq;
    a.NQ = a.pair_heads ? nqt : (nqt + 1) / 2;
    *grid = static_cast<long long>(a.NQ) * a.B * a.NH;
}

// Stage-ring depth and CTAs per SM for the decode kernel: two CTAs per SM
// when at least two 64-key stages fit in half of the SM's shared memory,
// otherwise one CTA with as many stages as fit.
template <int D>
bool decode_geometry(int G, int B, int* ns_out, int* ctas_per_sm, int* smem_out, bool vonly) {
    using Cfg = DecodeCfg<D>;
    const int half = (228 * 1024 - 2 * 1024) / 2;
    const int whole = 227 * 1024;
    const int max_ns = vonly ? 32 : 16;     // V-only stages are half as large: twice as many
    for (int per_sm : {2, 1}) {
        const int cap = per_sm == 2 ? half : whole;
        int ns = 0;
        while (ns < max_ns && Cfg::smem_bytes(G, B, ns + 1, vonly) <= cap) ++ns;
        if (ns >= 2) {
            *ns_out = ns;
            *ctas_per_sm = per_sm;
            *smem_out = Cfg::smem_bytes(G, B, ns, vonly);
            return true;
        }
    }
    return false;
}

template <int D>
attn_status_t launch_decode(const CUtensorMap& mk, const CUtensorMap& mv, DecodeArgs a,
                            int sms, long long items_max, cudaStream_t st, const int32_t* seqused_k,
                            int max_tokens, bool pdl = false) {
    static std::atomic<uint64_t> attr_mask{0};   // one bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_mask.load() & bit)) {
        const attn_status_t s = set_smem(decode_split_kernel<D>, 227 * 1024);
        if (s != ATTN_OK) return s;
        attr_mask.fetch_or(bit);
    }
    int ns = 0, per_sm = 0, smem = 0;
    if (!decode_geometry<D>(a.group, a.B, &ns, &per_sm, &smem, a.only_qv != 0)) return ATTN_ERR_UNSUPPORTED;
    a.nstages = ns;
    const int grid = (int)std::min<long long>((long long)sms * per_sm, std::max<long long>(items_max, 1));
    attn_status_t s = launch_maybe_pdl(decode_split_kernel<D>, dim3(grid), dim3(kDecThreads), smem, st,
                                       pdl, mk, mv, a);
    if (s != ATTN_OK || a.direct) return s;
    // The combine kernel is launched as a programmatic dependent of the split
    // kernel: it is scheduled while the split grid runs and waits on the grid
    // dependency before reading the partials.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B * a.Hq);
    cfg.blockDim = dim3(D);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, (const float*)a.o_part,
                           (const float*)a.lse_part, (const int*)seqused_k, a.B, a.Hq, a.num_splits,
                           a.tokens_per_split, max_tokens, a.window, a.o, a.lse) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

// One CTA waits on an mbarrier that nothing ever arrives on, bounded by
// limit_ns: the wait expires, records kErrSelftestWait in the device error word
// and the kernel returns (the failure-detection path of every kernel here,
// made to run out on purpose).
__global__ void wait_expiry_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_for(&bar, 0, kErrSelftestWait, limit_ns);
    __syncthreads();
}

// ------------------------------------------------------------------ allocation-free decode
// Fixed device scratch for attn_decode_paged_noalloc.  Every device that loads
// this library holds these bytes until the process exits.  Host code must not
// pass the symbol itself to a kernel (on the host it is only a stand-in for the
// device object); the device address is looked up once per device below.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
std::atomic<void*> g_noalloc_addr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch on the current device, resolved on first use
// (with that device current) and cached.  Returns nullptr on failure.
void* noalloc_scratch_address(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    void* p = g_noalloc_addr[dev].load(std::memory_order_acquire);
    if (p) return p;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    p = g_noalloc_addr[dev].load(std::memory_order_acquire);
    if (p) return p;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return nullptr;
    }
    g_noalloc_addr[dev].store(p, std::memory_order_release);
    return p;
}

template <int D, bool FP8, int NT, bool HQ = false>
attn_status_t launch_decode_pages(const CUtensorMap& mk, const CUtensorMap& mv, const DecodePagesArgs& a,
                                  int grid, cudaStream_t st, __nv_bfloat16* o, float* lse,
                                  bool pdl = false) {
    static std::atomic<uint64_t> attr_mask{0};   // one bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_mask.load() & bit)) {
        const attn_status_t s = set_smem(decode_pages_kernel<D, FP8, NT, HQ>, 227 * 1024);
        if (s != ATTN_OK) return s;
        attr_mask.fetch_or(bit);
    }
    const int smem = DecodePagesCfg<D, FP8>::smem_bytes(a.Hkv, a.B, a.nstages, a.only_qv != 0);
    attn_status_t s = launch_maybe_pdl(decode_pages_kernel<D, FP8, NT, HQ>, dim3(grid), dim3(32 * (a.Hkv + 1)),
                                       smem, st, pdl, mk, mv, a);
    if (s != ATTN_OK) return s;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B * a.Hq);
    cfg.blockDim = dim3(D);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_pages_combine_kernel<D>, (const float*)a.o_part,
                           (const float*)a.lse_part, (const int*)a.meta, a.B, a.Hq, o, lse) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

// Backward: Delta, then the dK/dV and the dQ kernels, on one stream.
template <int D>
attn_status_t launch_backward(const CUtensorMap& mq, const CUtensorMap& mdo, const CUtensorMap& mk,
                              const CUtensorMap& mv, const BwdArgs& a, const void* o,
                              const void* dout, float* delta, int sms, cudaStream_t st) {
    using Cfg = BwdCfg<D>;
    static std::atomic<uint64_t> attr_mask{0};   // one bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_mask.load() & bit)) {
        attn_status_t s = set_smem(bwd_dkdv_kernel<D>, Cfg::SMEM_A);
        if (s == ATTN_OK) s = set_smem(bwd_dq_kernel<D>, Cfg::SMEM_B);
        if (s != ATTN_OK) return s;
        attr_mask.fetch_or(bit);
    }
    const long long rows = (long long)a.total_q * a.Hq;
    const int dgrid = (int)std::max<long long>(1, std::min<long long>((rows + 7) / 8, (long long)sms * 32));
    bwd_delta_kernel<D><<<dgrid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(o),
                                                static_cast<const __nv_bfloat16*>(dout), delta,
                                                a.total_q, a.Hq);
    attn_status_t s = launch_status();
    if (s != ATTN_OK) return s;
    const long long g1 = (long long)a.nkt * a.B * a.Hkv;
    const long long g2 = (long long)a.nqt * a.B * a.Hq;
    if (g1 >= (1LL << 31) || g2 >= (1LL << 31)) return ATTN_ERR_UNSUPPORTED;
    if (g1 > 0) {
        bwd_dkdv_kernel<D><<<(unsigned)g1, kBwdThreads, Cfg::SMEM_A, st>>>(mq, mdo, mk, mv, a);
        if ((s = launch_status()) != ATTN_OK) return s;
    }
    if (g2 > 0) {
        bwd_dq_kernel<D><<<(unsigned)g2, kBwdThreads, Cfg::SMEM_B, st>>>(mq, mdo, mk, mv, a);
        if ((s = launch_status()) != ATTN_OK) return s;
    }
    return ATTN_OK;
}

}  // namespace

// ==================================================================== C ABI
template <int D>
static attn_status_t launch_patch_stream(const PatchMaps& maps, const PatchArgs& pa, int n_hg, int n_rg,
                                         cudaStream_t st) {
    static std::atomic<uint64_t> attr_mask{0};   // one bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_mask.load() & bit)) {
        const attn_status_t s = set_smem(patch_stream_kernel<D>, patch_stream_smem_bytes());
        if (s != ATTN_OK) return s;
        // kPsCtas CTAs share an SM: ask for the largest shared-memory carveout (a hint)
        if (cudaFuncSetAttribute(patch_stream_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            cudaGetLastError();
        attr_mask.fetch_or(bit);
    }
    patch_stream_kernel<D><<<(unsigned)(n_hg * n_rg), kPsThreads, patch_stream_smem_bytes(), st>>>(maps, pa, n_hg);
    return launch_status();
}

extern "C" {

const char* attn_status_string(attn_status_t s) {
    switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case ATTN_ERR_NO_KERNEL_IMAGE: return "device is not sm_100 (B200) or the kernel image does not load";
    case ATTN_ERR_TMA_ENCODE: return "TMA descriptor encoding failed";
    case ATTN_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case ATTN_ERR_CUDA: return "CUDA runtime error";
    case ATTN_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded wait";
    case ATTN_ERR_SCRATCH_LIMIT: return "request needs more than the library's fixed scratch (8 MiB)";
    case ATTN_ERR_DEVICE_RANGE: return "a kernel met an index outside its buffers (block table entry or append position)";
    default: return "unknown status";
    }
}

attn_status_t attn_check_device(int device) {
    int n = 0;
    if (cudaGetDeviceCount(&n) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    if (device < 0 || device >= n) return ATTN_ERR_INVALID_ARG;
    return check_device_uncached(device);
}

attn_status_t attn_device_error(int* code_out, attn_stream_t stream) {
    if (!code_out) return ATTN_ERR_INVALID_ARG;
    const attn_status_t dv = current_device_ok(nullptr);
    if (dv != ATTN_OK) return dv;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int wait_code = 0, data_code = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbolAsync(&wait_code, g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                  st) != cudaSuccess ||
        cudaMemcpyFromSymbolAsync(&data_code, g_data_error, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                  st) != cudaSuccess ||
        cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaMemcpyToSymbolAsync(g_data_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    if (wait_code != 0) {
        *code_out = wait_code;
        return ATTN_ERR_DEVICE_TIMEOUT;
    }
    *code_out = data_code;
    return data_code == 0 ? ATTN_OK : ATTN_ERR_DEVICE_RANGE;
}

attn_status_t attn_selftest_wait_expiry(long long limit_ns, attn_stream_t stream) {
    if (limit_ns < 0 || limit_ns > 10000000000LL) return ATTN_ERR_INVALID_ARG;
    const attn_status_t dvs = current_device_ok(nullptr);
    if (dvs != ATTN_OK) return dvs;
    wait_expiry_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<unsigned long long>(limit_ns));
    return launch_status();
}

// Sliding window and softcap: a window is defined for the causal mask only
// (any negative window_left means none); softcap must be finite and >= 0.
static attn_status_t check_score_mods(int mask, int window_left, float softcap) {
    if (!(softcap >= 0.0f) || !std::isfinite(softcap)) return ATTN_ERR_INVALID_ARG;
    if (window_left >= 0 && mask != ATTN_MASK_CAUSAL) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

// Keys a decode query can touch: the whole cache span, or its window plus the
// part of the first page before it.
static int decode_span(int max_tokens, int window) {
    if (window < 0) return max_tokens;
    return (int)std::min<long long>(max_tokens, (long long)window + 1 + kPageRows);
}

attn_status_t attn_fwd_dense(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int Lq, int Lk, int Hq, int Hkv, int D,
                             const int64_t* sq, const int64_t* sk, const int64_t* sv,
                             float softmax_scale, int mask, int window_left, float softcap,
                             int dtype, const float* dq, const float* dk, const float* dv,
                             attn_stream_t stream) {
    if (!q || !k || !v || !o || !sq || !sk || !sv) return ATTN_ERR_INVALID_ARG;
    if (B < 0 || Lq < 0 || Lk < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return ATTN_ERR_INVALID_ARG;
    if (mask != ATTN_MASK_NONE && mask != ATTN_MASK_CAUSAL) {
        return mask == ATTN_MASK_PATCH ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
    }
    {
        const attn_status_t ms = check_score_mods(mask, window_left, softcap);
        if (ms != ATTN_OK) return ms;
    }
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (dtype == ATTN_FP8_E4M3 && (!dq || !dk || !dv)) return ATTN_ERR_INVALID_ARG;
    const int E = elem_bytes(dtype);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i) {
        if (sq[i] <= 0 || sk[i] <= 0 || sv[i] <= 0) return ATTN_ERR_INVALID_ARG;
        if ((sq[i] * E) % 16 || (sk[i] * E) % 16 || (sv[i] * E) % 16) return ATTN_ERR_INVALID_ARG;
    }
    if (sq[2] < D || sk[2] < D || sv[2] < D) return ATTN_ERR_INVALID_ARG;
    if (Lq > (1 << 30) || Lk > (1 << 30)) return ATTN_ERR_UNSUPPORTED;
    const attn_status_t dvs = current_device_ok(nullptr);
    if (dvs != ATTN_OK) return dvs;
    if (B == 0 || Lq == 0) return ATTN_OK;

    const int chunk = std::min(128 / E, D);   // one swizzle column of a row
    CUtensorMap mq, mk, mv;
    const uint64_t dq4[4] = {(uint64_t)D, (uint64_t)Hq, (uint64_t)Lq, (uint64_t)B};
    const uint64_t sq3[3] = {(uint64_t)(sq[2] * E), (uint64_t)(sq[1] * E), (uint64_t)(sq[0] * E)};
    const uint32_t bq[4] = {(uint32_t)chunk, 1, (uint32_t)kBM, 1};
    const uint64_t dk4[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)std::max(Lk, 1), (uint64_t)B};
    const uint64_t sk3[3] = {(uint64_t)(sk[2] * E), (uint64_t)(sk[1] * E), (uint64_t)(sk[0] * E)};
    const uint64_t sv3[3] = {(uint64_t)(sv[2] * E), (uint64_t)(sv[1] * E), (uint64_t)(sv[0] * E)};
    const uint32_t bkv[4] = {(uint32_t)chunk, 1, (uint32_t)kBN, 1};
    attn_status_t s;
    if ((s = get_map(&mq, q, dtype, dq4, sq3, bq)) != ATTN_OK) return s;
    if ((s = get_map(&mk, k, dtype, dk4, sk3, bkv)) != ATTN_OK) return s;
    if ((s = get_map(&mv, v, dtype, dk4, sv3, bkv)) != ATTN_OK) return s;

    PrefillArgs a;
    std::memset(&a, 0, sizeof(a));
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.group = Hq / Hkv;
    a.mask = mask;
    a.window = window_left < 0 ? -1 : window_left;
    a.softcap = softcap;
    a.varlen = 0;
    a.paged = 0;
    a.Lq = Lq;
    a.Lk = Lk;
    a.scale = resolve_scale(softmax_scale, D);
    a.descale_q = dq;
    a.descale_k = dk;
    a.descale_v = dv;
    a.o = static_cast<__nv_bfloat16*>(o);
    a.lse = lse;
    a.o_stride_row = (long long)Hq * D;
    a.o_stride_b = (long long)Lq * Hq * D;
    a.lse_stride_h = Lq;
    a.lse_stride_b = (long long)Hq * Lq;
    long long grid;
    unit_grid(a, Lq, &grid);
    return launch_prefill(D, dtype, mq, mk, mv, a, grid, static_cast<cudaStream_t>(stream));
}

// The varlen / paged forward; with `only_qv` the score is q . v (k_cache is the
// value store, and the kernel reads the value tile as the score GEMM's operand).
static attn_status_t fwd_varlen_paged_impl(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
    int max_blocks_per_seq, int num_blocks, int block_size, const int32_t* cu_seqlens_q,
    const int32_t* cu_seqlens_k, const int32_t* seqused_k, int B, int total_q, int total_k,
    int max_seqlen_q, int Hq, int Hkv, int D, float softmax_scale, int mask,
    const int32_t* patch_kv_range, int window_left, float softcap, int dtype, const float* dq,
    const float* dk, const float* dv, void* o, float* lse, attn_stream_t stream, int only_qv,
    const void* qv = nullptr) {
    if (!q || !k_cache || !v_cache || !o || !cu_seqlens_q) return ATTN_ERR_INVALID_ARG;
    if (B < 0 || total_q < 0 || max_seqlen_q < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0)
        return ATTN_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return ATTN_ERR_INVALID_ARG;
    if (mask < ATTN_MASK_NONE || mask > ATTN_MASK_PATCH) return ATTN_ERR_INVALID_ARG;
    if (mask == ATTN_MASK_PATCH && !patch_kv_range) return ATTN_ERR_INVALID_ARG;
    {
        const attn_status_t ms = check_score_mods(mask, window_left, softcap);
        if (ms != ATTN_OK) return ms;
    }
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (qv && (dtype != ATTN_BF16 || only_qv)) return ATTN_ERR_UNSUPPORTED;
    if (dtype == ATTN_FP8_E4M3 && (!dq || !dk || !dv)) return ATTN_ERR_INVALID_ARG;
    const bool paged = block_table != nullptr;
    if (paged) {
        if (block_size != kPageRows) return ATTN_ERR_UNSUPPORTED;
        if (num_blocks <= 0 || max_blocks_per_seq <= 0) return ATTN_ERR_INVALID_ARG;
        if ((long long)num_blocks * block_size >= (1LL << 31)) return ATTN_ERR_UNSUPPORTED;
        if (!seqused_k && !cu_seqlens_k) return ATTN_ERR_INVALID_ARG;
    } else {
        if (!cu_seqlens_k || total_k < 0) return ATTN_ERR_INVALID_ARG;
    }
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
        return ATTN_ERR_INVALID_ARG;
    if (qv && !aligned16(qv)) return ATTN_ERR_INVALID_ARG;
    const int E = elem_bytes(dtype);
    if ((D * E) % 16) return ATTN_ERR_INVALID_ARG;
    const attn_status_t dvs = current_device_ok(nullptr);
    if (dvs != ATTN_OK) return dvs;
    if (B == 0 || total_q == 0 || max_seqlen_q == 0) return ATTN_OK;

    const int chunk = std::min(128 / E, D);   // one swizzle column of a row
    CUtensorMap mq, mk, mv;
    const uint64_t rowq = (uint64_t)Hq * D * E;
    const uint64_t dq4[4] = {(uint64_t)D, (uint64_t)Hq, (uint64_t)total_q, 1};
    const uint64_t sq3[3] = {(uint64_t)D * E, rowq, rowq * (uint64_t)total_q};
    const uint32_t bq[4] = {(uint32_t)chunk, 1, (uint32_t)kBM, 1};
    const uint64_t rowk = (uint64_t)Hkv * D * E;
    const uint64_t nrows = paged ? (uint64_t)num_blocks * block_size : (uint64_t)std::max(total_k, 1);
    const uint64_t dk4[4] = {(uint64_t)D, (uint64_t)Hkv, nrows, 1};
    const uint64_t sk3[3] = {(uint64_t)D * E, rowk, rowk * nrows};
    const uint32_t bkv[4] = {(uint32_t)chunk, 1, (uint32_t)(paged ? kPageRows : kBN), 1};
    attn_status_t s;
    if ((s = get_map(&mq, q, dtype, dq4, sq3, bq)) != ATTN_OK) return s;
    CUtensorMap mqv;
    if (qv && (s = get_map(&mqv, qv, dtype, dq4, sq3, bq)) != ATTN_OK) return s;
    if ((s = get_map(&mv, v_cache, dtype, dk4, sk3, bkv)) != ATTN_OK) return s;
    if (only_qv) mk = mv;   // no key store: its map is never used
    else if ((s = get_map(&mk, k_cache, dtype, dk4, sk3, bkv)) != ATTN_OK) return s;

    PrefillArgs a;
    std::memset(&a, 0, sizeof(a));
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.group = Hq / Hkv;
    a.mask = mask;
    a.window = window_left < 0 ? -1 : window_left;
    a.softcap = softcap;
    a.varlen = 1;
    a.paged = paged ? 1 : 0;
    a.only_qv = only_qv ? 1 : 0;
    a.cu_q = cu_seqlens_q;
    a.cu_k = cu_seqlens_k;
    a.seqused_k = seqused_k;
    a.block_table = block_table;
    a.max_blocks = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.patch = patch_kv_range;
    a.scale = resolve_scale(softmax_scale, D);
    a.descale_q = dq;
    a.descale_k = dk;
    a.descale_v = dv;
    a.o = static_cast<__nv_bfloat16*>(o);
    a.lse = lse;
    a.o_stride_row = (long long)Hq * D;
    a.o_stride_b = 0;
    a.lse_stride_h = total_q;
    a.lse_stride_b = 0;
    long long grid;
    unit_grid(a, max_seqlen_q, &grid);
    return launch_prefill(D, dtype, mq, mk, mv, a, grid, static_cast<cudaStream_t>(stream),
                          qv ? &mqv : nullptr);
}

attn_status_t attn_fwd_varlen_paged(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
    int max_blocks_per_seq, int num_blocks, int block_size, const int32_t* cu_seqlens_q,
    const int32_t* cu_seqlens_k, const int32_t* seqused_k, int B, int total_q, int total_k,
    int max_seqlen_q, int Hq, int Hkv, int D, float softmax_scale, int mask,
    const int32_t* patch_kv_range, int window_left, float softcap, int dtype, const float* dq,
    const float* dk, const float* dv, void* o, float* lse, void* workspace,
    size_t workspace_bytes, attn_stream_t stream) {
    (void)workspace;
    (void)workspace_bytes;
    return fwd_varlen_paged_impl(q, k_cache, v_cache, block_table, max_blocks_per_seq, num_blocks,
                                 block_size, cu_seqlens_q, cu_seqlens_k, seqused_k, B, total_q,
                                 total_k, max_seqlen_q, Hq, Hkv, D, softmax_scale, mask,
                                 patch_kv_range, window_left, softcap, dtype, dq, dk, dv, o, lse,
                                 stream, 0);
}

attn_status_t attn_fwd_varlen_paged_qv(
    const void* q, const void* qv, const void* k_cache, const void* v_cache,
    const int32_t* block_table, int max_blocks_per_seq, int num_blocks, int block_size,
    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const int32_t* seqused_k, int B,
    int total_q, int total_k, int max_seqlen_q, int Hq, int Hkv, int D, float softmax_scale,
    int mask, const int32_t* patch_kv_range, int window_left, float softcap, int dtype, void* o,
    float* lse, attn_stream_t stream) {
    if (!qv) return ATTN_ERR_INVALID_ARG;
    return fwd_varlen_paged_impl(q, k_cache, v_cache, block_table, max_blocks_per_seq, num_blocks,
                                 block_size, cu_seqlens_q, cu_seqlens_k, seqused_k, B, total_q,
                                 total_k, max_seqlen_q, Hq, Hkv, D, softmax_scale, mask,
                                 patch_kv_range, window_left, softcap, dtype, nullptr, nullptr,
                                 nullptr, o, lse, stream, 0, qv);
}

attn_status_t attn_fwd_varlen_paged_only_qv(
    const void* qv, const void* v_cache, const int32_t* block_table, int max_blocks_per_seq,
    int num_blocks, int block_size, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
    const int32_t* seqused_k, int B, int total_q, int total_k, int max_seqlen_q, int Hq, int Hkv,
    int D, float softmax_scale, int mask, const int32_t* patch_kv_range, int window_left,
    float softcap, int dtype, const float* descale_qv, const float* descale_v, void* o,
    float* lse, attn_stream_t stream) {
    // the value codes stand in the key slot, so the score's key descale is the value one
    return fwd_varlen_paged_impl(qv, v_cache, v_cache, block_table, max_blocks_per_seq, num_blocks,
                                 block_size, cu_seqlens_q, cu_seqlens_k, seqused_k, B, total_q,
                                 total_k, max_seqlen_q, Hq, Hkv, D, softmax_scale, mask,
                                 patch_kv_range, window_left, softcap, dtype, descale_qv, descale_v,
                                 descale_v, o, lse, stream, 1);
}

attn_status_t attn_fwd_patch(const void* q, const void* k, const void* v,
                             const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                             const int32_t* patch_kv_range, int B, int total_q, int total_k,
                             int max_seqlen_q, int Hq, int Hkv, int D, float softmax_scale,
                             int max_interval, int dtype, const float* dq, const float* dk,
                             const float* dv, void* o, float* lse, attn_stream_t stream) {
    if (max_interval < 0) return ATTN_ERR_INVALID_ARG;
    // Long intervals, or fp8: the tiled tensor-core kernel with the patch mask.
    if (max_interval > kPatchShortMax || dtype != ATTN_BF16)
        return fwd_varlen_paged_impl(q, k, v, nullptr, 0, 0, 0, cu_seqlens_q, cu_seqlens_k, nullptr, B,
                                     total_q, total_k, max_seqlen_q, Hq, Hkv, D, softmax_scale,
                                     ATTN_MASK_PATCH, patch_kv_range, -1, 0.0f, dtype, dq, dk, dv, o,
                                     lse, stream, 0);
    if (!q || !k || !v || !o || !cu_seqlens_q || !cu_seqlens_k || !patch_kv_range) return ATTN_ERR_INVALID_ARG;
    if (B < 0 || total_q < 0 || total_k < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0)
        return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    int dev = 0;
    const attn_status_t dvs = current_device_ok(&dev);
    if (dvs != ATTN_OK) return dvs;
    if (B == 0 || total_q == 0) return ATTN_OK;
    PatchArgs pa;
    std::memset(&pa, 0, sizeof(pa));
    pa.q = static_cast<const __nv_bfloat16*>(q);
    pa.k = static_cast<const __nv_bfloat16*>(k);
    pa.v = static_cast<const __nv_bfloat16*>(v);
    pa.cu_q = cu_seqlens_q;
    pa.cu_k = cu_seqlens_k;
    pa.range = patch_kv_range;
    pa.B = B;
    pa.Hq = Hq;
    pa.Hkv = Hkv;
    pa.group = Hq / Hkv;
    pa.total_q = total_q;
    pa.total_k = total_k;
    pa.scale = resolve_scale(softmax_scale, D);
    pa.o = static_cast<__nv_bfloat16*>(o);
    pa.lse = lse;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // no grouped heads: heads in 512-byte slices, each query's rows streamed through
    // shared memory by bulk copies
    if (Hq == Hkv && Hq % (256 / D) == 0) {
        const int n_hg = Hq / (256 / D);
        const int n_rg = std::max(1, kPsCtas * sm_count(dev) / n_hg);
        PatchMaps maps;
        const uint64_t C = (uint64_t)Hq * D;          // elements of a row (Hq == Hkv)
        const uint64_t dq4[4] = {C, (uint64_t)total_q, 1, 1};
        const uint64_t sq3[3] = {C * 2, C * 2 * (uint64_t)total_q, C * 2 * (uint64_t)total_q};
        const uint32_t bq4[4] = {256, (uint32_t)kPsQ, 1, 1};
        attn_status_t s;
        if ((s = get_map(&maps.q, q, ATTN_BF16, dq4, sq3, bq4)) != ATTN_OK) return s;
        const uint64_t nk = (uint64_t)std::max(total_k, 1);
        const uint64_t dk4[4] = {C, nk, 1, 1};
        const uint64_t sk3[3] = {C * 2, C * 2 * nk, C * 2 * nk};
        for (int pc = 0; pc < 4; ++pc) {
            const uint32_t bk4[4] = {256, (uint32_t)(8 << pc), 1, 1};
            if ((s = get_map(&maps.k[pc], k, ATTN_BF16, dk4, sk3, bk4)) != ATTN_OK) return s;
            if ((s = get_map(&maps.v[pc], v, ATTN_BF16, dk4, sk3, bk4)) != ATTN_OK) return s;
        }
        return D == 128 ? launch_patch_stream<128>(maps, pa, n_hg, n_rg, st)
                        : launch_patch_stream<64>(maps, pa, n_hg, n_rg, st);
    }
    // a warp per query (all heads) where a lane's share of the heads' columns is small;
    // otherwise a warp per (query, head)
    const long long qblocks = std::min<long long>((total_q + kPatchWarps - 1) / kPatchWarps,
                                                  (long long)sm_count(dev) * 16);
    if (Hq == 16 && D == 64) {
        patch_query_kernel<64, 16><<<(unsigned)qblocks, 32 * kPatchWarps, 0, st>>>(pa);
        return launch_status();
    }
    if (Hq == 8 && D == 128) {
        patch_query_kernel<128, 8><<<(unsigned)qblocks, 32 * kPatchWarps, 0, st>>>(pa);
        return launch_status();
    }
    if (Hq == 8 && D == 64) {
        patch_query_kernel<64, 8><<<(unsigned)qblocks, 32 * kPatchWarps, 0, st>>>(pa);
        return launch_status();
    }
    const long long items = (long long)total_q * Hq;
    const long long blocks = std::min<long long>((items + kPatchWarps - 1) / kPatchWarps, (long long)sm_count(dev) * 8);
    if (D == 128) patch_kernel<128><<<(unsigned)blocks, 32 * kPatchWarps, 0, st>>>(pa);
    else patch_kernel<64><<<(unsigned)blocks, 32 * kPatchWarps, 0, st>>>(pa);
    return launch_status();
}

// Split-KV heuristic: enough CTAs to fill every SM about twice with sequences
// of the maximum length, and at most ~512 keys per split for balance across
// ragged lengths; tokens per split is a multiple of the 64-key stage.
static void decode_splits(int B, int Hkv, int max_tokens, int requested, int* num_splits,
                          int* tps) {
    max_tokens = std::max(max_tokens, 1);
    int ns;
    if (requested > 0) {
        ns = requested;
    } else {
        const int for_balance = (max_tokens + 511) / 512;
        const int for_fill = (2 * 148 * 2 + B * Hkv - 1) / std::max(B * Hkv, 1);
        ns = std::max(for_balance, for_fill);
    }
    ns = std::max(1, std::min(ns, (max_tokens + kDecStageTok - 1) / kDecStageTok));
    ns = std::min(ns, kMaxSplits);
    int t = (max_tokens + ns - 1) / ns;
    t = (t + kDecStageTok - 1) / kDecStageTok * kDecStageTok;
    *tps = t;
    *num_splits = (max_tokens + t - 1) / t;
}

static int decode_pages_stages(int D, int Hkv, int B, bool vonly = false, bool fp8 = false) {
    const int cap = 227 * 1024;
    const int max_ns = (vonly || fp8) ? 16 : 8;   // V-only or e4m3 stages are half as large
    int ns = 0;
    if (fp8 && D == 128)
        while (ns < max_ns && DecodePagesCfg<128, true>::smem_bytes(Hkv, B, ns + 1, vonly) <= cap) ++ns;
    else if (fp8)
        while (ns < max_ns && DecodePagesCfg<64, true>::smem_bytes(Hkv, B, ns + 1, vonly) <= cap) ++ns;
    else if (D == 128)
        while (ns < max_ns && DecodePagesCfg<128>::smem_bytes(Hkv, B, ns + 1, vonly) <= cap) ++ns;
    else
        while (ns < max_ns && DecodePagesCfg<64>::smem_bytes(Hkv, B, ns + 1, vonly) <= cap) ++ns;
    return ns;
}

// The page-stream kernel serves the automatic split choice whenever a whole
// page of all KV heads fits a stage twice over; an explicit num_splits selects
// the per-(sequence, split, KV head) kernel.
static bool use_page_stream(int B, int Hq, int Hkv, int D, int num_splits) {
    return num_splits <= 0 && Hkv <= kPgMaxWarps && Hq / Hkv <= kDecRows && B <= kDecMaxSeqs &&
           decode_pages_stages(D, Hkv, B) >= 2;
}

static int current_sm_count_or(int fallback) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return fallback;
    }
    return n;
}

size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int D, int max_blocks_per_seq,
                                  int block_size, int num_splits) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_blocks_per_seq <= 0 || block_size <= 0)
        return 0;
    if (use_page_stream(B, Hq, Hkv, D, num_splits)) {
        // partial slots (grid + B), their LSEs, then the page prefix table
        const size_t slots = (size_t)current_sm_count_or(1024) + B;
        return slots * Hq * (D + 1) * sizeof(float) + (size_t)(B + 2) * sizeof(int) + 64;
    }
    int ns, tps;
    decode_splits(B, Hkv, max_blocks_per_seq * block_size, num_splits, &ns, &tps);
    if (ns <= 1) return 16;
    return (size_t)ns * B * Hq * (D + 1) * sizeof(float) + 16;
}

// The paged decode; with `pdl` its first kernel is launched as a programmatic
// dependent of the kernel launched before it on the stream (a KV append).
static attn_status_t decode_paged_impl(const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_table, int max_blocks_per_seq,
                                       int num_blocks, int block_size, const int32_t* seqused_k,
                                       int B, int Hq, int Hkv, int D, float softmax_scale,
                                       int window_left, float softcap, int num_splits, int dtype,
                                       const float* dq, const float* dk, const float* dv, void* o,
                                       float* lse, void* workspace, size_t workspace_bytes,
                                       attn_stream_t stream, bool pdl, int only_qv = 0,
                                       const void* qv = nullptr) {
    if (!q || !k_cache || !v_cache || !block_table || !seqused_k || !o) return ATTN_ERR_INVALID_ARG;
    {
        // the query is the newest token: the window is a causal one by construction
        const attn_status_t ms = check_score_mods(ATTN_MASK_CAUSAL, window_left, softcap);
        if (ms != ATTN_OK) return ms;
    }
    const int window = window_left < 0 ? -1 : window_left;
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (num_blocks <= 0 || max_blocks_per_seq <= 0) return ATTN_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return ATTN_ERR_INVALID_ARG;
    const bool fp8 = dtype == ATTN_FP8_E4M3;
    if (fp8) {
        // e4m3 q and cache: the page-stream decode (automatic split)
        if (only_qv || qv) return ATTN_ERR_UNSUPPORTED;
        if (!dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
        if (num_splits > 0) return ATTN_ERR_UNSUPPORTED;
    }
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (block_size != kPageRows) return ATTN_ERR_UNSUPPORTED;
    if (Hq / Hkv > kDecRows) return ATTN_ERR_UNSUPPORTED;
    if (B > kDecMaxSeqs) return ATTN_ERR_UNSUPPORTED;
    if ((long long)num_blocks * block_size >= (1LL << 31)) return ATTN_ERR_UNSUPPORTED;
    if ((long long)max_blocks_per_seq * block_size >= (1LL << 30)) return ATTN_ERR_UNSUPPORTED;
    if (fp8 && !use_page_stream(B, Hq, Hkv, D, num_splits)) return ATTN_ERR_UNSUPPORTED;
    if (qv) {
        // the extra Qv score term: bf16, the page-stream decode (automatic split)
        if (dtype != ATTN_BF16 || only_qv || !use_page_stream(B, Hq, Hkv, D, num_splits))
            return ATTN_ERR_UNSUPPORTED;
        if (!aligned16(qv)) return ATTN_ERR_INVALID_ARG;
    }
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
        return ATTN_ERR_INVALID_ARG;
    int ns, tps;
    decode_splits(B, Hkv, decode_span(max_blocks_per_seq * block_size, window), num_splits, &ns, &tps);
    const size_t need = attn_decode_workspace_size(B, Hq, Hkv, D, max_blocks_per_seq, block_size,
                                                   num_splits);
    if (ns > 1 && !use_page_stream(B, Hq, Hkv, D, num_splits)) {
        if (!workspace || !aligned16(workspace)) return ATTN_ERR_INVALID_ARG;
        if (workspace_bytes < need) return ATTN_ERR_WORKSPACE_TOO_SMALL;
    }
    int dev = 0;
    const attn_status_t dvs = current_device_ok(&dev);
    if (dvs != ATTN_OK) return dvs;
    if (B == 0) return ATTN_OK;

    CUtensorMap mk, mv;
    cudaStream_t stp = static_cast<cudaStream_t>(stream);
    if (use_page_stream(B, Hq, Hkv, D, num_splits)) {
        // {d, token, head, page} view: one box = a whole page's 128-byte column
        CUtensorMap pk, pv;
        const int E = elem_bytes(dtype);
        const uint64_t rowk = (uint64_t)Hkv * D * E;
        const uint64_t pd[4] = {(uint64_t)D, (uint64_t)kPageRows, (uint64_t)Hkv, (uint64_t)num_blocks};
        const uint64_t ps[3] = {rowk, (uint64_t)D * E, rowk * kPageRows};
        const uint32_t pbox[4] = {(uint32_t)std::min(128 / E, D), (uint32_t)kPageRows, (uint32_t)Hkv, 1};
        attn_status_t s;
        if ((s = get_map(&pv, v_cache, dtype, pd, ps, pbox)) != ATTN_OK) return s;
        if (only_qv) pk = pv;   // no key store: its map is never used
        else if ((s = get_map(&pk, k_cache, dtype, pd, ps, pbox)) != ATTN_OK) return s;
        const int grid = sm_count(dev);
        const size_t slots = (size_t)grid + B;
        const size_t need_pg = slots * Hq * (D + 1) * sizeof(float) + (size_t)(B + 2) * sizeof(int);
        if (!workspace || !aligned16(workspace)) return ATTN_ERR_INVALID_ARG;
        if (workspace_bytes < need_pg) return ATTN_ERR_WORKSPACE_TOO_SMALL;
        DecodePagesArgs pa;
        std::memset(&pa, 0, sizeof(pa));
        pa.B = B;
        pa.Hq = Hq;
        pa.Hkv = Hkv;
        pa.group = Hq / Hkv;
        pa.q = q;
        pa.qv = qv;
        pa.descale_q = dq;
        pa.descale_k = dk;
        pa.descale_v = dv;
        pa.block_table = block_table;
        pa.max_blocks = max_blocks_per_seq;
        pa.num_blocks = num_blocks;
        pa.seqused_k = seqused_k;
        pa.scale = resolve_scale(softmax_scale, D);
        pa.window = window;
        pa.softcap = softcap;
        pa.o_part = static_cast<float*>(workspace);
        pa.lse_part = pa.o_part + slots * Hq * D;
        pa.meta = reinterpret_cast<int*>(pa.lse_part + slots * Hq);
        pa.nstages = decode_pages_stages(D, Hkv, B, only_qv != 0, fp8);
        pa.only_qv = only_qv ? 1 : 0;
        __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(o);
        const bool wide = pa.group > 8;          // two n-tiles of 8 query heads
        if (qv) {
            if (D == 128)
                return wide ? launch_decode_pages<128, false, 2, true>(pk, pv, pa, grid, stp, ob, lse, pdl)
                            : launch_decode_pages<128, false, 1, true>(pk, pv, pa, grid, stp, ob, lse, pdl);
            return wide ? launch_decode_pages<64, false, 2, true>(pk, pv, pa, grid, stp, ob, lse, pdl)
                        : launch_decode_pages<64, false, 1, true>(pk, pv, pa, grid, stp, ob, lse, pdl);
        }
        if (fp8 && D == 128)
            return wide ? launch_decode_pages<128, true, 2>(pk, pv, pa, grid, stp, ob, lse, pdl)
                        : launch_decode_pages<128, true, 1>(pk, pv, pa, grid, stp, ob, lse, pdl);
        if (fp8)
            return wide ? launch_decode_pages<64, true, 2>(pk, pv, pa, grid, stp, ob, lse, pdl)
                        : launch_decode_pages<64, true, 1>(pk, pv, pa, grid, stp, ob, lse, pdl);
        if (D == 128)
            return wide ? launch_decode_pages<128, false, 2>(pk, pv, pa, grid, stp, ob, lse, pdl)
                        : launch_decode_pages<128, false, 1>(pk, pv, pa, grid, stp, ob, lse, pdl);
        return wide ? launch_decode_pages<64, false, 2>(pk, pv, pa, grid, stp, ob, lse, pdl)
                    : launch_decode_pages<64, false, 1>(pk, pv, pa, grid, stp, ob, lse, pdl);
    }

    const uint64_t rowk = (uint64_t)Hkv * D * 2;
    const uint64_t nrows = (uint64_t)num_blocks * block_size;
    const uint64_t dk4[4] = {(uint64_t)D, (uint64_t)Hkv, nrows, 1};
    const uint64_t sk3[3] = {(uint64_t)D * 2, rowk, rowk * nrows};
    const uint32_t bkv[4] = {64, 1, (uint32_t)kPageRows, 1};
    attn_status_t s;
    if ((s = get_map(&mv, v_cache, ATTN_BF16, dk4, sk3, bkv)) != ATTN_OK) return s;
    if (only_qv) mk = mv;
    else if ((s = get_map(&mk, k_cache, ATTN_BF16, dk4, sk3, bkv)) != ATTN_OK) return s;

    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.group = Hq / Hkv;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.block_table = block_table;
    a.max_blocks = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.seqused_k = seqused_k;
    a.tokens_per_split = tps;
    a.num_splits = ns;
    a.scale = resolve_scale(softmax_scale, D);
    a.window = window;
    a.softcap = softcap;
    a.o = static_cast<__nv_bfloat16*>(o);
    a.lse = lse;
    a.direct = ns == 1 ? 1 : 0;
    a.only_qv = only_qv ? 1 : 0;
    if (ns > 1) {
        a.o_part = static_cast<float*>(workspace);
        a.lse_part = a.o_part + (size_t)ns * B * Hq * D;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long items_max = (long long)B * Hkv * ns;
    if (D == 128)
        s = launch_decode<128>(mk, mv, a, sm_count(dev), items_max, st, seqused_k,
                               max_blocks_per_seq * block_size, pdl);
    else
        s = launch_decode<64>(mk, mv, a, sm_count(dev), items_max, st, seqused_k,
                              max_blocks_per_seq * block_size, pdl);
    if (s != ATTN_OK) return s;
    return launch_status();
}

attn_status_t attn_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* block_table, int max_blocks_per_seq, int num_blocks,
                                int block_size, const int32_t* seqused_k, int B, int Hq, int Hkv,
                                int D, float softmax_scale, int window_left, float softcap,
                                int num_splits, int dtype, const float* dq, const float* dk,
                                const float* dv, void* o, float* lse, void* workspace,
                                size_t workspace_bytes, attn_stream_t stream) {
    return decode_paged_impl(q, k_cache, v_cache, block_table, max_blocks_per_seq, num_blocks,
                             block_size, seqused_k, B, Hq, Hkv, D, softmax_scale, window_left,
                             softcap, num_splits, dtype, dq, dk, dv, o, lse, workspace,
                             workspace_bytes, stream, false);
}

attn_status_t attn_decode_paged_qv(const void* q, const void* qv, const void* k_cache,
                                   const void* v_cache, const int32_t* block_table,
                                   int max_blocks_per_seq, int num_blocks, int block_size,
                                   const int32_t* seqused_k, int B, int Hq, int Hkv, int D,
                                   float softmax_scale, int window_left, float softcap,
                                   int num_splits, int dtype, void* o, float* lse, void* workspace,
                                   size_t workspace_bytes, attn_stream_t stream) {
    if (!qv) return ATTN_ERR_INVALID_ARG;
    return decode_paged_impl(q, k_cache, v_cache, block_table, max_blocks_per_seq, num_blocks,
                             block_size, seqused_k, B, Hq, Hkv, D, softmax_scale, window_left,
                             softcap, num_splits, dtype, nullptr, nullptr, nullptr, o, lse,
                             workspace, workspace_bytes, stream, false, 0, qv);
}

attn_status_t attn_decode_paged_only_qv(const void* qv, const void* v_cache,
                                        const int32_t* block_table, int max_blocks_per_seq,
                                        int num_blocks, int block_size, const int32_t* seqused_k,
                                        int B, int Hq, int Hkv, int D, float softmax_scale,
                                        int window_left, float softcap, int num_splits, int dtype,
                                        void* o, float* lse, void* workspace,
                                        size_t workspace_bytes, attn_stream_t stream) {
    return decode_paged_impl(qv, v_cache, v_cache, block_table, max_blocks_per_seq, num_blocks,
                             block_size, seqused_k, B, Hq, Hkv, D, softmax_scale, window_left,
                             softcap, num_splits, dtype, nullptr, nullptr, nullptr, o, lse,
                             workspace, workspace_bytes, stream, false, 1);
}

// Shared checks and launch of the KV append; `one_per_seq` means
// cu_seqlens_new is absent and each sequence gets exactly one new token.
static attn_status_t kv_append_launch(const void* k_new, const void* v_new, void* k_cache,
                                      void* v_cache, const int32_t* block_table,
                                      int max_blocks_per_seq, int num_blocks, int block_size,
                                      const int32_t* cu_seqlens_new, const int32_t* seqused_k,
                                      int32_t* seqused_k_out, int B, int total_new, int Hkv, int D,
                                      int dtype, attn_stream_t stream) {
    if (!k_new || !v_new || !k_cache || !v_cache || !block_table || !seqused_k)
        return ATTN_ERR_INVALID_ARG;
    if (B < 0 || total_new < 0 || Hkv <= 0 || D <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0)
        return ATTN_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return ATTN_ERR_INVALID_ARG;
    if (!cu_seqlens_new && total_new != B) return ATTN_ERR_INVALID_ARG;
    if (seqused_k_out && (const void*)seqused_k_out == (const void*)seqused_k) return ATTN_ERR_INVALID_ARG;
    if (block_size != kPageRows) return ATTN_ERR_UNSUPPORTED;
    const long long row_bytes = (long long)D * elem_bytes(dtype);
    if (row_bytes % 16) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
        return ATTN_ERR_INVALID_ARG;
    if ((long long)num_blocks * block_size * Hkv * row_bytes / 16 >= (1LL << 62)) return ATTN_ERR_UNSUPPORTED;
    int dev = 0;
    const attn_status_t dvs = current_device_ok(&dev);
    if (dvs != ATTN_OK) return dvs;
    if (B == 0) return ATTN_OK;
    AppendArgs a;
    std::memset(&a, 0, sizeof(a));
    a.k_new = static_cast<const uint4*>(k_new);
    a.v_new = static_cast<const uint4*>(v_new);
    a.k_cache = static_cast<uint4*>(k_cache);
    a.v_cache = static_cast<uint4*>(v_cache);
    a.block_table = block_table;
    a.max_blocks = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.cu_new = cu_seqlens_new;
    a.seqused_k = seqused_k;
    a.seqused_k_out = seqused_k_out;
    a.B = B;
    a.total_new = total_new;
    a.pieces_per_token = (int)((long long)Hkv * row_bytes / 16);
    const int warps_per_block = kAppendThreads / 32;
    const long long want = std::max<long long>((long long)std::max(total_new, B) + warps_per_block - 1,
                                               warps_per_block) / warps_per_block;
    const int grid = (int)std::min<long long>(want, (long long)sm_count(dev) * 8);
    kv_append_kernel<<<grid, kAppendThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return launch_status();
}

attn_status_t attn_kv_append_paged(const void* k_new, const void* v_new, void* k_cache,
                                   void* v_cache, const int32_t* block_table,
                                   int max_blocks_per_seq, int num_blocks, int block_size,
                                   const int32_t* cu_seqlens_new, const int32_t* seqused_k,
                                   int32_t* seqused_k_out, int B, int total_new, int num_heads_kv,
                                   int head_dim, int dtype, attn_stream_t stream) {
    return kv_append_launch(k_new, v_new, k_cache, v_cache, block_table, max_blocks_per_seq,
                            num_blocks, block_size, cu_seqlens_new, seqused_k, seqused_k_out, B,
                            total_new, num_heads_kv, head_dim, dtype, stream);
}

attn_status_t attn_decode_paged_append(const void* q, const void* k_new, const void* v_new,
                                       void* k_cache, void* v_cache, const int32_t* block_table,
                                       int max_blocks_per_seq, int num_blocks, int block_size,
                                       const int32_t* seqused_k, int32_t* seqused_k_out, int B,
                                       int Hq, int Hkv, int D, float softmax_scale,
                                       int window_left, float softcap, int num_splits, int dtype,
                                       void* o, float* lse, void* workspace,
                                       size_t workspace_bytes, attn_stream_t stream) {
    if (!seqused_k_out) return ATTN_ERR_INVALID_ARG;
    // Validate the decode half before anything is launched (no partial work on a bad call).
    if (!q || !o) return ATTN_ERR_INVALID_ARG;
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (Hq / Hkv > kDecRows || B > kDecMaxSeqs) return ATTN_ERR_UNSUPPORTED;
    {
        const attn_status_t ms = check_score_mods(ATTN_MASK_CAUSAL, window_left, softcap);
        if (ms != ATTN_OK) return ms;
    }
    if (!aligned16(q) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    if (B > 0) {
        int ns, tps;
        const int span = decode_span(max_blocks_per_seq * block_size, window_left < 0 ? -1 : window_left);
        decode_splits(B, Hkv, span, num_splits, &ns, &tps);
        const bool stream_pages = use_page_stream(B, Hq, Hkv, D, num_splits);
        if (stream_pages || ns > 1) {
            const size_t need = attn_decode_workspace_size(B, Hq, Hkv, D, max_blocks_per_seq,
                                                           block_size, num_splits);
            if (!workspace || !aligned16(workspace)) return ATTN_ERR_INVALID_ARG;
            if (workspace_bytes < need) return ATTN_ERR_WORKSPACE_TOO_SMALL;
        }
    }
    attn_status_t s = kv_append_launch(k_new, v_new, k_cache, v_cache, block_table,
                                       max_blocks_per_seq, num_blocks, block_size, nullptr,
                                       seqused_k, seqused_k_out, B, B, Hkv, D, dtype, stream);
    if (s != ATTN_OK || B == 0) return s;
    return decode_paged_impl(q, k_cache, v_cache, block_table, max_blocks_per_seq, num_blocks,
                             block_size, seqused_k_out, B, Hq, Hkv, D, softmax_scale, window_left,
                             softcap, num_splits, dtype, nullptr, nullptr, nullptr, o, lse,
                             workspace, workspace_bytes, stream, true);
}

size_t attn_bwd_workspace_size(int num_heads_q, int total_q) {
    if (num_heads_q <= 0 || total_q < 0) return 0;
    return (size_t)num_heads_q * (size_t)total_q * sizeof(float) + 16;
}

attn_status_t attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                              int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int Hq,
                              int Hkv, int D, float softmax_scale, int mask, int window_left,
                              void* workspace, size_t workspace_bytes, attn_stream_t stream) {
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !cu_seqlens_q || !cu_seqlens_k)
        return ATTN_ERR_INVALID_ARG;
    if (B < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0 || Hq <= 0 ||
        Hkv <= 0 || Hq % Hkv != 0)
        return ATTN_ERR_INVALID_ARG;
    if (mask != ATTN_MASK_NONE && mask != ATTN_MASK_CAUSAL)
        return mask == ATTN_MASK_PATCH ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
    if (window_left >= 0 && mask != ATTN_MASK_CAUSAL) return ATTN_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return ATTN_ERR_INVALID_ARG;
    const size_t need = attn_bwd_workspace_size(Hq, total_q);
    if (!workspace || !aligned16(workspace)) return ATTN_ERR_INVALID_ARG;
    if (workspace_bytes < need) return ATTN_ERR_WORKSPACE_TOO_SMALL;
    if ((long long)total_q * Hq >= (1LL << 31) || (long long)total_k >= (1LL << 31))
        return ATTN_ERR_UNSUPPORTED;
    int dev = 0;
    const attn_status_t dvs = current_device_ok(&dev);
    if (dvs != ATTN_OK) return dvs;
    if (B == 0 || total_q == 0) return ATTN_OK;

    CUtensorMap mq, mdo, mk, mv;
    const uint64_t rowq = (uint64_t)Hq * D * 2;
    const uint64_t dq4[4] = {(uint64_t)D, (uint64_t)Hq, (uint64_t)total_q, 1};
    const uint64_t sq3[3] = {(uint64_t)D * 2, rowq, rowq * (uint64_t)total_q};
    const uint64_t rowk = (uint64_t)Hkv * D * 2;
    const uint64_t nk = (uint64_t)std::max(total_k, 1);
    const uint64_t dk4[4] = {(uint64_t)D, (uint64_t)Hkv, nk, 1};
    const uint64_t sk3[3] = {(uint64_t)D * 2, rowk, rowk * nk};
    const uint32_t box[4] = {64, 1, 128, 1};
    attn_status_t s;
    if ((s = get_map(&mq, q, ATTN_BF16, dq4, sq3, box)) != ATTN_OK) return s;
    if ((s = get_map(&mdo, dout, ATTN_BF16, dq4, sq3, box)) != ATTN_OK) return s;
    if ((s = get_map(&mk, k, ATTN_BF16, dk4, sk3, box)) != ATTN_OK) return s;
    if ((s = get_map(&mv, v, ATTN_BF16, dk4, sk3, box)) != ATTN_OK) return s;

    BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.group = Hq / Hkv;
    a.mask = mask;
    a.window = window_left < 0 ? -1 : window_left;
    a.cu_q = cu_seqlens_q;
    a.cu_k = cu_seqlens_k;
    a.lse = lse;
    a.delta = static_cast<float*>(workspace);
    a.scale = resolve_scale(softmax_scale, D);
    a.dq = static_cast<__nv_bfloat16*>(dq);
    a.dk = static_cast<__nv_bfloat16*>(dk);
    a.dv = static_cast<__nv_bfloat16*>(dv);
    a.total_q = total_q;
    a.nqt = (max_seqlen_q + 127) / 128;
    a.nkt = (max_seqlen_k + 127) / 128;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* delta = static_cast<float*>(workspace);
    if (D == 128) return launch_backward<128>(mq, mdo, mk, mv, a, o, dout, delta, sm_count(dev), st);
    return launch_backward<64>(mq, mdo, mk, mv, a, o, dout, delta, sm_count(dev), st);
}

attn_status_t attn_decode_paged_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                        const int32_t* block_table, int max_blocks_per_seq,
                                        int num_blocks, int block_size, const int32_t* seqused_k,
                                        int B, int Hq, int Hkv, int D, float softmax_scale, int dtype,
                                        void* o, float* lse, attn_stream_t stream) {
    // The argument checks of attn_decode_paged, in its order, so that a bad call
    // gets the same status from both entry points; then what decides whether the
    // fixed scratch can serve the request.
    if (!q || !k_cache || !v_cache || !block_table || !seqused_k || !o) return ATTN_ERR_INVALID_ARG;
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (num_blocks <= 0 || max_blocks_per_seq <= 0) return ATTN_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (block_size != kPageRows) return ATTN_ERR_UNSUPPORTED;
    if (Hq / Hkv > kDecRows) return ATTN_ERR_UNSUPPORTED;
    if (B > kDecMaxSeqs) return ATTN_ERR_UNSUPPORTED;
    if ((long long)num_blocks * block_size >= (1LL << 31)) return ATTN_ERR_UNSUPPORTED;
    if ((long long)max_blocks_per_seq * block_size >= (1LL << 30)) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
        return ATTN_ERR_INVALID_ARG;
    if (B == 0) {
        const attn_status_t dv0 = current_device_ok(nullptr);
        return dv0;
    }
    if (!use_page_stream(B, Hq, Hkv, D, 0)) return ATTN_ERR_UNSUPPORTED;
    int dev = 0;
    const attn_status_t dvs = current_device_ok(&dev);
    if (dvs != ATTN_OK) return dvs;
    const size_t need = (size_t)((size_t)sm_count(dev) + B) * Hq * (D + 1) * sizeof(float) +
                        (size_t)(B + 2) * sizeof(int);
    if (need > kNoAllocScratchBytes) return ATTN_ERR_SCRATCH_LIMIT;
    void* scratch = noalloc_scratch_address(dev);
    if (!scratch) return ATTN_ERR_CUDA;
    return attn_decode_paged(q, k_cache, v_cache, block_table, max_blocks_per_seq, num_blocks,
                             block_size, seqused_k, B, Hq, Hkv, D, softmax_scale, -1, 0.0f, 0, dtype,
                             nullptr, nullptr, nullptr, o, lse, scratch, kNoAllocScratchBytes,
                             stream);
}

}  // extern "C"
