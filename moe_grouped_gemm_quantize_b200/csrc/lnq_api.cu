// lnq_api.cu -- host layer of liblnq.so: argument checks, device checks, TMA
// descriptor encoding, tile-configuration choice and kernel launches behind
// the C ABI declared in include/lnq.h.
//
// The library allocates no device memory and never synchronizes a stream on
// the compute path.  Argument errors are returned before any CUDA call.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "lnq.h"
#include "lnq_gemm.cuh"
#include "lnq_mx.cuh"
#include "lnq_ptx.cuh"
#include "lnq_quantize.cuh"

namespace lnq {

// Device status word: timeout and bad-group bits set by the kernels.
__device__ unsigned int g_status;

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceInfo {
    bool ready = false;
    bool supported = false;
    int ordinal = 0;                 // device number, < kMaxDevices
    int sm_count = 0;
    unsigned int* status = nullptr;  // device address of g_status
};

std::mutex g_mutex;
// Dense GEMMs with M > 128 run on CTA pairs when set (1: 256x256, 2: 256x128 tiles).
std::atomic<int> g_dense_pairs{1};
// Grouped GEMMs in the prefix-sum layout with 256-row alignment run 256 x 256 tiles on
// CTA pairs when set (otherwise 128-row tiles, skipping those of pad rows only).
std::atomic<int> g_grouped_pairs{0};
// GEMMs may start streaming weights before the prior kernel completes.
std::atomic<int> g_weight_prefetch{0};
// Dense and grouped GEMM outputs go through shared memory and TMA stores when set.
std::atomic<int> g_tma_store{1};
DeviceInfo g_devices[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Raises a kernel's dynamic shared-memory limit once per device.  The per-device flags
// are atomic: first calls racing from several host threads may each set the attribute,
// which is harmless.
template <class Kernel>
lnq_status smem_attr_once(std::atomic<bool> (&done)[kMaxDevices], int ordinal, Kernel* kernel, int bytes) {
    if (!done[ordinal].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
            return LNQ_ERR_CUDA;
        done[ordinal].store(true, std::memory_order_release);
    }
    return LNQ_OK;
}
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Current device's capabilities; resolves the driver's tensor-map encoder once.
lnq_status device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LNQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return LNQ_ERR_UNSUPPORTED_ARCH;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& d = g_devices[dev];
    if (!d.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return LNQ_ERR_CUDA;
        d.supported = (major == 10 && minor == 0);
        d.ordinal = dev;
        d.sm_count = sms;
        if (d.supported) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return LNQ_ERR_CUDA;
            d.status = static_cast<unsigned int*>(p);
        }
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return LNQ_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        d.ready = true;
    }
    if (!d.supported) return LNQ_ERR_UNSUPPORTED_ARCH;
    *out = &d;
    return LNQ_OK;
}

// 2-D E4M3 tensor [rows][cols] (cols contiguous, row stride = cols bytes),
// box of 128 columns x box_rows rows, 128-byte swizzle, zero fill out of bounds.
lnq_status encode_e4m3_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                           int box_rows) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
    cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LNQ_OK : LNQ_ERR_CUDA;
}

// 2-D output tensor [rows][cols] of `elem_bytes`-byte elements (row stride = cols
// elements), box of 64 bytes x 128 rows in the 64-byte swizzle: one epilogue
// warpgroup's staging buffer of the TMA-store epilogue.
lnq_status encode_out_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int elem_bytes) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * elem_bytes)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(64 / elem_bytes), 128u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                          const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LNQ_OK : LNQ_ERR_CUDA;
}

// UE8M0 scale atoms viewed as rows of 128 32-bit words (one 512-byte atom per row), box
// of `box_rows` atoms, no swizzle: the CTA-pair block-scaled GEMM loads them by TMA.
lnq_status encode_atom_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows) {
    cuuint64_t dims[2] = {128u, static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {512u};
    cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LNQ_OK : LNQ_ERR_CUDA;
}

template <class C>
lnq_status launch_gemm(const DeviceInfo& dev, const void* act, int64_t act_rows,
                       const void* wgt, int64_t wgt_rows, int64_t K, GemmArgs args,
                       cudaStream_t stream) {
    CUtensorMap map_p, map_q;
    lnq_status st;
    if (C::SWAP) {
        st = encode_e4m3_map(&map_p, wgt, wgt_rows, K, C::kP);
        if (st == LNQ_OK) st = encode_e4m3_map(&map_q, act, act_rows, K, C::BNQ);
    } else {
        st = encode_e4m3_map(&map_p, act, act_rows, K, C::kP);
        if (st == LNQ_OK)
            st = encode_e4m3_map(&map_q, wgt, wgt_rows, K,
                                 C::SILU ? C::kQBoxRows : (C::PAIR ? C::kSliceQRows : C::kQRowsPerCta));
    }
    if (st != LNQ_OK) return st;
    // the output of the TMA-store epilogue (dense and grouped tiles; decode tiles store
    // their transposed rows directly and never read this map)
    CUtensorMap map_d;
    std::memset(&map_d, 0, sizeof map_d);
    if (!C::SWAP) {
        st = args.q_out != nullptr ? encode_out_map(&map_d, args.q_out, args.M, args.N, 1)
                                   : encode_out_map(&map_d, args.d, args.M, args.N, 2);
        if (st != LNQ_OK) return st;
    }
    static std::atomic<bool> attr_set[kMaxDevices];
    st = smem_attr_once(attr_set, dev.ordinal, k_fp8_block_gemm<C>, C::kSmemBytes);
    if (st != LNQ_OK) return st;
    args.status = dev.status;
    args.timeout_ns = kDefaultTimeoutNs;
    args.prefetch_weights = g_weight_prefetch.load(std::memory_order_relaxed);
    args.tma_store = g_tma_store.load(std::memory_order_relaxed);
    if (!C::SWAP) {
        // raster bands: grouped tiles 8 row blocks; dense tiles as many row tiles as keep
        // the band's activation rows within 32 MB of L2 (every weight column tile is
        // read once per band)
        int64_t band = 8;
        if (!C::GROUPED) {
            band = (int64_t{32} << 20) / (static_cast<int64_t>(C::kTileM) * K);
            if (band < 1) band = 1;
        }
        args.band = static_cast<int>(band < args.tiles_p ? band : (args.tiles_p > 0 ? args.tiles_p : 1));
    } else {
        args.band = 1;
    }
    if constexpr (C::PAIR) {
        // clusters of two CTAs sharing one MMA; as many pairs as can be resident
        constexpr int kCluster = 2;
        static std::atomic<int> max_clusters[kMaxDevices];
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.blockDim = dim3(C::kThreads, 1, 1);
        cfg.dynamicSmemBytes = C::kSmemBytes;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        int resident = max_clusters[dev.ordinal].load(std::memory_order_relaxed);
        if (resident == 0) {
            cfg.gridDim = dim3(2 * (dev.sm_count / 2), 1, 1);
            if (cudaOccupancyMaxActiveClusters(&resident, k_fp8_block_gemm<C>, &cfg) != cudaSuccess || resident <= 0)
                return LNQ_ERR_CUDA;
            max_clusters[dev.ordinal].store(resident, std::memory_order_relaxed);
        }
        const int clusters = args.num_tiles < resident ? args.num_tiles : resident;
        if (clusters <= 0) return LNQ_OK;
        cfg.gridDim = dim3(kCluster * clusters, 1, 1);
        if (cudaLaunchKernelEx(&cfg, k_fp8_block_gemm<C>, map_p, map_q, map_d, args) != cudaSuccess)
            return LNQ_ERR_CUDA;
        return cudaGetLastError() == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
    }
    // whole tiles per CTA, or (split) every CTA a run of the (tile, K block) units
    const long long work = C::SPLITK ? static_cast<long long>(args.num_tiles) * args.num_kb : args.num_tiles;
    const int grid = static_cast<int>(work < dev.sm_count ? work : dev.sm_count);
    if (grid <= 0) return LNQ_OK;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_fp8_block_gemm<C>, map_p, map_q, map_d, args) != cudaSuccess)
        return LNQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
}

// Tile configurations (P = MMA M slot, Q = MMA N slot).
using CfgDense256 = GemmCfg<256, 4, 2, false, false>;
using CfgPair256 = GemmCfg<256, 6, 2, false, false, true>;
using CfgPair128 = GemmCfg<128, 8, 2, false, false, true>;

using CfgDense128 = GemmCfg<128, 6, 2, false, false>;
using CfgGrouped256 = GemmCfg<256, 4, 2, false, true>;
using CfgGrouped128 = GemmCfg<128, 6, 2, false, true>;
using CfgGroupedPair256 = GemmCfg<256, 6, 2, false, true, true>;
using CfgSilu = GemmCfg<256, 4, 2, false, false, false, 1, false, true>;
using CfgSiluPair = GemmCfg<256, 6, 2, false, false, true, 1, false, true>;
using CfgSwap32 = GemmCfg<32, 5, 2, true, false>;
using CfgSwap64 = GemmCfg<64, 4, 2, true, false>;
using CfgSwap32Split = GemmCfg<32, 5, 2, true, false, false, 1, true>;
using CfgSwap64Split = GemmCfg<64, 4, 2, true, false, false, 1, true>;

constexpr int64_t kMaxRows = (int64_t{1} << 31) - 256;
// Split workspace: one int32 counter per weight tile in a fixed region at its start.
constexpr int64_t kSplitCounterBytes = 4096;

}  // namespace
}  // namespace lnq

using namespace lnq;

// Scratch of lnq_fp8_block_gemm_nt_static_ws: the decode K split's partial tiles and
// counters in a fixed device array (zero when the module loads; every call leaves the
// counters zero), so that entry point allocates nothing.  Calls on several streams
// would share it: they must not overlap.
static constexpr int64_t kStaticSplitBytes = int64_t{10} << 20;
static constexpr int kStaticSplitDevices = 64;
static __device__ __align__(256) unsigned char g_static_split_scratch[kStaticSplitBytes];
static void* g_static_split_addr[kStaticSplitDevices] = {};
static std::mutex g_static_split_mutex;

// Device address of the scratch array on device `devno` (the current device), looked
// up once per device; nullptr if the lookup fails.
static void* static_split_scratch(int devno) {
    std::lock_guard<std::mutex> lock(g_static_split_mutex);
    if (g_static_split_addr[devno] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_split_scratch) != cudaSuccess) return nullptr;
        g_static_split_addr[devno] = p;
    }
    return g_static_split_addr[devno];
}

// After a kernel gave up on a wait, a split may have left tile counters of the scratch
// array non-zero; later calls would then finish tiles early.  Zero the counter region
// (the first kSplitCounterBytes) of this device's array if it has been used.  Called
// with the stream already synchronized.
static lnq_status reset_static_split_counters(int devno, cudaStream_t stream) {
    void* p = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_static_split_mutex);
        if (devno >= 0 && devno < kStaticSplitDevices) p = g_static_split_addr[devno];
    }
    if (p == nullptr) return LNQ_OK;  // never used on this device: still all zero
    if (cudaMemsetAsync(p, 0, static_cast<size_t>(kSplitCounterBytes), stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return LNQ_ERR_CUDA;
    return LNQ_OK;
}

extern "C" {

int32_t lnq_abi_version(void) { return 10000; }

int32_t lnq_set_weight_prefetch(int32_t enable) { return g_weight_prefetch.exchange(enable ? 1 : 0); }

int32_t lnq_set_tma_store(int32_t enable) { return g_tma_store.exchange(enable ? 1 : 0); }

int32_t lnq_set_grouped_cta_pairs(int32_t enable) {
    return g_grouped_pairs.exchange(enable == 1 ? 1 : 0);
}

int32_t lnq_set_dense_cta_pairs(int32_t enable) {
    const int previous = g_dense_pairs.exchange(enable >= 0 && enable <= 2 ? enable : 0);
    return previous;
}

const char* lnq_status_string(lnq_status s) {
    switch (s) {
        case LNQ_OK: return "ok";
        case LNQ_ERR_INVALID_ARG: return "invalid argument";
        case LNQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case LNQ_ERR_MISALIGNED: return "misaligned pointer or stride";
        case LNQ_ERR_UNSUPPORTED_ARCH: return "device is not sm_100 (B200)";
        case LNQ_ERR_CUDA: return "CUDA call failed";
        case LNQ_ERR_TIMEOUT: return "a kernel wait timed out";
    }
    return "unknown status";
}

lnq_status lnq_quantize_fp8_groups(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x,
                                   void* q_e4m3, int64_t ld_q, float* sfa, int64_t M4,
                                   void* stream) {
    if (M < 0 || K <= 0) return LNQ_ERR_INVALID_ARG;
    if (K % 128 != 0) return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (ld_x < K || ld_q < K) return LNQ_ERR_INVALID_ARG;
    if (M4 < ((M + 3) / 4) * 4 || M4 % 4 != 0 || M4 > kMaxRows) return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (M4 == 0) return LNQ_OK;
    if (!sfa || (M > 0 && (!x_bf16 || !q_e4m3))) return LNQ_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(q_e4m3) || !aligned16(sfa) || ld_x % 8 != 0 ||
        ld_q % 16 != 0)
        return LNQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;
    if (M == 0) {
        // no rows: only the pad scales, which are zero
        return cudaMemsetAsync(sfa, 0, static_cast<size_t>(K / 128) * M4 * sizeof(float),
                               static_cast<cudaStream_t>(stream)) == cudaSuccess
                   ? LNQ_OK
                   : LNQ_ERR_CUDA;
    }
    // bf16 [M][ld_x] as a 2-D tensor of K columns, box of 256 columns x 32 rows
    CUtensorMap xmap;
    {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_x) * 2};
        cuuint32_t box[2] = {static_cast<cuuint32_t>(kQuantCols), static_cast<cuuint32_t>(kQuantRows)};
        cuuint32_t estr[2] = {1u, 1u};
        if (g_encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x_bf16), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return LNQ_ERR_CUDA;
    }
    QuantArgs qa{};
    qa.q = static_cast<uint8_t*>(q_e4m3);
    qa.sfa = sfa;
    qa.status = dev->status;
    qa.timeout_ns = kDefaultTimeoutNs;
    qa.M = M;
    qa.K = K;
    qa.ld_q = ld_q;
    qa.M4 = M4;
    qa.col_tiles = static_cast<int>((K + kQuantCols - 1) / kQuantCols);
    const long long tiles = ((M4 + kQuantRows - 1) / kQuantRows) * static_cast<long long>(qa.col_tiles);
    if (tiles > 0x7FFFFFFFLL) return LNQ_ERR_UNSUPPORTED_SHAPE;
    qa.num_tiles = static_cast<int>(tiles);
    static std::atomic<bool> attr_set[kMaxDevices];
    st = smem_attr_once(attr_set, dev->ordinal, k_quantize_groups, kQuantSmemBytes);
    if (st != LNQ_OK) return st;
    const long long max_ctas = 3LL * dev->sm_count;
    const int grid = static_cast<int>(tiles < max_ctas ? tiles : max_ctas);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kQuantThreads, 1, 1);
    cfg.dynamicSmemBytes = kQuantSmemBytes;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_quantize_groups, xmap, qa) != cudaSuccess) return LNQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
}

lnq_status lnq_quantize_fp8_blocks(const void* w_bf16, int64_t N, int64_t K, void* q_e4m3,
                                   float* sfb, void* stream) {
    if (N <= 0 || K <= 0) return LNQ_ERR_INVALID_ARG;
    if (K % 128 != 0 || N > kMaxRows || K / 128 > 65535) return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (!w_bf16 || !q_e4m3 || !sfb) return LNQ_ERR_INVALID_ARG;
    if (!aligned16(w_bf16) || !aligned16(q_e4m3) || !aligned4(sfb)) return LNQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;
    dim3 grid(static_cast<unsigned>((N + 127) / 128), static_cast<unsigned>(K / 128));
    k_quantize_blocks<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint16_t*>(w_bf16), N, K, static_cast<uint8_t*>(q_e4m3), sfb);
    return cudaGetLastError() == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
}

// ---------------------------------------------------------------- UE8M0 recipe

lnq_status lnq_quantize_ue8m0_groups(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, void* q_e4m3,
                                     int64_t ld_q, void* sfa_atoms, void* stream) {
    if (M <= 0 || K <= 0 || ld_x < K || ld_q < K) return LNQ_ERR_INVALID_ARG;
    if (K % 128 != 0 || M > kMaxRows || K > (int64_t{1} << 31)) return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (!x_bf16 || !q_e4m3 || !sfa_atoms) return LNQ_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(q_e4m3) || !aligned16(sfa_atoms) || ld_x % 8 != 0 || ld_q % 16 != 0)
        return LNQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;
    const int64_t Mpad = (M + 127) / 128 * 128;
    const int64_t units = Mpad * (K / 128);
    const int64_t want = (units + 15) / 16;  // 8 warps of two groups per CTA
    const int grid = static_cast<int>(want < 4 * dev->sm_count ? want : 4 * dev->sm_count);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_quantize_ue8m0_groups, static_cast<const uint16_t*>(x_bf16), static_cast<int>(M),
                           static_cast<int>(K), static_cast<long long>(ld_x), static_cast<uint8_t*>(q_e4m3),
                           static_cast<long long>(ld_q), static_cast<uint32_t*>(sfa_atoms),
                           static_cast<int>(Mpad)) != cudaSuccess)
        return LNQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
}

lnq_status lnq_quantize_ue8m0_blocks(const void* w_bf16, int64_t N, int64_t K, void* q_e4m3, void* sfb_atoms,
                                     void* stream) {
    if (N <= 0 || K <= 0) return LNQ_ERR_INVALID_ARG;
    if (K % 128 != 0 || N > kMaxRows || K > (int64_t{1} << 31) || ((N + 127) / 128) * (K / 128) > INT32_MAX)
        return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (!w_bf16 || !q_e4m3 || !sfb_atoms) return LNQ_ERR_INVALID_ARG;
    if (!aligned16(w_bf16) || !aligned16(q_e4m3) || !aligned16(sfb_atoms)) return LNQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;
    const int nblocks = static_cast<int>((N + 127) / 128);
    k_quantize_ue8m0_blocks<<<static_cast<unsigned>(nblocks * (K / 128)), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint16_t*>(w_bf16), static_cast<int>(N), static_cast<int>(K), static_cast<uint8_t*>(q_e4m3),
        static_cast<uint32_t*>(sfb_atoms), nblocks);
    return cudaGetLastError() == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
}

lnq_status lnq_quantize_mxfp8(const void* x_bf16, int64_t rows, int64_t K, int64_t ld_x, void* q_e4m3, int64_t ld_q,
                              void* sf_atoms, void* stream) {
    if (rows <= 0 || K <= 0 || ld_x < K || ld_q < K) return LNQ_ERR_INVALID_ARG;
    if (K % 128 != 0 || rows > kMaxRows || K > (int64_t{1} << 31)) return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (!x_bf16 || !q_e4m3 || !sf_atoms) return LNQ_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(q_e4m3) || !aligned16(sf_atoms) || ld_x % 8 != 0 || ld_q % 16 != 0)
        return LNQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;
    const int64_t Rpad = (rows + 127) / 128 * 128;
    const int64_t units = Rpad * (K / 128);
    const int64_t want = (units + 15) / 16;  // 8 warps of two four-group halves per CTA
    const int grid = static_cast<int>(want < 4 * dev->sm_count ? want : 4 * dev->sm_count);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_quantize_mxfp8, static_cast<const uint16_t*>(x_bf16), static_cast<int>(rows),
                           static_cast<int>(K), static_cast<long long>(ld_x), static_cast<uint8_t*>(q_e4m3),
                           static_cast<long long>(ld_q), static_cast<uint32_t*>(sf_atoms),
                           static_cast<int>(Rpad)) != cudaSuccess)
        return LNQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
}

}  // extern "C"

namespace {

// The block-scaled product of the UE8M0 recipes: gran-128 scales (GRAN32 false) or the
// MXFP8 gran-32 scales, dense or M-grouped contiguous (m_indices != nullptr).
// The UE8M0 / MXFP8 block-scaled GEMM: dense (m_indices and masked_m null), M-grouped
// contiguous (m_indices) or M-grouped masked (masked_m, groups of m_max rows, M the total).
template <bool GRAN32>
lnq_status mx_gemm(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3, const void* sfb_atoms,
                   const int32_t* m_indices, int32_t num_groups, void* d_bf16, int64_t M, int64_t N, int64_t K,
                   void* stream, const int32_t* masked_m = nullptr, int64_t m_max = 0) {
    using C = MxCfg<4>;
    using CP = MxCfg<6, true>;
    const bool grouped = m_indices != nullptr || masked_m != nullptr;
    if (M <= 0 || N <= 0 || K <= 0 || (grouped && num_groups <= 0)) return LNQ_ERR_INVALID_ARG;
    if (K % 128 != 0 || N % 16 != 0 || M > kMaxRows || N > kMaxRows || K > (int64_t{1} << 31))
        return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (grouped && (M % 128 != 0 || N % 128 != 0 || static_cast<int64_t>(num_groups) * N > kMaxRows))
        return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (masked_m != nullptr && (m_max <= 0 || m_max % 128 != 0 || M != static_cast<int64_t>(num_groups) * m_max))
        return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (!a_e4m3 || !sfa_atoms || !b_e4m3 || !sfb_atoms || !d_bf16) return LNQ_ERR_INVALID_ARG;
    if (!aligned16(a_e4m3) || !aligned16(sfa_atoms) || !aligned16(b_e4m3) || !aligned16(sfb_atoms) ||
        !aligned16(d_bf16) || (m_indices != nullptr && !aligned4(m_indices)) ||
        (masked_m != nullptr && !aligned4(masked_m)))
        return LNQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;
    // dense products of more than 128 rows run 256 x 256 tiles on CTA pairs unless the
    // dense configuration knob selects single CTAs
    const bool pair = !grouped && M > 128 && g_dense_pairs.load(std::memory_order_relaxed) != 0;
    const int64_t wrows = grouped ? static_cast<int64_t>(num_groups) * N : N;
    MxArgs args{};
    args.sfa = static_cast<const uint32_t*>(sfa_atoms);
    args.sfb = static_cast<const uint32_t*>(sfb_atoms);
    args.d = static_cast<uint16_t*>(d_bf16);
    args.status = dev->status;
    args.timeout_ns = kDefaultTimeoutNs;
    args.M = static_cast<int>(M);
    args.N = static_cast<int>(N);
    args.num_kb = static_cast<int>(K / 128);
    args.mblocks = static_cast<int>((M + 127) / 128);
    args.nblocks = static_cast<int>((wrows + 127) / 128);
    args.tiles_p = pair ? static_cast<int>((M + 255) / 256) : args.mblocks;
    args.tiles_q = static_cast<int>((N + 255) / 256);
    args.num_tiles = args.tiles_p * args.tiles_q;
    args.m_indices = m_indices;
    args.num_groups = grouped ? num_groups : 1;
    args.masked_m = masked_m;
    args.m_max = static_cast<int>(m_max);
    CUtensorMap map_a, map_b, map_sfa, map_sfb;
    std::memset(&map_sfa, 0, sizeof map_sfa);
    std::memset(&map_sfb, 0, sizeof map_sfb);
    st = encode_e4m3_map(&map_a, a_e4m3, M, K, 128);
    if (st == LNQ_OK) st = encode_e4m3_map(&map_b, b_e4m3, wrows, K, pair ? 128 : 256);
    if (st == LNQ_OK && pair) {
        st = encode_atom_map(&map_sfa, sfa_atoms, (K / 128) * args.mblocks, 1);
        if (st == LNQ_OK) st = encode_atom_map(&map_sfb, sfb_atoms, (K / 128) * args.nblocks, 2);
    }
    if (st != LNQ_OK) return st;
    static std::atomic<bool> attr_dense[kMaxDevices], attr_grouped[kMaxDevices], attr_pair[kMaxDevices];
    st = pair      ? smem_attr_once(attr_pair, dev->ordinal, k_mx_block_gemm<6, false, GRAN32, true>, CP::kSmemBytes)
         : grouped ? smem_attr_once(attr_grouped, dev->ordinal, k_mx_block_gemm<4, true, GRAN32>, C::kSmemBytes)
                   : smem_attr_once(attr_dense, dev->ordinal, k_mx_block_gemm<4, false, GRAN32>, C::kSmemBytes);
    if (st != LNQ_OK) return st;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cfg.attrs = attr;
    cudaError_t e;
    if (pair) {
        // clusters of two CTAs sharing one MMA; as many pairs as can be resident
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = 2;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
        cfg.dynamicSmemBytes = CP::kSmemBytes;
        static std::atomic<int> max_clusters[kMaxDevices];
        int resident = max_clusters[dev->ordinal].load(std::memory_order_relaxed);
        if (resident == 0) {
            cfg.gridDim = dim3(2 * (dev->sm_count / 2), 1, 1);
            if (cudaOccupancyMaxActiveClusters(&resident, k_mx_block_gemm<6, false, GRAN32, true>, &cfg) !=
                    cudaSuccess ||
                resident <= 0)
                return LNQ_ERR_CUDA;
            max_clusters[dev->ordinal].store(resident, std::memory_order_relaxed);
        }
        const int clusters = args.num_tiles < resident ? args.num_tiles : resident;
        cfg.gridDim = dim3(2 * clusters, 1, 1);
        e = cudaLaunchKernelEx(&cfg, k_mx_block_gemm<6, false, GRAN32, true>, map_a, map_b, map_sfa, map_sfb, args);
    } else {
        const int grid = args.num_tiles < dev->sm_count ? args.num_tiles : dev->sm_count;
        cfg.gridDim = dim3(grid, 1, 1);
        cfg.numAttrs = 1;
        cfg.dynamicSmemBytes = C::kSmemBytes;
        e = grouped ? cudaLaunchKernelEx(&cfg, k_mx_block_gemm<4, true, GRAN32>, map_a, map_b, map_sfa, map_sfb, args)
                    : cudaLaunchKernelEx(&cfg, k_mx_block_gemm<4, false, GRAN32>, map_a, map_b, map_sfa, map_sfb, args);
    }
    if (e != cudaSuccess) return LNQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
}

}  // namespace

extern "C" {

lnq_status lnq_mxfp8_gemm_nt(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3, const void* sfb_atoms,
                             void* d_bf16, int64_t M, int64_t N, int64_t K, void* stream) {
    return mx_gemm<true>(a_e4m3, sfa_atoms, b_e4m3, sfb_atoms, nullptr, 0, d_bf16, M, N, K, stream);
}

lnq_status lnq_m_grouped_mxfp8_gemm_contiguous(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3,
                                               const void* sfb_atoms, const int32_t* m_indices, int32_t num_groups,
                                               void* d_bf16, int64_t M_total, int64_t N, int64_t K, void* stream) {
    if (!m_indices) return LNQ_ERR_INVALID_ARG;
    return mx_gemm<true>(a_e4m3, sfa_atoms, b_e4m3, sfb_atoms, m_indices, num_groups, d_bf16, M_total, N, K,
                         stream);
}

lnq_status lnq_m_grouped_mx_gemm_masked(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3,
                                        const void* sfb_atoms, const int32_t* masked_m, int32_t num_groups,
                                        int64_t M_max, int64_t expected_m, void* d_bf16, int64_t N, int64_t K,
                                        void* stream) {
    if (!masked_m || expected_m < 0 || num_groups <= 0 || M_max <= 0) return LNQ_ERR_INVALID_ARG;
    return mx_gemm<false>(a_e4m3, sfa_atoms, b_e4m3, sfb_atoms, nullptr, num_groups, d_bf16,
                          static_cast<int64_t>(num_groups) * M_max, N, K, stream, masked_m, M_max);
}

lnq_status lnq_m_grouped_mxfp8_gemm_masked(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3,
                                           const void* sfb_atoms, const int32_t* masked_m, int32_t num_groups,
                                           int64_t M_max, int64_t expected_m, void* d_bf16, int64_t N, int64_t K,
                                           void* stream) {
    if (!masked_m || expected_m < 0 || num_groups <= 0 || M_max <= 0) return LNQ_ERR_INVALID_ARG;
    return mx_gemm<true>(a_e4m3, sfa_atoms, b_e4m3, sfb_atoms, nullptr, num_groups, d_bf16,
                         static_cast<int64_t>(num_groups) * M_max, N, K, stream, masked_m, M_max);
}

lnq_status lnq_mx_block_gemm_nt(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3,
                                const void* sfb_atoms, void* d_bf16, int64_t M, int64_t N, int64_t K,
                                void* stream) {
    return mx_gemm<false>(a_e4m3, sfa_atoms, b_e4m3, sfb_atoms, nullptr, 0, d_bf16, M, N, K, stream);
}

namespace {

// Layout of the split workspace for one decode product, or need_bytes == 0 when the
// product does not split: [counters: one int32 per tile in a fixed 4 KiB region]
// [partials: tiles * max_slots * 128 * BNQ fp32 from byte 4096].  The counters sit
// at the same place for every shape, so one workspace (zeroed once) serves any
// sequence of products: each call rezeroes the counters it used, and no call writes
// partial tiles over another shape's counters.
struct SplitPlan {
    int64_t need_bytes = 0;
    int64_t partials_offset = kSplitCounterBytes;
    int max_slots = 0;
};

SplitPlan plan_split(int64_t M, int64_t N, int64_t K, int64_t num_sms) {
    SplitPlan plan;
    if (M <= 0 || M > 64 || N <= 0 || K <= 0 || K % 128 != 0 || num_sms <= 0) return plan;
    const int64_t bnq = M <= 32 ? 32 : 64;
    const int64_t tiles = ((N + 127) / 128) * ((M + bnq - 1) / bnq);
    const int64_t nkb = K / 128;
    // only where whole tiles would leave SMs idle and a tile has K blocks to share
    if (tiles >= num_sms || nkb < 2 || tiles * 4 > kSplitCounterBytes) return plan;
    const int64_t U = tiles * nkb;
    const int64_t G = U < num_sms ? U : num_sms;
    auto owner = [&](int64_t x) { return ((x + 1) * G + U - 1) / U - 1; };
    int64_t slots = 0;
    for (int64_t t = 0; t < tiles; ++t) {
        const int64_t n = owner((t + 1) * nkb - 1) - owner(t * nkb) + 1;
        if (n > slots) slots = n;
    }
    auto round256 = [](int64_t b) { return (b + 255) / 256 * 256; };
    plan.max_slots = static_cast<int>(slots);
    plan.need_bytes = kSplitCounterBytes + round256(tiles * slots * 128 * bnq * 4);
    return plan;
}

// Output side of a dense product: bf16 D, or (fused) the E4M3 codes and 1 x 128
// scales of the bf16-rounded result; an optional bf16 bias per column.
struct Epilogue {
    const void* bias = nullptr;
    void* q_out = nullptr;
    float* sfa_out = nullptr;
    int64_t M4_out = 0;
};

// The argument checks of a dense product, made on the host before any CUDA call.
lnq_status check_gemm_args(const void* a_e4m3, const float* sfa, int64_t M4, const void* b_e4m3,
                           const float* sfb, const void* d_bf16, int64_t M, int64_t N, int64_t K,
                           const Epilogue& ep) {
    if (M <= 0 || N <= 0 || K <= 0) return LNQ_ERR_INVALID_ARG;
    if (K % 128 != 0 || N % 16 != 0 || N < 16 || M > kMaxRows || N > kMaxRows ||
        K > (int64_t{1} << 31))
        return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (M4 < ((M + 3) / 4) * 4 || M4 % 4 != 0) return LNQ_ERR_UNSUPPORTED_SHAPE;
    const bool fp8_out = ep.q_out != nullptr;
    if (!a_e4m3 || !sfa || !b_e4m3 || !sfb || (fp8_out ? (d_bf16 != nullptr) : (d_bf16 == nullptr)))
        return LNQ_ERR_INVALID_ARG;
    if (!aligned16(a_e4m3) || !aligned16(sfa) || !aligned16(b_e4m3) || !aligned4(sfb) ||
        (d_bf16 && !aligned16(d_bf16)) || (ep.bias && !aligned16(ep.bias)))
        return LNQ_ERR_MISALIGNED;
    if (fp8_out) {
        // each epilogue thread must hold one whole 1 x 128 group: dense 128 x 256 tiles
        if (M <= 64 || N % 128 != 0 || N < 256) return LNQ_ERR_UNSUPPORTED_SHAPE;
        if (!ep.sfa_out) return LNQ_ERR_INVALID_ARG;
        if (ep.M4_out < ((M + 3) / 4) * 4 || ep.M4_out % 4 != 0) return LNQ_ERR_UNSUPPORTED_SHAPE;
        if (!aligned16(ep.q_out) || !aligned16(ep.sfa_out)) return LNQ_ERR_MISALIGNED;
    }
    return LNQ_OK;
}

lnq_status gemm_nt(const void* a_e4m3, const float* sfa, int64_t M4, const void* b_e4m3,
                   const float* sfb, void* d_bf16, int64_t M, int64_t N, int64_t K,
                   void* workspace, int64_t workspace_bytes, void* stream,
                   const Epilogue& ep = Epilogue()) {
    lnq_status st = check_gemm_args(a_e4m3, sfa, M4, b_e4m3, sfb, d_bf16, M, N, K, ep);
    if (st != LNQ_OK) return st;
    const bool fp8_out = ep.q_out != nullptr;
    DeviceInfo* dev = nullptr;
    st = device_info(&dev);
    if (st != LNQ_OK) return st;

    GemmArgs args{};
    args.sfa = sfa;
    args.sfb = sfb;
    args.d = static_cast<uint16_t*>(d_bf16);
    args.bias = static_cast<const uint16_t*>(ep.bias);
    args.q_out = static_cast<uint8_t*>(ep.q_out);
    args.sfa_out = ep.sfa_out;
    args.M4_out = ep.M4_out;
    args.M4 = M4;
    args.M = static_cast<int>(M);
    args.N = static_cast<int>(N);
    args.num_kb = static_cast<int>(K / 128);
    args.nb = static_cast<int>((N + 127) / 128);
    args.num_groups = 1;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M <= 64) {
        // decode: weights in the MMA's 128-row slot, tokens padded to 32 or 64
        args.tiles_p = static_cast<int>((N + 127) / 128);
        const SplitPlan plan = plan_split(M, N, K, dev->sm_count);
        if (workspace != nullptr && plan.need_bytes > 0) {
            if (workspace_bytes < plan.need_bytes) return LNQ_ERR_INVALID_ARG;
            if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return LNQ_ERR_MISALIGNED;
            // all SMs share the (tile, K block) units; partial tiles meet in the workspace
            args.counters = static_cast<int*>(workspace);
            args.partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + plan.partials_offset);
            args.max_slots = plan.max_slots;
            if (M <= 32) {
                args.tiles_q = static_cast<int>((M + 31) / 32);
                args.num_tiles = args.tiles_p * args.tiles_q;
                return launch_gemm<CfgSwap32Split>(*dev, a_e4m3, M, b_e4m3, N, K, args, s);
            }
            args.tiles_q = static_cast<int>((M + 63) / 64);
            args.num_tiles = args.tiles_p * args.tiles_q;
            return launch_gemm<CfgSwap64Split>(*dev, a_e4m3, M, b_e4m3, N, K, args, s);
        }
        if (M <= 32) {
            args.tiles_q = static_cast<int>((M + 31) / 32);
            args.num_tiles = args.tiles_p * args.tiles_q;
            return launch_gemm<CfgSwap32>(*dev, a_e4m3, M, b_e4m3, N, K, args, s);
        }
        args.tiles_q = static_cast<int>((M + 63) / 64);
        args.num_tiles = args.tiles_p * args.tiles_q;
        return launch_gemm<CfgSwap64>(*dev, a_e4m3, M, b_e4m3, N, K, args, s);
    }
    int pairs = g_dense_pairs.load(std::memory_order_relaxed);
    if (fp8_out && pairs == 2) pairs = 1;  // 256 x 128 pair tiles split a thread's 128-column group
    if (N >= 256 && M > 128 && pairs == 1) {
        // pairs of CTAs on 256 x 256 tiles
        args.tiles_p = static_cast<int>((M + 255) / 256);
        args.tiles_q = static_cast<int>((N + 255) / 256);
        args.num_tiles = args.tiles_p * args.tiles_q;
        return launch_gemm<CfgPair256>(*dev, a_e4m3, M, b_e4m3, N, K, args, s);
    }
    if (N >= 128 && M > 128 && pairs == 2) {
        // pairs of CTAs on 256 x 128 tiles, four accumulators per CTA
        args.tiles_p = static_cast<int>((M + 255) / 256);
        args.tiles_q = static_cast<int>((N + 127) / 128);
        args.num_tiles = args.tiles_p * args.tiles_q;
        return launch_gemm<CfgPair128>(*dev, a_e4m3, M, b_e4m3, N, K, args, s);
    }
    args.tiles_p = static_cast<int>((M + 127) / 128);
    if (N >= 256) {
        args.tiles_q = static_cast<int>((N + 255) / 256);
        args.num_tiles = args.tiles_p * args.tiles_q;
        return launch_gemm<CfgDense256>(*dev, a_e4m3, M, b_e4m3, N, K, args, s);
    }
    args.tiles_q = static_cast<int>((N + 127) / 128);
    args.num_tiles = args.tiles_p * args.tiles_q;
    return launch_gemm<CfgDense128>(*dev, a_e4m3, M, b_e4m3, N, K, args, s);
}

}  // namespace

lnq_status lnq_fp8_block_gemm_nt(const void* a_e4m3, const float* sfa, int64_t M4,
                                 const void* b_e4m3, const float* sfb, void* d_bf16, int64_t M,
                                 int64_t N, int64_t K, void* stream) {
    return gemm_nt(a_e4m3, sfa, M4, b_e4m3, sfb, d_bf16, M, N, K, nullptr, 0, stream);
}

int64_t lnq_fp8_block_gemm_nt_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t num_sms) {
    return plan_split(M, N, K, num_sms).need_bytes;
}

lnq_status lnq_fp8_block_gemm_nt_epilogue(const void* a_e4m3, const float* sfa, int64_t M4,
                                          const void* b_e4m3, const float* sfb, const void* bias_bf16,
                                          void* d_bf16, void* q_e4m3, float* sfa_out, int64_t M4_out,
                                          int64_t M, int64_t N, int64_t K, void* stream) {
    Epilogue ep;
    ep.bias = bias_bf16;
    ep.q_out = q_e4m3;
    ep.sfa_out = sfa_out;
    ep.M4_out = M4_out;
    return gemm_nt(a_e4m3, sfa, M4, b_e4m3, sfb, d_bf16, M, N, K, nullptr, 0, stream, ep);
}

lnq_status lnq_fp8_block_gemm_nt_ws(const void* a_e4m3, const float* sfa, int64_t M4,
                                    const void* b_e4m3, const float* sfb, void* d_bf16, int64_t M,
                                    int64_t N, int64_t K, void* workspace, int64_t workspace_bytes,
                                    void* stream) {
    if (workspace_bytes < 0) return LNQ_ERR_INVALID_ARG;
    return gemm_nt(a_e4m3, sfa, M4, b_e4m3, sfb, d_bf16, M, N, K, workspace, workspace_bytes, stream);
}

lnq_status lnq_fp8_block_gemm_nt_static_ws(const void* a_e4m3, const float* sfa, int64_t M4,
                                           const void* b_e4m3, const float* sfb, void* d_bf16,
                                           int64_t M, int64_t N, int64_t K, void* stream) {
    // argument errors come back before any CUDA call, as for every other entry point
    lnq_status st = check_gemm_args(a_e4m3, sfa, M4, b_e4m3, sfb, d_bf16, M, N, K, Epilogue());
    if (st != LNQ_OK) return st;
    DeviceInfo* dev = nullptr;
    st = device_info(&dev);
    if (st != LNQ_OK) return st;
    const int devno = dev->ordinal;
    if (devno < 0 || devno >= kStaticSplitDevices) return LNQ_ERR_INVALID_ARG;
    const int64_t need = plan_split(M, N, K, dev->sm_count).need_bytes;
    if (need > kStaticSplitBytes) return LNQ_ERR_UNSUPPORTED_SHAPE;
    void* ws = nullptr;
    if (need > 0) {
        ws = static_split_scratch(devno);
        if (ws == nullptr) return LNQ_ERR_CUDA;
    }
    return gemm_nt(a_e4m3, sfa, M4, b_e4m3, sfb, d_bf16, M, N, K, ws, kStaticSplitBytes, stream);
}

lnq_status lnq_m_grouped_fp8_gemm_contiguous(const void* a_e4m3, const float* sfa,
                                             const void* b_e4m3, const float* sfb,
                                             const int32_t* m_indices, int32_t num_groups,
                                             void* d_bf16, int64_t M_total, int64_t N, int64_t K,
                                             void* stream) {
    if (M_total <= 0 || N <= 0 || K <= 0 || num_groups <= 0) return LNQ_ERR_INVALID_ARG;
    if (M_total % 128 != 0 || K % 128 != 0 || N % 16 != 0 || N < 16 || M_total > kMaxRows ||
        K > (int64_t{1} << 31) || static_cast<int64_t>(num_groups) * N > kMaxRows)
        return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (!a_e4m3 || !sfa || !b_e4m3 || !sfb || !m_indices || !d_bf16) return LNQ_ERR_INVALID_ARG;
    if (!aligned16(a_e4m3) || !aligned16(sfa) || !aligned16(b_e4m3) || !aligned4(sfb) ||
        !aligned16(d_bf16) || !aligned4(m_indices))
        return LNQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;

    GemmArgs args{};
    args.sfa = sfa;
    args.sfb = sfb;
    args.d = static_cast<uint16_t*>(d_bf16);
    args.m_indices = m_indices;
    args.M4 = M_total;
    args.M = static_cast<int>(M_total);
    args.N = static_cast<int>(N);
    args.num_kb = static_cast<int>(K / 128);
    args.nb = static_cast<int>((N + 127) / 128);
    args.num_groups = num_groups;
    args.tiles_p = static_cast<int>(M_total / 128);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t wrows = static_cast<int64_t>(num_groups) * N;
    if (N >= 256) {
        args.tiles_q = static_cast<int>((N + 255) / 256);
        args.num_tiles = args.tiles_p * args.tiles_q;
        return launch_gemm<CfgGrouped256>(*dev, a_e4m3, M_total, b_e4m3, wrows, K, args, s);
    }
    args.tiles_q = static_cast<int>((N + 127) / 128);
    args.num_tiles = args.tiles_p * args.tiles_q;
    return launch_gemm<CfgGrouped128>(*dev, a_e4m3, M_total, b_e4m3, wrows, K, args, s);
}

lnq_status lnq_fp8_block_gemm_nt_silu_mul(const void* a_e4m3, const float* sfa, int64_t M4,
                                          const void* b_e4m3, const float* sfb, void* h_bf16,
                                          int64_t M, int64_t I, int64_t K, void* stream) {
    if (M <= 0 || I <= 0 || K <= 0) return LNQ_ERR_INVALID_ARG;
    if (K % 128 != 0 || I % 128 != 0 || M > kMaxRows || 2 * I > kMaxRows || K > (int64_t{1} << 31))
        return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (M4 < ((M + 3) / 4) * 4 || M4 % 4 != 0) return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (!a_e4m3 || !sfa || !b_e4m3 || !sfb || !h_bf16) return LNQ_ERR_INVALID_ARG;
    if (!aligned16(a_e4m3) || !aligned16(sfa) || !aligned16(b_e4m3) || !aligned4(sfb) || !aligned16(h_bf16))
        return LNQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;

    // Dense tiles of 128 outputs: the MMA's 256 columns are the outputs' 128 gate
    // rows and their 128 up rows (I further on in the weight).
    GemmArgs args{};
    args.sfa = sfa;
    args.sfb = sfb;
    args.d = static_cast<uint16_t*>(h_bf16);
    args.M4 = M4;
    args.M = static_cast<int>(M);
    args.N = static_cast<int>(I);
    args.num_kb = static_cast<int>(K / 128);
    args.nb = static_cast<int>(2 * I / 128);
    args.num_groups = 1;
    args.tiles_q = static_cast<int>(I / 128);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M > 128 && g_dense_pairs.load(std::memory_order_relaxed) != 0) {
        args.tiles_p = static_cast<int>((M + 255) / 256);
        args.num_tiles = args.tiles_p * args.tiles_q;
        return launch_gemm<CfgSiluPair>(*dev, a_e4m3, M, b_e4m3, 2 * I, K, args, s);
    }
    args.tiles_p = static_cast<int>((M + 127) / 128);
    args.num_tiles = args.tiles_p * args.tiles_q;
    return launch_gemm<CfgSilu>(*dev, a_e4m3, M, b_e4m3, 2 * I, K, args, s);
}

lnq_status lnq_m_grouped_mx_gemm_contiguous(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3,
                                            const void* sfb_atoms, const int32_t* m_indices, int32_t num_groups,
                                            void* d_bf16, int64_t M_total, int64_t N, int64_t K, void* stream) {
    if (!m_indices) return LNQ_ERR_INVALID_ARG;
    return mx_gemm<false>(a_e4m3, sfa_atoms, b_e4m3, sfb_atoms, m_indices, num_groups, d_bf16, M_total, N, K,
                          stream);
}

lnq_status lnq_m_grouped_fp8_gemm_contiguous_psum(const void* a_e4m3, const float* sfa,
                                                  const void* b_e4m3, const float* sfb,
                                                  const int32_t* psum, int32_t num_groups,
                                                  int64_t alignment, void* d_bf16, int64_t M_total,
                                                  int64_t N, int64_t K, void* stream) {
    if (M_total <= 0 || N <= 0 || K <= 0 || num_groups <= 0) return LNQ_ERR_INVALID_ARG;
    if (alignment != 128 && alignment != 256) return LNQ_ERR_INVALID_ARG;
    if (M_total % alignment != 0 || K % 128 != 0 || N % 16 != 0 || N < 16 || M_total > kMaxRows ||
        K > (int64_t{1} << 31) || static_cast<int64_t>(num_groups) * N > kMaxRows)
        return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (!a_e4m3 || !sfa || !b_e4m3 || !sfb || !psum || !d_bf16) return LNQ_ERR_INVALID_ARG;
    if (!aligned16(a_e4m3) || !aligned16(sfa) || !aligned16(b_e4m3) || !aligned4(sfb) ||
        !aligned16(d_bf16) || !aligned4(psum))
        return LNQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;

    // The grouped kernel with each tile's group looked up in psum on the device (no
    // host synchronization, no per-row ids).  Groups aligned to 256 rows hold whole
    // 256-row tiles, which may run on CTA pairs like the dense ones; by default the
    // tiles are 128 rows and those holding pad rows only are skipped, so the rows
    // computed are the same as with 128-row alignment.
    GemmArgs args{};
    args.sfa = sfa;
    args.sfb = sfb;
    args.d = static_cast<uint16_t*>(d_bf16);
    args.m_indices = nullptr;
    args.psum = psum;
    args.align = static_cast<int>(alignment);
    args.M4 = M_total;
    args.M = static_cast<int>(M_total);
    args.N = static_cast<int>(N);
    args.num_kb = static_cast<int>(K / 128);
    args.nb = static_cast<int>((N + 127) / 128);
    args.num_groups = num_groups;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t wrows = static_cast<int64_t>(num_groups) * N;
    if (alignment == 256 && N >= 256 && g_grouped_pairs.load(std::memory_order_relaxed) != 0) {
        args.tiles_p = static_cast<int>(M_total / 256);
        args.tiles_q = static_cast<int>((N + 255) / 256);
        args.num_tiles = args.tiles_p * args.tiles_q;
        return launch_gemm<CfgGroupedPair256>(*dev, a_e4m3, M_total, b_e4m3, wrows, K, args, s);
    }
    args.tiles_p = static_cast<int>(M_total / 128);
    if (N >= 256) {
        args.tiles_q = static_cast<int>((N + 255) / 256);
        args.num_tiles = args.tiles_p * args.tiles_q;
        return launch_gemm<CfgGrouped256>(*dev, a_e4m3, M_total, b_e4m3, wrows, K, args, s);
    }
    args.tiles_q = static_cast<int>((N + 127) / 128);
    args.num_tiles = args.tiles_p * args.tiles_q;
    return launch_gemm<CfgGrouped128>(*dev, a_e4m3, M_total, b_e4m3, wrows, K, args, s);
}

lnq_status lnq_m_grouped_fp8_gemm_masked(const void* a_e4m3, const float* sfa, const void* b_e4m3,
                                         const float* sfb, const int32_t* masked_m,
                                         int32_t num_groups, int64_t M_max, int64_t expected_m,
                                         void* d_bf16, int64_t N, int64_t K, void* stream) {
    if (M_max <= 0 || N <= 0 || K <= 0 || num_groups <= 0 || expected_m < 0)
        return LNQ_ERR_INVALID_ARG;
    const int64_t M_total = static_cast<int64_t>(num_groups) * M_max;
    if (M_max % 128 != 0 || K % 128 != 0 || N % 16 != 0 || N < 16 || M_total > kMaxRows ||
        K > (int64_t{1} << 31) || static_cast<int64_t>(num_groups) * N > kMaxRows)
        return LNQ_ERR_UNSUPPORTED_SHAPE;
    if (!a_e4m3 || !sfa || !b_e4m3 || !sfb || !masked_m || !d_bf16) return LNQ_ERR_INVALID_ARG;
    if (!aligned16(a_e4m3) || !aligned16(sfa) || !aligned16(b_e4m3) || !aligned4(sfb) ||
        !aligned16(d_bf16) || !aligned4(masked_m))
        return LNQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;

    // The grouped kernel with the group of a 128-row block given by its position and
    // the block's real rows by masked_m, read on the device (no host synchronization).
    // expected_m is accepted as the callers' scheduling hint; the blocks past a
    // group's count are skipped by the CTA that owns them.
    GemmArgs args{};
    args.sfa = sfa;
    args.sfb = sfb;
    args.d = static_cast<uint16_t*>(d_bf16);
    args.m_indices = nullptr;
    args.masked_m = masked_m;
    args.m_max = static_cast<int>(M_max);
    args.M4 = M_total;
    args.M = static_cast<int>(M_total);
    args.N = static_cast<int>(N);
    args.num_kb = static_cast<int>(K / 128);
    args.nb = static_cast<int>((N + 127) / 128);
    args.num_groups = num_groups;
    args.tiles_p = static_cast<int>(M_total / 128);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t wrows = static_cast<int64_t>(num_groups) * N;
    if (N >= 256) {
        args.tiles_q = static_cast<int>((N + 255) / 256);
        args.num_tiles = args.tiles_p * args.tiles_q;
        return launch_gemm<CfgGrouped256>(*dev, a_e4m3, M_total, b_e4m3, wrows, K, args, s);
    }
    args.tiles_q = static_cast<int>((N + 127) / 128);
    args.num_tiles = args.tiles_p * args.tiles_q;
    return launch_gemm<CfgGrouped128>(*dev, a_e4m3, M_total, b_e4m3, wrows, K, args, s);
}

lnq_status lnq_get_last_device_error(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return LNQ_ERR_CUDA;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof v) != cudaSuccess) return LNQ_ERR_CUDA;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof zero) != cudaSuccess) return LNQ_ERR_CUDA;
    }
    if (v & kStatusTimeout) {
        st = reset_static_split_counters(dev->ordinal, static_cast<cudaStream_t>(stream));
        if (st != LNQ_OK) return st;
        return LNQ_ERR_TIMEOUT;
    }
    if (v & kStatusBadGroup) return LNQ_ERR_INVALID_ARG;
    return LNQ_OK;
}

lnq_status lnq_selftest_wait_timeout(int64_t timeout_ns, void* stream) {
    if (timeout_ns < 1000 || timeout_ns > 10000000000LL) return LNQ_ERR_INVALID_ARG;
    DeviceInfo* dev = nullptr;
    lnq_status st = device_info(&dev);
    if (st != LNQ_OK) return st;
    k_wait_timeout_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        dev->status, static_cast<unsigned long long>(timeout_ns));
    return cudaGetLastError() == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
}

}  // extern "C"
