// lnq_quantize.cuh -- E4M3 quantization kernels.
//
//  * k_quantize_groups: activations, one FP32 scale per 1 x 128 group of a row
//    (Linnet "Backend plugins", DeepGEMM plugin: "each 128 inputs of a row to
//    FP8 with a scale of their own"), scales written MN-major over rows padded
//    to a multiple of four.  amax, scale and E4M3 cast are fused in one pass
//    over tiles streamed into shared memory by TMA.
//  * k_quantize_blocks: weights, one FP32 scale per 128 x 128 block (Linnet
//    plugin docstring; deepgemm-rust README, "Quick start", sfb shape).
//
// Both use scale = amax / 448 (IEEE fp32 division) and code = E4M3
// round-to-nearest-even of the correctly rounded fp32 quotient x / scale,
// saturating at +-448; a group with amax == 0 gets scale 0 and codes +-0.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "lnq_ptx.cuh"

namespace lnq {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two fp32 values to two E4M3 codes (saturating, RNE); `lo` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float quotient(float x, float s, bool zero_group) {
    return zero_group ? x : __fdiv_rn(x, s);
}

// The correctly rounded amax / 448 from one multiplication and two FMAs: q0 =
// RN(amax * c) with c = RN(1/448), then one correction step with the exact
// remainder amax - 448 q0 (Markstein's division correction for a divisor known
// in advance).  Checked exhaustively against the IEEE quotient over every
// non-negative finite bf16 amax.
__device__ __forceinline__ float scale_of_amax(float amax) {
    constexpr float c = 1.0f / 448.0f;
    const float q0 = __fmul_rn(amax, c);
    const float rem = __fmaf_rn(-q0, 448.0f, amax);
    return __fmaf_rn(rem, c, q0);
}

// Approximate reciprocal (hardware rcp.approx, within a few ulps).
__device__ __forceinline__ float rcp_approx(float s) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    return r;
}


__device__ __forceinline__ uint2 pack8(const float (&t)[8]) {
    uint2 out;
    out.x = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
    out.y = e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16);
    return out;
}

// Eight E4M3 codes (packed, the first value in the low byte) of the correctly rounded
// quotients x/s of the bf16 values in `raw`.  r_lo and r_hi bracket 1/s: with r within
// 2^-21 of 1/s (rcp.approx), r_lo = RN(r (1 - 2^-18)) and r_hi = RN(r (1 + 2^-18)), so for
// every x the products RN(x r_lo) and RN(x r_hi) lie on either side of RN(x/s) (each
// within about 2^-18 of x/s, further than RN(x/s) can be).  E4M3 rounding with
// saturation is monotonic, so when both products take the same code, RN(x/s) takes it
// too; otherwise (a quotient within about 32 fp32 ulps of an E4M3 rounding boundary,
// about one value in 16000) the eight values take the IEEE division.  A product that is
// an fp32 subnormal codes to +-0 at both ends, as the quotient does.  Scales below 2^-125,
// whose reciprocal may overflow, take the division outright; an all-zero group (s = 0)
// keeps the signed zeros.
__device__ __forceinline__ uint2 codes8(const uint4& raw, float s, float r_lo, float r_hi, bool zero_group,
                                        bool exact_group) {
    float t[8];
    t[0] = bf16_lo(raw.x);
    t[1] = bf16_hi(raw.x);
    t[2] = bf16_lo(raw.y);
    t[3] = bf16_hi(raw.y);
    t[4] = bf16_lo(raw.z);
    t[5] = bf16_hi(raw.z);
    t[6] = bf16_lo(raw.w);
    t[7] = bf16_hi(raw.w);
    if (zero_group) return pack8(t);
    if (!exact_group) {
        float lo[8], hi[8];
        const float2 rl = make_float2(r_lo, r_lo), rh = make_float2(r_hi, r_hi);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 x = make_float2(t[2 * j], t[2 * j + 1]);
            const float2 a = __fmul2_rn(x, rl), b = __fmul2_rn(x, rh);
            lo[2 * j] = a.x;
            lo[2 * j + 1] = a.y;
            hi[2 * j] = b.x;
            hi[2 * j + 1] = b.y;
        }
        const uint2 a = pack8(lo), b = pack8(hi);
        if (a.x == b.x && a.y == b.y) return a;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j] = __fdiv_rn(t[j], s);
    return pack8(t);
}

// The two bracketing reciprocals of codes8 for a scale s >= 2^-125.
__device__ __forceinline__ void bracket_rcp(float s, float& r_lo, float& r_hi) {
    const float r = rcp_approx(s);
    r_lo = __fmul_rn(r, 1.0f - 0x1p-18f);
    r_hi = __fmul_rn(r, 1.0f + 0x1p-18f);
}

// Largest magnitude of two packed bf16 pairs, as a packed pair whose magnitudes are
// max(|a|, |b|) lane by lane (the sign bits are not meaningful); exact.
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Largest |x| of the eight bf16 values in `raw` (exact).
__device__ __forceinline__ float absmax8_packed(const uint4& raw) {
    const uint32_t m = maxabs_bf16x2(maxabs_bf16x2(raw.x, raw.y), maxabs_bf16x2(raw.z, raw.w));
    return fmaxf(fabsf(bf16_lo(m)), fabsf(bf16_hi(m)));
}

__device__ __forceinline__ float absmax8(const uint4& raw) {
    float m = fabsf(bf16_lo(raw.x));
    m = fmaxf(m, fabsf(bf16_hi(raw.x)));
    m = fmaxf(m, fabsf(bf16_lo(raw.y)));
    m = fmaxf(m, fabsf(bf16_hi(raw.y)));
    m = fmaxf(m, fabsf(bf16_lo(raw.z)));
    m = fmaxf(m, fabsf(bf16_hi(raw.z)));
    m = fmaxf(m, fabsf(bf16_lo(raw.w)));
    m = fmaxf(m, fabsf(bf16_hi(raw.w)));
    return m;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

constexpr int kQuantRows = 32;      // rows of one activation tile
constexpr int kQuantCols = 256;     // columns of one tile: two 128-groups
constexpr int kQuantStages = 4;     // tiles in flight per CTA
constexpr int kQuantTileBytes = kQuantRows * kQuantCols * 2;
constexpr int kQuantConsumerWarps = 8;
constexpr int kQuantThreads = 32 * (kQuantConsumerWarps + 1);
constexpr int kQuantSmemBytes = kQuantStages * kQuantTileBytes + 2 * kQuantStages * 8 + 16 + 128;

// Row and column tile of t = blockIdx.x + i * gridDim.x, advanced by the grid size
// (t = r * cols + c) without a division per tile.
struct TileWalk {
    int r, c, dr, dc;
    __device__ __forceinline__ explicit TileWalk(int cols)
        : r(static_cast<int>(blockIdx.x) / cols), c(static_cast<int>(blockIdx.x) % cols),
          dr(static_cast<int>(gridDim.x) / cols), dc(static_cast<int>(gridDim.x) % cols) {}
    __device__ __forceinline__ void next(int cols) {
        r += dr;
        c += dc;
        if (c >= cols) {
            c -= cols;
            ++r;
        }
    }
};

struct QuantArgs {
    uint8_t* q;
    float* sfa;
    unsigned int* status;
    unsigned long long timeout_ns;
    long long M, K, ld_q, M4;
    int num_tiles;   // ceil(M4 / 32) * ceil(K / 256)
    int col_tiles;   // ceil(K / 256)
};

// Persistent 1x128 activation quantize.  A producer warp streams 32 x 256 bf16
// tiles into a 4-stage shared-memory ring with TMA (rows past M arrive as
// zeros); eight consumer warps each own four consecutive rows of a tile.  The
// lanes of half h of a warp take the warp's rows 2h and 2h+1, lane j of the half
// holding columns 16j .. 16j+15 of both, so that eight lanes form a 128-group and
// every lane codes 32 values with two rows' worth of scale work.  The two rows'
// amaxes travel as one packed bf16 pair through a three-step shuffle; the first
// lane of every eight stores the pair of scales (rows 2h, 2h+1; M4 is a multiple
// of 4).  Consumer warps never wait for one another.  Tile indices advance by the
// grid size without a division per tile.
__global__ void __launch_bounds__(kQuantThreads)
    k_quantize_groups(const __grid_constant__ CUtensorMap xmap, const QuantArgs args) {
    extern __shared__ uint8_t qsmem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(qsmem_raw) + 127) & ~static_cast<uintptr_t>(127));
    uint8_t* bar_area = smem + kQuantStages * kQuantTileBytes;
    const uint32_t bars = smem_u32(bar_area);
    auto full_bar = [&](int st) { return bars + 8u * st; };
    auto empty_bar = [&](int st) { return bars + 8u * (kQuantStages + st); };
    volatile uint32_t* abort_flag =
        reinterpret_cast<volatile uint32_t*>(bar_area + 2 * kQuantStages * 8);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int st = 0; st < kQuantStages; ++st) {
            mbar_init(full_bar(st), 1);
            mbar_init(empty_bar(st), kQuantConsumerWarps);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    launch_dependents();
    wait_prior_grids();
    WaitCtx wctx;
    wctx.abort = abort_flag;
    wctx.status = args.status;
    wctx.timeout_ns = args.timeout_ns;

    if (warp == kQuantConsumerWarps) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            tma_prefetch_desc(&xmap);
            int stage = 0;
            uint32_t phase = 0, filled = 0, fill_parity = 0;
            bool ok = true;
            TileWalk tw(args.col_tiles);
            for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x, tw.next(args.col_tiles)) {
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, wctx)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(full_bar(stage), kQuantTileBytes);
                tma_load_2d(smem_u32(smem + stage * kQuantTileBytes), &xmap, full_bar(stage),
                            tw.c * kQuantCols, tw.r * kQuantRows);
                filled |= 1u << stage;
                fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == kQuantStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                WaitCtx drain = wctx;
                uint32_t never = 0u;
                drain.abort = &never;
                for (int st = 0; st < kQuantStages; ++st)
                    if (filled & (1u << st)) (void)mbar_wait(full_bar(st), (fill_parity >> st) & 1u, drain);
            }
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    constexpr int kRowsPerWarp = kQuantRows / kQuantConsumerWarps;
    static_assert(kRowsPerWarp == 4, "two rows per half-warp");
    constexpr int kRowBytes = kQuantCols * 2;
    const int half = lane >> 4;
    const int j = lane & 15;       // columns 16j .. 16j+15 of the tile
    const int gsel = j >> 3;       // the tile's first or second 128-group
    const long long k_groups = args.K >> 7;
    int stage = 0;
    uint32_t phase = 0;
    TileWalk tw(args.col_tiles);
    for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x, tw.next(args.col_tiles)) {
        // first of this lane's two rows, and its first column
        const long long row0 = static_cast<long long>(tw.r) * kQuantRows + warp * kRowsPerWarp + 2 * half;
        const long long col = static_cast<long long>(tw.c) * kQuantCols + 16 * j;
        const long long group = (col >> 7);
        const bool group_ok = group < k_groups;
        if (!mbar_wait(full_bar(stage), phase, wctx)) break;
        const uint8_t* src = smem + stage * kQuantTileBytes + (warp * kRowsPerWarp + 2 * half) * kRowBytes + 32 * j;
        uint4 raw[2][2];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            raw[p][0] = *reinterpret_cast<const uint4*>(src + p * kRowBytes);
            raw[p][1] = *reinterpret_cast<const uint4*>(src + p * kRowBytes + 16);
        }
        // each row's largest magnitude over this lane's 16 values (both bf16 halves of
        // m[p] are candidates), then row 0 in the low and row 1 in the high half of one
        // word, reduced over the group's eight lanes; exact throughout
        uint32_t m[2];
#pragma unroll
        for (int p = 0; p < 2; ++p)
            m[p] = maxabs_bf16x2(maxabs_bf16x2(maxabs_bf16x2(raw[p][0].x, raw[p][0].y),
                                               maxabs_bf16x2(raw[p][0].z, raw[p][0].w)),
                                 maxabs_bf16x2(maxabs_bf16x2(raw[p][1].x, raw[p][1].y),
                                               maxabs_bf16x2(raw[p][1].z, raw[p][1].w)));
        uint32_t z = maxabs_bf16x2(__byte_perm(m[0], m[1], 0x5410), __byte_perm(m[0], m[1], 0x7632));
#pragma unroll
        for (int off = 1; off <= 4; off <<= 1) z = maxabs_bf16x2(z, __shfl_xor_sync(0xFFFFFFFFu, z, off));
        const float sv[2] = {scale_of_amax(fabsf(bf16_lo(z))), scale_of_amax(fabsf(bf16_hi(z)))};
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const long long r = row0 + p;
            if (r < args.M && group_ok) {
                float r_lo, r_hi;
                bracket_rcp(sv[p], r_lo, r_hi);
                const bool zero_group = sv[p] == 0.0f, exact_group = !(sv[p] >= 0x1p-125f);
                const uint2 a = codes8(raw[p][0], sv[p], r_lo, r_hi, zero_group, exact_group);
                const uint2 b = codes8(raw[p][1], sv[p], r_lo, r_hi, zero_group, exact_group);
                *reinterpret_cast<uint4*>(args.q + r * args.ld_q + col) = make_uint4(a.x, a.y, b.x, b.y);
            }
        }
        if ((j & 7) == 0 && group_ok && row0 < args.M4)
            *reinterpret_cast<float2*>(args.sfa + group * args.M4 + row0) = make_float2(sv[0], sv[1]);
        // The stage goes back to the producer only now: every value this warp read from it
        // fed the stores above (codes, or through the shuffles the scales), so the reads
        // have completed, and the release orders them before the next TMA write.  An
        // arrival straight after the reads let a shared-memory read still queued behind
        // bank-conflicted ones see the next tile.
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(stage));
        if (++stage == kQuantStages) {
            stage = 0;
            phase ^= 1u;
        }
    }
}

// grid = (ceil(N / 128), K / 128), block = 256 threads: one 128 x 128 block.
// Warp w takes rows 16w .. 16w+15 of the block; lane l columns 4l .. 4l+3.
__global__ void __launch_bounds__(256)
    k_quantize_blocks(const uint16_t* __restrict__ w, int64_t N, int64_t K,
                      uint8_t* __restrict__ q, float* __restrict__ sfb) {
    __shared__ float s_warp_max[8];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 128 + warp * 16;
    const int64_t col = static_cast<int64_t>(blockIdx.y) * 128 + lane * 4;

    uint2 raw[16];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int64_t r = n0 + i;
        raw[i] = make_uint2(0u, 0u);
        if (r < N) raw[i] = *reinterpret_cast<const uint2*>(w + r * K + col);
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(raw[i].x)), fabsf(bf16_hi(raw[i].x))),
                                 fmaxf(fabsf(bf16_lo(raw[i].y)), fabsf(bf16_hi(raw[i].y)))));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    if (lane == 0) s_warp_max[warp] = amax;
    __syncthreads();
    amax = s_warp_max[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, s_warp_max[i]);
    const float s = __fdiv_rn(amax, 448.0f);
    const bool zero_block = amax == 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int64_t r = n0 + i;
        if (r < N) {
            const uint32_t c =
                e4m3x2(quotient(bf16_lo(raw[i].x), s, zero_block),
                       quotient(bf16_hi(raw[i].x), s, zero_block)) |
                (e4m3x2(quotient(bf16_lo(raw[i].y), s, zero_block),
                        quotient(bf16_hi(raw[i].y), s, zero_block))
                 << 16);
            *reinterpret_cast<uint32_t*>(q + r * K + col) = c;
        }
    }
    if (threadIdx.x == 0) sfb[static_cast<int64_t>(blockIdx.x) * (K >> 7) + blockIdx.y] = s;
}

}  // namespace lnq
