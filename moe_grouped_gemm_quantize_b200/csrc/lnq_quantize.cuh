// lnq_quantize.cuh -- E4M3 quantization kernels.
//
//  * k_quantize_groups: activations, one FP32 scale per 1 x 128 group of a row
//    (Linnet "Backend plugins", DeepGEMM plugin: "each 128 inputs of a row to
//    FP8 with a scale of their own"), scales written MN-major over rows padded
//    to a multiple of four.  amax, scale and E4M3 cast are fused in one pass:
//    128-bit bf16 loads, a half-warp shuffle reduction for amax, packed
//    e4m3x2 conversion, and the scale column staged through shared memory so
//    it is stored as contiguous 128-byte runs.
//  * k_quantize_blocks: weights, one FP32 scale per 128 x 128 block (Linnet
//    plugin docstring; deepgemm-rust README, "Quick start", sfb shape).
//
// Both use scale = amax / 448 (IEEE fp32 division) and code = E4M3
// round-to-nearest-even of the correctly rounded fp32 quotient x / scale,
// saturating at +-448; a group with amax == 0 gets scale 0 and codes +-0.
#pragma once

#include <cstdint>

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

// True when the E4M3 rounding of t could differ from the E4M3 rounding of a
// value at most 3 fp32 ulps away: t within 4 ulps of a rounding midpoint of the
// normal E4M3 range (the 20 fp32 mantissa bits below the 3 E4M3 mantissa bits
// within 4 of 0x80000), or 0 < |t| < 2^-6 (E4M3 subnormal range, where the
// midpoints sit elsewhere).  Binade edges hold no midpoint, so one test covers
// every exponent.
__device__ __forceinline__ bool near_e4m3_midpoint(float t) {
    const uint32_t b = __float_as_uint(t);
    const bool near_mid = ((b & 0xFFFFFu) - 0x7FFFCu) < 9u;
    const bool small = ((b & 0x7FFFFFFFu) - 1u) < 0x3C7FFFFFu;
    return near_mid || small;
}

// Eight quotients x/s whose E4M3 codes equal those of the correctly rounded
// quotients.  The fast path multiplies by r = RN(1/s): |x*r - x/s| is at most
// 2^-23 |x/s| + 2^-48 |x/s|, so x*r and RN(x/s) are at most 3 ulps apart and
// round to the same E4M3 code unless x*r lies within 4 ulps of an E4M3
// midpoint (a rounding test in the manner of Ziv's correctly rounded
// elementary functions).  Then, and for tiny scales where r is inexact or
// infinite, the eight values take the IEEE division instead.
__device__ __forceinline__ void quotients8(const uint4& raw, float s, float r, bool zero_group,
                                           bool exact_group, float (&t)[8]) {
    t[0] = bf16_lo(raw.x);
    t[1] = bf16_hi(raw.x);
    t[2] = bf16_lo(raw.y);
    t[3] = bf16_hi(raw.y);
    t[4] = bf16_lo(raw.z);
    t[5] = bf16_hi(raw.z);
    t[6] = bf16_lo(raw.w);
    t[7] = bf16_hi(raw.w);
    if (zero_group) return;  // all +-0: the codes keep the signs
    float f[8];
    bool risky = exact_group;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        f[j] = t[j] * r;
        risky |= near_e4m3_midpoint(f[j]);
    }
    if (risky) {
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = __fdiv_rn(t[j], s);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j] = f[j];
}

__device__ __forceinline__ uint2 pack8(const float (&t)[8]) {
    uint2 out;
    out.x = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
    out.y = e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16);
    return out;
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

constexpr int kQuantRowsPerCta = 32;   // rows of one activation tile
constexpr int kQuantColsPerCta = 256;  // two 128-groups
constexpr int kQuantRowsPerWarp = kQuantRowsPerCta / 8;

// grid = (ceil(M4 / 32), ceil(K / 256)), block = 256 threads.
// Warp w takes rows w, w+8, w+16, w+24 of the tile; lane l takes columns
// 8l .. 8l+7 of the 256, so lanes 0-15 form the first group, 16-31 the second.
__global__ void __launch_bounds__(256)
    k_quantize_groups(const uint16_t* __restrict__ x, int64_t M, int64_t K, int64_t ld_x,
                      uint8_t* __restrict__ q, int64_t ld_q, float* __restrict__ sfa, int64_t M4) {
    __shared__ float s_scale[2][kQuantRowsPerCta];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kQuantRowsPerCta;
    const int64_t col0 = static_cast<int64_t>(blockIdx.y) * kQuantColsPerCta;
    const int64_t groups = K >> 7;
    const bool group_ok = (col0 >> 7) + half < groups;
    const int64_t col = col0 + lane * 8;

    uint4 raw[kQuantRowsPerWarp];
#pragma unroll
    for (int i = 0; i < kQuantRowsPerWarp; ++i) {
        const int64_t r = row0 + warp + 8 * i;
        raw[i] = make_uint4(0u, 0u, 0u, 0u);
        if (r < M && group_ok) raw[i] = ld_nc_v4(x + r * ld_x + col);
    }
#pragma unroll
    for (int i = 0; i < kQuantRowsPerWarp; ++i) {
        float amax = absmax8(raw[i]);
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
        const float s = __fdiv_rn(amax, 448.0f);
        const int64_t r = row0 + warp + 8 * i;
        if (r < M && group_ok) {
            float t[8];
            quotients8(raw[i], s, __frcp_rn(s), amax == 0.0f, !(s >= 0x1p-125f), t);
            *reinterpret_cast<uint2*>(q + r * ld_q + col) = pack8(t);
        }
        if ((lane & 15) == 0) s_scale[half][warp + 8 * i] = s;
    }
    __syncthreads();
    if (threadIdx.x < 2 * kQuantRowsPerCta) {
        const int h = threadIdx.x / kQuantRowsPerCta;
        const int i = threadIdx.x % kQuantRowsPerCta;
        const int64_t g = (col0 >> 7) + h;
        const int64_t r = row0 + i;
        if (g < groups && r < M4) sfa[g * M4 + r] = s_scale[h][i];
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
