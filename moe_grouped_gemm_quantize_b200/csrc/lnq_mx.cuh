// lnq_mx.cuh -- the UE8M0 recipe: power-of-two scales consumed by the tensor core.
//
// The same 1 x 128 activation groups and 128 x 128 weight blocks as the FP32-scale
// recipe, with each scale a power of two stored as an 8-bit exponent (UE8M0, value
// 2^(e - 127)), applied inside tcgen05.mma kind::mxf8f6f4.block_scale instead of
// by FP32 promotion FMAs (deepgemm-rust README, "Blackwell-native FP4/FP8 (SM100a,
// tcgen05)": UE8M0 scales copied shared -> tensor memory with tcgen05.cp
// .32x128b.warpx4 and consumed directly by the block-scaled MMA; "What's
// implemented": gran-128 on either side).
//
// Scale of a group or block: the smallest power of two p with 448 p >= amax, so no
// code saturates; an all-zero group takes p = 1.  With amax = m 2^E (1 <= m < 2),
// p = 2^(E - 8) when m <= 1.75 and 2^(E - 7) otherwise; the exponent is clamped to
// [-127, 127].  Codes are the E4M3 RNE of x / p, exact products by 2^-e.
//
// Scale layout ("scale atoms"): for K block kb and 128-row block rb, 128 32-bit
// words; row r = r0 + 32 r1 of the block (r0 < 32, r1 < 4) owns word 4 r0 + r1,
// whose low byte is the row's exponent byte and whose other bytes are zero.  One
// atom is 512 contiguous bytes, the 32 x 128-bit source of one tcgen05.cp
// .32x128b.warpx4: tensor-memory lane r0 (and its copies in the other three lane
// quarters) receives words 4 r0 .. 4 r0 + 3 in four consecutive columns, and the
// MMA reads row r's scale at lane r, column base + r / 32, byte 0.
//   activations: [K/128][ceil(M/128)][128] words;
//   weights:     [K/128][ceil(N/128)][128] words, every row of a block the block's.
//
// The MXFP8 gran-32 recipe (deepgemm-rust README, benchmark block "SM100 FP8: DeepSeek
// gran-128 recipe and MXFP8 gran-32") uses the same scale rule per 1 x 32 block along K,
// on activations and weights alike, and the same atoms: the word of row r then holds
// the exponent bytes of the row's four 32-blocks of the K block, block j in byte j, and
// the j-th K = 32 MMA of the K block reads byte j (the scale-ID fields of the
// instruction descriptor).
#pragma once

#include <cstdint>
#include <cuda.h>

#include "lnq_ptx.cuh"
#include "lnq_quantize.cuh"

namespace lnq {

// ------------------------------------------------------------------ helpers

// Exponent e of the UE8M0 scale 2^e of a group with largest magnitude amax.
__device__ __forceinline__ int ue8m0_exponent(float amax) {
    const uint32_t b = __float_as_uint(amax);
    const int field = static_cast<int>((b >> 23) & 0xFFu);
    if (field == 0) return amax > 0.0f ? -127 : 0;  // subnormal amax: clamped; zero: p = 1
    const int e = field - 127 - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^-e as a float, e in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float pow2_neg(int e) {
    return e >= 127 ? __uint_as_float(0x00400000u) : __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

// Word of row r within its 128-row scale atom.
__host__ __device__ __forceinline__ int atom_word(int r) { return ((r & 31) << 2) | ((r >> 5) & 3); }

// 1-D bulk copy global -> shared of `bytes` (a multiple of 16, both addresses 16-byte
// aligned), completing its bytes on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

// Shared-memory descriptor of one 512-byte scale atom as the source of tcgen05.cp
// .32x128b: K-major, no swizzle, 32 rows of 16 bytes, 8-row core matrices 128 bytes
// apart (stride byte offset 128 >> 4 = 8 in bits 32-45), the fixed value 1 in bits
// 46-47, layout type 0 (no swizzle) in bits 61-63.
__device__ __forceinline__ uint64_t atom_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(128u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    return d;
}

// tcgen05.cp of a 32 x 128-bit scale atom into tensor-memory columns taddr ..
// taddr + 3 of lanes 0-31, copied to the other three lane quarters.
__device__ __forceinline__ void scale_copy(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// CTA pairs: the pair's leader copies a scale atom from each CTA's shared memory (the
// same offset in both) into the same tensor-memory columns of each CTA.
__device__ __forceinline__ void scale_copy_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Instruction descriptor of tcgen05.mma kind::mxf8f6f4.block_scale for E4M3 x E4M3,
// both K-major, UE8M0 scales: B scale byte id 0 (bits 4-5), A and B formats 0 (E4M3,
// bits 7-9 and 10-12), N >> 3 in bits 17-22, scale format 1 (E8M0) in bit 23,
// M >> 4 in bits 24-28, A scale byte id 0 (bits 29-30), K = 32 (bit 31 = 0).
__host__ __device__ constexpr uint32_t mxf8_idesc(int M, int N) {
    return (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) | (static_cast<uint32_t>(M >> 4) << 24);
}

// The same descriptor with scale byte j for both operands (A's scale ID in bits 29-30,
// B's in bits 4-5): the j-th K = 32 step of a K block under 1 x 32 scales.
__host__ __device__ constexpr uint32_t mxf8_idesc_byte(uint32_t idesc, int j) {
    return idesc | (static_cast<uint32_t>(j) << 29) | (static_cast<uint32_t>(j) << 4);
}

// D[tmem] (+)= (A * 2^sa) (B * 2^sb)^T over K = 32, the scales read from tensor memory.
__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// The same over a CTA pair (M = 256): each CTA holds its 128 rows of A, its half of B
// and, in its own tensor memory, the scales of its A rows and of all N columns of B.
__device__ __forceinline__ void mma_mxf8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// ------------------------------------------------------------------ quantize

// Activations: every half warp quantizes four consecutive 1 x 128 groups per step
// (8 inputs per lane and group; the four 16-byte loads of a lane are issued before
// any reduction, so they are in flight together).  Rows M .. Mpad-1 only get the
// scale word of p = 1.
__global__ void __launch_bounds__(256) k_quantize_ue8m0_groups(const uint16_t* __restrict__ x, int M, int K,
                                                               long long ld_x, uint8_t* __restrict__ q,
                                                               long long ld_q, uint32_t* __restrict__ sf,
                                                               int Mpad) {
    constexpr int kPerHalf = 4;
    wait_prior_grids();
    launch_dependents();
    const int G = K / 128;
    const long long units = static_cast<long long>(Mpad) * G;
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4, l16 = lane & 15;
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
    const long long warp = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int rblocks = Mpad / 128;
    for (long long base = warp * 2 * kPerHalf; base < units; base += warps * 2 * kPerHalf) {
        uint4 raw[kPerHalf];
        int m[kPerHalf], g[kPerHalf];
        bool valid[kPerHalf], real[kPerHalf];
#pragma unroll
        for (int j = 0; j < kPerHalf; ++j) {
            const long long u = base + half * kPerHalf + j;
            valid[j] = u < units;
            m[j] = valid[j] ? static_cast<int>(u / G) : 0;
            g[j] = valid[j] ? static_cast<int>(u % G) : 0;
            real[j] = valid[j] && m[j] < M;
            raw[j] = make_uint4(0u, 0u, 0u, 0u);
            if (real[j]) raw[j] = ld_nc_v4(x + m[j] * ld_x + g[j] * 128 + l16 * 8);
        }
#pragma unroll
        for (int j = 0; j < kPerHalf; ++j) {
            float amax = absmax8(raw[j]);
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const int e = ue8m0_exponent(amax);
            if (real[j]) {
                const float r = pow2_neg(e);
                float t[8];
                t[0] = bf16_lo(raw[j].x) * r;
                t[1] = bf16_hi(raw[j].x) * r;
                t[2] = bf16_lo(raw[j].y) * r;
                t[3] = bf16_hi(raw[j].y) * r;
                t[4] = bf16_lo(raw[j].z) * r;
                t[5] = bf16_hi(raw[j].z) * r;
                t[6] = bf16_lo(raw[j].w) * r;
                t[7] = bf16_hi(raw[j].w) * r;
                *reinterpret_cast<uint2*>(q + m[j] * ld_q + g[j] * 128 + l16 * 8) = pack8(t);
            }
            if (valid[j] && l16 == 0)
                sf[(static_cast<long long>(g[j]) * rblocks + m[j] / 128) * 128 + atom_word(m[j] & 127)] =
                    static_cast<uint32_t>(e + 127);
        }
    }
}

// Weights: one CTA of 256 threads per 128 x 128 block; rows past N take no part in
// the amax, and every row of the block's atom gets the block's exponent.
__global__ void __launch_bounds__(256) k_quantize_ue8m0_blocks(const uint16_t* __restrict__ w, int N, int K,
                                                               uint8_t* __restrict__ q, uint32_t* __restrict__ sf,
                                                               int nblocks) {
    __shared__ float warp_max[8];
    const int KB = K / 128;
    const int nb = blockIdx.x / KB, kb = blockIdx.x % KB;
    const int tid = threadIdx.x;
    const int col = kb * 128 + (tid & 15) * 8;
    uint4 raw[8];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int n = nb * 128 + (tid >> 4) + 16 * i;
        raw[i] = make_uint4(0u, 0u, 0u, 0u);
        if (n < N) raw[i] = ld_nc_v4(w + static_cast<long long>(n) * K + col);
        amax = fmaxf(amax, absmax8(raw[i]));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((tid & 31) == 0) warp_max[tid >> 5] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, warp_max[i]);
    const int e = ue8m0_exponent(amax);
    const float r = pow2_neg(e);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int n = nb * 128 + (tid >> 4) + 16 * i;
        if (n < N) {
            float t[8];
            t[0] = bf16_lo(raw[i].x) * r;
            t[1] = bf16_hi(raw[i].x) * r;
            t[2] = bf16_lo(raw[i].y) * r;
            t[3] = bf16_hi(raw[i].y) * r;
            t[4] = bf16_lo(raw[i].z) * r;
            t[5] = bf16_hi(raw[i].z) * r;
            t[6] = bf16_lo(raw[i].w) * r;
            t[7] = bf16_hi(raw[i].w) * r;
            *reinterpret_cast<uint2*>(q + static_cast<long long>(n) * K + col) = pack8(t);
        }
    }
    if (tid < 128) sf[(static_cast<long long>(kb) * nblocks + nb) * 128 + atom_word(tid)] = static_cast<uint32_t>(e + 127);
}

// MXFP8 gran-32: every row in 1 x 32 blocks.  As the gran-128 activation quantizer, a
// half warp takes four consecutive 128-groups of a row per step, 8 inputs per lane and
// group; the four lanes of a 32-block reduce its amax by two shuffles, and the block's
// first lane writes its exponent byte into byte (block within the group) of the row's
// atom word.  Rows R .. Rpad-1 get the word of p = 1 in all four bytes.
__global__ void __launch_bounds__(256) k_quantize_mxfp8(const uint16_t* __restrict__ x, int R, int K, long long ld_x,
                                                        uint8_t* __restrict__ q, long long ld_q,
                                                        uint32_t* __restrict__ sf, int Rpad) {
    constexpr int kPerHalf = 4;
    wait_prior_grids();
    launch_dependents();
    const int G = K / 128;
    const long long units = static_cast<long long>(Rpad) * G;
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4, l16 = lane & 15;
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
    const long long warp = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int rblocks = Rpad / 128;
    uint8_t* sf_bytes = reinterpret_cast<uint8_t*>(sf);
    for (long long base = warp * 2 * kPerHalf; base < units; base += warps * 2 * kPerHalf) {
        uint4 raw[kPerHalf];
        int m[kPerHalf], g[kPerHalf];
        bool valid[kPerHalf], real[kPerHalf];
#pragma unroll
        for (int j = 0; j < kPerHalf; ++j) {
            const long long u = base + half * kPerHalf + j;
            valid[j] = u < units;
            m[j] = valid[j] ? static_cast<int>(u / G) : 0;
            g[j] = valid[j] ? static_cast<int>(u % G) : 0;
            real[j] = valid[j] && m[j] < R;
            raw[j] = make_uint4(0u, 0u, 0u, 0u);
            if (real[j]) raw[j] = ld_nc_v4(x + m[j] * ld_x + g[j] * 128 + l16 * 8);
        }
#pragma unroll
        for (int j = 0; j < kPerHalf; ++j) {
            float amax = absmax8_packed(raw[j]);
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            const int e = ue8m0_exponent(amax);
            const long long word = (static_cast<long long>(g[j]) * rblocks + m[j] / 128) * 128 + atom_word(m[j] & 127);
            if (real[j]) {
                const float r = pow2_neg(e);
                float t[8];
                t[0] = bf16_lo(raw[j].x) * r;
                t[1] = bf16_hi(raw[j].x) * r;
                t[2] = bf16_lo(raw[j].y) * r;
                t[3] = bf16_hi(raw[j].y) * r;
                t[4] = bf16_lo(raw[j].z) * r;
                t[5] = bf16_hi(raw[j].z) * r;
                t[6] = bf16_lo(raw[j].w) * r;
                t[7] = bf16_hi(raw[j].w) * r;
                *reinterpret_cast<uint2*>(q + m[j] * ld_q + g[j] * 128 + l16 * 8) = pack8(t);
                if ((l16 & 3) == 0) sf_bytes[word * 4 + (l16 >> 2)] = static_cast<uint8_t>(e + 127);
            } else if (valid[j] && l16 == 0) {
                sf[word] = 0x7F7F7F7Fu;
            }
        }
    }
}

// ------------------------------------------------------------------ GEMM

struct MxArgs {
    const uint32_t* sfa;   // activation scale atoms [K/128][ceil(M/128)][128]
    const uint32_t* sfb;   // weight scale atoms [K/128][ceil(rows of B / 128)][128]
    uint16_t* d;           // [M][N] bf16 bits
    unsigned int* status;  // device status word
    unsigned long long timeout_ns;
    int M, N, num_kb;
    int mblocks, nblocks;  // ceil(M/128), ceil(rows of B / 128)
    int tiles_p, tiles_q, num_tiles;
    // M-grouped contiguous layout (GROUPED): each 128-row block of A takes the weights
    // of the group named by its first row's id (rows g*N .. g*N + N - 1 of B, N % 128
    // == 0); a block led by a negative id is skipped.
    const int32_t* m_indices;
    int num_groups;
    // M-grouped masked layout (GROUPED, m_indices == nullptr): group g owns rows
    // g*m_max .. g*m_max + m_max - 1 of A and D, of which the first masked_m[g] are real;
    // blocks past the count are skipped and stores stop at it.
    const int32_t* masked_m;  // [num_groups], on the device
    int m_max;                // rows per group, a multiple of 128
};

// One persistent CTA per SM, tiles of 128 rows x 256 columns (256 x 256 on CTA pairs), 384
// threads:
//   warp 0      TMA producer: per K block the A and B boxes and the three scale atoms
//               (A's, and B's two 128-row halves) of the tile on one barrier;
//   warp 1      tensor memory (512 columns) and the MMA issuer: per K block three
//               tcgen05.cp of the scale atoms into the stage's scale columns, then
//               four block-scaled MMAs of K = 32 into the tile's accumulator;
//   warps 4-11  epilogue: after the tile's last K block, read the 128 x 256 FP32
//               accumulator, release it, round to bf16 and store.
// With GROUPED, a 128-row block of A takes its group's weights (the M-grouped
// contiguous MoE layout, deepgemm-rust README, "Grouped (contiguous) MoE GEMM").
// Tensor memory: the accumulator in columns 0-255; stage s's A scales in columns
// 256 + 16 s .. + 3 and its B scales in 256 + 16 s + 4 .. + 11.  The scales are
// applied by the tensor core, so no promotion FMAs run and the accumulator is read
// once per tile; its single buffer costs the MMA one readout per tile.
// PAIR (dense): a cluster of two CTAs runs one tcgen05.mma.cta_group::2 of 256 x 256; each
// CTA loads its 128 rows of A, 128 of the 256 rows of B, its A rows' scale atom and both of
// B's atoms, all by TMA onto the first CTA's barrier, whose MMA warp copies the atoms
// into both CTAs' tensor memory and issues the pair's MMAs.  Each SM then loads 32 KB of
// operands per K block instead of 48 KB.
template <int STAGES, bool PAIR = false>
struct MxCfg {
    static constexpr int kBK = 128;
    static constexpr int kABytes = 128 * kBK;
    static constexpr int kBRows = PAIR ? 128 : 256;
    static constexpr int kBBytes = kBRows * kBK;
    static constexpr int kSfBytes = 3 * 512;
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + STAGES * kABytes;
    static constexpr int kOffSf = kOffB + STAGES * kBBytes;
    static constexpr int kOffBar = kOffSf + STAGES * kSfBytes;
    static constexpr int kNumBars = 2 * STAGES + 3;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
    static constexpr int kThreads = 384;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kSfCol0 = 256;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(kSfCol0 + 16 * STAGES <= kTmemCols, "scale columns");
};

// map_sfa and map_sfb (CTA pairs only) view the scale atoms as rows of 128 words: rows
// kb * mblocks + mb of A's, kb * nblocks + nb of B's.
template <int STAGES, bool GROUPED = false, bool GRAN32 = false, bool PAIR = false>
__global__ void __launch_bounds__(384, 1)
    k_mx_block_gemm(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                    const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
                    const MxArgs args) {
    static_assert(!(PAIR && GROUPED), "CTA pairs serve the dense product");
    using C = MxCfg<STAGES, PAIR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sA = s_base + C::kOffA;
    const uint32_t sB = s_base + C::kOffB;
    const uint32_t sSf = s_base + C::kOffSf;
    const uint32_t bars = s_base + C::kOffBar;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
    const uint32_t tfull_bar = bars + 8u * (2 * STAGES);
    const uint32_t tempty_bar = tfull_bar + 8u;
    const uint32_t drain_bar = tfull_bar + 16u;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile uint32_t* abort_flag = misc + 1;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // CTA pairs: rank in the pair; tiles are numbered per pair
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(tfull_bar, 1);
        mbar_init(tempty_bar, PAIR ? 16 : 8);
        mbar_init(drain_bar, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_u32(misc), C::kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(misc), C::kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if constexpr (PAIR) cluster_sync();  // the peer's barriers exist before any remote signal
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    launch_dependents();
    wait_prior_grids();

    WaitCtx wctx;
    wctx.abort = abort_flag;
    wctx.status = args.status;
    wctx.timeout_ns = args.timeout_ns;

    // banded raster, column-major inside bands of row tiles (16 dense, 8 grouped: the
    // blocks of a group walk its weight columns together).  Returns the tile's group
    // (0 dense; -1 for a grouped block to skip), its first row of B and the end of its
    // rows that are stored (rows from row_end on stay untouched).
    auto tile_rc = [&](int t, int& p0, int& q0, int& b_row, int& row_end) {
        constexpr int kBand = GROUPED ? 8 : 16;
        const int band_tiles = kBand * args.tiles_q;
        const int band = t / band_tiles;
        const int first = band * kBand;
        const int rows = min(args.tiles_p - first, kBand);
        const int r = t - band * band_tiles;
        p0 = (first + r % rows) * (PAIR ? 256 : 128) + static_cast<int>(rank) * 128;
        q0 = (r / rows) * 256;
        row_end = args.M;
        int g = 0;
        if constexpr (GROUPED) {
            if (args.m_indices != nullptr) {
                g = __ldg(args.m_indices + p0);
                if (g >= args.num_groups) {
                    atomicOr(args.status, kStatusBadGroup);
                    g = -1;
                }
            } else {
                // masked: group g's first masked_m[g] rows are real
                g = p0 / args.m_max;
                int count = __ldg(args.masked_m + g);
                if (count < 0 || count > args.m_max) {
                    atomicOr(args.status, kStatusBadGroup);
                    count = count < 0 ? 0 : args.m_max;
                }
                const int valid = g * args.m_max + count - p0;
                row_end = p0 + (valid < 128 ? valid : 128);
                if (valid <= 0) g = -1;
            }
        }
        b_row = (g < 0 ? 0 : g) * args.N + q0;
        return g;
    };

    if (warp < 4) {
        setmaxnreg_dec<56>();
        if (warp == 0) {
            // ---------------------------------------------------------------- producer
            if (elect_one()) {
                tma_prefetch_desc(&map_a);
                tma_prefetch_desc(&map_b);
                if constexpr (PAIR) {
                    tma_prefetch_desc(&map_sfa);
                    tma_prefetch_desc(&map_sfb);
                }
            }
            __syncwarp();
            int stage = 0;
            uint32_t phase = 0, filled = 0, fill_parity = 0;
            bool ok = true;
            for (int t = unit; ok && t < args.num_tiles; t += units) {
                int p0, q0, b_row, row_end;
                if (tile_rc(t, p0, q0, b_row, row_end) < 0) continue;
                const int mb = p0 / 128;
                const int nb0 = b_row / 128;
                const int nb1 = min(nb0 + 1, args.nblocks - 1);
                for (int kb = 0; kb < args.num_kb; ++kb) {
                    if (!mbar_wait_warp(empty_bar(stage), phase ^ 1u, wctx)) {
                        ok = false;
                        break;
                    }
                    if (elect_one()) {
                        const uint32_t sf = sSf + stage * C::kSfBytes;
                        if constexpr (PAIR) {
                            // both CTAs' bytes complete on the first CTA's full barrier; B's two
                            // atoms are adjacent rows of its atom view (a second row past the
                            // last block only scales columns past N, which are never stored)
                            const uint32_t fb = mapa_shared(full_bar(stage), 0);
                            if (rank == 0)
                                mbar_arrive_expect_tx(full_bar(stage), 2 * (C::kABytes + C::kBBytes + C::kSfBytes));
                            tma_load_2d_pair(sA + stage * C::kABytes, &map_a, fb, kb * C::kBK, p0);
                            tma_load_2d_pair(sB + stage * C::kBBytes, &map_b, fb, kb * C::kBK,
                                             b_row + static_cast<int>(rank) * 128);
                            tma_load_2d_pair(sf, &map_sfa, fb, 0, kb * args.mblocks + mb);
                            tma_load_2d_pair(sf + 512u, &map_sfb, fb, 0, kb * args.nblocks + nb0);
                        } else {
                            const uint32_t fb = full_bar(stage);
                            mbar_arrive_expect_tx(fb, C::kABytes + C::kBBytes + C::kSfBytes);
                            tma_load_2d(sA + stage * C::kABytes, &map_a, fb, kb * C::kBK, p0);
                            tma_load_2d(sB + stage * C::kBBytes, &map_b, fb, kb * C::kBK, b_row);
                            const long long kbase = static_cast<long long>(kb);
                            bulk_load(sf, args.sfa + (kbase * args.mblocks + mb) * 128, 512u, fb);
                            bulk_load(sf + 512u, args.sfb + (kbase * args.nblocks + nb0) * 128, 512u, fb);
                            bulk_load(sf + 1024u, args.sfb + (kbase * args.nblocks + nb1) * 128, 512u, fb);
                        }
                    }
                    __syncwarp();
                    filled |= 1u << stage;
                    fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // the copies already issued land before the CTA can leave (a pair's second
                // CTA cannot see the first's barriers: it waits out a fixed delay)
                const uint64_t t0 = global_timer_ns();
                if (PAIR && rank != 0) {
                    while (global_timer_ns() - t0 < 200000ull) {
                    }
                } else {
                    WaitCtx drain = wctx;
                    uint32_t never = 0u;
                    drain.abort = &never;
                    for (int s = 0; s < STAGES; ++s)
                        if (filled & (1u << s)) (void)mbar_wait_warp(full_bar(s), (fill_parity >> s) & 1u, drain);
                    if (PAIR) {
                        while (global_timer_ns() - t0 < 200000ull) {
                        }
                    }
                }
            }
        } else if (warp == 1 && rank == 0) {
            // ---------------------------------------------------------------- MMA
            constexpr uint32_t kIdesc = mxf8_idesc(PAIR ? 256 : 128, 256);
            const uint64_t adesc0 = sw128_kmajor_desc(sA);
            const uint64_t bdesc0 = sw128_kmajor_desc(sB);
            int stage = 0;
            uint32_t phase = 0, aphase = 0;
            bool ok = true;
            for (int t = unit; ok && t < args.num_tiles; t += units) {
                int p0, q0, b_row, row_end;
                if (tile_rc(t, p0, q0, b_row, row_end) < 0) continue;
                // the epilogue has read the previous tile's accumulator
                if (!mbar_wait_warp(tempty_bar, aphase ^ 1u, wctx)) break;
                tc_fence_after();
                for (int kb = 0; kb < args.num_kb; ++kb) {
                    if (!mbar_wait_warp(full_bar(stage), phase, wctx)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sfa_t = tmem_base + C::kSfCol0 + 16u * stage;
                    const uint32_t sfb_t = sfa_t + 4u;
                    if (elect_one()) {
                        const uint32_t sf = sSf + stage * C::kSfBytes;
                        const uint64_t adesc = adesc0 + static_cast<uint64_t>((stage * C::kABytes) >> 4);
                        const uint64_t bdesc = bdesc0 + static_cast<uint64_t>((stage * C::kBBytes) >> 4);
                        if constexpr (PAIR) {
                            scale_copy_pair(sfa_t, atom_desc(sf));
                            scale_copy_pair(sfb_t, atom_desc(sf + 512u));
                            scale_copy_pair(sfb_t + 4u, atom_desc(sf + 1024u));
#pragma unroll
                            for (int k = 0; k < C::kBK / 32; ++k)
                                mma_mxf8_pair(tmem_base, adesc + 2u * k, bdesc + 2u * k,
                                              GRAN32 ? mxf8_idesc_byte(kIdesc, k) : kIdesc, sfa_t, sfb_t,
                                              (kb > 0 || k > 0) ? 1u : 0u);
                            mma_commit_pair(mapa_shared(empty_bar(stage), 0));
                            mma_commit_pair(mapa_shared(empty_bar(stage), 1));
                            if (kb + 1 == args.num_kb) {
                                mma_commit_pair(mapa_shared(tfull_bar, 0));
                                mma_commit_pair(mapa_shared(tfull_bar, 1));
                            }
                        } else {
                            scale_copy(sfa_t, atom_desc(sf));
                            scale_copy(sfb_t, atom_desc(sf + 512u));
                            scale_copy(sfb_t + 4u, atom_desc(sf + 1024u));
#pragma unroll
                            for (int k = 0; k < C::kBK / 32; ++k)
                                mma_mxf8(tmem_base, adesc + 2u * k, bdesc + 2u * k,
                                         GRAN32 ? mxf8_idesc_byte(kIdesc, k) : kIdesc, sfa_t, sfb_t,
                                         (kb > 0 || k > 0) ? 1u : 0u);
                            mma_commit(empty_bar(stage));
                            if (kb + 1 == args.num_kb) mma_commit(tfull_bar);
                        }
                    }
                    __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                aphase ^= 1u;
            }
            // every MMA and copy completes before tensor memory is released
            if (elect_one()) {
                if constexpr (PAIR) mma_commit_pair(mapa_shared(drain_bar, 0));
                else mma_commit(drain_bar);
            }
            __syncwarp();
            WaitCtx drain = wctx;
            uint32_t never = 0u;
            drain.abort = &never;
            (void)mbar_wait_warp(drain_bar, 0u, drain);
        }
    } else {
        // -------------------------------------------------------------------- epilogue
        setmaxnreg_inc<224>();
        const int wg = (warp - 4) >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t aphase = 0;
        for (int t = unit; t < args.num_tiles; t += units) {
            int p0, q0, b_row, row_end;
            if (tile_rc(t, p0, q0, b_row, row_end) < 0) continue;
            if (!mbar_wait_warp(tfull_bar, aphase, wctx)) break;
            tc_fence_after();
            uint32_t ra[64], rb[64];
            const uint32_t taddr = tmem_base + t_lane + static_cast<uint32_t>(wg * 128);
            tmem_ld_async(taddr, ra);
            tmem_ld_async(taddr + 64u, rb);
            tmem_wait_ld(ra);
            tmem_wait_ld(rb);
            // the accumulator may take the next tile
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR) mbar_arrive_cluster_relaxed(mapa_shared(tempty_bar, 0));
                else mbar_arrive(tempty_bar);
            }
            aphase ^= 1u;
            const int m = p0 + row;
            const int n0 = q0 + wg * 128;
            if (m < row_end) {
                uint16_t* drow = args.d + static_cast<long long>(m) * args.N;
                auto store8 = [&](int n, const uint32_t (&r)[64], int i) {
                    if (n < args.N) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(r[i + 0]), __uint_as_float(r[i + 1]));
                        v.y = pack_bf16x2(__uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
                        v.z = pack_bf16x2(__uint_as_float(r[i + 4]), __uint_as_float(r[i + 5]));
                        v.w = pack_bf16x2(__uint_as_float(r[i + 6]), __uint_as_float(r[i + 7]));
                        *reinterpret_cast<uint4*>(drow + n) = v;
                    }
                };
#pragma unroll
                for (int c = 0; c < 8; ++c) store8(n0 + c * 8, ra, c * 8);
#pragma unroll
                for (int c = 0; c < 8; ++c) store8(n0 + 64 + c * 8, rb, c * 8);
            }
        }
    }

    if constexpr (PAIR) {
        // no CTA leaves while its peer may still signal its barriers or read its TMEM
        tc_fence_before();
        cluster_sync();
        if (warp == 1) {
            tc_fence_after();
            tmem_dealloc_pair(tmem_base, C::kTmemCols);
        }
    } else {
        __syncthreads();
        if (warp == 1) {
            tc_fence_after();
            tmem_dealloc(tmem_base, C::kTmemCols);
        }
    }
}

}  // namespace lnq
