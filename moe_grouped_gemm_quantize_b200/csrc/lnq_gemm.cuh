// lnq_gemm.cuh -- block-scaled FP8 GEMM "nt" on sm_100a tensor cores.
//
// D[m][n] = bf16( sum_g sfa[g][m] * sfb[n/128][g] * sum_{k in g} a[m][k] * b[n][k] )
// (deepgemm-rust README, "What's implemented": per-(1x128) activation scales
// x per-(128x128) weight scales, FP32 promotion, BF16 out).
//
// One persistent, warp-specialized kernel serves three shapes:
//   * dense (M > 64): the MMA's M slot ("P operand") holds 128 activation rows,
//     its N slot ("Q operand") BNQ weight rows;
//   * M-grouped contiguous (MoE): as dense, each 128-row block of activations
//     takes the weights of the group named by its first row's id
//     (deepgemm-rust README, "Grouped (contiguous) MoE GEMM");
//   * decode (M <= 64, "swap AB"): the weights fill the 128-row M slot and the
//     few tokens the N slot, so the tensor core is not idle on padding rows.
//
// Roles (warps of one CTA):
//   warp 0      TMA producer: P and Q tiles of one 128-wide K block per stage
//               into a ring of shared-memory stages (128-byte swizzle).
//   warp 1      allocates tensor memory; one lane issues tcgen05.mma
//               kind::f8f6f4 (E4M3 x E4M3 -> FP32), 4 MMAs of K=32 per K block,
//               into one of two TMEM accumulators that alternate per K block.
//   warp 2      scale producer: loads the K block's activation and weight
//               scales into a small shared-memory ring.
//   warps 4..   epilogue: per K block, reads the FP32 partial product from TMEM
//               (tcgen05.ld), multiplies it by sa*sb and adds it into FP32
//               registers (the per-K-block promotion); after the last K block
//               converts to bf16 (round to nearest even) and stores the tile.
// The two TMEM accumulators let the tensor core run the next K block while
// the epilogue promotes the previous one.  All waits are bounded (mbar_wait).
#pragma once

#include <cstdint>
#include <cuda.h>

#include "lnq_ptx.cuh"

namespace lnq {

struct GemmArgs {
    const float* sfa;         // [K/128][M4]
    const float* sfb;         // [groups * NB][K/128]
    uint16_t* d;              // [M][N] bf16 bits
    const int32_t* m_indices; // grouped only: [M]
    unsigned int* status;     // device status word
    unsigned long long timeout_ns;
    long long M4;
    int M;            // activation rows (M_total for grouped)
    int N;            // output columns (per group for grouped)
    int num_kb;       // K / 128
    int nb;           // ceil(N / 128): weight scale rows per group
    int num_groups;   // grouped only
    int tiles_p;      // tiles along the MMA M slot
    int tiles_q;      // tiles along the MMA N slot
    int num_tiles;
};

constexpr unsigned int kStatusBadGroup = 2u;

template <int BNQ_, int STAGES_, int EPI_WG_, bool SWAP_, bool GROUPED_>
struct GemmCfg {
    static constexpr int BNQ = BNQ_;
    static constexpr int STAGES = STAGES_;
    static constexpr int EPI_WG = EPI_WG_;
    static constexpr bool SWAP = SWAP_;
    static constexpr bool GROUPED = GROUPED_;
    static_assert(!(SWAP && GROUPED), "decode configuration is dense only");
    static_assert(BNQ % 16 == 0 && BNQ >= 16 && BNQ <= 256, "MMA N for M=128");
    static_assert(!SWAP || EPI_WG == 1, "decode epilogue: one thread per weight row");
    static_assert(!SWAP || BNQ % 32 == 0, "decode tiles read TMEM in 32-column chunks");
    static_assert(SWAP || BNQ % 128 == 0, "dense tiles cover whole 128-column scale blocks");

    static constexpr int kP = 128;                // MMA M
    static constexpr int kBK = 128;               // K elements (bytes) per stage
    static constexpr int kPBytes = kP * kBK;
    static constexpr int kQBytes = BNQ * kBK;
    static constexpr int kScaleStages = 8;
    static constexpr int kCW = BNQ / EPI_WG;      // accumulator columns per epilogue thread
    static constexpr int kEpiThreads = 128 * EPI_WG;
    static constexpr int kThreads = 128 + kEpiThreads;
    static constexpr int kTmemCols = (2 * BNQ < 32) ? 32 : 2 * BNQ;
    static constexpr int kSbPerTile = SWAP ? 1 : BNQ / 128;
    static constexpr int kSaPerTile = SWAP ? BNQ : kP;
    static constexpr uint32_t kIdesc = f8f6f4_e4m3_idesc(kP, BNQ);
    static constexpr bool kRegSplit = (!SWAP && kCW == 128);

    // shared-memory layout (offsets from a 1024-byte aligned base)
    static constexpr int kOffP = 0;
    static constexpr int kOffQ = kOffP + STAGES * kPBytes;
    static constexpr int kOffScale = kOffQ + STAGES * kQBytes;
    static constexpr int kScaleSlotFloats = 256 + 4;
    static constexpr int kOffBar = kOffScale + kScaleStages * kScaleSlotFloats * 4;
    static constexpr int kNumBars = 2 * STAGES + 4 + 2 * kScaleStages + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(kQBytes % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
};

struct TileCoord {
    int p0;     // first row of the P operand (activation row, or weight row for SWAP)
    int q0;     // first row of the Q operand (weight row within the group, or token)
    int group;  // grouped: group id of the tile, -1 skip; else 0
};

template <class C>
__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& a, int t) {
    TileCoord c;
    if constexpr (C::SWAP) {
        c.p0 = (t % a.tiles_p) * C::kP;
        c.q0 = (t / a.tiles_p) * C::BNQ;
        c.group = 0;
    } else if constexpr (C::GROUPED) {
        // row-major over (128-row block, column tile): consecutive tiles share
        // the activation block and walk one group's weights, which stay in L2
        c.p0 = (t / a.tiles_q) * C::kP;
        c.q0 = (t % a.tiles_q) * C::BNQ;
        c.group = __ldg(a.m_indices + c.p0);
        if (c.group >= a.num_groups) {
            atomicOr(a.status, kStatusBadGroup);
            c.group = -1;
        }
    } else {
        // bands of 16 row blocks: a wave of tiles shares 16 activation blocks
        // and a few weight column tiles
        constexpr int kBand = 16;
        const int band_tiles = kBand * a.tiles_q;
        const int band = t / band_tiles;
        const int first = band * kBand;
        const int rows = min(a.tiles_p - first, kBand);
        const int r = t - band * band_tiles;
        c.p0 = (first + r % rows) * C::kP;
        c.q0 = (r / rows) * C::BNQ;
        c.group = 0;
    }
    return c;
}

// One K block of the per-block FP32 promotion: acc += partial * scale, where
// the partial is this thread's TMEM lane (kCW columns starting at taddr).
// TMEM loads are issued one 32-column chunk ahead of the packed (f32x2) FMAs
// that consume the previous chunk.
//   dense:  scale = sa[row] * sb[column block of this warpgroup]
//   decode: scale = sa[token j] * sb[weight block of the tile], per column j
template <class C>
__device__ __forceinline__ void promote_k_block(float2 (&acc)[C::kCW / 2], uint32_t taddr,
                                                const float* slot, int row, int wg) {
    constexpr int NC = C::kCW / 32;
    float2 s2;
    float sb = 0.f;
    if constexpr (!C::SWAP) {
        const float s = slot[row] * slot[256 + (wg * C::kCW) / 128];
        s2 = make_float2(s, s);
    } else {
        sb = slot[256];
        s2 = make_float2(sb, sb);
    }
    uint32_t ra[32], rb[32];
    tmem_ld32_async(taddr, ra);
    tmem_wait_ld(ra);
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        if (c + 1 < NC) {
            if (c & 1) tmem_ld32_async(taddr + (c + 1) * 32, ra);
            else tmem_ld32_async(taddr + (c + 1) * 32, rb);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t lo = (c & 1) ? rb[2 * i] : ra[2 * i];
            const uint32_t hi = (c & 1) ? rb[2 * i + 1] : ra[2 * i + 1];
            const float2 v = make_float2(__uint_as_float(lo), __uint_as_float(hi));
            float2 sc = s2;
            if constexpr (C::SWAP) {
                const float2 sa = *reinterpret_cast<const float2*>(slot + c * 32 + 2 * i);
                sc = __fmul2_rn(sa, s2);
            }
            acc[c * 16 + i] = __ffma2_rn(v, sc, acc[c * 16 + i]);
        }
        if (c + 1 < NC) {
            if (c & 1) tmem_wait_ld(ra);
            else tmem_wait_ld(rb);
        }
    }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    k_fp8_block_gemm(const __grid_constant__ CUtensorMap map_p,
                     const __grid_constant__ CUtensorMap map_q, const GemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sP = s_base + C::kOffP;
    const uint32_t sQ = s_base + C::kOffQ;
    float* scale_slots = reinterpret_cast<float*>(smem + C::kOffScale);
    const uint32_t bars = s_base + C::kOffBar;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (C::STAGES + s); };
    auto tfull_bar = [&](int b) { return bars + 8u * (2 * C::STAGES + b); };
    auto tempty_bar = [&](int b) { return bars + 8u * (2 * C::STAGES + 2 + b); };
    auto sfull_bar = [&](int s) { return bars + 8u * (2 * C::STAGES + 4 + s); };
    auto sempty_bar = [&](int s) { return bars + 8u * (2 * C::STAGES + 4 + C::kScaleStages + s); };
    const uint32_t drain_bar = bars + 8u * (2 * C::STAGES + 4 + 2 * C::kScaleStages);
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile uint32_t* abort_flag = misc + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), C::kEpiThreads / 32);
        }
        for (int s = 0; s < C::kScaleStages; ++s) {
            mbar_init(sfull_bar(s), 32);
            mbar_init(sempty_bar(s), C::kEpiThreads / 32);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(misc), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];

    WaitCtx wctx;
    wctx.abort = abort_flag;
    wctx.status = args.status;
    wctx.timeout_ns = args.timeout_ns;

    if (warp < 4) {
    // control warpgroup: registers handed to the epilogue warpgroups
    if constexpr (C::kRegSplit) setmaxnreg_dec<56>();
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&map_p);
            tma_prefetch_desc(&map_q);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0, fill_parity = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
                const TileCoord tc = tile_coord<C>(args, t);
                if (tc.group < 0) continue;
                int p_row, q_row;
                if constexpr (C::SWAP) {
                    p_row = tc.p0;
                    q_row = tc.q0;
                } else {
                    p_row = tc.p0;
                    q_row = tc.group * args.N + tc.q0;
                }
                for (int kb = 0; kb < args.num_kb; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, wctx)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full_bar(stage), C::kPBytes + C::kQBytes);
                    tma_load_2d(sP + stage * C::kPBytes, &map_p, full_bar(stage), kb * C::kBK, p_row);
                    tma_load_2d(sQ + stage * C::kQBytes, &map_q, full_bar(stage), kb * C::kBK, q_row);
                    filled |= 1u << stage;
                    fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA can exit
                WaitCtx drain = wctx;
                uint32_t never = 0u;
                drain.abort = &never;
                for (int s = 0; s < C::STAGES; ++s)
                    if (filled & (1u << s)) (void)mbar_wait(full_bar(s), (fill_parity >> s) & 1u, drain);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, abuf = 0;
            uint32_t phase = 0, aphase = 0;
            bool ok = true, issued = false;
            for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
                const TileCoord tc = tile_coord<C>(args, t);
                if (tc.group < 0) continue;
                for (int kb = 0; kb < args.num_kb; ++kb) {
                    if (!mbar_wait(tempty_bar(abuf), aphase ^ 1u, wctx) ||
                        !mbar_wait(full_bar(stage), phase, wctx)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * C::BNQ);
                    const uint64_t adesc = sw128_kmajor_desc(sP + stage * C::kPBytes);
                    const uint64_t bdesc = sw128_kmajor_desc(sQ + stage * C::kQBytes);
#pragma unroll
                    for (int k = 0; k < C::kBK / 32; ++k)
                        mma_f8f6f4(d_tmem, adesc + 2u * k, bdesc + 2u * k, C::kIdesc, k > 0 ? 1u : 0u);
                    mma_commit(empty_bar(stage));
                    mma_commit(tfull_bar(abuf));
                    issued = true;
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    abuf ^= 1;
                    if (abuf == 0) aphase ^= 1u;
                }
            }
            if (issued) {
                // every MMA this thread issued completes before TMEM is released
                mma_commit(drain_bar);
                WaitCtx drain = wctx;
                uint32_t never = 0u;
                drain.abort = &never;
                (void)mbar_wait(drain_bar, 0u, drain);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ scale producer
        int sstage = 0;
        uint32_t sphase = 0;
        bool ok = true;
        constexpr int kBatch = 4;
        constexpr int kSaLanes = C::kSaPerTile / 4;  // lanes that load a float4 of sa
        for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
            const TileCoord tc = tile_coord<C>(args, t);
            if (tc.group < 0) continue;
            // activation rows of the tile (tokens for SWAP) and weight scale rows
            const long long a_row0 = C::SWAP ? tc.q0 : tc.p0;
            const int sb_row0 = C::SWAP ? tc.p0 / 128 : tc.group * args.nb + tc.q0 / 128;
            const int sb_valid = C::SWAP ? 1 : min(C::kSbPerTile, args.nb - tc.q0 / 128);
            const bool sa_ok = lane < kSaLanes && a_row0 + lane * 4 < args.M4;
            for (int kb0 = 0; kb0 < args.num_kb && ok; kb0 += kBatch) {
                float4 va[kBatch];
                float vb[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int kb = kb0 + u;
                    va[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                    vb[u] = 0.f;
                    if (kb < args.num_kb) {
                        if (sa_ok)
                            va[u] = __ldg(reinterpret_cast<const float4*>(
                                args.sfa + static_cast<long long>(kb) * args.M4 + a_row0 + lane * 4));
                        if (lane < sb_valid)
                            vb[u] = __ldg(args.sfb + static_cast<long long>(sb_row0 + lane) * args.num_kb + kb);
                    }
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    if (kb0 + u >= args.num_kb) break;
                    if (!mbar_wait(sempty_bar(sstage), sphase ^ 1u, wctx)) {
                        ok = false;
                        break;
                    }
                    float* slot = scale_slots + sstage * C::kScaleSlotFloats;
                    if (lane < kSaLanes) reinterpret_cast<float4*>(slot)[lane] = va[u];
                    if (lane < C::kSbPerTile) slot[256 + lane] = vb[u];
                    mbar_arrive(sfull_bar(sstage));
                    if (++sstage == C::kScaleStages) {
                        sstage = 0;
                        sphase ^= 1u;
                    }
                }
            }
        }
    }
    } else {
        // ------------------------------------------------------------ epilogue
        if constexpr (C::kRegSplit) setmaxnreg_inc<224>();
        const int ew = warp - 4;
        const int wg = ew >> 2;           // epilogue warpgroup
        const int quarter = warp & 3;     // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;  // accumulator lane = P-operand row
        const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
        int sstage = 0, abuf = 0;
        uint32_t sphase = 0, aphase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
            const TileCoord tc = tile_coord<C>(args, t);
            if (tc.group < 0) continue;
            float2 acc[C::kCW / 2];
#pragma unroll
            for (int i = 0; i < C::kCW / 2; ++i) acc[i] = make_float2(0.f, 0.f);
            for (int kb = 0; kb < args.num_kb; ++kb) {
                if (!mbar_wait(sfull_bar(sstage), sphase, wctx) ||
                    !mbar_wait(tfull_bar(abuf), aphase, wctx)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float* slot = scale_slots + sstage * C::kScaleSlotFloats;
                const uint32_t taddr = tmem_base + t_lane + static_cast<uint32_t>(abuf * C::BNQ + wg * C::kCW);
                promote_k_block<C>(acc, taddr, slot, row, wg);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(tempty_bar(abuf));
                    mbar_arrive(sempty_bar(sstage));
                }
                if (++sstage == C::kScaleStages) {
                    sstage = 0;
                    sphase ^= 1u;
                }
                abuf ^= 1;
                if (abuf == 0) aphase ^= 1u;
            }
            if (!ok) break;
            // ---- store the tile
            if constexpr (!C::SWAP) {
                const int m = tc.p0 + row;
                if (m < args.M) {
                    uint16_t* drow = args.d + static_cast<long long>(m) * args.N;
#pragma unroll
                    for (int c = 0; c < C::kCW / 8; ++c) {
                        const int n = tc.q0 + wg * C::kCW + c * 8;
                        if (n < args.N) {
                            uint4 w;
                            w.x = pack_bf16x2(acc[c * 4 + 0].x, acc[c * 4 + 0].y);
                            w.y = pack_bf16x2(acc[c * 4 + 1].x, acc[c * 4 + 1].y);
                            w.z = pack_bf16x2(acc[c * 4 + 2].x, acc[c * 4 + 2].y);
                            w.w = pack_bf16x2(acc[c * 4 + 3].x, acc[c * 4 + 3].y);
                            *reinterpret_cast<uint4*>(drow + n) = w;
                        }
                    }
                }
            } else {
                const int n = tc.p0 + row;
                if (n < args.N) {
#pragma unroll
                    for (int j = 0; j < C::kCW; ++j) {
                        const int m = tc.q0 + j;
                        const float v = (j & 1) ? acc[j >> 1].y : acc[j >> 1].x;
                        if (m < args.M)
                            args.d[static_cast<long long>(m) * args.N + n] =
                                static_cast<uint16_t>(pack_bf16x2(v, 0.f) & 0xFFFFu);
                    }
                }
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// Self-test of the bounded wait: one warp waits on a barrier that nobody
// arrives on; the wait gives up after timeout_ns and records the timeout.
__global__ void k_wait_timeout_selftest(unsigned int* status, unsigned long long timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t abort_word;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_word = 0u;
        fence_barrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        WaitCtx w;
        w.abort = &abort_word;
        w.status = status;
        w.timeout_ns = timeout_ns;
        (void)mbar_wait(smem_u32(&bar), 0u, w);
    }
}

}  // namespace lnq
