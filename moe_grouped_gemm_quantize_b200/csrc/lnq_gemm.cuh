// lnq_gemm.cuh -- block-scaled FP8 GEMM "nt" on sm_100a tensor cores.
//
// D[m][n] = bf16( sum_g sfa[g][m] * sfb[n/128][g] * sum_{k in g} a[m][k] * b[n][k] )
// (deepgemm-rust README, "What's implemented": per-(1x128) activation scales
// x per-(128x128) weight scales, FP32 promotion, BF16 out).
//
// One persistent, warp-specialized kernel serves four shapes:
//   * dense, CTA pairs (M > 64, PAIR): two CTAs of a cluster run one
//     tcgen05.mma.cta_group::2 of 256 x 256; each CTA loads its own 128
//     activation rows and 128 of the 256 weight rows per K block, so each
//     CTA streams 32 KB instead of 48 KB per 128 x 256 of output;
//   * dense, single CTA: 128 activation rows in the MMA's M slot ("P
//     operand"), BNQ weight rows in its N slot ("Q operand");
//   * M-grouped contiguous (MoE): as single-CTA dense, each 128-row block of
//     activations takes the weights of the group named by its first row's id
//     (deepgemm-rust README, "Grouped (contiguous) MoE GEMM"), or of the group
//     whose aligned rows hold it in the prefix-sum layout; with 256-row group
//     alignment the grouped tiles run on CTA pairs as dense ones do
//     (deepgemm-rust README, "The mk_alignment knob (MoE tile width)");
//   * decode (M <= 64, "swap AB"): the weights fill the 128-row M slot and the
//     few tokens the N slot, so the tensor core is not idle on padding rows;
//   * gate_up with SiLU.mul (SILU, dense, single CTA or pair): the weight holds I
//     gate rows over I up rows; a tile's 256 MMA columns are 128 gate columns and
//     the 128 up columns of the same outputs, and the epilogue stores
//     h = silu(gate) * up (deepgemm-rust README, "What's implemented",
//     moe_fp8_layer: grouped GEMM -> SiLU.mul -> grouped GEMM).
//
// Roles (warps of one CTA):
//   warp 0      TMA producer: P and Q tiles of one 128-wide K block per stage
//               into a ring of shared-memory stages (128-byte swizzle).
//   warp 1      allocates tensor memory; one lane (of the pair's first CTA)
//               issues tcgen05.mma kind::f8f6f4 (E4M3 x E4M3 -> FP32), 4 MMAs
//               of K=32 per K block, into one of two TMEM accumulators that
//               alternate per K block.
//   warp 2      scale producer: loads the K block's activation and weight
//               scales into a small shared-memory ring.
//   warps 4..   epilogue: per K block, reads the FP32 partial product from TMEM
//               (tcgen05.ld), multiplies it by sa*sb and adds it into FP32
//               registers (the per-K-block promotion); after the last K block
//               converts to bf16 (round to nearest even) and stores the tile.
// The TMEM accumulators (as many as fit: 2 of 256 columns, 4 of 128, up to 16 of
// 32) let the tensor core run ahead of the epilogue's promotion; the depth
// hides the MMA -> epilogue -> MMA handshake latency.  All waits are bounded
// (mbar_wait).
#pragma once

#include <cstdint>
#include <cuda.h>

#include "lnq_ptx.cuh"
#include "lnq_quantize.cuh"

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
    int tiles_p;      // tiles along the MMA M slot (of 256 rows for PAIR)
    int tiles_q;      // tiles along the MMA N slot
    int num_tiles;
    int band;         // dense and grouped raster: row tiles per band (>= 1)
    int prefetch_weights;  // issue the first weight stages before waiting on the prior kernel
    // Split configuration only: the grid's CTAs share the num_tiles * num_kb (tile, K
    // block) units in contiguous runs; a CTA that covers part of a tile leaves an FP32
    // partial tile in `partials` and counts itself in `counters`.
    float* partials;  // [num_tiles][max_slots][128][BNQ]
    int* counters;    // [num_tiles], zero before and after every launch
    int max_slots;    // most CTAs sharing one tile
    // Grouped, masked layout only (m_indices == nullptr): group g owns rows
    // g*m_max .. g*m_max + m_max - 1, of which the first masked_m[g] are real.
    const int32_t* masked_m;  // [num_groups], on the device
    int m_max;                // rows per group, a multiple of 128
    // Grouped, prefix-sum layout only (m_indices == nullptr, psum != nullptr): psum[g]
    // counts the tokens of groups 0..g; group g's tokens start at the row
    // sum_{j<g} align_up(count_j, align), align a multiple of the tile's rows.
    const int32_t* psum;      // [num_groups], on the device
    int align;
    // Fused epilogue (dense and decode tiles): an optional bf16 bias per output
    // column added in FP32; and, instead of the bf16 D, the output quantized for a
    // next linear (dense 128 x 256 tiles only): E4M3 codes [M][N] and FP32 scales
    // [N/128][M4_out] of each 1 x 128 group of the bf16-rounded result.
    const uint16_t* bias;  // [N] bf16 bits, or nullptr
    uint8_t* q_out;        // [M][N] E4M3, or nullptr (bf16 D)
    float* sfa_out;        // [N/128][M4_out]
    long long M4_out;
    // dense and grouped tiles: 1 = output through shared memory and TMA stores, 0 = each
    // thread stores its own row
    int tma_store;
};

template <int BNQ_, int STAGES_, int EPI_WG_, bool SWAP_, bool GROUPED_, bool PAIR_ = false,
          int SLICES_ = 1, bool SPLITK_ = false, bool SILU_ = false>
struct GemmCfg {
    static constexpr int BNQ = BNQ_;   // MMA N (the whole pair's N for PAIR)
    static constexpr int STAGES = STAGES_;
    static constexpr int EPI_WG = EPI_WG_;
    static constexpr bool SWAP = SWAP_;
    static constexpr bool GROUPED = GROUPED_;
    static constexpr bool PAIR = PAIR_;
    // decode only: (tile, K block) units shared in contiguous runs by all CTAs
    static constexpr bool SPLITK = SPLITK_;
    static_assert(!SPLITK || SWAP, "the K split serves the decode configuration");
    // gate_up with SiLU.mul: a tile covers 128 outputs, i.e. 128 gate and 128 up columns
    static constexpr bool SILU = SILU_;
    static_assert(!SILU || (!SWAP && !GROUPED && !SPLITK && BNQ == 256 && EPI_WG_ == 2 && SLICES_ == 1),
                  "SiLU.mul tiles are dense 128 x 256 (or 256 x 256 on pairs) with two epilogue warpgroups");
    static_assert(!(SWAP && GROUPED), "decode configuration is dense only");
    static_assert(!(PAIR && SWAP), "CTA pairs serve the dense and grouped configurations");
    static_assert(BNQ % 16 == 0 && BNQ >= 16 && BNQ <= 256, "MMA N for M=128/256");
    static_assert(!SWAP || (BNQ / EPI_WG) % 16 == 0, "decode threads read TMEM in 16-column loads");
    static_assert(SWAP || BNQ % 128 == 0, "dense tiles cover whole 128-column scale blocks");

    static constexpr int kP = 128;                // P rows per CTA (MMA M per CTA)
    static constexpr int kTileM = PAIR ? 256 : 128;  // P rows per tile
    static constexpr int kBK = 128;               // K elements (bytes) per K block
    // K blocks per pipeline stage: decode tiles stream two weight boxes per stage (one
    // barrier wait, one expect-tx arrival and one commit for 32 KB of weights), and the
    // epilogue promotes the stage's two K blocks together
    static constexpr int kKbPerStage = SWAP ? 2 : 1;
    static constexpr int kPBytes = kP * kBK;
    static constexpr int kQRowsPerCta = PAIR ? BNQ / 2 : BNQ;
    static constexpr int kQBytes = kQRowsPerCta * kBK;
    // rows of one weight TMA box: a single-CTA SiLU.mul tile loads its gate and up
    // halves as two boxes
    static constexpr int kQBoxRows = (PAIR || SILU) ? 128 : kQRowsPerCta;
    // output columns per tile
    static constexpr int kTileN = SILU ? 128 : BNQ;
    // Scale ring.  Each slot holds the scales of kScaleBatch consecutive K blocks of
    // a tile, so the epilogue waits on (and releases) a slot once per batch.  Scale
    // copies travel the load/store path and take several microseconds to land under
    // a full operand stream, so the ring holds 32 K blocks' worth.
    static constexpr int kScaleBatch = 4;
    static constexpr int kScaleStages = 32 / kScaleBatch;
    // per K block: activation scales (128 rows, or BNQ tokens), then the weight scales
    static constexpr int kSbOffset = SWAP ? BNQ : 128;
    static constexpr int kScaleKbFloats = kSbOffset + 4;
    static constexpr int kScaleSlotFloats = kScaleBatch * kScaleKbFloats;
    static_assert(kScaleKbFloats % 4 == 0, "16-byte aligned scale runs");
    static constexpr int kCW = BNQ / EPI_WG;      // accumulator columns per epilogue thread
    // TMEM columns per load in the promotion: a decode thread loads all of its columns of
    // a K block at once; dense and grouped threads in chunks of 64 columns, each waited for
    // before its FMAs (a tcgen05.ld wait covers every load in flight, so a second chunk
    // loaded ahead would hide nothing; with 64 columns the load latency is paid twice per
    // K block for 128 columns instead of four times)
    static constexpr int kLdCols = SWAP ? kCW : (kCW >= 64 ? 64 : 32);
    static_assert(kCW % kLdCols == 0, "promotion chunks tile the thread's columns");
    // TMEM column of the thread's promotion chunk c, from its first column: SiLU.mul
    // threads take kCW/2 gate columns and the kCW/2 up columns 128 further on
    __host__ __device__ static constexpr int chunk_col(int c) {
        return SILU ? (c < kCW / kLdCols / 2 ? c * kLdCols : 128 + (c - kCW / kLdCols / 2) * kLdCols)
                    : c * kLdCols;
    }
    // first TMEM column of epilogue warpgroup wg's chunks
    __host__ __device__ static constexpr int wg_col(int wg) { return SILU ? wg * (kCW / 2) : wg * kCW; }
    static constexpr int kEpiThreads = 128 * EPI_WG;
    static constexpr int kThreads = 128 + kEpiThreads;
    // TMEM accumulators of BNQ columns each, as many as the 512 columns hold (at
    // most 16): the tensor core may run kAccBufs-1 K blocks ahead of the promotion.
    static constexpr int kAccBufs = (512 / BNQ) > 16 ? 16 : (512 / BNQ);
    static constexpr int kTmemCols = kAccBufs * BNQ;
    static constexpr int kSbPerTile = SWAP ? 1 : BNQ / 128;
    static constexpr int kSaPerTile = SWAP ? BNQ : kP;
    static constexpr bool kRegSplit = (!SWAP && kCW == 128);
    // With kSlices > 1 each epilogue warpgroup owns one column slice of the
    // accumulator: the MMA of a K block is issued slice by slice (N = BNQ /
    // kSlices), each slice with its own full/empty barriers, so the tensor core
    // may run up to 2*kSlices-1 slices ahead of the promotion.  With kSlices = 1
    // one MMA of N = BNQ covers the K block and all epilogue warps release it.
    static constexpr int kSlices = SLICES_;
    static_assert(kSlices == 1 || kSlices == EPI_WG, "slices follow the epilogue warpgroups");
    static constexpr int kSliceN = BNQ / kSlices;                   // MMA N per slice
    static constexpr int kSliceQRows = PAIR ? kSliceN / 2 : kSliceN;  // B rows per slice per CTA
    static constexpr int kEpiWarpsPerSlice = (PAIR ? 2 : 1) * 4 * (EPI_WG / kSlices);
    static constexpr uint32_t kIdesc = f8f6f4_e4m3_idesc(PAIR ? 256 : 128, kSliceN);
    static_assert(kSliceN % 16 == 0 && kSliceQRows % 8 == 0, "slice shapes");

    // shared-memory layout (offsets from a 1024-byte aligned base)
    static constexpr int kOffP = 0;
    static constexpr int kOffQ = kOffP + STAGES * kKbPerStage * kPBytes;
    static constexpr int kOffScale = kOffQ + STAGES * kKbPerStage * kQBytes;
    // Output staging for the TMA-store epilogue (dense and grouped tiles): per epilogue
    // warpgroup one 8 KB buffer of 128 rows x 64 bytes (32 bf16 columns, or 64 E4M3
    // codes) in the 64-byte swizzle, sent out by one TMA store per round.
    static constexpr int kStageRowBytes = 64;
    static constexpr int kStageBytes = 128 * kStageRowBytes;
    static constexpr int kOffStage = (kOffScale + kScaleStages * kScaleSlotFloats * 4 + 1023) / 1024 * 1024;
    static constexpr int kOffBar = kOffStage + (SWAP ? 0 : EPI_WG * kStageBytes);
    static constexpr int kNumBars = 2 * STAGES + 2 * kAccBufs * kSlices + 2 * kScaleStages + 1 + (SPLITK ? 2 : 0);
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(kTmemCols >= 32 && (kTmemCols & (kTmemCols - 1)) == 0 && kTmemCols <= 512,
                  "TMEM allocation is a power of two between 32 and 512 columns");
    static_assert(kQBytes % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
};

// A run of K blocks [kb_lo, kb_hi) of tile t.  Without the split each CTA takes
// whole tiles unit, unit + units, ...; with it, CTA `unit` of `units` takes the
// (tile, K block) units [unit*U/units, (unit+1)*U/units), U = num_tiles * num_kb,
// which covers at most two tiles partly.
struct Segment {
    int t;
    int kb_lo;
    int kb_hi;
};

template <class C>
__device__ __forceinline__ bool segment(const GemmArgs& a, int unit, int units, int i, Segment& s) {
    if constexpr (C::SPLITK) {
        const long long nkb = a.num_kb;
        const long long U = static_cast<long long>(a.num_tiles) * nkb;
        const long long u0 = static_cast<long long>(unit) * U / units;
        const long long u1 = static_cast<long long>(unit + 1) * U / units;
        const long long t = u0 / nkb + i;
        if (t * nkb >= u1) return false;
        s.t = static_cast<int>(t);
        s.kb_lo = static_cast<int>(u0 > t * nkb ? u0 - t * nkb : 0);
        s.kb_hi = static_cast<int>(u1 - t * nkb < nkb ? u1 - t * nkb : nkb);
        return true;
    } else {
        const int t = unit + i * units;
        if (t >= a.num_tiles) return false;
        s.t = t;
        s.kb_lo = 0;
        s.kb_hi = a.num_kb;
        return true;
    }
}

// The CTA whose run holds unit x: the largest c with floor(c*U/units) <= x.
__device__ __forceinline__ int unit_owner(long long x, long long U, int units) {
    return static_cast<int>(((x + 1) * units + U - 1) / U) - 1;
}

struct TileCoord {
    int p0;       // first row of this CTA's P operand (activation row, or weight row for SWAP)
    int q0;       // first output column of the tile (weight row within the group, or token)
    int group;    // grouped: group id of the tile, -1 skip; else 0
    int row_end;  // output rows from row_end on are not stored (dense and grouped tiles)
};

// Prefix-sum layout: the tiles of TILE_M rows that hold tokens, numbered group by
// group (group g has ceil(count_g / TILE_M) of them, from its first aligned row on).
// Tile v's group, first arena row and end of its group's tokens; group -1 past the
// last tile.  Numbering only the tiles with tokens keeps the pad rows of a coarse
// alignment out of the schedule: every CTA gets its share of real tiles.  Runs on a
// whole warp: each lane takes one group of a run of 32, the run's aligned row counts
// and tile counts are summed by warp scans, and the run whose tiles reach past v
// holds the group.  A count below zero (a decreasing psum) is reported and taken as
// zero.  Returns the first row after the runs scanned (after all groups when v lies
// past the last tile).
template <int TILE_M>
__device__ __forceinline__ long long psum_tile(const GemmArgs& a, int v, int& group, long long& p0,
                                               int& row_end) {
    const int lane = static_cast<int>(threadIdx.x & 31u);
    const long long align = a.align;
    long long base = 0;   // first row of the run's first group
    int base_tiles = 0;   // tiles of the groups before the run
    int prev_psum = 0;    // psum of the group before the run
    group = -1;
    p0 = 0;
    row_end = 0;
    for (int g0 = 0; g0 < a.num_groups && base_tiles <= v; g0 += 32) {
        const int g = g0 + lane;
        const bool real = g < a.num_groups;
        const int ps = real ? __ldg(a.psum + g) : 0;
        int before = __shfl_up_sync(0xffffffffu, ps, 1);
        if (lane == 0) before = prev_psum;
        long long count = real ? static_cast<long long>(ps) - before : 0;
        if (count < 0) {
            atomicOr(a.status, kStatusBadGroup);
            count = 0;
        }
        const long long padded = (count + align - 1) / align * align;
        const int tiles = static_cast<int>((count + TILE_M - 1) / TILE_M);
        long long end = padded;  // inclusive scans of the aligned rows and of the tiles
        int tend = tiles;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const long long x = __shfl_up_sync(0xffffffffu, end, d);
            const int y = __shfl_up_sync(0xffffffffu, tend, d);
            if (lane >= d) {
                end += x;
                tend += y;
            }
        }
        end += base;
        tend += base_tiles;
        const long long start = end - padded;
        const int tstart = tend - tiles;
        const unsigned hit = __ballot_sync(0xffffffffu, tiles > 0 && tstart <= v && v < tend);
        if (hit != 0u) {
            const int src = __ffs(hit) - 1;
            group = g0 + src;
            p0 = __shfl_sync(0xffffffffu, start + static_cast<long long>(v - tstart) * TILE_M, src);
            const long long tok_end = __shfl_sync(0xffffffffu, start + count, src);
            row_end = static_cast<int>(tok_end < a.M ? tok_end : a.M);
            if (tok_end > a.M) atomicOr(a.status, kStatusBadGroup);
            break;
        }
        base = __shfl_sync(0xffffffffu, end, 31);
        base_tiles = __shfl_sync(0xffffffffu, tend, 31);
        prev_psum = __shfl_sync(0xffffffffu, ps, 31);
    }
    return base;
}

// Tile t of this CTA (or of this CTA pair; `rank` is the CTA's rank in the pair).
template <class C>
__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& a, int t, uint32_t rank) {
    TileCoord c;
    if constexpr (C::SWAP) {
        c.p0 = (t % a.tiles_p) * C::kP;
        c.q0 = (t / a.tiles_p) * C::BNQ;
        c.group = 0;
        c.row_end = a.M;
    } else {
        // Bands of row tiles, column-major inside a band: a wave of tiles shares a
        // band of activation rows and a few weight column tiles, and every weight
        // column tile is read once per band.  The host sizes the band so that its
        // activation rows stay within a share of L2.  Grouped: the 128-row blocks of
        // one group sit next to each other, so a band's blocks of a group walk that
        // group's weight columns together (a narrow band keeps the weights of the
        // groups in flight within L2).
        const int kBand = a.band;
        const int band_tiles = kBand * a.tiles_q;
        const int band = t / band_tiles;
        const int first = band * kBand;
        const int rows = min(a.tiles_p - first, kBand);
        const int r = t - band * band_tiles;
        c.p0 = (first + r % rows) * C::kTileM + static_cast<int>(rank) * C::kP;
        c.q0 = (r / rows) * C::kTileN;
        c.row_end = a.M;
        if constexpr (C::GROUPED) {
            if (a.psum != nullptr) {
                // prefix-sum layout: the raster's row tile is the index among the tiles
                // that hold tokens (the same for both CTAs of a pair); a tile that would
                // start past the arena (groups that overrun it) is skipped
                int g, end;
                long long base_row;
                psum_tile<C::kTileM>(a, c.p0 / C::kTileM, g, base_row, end);
                c.group = base_row < a.M ? g : -1;
                c.p0 = static_cast<int>(base_row < a.M ? base_row : 0) + static_cast<int>(rank) * C::kP;
                c.row_end = end;
            } else if (a.m_indices != nullptr) {
                // contiguous: the block's group is that of its first row
                c.group = __ldg(a.m_indices + c.p0);
                if (c.group >= a.num_groups) {
                    atomicOr(a.status, kStatusBadGroup);
                    c.group = -1;
                }
            } else {
                // masked: group g's first masked_m[g] rows are real; a block past
                // them is skipped, a block that holds the last of them stops there
                const int g = c.p0 / a.m_max;
                int count = __ldg(a.masked_m + g);
                if (count < 0 || count > a.m_max) {
                    atomicOr(a.status, kStatusBadGroup);
                    count = count < 0 ? 0 : a.m_max;
                }
                const int valid = g * a.m_max + count - c.p0;
                c.group = valid > 0 ? g : -1;
                c.row_end = c.p0 + (valid < C::kP ? valid : C::kP);
            }
        } else {
            c.group = 0;
        }
    }
    return c;
}

// One K block of the per-block FP32 promotion: acc += partial * scale, where
// the partial is this thread's TMEM lane (kCW columns starting at taddr).  The
// columns are read in chunks of kLdCols; `release`
// runs as soon as the last chunk has arrived in registers, before its FMAs, so
// the tensor core may overwrite the slice early.
//   dense:  scale = sa[row] * sb[column block of this warpgroup]
//   decode: scale = sa[token j] * sb[weight block of the tile], per column j
template <class C, int W>
__device__ __forceinline__ void promote_chunk(float2 (&acc)[C::kCW / 2], const uint32_t (&r)[W],
                                              int col0, const float* slot, float2 s2) {
#pragma unroll
    for (int i = 0; i < W / 2; ++i) {
        const float2 v = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        float2 sc = s2;
        if constexpr (C::SWAP) {
            const float2 sa = *reinterpret_cast<const float2*>(slot + col0 + 2 * i);
            sc = __fmul2_rn(sa, s2);
        }
        acc[col0 / 2 + i] = __ffma2_rn(v, sc, acc[col0 / 2 + i]);
    }
}

template <class C, class Release>
__device__ __forceinline__ void promote_k_block(float2 (&acc)[C::kCW / 2], uint32_t taddr,
                                                const float* slot, int row, int wg,
                                                Release&& release) {
    // chunks of kLdCols columns, each load issued one chunk ahead of the FMAs
    constexpr int X = C::kLdCols;
    constexpr int NC = C::kCW / X;
    float2 s2, s2_up;
    if constexpr (C::SILU) {
        // gate columns take the gate block's weight scale, up columns the up block's
        const float sa = slot[row];
        const float sg = sa * slot[C::kSbOffset];
        const float su = sa * slot[C::kSbOffset + 1];
        s2 = make_float2(sg, sg);
        s2_up = make_float2(su, su);
    } else if constexpr (!C::SWAP) {
        const float s = slot[row] * slot[C::kSbOffset + (wg * C::kCW) / 128];
        s2 = make_float2(s, s);
        s2_up = s2;
    } else {
        const float sb = slot[C::kSbOffset];
        s2 = make_float2(sb, sb);
        s2_up = s2;
    }
    if constexpr (X == 64) {
        // one 64-column chunk at a time: load, wait, (after the last load) release, FMAs
        uint32_t r[X];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            tmem_ld_async(taddr + C::chunk_col(c), r);
            tmem_wait_ld(r);
            if (NC > 1 && c + 1 == NC) release();
            const float2 sc = (C::SILU && c >= NC / 2) ? s2_up : s2;
            promote_chunk<C, X>(acc, r, c * X, slot, sc);
            // one chunk: release once the FMAs have consumed the scale slot's values
            if (NC == 1) release();
        }
    } else {
        uint32_t ra[X], rb[X];
        tmem_ld_async(taddr + C::chunk_col(0), ra);
        tmem_wait_ld(ra);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            if (c + 1 < NC) {
                if (c & 1) tmem_ld_async(taddr + C::chunk_col(c + 1), ra);
                else tmem_ld_async(taddr + C::chunk_col(c + 1), rb);
            }
            const float2 sc = (C::SILU && c >= NC / 2) ? s2_up : s2;
            if (c & 1) promote_chunk<C, X>(acc, rb, c * X, slot, sc);
            else promote_chunk<C, X>(acc, ra, c * X, slot, sc);
            if (NC == 1) release();  // after the FMAs that consumed the scale slot's values
            if (c + 1 < NC) {
                if (c & 1) tmem_wait_ld(ra);
                else tmem_wait_ld(rb);
                if (c + 2 == NC) release();
            }
        }
    }
}

// Decode tile store: this thread holds weight row n = p0 + row for the tile's
// tokens q0 + col0 .. q0 + col0 + kCW - 1; D is [M][N], so each token's row gets one bf16.
template <class C>
__device__ __forceinline__ void store_decode_tile(const GemmArgs& args, const TileCoord& tc, int row, int col0,
                                                  const float2 (&acc)[C::kCW / 2]) {
    const int n = tc.p0 + row;
    if (n >= args.N) return;
    const float bias = args.bias != nullptr ? bf16_lo(static_cast<uint32_t>(args.bias[n])) : 0.f;
#pragma unroll
    for (int j = 0; j < C::kCW; ++j) {
        const int m = tc.q0 + col0 + j;
        const float v = ((j & 1) ? acc[j >> 1].y : acc[j >> 1].x) + bias;
        if (m < args.M)
            args.d[static_cast<long long>(m) * args.N + n] =
                static_cast<uint16_t>(pack_bf16x2(v, 0.f) & 0xFFFFu);
    }
}

// One round of the TMA-store epilogue for one epilogue warpgroup: its 128 rows (thread
// = row) of 64 bytes each go into the warpgroup's staging buffer `buf` (64-byte swizzle:
// 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3)) and out with one TMA store
// of the box at (x, y), issued by the warpgroup's first thread.  The buffer is rewritten
// only after the previous round's store has read it.  Named barrier `bar` (128 threads)
// orders the rounds.
__device__ __forceinline__ void stage_store_round(uint32_t buf, int row, bool leader, uint32_t bar,
                                                  const uint32_t (&w)[16], const CUtensorMap* map, int x, int y) {
    if (leader) bulk_wait_read_all();
    asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
    const uint32_t rowaddr = buf + static_cast<uint32_t>(row * 64);
    const uint32_t sw = static_cast<uint32_t>((row >> 1) & 3);
#pragma unroll
    for (int c = 0; c < 4; ++c)
        st_shared_v4(rowaddr + ((static_cast<uint32_t>(c) ^ sw) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2],
                     w[4 * c + 3]);
    fence_proxy_async_shared();
    asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
    if (leader) {
        tma_store_2d(map, buf, x, y);
        bulk_commit();
    }
}

// Spin for `ns` nanoseconds (bounded); lets copies already issued by a CTA
// that gave up land before it leaves.
__device__ __forceinline__ void settle_ns(uint64_t ns) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < ns) {
    }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    k_fp8_block_gemm(const __grid_constant__ CUtensorMap map_p,
                     const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_d,
                     const GemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t sP = s_base + C::kOffP;
    const uint32_t sQ = s_base + C::kOffQ;
    // K block h of ring stage s, P and Q operands
    auto p_at = [&](int s, int h) { return sP + static_cast<uint32_t>((s * C::kKbPerStage + h) * C::kPBytes); };
    auto q_at = [&](int s, int h) { return sQ + static_cast<uint32_t>((s * C::kKbPerStage + h) * C::kQBytes); };
    float* scale_slots = reinterpret_cast<float*>(smem + C::kOffScale);
    const uint32_t bars = s_base + C::kOffBar;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (C::STAGES + s); };
    // accumulator slot = buffer * kSlices + slice
    constexpr int kSlots = C::kAccBufs * C::kSlices;
    auto tfull_bar = [&](int b) { return bars + 8u * (2 * C::STAGES + b); };
    auto tempty_bar = [&](int b) { return bars + 8u * (2 * C::STAGES + kSlots + b); };
    auto sfull_bar = [&](int s) { return bars + 8u * (2 * C::STAGES + 2 * kSlots + s); };
    auto sempty_bar = [&](int s) {
        return bars + 8u * (2 * C::STAGES + 2 * kSlots + C::kScaleStages + s);
    };
    const uint32_t drain_bar = bars + 8u * (2 * C::STAGES + 2 * kSlots + 2 * C::kScaleStages);
    // split configuration: partial tile written by every epilogue warp; count taken
    const uint32_t fix_bar = drain_bar + 8u;
    const uint32_t dec_bar = drain_bar + 16u;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile uint32_t* abort_flag = misc + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // CTA pairs: rank in the pair; tiles are numbered per pair
    const uint32_t rank = C::PAIR ? cluster_ctarank() : 0u;
    const int unit = C::PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int units = C::PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

    if (warp == 0) {
        // The barriers lie in one array in this order: stage full and empty, accumulator
        // full and empty, scale full and empty, drain (and the split's two); the lanes of
        // warp 0 initialize them together (a decode CTA has about sixty).
        auto arrivals = [](int i) -> uint32_t {
            if (i < 2 * C::STAGES) return 1u;
            i -= 2 * C::STAGES;
            if (i < kSlots) return 1u;
            i -= kSlots;
            if (i < kSlots) return static_cast<uint32_t>(C::kEpiWarpsPerSlice);
            i -= kSlots;
            if (i < C::kScaleStages) return 32u;
            i -= C::kScaleStages;
            if (i < C::kScaleStages) return static_cast<uint32_t>(C::kEpiThreads / 32);
            i -= C::kScaleStages;
            if (i == 0) return 2u;                                             // drain
            return i == 1 ? static_cast<uint32_t>(C::kEpiThreads / 32) : 1u;  // split: fix, count
        };
        for (int i = lane; i < C::kNumBars; i += 32) mbar_init(bars + 8u * static_cast<uint32_t>(i), arrivals(i));
        if (lane == 0) *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 1) {
        if constexpr (C::PAIR) {
            tmem_alloc_pair(smem_u32(misc), C::kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(misc), C::kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if constexpr (C::PAIR) cluster_sync();  // the peer's barriers exist before any remote signal
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    // the prologue above touches no global memory: the next kernel may start its
    // own, and this one waits for the previous kernel before reading any input
    // (the producer may first prefetch weights, see below)
    launch_dependents();
    if (!(args.prefetch_weights && warp == 0)) wait_prior_grids();

    WaitCtx wctx;
    wctx.abort = abort_flag;
    wctx.status = args.status;
    wctx.timeout_ns = args.timeout_ns;

    if (warp < 4) {
    // control warpgroup: registers handed to the epilogue warpgroups
    if constexpr (C::kRegSplit) setmaxnreg_dec<56>();
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp runs the loop; one elected lane issues the copies.
        {
            if (elect_one()) {
                tma_prefetch_desc(&map_p);
                tma_prefetch_desc(&map_q);
            }
            __syncwarp();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0, fill_parity = 0;
            bool ok = true;
            // Weight prefetch (caller asserts that the weights and their scales are not
            // written by the kernels still running before this one): the weight halves of
            // the first ring stages of the first tile are issued before the wait on the
            // prior kernel, the activation halves after it.
            int prefetched = 0;
            if (args.prefetch_weights) {
                // dense tiles only: a grouped tile's weights depend on group ids or
                // counts that the prior kernel may still be writing
                if constexpr (!C::PAIR && !C::GROUPED) {
                    Segment sg0;
                    if (segment<C>(args, unit, units, 0, sg0)) {
                        const TileCoord tc = tile_coord<C>(args, sg0.t, rank);
                        constexpr int KBS = C::kKbPerStage;
                        prefetched = min(C::STAGES, (sg0.kb_hi - sg0.kb_lo + KBS - 1) / KBS);
                        if (elect_one()) {
                            for (int s = 0; s < prefetched; ++s) {
                                const int kb0 = sg0.kb_lo + s * KBS;
                                const int nk = min(KBS, sg0.kb_hi - kb0);
                                mbar_arrive_expect_tx(full_bar(s), nk * (C::kPBytes + C::kQBytes));
                                for (int h = 0; h < nk; ++h) {
                                    if constexpr (C::SWAP) {
                                        tma_load_2d(p_at(s, h), &map_p, full_bar(s), (kb0 + h) * C::kBK, tc.p0);
                                    } else {
                                        tma_load_2d(q_at(s, h), &map_q, full_bar(s), (kb0 + h) * C::kBK, tc.q0);
                                        if constexpr (C::SILU)  // the up rows of the same outputs
                                            tma_load_2d(q_at(s, h) + C::kQBoxRows * C::kBK, &map_q, full_bar(s),
                                                        (kb0 + h) * C::kBK, tc.q0 + args.N);
                                    }
                                }
                            }
                        }
                        __syncwarp();
                    }
                }
                wait_prior_grids();
            }
            Segment sg;
            for (int i = 0; ok && segment<C>(args, unit, units, i, sg); ++i) {
                const TileCoord tc = tile_coord<C>(args, sg.t, rank);
                if (tc.group < 0) continue;
                int p_row, q_row;
                if constexpr (C::SWAP) {
                    p_row = tc.p0;
                    q_row = tc.q0;
                } else if constexpr (C::SILU) {
                    // gate rows q0.. (and, on a pair's second CTA, the up rows I + q0..)
                    p_row = tc.p0;
                    q_row = tc.q0 + static_cast<int>(rank) * args.N;
                } else {
                    p_row = tc.p0;
                    q_row = tc.group * args.N + tc.q0 + static_cast<int>(rank) * C::kSliceQRows;
                }
                for (int kb = sg.kb_lo; kb < sg.kb_hi; kb += C::kKbPerStage) {
                    const int nk = min(C::kKbPerStage, sg.kb_hi - kb);
                    if (prefetched > 0) {
                        // stage already armed and its weight half in flight: load the activations
                        if constexpr (!C::PAIR) {
                            if (elect_one()) {
                                for (int h = 0; h < nk; ++h) {
                                    if constexpr (C::SWAP)
                                        tma_load_2d(q_at(stage, h), &map_q, full_bar(stage), (kb + h) * C::kBK, q_row);
                                    else
                                        tma_load_2d(p_at(stage, h), &map_p, full_bar(stage), (kb + h) * C::kBK, p_row);
                                }
                            }
                            __syncwarp();
                        }
                        --prefetched;
                    } else {
                        if (!mbar_wait_warp(empty_bar(stage), phase ^ 1u, wctx)) {
                            ok = false;
                            break;
                        }
                        if (elect_one()) {
                            if constexpr (C::PAIR) {
                                // both CTAs' bytes complete on the first CTA's full barrier
                                if (rank == 0)
                                    mbar_arrive_expect_tx(full_bar(stage), 2 * (C::kPBytes + C::kQBytes));
                                const uint32_t leader_full = mapa_shared(full_bar(stage), 0);
                                tma_load_2d_pair(p_at(stage, 0), &map_p, leader_full, kb * C::kBK, p_row);
                                // slice h of the tile's N: this CTA holds its kSliceQRows rows of it
#pragma unroll
                                for (int h = 0; h < C::kSlices; ++h)
                                    tma_load_2d_pair(q_at(stage, 0) + h * C::kSliceQRows * C::kBK, &map_q,
                                                     leader_full, kb * C::kBK, q_row + h * C::kSliceN);
                            } else {
                                mbar_arrive_expect_tx(full_bar(stage), nk * (C::kPBytes + C::kQBytes));
                                for (int h = 0; h < nk; ++h) {
                                    tma_load_2d(p_at(stage, h), &map_p, full_bar(stage), (kb + h) * C::kBK, p_row);
                                    tma_load_2d(q_at(stage, h), &map_q, full_bar(stage), (kb + h) * C::kBK, q_row);
                                    if constexpr (C::SILU && !C::PAIR)  // the up rows of the same outputs
                                        tma_load_2d(q_at(stage, h) + C::kQBoxRows * C::kBK, &map_q, full_bar(stage),
                                                    (kb + h) * C::kBK, q_row + args.N);
                                }
                            }
                        }
                        __syncwarp();
                    }
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
                if (C::PAIR && rank != 0) {
                    settle_ns(200000);
                } else {
                    WaitCtx drain = wctx;
                    uint32_t never = 0u;
                    drain.abort = &never;
                    for (int s = 0; s < C::STAGES; ++s)
                        if (filled & (1u << s))
                            (void)mbar_wait_warp(full_bar(s), (fill_parity >> s) & 1u, drain);
                    if (C::PAIR) settle_ns(200000);
                }
            }
        }
    } else if (warp == 1 || warp == 3) {
        // ------------------------------------------------------------ MMA issuers
        // The whole warp runs the loop (operands stay warp-uniform); one elected
        // lane issues the MMAs and commits.  Issuing a K block (two barrier waits,
        // four MMAs, two commits) keeps a warp busy about as long as the tensor core
        // needs for a 128 x 256 K block, and longer for the narrow decode tiles, so
        // warps 1 and 3 take alternate K blocks (each K block has its own stage and
        // accumulator: the two streams are independent).
        const int midx = (warp == 1) ? 0 : 1;
        constexpr int kIssuers = 2;
        if (rank == 0) {
            int stage = 0, abuf = 0;
            int gs = 0;  // ring stages seen, for the alternation
            uint32_t phase = 0, aphase = 0;
            bool ok = true;
            const uint64_t adesc0 = sw128_kmajor_desc(sP);
            const uint64_t bdesc0 = sw128_kmajor_desc(sQ);
            auto next_acc = [&]() {
                if (++abuf == C::kAccBufs) {
                    abuf = 0;
                    aphase ^= 1u;
                }
            };
            Segment sg;
            for (int i = 0; ok && segment<C>(args, unit, units, i, sg); ++i) {
                const TileCoord tc = tile_coord<C>(args, sg.t, 0);
                if (tc.group < 0) continue;
                for (int kb = sg.kb_lo; kb < sg.kb_hi && ok; kb += C::kKbPerStage) {
                    const int nk = min(C::kKbPerStage, sg.kb_hi - kb);
                    if (gs++ % kIssuers != midx) {
                        // the other issuer's stage and its K blocks' accumulators
                        if (++stage == C::STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                        for (int hk = 0; hk < nk; ++hk) next_acc();
                        continue;
                    }
                    if (!mbar_wait_warp(full_bar(stage), phase, wctx)) {
                        ok = false;
                        break;
                    }
                    for (int hk = 0; hk < nk && ok; ++hk) {
                        // descriptor start fields advance by (byte offset >> 4)
                        const int sk = stage * C::kKbPerStage + hk;
                        const uint64_t adesc = adesc0 + static_cast<uint64_t>((sk * C::kPBytes) >> 4);
#pragma unroll
                        for (int h = 0; h < C::kSlices; ++h) {
                            const int slot = abuf * C::kSlices + h;
                            if (!mbar_wait_warp(tempty_bar(slot), aphase ^ 1u, wctx)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * C::BNQ + h * C::kSliceN);
                            const uint64_t bdesc =
                                bdesc0 + static_cast<uint64_t>((sk * C::kQBytes + h * C::kSliceQRows * C::kBK) >> 4);
                            if (elect_one()) {
                                if constexpr (C::PAIR) {
#pragma unroll
                                    for (int k = 0; k < C::kBK / 32; ++k)
                                        mma_f8f6f4_pair(d_tmem, adesc + 2u * k, bdesc + 2u * k, C::kIdesc,
                                                        k > 0 ? 1u : 0u);
                                    mma_commit_pair(mapa_shared(tfull_bar(slot), 0));
                                    mma_commit_pair(mapa_shared(tfull_bar(slot), 1));
                                } else {
#pragma unroll
                                    for (int k = 0; k < C::kBK / 32; ++k)
                                        mma_f8f6f4(d_tmem, adesc + 2u * k, bdesc + 2u * k, C::kIdesc,
                                                   k > 0 ? 1u : 0u);
                                    mma_commit(tfull_bar(slot));
                                }
                            }
                            __syncwarp();
                        }
                        next_acc();
                    }
                    if (!ok) break;
                    // the stage is free once every slice's MMAs have read it
                    if (elect_one()) {
                        if constexpr (C::PAIR) {
                            mma_commit_pair(mapa_shared(empty_bar(stage), 0));
                            mma_commit_pair(mapa_shared(empty_bar(stage), 1));
                        } else {
                            mma_commit(empty_bar(stage));
                        }
                    }
                    __syncwarp();
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            {
                // every MMA this warp issued completes before TMEM is released (both
                // issuers always commit: the barrier counts two arrivals)
                if (elect_one()) {
                    if constexpr (C::PAIR) mma_commit_pair(mapa_shared(drain_bar, 0));
                    else mma_commit(drain_bar);
                }
                __syncwarp();
                WaitCtx drain = wctx;
                uint32_t never = 0u;
                drain.abort = &never;
                (void)mbar_wait_warp(drain_bar, 0u, drain);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ scale producer
        // Copies each K block's activation scales (one 16-byte run per lane) and the
        // tile's weight scales straight into the scale ring with cp.async; each lane's
        // arrival on the slot's barrier fires when its copies have landed, so the warp
        // runs up to the ring's depth ahead without holding anything in registers.
        // Rows past M4 and weight blocks past N read clamped addresses: they only feed
        // accumulator rows or columns that are never stored.
        int sstage = 0;
        uint32_t sphase = 0;
        bool ok = true;
        constexpr int kSaLanes = C::kSaPerTile / 4;  // lanes that copy 16 bytes of sa
        if constexpr (C::GROUPED) {
            // prefix-sum layout: groups whose aligned rows run past the arena are
            // reported once per launch (tiles that would start past it are skipped)
            if (args.psum != nullptr && blockIdx.x == 0) {
                int g, e;
                long long r0;
                if (psum_tile<C::kTileM>(args, 0x7fffffff, g, r0, e) > args.M) atomicOr(args.status, kStatusBadGroup);
            }
        }
        Segment sg;
        for (int i = 0; ok && segment<C>(args, unit, units, i, sg); ++i) {
            const TileCoord tc = tile_coord<C>(args, sg.t, rank);
            if (tc.group < 0) continue;
            // activation rows of the tile (tokens for SWAP) and weight scale rows
            long long a_row = (C::SWAP ? tc.q0 : tc.p0) + lane * 4;
            if (a_row > args.M4 - 4) a_row = args.M4 - 4;
            const int nb_first = C::SWAP ? tc.p0 / 128 : tc.q0 / 128;
            // SiLU.mul: lane 0 the gate block's scales, lane 1 the up block's (I/128 further)
            const int nb_lane = min(C::SILU ? nb_first + lane * (args.N / 128) : nb_first + lane, args.nb - 1);
            const long long sb_row = static_cast<long long>(C::SWAP ? 0 : tc.group) * args.nb + nb_lane;
            const float* sa_src = args.sfa + a_row;
            const float* sb_src = args.sfb + sb_row * args.num_kb;
            for (int kb0 = sg.kb_lo; kb0 < sg.kb_hi; kb0 += C::kScaleBatch) {
                if (!mbar_wait(sempty_bar(sstage), sphase ^ 1u, wctx)) {
                    ok = false;
                    break;
                }
                const uint32_t slot = smem_u32(scale_slots + sstage * C::kScaleSlotFloats);
                const int nkb = min(C::kScaleBatch, sg.kb_hi - kb0);
                for (int j = 0; j < nkb; ++j) {
                    const int kb = kb0 + j;
                    const uint32_t sub = slot + static_cast<uint32_t>(j * C::kScaleKbFloats * 4);
                    if (lane < kSaLanes) cp_async_16(sub + lane * 16, sa_src + static_cast<long long>(kb) * args.M4);
                    if (lane < C::kSbPerTile) cp_async_4(sub + (C::kSbOffset + lane) * 4, sb_src + kb);
                }
                cp_async_arrive(sfull_bar(sstage));
                if (++sstage == C::kScaleStages) {
                    sstage = 0;
                    sphase ^= 1u;
                }
            }
        }
        // no copy may still be landing when the CTA leaves
        asm volatile("cp.async.wait_all;" ::: "memory");
    }
    } else {
        // ------------------------------------------------------------ epilogue
        if constexpr (C::kRegSplit) setmaxnreg_inc<224>();
        const int ew = warp - 4;
        const int wg = ew >> 2;           // epilogue warpgroup
        const int quarter = warp & 3;     // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;  // accumulator lane = P-operand row
        const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
        // the warpgroup's staging buffer, and the thread that issues its TMA stores
        const uint32_t stage_buf = s_base + static_cast<uint32_t>(C::kOffStage + wg * C::kStageBytes);
        const bool stage_leader = (ew & 3) == 0 && lane == 0;
        if constexpr (!C::SWAP) {
            if (ew == 0 && lane == 0) tma_prefetch_desc(&map_d);
        }
        int sstage = 0, abuf = 0;
        uint32_t sphase = 0, aphase = 0;
        uint32_t fix_phase = 0;
        bool ok = true;
        Segment sg;
        for (int i = 0; ok && segment<C>(args, unit, units, i, sg); ++i) {
            const TileCoord tc = tile_coord<C>(args, sg.t, rank);
            if (tc.group < 0) continue;
            float2 acc[C::kCW / 2];
#pragma unroll
            for (int i = 0; i < C::kCW / 2; ++i) acc[i] = make_float2(0.f, 0.f);
            int j = 0;  // K block within the scale slot's batch
            for (int kb = sg.kb_lo; kb < sg.kb_hi; kb += C::kKbPerStage) {
                if constexpr (C::SWAP) {
                    // Decode: the ring stage's K blocks (two, or one at the end of a run) are
                    // promoted together: both partials are loaded before either is waited
                    // on, both accumulators released, then both multiplied in.  This
                    // thread's columns are tokens wg*kCW .. wg*kCW + kCW - 1 of the tile.
                    const int nk = min(C::kKbPerStage, sg.kb_hi - kb);
                    const bool batch_last = (j + nk == C::kScaleBatch) || (kb + nk == sg.kb_hi);
                    int abuf1 = abuf + 1;
                    uint32_t aphase1 = aphase;
                    if (abuf1 == C::kAccBufs) {
                        abuf1 = 0;
                        aphase1 ^= 1u;
                    }
                    if ((j == 0 && !mbar_wait(sfull_bar(sstage), sphase, wctx)) ||
                        !mbar_wait(tfull_bar(abuf), aphase, wctx) ||
                        (nk > 1 && !mbar_wait(tfull_bar(abuf1), aphase1, wctx))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float* slot = scale_slots + sstage * C::kScaleSlotFloats + j * C::kScaleKbFloats;
                    const uint32_t col = static_cast<uint32_t>(C::wg_col(wg));
                    uint32_t r0[C::kCW], r1[C::kCW];
                    tmem_ld_async(tmem_base + t_lane + static_cast<uint32_t>(abuf * C::BNQ) + col, r0);
                    if (nk > 1) tmem_ld_async(tmem_base + t_lane + static_cast<uint32_t>(abuf1 * C::BNQ) + col, r1);
                    tmem_wait_ld(r0);
                    if (nk > 1) tmem_wait_ld(r1);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive_relaxed(tempty_bar(abuf));
                        if (nk > 1) mbar_arrive_relaxed(tempty_bar(abuf1));
                    }
                    {
                        const float sb = slot[C::kSbOffset];
                        promote_chunk<C, C::kCW>(acc, r0, 0, slot + wg * C::kCW, make_float2(sb, sb));
                    }
                    if (nk > 1) {
                        const float* slot1 = slot + C::kScaleKbFloats;
                        const float sb = slot1[C::kSbOffset];
                        promote_chunk<C, C::kCW>(acc, r1, 0, slot1 + wg * C::kCW, make_float2(sb, sb));
                    }
                    // the per-token scales were read by the FMAs above: the slot may go
                    if (batch_last) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive_relaxed(sempty_bar(sstage));
                        j = 0;
                        if (++sstage == C::kScaleStages) {
                            sstage = 0;
                            sphase ^= 1u;
                        }
                    } else {
                        j += nk;
                    }
                    abuf = abuf1;
                    aphase = aphase1;
                    if (nk > 1 && ++abuf == C::kAccBufs) {
                        abuf = 0;
                        aphase ^= 1u;
                    }
                    continue;
                } else {
                const bool batch_last = (j == C::kScaleBatch - 1) || (kb + 1 == sg.kb_hi);
                const int slot_id = abuf * C::kSlices + (C::kSlices == 1 ? 0 : wg);
                if ((j == 0 && !mbar_wait(sfull_bar(sstage), sphase, wctx)) ||
                    !mbar_wait(tfull_bar(slot_id), aphase, wctx)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float* slot = scale_slots + sstage * C::kScaleSlotFloats + j * C::kScaleKbFloats;
                const uint32_t taddr = tmem_base + t_lane + static_cast<uint32_t>(abuf * C::BNQ + C::wg_col(wg));
                // the accumulator slice and the scale slot are only read, and each arrival
                // follows the completion of those reads: the TMEM loads are waited for, and
                // the scale values have fed FMAs issued before the arrival.  No release fence
                // is needed (one would also wait for this warp's outstanding output stores).
                // The slice is released as soon as its last chunk is in registers (with a
                // single chunk, after its FMAs), the scale slot after the last K block of its
                // batch.
                const uint32_t sempty = sempty_bar(sstage);
                promote_k_block<C>(acc, taddr, slot, row, wg, [&]() {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if constexpr (C::PAIR) mbar_arrive_cluster_relaxed(mapa_shared(tempty_bar(slot_id), 0));
                        else mbar_arrive_relaxed(tempty_bar(slot_id));
                        // the scale values were consumed by FMAs issued before this arrival
                        if (batch_last) mbar_arrive_relaxed(sempty);
                    }
                });
                if (batch_last) {
                    j = 0;
                    if (++sstage == C::kScaleStages) {
                        sstage = 0;
                        sphase ^= 1u;
                    }
                } else {
                    ++j;
                }
                if (++abuf == C::kAccBufs) {
                    abuf = 0;
                    aphase ^= 1u;
                }
                }
            }
            if (!ok) break;
            if constexpr (C::SPLITK) {
                if (sg.kb_lo != 0 || sg.kb_hi != args.num_kb) {
                    // Part of the tile's K range: leave the FP32 partial in this CTA's slot
                    // of the tile and count it; the CTA that completes the count sums the
                    // slots in order of their K ranges (so the result does not depend on
                    // which CTA finishes last), stores the tile and rezeroes the count.
                    const long long nkb = args.num_kb;
                    const long long U = static_cast<long long>(args.num_tiles) * nkb;
                    const int first = unit_owner(static_cast<long long>(sg.t) * nkb, U, units);
                    const int last = unit_owner(static_cast<long long>(sg.t + 1) * nkb - 1, U, units);
                    const int n_parts = last - first + 1;
                    const int slot = unit - first;
                    auto part = [&](int sl) {
                        return reinterpret_cast<float4*>(
                            args.partials +
                            ((static_cast<long long>(sg.t) * args.max_slots + sl) * C::kP + row) * C::BNQ +
                            wg * C::kCW);
                    };
                    float4* mine = part(slot);
#pragma unroll
                    for (int i4 = 0; i4 < C::kCW / 4; ++i4)
                        mine[i4] = make_float4(acc[2 * i4].x, acc[2 * i4].y, acc[2 * i4 + 1].x, acc[2 * i4 + 1].y);
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(fix_bar);
                    if (ew == 0) {
                        // every epilogue warp has written and fenced its rows: count this CTA
                        if (mbar_wait_warp(fix_bar, fix_phase, wctx)) {
                            if (lane == 0) {
                                const int before = atomicAdd(args.counters + sg.t, 1);
                                const bool completes = (before == n_parts - 1);
                                if (completes) args.counters[sg.t] = 0;
                                misc[2] = completes ? 1u : 0u;
                                __threadfence();
                            }
                            __syncwarp();
                            if (lane == 0) mbar_arrive(dec_bar);
                        } else {
                            ok = false;
                        }
                    }
                    if (ok) ok = mbar_wait(dec_bar, fix_phase, wctx);
                    fix_phase ^= 1u;
                    if (!ok) break;
                    if (*reinterpret_cast<volatile uint32_t*>(misc + 2) == 0u) continue;  // another CTA stores
                    __threadfence();
                    // every slot of the tile, in order of K
                    for (int sl = 0; sl < n_parts; ++sl) {
                        const float4* p = part(sl);
#pragma unroll
                        for (int i4 = 0; i4 < C::kCW / 4; ++i4) {
                            const float4 v = __ldcg(p + i4);
                            if (sl == 0) {
                                acc[2 * i4] = make_float2(v.x, v.y);
                                acc[2 * i4 + 1] = make_float2(v.z, v.w);
                            } else {
                                acc[2 * i4] = __fadd2_rn(acc[2 * i4], make_float2(v.x, v.y));
                                acc[2 * i4 + 1] = __fadd2_rn(acc[2 * i4 + 1], make_float2(v.z, v.w));
                            }
                        }
                    }
                }
            }
            // ---- store the tile
            // Dense and grouped tiles, TMA-store mode: each epilogue warpgroup sends its 128
            // rows out through its staging buffer, 32 bf16 columns (or 64 E4M3 codes) per TMA
            // store, which the tensor map clips at the M and N edges.  A tile whose rows end
            // at a row_end inside the output (a masked or prefix-sum group's last rows), and
            // every tile in direct mode, is stored row by row from the registers instead
            // (16-byte stores; rows from row_end on stay untouched).
            const bool whole_tile = args.tma_store != 0 && (tc.row_end >= args.M || tc.p0 + C::kP <= tc.row_end);
            // the 64 bytes of this thread's row from column x; elem_bytes 2 (bf16) or 1 (E4M3)
            auto out_round = [&](const uint32_t (&w)[16], int x, void* row_ptr, int elem_bytes) {
                if (whole_tile) {
                    stage_store_round(stage_buf, row, stage_leader, 1u + static_cast<uint32_t>(wg), w, &map_d, x, tc.p0);
                } else if (row_ptr != nullptr) {
                    // 16-byte chunks that lie inside the row (N is a multiple of 16)
                    const int chunks = min(4, (args.N - x) * elem_bytes / 16);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        if (c < chunks)
                            reinterpret_cast<uint4*>(row_ptr)[c] =
                                make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                }
            };
            if constexpr (C::SILU) {
                // h[m][q0 + wg*64 + i] = silu(gate_i) * up_i: acc[0 .. kCW/4) hold the gate
                // columns in pairs, acc[kCW/4 ..) the up columns of the same outputs
                const int m = tc.p0 + row;
                const int n0 = tc.q0 + wg * (C::kCW / 2);
                if (n0 < args.N) {
#pragma unroll
                    for (int rr = 0; rr < C::kCW / 64; ++rr) {
                        uint32_t w[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float2 g = acc[rr * 16 + i];
                            const float2 u = acc[C::kCW / 4 + rr * 16 + i];
                            w[i] = pack_bf16x2(g.x / (1.0f + expf(-g.x)) * u.x, g.y / (1.0f + expf(-g.y)) * u.y);
                        }
                        const int n = n0 + 32 * rr;
                        out_round(w, n, m < tc.row_end ? args.d + static_cast<long long>(m) * args.N + n : nullptr, 2);
                    }
                }
            } else if constexpr (!C::SWAP) {
                const int m = tc.p0 + row;
                const int n0 = tc.q0 + wg * C::kCW;
                if (args.bias != nullptr) {
#pragma unroll
                    for (int c = 0; c < C::kCW / 8; ++c) {
                        if (n0 + c * 8 < args.N) {
                            const uint4 b = *reinterpret_cast<const uint4*>(args.bias + n0 + c * 8);
                            acc[c * 4 + 0] = __fadd2_rn(acc[c * 4 + 0], make_float2(bf16_lo(b.x), bf16_hi(b.x)));
                            acc[c * 4 + 1] = __fadd2_rn(acc[c * 4 + 1], make_float2(bf16_lo(b.y), bf16_hi(b.y)));
                            acc[c * 4 + 2] = __fadd2_rn(acc[c * 4 + 2], make_float2(bf16_lo(b.z), bf16_hi(b.z)));
                            acc[c * 4 + 3] = __fadd2_rn(acc[c * 4 + 3], make_float2(bf16_lo(b.w), bf16_hi(b.w)));
                        }
                    }
                }
                if (args.q_out != nullptr) {
                    if constexpr (C::kCW == 128) {
                        // this thread's 128 columns are one 1 x 128 group of row m: round
                        // to bf16 as the D store would, then quantize exactly as the
                        // activation quantize kernel does (rows past M hold zeros and are
                        // clipped by the store)
                        if (n0 < args.N) {
                            uint32_t h[64];
#pragma unroll
                            for (int i = 0; i < 64; ++i) h[i] = pack_bf16x2(acc[i].x, acc[i].y);
                            float amax = 0.f;
#pragma unroll
                            for (int i = 0; i < 64; ++i)
                                amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(h[i])), fabsf(bf16_hi(h[i]))));
                            const float sv = scale_of_amax(amax);
                            float r_lo = 0.f, r_hi = 0.f;
                            if (sv >= 0x1p-125f) bracket_rcp(sv, r_lo, r_hi);
                            const bool zero_group = sv == 0.0f, exact_group = !(sv >= 0x1p-125f);
#pragma unroll
                            for (int rr = 0; rr < 2; ++rr) {
                                // codes of columns 64 rr .. 64 rr + 63
                                uint32_t w[16];
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const int k = 32 * rr + 4 * j;
                                    const uint2 c = codes8(make_uint4(h[k], h[k + 1], h[k + 2], h[k + 3]), sv, r_lo, r_hi,
                                                           zero_group, exact_group);
                                    w[2 * j] = c.x;
                                    w[2 * j + 1] = c.y;
                                }
                                out_round(w, n0 + 64 * rr,
                                          m < tc.row_end ? args.q_out + static_cast<long long>(m) * args.N + n0 + 64 * rr
                                                         : nullptr,
                                          1);
                            }
                            if (m < tc.row_end) {
                                args.sfa_out[static_cast<long long>(n0 >> 7) * args.M4_out + m] = sv;
                            } else if (m >= args.M && m < args.M4_out) {
                                // rows past M up to the padded scale count carry a zero scale
                                args.sfa_out[static_cast<long long>(n0 >> 7) * args.M4_out + m] = 0.f;
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int rr = 0; rr < C::kCW / 32; ++rr) {
                        const int n = n0 + 32 * rr;
                        if (n < args.N) {
                            uint32_t w[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(acc[16 * rr + i].x, acc[16 * rr + i].y);
                            out_round(w, n, m < tc.row_end ? args.d + static_cast<long long>(m) * args.N + n : nullptr, 2);
                        }
                    }
                }
            } else {
                store_decode_tile<C>(args, tc, row, wg * C::kCW, acc);
            }
        }
        // every TMA store of this warpgroup has completed before the CTA may leave
        if constexpr (!C::SWAP) {
            if (stage_leader) bulk_wait_all();
            __syncwarp();
        }
    }

    if constexpr (C::PAIR) {
        // no CTA leaves while its peer may still signal its barriers or read TMEM
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
