/*
 * lnq.h -- C ABI of liblnq.so: the fine-grained block-scaled FP8 linear
 * D = A . B^T on NVIDIA B200 (sm_100a), and its M-grouped contiguous MoE
 * variant.
 *
 * Numerics (the "DeepSeek gran-128" recipe):
 *   - activations are quantized per row in groups of 128 consecutive inputs,
 *     each group with its own FP32 scale s = amax / 448 and E4M3 codes
 *     q = E4M3_RNE_saturating(x / s)
 *       (Linnet "Backend plugins", DeepGEMM plugin source, docstring and
 *        _BlockProduct.execute; deepgemm-rust README, "What's implemented",
 *        fp8_gemm_nt row);
 *   - weights are E4M3 in 128 x 128 blocks with one FP32 scale per block
 *       (Linnet plugin docstring; deepgemm-rust README, "Quick start");
 *   - the product of each 128-wide K block is accumulated in FP32 on the
 *     tensor cores, multiplied by sa * sb and added into an FP32 accumulator;
 *     the output is BF16 (deepgemm-rust README, "What's implemented":
 *     "FP32 promotion, BF16 out").
 *
 * Conventions shared by every call:
 *   - All pointers are device pointers (cudaMalloc / PyTorch CUDA memory) on
 *     the current device, 16-byte aligned, except the weight-scale tensor
 *     sfb and the group ids m_indices, which need 4-byte alignment.  The
 *     library never takes ownership, never allocates device memory and
 *     never synchronizes the stream (except lnq_get_last_device_error).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on that stream.
 *   - Argument errors are detected on the host and returned before any CUDA
 *     call; on such an error nothing is launched and no output is written.
 *     LNQ_ERR_CUDA reports a failed CUDA runtime/driver call (launch or
 *     descriptor encoding).  A kernel whose bounded wait expired reports it
 *     through lnq_get_last_device_error.
 *   - K must be a multiple of 128 (deepgemm-rust README, "Quick start":
 *     "k must be a multiple of 128").
 *   - E4M3 tensors are OCP FP8 E4M3 ("e4m3fn") bytes, BF16 tensors raw
 *     bfloat16, all row-major.
 */
#ifndef LNQ_H
#define LNQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lnq_status {
    LNQ_OK = 0,
    LNQ_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad stride */
    LNQ_ERR_UNSUPPORTED_SHAPE = 2, /* K % 128 != 0, N % 16 != 0, M4 < ceil4(M), ... */
    LNQ_ERR_MISALIGNED = 3,        /* a pointer not 16-byte aligned */
    LNQ_ERR_UNSUPPORTED_ARCH = 4,  /* current device is not compute capability 10.0 */
    LNQ_ERR_CUDA = 5,              /* a CUDA call failed */
    LNQ_ERR_TIMEOUT = 6            /* a kernel's bounded wait expired (device-reported) */
} lnq_status;

/*
 * Activation quantization, 1 x 128 groups (amax, scale and E4M3 cast fused in
 * one pass over the input).
 *
 *   x_bf16  [M][ld_x] bf16; the first K columns of each row are read.
 *   q_e4m3  [M][ld_q] E4M3; the first K columns of each row are written.
 *   sfa     [K/128][M4] fp32, MN-major ("column by column"): the scale of
 *           row m, group g is sfa[g*M4 + m].  Entries m in [M, M4) are
 *           written as 0.0f.  M4 >= ceil4(M) and M4 % 4 == 0, so each scale
 *           column starts 16-byte aligned (Linnet plugin: "the rows padded
 *           to a multiple of four and the scales column by column";
 *           _BlockProduct.execute, `padded`).
 *   Scale s = amax/448 as an IEEE fp32 division; q = E4M3 round-to-nearest-
 *   even of the correctly rounded fp32 quotient x/s, saturating at +-448.  A
 *   group with amax == 0 gets s = 0.0f and codes 0x00 (0x80 for -0.0).
 *
 *   Requires: M >= 0 (M == 0 writes nothing), K % 128 == 0, ld_x >= K,
 *   ld_x % 8 == 0, ld_q >= K, ld_q % 16 == 0, pointers 16-byte aligned.
 */
lnq_status lnq_quantize_fp8_groups(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x,
                                   void* q_e4m3, int64_t ld_q, float* sfa, int64_t M4,
                                   void* stream);

/*
 * Weight quantization, 128 x 128 blocks (offline preparation of the weight
 * operand; Linnet plugin docstring, "weight blocks of 128 by 128";
 * deepgemm-rust README, "Quick start", sfb shape (n/128, k/128)).
 *
 *   w_bf16  [N][K] bf16 row-major.
 *   q_e4m3  [N][K] E4M3.
 *   sfb     [ceil(N/128)][K/128] fp32 row-major: the scale of the block
 *           (nb, kb) is sfb[nb*(K/128) + kb].  A ragged last row block takes
 *           its amax over the rows that exist.
 *   Same scale and rounding rule as lnq_quantize_fp8_groups.
 *   Grouped weights [G*N][K] whose N is not a multiple of 128 are quantized
 *   one group at a time (w + g*N*K, q + g*N*K, sfb + g*ceil(N/128)*(K/128)),
 *   so that no 128 x 128 block spans two groups.
 *   Requires: N >= 1, K % 128 == 0, w and q 16-byte aligned, sfb 4-byte
 *   aligned.
 */
lnq_status lnq_quantize_fp8_blocks(const void* w_bf16, int64_t N, int64_t K, void* q_e4m3,
                                   float* sfb, void* stream);

/*
 * Block-scaled FP8 GEMM, "nt" (both operands K-major):
 *   D[m][n] = bf16_RN( sum_g  sfa[g*M4+m] * sfb[(n/128)*(K/128)+g]
 *                              * sum_{k in block g} a[m][k] * b[n][k] )
 * with the inner sums on the tensor cores (FP32) and the promotion in FP32
 * (deepgemm-rust README, "What's implemented", fp8_gemm_nt; Linnet plugin,
 * _BlockProduct.execute, deep_gemm.fp8_gemm_nt((q, scales), (weight, f32
 * scale), out, disable_ue8m0_cast=True)).
 *
 *   a_e4m3  [M][K] E4M3 (activations, row stride K).
 *   sfa     [K/128][M4] fp32 MN-major, as written by lnq_quantize_fp8_groups.
 *   b_e4m3  [N][K] E4M3 (weights, row stride K).
 *   sfb     [ceil(N/128)][K/128] fp32, as written by lnq_quantize_fp8_blocks.
 *   d_bf16  [M][N] bf16 row-major (row stride N), fully overwritten.
 *   Requires: M >= 1, N >= 16, N % 16 == 0, K % 128 == 0, M4 >= ceil4(M),
 *   M4 % 4 == 0, sfb 4-byte aligned, the other pointers 16-byte aligned.
 *   M <= 64 runs the decode configuration (weights in the MMA's M slot);
 *   larger M runs the persistent 128 x BN tile kernel.
 */
lnq_status lnq_fp8_block_gemm_nt(const void* a_e4m3, const float* sfa, int64_t M4,
                                 const void* b_e4m3, const float* sfb, void* d_bf16, int64_t M,
                                 int64_t N, int64_t K, void* stream);

/*
 * lnq_fp8_block_gemm_nt with a fused epilogue: an optional bias, and the output
 * either in bf16 or already quantized for a next linear (deepgemm-rust README,
 * "Key techniques": fused epilogues; Linnet plugin, _BlockProduct.execute adds
 * the bias after the product).
 *
 *   bias_bf16  [N] bf16 or NULL (16-byte aligned): added to every row in FP32
 *              before the output rounding.
 *   d_bf16     [M][N] bf16 output, or NULL when q_e4m3 is given.
 *   q_e4m3     [M][N] E4M3 output, or NULL: the result is rounded to bf16 (the
 *              values d_bf16 would hold) and quantized per row in 1 x 128 groups
 *              exactly as lnq_quantize_fp8_groups quantizes a bf16 input.
 *   sfa_out    [N/128][M4_out] fp32 scales of q_e4m3 (MN-major; rows M ..
 *              M4_out-1 get 0.0f), as lnq_quantize_fp8_groups writes them.
 *   M4_out     >= ceil4(M), a multiple of 4.
 *   Exactly one of d_bf16 and q_e4m3 is given.  The quantized output needs
 *   M > 64, N >= 256 and N % 128 == 0 (LNQ_ERR_UNSUPPORTED_SHAPE otherwise);
 *   q_e4m3 and sfa_out 16-byte aligned.  Other arguments as
 *   lnq_fp8_block_gemm_nt.
 */
lnq_status lnq_fp8_block_gemm_nt_epilogue(const void* a_e4m3, const float* sfa, int64_t M4,
                                          const void* b_e4m3, const float* sfb, const void* bias_bf16,
                                          void* d_bf16, void* q_e4m3, float* sfa_out, int64_t M4_out,
                                          int64_t M, int64_t N, int64_t K, void* stream);

/*
 * Gate_up linear with SiLU.mul fused into its epilogue (deepgemm-rust README,
 * "What's implemented", moe_fp8_layer: grouped GEMM -> SiLU.mul -> grouped GEMM):
 *     h[m][j] = bf16( silu(D[m][j]) * D[m][I + j] ),  silu(x) = x / (1 + e^-x),
 * D = A . B^T promoted in FP32 as in lnq_fp8_block_gemm_nt; gate and up values
 * are the FP32 products (D is never rounded to bf16).
 *
 *   b_e4m3   [2I][K] E4M3: the I gate rows, then the I up rows.
 *   sfb      [2I/128][K/128] fp32, as lnq_quantize_fp8_blocks writes for 2I rows.
 *   h_bf16   [M][I] bf16 row-major, fully overwritten.
 *   Requires: M >= 1, I % 128 == 0, K % 128 == 0, M4 >= ceil4(M), M4 % 4 == 0,
 *   sfb 4-byte aligned, the other pointers 16-byte aligned.  M > 128 runs
 *   256-row tiles on CTA pairs (unless lnq_set_dense_cta_pairs(0)).
 */
lnq_status lnq_fp8_block_gemm_nt_silu_mul(const void* a_e4m3, const float* sfa, int64_t M4,
                                          const void* b_e4m3, const float* sfb, void* h_bf16,
                                          int64_t M, int64_t I, int64_t K, void* stream);

/*
 * Bytes of workspace that lnq_fp8_block_gemm_nt_ws needs to split the K range of
 * a decode product (M <= 64) over `num_sms` CTAs, or 0 when the product does not
 * split (M > 64, K == 128, or at least one weight tile per SM already).  A pure
 * host computation: no device is touched.
 */
int64_t lnq_fp8_block_gemm_nt_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t num_sms);

/*
 * lnq_fp8_block_gemm_nt with a caller-owned workspace for the decode split.
 *
 * Decode products have fewer 128-row weight tiles than the GPU has SMs (96 for
 * N = 12288).  With a workspace, every SM takes an equal contiguous run of the
 * (weight tile, 128-wide K block) units; a CTA that covers part of a tile's K
 * range writes its FP32 partial tile into the workspace and counts itself in the
 * tile's counter, and the CTA that completes the count adds the tile's partials
 * in order of their K ranges (a fixed order: the result does not depend on
 * timing), stores the bf16 tile and resets the counter.  The FP32 promotion per
 * 128-wide K block is the same as in lnq_fp8_block_gemm_nt; only the grouping of
 * the block sums differs, so results agree within FP32 rounding.
 *
 *   workspace        device memory of at least
 *                    lnq_fp8_block_gemm_nt_workspace_bytes(M, N, K, SMs of the
 *                    current device) bytes, 256-byte aligned, ZEROED before its
 *                    first use.  Its first 4 KiB hold one counter per weight tile
 *                    and every call leaves them zero again; the partial tiles
 *                    follow.  So one workspace, sized for the largest product, serves
 *                    any sequence of products.  The caller owns it.  Calls that share
 *                    a workspace must be ordered (one stream); after an error
 *                    (LNQ_ERR_TIMEOUT) zero it again.
 *   workspace_bytes  its size.
 *   Other arguments and requirements as lnq_fp8_block_gemm_nt.  With workspace ==
 *   NULL, or for products that do not split, this is lnq_fp8_block_gemm_nt.  A
 *   workspace smaller than needed returns LNQ_ERR_INVALID_ARG, a misaligned one
 *   LNQ_ERR_MISALIGNED, before any launch.
 */
lnq_status lnq_fp8_block_gemm_nt_ws(const void* a_e4m3, const float* sfa, int64_t M4,
                                    const void* b_e4m3, const float* sfb, void* d_bf16, int64_t M,
                                    int64_t N, int64_t K, void* workspace, int64_t workspace_bytes,
                                    void* stream);

/*
 * lnq_fp8_block_gemm_nt_ws with the library's own fixed scratch instead of a
 * caller's workspace: this entry point allocates nothing.  The pages have no
 * counterpart; it exists for callers that may not allocate device memory around
 * the call.
 *
 * The scratch is one file-scope device array of 10 MiB (10485760 bytes) per
 * device, whose address is looked up once per device.  Products whose split needs
 * more (lnq_fp8_block_gemm_nt_workspace_bytes above 10 MiB; M = 64, N = 12288,
 * K = 4096 needs 9.0 MiB) return LNQ_ERR_UNSUPPORTED_SHAPE before any launch;
 * products that do not split run lnq_fp8_block_gemm_nt.
 *
 * The array is shared by every call on the device: calls that overlap in time (on
 * different streams, or from several threads without ordering) race on it and
 * must not be issued.  After a call the array keeps that call's partial tiles
 * (its counters are zero again).  A call that gave up on a wait may leave tile
 * counters non-zero; lnq_get_last_device_error, when it reports LNQ_ERR_TIMEOUT,
 * zeroes the counter region of the array on the current device (a memset of its
 * first 4 KiB; nothing is allocated), so later calls are correct again.
 * Argument errors are returned before any CUDA call, as for lnq_fp8_block_gemm_nt;
 * a device numbered 64 or above returns LNQ_ERR_INVALID_ARG.
 */
lnq_status lnq_fp8_block_gemm_nt_static_ws(const void* a_e4m3, const float* sfa, int64_t M4,
                                           const void* b_e4m3, const float* sfb, void* d_bf16,
                                           int64_t M, int64_t N, int64_t K, void* stream);

/*
 * M-grouped contiguous block-scaled FP8 GEMM (MoE experts): tokens of all
 * groups concatenated along M, every group starting at a multiple of 128
 * rows, a per-row group id (deepgemm-rust README, "Grouped (contiguous) MoE
 * GEMM" and "What's implemented", m_grouped_fp8_gemm_nt_contiguous;
 * Triton_Grouped_GEMM README, "Example DeepGEMM layout creation").
 *
 *   a_e4m3     [M_total][K] E4M3.
 *   sfa        [K/128][M_total] fp32 MN-major.
 *   b_e4m3     [num_groups*N][K] E4M3: rows g*N .. g*N+N-1 are group g's weights.
 *   sfb        [num_groups*ceil(N/128)][K/128] fp32: row g*ceil(N/128)+nb
 *              (each group's weights quantized on their own).
 *   m_indices  [M_total] int32: group of each row, or -1 for a pad row.  Each
 *              128-row block takes the group of its first row; a block whose
 *              first row is -1 is skipped (its D rows are not written).  Pad
 *              rows inside a block are computed with the block's group and
 *              their D rows are unspecified.
 *   d_bf16     [M_total][N] bf16.
 *   Requires: M_total >= 128, M_total % 128 == 0, num_groups >= 1,
 *   N % 16 == 0, K % 128 == 0, ids < num_groups (a block whose id is out of
 *   range is skipped and reported by lnq_get_last_device_error as
 *   LNQ_ERR_INVALID_ARG), sfb and m_indices 4-byte aligned, the other
 *   pointers 16-byte aligned.
 */
lnq_status lnq_m_grouped_fp8_gemm_contiguous(const void* a_e4m3, const float* sfa,
                                             const void* b_e4m3, const float* sfb,
                                             const int32_t* m_indices, int32_t num_groups,
                                             void* d_bf16, int64_t M_total, int64_t N, int64_t K,
                                             void* stream);

/*
 * M-grouped contiguous block-scaled FP8 GEMM with the prefix-sum group layout
 * (deepgemm-rust README: the device-level m_grouped contiguous entry point
 * "(psum layout)", and "The mk_alignment knob (MoE tile width)": each group's
 * tokens start at an aligned row of the A arena; on SM100 the alignment may be
 * 256 so that tiles run at the MMA's full 256-row width).  The group boundaries
 * stay on the device: no per-row ids and no host synchronization.
 *
 *   psum        [num_groups] int32 on the device: psum[g] = tokens of groups
 *               0..g (non-decreasing).  Group g has count_g = psum[g] -
 *               psum[g-1] tokens (psum[-1] = 0) at rows start_g .. start_g +
 *               count_g - 1 of the arena, start_0 = 0 and start_{g+1} = start_g +
 *               align_up(count_g, alignment).
 *   alignment   128 or 256 (the mk_alignment of the layout).  Tiles are 128
 *               rows; those holding pad rows only are skipped, so both
 *               alignments compute the same rows.  With 256, N >= 256 and
 *               lnq_set_grouped_cta_pairs(1) the tiles are 256 x 256 on CTA pairs.
 *   a_e4m3      [M_total][K] E4M3 arena; sfa [K/128][M_total] fp32 MN-major.
 *   b_e4m3      [num_groups*N][K] E4M3, sfb [num_groups*ceil(N/128)][K/128] fp32:
 *               as in lnq_m_grouped_fp8_gemm_contiguous.
 *   d_bf16      [M_total][N] bf16: the rows of each group's tokens are written;
 *               pad rows and rows past the last group are left untouched.
 *   Requires: alignment in {128, 256} (else LNQ_ERR_INVALID_ARG), M_total %
 *   alignment == 0, N % 16 == 0, K % 128 == 0, sfb and psum 4-byte aligned, the
 *   other pointers 16-byte aligned.  A decreasing psum (its negative counts are
 *   taken as zero) or groups that overrun M_total (rows from M_total on are not
 *   written) are reported by lnq_get_last_device_error as LNQ_ERR_INVALID_ARG.
 */
lnq_status lnq_m_grouped_fp8_gemm_contiguous_psum(const void* a_e4m3, const float* sfa,
                                                  const void* b_e4m3, const float* sfb,
                                                  const int32_t* psum, int32_t num_groups,
                                                  int64_t alignment, void* d_bf16, int64_t M_total,
                                                  int64_t N, int64_t K, void* stream);

/*
 * M-grouped masked block-scaled FP8 GEMM (MoE experts fed by a token dispatch):
 * every group has a fixed buffer of M_max rows, of which only the first
 * masked_m[g] hold tokens; the counts stay on the device, so no host
 * synchronization is needed (deepgemm-rust README, "What's implemented",
 * m_grouped_fp8_gemm_nt_masked: masked_m scheduler, DeepEP-style dispatch
 * output, expected_m scheduling, zero CPU sync).
 *
 *   a_e4m3      [num_groups*M_max][K] E4M3: rows g*M_max .. g*M_max + M_max - 1
 *               are group g's buffer (a [num_groups][M_max][K] tensor).
 *   sfa         [K/128][num_groups*M_max] fp32 MN-major over all those rows, as
 *               lnq_quantize_fp8_groups writes for M = num_groups*M_max.
 *   b_e4m3      [num_groups*N][K] E4M3, sfb [num_groups*ceil(N/128)][K/128] fp32:
 *               as in lnq_m_grouped_fp8_gemm_contiguous.
 *   masked_m    [num_groups] int32 on the device: real rows of each group,
 *               0 .. M_max.  A count outside that range is clamped and reported
 *               by lnq_get_last_device_error as LNQ_ERR_INVALID_ARG.
 *   expected_m  the caller's estimate of the rows per group (>= 0); a scheduling
 *               hint only, results do not depend on it.
 *   d_bf16      [num_groups*M_max][N] bf16: rows g*M_max + m for m < masked_m[g]
 *               are written; the other rows are left untouched.
 *   Requires: M_max % 128 == 0, N % 16 == 0, K % 128 == 0, sfb and masked_m
 *   4-byte aligned, the other pointers 16-byte aligned.
 */
lnq_status lnq_m_grouped_fp8_gemm_masked(const void* a_e4m3, const float* sfa, const void* b_e4m3,
                                         const float* sfb, const int32_t* masked_m,
                                         int32_t num_groups, int64_t M_max, int64_t expected_m,
                                         void* d_bf16, int64_t N, int64_t K, void* stream);

/*
 * UE8M0 recipe (deepgemm-rust README, "Blackwell-native FP4/FP8 (SM100a,
 * tcgen05)": UE8M0 power-of-two scales copied into tensor memory and consumed
 * by the block-scaled MMA; "What's implemented": gran-128 on either side).
 * The same 1 x 128 activation groups and 128 x 128 weight blocks as the
 * FP32-scale recipe; each scale is the smallest power of two p with
 * 448 p >= amax (no code saturates; an all-zero group takes p = 1), stored as
 * the byte e + 127 of p = 2^e, e clamped to [-127, 127].  Codes are the E4M3
 * round-to-nearest-even of x / p.
 *
 * Scale atoms: for each K block kb and 128-row block rb, 128 uint32 words; row
 * r = r0 + 32 r1 of the block (r0 < 32, r1 < 4) owns word 4 r0 + r1, whose low
 * byte is the row's exponent byte (the other bytes 0).  Each atom is 512
 * contiguous bytes, the layout the tensor core's scale copy reads.
 *
 * lnq_quantize_ue8m0_groups: x bf16 [M][ld_x] -> q E4M3 [M][ld_q] and
 *   sfa_atoms uint32 [K/128][ceil(M/128)][128] (rows M .. of the last block get
 *   p = 1).  Requires K % 128 == 0, ld_x % 8 == 0, ld_q % 16 == 0, pointers
 *   16-byte aligned.
 * lnq_quantize_ue8m0_blocks: w bf16 [N][K] -> q E4M3 [N][K] and sfb_atoms uint32
 *   [K/128][ceil(N/128)][128], every row of a block carrying the block's byte.
 *   Requires K % 128 == 0, pointers 16-byte aligned.
 * lnq_mx_block_gemm_nt: D[m][n] = bf16( sum_k a[m][k] 2^ea[m][k/128] *
 *   b[n][k] 2^eb[n/128][k/128] ), the scales applied by the tensor core
 *   (tcgen05.mma kind::mxf8f6f4.block_scale) and the sum accumulated in FP32
 *   over the whole K range.  a_e4m3 [M][K], b_e4m3 [N][K] (K-major), d_bf16
 *   [M][N] fully overwritten.  Requires N % 16 == 0, K % 128 == 0, pointers
 *   16-byte aligned.  M > 128 runs 256 x 256 tiles on CTA pairs (unless
 *   lnq_set_dense_cta_pairs(0)).
 */
lnq_status lnq_quantize_ue8m0_groups(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, void* q_e4m3,
                                     int64_t ld_q, void* sfa_atoms, void* stream);
lnq_status lnq_quantize_ue8m0_blocks(const void* w_bf16, int64_t N, int64_t K, void* q_e4m3, void* sfb_atoms,
                                     void* stream);
lnq_status lnq_mx_block_gemm_nt(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3,
                                const void* sfb_atoms, void* d_bf16, int64_t M, int64_t N, int64_t K,
                                void* stream);

/*
 * lnq_mx_block_gemm_nt for the M-grouped contiguous MoE layout (deepgemm-rust
 * README, "Grouped (contiguous) MoE GEMM"): each 128-row block of the A arena
 * takes the weights of the group named by its first row's id, as in
 * lnq_m_grouped_fp8_gemm_contiguous.
 *   a_e4m3 [M_total][K], sfa_atoms from lnq_quantize_ue8m0_groups over M_total rows;
 *   b_e4m3 [num_groups*N][K], sfb_atoms from lnq_quantize_ue8m0_blocks over all
 *   num_groups*N rows (N % 128 == 0, so no weight block spans two groups);
 *   m_indices int32 [M_total]: a block whose first id is negative is skipped (its
 *   rows of D untouched); pad rows inside a block are computed with the block's
 *   group and their rows of D are unspecified; an id >= num_groups skips the
 *   block and is reported by lnq_get_last_device_error as LNQ_ERR_INVALID_ARG.
 *   Requires M_total % 128 == 0, N % 128 == 0, K % 128 == 0, m_indices 4-byte
 *   aligned, the other pointers 16-byte aligned.
 */
lnq_status lnq_m_grouped_mx_gemm_contiguous(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3,
                                            const void* sfb_atoms, const int32_t* m_indices, int32_t num_groups,
                                            void* d_bf16, int64_t M_total, int64_t N, int64_t K, void* stream);

/*
 * MXFP8 gran-32 recipe (deepgemm-rust README, benchmark block "SM100 FP8:
 * DeepSeek gran-128 recipe and MXFP8 gran-32"; kernel table, kind::mxf8f6f4
 * with UE8M0 scales).  Every row of an operand, activations and weights alike,
 * is quantized in 1 x 32 blocks along K, each block with its own UE8M0 scale
 * chosen by the rule of the gran-128 recipe above (the smallest power of two p
 * with 448 p >= amax; p = 1 for an all-zero block), codes the E4M3 RNE of x / p.
 *
 * Scale atoms as for the gran-128 recipe ([K/128][ceil(rows/128)][128] uint32
 * words, row r = r0 + 32 r1 of a 128-row block in word 4 r0 + r1), except that
 * the word of a row holds the exponent bytes of its four 32-blocks of the 128-wide
 * K block: 32-block j in byte j.  The tensor core reads byte j for the j-th K = 32
 * step (the scale-ID fields of the block-scaled MMA).
 *
 * lnq_quantize_mxfp8: x bf16 [rows][ld_x] -> q E4M3 [rows][ld_q] and sf_atoms
 *   uint32 [K/128][ceil(rows/128)][128]; rows past `rows` in the last 128-row
 *   block get p = 1 in all four bytes.  The same call quantizes activations and
 *   weights.  Requires K % 128 == 0, ld_x % 8 == 0, ld_q % 16 == 0, pointers
 *   16-byte aligned.
 * lnq_mxfp8_gemm_nt: D[m][n] = bf16( sum_k a[m][k] 2^ea[m][k/32] b[n][k]
 *   2^eb[n][k/32] ), the scales applied by the tensor core
 *   (tcgen05.mma kind::mxf8f6f4.block_scale, one scale byte per row per K = 32)
 *   and the sum accumulated in FP32 over the whole K range.  a_e4m3 [M][K],
 *   b_e4m3 [N][K], d_bf16 [M][N] fully overwritten.  Requires N % 16 == 0,
 *   K % 128 == 0, pointers 16-byte aligned.
 * lnq_m_grouped_mxfp8_gemm_contiguous: the same for the M-grouped contiguous
 *   layout, with the arguments and requirements of
 *   lnq_m_grouped_mx_gemm_contiguous (sfb_atoms from lnq_quantize_mxfp8 over all
 *   num_groups*N weight rows).
 */
lnq_status lnq_quantize_mxfp8(const void* x_bf16, int64_t rows, int64_t K, int64_t ld_x, void* q_e4m3, int64_t ld_q,
                              void* sf_atoms, void* stream);
lnq_status lnq_mxfp8_gemm_nt(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3, const void* sfb_atoms,
                             void* d_bf16, int64_t M, int64_t N, int64_t K, void* stream);
lnq_status lnq_m_grouped_mxfp8_gemm_contiguous(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3,
                                               const void* sfb_atoms, const int32_t* m_indices, int32_t num_groups,
                                               void* d_bf16, int64_t M_total, int64_t N, int64_t K, void* stream);

/*
 * The UE8M0 (gran-128) and MXFP8 (gran-32) recipes in the M-grouped masked layout
 * (deepgemm-rust README, "What's implemented": the masked_m scheduler of the
 * DeepEP-style dispatch output, zero CPU sync; "Full recipes": gran-32 and
 * gran-128 on either side): as lnq_m_grouped_fp8_gemm_masked, with the scales in
 * atoms.
 *   a_e4m3      [num_groups*M_max][K] E4M3, group g's buffer in rows g*M_max ..
 *               g*M_max + M_max - 1; sfa_atoms over all num_groups*M_max rows, from
 *               lnq_quantize_ue8m0_groups (lnq_m_grouped_mx_gemm_masked) or
 *               lnq_quantize_mxfp8 (lnq_m_grouped_mxfp8_gemm_masked).
 *   b_e4m3      [num_groups*N][K] E4M3 and sfb_atoms over all num_groups*N rows, from
 *               lnq_quantize_ue8m0_blocks or lnq_quantize_mxfp8.
 *   masked_m    [num_groups] int32 on the device: real rows of each group, 0 .. M_max;
 *               a count outside that range is clamped and reported by
 *               lnq_get_last_device_error as LNQ_ERR_INVALID_ARG.
 *   expected_m  a scheduling hint (>= 0); results do not depend on it.
 *   d_bf16      [num_groups*M_max][N] bf16: rows g*M_max + m for m < masked_m[g] are
 *               written, the other rows left untouched.
 *   Requires M_max % 128 == 0, N % 128 == 0, K % 128 == 0, masked_m 4-byte aligned,
 *   the other pointers 16-byte aligned.
 */
lnq_status lnq_m_grouped_mx_gemm_masked(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3,
                                        const void* sfb_atoms, const int32_t* masked_m, int32_t num_groups,
                                        int64_t M_max, int64_t expected_m, void* d_bf16, int64_t N, int64_t K,
                                        void* stream);
lnq_status lnq_m_grouped_mxfp8_gemm_masked(const void* a_e4m3, const void* sfa_atoms, const void* b_e4m3,
                                           const void* sfb_atoms, const int32_t* masked_m, int32_t num_groups,
                                           int64_t M_max, int64_t expected_m, void* d_bf16, int64_t N, int64_t K,
                                           void* stream);

/* Static text for a status code. */
const char* lnq_status_string(lnq_status status);

/*
 * Synchronizes `stream`, then reads and clears the library's device status
 * word on the current device.  Returns LNQ_ERR_TIMEOUT if a kernel launched
 * since the last call gave up on a bounded wait (the kernel then skipped its
 * remaining work and released its tensor memory; its outputs are
 * unspecified), LNQ_ERR_CUDA if the synchronization failed, else LNQ_OK.
 * On a timeout it also zeroes the tile counters of the scratch array that
 * lnq_fp8_block_gemm_nt_static_ws uses on this device (on `stream`, then
 * synchronizes it again).
 */
lnq_status lnq_get_last_device_error(void* stream);

/*
 * Diagnostic: launches one tiny kernel that waits on a barrier nobody
 * arrives on, with a limit of `timeout_ns` nanoseconds (1e3 .. 1e10), then
 * records LNQ_ERR_TIMEOUT in the device status word exactly as the GEMM
 * kernels do when one of their waits expires.  Used to test the timeout path
 * without faulting or hanging the GPU.  Returns the launch status.
 */
lnq_status lnq_selftest_wait_timeout(int64_t timeout_ns, void* stream);

/*
 * Tuning knob (process-wide, default 1) for dense GEMMs with M > 128:
 *   0  one CTA per 128 x 256 tile (N >= 256);
 *   1  pairs of CTAs (a cluster of two sharing one tcgen05 MMA) on 256 x 256
 *      tiles, each CTA loading half of the weight tile (N >= 256); the
 *      default: it halves the weight bytes each SM loads per K block;
 *   2  pairs of CTAs on 256 x 128 tiles with four accumulators per CTA
 *      (N >= 128).
 * Other values select 0.  Results are the same up to FP32 summation order.
 * The same knob serves the dense UE8M0 and MXFP8 GEMMs (lnq_mx_block_gemm_nt,
 * lnq_mxfp8_gemm_nt) with M > 128: 0 one CTA per 128 x 256 tile, any other mode pairs
 * of CTAs on 256 x 256 tiles (tcgen05.mma.cta_group::2 with block scaling).
 * Returns the previous setting.
 */
int32_t lnq_set_dense_cta_pairs(int32_t enable);

/*
 * Tuning knob (process-wide, default 0) for lnq_m_grouped_fp8_gemm_contiguous_psum
 * with alignment 256 and N >= 256: 1 runs its 256 x 256 tiles on CTA pairs (each
 * CTA loading half of the weight tile, as for dense tiles), any other value
 * 128-row tiles on single CTAs, skipping tiles of pad rows only.  Results are the
 * same up to FP32 summation order.  Returns the previous setting.
 */
int32_t lnq_set_grouped_cta_pairs(int32_t enable);

/*
 * Weight prefetch (process-wide, default 0).  Every kernel of this library is
 * launched with programmatic stream serialization: it may start while the
 * previous kernel of the stream is still running, and waits for that kernel
 * to complete before it reads any input.  When this knob is non-zero, the
 * single-CTA dense and decode GEMMs issue the weight halves of their first
 * pipeline stages before that wait.  Enable it only when the weights and the
 * weight scales passed to the GEMM are not written by kernels that may still
 * be running when the GEMM starts (e.g. they are model parameters prepared
 * before the forward pass).  Returns the previous setting.
 */
int32_t lnq_set_weight_prefetch(int32_t enable);

/*
 * Output path of the dense and grouped GEMMs (process-wide, default 1).  Non-zero:
 * each epilogue warpgroup converts its 128 rows x 32 columns of the tile to bf16 (or
 * its 64 E4M3 codes for the fused FP8 output) into an 8 KB shared-memory buffer in the
 * 64-byte swizzle and writes it with one TMA store (cp.async.bulk.tensor), the box
 * clipped at the M and N edges; 0: every epilogue thread writes its own output row
 * with 16-byte stores.  Tiles of the masked and prefix-sum layouts whose rows end
 * inside the output are always stored row by row.  Results are identical bit for bit;
 * only the speed differs (the TMA stores were measured 1-7% faster per GEMM on the
 * prefill, square and MoE workloads).  Decode tiles (M <= 64) always store directly.
 * Returns the previous setting.
 */
int32_t lnq_set_tma_store(int32_t enable);

/* Version of this ABI (major*10000 + minor*100 + patch). */
int32_t lnq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LNQ_H */
