/*
 * sdattn.h -- C ABI of libsdattn, B200 (sm_100a) attention for the
 * transformer blocks of Stable Diffusion's UNet:  O = softmax(scale Q K^T) V.
 *
 * Source of the method: "Speed Is All You Need: On-Device Acceleration of
 * Large Diffusion Models via GPU-Aware Optimizations" (Chen et al., CVPR
 * Workshops 2023), as summarised in the news page on m.danchuang.com.cn,
 * section on the three optimisations ("improving attention efficiency").
 * That section describes two forms of attention:
 *
 *   1. Partially fused softmax.  Instead of running a full softmax over the
 *      large score matrix A, one kernel reduces A to per-row vectors L and S
 *      (an N x 2 tensor), the reduction split over blocks of A with the
 *      partial results reduced to the final ones; a second kernel fuses the
 *      softmax normalisation with the multiplication by V.
 *      -> sdattn_qk_stats, sdattn_softmax_av
 *   2. FlashAttention: exact attention computed tile by tile in one kernel
 *      without writing A to memory.
 *      -> sdattn_flash (and sdattn_flash_f32o: fp32 O, for bf16 inputs;
 *         sdattn_flash_tf32: fp32 inputs, tf32 products, fp32 O)
 *
 * Variants of the partially fused form, measured against it:
 *   - the page's reduction as a kernel of its own that reads A back
 *     (three passes over A instead of two):
 *      -> sdattn_qk_scores, sdattn_row_stats, sdattn_softmax_av
 *   - A stored in fp16, halving the bytes of A written and read:
 *      -> sdattn_qk_stats_f16a, sdattn_softmax_av_f16a
 *
 * The two specialised kernels the same section names beside attention:
 * group normalisation in one command, and GELU fused with its split and
 * multiplication (the UNet's gated feed-forward activation):
 *      -> sdattn_group_norm, sdattn_geglu
 *
 * The section's third optimisation, 3x3 convolutions by Winograd's minimal
 * filtering with 4x4 tiles:
 *      -> sdattn_wino_filter, sdattn_wino_conv3x3
 *
 * The page gives no formula for L and S.  This library reads them as
 *      L_i = max_j A_ij,     S_i = sum_j exp(A_ij - L_i)      (natural base)
 * with A = scale * Q K^T, so that softmax(A)_ij = exp(A_ij - L_i) / S_i.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensors are caller-owned DEVICE buffers, row-major and contiguous:
 *        Q  [B][H][N][d]      element type desc->dtype
 *        K  [B][H][M][d]      element type desc->dtype
 *        V  [B][H][M][d]      element type desc->dtype
 *        O  [B][H][N][d]      element type desc->dtype
 *        A  [B][H][N][lda]    float32, lda = sdattn_a_ld(desc) >= M; only the
 *                             first M entries of each row are read or written
 *        A16 [B][H][N][lda16] float16 (the fp16-A variant), lda16 =
 *                             sdattn_a16_ld(desc) >= M
 *        LS [B][H][N][2]      float32, (L_i, S_i) pairs
 *  - Every pointer must be 16-byte aligned.  Buffers must not overlap.
 *  - Calls only enqueue work on `stream` (a cudaStream_t, or NULL for the
 *    legacy default stream) and return; results are ready when the stream
 *    reaches them.  Argument errors are detected on the host before anything
 *    is enqueued and nothing is written.  The library allocates no memory,
 *    never calls exit/abort/__trap, and lets no C++ exception cross the ABI.
 *  - The library keeps one device-resident error word per device.  A kernel
 *    whose internal wait exceeds its time limit (about one second) records
 *    SDATTN_ERR_TIMEOUT there and returns early; sdattn_device_error() reads
 *    and clears it.
 *  - Supported: d in {40, 80, 160} (the UNet's head widths), dtype F16 or
 *    BF16, B*H*N and B*H*M below 2^31, M and N at least 1, scale > 0.
 *  - Thread safety: calls on different streams may run concurrently; calls
 *    that share a workspace must be ordered on one stream.
 */
#ifndef SDATTN_H
#define SDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SDATTN_F16 = 0,   /* IEEE binary16 */
    SDATTN_BF16 = 1,  /* bfloat16 */
    SDATTN_F32 = 2    /* IEEE binary32: sdattn_flash_tf32 only */
} sdattn_dtype;

/* Shape of one attention call.  scale is applied to Q K^T (1/sqrt(d) in SD). */
typedef struct {
    int32_t B;        /* batch (2 for a classifier-free-guidance pair) */
    int32_t H;        /* heads */
    int32_t N;        /* query rows per (b, h) */
    int32_t M;        /* key / value rows per (b, h) */
    int32_t d;        /* head width: 40, 80 or 160 */
    int32_t dtype;    /* sdattn_dtype of Q, K, V and O */
    float scale;      /* finite, positive score scale */
} sdattn_desc;

typedef enum {
    SDATTN_OK = 0,
    SDATTN_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, scale not finite and > 0 */
    SDATTN_ERR_UNSUPPORTED = 2,   /* d or dtype outside the supported set */
    SDATTN_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
    SDATTN_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
    SDATTN_ERR_CUDA = 5,          /* a CUDA runtime / driver call failed */
    SDATTN_ERR_TIMEOUT = 6        /* a kernel's bounded wait ran out (device error word) */
} sdattn_status;

/* Row stride of A in floats: M rounded up to a multiple of 4 (16-byte rows).
 * Returns -1 for an invalid descriptor. */
int64_t sdattn_a_ld(const sdattn_desc *desc);

/* Bytes of workspace that sdattn_qk_stats, sdattn_qk_stats_f16a,
 * sdattn_row_stats and sdattn_flash need for this shape on the current device
 * (split-reduction partials plus arrival counters): enough for each of these
 * calls.  The same workspace serves all of them and any shape whose need is
 * at most its size.  It must be zero-filled once before its first use; every
 * completed call leaves all of it zero again.  After SDATTN_ERR_TIMEOUT it
 * must be zero-filled anew.
 * Returns 0 for an invalid descriptor. */
size_t sdattn_workspace_bytes(const sdattn_desc *desc);

/* Partially fused softmax, first kernel: the score matrix and its row
 * statistics, in one launch.
 *   A[b][h][i][j] = scale * sum_k Q[b][h][i][k] K[b][h][j][k]   (fp32, j < M)
 *   LS[b][h][i]   = (L_i, S_i) as defined above.
 * The reduction follows the page's split: each 128-column block of a row is
 * reduced to a partial (m, s) pair, partial pairs are merged per column split,
 * and the last split to finish merges the splits into LS.
 * Q, K: inputs; A, LS: outputs; ws: workspace of ws_bytes >=
 * sdattn_workspace_bytes(desc) bytes, zero-filled before first use. */
sdattn_status sdattn_qk_stats(const sdattn_desc *desc, const void *Q, const void *K,
                              float *A, float *LS, void *ws, size_t ws_bytes,
                              void *stream);

/* Partially fused softmax, second kernel: normalisation fused with the
 * multiplication by V.
 *   O[b][h][i][c] = (sum_j exp(A_ij - L_i) V[b][h][j][c]) / S_i
 * A, LS (as written by sdattn_qk_stats, or by sdattn_qk_scores followed by
 * sdattn_row_stats), V: inputs; O: output.  Needs no workspace: when the
 * 128-row tiles fill under half the SMs, a thread-block cluster of up to 8
 * CTAs shares each tile's key blocks and adds the partial products through
 * distributed shared memory in a fixed order. */
sdattn_status sdattn_softmax_av(const sdattn_desc *desc, const float *A, const float *LS,
                                const void *V, void *O, void *stream);

/* Three-pass variant, first pass: the score matrix alone,
 *   A[b][h][i][j] = scale * sum_k Q[b][h][i][k] K[b][h][j][k]   (fp32, j < M),
 * bit for bit the A that sdattn_qk_stats writes.  Q, K: inputs; A: output.
 * Needs no workspace. */
sdattn_status sdattn_qk_scores(const sdattn_desc *desc, const void *Q, const void *K, float *A,
                               void *stream);

/* Three-pass variant, second pass: the page's stand-alone reduction of a
 * materialised A to LS[b][h][i] = (L_i, S_i), reading A once (summary of the
 * paper, partially fused softmax paragraph: blocks of A reduced to partial
 * results, which are reduced to the final ones, one GPU command).  Each row,
 * or each column split of a row when rows are few, is reduced by one warp
 * with coalesced 16-byte loads and warp shuffles; the splits of a row are
 * merged by the last one to finish.
 * A: input (layout of sdattn_qk_stats' A); LS: output.  ws / ws_bytes: the
 * workspace (zero-filled before first use, left zero by every completed
 * call) of at least sdattn_workspace_bytes(desc) bytes; it may be NULL / 0
 * when B*H*N is at least 32 times the SM count (no row is split then), and a
 * split call without one returns SDATTN_ERR_WORKSPACE. */
sdattn_status sdattn_row_stats(const sdattn_desc *desc, const float *A, float *LS, void *ws,
                               size_t ws_bytes, void *stream);

/* Row stride of fp16-stored A, in elements: M rounded up to a multiple of 8
 * (16-byte rows).  Returns -1 for an invalid descriptor. */
int64_t sdattn_a16_ld(const sdattn_desc *desc);

/* fp16-A variant, first kernel: as sdattn_qk_stats, but A is rounded to fp16
 * (nearest even) when stored, A16 = fp16(scale * Q K^T), and L, S are the
 * statistics of the stored values (L_i = max_j A16_ij, S_i = sum_j
 * exp(A16_ij - L_i)), so that the second kernel's weights sum to S_i.
 * Q, K: inputs; A16 [B][H][N][sdattn_a16_ld(desc)] and LS: outputs; ws as
 * for sdattn_qk_stats. */
sdattn_status sdattn_qk_stats_f16a(const sdattn_desc *desc, const void *Q, const void *K, void *A16,
                                   float *LS, void *ws, size_t ws_bytes, void *stream);

/* fp16-A variant, second kernel: as sdattn_softmax_av, reading fp16 A16
 * (as written by sdattn_qk_stats_f16a).  Needs no workspace. */
sdattn_status sdattn_softmax_av_f16a(const sdattn_desc *desc, const void *A16, const float *LS,
                                     const void *V, void *O, void *stream);

/* FlashAttention form: one kernel, tiled over keys with an online softmax,
 * A never stored.  Q, K, V: inputs; O: output.  LS_or_null: if not NULL,
 * also receives (L_i, S_i) as defined above.
 * ws / ws_bytes: optional workspace (may be NULL / 0).  When given it must
 * be zero-filled before first use and hold at least sdattn_workspace_bytes
 * (desc) bytes; a short one returns SDATTN_ERR_WORKSPACE.  The flash part of
 * that need grows with the SM count and d, not with B, H, N or M.  With a
 * workspace the kernel may cut the key range of a block of query rows
 * between two CTAs and merge the two halves' partial results (an
 * online-softmax merge, in a fixed order, so repeated calls give identical
 * results); this evens out the last wave of work when the row blocks do not
 * divide evenly among the SMs.  Without it every block of rows runs whole in
 * one CTA.  The two schedules agree within rounding.  Independently of the
 * workspace, when the blocks of query rows fill under half the SMs (small
 * latents, d = 80 and 160), a thread-block cluster of up to 8 CTAs shares
 * each block's key range and merges the pieces through distributed shared
 * memory in a fixed order (deterministic results). */
sdattn_status sdattn_flash(const sdattn_desc *desc, const void *Q, const void *K,
                           const void *V, void *O, float *LS_or_null, void *ws,
                           size_t ws_bytes, void *stream);

/* FlashAttention form with fp32 output and 16 more bits of P: the same
 * kernel with one query tile per CTA, where each weight p is carried as its
 * 16-bit rounding plus the 16-bit rounding of the residual, P V is the sum of
 * two tensor-core products, and O [B][H][N][d] is written in float32.  This
 * is the form that holds bf16 inputs to the accuracy bar of fp16 ones (with
 * 8-bit mantissas, a 16-bit P and a bf16 O would each cost about 1e-3 of
 * relative error).  Q, K, V: inputs (desc->dtype); O: float32 output;
 * LS_or_null as for sdattn_flash.  Needs no workspace (no key-range split). */
sdattn_status sdattn_flash_f32o(const sdattn_desc *desc, const void *Q, const void *K,
                                const void *V, float *O, float *LS_or_null, void *stream);

/* FlashAttention form for fp32 inputs (desc->dtype = SDATTN_F32), without
 * rounding them to 16 bits first: Q, K, V [B][H][*][d] float32 are read as
 * fp32 and multiplied on the tensor cores as tf32 (10-bit mantissas); the
 * weights P are rounded to tf32 (nearest) before P V; every sum is fp32 and
 * O [B][H][N][d] is written in float32.  LS_or_null as for sdattn_flash.
 * One 128-row query tile per CTA, no workspace; d in {40, 80, 160}; any
 * other dtype returns SDATTN_ERR_UNSUPPORTED. */
sdattn_status sdattn_flash_tf32(const sdattn_desc *desc, const void *Q, const void *K, const void *V,
                                float *O, float *LS_or_null, void *stream);

/* Allocation-free variant of sdattn_qk_stats.  It has no counterpart in the
 * paper; it exists for callers that cannot allocate device memory (for
 * instance code running under a framework that owns the allocator, or a
 * plug-in that is handed only its input and output buffers).
 * Same inputs, outputs and results as sdattn_qk_stats, but the scratch of the
 * split reduction is a 2 MiB array inside the library, present on every GPU
 * that loads it until the process exits.  The call allocates nothing and
 * calls no allocating routine.
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current); make that first call before any
 *    stream capture on the device.  After a device reset (a new primary
 *    context) the next call looks the address up again, so that first call
 *    after the reset, too, belongs before any capture.
 *  - Each call clears the part of the array that must start at zero.  All
 *    calls share the one array, which keeps the last call's contents, so calls
 *    that may overlap on the GPU (different streams, different threads) race
 *    and must not be issued; order them on one stream.
 *  - Shapes whose split scratch would exceed 2 MiB return
 *    SDATTN_ERR_WORKSPACE (use sdattn_qk_stats with a caller workspace). */
sdattn_status sdattn_qk_stats_noalloc(const sdattn_desc *desc, const void *Q, const void *K,
                                      float *A, float *LS, void *stream);

/* Shape of one group normalisation: X and Y are [B][C][H][W] (NCHW,
 * contiguous), element type dtype; the C channels form G groups of C/G
 * consecutive channels. */
typedef struct {
    int32_t B, C, H, W;   /* batch, channels, height, width */
    int32_t G;            /* groups; C must be a multiple of G */
    int32_t dtype;        /* sdattn_dtype of X and Y */
    float eps;            /* finite, >= 0; added to the variance (1e-6 in SD's UNet) */
} sdattn_gn_desc;

/* Group normalisation in one launch (summary of the paper, specialised-
 * kernels paragraphs: channels split into groups, each group normalised on
 * its own, one GPU command without intermediate tensors).  Each group is
 * held in registers by a thread-block cluster that combines its partial sums
 * through distributed shared memory, so x is read once and y written once.  For each batch b
 * and group g, over the group's (C/G) H W values:
 *   mean = sum x / n,  var = sum (x - mean)^2 / n   (biased, fp32),
 *   Y[b][c][h][w] = (X[b][c][h][w] - mean) / sqrt(var + eps) * gamma[c] + beta[c].
 * X: input; gamma, beta: float32 [C] (4-byte aligned); Y: output (may not
 * overlap X).  H*W must be a multiple of 8 and a group at most 262144 values;
 * other shapes return SDATTN_ERR_UNSUPPORTED.  Needs no workspace. */
sdattn_status sdattn_group_norm(const sdattn_gn_desc *desc, const void *X, const float *gamma,
                                const float *beta, void *Y, void *stream);

/* The gated GELU of the UNet's feed-forward layers in one launch (summary of
 * the paper, specialised-kernels paragraphs: GELU's Gaussian error function
 * fused with the split and multiplication around it).  X [T][2F] is the
 * projection's output; its first F columns are h, the last F the gate g:
 *   Y[t][f] = h[t][f] * g/2 * (1 + erf(g / sqrt(2))),   g = X[t][F + f]
 * (fp32 arithmetic, Y rounded to dtype).  X: input; Y [T][F]: output.
 * F must be a multiple of 8 (SDATTN_ERR_UNSUPPORTED otherwise), T >= 1. */
sdattn_status sdattn_geglu(int64_t T, int32_t F, int32_t dtype, const void *X, void *Y, void *stream);

/* The UNet's 3x3 convolution by Winograd's minimal filtering (summary of the
 * paper, Winograd paragraphs: 3x3 convolutions as Winograd convolutions, a
 * 4x4 tile as the best balance of compute and memory), read as F(4x4, 3x3):
 * 4x4 output tiles from 6x6 input tiles.  Stride 1, zero padding 1 (Y has
 * X's H x W), cross-correlation as in the UNet, optional bias:
 *   Y[n][k][h][w] = bias[k] + sum_{c,r,s} Wt[k][c][r][s] X[n][c][h+r-1][w+s-1]
 * X [N][C][H][W], Wt [K][C][3][3] and Y [N][K][H][W] of element type dtype;
 * bias float32 [K] or NULL.  C must be a multiple of 8 and W at most 4096
 * (SDATTN_ERR_UNSUPPORTED otherwise). */
typedef struct {
    int32_t N, C, K, H, W;   /* batch, input channels, output channels, height, width; all >= 1 */
    int32_t dtype;           /* sdattn_dtype of X, Wt, U and Y */
} sdattn_conv_desc;

/* Bytes of the transformed filter U [36][K][C] (dtype); 0 for an invalid desc. */
size_t sdattn_wino_filter_bytes(const sdattn_conv_desc *desc);

/* Bytes of the workspace a convolution needs: the transformed input
 * [36][T][C] (dtype) and the 36 products [36][K][ldm] (float32), T = N
 * ceil(H/4) ceil(W/4) tiles, ldm = T rounded up to 4.  0 for an invalid desc. */
size_t sdattn_wino_workspace_bytes(const sdattn_conv_desc *desc);

/* Filter transform, once per filter: U[xi][k][c] = (G Wt[k][c] G^T)[xi] in
 * fp32, rounded to dtype (G the 6x3 transform of F(4, 3)).  Wt needs 2-byte,
 * U 16-byte alignment; U holds sdattn_wino_filter_bytes(desc) bytes. */
sdattn_status sdattn_wino_filter(const sdattn_conv_desc *desc, const void *Wt, void *U, void *stream);

/* The convolution from a transformed filter U: input transform (B^T d B per
 * tile, fp32, rounded to dtype), a batched tensor-core product over the 36
 * transformed positions (fp32 accumulation), output transform (A^T m A, fp32)
 * plus bias, rounded to dtype: three launches on `stream`.  ws: at least
 * sdattn_wino_workspace_bytes(desc) bytes, 16-byte aligned, caller-owned,
 * fully overwritten (no state between calls).  X, U, Y 16-byte aligned; bias
 * 4-byte aligned.  Y may not overlap X, U or ws. */
sdattn_status sdattn_wino_conv3x3(const sdattn_conv_desc *desc, const void *X, const void *U, const float *bias,
                                  void *Y, void *ws, size_t ws_bytes, void *stream);

/* Reads and clears this device's error word (synchronises the device).
 * Returns SDATTN_OK, SDATTN_ERR_TIMEOUT, or SDATTN_ERR_CUDA if it cannot be
 * read.  If detail is not NULL it receives a code naming the wait that ran
 * out (0 when none). */
sdattn_status sdattn_device_error(uint32_t *detail);

/* Static, human-readable name of a status. */
const char *sdattn_status_string(sdattn_status status);

/* Library version, e.g. 100 for 0.1.0. */
int32_t sdattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SDATTN_H */
