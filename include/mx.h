/*
 * mx.h -- C ABI of the B200 (sm_100a) MXFP8 GEMM library.
 *
 * What the library computes
 * -------------------------
 * MXFP8 ("PyTorch and Nebius optimise DeepSeek-V3 MoE training on B200
 * clusters", glossary entry on microscaling FP8, and the OCP Microscaling
 * specification it cites): 8-bit E4M3 elements that share one UE8M0
 * power-of-two scale per block of 32 consecutive elements along K.  The
 * pipeline is BF16 -> MXFP8 -> (grouped) GEMM with FP32 accumulation -> BF16
 * (same page, diagram of the MXFP8 flow from router input to the all-to-all
 * combine).  The GEMM family -- one dense GEMM and MoE grouped GEMMs in a
 * contiguous and a masked layout -- is the one the DeepGEMM pages describe
 * ("DeepGEMM" summary page, introduction and the MoE grouped GEMM note;
 * DeepGEMM release page, section 4 "MoE optimisation").
 *
 * Conventions for every call
 * --------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The
 *    library allocates no memory per call and keeps no reference to any
 *    pointer after the call returns.
 *  - Row-major layouts with K contiguous.  A is [M, K], B is [N, K] (one
 *    expert) or [E, N, K]; the product is D = A * B^T, [M, N] BF16.
 *  - Quantised elements: one byte per element (E4M3), same shape as the
 *    BF16 source.
 *  - Scales: UE8M0 bytes (value 2^(c-127), 0xFF = NaN) in the tiled layout
 *    the tensor cores consume.  For a matrix of R rows and Kb = K/32 blocks,
 *    rows are padded to a multiple of 128 and Kb to a multiple of 4; the
 *    scale of row r, block c sits at byte
 *        ((r/128)*(Kb_pad/4) + c/4) * 512 + (r%32)*16 + ((r%128)/32)*4 + c%4.
 *    Padding bytes are written as 0x00 by the quantiser.  For 3-D operands
 *    each group has its own such region of mx_scale_bytes(rows, K) bytes,
 *    placed back to back.
 *  - Every call is asynchronous on `stream` (NULL = legacy default stream).
 *    Argument errors are reported synchronously through the return value
 *    and nothing is launched.  Data-dependent errors found on the device
 *    (bad group offsets, masked_m out of range, an internal wait that timed
 *    out) are OR-ed into *dev_status as MX_DEV_* bits when dev_status is
 *    not NULL, otherwise into a library-internal word readable with
 *    mx_read_internal_status().  Kernels never trap.
 *  - No exceptions cross this boundary.
 */
#ifndef MX_H
#define MX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *mx_stream_t;

typedef enum mx_status {
    MX_OK = 0,
    MX_ERR_INVALID_ARGUMENT = 1, /* NULL pointer, negative size, bad count */
    MX_ERR_UNSUPPORTED_SHAPE = 2, /* K not a multiple of 32 (quantiser) / 128 (GEMM), N % 16 != 0 */
    MX_ERR_MISALIGNED = 3,       /* a pointer not 16-byte aligned */
    MX_ERR_CUDA = 4              /* a CUDA runtime / driver call failed */
} mx_status;

/* Device-side status bits (OR-ed into *dev_status). */
#define MX_DEV_BAD_OFFSETS 0x1 /* group_offsets not monotone, not multiples of 128, or > m_total */
#define MX_DEV_BAD_MASK 0x2    /* masked_m[e] outside [0, max_m] (clamped) */
#define MX_DEV_TIMEOUT 0x4     /* an internal pipeline wait exceeded its limit; output invalid */
#define MX_DEV_BAD_INDEX 0x8   /* a row index read from device memory was out of range (access skipped) */

/* Human-readable name of a status code; never NULL. */
const char *mx_status_string(int status);

/* Bytes of the tiled scale region for a [rows, k] operand:
 * ceil(rows/128)*128 * ceil(k/32/4)*4.  Returns 0 for rows <= 0 or k <= 0. */
size_t mx_scale_bytes(int64_t rows, int64_t k);

/*
 * BF16 -> MXFP8 quantisation along K.
 *   x_bf16   [rows, k] BF16, row-major, 16-byte aligned.
 *   q_e4m3   [rows, k] bytes out, 16-byte aligned.
 *   sf_ue8m0 mx_scale_bytes(rows, k) bytes out (tiled layout above).
 * Per 32-element block: amax over |x|; X = floor(log2 amax) - 8 clamped to
 * [-127, 127] (amax = 0 gives X = -127); scale byte X+127; each element
 * x*2^-X rounded to nearest-even and saturated to +-448.  A block holding a
 * NaN or +-Inf gets scale 0xFF and elements 0x7F.  Requires k % 32 == 0.
 * rows == 0 is a no-op.
 */
mx_status mx_quantize_bf16_to_e4m3(const void *x_bf16, int64_t rows, int64_t k, void *q_e4m3,
                                   void *sf_ue8m0, mx_stream_t stream);

/*
 * Same as mx_quantize_bf16_to_e4m3 for a 3-D [groups, rows, k] tensor whose
 * scales are stored per group: group g's scales start at
 * g * mx_scale_bytes(rows, k).  (When rows % 128 == 0 this equals the 2-D
 * call on groups*rows rows.)
 */
mx_status mx_quantize_bf16_to_e4m3_grouped(const void *x_bf16, int64_t groups, int64_t rows,
                                           int64_t k, void *q_e4m3, void *sf_ue8m0,
                                           mx_stream_t stream);

/*
 * Several quantisations in one kernel launch (for the operands of one step:
 * fewer launches, one launch latency).  Each job is exactly the
 * mx_quantize_bf16_to_e4m3_grouped call with the same fields (groups == 1
 * for a 2-D tensor); jobs with a zero extent are skipped.  Every job is
 * validated before anything is launched; up to 8 jobs share a launch.  The
 * jobs must not overlap in memory.
 */
typedef struct mx_quant_job {
    const void *x_bf16; /* [groups, rows, k] BF16 */
    int64_t groups;
    int64_t rows;
    int64_t k;
    void *q_e4m3;       /* [groups, rows, k] bytes out */
    void *sf_ue8m0;     /* groups * mx_scale_bytes(rows, k) bytes out */
} mx_quant_job;

mx_status mx_quantize_bf16_to_e4m3_multi(const mx_quant_job *jobs, int32_t count, mx_stream_t stream);

/*
 * The same jobs, the same bytes out and the same argument checks as
 * mx_quantize_bf16_to_e4m3_multi, from a form of the kernel that uses no
 * shared memory and one CTA per SM.  It is meant to run concurrently with a
 * GEMM launched on another stream: the GEMM's CTAs hold nearly all of each
 * SM's shared memory, so the normal form cannot share an SM with them, and
 * the quantisation (HBM-bound) then proceeds underneath the GEMM
 * (tensor-bound) instead of before or after it.  Alone it is slower than the
 * normal form.
 */
mx_status mx_quantize_bf16_to_e4m3_multi_lean(const mx_quant_job *jobs, int32_t count, mx_stream_t stream);

/*
 * Dense MXFP8 GEMM, D = A * B^T ("DeepGEMM" summary page: the plain FP8
 * GEMM; the dense shapes of its CUTLASS comparison table).
 *   qa [m, k], sfa = scales of A (mx_scale_bytes(m, k));
 *   qb [n, k], sfb = scales of B (mx_scale_bytes(n, k));
 *   d_bf16 [m, n] BF16 out.  FP32 accumulation, BF16 round-to-nearest-even.
 * Requires k % 128 == 0, k > 0, n % 16 == 0, 16-byte aligned pointers.
 * m == 0 or n == 0 is a no-op.
 */
mx_status mx_gemm(const void *qa, const void *sfa, const void *qb, const void *sfb, void *d_bf16,
                  int64_t m, int64_t n, int64_t k, int32_t *dev_status, mx_stream_t stream);

/*
 * Several independent dense MXFP8 GEMMs in ONE launch: D_i = A_i * B_i^T for
 * i < count ("DeepGEMM" summary page, CUTLASS comparison table: the dense
 * shapes it lists are separate small-M problems of one model, e.g.
 * 64x2112x7168, 64x24576x1536 and 128x7168x2048).  Each problem follows
 * mx_gemm's contract (layouts, alignment, k % 128 == 0, n % 16 == 0, the
 * same result up to FP32 summation order); problems with m == 0 or n == 0
 * are no-ops.  The GPU is shared among the problems so that all of them
 * stream their operands at once instead of one launch after another: each
 * gets a share of the SMs sized to its bytes, with K split across a cluster
 * where that shortens it.  Meant for problems too small to fill the GPU
 * alone; every problem uses one-CTA tiles of 128 rows (128 or 256 columns,
 * one width for the whole batch).
 *   problems  host array of `count` descriptors, read during the call;
 *   1 <= count <= MX_GEMM_BATCH_MAX (else MX_ERR_INVALID_ARGUMENT).
 * One status word for all problems (dev_status, nullable).
 */
#define MX_GEMM_BATCH_MAX 4
typedef struct {
    const void *qa;   /* [m, k] E4M3 */
    const void *sfa;  /* mx_scale_bytes(m, k) tiled scales of A */
    const void *qb;   /* [n, k] E4M3 */
    const void *sfb;  /* mx_scale_bytes(n, k) tiled scales of B */
    void *d_bf16;     /* [m, n] BF16 out */
    int64_t m, n, k;
} mx_gemm_problem;

mx_status mx_gemm_batch(const mx_gemm_problem *problems, int32_t count, int32_t *dev_status, mx_stream_t stream);

/*
 * Contiguous-layout MoE grouped GEMM ("DeepGEMM" release page, section 4:
 * token sequences of all experts grouped into one M dimension).
 *   qa [m_total, k] holds the groups back to back; group e owns rows
 *   [group_offsets[e], group_offsets[e+1]).  Every offset must be a multiple
 *   of 128 (pad each group with rows; padded rows are multiplied like any
 *   other row).  sfa = scales of the whole [m_total, k] operand.
 *   qb [groups, n, k], sfb = groups back-to-back regions of
 *   mx_scale_bytes(n, k) bytes.
 *   group_offsets: DEVICE int32[groups + 1], read by the kernel (no host
 *   synchronisation).
 *   d_bf16 [m_total, n]: rows inside a group are written; rows at or beyond
 *   group_offsets[groups] are left untouched.
 */
mx_status mx_grouped_gemm_contiguous(const void *qa, const void *sfa, const void *qb,
                                     const void *sfb, const int32_t *group_offsets,
                                     int32_t groups, int64_t m_total, int64_t n, int64_t k,
                                     void *d_bf16, int32_t *dev_status, mx_stream_t stream);

/*
 * Masked-layout MoE grouped GEMM ("DeepGEMM" release page, section 4:
 * efficient when expert activation is sparse).
 *   qa [groups, max_m, k], sfa = groups back-to-back regions of
 *   mx_scale_bytes(max_m, k) bytes; qb [groups, n, k], sfb likewise with
 *   mx_scale_bytes(n, k).  masked_m: DEVICE int32[groups], valid rows of
 *   each group.  d_bf16 [groups, max_m, n]: for group e only rows
 *   r < masked_m[e] are written; all other rows are left untouched (their
 *   A rows may hold anything, NaN included).
 */
mx_status mx_grouped_gemm_masked(const void *qa, const void *sfa, const void *qb,
                                 const void *sfb, const int32_t *masked_m, int32_t groups,
                                 int64_t max_m, int64_t n, int64_t k, void *d_bf16,
                                 int32_t *dev_status, mx_stream_t stream);

/*
 * Quantisation along the ROW dimension, written transposed: for x
 * [groups, rows, cols] BF16 (row-major) the output is q [groups, cols, rows]
 * E4M3, each 32 consecutive rows of a column sharing one UE8M0 scale, with
 * per-group tiled scales of the [cols, rows] operand
 * (groups * mx_scale_bytes(cols, rows) bytes; rows play the role of K).
 * Same scale and rounding rule as mx_quantize_bf16_to_e4m3.  Used for the
 * training-side MoE GEMMs (the B200 MoE-training page applies MXFP8 to
 * DeepSeek-V3 training): the weight gradient reduces over tokens, so the
 * output gradient and the layer input [tokens, features] are quantised along
 * tokens; the input gradient reduces over the layer's output features, so the
 * expert weights [E, N, K] are quantised along N into [E, K, N].
 * Requires rows % 32 == 0, cols % 8 == 0, 16-byte aligned pointers.  Scale
 * padding bytes are written as 0x00.
 */
mx_status mx_quantize_bf16_to_e4m3_transposed(const void *x_bf16, int64_t groups, int64_t rows, int64_t cols,
                                              void *q_e4m3, void *sf_ue8m0, mx_stream_t stream);

/*
 * K-grouped MoE GEMM: the weight gradient of an expert layer, where the
 * reduction runs over tokens and each expert owns a contiguous range of them
 * (the contiguous layout of mx_grouped_gemm_contiguous, seen from the
 * backward pass).  For expert e and k in [group_offsets[e], group_offsets[e+1]):
 *   D[e, i, j] = sum_k deq(A[i, k]) * deq(B[j, k])   (FP32 accumulation, BF16 out)
 *   qa [m, k_total] E4M3 (e.g. the output gradient transposed, m = N of the
 *   layer), sfa = mx_scale_bytes(m, k_total) tiled scales (blocks of 32
 *   tokens); qb [n, k_total] (e.g. the layer input transposed), sfb
 *   likewise; both from mx_quantize_bf16_to_e4m3_transposed.
 *   group_offsets: DEVICE int32[groups + 1], multiples of 128, non-decreasing,
 *   at most k_total (else MX_DEV_BAD_OFFSETS and nothing is written).
 *   d_bf16 [groups, m, n]: every expert's block is written; an expert with
 *   no tokens gets zeros.
 * Requires k_total > 0, k_total % 128 == 0, n % 16 == 0, 16-byte aligned
 * pointers.
 */
mx_status mx_grouped_gemm_kgrouped(const void *qa, const void *sfa, const void *qb, const void *sfb,
                                   const int32_t *group_offsets, int32_t groups, int64_t m, int64_t n,
                                   int64_t k_total, void *d_bf16, int32_t *dev_status, mx_stream_t stream);

/*
 * Fused first half of an MoE expert MLP: the gate/up GEMM, SwiGLU, and MXFP8
 * requantisation of the result in one kernel, so the activation never goes
 * to memory in BF16 (the B200 MoE-training page describes MXFP8 expert
 * layers between a BF16 -> MXFP8 quantise and the BF16 restore; the
 * activation between the two expert GEMMs is DeepSeek-V3's SwiGLU).
 *
 *   G = A * gate^T, U = A * up^T (FP32 accumulation, as in mx_gemm);
 *   H = silu(G) * U with silu(x) = x / (1 + e^-x), in FP32;
 *   H is quantised along its columns in 32-element blocks by the rule of
 *   mx_quantize_bf16_to_e4m3 applied to the FP32 values.
 *
 * qb holds, per expert, the 2*i_dim rows of the gate/up projection stacked as
 * [gate (i_dim rows); up (i_dim rows)], row-major [groups, 2*i_dim, k]; sfb
 * its scales (groups regions of mx_scale_bytes(2*i_dim, k) bytes).  qa/sfa
 * as in the matching plain call.  Outputs: qh E4M3 [rows, i_dim] (row
 * layout of the matching plain call's D) and sfh its tiled scales
 * (mx_scale_bytes(rows, i_dim) bytes; per expert for the masked form).
 * (qh, sfh) is directly the A operand of the down GEMM (K = i_dim).
 *
 * Requires k % 128 == 0, i_dim % 128 == 0, 16-byte aligned pointers.  Rows
 * the plain call leaves untouched (contiguous: at or beyond
 * group_offsets[groups]; masked: at or beyond masked_m[e]) are left
 * untouched in qh and sfh too; the dense form writes 0x00 into the scale
 * padding rows of its last 128-row block.  Errors as for the plain calls.
 */
mx_status mx_gemm_swiglu_quant(const void *qa, const void *sfa, const void *qb, const void *sfb, void *qh,
                               void *sfh, int64_t m, int64_t i_dim, int64_t k, int32_t *dev_status,
                               mx_stream_t stream);

mx_status mx_grouped_gemm_contiguous_swiglu_quant(const void *qa, const void *sfa, const void *qb,
                                                  const void *sfb, const int32_t *group_offsets,
                                                  int32_t groups, int64_t m_total, int64_t i_dim, int64_t k,
                                                  void *qh, void *sfh, int32_t *dev_status,
                                                  mx_stream_t stream);

mx_status mx_grouped_gemm_masked_swiglu_quant(const void *qa, const void *sfa, const void *qb,
                                              const void *sfb, const int32_t *masked_m, int32_t groups,
                                              int64_t max_m, int64_t i_dim, int64_t k, void *qh, void *sfh,
                                              int32_t *dev_status, mx_stream_t stream);

/*
 * Tile-wise FP32-scaled FP8: the format with fine-grained FP32 scales that
 * DeepGEMM's GEMMs take (the pages: "tile-wise" scaling in the FP8
 * mixed-precision recipe; DeepGEMM's FP32 two-level accumulation), with
 * DeepSeek-V3's tiles: 1 x 128 for activations, 128 x 128 for weights.
 * Per tile: s = amax / 448 in FP32 (IEEE division), element x / s (IEEE FP32
 * division) as E4M3 with saturating round-to-nearest-even; an all-zero tile
 * gets s = 1, a tile holding NaN or +-Inf gets s = NaN (0x7FC00000) and
 * elements 0x7F.  Scales are plain FP32 arrays:
 *   1 x 128:   scales [k/128, rows]          (K-tile major)
 *   128 x 128: scales [ceil(rows/128), k/128]
 * x [rows, k] BF16 16-byte aligned, q [rows, k], scales 4-byte aligned;
 * requires k % 128 == 0 (else MX_ERR_UNSUPPORTED_SHAPE), rows and k at most
 * 2^31 - 1 and fewer than 2^32 - 16 groups of 8 rows x 128 columns (else
 * MX_ERR_UNSUPPORTED_SHAPE).  rows == 0 is a no-op.  Null pointers give
 * MX_ERR_INVALID_ARGUMENT, misaligned ones MX_ERR_MISALIGNED.
 */
mx_status mx_quantize_bf16_to_e4m3_tile1x128(const void *x_bf16, int64_t rows, int64_t k, void *q_e4m3,
                                             float *scales, mx_stream_t stream);
mx_status mx_quantize_bf16_to_e4m3_block128x128(const void *x_bf16, int64_t rows, int64_t k, void *q_e4m3,
                                                float *scales, mx_stream_t stream);

/*
 * GEMM on tile-wise FP32-scaled FP8 operands:
 *   D[i, j] = sum_kt sa[kt, i] * sb[j/128, kt] * sum_{k in K tile kt} e4m3(a[i,k]) * e4m3(b[j,k])
 * qa [m, k] with sa [k/128, m] (1 x 128 tiles); qb [n, k] with sb
 * [ceil(n/128), k/128] (128 x 128 blocks); d_bf16 [m, n].  Each K tile's
 * products are summed by the tensor core into a TMEM accumulator and
 * promoted into FP32 with its two scales (DeepGEMM's two-level accumulation,
 * "DeepSeek drops DeepGEMM" page, section 1).  Requires k % 128 == 0,
 * n % 16 == 0, 16-byte aligned qa/qb/d, 4-byte aligned scales.
 * The contiguous grouped form follows mx_grouped_gemm_contiguous: qb
 * [groups, n, k], sb [groups, ceil(n/128), k/128], device group_offsets
 * (multiples of 128), sa [k/128, m_total].
 */
mx_status mx_gemm_tilewise(const void *qa, const float *sa, const void *qb, const float *sb, void *d_bf16,
                           int64_t m, int64_t n, int64_t k, int32_t *dev_status, mx_stream_t stream);
mx_status mx_grouped_gemm_contiguous_tilewise(const void *qa, const float *sa, const void *qb, const float *sb,
                                              const int32_t *group_offsets, int32_t groups, int64_t m_total,
                                              int64_t n, int64_t k, void *d_bf16, int32_t *dev_status,
                                              mx_stream_t stream);

/* ------------------------------------------------------------------ MoE expert layer
 *
 * The data movement around the grouped GEMM in a mixture-of-experts layer:
 * the B200 MoE-training page's MXFP8 expert layer (router output -> BF16 ->
 * MXFP8 -> grouped GEMM -> BF16 -> all-to-all combine; glossary entry on
 * all-to-all: tokens are sent to their experts and the results gathered
 * back) and DeepGEMM's contiguous layout (release page, section 4).  The
 * router is not part of the path: expert ids and gate weights are inputs.
 * For expert parallelism the same calls build and unpack the all-to-all
 * buffers (route with pad = 1 orders entries by expert, i.e. by the rank that
 * owns the expert).
 */

/* Upper bound of the rows a routing plan of n entries over `experts` groups
 * padded to `pad` occupies, rounded up to a multiple of 128 (the scale-tile
 * height): allocate the grouped operand with this many rows. */
int64_t mx_moe_max_rows(int64_t n, int32_t experts, int32_t pad);

/* Routing plan of a [tokens, topk] expert-id table (n = tokens*topk int32
 * entries, token-major, device).  Expert e's rows are its entries in entry
 * order starting at offsets[e]; every group is padded to a multiple of `pad`
 * rows: offsets[e+1] = offsets[e] + ceil(counts[e]/pad)*pad.  Outputs
 * (device, caller-owned): counts int32 [experts], offsets int32 [experts+1],
 * row int32 [n] (the entry's row; -1 for an id outside [0, experts), which is
 * dropped), dropped int32 [1] (nullable: the number of dropped entries).
 * One CTA; 1 <= experts <= 1024, 1 <= pad <= 128, n < 2^31 - 1024. */
mx_status mx_moe_route(const int32_t *ids, int64_t n, int32_t experts, int32_t pad, int32_t *counts,
                       int32_t *offsets, int32_t *row, int32_t *dropped, mx_stream_t stream);

/* Dispatch: each token row of x_bf16 [tokens, k] is quantised to MXFP8 once
 * (the rule of mx_quantize_bf16_to_e4m3, bit for bit) and written to row
 * row[t*topk + j] of q_e4m3 [m_rows, k] for every j with row >= 0; its k/32
 * scale bytes go to the same row of sf: the tiled layout over m_rows rows
 * (mx_scale_bytes(m_rows, k) bytes; the GEMM operand) when sf_row_major == 0,
 * else row-major [m_rows, k/32] (an all-to-all send buffer).  When pad > 1 the
 * padding rows of every group ([offsets[e] + counts[e], offsets[e+1]), from
 * mx_moe_route with the same pad) are set to the quantisation of a zero row
 * (E4M3 0x00, scale 0x00).  k % 128 == 0; m_rows % 128 == 0 for the tiled
 * layout; 16-byte aligned x, q and sf.  A row >= m_rows is skipped and sets
 * MX_DEV_BAD_INDEX.  The rows of different entries must be distinct (as
 * mx_moe_route makes them); two entries sharing a row leave either one's data. */
mx_status mx_moe_dispatch_quant(const void *x_bf16, int64_t tokens, int64_t k, const int32_t *row, int32_t topk,
                                const int32_t *counts, const int32_t *offsets, int32_t experts, int32_t pad,
                                int64_t m_rows, void *q_e4m3, void *sf, int32_t sf_row_major,
                                int32_t *dev_status, mx_stream_t stream);

/* Scatter of already quantised rows (an all-to-all receive buffer): row i of
 * q_src [n_src, k] with its row-major scales sf_src [n_src, k/32] goes to row
 * dst_row[i] of q_dst [m_rows, k] / the tiled scales sf_dst (mx_scale_bytes(
 * m_rows, k) bytes); padding rows of the plan (counts, offsets, pad) are
 * cleared as in mx_moe_dispatch_quant.  Same shape, alignment and index rules. */
mx_status mx_moe_scatter_rows(const void *q_src, const void *sf_src, int64_t n_src, int64_t k,
                              const int32_t *dst_row, const int32_t *counts, const int32_t *offsets,
                              int32_t experts, int32_t pad, int64_t m_rows, void *q_dst, void *sf_dst,
                              int32_t *dev_status, mx_stream_t stream);

/* Row gather: dst[i] = src[idx[i]] for i < n, rows of row_bytes bytes
 * (row_bytes % 16 == 0, 16-byte aligned src and dst); an index outside
 * [0, src_rows) gives a zero row and sets MX_DEV_BAD_INDEX. */
mx_status mx_gather_rows(const void *src, int64_t src_rows, int64_t row_bytes, const int32_t *idx, int64_t n,
                         void *dst, int32_t *dev_status, mx_stream_t stream);

/* Combine: out[t, :] = sum_j w[t, j] * y[row[t*topk + j], :] for t < tokens,
 * over the entries with row >= 0, FP32 fused multiply-adds in j order and one
 * rounding to BF16 (RNE).  y_bf16 [y_rows, n_cols], w float32 [tokens, topk],
 * row int32 [tokens*topk], out_bf16 [tokens, n_cols]; n_cols % 8 == 0,
 * 16-byte aligned y and out, 1 <= topk <= 64.  A row >= y_rows is skipped and
 * sets MX_DEV_BAD_INDEX. */
mx_status mx_moe_combine(const void *y_bf16, int64_t y_rows, int64_t n_cols, const int32_t *row, const float *w,
                         int64_t tokens, int32_t topk, void *out_bf16, int32_t *dev_status, mx_stream_t stream);

/*
 * Expert parallelism over peer memory (the DeepEP role on the B200
 * MoE-training page: tokens are sent to the ranks that hold their experts and
 * the results gathered back), with the exchange fused into the dispatch and
 * the combine: the dispatch quantises each token once and stores its MXFP8
 * row straight into the receive buffer of the rank that owns the expert, and
 * the combine loads the expert outputs straight from their owners' buffers.
 * "Rank r's buffer" is any device pointer this process can dereference:
 * another GPU's memory mapped for peer access (NVLink), or, to emulate several
 * ranks on one GPU, a local buffer.  Pointer tables (q_peers, sf_peers,
 * y_peers) are DEVICE arrays of `ranks` pointers, every buffer 16-byte aligned
 * and of the same shape on every rank.  The calls only load and store: the
 * caller orders the phases across ranks (every rank's dispatch complete
 * before any owner's GEMM reads its receive buffer; every owner's GEMM
 * complete before any combine reads its output; every combine complete before
 * the buffers are written again), e.g. with a collective barrier on the stream.
 * Rank r of R owns the experts [r*E/R, (r+1)*E/R).
 */

/* Placement plan of this rank's entries (n = tokens*topk, device).  ids are
 * global expert ids; row_send is mx_moe_route(ids, experts, pad = 1)'s row
 * output; count_table int32 [ranks, experts] holds every rank's counts from
 * that route (e.g. all-gathered).  On the owner of expert e, e's rows come
 * source rank by source rank, each source's rows in its entry order, and each
 * local expert's group is padded to `pad` rows.  Outputs (device):
 * dst_rank/dst_row int32 [n] (the owner and the row in its receive buffer;
 * -1/-1 for an id outside [0, experts)), and this rank's own receive plan:
 * counts_local int32 [experts/ranks] (rows from all sources) and
 * offsets_local int32 [experts/ranks + 1] (padded group starts, the
 * group_offsets of the grouped GEMMs; offsets_local[E/R] = rows in use).
 * experts % ranks == 0; 1 <= experts, ranks <= 1024; 1 <= pad <= 128;
 * n * ranks + experts * (pad - 1) < 2^31 (the largest padded offset the plan
 * can produce), else MX_ERR_UNSUPPORTED_SHAPE.  A row_send inconsistent with count_table sets
 * MX_DEV_BAD_INDEX and gives -1/-1. */
mx_status mx_moe_peer_plan(const int32_t *ids, const int32_t *row_send, int64_t n, const int32_t *count_table,
                           int32_t ranks, int32_t rank, int32_t experts, int32_t pad, int32_t *dst_rank,
                           int32_t *dst_row, int32_t *counts_local, int32_t *offsets_local, int32_t *dev_status,
                           mx_stream_t stream);

/* Dispatch over peer memory: each token row of x_bf16 [tokens, k] is
 * quantised to MXFP8 once (mx_quantize_bf16_to_e4m3's rule, bit for bit) and,
 * for every j with dst_row[t*topk + j] >= 0, written to row dst_row of
 * q_peers[dst_rank] [m_rows, k] with its scale bytes in the tiled layout of
 * sf_peers[dst_rank] (mx_scale_bytes(m_rows, k) bytes).  This rank's own
 * receive buffer q_local / sf_local (the entries of the tables for this rank)
 * gets the padding rows of its plan (counts_local, offsets_local,
 * experts_local, pad from mx_moe_peer_plan) set to the quantisation of a zero
 * row.  k % 128 == 0, m_rows % 128 == 0, 16-byte aligned buffers.  A
 * dst_rank outside [0, ranks) or a dst_row >= m_rows is skipped and sets
 * MX_DEV_BAD_INDEX. */
mx_status mx_moe_dispatch_quant_peer(const void *x_bf16, int64_t tokens, int64_t k, const int32_t *dst_rank,
                                     const int32_t *dst_row, int32_t topk, void *const *q_peers,
                                     void *const *sf_peers, int32_t ranks, int64_t m_rows, void *q_local,
                                     void *sf_local, const int32_t *counts_local, const int32_t *offsets_local,
                                     int32_t experts_local, int32_t pad, int32_t *dev_status, mx_stream_t stream);

/* Combine over peer memory: out[t, :] = sum_j w[t, j] * y_peers[src_rank[t*topk+j]][src_row[t*topk+j], :]
 * over the entries with src_row >= 0, with mx_moe_combine's arithmetic (FP32
 * fused multiply-adds in j order, one rounding to BF16).  Every rank's output
 * buffer is BF16 [y_rows, n_cols]; src_rank/src_row are the dispatch's
 * dst_rank/dst_row.  A rank outside [0, ranks) or a row >= y_rows is skipped
 * and sets MX_DEV_BAD_INDEX. */
mx_status mx_moe_combine_peer(const void *const *y_peers, int32_t ranks, int64_t y_rows, int64_t n_cols,
                              const int32_t *src_rank, const int32_t *src_row, const float *w, int64_t tokens,
                              int32_t topk, void *out_bf16, int32_t *dev_status, mx_stream_t stream);

/* Failure detection (no counterpart on the pages; a property of this
 * implementation).  Every wait inside the GEMM kernels (a pipeline stage
 * landing, an accumulator being drained, ...) is bounded: a wait that runs
 * longer than the limit gives up, the kernel sets MX_DEV_TIMEOUT in the
 * status word, stops issuing work, waits for the tensor-core work and copies
 * it already issued, frees its tensor memory and returns -- it never traps or
 * hangs, and the context stays usable; the output of that call is invalid.
 * The limit defaults to 2 s (far above any legitimate wait).  This sets it,
 * in nanoseconds, for the GEMM launches that follow, from any thread
 * (ns == 0 restores the default); a limit below a kernel's legitimate waits
 * makes its calls fail with MX_DEV_TIMEOUT, which is how the failure path is
 * tested.  Never fails. */
mx_status mx_set_wait_limit_ns(uint64_t ns);
/* The current limit in nanoseconds. */
uint64_t mx_wait_limit_ns(void);

/* Copies the library-internal device status word (used when a call got
 * dev_status == NULL) to *host_out and, if clear != 0, resets it.
 * Synchronises the device. */
mx_status mx_read_internal_status(int32_t *host_out, int clear);

#ifdef __cplusplus
}
#endif
#endif /* MX_H */
