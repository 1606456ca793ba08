/*
 * svq.h -- C ABI of libsvq, the B200 (sm_100a) library for SAGE's 2-bit
 * spherical vector quantization (SVQ) linear layer, y = W x.
 *
 * The method ("SAGE: Pushing 2-Bit Vector-Quantized LLMs toward Real-World
 * Usability", arXiv 2610.14745):
 *   - Figure 2 caption: each subvector of eight weights is stored as eight
 *     signs, a direction index into a per-matrix codebook and a quantized
 *     radius, 18 bits per eight weights; the 10 non-sign bits are split
 *     between direction (b_d) and radius (b_r = 10 - b_d) per matrix (ABS).
 *   - Figure 6 caption: the kernel multiplies each decoded subvector by eight
 *     reordered activations (the ESG input-channel permutation).
 *   - Figures 1 and 5 captions: weights are reconstructed on demand; no dense
 *     copy of W is kept (svq_linear_gemm from 4 tiles of 256 tokens on decodes
 *     the matrix into its caller-owned workspace for the duration of the call).
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller, except where
 *     a parameter says "host".  The library never allocates or frees memory
 *     and never synchronises the device (svq_get_device_status excepted).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy stream) and
 *     runs asynchronously; the return value reports argument validation and
 *     launch errors only.
 *   - fp16 / bf16 values are passed as 16-bit bit patterns (uint16_t).
 *   - Shapes: K % 8 == 0 (the format's own rule), N >= 1, 1 <= b_d <= 10.
 *     Shapes with N % 4 != 0 or K % 128 != 0 are stored padded to the next
 *     multiple of 4 rows and 128 columns (zero codes, svq_packed_bytes counts
 *     them); the padding never contributes to an output.  svq_moe_grouped_gemv
 *     takes only K % 128 == 0 and N % 4 == 0.
 *   - Return codes: SVQ_OK or one of the SVQ_ERR_* values below; nothing is
 *     enqueued when an error is returned.
 */
#ifndef SVQ_H_
#define SVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SVQ_API __attribute__((visibility("default")))
#else
#define SVQ_API
#endif

typedef struct CUstream_st* svq_stream_t; /* same type as cudaStream_t */

enum svq_status {
  SVQ_OK = 0,
  SVQ_ERR_INVALID_ARG = 1,       /* NULL or misaligned pointer, bad enum, M out of range */
  SVQ_ERR_UNSUPPORTED_SHAPE = 2, /* N, K or b_d outside what the kernels handle */
  SVQ_ERR_WORKSPACE = 3,         /* workspace NULL or smaller than the *_workspace_size query */
  SVQ_ERR_CUDA = 4,              /* a CUDA runtime call failed (launch, attribute) */
  SVQ_ERR_TIMEOUT = 5            /* a kernel's bounded wait ran out (read by svq_get_device_status) */
};

enum svq_dtype { SVQ_F16 = 1, SVQ_BF16 = 2, SVQ_F32 = 3 };

/* One SVQ matrix W[N][K].  Column j of the stored order multiplies x[perm[j]].
 * perm may be NULL: the caller then supplies x already in the stored column
 * order (the producer of x applied the permutation, as a decoder layer does
 * when the previous kernel writes its output permuted), every call below reads
 * x[m][j] for column j, and the permutation pass of svq_linear_gemm is
 * skipped.
 * The quantized radius (Figure 2 caption) of row n and radius code c is
 *   r = fmaf(radius_scale[n], c, radius_offset[n])  (fp32, affine form), or,
 *   when radius_lut is not NULL, r = radius_lut[n][c] (a per-row table of
 *   2^b_r fp16 levels: levels fitted freely, as the pages optimise them; then
 *   radius_scale and radius_offset are not read and may be NULL).  The table
 *   form needs b_r <= 4 (b_d >= 6); svq_moe_grouped_gemv does not take it. */
typedef struct svq_matrix {
  int32_t N;                      /* output features (rows of W)                            */
  int32_t K;                      /* input features                                         */
  int32_t b_d;                    /* direction-index bits; radius code has 10 - b_d bits    */
  int32_t reserved;               /* must be 0                                              */
  const void* packed;             /* device layout written by svq_repack, svq_packed_bytes  */
  const uint16_t* codebook;       /* fp16 [1 << b_d][8], 16-byte aligned                    */
  const uint16_t* radius_scale;   /* fp16 [N]                                               */
  const uint16_t* radius_offset;  /* fp16 [N]                                               */
  const int32_t* perm;            /* [K], a permutation of 0..K-1, 4-byte aligned, or NULL  */
  const uint16_t* radius_lut;     /* fp16 [N][1 << (10 - b_d)], 2-byte aligned, or NULL      */
} svq_matrix;

/* Message for a status code (static string). */
SVQ_API const char* svq_status_string(int status);

/* Library version, e.g. 100 for 0.1.0. */
SVQ_API int svq_version(void);

/* Bytes of the device layout of an N x K matrix: exactly N * K * 9 / 32 (18 bits
 * per 8 weights, Figure 2 caption), the same size as the canonical stream, for
 * N % 4 == 0 and K % 128 == 0; otherwise Np * Kp * 9 / 32 with N and K rounded
 * up to multiples of 4 and 128 (padding).  Returns 0 when K % 8 != 0. */
SVQ_API size_t svq_packed_bytes(int N, int K);

/* Bytes of the canonical stream: N * ceil(18 * (K/8) / 8). */
SVQ_API size_t svq_canonical_bytes(int N, int K);

/*
 * svq_repack -- lossless conversion of the canonical code stream into the
 * device layout used by every kernel (done once per matrix, offline).
 *
 * canonical [N][ceil(18*(K/8)/8)] bytes: row n, subvector g occupies stream bits
 *   [18g, 18g+18) of the row, stream bit b = bit (b mod 8) of byte b/8 (LSB
 *   first); code word bits 0..7 = signs (bit i -> element i, 1 = negative),
 *   bits 8..8+b_d-1 = direction index, the remaining b_r bits = radius code.
 *   (The pages give the 18-bit budget and the three fields, Figure 2 caption;
 *   the bit order is this library's interchange reading.)
 * packed_out: svq_packed_bytes(N, K) bytes, 16-byte aligned.
 * The device layout groups 4 rows x 16 subvectors (144 bytes) per lane so that a
 * warp streams 16-byte coalesced loads; it holds exactly the same bits.
 */
SVQ_API int svq_repack(const uint8_t* canonical, int N, int K, int b_d, void* packed_out,
               svq_stream_t stream);

/*
 * svq_unpack_fields -- decode the device layout back into per-subvector fields
 * (test and inspection aid).  signs [N][K/8] uint8, idx [N][K/8] uint16,
 * code [N][K/8] uint16.  Bit-exact inverse of svq_repack.
 */
SVQ_API int svq_unpack_fields(const void* packed, int N, int K, int b_d, uint8_t* signs,
                      uint16_t* idx, uint16_t* code, svq_stream_t stream);

/*
 * svq_dequantize -- export the dense weights in the stored (permuted) column
 * order, w_out [N][K] of out_dtype SVQ_F16 or SVQ_BF16.  Per element:
 *   r = fmaf(scale_n, code, offset_n) in fp32 (the quantized radius, Figure 2),
 *   w = round_to_nearest_even(r * c_{idx,i}) (binary32 product, then fp16/bf16),
 *   then the sign bit is set when the code's sign bit is 1 (a zero becomes -0).
 * Bit-exact against the reference decoder.
 */
SVQ_API int svq_dequantize(const svq_matrix* W /* host struct */, int out_dtype, void* w_out,
                   svq_stream_t stream);

/*
 * Workspace for svq_linear_gemv / svq_linear_gemv_batched (0 bytes when no
 * 128-row tile is split across CTAs): completion counters in its first 64 KiB,
 * then partial sums of the split tiles.  The counters must be zero before the
 * first call that uses a workspace (svq_workspace_init zero-fills it); every
 * completed call leaves them zero again, so one workspace can serve a stream of
 * calls of any shapes it is large enough for.  Calls that share a workspace
 * must not overlap on the GPU.
 */
SVQ_API int svq_linear_gemv_workspace_size(const svq_matrix* W /* host */, int M, size_t* bytes);
SVQ_API int svq_workspace_init(void* workspace, size_t bytes, svq_stream_t stream);

/*
 * svq_linear_gemv -- decode-and-multiply for batch 1 to 16:
 *   y[m][n] = sum_j W[n][j] * x[m][perm[j]],  m < M, with W decoded on the fly.
 * x: fp16 [M][K] (natural input order; the kernel applies perm, Figure 6;
 * stored order when perm is NULL).
 * y: [M][N] of y_dtype SVQ_F16 or SVQ_F32.  Each subvector's eight products
 * of fp16 codeword entries and fp16 activations are formed exactly and
 * accumulated in fp32 (one rounding per addition), scaled by the radius and
 * accumulated across subvectors in fp32, so any finite fp16 x is safe from
 * overflow.
 * Error bound used by the tests: |y - y_ref| <= 1e-3 * sum_j |W[n][j]||x[m][perm[j]]|.
 * Launch: the kernel is launched as a programmatic dependent of the previous
 * kernel on `stream`; it reads x only after that kernel has completed, but may
 * read the weights (packed codes, codebook, radius parameters, perm) as soon as
 * every block of that kernel has exited.  svq_repack makes its stores visible
 * before its blocks exit; a caller whose own kernel writes the weights right
 * before a GEMV on the same stream must do the same (e.g. end it with
 * __threadfence()).
 */
SVQ_API int svq_linear_gemv(const svq_matrix* W /* host */, const uint16_t* x, int M, void* y,
                    int y_dtype, void* workspace, size_t workspace_bytes, svq_stream_t stream);

/*
 * svq_linear_gemv_batched -- several independent layers in one launch
 * (e.g. the seven linears of a decoder layer, or q|k|v sharing one x):
 *   y_i = W_i x_i for i < n_mats (n_mats <= 8), each with its own M-row input.
 * mats, x, y are HOST arrays of n_mats entries (x[i], y[i] device pointers).
 * The launch shares the GPU's SMs among the matrices in proportion to their
 * sizes, so its workspace depends on the whole group:
 * svq_linear_gemv_batched_workspace_size.
 */
SVQ_API int svq_linear_gemv_batched_workspace_size(const svq_matrix* mats, int n_mats, int M,
                                           size_t* bytes);
SVQ_API int svq_linear_gemv_batched(const svq_matrix* mats, int n_mats, const uint16_t* const* x,
                            int M, void* const* y, int y_dtype, void* workspace,
                            size_t workspace_bytes, svq_stream_t stream);

/*
 * svq_linear_gemv_batched_host -- svq_linear_gemv_batched for a decode step
 * whose activations come from and whose results go to host memory: one call
 * enqueues on `stream` the copy of x_host into x_dev, the grouped launch and
 * the copy of y_dev into y_host (cudaMemcpyAsync each; nothing is allocated).
 * x_host, x_dev: the n_mats inputs back to back, input i = M rows of
 *   mats[i].K fp16 values (natural input order, as for svq_linear_gemv_batched).
 * y_host, y_dev: the n_mats outputs back to back, output i = M rows of
 *   mats[i].N values of y_dtype (SVQ_F16 or SVQ_F32).
 * x_dev and y_dev are device buffers the caller owns; x_host and y_host should
 * be page-locked, otherwise the copies are not asynchronous.  Every check of
 * svq_linear_gemv_batched runs before anything is enqueued; the call returns
 * once the three operations are enqueued, so y_host holds the results only
 * after the stream has reached them (e.g. cudaStreamSynchronize).
 */
SVQ_API int svq_linear_gemv_batched_host(const svq_matrix* mats, int n_mats, const uint16_t* x_host,
                                         uint16_t* x_dev, int M, void* y_host, void* y_dev, int y_dtype,
                                         void* workspace, size_t workspace_bytes, svq_stream_t stream);

/*
 * svq_linear_gemv_noalloc -- svq_linear_gemv for callers that cannot allocate
 * device memory.  The paper has no counterpart; this is a deployment aid.  Some
 * callers have no allocator to get a workspace from: a plugin that is handed
 * only a stream, code that runs after its host has frozen its memory pools, or
 * a real-time loop where a cudaMalloc could stall.  This entry point takes the
 * same inputs and outputs as svq_linear_gemv (x fp16 [M][K], y [M][N] of
 * SVQ_F16 or SVQ_F32, M 1..16) but keeps its split-K scratch in a fixed 1 MiB
 * array inside the library, which every GPU that loads the library holds
 * until the process exits.  It allocates nothing and calls no allocating
 * routine.
 *   - A call whose scratch need (svq_linear_gemv_workspace_size) exceeds
 *     1 MiB returns SVQ_ERR_WORKSPACE and enqueues nothing (e.g. M = 8 on a
 *     32768 x 2560 matrix; split such a call into passes of fewer rows).
 *   - The first call on a device looks up the array's device address and
 *     zero-fills it on `stream`; under lazy module loading that first call may
 *     also be what loads the library's device code, which reserves the array
 *     and the kernels' code on that device.  Make the first call on each
 *     device at set-up time: before the host freezes its memory pools and
 *     before any stream capture.  The first-call set-up is guarded, so host
 *     threads may make their first calls concurrently.
 *   - All calls share the one array: calls that overlap on the GPU (other
 *     streams, other threads) race and give wrong results; serialise them.
 *   - The array keeps the last call's contents; the counters that must start
 *     at zero are zeroed at set-up and left zero by every completed call.
 */
SVQ_API int svq_linear_gemv_noalloc(const svq_matrix* W /* host */, const uint16_t* x, int M, void* y,
                                    int y_dtype, svq_stream_t stream);

/*
 * svq_linear_gemm -- prefill / batched layer on the tensor cores (tcgen05):
 *   y[m][n] = sum_j W[n][j] * x[m][perm[j]],  any M >= 1.
 * The pages' prefill kernel is a 64-row GEMM loop that accumulates mma products
 * (Figure 6(b) caption); here weight tiles are decoded from the codes into
 * shared memory as bf16 (x_dtype SVQ_BF16) or fp16 (x_dtype SVQ_F16) -- the
 * weights are the same rounded values svq_dequantize exports -- and multiplied
 * with fp32 accumulation in tensor memory.  x: [M][K] of x_dtype (natural input
 * order; stored order when perm is NULL, x then 16-byte aligned because the
 * Tensor Memory Accelerator (TMA) reads it directly).  y: [M][N] of y_dtype SVQ_F32
 * or SVQ_BF16.
 * Workspace (svq_linear_gemm_workspace_size): the permuted activations
 * x[:, perm] (unused when perm is NULL); from two token tiles on (M > 128,
 * except M = 256, one tile) the matrix decoded once (N x K values of x_dtype, the weights
 * svq_dequantize exports), which the tensor cores then read in place of
 * decoding every weight tile once per token tile; and, when tiles are split
 * along K across CTAs (the tiles of a last, partial round over the SMs, or all
 * of them), the fp32 partial sums of those tiles (summed by a second kernel in
 * slice order).  It
 * carries no state between calls and needs no initialisation.  Error bound used by the tests:
 * |y - y_ref| <= 1e-2 * sum_j |W[n][j]||x[m][perm[j]]|.
 */
SVQ_API int svq_linear_gemm_workspace_size(const svq_matrix* W /* host */, int M, size_t* bytes);
SVQ_API int svq_linear_gemm(const svq_matrix* W /* host */, const uint16_t* x, int x_dtype, int M, void* y,
                            int y_dtype, void* workspace, size_t workspace_bytes, svq_stream_t stream);

/*
 * svq_moe_grouped_gemv -- many SVQ matrices applied to many rows in one call,
 * driven by a DEVICE-side item list (mixture-of-experts layers, whose routing
 * is produced on the GPU).  The pages evaluate SVQ on an MoE model
 * (Qwen3-30B-A3B, abstract) without describing an MoE kernel; each expert
 * matrix is an SVQ matrix as in Figure 2 with its own permutation (Figure 6).
 *
 *   for every item i:  v_i = out_scale_i * W[matrix_i] * in(x_row_i)
 *   accumulate == 0:   y[out_row_i] = v_i          (out rows must be distinct)
 *   accumulate == 1:   y[r] = sum of v_i over the items with out_row == r, in
 *                      item order (rows with no item are left untouched)
 * in(row): x_mode SVQ_X_F16 -> x is fp16 [n_x_rows][K], in(row) = x[row];
 *          x_mode SVQ_X_SWIGLU_F32 -> x is fp32 [n_x_rows][2K] holding [gate | up],
 *          in(row) = fp16(silu(gate) * up) computed per element in fp32.
 * Item fields are checked on the device: an item whose x_row lies outside
 *   0..n_x_rows-1 reads zeros, one whose out_row lies outside 0..n_out_rows-1
 *   (accumulate == 0) is not written, an item whose matrix lies outside
 *   0..n_mats-1 is skipped; each of these sets the device status word to
 *   SVQ_ERR_INVALID_ARG (svq_get_device_status).  With accumulate == 1 the
 *   items of one output row are summed in item order by one CTA per row, linear
 *   in the number of items.
 * mats: DEVICE array of n_mats descriptors (same layout as svq_matrix), every
 *   one N x K with b_d <= max_b_d; the host cannot read them, so the caller
 *   guarantees them (the host checks N, K, max_b_d and the pointers it sees).
 * items: DEVICE array of n_items.  Each touched matrix is decoded once per
 *   pass and applied to up to P of its items in that pass, P = 1, 2 or 4 chosen
 *   from max_items_per_matrix (1 -> 1, 2 -> 2, else 4); a matrix with more
 *   items takes more passes.  The grouping of items by matrix (routing) is done
 *   on the device, by every CTA in shared memory for up to 2048 matrices and
 *   4096 items, else by a separate routing kernel through the workspace.
 * y: fp32 [n_out_rows][N].  Workspace: svq_moe_grouped_gemv_workspace_size.
 * Tolerance used by the tests: as svq_linear_gemv (1e-3 of sum |W| |in|).
 */
typedef struct svq_group_item {
  int32_t matrix;    /* index into mats                         */
  int32_t x_row;     /* input row                               */
  int32_t out_row;   /* output row of y                         */
  float out_scale;   /* multiplies W * in before it is written  */
} svq_group_item;

enum svq_x_mode { SVQ_X_F16 = 0, SVQ_X_SWIGLU_F32 = 1 };

SVQ_API int svq_moe_grouped_gemv_workspace_size(int n_mats, int n_items, int N, int accumulate, size_t* bytes);
SVQ_API int svq_moe_grouped_gemv(const svq_matrix* mats, int n_mats, int N, int K, int max_b_d,
                                 const svq_group_item* items, int n_items, int max_items_per_matrix,
                                 const void* x, int x_mode, int n_x_rows, float* y, int n_out_rows, int accumulate,
                                 void* workspace, size_t workspace_bytes, svq_stream_t stream);

/*
 * Decoder-layer producers: kernels that write a linear layer's input directly
 * in the stored column order of its SVQ matrices, so those matrices can be
 * called with perm NULL.  Each subvector multiplies eight reordered activations
 * (Figure 6 caption); the pages leave open where the reordering happens.  The
 * two producers of a Qwen3-style decoder layer (the models the pages evaluate)
 * are below.  Both are launched as programmatic dependents like the GEMV: they
 * read their input only after the previous kernel on `stream` has completed,
 * and the kernel after them may start its weight-only prologue early (its own
 * wait still covers their writes).  Results are deterministic.
 *
 * svq_rmsnorm_permute -- RMS normalisation of M rows of the residual stream h,
 * written once for each of n_out consumers (1..8):
 *   inv_m = 1 / sqrt( (1/K) sum_k h[m][k]^2 + eps )          (fp32)
 *   outs[g][m][j] = fp16( (h[m][s] * inv_m) * gamma[s] ),  s = perms[g][j]
 * (s = j when perms is NULL or perms[g] is NULL).  h: [M][K] of h_dtype
 * SVQ_F16 or SVQ_BF16, 16-byte aligned; gamma: fp16 [K], 16-byte aligned;
 * perms: HOST array of n_out device pointers ([K] int32, 4-byte aligned) or
 * NULL; outs: HOST array of n_out device pointers, fp16 [M][K], 16-byte
 * aligned, not overlapping h.  K a multiple of 8, 0 <= M <= 65535, eps finite
 * and >= 0.  M = 0 returns SVQ_OK without looking at any pointer.  Tolerance used by the tests: 1 fp16 unit in the last place of the
 * fp64 value rounded once.
 *
 * svq_swiglu_permute -- the gated activation in front of an MLP's down
 * projection, written in that matrix's stored column order:
 *   x[m][j] = fp16( silu(gate[m][s]) * up[m][s] ),  s = perm[j] (or j if NULL),
 *   silu(v) = v / (1 + e^-v) in fp32 (the expression SVQ_X_SWIGLU_F32 uses).
 * gate, up: fp32 [M][I] (e.g. the fp32 outputs of the gate and up GEMVs),
 * 16-byte aligned; perm: [I] int32, 4-byte aligned, or NULL; x: fp16 [M][I],
 * 16-byte aligned.  I a multiple of 8, 0 <= M <= 65535 (M = 0: SVQ_OK, no
 * pointer looked at).  Tolerance: as above.
 */
SVQ_API int svq_rmsnorm_permute(const uint16_t* h, int h_dtype, const uint16_t* gamma, float eps, int M, int K,
                                const int32_t* const* perms /* host array */, uint16_t* const* outs /* host array */,
                                int n_out, svq_stream_t stream);
SVQ_API int svq_swiglu_permute(const float* gate, const float* up, int M, int I, const int32_t* perm, uint16_t* x,
                               svq_stream_t stream);

/*
 * Calibration side (offline, before svq_repack): Energy-Stratified Grouping,
 * the per-row radius grid, the activation-weighted encoder and Adaptive Bit
 * Split ("SAGE", abstract; Figure 2 caption: signs, direction index and
 * quantized radius fitted under activation-energy weights; Figure 4(a): the
 * energy exponent gamma).  The pages give no formulas; the readings are stated
 * with each call.  Every integer result (permutation, signs, direction indices,
 * radius codes, the chosen split) is decided from fp64 values computed with one
 * rounding per operation in a fixed order, so it is reproducible bit for bit.
 * Inputs must be finite.  All pointers are device pointers; nothing is
 * allocated; every call is asynchronous on `stream`.
 *
 * svq_esg -- channel energies e_k = (sum_t x_cal[t][k]^2) / T (fp64, t
 * ascending), the ESG permutation and the fitting weights.  The channels are
 * ordered by energy, highest first (equal energies: lower index first) and cut
 * into 8 tiers of K/8; stored column 8g + t takes the g-th channel of tier t:
 * perm[8g + t] = order[t * K/8 + g].  weights[k] = (float) pow(e_k, gamma)
 * (NULL: not written; pow is CUDA's, within 2 ulp in fp64).
 * x_cal: fp32 [T][K], 4-byte aligned; energy: fp64 [K] out, 8-byte aligned;
 * perm: int32 [K] out; weights: fp32 [K] out or NULL.  T >= 1, K a multiple of
 * 8.  Cost O(K^2) comparisons (ranking).
 *
 * svq_radius_grid -- per-row uniform radius grid: with the row's subvector
 * norms in stored order (W[n][perm[8g..8g+7]], squares summed in element order,
 * correctly rounded sqrt) and their minimum lo and maximum hi,
 * offset[n] = fp16(lo) and scale[n] = fp16((hi - lo) / (2^b_r - 1)) (0 when
 * b_r = 0), each rounded once to nearest even.  W: fp32 [N][K], natural column
 * order; perm: [K] or NULL (identity).
 *
 * svq_encode -- encodes W (fp32 [N][K], natural column order) as the
 * canonical stream of an SVQ matrix with stored column j = perm[j] (identity
 * when perm is NULL).  Per subvector (stored columns 8g..8g+7, w = those
 * weights, e = weights[perm[...]], all 1 when weights is NULL): sign bit
 * s_i = (w_i < 0); (idx, code) minimises
 *   X = sum_i e_i (|w_i| - r_code c_idx,i)^2,  r_code = fma(scale[n], code, offset[n]) (fp32)
 * evaluated term by term in fp64 (i ascending), ties to the lowest idx, then
 * the lowest code -- the brute-force choice, reached without evaluating every
 * pair (a filter with a proven error bound skips pairs that cannot win).
 * With radius_lut (fp16 [N][2^b_r], b_r <= 4) the levels are r_code =
 * radius_lut[n][code] and scale/offset are not read (may be NULL).
 * codebook: fp16 [2^b_d][8]; scale, offset: fp16 [N]; canonical: [N][row
 * bytes of svq_canonical_bytes] out, pad bits zero; row_err: fp64 [N] out or
 * NULL: sum_j e_j (W[n][perm[j]] - What[n][j])^2 over the row (What the exact
 * decoded weight), per subvector in element order, then in a fixed tree over
 * each 32 subvectors and in order over those chunks.  1 <= b_d <= 10, K a
 * multiple of 8.
 *
 * svq_abs_select -- Adaptive Bit Split: totals[k] = sum_n row_err[k][n] (fixed
 * order) for n_cand (1..64) candidate encodings of one matrix (row_err: fp64
 * [n_cand][N], each written by svq_encode under one split), and *best = the
 * first candidate with the least total.  totals may be NULL; best: int32 [1].
 */
SVQ_API int svq_esg(const float* x_cal, int T, int K, double gamma, double* energy, int32_t* perm, float* weights,
                    svq_stream_t stream);
SVQ_API int svq_radius_grid(const float* W, int N, int K, const int32_t* perm, int b_d, uint16_t* scale,
                            uint16_t* offset, svq_stream_t stream);
SVQ_API int svq_encode(const float* W, int N, int K, int b_d, const int32_t* perm, const float* weights,
                       const uint16_t* codebook, const uint16_t* scale, const uint16_t* offset,
                       const uint16_t* radius_lut, uint8_t* canonical, double* row_err, svq_stream_t stream);
SVQ_API int svq_abs_select(const double* row_err, int n_cand, int N, double* totals, int32_t* best,
                           svq_stream_t stream);

/*
 * Synchronising read-and-clear of the device status word that kernels set
 * when a bounded wait runs out (SVQ_ERR_TIMEOUT) or a device-side argument
 * check fails (SVQ_ERR_INVALID_ARG); SVQ_OK when neither happened.  Tests only.
 */
SVQ_API int svq_get_device_status(svq_stream_t stream);

/*
 * Test aid for the failure path of the bounded waits (no counterpart in the
 * paper).  Every wait of svq_linear_gemm on a pipeline barrier polls at most
 * `polls` times (default 2^21) before it gives up: the kernel then sets the
 * status word to SVQ_ERR_TIMEOUT, lets the copies it already issued land,
 * releases its tensor memory and returns (no trap, no hang).  polls == 0 makes
 * the first wait give up at once.  Applies to launches enqueued after the
 * call, process-wide; returns the previous bound.  Restore the default before
 * relying on results.
 */
SVQ_API unsigned svq_debug_set_wait_polls(unsigned polls);

#ifdef __cplusplus
}
#endif

#endif /* SVQ_H_ */
