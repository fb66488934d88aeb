/*
 * qamw.h -- C ABI of libqamw.so, the sm_100a (B200) QAM-W weight codec.
 *
 * The method: "QAM-W: Joint 2D Codebook Quantization for LLM Weights via
 * Hadamard Rotation and Activation-Aware Scaling" (gist.science/paper/2605.26339),
 * Technical Summary, "Methodology: The QAM-W Codec", steps
 *   (1) Separation of Scale and Direction  (2) Deterministic Rotation
 *   (3) Pairing and Calibration            (4) Joint 2D Quantization
 *   (5) Activation-Aware Scaling           (6) Decoding.
 * Step (5) is applied before quantization, so a row is coded as
 *   w'_j = w_j * s_j                     s_j = RN32(act_rms_j ^ alpha), pow in fp64   (5)
 *   r    = RN32(||w'||_2)                stored row norm                               (1)
 *   y    = H_b (d * w'/r) / sqrt(b)      per block of b columns, d_j = +-1 mask         (2)
 *   z_k  = (y_2k, y_2k+1),  x_k = RN32(z_k / sigma_k)                                  (3)
 *   idx_k = argmin_c |x_k - C_c|^2       lowest index on ties                          (4)
 * and decoded as w_hat = r * d * (H_b (sigma (.) C[idx])) / (sqrt(b) * s)           (6).
 * H_b is the Sylvester (natural order) Hadamard matrix; d_j = -1 exactly when
 * bit 63 of the (j+1)-th SplitMix64 output for sign_seed is set (one mask per
 * matrix, shared by all rows).
 *
 * Conventions shared by every entry point
 *   - Every array pointer is a DEVICE pointer owned by the caller. The
 *     library allocates nothing; between calls it keeps only caches of device
 *     attributes (SM count, shared-memory opt-in) and the fixed scratch area
 *     of qamw_calibrate_sigma_noalloc, none of which affects results.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and return once the kernels are enqueued.
 *   - Arguments are validated on the host before anything is launched; on a
 *     validation error nothing is enqueued and the status code says why.
 *   - Shapes: W is M x K, row-major with leading dimension ld >= K (elements).
 *     K must be even and a multiple of the block size b; b is a power of two
 *     in [2, 1024]; 1 <= bits_per_pair <= 16; 1 <= N <= min(2^bits, 8192).
 *   - Packed index stream: uint32 [M][qamw_words_per_row(K, bits)], each row
 *     starting on a fresh word; index k of a row occupies stream bits
 *     k*bits .. k*bits+bits-1, least significant bit first, and stream bit t is
 *     bit (t mod 32) of word t/32 (little-endian words).
 *   - Codebook: float32 [N][2] (x, y) centroids, row-major.
 *   - `status` (nullable) is a device int32 the kernels OR bits into
 *     (QAMW_STATUS_*); the caller clears it and reads it after syncing.
 *   - Return value: QAMW_OK or an error code below; qamw_last_error() gives a
 *     message for the most recent failing call on the calling host thread.
 */
#ifndef QAMW_H_
#define QAMW_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *qamw_stream_t; /* same type as cudaStream_t */

typedef enum { QAMW_F32 = 0, QAMW_BF16 = 1 } qamw_dtype;

/* Return codes. */
enum {
  QAMW_OK = 0,
  QAMW_EINVAL = 1,       /* bad shape or argument value */
  QAMW_ENULL = 2,        /* a required pointer is NULL */
  QAMW_EUNSUPPORTED = 3, /* valid for the method but beyond this build's limits */
  QAMW_ECUDA = 4,        /* a CUDA call failed (see qamw_last_error) */
  QAMW_EWORKSPACE = 5    /* workspace missing or smaller than required */
};

/* Device status bits (ORed into *status by the kernels). */
#define QAMW_STATUS_BAD_INDEX 1u        /* decode: an index >= N (decoded as 0) */
#define QAMW_STATUS_NONFINITE_NORM 2u   /* a row norm is Inf/NaN */
#define QAMW_STATUS_BAD_ACT_RMS 4u      /* an act_rms entry is not finite and > 0 */
#define QAMW_STATUS_NONFINITE_INPUT 8u  /* encode: a row norm is Inf/NaN (the row is coded as zero pairs) or a sigma_k gives no finite fp32 pair (1/sigma_k not finite or beyond the fp32 range) */
#define QAMW_STATUS_TIMEOUT 16u         /* a bounded wait on an asynchronous copy ran out; output incomplete */

/* Maximum sizes of this build. */
#define QAMW_MAX_CENTROIDS 8192
#define QAMW_MAX_BLOCK 1024

/* Words per row of the packed stream: ceil((K/2) * bits / 32); -1 if invalid. */
int64_t qamw_words_per_row(int64_t K, int32_t bits_per_pair);

/* Message for a return code (static string). */
const char *qamw_status_string(int code);

/* Message of the most recent failing call on this host thread ("" if none). */
const char *qamw_last_error(void);

/* Version string of the library. */
const char *qamw_version(void);

/*
 * qamw_channel_scale -- Methodology (5) Activation-Aware Scaling.
 * s_out[j] = RN32(pow((double)act_rms[j], (double)alpha)) for j < K; the
 * proportionality constant is 1. act_rms == NULL writes s = 1. Entries that
 * are not finite and > 0 give s = 1 and set QAMW_STATUS_BAD_ACT_RMS.
 *   act_rms  : device float32 [K] or NULL      s_out : device float32 [K]
 */
int qamw_channel_scale(const float *act_rms, float alpha, int64_t K, float *s_out,
                       int32_t *status, qamw_stream_t stream);

/*
 * qamw_calibrate_workspace_bytes -- scratch needed by qamw_calibrate_sigma
 * (and qamw_calibrate_partial_sums, qamw_calibrate_encode): s_j [K] and r_i
 * [M] in fp32, then the fp64 partial sums of |z| [ceil(M/28)][K/2], each
 * section 256-byte aligned. 0 for M < 1 or K < 2.
 */
size_t qamw_calibrate_workspace_bytes(int64_t M, int64_t K);

/*
 * qamw_calibrate_sigma -- Methodology (3) Pairing and Calibration.
 * sigma_out[k] = RN32(sqrt(2/pi) * (1/M) * sum_i |z_ik|) for k < K/2, the
 * Rayleigh mean-amplitude estimate that maps pair k onto the unit circular
 * Gaussian; a pair position that is zero in every row gets 1.0. z is computed
 * exactly as in qamw_encode (steps 5, 1, 2). The sum runs in fp64 over fixed
 * row groups and is reduced in a fixed order, so the result is deterministic.
 *   W        : device [M][ldw] of w_dtype        act_rms : device float32 [K] or NULL (s = 1)
 *   sigma_out: device float32 [K/2]              workspace: device, >= qamw_calibrate_workspace_bytes(M, K)
 * Errors: QAMW_ENULL (W, sigma_out, workspace), QAMW_EINVAL (shape, alpha not
 * finite, M < 1), QAMW_EWORKSPACE.
 */
int qamw_calibrate_sigma(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                         const float *act_rms, float alpha, int32_t block, uint64_t sign_seed,
                         float *sigma_out, void *workspace, size_t workspace_bytes,
                         int32_t *status, qamw_stream_t stream);

/*
 * qamw_calibrate_partial_sums / qamw_sigma_from_partial_sums -- the calibration
 * of one matrix whose rows are split across devices (or calls). sigma_k is a
 * mean over all M rows, so each shard of rows contributes its sum of |z_ik|
 * (Methodology (3)); the shards' sums are exchanged (one all-gather) and
 * combined:
 *   qamw_calibrate_partial_sums: sums_out[k] = sum over the shard's rows i of
 *     |z_ik| in fp64, in the fixed order qamw_calibrate_sigma uses (same
 *     arguments and workspace as qamw_calibrate_sigma; sums_out: device
 *     float64 [K/2]);
 *   qamw_sigma_from_partial_sums: sums = device float64 [R][P] (shard r's sums
 *     in row r), added in shard order; sigma_out[k] = RN32(sqrt(2/pi) *
 *     total_k / M_total), 0 -> 1.
 * With one shard (R = 1, M_total = M) the result equals qamw_calibrate_sigma's
 * bit for bit. Errors: as qamw_calibrate_sigma; QAMW_EINVAL for R, P or
 * M_total < 1.
 */
int qamw_calibrate_partial_sums(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                                const float *act_rms, float alpha, int32_t block, uint64_t sign_seed,
                                double *sums_out, void *workspace, size_t workspace_bytes, int32_t *status,
                                qamw_stream_t stream);
int qamw_sigma_from_partial_sums(const double *sums, int32_t R, int64_t P, int64_t M_total, float *sigma_out,
                                 qamw_stream_t stream);

/*
 * qamw_calibrate_sigma_noalloc -- qamw_calibrate_sigma for callers that cannot
 * allocate device memory.
 * (An interface of this library; the QAM-W page has no counterpart.)
 * Some callers cannot provide the calibration workspace: an inference engine
 * that freezes its device memory pool after start-up, a plug-in whose host
 * framework owns all device memory and offers no allocator, or a
 * latency-critical path on which cudaMalloc (which may synchronize the
 * device) is not acceptable. This entry point computes exactly what
 * qamw_calibrate_sigma computes, with the same arguments minus the
 * workspace, using a fixed scratch area of QAMW_NOALLOC_SCRATCH_BYTES bytes
 * built into the library; neither it nor the library allocates anything.
 *   - Limit: qamw_calibrate_workspace_bytes(M, K) must not exceed
 *     QAMW_NOALLOC_SCRATCH_BYTES, i.e.
 *       align256(4K) + align256(4M) + align256(ceil(M/28) * (K/2) * 8) <= 8 MiB
 *     (align256 rounds up to a multiple of 256). For large M this is about
 *     M*K <= 58 million weights; for M < 28 the partial sums alone take 4K
 *     bytes, so K is at most about 2 million. Larger shapes return
 *     QAMW_EUNSUPPORTED with a message that says so.
 *   - The area is reserved on every GPU that loads the library, until the
 *     process exits.
 *   - Set-up: the first call made in a given context (device) looks up the
 *     area's device address (cudaGetSymbolAddress) and caches it with that
 *     context; a call in another context (after cudaDeviceReset, or with a
 *     non-primary context current) looks it up again. Make the first call
 *     in a context before any stream capture in it.
 *   - All calls share the one area and it keeps the last call's contents;
 *     nothing in it needs to start at zero (each call writes every byte it
 *     reads). Calls whose kernels overlap on the GPU (different streams, or
 *     different host threads) race on the area: serialize them.
 * Errors: as qamw_calibrate_sigma (except EWORKSPACE), plus QAMW_EUNSUPPORTED
 * for shapes beyond the limit and QAMW_ECUDA if the address lookup fails.
 */
#define QAMW_NOALLOC_SCRATCH_BYTES (8u << 20)
int qamw_calibrate_sigma_noalloc(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                                 const float *act_rms, float alpha, int32_t block, uint64_t sign_seed,
                                 float *sigma_out, int32_t *status, qamw_stream_t stream);

/*
 * qamw_encode -- Methodology steps (5), (1), (2), (3), (4) and bit packing.
 * For every row: s_j (step 5), r_i = RN32(||w' ||) written to row_norm_out
 * (step 1), the sign-masked block Hadamard rotation (step 2, in fp64, so that
 * x_k = RN32(z_k / sigma_k) is the correctly rounded value), pairing with the
 * given sigma (step 3), the nearest centroid by fp32 direct-difference squared
 * distance (x0-c0)^2 + (x1-c1)^2 with the lowest index on ties (step 4), and
 * the packed stream described above. A zero row codes x = 0.
 *   W           : device [M][ldw] of w_dtype       act_rms : device float32 [K] or NULL
 *   sigma       : device float32 [K/2] (from qamw_calibrate_sigma, all > 0)
 *   codebook    : device float32 [N][2]
 *   search_table: device table from qamw_build_search_table for this codebook,
 *                 or NULL for the brute-force search over all N centroids.
 *                 Both searches return the same index. The table is used for
 *                 b <= 512 and N <= 2048; other shapes take the brute-force
 *                 search (same result). A table that does not match the
 *                 codebook (another N, a corrupt header) makes every pair
 *                 scan all N centroids, still exact.
 *   packed_out  : device uint32 [M][qamw_words_per_row(K, bits)]
 *   row_norm_out: device float32 [M]                 col_scale_out: device float32 [K] (s_j)
 * row_norm_out and col_scale_out are the metadata qamw_decode needs; the
 * encode also reads them back between its kernels (no other scratch).
 * Errors: QAMW_ENULL, QAMW_EINVAL (shape, code size, alpha), QAMW_EUNSUPPORTED.
 */
int qamw_encode(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                const float *act_rms, float alpha, int32_t block, uint64_t sign_seed,
                const float *sigma, const float *codebook, int32_t N, int32_t bits_per_pair,
                const void *search_table, uint32_t *packed_out, float *row_norm_out,
                float *col_scale_out, int32_t *status, qamw_stream_t stream);

/*
 * qamw_encode_prepared -- qamw_encode with the channel scales and row norms
 * given: steps (2), (3), (4) and bit packing of Methodology, reading s_j and
 * r_i instead of computing them (steps (5) and (1)), e.g. the col_scale_out
 * and row_norm_out of an earlier qamw_encode or qamw_calibrate_encode of the
 * same matrix, or stored metadata. One kernel; its packed stream equals
 * qamw_encode's bit for bit when s and r are the ones qamw_encode writes.
 * (An interface of this library; the QAM-W page has no counterpart.)
 *   col_scale: device float32 [K] (s_j)   row_norm: device float32 [M] (r_i; a zero
 *              row codes x = 0, a non-finite one sets QAMW_STATUS_NONFINITE_INPUT)
 *   other arguments as qamw_encode.
 * Errors: QAMW_ENULL, QAMW_EINVAL (shape, code size), QAMW_EUNSUPPORTED.
 */
int qamw_encode_prepared(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                         const float *col_scale, const float *row_norm, int32_t block, uint64_t sign_seed,
                         const float *sigma, const float *codebook, int32_t N, int32_t bits_per_pair,
                         const void *search_table, uint32_t *packed_out, int32_t *status, qamw_stream_t stream);

/*
 * qamw_calibrate_encode -- qamw_calibrate_sigma followed by qamw_encode on the
 * same matrix, as one call: Methodology (3) calibrates sigma over the rows of
 * W, then steps (5), (1), (2), (3), (4) code them with that sigma. The channel
 * scales s_j (step 5) and the row norms r_i (step 1) are computed once, into
 * col_scale_out and row_norm_out, and read by both passes; the two separate
 * calls compute each of them twice. Every output equals, bit for bit, what
 * qamw_calibrate_sigma and then qamw_encode (with sigma_out as its sigma)
 * write.
 * (An interface of this library; the QAM-W page has no counterpart.)
 *   sigma_out : device float32 [K/2]   workspace: device, 256-byte aligned,
 *               >= qamw_calibrate_workspace_bytes(M, K)
 *   other arguments as qamw_encode; packed_out, row_norm_out and
 *   col_scale_out are qamw_encode's outputs, and the calibration reads
 *   row_norm_out and col_scale_out after writing them.
 * Errors: as qamw_encode, plus QAMW_EWORKSPACE.
 */
int qamw_calibrate_encode(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                          const float *act_rms, float alpha, int32_t block, uint64_t sign_seed,
                          const float *codebook, int32_t N, int32_t bits_per_pair, const void *search_table,
                          float *sigma_out, uint32_t *packed_out, float *row_norm_out, float *col_scale_out,
                          void *workspace, size_t workspace_bytes, int32_t *status, qamw_stream_t stream);

/*
 * qamw_search_table_bytes / qamw_build_search_table -- an exact pruned search
 * for Methodology (4): a grid over the plane of normalised pairs, each cell
 * listing (in ascending index order) every centroid that can be the fp32
 * nearest one for a pair in that cell. qamw_encode given the table returns
 * the same indices as without it (the brute-force search), faster. The table
 * depends only on the codebook; build it once per codebook.
 *   codebook : device float32 [N][2]      table: device, 16-byte aligned,
 *   >= qamw_search_table_bytes(N) bytes (0 if N is out of range).
 * A codebook whose lists overflow the table's capacity yields a table marked
 * invalid, with which qamw_encode uses the brute-force search.
 */
size_t qamw_search_table_bytes(int32_t N);
int qamw_build_search_table(const float *codebook, int32_t N, void *table, size_t table_bytes,
                            qamw_stream_t stream);

/*
 * qamw_search_cells -- test hook for the pruned search of Methodology (4):
 * the grid cell the encode assigns to each normalised pair, computed by the
 * encode's own device function (cell_out[i] = iy * G + ix of the table's
 * grid, or -1 for a pair outside the grid or an invalid table). With the
 * table's lists it lets a test check that every pair's exact nearest
 * centroid is listed in the cell the encode actually looks in.
 * (An interface of this library; the QAM-W page has no counterpart.)
 *   x: device float32 [n][2]   table: as for qamw_encode   cell_out: device int32 [n]
 * Errors: QAMW_ENULL, QAMW_EINVAL (n < 0, table not 16-byte aligned).
 */
int qamw_search_cells(const float *x, int64_t n, const void *table, int32_t *cell_out, qamw_stream_t stream);

/*
 * qamw_encode_polar -- the polar baseline codec ("Joint 2D vs. Polar", Results
 * of the QAM-W page): steps (5), (1), (2), (3) exactly as qamw_encode, then
 * the amplitude and the phase of each normalised pair are quantized
 * independently, at the rate of a joint codebook of A*P points:
 *   a = number of edges (amps[i] + amps[i+1]) / 2 below hypot(x0, x1),
 *   p = floor((atan2(x1, x0) mod 2 pi) / (2 pi / P)) mod P,  index = a * P + p,
 * decided in fp64 from the fp32 pair. The stream decodes with qamw_decode
 * given the A*P reconstruction points amps[a] * (cos, sin)(2 pi (p + 1/2) / P),
 * in index order, as the codebook.
 *   amps: device float64 [A], ascending, 8-byte aligned; 1 <= A*P <= 2^bits.
 * Other arguments as qamw_encode (block <= 512; larger blocks return
 * QAMW_EUNSUPPORTED).
 */
int qamw_encode_polar(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                      const float *act_rms, float alpha, int32_t block, uint64_t sign_seed,
                      const float *sigma, const double *amps, int32_t A, int32_t P, int32_t bits_per_pair,
                      uint32_t *packed_out, float *row_norm_out, float *col_scale_out, int32_t *status,
                      qamw_stream_t stream);

/*
 * qamw_decode -- Methodology (6) Decoding.
 * w_hat_ij = r_i * d_j * (H_b (sigma (.) C[idx]))_j / (sqrt(b) * s_j): unpack,
 * look up centroids, rescale by sigma_k, inverse rotation, multiply by the
 * stored row norm, divide by the stored channel scale. fp32 arithmetic; the
 * output is rounded (RNE) to out_dtype. bf16 output is what the page's pipeline
 * feeds to the matrix multiply ("Significance and Claims").
 *   packed   : device uint32 [M][qamw_words_per_row(K, bits)]
 *   row_norm : device float32 [M]      sigma : device float32 [K/2]
 *   col_scale: device float32 [K] (s_j as written by qamw_encode) or NULL (s = 1)
 *   codebook : device float32 [N][2]   W_out : device [M][ldo] of out_dtype
 * An index >= N decodes as centroid 0 and sets QAMW_STATUS_BAD_INDEX; a
 * non-finite row norm sets QAMW_STATUS_NONFINITE_NORM.
 */
int qamw_decode(const uint32_t *packed, const float *row_norm, const float *sigma,
                const float *col_scale, int64_t M, int64_t K, int32_t block,
                uint64_t sign_seed, const float *codebook, int32_t N, int32_t bits_per_pair,
                void *W_out, qamw_dtype out_dtype, int64_t ldo, int32_t *status,
                qamw_stream_t stream);

/*
 * qamw_decode_matmul -- Methodology (6) Decoding fused with the matrix
 * multiply that consumes the weights ("Significance and Claims": the bit
 * savings reach inference latency once decoding is fused into the matmul):
 *   Y[t][m] = sum_j X[t][j] * w_hat[m][j],   w_hat as qamw_decode defines it,
 * without forming w_hat. The decode's steps after the codebook lookup are
 * linear and shared by all rows, and H_b is symmetric, so they are applied to
 * the activations instead:
 *   Y[t][m] = r_m * sum_i a_t[i] * C[idx(m, i/2)][i % 2],
 *   a_t[i]  = sigma_{i/2} * (H_b (d (.) X[t] / s))_i / sqrt(b)   (per block of b columns).
 * A first kernel computes a_t in fp32 and stores it in the workspace as fp16,
 * scaled by a power of two 2^-e_t per token (its largest |a| lands in
 * (2^13, 2^14]); a second streams the packed indices, looks up the centroids
 * as fp16 pairs and stores them straight into the tensor-core A operand in
 * tensor memory, multiplies on the tensor cores (tcgen05, fp32 accumulation in
 * tensor memory) and scales by r_m 2^e_t. The weights never reach device
 * memory, nor shared memory.
 * Accuracy: with S[t][m] = r_m sum_i |a_t[i] C[idx(m,i/2)][i%2]| and
 * Q[t][m] = r_m sum_i sigma_{i/2} |C[..]| sum_{j in block(i)} |X[t][j] / s_j| / sqrt(b),
 *   |Y - Y_exact| <= (2^-10 + K 2^-22) S + 2^-19 Q + (tiny fp16-subnormal terms),
 * i.e. two fp16 roundings per product (2^-11 each) against the one bf16
 * rounding (2^-8) of decoding to bf16 first.
 *   packed, row_norm, sigma, col_scale, codebook: as qamw_decode (packed 8-byte, sigma 16-byte aligned)
 *   X : device bf16 [T][ldx] (activations, row-major; 16-byte aligned, ldx a multiple of 8)
 *   Y : device float32 [T][ldy] (written for t < T, m < M)
 *   workspace : device, 256-byte aligned, >= qamw_decode_matmul_workspace_bytes(M, K, T)
 *               bytes (the fp16 a_t, the per-token powers of two, and the partial sums
 *               of output tiles whose K range is split between CTAs); owned by the caller
 * Limits of this build: K a multiple of 128 and at most 32768
 * (QAMW_EUNSUPPORTED otherwise). Status bits as qamw_decode, plus
 * QAMW_STATUS_TIMEOUT if a bounded wait for a copy or a tensor-core result
 * ran out. NaN or Inf activations propagate into Y as in any matrix product.
 * Errors: QAMW_ENULL, QAMW_EINVAL (shape, T outside [1, 2^24], ldx / ldy,
 * alignment, workspace too small), QAMW_EUNSUPPORTED.
 */
int qamw_decode_matmul(const uint32_t *packed, const float *row_norm, const float *sigma, const float *col_scale,
                       int64_t M, int64_t K, int32_t block, uint64_t sign_seed, const float *codebook, int32_t N,
                       int32_t bits_per_pair, const void *X, int64_t T, int64_t ldx, float *Y, int64_t ldy,
                       void *workspace, size_t workspace_bytes, int32_t *status, qamw_stream_t stream);
/* Workspace bytes qamw_decode_matmul needs for M rows, K columns and T tokens
 * (0 unless M, K >= 1 and 1 <= T <= 2^24). */
size_t qamw_decode_matmul_workspace_bytes(int64_t M, int64_t K, int64_t T);

/*
 * qamw_rotate_rows -- the rotation alone, for tests of step (2).
 * inverse == 0: Y = H_b (d * U) / sqrt(b); inverse != 0: Y = d * (H_b U) / sqrt(b),
 * per block of b columns, in fp64 (the encode path's arithmetic).
 *   U, Y : device float64 [M][K] (dense, ld = K)
 */
int qamw_rotate_rows(const double *U, double *Y, int64_t M, int64_t K, int32_t block,
                     uint64_t sign_seed, int32_t inverse, qamw_stream_t stream);

/*
 * qamw_selftest_wait_timeout -- test hook for failure detection (an interface
 * of this library; the QAM-W page has no counterpart). Launches one warp that
 * waits, with the bounded mbarrier wait the TMA decode uses (at most `tries`
 * attempts), on a barrier no one arrives on; when the wait runs out it sets
 * QAMW_STATUS_TIMEOUT in *status (device int32) and returns. Nothing hangs or
 * faults; the context stays usable.
 * Errors: QAMW_ENULL (status), QAMW_EINVAL (tries not in [1, 2^20]).
 */
int qamw_selftest_wait_timeout(uint32_t tries, int32_t *status, qamw_stream_t stream);

/*
 * Lloyd training of the 2D codebook -- Methodology (4) Joint 2D Quantization
 * and "Significance and Claims" (the codebook is a 2D Lloyd-Max quantizer
 * trained once on samples of the unit circular Gaussian). One iteration:
 * assign every sample to its nearest centroid (Euclidean, lowest index on
 * ties), then move every centroid to the mean of its samples (a centroid
 * with no sample keeps its place). Everything is fp64.
 *   points    : device float64 [T][2], 16-byte aligned (the samples; drawn by
 *               the caller)
 *   centroids : device float64 [N][2], 16-byte aligned, 1 <= N <= QAMW_MAX_CENTROIDS
 *   idx       : device int32 [T]
 *   workspace : device, 256-byte aligned, >= qamw_lloyd_workspace_bytes(T, N)
 * Sums are formed in a fixed order, so results do not depend on the device.
 *
 * qamw_lloyd_assign writes the nearest index of every sample into idx_inout
 * and, if `changed` (device uint64) is not NULL, adds the number of samples
 * whose index differs from what idx_inout held before.
 * qamw_lloyd_update moves the centroids (in place) to the means of their
 * samples under idx.
 * qamw_lloyd_train runs idx = assign(C); then, up to max_iter times,
 * C = update(idx), idx' = assign(C), stopping when no index changed. It writes
 * the trained centroids in place, the final assignment, and (host pointers,
 * nullable) the iteration count and whether it converged. It synchronizes
 * `stream` once per iteration.
 * Errors: QAMW_ENULL, QAMW_EINVAL (T < 1, N out of range, alignment,
 * max_iter < 0), QAMW_EWORKSPACE, QAMW_ECUDA.
 */
size_t qamw_lloyd_workspace_bytes(int64_t T, int32_t N);
int qamw_lloyd_assign(const double *points, int64_t T, const double *centroids, int32_t N, int32_t *idx_inout,
                      unsigned long long *changed, qamw_stream_t stream);
int qamw_lloyd_update(const double *points, int64_t T, const int32_t *idx, int32_t N, double *centroids_inout,
                      void *workspace, size_t workspace_bytes, qamw_stream_t stream);
int qamw_lloyd_train(const double *points, int64_t T, double *centroids, int32_t N, int32_t max_iter,
                     int32_t *idx_out, void *workspace, size_t workspace_bytes, int32_t *iterations_out,
                     int32_t *converged_out, qamw_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QAMW_H_ */
