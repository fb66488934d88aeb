// qamw_internal.h -- launcher interface between the C-ABI layer (qamw_api.cu)
// and the kernel translation units. Arguments here are already validated.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "qamw.h"

namespace qamw {

// Rows per calibration row group (fixed, so the fp64 reduction order -- and
// hence sigma -- does not depend on the device or the grid size).
constexpr int kCalibRowGroup = 28;
// Columns handled by one warp in the encode / calibrate kernels (32 lanes x 32).
constexpr int kUnitCols = 1024;

// Header of a search table (see qamw_search.cu).
constexpr uint32_t kSearchMagic = 0x34574D51u;   // "QMW4": table layout version 4 (8-byte cell records)
constexpr int kSearchMaxG = 181;                 // the scan kernel's limit (32768 cells)
constexpr int kSearchInline = 3;                 // candidates held in a cell record
constexpr int kSearchImageOffset = 64;           // bytes from the table's start to the records
struct SearchHeader {
  uint32_t magic;
  int32_t N, G, total;     // total: overflow entries used
  int32_t valid, capacity; // capacity: overflow entries the table holds
  // The grid is uniform in u = T(x) = x / (a + |x|) on each axis: cell index
  // floor((T(x) + UL) * inv_cw), UL = T(L); it covers [-L, L]^2 in x.
  float a, UL, inv_cw, L;
  int32_t image_bytes;     // records + overflow, a multiple of 16: the bytes the encode copies
  int32_t pad;
};
static_assert(sizeof(SearchHeader) == 48, "search header is 48 bytes");
// A cell record: four 16-bit fields e0, e1, e2, meta. meta & 3 = n in 1..3:
// the cell's list is e0..e(n-1) (ascending; unused fields repeat e0). n = 0:
// the list is e0, e1, e2 followed by ovf[o + 1 .. o + ovf[o]] (o = meta >> 2,
// ascending), in the table's overflow array.
__host__ __device__ __forceinline__ uint64_t search_record(uint32_t e0, uint32_t e1, uint32_t e2, uint32_t meta) {
  return (uint64_t)e0 | ((uint64_t)e1 << 16) | ((uint64_t)e2 << 32) | ((uint64_t)meta << 48);
}
int search_grid(int N);

// The encode's cell of a normalised pair: per axis c = round(T(x) * inv_cw +
// (G - 1) / 2) with T(x) = x / (a + |x|), which for odd G is floor((T(x) + UL)
// * inv_cw), the grid of the table; -1 outside the grid (|x| > L on an axis,
// or a non-finite x). The rounding to an integer is that of one fp32 fma at
// the magnitude 1.5 * 2^23 (unit spacing), cbias = 1.5 * 2^23 + (G - 1) / 2,
// and the integer is read from the float's bits: no conversion instruction.
// Its error in cells (approximate reciprocal, two fp32 roundings) is below
// 1e-4, inside the 1e-3-cell margin every list is built with.
constexpr float kCellMagic = 12582912.0f;        // 1.5 * 2^23
constexpr int kCellMagicBits = 0x4B400000;       // its fp32 bits
__device__ __forceinline__ int search_cell(float x0, float x1, float a, float inv_cw, float cbias, float L, int G) {
  const float u0 = __fdividef(x0, __fadd_rn(a, fabsf(x0)));
  const float u1 = __fdividef(x1, __fadd_rn(a, fabsf(x1)));
  const int cx = __float_as_int(__fmaf_rn(u0, inv_cw, cbias)) - kCellMagicBits;
  const int cy = __float_as_int(__fmaf_rn(u1, inv_cw, cbias)) - kCellMagicBits;
  const bool in = fmaxf(fabsf(x0), fabsf(x1)) <= L && (unsigned)cx < (unsigned)G && (unsigned)cy < (unsigned)G;
  return in ? cy * G + cx : -1;
}
int64_t search_capacity(int N);
size_t search_table_bytes(int N);
cudaError_t launch_build_search_table(const float *codebook, int N, void *table, cudaStream_t s);
// Test hook: the encode's cell of n pairs (float32 [n][2]) for a table (-1 off the grid or for an invalid table).
cudaError_t launch_search_cells(const float *x, int64_t n, const void *table, int32_t *cell_out, cudaStream_t s);

struct ScaleArgs {
  const float *act_rms;  // [K] or nullptr
  float alpha;
  int64_t K;
  float *s_out;          // [K]
  int32_t *status;
};

struct RowNormArgs {
  const void *W;
  qamw_dtype wt;
  int64_t M, K, ldw;
  const float *s;        // [K]
  float *r_out;          // [M]
  int32_t *status;
};

struct RotateArgs {       // shared by encode and calibrate
  const void *W;
  qamw_dtype wt;
  int64_t M, K, ldw;
  int32_t log2b;
  uint64_t seed;
  const float *s;        // [K] channel scales
  const float *r;        // [M] stored row norms
};

struct CalibArgs {
  RotateArgs rot;
  double *partials;      // [G][K/2]
  int64_t groups;        // G = ceil(M / kCalibRowGroup)
  float *sigma_out;      // [K/2]
  double *sum_out = nullptr;  // [K/2]: if set, the fp64 sums are written instead of sigma
};

struct EncodeArgs {
  RotateArgs rot;
  const float *sigma;    // [K/2]
  const float *codebook; // [N][2]
  int32_t N;
  int32_t bits;
  int64_t wpr;           // words per row
  uint32_t *packed;      // [M][wpr]
  const void *table;     // search table or nullptr (brute force)
  int32_t *status;
  const double *polar_amps = nullptr;   // polar baseline: A amplitude levels (ascending), P sectors
  int32_t polar_A = 0, polar_P = 0;
};

struct DecodeArgs {
  const uint32_t *packed;
  const float *row_norm;
  const float *sigma;
  const float *col_scale;  // nullable
  int64_t M, K;
  int32_t log2b;
  uint64_t seed;
  const float *codebook;
  int32_t N;
  int32_t bits;
  int64_t wpr;
  void *out;
  qamw_dtype out_t;
  int64_t ldo;
  int32_t *status;
};

struct RotateTestArgs {
  const double *U;
  double *Y;
  int64_t M, K;
  int32_t log2b;
  uint64_t seed;
  int32_t inverse;
};

// Each launcher returns cudaSuccess or the launch error.
cudaError_t launch_channel_scale(const ScaleArgs &a, cudaStream_t s);
cudaError_t launch_row_norms(const RowNormArgs &a, cudaStream_t s);
cudaError_t launch_calibrate(const CalibArgs &a, cudaStream_t s);
// sigma_k from R row shards' sums [R][P] added in rank order.
cudaError_t launch_sigma_from_sums(const double *sums, int R, int64_t P, int64_t M, float *sigma_out,
                                   cudaStream_t s);
// The partial sums of the calibration for b <= 512 (qamw_calibrate.cu).
cudaError_t launch_calibrate_partials512(const CalibArgs &a, cudaStream_t s);
cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t s);
// Encode with the pruned search (qamw_encode_pruned.cu): a table given,
// b <= 512 and N <= kPrunedMaxN; otherwise launch_encode takes the brute-force
// kernel.
constexpr int kPrunedMaxN = 2048;
bool encode_pruned_applicable(const EncodeArgs &a);
cudaError_t launch_encode_pruned(const EncodeArgs &a, cudaStream_t s);
// The polar baseline encode (qamw_encode_polar.cu), b <= 512.
cudaError_t launch_encode_polar(const EncodeArgs &a, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
// bf16 decode with TMA tensor loads/stores (qamw_decode_tma.cu).
bool decode_tma_applicable(const DecodeArgs &a);
cudaError_t launch_decode_tma(const DecodeArgs &a, cudaStream_t s);
cudaError_t launch_rotate_test(const RotateTestArgs &a, cudaStream_t s);
// Decode fused with the matrix multiply Y = X W_hat^T on the tensor cores
// (qamw_decode_gemm.cu): X bf16 [T][ldx], Y fp32 [T][ldy], workspace of
// decode_matmul_workspace_bytes(M, K, T) bytes (256-byte aligned); K % 128 == 0,
// K <= 32768, N <= QAMW_MAX_CENTROIDS, T <= 2^24.
size_t decode_matmul_workspace_bytes(int64_t M, int64_t K, int64_t T);
cudaError_t launch_decode_gemm(const DecodeArgs &d, const uint16_t *X, int64_t T, int64_t ldx, float *Y, int64_t ldy,
                               void *workspace, cudaStream_t s);
// The same for b <= 512 with the 512-column rotation of the encode and calibrate kernels.
cudaError_t launch_rotate_test512(const RotateTestArgs &a, cudaStream_t s);

// Lloyd training of the 2D codebook (qamw_lloyd.cu); points and centroids are
// fp64 [.][2], 16-byte aligned.
size_t lloyd_workspace_bytes(int64_t T, int N);
cudaError_t launch_lloyd_assign(const double *pts, int64_t T, const double *cent, int N, int32_t *idx,
                                unsigned long long *changed, cudaStream_t s);
cudaError_t launch_lloyd_update(const double *pts, int64_t T, const int32_t *idx, int N, double *cent,
                                void *workspace, int32_t *empty_count, cudaStream_t s);

// Test hook: a bounded wait on an mbarrier that never completes (qamw_selftest.cu).
cudaError_t launch_wait_timeout(uint32_t tries, int32_t *status, cudaStream_t s);

// cudaFuncSetAttribute(func, MaxDynamicSharedMemorySize, bytes) on the current
// device, once per (kernel, device) and size: later calls with a size already
// set cost a lookup instead of a driver call.
cudaError_t set_max_dynamic_smem(const void *func, size_t bytes);

// Number of SMs of the current device (cached per device).
int sm_count();

// Sets the message qamw_last_error() returns on this host thread.
void set_last_error(const char *msg);

}  // namespace qamw
