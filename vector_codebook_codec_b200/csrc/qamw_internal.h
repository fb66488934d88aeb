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
constexpr uint32_t kSearchMagic = 0x32574D51u;   // "QMW2": table layout version 2
struct SearchHeader {
  uint32_t magic;
  int32_t N, G, total;
  int32_t valid, capacity;
  // The grid is uniform in u = T(x) = x / (a + |x|) on each axis: cell index
  // floor((T(x) + UL) * inv_cw), UL = T(L); it covers [-L, L]^2 in x.
  float a, UL, inv_cw, L;
  int32_t pad[2];
};
static_assert(sizeof(SearchHeader) == 48, "search header is 48 bytes");
int search_grid(int N);
int64_t search_capacity(int N);
size_t search_table_bytes(int N);
cudaError_t launch_build_search_table(const float *codebook, int N, void *table, cudaStream_t s);

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
