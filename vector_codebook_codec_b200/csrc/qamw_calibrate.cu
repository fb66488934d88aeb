// qamw_calibrate.cu -- sigma_k partial sums (step 3 of "Methodology: The
// QAM-W Codec", QAM-W Technical Summary) for Hadamard blocks b <= 512.
//
// sigma_k = RN32(sqrt(2/pi) * (1/M) * sum_i ||z_ik||) over the rotated unit
// rows. A CTA of 28 warps takes a contiguous range of tiles (28 rows x one
// 512-column chunk) in chunk-major order, warp w holding row 28g + w with the
// 512-column unit of qamw_rotate16.cuh. The 28 rows' ||z_ik|| are added in
// shared memory in row order (w = 0..27) and written as the row group's fp64
// partial sum; sigma_reduce (qamw_encode.cu) adds the groups in a fixed order.
// The sums are the same, in the same order, as those of the 1024-column
// calibrate kernel, so both give the same sigma.
#include <algorithm>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"
#include "qamw_rotate16.cuh"

namespace qamw {
namespace {

constexpr int kWarps = kTileRows;
constexpr int kThreads = kWarps * 32;
static_assert(kCalibRowGroup == kTileRows, "one calibration row group per tile");

struct CalibSmem {
  double sd[32 * kSdPitch];
  double part[2][kWarps][32 * kIsPitch];   // double-buffered per-row |z| of the tile
};

template <int WT>
__global__ void __launch_bounds__(kThreads, 1) calibrate512_kernel(CalibArgs a, int vec_ok) {
  extern __shared__ __align__(16) unsigned char smem[];
  CalibSmem &sm = *reinterpret_cast<CalibSmem *>(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const RotateArgs &ra = a.rot;
  const int64_t M = ra.M, K = ra.K, P = K >> 1;
  const int64_t n_chunks = (K + kUnit - 1) / kUnit;
  const int64_t RG = (M + kTileRows - 1) / kTileRows;
  const int64_t T = n_chunks * RG;
  const int64_t t0 = (int64_t)blockIdx.x * T / gridDim.x, t1 = ((int64_t)blockIdx.x + 1) * T / gridDim.x;
  const double inv_sqrt_b = 1.0 / sqrt((double)(1 << ra.log2b));

  auto prefetch = [&](int64_t chunk, int64_t g, WRegs<WT> &w, float &rn) -> bool {
    const int64_t row = g * kTileRows + warp;
    rn = 0.0f;
    if (row >= M) return false;
    rn = ra.r[row];
    return load_unit16<WT>(w, ra.W, ra.ldw, K, row, chunk * kUnit + 16 * lane, vec_ok);
  };

  WRegs<WT> wn;
  float rn_next = 0.0f;
  // tile t = chunk * RG + g, walked incrementally (no 64-bit division per tile)
  int64_t chunk = t0 / RG, g = t0 % RG, next_chunk = chunk, next_g = g;
  bool full_next = (t0 < t1) ? prefetch(chunk, g, wn, rn_next) : false;
  int64_t cur_chunk = -1;
  int buf = 0;
  for (int64_t t = t0; t < t1; ++t, buf ^= 1, chunk = next_chunk, g = next_g) {
    next_g = g + 1;
    next_chunk = chunk;
    if (next_g == RG) { next_g = 0; ++next_chunk; }
    if (chunk != cur_chunk) {
      __syncthreads();
      if (threadIdx.x < kUnit) load_sd512(sm.sd, ra.s, ra.seed, K, chunk, threadIdx.x);
      __syncthreads();
      cur_chunk = chunk;
    }
    const WRegs<WT> wc = wn;
    const bool full = full_next;
    const float r = rn_next;
    if (t + 1 < t1) full_next = prefetch(next_chunk, next_g, wn, rn_next);

    const int64_t row = g * kTileRows + warp;
    double acc[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) acc[p] = 0.0;
    if (row < M && r > 0.0f && isfinite(r)) {   // a zero (or non-finite) row adds nothing
      double v[16];
      scaled16<WT>(v, wc, full, ra.W, ra.ldw, K, row, chunk * kUnit + 16 * lane, &sm.sd[lane * kSdPitch]);
      fwht16_fp64(v, ra.log2b, lane);
      const double q = inv_sqrt_b / (double)r;
#pragma unroll
      for (int p = 0; p < 8; ++p)
        acc[p] = q * sqrt(__dadd_rn(__dmul_rn(v[2 * p], v[2 * p]), __dmul_rn(v[2 * p + 1], v[2 * p + 1])));
    }
    double2 *dst = reinterpret_cast<double2 *>(&sm.part[buf][warp][lane * kIsPitch]);
#pragma unroll
    for (int h = 0; h < 4; ++h) dst[h] = make_double2(acc[2 * h], acc[2 * h + 1]);
    __syncthreads();
    if (threadIdx.x < kUnit / 2) {
      const int i = threadIdx.x;
      const int64_t pair = chunk * (kUnit / 2) + i;
      double s = 0.0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += sm.part[buf][w][(i >> 3) * kIsPitch + (i & 7)];
      if (pair < P) a.partials[g * P + pair] = s;
    }
    // part[buf] is written again two tiles later, after the next tile's barrier
  }
}

template <typename Kern>
cudaError_t set_smem(Kern k, size_t bytes) {
  return set_max_dynamic_smem(reinterpret_cast<const void *>(k), bytes);
}

template <int WT>
cudaError_t launch_t(const CalibArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(CalibSmem);
  cudaError_t e = set_smem(calibrate512_kernel<WT>, smem);
  if (e != cudaSuccess) return e;
  const int64_t n_chunks = (a.rot.K + kUnit - 1) / kUnit;
  const int64_t tiles = n_chunks * ((a.rot.M + kTileRows - 1) / kTileRows);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(tiles, sm_count()));
  const size_t es = (WT == QAMW_BF16) ? 2 : 4;
  const int vec = ((reinterpret_cast<uintptr_t>(a.rot.W) % 16) == 0 && (a.rot.ldw * (int64_t)es) % 16 == 0) ? 1 : 0;
  calibrate512_kernel<WT><<<(int)blocks, kThreads, smem, s>>>(a, vec);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_calibrate_partials512(const CalibArgs &a, cudaStream_t s) {
  return (a.rot.wt == QAMW_BF16) ? launch_t<QAMW_BF16>(a, s) : launch_t<QAMW_F32>(a, s);
}

}  // namespace qamw
