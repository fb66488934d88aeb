// qamw_calibrate.cu -- sigma_k partial sums (step 3 of "Methodology: The
// QAM-W Codec", QAM-W Technical Summary) for Hadamard blocks b <= 512.
//
// sigma_k = RN32(sqrt(2/pi) * (1/M) * sum_i ||z_ik||) over the rotated unit
// rows. A CTA of 14 warps takes a contiguous range of tiles (28 rows x one
// 512-column chunk) in chunk-major order; warp w rotates rows 28g + w and
// 28g + w + 14 with the 512-column unit of qamw_rotate16.cuh (one-pass
// transposes; the block size fixed at compile time for bf16 weights). The 28
// rows' ||z_ik|| are added in shared memory in row order (0..27) and written
// as the row group's fp64 partial sum; sigma_reduce (qamw_encode.cu) adds the
// groups in a fixed order.
// The sums are the same, in the same order, as those of the 1024-column
// calibrate kernel (b = 1024), so sigma does not depend on the kernel.
#include <algorithm>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"
#include "qamw_rotate16.cuh"

namespace qamw {
namespace {

#ifndef QAMW_CAL_WARPS
#define QAMW_CAL_WARPS 14
#endif
constexpr int kWarps = QAMW_CAL_WARPS;     // warps per CTA
constexpr int kRows = kTileRows / kWarps;  // rows of a tile per warp (warp w: rows w, w + kWarps, ...)
constexpr int kThreads = kWarps * 32;
static_assert(kCalibRowGroup == kTileRows, "one calibration row group per tile");
static_assert(kRows * kWarps == kTileRows, "the tile's rows split evenly over the warps");

struct CalibSmem {
  double sd[32 * kSdPitch];
  double part[2][kTileRows][32 * kIsPitch];   // double-buffered per-row |z| of the tile (pair layout)
  double xbuf[kWarps][kXbufFull];             // per-warp transpose buffers
};

template <int WT, int LB>
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

  auto prefetch = [&](int64_t chunk, int64_t g, int rr, WRegs<WT> &w, float &rn) -> bool {
    const int64_t row = g * kTileRows + warp + rr * kWarps;
    rn = 0.0f;
    if (row >= M) return false;
    rn = ra.r[row];
    return load_unit16<WT>(w, ra.W, ra.ldw, K, row, chunk * kUnit + 16 * lane, vec_ok);
  };

  WRegs<WT> wn[kRows];
  float rn_next[kRows];
  bool full_next[kRows];
  // tile t = chunk * RG + g, walked incrementally (no 64-bit division per tile)
  int64_t chunk = t0 / RG, g = t0 % RG, next_chunk = chunk, next_g = g;
#pragma unroll
  for (int rr = 0; rr < kRows; ++rr) {
    rn_next[rr] = 0.0f;
    full_next[rr] = (t0 < t1) ? prefetch(chunk, g, rr, wn[rr], rn_next[rr]) : false;
  }
  int64_t cur_chunk = -1;
  int buf = 0;
  for (int64_t t = t0; t < t1; ++t, buf ^= 1, chunk = next_chunk, g = next_g) {
    next_g = g + 1;
    next_chunk = chunk;
    if (next_g == RG) { next_g = 0; ++next_chunk; }
    if (chunk != cur_chunk) {
      __syncthreads();
      for (int c = threadIdx.x; c < kUnit; c += kThreads) load_sd512(sm.sd, ra.s, ra.seed, K, chunk, c);
      __syncthreads();
      cur_chunk = chunk;
    }
#pragma unroll
    for (int rr = 0; rr < kRows; ++rr) {
      const WRegs<WT> wc = wn[rr];
      const bool full = full_next[rr];
      const float r = rn_next[rr];
      if (t + 1 < t1) full_next[rr] = prefetch(next_chunk, next_g, rr, wn[rr], rn_next[rr]);

      const int64_t row = g * kTileRows + warp + rr * kWarps;
      double acc[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) acc[p] = 0.0;
      if (row < M && r > 0.0f && isfinite(r)) {   // a zero (or non-finite) row adds nothing; uniform per warp
        double u[16];
        rotate_unit16<WT, false, LB>(u, wc, full, ra.W, ra.ldw, K, row, chunk * kUnit + 16 * lane,
                                     &sm.sd[lane * kSdPitch], ra.log2b, sm.xbuf[warp], lane);
        const double q = inv_sqrt_b / (double)r;
#pragma unroll
        for (int m = 0; m < 8; ++m)
          acc[m] = q * sqrt(__dadd_rn(__dmul_rn(u[2 * m], u[2 * m]), __dmul_rn(u[2 * m + 1], u[2 * m + 1])));
      }
      double2 *dst = reinterpret_cast<double2 *>(&sm.part[buf][warp + rr * kWarps][lane * kIsPitch]);
#pragma unroll
      for (int h = 0; h < 4; ++h) dst[h] = make_double2(acc[2 * h], acc[2 * h + 1]);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kUnit / 2; i += kThreads) {
      const int64_t pair = chunk * (kUnit / 2) + i;
      double s = 0.0;
      const int slot = pair_slot(i);
#pragma unroll 4
      for (int w = 0; w < kTileRows; ++w) s += sm.part[buf][w][slot];   // the tile's rows in row order
      if (pair < P) a.partials[g * P + pair] = s;
    }
    // part[buf] is written again two tiles later, after the next tile's barrier
  }
}

template <typename Kern>
cudaError_t set_smem(Kern k, size_t bytes) {
  return set_max_dynamic_smem(reinterpret_cast<const void *>(k), bytes);
}

template <int WT, int LB>
cudaError_t launch_t(const CalibArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(CalibSmem);
  cudaError_t e = set_smem(calibrate512_kernel<WT, LB>, smem);
  if (e != cudaSuccess) return e;
  const int64_t n_chunks = (a.rot.K + kUnit - 1) / kUnit;
  const int64_t tiles = n_chunks * ((a.rot.M + kTileRows - 1) / kTileRows);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(tiles, sm_count()));
  const size_t es = (WT == QAMW_BF16) ? 2 : 4;
  const int vec = ((reinterpret_cast<uintptr_t>(a.rot.W) % 16) == 0 && (a.rot.ldw * (int64_t)es) % 16 == 0) ? 1 : 0;
  calibrate512_kernel<WT, LB><<<(int)blocks, kThreads, smem, s>>>(a, vec);
  return cudaGetLastError();
}

// block sizes 128 and 256 (the bf16 workloads) compiled for their size
template <int WT>
cudaError_t launch_wt(const CalibArgs &a, cudaStream_t s) {
  if (WT == QAMW_BF16 && a.rot.log2b == 7) return launch_t<WT, 7>(a, s);
  if (WT == QAMW_BF16 && a.rot.log2b == 8) return launch_t<WT, 8>(a, s);
  return launch_t<WT, 0>(a, s);
}

// Test hook (qamw_rotate_rows) for b <= 512: the encode's and calibrate's
// 512-column rotation applied to fp64 rows. Forward: Y = H_b (d U) / sqrt(b);
// inverse: Y = d (H_b U) / sqrt(b). The first butterfly is the same fma as in
// scaled16 with s = 1 (one rounding, like the add).
constexpr int kRotWarps = 8;
__global__ void __launch_bounds__(kRotWarps * 32) rotate_test512_kernel(RotateTestArgs a) {
  __shared__ __align__(16) double xbuf[kRotWarps][kXbufFull];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_chunks = (a.K + kUnit - 1) / kUnit;
  const int64_t U = n_chunks * a.M;
  const double inv_sqrt_b = 1.0 / sqrt((double)(1 << a.log2b));
  for (int64_t unit = (int64_t)blockIdx.x * kRotWarps + warp; unit < U; unit += (int64_t)gridDim.x * kRotWarps) {
    const int64_t chunk = unit / a.M, row = unit % a.M;
    const int64_t col0 = chunk * kUnit + 16 * lane;
    double x[16], v[16], u[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int64_t col = col0 + e;
      double t = (col < a.K) ? a.U[row * a.K + col] : 0.0;
      if (!a.inverse && col < a.K && mask_is_negative(a.seed, col)) t = -t;
      x[e] = t;
    }
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const double b = x[2 * h + 1] * 1.0;
      v[2 * h] = fma(x[2 * h], 1.0, b);
      v[2 * h + 1] = fma(x[2 * h], 1.0, -b);
    }
    fwht16_low<0>(v, a.log2b);
    transpose16<false>(v, u, xbuf[warp], lane);
    fwht16_high<0>(u, a.log2b, lane);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int64_t col = chunk * kUnit + 128 * (lane >> 3) + 16 * m + 2 * (lane & 7) + e;
        if (col < a.K) {
          double y = u[2 * m + e] * inv_sqrt_b;
          if (a.inverse && mask_is_negative(a.seed, col)) y = -y;
          a.Y[row * a.K + col] = y;
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_rotate_test512(const RotateTestArgs &a, cudaStream_t s) {
  const int64_t n_chunks = (a.K + kUnit - 1) / kUnit;
  const int64_t units = n_chunks * a.M;
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((units + kRotWarps - 1) / kRotWarps, 4096));
  rotate_test512_kernel<<<(int)blocks, kRotWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_calibrate_partials512(const CalibArgs &a, cudaStream_t s) {
  return (a.rot.wt == QAMW_BF16) ? launch_wt<QAMW_BF16>(a, s) : launch_wt<QAMW_F32>(a, s);
}

}  // namespace qamw
