// qamw_rotate16.cuh -- the 512-column unit of the encode and calibrate
// kernels for Hadamard blocks b <= 512: one warp holds one row x 512 columns,
// lane l owning columns [16l, 16l + 16) (8 pairs), in fp64.
//
// Step (2) of "Methodology: The QAM-W Codec" (QAM-W Technical Summary):
// y = H_b (d (.) w') / sqrt(b) per block, Sylvester H_b. The butterflies of
// block bits 0..3 run in registers, those of bits 4..8 across lanes (lane bit
// t - 4) with warp shuffles. Every stage is one fp64 add or subtract of the
// same two operands, in the same bit order, as the 1024-column unit of
// qamw_encode.cu, so the two produce identical values. The products
// w_j * (d_j s_j) are exact in fp64 (bf16 or fp32 times fp32).
#pragma once

#include <cstdint>

#include "qamw_device.cuh"

namespace qamw {

constexpr int kUnit = 512;        // columns per unit
constexpr int kTileRows = 28;     // calibration rows per tile: one per warp (896-thread CTA; 28 measured fastest)
constexpr int kSdPitch = 18;      // doubles per lane row of a d_j s_j table: 16 used (144-byte rows keep 16-byte loads conflict-free)
constexpr int kIsPitch = 10;      // doubles per lane row of a per-pair table: 8 used (80-byte rows)

template <int WT>
struct WRegs {
  uint4 q[WT == QAMW_BF16 ? 2 : 4];   // the lane's 16 weights as loaded
};

template <int WT>
__device__ __forceinline__ double load_scalar(const void *W, int64_t off) {
  if (WT == QAMW_BF16) return bf16_bits_to_double(reinterpret_cast<const uint16_t *>(W)[off]);
  return (double)reinterpret_cast<const float *>(W)[off];
}

// The lane's 16 weights of (row, col..col+15): vector loads (16-byte aligned
// and in range), returns false if the caller must read them scalar.
template <int WT>
__device__ __forceinline__ bool load_unit16(WRegs<WT> &w, const void *W, int64_t ldw, int64_t K, int64_t row,
                                            int64_t col, int vec_ok) {
  if (!(vec_ok && col + 16 <= K)) return false;
  constexpr int es = (WT == QAMW_BF16) ? 2 : 4;
  const uint4 *p = reinterpret_cast<const uint4 *>(reinterpret_cast<const unsigned char *>(W) + (row * ldw + col) * es);
#pragma unroll
  for (int q = 0; q < (WT == QAMW_BF16 ? 2 : 4); ++q) w.q[q] = __ldg(p + q);
  return true;
}

// The lane's 16 weights times d_j s_j, with the butterflies of block bit 0
// applied (every block has b >= 2): v[2i] = w0 a0 + w1 a1, v[2i+1] = w0 a0 -
// w1 a1. The products are exact in fp64 (at most 24 x 24 significant bits), so
// fma(w0, a0, +-w1 a1) rounds the same as the sum of the two rounded products.
// Columns past K count as 0.
template <int WT>
__device__ __forceinline__ void scaled16(double (&v)[16], const WRegs<WT> &w, bool full, const void *W,
                                         int64_t ldw, int64_t K, int64_t row, int64_t col, const double *sd_lane) {
  double x[16];
  if (full) {
    if (WT == QAMW_BF16) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const uint32_t w4[4] = {w.q[q].x, w.q[q].y, w.q[q].z, w.q[q].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          x[8 * q + 2 * h] = bf16_bits_to_double(w4[h] & 0xffffu);
          x[8 * q + 2 * h + 1] = bf16_bits_to_double(w4[h] >> 16);
        }
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        x[4 * q] = (double)__uint_as_float(w.q[q].x);
        x[4 * q + 1] = (double)__uint_as_float(w.q[q].y);
        x[4 * q + 2] = (double)__uint_as_float(w.q[q].z);
        x[4 * q + 3] = (double)__uint_as_float(w.q[q].w);
      }
    }
  } else {
    const int64_t off = row * ldw + col;
#pragma unroll
    for (int e = 0; e < 16; ++e) x[e] = (col + e < K) ? load_scalar<WT>(W, off + e) : 0.0;
  }
  const double2 *sd2 = reinterpret_cast<const double2 *>(sd_lane);
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    const double2 s = sd2[h];
    const double b = x[2 * h + 1] * s.y;
    v[2 * h] = fma(x[2 * h], s.x, b);
    v[2 * h + 1] = fma(x[2 * h], s.x, -b);
  }
}

// Butterflies of block bits 1..log2b-1 (bit 0 is applied by scaled16); the
// partner with block bit t clear keeps a + b, the other keeps a - b. Across
// lanes both are one fma(+-1, own, partner's), rounded once like the add.
__device__ __forceinline__ void fwht16_fp64(double (&v)[16], int log2b, int lane) {
#pragma unroll
  for (int t = 1; t < 4; ++t) {
    if (t < log2b) {
      const int h = 1 << t;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if ((i & h) == 0) {
          const double a0 = v[i], a1 = v[i | h];
          v[i] = a0 + a1;
          v[i | h] = a0 - a1;
        }
      }
    }
  }
#pragma unroll
  for (int t = 4; t < 9; ++t) {
    if (t < log2b) {
      const int h = 1 << (t - 4);
      const double sgn = (lane & h) ? -1.0 : 1.0;
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = fma(sgn, v[i], __shfl_xor_sync(0xffffffffu, v[i], h));
    }
  }
}

// d_j s_j of the chunk's 512 columns into a [32][kSdPitch] table, one column
// per thread of a 512-thread CTA.
__device__ __forceinline__ void load_sd512(double *sd, const float *s, uint64_t seed, int64_t K, int64_t chunk,
                                           int tid) {
  const int64_t col = chunk * kUnit + tid;
  double v = 0.0;
  if (col < K) {
    v = (double)s[col];
    if (mask_is_negative(seed, col)) v = -v;
  }
  sd[(tid >> 4) * kSdPitch + (tid & 15)] = v;
}

}  // namespace qamw
