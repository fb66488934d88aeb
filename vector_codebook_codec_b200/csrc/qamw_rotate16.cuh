// qamw_rotate16.cuh -- the 512-column unit of the encode and calibrate
// kernels for Hadamard blocks b <= 512: one warp rotates one row x 512
// columns in fp64.
//
// Step (2) of "Methodology: The QAM-W Codec" (QAM-W Technical Summary):
// y = H_b (d (.) w') / sqrt(b) per block, Sylvester H_b, i.e. one butterfly
// per block bit t (columns differing in bit t; the lower keeps a + b, the
// upper a - b). The products w_j * (d_j s_j) are exact in fp64 (bf16 or fp32
// times fp32) and every butterfly is one fp64 add or subtract of the same two
// operands in the same bit order as the 1024-column unit of qamw_encode.cu,
// so the two layouts produce identical values.
//
// Layout. At load, lane l holds columns 16l .. 16l+15 of the unit (column bits
// 0..3 in registers, bits 4..8 = lane bits 0..4). Bits 0..3 are butterflied
// in registers, then the warp transposes through shared memory so that lane
// l' = 8 h + q (h = column bits 7..8, q = column bits 1..3) holds the 16
// columns 128 h + 16 m + 2 q + e (m = 0..7, e = 0..1) as u[2m + e]: bits 4..6
// are butterflied in registers and bits 7..8 (b >= 256) across lanes with
// shuffles. Lane l' then owns the 8 pairs k_m = 64 h + 8 m + q of the unit.
// The transpose costs 8 stores + 8 loads of 16 bytes per lane (or 16 + 8
// with the half-size buffer), conflict-free with a XOR swizzle, against 96
// shuffles for the three cross-lane stages it replaces (b = 128).
#pragma once

#include <cstdint>

#include "qamw_device.cuh"

namespace qamw {

constexpr int kUnit = 512;        // columns per unit
constexpr int kTileRows = 28;     // calibration rows per tile: one per warp (896-thread CTA)
constexpr int kSdPitch = 18;      // doubles per lane row of a d_j s_j table: 16 used (144-byte rows keep 16-byte loads conflict-free)
constexpr int kIsPitch = 10;      // doubles per lane row of a per-pair table: 8 used (80-byte rows)
constexpr int kXbufFull = 512;    // doubles per warp for a one-pass transpose (4 KB)
constexpr int kXbufHalf = 256;    // doubles per warp for a two-pass transpose (2 KB)

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

// Butterflies of block bits 1..3 (register bits 1..3 of the load layout).
// LB > 0 fixes log2 b at compile time (a stage guarded by a run-time block
// size costs register copies where the two paths join); LB = 0 reads log2b.
template <int LB>
__device__ __forceinline__ void fwht16_low(double (&v)[16], int log2b) {
  if (LB > 0) log2b = LB;
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
}

// Load layout -> pair layout (see the file comment). Row r = 4 h + (m mod 4)
// of a half (or 8 h + m of the whole buffer) holds the 8 16-byte chunks q of
// writer lane 8 h + m; chunk q sits at slot q ^ (r & 7), so that the 8 lanes
// of a quarter-warp touch 8 different 16-byte slots of a 128-byte line in
// both directions. HALF: the m < 4 writers go first, then m >= 4, through a
// buffer of half the size (16 stores + 8 loads per lane instead of 8 + 8).
template <bool HALF>
__device__ __forceinline__ void transpose16(const double (&v)[16], double (&u)[16], double *buf, int lane) {
  const int h = lane >> 3, m_w = lane & 7, q_r = lane & 7;
  double2 *b2 = reinterpret_cast<double2 *>(buf);
  if (!HALF) {
    const int r = 8 * h + m_w;
#pragma unroll
    for (int q = 0; q < 8; ++q) b2[r * 8 + (q ^ (r & 7))] = make_double2(v[2 * q], v[2 * q + 1]);
    __syncwarp();
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int rr = 8 * h + m;
      const double2 t = b2[rr * 8 + (q_r ^ (rr & 7))];
      u[2 * m] = t.x;
      u[2 * m + 1] = t.y;
    }
    __syncwarp();
  } else {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if ((m_w >> 2) == half) {
        const int r = 4 * h + (m_w & 3);
#pragma unroll
        for (int q = 0; q < 8; ++q) b2[r * 8 + (q ^ (r & 7))] = make_double2(v[2 * q], v[2 * q + 1]);
      }
      __syncwarp();
#pragma unroll
      for (int mm = 0; mm < 4; ++mm) {
        const int rr = 4 * h + mm;
        const double2 t = b2[rr * 8 + (q_r ^ (rr & 7))];
        u[2 * (4 * half + mm)] = t.x;
        u[2 * (4 * half + mm) + 1] = t.y;
      }
      __syncwarp();
    }
  }
}

// Butterflies of block bits 4..6 (register index bits 1..3 of the pair
// layout) and 7..8 (lane bits 3..4, shuffles; across lanes one
// fma(+-1, own, partner's), rounded once like the add).
template <int LB>
__device__ __forceinline__ void fwht16_high(double (&u)[16], int log2b, int lane) {
  if (LB > 0) log2b = LB;
#pragma unroll
  for (int t = 4; t < 7; ++t) {
    if (t < log2b) {
      const int h = 2 << (t - 4);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if ((i & h) == 0) {
          const double a0 = u[i], a1 = u[i | h];
          u[i] = a0 + a1;
          u[i | h] = a0 - a1;
        }
      }
    }
  }
#pragma unroll
  for (int t = 7; t < 9; ++t) {
    if (t < log2b) {
      const int h = 8 << (t - 7);
      const double sgn = (lane & h) ? -1.0 : 1.0;
#pragma unroll
      for (int i = 0; i < 16; ++i) u[i] = fma(sgn, u[i], __shfl_xor_sync(0xffffffffu, u[i], h));
    }
  }
}

// The whole rotation of the lane's 16 loaded columns: u (pair layout) =
// H_b (d s w) per block, unnormalised (the caller divides by r sqrt(b)).
template <int WT, bool HALF, int LB>
__device__ __forceinline__ void rotate_unit16(double (&u)[16], const WRegs<WT> &w, bool full, const void *W,
                                              int64_t ldw, int64_t K, int64_t row, int64_t col,
                                              const double *sd_lane, int log2b, double *xbuf, int lane) {
  double v[16];
  scaled16<WT>(v, w, full, W, ldw, K, row, col, sd_lane);
  fwht16_low<LB>(v, log2b);
  transpose16<HALF>(v, u, xbuf, lane);
  fwht16_high<LB>(u, log2b, lane);
}

// Index within the unit of pair m (0..7) of lane l' in the pair layout.
__device__ __forceinline__ int unit_pair(int lane, int m) { return 64 * (lane >> 3) + 8 * m + (lane & 7); }

// d_j s_j of the chunk's 512 columns into a [32][kSdPitch] table (load
// layout), one column per thread of a 512-thread group.
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

// Slot of unit pair k (0..255) in a [32][kIsPitch] per-pair table in the pair
// layout: lane 8 (k >> 6) + (k & 7), entry (k >> 3) & 7.
__device__ __forceinline__ int pair_slot(int k) { return (8 * (k >> 6) + (k & 7)) * kIsPitch + ((k >> 3) & 7); }

}  // namespace qamw
