// qamw_encode.cu -- QAM-W encode side on sm_100a: channel scale (step 5),
// row norms (step 1), the sign-masked block Hadamard rotation (step 2), sigma
// calibration (step 3), nearest-centroid search (step 4) and bit packing.
//
// Method: "QAM-W: Joint 2D Codebook Quantization for LLM Weights via Hadamard
// Rotation and Activation-Aware Scaling", Technical Summary, "Methodology:
// The QAM-W Codec" (steps numbered as on that page).
//
// Work decomposition. A *unit* is one row x 1024 consecutive columns, handled
// by one warp: lane l owns columns [32l, 32l+32) of the unit, i.e. 16 pairs.
// The rotation runs in fp64: the lane applies the butterflies of the block
// bits it holds (bits 0..4) in registers and the higher block bits (5..9) with
// warp shuffles, so a Hadamard block never leaves the warp (b <= 1024).
// Because every product w_j * (d_j s_j) is exact in fp64 and the butterflies
// add only log2(b) roundings of ~1e-16, x = RN32(z / sigma) comes out as the
// correctly rounded value except within ~1e-15 of an fp32 rounding midpoint.
// Units are taken in column-major order (all rows of column chunk 0, then
// chunk 1, ...) so a warp's per-column tables change rarely.
#include <algorithm>
#include <cfloat>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"

namespace qamw {
namespace {

constexpr int kWarps = 8;           // warps per CTA for the unit kernels
constexpr int kThreads = kWarps * 32;
constexpr int kSdPitch = 36;        // floats per lane row of the per-warp scale table
constexpr int kInvPitch = 18;       // doubles per lane row of the per-warp 1/sigma table
constexpr float kFarCentroid = 3.0e18f;  // padding centroid: never the nearest for |x| < 1e18

// ----------------------------------------------------------------------------
// Step (5): s_j = RN32(pow(act_rms_j, alpha)) with the power in fp64.
// ----------------------------------------------------------------------------
__global__ void channel_scale_kernel(ScaleArgs a) {
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < a.K;
       j += (int64_t)gridDim.x * blockDim.x) {
    float s = 1.0f;
    if (a.act_rms != nullptr) {
      const float r = a.act_rms[j];
      if (isfinite(r) && r > 0.0f) {
        s = (float)pow((double)r, (double)a.alpha);
      } else {
        status_or(a.status, QAMW_STATUS_BAD_ACT_RMS);
      }
    }
    a.s_out[j] = s;
  }
}

// ----------------------------------------------------------------------------
// Step (1): r_i = RN32(sqrt(sum_j (w_ij s_j)^2)), fp64 accumulation, one warp
// per row, fixed lane->column mapping and reduction tree (deterministic).
// ----------------------------------------------------------------------------
template <int WT>
__device__ __forceinline__ double load_w(const void *W, int64_t off) {
  if (WT == QAMW_BF16) {
    const uint16_t b = reinterpret_cast<const uint16_t *>(W)[off];
    return bf16_bits_to_double(b);
  } else {
    return (double)reinterpret_cast<const float *>(W)[off];
  }
}

template <int WT>
__global__ void __launch_bounds__(256) row_norm_kernel(RowNormArgs a, int vec_ok) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  constexpr int kEpv = (WT == QAMW_BF16) ? 8 : 4;   // elements per 16-byte load
  for (int64_t row = gw; row < a.M; row += nw) {
    const int64_t base = row * a.ldw;
    double acc = 0.0;
    if (vec_ok) {   // K % kEpv == 0, W rows and s 16-byte aligned
#pragma unroll 4
      for (int64_t j = (int64_t)lane * kEpv; j < a.K; j += 32 * kEpv) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(reinterpret_cast<const unsigned char *>(a.W) +
                                                              (base + j) * (WT == QAMW_BF16 ? 2 : 4)));
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
        if (WT == QAMW_BF16) {
          const float4 s0 = __ldg(reinterpret_cast<const float4 *>(a.s + j));
          const float4 s1 = __ldg(reinterpret_cast<const float4 *>(a.s + j + 4));
          const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const double v0 = bf16_bits_to_double(w4[h] & 0xffffu) * (double)sv[2 * h];
            const double v1 = bf16_bits_to_double(w4[h] >> 16) * (double)sv[2 * h + 1];
            acc = fma(v0, v0, acc);
            acc = fma(v1, v1, acc);
          }
        } else {
          const float4 s0 = __ldg(reinterpret_cast<const float4 *>(a.s + j));
          const float sv[4] = {s0.x, s0.y, s0.z, s0.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const double v = (double)__uint_as_float(w4[h]) * (double)sv[h];
            acc = fma(v, v, acc);
          }
        }
      }
    } else {
      for (int64_t j = lane; j < a.K; j += 32) {
        const double v = load_w<WT>(a.W, base + j) * (double)a.s[j];
        acc = fma(v, v, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float r = (float)sqrt(acc);
      if (!isfinite(r)) status_or(a.status, QAMW_STATUS_NONFINITE_NORM);
      a.r_out[row] = r;
    }
  }
}

// ----------------------------------------------------------------------------
// Step (2): Sylvester Hadamard butterflies over a lane's 32 values plus the
// cross-lane block bits. Element e of lane l is column 32l + e of the unit;
// block bit t pairs columns differing in bit t. Lower partner keeps a+b,
// upper keeps a-b.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void fwht_unit_fp64(double (&v)[32], int log2b, int lane) {
#pragma unroll
  for (int t = 0; t < 5; ++t) {
    if (t < log2b) {
      const int h = 1 << t;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if ((i & h) == 0) {
          const double a0 = v[i], a1 = v[i | h];
          v[i] = a0 + a1;
          v[i | h] = a0 - a1;
        }
      }
    }
  }
#pragma unroll
  for (int t = 5; t < 10; ++t) {
    if (t < log2b) {
      const int h = 1 << (t - 5);
      const bool upper = (lane & h) != 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const double p = __shfl_xor_sync(0xffffffffu, v[i], h);
        v[i] = upper ? (p - v[i]) : (v[i] + p);
      }
    }
  }
}

// Per-warp column tables for one 1024-column chunk.
struct WarpTables {
  float sd[32 * kSdPitch];       // d_j * s_j for the lane's 32 columns (0 past K)
  double inv_sigma[32 * kInvPitch];  // 1/sigma_k for the lane's 16 pairs
  uint16_t idx[512];             // unit indices for packing
};

__device__ __forceinline__ void load_chunk_tables(WarpTables &t, const RotateArgs &a,
                                                  const float *sigma, int64_t chunk, int lane) {
  const int64_t c0 = chunk * kUnitCols;
#pragma unroll 4
  for (int i = 0; i < 32; ++i) {
    const int64_t col = c0 + 32 * i + lane;
    float v = 0.0f;
    if (col < a.K) {
      v = a.s[col];
      if (mask_is_negative(a.seed, col)) v = -v;
    }
    t.sd[i * kSdPitch + lane] = v;
  }
  if (sigma != nullptr) {
    const int64_t p0 = chunk * (kUnitCols / 2);
    const int64_t P = a.K >> 1;
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
      const int pl = 32 * i + lane;
      const int64_t p = p0 + pl;
      t.inv_sigma[(pl >> 4) * kInvPitch + (pl & 15)] = (p < P) ? 1.0 / (double)sigma[p] : 0.0;
    }
  }
  __syncwarp();
}

// Loads the lane's 32 weights of `row`, multiplies by d_j s_j (exact in fp64)
// and applies the forward butterflies. Columns past K read as zero.
template <int WT>
__device__ __forceinline__ void rotate_row_lane(double (&v)[32], const RotateArgs &a,
                                                const float *sd_lane, int64_t row,
                                                int64_t col_lane, bool vec_ok, int lane) {
  const int64_t off = row * a.ldw + col_lane;
  if (col_lane + 32 <= a.K && vec_ok) {
    if (WT == QAMW_BF16) {
      const uint4 *p = reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(a.W) + off);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 u = __ldg(p + q);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          v[8 * q + 2 * h] = bf16_bits_to_double(w4[h] & 0xffffu);
          v[8 * q + 2 * h + 1] = bf16_bits_to_double(w4[h] >> 16);
        }
      }
    } else {
      const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.W) + off);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 f = __ldg(p + q);
        v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = (col_lane + e < a.K) ? load_w<WT>(a.W, off + e) : 0.0;
  }
#pragma unroll
  for (int e = 0; e < 32; ++e) v[e] *= (double)sd_lane[e];
  fwht_unit_fp64(v, a.log2b, lane);
}

// ----------------------------------------------------------------------------
// Step (3): per-row-group partial sums of |z_k| (fp64), then a fixed-order
// reduction: sigma_k = RN32(sqrt(2/pi) * (sum / M)); 0 -> 1.
// ----------------------------------------------------------------------------
template <int WT>
__global__ void __launch_bounds__(kThreads, 1) calibrate_kernel(CalibArgs a, int vec_ok) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WarpTables &tab = reinterpret_cast<WarpTables *>(smem_raw)[warp];
  const RotateArgs &ra = a.rot;
  const int64_t n_chunks = (ra.K + kUnitCols - 1) / kUnitCols;
  const int64_t U = n_chunks * a.groups;
  const int64_t gw = (int64_t)blockIdx.x * kWarps + warp;
  const int64_t GW = (int64_t)gridDim.x * kWarps;
  const int64_t u0 = gw * U / GW, u1 = (gw + 1) * U / GW;
  const double inv_sqrt_b = 1.0 / sqrt((double)(1 << ra.log2b));
  const int64_t P = ra.K >> 1;
  int64_t cur_chunk = -1;
  for (int64_t u = u0; u < u1; ++u) {
    const int64_t chunk = u / a.groups, g = u % a.groups;
    if (chunk != cur_chunk) {
      __syncwarp();
      load_chunk_tables(tab, ra, nullptr, chunk, lane);
      cur_chunk = chunk;
    }
    const int64_t col_lane = chunk * kUnitCols + 32 * lane;
    double acc[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) acc[p] = 0.0;
    const int64_t r0 = g * kCalibRowGroup;
    for (int64_t row = r0; row < r0 + kCalibRowGroup && row < ra.M; ++row) {
      const float r = ra.r[row];
      if (!(r > 0.0f) || !isfinite(r)) continue;  // a zero row adds nothing
      double v[32];
      rotate_row_lane<WT>(v, ra, &tab.sd[lane * kSdPitch], row, col_lane, vec_ok != 0, lane);
      const double q = inv_sqrt_b / (double)r;
#pragma unroll
      for (int p = 0; p < 16; ++p)
        acc[p] += q * sqrt(__dadd_rn(__dmul_rn(v[2 * p], v[2 * p]), __dmul_rn(v[2 * p + 1], v[2 * p + 1])));
    }
    const int64_t pbase = col_lane >> 1;
#pragma unroll
    for (int p = 0; p < 16; ++p)
      if (pbase + p < P) a.partials[g * P + pbase + p] = acc[p];
  }
}

// One CTA per 32 consecutive pair positions; warp w sums row groups
// g = w, w + 32, ... in order, then lane k of warp 0 adds the 32 warp sums in
// order. The order depends only on the shape, never on the device.
constexpr int kReduceWarps = 32;
// With sum_out set, the kernel writes the fp64 sum instead of sigma (the
// row-sharded calibration; see sigma_from_sums_kernel).
__global__ void __launch_bounds__(kReduceWarps * 32) sigma_reduce_kernel(const double *partials, int64_t groups,
                                                                         int64_t P, int64_t M, float *sigma_out,
                                                                         double *sum_out) {
  __shared__ double part[kReduceWarps][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t k = (int64_t)blockIdx.x * 32 + lane;
  double s = 0.0;
  if (k < P)
    for (int64_t g = warp; g < groups; g += kReduceWarps) s += partials[g * P + k];
  part[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && k < P) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w) t += part[w][lane];
    if (sum_out != nullptr) {
      sum_out[k] = t;
    } else {
      const double c = 0.79788456080286535588;  // sqrt(2/pi)
      float sg = (float)(c * (t / (double)M));
      if (sg == 0.0f) sg = 1.0f;
      sigma_out[k] = sg;
    }
  }
}

// sigma_k from the sums of R row shards (rank order); R = 1 gives exactly the
// value sigma_reduce_kernel writes for the whole matrix.
__global__ void sigma_from_sums_kernel(const double *sums, int R, int64_t P, int64_t M, float *sigma_out) {
  const int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (k >= P) return;
  double t = 0.0;
  for (int r = 0; r < R; ++r) t += sums[(int64_t)r * P + k];
  const double c = 0.79788456080286535588;  // sqrt(2/pi)
  float sg = (float)(c * (t / (double)M));
  if (sg == 0.0f) sg = 1.0f;
  sigma_out[k] = sg;
}

// ----------------------------------------------------------------------------
// Step (4): brute-force nearest centroid for 16 pairs per lane.
// The codebook sits in shared memory as (c0, c0, c1, c1) so one broadcast
// 16-byte load feeds the packed fp32x2 distance pipeline for 16 pairs.
// Pass 1 keeps the running minimum (fminf) and the CHUNK-aligned block in
// which each pair's minimum first strictly dropped; pass 2 rescans that block
// for the first index whose distance equals the minimum -- exactly the lowest
// index among the fp32 minimisers.
// ----------------------------------------------------------------------------
template <int CHUNK>
__device__ __forceinline__ void search_brute16(const float4 *__restrict__ cb4, int n_pad,
                                               const float (&x0)[16], const float (&x1)[16],
                                               int (&out)[16]) {
  float2 X0[8], X1[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    X0[g] = make_float2(x0[2 * g], x0[2 * g + 1]);
    X1[g] = make_float2(x1[2 * g], x1[2 * g + 1]);
  }
  float m[16];
  int best[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) { m[i] = INFINITY; best[i] = 0; }
  for (int cb = 0; cb < n_pad; cb += CHUNK) {
    float mp[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) mp[i] = m[i];
#pragma unroll
    for (int c = 0; c < CHUNK; ++c) {
      const float4 cc = cb4[cb + c];
      const float2 C0 = make_float2(cc.x, cc.y), C1 = make_float2(cc.z, cc.w);
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float2 dx = sub2(X0[g], C0);
        const float2 dy = sub2(X1[g], C1);
        const float2 d = fma2(dy, dy, mul2(dx, dx));
        m[2 * g] = fminf(m[2 * g], d.x);
        m[2 * g + 1] = fminf(m[2 * g + 1], d.y);
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) best[i] = (m[i] < mp[i]) ? cb : best[i];
  }
  // Rescan: lane l visits the CHUNK entries of its block starting at offset l
  // (mod CHUNK), so the 32 lanes of a load spread over all banks instead of
  // hitting one (every block starts at a multiple of CHUNK); the smallest
  // matching index is kept, which gives the same answer as an ascending scan.
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int base = best[i];
    int found = 0x7fffffff;
#pragma unroll 4
    for (int j = 0; j < CHUNK; ++j) {
      const int c = base + ((j + lane) & (CHUNK - 1));
      const float4 cc = cb4[c];
      if (dist2_scalar(x0[i], x1[i], cc.x, cc.z) == m[i]) found = min(found, c);
    }
    out[i] = (found == 0x7fffffff) ? base : found;
  }
}

template <int WT, int CHUNK>
__global__ void __launch_bounds__(kThreads, 1) encode_kernel(EncodeArgs a, int vec_ok) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_pad = (a.N + CHUNK - 1) / CHUNK * CHUNK;
  // (c0, c0, c1, c1) per centroid for the packed fp32x2 pipeline
  float4 *cb4 = reinterpret_cast<float4 *>(smem_raw);
  WarpTables &tab = reinterpret_cast<WarpTables *>(smem_raw + (size_t)n_pad * sizeof(float4))[warp];
  for (int c = threadIdx.x; c < n_pad; c += blockDim.x) {
    float c0 = kFarCentroid, c1 = kFarCentroid;
    if (c < a.N) { c0 = a.codebook[2 * c]; c1 = a.codebook[2 * c + 1]; }
    cb4[c] = make_float4(c0, c0, c1, c1);
  }
  __syncthreads();

  const RotateArgs &ra = a.rot;
  const int64_t n_chunks = (ra.K + kUnitCols - 1) / kUnitCols;
  const int64_t U = n_chunks * ra.M;
  const int64_t gw = (int64_t)blockIdx.x * kWarps + warp;
  const int64_t GW = (int64_t)gridDim.x * kWarps;
  const int64_t u0 = gw * U / GW, u1 = (gw + 1) * U / GW;
  const double inv_sqrt_b = 1.0 / sqrt((double)(1 << ra.log2b));
  const int64_t P = ra.K >> 1;
  int64_t cur_chunk = -1;
  for (int64_t u = u0; u < u1; ++u) {
    const int64_t chunk = u / ra.M, row = u % ra.M;
    if (chunk != cur_chunk) {
      __syncwarp();
      load_chunk_tables(tab, ra, a.sigma, chunk, lane);
      cur_chunk = chunk;
    }
    const int64_t col_lane = chunk * kUnitCols + 32 * lane;
    const float r = ra.r[row];
    float x0[16], x1[16];
    uint32_t bad = 0;
    if (r > 0.0f && isfinite(r)) {
      double v[32];
      rotate_row_lane<WT>(v, ra, &tab.sd[lane * kSdPitch], row, col_lane, vec_ok != 0, lane);
      const double q = inv_sqrt_b / (double)r;
      const double *is = &tab.inv_sigma[lane * kInvPitch];
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        const double f = q * is[p];
        x0[p] = (float)(v[2 * p] * f);
        x1[p] = (float)(v[2 * p + 1] * f);
        if (!isfinite(x0[p]) || !isfinite(x1[p])) bad = 1;
      }
    } else {
      if (!(r == 0.0f)) bad = 1;  // NaN / Inf row norm
#pragma unroll
      for (int p = 0; p < 16; ++p) { x0[p] = 0.0f; x1[p] = 0.0f; }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) status_or(a.status, QAMW_STATUS_NONFINITE_INPUT);
    int idx[16];
    search_brute16<CHUNK>(cb4, n_pad, x0, x1, idx);
    // pack: stage the unit's 512 indices, then build the unit's words
    __syncwarp();
#pragma unroll
    for (int p = 0; p < 16; ++p) tab.idx[lane * 16 + p] = (uint16_t)idx[p];
    __syncwarp();
    const int64_t pair0 = chunk * (kUnitCols / 2);
    const int np = (int)((P - pair0) < (kUnitCols / 2) ? (P - pair0) : (kUnitCols / 2));
    const int B = a.bits;
    const int nw = (np * B + 31) >> 5;
    uint32_t *dst = a.packed + row * a.wpr + chunk * (int64_t)(16 * B);
    for (int w = lane; w < nw; w += 32) {
      const int bit0 = w * 32;
      const int k0 = bit0 / B;
      const int k1 = min((bit0 + 31) / B, np - 1);
      uint32_t word = 0;
      for (int k = k0; k <= k1; ++k) {
        const int off = k * B - bit0;
        const uint32_t iv = tab.idx[k];
        word |= (off >= 0) ? (iv << off) : (iv >> (-off));
      }
      dst[w] = word;
    }
  }
}

// Test hook: the rotation alone on fp64 rows (forward or inverse).
__global__ void __launch_bounds__(kThreads) rotate_test_kernel(RotateTestArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_chunks = (a.K + kUnitCols - 1) / kUnitCols;
  const int64_t U = n_chunks * a.M;
  const double inv_sqrt_b = 1.0 / sqrt((double)(1 << a.log2b));
  for (int64_t u = (int64_t)blockIdx.x * kWarps + warp; u < U; u += (int64_t)gridDim.x * kWarps) {
    const int64_t chunk = u / a.M, row = u % a.M;
    const int64_t col_lane = chunk * kUnitCols + 32 * lane;
    double v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int64_t col = col_lane + e;
      double x = (col < a.K) ? a.U[row * a.K + col] : 0.0;
      if (!a.inverse && col < a.K && mask_is_negative(a.seed, col)) x = -x;
      v[e] = x;
    }
    fwht_unit_fp64(v, a.log2b, lane);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int64_t col = col_lane + e;
      if (col < a.K) {
        double y = v[e] * inv_sqrt_b;
        if (a.inverse && mask_is_negative(a.seed, col)) y = -y;
        a.Y[row * a.K + col] = y;
      }
    }
  }
}

template <typename Kern>
cudaError_t set_smem(Kern k, size_t bytes) {
  return set_max_dynamic_smem(reinterpret_cast<const void *>(k), bytes);
}

bool w_vec_ok(const void *W, qamw_dtype wt, int64_t ldw) {
  const size_t es = (wt == QAMW_BF16) ? 2 : 4;
  return (reinterpret_cast<uintptr_t>(W) % 16 == 0) && ((ldw * (int64_t)es) % 16 == 0);
}

}  // namespace

cudaError_t launch_channel_scale(const ScaleArgs &a, cudaStream_t s) {
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>((a.K + threads - 1) / threads, 4096);
  channel_scale_kernel<<<(int)std::max<int64_t>(blocks, 1), threads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_row_norms(const RowNormArgs &a, cudaStream_t s) {
  const int epv = (a.wt == QAMW_BF16) ? 8 : 4;
  const int vec = (w_vec_ok(a.W, a.wt, a.ldw) && a.K % epv == 0 && reinterpret_cast<uintptr_t>(a.s) % 16 == 0) ? 1 : 0;
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>((a.M + 7) / 8, (int64_t)sm_count() * 8);
  if (a.wt == QAMW_BF16)
    row_norm_kernel<QAMW_BF16><<<(int)blocks, threads, 0, s>>>(a, vec);
  else
    row_norm_kernel<QAMW_F32><<<(int)blocks, threads, 0, s>>>(a, vec);
  return cudaGetLastError();
}

cudaError_t launch_calibrate(const CalibArgs &a, cudaStream_t s) {
  cudaError_t e;
  if (a.rot.log2b <= 9) {
    if ((e = launch_calibrate_partials512(a, s)) != cudaSuccess) return e;
  } else {
    const size_t smem = sizeof(WarpTables) * kWarps;
    const int64_t n_chunks = (a.rot.K + kUnitCols - 1) / kUnitCols;
    const int64_t units = n_chunks * a.groups;
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((units + kWarps - 1) / kWarps, sm_count()));
    const int vec = w_vec_ok(a.rot.W, a.rot.wt, a.rot.ldw) ? 1 : 0;
    if (a.rot.wt == QAMW_BF16) {
      if ((e = set_smem(calibrate_kernel<QAMW_BF16>, smem)) != cudaSuccess) return e;
      calibrate_kernel<QAMW_BF16><<<(int)blocks, kThreads, smem, s>>>(a, vec);
    } else {
      if ((e = set_smem(calibrate_kernel<QAMW_F32>, smem)) != cudaSuccess) return e;
      calibrate_kernel<QAMW_F32><<<(int)blocks, kThreads, smem, s>>>(a, vec);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int64_t P = a.rot.K >> 1;
  sigma_reduce_kernel<<<(int)((P + 31) / 32), kReduceWarps * 32, 0, s>>>(a.partials, a.groups, P, a.rot.M,
                                                                          a.sigma_out, a.sum_out);
  return cudaGetLastError();
}

cudaError_t launch_sigma_from_sums(const double *sums, int R, int64_t P, int64_t M, float *sigma_out,
                                   cudaStream_t s) {
  sigma_from_sums_kernel<<<(int)((P + 255) / 256), 256, 0, s>>>(sums, R, P, M, sigma_out);
  return cudaGetLastError();
}

template <int WT, int CHUNK>
static cudaError_t launch_encode_t(const EncodeArgs &a, cudaStream_t s) {
  const int n_pad = (a.N + CHUNK - 1) / CHUNK * CHUNK;
  const size_t smem = (size_t)n_pad * sizeof(float4) + sizeof(WarpTables) * kWarps;
  cudaError_t e = set_smem(encode_kernel<WT, CHUNK>, smem);
  if (e != cudaSuccess) return e;
  const int64_t n_chunks = (a.rot.K + kUnitCols - 1) / kUnitCols;
  const int64_t units = n_chunks * a.rot.M;
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((units + kWarps - 1) / kWarps, sm_count()));
  const int vec = w_vec_ok(a.rot.W, a.rot.wt, a.rot.ldw) ? 1 : 0;
  encode_kernel<WT, CHUNK><<<(int)blocks, kThreads, smem, s>>>(a, vec);
  return cudaGetLastError();
}

template <int WT>
static cudaError_t launch_encode_wt(const EncodeArgs &a, cudaStream_t s) {
  return (a.N >= 512) ? launch_encode_t<WT, 32>(a, s) : launch_encode_t<WT, 8>(a, s);
}

cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t s) {
  if (encode_pruned_applicable(a)) return launch_encode_pruned(a, s);
  return (a.rot.wt == QAMW_BF16) ? launch_encode_wt<QAMW_BF16>(a, s) : launch_encode_wt<QAMW_F32>(a, s);
}

cudaError_t launch_rotate_test(const RotateTestArgs &a, cudaStream_t s) {
  const int64_t n_chunks = (a.K + kUnitCols - 1) / kUnitCols;
  const int64_t units = n_chunks * a.M;
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((units + kWarps - 1) / kWarps, 4096));
  rotate_test_kernel<<<(int)blocks, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace qamw
