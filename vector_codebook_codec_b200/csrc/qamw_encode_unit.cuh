// qamw_encode_unit.cuh -- the 512-column encode pipeline shared by the
// pruned-search encode (qamw_encode_pruned.cu) and the polar baseline encode
// (qamw_encode_polar.cu), for Hadamard blocks b <= 512.
//
// Method: "QAM-W: Joint 2D Codebook Quantization for LLM Weights via Hadamard
// Rotation and Activation-Aware Scaling", Technical Summary, "Methodology:
// The QAM-W Codec": normalise by the stored row norm (step 1), sign-masked
// block Hadamard rotation (step 2), x = z / sigma (step 3), quantization of
// each pair (step 4; the search policy) with the channel scale s_j applied
// first (step 5), then bit packing.
//
// Work decomposition. A *unit* is one row x 512 consecutive columns handled by
// one warp: lane l owns columns [16l, 16l + 16) of the unit (8 pairs); the
// rotation is the fp64 one of qamw_rotate16.cuh, which gives the same x bit
// for bit as the 1024-column kernel of qamw_encode.cu. A CTA of 28 warps takes
// a contiguous range of *tiles* (one row per warp x one 512-column chunk) in
// chunk-major order; the chunk's d_j * s_j and 1 / sigma_k live once per CTA in
// shared memory. The next unit's weights are loaded while the current one is
// quantized. The search policy S maps the 8 pairs (x0[p], x1[p]) of a lane to
// 8 indices: S.search8(x0, x1, idx).
#pragma once

#include <cfloat>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"
#include "qamw_rotate16.cuh"

namespace qamw {

constexpr int kUnitWarps = 28;  // warps per CTA = rows per tile; 4096^2 encode: 16 warps 146 us, 20 137, 24 132, 28 126
constexpr int kUnitThreads = kUnitWarps * 32;

struct ChunkTables {
  double sd[32 * kSdPitch];         // d_j * s_j of the lane's 16 columns (0 past K)
  double inv_sigma[32 * kIsPitch];  // 1 / sigma_k of the lane's 8 pairs (0 past K/2)
};
constexpr int kStageBytes = 512;    // per warp: 256 uint16 indices of the unit
// shared memory the pipeline uses at the start of the dynamic area
constexpr size_t kUnitSmemBytes = sizeof(ChunkTables) + (size_t)kUnitWarps * kStageBytes;

template <int WT, class Search>
__device__ __forceinline__ void encode_units(const EncodeArgs &a, int vec_ok, unsigned char *smem,
                                             const Search &S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const RotateArgs &ra = a.rot;
  ChunkTables &ct = *reinterpret_cast<ChunkTables *>(smem);
  uint16_t *stage = reinterpret_cast<uint16_t *>(smem + sizeof(ChunkTables) + warp * kStageBytes);
  const int64_t M = ra.M, K = ra.K, P = K >> 1;
  const int64_t n_chunks = (K + kUnit - 1) / kUnit;
  const int64_t RG = (M + kUnitWarps - 1) / kUnitWarps;
  const int64_t T = n_chunks * RG;
  const int64_t t0 = (int64_t)blockIdx.x * T / gridDim.x, t1 = ((int64_t)blockIdx.x + 1) * T / gridDim.x;
  const double inv_sqrt_b = 1.0 / sqrt((double)(1 << ra.log2b));
  const int B = a.bits;
  // floor(n / B) = (n * divB) >> 32 exactly for 0 <= n < 2^14 and 1 <= B <= 16
  // (checked exhaustively); the packing needs n < 256 * 16 + 32
  const uint64_t divB = (0x100000000ull / (uint64_t)B) + 1ull;

  // the next unit's weights and row norm, loaded while the current one is searched
  auto prefetch = [&](int64_t chunk, int64_t g, WRegs<WT> &w, float &rn) -> bool {
    const int64_t row = g * kUnitWarps + warp;
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
  for (int64_t t = t0; t < t1; ++t, chunk = next_chunk, g = next_g) {
    next_g = g + 1;
    next_chunk = chunk;
    if (next_g == RG) { next_g = 0; ++next_chunk; }
    if (chunk != cur_chunk) {
      __syncthreads();   // every warp is done with the previous chunk's tables (and the table copy is complete)
      if (threadIdx.x < kUnit) load_sd512(ct.sd, ra.s, ra.seed, K, chunk, threadIdx.x);
      if (threadIdx.x < kUnit / 2) {
        // a rotated unit row has |y_j| <= 1 (to within the fp32 rounding of r),
        // so |x| <= 1 / sigma_k: every x of the column is a finite fp32 when
        // 1 / sigma_k is at most half the fp32 range (else the status says so)
        const int i = threadIdx.x;
        const int64_t p = chunk * (kUnit / 2) + i;
        const double is = (p < P) ? 1.0 / (double)a.sigma[p] : 0.0;
        ct.inv_sigma[(i >> 3) * kIsPitch + (i & 7)] = is;
        if (!(fabs(is) <= 0.5 * (double)FLT_MAX)) status_or(a.status, QAMW_STATUS_NONFINITE_INPUT);
      }
      __syncthreads();
      cur_chunk = chunk;
    }
    const WRegs<WT> wc = wn;
    const bool full = full_next;
    const float r = rn_next;
    if (t + 1 < t1) full_next = prefetch(next_chunk, next_g, wn, rn_next);

    const int64_t row = g * kUnitWarps + warp;
    if (row >= M) continue;
    const int64_t col = chunk * kUnit + 16 * lane;

    float x0[8], x1[8];
    uint32_t bad = 0;
    if (r > 0.0f && isfinite(r)) {
      double v[16];
      scaled16<WT>(v, wc, full, ra.W, ra.ldw, K, row, col, &ct.sd[lane * kSdPitch]);
      fwht16_fp64(v, ra.log2b, lane);
      const double qn = inv_sqrt_b / (double)r;
      const double2 *is2 = reinterpret_cast<const double2 *>(&ct.inv_sigma[lane * kIsPitch]);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const double2 is = is2[h];
        const double f0 = qn * is.x, f1 = qn * is.y;
        x0[2 * h] = (float)(v[4 * h] * f0);
        x1[2 * h] = (float)(v[4 * h + 1] * f0);
        x0[2 * h + 1] = (float)(v[4 * h + 2] * f1);
        x1[2 * h + 1] = (float)(v[4 * h + 3] * f1);
      }
    } else {
      if (!(r == 0.0f)) bad = 1;   // NaN / Inf row norm; a zero row codes every pair as x = 0
#pragma unroll
      for (int p = 0; p < 8; ++p) { x0[p] = 0.0f; x1[p] = 0.0f; }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) status_or(a.status, QAMW_STATUS_NONFINITE_INPUT);

    int idx[8];
    S.search8(x0, x1, idx);

    // pack: stage the unit's 256 indices, then build the unit's words
    __syncwarp();
    reinterpret_cast<uint4 *>(stage)[lane] =
        make_uint4((uint32_t)idx[0] | ((uint32_t)idx[1] << 16), (uint32_t)idx[2] | ((uint32_t)idx[3] << 16),
                   (uint32_t)idx[4] | ((uint32_t)idx[5] << 16), (uint32_t)idx[6] | ((uint32_t)idx[7] << 16));
    __syncwarp();
    const int64_t pair0 = chunk * (kUnit / 2);
    const int np = (int)((P - pair0) < (kUnit / 2) ? (P - pair0) : (kUnit / 2));
    const int nw = (np * B + 31) >> 5;
    uint32_t *dst = a.packed + row * a.wpr + chunk * (int64_t)(8 * B);
    for (int w = lane; w < nw; w += 32) {
      const int bit0 = w * 32;
      const int k0 = (int)(((uint64_t)bit0 * divB) >> 32);               // bit0 / B
      const int k1 = min((int)(((uint64_t)(bit0 + 31) * divB) >> 32), np - 1);
      uint32_t word = 0;
#pragma unroll 1   // 2 to 4 indices per word: unrolling measured slower
      for (int k = k0; k <= k1; ++k) {
        const int off = k * B - bit0;
        const uint32_t iv = stage[k];
        word |= (off >= 0) ? (iv << off) : (iv >> (-off));
      }
      dst[w] = word;
    }
  }
}

}  // namespace qamw
