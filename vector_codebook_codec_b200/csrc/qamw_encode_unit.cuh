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
// one warp with the rotation of qamw_rotate16.cuh (the same x, bit for bit,
// as the 1024-column kernel of qamw_encode.cu). A CTA of kEncWarps warps takes
// a contiguous range of *tiles* (one row per warp x one 512-column chunk) in
// chunk-major order; the chunk's d_j * s_j and 1 / sigma_k live once per CTA
// in shared memory. The next unit's weights are loaded while the current one
// is quantized. After the rotation lane l' holds the unit's pairs
// 64 (l' >> 3) + 8 m + (l' & 7), m = 0..7; the search policy S maps them to 8
// indices: S.search8(x0, x1, idx). The indices are staged in the warp's
// transpose buffer and packed into whole words of the stream.
#pragma once

#include <cfloat>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"
#include "qamw_rotate16.cuh"

namespace qamw {

#ifndef QAMW_ENC_WARPS
#define QAMW_ENC_WARPS 16
#endif
constexpr int kEncWarps = QAMW_ENC_WARPS;   // warps per CTA (one tile row each)
constexpr int kEncThreads = kEncWarps * 32;

struct ChunkTables {
  double sd[32 * kSdPitch];         // d_j * s_j of the lane's 16 columns, load layout (0 past K)
  double inv_sigma[32 * kIsPitch];  // 1 / sigma_k of the lane's 8 pairs, pair layout (0 past K/2)
};
// shared memory the pipeline uses at the start of the dynamic area
constexpr size_t kUnitSmemBytes = sizeof(ChunkTables) + (size_t)kEncWarps * kXbufHalf * sizeof(double);

// Packs the unit's np staged indices (stage[k] = index of unit pair k, 0
// for k >= np) into its words dst[0 .. ceil(np B / 32)). BB > 0 fixes the
// code size B at compile time (constant divisions and shifts, no inner loop).
template <int BB>
__device__ __forceinline__ void pack_unit(const uint16_t *stage, uint32_t *dst, int np, int B, uint64_t divB,
                                          int lane) {
  const int nw = (np * B + 31) >> 5;
  if (BB > 0) {
    constexpr int kB = BB > 0 ? BB : 1;
    constexpr int kMore = (32 + kB - 1) / kB;   // indices after the first that can start inside a word
    for (int w = lane; w < nw; w += 32) {
      const int bit0 = w * 32;
      const int k0 = bit0 / kB;
      const int off0 = k0 * kB - bit0;          // in (-B, 0]
      uint32_t word = (uint32_t)stage[k0] >> (-off0);
#pragma unroll
      for (int i = 1; i <= kMore; ++i) {
        const int off = off0 + i * kB;          // > 0
        if (off < 32) word |= (uint32_t)stage[k0 + i] << off;
      }
      dst[w] = word;
    }
  } else {
    for (int w = lane; w < nw; w += 32) {
      const int bit0 = w * 32;
      const int k0 = (int)(((uint64_t)bit0 * divB) >> 32);               // bit0 / B
      const int k1 = min((int)(((uint64_t)(bit0 + 31) * divB) >> 32), np - 1);
      uint32_t word = 0;
#pragma unroll 1   // 2 to 4 indices per word
      for (int k = k0; k <= k1; ++k) {
        const int off = k * B - bit0;
        const uint32_t iv = stage[k];
        word |= (off >= 0) ? (iv << off) : (iv >> (-off));
      }
      dst[w] = word;
    }
  }
}

// LB > 0 fixes log2 b, BB > 0 the code size, at compile time (0: read at run time).
template <int WT, int LB, int BB, class Search>
__device__ __forceinline__ void encode_units(const EncodeArgs &a, int vec_ok, unsigned char *smem,
                                             const Search &S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const RotateArgs &ra = a.rot;
  ChunkTables &ct = *reinterpret_cast<ChunkTables *>(smem);
  double *xbuf = reinterpret_cast<double *>(smem + sizeof(ChunkTables)) + warp * kXbufHalf;
  uint16_t *stage = reinterpret_cast<uint16_t *>(xbuf);
  const int64_t M = ra.M, K = ra.K, P = K >> 1;
  const int64_t n_chunks = (K + kUnit - 1) / kUnit;
  const int64_t RG = (M + kEncWarps - 1) / kEncWarps;
  const int64_t T = n_chunks * RG;
  const int64_t t0 = (int64_t)blockIdx.x * T / gridDim.x, t1 = ((int64_t)blockIdx.x + 1) * T / gridDim.x;
  const double inv_sqrt_b = 1.0 / sqrt((double)(1 << ra.log2b));
  const int B = a.bits;
  // floor(n / B) = (n * divB) >> 32 exactly for 0 <= n < 2^14 and 1 <= B <= 16
  // (checked exhaustively); the packing needs n < 256 * 16 + 32
  const uint64_t divB = (0x100000000ull / (uint64_t)B) + 1ull;

  // the next unit's weights and row norm, loaded while the current one is searched
  auto prefetch = [&](int64_t chunk, int64_t g, WRegs<WT> &w, float &rn) -> bool {
    const int64_t row = g * kEncWarps + warp;
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
        const int k = threadIdx.x;
        const int64_t p = chunk * (kUnit / 2) + k;
        const double is = (p < P) ? 1.0 / (double)a.sigma[p] : 0.0;
        ct.inv_sigma[pair_slot(k)] = is;
        if (!(fabs(is) <= 0.5 * (double)FLT_MAX)) status_or(a.status, QAMW_STATUS_NONFINITE_INPUT);
      }
      __syncthreads();
      cur_chunk = chunk;
    }
    const WRegs<WT> wc = wn;
    const bool full = full_next;
    const float r = rn_next;
    if (t + 1 < t1) full_next = prefetch(next_chunk, next_g, wn, rn_next);

    const int64_t row = g * kEncWarps + warp;
    if (row >= M) continue;
    const int64_t col = chunk * kUnit + 16 * lane;

    float x0[8], x1[8];
    const bool ok = r > 0.0f && isfinite(r);   // uniform across the warp (one row)
    if (ok) {
      double u[16];
      rotate_unit16<WT, true, LB>(u, wc, full, ra.W, ra.ldw, K, row, col, &ct.sd[lane * kSdPitch], ra.log2b,
                                  xbuf, lane);
      const double qn = inv_sqrt_b / (double)r;
      const double2 *is2 = reinterpret_cast<const double2 *>(&ct.inv_sigma[lane * kIsPitch]);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const double2 is = is2[h];
        const double f0 = qn * is.x, f1 = qn * is.y;
        x0[2 * h] = (float)(u[4 * h] * f0);
        x1[2 * h] = (float)(u[4 * h + 1] * f0);
        x0[2 * h + 1] = (float)(u[4 * h + 2] * f1);
        x1[2 * h + 1] = (float)(u[4 * h + 3] * f1);
      }
    } else {
      // NaN / Inf row norm: status; a zero row codes every pair as x = 0
      if (!(r == 0.0f) && lane == 0) status_or(a.status, QAMW_STATUS_NONFINITE_INPUT);
#pragma unroll
      for (int p = 0; p < 8; ++p) { x0[p] = 0.0f; x1[p] = 0.0f; }
    }

    int idx[8];
    S.search8(x0, x1, idx);

    // pack: stage the unit's 256 indices (in pair order; 0 past the last pair),
    // then build the unit's words
    const int64_t pair0 = chunk * (kUnit / 2);
    const int np = (int)((P - pair0) < (kUnit / 2) ? (P - pair0) : (kUnit / 2));
    __syncwarp();   // the transpose buffer is free again
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int k = unit_pair(lane, m);
      stage[k] = (uint16_t)(k < np ? idx[m] : 0);
    }
    __syncwarp();
    pack_unit<BB>(stage, a.packed + row * a.wpr + chunk * (int64_t)(8 * B), np, B, divB, lane);
    __syncwarp();   // the stage is read before the next unit's transpose overwrites it
  }
}

}  // namespace qamw
