// qamw_decode.cu -- QAM-W decode on sm_100a ("QAM-W: Joint 2D Codebook
// Quantization for LLM Weights ...", Methodology (6) Decoding):
//   w_hat_ij = r_i * d_j * (H_b (sigma (.) C[idx]))_j / (sqrt(b) * s_j).
//
// Decode is bound by HBM: it reads bits/16 bytes per weight of packed indices
// and writes 2 (bf16) or 4 (fp32) bytes per weight. The design keeps every
// other byte on chip:
//   * one lane owns one 128-column *segment* of one row: its 64 indices are
//     unpacked from 2*bits registers with constant shifts, looked up in a
//     shared-memory table C'[c] = (c0 + c1, c0 - c1) -- the first butterfly
//     of H_b folded into the table -- and scaled by sigma_k * r_i with one
//     packed fp32x2 multiply per pair;
//   * the remaining butterflies of the segment (block bits 1..6) run in
//     registers on packed fp32x2 adds; blocks wider than 128 (b = 256..1024)
//     span 2..8 lanes of the same row and finish with warp shuffles;
//   * the column factor d_j / (sqrt(b) s_j) comes from a per-warp table;
//   * results are staged in shared memory (rows padded by 16 bytes, so the
//     8 lanes of each 16-byte store phase hit distinct banks) and written
//     back as fully coalesced 16-byte stores, 256 or 512 contiguous bytes
//     per row segment.
// A warp handles a *task* of ROWS = 32/SEGS rows x SEGS segments (SEGS =
// max(1, b/128)); tasks are ordered column-strip major and split evenly over
// a persistent grid of one CTA per SM, so each warp rebuilds its column
// tables only when its strip changes.
#include <algorithm>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"

namespace qamw {
namespace {

constexpr int kSeg = 128;  // columns per lane

// Data-movement choices (complete implementations either way):
//   QAMW_DEC_PREFETCH     1: packed words + row norm of the next task are copied
//                            to shared memory with cp.async while the current
//                            task computes; 0 (default, measured faster): plain
//                            loads at the start of a task.
//   QAMW_DEC_DIRECT_STORE 1: each lane stores its bf16 row segment straight from
//                            registers (16-byte stores); 0: stage in shared
//                            memory and write fully coalesced rows.
#ifndef QAMW_DEC_PREFETCH
#define QAMW_DEC_PREFETCH 0
#endif
#ifndef QAMW_DEC_DIRECT_STORE
#define QAMW_DEC_DIRECT_STORE 0
#endif

template <bool BF16OUT>
struct OutTraits;
template <>
struct OutTraits<true> {
  static constexpr int kWarps = 12;   // 384 threads x 168 registers: one CTA per SM
  static constexpr int kEsize = 2;
};
template <>
struct OutTraits<false> {
  static constexpr int kWarps = 4;
  static constexpr int kEsize = 4;
};

// The C' table is stored R times, entry-major (entry i occupies 8R bytes, copy
// r at byte 8(iR + r)); lane l reads copy l mod R. An 8-byte word at byte A
// sits in bank pair (A/8) mod 16, so lane classes l mod R never share a bank
// pair and the random lookups of a half-warp collide only within a class
// (16/R lanes) instead of across all 16 lanes.
__host__ __device__ inline int table_copies(int N) {
  int r = 16;
  while (r > 1 && (size_t)N * 8 * r > 65536) r >>= 1;
  return r;
}

struct DecodeGeom {
  int copies, log2copies;     // codebook table replication
  int segs, rows, log2rows;   // SEGS, ROWS = 32/SEGS
  int pitch;                  // staging row pitch in bytes
  int warp_bytes;             // per-warp shared memory
  int64_t n_segcols, n_bands, n_tasks;
};

__host__ __device__ inline int geom_warp_bytes(int segs, int esize) {
  const int rows = 32 / segs;
  const int pitch = segs * kSeg * esize + 16;
  return segs * kSeg * 4 /*cf*/ + segs * (kSeg / 2) * 8 /*sigma, duplicated*/ + rows * pitch;
}

// Prefetch slot of one lane: the 2*BITS packed words of its segment, padded to
// an odd number of 8-byte units so that the 32 lanes' 64-bit reads fall in
// distinct bank pairs.
__host__ __device__ constexpr int prefetch_words(int bits) {
  return (bits > 0 && QAMW_DEC_PREFETCH) ? 2 * (bits | 1) : 0;
}
__host__ __device__ constexpr int prefetch_bytes(int bits) {
  return (bits > 0 && QAMW_DEC_PREFETCH) ? 2 * 32 * (prefetch_words(bits) + 1) * 4 : 0;  // 2 stages x 32 lanes x (words + norm)
}

template <int BITS>
__device__ __forceinline__ uint32_t extract_idx(const uint32_t *w, int q) {
  constexpr uint32_t mask = (BITS >= 32) ? 0xffffffffu : ((1u << BITS) - 1u);
  const int o = q * BITS, wi = o >> 5, sh = o & 31;
  if (sh + BITS <= 32) return (w[wi] >> sh) & mask;
  return __funnelshift_r(w[wi], w[wi + 1], sh) & mask;
}

// Byte offset idx * 8 of index q, extracted with the shift folded in.
template <int BITS>
__device__ __forceinline__ uint32_t extract_off8(const uint32_t *w, int q) {
  constexpr uint32_t mask8 = ((1u << BITS) - 1u) << 3;
  const int o = q * BITS, wi = o >> 5, sh = o & 31;
  if (sh + BITS <= 32) {
    if (sh >= 3) return (w[wi] >> (sh - 3)) & mask8;
    return (w[wi] << (3 - sh)) & mask8;
  }
  return __funnelshift_r(w[wi], w[wi + 1], sh - 3) & mask8;   // sh >= 22 here
}

// One butterfly stage on block bit TB (1..6) of the lane's 128 values, on
// packed fp32x2 pairs (elements 2k and 2k+1 share a register pair).
template <int TB>
__device__ __forceinline__ void bfly_stage(float (&v)[kSeg]) {
  constexpr int h = 1 << TB;
#pragma unroll
  for (int i = 0; i < kSeg; i += 2) {
    if ((i & h) == 0) {
      const float2 A = make_float2(v[i], v[i + 1]);
      const float2 B = make_float2(v[i | h], v[(i | h) + 1]);
      const float2 s = add2(A, B), d = sub2(A, B);
      v[i] = s.x; v[i + 1] = s.y;
      v[i | h] = d.x; v[(i | h) + 1] = d.y;
    }
  }
}

// Block bits 1 .. min(LB,7)-1 inside the lane (bit 0 is folded into C').
template <int LB>
__device__ __forceinline__ void inlane_stages(float (&v)[kSeg]) {
  if constexpr (LB > 1) bfly_stage<1>(v);
  if constexpr (LB > 2) bfly_stage<2>(v);
  if constexpr (LB > 3) bfly_stage<3>(v);
  if constexpr (LB > 4) bfly_stage<4>(v);
  if constexpr (LB > 5) bfly_stage<5>(v);
  if constexpr (LB > 6) bfly_stage<6>(v);
}

// Block bit TB >= 7: the partner segment sits in lane ^ (ROWS << (TB-7)).
template <int TB, int ROWS>
__device__ __forceinline__ void xlane_stage(float (&v)[kSeg], int lane) {
  constexpr int h = ROWS << (TB - 7);
  const bool upper = (lane & h) != 0;
#pragma unroll
  for (int i = 0; i < kSeg; ++i) {
    const float p = __shfl_xor_sync(0xffffffffu, v[i], h);
    v[i] = upper ? __fsub_rn(p, v[i]) : __fadd_rn(v[i], p);
  }
}

template <int LB, int ROWS>
__device__ __forceinline__ void xlane_stages(float (&v)[kSeg], int lane) {
  if constexpr (LB > 7) xlane_stage<7, ROWS>(v, lane);
  if constexpr (LB > 8) xlane_stage<8, ROWS>(v, lane);
  if constexpr (LB > 9) xlane_stage<9, ROWS>(v, lane);
}

template <int LB>
struct SegGeom {
  static constexpr int kSegs = (LB > 7) ? (1 << (LB - 7)) : 1;  // segments per block
  static constexpr int kRows = 32 / kSegs;                       // rows per warp task
  static constexpr int kLog2Rows = 5 - ((LB > 7) ? (LB - 7) : 0);
};

// BITS > 0: compile-time width, words held in registers. BITS == 0: any width
// (runtime), indices read through a 64-bit window from global memory.
// LB = log2(block size).
template <int BITS, int LB, bool BF16OUT>
__global__ void __launch_bounds__(OutTraits<BF16OUT>::kWarps * 32, 1)
    decode_kernel(DecodeArgs a, DecodeGeom g, int fast_store, int vec_words) {
  constexpr int kEs = OutTraits<BF16OUT>::kEsize;
  constexpr int SEGS = SegGeom<LB>::kSegs;
  constexpr int ROWS = SegGeom<LB>::kRows;
  constexpr int kPitch = SEGS * kSeg * kEs + 16;
  constexpr int kSegCols = SEGS * kSeg;
  constexpr int kRowBytes = kSegCols * kEs;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float2 *cbp = reinterpret_cast<float2 *>(smem_raw);
  unsigned char *wbase = smem_raw + (size_t)a.N * g.copies * sizeof(float2) + (size_t)warp * g.warp_bytes;
  float *cf = reinterpret_cast<float *>(wbase);
  float2 *sg = reinterpret_cast<float2 *>(cf + kSegCols);   // (sigma_k, sigma_k)
  unsigned char *stage = reinterpret_cast<unsigned char *>(sg + kSegCols / 2);
  constexpr int WS = prefetch_words(BITS);
  uint32_t *wbuf = reinterpret_cast<uint32_t *>(stage + ROWS * kPitch);   // [2][32][WS]
  float *rnbuf = reinterpret_cast<float *>(wbuf + 2 * 32 * WS);            // [2][32]

  for (int c = threadIdx.x; c < a.N; c += blockDim.x) {
    const float c0 = a.codebook[2 * c], c1 = a.codebook[2 * c + 1];
    const float2 e = make_float2(__fadd_rn(c0, c1), __fsub_rn(c0, c1));
    for (int r = 0; r < g.copies; ++r) cbp[c * g.copies + r] = e;
  }
  __syncthreads();
  // this lane's copy of the table: entry i at cbl[i << log2copies]
  const float2 *cbl = cbp + (lane & (g.copies - 1));
  const int lgc = g.log2copies;

  const int bits = (BITS > 0) ? BITS : a.bits;
  const uint32_t imask = (bits >= 32) ? 0xffffffffu : ((1u << bits) - 1u);
  const int rr = lane & (ROWS - 1);
  const int sgi = lane >> SegGeom<LB>::kLog2Rows;
  const int nwarps = blockDim.x >> 5;
  const int64_t gw = (int64_t)blockIdx.x * nwarps + warp;
  const int64_t GW = (int64_t)gridDim.x * nwarps;
  const int64_t t0 = gw * g.n_tasks / GW, t1 = (gw + 1) * g.n_tasks / GW;
  const double inv_sqrt_b = 1.0 / sqrt((double)(1 << LB));
  const int64_t P = a.K >> 1;
  int64_t cur = -1;
  uint32_t bad = 0;
  const bool check_idx = a.N < (1 << bits);   // with N == 2^bits every index is valid

  // Copy task t's packed words and row norm for this lane into stage st.
  auto prefetch = [&](int64_t t, int st) {
    if constexpr (BITS > 0 && QAMW_DEC_PREFETCH) {
      const int64_t sc = t / g.n_bands, bd = t - sc * g.n_bands;
      const int64_t row = bd * ROWS + rr;
      const int64_t c0 = sc * kSegCols + (int64_t)sgi * kSeg;
      if (row < a.M) {
        const uint32_t *src = a.packed + row * a.wpr + (c0 >> 1) * BITS / 32;
        uint32_t *dst = wbuf + (st * 32 + lane) * WS;
        const int vcp = (int)std::min<int64_t>(kSeg, a.K - c0);
        if (vcp == kSeg && vec_words) {
#pragma unroll
          for (int i = 0; i < BITS; ++i) cp_async8(dst + 2 * i, src + 2 * i);
        } else {
          const int nvw = ((vcp >> 1) * BITS + 31) >> 5;
          for (int i = 0; i < nvw; ++i) cp_async4(dst + i, src + i);
        }
        cp_async4(rnbuf + st * 32 + lane, a.row_norm + row);
      }
      cp_async_commit();
    }
  };
  if (t0 < t1) prefetch(t0, 0);

  for (int64_t t = t0; t < t1; ++t) {
    const int64_t segcol = t / g.n_bands, band = t - (t / g.n_bands) * g.n_bands;
    const int64_t colbase = segcol * kSegCols;
    const int st = (int)((t - t0) & 1);
    if constexpr (BITS > 0 && QAMW_DEC_PREFETCH) {
      if (t + 1 < t1) {
        prefetch(t + 1, st ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
    }
    if (segcol != cur) {
      __syncwarp();
      for (int j = lane; j < kSegCols; j += 32) {
        const int64_t col = colbase + j;
        float f = 0.0f;
        if (col < a.K) {
          const double s = (a.col_scale != nullptr) ? (double)a.col_scale[col] : 1.0;
          double v = inv_sqrt_b / s;
          if (mask_is_negative(a.seed, col)) v = -v;
          f = (float)v;
        }
        cf[j] = f;
      }
      for (int p = lane; p < kSegCols / 2; p += 32) {
        const int64_t k = (colbase >> 1) + p;
        const float sk = (k < P) ? a.sigma[k] : 0.0f;
        sg[p] = make_float2(sk, sk);
      }
      __syncwarp();
      cur = segcol;
    }
    const int64_t row = band * ROWS + rr;
    const bool row_ok = row < a.M;
    const int64_t col0 = colbase + (int64_t)sgi * kSeg;
    const int vc = (int)std::min<int64_t>(kSeg, a.K - col0);  // valid columns (>= 1)
    const int vp = vc >> 1;

    float rn = 0.0f;
    if (row_ok) {
      if constexpr (BITS > 0 && QAMW_DEC_PREFETCH) rn = rnbuf[st * 32 + lane];
      else rn = a.row_norm[row];
      if (!isfinite(rn)) bad |= QAMW_STATUS_NONFINITE_NORM;
    }

    float v[kSeg];
    const float2 *sgl = sg + sgi * (kSeg / 2);
    const float2 rn2 = make_float2(rn, rn);
    if constexpr (BITS > 0) {
      constexpr int NW = 2 * BITS;
      uint32_t w[NW + 1];
      const int nvw = (vp * BITS + 31) >> 5;
#if QAMW_DEC_PREFETCH
      const uint32_t *wsrc = wbuf + (st * 32 + lane) * WS;
      if (row_ok && vc == kSeg) {
#pragma unroll
        for (int i = 0; i < NW / 2; ++i) {
          const uint2 u = *reinterpret_cast<const uint2 *>(wsrc + 2 * i);
          w[2 * i] = u.x;
          w[2 * i + 1] = u.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) w[i] = (row_ok && i < nvw) ? wsrc[i] : 0u;
      }
#else
      const uint32_t *gsrc = a.packed + (row_ok ? row : 0) * a.wpr + (col0 >> 1) * BITS / 32;
      if (row_ok && vc == kSeg && vec_words) {
#pragma unroll
        for (int i = 0; i < NW / 2; ++i) {
          const uint2 u = __ldg(reinterpret_cast<const uint2 *>(gsrc) + i);
          w[2 * i] = u.x;
          w[2 * i + 1] = u.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) w[i] = (row_ok && i < nvw) ? __ldg(gsrc + i) : 0u;
      }
#endif
      w[NW] = 0u;
      if (check_idx) {
#pragma unroll
        for (int q = 0; q < kSeg / 2; ++q) {
          uint32_t idx = extract_idx<BITS>(w, q);
          if (idx >= (uint32_t)a.N) { if (row_ok && q < vp) bad |= QAMW_STATUS_BAD_INDEX; idx = 0; }
          const float2 s2 = mul2(sgl[q], rn2);
          const float2 y = mul2(s2, cbl[idx << lgc]);
          v[2 * q] = y.x;
          v[2 * q + 1] = y.y;
        }
      } else {
        const unsigned char *cbb = reinterpret_cast<const unsigned char *>(cbl);
#pragma unroll
        for (int q = 0; q < kSeg / 2; ++q) {
          const uint32_t off = extract_off8<BITS>(w, q) << lgc;
          const float2 s2 = mul2(sgl[q], rn2);
          const float2 y = mul2(s2, *reinterpret_cast<const float2 *>(cbb + off));
          v[2 * q] = y.x;
          v[2 * q + 1] = y.y;
        }
      }
    } else {
      const uint32_t *src = a.packed + (row_ok ? row : 0) * a.wpr;
      const int64_t pbase = col0 >> 1;
#pragma unroll
      for (int q = 0; q < kSeg / 2; ++q) {
        uint32_t idx = 0;
        if (row_ok && q < vp) {
          const int64_t o = (pbase + q) * bits;
          const int64_t wi = o >> 5;
          const int sh = (int)(o & 31);
          const uint32_t lo = __ldg(src + wi);
          const uint32_t hi = (sh + bits > 32) ? __ldg(src + wi + 1) : 0u;
          idx = __funnelshift_r(lo, hi, sh) & imask;
          if (idx >= (uint32_t)a.N) { bad |= QAMW_STATUS_BAD_INDEX; idx = 0; }
        }
        const float2 y = mul2(mul2(sgl[q], rn2), cbl[idx << lgc]);
        v[2 * q] = y.x;
        v[2 * q + 1] = y.y;
      }
    }

    inlane_stages<LB>(v);
    xlane_stages<LB, ROWS>(v, lane);

    // column factor, round to the output type, stage
    const float *cfl = cf + sgi * kSeg;
    unsigned char *srow = stage + rr * kPitch + sgi * (kSeg * kEs);
    const bool full = (colbase + kSegCols <= a.K);
#if QAMW_DEC_DIRECT_STORE
    if constexpr (BF16OUT) {
      if (fast_store && full) {
        unsigned char *gdst = reinterpret_cast<unsigned char *>(a.out) + (row_ok ? row : 0) * a.ldo * kEs + col0 * kEs;
#pragma unroll
        for (int c = 0; c < kSeg; c += 8) {
          const float4 f0 = *reinterpret_cast<const float4 *>(cfl + c);
          const float4 f1 = *reinterpret_cast<const float4 *>(cfl + c + 4);
          const float2 o0 = mul2(make_float2(v[c], v[c + 1]), make_float2(f0.x, f0.y));
          const float2 o1 = mul2(make_float2(v[c + 2], v[c + 3]), make_float2(f0.z, f0.w));
          const float2 o2 = mul2(make_float2(v[c + 4], v[c + 5]), make_float2(f1.x, f1.y));
          const float2 o3 = mul2(make_float2(v[c + 6], v[c + 7]), make_float2(f1.z, f1.w));
          __nv_bfloat162 b0 = __floats2bfloat162_rn(o0.x, o0.y);
          __nv_bfloat162 b1 = __floats2bfloat162_rn(o1.x, o1.y);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(o2.x, o2.y);
          __nv_bfloat162 b3 = __floats2bfloat162_rn(o3.x, o3.y);
          uint4 pk;
          pk.x = *reinterpret_cast<uint32_t *>(&b0);
          pk.y = *reinterpret_cast<uint32_t *>(&b1);
          pk.z = *reinterpret_cast<uint32_t *>(&b2);
          pk.w = *reinterpret_cast<uint32_t *>(&b3);
          if (row_ok) *reinterpret_cast<uint4 *>(gdst + c * 2) = pk;
        }
        continue;
      }
    }
#endif
#pragma unroll
    for (int c = 0; c < kSeg; c += 8) {
      const float4 f0 = *reinterpret_cast<const float4 *>(cfl + c);
      const float4 f1 = *reinterpret_cast<const float4 *>(cfl + c + 4);
      const float2 o0 = mul2(make_float2(v[c], v[c + 1]), make_float2(f0.x, f0.y));
      const float2 o1 = mul2(make_float2(v[c + 2], v[c + 3]), make_float2(f0.z, f0.w));
      const float2 o2 = mul2(make_float2(v[c + 4], v[c + 5]), make_float2(f1.x, f1.y));
      const float2 o3 = mul2(make_float2(v[c + 6], v[c + 7]), make_float2(f1.z, f1.w));
      if constexpr (BF16OUT) {
        uint4 pk;
        __nv_bfloat162 b0 = __floats2bfloat162_rn(o0.x, o0.y);
        __nv_bfloat162 b1 = __floats2bfloat162_rn(o1.x, o1.y);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(o2.x, o2.y);
        __nv_bfloat162 b3 = __floats2bfloat162_rn(o3.x, o3.y);
        pk.x = *reinterpret_cast<uint32_t *>(&b0);
        pk.y = *reinterpret_cast<uint32_t *>(&b1);
        pk.z = *reinterpret_cast<uint32_t *>(&b2);
        pk.w = *reinterpret_cast<uint32_t *>(&b3);
        *reinterpret_cast<uint4 *>(srow + c * 2) = pk;
      } else {
        *reinterpret_cast<float4 *>(srow + c * 4) = make_float4(o0.x, o0.y, o1.x, o1.y);
        *reinterpret_cast<float4 *>(srow + c * 4 + 16) = make_float4(o2.x, o2.y, o3.x, o3.y);
      }
    }
    __syncwarp();
    // write back
    const int64_t row0 = band * ROWS;
    const int64_t ldo_bytes = a.ldo * kEs;
    unsigned char *obase = reinterpret_cast<unsigned char *>(a.out) + colbase * kEs;
    if (fast_store && full) {
      constexpr int cpr = kRowBytes >> 4;
#pragma unroll 4
      for (int f = lane; f < ROWS * cpr; f += 32) {
        const int r = f / cpr, c = f - r * cpr;
        if (row0 + r < a.M)
          *reinterpret_cast<uint4 *>(obase + (row0 + r) * ldo_bytes + c * 16) =
              *reinterpret_cast<const uint4 *>(stage + r * kPitch + c * 16);
      }
    } else {
      const int vcols = (int)std::min<int64_t>(kSegCols, a.K - colbase);
      const int total = ROWS * vcols;
      for (int f = lane; f < total; f += 32) {
        const int r = f / vcols, j = f - r * vcols;
        if (row0 + r < a.M) {
          if constexpr (BF16OUT)
            *reinterpret_cast<uint16_t *>(obase + (row0 + r) * ldo_bytes + j * 2) =
                *reinterpret_cast<const uint16_t *>(stage + r * kPitch + j * 2);
          else
            *reinterpret_cast<float *>(obase + (row0 + r) * ldo_bytes + j * 4) =
                *reinterpret_cast<const float *>(stage + r * kPitch + j * 4);
        }
      }
    }
    __syncwarp();
  }
  bad = __reduce_or_sync(0xffffffffu, bad);
  if (lane == 0) status_or(a.status, bad);
}

template <int BITS, int LB, bool BF16OUT>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s) {
  constexpr int kWarps = OutTraits<BF16OUT>::kWarps;
  constexpr int kEs = OutTraits<BF16OUT>::kEsize;
  DecodeGeom g;
  g.copies = table_copies(a.N);
  g.log2copies = 0;
  while ((1 << g.log2copies) < g.copies) ++g.log2copies;
  g.segs = SegGeom<LB>::kSegs;
  g.rows = SegGeom<LB>::kRows;
  g.log2rows = SegGeom<LB>::kLog2Rows;
  g.pitch = g.segs * kSeg * kEs + 16;
  g.warp_bytes = geom_warp_bytes(g.segs, kEs) + prefetch_bytes(BITS);
  g.n_segcols = (a.K + g.segs * kSeg - 1) / (g.segs * kSeg);
  g.n_bands = (a.M + g.rows - 1) / g.rows;
  g.n_tasks = g.n_segcols * g.n_bands;
  // Warps per CTA: kWarps unless the codebook table plus per-warp buffers
  // would exceed the shared memory a CTA may use.
  const size_t cb_bytes = (size_t)a.N * g.copies * sizeof(float2);
  int dev = 0, smem_max = 0;
  cudaGetDevice(&dev);
  cudaError_t e = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  int warps = kWarps;
  while (warps > 1 && cb_bytes + (size_t)warps * g.warp_bytes > (size_t)smem_max) --warps;
  const size_t smem = cb_bytes + (size_t)warps * g.warp_bytes;
  if (smem > (size_t)smem_max) return cudaErrorInvalidConfiguration;
  e = set_max_dynamic_smem(reinterpret_cast<const void *>(decode_kernel<BITS, LB, BF16OUT>), smem);
  if (e != cudaSuccess) return e;
  const int fast_store = (reinterpret_cast<uintptr_t>(a.out) % 16 == 0) && ((a.ldo * kEs) % 16 == 0);
  const int vec_words = (reinterpret_cast<uintptr_t>(a.packed) % 8 == 0) && (a.wpr % 2 == 0);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((g.n_tasks + warps - 1) / warps, sm_count()));
  decode_kernel<BITS, LB, BF16OUT><<<(int)blocks, warps * 32, smem, s>>>(a, g, fast_store, vec_words);
  return cudaGetLastError();
}

template <int LB, bool BF16OUT>
cudaError_t launch_lb(const DecodeArgs &a, cudaStream_t s) {
  if constexpr (LB >= 6 && LB <= 8) {
    switch (a.bits) {
      case 7: return launch_t<7, LB, BF16OUT>(a, s);
      case 8: return launch_t<8, LB, BF16OUT>(a, s);
      case 10: return launch_t<10, LB, BF16OUT>(a, s);
      case 11: return launch_t<11, LB, BF16OUT>(a, s);
      default: break;
    }
  }
  return launch_t<0, LB, BF16OUT>(a, s);
}

template <bool BF16OUT>
cudaError_t launch_out(const DecodeArgs &a, cudaStream_t s) {
  switch (a.log2b) {
    case 1: return launch_lb<1, BF16OUT>(a, s);
    case 2: return launch_lb<2, BF16OUT>(a, s);
    case 3: return launch_lb<3, BF16OUT>(a, s);
    case 4: return launch_lb<4, BF16OUT>(a, s);
    case 5: return launch_lb<5, BF16OUT>(a, s);
    case 6: return launch_lb<6, BF16OUT>(a, s);
    case 7: return launch_lb<7, BF16OUT>(a, s);
    case 8: return launch_lb<8, BF16OUT>(a, s);
    case 9: return launch_lb<9, BF16OUT>(a, s);
    default: return launch_lb<10, BF16OUT>(a, s);
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
#ifndef QAMW_DEC_NO_TMA
  if (decode_tma_applicable(a)) {
    const cudaError_t e = launch_decode_tma(a, s);
    if (e != cudaErrorNotSupported) return e;
  }
#endif
  return (a.out_t == QAMW_BF16) ? launch_out<true>(a, s) : launch_out<false>(a, s);
}

}  // namespace qamw
