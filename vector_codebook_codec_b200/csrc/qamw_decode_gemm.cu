// qamw_decode_gemm.cu -- QAM-W decode fused with the matrix multiply that
// consumes the weights, on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "QAM-W: Joint 2D Codebook Quantization for LLM Weights ...", Methodology (6)
// Decoding, and "Significance and Claims": the decoded weights are rounded to
// BF16 and fed to the matrix multiply; the bit savings reach latency only
// with a fused kernel. Here
//   Y[t][m] = sum_k X[t][k] * W_bf16[m][k],   W_bf16 = RN_bf16(w_hat),
//   w_hat[m][j] = r_m * d_j * (H_b (sigma (.) C[idx]))_j / (sqrt(b) s_j),
// with the weights never leaving the chip: each CTA owns 128 output rows
// (features) and one tile of NT tokens, and walks K in chunks of 128 columns.
// For every chunk its 8 warps unpack the chunk's indices, look up and rescale
// the centroids, apply the inverse Hadamard butterflies in fp32 (block bits
// 0..4 in registers, 5..6 across the 4 lanes of a row), scale by r_m d_j /
// (sqrt(b) s_j) and write the bf16 tile into shared memory in the 128-byte
// swizzled K-major layout of the tensor cores; one TMA tensor copy (no
// multicast) brings the matching X tile in the same layout. One thread then
// issues the chunk's eight 128 x NT x 16 tcgen05.mma (bf16 in, fp32
// accumulated in tensor memory) and commits them to an mbarrier; the next
// chunk is decoded into the other stage meanwhile. At the end the accumulator
// is read from tensor memory (tcgen05.ld) and written as fp32 Y.
//
// Every wait (TMA arrival, MMA completion) is a bounded mbarrier wait; a wait
// that runs out sets QAMW_STATUS_TIMEOUT and the CTA stops, frees its tensor
// memory and returns.
#include <algorithm>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"
#include "qamw_mbarrier.cuh"
#include "qamw_tensor_map.h"

namespace qamw {
namespace {

constexpr int kBM = 128;              // output rows per CTA (tensor-memory lanes)
constexpr int kBK = 128;              // columns per chunk (whole Hadamard blocks, b <= 128)
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kAtomBytesA = kBM * 128;                // one 64-column swizzle atom of the weight tile
constexpr int kStageBytesA = 2 * kAtomBytesA;         // 128 columns = 2 atoms
constexpr uint32_t kWaitLimit = 1u << 22;             // mbarrier try_wait attempts

struct GemmArgs {
  DecodeArgs d;          // packed, row_norm, sigma, col_scale, M, K, log2b, seed, codebook, N, bits, wpr, status
  int64_t T;             // tokens
  int NT;                // tokens per CTA tile (16..256, multiple of 16)
  float *Y;              // [T][ldy] fp32
  int64_t ldy;
};

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  // start address >> 4 | leading offset 16 B (ignored for swizzled K-major) |
  // stride offset 1024 B (8 rows of 128 B) | descriptor version 1 | 128-byte swizzle
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Index of pair kk of a row (LSB-first stream of B-bit fields).
__device__ __forceinline__ uint32_t unpack_index(const uint32_t *row, int64_t kk, int B) {
  const int64_t bit = kk * B;
  const int64_t w = bit >> 5;
  const int off = (int)(bit & 31);
  uint64_t v = row[w];
  if (off + B > 32) v |= (uint64_t)row[w + 1] << 32;
  return (uint32_t)(v >> off) & ((1u << B) - 1u);
}

__global__ void __launch_bounds__(kThreads, 1) decode_gemm_kernel(const __grid_constant__ CUtensorMap xmap, GemmArgs g) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // 1024-byte alignment for the swizzled operand tiles
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const DecodeArgs &a = g.d;
  const int NT = g.NT;
  const int stage_b = NT * 256;                 // 2 atoms of NT rows x 128 B
  unsigned char *A0 = smem;                     // [2][kStageBytesA]
  unsigned char *B0 = smem + 2 * kStageBytesA;  // [2][stage_b]
  float2 *cb = reinterpret_cast<float2 *>(B0 + 2 * stage_b);
  float *fac = reinterpret_cast<float *>(cb + a.N);   // [kBK] d_j / (sqrt(b) s_j) of the chunk

  __shared__ __align__(8) uint64_t bar_x[2], bar_mma[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.x * kBM;
  const int64_t t0 = (int64_t)blockIdx.y * NT;
  const int64_t n_chunks = a.K / kBK;
  const int B = a.bits;
  const int log2b = a.log2b;
  const double inv_sqrt_b = 1.0 / sqrt((double)(1 << log2b));
  const uint32_t tmem_cols = NT <= 32 ? 32 : (NT <= 64 ? 64 : (NT <= 128 ? 128 : 256));

  for (int i = threadIdx.x; i < a.N; i += kThreads) cb[i] = make_float2(a.codebook[2 * i], a.codebook[2 * i + 1]);
  if (threadIdx.x == 0) {
    mbar_init(&bar_x[0], 1);
    mbar_init(&bar_x[1], 1);
    mbar_init(&bar_mma[0], 1);
    mbar_init(&bar_mma[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_fail = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  // instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, N = NT, M = 128
  const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

  // the two rows a thread decodes per chunk: rows 16 w + 8 i + (lane / 4), quarter q = lane % 4
  const int q = lane & 3;
  uint32_t bad = 0;
  float rn[2];
  bool rin[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int64_t m = m0 + 16 * warp + 8 * i + (lane >> 2);
    rin[i] = m < a.M;
    rn[i] = rin[i] ? a.row_norm[m] : 0.0f;
    if (rin[i] && !isfinite(rn[i])) bad |= QAMW_STATUS_NONFINITE_NORM;
  }

  bool failed = false;
  for (int64_t c = 0; c < n_chunks && !failed; ++c) {
    const int s = (int)(c & 1);
    unsigned char *As = A0 + s * kStageBytesA;
    unsigned char *Bs = B0 + s * stage_b;
    if (c >= 2) {   // stage s was read by the MMAs of chunk c - 2
      if (!mbar_wait(&bar_mma[s], (uint32_t)(((c - 2) >> 1) & 1), kWaitLimit)) bad |= QAMW_STATUS_TIMEOUT;
    }
    if (__syncthreads_or(bad & QAMW_STATUS_TIMEOUT)) { failed = true; break; }
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(&bar_x[s], (uint32_t)stage_b);
      tma_load_2d(Bs, &xmap, (int)(c * kBK), (int)t0, &bar_x[s]);
      tma_load_2d(Bs + NT * 128, &xmap, (int)(c * kBK + 64), (int)t0, &bar_x[s]);
    }
    // the chunk's column factors d_j / (sqrt(b) s_j)
    if (threadIdx.x < kBK) {
      const int64_t j = c * kBK + threadIdx.x;
      double f = inv_sqrt_b / (a.col_scale != nullptr ? (double)a.col_scale[j] : 1.0);
      if (mask_is_negative(a.seed, j)) f = -f;
      fac[threadIdx.x] = (float)f;
    }
    __syncthreads();
#pragma unroll 1
    for (int i = 0; i < 2; ++i) {
      const int rl = 16 * warp + 8 * i + (lane >> 2);
      const int64_t m = m0 + rl;
      float v[32];
      if (rin[i]) {
        const uint32_t *prow = a.packed + m * a.wpr;
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const int64_t kk = c * (kBK / 2) + 16 * q + p;
          uint32_t idx = unpack_index(prow, kk, B);
          if (idx >= (uint32_t)a.N) { bad |= QAMW_STATUS_BAD_INDEX; idx = 0; }
          const float2 cc = cb[idx];
          const float sg = a.sigma[kk];
          v[2 * p] = cc.x * sg;
          v[2 * p + 1] = cc.y * sg;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.0f;
      }
      // inverse Hadamard butterflies: block bits 0..4 in registers, 5..6 across lanes
#pragma unroll
      for (int t = 0; t < 5; ++t) {
        if (t < log2b) {
          const int h = 1 << t;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if ((e & h) == 0) {
              const float x0 = v[e], x1 = v[e | h];
              v[e] = x0 + x1;
              v[e | h] = x0 - x1;
            }
          }
        }
      }
#pragma unroll
      for (int t = 5; t < 7; ++t) {
        if (t < log2b) {
          const int hb = 1 << (t - 5);
          const float sgn = (lane & hb) ? -1.0f : 1.0f;
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __fmaf_rn(sgn, v[e], __shfl_xor_sync(0xffffffffu, v[e], hb));
        }
      }
      // scale, round to bf16 and store into the swizzled K-major tile:
      // row rl, columns 32 q .. 32 q + 31 = atom q / 2, 16-byte chunks 4 (q % 2) .. + 3
      const float r = rn[i];
      unsigned char *arow = As + (q >> 1) * kAtomBytesA + rl * 128;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t pk[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int e = 8 * ch + 2 * h;
          const float w0 = (v[e] * r) * fac[32 * q + e];
          const float w1 = (v[e + 1] * r) * fac[32 * q + e + 1];
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(w0, w1);
          pk[h] = *reinterpret_cast<const uint32_t *>(&b2);
        }
        const int chunk16 = 4 * (q & 1) + ch;
        *reinterpret_cast<uint4 *>(arow + ((chunk16 ^ (rl & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
    fence_proxy_async_smem();   // the tile's generic stores become visible to the tensor cores
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      if (!mbar_wait(&bar_x[s], (uint32_t)((c >> 1) & 1), kWaitLimit)) {
        bad |= QAMW_STATUS_TIMEOUT;
        s_fail = 1;
      } else {
        tc_fence_after();
        const uint32_t a_base = smem_u32(As), b_base = smem_u32(Bs);
#pragma unroll
        for (int k16 = 0; k16 < kBK / 16; ++k16) {
          const uint32_t atom = k16 >> 2, koff = (k16 & 3) * 32;
          const uint64_t ad = smem_desc_sw128(a_base + atom * kAtomBytesA + koff);
          const uint64_t bd = smem_desc_sw128(b_base + atom * (NT * 128) + koff);
          mma_bf16(tmem, ad, bd, idesc, (c > 0 || k16 > 0) ? 1u : 0u);
        }
        mma_commit(&bar_mma[s]);
      }
    }
  }
  __syncthreads();
  if (s_fail) failed = true;
  // the last chunk's commit covers every MMA before it
  if (!failed && n_chunks > 0) {
    const int64_t c = n_chunks - 1;
    if (!mbar_wait(&bar_mma[c & 1], (uint32_t)((c >> 1) & 1), kWaitLimit)) {
      bad |= QAMW_STATUS_TIMEOUT;
      failed = true;
    }
  }
  failed = __syncthreads_or(failed ? 1 : 0) != 0;
  if (!failed) {
    tc_fence_after();
    // warps w and w + 4 read tensor-memory lanes 32 (w % 4) .. + 31 (rows), each half of the columns
    const int wq = warp & 3;
    const int64_t m = m0 + 32 * wq + lane;
    const int half = warp >> 2;
    const int ncol = NT / 2;   // a multiple of 8
    const int cend = (half + 1) * ncol;
    // 16 columns per load; a load may reach 8 columns past the half (never
    // past the allocated columns: NT + 8 <= the allocation for NT = 16 * odd)
    for (int c0 = half * ncol; c0 < cend; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + ((uint32_t)(32 * wq) << 16) + (uint32_t)c0, v);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int64_t t = t0 + c0 + j;
        if (c0 + j < cend && m < a.M && t < g.T) g.Y[t * g.ldy + m] = v[j];
      }
    }
  } else {
    // a wait ran out: give the copies and MMAs in flight a second bounded wait before freeing
    if (threadIdx.x == 0) {
      mbar_wait(&bar_x[0], 0, kWaitLimit);
      mbar_wait(&bar_mma[0], 0, kWaitLimit);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols)
                              : "memory");
  bad = __reduce_or_sync(0xffffffffu, bad);
  if (lane == 0) status_or(a.status, bad);
}

}  // namespace

size_t decode_gemm_smem_bytes(int NT, int N) {
  return 1024 + 2 * (size_t)kStageBytesA + 2 * (size_t)NT * 256 + (size_t)N * 8 + kBK * 4;
}

cudaError_t launch_decode_gemm(const DecodeArgs &d, const uint16_t *X, int64_t T, int64_t ldx, float *Y, int64_t ldy,
                               cudaStream_t s) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  int NT = (int)std::min<int64_t>(256, (T + 15) / 16 * 16);
  CUtensorMap xmap;
  {
    cuuint64_t dims[2] = {(cuuint64_t)d.K, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)NT};
    cuuint32_t es[2] = {1, 1};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(X), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  GemmArgs g;
  g.d = d;
  g.T = T;
  g.NT = NT;
  g.Y = Y;
  g.ldy = ldy;
  const size_t smem = decode_gemm_smem_bytes(NT, d.N);
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(decode_gemm_kernel), smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((d.M + kBM - 1) / kBM), (unsigned)((T + NT - 1) / NT));
  decode_gemm_kernel<<<grid, kThreads, smem, s>>>(xmap, g);
  return cudaGetLastError();
}

}  // namespace qamw
