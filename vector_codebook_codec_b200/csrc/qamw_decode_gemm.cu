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
constexpr int kWarps = 16;            // one (row, 32-column quarter) of the chunk per thread
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

// shared-memory layout after the 1024-aligned operand stages
struct GemmSmem {
  int stage_b, words_row, words_stage;
  size_t off_b, off_words, off_cb, off_fac, off_sig, total;
};
constexpr int kWordStages = 3;   // packed words of a chunk are fetched two chunks ahead
__host__ __device__ __forceinline__ GemmSmem gemm_smem(int NT, int N, int B, int64_t K) {
  GemmSmem g;
  g.stage_b = NT * 256;                          // 2 atoms of NT rows x 128 B
  g.words_row = 2 * B;                           // a row's packed words of one chunk (64 pairs)
  g.words_stage = kBM * g.words_row + 4;         // + 4: the unpacking reads one word past a row
  g.off_b = 2 * (size_t)kStageBytesA;
  g.off_words = g.off_b + 2 * (size_t)g.stage_b;
  g.off_cb = g.off_words + kWordStages * (size_t)g.words_stage * 4;
  g.off_fac = (g.off_cb + (size_t)N * 8 + 15) & ~(size_t)15;   // 16-byte loads of the factors
  g.off_sig = g.off_fac + (size_t)K * 4;                        // every column's factor, computed once
  g.total = g.off_sig + kWordStages * (kBK / 2) * 4;
  return g;
}

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

// The 16 indices of pairs 16 q .. 16 q + 15 of a row's chunk, from its 2B
// staged words (LSB-first B-bit fields). BB > 0: B fixed at compile time (the
// quarter's first field starts at bit 0 or 16 of a word; a 16-bit funnel
// shift aligns it, and every later position is a constant).
template <int BB>
__device__ __forceinline__ void unpack16(const uint32_t *rw, int q, int B, uint32_t (&idx)[16]) {
  if (BB > 0) {
    constexpr int kNW = (16 * BB + 31) / 32 + 1;
    const int bit0 = 16 * q * BB;
    const uint32_t *p = rw + (bit0 >> 5);
    uint32_t w[kNW + 1];
#pragma unroll
    for (int i = 0; i <= kNW; ++i) w[i] = p[i];
    if (bit0 & 31) {
#pragma unroll
      for (int i = 0; i < kNW; ++i) w[i] = __funnelshift_r(w[i], w[i + 1], 16);
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int b = k * BB, wi = b >> 5, sh = b & 31;
      uint32_t v = w[wi] >> sh;
      if (sh + BB > 32) v |= w[wi + 1] << (32 - sh);
      idx[k] = v & ((1u << BB) - 1u);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int b = (16 * q + k) * B, wi = b >> 5, sh = b & 31;
      uint64_t v = rw[wi];
      if (sh + B > 32) v |= (uint64_t)rw[wi + 1] << 32;
      idx[k] = (uint32_t)(v >> sh) & ((1u << B) - 1u);
    }
  }
}

// BB > 0 fixes the code size, LB > 0 log2 b, at compile time (a butterfly
// stage guarded by a run-time block size costs register copies where the two
// paths join); 0 reads them at run time.
template <int BB, int LB>
__global__ void __launch_bounds__(kThreads, 1) decode_gemm_kernel(const __grid_constant__ CUtensorMap xmap, GemmArgs g) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // 1024-byte alignment for the swizzled operand tiles
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const DecodeArgs &a = g.d;
  const int NT = g.NT;
  const int B = BB > 0 ? BB : a.bits;
  const GemmSmem L = gemm_smem(NT, a.N, B, a.K);
  unsigned char *A0 = smem;                                          // [2][kStageBytesA]
  unsigned char *B0 = smem + L.off_b;                                // [2][stage_b]
  uint32_t *W0 = reinterpret_cast<uint32_t *>(smem + L.off_words);   // [2][words_stage] packed words of a chunk
  float2 *cbf = reinterpret_cast<float2 *>(smem + L.off_cb);         // (c0 + c1, c0 - c1): the first butterfly folded in
  float *fac = reinterpret_cast<float *>(smem + L.off_fac);          // [K] d_j / (sqrt(b) s_j)
  float *S0 = reinterpret_cast<float *>(smem + L.off_sig);           // [kWordStages][64] sigma of a chunk

  __shared__ __align__(8) uint64_t bar_x[2], bar_mma[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.x * kBM;
  const int64_t t0 = (int64_t)blockIdx.y * NT;
  const int64_t n_chunks = a.K / kBK;
  const int log2b = LB > 0 ? LB : a.log2b;
  const float inv_sqrt_b = (float)(1.0 / sqrt((double)(1 << log2b)));
  const uint32_t tmem_cols = NT <= 32 ? 32 : (NT <= 64 ? 64 : (NT <= 128 ? 128 : 256));

  // packed words and sigma of chunk c into staging buffer c % 3 (cp.async, 8 bytes
  // at a time: a row's 2B words of a chunk start 8B-byte aligned; four threads
  // per row; rows past M read as 0)
  auto stage_chunk = [&](int64_t c) {
    const int ws = (int)(c % kWordStages);
    uint32_t *dw = W0 + ws * L.words_stage;
    const int row = threadIdx.x >> 2, part = threadIdx.x & 3;
    const int64_t m = m0 + row;
    uint32_t *drow = dw + row * L.words_row;
    if (m < a.M) {
      const uint32_t *src = a.packed + m * a.wpr + c * L.words_row;
      for (int k = part; k < B; k += 4) cp_async8(drow + 2 * k, src + 2 * k);
    } else {
      for (int k = part; k < B; k += 4) *reinterpret_cast<uint2 *>(drow + 2 * k) = make_uint2(0u, 0u);
    }
    if (threadIdx.x < kBK / 8)
      cp_async16(S0 + ws * (kBK / 2) + 4 * threadIdx.x, a.sigma + c * (kBK / 2) + 4 * threadIdx.x);
    cp_async_commit();
  };

  for (int i = threadIdx.x; i < a.N; i += kThreads) {
    const float c0 = a.codebook[2 * i], c1 = a.codebook[2 * i + 1];
    cbf[i] = make_float2(c0 + c1, c0 - c1);
  }
  if (threadIdx.x < 4 * kWordStages) {   // the padding words past the last row of each staging buffer
    W0[(threadIdx.x >> 2) * L.words_stage + kBM * L.words_row + (threadIdx.x & 3)] = 0u;
  }
  // every column's factor d_j / (sqrt(b) s_j), once
  for (int64_t j = threadIdx.x; j < a.K; j += kThreads) {
    float f = __fdiv_rn(inv_sqrt_b, a.col_scale != nullptr ? a.col_scale[j] : 1.0f);
    if (mask_is_negative(a.seed, j)) f = -f;
    fac[j] = f;
  }
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
  if (n_chunks > 0) stage_chunk(0);
  if (n_chunks > 1) stage_chunk(1);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  // instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, N = NT, M = 128
  const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

  // this thread's item of every chunk: row rl = 8 w + lane / 4, columns 32 q .. 32 q + 31
  const int q = lane & 3;
  const int rl = 8 * warp + (lane >> 2);
  const int64_t mrow = m0 + rl;
  const bool rin = mrow < a.M;
  const float rn = rin ? a.row_norm[mrow] : 0.0f;
  uint32_t bad = (rin && !isfinite(rn)) ? QAMW_STATUS_NONFINITE_NORM : 0u;
  const bool check_idx = a.N < (1 << B);
  unsigned char *arow0 = A0 + (q >> 1) * kAtomBytesA + rl * 128;

  bool failed = false;
  for (int64_t c = 0; c < n_chunks && !failed; ++c) {
    const int s = (int)(c & 1);
    unsigned char *Bs = B0 + s * L.stage_b;
    if (c >= 2) {   // stage s was read by the MMAs of chunk c - 2 (every thread waits before overwriting it)
      if (!mbar_wait(&bar_mma[s], (uint32_t)(((c - 2) >> 1) & 1), kWaitLimit)) bad |= QAMW_STATUS_TIMEOUT;
    }
    if (threadIdx.x == 0 && !(bad & QAMW_STATUS_TIMEOUT)) {
      mbar_arrive_expect_tx(&bar_x[s], (uint32_t)L.stage_b);
      tma_load_2d(Bs, &xmap, (int)(c * kBK), (int)t0, &bar_x[s]);
      tma_load_2d(Bs + NT * 128, &xmap, (int)(c * kBK + 64), (int)t0, &bar_x[s]);
    }
    // the words of chunk c + 2 in flight while this one is decoded (its
    // buffer held chunk c - 1, decoded before the previous barrier)
    if (c + 2 < n_chunks) stage_chunk(c + 2);
    if (c + 2 < n_chunks) cp_async_wait<2>();   // chunk c's words and sigma have landed
    else if (c + 1 < n_chunks) cp_async_wait<1>();
    else cp_async_wait<0>();
    __syncthreads();

    const int ws = (int)(c % kWordStages);
    const uint32_t *rw = W0 + ws * L.words_stage + rl * L.words_row;
    const float4 *sg4 = reinterpret_cast<const float4 *>(S0 + ws * (kBK / 2) + 16 * q);
    uint32_t idx[16];
    unpack16<BB>(rw, q, B, idx);
    if (check_idx) {   // a codebook smaller than 2^B: out-of-range indices decode as centroid 0
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        if (idx[p] >= (uint32_t)a.N) { bad |= QAMW_STATUS_BAD_INDEX; idx[p] = 0; }
      }
    }
    float2 v[16];   // v[p] = r sigma_k (c0 + c1, c0 - c1): block bit 0 done, the row norm applied
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float4 sk = sg4[h];
      const float sr[4] = {sk.x * rn, sk.y * rn, sk.z * rn, sk.w * rn};
#pragma unroll
      for (int u = 0; u < 4; ++u) v[4 * h + u] = mul2(cbf[idx[4 * h + u]], make_float2(sr[u], sr[u]));
    }
    // block bits 1..4 in registers (pairs p and p | h/2), 5..6 across the 4 lanes of the row
#pragma unroll
    for (int t = 1; t < 5; ++t) {
      if (t < log2b) {
        const int h = 1 << (t - 1);
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          if ((p & h) == 0) {
            const float2 x0 = v[p], x1 = v[p | h];
            v[p] = add2(x0, x1);
            v[p | h] = sub2(x0, x1);
          }
        }
      }
    }
#pragma unroll
    for (int t = 5; t < 7; ++t) {
      if (t < log2b) {
        const int hb = 1 << (t - 5);
        const float sgn = (lane & hb) ? -1.0f : 1.0f;
        const float2 sg2 = make_float2(sgn, sgn);
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, v[p].x, hb), __shfl_xor_sync(0xffffffffu, v[p].y, hb));
          v[p] = fma2(sg2, v[p], o);
        }
      }
    }
    if (!rin) {
#pragma unroll
      for (int p = 0; p < 16; ++p) v[p] = make_float2(0.0f, 0.0f);
    }
    // scale by r d_j / (sqrt(b) s_j), round to bf16, store into the swizzled K-major tile:
    // row rl, columns 32 q .. 32 q + 31 = atom q / 2, 16-byte chunks 4 (q % 2) .. + 3
    unsigned char *arow = arow0 + s * kStageBytesA;
    const float4 *f4 = reinterpret_cast<const float4 *>(fac + c * kBK + 32 * q);
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t pk[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float4 f = f4[2 * ch + h];
        const float2 w0 = mul2(v[4 * ch + 2 * h], make_float2(f.x, f.y));
        const float2 w1 = mul2(v[4 * ch + 2 * h + 1], make_float2(f.z, f.w));
        const __nv_bfloat162 b0 = __floats2bfloat162_rn(w0.x, w0.y), b1 = __floats2bfloat162_rn(w1.x, w1.y);
        pk[2 * h] = *reinterpret_cast<const uint32_t *>(&b0);
        pk[2 * h + 1] = *reinterpret_cast<const uint32_t *>(&b1);
      }
      const int chunk16 = 4 * (q & 1) + ch;
      *reinterpret_cast<uint4 *>(arow + ((chunk16 ^ (rl & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    fence_proxy_async_smem();   // the tile's generic stores become visible to the tensor cores
    tc_fence_before();
    if (__syncthreads_or(bad & QAMW_STATUS_TIMEOUT)) { failed = true; break; }
    if (threadIdx.x == 0) {
      if (!mbar_wait(&bar_x[s], (uint32_t)((c >> 1) & 1), kWaitLimit)) {
        bad |= QAMW_STATUS_TIMEOUT;
        s_fail = 1;
      } else {
        tc_fence_after();
        const uint32_t a_base = smem_u32(A0 + s * kStageBytesA), b_base = smem_u32(Bs);
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
  cp_async_wait<0>();
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
    // warps w, w + 4, w + 8, w + 12 read tensor-memory lanes 32 (w % 4) .. + 31 (rows), a quarter of the columns each
    const int wq = warp & 3, grp = warp >> 2;
    const int64_t m = m0 + 32 * wq + lane;
    const int ncol = NT / 4;   // a multiple of 4
    const int cbeg = grp * ncol, cend = cbeg + ncol;
    // 16 columns per load; a load may reach 12 columns past the quarter (never
    // past the allocated columns, which exceed NT by at least 16 unless the quarters are multiples of 16)
    for (int c0 = cbeg; c0 < cend; c0 += 16) {
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

size_t decode_gemm_smem_bytes(int NT, int N, int B, int64_t K) { return 1024 + gemm_smem(NT, N, B, K).total; }

cudaError_t launch_decode_gemm(const DecodeArgs &d, const uint16_t *X, int64_t T, int64_t ldx, float *Y, int64_t ldy,
                               cudaStream_t s) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  int dev = 0, smem_max = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  // the widest token tile (<= 256, a multiple of 16) whose stages fit
  int NT = (int)std::min<int64_t>(256, (T + 15) / 16 * 16);
  while (NT > 16 && decode_gemm_smem_bytes(NT, d.N, d.bits, d.K) + 256 > (size_t)smem_max) NT -= 16;
  if (decode_gemm_smem_bytes(NT, d.N, d.bits, d.K) + 256 > (size_t)smem_max) return cudaErrorNotSupported;
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
  const size_t smem = decode_gemm_smem_bytes(NT, d.N, d.bits, d.K);
  const dim3 grid((unsigned)((d.M + kBM - 1) / kBM), (unsigned)((T + NT - 1) / NT));
  // 11- and 10-bit codes with 128-column blocks compiled for their shape; anything else at run time
  auto run = [&](auto kern) -> cudaError_t {
    cudaError_t err = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), smem);
    if (err != cudaSuccess) return err;
    kern<<<grid, kThreads, smem, s>>>(xmap, g);
    return cudaGetLastError();
  };
  if (d.bits == 11 && d.log2b == 7) return run(decode_gemm_kernel<11, 7>);
  if (d.bits == 10 && d.log2b == 7) return run(decode_gemm_kernel<10, 7>);
  return run(decode_gemm_kernel<0, 0>);
}

}  // namespace qamw
