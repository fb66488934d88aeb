// qamw_decode_gemm.cu -- QAM-W decode fused with the matrix multiply that
// consumes the weights, on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "QAM-W: Joint 2D Codebook Quantization for LLM Weights ...", Methodology (6)
// Decoding, and "Significance and Claims" (the bit savings reach inference
// latency only once decoding is fused into the matrix multiply). The product
//   Y[t][m] = sum_j X[t][j] w_hat[m][j],
//   w_hat[m][j] = r_m d_j (H_b y_m)_j / (sqrt(b) s_j),  y_m[2k+e] = sigma_k C[idx(m,k)][e],
// is formed without w_hat. Every decode step after the codebook lookup is
// linear and the same for all rows, and H_b is symmetric, so those steps move
// to the activations:
//   Y[t][m] = r_m sum_i a_t[i] C[idx(m, i/2)][i%2],
//   a_t[i]  = sigma_{i/2} (H_b (d (.) X[t] / s))_i / sqrt(b)      (per block of b columns),
// which costs log2 b adds per activation instead of per weight.
//
// Kernel 1 (prepare_x_kernel): a cluster of up to 8 CTAs per token (one CTA
// from 512 tokens on) computes a_t in fp32 (each CTA a share of the columns),
// agrees on the token's largest |a| through distributed shared memory,
// scales by 2^-e_t so that it lies in (2^13, 2^14], and stores fp16 a_t and
// 2^e_t. It also clears the tile counters of kernel 2.
//
// Kernel 2 (decode_gemm_kernel), persistent: one CTA per SM. The work is the
// list of (output tile, K chunk) units -- an output tile is 128 rows m x NT
// tokens, a chunk 128 columns (64 pairs) -- split into equal contiguous
// ranges, one per CTA ("stream-K"), so every SM gets the same number of
// chunks whatever the number of tiles. Warp roles:
//   warps 0-15  two groups of 8; a group unpacks the chunk's indices of the
//               128 rows (two threads per row, one 64-column half each), looks
//               the centroids up as fp16 pairs and stores the 128 x 128-column
//               operand tile straight into tensor memory (tcgen05.st: row m in
//               lane m, pair k in column k), where the MMA reads it -- the
//               decoded weights never touch shared memory;
//   warp 16     streams the packed indices into a ring of word stages (one TMA
//               tensor copy per chunk, or cp.async when the row pitch is not a
//               multiple of 16 bytes);
//   warp 17     streams the fp16 a tile of the chunk (two TMA copies, 128-byte
//               swizzle, two atoms of 64 columns) into the shared-memory
//               activation stage that goes with the group's operand stage; its
//               bytes complete the same full barrier, so the MMA warp waits
//               once per chunk;
//   warp 18     issues the chunk's eight 128 x NT x 16 tcgen05.mma (A from
//   (and 23)    tensor memory, B from shared memory, fp16 in, fp32 accumulated
//               in tensor memory, two accumulator buffers used in turn for
//               NT <= 128) and commits them to the stage's empty barrier (that
//               commit frees both tiles); for NT <= 64 warp 23 issues the four
//               of the chunk's second atom into an accumulator of its own;
//   warps 19-22 read a finished accumulator (tcgen05.ld) and write
//               Y = r_m 2^e_t acc; a tile whose chunks were split between CTAs
//               is written as partial sums to the workspace, and the CTA that
//               finishes it last adds the parts in a fixed order (its own
//               from its accumulator when there are two).
// Stages hand over through mbarriers (full / empty per stage), so the roles
// run ahead of one another by up to the ring depth; no CTA-wide barrier sits
// in the loop.
//
// Every wait is a bounded mbarrier wait; one that runs out sets
// QAMW_STATUS_TIMEOUT, the other roles see the CTA's failure flag and stop,
// the copies and MMAs already in flight are waited for (again bounded), the
// tensor memory is freed and the kernel returns.
#include <algorithm>
#include <cmath>
#include <cuda_fp16.h>

#include "qamw_device.cuh"
#include "qamw_internal.h"
#include "qamw_mbarrier.cuh"
#include "qamw_tensor_map.h"

namespace qamw {
namespace {

constexpr int kBM = 128;                   // output rows per tile (tensor-memory lanes)
constexpr int kBK = 128;                   // columns (64 pairs) per chunk: two 128-byte swizzle atoms
constexpr int kAtom = 64;                  // columns of one swizzle atom (128 bytes of fp16)
constexpr int kDecWarps = 16;              // 2 groups of 8; a group decodes one unit at a time
constexpr int kWarpWords = kDecWarps;      // streams the packed words
constexpr int kWarpX = kDecWarps + 1;      // streams the activation tiles
constexpr int kWarpMma = kDecWarps + 2;    // issues the MMAs
constexpr int kWarpEpi = kDecWarps + 3;    // first of the 4 epilogue warps
constexpr int kWarpMma2 = kDecWarps + 7;   // the second MMA issuer for token tiles of <= 64
constexpr int kThreads = (kDecWarps + 8) * 32;
constexpr int kMaxStages = 8;
constexpr int kMaxCtas = 160;              // persistent CTAs at most (the partial-sum slots are sized for it)
constexpr uint32_t kWaitTries = 1u << 22;  // try_wait attempts before a spinning wait gives up
constexpr uint32_t kSleepTries = 1u << 21; // attempts (<= 512 ns apart) before a sleeping wait gives up
constexpr int kPrepThreads = 128;          // small enough to share an SM with a CTA of kernel 2
constexpr int kPrepCluster = 8;            // CTAs per token in kernel 1 (portable cluster size)

// ---------------------------------------------------------------------------
// workspace: [a: T x K fp16][2^e_t: T fp32][tile counters][partial sums]
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }
__host__ __device__ __forceinline__ int nt_cap(int64_t T) { return (int)(T >= 256 ? 256 : (T + 15) / 16 * 16); }
struct WsLayout {
  size_t off_scale, off_cnt, off_part, total;
};
__host__ __device__ __forceinline__ WsLayout ws_layout(int64_t M, int64_t K, int64_t T) {
  WsLayout w;
  const int64_t tiles = ((M + kBM - 1) / kBM) * ((T + 15) / 16);   // tiles for the narrowest token tile
  w.off_scale = align256((size_t)T * (size_t)K * 2);
  w.off_cnt = w.off_scale + align256((size_t)T * 4);
  w.off_part = w.off_cnt + align256((size_t)tiles * 4);
  w.total = w.off_part + (size_t)2 * kMaxCtas * (size_t)nt_cap(T) * kBM * 4;
  return w;
}

struct GemmArgs {
  const uint32_t *packed;   // [M][wpr]
  const float *row_norm;    // [M]
  const float *codebook;    // [N][2] fp32
  const float *tok_scale;   // [T] 2^e_t
  uint32_t *counters;       // [tiles] contributions received (cleared by kernel 1)
  float *part;              // [2 * CTAs][NT][128] partial sums
  float *Y;                 // [T][ldy]
  int64_t ldy, M, K, T, wpr;
  int64_t n_m;              // row tiles
  int64_t n_units;          // tiles x chunks
  int N, bits;
  int NT;                   // tokens per tile (16..256, a multiple of 16)
  int SA;                   // weight-tile stages = decode groups (2)
  int SW;                   // word stages (a multiple of SA)
  int BW;                   // staged words per row and chunk
  int words_tma;            // 1: words by TMA; 0: by cp.async
  int32_t *status;
};

// shared-memory layout (after 1024-byte alignment): SA activation tiles, SW
// word stages, the fp16 codebook (the operand tiles live in tensor memory)
struct GemmSmem {
  int stage_x, wpitch;
  size_t off_x, off_w, off_cb, total;
};
__host__ __device__ __forceinline__ GemmSmem gemm_smem(int NT, int SA, int SW, int BW, int N) {
  GemmSmem g;
  g.stage_x = NT * 256;                                  // two atoms of NT rows x 128 B
  g.wpitch = (kBM * BW * 4 + 127) & ~127;
  g.off_x = 0;
  g.off_w = g.off_x + (size_t)SA * g.stage_x;
  g.off_cb = g.off_w + (size_t)SW * g.wpitch;
  g.total = g.off_cb + (size_t)N * 4;
  return g;
}

// the contiguous unit range [u0, u1) of CTA b of G, and the CTA holding unit u
__host__ __device__ __forceinline__ int64_t range_start(int64_t b, int64_t G, int64_t total) { return b * total / G; }
__host__ __device__ __forceinline__ int64_t cta_of_unit(int64_t u, int64_t G, int64_t total) {
  return ((u + 1) * G - 1) / total;
}

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  // start address >> 4 | leading offset 16 B (ignored for swizzled K-major) |
  // stride offset 1024 B (8 rows of 128 B) | descriptor version 1 | 128-byte swizzle
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }   // the 4 epilogue warps
__device__ __forceinline__ void dec_sync() { asm volatile("bar.sync 2, 512;" ::: "memory"); }   // the 16 decode warps
// barrier of the 4 epilogue warps that returns whether any of their threads passed true
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile("{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, 1, 128, p; selp.u32 %0, 1, 0, q; }"
               : "=r"(r)
               : "r"((uint32_t)v)
               : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// arrive once all of this thread's earlier cp.async copies have landed (the
// barrier's expected count includes this arrival)
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// programmatic dependent launch: kernel 2 starts while kernel 1 runs, and
// waits for kernel 1's results only where it reads them
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

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

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 accumulator columns of this warp's lanes: the sum of the ni accumulators
// (acc_cols apart) that the MMA warps filled
__device__ __forceinline__ void tmem_ld_acc(uint32_t taddr, uint32_t ni, uint32_t acc_cols, float (&v)[16]) {
  tmem_ld16(taddr, v);
  if (ni == 2) {
    float v2[16];
    tmem_ld16(taddr + acc_cols, v2);
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] += v2[j];
  }
}

// Bounded waits that also give up once another role of the CTA has failed:
// 0 = the phase completed, 1 = the CTA failed elsewhere, 2 = this wait ran out
// (it then raises the CTA's failure flag). wait_phase spins (the pipeline's
// hand-overs); wait_phase_sleep backs off with nanosleep (the epilogue's wait
// for a whole tile), leaving the issue slots to the decode warps.
__device__ __forceinline__ int wait_phase(uint64_t *bar, uint32_t parity, volatile int *fail) {
  for (uint32_t i = 0; i < kWaitTries; ++i) {
    if (mbar_try_wait(bar, parity)) return 0;
    if ((i & 63u) == 63u && *fail) return 1;
  }
  *fail = 1;
  return 2;
}
__device__ __forceinline__ int wait_phase_sleep(uint64_t *bar, uint32_t parity, volatile int *fail) {
  uint32_t ns = 32;
  for (uint32_t i = 0; i < kSleepTries; ++i) {
    if (mbar_try_wait(bar, parity)) return 0;
    if (*fail) return 1;
    __nanosleep(ns);
    if (ns < 512) ns <<= 1;
  }
  *fail = 1;
  return 2;
}

// position of a unit: tile = mt + n_m tt (row tile mt, token tile tt), chunk c;
// walked incrementally (no 64-bit division per unit)
struct Cursor {
  int64_t tile, mt, tt;
  int c;
  __device__ __forceinline__ Cursor(int64_t u, int n_chunks, int64_t n_m) {
    tile = u / n_chunks;
    c = (int)(u - tile * n_chunks);
    tt = tile / n_m;
    mt = tile - tt * n_m;
  }
  __device__ __forceinline__ void next(int n_chunks, int64_t n_m) {
    if (++c == n_chunks) {
      c = 0;
      ++tile;
      if (++mt == n_m) { mt = 0; ++tt; }
    }
  }
};

// One half of an operand row: the 32 fp16 centroid pairs of one 64-column
// half of the unit, stored into tensor-memory columns ta .. ta + 31 of the
// thread's lane (pair k in column k: the K-major layout of an A operand read
// from tensor memory, two fp16 per 32-bit column). Field k of the half is bits
// 32 REM + k BB .. of the staged words w. Warp-collective (tcgen05.st); returns
// the status bits.
template <int BB>
struct RowWords {
  static constexpr int kNW4 = (96 + 32 * BB + 127) / 128;   // 16-byte loads that cover REM <= 3 plus 32 fields
};
// CHECK: the codebook has fewer than 2^B entries, so a field may be out of range.
template <int BB, int REM, bool CHECK>
__device__ __forceinline__ uint32_t write_row(const uint32_t (&w)[4 * RowWords<BB>::kNW4], const uint32_t *cb,
                                              uint32_t ta, int N, bool rin) {
  constexpr uint32_t kMask4 = ((1u << BB) - 1u) << 2;   // the field times 4: its byte offset in the table
  const unsigned char *cbb = reinterpret_cast<const unsigned char *>(cb);
  uint32_t bad = 0;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t e[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      const int b = 32 * REM + (16 * j + p) * BB, wi = b >> 5, sh = b & 31;
      // the byte offset 4 id straight from the words: one shift (a funnel
      // shift for a field that spans two words) and one mask
      uint32_t off = (sh + BB > 32) ? (__funnelshift_r(w[wi], w[wi + 1], sh - 2) & kMask4)
                     : (sh >= 2)    ? ((w[wi] >> (sh - 2)) & kMask4)
                                    : ((w[wi] << (2 - sh)) & kMask4);
      if (CHECK && off >= ((uint32_t)N << 2)) {   // decode as centroid 0
        if (rin) bad |= QAMW_STATUS_BAD_INDEX;
        off = 0;
      }
      e[p] = *reinterpret_cast<const uint32_t *>(cbb + off);
    }
    tmem_st16(ta + 16 * j, e);   // pairs 16 j .. 16 j + 15 = tensor-memory columns
  }
  return bad;
}
// the same for a code size known only at run time (fields read from shared memory)
__device__ __forceinline__ uint32_t write_row_any(const uint32_t *rowp, int rem, int B, const uint32_t *cb,
                                                  uint32_t ta, bool check_idx, int N, bool rin) {
  uint32_t bad = 0;
  for (int j = 0; j < 2; ++j) {
    uint32_t e[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      const int b = 32 * rem + (16 * j + p) * B, wi = b >> 5, sh = b & 31;
      uint64_t v = rowp[wi];
      if (sh + B > 32) v |= (uint64_t)rowp[wi + 1] << 32;
      uint32_t id = (uint32_t)(v >> sh) & ((1u << B) - 1u);
      if (check_idx && id >= (uint32_t)N) {
        if (rin) bad |= QAMW_STATUS_BAD_INDEX;
        id = 0;
      }
      e[p] = cb[id];
    }
    tmem_st16(ta + 16 * j, e);
  }
  return bad;
}

// ----------------------------------------------------------------------------
// Kernel 1: a_t = sigma (.) H_b (d (.) x_t / s) / sqrt(b), fp16 with 2^e_t.
// Cluster of S CTAs per token (blocks S t .. S t + S - 1); CTA rank c takes the column units
// c, c + S, ... (a unit is 512 columns, or one block when b = 1024) and keeps
// them in shared memory as fp32.
// ----------------------------------------------------------------------------
struct PrepArgs {
  const uint16_t *X;        // bf16 [T][ldx]
  int64_t ldx, T, K;
  const float *sigma;       // [K/2]
  const float *col_scale;   // [K] or nullptr
  uint64_t seed;
  int log2b;
  int S;                    // CTAs per token (cluster size)
  __half *A;                // fp16 [T][K]
  float *tok_scale;         // [T]
  uint32_t *counters;       // cleared here
  int64_t n_counters;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(const float *local, uint32_t rank) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// 48 registers, no spills. A CTA does not fit beside a CTA of kernel 2 (24
// warps x 80 registers leave 1024 registers per SM sub-partition): kernel 2's
// CTAs on the few SMs that run kernel 1 start when it ends. A 32-register
// build that fits beside it was measured no faster (its spills).
__global__ void __launch_bounds__(kPrepThreads, 10) prepare_x_kernel(PrepArgs p) {
  extern __shared__ __align__(16) float vloc[];   // the CTA's units, fp32, one after the other
  __shared__ float red[kPrepThreads / 32];
  __shared__ float cta_max;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S;
  const int64_t t = blockIdx.x / S;
  const int64_t K = p.K;
  const int lb = p.log2b;
  const int rank = (int)cluster_rank();
  const int ucols = lb > 9 ? (1 << lb) : 512;       // columns per unit
  const int64_t n_units = (K + ucols - 1) / ucols;
  const int64_t n_mine = n_units > rank ? (n_units - rank + S - 1) / S : 0;
  const int lreg = lb < 4 ? lb : 4, lshf = lb < 9 ? lb : 9;
  const uint16_t *xr = p.X + t * p.ldx;

  griddep_launch_dependents();
  if (t == 0 && rank == 0)
    for (int64_t i = threadIdx.x; i < p.n_counters; i += kPrepThreads) p.counters[i] = 0u;
  const float inv_sqrt_b = (float)(1.0 / sqrt((double)(1 << lb)));
  float mx = 0.0f;   // the largest |a| of the CTA's columns

  // block bits 0..3 in registers (16 consecutive columns per lane), 4..8
  // across the lanes of a warp (a 512-column span per warp), 9 in shared memory
  const int64_t n_spans = n_mine * (ucols / 512);
  for (int64_t sp = warp; sp < n_spans; sp += kPrepThreads / 32) {
    const int64_t li = sp / (ucols / 512), part = sp % (ucols / 512);
    const int64_t col = (rank + li * S) * (int64_t)ucols + part * 512 + 16 * lane;
    float *dst = vloc + li * ucols + part * 512 + 16 * lane;
    const bool in = col < K;   // K % 16 == 0: a lane's 16 columns are all in or all out
    float4 sg4[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    if (lb <= 9 && in) {   // sigma of the lane's 8 pairs, loaded early (col % 16 == 0: 32-byte aligned)
      const float4 *sg = reinterpret_cast<const float4 *>(p.sigma + (col >> 1));
      sg4[0] = sg[0];
      sg4[1] = sg[1];
    }
    float u[16];
    if (in) {
      const uint4 *src = reinterpret_cast<const uint4 *>(xr + col);
      const uint4 q0 = src[0], q1 = src[1];
      const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x = __uint_as_float(((e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xffffu)) << 16);
        float v = p.col_scale != nullptr ? __fdiv_rn(x, p.col_scale[col + e]) : x;
        if (mask_is_negative(p.seed, col + e)) v = -v;
        u[e] = v;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) u[e] = 0.0f;
    }
#pragma unroll
    for (int tb = 0; tb < 4; ++tb) {
      if (tb < lreg) {
        const int h = 1 << tb;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          if ((e & h) == 0) {
            const float a0 = u[e], a1 = u[e | h];
            u[e] = a0 + a1;
            u[e | h] = a0 - a1;
          }
        }
      }
    }
    for (int tb = 4; tb < lshf; ++tb) {   // warp-uniform
      const int h = 1 << (tb - 4);
      const float sgn = (lane & h) ? -1.0f : 1.0f;
#pragma unroll
      for (int e = 0; e < 16; ++e) u[e] = __fmaf_rn(sgn, u[e], __shfl_xor_sync(0xffffffffu, u[e], h));
    }
    if (lb <= 9 && in) {   // every butterfly done: times sigma_k / sqrt(b) here
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float4 s4 = sg4[h];
        const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float gk = __fmul_rn(sv[k], inv_sqrt_b);
          u[8 * h + 2 * k] = __fmul_rn(u[8 * h + 2 * k], gk);
          u[8 * h + 2 * k + 1] = __fmul_rn(u[8 * h + 2 * k + 1], gk);
          mx = fmaxf(mx, fmaxf(fabsf(u[8 * h + 2 * k]), fabsf(u[8 * h + 2 * k + 1])));
        }
      }
    }
    float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d4[i] = make_float4(u[4 * i], u[4 * i + 1], u[4 * i + 2], u[4 * i + 3]);
  }
  __syncthreads();
  const int64_t n_loc = n_mine * ucols;
  if (lb > 9) {   // b = 1024: bit 9 pairs the two halves of every unit, then sigma_k / sqrt(b)
    const int h = 512;
    for (int64_t i = threadIdx.x; i < n_mine * h; i += kPrepThreads) {
      const int64_t li = i / h, o = i % h;
      float *v = vloc + li * ucols + o;
      const float a0 = v[0], a1 = v[h];
      v[0] = a0 + a1;
      v[h] = a0 - a1;
    }
    __syncthreads();
    for (int64_t i = 2 * threadIdx.x; i < n_loc; i += 2 * kPrepThreads) {
      const int64_t li = i / ucols, o = i % ucols;
      const int64_t col = (rank + li * S) * (int64_t)ucols + o;   // K % 1024 == 0: always < K
      const float gk = __fmul_rn(p.sigma[col >> 1], inv_sqrt_b);
      float2 v = *reinterpret_cast<float2 *>(vloc + i);
      v.x = __fmul_rn(v.x, gk);
      v.y = __fmul_rn(v.y, gk);
      *reinterpret_cast<float2 *>(vloc + i) = v;
      mx = fmaxf(mx, fmaxf(fabsf(v.x), fabsf(v.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int w = 1; w < kPrepThreads / 32; ++w) m = fmaxf(m, red[w]);
    cta_max = m;
  }
  cluster_sync();   // every CTA of the token has published its largest |a|
  if (warp == 0) {
    float m = lane < S ? ld_cluster_f32(&cta_max, (uint32_t)lane) : 0.0f;
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[0] = m;
  }
  __syncthreads();
  mx = red[0];
  // e = ceil(log2 mx) - 14, so that mx 2^-e lies in (2^13, 2^14]; 0 for a zero
  // or non-finite token (the latter then propagates into Y as in any product)
  int e = 0;
  if (mx > 0.0f && mx <= 3.0e38f) {
    int ex;
    const float fr = frexpf(mx, &ex);   // mx = fr 2^ex, fr in [0.5, 1)
    e = (fr == 0.5f ? ex - 1 : ex) - 14;
    e = max(-112, min(112, e));
  }
  const float down = __int_as_float((127 - e) << 23);   // 2^-e, exact
  if (rank == 0 && threadIdx.x == 0) p.tok_scale[t] = __int_as_float((127 + e) << 23);
  __half *ar = p.A + t * K;
  for (int64_t i = 8 * (int64_t)threadIdx.x; i < n_loc; i += 8 * kPrepThreads) {
    const int64_t li = i / ucols, o = i % ucols;
    const int64_t col = (rank + li * S) * (int64_t)ucols + o;
    if (col >= K) continue;
    const float4 v0 = *reinterpret_cast<const float4 *>(vloc + i), v1 = *reinterpret_cast<const float4 *>(vloc + i + 4);
    const __half2 h0 = __floats2half2_rn(v0.x * down, v0.y * down), h1 = __floats2half2_rn(v0.z * down, v0.w * down);
    const __half2 h2 = __floats2half2_rn(v1.x * down, v1.y * down), h3 = __floats2half2_rn(v1.z * down, v1.w * down);
    uint4 o4;
    o4.x = *reinterpret_cast<const uint32_t *>(&h0);
    o4.y = *reinterpret_cast<const uint32_t *>(&h1);
    o4.z = *reinterpret_cast<const uint32_t *>(&h2);
    o4.w = *reinterpret_cast<const uint32_t *>(&h3);
    *reinterpret_cast<uint4 *>(ar + col) = o4;
  }
  cluster_sync();   // no CTA leaves while another may still read its cta_max
}

// ----------------------------------------------------------------------------
// Kernel 2: unpack + lookup into the operand tile, tcgen05 MMA, epilogue.
// ----------------------------------------------------------------------------
template <int BB>
__global__ void __launch_bounds__(kThreads, 1)
    decode_gemm_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap, GemmArgs g) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // 1024-byte alignment for the swizzled operand tiles
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int B = BB > 0 ? BB : g.bits;
  const int NT = g.NT, SA = g.SA, SW = g.SW;
  const GemmSmem L = gemm_smem(NT, SA, SW, g.BW, g.N);
  unsigned char *X0 = smem + L.off_x;                                // [SA][stage_x]
  unsigned char *W0 = smem + L.off_w;                                // [SW][wpitch]
  uint32_t *cb = reinterpret_cast<uint32_t *>(smem + L.off_cb);      // [N] fp16 pairs

  __shared__ __align__(8) uint64_t full_w[kMaxStages], empty_w[kMaxStages];
  __shared__ __align__(8) uint64_t full_a[kMaxStages], empty_a[kMaxStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_fail;
  __shared__ int s_last;
  volatile int *fail = &s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_chunks = (int)(g.K / kBK);
  const int64_t G = gridDim.x;
  const int64_t u0 = range_start(blockIdx.x, G, g.n_units), u1 = range_start(blockIdx.x + 1, G, g.n_units);
  // tensor memory: nbuf accumulator buffers (two, so that the epilogue of one
  // tile overlaps the MMAs of the next, unless NT > 128), each of ni
  // accumulators of acc_cols columns (two for NT <= 64: the two MMA warps
  // each sum one 64-column half of every unit, and the epilogue adds them),
  // then the SA operand stages of 64 columns (128 fp16 per lane)
  const uint32_t acc_cols = NT <= 32 ? 32 : (NT <= 64 ? 64 : (NT <= 128 ? 128 : 256));
  const uint32_t ni = NT <= 64 ? 2 : 1;
  const uint32_t lbuf = 2 * ni * acc_cols + 64 * SA <= 512 ? 1 : 0;   // log2 of the buffer count
  const uint32_t nbuf = 1u << lbuf;
  const uint32_t a_col0 = nbuf * ni * acc_cols;
  const uint32_t tmem_cols = a_col0 + 64 * SA <= 256 ? 256 : 512;

  // each decode thread requests its first 4 codebook entries before the setup,
  // so that their latency overlaps it (and comes before the copies' burst)
  constexpr int kCbPre = 4;
  const bool cb_vec = (reinterpret_cast<uintptr_t>(g.codebook) & 7) == 0;
  float2 cpre[kCbPre];
#pragma unroll
  for (int k = 0; k < kCbPre; ++k) {
    const int i = threadIdx.x + k * kDecWarps * 32;
    cpre[k] = (warp < kDecWarps && cb_vec && i < g.N) ? reinterpret_cast<const float2 *>(g.codebook)[i]
                                                       : make_float2(0.0f, 0.0f);
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < SW; ++s) {
      mbar_init(&full_w[s], g.words_tma ? 1 : 32);
      mbar_init(&empty_w[s], kDecWarps / SA);   // the warps of the group that decodes the stage's units
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(&full_a[s], kDecWarps / SA + 1);   // the group's warps + the activation warp (with its bytes)
      mbar_init(&empty_a[s], ni);   // a commit of each MMA warp
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], ni);
      mbar_init(&acc_empty[s], 4);
    }
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
  uint32_t bad = 0;
  bool failed = false;

  if (warp < kDecWarps) {
    // the fp16 codebook, filled by the decode warps alone while the copy
    // warps already start streaming the first stages
    if (cb_vec) {   // 8-byte loads: the first kCbPre per thread already in registers
#pragma unroll
      for (int k = 0; k < kCbPre; ++k) {
        const int i = threadIdx.x + k * kDecWarps * 32;
        const __half2 h = __floats2half2_rn(cpre[k].x, cpre[k].y);
        if (i < g.N) cb[i] = *reinterpret_cast<const uint32_t *>(&h);
      }
#pragma unroll 4
      for (int i = threadIdx.x + kCbPre * kDecWarps * 32; i < g.N; i += kDecWarps * 32) {
        const float2 c2 = reinterpret_cast<const float2 *>(g.codebook)[i];
        const __half2 h = __floats2half2_rn(c2.x, c2.y);
        cb[i] = *reinterpret_cast<const uint32_t *>(&h);
      }
    } else {
      for (int i = threadIdx.x; i < g.N; i += kDecWarps * 32) {
        const __half2 h = __floats2half2_rn(g.codebook[2 * i], g.codebook[2 * i + 1]);
        cb[i] = *reinterpret_cast<const uint32_t *>(&h);
      }
    }
    dec_sync();
    // ---- decode: SA = 2 groups of 8 warps; group grp takes the CTA's units
    // u0 + grp, u0 + grp + SA, ... into operand stage grp and word stages
    // grp, grp + SA, ... (each stage is used by one group, in order), so SA
    // units are decoded at once. In a unit, thread tg of the group owns row
    // rl = tg % 128 and half hf = tg / 128 of it: the 32 pairs of columns
    // 64 hf .. 64 hf + 63, whose B words start hf B words after the unit's
    // first word. Row rl is tensor-memory lane rl (32 (warp % 4) + lane, the
    // lanes this warp may access); stage grp's half hf is columns
    // a_col0 + 64 grp + 32 hf .. + 31.
    const int wpg = kDecWarps / SA;
    const int grp = warp / wpg;
    const int tg = (warp % wpg) * 32 + lane;
    const int rl = tg & (kBM - 1);
    const int hf = tg >> 7;
    const bool check_idx = g.N < (1 << B);
    int sw = grp;
    uint32_t qa = 0, qw = 0;   // stage use counts (phase = count & 1)
    const uint32_t ta = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + a_col0 + 64 * grp + 32 * hf;
    Cursor cur(u0 + grp, n_chunks, g.n_m);
    for (int64_t u = u0 + grp; u < u1; u += SA) {
      const int c = cur.c;
      const bool rin = cur.mt * kBM + rl < g.M;
      // every failure decision is taken by the whole warp (the loop holds warp-wide syncs)
      int r = wait_phase(&full_w[sw], qw & 1u, fail);
      if (__reduce_max_sync(0xffffffffu, (unsigned)r)) { if (r == 2) bad |= QAMW_STATUS_TIMEOUT; failed = true; break; }
      // the half's first word in the staged row: the unit's 2B words start 0..3
      // words into it (TMA) or at its start (cp.async)
      const int s0 = (g.words_tma ? ((c * 2 * B) & 3) : 0) + hf * B;
      const int rem = s0 & 3;
      const uint32_t *rowp = reinterpret_cast<const uint32_t *>(W0 + (size_t)sw * L.wpitch) + rl * g.BW + (s0 & ~3);
      if (BB > 0) {
        constexpr int kNW4 = RowWords<BB>::kNW4;
        uint32_t w[4 * kNW4];
        const uint4 *src = reinterpret_cast<const uint4 *>(rowp);   // 16-byte rows, BW / 4 odd: no bank conflict
#pragma unroll
        for (int i = 0; i < kNW4; ++i) {
          const uint4 v = src[i];
          w[4 * i] = v.x;
          w[4 * i + 1] = v.y;
          w[4 * i + 2] = v.z;
          w[4 * i + 3] = v.w;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_w[sw]);
        if (qa > 0) {   // the stage's previous MMAs are done with it
          r = wait_phase(&empty_a[grp], (qa & 1u) ^ 1u, fail);
          if (__reduce_max_sync(0xffffffffu, (unsigned)r)) { if (r == 2) bad |= QAMW_STATUS_TIMEOUT; failed = true; break; }
          tc_fence_after();
        }
        if (check_idx) {
          switch (rem) {
            case 0: bad |= write_row<BB, 0, true>(w, cb, ta, g.N, rin); break;
            case 1: bad |= write_row<BB, 1, true>(w, cb, ta, g.N, rin); break;
            case 2: bad |= write_row<BB, 2, true>(w, cb, ta, g.N, rin); break;
            default: bad |= write_row<BB, 3, true>(w, cb, ta, g.N, rin); break;
          }
        } else {
          switch (rem) {
            case 0: write_row<BB, 0, false>(w, cb, ta, g.N, rin); break;
            case 1: write_row<BB, 1, false>(w, cb, ta, g.N, rin); break;
            case 2: write_row<BB, 2, false>(w, cb, ta, g.N, rin); break;
            default: write_row<BB, 3, false>(w, cb, ta, g.N, rin); break;
          }
        }
      } else {
        if (qa > 0) {
          r = wait_phase(&empty_a[grp], (qa & 1u) ^ 1u, fail);
          if (__reduce_max_sync(0xffffffffu, (unsigned)r)) { if (r == 2) bad |= QAMW_STATUS_TIMEOUT; failed = true; break; }
          tc_fence_after();
        }
        bad |= write_row_any(rowp, rem, B, cb, ta, check_idx, g.N, rin);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_w[sw]);
      }
      tmem_st_wait();   // the tile's tensor-memory stores are done
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_a[grp]);
      for (int k = 0; k < SA; ++k) cur.next(n_chunks, g.n_m);
      ++qa;
      sw += SA;
      if (sw >= SW) { sw -= SW; ++qw; }
    }
  } else if (warp == kWarpWords) {
    // ---- packed words of each unit -> word stage (u - u0) % SW
    int sw = 0;
    uint32_t pw = 0;
    int64_t issued = 0;
    Cursor cur(u0, n_chunks, g.n_m);
    for (int64_t u = u0; u < u1; ++u, cur.next(n_chunks, g.n_m)) {
      const int c = cur.c;
      const int64_t m0 = cur.mt * kBM;
      if (u - u0 >= SW) {
        const int r = wait_phase(&empty_w[sw], pw ^ 1u, fail);
        if (__reduce_max_sync(0xffffffffu, (unsigned)r)) { if (r == 2) bad |= QAMW_STATUS_TIMEOUT; failed = true; break; }
      }
      unsigned char *dst = W0 + (size_t)sw * L.wpitch;
      if (g.words_tma) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&full_w[sw], (uint32_t)(kBM * g.BW * 4));
          tma_load_2d(dst, &wmap, (c * 2 * B) & ~3, (int)m0, &full_w[sw]);
        }
      } else {
        // a row's 2B words of the chunk, 4 bytes at a time; rows past M are
        // not copied (their stale words decode to centroids of rows that are
        // never written)
        for (int row = lane; row < kBM; row += 32) {
          if (m0 + row < g.M) {
            const uint32_t *src = g.packed + (m0 + row) * g.wpr + (int64_t)c * 2 * B;
            uint32_t *d = reinterpret_cast<uint32_t *>(dst) + row * g.BW;
            for (int k = 0; k < 2 * B; ++k) cp_async4(d + k, src + k);
          }
        }
        cp_async_arrive_noinc(&full_w[sw]);
      }
      issued = u - u0 + 1;
      if (++sw == SW) { sw = 0; pw ^= 1u; }
    }
    if (failed) {   // copies still in flight land before the CTA exits
      if (g.words_tma) {
        if (lane == 0)
          for (int64_t i = (issued > SW ? issued - SW : 0); i < issued; ++i)
            mbar_wait(&full_w[i % SW], (uint32_t)((i / SW) & 1), kWaitTries);
      } else {
        cp_async_wait<0>();
      }
    }
  } else if (warp == kWarpX) {
    // ---- activation tile of each unit -> activation stage (u - u0) % SA, the
    // one beside the unit's operand stage: its copies complete on the same
    // full barrier as the decode group's tile (one wait for the MMA warp), and
    // the stage is free again when that tile's MMAs are (empty_a)
    if (lane == 0) {
      int sx = 0;
      uint32_t px = 0;
      int64_t issued = 0;
      griddep_wait();   // the a tiles are kernel 1's output
      Cursor cur(u0, n_chunks, g.n_m);
      for (int64_t u = u0; u < u1; ++u, cur.next(n_chunks, g.n_m)) {
        const int c = cur.c;
        const int64_t t0 = cur.tt * NT;
        if (u - u0 >= SA) {
          const int r = wait_phase(&empty_a[sx], px ^ 1u, fail);
          if (r) { if (r == 2) bad |= QAMW_STATUS_TIMEOUT; failed = true; break; }
        }
        unsigned char *dst = X0 + (size_t)sx * L.stage_x;
        mbar_arrive_expect_tx(&full_a[sx], (uint32_t)L.stage_x);
        tma_load_2d(dst, &xmap, c * kBK, (int)t0, &full_a[sx]);                   // atom 0: NT x 64 columns
        tma_load_2d(dst + NT * 128, &xmap, c * kBK + kAtom, (int)t0, &full_a[sx]);  // atom 1
        issued = u - u0 + 1;
        if (++sx == SA) { sx = 0; px ^= 1u; }
      }
      // copies still in flight land before the CTA exits (bounded: the phase
      // also waits for the decode group, which may have stopped)
      if (failed)
        for (int64_t i = (issued > SA ? issued - SA : 0); i < issued; ++i)
          mbar_wait(&full_a[i % SA], (uint32_t)((i / SA) & 1), kWaitTries);
    }
  } else if (warp == kWarpMma || warp == kWarpMma2) {
    // ---- MMA issue; segment = the CTA's units of one tile, accumulated in
    // buffer seg % nbuf. With ni = 2 MMA warp mi issues the 4 MMAs of atom mi
    // of every unit into accumulator mi: two issuers halve the serial chain of
    // one thread (each of its tensor and shared-memory instructions queues
    // behind the decode warps' gathers)
    const int mi = warp == kWarpMma ? 0 : 1;
    if (lane == 0 && mi < (int)ni) {
      // instruction descriptor: fp32 accumulator, fp16 A and B, both K-major, N = NT, M = 128
      const uint32_t idesc = (1u << 4) | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
      int sa = 0;
      uint32_t pa = 0;
      int64_t seg = 0;
      bool any = false;
      int c = (int)(u0 % n_chunks);
      for (int64_t u = u0; u < u1; ++u, c = (c + 1 == n_chunks) ? 0 : c + 1) {
        const bool first = (u == u0) || (c == 0);
        const bool last = (u + 1 == u1) || (c == n_chunks - 1);
        const uint32_t buf = (uint32_t)seg & (nbuf - 1);
        int r = 0;
        if (first && seg >= nbuf) r = wait_phase(&acc_empty[buf], (uint32_t)(((seg >> lbuf) - 1) & 1), fail);
        if (!r) r = wait_phase(&full_a[sa], pa, fail);   // the operand tile and the activation tile
        if (r) { if (r == 2) bad |= QAMW_STATUS_TIMEOUT; failed = true; break; }
        tc_fence_after();
        // descriptors of the stage's first atoms; a step along K adds its byte
        // offset / 16 to the start-address field (no carry: shared-memory
        // addresses stay below 2^18)
        const uint32_t ta0 = tmem + a_col0 + 64 * sa;
        const uint64_t bd0 = smem_desc_sw128(smem_u32(X0 + (size_t)sa * L.stage_x));
        const uint32_t d = tmem + (buf * ni + mi) * acc_cols;
        const int kb = 4 * mi, nk = (kBK / 16) / ni;   // this warp's K steps: kb .. kb + nk - 1
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          if (kk >= nk) break;
          const int k16 = kb + kk;
          // atom k16 / 4 (16 KB apart in A, NT x 128 B in the activations);
          // 16 columns = 32 bytes along its swizzled rows
          const uint64_t bd = bd0 + (uint64_t)((k16 >> 2) * (NT * 128 / 16) + (k16 & 3) * 2);
          mma_f16_ts(d, ta0 + 8 * k16, bd, idesc, (!first || kk > 0) ? 1u : 0u);   // 16 columns of A = 8 tensor-memory columns
        }
        mma_commit(&empty_a[sa]);   // frees the operand stage and the activation stage
        any = true;
        if (last) {
          mma_commit(&acc_full[buf]);
          ++seg;
        }
        if (++sa == SA) { sa = 0; pa ^= 1u; }
      }
      if (any) {   // every MMA issued completes before the tensor memory is freed
        const int ls = (sa + SA - 1) % SA;                  // stage of the last committed unit
        mbar_wait(&empty_a[ls], sa == 0 ? (pa ^ 1u) : pa, kWaitTries);
      }
    }
  } else {
    // ---- epilogue warps: lanes 32 (warp % 4) .. + 31 of tensor memory = rows of the tile
    const int wq = warp & 3;
    const int row = 32 * wq + lane;
    int64_t seg = 0;
    int64_t u = u0;
    griddep_wait();   // the token factors and the cleared counters are kernel 1's output
    while (u < u1) {
      const int64_t tile = u / n_chunks, c_begin = u - tile * n_chunks;
      const int64_t seg_end = (u1 < (tile + 1) * n_chunks) ? u1 : (tile + 1) * n_chunks;
      const bool whole = c_begin == 0 && seg_end == (tile + 1) * n_chunks;
      const uint32_t buf = (uint32_t)seg & (nbuf - 1);
      // one decision for all 4 warps: the partial-sum path below holds their named barriers
      const int r = wait_phase_sleep(&acc_full[buf], (uint32_t)((seg >> lbuf) & 1), fail);
      if (epi_any(r != 0)) { if (r == 2) bad |= QAMW_STATUS_TIMEOUT; failed = true; break; }
      tc_fence_after();
      const int64_t tt = tile / g.n_m;
      const int64_t m = (tile - tt * g.n_m) * kBM + row;
      const int64_t t0 = tt * NT;
      const float rn = m < g.M ? g.row_norm[m] : 0.0f;
      if (m < g.M && !isfinite(rn)) bad |= QAMW_STATUS_NONFINITE_NORM;
      const uint32_t taddr = tmem + buf * ni * acc_cols + ((uint32_t)(32 * wq) << 16);
      if (whole) {
        for (int c0 = 0; c0 < NT; c0 += 16) {
          float v[16];
          tmem_ld_acc(taddr + (uint32_t)c0, ni, acc_cols, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int64_t t = t0 + c0 + j;
            if (m < g.M && t < g.T) g.Y[t * g.ldy + m] = (v[j] * rn) * g.tok_scale[t];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
      } else {
        // a part of the tile: this CTA's slot is 0 if the part is its first
        // segment, else 1; the CTA that completes the tile adds all parts in
        // the order of their CTAs
        const int slot = (u == u0) ? 0 : 1;
        float *mine = g.part + ((size_t)(2 * blockIdx.x + slot) * NT) * kBM;
        for (int c0 = 0; c0 < NT; c0 += 16) {
          float v[16];
          tmem_ld_acc(taddr + (uint32_t)c0, ni, acc_cols, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) mine[(size_t)(c0 + j) * kBM + row] = v[j];
        }
        // with two accumulator buffers this one stays held until the part sum
        // below, which then reads this CTA's own part from tensor memory
        // instead of back from the workspace (the same values); with one, the
        // next tile's MMAs need it at once
        const bool hold = nbuf == 2;
        if (!hold) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
        const int64_t b_first = cta_of_unit(tile * n_chunks, G, g.n_units);
        const int64_t b_last = cta_of_unit((tile + 1) * n_chunks - 1, G, g.n_units);
        epi_sync();   // the 4 warps' partial sums are written
        if (threadIdx.x == kWarpEpi * 32) {
          // release: this CTA's partial sums (ordered before it by the barrier)
          // are visible with its count; acquire: the last contributor sees all
          // the others' (and passes them on to its warps through the barrier)
          const uint32_t old = atom_add_acq_rel(&g.counters[tile], 1u);
          s_last = (old == (uint32_t)(b_last - b_first)) ? 1 : 0;
        }
        epi_sync();
        if (s_last) {
          for (int c0 = 0; c0 < NT; c0 += 16) {
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
            for (int64_t b = b_first; b <= b_last; ++b) {
              if (hold && b == (int64_t)blockIdx.x) {   // 8 columns at a time: few live registers
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  float v[8];
                  tmem_ld8(taddr + (uint32_t)(c0 + 8 * h), v);
                  if (ni == 2) {
                    float v2[8];
                    tmem_ld8(taddr + acc_cols + (uint32_t)(c0 + 8 * h), v2);
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[j] += v2[j];
                  }
#pragma unroll
                  for (int j = 0; j < 8; ++j) acc[8 * h + j] += v[j];
                }
                continue;
              }
              // CTA b holds this tile in its first segment unless its range
              // began in an earlier tile (only b_first can have)
              const int sl = (b == b_first && range_start(b, G, g.n_units) < tile * n_chunks) ? 1 : 0;
              const float *pp = g.part + ((size_t)(2 * b + sl) * NT) * kBM;
#pragma unroll
              for (int j = 0; j < 16; ++j) acc[j] += __ldcg(pp + (size_t)(c0 + j) * kBM + row);
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int64_t t = t0 + c0 + j;
              if (m < g.M && t < g.T) g.Y[t * g.ldy + m] = (acc[j] * rn) * g.tok_scale[t];
            }
          }
        }
        if (hold) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
        epi_sync();   // s_last is read by all before the next part overwrites it
      }
      ++seg;
      u = seg_end;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols)
                              : "memory");
  bad = __reduce_or_sync(0xffffffffu, bad);
  if (lane == 0) status_or(g.status, bad);
}

}  // namespace

size_t decode_matmul_workspace_bytes(int64_t M, int64_t K, int64_t T) { return ws_layout(M, K, T).total; }

cudaError_t launch_decode_gemm(const DecodeArgs &d, const uint16_t *X, int64_t T, int64_t ldx, float *Y, int64_t ldy,
                               void *workspace, cudaStream_t s) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  int dev = 0, smem_max = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const WsLayout W = ws_layout(d.M, d.K, T);
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  __half *A = reinterpret_cast<__half *>(ws);
  float *tok_scale = reinterpret_cast<float *>(ws + W.off_scale);
  uint32_t *counters = reinterpret_cast<uint32_t *>(ws + W.off_cnt);
  float *part = reinterpret_cast<float *>(ws + W.off_part);

  // ---- kernel 2 shapes (kernel 1 clears its tile counters)
  GemmArgs g;
  g.packed = d.packed;
  g.row_norm = d.row_norm;
  g.codebook = d.codebook;
  g.tok_scale = tok_scale;
  g.counters = counters;
  g.part = part;
  g.Y = Y;
  g.ldy = ldy;
  g.M = d.M;
  g.K = d.K;
  g.T = T;
  g.wpr = d.wpr;
  g.N = d.N;
  g.bits = d.bits;
  g.status = d.status;
  const int B = d.bits;
  // the packed words by TMA when the row pitch is a multiple of 16 bytes: a
  // chunk's 2B words start at word 2Bc, 0 to 3 words past a 16-byte boundary;
  // cp.async copies place them at the start of the staged row. The thread of
  // the second half reads 16-byte groups from the one holding word B + 3 at
  // most, enough of them to cover 3 + B words: the row holds both reads.
  g.words_tma = ((d.wpr * 4) % 16 == 0 && reinterpret_cast<uintptr_t>(d.packed) % 16 == 0) ? 1 : 0;
  g.BW = ((B + 3) & ~3) + ((B + 3 + 3) & ~3);
  if ((g.BW / 4) % 2 == 0) g.BW += 4;   // an odd number of 16-byte groups per row: rows hit different banks
  // kernel 1's CTA shape: a cluster of up to 8 CTAs per token for few tokens
  // (its latency is on the critical path), one CTA per token from 512 tokens
  // on (enough CTAs to fill the GPU without clusters); for few tokens kernel
  // 2 leaves shared memory to one CTA of kernel 1, so that it can start
  // beside it
  const int ucols = d.log2b > 9 ? (1 << d.log2b) : 512;
  const int64_t prep_units = (d.K + ucols - 1) / ucols;
  const int prep_S = T >= 512 ? 1 : (int)std::min<int64_t>(kPrepCluster, prep_units);
  const size_t prep_smem = (size_t)((prep_units + prep_S - 1) / prep_S) * ucols * 4;
  const int64_t budget = (int64_t)smem_max - 1024 - 256 - (prep_S > 1 ? (int64_t)prep_smem + 2048 : 0);
  // two decode groups, each with its operand stage (tensor memory) and
  // activation stage (shared memory); the widest token tile (<= 256, a
  // multiple of 16) and, for it, the most word stages per group (4, 2, 1)
  // that fit (the smallest shape fits every code size and N <= 8192 at
  // NT = 16: at most 76 KB)
  const int SA = 2;
  auto fits = [&](int nt, int sw) { return (int64_t)gemm_smem(nt, SA, sw, g.BW, d.N).total <= budget; };
  int NT = nt_cap(T), SW = 0;
  for (; NT >= 16 && SW == 0; NT -= 16) {
    for (const int sw : {4 * SA, 2 * SA, SA}) {
      if (fits(NT, sw)) {
        SW = sw;
        break;
      }
    }
    if (SW != 0) break;
  }
  if (SW == 0) return cudaErrorNotSupported;
  g.NT = NT;
  g.SA = SA;
  g.SW = SW;
  g.n_m = (d.M + kBM - 1) / kBM;
  const int64_t n_tiles = g.n_m * ((T + NT - 1) / NT);
  g.n_units = n_tiles * (d.K / kBK);
  const int64_t G = std::min<int64_t>(std::min<int64_t>(sm_count(), kMaxCtas), g.n_units);

  // everything on the host first (tensor maps, attributes), so that the two
  // launches follow each other at once: kernel 2 starts beside kernel 1
  CUtensorMap xmap, wmap;
  {
    cuuint64_t dims[2] = {(cuuint64_t)d.K, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)d.K * 2};
    cuuint32_t box[2] = {(cuuint32_t)kAtom, (cuuint32_t)NT};
    cuuint32_t es[2] = {1, 1};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, A, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (g.words_tma) {
    cuuint64_t dims[2] = {(cuuint64_t)d.wpr, (cuuint64_t)d.M};
    cuuint64_t strides[1] = {(cuuint64_t)d.wpr * 4};
    cuuint32_t box[2] = {(cuuint32_t)g.BW, (cuuint32_t)kBM};
    cuuint32_t es[2] = {1, 1};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(d.packed), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    wmap = xmap;   // unused
  }
  const size_t smem = 1024 + gemm_smem(NT, SA, SW, g.BW, d.N).total;
  // 11- and 10-bit codes compiled for their shape; anything else at run time
  const void *kfn = B == 11   ? reinterpret_cast<const void *>(decode_gemm_kernel<11>)
                    : B == 10 ? reinterpret_cast<const void *>(decode_gemm_kernel<10>)
                              : reinterpret_cast<const void *>(decode_gemm_kernel<0>);
  if ((e = set_max_dynamic_smem(kfn, smem)) != cudaSuccess) return e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void *>(prepare_x_kernel), prep_smem)) != cudaSuccess) return e;

  // ---- kernel 1: a cluster of S CTAs per token
  {
    PrepArgs p;
    p.X = X;
    p.ldx = ldx;
    p.T = T;
    p.K = d.K;
    p.sigma = d.sigma;
    p.col_scale = d.col_scale;
    p.seed = d.seed;
    p.log2b = d.log2b;
    p.A = A;
    p.tok_scale = tok_scale;
    p.counters = counters;
    p.n_counters = n_tiles;
    p.S = prep_S;
    const size_t smem = prep_smem;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.S * T), 1, 1);
    cfg.blockDim = dim3(kPrepThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p.S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, prepare_x_kernel, p)) != cudaSuccess) return e;
  }


  auto run = [&](auto kern) -> cudaError_t {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)G, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, xmap, wmap, g);
  };
  if (B == 11) return run(decode_gemm_kernel<11>);
  if (B == 10) return run(decode_gemm_kernel<10>);
  return run(decode_gemm_kernel<0>);
}

}  // namespace qamw
