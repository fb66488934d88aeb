// qamw_encode_pruned.cu -- QAM-W encode with the exact pruned
// nearest-centroid search, for Hadamard blocks b <= 512.
//
// Method: "QAM-W: Joint 2D Codebook Quantization for LLM Weights via Hadamard
// Rotation and Activation-Aware Scaling", Technical Summary, "Methodology:
// The QAM-W Codec": normalise by the stored row norm (step 1), sign-masked
// block Hadamard rotation (step 2), x = z / sigma (step 3), nearest centroid
// (step 4) with the channel scale s_j applied first (step 5), then bit packing.
//
// Work decomposition: the 512-column pipeline of qamw_encode_unit.cuh (a
// unit is one row x 512 columns per warp, rotated in fp64 so that x is the
// correctly rounded value; 16 warps per CTA, tiles in chunk-major order).
//
// Search. The pair's grid cell (search_cell, qamw_internal.h) has a record of
// the search table (qamw_search.cu) listing, in ascending index order, every
// centroid that can be an fp32 minimiser for a pair in the cell: up to three
// inline, longer lists continuing in an overflow array. A one-entry list is
// the answer without a distance; otherwise a strict "<" over the list keeps
// the lowest index among equal distances, which is the brute-force result. A
// pair outside the grid, or every pair if the table is invalid or does not
// fit, scans all N centroids. The records and overflow lists are copied once
// per CTA into shared memory with bulk asynchronous copies (one thread, an
// mbarrier with a bounded wait); the codebook is copied from the codebook
// argument.
#include <algorithm>
#include <cfloat>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"
#include "qamw_encode_unit.cuh"
#include "qamw_mbarrier.cuh"

namespace qamw {
namespace {

constexpr int kThreads = kEncThreads;


// The exact pruned search over the codebook's grid table (see the file comment).
struct PrunedSearch {
  const float2 *cb2;
  const uint64_t *rec;
  const uint16_t *ovf;
  bool use;
  int G, N, total;
  float a_ax, inv_cw, cbias, L;

  __device__ __forceinline__ void search8(const float (&x0)[8], const float (&x1)[8], int (&idx)[8]) const {
    // Every pair evaluates the three inline entries of its cell's record
    // without a branch: a list of one or two repeats its first entry there,
    // and a repeated entry never wins a strict "<". Listed entries are in
    // ascending index order, so the strict "<" keeps the lowest index among
    // equal distances: the brute-force result. Pairs whose list continues in
    // the overflow array, and pairs outside the grid (whose record reads as
    // "0, 0, 0" and continue over all N centroids), finish in a loop that the
    // warp enters only if one of its lanes needs it.
    float best[8];
    int meta[8];
    uint32_t more = 0;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const int cell = use ? search_cell(x0[p], x1[p], a_ax, inv_cw, cbias, L, G) : -1;
      const uint2 r = cell >= 0 ? reinterpret_cast<const uint2 *>(rec)[cell] : make_uint2(0u, 0u);
      // indices clamped below N, so that no table content can read outside the codebook
      const int e0 = min((int)(r.x & 0xffffu), N - 1), e1 = min((int)(r.x >> 16), N - 1),
                e2 = min((int)(r.y & 0xffffu), N - 1);
      meta[p] = cell >= 0 ? (int)(r.y >> 16) : -1;
      const float2 c0 = cb2[e0], c1 = cb2[e1], c2 = cb2[e2];
      float b = dist2_scalar(x0[p], x1[p], c0.x, c0.y);
      int bi = e0;
      const float d1 = dist2_scalar(x0[p], x1[p], c1.x, c1.y);
      const float d2 = dist2_scalar(x0[p], x1[p], c2.x, c2.y);
      if (d1 < b) { b = d1; bi = e1; }
      if (d2 < b) { b = d2; bi = e2; }
      best[p] = b;
      idx[p] = bi;
      if (meta[p] < 0 || (meta[p] & 3) == 0) more |= 1u << p;   // off the grid (meta = -1) or an overflow list
    }
    if (__any_sync(0xffffffffu, more != 0)) {
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        if (more & (1u << p)) {
          const bool off_grid = meta[p] < 0;
          // (clamped to the copied overflow entries)
          const int o = min(meta[p] >> 2, total - 1);
          const int kb = off_grid ? 0 : o + 1, ke = off_grid ? N : min(o + 1 + (int)ovf[max(o, 0)], total);
          float b = best[p];
          int bi = idx[p];
#pragma unroll 1
          for (int k = kb; k < ke; ++k) {
            const int ik = off_grid ? k : min((int)ovf[k], N - 1);
            const float2 c = cb2[ik];
            const float d = dist2_scalar(x0[p], x1[p], c.x, c.y);
            if (d < b) { b = d; bi = ik; }
          }
          idx[p] = bi;
        }
      }
    }
  }
};

// Shared memory after the encode pipeline's: the codebook (float2 [N], from
// the codebook argument), then the table's image (records and overflow
// lists), copied by one thread with bulk asynchronous copies.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
constexpr uint32_t kTableWaitLimit = 1u << 22;   // try_wait attempts for the table copy (far beyond its ~2 us)

template <int WT, int LB, int BB>
__global__ void __launch_bounds__(kThreads, 1) encode_pruned_kernel(EncodeArgs a, int vec_ok, int image_cap) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = a.N;
  const int n2 = (N + 1) & ~1;
  float2 *cb2 = reinterpret_cast<float2 *>(smem + kUnitSmemBytes);
  unsigned char *image = reinterpret_cast<unsigned char *>(cb2 + n2);

  __shared__ __align__(8) uint64_t s_bar;
  __shared__ int s_use, s_G, s_total;
  __shared__ float s_a, s_inv, s_L;
  if (threadIdx.x == 0) {
    const SearchHeader h = *reinterpret_cast<const SearchHeader *>(a.table);
    const int64_t rec_bytes = (int64_t)h.G * h.G * 8;
    const int64_t copy = (rec_bytes + 2 * (int64_t)h.total + 15) & ~(int64_t)15;
    bool ok = h.magic == kSearchMagic && h.valid == 1 && h.N == N && h.G >= 1 && h.G <= kSearchMaxG &&
              (h.G & 1) == 1 && h.total >= 0 && h.total <= h.capacity && copy <= h.image_bytes &&
              copy <= (int64_t)image_cap && h.a > 0.0f && h.UL > 0.0f && h.UL < 1.0f && h.inv_cw > 0.0f &&
              h.L > 0.0f;
    if (ok) {
      mbar_init(&s_bar, 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      mbar_arrive_expect_tx(&s_bar, (uint32_t)copy);
      const unsigned char *src = reinterpret_cast<const unsigned char *>(a.table) + kSearchImageOffset;
      for (int64_t o = 0; o < copy; o += 32768) {
        const uint32_t nb = (uint32_t)((copy - o) < 32768 ? (copy - o) : 32768);
        bulk_copy_g2s(image + o, src + o, nb, &s_bar);
      }
      if (!mbar_wait(&s_bar, 0, kTableWaitLimit)) {
        status_or(a.status, QAMW_STATUS_TIMEOUT);
        mbar_wait(&s_bar, 0, kTableWaitLimit);   // give the copy a second bounded chance to land
        ok = false;
      }
    }
    s_use = ok ? 1 : 0;
    s_G = ok ? h.G : 1;
    s_total = ok ? h.total : 0;
    s_a = h.a;
    s_inv = h.inv_cw;
    s_L = h.L;
  }
  for (int c = threadIdx.x; c < n2; c += kThreads)
    cb2[c] = (c < N) ? make_float2(a.codebook[2 * c], a.codebook[2 * c + 1]) : make_float2(0.0f, 0.0f);
  __syncthreads();
  const bool use = s_use != 0;
  const int G = s_G;
  const uint64_t *rec = reinterpret_cast<const uint64_t *>(image);
  const uint16_t *ovf = reinterpret_cast<const uint16_t *>(image + (size_t)G * G * 8);
  const float a_ax = s_a, inv_cw = s_inv, L = s_L;
  const float cbias = kCellMagic + (float)((G - 1) / 2);

  const PrunedSearch S{cb2, rec, ovf, use, G, N, s_total, a_ax, inv_cw, cbias, L};
  encode_units<WT, LB, BB>(a, vec_ok, smem, S);
}

template <typename Kern>
cudaError_t set_smem(Kern k, size_t bytes) {
  return set_max_dynamic_smem(reinterpret_cast<const void *>(k), bytes);
}

template <int WT, int LB, int BB>
cudaError_t launch_t(const EncodeArgs &a, cudaStream_t s) {
  int dev = 0, smem_max = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const int n2 = (a.N + 1) & ~1;
  const size_t base = kUnitSmemBytes + (size_t)n2 * sizeof(float2);
  const int64_t room = ((int64_t)smem_max - 256 /*static*/ - (int64_t)base) & ~(int64_t)15;
  if (room < 16) return cudaErrorInvalidConfiguration;
  // the image of the table (or as much of it as fits; a table that does not
  // fit makes every pair take the brute-force loop)
  const int image_cap = (int)std::min<int64_t>(room, (int64_t)search_table_bytes(a.N));
  const size_t smem = base + (size_t)image_cap;
  if ((e = set_smem(encode_pruned_kernel<WT, LB, BB>, smem)) != cudaSuccess) return e;
  const int64_t n_chunks = (a.rot.K + kUnit - 1) / kUnit;
  const int64_t tiles = n_chunks * ((a.rot.M + kEncWarps - 1) / kEncWarps);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(tiles, sm_count()));
  const size_t es = (WT == QAMW_BF16) ? 2 : 4;
  const int vec = ((reinterpret_cast<uintptr_t>(a.rot.W) % 16) == 0 && (a.rot.ldw * (int64_t)es) % 16 == 0) ? 1 : 0;
  encode_pruned_kernel<WT, LB, BB><<<(int)blocks, kThreads, smem, s>>>(a, vec, image_cap);
  return cudaGetLastError();
}

// The bf16 workloads' shapes compiled for their block size (128, 256) and
// code size (10, 11 bits); every other shape takes the run-time version.
template <int WT>
cudaError_t launch_wt(const EncodeArgs &a, cudaStream_t s) {
  if (WT == QAMW_BF16) {
    if (a.rot.log2b == 7 && a.bits == 11) return launch_t<WT, 7, 11>(a, s);
    if (a.rot.log2b == 8 && a.bits == 11) return launch_t<WT, 8, 11>(a, s);
    if (a.rot.log2b == 7 && a.bits == 10) return launch_t<WT, 7, 10>(a, s);
    if (a.rot.log2b == 8 && a.bits == 10) return launch_t<WT, 8, 10>(a, s);
  }
  return launch_t<WT, 0, 0>(a, s);
}

}  // namespace

bool encode_pruned_applicable(const EncodeArgs &a) {
  return a.table != nullptr && a.rot.log2b <= 9 && a.N <= kPrunedMaxN;
}

cudaError_t launch_encode_pruned(const EncodeArgs &a, cudaStream_t s) {
  return (a.rot.wt == QAMW_BF16) ? launch_wt<QAMW_BF16>(a, s) : launch_wt<QAMW_F32>(a, s);
}

}  // namespace qamw
