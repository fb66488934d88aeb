// qamw_encode_pruned.cu -- QAM-W encode with the exact pruned
// nearest-centroid search, for Hadamard blocks b <= 512.
//
// Method: "QAM-W: Joint 2D Codebook Quantization for LLM Weights via Hadamard
// Rotation and Activation-Aware Scaling", Technical Summary, "Methodology:
// The QAM-W Codec": normalise by the stored row norm (step 1), sign-masked
// block Hadamard rotation (step 2), x = z / sigma (step 3), nearest centroid
// (step 4) with the channel scale s_j applied first (step 5), then bit packing.
//
// Work decomposition. A *unit* is one row x 512 consecutive columns handled by
// one warp: lane l owns columns [16l, 16l + 16) of the unit (8 pairs); the
// rotation is the fp64 one of qamw_rotate16.cuh, which gives the same x bit
// for bit as the 1024-column kernel of qamw_encode.cu. A CTA of 28 warps takes a contiguous
// range of *tiles* (28 rows x one 512-column chunk) in chunk-major order; the
// chunk's d_j * s_j and 1 / sigma_k live once per CTA in shared memory, next
// to the codebook and the search table. The next unit's weights are loaded
// while the current one is searched.
//
// Search. The pair's cell of the search table (qamw_search.cu) lists every
// centroid that can be an fp32 minimiser, in ascending index order; a strict
// "<" over the list keeps the lowest index among equal distances, which is the
// brute-force result. In shared memory the lists follow an identity list
// 0..N-1, which a pair outside the grid (or every pair, if the table does not
// fit or does not match the codebook) scans instead.
#include <algorithm>
#include <cfloat>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"
#include "qamw_encode_unit.cuh"

namespace qamw {
namespace {

constexpr int kThreads = kUnitThreads;

// The exact pruned search over the codebook's grid table (see the file comment).
struct PrunedSearch {
  const float2 *cb2;
  const uint16_t *toff, *lst;
  bool use;
  int G, N;
  float a_ax, UL, inv_cw, Gf;

  __device__ __forceinline__ void search8(const float (&x0)[8], const float (&x1)[8], int (&idx)[8]) const {
    // candidate ranges of the 8 pairs (cell lists, or the identity list),
    // without branches: an off-grid pair reads cell 0 and discards it
    int beg[8], end[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const float u0 = __fdividef(x0[p], __fadd_rn(a_ax, fabsf(x0[p])));
      const float u1 = __fdividef(x1[p], __fadd_rn(a_ax, fabsf(x1[p])));
      const float fx = __fmul_rn(__fadd_rn(u0, UL), inv_cw);
      const float fy = __fmul_rn(__fadd_rn(u1, UL), inv_cw);
      const bool in = use && fx >= 0.0f && fx < Gf && fy >= 0.0f && fy < Gf;
      const int cell = in ? (int)fy * G + (int)fx : 0;
      const int b0 = toff[cell], e0 = toff[cell + 1];
      beg[p] = in ? b0 : 0;
      end[p] = in ? e0 : N;
    }
    // Every list has at least one entry. A single-entry list is the answer
    // without a distance (30% of the pairs on the 4096^2 projection, whose
    // lanes then issue no codebook read); otherwise the first entry's distance
    // starts the strict "<" scan of the rest. The first entry of the identity
    // list is index 0, so an off-grid pair whose distances all overflow to
    // +inf still gets index 0, as in the brute-force search.
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const int e = end[p];
      int j = beg[p];
      int bi = lst[j];
      if (e - j > 1) {
        const float2 c0 = cb2[bi];
        float best = dist2_scalar(x0[p], x1[p], c0.x, c0.y);
        // one to a few iterations: not unrolled (an unrolled body with its
        // remainder loop measured 6 us slower on the 4096^2 projection)
#pragma unroll 1
        for (++j; j < e; ++j) {
          const int i0 = lst[j];
          const float2 c = cb2[i0];
          const float d0 = dist2_scalar(x0[p], x1[p], c.x, c.y);
          if (d0 < best) { best = d0; bi = i0; }
        }
      }
      idx[p] = bi;
    }
  }
};

template <int WT>
__global__ void __launch_bounds__(kThreads, 1)
    encode_pruned_kernel(EncodeArgs a, int vec_ok, int tab_cap, int toff_slots) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = a.N;
  const int n2 = (N + 1) & ~1;
  float2 *cb2 = reinterpret_cast<float2 *>(smem + kUnitSmemBytes);
  uint16_t *toff = reinterpret_cast<uint16_t *>(cb2 + n2);
  uint16_t *lst = toff + toff_slots;   // identity list 0..N-1, then the cell lists

  __shared__ int s_use, s_G;
  __shared__ float s_a, s_UL, s_inv;
  if (threadIdx.x == 0) {
    const SearchHeader h = *reinterpret_cast<const SearchHeader *>(a.table);
    const bool ok = h.magic == kSearchMagic && h.valid == 1 && h.N == N && h.G >= 1 && h.G <= 181 &&
                    h.G * h.G + 1 <= toff_slots && h.total >= 0 && h.total <= tab_cap - N &&
                    h.total + N < 65536 && h.a > 0.0f && h.UL > 0.0f && h.UL < 1.0f && h.inv_cw > 0.0f;
    s_use = ok ? 1 : 0;
    s_G = h.G;
    s_a = h.a;
    s_UL = h.UL;
    s_inv = h.inv_cw;
  }
  for (int c = threadIdx.x; c < n2; c += kThreads)
    cb2[c] = (c < N) ? make_float2(a.codebook[2 * c], a.codebook[2 * c + 1]) : make_float2(0.0f, 0.0f);
  for (int i = threadIdx.x; i < N; i += kThreads) lst[i] = (uint16_t)i;
  __syncthreads();
  const bool use = s_use != 0;
  const int G = s_G;
  if (use) {
    const uint32_t *goff = reinterpret_cast<const uint32_t *>(reinterpret_cast<const unsigned char *>(a.table) +
                                                              sizeof(SearchHeader));
    const uint16_t *gcand = reinterpret_cast<const uint16_t *>(goff + G * G + 1);
    // clamped on the copy, so that no table content can index outside the
    // lists or the codebook
    const uint32_t total = goff[G * G] < (uint32_t)(tab_cap - N) ? goff[G * G] : (uint32_t)(tab_cap - N);
    for (int i = threadIdx.x; i <= G * G; i += kThreads)
      toff[i] = (uint16_t)((goff[i] < total ? goff[i] : total) + (uint32_t)N);
    for (int i = threadIdx.x; i < (int)total; i += kThreads)
      lst[N + i] = (gcand[i] < (uint16_t)N) ? gcand[i] : (uint16_t)(N - 1);
  }
  const float a_ax = s_a, UL = s_UL, inv_cw = s_inv, Gf = (float)G;

  const PrunedSearch S{cb2, toff, lst, use, G, N, a_ax, UL, inv_cw, Gf};
  encode_units<WT>(a, vec_ok, smem, S);
}

template <typename Kern>
cudaError_t set_smem(Kern k, size_t bytes) {
  return set_max_dynamic_smem(reinterpret_cast<const void *>(k), bytes);
}

template <int WT>
cudaError_t launch_t(const EncodeArgs &a, cudaStream_t s) {
  int dev = 0, smem_max = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const int G = search_grid(a.N);
  const int toff_slots = (G * G + 1 + 7) & ~7;
  const int n2 = (a.N + 1) & ~1;
  const size_t base = kUnitSmemBytes + (size_t)n2 * sizeof(float2) + (size_t)toff_slots * 2;
  const int64_t room = ((int64_t)smem_max - 128 /*static*/ - (int64_t)base) / 2;
  int tab_cap = (int)std::max<int64_t>(0, std::min<int64_t>(room, 65535));
  tab_cap &= ~7;
  if (tab_cap < a.N) return cudaErrorInvalidConfiguration;   // the launcher only comes here for N <= 2048
  const size_t smem = base + (size_t)tab_cap * 2;
  if ((e = set_smem(encode_pruned_kernel<WT>, smem)) != cudaSuccess) return e;
  const int64_t n_chunks = (a.rot.K + kUnit - 1) / kUnit;
  const int64_t tiles = n_chunks * ((a.rot.M + kUnitWarps - 1) / kUnitWarps);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(tiles, sm_count()));
  const size_t es = (WT == QAMW_BF16) ? 2 : 4;
  const int vec = ((reinterpret_cast<uintptr_t>(a.rot.W) % 16) == 0 && (a.rot.ldw * (int64_t)es) % 16 == 0) ? 1 : 0;
  encode_pruned_kernel<WT><<<(int)blocks, kThreads, smem, s>>>(a, vec, tab_cap, toff_slots);
  return cudaGetLastError();
}

}  // namespace

bool encode_pruned_applicable(const EncodeArgs &a) {
  return a.table != nullptr && a.rot.log2b <= 9 && a.N <= kPrunedMaxN;
}

cudaError_t launch_encode_pruned(const EncodeArgs &a, cudaStream_t s) {
  return (a.rot.wt == QAMW_BF16) ? launch_t<QAMW_BF16>(a, s) : launch_t<QAMW_F32>(a, s);
}

}  // namespace qamw
