// qamw_lloyd.cu -- Lloyd training of the 2D codebook on the GPU.
//
// "QAM-W: Joint 2D Codebook Quantization for LLM Weights via Hadamard
// Rotation and Activation-Aware Scaling", Technical Summary, Methodology (4)
// Joint 2D Quantization, and "Significance and Claims": the codebook is a 2D
// Lloyd-Max quantizer trained once on samples of the unit circular Gaussian.
// One Lloyd iteration alternates
//   * assignment: every sample goes to its nearest centroid (Euclidean,
//     lowest index on ties), and
//   * update: every centroid moves to the mean of its samples; a centroid
//     with no sample keeps its place;
// training stops when an assignment pass changes no sample (or after
// max_iter passes). Samples and centroids are fp64, as the distances and means
// are defined on real numbers.
//
// Assignment: one thread per sample, brute force over the N centroids held in
// shared memory, d = dx*dx + dy*dy in fp64, strict "<" (lowest index). The
// pass also counts the samples whose index changed.
// Update, deterministic: the samples are cut into B contiguous ranges, one per
// CTA; thread t of a CTA owns centroids t, t + 1024, ... and adds, in sample
// order, the samples of the range assigned to them (the range is staged in
// shared memory chunk by chunk); the B partial sums of a centroid are then
// added in range order by one thread. The result does not depend on the GPU
// or the launch.
#include <algorithm>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"

namespace qamw {
namespace {

constexpr int kAssignThreads = 256;
constexpr int kUpdThreads = 1024;
constexpr int kUpdChunk = 1024;          // samples staged per step
constexpr int kMaxOwned = QAMW_MAX_CENTROIDS / kUpdThreads;   // centroids per thread at most

__global__ void __launch_bounds__(kAssignThreads) lloyd_assign_kernel(const double2 *__restrict__ pts, int64_t T,
                                                                      const double2 *__restrict__ cent, int N,
                                                                      int32_t *__restrict__ idx,
                                                                      unsigned long long *changed) {
  extern __shared__ double2 c_sh[];
  for (int i = threadIdx.x; i < N; i += blockDim.x) c_sh[i] = cent[i];
  __syncthreads();
  unsigned int chg = 0;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < T; t += (int64_t)gridDim.x * blockDim.x) {
    const double2 p = pts[t];
    double best = INFINITY;
    int bi = 0;
#pragma unroll 4
    for (int c = 0; c < N; ++c) {
      const double2 q = c_sh[c];
      const double dx = p.x - q.x, dy = p.y - q.y;
      const double d = __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy));
      if (d < best) {
        best = d;
        bi = c;
      }
    }
    if (idx[t] != bi) ++chg;
    idx[t] = bi;
  }
  for (int o = 16; o > 0; o >>= 1) chg += __shfl_xor_sync(0xffffffffu, chg, o);
  if ((threadIdx.x & 31) == 0 && chg != 0 && changed != nullptr) atomicAdd(changed, (unsigned long long)chg);
}

// Partial sums {sum x, sum y, count} of range b for every centroid; each
// thread owns KO centroids (KO = ceil(N / 1024)).
template <int KO>
__global__ void __launch_bounds__(kUpdThreads) lloyd_partial_kernel(const double2 *__restrict__ pts, int64_t T,
                                                                    const int32_t *__restrict__ idx, int N,
                                                                    double *__restrict__ part) {
  __shared__ double2 s_pts[kUpdChunk];
  __shared__ int32_t s_idx[kUpdChunk];
  const int64_t lo = blockIdx.x * T / gridDim.x, hi = (blockIdx.x + 1) * T / gridDim.x;
  double sx[KO], sy[KO], cn[KO];
#pragma unroll
  for (int k = 0; k < KO; ++k) { sx[k] = 0.0; sy[k] = 0.0; cn[k] = 0.0; }
  for (int64_t base = lo; base < hi; base += kUpdChunk) {
    const int n = (int)std::min<int64_t>(kUpdChunk, hi - base);
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += kUpdThreads) {
      s_pts[j] = pts[base + j];
      s_idx[j] = idx[base + j];
    }
    __syncthreads();
    for (int j = 0; j < n; ++j) {
      const int id = s_idx[j];
      if (id >= 0 && id < N && (id & (kUpdThreads - 1)) == (int)threadIdx.x) {
        const int k = id / kUpdThreads;
        const double2 p = s_pts[j];
#pragma unroll
        for (int q = 0; q < KO; ++q)
          if (q == k) { sx[q] += p.x; sy[q] += p.y; cn[q] += 1.0; }
      }
    }
  }
#pragma unroll
  for (int k = 0; k < KO; ++k) {
    const int c = (int)threadIdx.x + k * kUpdThreads;
    if (c < N) {
      double *d = part + ((int64_t)blockIdx.x * N + c) * 3;
      d[0] = sx[k];
      d[1] = sy[k];
      d[2] = cn[k];
    }
  }
}

// Centroid c = mean of its samples (ranges added in order); empty keeps c.
__global__ void lloyd_reduce_kernel(const double *__restrict__ part, int B, int N, double2 *cent,
                                    int32_t *empty_count) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= N) return;
  double sx = 0.0, sy = 0.0, cn = 0.0;
  for (int b = 0; b < B; ++b) {
    const double *d = part + ((int64_t)b * N + c) * 3;
    sx += d[0];
    sy += d[1];
    cn += d[2];
  }
  if (cn > 0.0) {
    cent[c] = make_double2(sx / cn, sy / cn);
  } else if (empty_count != nullptr) {
    atomicAdd(empty_count, 1);
  }
}

// About 16 k samples per range, at most 256 ranges: a function of T alone, so
// the order of every sum is the same on any GPU.
int update_ranges(int64_t T) {
  const int64_t r = (T + 16383) / 16384;
  return (int)std::max<int64_t>(1, std::min<int64_t>(r, 256));
}

}  // namespace

size_t lloyd_workspace_bytes(int64_t T, int N) {
  // partials [B][N][3] doubles | changed counter (8) | empty counter (4), 256-byte aligned
  const size_t part = (size_t)update_ranges(T) * (size_t)N * 3 * sizeof(double);
  return ((part + 255) & ~size_t(255)) + 256;
}

cudaError_t launch_lloyd_assign(const double *pts, int64_t T, const double *cent, int N, int32_t *idx,
                                unsigned long long *changed, cudaStream_t s) {
  const size_t smem = (size_t)N * sizeof(double2);
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(lloyd_assign_kernel), smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((T + kAssignThreads - 1) / kAssignThreads,
                                                                (int64_t)sm_count() * 8));
  lloyd_assign_kernel<<<(int)blocks, kAssignThreads, smem, s>>>(reinterpret_cast<const double2 *>(pts), T,
                                                              reinterpret_cast<const double2 *>(cent), N, idx,
                                                              changed);
  return cudaGetLastError();
}

cudaError_t launch_lloyd_update(const double *pts, int64_t T, const int32_t *idx, int N, double *cent,
                                void *workspace, int32_t *empty_count, cudaStream_t s) {
  const int B = update_ranges(T);
  double *part = static_cast<double *>(workspace);
  const double2 *p2 = reinterpret_cast<const double2 *>(pts);
  const int ko = (N + kUpdThreads - 1) / kUpdThreads;
  if (ko <= 1) lloyd_partial_kernel<1><<<B, kUpdThreads, 0, s>>>(p2, T, idx, N, part);
  else if (ko <= 2) lloyd_partial_kernel<2><<<B, kUpdThreads, 0, s>>>(p2, T, idx, N, part);
  else if (ko <= 4) lloyd_partial_kernel<4><<<B, kUpdThreads, 0, s>>>(p2, T, idx, N, part);
  else lloyd_partial_kernel<kMaxOwned><<<B, kUpdThreads, 0, s>>>(p2, T, idx, N, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  lloyd_reduce_kernel<<<(N + 255) / 256, 256, 0, s>>>(part, B, N, reinterpret_cast<double2 *>(cent), empty_count);
  return cudaGetLastError();
}

}  // namespace qamw
