// qamw_encode_polar.cu -- the polar baseline codec's encode ("QAM-W: Joint 2D
// Codebook Quantization for LLM Weights ...", Results, "Joint 2D vs. Polar":
// amplitude and phase of each normalised pair quantized independently, at
// the same rate as the joint 2D codebook).
//
// Steps (5), (1), (2), (3) are the 512-column pipeline of
// qamw_encode_unit.cuh, bit for bit the same x as the joint codec; step (4)
// is replaced by the polar quantizer, decided in fp64 from the fp32 pair:
//   a = number of amplitude edges e_i = (amp_i + amp_{i+1}) / 2 below
//       hypot(x0, x1)                      (nearest of the A levels),
//   p = floor(atan2(x1, x0) mod 2 pi / (2 pi / P)) mod P   (the phase sector),
//   index = a * P + p.
// The reconstruction point of index a*P + p is amp_a * (cos, sin)(2 pi (p + 1/2) / P),
// so the joint codec's decode (qamw_decode) decodes this stream given those
// points as its codebook.
#include <algorithm>
#include <cmath>

#include "qamw_encode_unit.cuh"

namespace qamw {
namespace {

constexpr double kTwoPi = 2.0 * 3.141592653589793;

struct PolarSearch {
  const double *edges;   // A - 1 amplitude decision edges, ascending
  int A1, P;
  double w;              // sector width 2 pi / P

  __device__ __forceinline__ void search8(const float (&x0)[8], const float (&x1)[8], int (&idx)[8]) const {
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const double X = (double)x0[p], Y = (double)x1[p];
      const double rad = hypot(X, Y);
      int lo = 0, hi = A1;   // count of edges < rad, by bisection
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (edges[mid] < rad) lo = mid + 1;
        else hi = mid;
      }
      double ang = atan2(Y, X);
      if (ang < 0.0) ang += kTwoPi;
      int sp = (int)floor(ang / w);
      sp %= P;
      if (sp < 0) sp += P;
      idx[p] = lo * P + sp;
    }
  }
};

template <int WT>
__global__ void __launch_bounds__(kEncThreads, 1) encode_polar_kernel(EncodeArgs a, int vec_ok) {
  extern __shared__ __align__(16) unsigned char smem[];
  double *edges = reinterpret_cast<double *>(smem + kUnitSmemBytes);
  const int A1 = a.polar_A - 1;
  for (int i = threadIdx.x; i < A1; i += kEncThreads) edges[i] = (a.polar_amps[i] + a.polar_amps[i + 1]) * 0.5;
  // encode_units synchronises the CTA before the first pair is quantized
  const PolarSearch S{edges, A1, a.polar_P, kTwoPi / (double)a.polar_P};
  encode_units<WT, 0, 0>(a, vec_ok, smem, S);
}

template <int WT>
cudaError_t launch_t(const EncodeArgs &a, cudaStream_t s) {
  const size_t smem = kUnitSmemBytes + (size_t)std::max(a.polar_A - 1, 1) * sizeof(double);
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(encode_polar_kernel<WT>), smem);
  if (e != cudaSuccess) return e;
  const int64_t n_chunks = (a.rot.K + kUnit - 1) / kUnit;
  const int64_t tiles = n_chunks * ((a.rot.M + kEncWarps - 1) / kEncWarps);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(tiles, sm_count()));
  const size_t es = (WT == QAMW_BF16) ? 2 : 4;
  const int vec = ((reinterpret_cast<uintptr_t>(a.rot.W) % 16) == 0 && (a.rot.ldw * (int64_t)es) % 16 == 0) ? 1 : 0;
  encode_polar_kernel<WT><<<(int)blocks, kEncThreads, smem, s>>>(a, vec);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode_polar(const EncodeArgs &a, cudaStream_t s) {
  return (a.rot.wt == QAMW_BF16) ? launch_t<QAMW_BF16>(a, s) : launch_t<QAMW_F32>(a, s);
}

}  // namespace qamw
