// qamw_decode_tma.cu -- the bf16 decode with Tensor Memory Accelerator I/O.
//
// Same arithmetic as qamw_decode.cu ("QAM-W: Joint 2D Codebook Quantization
// for LLM Weights ...", Methodology (6) Decoding), different data movement:
//   * packed words reach shared memory through one 2D TMA tensor load per
//     task (a box of ROWS rows x SEGS*64 columns worth of words), double
//     buffered and tracked by an mbarrier per stage;
//   * bf16 results are written into a 128-byte-swizzled staging tile and leave
//     through 2D TMA tensor stores (one per 64 columns), which clip rows and
//     columns past the matrix.
// Neither transfer occupies the load/store unit, which profiling showed to be
// the limiter of the plain-load / plain-store kernel (scattered 8-byte word
// loads touched one sector per lane; the coalescing copy-out doubled the
// shared-memory traffic of the staging).
//
// Task geometry: a warp decodes ROWS rows x SEGS segments of 64 columns with
// lane = row + ROWS * segment; each lane owns one segment of one row: 32
// indices, i.e. exactly `bits` packed words starting on a word boundary, and
// 64 fp32 values (128 registers, 16 warps per SM). SEGS is the larger
// of b/64 (the lanes of one block) and the segments whose words make a
// multiple of 16 bytes (a TMA box row must): 1 for bits % 4 == 0, 2 for even
// bits, 4 for odd bits. Block bits 1..5 are butterflies inside the lane, bits
// >= 6 across lanes (lane xor ROWS << (t - 6)) as fma(+-1, own, partner's),
// which rounds exactly like the add or subtract.
//
// Every mbarrier wait is bounded; a wait that runs out sets
// QAMW_STATUS_TIMEOUT and the kernel stops issuing work.
#include <algorithm>
#include <cmath>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "qamw_device.cuh"
#include "qamw_internal.h"
#include "qamw_mbarrier.cuh"
#include "qamw_tensor_map.h"

namespace qamw {
namespace {

constexpr int kSeg = 64;
constexpr int kMaxWarps = 16;
constexpr uint32_t kWaitLimit = 1u << 22;   // try_wait attempts before giving up

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, int x, int y, const void *src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(x),
               "r"(y), "r"(smem_u32(src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

template <int BITS>
__device__ __forceinline__ uint32_t extract_off8(const uint32_t *w, int q) {
  constexpr uint32_t mask8 = ((1u << BITS) - 1u) << 3;
  const int o = q * BITS, wi = o >> 5, sh = o & 31;
  if (sh + BITS <= 32) {
    if (sh >= 3) return (w[wi] >> (sh - 3)) & mask8;
    return (w[wi] << (3 - sh)) & mask8;
  }
  return __funnelshift_r(w[wi], w[wi + 1], sh - 3) & mask8;
}

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

template <int LB>
__device__ __forceinline__ void inlane_stages(float (&v)[kSeg]) {
  if constexpr (LB > 1) bfly_stage<1>(v);
  if constexpr (LB > 2) bfly_stage<2>(v);
  if constexpr (LB > 3) bfly_stage<3>(v);
  if constexpr (LB > 4) bfly_stage<4>(v);
  if constexpr (LB > 5) bfly_stage<5>(v);
}

// Block bit TB >= 6 across lanes: the partner holds the same columns of the
// other half; the lower lane keeps own + partner's, the upper partner's - own.
template <int TB, int ROWS>
__device__ __forceinline__ void xlane_stage(float (&v)[kSeg], int lane) {
  constexpr int h = ROWS << (TB - 6);
  const float sg = (lane & h) ? -1.0f : 1.0f;
  const float2 S = make_float2(sg, sg);
#pragma unroll
  for (int i = 0; i < kSeg; i += 2) {
    const float2 V = make_float2(v[i], v[i + 1]);
    const float2 P = make_float2(__shfl_xor_sync(0xffffffffu, v[i], h), __shfl_xor_sync(0xffffffffu, v[i + 1], h));
    const float2 o = fma2(S, V, P);
    v[i] = o.x;
    v[i + 1] = o.y;
  }
}

template <int LB, int ROWS>
__device__ __forceinline__ void xlane_stages(float (&v)[kSeg], int lane) {
  if constexpr (LB > 6) xlane_stage<6, ROWS>(v, lane);
  if constexpr (LB > 7) xlane_stage<7, ROWS>(v, lane);
  if constexpr (LB > 8) xlane_stage<8, ROWS>(v, lane);
}

#ifndef QAMW_DEC_STAGES
#define QAMW_DEC_STAGES 1
#endif
constexpr int kStages = QAMW_DEC_STAGES;   // input pipeline depth; 1 measured fastest (more stages cost warps)

template <int BITS, int LB>
struct TmaGeom {
  static constexpr int kSegsBlock = (LB > 6) ? (1 << (LB - 6)) : 1;
  static constexpr int kSegsAlign = (BITS % 4 == 0) ? 1 : ((BITS % 2 == 0) ? 2 : 4);
  static constexpr int kSegs = (kSegsBlock > kSegsAlign) ? kSegsBlock : kSegsAlign;
  static constexpr int kRows = 32 / kSegs;
  static constexpr int kLog2Rows = (kRows == 32) ? 5 : (kRows == 16) ? 4 : (kRows == 8) ? 3 : 2;
  static constexpr int kBoxWords = kSegs * BITS;              // words per row of the input box
  static constexpr int kInBytes = kRows * kBoxWords * 4;      // one input stage
  static constexpr int kOutBoxes = kSegs;                     // 64-column output boxes per task
  static constexpr int kOutBoxBytes = kRows * 128;            // one swizzled output box
  // per-warp layout (byte offsets); the staging tile first (1024-byte aligned)
  static constexpr int kOffStage = 0;
  static constexpr int kOffIn = kOffStage + kOutBoxes * kOutBoxBytes;
  static constexpr int kStageBytes = kInBytes + ((kRows * 4 + 127) & ~127);  // words + row norms
  static constexpr int kOffCf = kOffIn + kStages * kStageBytes;        // kSegs x (64 + 4) floats
  static constexpr int kOffSg = kOffCf + kSegs * (kSeg + 4) * 4;       // kSegs x (32 + 2) float2
  static constexpr int kOffBar = kOffSg + kSegs * (kSeg / 2 + 2) * 8;  // kStages mbarriers
  static constexpr int kWarpBytes = (kOffBar + 8 * kStages + 1023) & ~1023;
};

struct TmaArgs {
  DecodeArgs a;
  int copies, log2copies;
  int64_t n_segcols, n_bands, n_tasks;
};

template <int BITS, int LB>
__global__ void __launch_bounds__(kMaxWarps * 32, 1)
    decode_tma_kernel(TmaArgs ta, const __grid_constant__ CUtensorMap in_map,
                      const __grid_constant__ CUtensorMap rn_map, const __grid_constant__ CUtensorMap out_map) {
  using G = TmaGeom<BITS, LB>;
  constexpr int SEGS = G::kSegs, ROWS = G::kRows, NW = BITS;
  const DecodeArgs &a = ta.a;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  // per-warp regions first (1024-byte aligned: the swizzled TMA boxes need it;
  // the launch reserves 1 KB of slack), then the codebook table
  unsigned char *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char *wb = base + (size_t)warp * G::kWarpBytes;
  unsigned char *stage = wb + G::kOffStage;
  unsigned char *inbase = wb + G::kOffIn;   // stage st: words, then row norms
  float *cf = reinterpret_cast<float *>(wb + G::kOffCf);
  float2 *sg = reinterpret_cast<float2 *>(wb + G::kOffSg);
  uint64_t *bars = reinterpret_cast<uint64_t *>(wb + G::kOffBar);
  float2 *cbp = reinterpret_cast<float2 *>(base + (size_t)nwarps * G::kWarpBytes);

  for (int c = threadIdx.x; c < a.N; c += blockDim.x) {
    const float c0 = a.codebook[2 * c], c1 = a.codebook[2 * c + 1];
    const float2 e = make_float2(__fadd_rn(c0, c1), __fsub_rn(c0, c1));
    for (int r = 0; r < ta.copies; ++r) cbp[c * ta.copies + r] = e;
  }
  if (lane == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&bars[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  const float2 *cbl = cbp + (lane & (ta.copies - 1));
  const int lgc = ta.log2copies;
  const int rr = lane & (ROWS - 1);
  const int sgi = lane >> G::kLog2Rows;
  // Work split: warp g keeps column strip g % n_strips for its whole life (its
  // column tables are built once) and takes the bands slot, slot + per_strip,
  // slot + 2 per_strip, ... with slot = g / n_strips. All warps therefore move
  // down the matrix together and the reads and writes of any moment fall in
  // one band of consecutive rows, which keeps DRAM pages open; giving each
  // warp a contiguous run of tasks instead scattered the writes over the whole
  // matrix and halved the store throughput.
  const int gw = blockIdx.x * nwarps + warp;
  const int GW = gridDim.x * nwarps;
  const int nsc = (int)ta.n_segcols, nb = (int)ta.n_bands;
  const int per_strip = GW / nsc;           // >= 1 (checked on the host)
  const int my_strip = gw % nsc, slot = gw / nsc;
  const bool active = slot < per_strip;
  // tasks of this warp: k = 0, 1, ... with band = slot + k * per_strip
  const int t0 = 0, t1 = active ? (nb - slot + per_strip - 1) / per_strip : 0;
  const double inv_sqrt_b = 1.0 / sqrt((double)(1 << LB));
  const int64_t P = a.K >> 1;
  const bool check_idx = a.N < (1 << BITS);
  uint32_t bad = 0;
  bool timed_out = false;
  int cur = -1;

  // Input pipeline: kStages buffers of (packed words, row norms). The prologue
  // fills all of them; as soon as every lane has copied task t's words to
  // registers, its buffer is reloaded with task t + kStages, so each load has
  // about kStages tasks of compute time to arrive.
  auto issue_load = [&](int t) {
    const int st = (t - t0) % kStages;
    const int sc = my_strip, bd = slot + t * per_strip;
    unsigned char *buf = inbase + st * G::kStageBytes;
    mbar_arrive_expect_tx(&bars[st], (uint32_t)(G::kInBytes + ROWS * 4));
    tma_load_2d(buf, &in_map, sc * G::kBoxWords, bd * ROWS, &bars[st]);
    asm volatile(
        "cp.async.bulk.tensor.1d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2}], [%3];" ::"r"(
            smem_u32(buf + G::kInBytes)),
        "l"(&rn_map), "r"(bd * ROWS), "r"(smem_u32(&bars[st]))
        : "memory");
  };
  if (lane == 0)
    for (int t = t0; t < t1 && t < t0 + kStages; ++t) issue_load(t);

  for (int t = t0; t < t1; ++t) {
    const int segcol = my_strip, band = slot + t * per_strip;
    const int64_t colbase = (int64_t)segcol * (SEGS * kSeg);
    const int st = (t - t0) % kStages;
    const uint32_t parity = (uint32_t)(((t - t0) / kStages) & 1);
    const uint32_t *inbuf = reinterpret_cast<const uint32_t *>(inbase + st * G::kStageBytes);
    const float *rnbuf = reinterpret_cast<const float *>(inbase + st * G::kStageBytes + G::kInBytes);
    if (segcol != cur) {
      for (int j = lane; j < SEGS * kSeg; j += 32) {
        const int64_t col = colbase + j;
        float f = 0.0f;
        if (col < a.K) {
          const double s = (a.col_scale != nullptr) ? (double)a.col_scale[col] : 1.0;
          double v = inv_sqrt_b / s;
          if (mask_is_negative(a.seed, col)) v = -v;
          f = (float)v;
        }
        cf[(j >> 6) * (kSeg + 4) + (j & 63)] = f;
      }
      for (int p = lane; p < SEGS * kSeg / 2; p += 32) {
        const int64_t k = (colbase >> 1) + p;
        const float sk = (k < P) ? a.sigma[k] : 0.0f;
        sg[(p >> 5) * (kSeg / 2 + 2) + (p & 31)] = make_float2(sk, sk);
      }
      __syncwarp();
      cur = segcol;
    }
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[st], parity, kWaitLimit))) {
      timed_out = true;
      break;
    }
    const int64_t row = (int64_t)band * ROWS + rr;
    const bool row_ok = row < a.M;
    float rn = 0.0f;
    if (row_ok) {
      rn = rnbuf[rr];
      if (!isfinite(rn)) bad |= QAMW_STATUS_NONFINITE_NORM;
    }
    // words of this lane's segment
    uint32_t w[NW + 1];
    const uint32_t *wsrc = inbuf + rr * G::kBoxWords + sgi * NW;
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = wsrc[i];
    w[NW] = 0u;
    __syncwarp();
    if (lane == 0 && t + kStages < t1) {
      fence_proxy_async();
      issue_load(t + kStages);
    }
    const int64_t col0 = colbase + (int64_t)sgi * kSeg;
    const int vp = (int)std::min<int64_t>(kSeg, std::max<int64_t>(0, a.K - col0)) >> 1;
    const float2 rn2 = make_float2(rn, rn);
    const float2 *sgl = sg + sgi * (kSeg / 2 + 2);
    float v[kSeg];
    if (check_idx) {
#pragma unroll
      for (int q = 0; q < kSeg / 2; ++q) {
        uint32_t off = extract_off8<BITS>(w, q);
        if ((off >> 3) >= (uint32_t)a.N) {
          if (row_ok && q < vp) bad |= QAMW_STATUS_BAD_INDEX;
          off = 0;
        }
        const float2 y = mul2(mul2(sgl[q], rn2),
                              *reinterpret_cast<const float2 *>(reinterpret_cast<const unsigned char *>(cbl) + (off << lgc)));
        v[2 * q] = y.x;
        v[2 * q + 1] = y.y;
      }
    } else {
      const unsigned char *cbb = reinterpret_cast<const unsigned char *>(cbl);
#pragma unroll
      for (int q = 0; q < kSeg / 2; ++q) {
        const uint32_t off = extract_off8<BITS>(w, q) << lgc;
        const float2 y = mul2(mul2(sgl[q], rn2), *reinterpret_cast<const float2 *>(cbb + off));
        v[2 * q] = y.x;
        v[2 * q + 1] = y.y;
      }
    }
    inlane_stages<LB>(v);
    xlane_stages<LB, ROWS>(v, lane);

    // the previous task's stores must have finished reading the staging tile
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
    const float *cfl = cf + sgi * (kSeg + 4);
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
      // column c of this lane's segment -> output box sgi, 16-byte chunk c/8,
      // stored at chunk ^ (row % 8) (the 128-byte swizzle of the TMA box)
      const int box = sgi;
      const int chunk = (c >> 3) ^ (rr & 7);
      *reinterpret_cast<uint4 *>(stage + box * G::kOutBoxBytes + rr * 128 + chunk * 16) = pk;
    }
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int bx = 0; bx < G::kOutBoxes; ++bx)
        if (colbase + 64 * bx < a.K)
          tma_store_2d(&out_map, (int)(colbase + 64 * bx), band * ROWS, stage + bx * G::kOutBoxBytes);
      bulk_commit();
    }
    __syncwarp();
  }
  if (lane == 0) bulk_wait_all();
  if (timed_out) bad |= QAMW_STATUS_TIMEOUT;
  bad = __reduce_or_sync(0xffffffffu, bad);
  if (lane == 0) status_or(a.status, bad);
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------
}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

namespace {

template <int BITS, int LB>
cudaError_t launch_tma_t(const DecodeArgs &a, cudaStream_t s) {
  using G = TmaGeom<BITS, LB>;
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  CUtensorMap in_map, rn_map, out_map;
  {
    cuuint64_t dims[1] = {(cuuint64_t)a.M};
    cuuint64_t strides[1] = {4};
    cuuint32_t box[1] = {(cuuint32_t)G::kRows};
    cuuint32_t es[1] = {1};
    if (enc(&rn_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, const_cast<float *>(a.row_norm), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)a.wpr, (cuuint64_t)a.M};
    cuuint64_t strides[1] = {(cuuint64_t)a.wpr * 4};
    cuuint32_t box[2] = {(cuuint32_t)G::kBoxWords, (cuuint32_t)G::kRows};
    cuuint32_t es[2] = {1, 1};
    if (enc(&in_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(a.packed), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M};
    cuuint64_t strides[1] = {(cuuint64_t)a.ldo * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)G::kRows};
    cuuint32_t es[2] = {1, 1};
    if (enc(&out_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.out, dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  TmaArgs ta;
  ta.a = a;
  ta.copies = 16;
  while (ta.copies > 1 && (size_t)a.N * 8 * ta.copies > 65536) ta.copies >>= 1;
  int dev = 0, smem_max = 0;
  cudaGetDevice(&dev);
  cudaError_t e = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  int warps = kMaxWarps;
  auto need = [&](int w, int copies) { return 1024 + (size_t)w * G::kWarpBytes + (size_t)a.N * copies * 8; };
  // prefer kMaxWarps warps; shrink the table replication, then the warp count, to fit
  while (need(warps, ta.copies) > (size_t)smem_max && ta.copies > 4) ta.copies >>= 1;
  while (warps > 4 && need(warps, ta.copies) > (size_t)smem_max) --warps;
  while (need(warps, ta.copies) > (size_t)smem_max && ta.copies > 1) ta.copies >>= 1;
  if (need(warps, ta.copies) > (size_t)smem_max) return cudaErrorNotSupported;
  ta.log2copies = 0;
  while ((1 << ta.log2copies) < ta.copies) ++ta.log2copies;
  ta.n_segcols = (a.K + G::kSegs * kSeg - 1) / (G::kSegs * kSeg);
  ta.n_bands = (a.M + G::kRows - 1) / G::kRows;
  ta.n_tasks = ta.n_segcols * ta.n_bands;
  const size_t smem = need(warps, ta.copies);
  e = set_max_dynamic_smem(reinterpret_cast<const void *>(decode_tma_kernel<BITS, LB>), smem);
  if (e != cudaSuccess) return e;
  // one CTA per SM; every column strip needs at least one warp
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((ta.n_tasks + warps - 1) / warps, sm_count()));
  if (blocks * warps < ta.n_segcols) return cudaErrorNotSupported;
  decode_tma_kernel<BITS, LB><<<(int)blocks, warps * 32, smem, s>>>(ta, in_map, rn_map, out_map);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_tma_bits(const DecodeArgs &a, cudaStream_t s) {
  switch (a.log2b) {
    case 6: return launch_tma_t<BITS, 6>(a, s);
    case 7: return launch_tma_t<BITS, 7>(a, s);
    case 8: return launch_tma_t<BITS, 8>(a, s);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

bool decode_tma_applicable(const DecodeArgs &a) {
  if (a.out_t != QAMW_BF16) return false;
  if (a.bits != 7 && a.bits != 8 && a.bits != 10 && a.bits != 11) return false;
  if (a.log2b < 6 || a.log2b > 8) return false;
  if (reinterpret_cast<uintptr_t>(a.packed) % 16 || reinterpret_cast<uintptr_t>(a.out) % 16) return false;
  if ((a.wpr * 4) % 16 || (a.ldo * 2) % 16) return false;
  if (a.K % 64) return false;
  if (a.M > (int64_t(1) << 30) || a.wpr > (int64_t(1) << 30)) return false;
  if (reinterpret_cast<uintptr_t>(a.row_norm) % 16) return false;
  // task indices are 32-bit
  const int64_t sb = (a.log2b > 6) ? (int64_t(1) << (a.log2b - 6)) : 1;
  const int64_t sa = (a.bits % 4 == 0) ? 1 : ((a.bits % 2 == 0) ? 2 : 4);
  const int64_t segs = sb > sa ? sb : sa;
  if (((a.K + segs * 64 - 1) / (segs * 64)) * ((a.M + 31) / (32 / segs)) > (int64_t(1) << 30)) return false;
  return tensor_map_encoder() != nullptr;
}

cudaError_t launch_decode_tma(const DecodeArgs &a, cudaStream_t s) {
  switch (a.bits) {
    case 7: return launch_tma_bits<7>(a, s);
    case 8: return launch_tma_bits<8>(a, s);
    case 10: return launch_tma_bits<10>(a, s);
    case 11: return launch_tma_bits<11>(a, s);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace qamw
