// qamw_api.cu -- the extern "C" entry points of libqamw.so (declared in
// include/qamw.h): host-side argument validation, workspace carving and the
// kernel launches. Nothing is allocated; nothing is launched when an argument
// is rejected.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "qamw.h"
#include "qamw_internal.h"

namespace qamw {

namespace {
thread_local char g_last_error[512] = {0};

int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char *where) {
  return fail(QAMW_ECUDA, "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

int log2i(int64_t v) {
  int l = 0;
  while ((int64_t(1) << l) < v) ++l;
  return l;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// An NVTX range around one C-ABI call (visible to nsys / ncu when attached;
// a few nanoseconds otherwise).
struct CallRange {
  explicit CallRange(const char *name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange &) = delete;
  CallRange &operator=(const CallRange &) = delete;
};

// Shape checks common to calibrate / encode / decode.
int check_shape(int64_t M, int64_t K, int32_t block, const char *fn) {
  if (M < 1) return fail(QAMW_EINVAL, "%s: M must be >= 1 (got %lld)", fn, (long long)M);
  if (K < 2 || (K & 1)) return fail(QAMW_EINVAL, "%s: K must be even and >= 2 (got %lld)", fn, (long long)K);
  if (!is_pow2(block) || block < 2)
    return fail(QAMW_EINVAL, "%s: block must be a power of two >= 2 (got %d)", fn, block);
  if (block > QAMW_MAX_BLOCK)
    return fail(QAMW_EUNSUPPORTED, "%s: block %d exceeds %d", fn, block, QAMW_MAX_BLOCK);
  if (K % block) return fail(QAMW_EINVAL, "%s: K (%lld) must be a multiple of block (%d)", fn, (long long)K, block);
  if (M > (int64_t(1) << 40) || K > (int64_t(1) << 31))
    return fail(QAMW_EUNSUPPORTED, "%s: shape too large", fn);
  return QAMW_OK;
}

int check_code(int32_t N, int32_t bits, const char *fn) {
  if (bits < 1 || bits > 16) return fail(QAMW_EINVAL, "%s: bits_per_pair must be in [1, 16] (got %d)", fn, bits);
  if (N < 1 || (int64_t)N > (int64_t(1) << bits))
    return fail(QAMW_EINVAL, "%s: need 1 <= N <= 2^bits (N=%d, bits=%d)", fn, N, bits);
  if (N > QAMW_MAX_CENTROIDS)
    return fail(QAMW_EUNSUPPORTED, "%s: N=%d exceeds %d centroids", fn, N, QAMW_MAX_CENTROIDS);
  return QAMW_OK;
}

int check_dtype(qamw_dtype t, const char *fn) {
  if (t != QAMW_F32 && t != QAMW_BF16) return fail(QAMW_EINVAL, "%s: unknown dtype %d", fn, (int)t);
  return QAMW_OK;
}

std::mutex g_sm_mu;
int g_sm_count[64] = {0};
}  // namespace

void set_last_error(const char *msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

cudaError_t set_max_dynamic_smem(const void *func, size_t bytes) {
  static std::mutex mu;
  static std::vector<std::pair<std::pair<const void *, int>, size_t>> done;   // (kernel, device) -> bytes set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (auto &d : done)
    if (d.first.first == func && d.first.second == dev) {
      if (d.second >= bytes) return cudaSuccess;
      if ((e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) == cudaSuccess)
        d.second = bytes;
      return e;
    }
  if ((e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) == cudaSuccess)
    done.push_back({{func, dev}, bytes});
  return e;
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(g_sm_mu);
  if (g_sm_count[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    g_sm_count[dev] = v;
  }
  return g_sm_count[dev];
}

}  // namespace qamw

using namespace qamw;

extern "C" {

const char *qamw_version(void) { return "qamw 0.1.0 (sm_100a)"; }

const char *qamw_status_string(int code) {
  switch (code) {
    case QAMW_OK: return "ok";
    case QAMW_EINVAL: return "invalid argument";
    case QAMW_ENULL: return "null pointer";
    case QAMW_EUNSUPPORTED: return "unsupported by this build";
    case QAMW_ECUDA: return "CUDA error";
    case QAMW_EWORKSPACE: return "workspace too small";
    default: return "unknown status";
  }
}

const char *qamw_last_error(void) { return g_last_error; }

int64_t qamw_words_per_row(int64_t K, int32_t bits_per_pair) {
  if (K < 2 || (K & 1) || bits_per_pair < 1 || bits_per_pair > 16) return -1;
  return ((K / 2) * bits_per_pair + 31) / 32;
}

int qamw_channel_scale(const float *act_rms, float alpha, int64_t K, float *s_out, int32_t *status,
                       qamw_stream_t stream) {
  g_last_error[0] = 0;
  if (s_out == nullptr) return fail(QAMW_ENULL, "qamw_channel_scale: s_out is NULL");
  if (K < 1) return fail(QAMW_EINVAL, "qamw_channel_scale: K must be >= 1");
  if (!std::isfinite(alpha)) return fail(QAMW_EINVAL, "qamw_channel_scale: alpha must be finite");
  ScaleArgs a{act_rms, alpha, K, s_out, status};
  cudaError_t e = launch_channel_scale(a, (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, "qamw_channel_scale");
}

size_t qamw_calibrate_workspace_bytes(int64_t M, int64_t K) {
  if (M < 1 || K < 2) return 0;
  const int64_t groups = (M + kCalibRowGroup - 1) / kCalibRowGroup;
  return align256((size_t)K * 4) + align256((size_t)M * 4) + align256((size_t)groups * (size_t)(K / 2) * 8);
}

// Calibration of W's rows: sigma (sigma_out) or the fp64 sums of |z| per pair
// position (sum_out) -- qamw_calibrate_sigma and qamw_calibrate_partial_sums.
static int calibrate_impl(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                          const float *act_rms, float alpha, int32_t block, uint64_t sign_seed, float *sigma_out,
                          double *sum_out, void *workspace, size_t workspace_bytes, int32_t *status,
                          qamw_stream_t stream, const char *fn) {
  int rc;
  if (W == nullptr || (sigma_out == nullptr && sum_out == nullptr))
    return fail(QAMW_ENULL, "%s: W and the output must be non-NULL", fn);
  if ((rc = check_dtype(w_dtype, fn))) return rc;
  if ((rc = check_shape(M, K, block, fn))) return rc;
  if (ldw < K) return fail(QAMW_EINVAL, "%s: ldw (%lld) < K (%lld)", fn, (long long)ldw, (long long)K);
  if (!std::isfinite(alpha)) return fail(QAMW_EINVAL, "%s: alpha must be finite", fn);
  const size_t need = qamw_calibrate_workspace_bytes(M, K);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(QAMW_EWORKSPACE, "%s: workspace of %zu bytes needed (got %zu)", fn, need, workspace_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(QAMW_EINVAL, "%s: workspace must be 256-byte aligned", fn);
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  float *s = reinterpret_cast<float *>(ws);
  float *r = reinterpret_cast<float *>(ws + align256((size_t)K * 4));
  double *partials = reinterpret_cast<double *>(ws + align256((size_t)K * 4) + align256((size_t)M * 4));
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if ((e = launch_channel_scale(ScaleArgs{act_rms, alpha, K, s, status}, st)) != cudaSuccess) return cuda_fail(e, fn);
  if ((e = launch_row_norms(RowNormArgs{W, w_dtype, M, K, ldw, s, r, status}, st)) != cudaSuccess)
    return cuda_fail(e, fn);
  CalibArgs ca;
  ca.rot = RotateArgs{W, w_dtype, M, K, ldw, log2i(block), sign_seed, s, r};
  ca.partials = partials;
  ca.groups = (M + kCalibRowGroup - 1) / kCalibRowGroup;
  ca.sigma_out = sigma_out;
  ca.sum_out = sum_out;
  if ((e = launch_calibrate(ca, st)) != cudaSuccess) return cuda_fail(e, fn);
  return QAMW_OK;
}

int qamw_calibrate_sigma(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                         const float *act_rms, float alpha, int32_t block, uint64_t sign_seed,
                         float *sigma_out, void *workspace, size_t workspace_bytes, int32_t *status,
                         qamw_stream_t stream) {
  static const char *fn = "qamw_calibrate_sigma";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  if (sigma_out == nullptr) return fail(QAMW_ENULL, "%s: W and sigma_out must be non-NULL", fn);
  return calibrate_impl(W, w_dtype, M, K, ldw, act_rms, alpha, block, sign_seed, sigma_out, nullptr, workspace,
                        workspace_bytes, status, stream, fn);
}

int qamw_calibrate_partial_sums(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                                const float *act_rms, float alpha, int32_t block, uint64_t sign_seed,
                                double *sums_out, void *workspace, size_t workspace_bytes, int32_t *status,
                                qamw_stream_t stream) {
  static const char *fn = "qamw_calibrate_partial_sums";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  if (sums_out == nullptr) return fail(QAMW_ENULL, "%s: W and sums_out must be non-NULL", fn);
  return calibrate_impl(W, w_dtype, M, K, ldw, act_rms, alpha, block, sign_seed, nullptr, sums_out, workspace,
                        workspace_bytes, status, stream, fn);
}

int qamw_sigma_from_partial_sums(const double *sums, int32_t R, int64_t P, int64_t M_total, float *sigma_out,
                                 qamw_stream_t stream) {
  static const char *fn = "qamw_sigma_from_partial_sums";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  if (!sums || !sigma_out) return fail(QAMW_ENULL, "%s: sums and sigma_out must be non-NULL", fn);
  if (R < 1 || P < 1 || M_total < 1)
    return fail(QAMW_EINVAL, "%s: R (%d), P (%lld) and M_total (%lld) must be >= 1", fn, R, (long long)P,
                (long long)M_total);
  cudaError_t e = launch_sigma_from_sums(sums, R, P, M_total, sigma_out, (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, fn);
}

int qamw_encode(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                const float *act_rms, float alpha, int32_t block, uint64_t sign_seed,
                const float *sigma, const float *codebook, int32_t N, int32_t bits_per_pair,
                const void *search_table, uint32_t *packed_out, float *row_norm_out,
                float *col_scale_out, int32_t *status, qamw_stream_t stream) {
  static const char *fn = "qamw_encode";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  int rc;
  if (!W || !sigma || !codebook || !packed_out || !row_norm_out || !col_scale_out)
    return fail(QAMW_ENULL, "%s: W, sigma, codebook, packed_out, row_norm_out, col_scale_out must be non-NULL", fn);
  if ((rc = check_dtype(w_dtype, fn))) return rc;
  if ((rc = check_shape(M, K, block, fn))) return rc;
  if ((rc = check_code(N, bits_per_pair, fn))) return rc;
  if (ldw < K) return fail(QAMW_EINVAL, "%s: ldw (%lld) < K (%lld)", fn, (long long)ldw, (long long)K);
  if (!std::isfinite(alpha)) return fail(QAMW_EINVAL, "%s: alpha must be finite", fn);
  if (search_table != nullptr && reinterpret_cast<uintptr_t>(search_table) % 16)
    return fail(QAMW_EINVAL, "%s: search_table must be 16-byte aligned", fn);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if ((e = launch_channel_scale(ScaleArgs{act_rms, alpha, K, col_scale_out, status}, st)) != cudaSuccess)
    return cuda_fail(e, fn);
  if ((e = launch_row_norms(RowNormArgs{W, w_dtype, M, K, ldw, col_scale_out, row_norm_out, status}, st)) !=
      cudaSuccess)
    return cuda_fail(e, fn);
  EncodeArgs ea;
  ea.rot = RotateArgs{W, w_dtype, M, K, ldw, log2i(block), sign_seed, col_scale_out, row_norm_out};
  ea.sigma = sigma;
  ea.codebook = codebook;
  ea.N = N;
  ea.bits = bits_per_pair;
  ea.wpr = qamw_words_per_row(K, bits_per_pair);
  ea.packed = packed_out;
  ea.table = search_table;
  ea.status = status;
  if ((e = launch_encode(ea, st)) != cudaSuccess) return cuda_fail(e, fn);
  return QAMW_OK;
}

int qamw_encode_prepared(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                         const float *col_scale, const float *row_norm, int32_t block, uint64_t sign_seed,
                         const float *sigma, const float *codebook, int32_t N, int32_t bits_per_pair,
                         const void *search_table, uint32_t *packed_out, int32_t *status, qamw_stream_t stream) {
  static const char *fn = "qamw_encode_prepared";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  int rc;
  if (!W || !col_scale || !row_norm || !sigma || !codebook || !packed_out)
    return fail(QAMW_ENULL, "%s: W, col_scale, row_norm, sigma, codebook, packed_out must be non-NULL", fn);
  if ((rc = check_dtype(w_dtype, fn))) return rc;
  if ((rc = check_shape(M, K, block, fn))) return rc;
  if ((rc = check_code(N, bits_per_pair, fn))) return rc;
  if (ldw < K) return fail(QAMW_EINVAL, "%s: ldw (%lld) < K (%lld)", fn, (long long)ldw, (long long)K);
  if (search_table != nullptr && reinterpret_cast<uintptr_t>(search_table) % 16)
    return fail(QAMW_EINVAL, "%s: search_table must be 16-byte aligned", fn);
  EncodeArgs ea;
  ea.rot = RotateArgs{W, w_dtype, M, K, ldw, log2i(block), sign_seed, col_scale, row_norm};
  ea.sigma = sigma;
  ea.codebook = codebook;
  ea.N = N;
  ea.bits = bits_per_pair;
  ea.wpr = qamw_words_per_row(K, bits_per_pair);
  ea.packed = packed_out;
  ea.table = search_table;
  ea.status = status;
  cudaError_t e = launch_encode(ea, (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, fn);
}

int qamw_calibrate_encode(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                          const float *act_rms, float alpha, int32_t block, uint64_t sign_seed,
                          const float *codebook, int32_t N, int32_t bits_per_pair, const void *search_table,
                          float *sigma_out, uint32_t *packed_out, float *row_norm_out, float *col_scale_out,
                          void *workspace, size_t workspace_bytes, int32_t *status, qamw_stream_t stream) {
  static const char *fn = "qamw_calibrate_encode";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  int rc;
  if (!W || !codebook || !sigma_out || !packed_out || !row_norm_out || !col_scale_out)
    return fail(QAMW_ENULL,
                "%s: W, codebook, sigma_out, packed_out, row_norm_out, col_scale_out must be non-NULL", fn);
  if ((rc = check_dtype(w_dtype, fn))) return rc;
  if ((rc = check_shape(M, K, block, fn))) return rc;
  if ((rc = check_code(N, bits_per_pair, fn))) return rc;
  if (ldw < K) return fail(QAMW_EINVAL, "%s: ldw (%lld) < K (%lld)", fn, (long long)ldw, (long long)K);
  if (!std::isfinite(alpha)) return fail(QAMW_EINVAL, "%s: alpha must be finite", fn);
  if (search_table != nullptr && reinterpret_cast<uintptr_t>(search_table) % 16)
    return fail(QAMW_EINVAL, "%s: search_table must be 16-byte aligned", fn);
  const size_t need = qamw_calibrate_workspace_bytes(M, K);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(QAMW_EWORKSPACE, "%s: workspace of %zu bytes needed (got %zu)", fn, need, workspace_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(QAMW_EINVAL, "%s: workspace must be 256-byte aligned", fn);
  // the partials sit where qamw_calibrate_sigma puts them; s and r go straight
  // to the caller's metadata arrays, which both passes read
  double *partials = reinterpret_cast<double *>(static_cast<unsigned char *>(workspace) + align256((size_t)K * 4) +
                                                align256((size_t)M * 4));
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if ((e = launch_channel_scale(ScaleArgs{act_rms, alpha, K, col_scale_out, status}, st)) != cudaSuccess)
    return cuda_fail(e, fn);
  if ((e = launch_row_norms(RowNormArgs{W, w_dtype, M, K, ldw, col_scale_out, row_norm_out, status}, st)) !=
      cudaSuccess)
    return cuda_fail(e, fn);
  const RotateArgs rot{W, w_dtype, M, K, ldw, log2i(block), sign_seed, col_scale_out, row_norm_out};
  CalibArgs ca;
  ca.rot = rot;
  ca.partials = partials;
  ca.groups = (M + kCalibRowGroup - 1) / kCalibRowGroup;
  ca.sigma_out = sigma_out;
  ca.sum_out = nullptr;
  if ((e = launch_calibrate(ca, st)) != cudaSuccess) return cuda_fail(e, fn);
  EncodeArgs ea;
  ea.rot = rot;
  ea.sigma = sigma_out;
  ea.codebook = codebook;
  ea.N = N;
  ea.bits = bits_per_pair;
  ea.wpr = qamw_words_per_row(K, bits_per_pair);
  ea.packed = packed_out;
  ea.table = search_table;
  ea.status = status;
  if ((e = launch_encode(ea, st)) != cudaSuccess) return cuda_fail(e, fn);
  return QAMW_OK;
}

int qamw_encode_polar(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K, int64_t ldw,
                      const float *act_rms, float alpha, int32_t block, uint64_t sign_seed, const float *sigma,
                      const double *amps, int32_t A, int32_t P, int32_t bits_per_pair, uint32_t *packed_out,
                      float *row_norm_out, float *col_scale_out, int32_t *status, qamw_stream_t stream) {
  static const char *fn = "qamw_encode_polar";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  int rc;
  if (!W || !sigma || !amps || !packed_out || !row_norm_out || !col_scale_out)
    return fail(QAMW_ENULL, "%s: W, sigma, amps, packed_out, row_norm_out, col_scale_out must be non-NULL", fn);
  if ((rc = check_dtype(w_dtype, fn))) return rc;
  if ((rc = check_shape(M, K, block, fn))) return rc;
  if (A < 1 || P < 1 || (int64_t)A * P > QAMW_MAX_CENTROIDS)
    return fail(QAMW_EINVAL, "%s: A (%d) and P (%d) must be >= 1 with A*P <= %d", fn, A, P, QAMW_MAX_CENTROIDS);
  if ((rc = check_code(A * P, bits_per_pair, fn))) return rc;
  if (ldw < K) return fail(QAMW_EINVAL, "%s: ldw (%lld) < K (%lld)", fn, (long long)ldw, (long long)K);
  if (!std::isfinite(alpha)) return fail(QAMW_EINVAL, "%s: alpha must be finite", fn);
  if (reinterpret_cast<uintptr_t>(amps) % 8) return fail(QAMW_EINVAL, "%s: amps must be 8-byte aligned", fn);
  if (block > 512) return fail(QAMW_EUNSUPPORTED, "%s: block %d > 512 is not supported", fn, block);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if ((e = launch_channel_scale(ScaleArgs{act_rms, alpha, K, col_scale_out, status}, st)) != cudaSuccess)
    return cuda_fail(e, fn);
  if ((e = launch_row_norms(RowNormArgs{W, w_dtype, M, K, ldw, col_scale_out, row_norm_out, status}, st)) !=
      cudaSuccess)
    return cuda_fail(e, fn);
  EncodeArgs ea;
  ea.rot = RotateArgs{W, w_dtype, M, K, ldw, log2i(block), sign_seed, col_scale_out, row_norm_out};
  ea.sigma = sigma;
  ea.codebook = nullptr;
  ea.N = A * P;
  ea.bits = bits_per_pair;
  ea.wpr = qamw_words_per_row(K, bits_per_pair);
  ea.packed = packed_out;
  ea.table = nullptr;
  ea.status = status;
  ea.polar_amps = amps;
  ea.polar_A = A;
  ea.polar_P = P;
  if ((e = launch_encode_polar(ea, st)) != cudaSuccess) return cuda_fail(e, fn);
  return QAMW_OK;
}

int qamw_decode_matmul(const uint32_t *packed, const float *row_norm, const float *sigma, const float *col_scale,
                       int64_t M, int64_t K, int32_t block, uint64_t sign_seed, const float *codebook, int32_t N,
                       int32_t bits_per_pair, const void *X, int64_t T, int64_t ldx, float *Y, int64_t ldy,
                       void *workspace, size_t workspace_bytes, int32_t *status, qamw_stream_t stream) {
  static const char *fn = "qamw_decode_matmul";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  int rc;
  if (!packed || !row_norm || !sigma || !codebook || !X || !Y || !workspace)
    return fail(QAMW_ENULL, "%s: packed, row_norm, sigma, codebook, X, Y and workspace must be non-NULL", fn);
  if ((rc = check_shape(M, K, block, fn))) return rc;
  if ((rc = check_code(N, bits_per_pair, fn))) return rc;
  if (T < 1 || T > (int64_t)1 << 24) return fail(QAMW_EINVAL, "%s: T (%lld) must be in [1, 2^24]", fn, (long long)T);
  if (ldx < K || ldy < M)
    return fail(QAMW_EINVAL, "%s: ldx (%lld) must be >= K and ldy (%lld) >= M", fn, (long long)ldx, (long long)ldy);
  if (K % 128 != 0 || K > 32768)
    return fail(QAMW_EUNSUPPORTED, "%s: needs K a multiple of 128 and at most 32768", fn);
  if (reinterpret_cast<uintptr_t>(X) % 16 != 0 || ldx % 8 != 0)
    return fail(QAMW_EINVAL, "%s: X must be 16-byte aligned with ldx a multiple of 8", fn);
  if (reinterpret_cast<uintptr_t>(packed) % 8 != 0 || reinterpret_cast<uintptr_t>(sigma) % 16 != 0)
    return fail(QAMW_EINVAL, "%s: packed must be 8-byte and sigma 16-byte aligned", fn);
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0 || workspace_bytes < decode_matmul_workspace_bytes(M, K, T))
    return fail(QAMW_EINVAL, "%s: workspace must be 256-byte aligned and hold %zu bytes (got %zu)", fn,
                decode_matmul_workspace_bytes(M, K, T), workspace_bytes);
  DecodeArgs a;
  a.packed = packed;
  a.row_norm = row_norm;
  a.sigma = sigma;
  a.col_scale = col_scale;
  a.M = M;
  a.K = K;
  a.log2b = log2i(block);
  a.seed = sign_seed;
  a.codebook = codebook;
  a.N = N;
  a.bits = bits_per_pair;
  a.wpr = qamw_words_per_row(K, bits_per_pair);
  a.out = nullptr;
  a.out_t = QAMW_BF16;
  a.ldo = 0;
  a.status = status;
  cudaError_t e = launch_decode_gemm(a, static_cast<const uint16_t *>(X), T, ldx, Y, ldy, workspace,
                                     (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, fn);
}

size_t qamw_decode_matmul_workspace_bytes(int64_t M, int64_t K, int64_t T) {
  if (M < 1 || K < 1 || T < 1 || T > (int64_t)1 << 24) return 0;
  return decode_matmul_workspace_bytes(M, K, T);
}

int qamw_decode(const uint32_t *packed, const float *row_norm, const float *sigma, const float *col_scale,
                int64_t M, int64_t K, int32_t block, uint64_t sign_seed, const float *codebook, int32_t N,
                int32_t bits_per_pair, void *W_out, qamw_dtype out_dtype, int64_t ldo, int32_t *status,
                qamw_stream_t stream) {
  static const char *fn = "qamw_decode";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  int rc;
  if (!packed || !row_norm || !sigma || !codebook || !W_out)
    return fail(QAMW_ENULL, "%s: packed, row_norm, sigma, codebook, W_out must be non-NULL", fn);
  if ((rc = check_dtype(out_dtype, fn))) return rc;
  if ((rc = check_shape(M, K, block, fn))) return rc;
  if ((rc = check_code(N, bits_per_pair, fn))) return rc;
  if (ldo < K) return fail(QAMW_EINVAL, "%s: ldo (%lld) < K (%lld)", fn, (long long)ldo, (long long)K);
  DecodeArgs a;
  a.packed = packed;
  a.row_norm = row_norm;
  a.sigma = sigma;
  a.col_scale = col_scale;
  a.M = M;
  a.K = K;
  a.log2b = log2i(block);
  a.seed = sign_seed;
  a.codebook = codebook;
  a.N = N;
  a.bits = bits_per_pair;
  a.wpr = qamw_words_per_row(K, bits_per_pair);
  a.out = W_out;
  a.out_t = out_dtype;
  a.ldo = ldo;
  a.status = status;
  cudaError_t e = launch_decode(a, (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, fn);
}

size_t qamw_search_table_bytes(int32_t N) {
  if (N < 1 || N > QAMW_MAX_CENTROIDS) return 0;
  return search_table_bytes(N);
}

int qamw_build_search_table(const float *codebook, int32_t N, void *table, size_t table_bytes,
                            qamw_stream_t stream) {
  static const char *fn = "qamw_build_search_table";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  if (!codebook || !table) return fail(QAMW_ENULL, "%s: codebook and table must be non-NULL", fn);
  if (N < 1) return fail(QAMW_EINVAL, "%s: N must be >= 1 (got %d)", fn, N);
  if (N > QAMW_MAX_CENTROIDS) return fail(QAMW_EUNSUPPORTED, "%s: N=%d exceeds %d", fn, N, QAMW_MAX_CENTROIDS);
  const size_t need = search_table_bytes(N);
  if (table_bytes < need) return fail(QAMW_EWORKSPACE, "%s: table of %zu bytes needed (got %zu)", fn, need, table_bytes);
  if (reinterpret_cast<uintptr_t>(table) % 16) return fail(QAMW_EINVAL, "%s: table must be 16-byte aligned", fn);
  cudaError_t e = launch_build_search_table(codebook, N, table, (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, fn);
}

int qamw_rotate_rows(const double *U, double *Y, int64_t M, int64_t K, int32_t block, uint64_t sign_seed,
                     int32_t inverse, qamw_stream_t stream) {
  static const char *fn = "qamw_rotate_rows";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  int rc;
  if (!U || !Y) return fail(QAMW_ENULL, "%s: U and Y must be non-NULL", fn);
  if ((rc = check_shape(M, K, block, fn))) return rc;
  RotateTestArgs a{U, Y, M, K, log2i(block), sign_seed, inverse};
  cudaError_t e = (a.log2b <= 9) ? launch_rotate_test512(a, (cudaStream_t)stream)
                                 : launch_rotate_test(a, (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, fn);
}

int qamw_search_cells(const float *x, int64_t n, const void *table, int32_t *cell_out, qamw_stream_t stream) {
  static const char *fn = "qamw_search_cells";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  if (!x || !table || !cell_out) return fail(QAMW_ENULL, "%s: x, table and cell_out must be non-NULL", fn);
  if (n < 0) return fail(QAMW_EINVAL, "%s: n must be >= 0", fn);
  if (n == 0) return QAMW_OK;
  if (reinterpret_cast<uintptr_t>(table) % 16) return fail(QAMW_EINVAL, "%s: table must be 16-byte aligned", fn);
  cudaError_t e = launch_search_cells(x, n, table, cell_out, (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, fn);
}

size_t qamw_lloyd_workspace_bytes(int64_t T, int32_t N) {
  if (T < 1 || N < 1 || N > QAMW_MAX_CENTROIDS) return 0;
  return qamw::lloyd_workspace_bytes(T, N);
}

static int check_lloyd(const void *points, int64_t T, const void *centroids, int32_t N, const char *fn) {
  if (!points || !centroids) return fail(QAMW_ENULL, "%s: points and centroids must be non-NULL", fn);
  if (T < 1) return fail(QAMW_EINVAL, "%s: T (%lld) must be >= 1", fn, (long long)T);
  if (N < 1 || N > QAMW_MAX_CENTROIDS)
    return fail(QAMW_EINVAL, "%s: N (%d) must be in [1, %d]", fn, N, QAMW_MAX_CENTROIDS);
  if (reinterpret_cast<uintptr_t>(points) % 16 || reinterpret_cast<uintptr_t>(centroids) % 16)
    return fail(QAMW_EINVAL, "%s: points and centroids must be 16-byte aligned", fn);
  return QAMW_OK;
}

int qamw_lloyd_assign(const double *points, int64_t T, const double *centroids, int32_t N, int32_t *idx_inout,
                      unsigned long long *changed, qamw_stream_t stream) {
  static const char *fn = "qamw_lloyd_assign";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  int rc;
  if ((rc = check_lloyd(points, T, centroids, N, fn))) return rc;
  if (!idx_inout) return fail(QAMW_ENULL, "%s: idx_inout must be non-NULL", fn);
  cudaError_t e = launch_lloyd_assign(points, T, centroids, N, idx_inout, changed, (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, fn);
}

int qamw_lloyd_update(const double *points, int64_t T, const int32_t *idx, int32_t N, double *centroids_inout,
                      void *workspace, size_t workspace_bytes, qamw_stream_t stream) {
  static const char *fn = "qamw_lloyd_update";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  int rc;
  if ((rc = check_lloyd(points, T, centroids_inout, N, fn))) return rc;
  if (!idx) return fail(QAMW_ENULL, "%s: idx must be non-NULL", fn);
  const size_t need = qamw_lloyd_workspace_bytes(T, N);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(QAMW_EWORKSPACE, "%s: workspace of %zu bytes needed (got %zu)", fn, need, workspace_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(QAMW_EINVAL, "%s: workspace must be 256-byte aligned", fn);
  cudaError_t e = launch_lloyd_update(points, T, idx, N, centroids_inout, workspace, nullptr, (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, fn);
}

int qamw_lloyd_train(const double *points, int64_t T, double *centroids, int32_t N, int32_t max_iter,
                     int32_t *idx_out, void *workspace, size_t workspace_bytes, int32_t *iterations_out,
                     int32_t *converged_out, qamw_stream_t stream) {
  static const char *fn = "qamw_lloyd_train";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  int rc;
  if ((rc = check_lloyd(points, T, centroids, N, fn))) return rc;
  if (!idx_out) return fail(QAMW_ENULL, "%s: idx_out must be non-NULL", fn);
  if (max_iter < 0) return fail(QAMW_EINVAL, "%s: max_iter (%d) must be >= 0", fn, max_iter);
  const size_t need = qamw_lloyd_workspace_bytes(T, N);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(QAMW_EWORKSPACE, "%s: workspace of %zu bytes needed (got %zu)", fn, need, workspace_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(QAMW_EINVAL, "%s: workspace must be 256-byte aligned", fn);
  cudaStream_t st = (cudaStream_t)stream;
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  unsigned long long *changed = reinterpret_cast<unsigned long long *>(ws + need - 256);
  cudaError_t e;
  // idx = assign(C0) (every sample counts as changed: idx starts at -1)
  if ((e = cudaMemsetAsync(idx_out, 0xff, (size_t)T * sizeof(int32_t), st)) != cudaSuccess) return cuda_fail(e, fn);
  if ((e = launch_lloyd_assign(points, T, centroids, N, idx_out, nullptr, st)) != cudaSuccess) return cuda_fail(e, fn);
  int32_t it = 0, conv = 0;
  for (it = 1; it <= max_iter; ++it) {
    if ((e = launch_lloyd_update(points, T, idx_out, N, centroids, workspace, nullptr, st)) != cudaSuccess)
      return cuda_fail(e, fn);
    if ((e = cudaMemsetAsync(changed, 0, sizeof(unsigned long long), st)) != cudaSuccess) return cuda_fail(e, fn);
    if ((e = launch_lloyd_assign(points, T, centroids, N, idx_out, changed, st)) != cudaSuccess)
      return cuda_fail(e, fn);
    unsigned long long h = 0;
    if ((e = cudaMemcpyAsync(&h, changed, sizeof(h), cudaMemcpyDeviceToHost, st)) != cudaSuccess)
      return cuda_fail(e, fn);
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, fn);
    if (h == 0) {
      conv = 1;
      break;
    }
  }
  if (it > max_iter) it = max_iter;
  if (iterations_out) *iterations_out = it;
  if (converged_out) *converged_out = conv;
  return QAMW_OK;
}

int qamw_selftest_wait_timeout(uint32_t tries, int32_t *status, qamw_stream_t stream) {
  static const char *fn = "qamw_selftest_wait_timeout";
  CallRange nvtx_range(fn);
  g_last_error[0] = 0;
  if (status == nullptr) return fail(QAMW_ENULL, "%s: status must be non-NULL", fn);
  if (tries < 1 || tries > (1u << 20)) return fail(QAMW_EINVAL, "%s: tries (%u) must be in [1, 2^20]", fn, tries);
  cudaError_t e = launch_wait_timeout(tries, status, (cudaStream_t)stream);
  return e == cudaSuccess ? QAMW_OK : cuda_fail(e, fn);
}

}  // extern "C"
