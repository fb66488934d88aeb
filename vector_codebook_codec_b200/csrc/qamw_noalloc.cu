// qamw_noalloc.cu -- sigma calibration for callers that cannot allocate.
//
// qamw_calibrate_sigma needs a caller-provided device workspace (channel
// scales, row norms and fp64 partial sums). Some callers cannot provide one:
// an inference engine that freezes its device memory pool after start-up, a
// plug-in hosted by a framework that owns all device memory and exposes no
// allocator, or a latency-critical path where cudaMalloc (which may
// synchronize the device) is not acceptable. For them,
// qamw_calibrate_sigma_noalloc runs the same kernels on a fixed scratch area
// that lives in this module: no cudaMalloc, cudaFree or other allocating call
// is made, by the caller or by the library.
//
// The area is a file-scope device array of QAMW_NOALLOC_SCRATCH_BYTES bytes;
// every GPU that loads the library reserves it until the process exits. In
// host code its name is only a handle for the symbol, not a device address,
// so the address is looked up once per device with cudaGetSymbolAddress (on
// the first call made with that device current) and cached.
#include <cstdio>
#include <mutex>

#include "qamw.h"
#include "qamw_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_calib_scratch[QAMW_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of this module's scratch area on the current device.
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_calib_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int qamw_calibrate_sigma_noalloc(const void *W, qamw_dtype w_dtype, int64_t M, int64_t K,
                                            int64_t ldw, const float *act_rms, float alpha, int32_t block,
                                            uint64_t sign_seed, float *sigma_out, int32_t *status,
                                            qamw_stream_t stream) {
  // Argument validation of the workspace version: with no workspace it returns
  // before any CUDA call, QAMW_EWORKSPACE meaning "every other argument is valid".
  const int rc = qamw_calibrate_sigma(W, w_dtype, M, K, ldw, act_rms, alpha, block, sign_seed, sigma_out, nullptr,
                                      0, status, stream);
  if (rc != QAMW_EWORKSPACE) return rc;
  const size_t need = qamw_calibrate_workspace_bytes(M, K);
  if (need > (size_t)QAMW_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "qamw_calibrate_sigma_noalloc: M=%lld x K=%lld needs %zu bytes of scratch; the built-in area holds %u "
             "(use qamw_calibrate_sigma with a workspace)",
             (long long)M, (long long)K, need, (unsigned)QAMW_NOALLOC_SCRATCH_BYTES);
    qamw::set_last_error(msg);
    return QAMW_EUNSUPPORTED;
  }
  void *scratch = nullptr;
  const cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "qamw_calibrate_sigma_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    qamw::set_last_error(msg);
    return QAMW_ECUDA;
  }
  // Every byte of the scratch that the calibration reads is written earlier in
  // the same call, so nothing has to be cleared between calls.
  return qamw_calibrate_sigma(W, w_dtype, M, K, ldw, act_rms, alpha, block, sign_seed, sigma_out, scratch,
                              (size_t)QAMW_NOALLOC_SCRATCH_BYTES, status, stream);
}
