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
// so the address is looked up with cudaGetSymbolAddress (on the first call
// made with a device current) and cached. The cache entry remembers the
// driver context it was looked up in: after cudaDeviceReset, or with another
// context current on the same device, the module is loaded anew at another
// address, so a call in a new context looks the address up again.
#include <cstdio>
#include <mutex>

#include <cuda.h>

#include "qamw.h"
#include "qamw_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_calib_scratch[QAMW_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
struct ScratchEntry {
  CUcontext ctx;
  void *addr;
};
ScratchEntry g_scratch[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// The driver's cuCtxGetCurrent, reached through the runtime (no -lcuda).
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of this module's scratch area in the current context.
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CtxGetCurrentFn get = ctx_get_current();
  if (get == nullptr) return cudaErrorDeviceUninitialized;
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;   // NULL before the runtime's first use
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchEntry &ent = g_scratch[dev];
  if (ctx == nullptr || ent.addr == nullptr || ent.ctx != ctx) {
    void *p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_calib_scratch)) != cudaSuccess) return e;   // sets a context current
    if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
    ent.ctx = ctx;
    ent.addr = p;
  }
  *out = ent.addr;
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
