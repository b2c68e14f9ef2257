// eqlin_noalloc.cu -- weight/bias gradient for callers that cannot allocate.
//
// Some callers cannot call cudaMalloc at all: code that runs while a custom
// allocator owns the device memory, runtimes that forbid allocation after
// start-up, or plug-ins loaded into a host that manages memory itself.  Such a
// caller cannot create an eqlin_t (that allocates the Fourier weights and the
// workspace), but the weight gradient needs no weights: it depends only on x
// and gy.  eqlin_backward_dw_noalloc computes dW and db with the same
// tensor-core kernels as eqlin_backward_dw and keeps its per-chunk partial
// sums in the fixed-size device array below instead of an allocated workspace.
//
// The array is a file-scope __device__ object: the CUDA runtime reserves it on
// a device when this module's device code is loaded there and holds it until
// the process exits.  Module loading is lazy, so that happens at the first
// call on each device -- inside cudaGetSymbolAddress, which this file calls
// once per device, with that device current, to turn the host-side stand-in
// `g_dw_scratch` into the array's device address.  A device without room for
// the array makes that lookup fail with cudaErrorMemoryAllocation, reported
// as EQLIN_ERR_OOM.
#include <mutex>

#include "eqlin_internal.cuh"

namespace {

constexpr size_t kPartialBytes = size_t(64) << 20;       // per-chunk partial planes
constexpr size_t kScratchBytes = kPartialBytes + 256;     // + the kernels' error record

static __device__ __align__(256) unsigned char g_dw_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_dw_scratch on the current device (looked up once per device).
cudaError_t scratch_address(int dev, unsigned char** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_dw_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_addr[dev]);
  return cudaSuccess;
}

}  // namespace

extern "C" eqlin_status_t eqlin_backward_dw_noalloc(int T, int64_t Cp, int64_t Dp,
                                                    eqlin_dtype_t dtype, const void* x,
                                                    const void* gy, float* dW, float* db,
                                                    int64_t N, void* stream) {
  if (dtype != EQLIN_F32 && dtype != EQLIN_F16 && dtype != EQLIN_BF16) return EQLIN_ERR_INVALID_ARG;
  if (Cp < 1 || Dp < 1 || N < 0 || !dW) return EQLIN_ERR_INVALID_ARG;
  if (T != 1 && T != 2 && T != 4 && T != 8) return EQLIN_ERR_UNSUPPORTED;
  if (dtype == EQLIN_F32 || Cp > 65536 || Dp > 65536) return EQLIN_ERR_UNSUPPORTED;
  if ((Cp * T * 2) % 16 || (Dp * T * 2) % 16) return EQLIN_ERR_MISALIGNED;
  if (((uintptr_t)dW & 15u) || (db && ((uintptr_t)db & 15u))) return EQLIN_ERR_MISALIGNED;
  if (N > 0 && (!x || !gy)) return EQLIN_ERR_INVALID_ARG;
  if (N > 0 && (((uintptr_t)x & 15u) || ((uintptr_t)gy & 15u))) return EQLIN_ERR_MISALIGNED;

  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return EQLIN_ERR_CUDA;
  // makes the device's primary context current in this host thread (the
  // tensor-map encoding needs one; a thread may have selected the device only)
  if (cudaSetDevice(dev) != cudaSuccess) return EQLIN_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return EQLIN_ERR_CUDA;
  // The partials of the largest token split this shape can use must fit.
  if (eqlin::tc_dw_workspace_bytes(T, Cp, Dp, sms) > kPartialBytes) return EQLIN_ERR_UNSUPPORTED;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (N == 0) {
    cudaError_t e = cudaMemsetAsync(dW, 0, (size_t)Dp * Cp * T * sizeof(float), st);
    if (e == cudaSuccess && db) e = cudaMemsetAsync(db, 0, (size_t)Dp * sizeof(float), st);
    return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
  }

  unsigned char* scratch = nullptr;
  {
    const cudaError_t e = scratch_address(dev, &scratch);
    if (e != cudaSuccess) {
      cudaGetLastError();   // a failed lazy load leaves no sticky error behind
      return e == cudaErrorMemoryAllocation ? EQLIN_ERR_OOM : EQLIN_ERR_CUDA;
    }
  }

  eqlin::Handle h;                       // a description of the call; owns nothing
  h.T = T;
  h.Cp = Cp;
  h.Dp = Dp;
  h.dtype = dtype;
  h.device = dev;
  h.sm_count = sms;
  h.ws = reinterpret_cast<float*>(scratch);
  h.ws_bytes = kPartialBytes;
  h.err = reinterpret_cast<int*>(scratch + kPartialBytes);
  // The error word keeps the previous call's value; it must start at zero.
  if (cudaMemsetAsync(h.err, 0, 4 * sizeof(int), st) != cudaSuccess) return EQLIN_ERR_CUDA;
  const cudaError_t e = eqlin::launch_tc_dw(h, x, gy, dW, db, N, st);
  return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
}
