// eqlin_api.cu -- the C ABI: handle lifetime, argument checks, dispatch.
//
// Every entry point validates its arguments on the host, returns a status and
// enqueues kernels on the caller's stream.  No entry point synchronises except
// eqlin_get_error (which reads the device error word) and eqlin_destroy.
#include <stdlib.h>
#include <string.h>
#include <stdio.h>
#include <atomic>
#include <mutex>
#include <new>
#include <set>
#include <utility>

#include "eqlin_internal.cuh"

using eqlin::Handle;

namespace eqlin {
static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

cudaError_t set_smem_limit(const void* kernel, int bytes) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev})) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.insert({kernel, dev});
  return e;
}

void* tensor_map_encoder() {
  // function-local static: initialised once, thread-safe
  static void* const fn = []() -> void* {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return ptr;
    return nullptr;
  }();
  return fn;
}
}  // namespace eqlin

struct eqlin_handle {
  Handle h;
};

namespace {

size_t elem_size(eqlin_dtype_t dt) { return dt == EQLIN_F32 ? 4 : 2; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Make the handle's device current for the duration of a call.  The set is
// unconditional: besides selecting the device it makes the device's primary
// context current in this host thread, which a thread that has only selected
// the device (an autograd worker, say) may not have yet, and which the
// tensor-map encoding needs.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
    if (cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

void free_split(Handle& h) {
  for (int pass = 0; pass < 2; ++pass) {
    cudaFree(h.split_ws[pass]);
    cudaFree(h.split_flags[pass]);
    h.split_ws[pass] = nullptr;
    h.split_flags[pass] = nullptr;
    h.split_pairs[pass] = h.split_cols[pass] = 0;
  }
}

// The tail-split workspaces (tc_split_tiles) of the f16/bf16 tensor-core
// passes long enough to split: one FP32 accumulator per pair of CTAs, with
// its flags.
bool alloc_split(Handle& h) {
  for (int pass = 0; pass < 2; ++pass) {
    const int64_t K = pass ? h.Dp : h.Cp;
    if (h.split_ws[pass] || (K + eqlin::TC_BK - 1) / eqlin::TC_BK < eqlin::kSplitMinStages ||
        !eqlin::tc_supported(h, pass == 1))
      continue;
    int cols = h.T * (pass ? h.bo_bwd : h.bo_fwd);
    if (pass == 0 && h.bo_gauss && 5 * h.bo_gauss > cols) cols = 5 * h.bo_gauss;
    const int pairs = h.sm_count / 2;
    const size_t nflags = (size_t)2 * pairs + 1;
    const bool ok = cudaMalloc(&h.split_ws[pass], (size_t)pairs * 128 * cols * sizeof(float)) == cudaSuccess &&
                    cudaMalloc(&h.split_flags[pass], nflags * sizeof(int)) == cudaSuccess &&
                    cudaMemset(h.split_flags[pass], 0, nflags * sizeof(int)) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      free_split(h);
      return false;
    }
    h.split_pairs[pass] = pairs;
    h.split_cols[pass] = cols;
  }
  return true;
}

void free_all(Handle& h) {
  cudaFree(h.wf_fwd);
  cudaFree(h.wf_bwd);
  cudaFree(h.wt_fwd);
  cudaFree(h.wt_bwd);
  cudaFree(h.bias);
  cudaFree(h.ws);
  cudaFree(h.err);
  cudaFree(h.wt_gauss);
  h.wt_gauss = nullptr;
  free_split(h);
  h.wf_fwd = h.wf_bwd = nullptr;
  h.wt_fwd = h.wt_bwd = nullptr;
  h.bias = h.ws = nullptr;
  h.err = nullptr;
}

eqlin_status_t check_io(const Handle& h, const void* a, const void* b, int64_t N) {
  if (N < 0) return EQLIN_ERR_INVALID_ARG;
  if (N == 0) return EQLIN_OK;
  if (!a || !b) return EQLIN_ERR_INVALID_ARG;
  if (!h.has_weights) return EQLIN_ERR_NO_WEIGHTS;
  if (!aligned16(a) || !aligned16(b)) return EQLIN_ERR_MISALIGNED;
  return EQLIN_OK;
}

}  // namespace

extern "C" {

const char* eqlin_status_string(eqlin_status_t s) {
  switch (s) {
    case EQLIN_OK: return "ok";
    case EQLIN_ERR_INVALID_ARG: return "invalid argument";
    case EQLIN_ERR_UNSUPPORTED: return "unsupported group order or size";
    case EQLIN_ERR_MISALIGNED: return "pointer or row not 16-byte aligned";
    case EQLIN_ERR_CUDA: return "CUDA error";
    case EQLIN_ERR_NO_WEIGHTS: return "weights not set";
    case EQLIN_ERR_TIMEOUT: return "device-side wait timed out";
    case EQLIN_ERR_OOM: return "device out of memory";
  }
  return "unknown status";
}

eqlin_status_t eqlin_create(int T, int64_t Cp, int64_t Dp, eqlin_dtype_t dtype, eqlin_t* out) {
  return eqlin_create_group(EQLIN_GROUP_CYCLIC, T, Cp, Dp, dtype, out);
}

eqlin_status_t eqlin_create_group(eqlin_group_t group, int m, int64_t Cp, int64_t Dp, eqlin_dtype_t dtype,
                                  eqlin_t* out) {
  if (!out) return EQLIN_ERR_INVALID_ARG;
  *out = nullptr;
  if (dtype != EQLIN_F32 && dtype != EQLIN_F16 && dtype != EQLIN_BF16) return EQLIN_ERR_INVALID_ARG;
  if (group != EQLIN_GROUP_CYCLIC && group != EQLIN_GROUP_DIHEDRAL) return EQLIN_ERR_INVALID_ARG;
  if (Cp < 1 || Dp < 1) return EQLIN_ERR_INVALID_ARG;
  const bool dihedral = group == EQLIN_GROUP_DIHEDRAL;
  if (dihedral && !eqlin::dihedral_supported(m)) return EQLIN_ERR_UNSUPPORTED;
  const int T = dihedral ? 2 * m : m;      // group order
  if (!dihedral && T != 1 && T != 2 && T != 3 && T != 4 && T != 6 && T != 8) return EQLIN_ERR_UNSUPPORTED;
  if (Cp > 65536 || Dp > 65536) return EQLIN_ERR_UNSUPPORTED;
  const size_t e = elem_size(dtype);
  if ((Cp * T * e) % 16 || (Dp * T * e) % 16) return EQLIN_ERR_MISALIGNED;

  eqlin_handle* hh = new (std::nothrow) eqlin_handle();
  if (!hh) return EQLIN_ERR_OOM;
  Handle& h = hh->h;
  h.T = T;
  h.group = group;
  h.m = m;
  h.Cp = Cp;
  h.Dp = Dp;
  h.dtype = dtype;
  if (cudaGetDevice(&h.device) != cudaSuccess) { delete hh; return EQLIN_ERR_CUDA; }
  if (cudaDeviceGetAttribute(&h.sm_count, cudaDevAttrMultiProcessorCount, h.device) != cudaSuccess) {
    delete hh;
    return EQLIN_ERR_CUDA;
  }
  const size_t planes = (size_t)T * Cp * Dp;
  h.ws_bytes = eqlin::simt_dw_workspace_bytes(T, Cp, Dp);
  if (!dihedral && dtype == EQLIN_F32 && eqlin::tc32_dw_supported(h)) {
    const size_t tcb = eqlin::tc32_dw_workspace_bytes(T, Cp, Dp, h.sm_count);
    if (tcb > h.ws_bytes) h.ws_bytes = tcb;
  }
  if (!dihedral && dtype != EQLIN_F32) {
    const size_t tcb = eqlin::tc_dw_workspace_bytes(T, Cp, Dp, h.sm_count);
    if (tcb > h.ws_bytes) h.ws_bytes = tcb;
    const size_t tcs = eqlin::tc_dws_workspace_bytes(T, Cp, Dp, h.sm_count);
    if (tcs > h.ws_bytes) h.ws_bytes = tcs;
  }
  bool ok = cudaMalloc(&h.wf_fwd, planes * 4) == cudaSuccess &&
            cudaMalloc(&h.wf_bwd, planes * 4) == cudaSuccess &&
            cudaMalloc(&h.bias, (size_t)Dp * 4) == cudaSuccess &&
            cudaMalloc(&h.ws, h.ws_bytes) == cudaSuccess &&
            cudaMalloc(&h.err, 4 * sizeof(int)) == cudaSuccess;
  // tensor-core weight tiles only where a tensor-core pass exists (T | 8)
  if (ok && !dihedral && dtype != EQLIN_F32 && (eqlin::tc_supported(h, false) || eqlin::tc_supported(h, true))) {
    h.bo_fwd = eqlin::tc_pick_bo(T, Dp);
    h.bo_bwd = eqlin::tc_pick_bo(T, Cp);
    const size_t nf = (size_t)eqlin::wtile_elems(T, h.bo_fwd, Dp, Cp);
    const size_t nb = (size_t)eqlin::wtile_elems(T, h.bo_bwd, Cp, Dp);
    ok = cudaMalloc(&h.wt_fwd, nf * e) == cudaSuccess && cudaMalloc(&h.wt_bwd, nb * e) == cudaSuccess;
    // padding rows and K columns of the tiles stay zero
    if (ok) ok = cudaMemset(h.wt_fwd, 0, nf * e) == cudaSuccess && cudaMemset(h.wt_bwd, 0, nb * e) == cudaSuccess;
    // the p4 three-product forward image (eqlin_forward_gauss)
    if (ok && T == 4 && eqlin::tc_supported(h, false) && eqlin::tc_supported(h, true)) {
      h.bo_gauss = eqlin::tc_pick_bo_gauss(Dp);
      const size_t ng = (size_t)eqlin::wtile_elems(T, h.bo_gauss, Dp, Cp);
      ok = cudaMalloc(&h.wt_gauss, ng * e) == cudaSuccess && cudaMemset(h.wt_gauss, 0, ng * e) == cudaSuccess;
    }
  }
  // FP32: the 3xTF32 hi/lo images, for the passes whose reduction is short
  // enough (tc32_pass_ok); the other pass keeps the FP32 SIMT planes
  const bool tc32_f = ok && eqlin::tc32_pass_ok(h, false), tc32_b = ok && eqlin::tc32_pass_ok(h, true);
  if (tc32_f || tc32_b) {
    h.bo_fwd = eqlin::tc32_pick_bo(T, Dp);
    h.bo_bwd = eqlin::tc32_pick_bo(T, Cp);
    const size_t nf = (size_t)eqlin::wtile32_elems(T, h.bo_fwd, Dp, Cp);
    const size_t nb = (size_t)eqlin::wtile32_elems(T, h.bo_bwd, Cp, Dp);
    ok = cudaMalloc(&h.wt_fwd, nf * 4) == cudaSuccess && cudaMalloc(&h.wt_bwd, nb * 4) == cudaSuccess;
    if (ok) ok = cudaMemset(h.wt_fwd, 0, nf * 4) == cudaSuccess && cudaMemset(h.wt_bwd, 0, nb * 4) == cudaSuccess;
  }
  if (ok) ok = cudaMemset(h.err, 0, 4 * sizeof(int)) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    free_all(h);
    delete hh;
    return EQLIN_ERR_OOM;
  }
  h.need_simt_fwd = dihedral || (dtype == EQLIN_F32 ? !tc32_f : !eqlin::tc_supported(h, false));
  h.need_simt_bwd = dihedral || (dtype == EQLIN_F32 ? !tc32_b : !eqlin::tc_supported(h, true));
  snprintf(h.backend, sizeof(h.backend), "fwd=%s dx=%s dw=%s", h.need_simt_fwd ? "simt" : "tcgen05",
           h.need_simt_bwd ? "simt" : "tcgen05",
           eqlin::tc_dw_supported(h) || eqlin::tc32_dw_supported(h) ? "tcgen05" : "simt");
  *out = hh;
  return EQLIN_OK;
}

void eqlin_destroy(eqlin_t hh) {
  if (!hh) return;
  DeviceGuard g(hh->h.device);
  cudaDeviceSynchronize();
  free_all(hh->h);
  delete hh;
}

eqlin_status_t eqlin_set_weights(eqlin_t hh, const void* W, const void* b, void* stream) {
  if (!hh || !W) return EQLIN_ERR_INVALID_ARG;
  Handle& h = hh->h;
  if (!aligned16(W) || (b && ((uintptr_t)b % elem_size(h.dtype)))) return EQLIN_ERR_MISALIGNED;
  DeviceGuard g(h.device);
  if (!g.ok) return EQLIN_ERR_CUDA;
  cudaError_t e = h.group == EQLIN_GROUP_DIHEDRAL ? eqlin::launch_dihedral_pretransform(h, W, b, (cudaStream_t)stream)
                                                  : eqlin::launch_pretransform(h, W, b, (cudaStream_t)stream);
  if (e != cudaSuccess) return EQLIN_ERR_CUDA;
  h.has_weights = true;
  return EQLIN_OK;
}

eqlin_status_t eqlin_forward(eqlin_t hh, const void* x, void* y, int64_t N, void* stream) {
  if (!hh) return EQLIN_ERR_INVALID_ARG;
  Handle& h = hh->h;
  eqlin_status_t s = check_io(h, x, y, N);
  if (s != EQLIN_OK || N == 0) return s;
  DeviceGuard g(h.device);
  if (!g.ok) return EQLIN_ERR_CUDA;
  cudaError_t e;
  if (h.group == EQLIN_GROUP_DIHEDRAL)
    e = eqlin::launch_dihedral_apply(h, false, x, y, N, (cudaStream_t)stream);
  else if (h.dtype != EQLIN_F32 && eqlin::tc_supported(h, false))
    e = eqlin::launch_tc_apply(h, false, x, y, nullptr, N, (cudaStream_t)stream);
  else if (h.dtype == EQLIN_F32 && !h.need_simt_fwd)
    e = eqlin::launch_tc32_apply(h, false, x, y, N, (cudaStream_t)stream);
  else
    e = eqlin::launch_simt_apply(h, false, x, y, N, (cudaStream_t)stream);
  return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
}

eqlin_status_t eqlin_forward_gauss(eqlin_t hh, const void* x, void* y, int64_t N, void* stream) {
  if (!hh) return EQLIN_ERR_INVALID_ARG;
  Handle& h = hh->h;
  if (h.group != EQLIN_GROUP_CYCLIC || h.T != 4 || !h.wt_gauss) return EQLIN_ERR_UNSUPPORTED;
  eqlin_status_t s = check_io(h, x, y, N);
  if (s != EQLIN_OK || N == 0) return s;
  DeviceGuard g(h.device);
  if (!g.ok) return EQLIN_ERR_CUDA;
  const cudaError_t e = eqlin::launch_tc_apply_gauss(h, x, y, N, (cudaStream_t)stream);
  return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
}

eqlin_status_t eqlin_backward_dx(eqlin_t hh, const void* gy, void* dx, int64_t N, void* stream) {
  if (!hh) return EQLIN_ERR_INVALID_ARG;
  Handle& h = hh->h;
  eqlin_status_t s = check_io(h, gy, dx, N);
  if (s != EQLIN_OK || N == 0) return s;
  DeviceGuard g(h.device);
  if (!g.ok) return EQLIN_ERR_CUDA;
  cudaError_t e;
  if (h.group == EQLIN_GROUP_DIHEDRAL)
    e = eqlin::launch_dihedral_apply(h, true, gy, dx, N, (cudaStream_t)stream);
  else if (h.dtype != EQLIN_F32 && eqlin::tc_supported(h, true))
    e = eqlin::launch_tc_apply(h, true, gy, dx, nullptr, N, (cudaStream_t)stream);
  else if (h.dtype == EQLIN_F32 && !h.need_simt_bwd)
    e = eqlin::launch_tc32_apply(h, true, gy, dx, N, (cudaStream_t)stream);
  else
    e = eqlin::launch_simt_apply(h, true, gy, dx, N, (cudaStream_t)stream);
  return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
}

eqlin_status_t eqlin_backward_dw(eqlin_t hh, const void* x, const void* gy, float* dW, float* db,
                                 int64_t N, void* stream) {
  if (!hh) return EQLIN_ERR_INVALID_ARG;
  Handle& h = hh->h;
  if (!dW || N < 0) return EQLIN_ERR_INVALID_ARG;
  if (!aligned16(dW) || (db && !aligned16(db))) return EQLIN_ERR_MISALIGNED;
  DeviceGuard g(h.device);
  if (!g.ok) return EQLIN_ERR_CUDA;
  if (N == 0) {
    cudaError_t e = cudaMemsetAsync(dW, 0, (size_t)h.Dp * h.Cp * h.T * 4, (cudaStream_t)stream);
    if (e == cudaSuccess && db) e = cudaMemsetAsync(db, 0, (size_t)h.Dp * 4, (cudaStream_t)stream);
    return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
  }
  eqlin_status_t s = check_io(h, x, gy, N);
  if (s != EQLIN_OK) return s;
  cudaError_t e = h.group == EQLIN_GROUP_DIHEDRAL ? eqlin::launch_dihedral_dw(h, x, gy, dW, db, N, (cudaStream_t)stream)
                  : eqlin::tc_dw_supported(h)      ? eqlin::launch_tc_dw(h, x, gy, dW, db, N, (cudaStream_t)stream)
                  : eqlin::tc32_dw_supported(h)    ? eqlin::launch_tc32_dw(h, x, gy, dW, db, N, (cudaStream_t)stream)
                                                   : eqlin::launch_simt_dw(h, x, gy, dW, db, N, (cudaStream_t)stream);
  return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
}

// The stash forms and the weight gradient from spectra serve cyclic f16/bf16
// layers of order T | 8 (the tensor-core kernels for T = 3 and 6 have no
// stash form).
static bool stash_order(const Handle& h) {
  return h.group == EQLIN_GROUP_CYCLIC && h.dtype != EQLIN_F32 &&
         (h.T == 1 || h.T == 2 || h.T == 4 || h.T == 8);
}

int64_t eqlin_spectra_ld(int64_t N) { return N < 0 ? -1 : eqlin::spectra_ld(N); }

eqlin_status_t eqlin_forward_stash(eqlin_t hh, const void* x, void* y, void* xs, int64_t N, void* stream) {
  if (!hh) return EQLIN_ERR_INVALID_ARG;
  Handle& h = hh->h;
  eqlin_status_t s = check_io(h, x, y, N);
  if (s != EQLIN_OK || N == 0) return s;
  if (!xs) return EQLIN_ERR_INVALID_ARG;
  if (!aligned16(xs)) return EQLIN_ERR_MISALIGNED;
  if (!stash_order(h) || !eqlin::tc_supported(h, false))
    return EQLIN_ERR_UNSUPPORTED;
  DeviceGuard g(h.device);
  if (!g.ok) return EQLIN_ERR_CUDA;
  const cudaError_t e = eqlin::launch_tc_apply(h, false, x, y, xs, N, (cudaStream_t)stream);
  return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
}

eqlin_status_t eqlin_backward_dx_stash(eqlin_t hh, const void* gy, void* dx, void* gs, int64_t N, void* stream) {
  if (!hh) return EQLIN_ERR_INVALID_ARG;
  Handle& h = hh->h;
  eqlin_status_t s = check_io(h, gy, dx, N);
  if (s != EQLIN_OK || N == 0) return s;
  if (!gs) return EQLIN_ERR_INVALID_ARG;
  if (!aligned16(gs)) return EQLIN_ERR_MISALIGNED;
  if (!stash_order(h) || !eqlin::tc_supported(h, true))
    return EQLIN_ERR_UNSUPPORTED;
  DeviceGuard g(h.device);
  if (!g.ok) return EQLIN_ERR_CUDA;
  const cudaError_t e = eqlin::launch_tc_apply(h, true, gy, dx, gs, N, (cudaStream_t)stream);
  return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
}

eqlin_status_t eqlin_backward_dw_spectra(eqlin_t hh, const void* xs, const void* gs, float* dW, float* db,
                                         int64_t N, void* stream) {
  if (!hh) return EQLIN_ERR_INVALID_ARG;
  Handle& h = hh->h;
  if (!dW || N < 0) return EQLIN_ERR_INVALID_ARG;
  if (!aligned16(dW) || (db && !aligned16(db))) return EQLIN_ERR_MISALIGNED;
  if (!stash_order(h) || !eqlin::tc_dw_supported(h))
    return EQLIN_ERR_UNSUPPORTED;
  DeviceGuard g(h.device);
  if (!g.ok) return EQLIN_ERR_CUDA;
  if (N == 0) {
    cudaError_t e = cudaMemsetAsync(dW, 0, (size_t)h.Dp * h.Cp * h.T * 4, (cudaStream_t)stream);
    if (e == cudaSuccess && db) e = cudaMemsetAsync(db, 0, (size_t)h.Dp * 4, (cudaStream_t)stream);
    return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
  }
  eqlin_status_t s = check_io(h, xs, gs, N);
  if (s != EQLIN_OK) return s;
  const cudaError_t e = eqlin::launch_tc_dw_spectra(h, xs, gs, dW, db, N, (cudaStream_t)stream);
  return e == cudaSuccess ? EQLIN_OK : EQLIN_ERR_CUDA;
}

eqlin_status_t eqlin_backward(eqlin_t hh, const void* gy, const void* xs, void* dx, void* gs, float* dW,
                              float* db, int64_t N, void* stream) {
  eqlin_status_t s = eqlin_backward_dx_stash(hh, gy, dx, gs, N, stream);
  if (s != EQLIN_OK) return s;
  return eqlin_backward_dw_spectra(hh, xs, gs, dW, db, N, stream);
}

eqlin_status_t eqlin_get_error(eqlin_t hh) {
  if (!hh) return EQLIN_ERR_INVALID_ARG;
  Handle& h = hh->h;
  DeviceGuard g(h.device);
  int rec[4] = {0, 0, 0, 0};
  if (cudaMemcpy(rec, h.err, sizeof(rec), cudaMemcpyDeviceToHost) != cudaSuccess) return EQLIN_ERR_CUDA;
  const int v = rec[0];
  if (v != eqlin::DEV_OK) {
    for (int i = 0; i < 4; ++i) h.last_error[i] = (uint32_t)rec[i];
    const int zero[4] = {0, 0, 0, 0};
    if (cudaMemcpy(h.err, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return EQLIN_ERR_CUDA;
  }
  return v == eqlin::DEV_OK ? EQLIN_OK : v == eqlin::DEV_TIMEOUT ? EQLIN_ERR_TIMEOUT : EQLIN_ERR_CUDA;
}

eqlin_status_t eqlin_error_detail(eqlin_t hh, uint32_t detail[4]) {
  if (!hh || !detail) return EQLIN_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i) detail[i] = hh->h.last_error[i];
  return EQLIN_OK;
}

eqlin_status_t eqlin_set_tail_split(eqlin_t hh, int enable) {
  if (!hh) return EQLIN_ERR_INVALID_ARG;
  Handle& h = hh->h;
  DeviceGuard g(h.device);
  // the workspaces may still be in use by this handle's queued launches
  if (cudaDeviceSynchronize() != cudaSuccess) return EQLIN_ERR_CUDA;
  if (!enable) {
    free_split(h);
    return EQLIN_OK;
  }
  if (h.group != EQLIN_GROUP_CYCLIC || h.dtype == EQLIN_F32) return EQLIN_OK;   // no tensor-core split there
  return alloc_split(h) ? EQLIN_OK : EQLIN_ERR_OOM;
}

eqlin_status_t eqlin_set_wait_limit(eqlin_t hh, uint32_t iterations) {
  if (!hh) return EQLIN_ERR_INVALID_ARG;
  hh->h.wait_limit = iterations;
  return EQLIN_OK;
}

const char* eqlin_backend_name(eqlin_t hh) { return hh ? hh->h.backend : "none"; }

uint64_t eqlin_launch_count(void) { return eqlin::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
