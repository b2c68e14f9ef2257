// eqlin_internal.cuh -- shared declarations of the Flash EQ-Linear CUDA library.
//
// Group-axis transforms used by every kernel ("Flash EQ-Linear", technical
// summary, section "Abordagem Algoritmica"): with theta = 2*pi*k*t/T,
//
//   forward DFT   V_k = sum_t v_t (cos theta - i sin theta),   k = 0 .. floor(T/2)
//   inverse DFT   v_s = (1/T) [ V_0 + (-1)^s V_{T/2} + 2 sum_{0<k<T/2} Re(V_k e^{+i theta_s}) ]
//
// Real inputs give a Hermitian spectrum, so only the half spectrum is kept
// (item 2 of the same section).  A T-vector is held as T real "planes":
//   plane 0             Re V_0
//   plane 1 (T even)    Re V_{T/2}
//   plane nreal+2(k-1)  Re V_k,  plane nreal+2(k-1)+1  Im V_k,  k = 1 .. T/2-1
// For p4 that is [V0, V2, Re V1, Im V1], and the transforms need only adds,
// subtracts and power-of-two scales (section "Especializacao ... p4").
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/eqlin.h"

namespace eqlin {

// ------------------------------------------------------------- element types
template <typename E> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__half> {
  static __device__ __forceinline__ float to_f(__half v) { return __half2float(v); }
  static __device__ __forceinline__ __half from_f(float v) { return __float2half_rn(v); }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// --------------------------------------------------- group-axis plane tables
// cos/sin of 2*pi*j/8 for T in {1,2,4,8} (entry j * 8/T), and of 2*pi*j/12
// for T in {3,6} (entry j * 12/T).  The only inexact entries are sqrt(2)/2
// (T = 8) and sqrt(3)/2 (T = 3, 6), each rounded once to float; the others
// are 0, +-1/2 and +-1.
#define EQLIN_RSQRT2 0.70710678118654752440f
#define EQLIN_SQRT3_2 0.86602540378443864676f

template <int T> struct Group {
  static_assert(8 % T == 0 || 12 % T == 0, "T in {1, 2, 3, 4, 6, 8}");
  static constexpr int nreal = (T % 2) ? 1 : 2;         // k = 0, and k = T/2 for even T
  static constexpr int ncomplex = (T - nreal) / 2;      // k = 1 .. ceil(T/2)-1
  static constexpr int planes = T;                      // real planes of the half spectrum
  // Real GEMM count R(T): one per real frequency, four per complex one.
  static constexpr int gemms = nreal + 4 * ncomplex;

  static __host__ __device__ __forceinline__ float cos8(int j) {
    j &= 7;
    return j == 0 ? 1.f : j == 1 ? EQLIN_RSQRT2 : j == 2 ? 0.f : j == 3 ? -EQLIN_RSQRT2
         : j == 4 ? -1.f : j == 5 ? -EQLIN_RSQRT2 : j == 6 ? 0.f : EQLIN_RSQRT2;
  }
  static __host__ __device__ __forceinline__ float sin8(int j) { return cos8(j - 2); }
  static __host__ __device__ __forceinline__ float cos12(int j) {
    j = ((j % 12) + 12) % 12;
    return j == 0 ? 1.f : j == 1 ? EQLIN_SQRT3_2 : j == 2 ? 0.5f : j == 3 ? 0.f : j == 4 ? -0.5f
         : j == 5 ? -EQLIN_SQRT3_2 : j == 6 ? -1.f : j == 7 ? -EQLIN_SQRT3_2 : j == 8 ? -0.5f
         : j == 9 ? 0.f : j == 10 ? 0.5f : EQLIN_SQRT3_2;
  }
  static __host__ __device__ __forceinline__ float sin12(int j) { return cos12(j - 3); }
  // cos / sin of 2*pi*k*t/T
  static __host__ __device__ __forceinline__ float c(int k, int t) {
    if constexpr (8 % T == 0) return cos8(k * t * (8 / T));
    else return cos12(k * t * (12 / T));
  }
  static __host__ __device__ __forceinline__ float s(int k, int t) {
    if constexpr (8 % T == 0) return sin8(k * t * (8 / T));
    else return sin12(k * t * (12 / T));
  }

  // Forward real DFT of v[0..T) into planes P[0..T).
  static __host__ __device__ __forceinline__ void dft(const float* v, float* P) {
    float a = 0.f;
#pragma unroll
    for (int t = 0; t < T; ++t) a += v[t];
    P[0] = a;
    if constexpr (T % 2 == 0) {
      float h = 0.f;
#pragma unroll
      for (int t = 0; t < T; ++t) h += (t & 1) ? -v[t] : v[t];
      P[1] = h;
    }
#pragma unroll
    for (int k = 1; k <= ncomplex; ++k) {
      float re = 0.f, im = 0.f;
#pragma unroll
      for (int t = 0; t < T; ++t) {
        const float ct = c(k, t), st = s(k, t);
        if (ct != 0.f) re += (ct == 1.f ? v[t] : ct == -1.f ? -v[t] : ct * v[t]);
        if (st != 0.f) im -= (st == 1.f ? v[t] : st == -1.f ? -v[t] : st * v[t]);
      }
      P[nreal + 2 * (k - 1)] = re;
      P[nreal + 2 * (k - 1) + 1] = im;
    }
  }

  // Inverse real DFT of planes that already carry the scales 1/T (real
  // frequencies) and 2/T (complex ones): v_s = P0 + (-1)^s P1 + sum_k
  // (Re_k cos - Im_k sin), plus `add` on every output.
  static __host__ __device__ __forceinline__ void idft_scaled(const float* P, float add, float* v) {
    const float a = P[0] + add;
    if (T == 1) { v[0] = a; return; }
    // even T: + (-1)^s P1 (the k = T/2 plane); odd T has none
    const float ep = (T % 2 == 0) ? a + P[1] : a, em = (T % 2 == 0) ? a - P[1] : a;
#pragma unroll
    for (int s_ = 0; s_ < T; ++s_) {
      float acc = (s_ & 1) ? em : ep;
#pragma unroll
      for (int k = 1; k <= ncomplex; ++k) {
        const float cs = c(k, s_), sn = s(k, s_);
        const float re = P[nreal + 2 * (k - 1)], im = P[nreal + 2 * (k - 1) + 1];
        if (cs != 0.f) acc += (cs == 1.f ? re : cs == -1.f ? -re : cs * re);
        if (sn != 0.f) acc -= (sn == 1.f ? im : sn == -1.f ? -im : sn * im);
      }
      v[s_] = acc;
    }
  }

  // Inverse real DFT of planes P into v[0..T), including the 1/T.
  static __host__ __device__ __forceinline__ void idft(const float* P, float* v) {
#pragma unroll
    for (int s_ = 0; s_ < T; ++s_) {
      float a = P[0];
      if constexpr (T % 2 == 0) a += (s_ & 1) ? -P[1] : P[1];
      float acc2 = 0.f;
#pragma unroll
      for (int k = 1; k <= ncomplex; ++k) {
        const float cs = c(k, s_), sn = s(k, s_);
        const float re = P[nreal + 2 * (k - 1)], im = P[nreal + 2 * (k - 1) + 1];
        if (cs != 0.f) acc2 += (cs == 1.f ? re : cs == -1.f ? -re : cs * re);
        if (sn != 0.f) acc2 -= (sn == 1.f ? im : sn == -1.f ? -im : sn * im);
      }
      v[s_] = (a + 2.f * acc2) * (1.f / T);
    }
  }
};

// --------------------------------------------- tensor-core weight tiles
// The tensor-core kernels read the Fourier weight planes as tiles of BO
// output rows x 16 K (input channels), one per (output tile, K stage) and
// plane, stored in the exact 32-byte-swizzled image the MMA reads from shared
// memory, so that one contiguous bulk copy fetches a stage.  For K-major rows
// of 32 bytes, 16-byte chunk j of row r sits at chunk j ^ ((r >> 2) & 1).
//
// BO, the output channels of a tile, is chosen per pass from the pass's
// output width O.  The accumulator of a tile takes T * BO TMEM columns (of
// 512), a complex frequency's block product is an N = 2 * BO MMA (N <= 256),
// and the epilogue stores 64 / T channels per chunk in an even number of
// chunks.  For T = 4 the candidates are 128, 96, 64 and 32: the one that pads
// O least, the wider on a tie (fewer output tiles, so fewer repeats of the
// input transform).  Other T use one width.
constexpr int TC_BK = 16;
__host__ __device__ constexpr int tc_planes(int T) {
  return (T % 2 ? 1 : 2) + 3 * ((T - (T % 2 ? 1 : 2)) / 2);
}
// Tile width of the p4 three-product form: 96, 64 or 32, padding O least
// (wider on a tie).
inline int tc_pick_bo_gauss(int64_t O) {
  int best = 96;
  int64_t best_pad = (O + 95) / 96 * 96;
  for (int bo : {64, 32}) {
    const int64_t pad = (O + bo - 1) / bo * bo;
    if (pad < best_pad) { best = bo; best_pad = pad; }
  }
  return best;
}
inline int tc_pick_bo(int T, int64_t O) {
  if (T == 1) return 256;
  if (T == 2) return 128;
  if (T == 3) return 128;
  if (T == 6) return 64;
  if (T == 8) return 32;
  int best = 128;
  int64_t best_pad = (O + 127) / 128 * 128;
  for (int bo : {96, 64, 32}) {
    const int64_t pad = (O + bo - 1) / bo * bo;
    if (pad < best_pad) { best = bo; best_pad = pad; }
  }
  return best;
}
// Tail split of a tc_apply launch.  With ctas persistent CTAs taking tiles
// round-robin, the last wave holds r = n_tiles mod ctas tiles and leaves the
// other SMs idle for a whole tile.  When 2r <= ctas, each of those r tiles is
// split in two along the reduction (stages [0, 3nk/8) and [3nk/8, nk)), so
// the last wave takes 5/8 of a tile.  The half whose MMAs finish first
// (usually the shorter) leaves its FP32 accumulator in the handle's
// workspace; the other adds it before the inverse DFT and stores the tile.
// Only reductions of at least kSplitMinStages stages are split: the
// hand-over of a 128 x 384-column accumulator costs a few microseconds.  The
// split shortens a lone call, but the hand-over is extra work: where other
// kernels (another stream's) would fill the idle SMs, it costs throughput.
// So it is off by default (eqlin_set_tail_split).
constexpr int kSplitMinStages = 16;
inline int tc_split_tiles(int64_t n_tiles, int ctas, int nk, int pairs) {
  if (nk < kSplitMinStages || ctas < 2 || n_tiles < 1) return 0;
  const int64_t r = n_tiles % ctas;
  return (r > 0 && 2 * r <= ctas && r <= pairs) ? (int)r : 0;
}
// Element index of (row, k, plane q) in a tiled weight buffer with tile width
// bo and n_kb K stages.
__host__ __device__ inline int64_t wtile_index(int T, int bo, int64_t n_kb, int64_t row, int64_t k, int q) {
  const int Q = tc_planes(T);
  const int64_t ot = row / bo, kb = k / TC_BK;
  const int r = (int)(row % bo), kk = (int)(k % TC_BK);
  const int64_t tile = (ot * n_kb + kb) * Q + q;
  const int64_t byte = tile * bo * 32 + r * 32 + ((((kk >> 3) ^ ((r >> 2) & 1))) << 4) + (kk & 7) * 2;
  return byte / 2;
}
// Elements of a tiled buffer for `rows` output rows and K = `kdim`.
__host__ __device__ inline int64_t wtile_elems(int T, int bo, int64_t rows, int64_t kdim) {
  return ((rows + bo - 1) / bo) * ((kdim + TC_BK - 1) / TC_BK) * tc_planes(T) * bo * TC_BK;
}

// FP32 handles (the 3xTF32 kernel, eqlin_tc32.cu): K stages of 8 input
// channels (one kind::tf32 MMA step, 32-byte rows of f32), and per stage 2Q
// planes: the Q planes above rounded to TF32 ("hi", planes 0 .. Q-1), then
// the TF32 rounding of what that rounding left over ("lo", planes Q .. 2Q-1).
// Same 32-byte-swizzled row image: 16-byte chunk j (4 floats) of row r at
// chunk j ^ ((r >> 2) & 1).  Tile widths: the widest MMAs that fit (an
// N = 128 TF32 MMA already reads its operands at the SM's shared-memory rate,
// so narrower tiles are bandwidth-bound): 256 (T = 1), 256 or 128 (T = 2),
// 128, 64 or 32 (T = 4), the one that pads O least, the wider on a tie; 32
// for T = 8 (its 16 hi/lo A planes fill most of shared memory).
constexpr int TC32_BK = 8;
inline int tc32_pick_bo(int T, int64_t O) {
  if (T == 1) return 256;
  if (T == 8) return 32;
  const int widths2[2] = {256, 128}, widths4[3] = {128, 64, 32};
  const int* w = T == 2 ? widths2 : widths4;
  const int n = T == 2 ? 2 : 3;
  int best = w[0];
  for (int i = 1; i < n; ++i)
    if ((O + w[i] - 1) / w[i] * w[i] < (O + best - 1) / best * best) best = w[i];
  return best;
}
__host__ __device__ inline int64_t wtile32_index(int T, int bo, int64_t n_kb, int64_t row, int64_t k, int plane) {
  const int64_t ot = row / bo, kb = k / TC32_BK;
  const int r = (int)(row % bo), kk = (int)(k % TC32_BK);
  const int64_t tile = (ot * n_kb + kb) * 2 * tc_planes(T) + plane;
  const int64_t byte = tile * bo * 32 + r * 32 + ((((kk >> 2) ^ ((r >> 2) & 1))) << 4) + (kk & 3) * 4;
  return byte / 4;
}
__host__ __device__ inline int64_t wtile32_elems(int T, int bo, int64_t rows, int64_t kdim) {
  return ((rows + bo - 1) / bo) * ((kdim + TC32_BK - 1) / TC32_BK) * 2 * tc_planes(T) * bo * TC32_BK;
}

// ------------------------------------------------------------ spectra
// The stash forms of the forward and the input gradient also write the group
// DFT of their input -- X = DFT(x) [T][C'][ld], G = DFT(gy) [T][D'][ld] --
// which the weight gradient then reads instead of x and gy.  Planes in the
// order above, unscaled, in the handle's dtype, tokens contiguous; the row
// pitch ld is N rounded up to a multiple of 64 tokens (128-byte rows).
inline int64_t spectra_ld(int64_t N) { return (N + 63) / 64 * 64; }

// ------------------------------------------------------------------ handle
struct Handle {
  int T = 0;                      // group order (cyclic: T; dihedral D_m: 2m)
  int group = EQLIN_GROUP_CYCLIC;
  int m = 0;                      // dihedral groups: D_m
  int64_t Cp = 0, Dp = 0;
  eqlin_dtype_t dtype = EQLIN_F32;
  int device = 0;
  int sm_count = 0;
  bool has_weights = false;
  // FP32 Fourier planes for the SIMT kernels: fwd [T][Cp][Dp] (row = input
  // channel, contiguous over output channel); bwd [T][Dp][Cp], conjugated.
  float* wf_fwd = nullptr;
  float* wf_bwd = nullptr;
  // Fourier planes in the handle dtype for the tensor-core kernels, tiled as
  // above: fwd rows D' x K C', bwd rows C' x K D' (conjugated); Q = real
  // freqs + 3 per complex freq (-Im, Re, Im stacked so that [Re;Im] and
  // [-Im;Re] are contiguous windows of a stage).  FP32 handles hold the
  // 3xTF32 hi/lo images here instead (wtile32_index).
  void* wt_fwd = nullptr;
  void* wt_bwd = nullptr;
  int bo_fwd = 0, bo_bwd = 0;     // tile widths (output channels) of the two layouts
  // p4 forward image for the three-product (Gauss) complex products, tile
  // width bo_gauss (its five accumulators fit TMEM up to 96 channels);
  // present for T = 4 handles whose passes both run on the tensor cores
  void* wt_gauss = nullptr;
  int bo_gauss = 0;
  bool need_simt_fwd = true;      // FP32 planes needed (SIMT serves forward / dx)
  bool need_simt_bwd = true;
  float* bias = nullptr;          // [Dp] float32 (zeros when no bias)
  float* ws = nullptr;            // dW split partials
  size_t ws_bytes = 0;
  // tc_apply tail split (tc_split_tiles), off unless eqlin_set_tail_split
  // turned it on; then, per pass (0 forward, 1 dx) of at least
  // kSplitMinStages stages: split_ws [pairs][cols / 4][128 rows][4] FP32
  // accumulators; split_flags [pairs] claims, [pairs] ready flags and a count
  // of finished CTAs, all zero between launches.
  float* split_ws[2] = {nullptr, nullptr};
  int* split_flags[2] = {nullptr, nullptr};
  int split_pairs[2] = {0, 0};
  int split_cols[2] = {0, 0};
  int* err = nullptr;             // device error record, 4 words (eqlin_wait.cuh)
  uint32_t last_error[4] = {0, 0, 0, 0};   // the record eqlin_get_error last read, when not OK
  uint32_t wait_limit = 0;        // 0 = default
  // kernel family of each pass, "fwd=<k> dx=<k> dw=<k>" (<k>: tcgen05 or simt)
  char backend[48] = "fwd=simt dx=simt dw=simt";
};

// Device error codes written into Handle::err (first writer wins).
enum : int { DEV_OK = 0, DEV_TIMEOUT = 1 };

// Default poll cap of a wait; the wall-time cap (2 s per wait) binds first.
constexpr uint32_t kDefaultWaitLimit = 0xFFFFFFFFu;

// Count kernels enqueued by this library (reported by eqlin_launch_count).
void count_launches(int n);

// Raise `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device.  The attribute belongs to the device's context, so it is set once
// per (kernel, device) pair in this process; safe to call from any host thread.
cudaError_t set_smem_limit(const void* kernel, int bytes);

// cuTensorMapEncodeTiled from the driver, looked up once (nullptr if absent).
void* tensor_map_encoder();

// ------------------------------------------- programmatic dependent launch
// Every kernel of this library is launched with programmatic stream
// serialization: its CTAs may start on SMs that the previous kernel in the
// stream has already left, and run their prologue (barrier set-up, tensor
// memory allocation) while that kernel finishes.  Each kernel therefore
// calls grid_dep_wait() -- which returns once the previous grid has
// completed and its memory is visible -- before its first global memory
// access, and grid_dep_launch(), which lets the next kernel be scheduled
// once every CTA of this one has issued it: at the start of short kernels,
// after the main loop where a waiting dependent would slow the loop.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// ------------------------------------------------------- launch wrappers
// SIMT path (any T in {1,2,4,8}, any dtype).
cudaError_t launch_pretransform(const Handle& h, const void* W, const void* b, cudaStream_t st);
cudaError_t launch_simt_apply(const Handle& h, bool backward, const void* in, void* out,
                              int64_t N, cudaStream_t st);
cudaError_t launch_simt_dw(const Handle& h, const void* x, const void* gy, float* dW, float* db,
                           int64_t N, cudaStream_t st);
size_t simt_dw_workspace_bytes(int T, int64_t Cp, int64_t Dp);
// Token splits of the SIMT weight gradients (32 x 32 channel tiles).
int simt_dw_splits(int64_t Cp, int64_t Dp, int64_t N);

// Dihedral groups D_m (eqlin_dihedral.cu), FP32 CUDA-core kernels, every dtype.
bool dihedral_supported(int m);
cudaError_t launch_dihedral_pretransform(const Handle& h, const void* W, const void* b, cudaStream_t st);
cudaError_t launch_dihedral_apply(const Handle& h, bool backward, const void* in, void* out, int64_t N,
                                  cudaStream_t st);
cudaError_t launch_dihedral_dw(const Handle& h, const void* x, const void* gy, float* dW, float* db, int64_t N,
                               cudaStream_t st);
// Sum per-split partial Fourier planes ([splits][T][Dp][Cp], or
// [splits][T][Cp][Dp] when cd_layout) and db partials [splits][Dp] in split
// order and apply the inverse DFT -> dW [Dp][Cp][T].
cudaError_t launch_dw_reduce(const Handle& h, int splits, const float* part, const float* dbpart,
                             float* dW, float* db, bool cd_layout, cudaStream_t st);

// tcgen05 path (f16/bf16).  Returns cudaErrorNotSupported when the shape is
// outside what the kernel handles, so the caller can fall back to SIMT.
bool tc_supported(const Handle& h, bool backward);
// Forward (backward = false) or input gradient; with `stash` non-null, also
// writes the input's spectrum there (see spectra_ld).
cudaError_t launch_tc_apply(const Handle& h, bool backward, const void* in, void* out, void* stash,
                            int64_t N, cudaStream_t st);
// The p4 forward with the complex products in three real GEMMs (Gauss), for
// comparison; needs the handle's Gauss image (h.wt_gauss).
cudaError_t launch_tc_apply_gauss(const Handle& h, const void* in, void* out, int64_t N, cudaStream_t st);
// FP32 handles on the tensor cores, 3xTF32 (eqlin_tc32.cu): T in {1, 2, 4, 8};
// forward and input gradient, and the pretransform into the hi/lo images.
// tc32_pass_ok: the pass's reduction is short enough for the FP32-level
// error bound (at most 256 MMAs into one accumulator: K <= 680 for T = 1,
// 2 and K <= 336 for T = 4, 8, whose complex accumulators take two block
// products per stage).
bool tc32_supported(const Handle& h);
bool tc32_pass_ok(const Handle& h, bool backward);
// dW, db (eqlin_tc32_dw.cu) for T in {1, 2, 4}, token chunks of at most 256
// MMAs per accumulator
bool tc32_dw_supported(const Handle& h);
size_t tc32_dw_workspace_bytes(int T, int64_t Cp, int64_t Dp, int sm_count);
cudaError_t launch_tc32_dw(const Handle& h, const void* x, const void* gy, float* dW, float* db, int64_t N,
                           cudaStream_t st);
cudaError_t launch_tc32_apply(const Handle& h, bool backward, const void* in, void* out, int64_t N,
                              cudaStream_t st);
cudaError_t launch_tc32_pretransform(const Handle& h, const float* W, const float* b, cudaStream_t st);
bool tc_dw_supported(const Handle& h);
// dW, db from the spectra written by the stash forms (eqlin_tc_dws.cu).
size_t tc_dws_workspace_bytes(int T, int64_t Cp, int64_t Dp, int sm_count);
cudaError_t launch_tc_dw_spectra(const Handle& h, const void* xs, const void* gs, float* dW, float* db, int64_t N,
                                 cudaStream_t st);
size_t tc_dw_workspace_bytes(int T, int64_t Cp, int64_t Dp, int sm_count);
cudaError_t launch_tc_dw(const Handle& h, const void* x, const void* gy, float* dW, float* db,
                         int64_t N, cudaStream_t st);

}  // namespace eqlin
