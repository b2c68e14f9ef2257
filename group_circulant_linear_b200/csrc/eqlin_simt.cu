// eqlin_simt.cu -- weight pre-transform and the SIMT (CUDA-core) kernels.
//
// These kernels serve every T in {1,2,4,8} and every dtype.  They are the
// FP32 path (FFMA, FP32 accumulation) and the reference structure the
// tensor-core kernels follow:
//
//   prologue  DFT of each input row along t, one T-vector per channel
//   mainloop  per-frequency channel products on the half spectrum: one real
//             product per real frequency, a complex product (4 real ones)
//             per complex frequency -- R(T) real GEMMs in all
//   epilogue  inverse DFT along the frequency axis, 1/T, bias, cast, store
//
// ("Flash EQ-Linear", technical summary, sections "Abordagem Algoritmica" and
// "Implementacao": fused data flow, no intermediate global writes.)
#include "eqlin_internal.cuh"

namespace eqlin {

// ========================================================== weight transform
// One 32 (c) x 32 (d) tile per block: the DFT of W[d, c, 0..T) along tau,
// written as
//   wf_fwd[p][c][d]  (FP32, forward planes; SIMT kernels only)
//   wf_bwd[p][d][c]  (FP32, conjugated: the dx product uses conj(W_hat))
//   wt_fwd (rows d, K c), wt_bwd (rows c, K d): handle dtype, tensor-core
//   operand tiles (see wtile_index) scaled by 1/T (real) or 2/T (complex);
//   q enumerates real frequencies, then (-Im, Re, Im) triples
// The FP32 planes are written with consecutive threads on consecutive
// addresses; the transposed ones go through a shared-memory tile.
namespace pt {
constexpr int TILE = 32, ROWS = 8;   // block = 32 x 8 threads
}

template <int T, typename E>
__global__ void __launch_bounds__(pt::TILE * pt::ROWS)
pretransform_kernel(const E* __restrict__ W, const E* __restrict__ b, float* __restrict__ wf_fwd,
                    float* __restrict__ wf_bwd, E* __restrict__ wt_fwd, E* __restrict__ wt_bwd,
                    float* __restrict__ bias, int Cp, int Dp, int bo_f, int bo_b) {
  using G = Group<T>;
  using namespace pt;
  grid_dep_launch();
  grid_dep_wait();
  constexpr int Q = G::nreal + 3 * G::ncomplex;
  __shared__ float sP[T][TILE][TILE + 1];        // planes of the tile, [p][d][c]
  const int c0 = blockIdx.x * TILE, d0 = blockIdx.y * TILE;
  const int tx = threadIdx.x, ty = threadIdx.y;
  if (blockIdx.x == 0 && ty == 0)
    for (int d = d0 + tx; d < d0 + TILE && d < Dp; d += TILE) bias[d] = b ? Elem<E>::to_f(b[d]) : 0.f;
  const int64_t plane = (int64_t)Cp * Dp;
  // pass 1: thread (tx = c, rows d): DFT, write the [d][c]-ordered planes
#pragma unroll
  for (int i = 0; i < TILE / ROWS; ++i) {
    const int dl = ty + i * ROWS, d = d0 + dl, c = c0 + tx;
    float v[T], P[T];
    const bool ok = d < Dp && c < Cp;
#pragma unroll
    for (int t = 0; t < T; ++t) v[t] = ok ? Elem<E>::to_f(W[((int64_t)d * Cp + c) * T + t]) : 0.f;
    G::dft(v, P);
#pragma unroll
    for (int q = 0; q < T; ++q) sP[q][dl][tx] = P[q];
    if (!ok) continue;
    if (wf_bwd) {
#pragma unroll
      for (int q = 0; q < T; ++q) {
        const bool imag = q >= G::nreal && ((q - G::nreal) & 1);
        wf_bwd[q * plane + (int64_t)d * Cp + c] = imag ? -P[q] : P[q];
      }
    }
    if (wt_fwd) {
      // forward tiles: rows d, K = c
      const float sr = 1.f / T, sc = 2.f / T;
      const int64_t nkb = (Cp + TC_BK - 1) / TC_BK;
#pragma unroll
      for (int f = 0; f < G::nreal; ++f) wt_fwd[wtile_index(T, bo_f, nkb, d, c, f)] = Elem<E>::from_f(P[f] * sr);
#pragma unroll
      for (int k = 1; k <= G::ncomplex; ++k) {
        const float re = P[G::nreal + 2 * (k - 1)] * sc, im = P[G::nreal + 2 * (k - 1) + 1] * sc;
        const int q = G::nreal + 3 * (k - 1);
        wt_fwd[wtile_index(T, bo_f, nkb, d, c, q + 0)] = Elem<E>::from_f(-im);
        wt_fwd[wtile_index(T, bo_f, nkb, d, c, q + 1)] = Elem<E>::from_f(re);
        wt_fwd[wtile_index(T, bo_f, nkb, d, c, q + 2)] = Elem<E>::from_f(im);
      }
    }
  }
  __syncthreads();
  // pass 2: thread (tx = d, rows c): the [c][d]-ordered planes
#pragma unroll
  for (int i = 0; i < TILE / ROWS; ++i) {
    const int cl = ty + i * ROWS, c = c0 + cl, d = d0 + tx;
    if (d >= Dp || c >= Cp) continue;
    float P[T];
#pragma unroll
    for (int q = 0; q < T; ++q) P[q] = sP[q][tx][cl];
    if (wf_fwd) {
#pragma unroll
      for (int q = 0; q < T; ++q) wf_fwd[q * plane + (int64_t)c * Dp + d] = P[q];
    }
    if (wt_bwd) {
      // input-gradient tiles: rows c, K = d; conj(W_hat): Im -> -Im
      const float sr = 1.f / T, sc = 2.f / T;
      const int64_t nkb = (Dp + TC_BK - 1) / TC_BK;
#pragma unroll
      for (int f = 0; f < G::nreal; ++f) wt_bwd[wtile_index(T, bo_b, nkb, c, d, f)] = Elem<E>::from_f(P[f] * sr);
#pragma unroll
      for (int k = 1; k <= G::ncomplex; ++k) {
        const float re = P[G::nreal + 2 * (k - 1)] * sc, im = P[G::nreal + 2 * (k - 1) + 1] * sc;
        const int q = G::nreal + 3 * (k - 1);
        wt_bwd[wtile_index(T, bo_b, nkb, c, d, q + 0)] = Elem<E>::from_f(im);
        wt_bwd[wtile_index(T, bo_b, nkb, c, d, q + 1)] = Elem<E>::from_f(re);
        wt_bwd[wtile_index(T, bo_b, nkb, c, d, q + 2)] = Elem<E>::from_f(-im);
      }
    }
  }
  (void)Q;
}

// Tensor-core weight images only, for handles that need no FP32 planes.
// One thread makes 8 K-consecutive entries of one row of one image; those sit
// in 16 contiguous bytes of a tile (see wtile_index), so every plane is one
// 16-byte store.  Threads [0, nA) build the forward image (rows d, K c), the
// rest the input-gradient image (rows c, K d), with consecutive threads on
// consecutive c so that the W reads stay coalesced.  The values are those of
// pretransform_kernel; K entries past the end are written as zeros.
template <typename E>
__device__ __forceinline__ uint16_t bits16(E v) {
  uint16_t u;
  __builtin_memcpy(&u, &v, 2);
  return u;
}

template <typename E>
__device__ __forceinline__ void store8(E* dst, const float (&v)[8]) {
  uint4 u;
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = (uint32_t)bits16(Elem<E>::from_f(v[2 * i])) | ((uint32_t)bits16(Elem<E>::from_f(v[2 * i + 1])) << 16);
  u.x = w[0]; u.y = w[1]; u.z = w[2]; u.w = w[3];
  *reinterpret_cast<uint4*>(dst) = u;
}

template <int T, typename E>
__global__ void __launch_bounds__(256)
pretransform_tc_kernel(const E* __restrict__ W, const E* __restrict__ b, E* __restrict__ wt_fwd,
                       E* __restrict__ wt_bwd, float* __restrict__ bias, int Cp, int Dp, int bo_f, int bo_b,
                       E* __restrict__ wt_gauss, int bo_g) {
  using G = Group<T>;
  static_assert(sizeof(E) == 2, "tensor-core images hold 16-bit elements");
  grid_dep_launch();
  grid_dep_wait();
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid < Dp) bias[tid] = b ? Elem<E>::to_f(b[tid]) : 0.f;
  const int64_t gA = (Cp + 7) / 8, gB = (Dp + 7) / 8;
  const int64_t nA = (int64_t)Dp * gA, nB = (int64_t)Cp * gB;
  bool fwd;
  int64_t row, k0;
  if (tid < nA) {
    fwd = true; row = tid / gA; k0 = (tid % gA) * 8;
  } else if (tid < nA + nB) {
    const int64_t j = tid - nA;
    fwd = false; k0 = (j / Cp) * 8; row = j % Cp;
  } else {
    return;
  }
  const int64_t K = fwd ? Cp : Dp;
  // W[d, c, 0..T): the forward image reads 8 consecutive c of one d (8T
  // contiguous elements), the input-gradient image the same c of 8
  // consecutive d (8 runs of T).  Whole groups with C' a multiple of 8 (as
  // every tensor-core handle has) load in 16-byte / T-element vectors: W is
  // 16-byte aligned and (d*C' + c) a multiple of 8 for the forward image.
  alignas(16) E w[8][T];
  if (k0 + 8 <= K && Cp % 8 == 0) {
    if (fwd) {
      const uint4* src = reinterpret_cast<const uint4*>(W + (row * Cp + k0) * T);
#pragma unroll
      for (int v = 0; v < T; ++v) reinterpret_cast<uint4*>(&w[0][0])[v] = __ldg(src + v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const E* src = W + ((k0 + i) * Cp + row) * T;
        if constexpr (T == 8) {
          *reinterpret_cast<uint4*>(w[i]) = __ldg(reinterpret_cast<const uint4*>(src));
        } else if constexpr (T == 4) {
          *reinterpret_cast<uint2*>(w[i]) = __ldg(reinterpret_cast<const uint2*>(src));
        } else if constexpr (T == 2) {
          *reinterpret_cast<uint32_t*>(w[i]) = __ldg(reinterpret_cast<const unsigned int*>(src));
        } else {
#pragma unroll
          for (int t = 0; t < T; ++t) w[i][t] = src[t];
        }
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t k = k0 + i;
      const int64_t base = fwd ? (row * Cp + k) * T : (k * Cp + row) * T;
#pragma unroll
      for (int t = 0; t < T; ++t) w[i][t] = k < K ? W[base + t] : Elem<E>::from_f(0.f);
    }
  }
  float P[8][T];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float v[T];
#pragma unroll
    for (int t = 0; t < T; ++t) v[t] = Elem<E>::to_f(w[i][t]);
    G::dft(v, P[i]);
  }
  E* out = fwd ? wt_fwd : wt_bwd;
  const int bo = fwd ? bo_f : bo_b;
  const int64_t nkb = (K + TC_BK - 1) / TC_BK;
  const float sr = 1.f / T, sc = 2.f / T;
  float o[8];
#pragma unroll
  for (int f = 0; f < G::nreal; ++f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = k0 + i < K ? P[i][f] * sr : 0.f;
    store8(out + wtile_index(T, bo, nkb, row, k0, f), o);
  }
#pragma unroll
  for (int k = 1; k <= G::ncomplex; ++k) {
    const int pr = G::nreal + 2 * (k - 1), q = G::nreal + 3 * (k - 1);
    // forward: (-Im, Re, Im); input gradient, conj(W_hat): (Im, Re, -Im)
    const float s0 = fwd ? -1.f : 1.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = k0 + i < K ? s0 * (P[i][pr + 1] * sc) : 0.f;
    store8(out + wtile_index(T, bo, nkb, row, k0, q + 0), o);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = k0 + i < K ? P[i][pr] * sc : 0.f;
    store8(out + wtile_index(T, bo, nkb, row, k0, q + 1), o);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = k0 + i < K ? -s0 * (P[i][pr + 1] * sc) : 0.f;
    store8(out + wtile_index(T, bo, nkb, row, k0, q + 2), o);
  }
  // The forward image for the three-product (Gauss) form of the complex
  // products: real planes as above; per complex frequency (Re W, Im W - Re W,
  // Re W + Im W), each formed in FP32 and rounded once.
  if (fwd && wt_gauss) {
#pragma unroll
    for (int f = 0; f < G::nreal; ++f) {
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = k0 + i < K ? P[i][f] * sr : 0.f;
      store8(wt_gauss + wtile_index(T, bo_g, nkb, row, k0, f), o);
    }
#pragma unroll
    for (int k = 1; k <= G::ncomplex; ++k) {
      const int pr = G::nreal + 2 * (k - 1), q = G::nreal + 3 * (k - 1);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = k0 + i < K ? P[i][pr] * sc : 0.f;
      store8(wt_gauss + wtile_index(T, bo_g, nkb, row, k0, q + 0), o);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = k0 + i < K ? (P[i][pr + 1] - P[i][pr]) * sc : 0.f;
      store8(wt_gauss + wtile_index(T, bo_g, nkb, row, k0, q + 1), o);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = k0 + i < K ? (P[i][pr] + P[i][pr + 1]) * sc : 0.f;
      store8(wt_gauss + wtile_index(T, bo_g, nkb, row, k0, q + 2), o);
    }
  }
}

template <int T, typename E>
static cudaError_t pretransform_t(const Handle& h, const void* W, const void* b, cudaStream_t st) {
  if constexpr (sizeof(E) == 2) {
    if (!h.need_simt_fwd && !h.need_simt_bwd && h.wt_fwd && h.wt_bwd) {
      const int64_t n = h.Dp * ((h.Cp + 7) / 8) + h.Cp * ((h.Dp + 7) / 8);
      const int64_t threads = n > h.Dp ? n : h.Dp;
      const cudaError_t e = launch_pdl(pretransform_tc_kernel<T, E>, dim3((unsigned)((threads + 255) / 256)),
                                       dim3(256), 0, st, (const E*)W, (const E*)b, (E*)h.wt_fwd, (E*)h.wt_bwd,
                                       h.bias, (int)h.Cp, (int)h.Dp, h.bo_fwd, h.bo_bwd, (E*)h.wt_gauss,
                                       h.bo_gauss);
      count_launches(1);
      return e;
    }
  }
  dim3 grid((unsigned)((h.Cp + pt::TILE - 1) / pt::TILE), (unsigned)((h.Dp + pt::TILE - 1) / pt::TILE));
  dim3 block(pt::TILE, pt::ROWS);
  const cudaError_t e = launch_pdl(
      pretransform_kernel<T, E>, grid, block, 0, st, (const E*)W, (const E*)b,
      h.need_simt_fwd ? h.wf_fwd : nullptr, h.need_simt_bwd ? h.wf_bwd : nullptr,
      sizeof(E) == 2 ? (E*)h.wt_fwd : nullptr, sizeof(E) == 2 ? (E*)h.wt_bwd : nullptr,   // f32: 3xTF32 images
      h.bias, (int)h.Cp, (int)h.Dp, h.bo_fwd, h.bo_bwd);
  count_launches(1);
  return e;
}

template <typename E>
static cudaError_t pretransform_e(const Handle& h, const void* W, const void* b, cudaStream_t st) {
  switch (h.T) {
    case 1: return pretransform_t<1, E>(h, W, b, st);
    case 2: return pretransform_t<2, E>(h, W, b, st);
    case 3: return pretransform_t<3, E>(h, W, b, st);
    case 6: return pretransform_t<6, E>(h, W, b, st);
    case 4: return pretransform_t<4, E>(h, W, b, st);
    case 8: return pretransform_t<8, E>(h, W, b, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_pretransform(const Handle& h, const void* W, const void* b, cudaStream_t st) {
  switch (h.dtype) {
    case EQLIN_F32:
      // the 3xTF32 tensor-core images (and the bias); the FP32 planes as well
      // when a pass runs on the SIMT kernels
      if (h.wt_fwd && h.wt_bwd) {
        const cudaError_t e = launch_tc32_pretransform(h, (const float*)W, (const float*)b, st);
        if (e != cudaSuccess || (!h.need_simt_fwd && !h.need_simt_bwd)) return e;
      }
      return pretransform_e<float>(h, W, b, st);
    case EQLIN_F16: return pretransform_e<__half>(h, W, b, st);
    case EQLIN_BF16: return pretransform_e<__nv_bfloat16>(h, W, b, st);
  }
  return cudaErrorInvalidValue;
}

// ============================================================ apply (fwd/dx)
// out[n, o*T+s] = bias[o] + IDFT_s( sum_i planes[.][i][o] (*) DFT(in[n, i*T+.]) )
// planes [T][K][O] FP32.  Forward: in = x, K = C', O = D', forward planes.
// dx: in = gy, K = D', O = C', conjugated planes, no bias.
namespace simt {
constexpr int BM = 64, BO = 32, BK = 8, THREADS = 256;
}

template <int T, typename E>
__global__ void __launch_bounds__(simt::THREADS)
simt_apply_kernel(const E* __restrict__ in, const float* __restrict__ planes,
                  const float* __restrict__ bias, E* __restrict__ out, int64_t N, int K, int O) {
  using G = Group<T>;
  using namespace simt;
  grid_dep_launch();
  grid_dep_wait();
  __shared__ float Xs[T][BK][BM];
  __shared__ __align__(16) float Ws[T][BK][BO];

  const int tid = threadIdx.x;
  const int to = tid % 8, tn = tid / 8;              // 4 outputs x 2 tokens per thread
  const int64_t n0 = (int64_t)blockIdx.x * BM;
  const int o0 = blockIdx.y * BO;
  const int64_t plane = (int64_t)K * O;

  float acc[2][4][T];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int p = 0; p < T; ++p) acc[i][j][p] = 0.f;

  for (int k0 = 0; k0 < K; k0 += BK) {
    // prologue: DFT of BM x BK input T-vectors into the planes Xs
#pragma unroll
    for (int r = 0; r < (BM * BK) / THREADS; ++r) {
      const int q = tid + r * THREADS;
      const int kk = q % BK, nn = q / BK;
      const int64_t n = n0 + nn;
      const int k = k0 + kk;
      float v[T], P[T];
      if (n < N && k < K) {
        const E* src = in + n * (int64_t)K * T + (int64_t)k * T;
#pragma unroll
        for (int t = 0; t < T; ++t) v[t] = Elem<E>::to_f(src[t]);
      } else {
#pragma unroll
        for (int t = 0; t < T; ++t) v[t] = 0.f;
      }
      G::dft(v, P);
#pragma unroll
      for (int p = 0; p < T; ++p) Xs[p][kk][nn] = P[p];
    }
    // Fourier weight planes
    for (int q = tid; q < T * BK * BO; q += THREADS) {
      const int oo = q % BO, kk = (q / BO) % BK, p = q / (BO * BK);
      const int o = o0 + oo, k = k0 + kk;
      Ws[p][kk][oo] = (o < O && k < K) ? planes[p * plane + (int64_t)k * O + o] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float xv[2][T], wv[4][T];
#pragma unroll
      for (int p = 0; p < T; ++p) {
#pragma unroll
        for (int i = 0; i < 2; ++i) xv[i][p] = Xs[p][kk][tn + 32 * i];
        const float4 w4 = *reinterpret_cast<const float4*>(&Ws[p][kk][to * 4]);
        wv[0][p] = w4.x; wv[1][p] = w4.y; wv[2][p] = w4.z; wv[3][p] = w4.w;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int f = 0; f < G::nreal; ++f) acc[i][j][f] = fmaf(xv[i][f], wv[j][f], acc[i][j][f]);
#pragma unroll
          for (int m = 0; m < G::ncomplex; ++m) {
            const int pr = G::nreal + 2 * m, pi = pr + 1;
            acc[i][j][pr] = fmaf(xv[i][pr], wv[j][pr], acc[i][j][pr]);
            acc[i][j][pr] = fmaf(-xv[i][pi], wv[j][pi], acc[i][j][pr]);
            acc[i][j][pi] = fmaf(xv[i][pr], wv[j][pi], acc[i][j][pi]);
            acc[i][j][pi] = fmaf(xv[i][pi], wv[j][pr], acc[i][j][pi]);
          }
        }
    }
    __syncthreads();
  }
  // epilogue: inverse DFT, bias, store T contiguous outputs per (n, o)
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int64_t n = n0 + tn + 32 * i;
    if (n >= N) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = o0 + to * 4 + j;
      if (o >= O) continue;
      float v[T];
      G::idft(acc[i][j], v);
      const float bo = bias ? bias[o] : 0.f;
      E* dst = out + n * (int64_t)O * T + (int64_t)o * T;
#pragma unroll
      for (int s = 0; s < T; ++s) dst[s] = Elem<E>::from_f(v[s] + bo);
    }
  }
}

template <int T, typename E>
static cudaError_t simt_apply_t(const Handle& h, bool backward, const void* in, void* out,
                                int64_t N, cudaStream_t st) {
  const int K = (int)(backward ? h.Dp : h.Cp);
  const int O = (int)(backward ? h.Cp : h.Dp);
  const int64_t tiles_n = (N + simt::BM - 1) / simt::BM;
  if (tiles_n > 0x7fffffff) return cudaErrorInvalidValue;
  dim3 grid((unsigned)tiles_n, (unsigned)((O + simt::BO - 1) / simt::BO));
  const cudaError_t e = launch_pdl(simt_apply_kernel<T, E>, grid, dim3(simt::THREADS), 0, st, (const E*)in,
                                   (const float*)(backward ? h.wf_bwd : h.wf_fwd),
                                   (const float*)(backward ? nullptr : h.bias), (E*)out, N, K, O);
  count_launches(1);
  return e;
}

template <typename E>
static cudaError_t simt_apply_e(const Handle& h, bool bwd, const void* in, void* out, int64_t N,
                                cudaStream_t st) {
  switch (h.T) {
    case 1: return simt_apply_t<1, E>(h, bwd, in, out, N, st);
    case 2: return simt_apply_t<2, E>(h, bwd, in, out, N, st);
    case 3: return simt_apply_t<3, E>(h, bwd, in, out, N, st);
    case 6: return simt_apply_t<6, E>(h, bwd, in, out, N, st);
    case 4: return simt_apply_t<4, E>(h, bwd, in, out, N, st);
    case 8: return simt_apply_t<8, E>(h, bwd, in, out, N, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_simt_apply(const Handle& h, bool backward, const void* in, void* out,
                              int64_t N, cudaStream_t st) {
  switch (h.dtype) {
    case EQLIN_F32: return simt_apply_e<float>(h, backward, in, out, N, st);
    case EQLIN_F16: return simt_apply_e<__half>(h, backward, in, out, N, st);
    case EQLIN_BF16: return simt_apply_e<__nv_bfloat16>(h, backward, in, out, N, st);
  }
  return cudaErrorInvalidValue;
}

// ================================================================= dW and db
// Fourier form of the weight gradient (derived from the definition; the
// pages give no formula): dW_hat_k[d, c] = sum_n G_k[n, d] conj(X_k[n, c]),
// G = DFT(gy), X = DFT(x); dW = IDFT_tau(dW_hat) with the 1/T.  db[d] =
// sum_n G_0[n, d].  Stage 1 writes per-split partial planes; stage 2 sums the
// splits in a fixed order and applies the inverse DFT (deterministic).
namespace simtdw {
constexpr int BD = 32, BC = 32, BK = 16, THREADS = 256, MAX_SPLITS = 64, TARGET_CTAS = 4 * 148;
}

static int dw_splits(int64_t Cp, int64_t Dp, int64_t N) {
  using namespace simtdw;
  const int64_t tiles = ((Cp + BC - 1) / BC) * ((Dp + BD - 1) / BD);
  int64_t s = (TARGET_CTAS + tiles - 1) / tiles;
  const int64_t max_by_n = (N + BK - 1) / BK;
  if (s > MAX_SPLITS) s = MAX_SPLITS;
  if (s > max_by_n) s = max_by_n;
  return s < 1 ? 1 : (int)s;
}

int simt_dw_splits(int64_t Cp, int64_t Dp, int64_t N) { return dw_splits(Cp, Dp, N); }

size_t simt_dw_workspace_bytes(int T, int64_t Cp, int64_t Dp) {
  const int64_t s = dw_splits(Cp, Dp, INT64_MAX / 2);
  return (size_t)s * ((size_t)T * Cp * Dp + Dp) * sizeof(float);
}

template <int T, typename E>
__global__ void __launch_bounds__(simtdw::THREADS)
simt_dw_kernel(const E* __restrict__ x, const E* __restrict__ gy, float* __restrict__ part,
               float* __restrict__ dbpart, int64_t N, int Cp, int Dp, int64_t tok_per_split) {
  using G = Group<T>;
  using namespace simtdw;
  grid_dep_launch();
  grid_dep_wait();
  __shared__ float Gs[T][BK][BD];
  __shared__ __align__(16) float Xs[T][BK][BC];
  const int tid = threadIdx.x;
  const int tc = tid % 8, td = tid / 8;             // 4 c x 1 d per thread
  const int c0 = blockIdx.x * BC, d0 = blockIdx.y * BD;
  const int z = blockIdx.z;
  const int64_t nbeg = (int64_t)z * tok_per_split;
  int64_t nend = nbeg + tok_per_split;
  if (nend > N) nend = N;

  float acc[4][T];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int p = 0; p < T; ++p) acc[j][p] = 0.f;
  float dbacc = 0.f;

  for (int64_t nb = nbeg; nb < nend; nb += BK) {
#pragma unroll
    for (int r = 0; r < (BK * BD) / THREADS; ++r) {
      const int q = tid + r * THREADS;
      const int dd = q % BD, nn = q / BD;
      const int64_t n = nb + nn;
      const int d = d0 + dd;
      float v[T], P[T];
      if (n < nend && d < Dp) {
        const E* src = gy + n * (int64_t)Dp * T + (int64_t)d * T;
#pragma unroll
        for (int t = 0; t < T; ++t) v[t] = Elem<E>::to_f(src[t]);
      } else {
#pragma unroll
        for (int t = 0; t < T; ++t) v[t] = 0.f;
      }
      G::dft(v, P);
#pragma unroll
      for (int p = 0; p < T; ++p) Gs[p][nn][dd] = P[p];
    }
#pragma unroll
    for (int r = 0; r < (BK * BC) / THREADS; ++r) {
      const int q = tid + r * THREADS;
      const int cc = q % BC, nn = q / BC;
      const int64_t n = nb + nn;
      const int c = c0 + cc;
      float v[T], P[T];
      if (n < nend && c < Cp) {
        const E* src = x + n * (int64_t)Cp * T + (int64_t)c * T;
#pragma unroll
        for (int t = 0; t < T; ++t) v[t] = Elem<E>::to_f(src[t]);
      } else {
#pragma unroll
        for (int t = 0; t < T; ++t) v[t] = 0.f;
      }
      G::dft(v, P);
#pragma unroll
      for (int p = 0; p < T; ++p) Xs[p][nn][cc] = P[p];
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float gv[T], xv[4][T];
#pragma unroll
      for (int p = 0; p < T; ++p) {
        gv[p] = Gs[p][kk][td];
        const float4 x4 = *reinterpret_cast<const float4*>(&Xs[p][kk][tc * 4]);
        xv[0][p] = x4.x; xv[1][p] = x4.y; xv[2][p] = x4.z; xv[3][p] = x4.w;
      }
      dbacc += gv[0];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int f = 0; f < G::nreal; ++f) acc[j][f] = fmaf(gv[f], xv[j][f], acc[j][f]);
#pragma unroll
        for (int m = 0; m < G::ncomplex; ++m) {
          const int pr = G::nreal + 2 * m, pi = pr + 1;
          // G * conj(X)
          acc[j][pr] = fmaf(gv[pr], xv[j][pr], acc[j][pr]);
          acc[j][pr] = fmaf(gv[pi], xv[j][pi], acc[j][pr]);
          acc[j][pi] = fmaf(gv[pi], xv[j][pr], acc[j][pi]);
          acc[j][pi] = fmaf(-gv[pr], xv[j][pi], acc[j][pi]);
        }
      }
    }
    __syncthreads();
  }
  const int d = d0 + td;
  if (d >= Dp) return;
  const int64_t plane = (int64_t)Cp * Dp;
  float* base = part + (int64_t)z * T * plane;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = c0 + tc * 4 + j;
    if (c >= Cp) continue;
#pragma unroll
    for (int p = 0; p < T; ++p) base[p * plane + (int64_t)d * Cp + c] = acc[j][p];
  }
  if (blockIdx.x == 0 && tc == 0) dbpart[(int64_t)z * Dp + d] = dbacc;
}

// Sum the splits in index order, then inverse DFT along the frequency planes.
// Partials are [splits][T][Dp][Cp] (cd_layout false) or [splits][T][Cp][Dp]
// (cd_layout true).  One block of 256 threads per tile of 32 (d) x 8 (c)
// (cd_layout) or 8 (d) x 32 (c) channels, one element per thread, with the
// warp's 32 lanes along the partials' contiguous index.  A thread sums the
// splits in index order, eight at a time with all of a group's T x 8 loads
// issued before any is added (the reduction is latency bound), in a fixed
// order; takes the inverse DFT; and stages the tile in shared memory so that
// dW [Dp][Cp][T] is written row by row.
template <int T, bool CD>
__global__ void __launch_bounds__(256)
dw_reduce_kernel(const float* __restrict__ part, const float* __restrict__ dbpart, float* __restrict__ dW,
                 float* __restrict__ db, int splits, int Cp, int Dp) {
  using G = Group<T>;
  grid_dep_launch();
  grid_dep_wait();
  constexpr int DT = CD ? 32 : 8, CT = CD ? 8 : 32;  // tile: d x c
  constexpr int ZG = 8;                               // splits per load group
  __shared__ float sV[DT][CT * T + 1];                // [d][c*T + t] of the tile
  const int c0 = blockIdx.x * CT, d0 = blockIdx.y * DT;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
  const int64_t plane = (int64_t)Cp * Dp;
  const int d = CD ? d0 + tx : d0 + ty;
  const int c = CD ? c0 + ty : c0 + tx;
  float P[T], v[T];
#pragma unroll
  for (int q = 0; q < T; ++q) P[q] = 0.f;
  if (d < Dp && c < Cp) {
    const float* src = part + (CD ? (int64_t)c * Dp + d : (int64_t)d * Cp + c);
    const int64_t zs = (int64_t)T * plane;
    for (int z0 = 0; z0 < splits; z0 += ZG) {
      float val[ZG][T];
#pragma unroll
      for (int i = 0; i < ZG; ++i)
#pragma unroll
        for (int q = 0; q < T; ++q)
          val[i][q] = (z0 + i < splits) ? __ldg(src + (int64_t)(z0 + i) * zs + (int64_t)q * plane) : 0.f;
#pragma unroll
      for (int q = 0; q < T; ++q) {
        const float g = ((val[0][q] + val[1][q]) + (val[2][q] + val[3][q])) +
                        ((val[4][q] + val[5][q]) + (val[6][q] + val[7][q]));
        P[q] += g;
      }
    }
  }
  G::idft(P, v);
  const int dl = d - d0, cl = c - c0;
#pragma unroll
  for (int t = 0; t < T; ++t) sV[dl][cl * T + t] = v[t];
  __syncthreads();
  // rows of CT*T contiguous floats, one warp per row at a time
  const int ncol = min(CT, Cp - c0) * T;
  for (int r = ty; r < DT; r += 8) {
    const int dd = d0 + r;
    if (dd >= Dp) continue;
    float* dst = dW + ((int64_t)dd * Cp + c0) * T;
    for (int j = tx; j < ncol; j += 32) dst[j] = sV[r][j];
  }
  if (db && blockIdx.x == 0 && threadIdx.x < DT) {
    const int dd = d0 + threadIdx.x;
    if (dd < Dp) {
      float s = 0.f;
      for (int z = 0; z < splits; ++z) s += dbpart[(int64_t)z * Dp + dd];
      db[dd] = s;
    }
  }
}

template <int T>
static cudaError_t dw_reduce_t(const Handle& h, int splits, const float* part, const float* dbpart,
                               float* dW, float* db, bool cd_layout, cudaStream_t st) {
  cudaError_t e;
  if (cd_layout) {
    dim3 grid((unsigned)((h.Cp + 7) / 8), (unsigned)((h.Dp + 31) / 32));
    e = launch_pdl(dw_reduce_kernel<T, true>, grid, dim3(256), 0, st, part, dbpart, dW, db, splits, (int)h.Cp,
                   (int)h.Dp);
  } else {
    dim3 grid((unsigned)((h.Cp + 31) / 32), (unsigned)((h.Dp + 7) / 8));
    e = launch_pdl(dw_reduce_kernel<T, false>, grid, dim3(256), 0, st, part, dbpart, dW, db, splits, (int)h.Cp,
                   (int)h.Dp);
  }
  count_launches(1);
  return e;
}

cudaError_t launch_dw_reduce(const Handle& h, int splits, const float* part, const float* dbpart,
                             float* dW, float* db, bool cd_layout, cudaStream_t st) {
  switch (h.T) {
    case 1: return dw_reduce_t<1>(h, splits, part, dbpart, dW, db, cd_layout, st);
    case 2: return dw_reduce_t<2>(h, splits, part, dbpart, dW, db, cd_layout, st);
    case 3: return dw_reduce_t<3>(h, splits, part, dbpart, dW, db, cd_layout, st);
    case 6: return dw_reduce_t<6>(h, splits, part, dbpart, dW, db, cd_layout, st);
    case 4: return dw_reduce_t<4>(h, splits, part, dbpart, dW, db, cd_layout, st);
    case 8: return dw_reduce_t<8>(h, splits, part, dbpart, dW, db, cd_layout, st);
  }
  return cudaErrorInvalidValue;
}

template <int T, typename E>
static cudaError_t simt_dw_t(const Handle& h, const void* x, const void* gy, float* dW, float* db,
                             int64_t N, cudaStream_t st) {
  using namespace simtdw;
  const int splits = dw_splits(h.Cp, h.Dp, N);
  const int64_t tps = ((N + splits - 1) / splits + BK - 1) / BK * BK;
  const int64_t plane = h.Cp * h.Dp;
  float* part = h.ws;
  float* dbpart = h.ws + (int64_t)splits * T * plane;
  if ((size_t)splits * ((size_t)T * plane + h.Dp) * sizeof(float) > h.ws_bytes)
    return cudaErrorInvalidValue;
  dim3 grid((unsigned)((h.Cp + BC - 1) / BC), (unsigned)((h.Dp + BD - 1) / BD), (unsigned)splits);
  cudaError_t e = launch_pdl(simt_dw_kernel<T, E>, grid, dim3(THREADS), 0, st, (const E*)x, (const E*)gy, part,
                             dbpart, N, (int)h.Cp, (int)h.Dp, tps);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return launch_dw_reduce(h, splits, part, dbpart, dW, db, /*cd_layout=*/false, st);
}

template <typename E>
static cudaError_t simt_dw_e(const Handle& h, const void* x, const void* gy, float* dW, float* db,
                             int64_t N, cudaStream_t st) {
  switch (h.T) {
    case 1: return simt_dw_t<1, E>(h, x, gy, dW, db, N, st);
    case 2: return simt_dw_t<2, E>(h, x, gy, dW, db, N, st);
    case 3: return simt_dw_t<3, E>(h, x, gy, dW, db, N, st);
    case 6: return simt_dw_t<6, E>(h, x, gy, dW, db, N, st);
    case 4: return simt_dw_t<4, E>(h, x, gy, dW, db, N, st);
    case 8: return simt_dw_t<8, E>(h, x, gy, dW, db, N, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_simt_dw(const Handle& h, const void* x, const void* gy, float* dW, float* db,
                           int64_t N, cudaStream_t st) {
  switch (h.dtype) {
    case EQLIN_F32: return simt_dw_e<float>(h, x, gy, dW, db, N, st);
    case EQLIN_F16: return simt_dw_e<__half>(h, x, gy, dW, db, N, st);
    case EQLIN_BF16: return simt_dw_e<__nv_bfloat16>(h, x, gy, dW, db, N, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace eqlin
