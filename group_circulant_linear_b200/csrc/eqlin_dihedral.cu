// eqlin_dihedral.cu -- the layer over the dihedral groups D_m (reflections and
// rotations of a regular m-gon), FP32 CUDA-core kernels.
//
// The paper names reflection groups as future work ("Flash EQ-Linear",
// technical summary, section "Limitacoes e Trabalho Futuro") without a
// formula.  The layer taken is the group convolution
//
//   y[n, d*|G|+g] = b[d] + sum_c sum_h W[d, c, h^-1 g] x[n, c*|G|+h]
//
// over D_m (|G| = 2m, element r^a s^f at index f*m + a), which on the cyclic
// group is the paper's (s - t) mod T.  It is evaluated the way the paper
// evaluates the cyclic case, with the DFT replaced by the Fourier transform
// over D_m's real irreducible representations rho (the trivial one, the
// reflection sign (-1)^f, for even m also (-1)^a and (-1)^(a+f), and the
// planar rho_k(r^a s^f) = rotation by 2 pi k a / m then diag(1, -1)^f,
// k = 1 .. ceil(m/2)-1):
//
//   x^(rho) = sum_g x(g) rho(g)                 (d_rho x d_rho per channel)
//   y^(rho) = sum_c x^(rho)[c] W^(rho)[d, c]     (matrix products per irrep)
//   y(g)    = (1/|G|) sum_rho d_rho tr(rho(g)^T y^(rho))
//
// so each 1-dimensional irrep is one real channel GEMM and each planar one
// eight (a 2 x 2 matrix product): 12 for D_4 against the 64 of the unrolled
// dense layer.  The gradients (derived from the definition):
//   dx^(rho) = sum_d G^(rho)[d] W^(rho)[d, c]^T,   G = transform of gy
//   dW^(rho) = sum_n x^(rho)^T G^(rho),            db = sum_n G^(trivial)
//
// A channel's transform is held as |G| real planes: first the 1-dimensional
// irreps, then for each planar irrep its entries (0,0), (0,1), (1,0), (1,1).
// The forward and the input gradient share one kernel: the input gradient's
// weight planes hold each planar block transposed.
#include "eqlin_internal.cuh"

namespace eqlin {
namespace dih {

template <int M>
struct Dih {
  static constexpr int n = 2 * M;                      // group order
  static constexpr int n1 = (M % 2 == 0) ? 4 : 2;      // 1-dimensional irreps
  static constexpr int K2 = (M + 1) / 2 - 1;           // planar irreps
  static_assert(n1 + 4 * K2 == n, "sum of d^2 is the group order");
};

// F[r][g] = rho(g)_ij of plane r = (rho, i, j); Fi[g][r] = (d_rho / |G|) rho(g)_ij.
template <int M>
__device__ void make_tables(float (*F)[2 * M], float (*Fi)[2 * M]) {
  using D = Dih<M>;
  for (int g = threadIdx.x; g < D::n; g += blockDim.x) {
    const int f = g / M, a = g % M;
    float col[D::n];
    col[0] = 1.f;
    col[1] = f ? -1.f : 1.f;
    if constexpr (D::n1 == 4) {
      col[2] = (a & 1) ? -1.f : 1.f;
      col[3] = ((a + f) & 1) ? -1.f : 1.f;
    }
#pragma unroll
    for (int k = 1; k <= D::K2; ++k) {
      float s, c;
      sincospif(2.f * (float)(k * a % M) / (float)M, &s, &c);
      const int b = D::n1 + 4 * (k - 1);
      col[b + 0] = c;
      col[b + 1] = f ? s : -s;
      col[b + 2] = s;
      col[b + 3] = f ? -c : c;
    }
#pragma unroll
    for (int r = 0; r < D::n; ++r) {
      F[r][g] = col[r];
      Fi[g][r] = (r < D::n1 ? 1.f : 2.f) / (float)D::n * col[r];
    }
  }
}

// acc += the irrep-blockwise product of x and w (planes r), x on the left:
// 1-dim planes x_r w_r; planar blocks (x w)_ij = sum_k x_ik w_kj.
template <int M>
__device__ __forceinline__ void block_mac(float* acc, const float* x, const float* w) {
  using D = Dih<M>;
#pragma unroll
  for (int r = 0; r < D::n1; ++r) acc[r] = fmaf(x[r], w[r], acc[r]);
#pragma unroll
  for (int k = 0; k < D::K2; ++k) {
    const int b = D::n1 + 4 * k;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float s = acc[b + 2 * i + j];
        s = fmaf(x[b + 2 * i + 0], w[b + 0 * 2 + j], s);
        s = fmaf(x[b + 2 * i + 1], w[b + 1 * 2 + j], s);
        acc[b + 2 * i + j] = s;
      }
  }
}

// ---------------------------------------------------------- weight transform
// wf[r][c][d] = W^(rho)_r[d, c] (forward); wb[r][d][c] = the same with each
// planar block transposed (input gradient).  One thread per (d, c).
template <int M, typename E>
__global__ void __launch_bounds__(256)
dih_pretransform_kernel(const E* __restrict__ W, const E* __restrict__ b, float* __restrict__ wf,
                        float* __restrict__ wb, float* __restrict__ bias, int Cp, int Dp) {
  using D = Dih<M>;
  __shared__ float F[D::n][D::n], Fi[D::n][D::n];
  grid_dep_launch();
  make_tables<M>(F, Fi);
  __syncthreads();
  grid_dep_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < Dp) bias[i] = b ? Elem<E>::to_f(b[i]) : 0.f;
  if (i >= (int64_t)Cp * Dp) return;
  const int d = (int)(i / Cp), c = (int)(i % Cp);
  float v[D::n];
#pragma unroll
  for (int g = 0; g < D::n; ++g) v[g] = Elem<E>::to_f(W[i * D::n + g]);
  const int64_t plane = (int64_t)Cp * Dp;
#pragma unroll
  for (int r = 0; r < D::n; ++r) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < D::n; ++g) s = fmaf(F[r][g], v[g], s);
    wf[r * plane + (int64_t)c * Dp + d] = s;
    // transposed planar block: plane (i, j) of wb holds entry (j, i)
    int rt = r;
    if (r >= D::n1) {
      const int q = (r - D::n1) & 3;
      rt = r - q + ((q & 1) << 1) + (q >> 1);
    }
    wb[rt * plane + (int64_t)d * Cp + c] = s;
  }
}

// ------------------------------------------------------------ forward / dx
// out[n, o*|G|+g] = bias[o] + inverse transform of sum_k in^(rho)[n, k] planes[r][k][o].
namespace ap {
constexpr int BM = 64, BO = 16, BK = 8, THREADS = 256;   // thread: 1 token x 4 outputs
}

template <int M, typename E>
__global__ void __launch_bounds__(ap::THREADS)
dih_apply_kernel(const E* __restrict__ in, const float* __restrict__ planes, const float* __restrict__ bias,
                 E* __restrict__ out, int64_t N, int K, int O) {
  using D = Dih<M>;
  using namespace ap;
  __shared__ float F[D::n][D::n], Fi[D::n][D::n];
  __shared__ float Xs[D::n][BK][BM];
  __shared__ float Ws[D::n][BK][BO];
  grid_dep_launch();
  make_tables<M>(F, Fi);
  grid_dep_wait();
  const int tid = threadIdx.x;
  const int tm = tid % BM, to = (tid / BM) * 4;
  const int64_t n0 = (int64_t)blockIdx.x * BM;
  const int o0 = blockIdx.y * BO;
  const int64_t plane = (int64_t)K * O;
  float acc[4][D::n];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int r = 0; r < D::n; ++r) acc[j][r] = 0.f;
  __syncthreads();
  for (int k0 = 0; k0 < K; k0 += BK) {
    // prologue: transform BM x BK input vectors
    for (int q = tid; q < BM * BK; q += THREADS) {
      const int kk = q % BK, mm = q / BK;
      const int64_t nn = n0 + mm;
      const int k = k0 + kk;
      float v[D::n];
      const bool ok = nn < N && k < K;
#pragma unroll
      for (int g = 0; g < D::n; ++g) v[g] = ok ? Elem<E>::to_f(in[(nn * K + k) * D::n + g]) : 0.f;
#pragma unroll
      for (int r = 0; r < D::n; ++r) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < D::n; ++g) s = fmaf(F[r][g], v[g], s);
        Xs[r][kk][mm] = s;
      }
    }
    for (int q = tid; q < D::n * BK * BO; q += THREADS) {
      const int oo = q % BO, kk = (q / BO) % BK, r = q / (BO * BK);
      const int o = o0 + oo, k = k0 + kk;
      Ws[r][kk][oo] = (o < O && k < K) ? planes[r * plane + (int64_t)k * O + o] : 0.f;
    }
    __syncthreads();
#pragma unroll 1
    for (int kk = 0; kk < BK; ++kk) {
      float x[D::n];
#pragma unroll
      for (int r = 0; r < D::n; ++r) x[r] = Xs[r][kk][tm];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float w[D::n];
#pragma unroll
        for (int r = 0; r < D::n; ++r) w[r] = Ws[r][kk][to + j];
        block_mac<M>(acc[j], x, w);
      }
    }
    __syncthreads();
  }
  const int64_t nn = n0 + tm;
  if (nn >= N) return;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int o = o0 + to + j;
    if (o >= O) continue;
    const float bo = bias ? bias[o] : 0.f;
    E* dst = out + (nn * O + o) * D::n;
#pragma unroll
    for (int g = 0; g < D::n; ++g) {
      float s = bo;
#pragma unroll
      for (int r = 0; r < D::n; ++r) s = fmaf(Fi[g][r], acc[j][r], s);
      dst[g] = Elem<E>::from_f(s);
    }
  }
}

// --------------------------------------------------------------- dW and db
// part[z][r][d][c] = sum over the split's tokens of (x^(rho)^T G^(rho))_r;
// dbpart[z][d] = sum of G's trivial plane.  Tile 32 d x 32 c; thread: 1 d x 4 c.
namespace dw {
constexpr int BD = 32, BC = 32, BKN = 8, THREADS = 256;
}

template <int M, typename E>
__global__ void __launch_bounds__(dw::THREADS)
dih_dw_kernel(const E* __restrict__ x, const E* __restrict__ gy, float* __restrict__ part,
              float* __restrict__ dbpart, int64_t N, int Cp, int Dp, int64_t tok_per_split) {
  using D = Dih<M>;
  using namespace dw;
  __shared__ float F[D::n][D::n], Fi[D::n][D::n];
  __shared__ float Gs[D::n][BKN][BD];
  __shared__ float Xs[D::n][BKN][BC];
  grid_dep_launch();
  make_tables<M>(F, Fi);
  grid_dep_wait();
  const int tid = threadIdx.x;
  const int td = tid / 8, tc = (tid % 8) * 4;
  const int c0 = blockIdx.x * BC, d0 = blockIdx.y * BD, z = blockIdx.z;
  const int64_t nbeg = (int64_t)z * tok_per_split;
  const int64_t nend = nbeg + tok_per_split < N ? nbeg + tok_per_split : N;
  float acc[4][D::n];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int r = 0; r < D::n; ++r) acc[j][r] = 0.f;
  float dbacc = 0.f;
  __syncthreads();
  for (int64_t nb = nbeg; nb < nend; nb += BKN) {
    // one (token, d) and one (token, c) transform per thread
    {
      const int kk = tid / BD, dd = tid % BD;
      const int64_t nn = nb + kk;
      const bool ok = nn < nend && d0 + dd < Dp;
      float v[D::n];
#pragma unroll
      for (int g = 0; g < D::n; ++g) v[g] = ok ? Elem<E>::to_f(gy[(nn * Dp + d0 + dd) * D::n + g]) : 0.f;
#pragma unroll
      for (int r = 0; r < D::n; ++r) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < D::n; ++g) s = fmaf(F[r][g], v[g], s);
        Gs[r][kk][dd] = s;
      }
    }
    {
      const int kk = tid / BC, cc = tid % BC;
      const int64_t nn = nb + kk;
      const bool ok = nn < nend && c0 + cc < Cp;
      float v[D::n];
#pragma unroll
      for (int g = 0; g < D::n; ++g) v[g] = ok ? Elem<E>::to_f(x[(nn * Cp + c0 + cc) * D::n + g]) : 0.f;
#pragma unroll
      for (int r = 0; r < D::n; ++r) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < D::n; ++g) s = fmaf(F[r][g], v[g], s);
        Xs[r][kk][cc] = s;
      }
    }
    __syncthreads();
#pragma unroll 1
    for (int kk = 0; kk < BKN; ++kk) {
      float gv[D::n];
#pragma unroll
      for (int r = 0; r < D::n; ++r) gv[r] = Gs[r][kk][td];
      dbacc += gv[0];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float xv[D::n], xt[D::n];
#pragma unroll
        for (int r = 0; r < D::n; ++r) xv[r] = Xs[r][kk][tc + j];
        // x^T: transpose each planar block, then the same blockwise product
#pragma unroll
        for (int r = 0; r < D::n1; ++r) xt[r] = xv[r];
#pragma unroll
        for (int k = 0; k < D::K2; ++k) {
          const int b = D::n1 + 4 * k;
          xt[b + 0] = xv[b + 0];
          xt[b + 1] = xv[b + 2];
          xt[b + 2] = xv[b + 1];
          xt[b + 3] = xv[b + 3];
        }
        block_mac<M>(acc[j], xt, gv);
      }
    }
    __syncthreads();
  }
  const int d = d0 + td;
  if (d >= Dp) return;
  const int64_t plane = (int64_t)Cp * Dp;
  float* base = part + (int64_t)z * D::n * plane;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = c0 + tc + j;
    if (c >= Cp) continue;
#pragma unroll
    for (int r = 0; r < D::n; ++r) base[r * plane + (int64_t)d * Cp + c] = acc[j][r];
  }
  if (blockIdx.x == 0 && tc == 0) dbpart[(int64_t)z * Dp + d] = dbacc;
}

// Sum the splits in index order, then the inverse transform: dW[d, c, u] =
// sum_r Fi[u][r] P_r[d, c]; db[d] = sum of the db partials.
template <int M>
__global__ void __launch_bounds__(256)
dih_reduce_kernel(const float* __restrict__ part, const float* __restrict__ dbpart, float* __restrict__ dW,
                  float* __restrict__ db, int splits, int Cp, int Dp) {
  using D = Dih<M>;
  __shared__ float F[D::n][D::n], Fi[D::n][D::n];
  grid_dep_launch();
  make_tables<M>(F, Fi);
  __syncthreads();
  grid_dep_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t plane = (int64_t)Cp * Dp;
  if (i < plane) {
    float P[D::n];
#pragma unroll
    for (int r = 0; r < D::n; ++r) P[r] = 0.f;
    for (int z = 0; z < splits; ++z)
#pragma unroll
      for (int r = 0; r < D::n; ++r) P[r] += part[((int64_t)z * D::n + r) * plane + i];
    // i = d * Cp + c: dW [d][c][u] is contiguous in u
#pragma unroll
    for (int u = 0; u < D::n; ++u) {
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < D::n; ++r) s = fmaf(Fi[u][r], P[r], s);
      dW[i * D::n + u] = s;
    }
  }
  if (db && i < Dp) {
    float s = 0.f;
    for (int z = 0; z < splits; ++z) s += dbpart[(int64_t)z * Dp + i];
    db[i] = s;
  }
}

// -------------------------------------------------------------------- host
template <int M, typename E>
static cudaError_t pretransform_t(const Handle& h, const void* W, const void* b, cudaStream_t st) {
  const int64_t n = h.Cp * h.Dp > h.Dp ? h.Cp * h.Dp : h.Dp;
  const cudaError_t e = launch_pdl(dih_pretransform_kernel<M, E>, dim3((unsigned)((n + 255) / 256)), dim3(256), 0,
                                   st, (const E*)W, (const E*)b, h.wf_fwd, h.wf_bwd, h.bias, (int)h.Cp, (int)h.Dp);
  count_launches(1);
  return e;
}

template <int M, typename E>
static cudaError_t apply_t(const Handle& h, bool backward, const void* in, void* out, int64_t N, cudaStream_t st) {
  const int K = (int)(backward ? h.Dp : h.Cp), O = (int)(backward ? h.Cp : h.Dp);
  const int64_t tiles_n = (N + ap::BM - 1) / ap::BM;
  if (tiles_n > 0x7fffffff) return cudaErrorInvalidValue;
  dim3 grid((unsigned)tiles_n, (unsigned)((O + ap::BO - 1) / ap::BO));
  const cudaError_t e = launch_pdl(dih_apply_kernel<M, E>, grid, dim3(ap::THREADS), 0, st, (const E*)in,
                                   (const float*)(backward ? h.wf_bwd : h.wf_fwd),
                                   (const float*)(backward ? nullptr : h.bias), (E*)out, N, K, O);
  count_launches(1);
  return e;
}

template <int M, typename E>
static cudaError_t dw_t(const Handle& h, const void* x, const void* gy, float* dW, float* db, int64_t N,
                        cudaStream_t st) {
  constexpr int n = Dih<M>::n;
  const int splits = simt_dw_splits(h.Cp, h.Dp, N);
  const int64_t tps = ((N + splits - 1) / splits + dw::BKN - 1) / dw::BKN * dw::BKN;
  const int64_t plane = h.Cp * h.Dp;
  if ((size_t)splits * ((size_t)n * plane + h.Dp) * sizeof(float) > h.ws_bytes) return cudaErrorInvalidValue;
  float* part = h.ws;
  float* dbpart = h.ws + (int64_t)splits * n * plane;
  dim3 grid((unsigned)((h.Cp + dw::BC - 1) / dw::BC), (unsigned)((h.Dp + dw::BD - 1) / dw::BD), (unsigned)splits);
  cudaError_t e = launch_pdl(dih_dw_kernel<M, E>, grid, dim3(dw::THREADS), 0, st, (const E*)x, (const E*)gy, part,
                             dbpart, N, (int)h.Cp, (int)h.Dp, tps);
  if (e != cudaSuccess) return e;
  count_launches(1);
  const int64_t cnt = plane > h.Dp ? plane : h.Dp;
  e = launch_pdl(dih_reduce_kernel<M>, dim3((unsigned)((cnt + 255) / 256)), dim3(256), 0, st, (const float*)part,
                 (const float*)dbpart, dW, db, splits, (int)h.Cp, (int)h.Dp);
  count_launches(1);
  return e;
}

template <typename E>
static cudaError_t dispatch(const Handle& h, int what, const void* a, const void* b, void* c, float* dW, float* db,
                            int64_t N, cudaStream_t st) {
#define EQLIN_DIH_CASE(MM)                                                                   \
  case MM:                                                                                   \
    if (what == 0) return pretransform_t<MM, E>(h, a, b, st);                                \
    if (what == 1) return apply_t<MM, E>(h, false, a, c, N, st);                             \
    if (what == 2) return apply_t<MM, E>(h, true, a, c, N, st);                              \
    return dw_t<MM, E>(h, a, b, dW, db, N, st);
  switch (h.m) {
    EQLIN_DIH_CASE(1)
    EQLIN_DIH_CASE(2)
    EQLIN_DIH_CASE(3)
    EQLIN_DIH_CASE(4)
    EQLIN_DIH_CASE(5)
    EQLIN_DIH_CASE(6)
    EQLIN_DIH_CASE(8)
  }
#undef EQLIN_DIH_CASE
  return cudaErrorInvalidValue;
}

static cudaError_t dispatch_dtype(const Handle& h, int what, const void* a, const void* b, void* c, float* dW,
                                  float* db, int64_t N, cudaStream_t st) {
  switch (h.dtype) {
    case EQLIN_F32: return dispatch<float>(h, what, a, b, c, dW, db, N, st);
    case EQLIN_F16: return dispatch<__half>(h, what, a, b, c, dW, db, N, st);
    case EQLIN_BF16: return dispatch<__nv_bfloat16>(h, what, a, b, c, dW, db, N, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dih

bool dihedral_supported(int m) { return m == 1 || m == 2 || m == 3 || m == 4 || m == 5 || m == 6 || m == 8; }

cudaError_t launch_dihedral_pretransform(const Handle& h, const void* W, const void* b, cudaStream_t st) {
  return dih::dispatch_dtype(h, 0, W, b, nullptr, nullptr, nullptr, 0, st);
}
cudaError_t launch_dihedral_apply(const Handle& h, bool backward, const void* in, void* out, int64_t N,
                                  cudaStream_t st) {
  return dih::dispatch_dtype(h, backward ? 2 : 1, in, nullptr, out, nullptr, nullptr, N, st);
}
cudaError_t launch_dihedral_dw(const Handle& h, const void* x, const void* gy, float* dW, float* db, int64_t N,
                               cudaStream_t st) {
  return dih::dispatch_dtype(h, 3, x, gy, nullptr, dW, db, N, st);
}

}  // namespace eqlin
