// eqlin_tc_dw.cu -- tcgen05 kernel for the weight gradient dW and db.
//
// In the Fourier domain the weight gradient of every frequency k is a channel
// GEMM that reduces over tokens (derived from the layer's definition; the
// pages print no backward formula):
//
//   dW_hat_k[d, c] = sum_n G_k[n, d] * conj(X_k[n, c]),   G = DFT_t(gy), X = DFT_t(x)
//   dW[d, c, tau]  = IDFT_k(dW_hat)[tau]   (with the 1/T),   db[d] = sum_n G_0[n, d]
//
// For a complex frequency the two real outputs come from two block products
// of N = 2*BC columns:  [Re | Im] = Re G [Re X ; -Im X] + Im G [Im X ; Re X],
// so p4 again needs six real GEMMs.
//
// Work unit of one CTA: 128 output channels d x BC input channels c x one
// contiguous chunk of tokens.  Roles:
//   warps 0-3  (one thread per d)  load gy[n, d*T .. d*T+T) straight from
//              global memory -- a warp reads 256 contiguous bytes per token --,
//              one stage ahead of use (double-buffered in registers), take the
//              DFT on packed pairs of tokens (T <= 4; FP32 with one rounding
//              for T = 8), keep sum_n G_0 in FP32 for db and write the K-major
//              (token-contiguous) operand planes;
//              after the main loop they read the accumulators out of TMEM
//   warps 4-7  (one thread per c)  the same for x, writing the B planes
//              (real frequencies, then Im X, Re X, -Im X per complex one)
//   warp 8     allocates TMEM; one thread issues the MMAs and, several
//              stages ahead, L2 prefetches (TMA) of the gy and x rows
// The per-chunk partial planes go to the handle's workspace; a second kernel
// sums the chunks in a fixed order and applies the inverse DFT
// (deterministic, no atomics).  All waits are bounded as in eqlin_tc.cu.
#include <cudaTypedefs.h>

#include <type_traits>

#include "eqlin_internal.cuh"
#include "eqlin_packed.cuh"
#include "eqlin_ptx.cuh"

namespace eqlin {
namespace tcdw {

using namespace ptx;

template <int T>
struct Cfg {
  using G = Group<T>;
  static constexpr int BM = 128;                          // output channels d per tile (MMA M)
  static constexpr int BKN = 32;                          // tokens per stage (MMA K = 2 x 16)
  static constexpr int ROWB = BKN * 2;                    // 64-byte K-major rows, 64B swizzle
  static constexpr int BC_MAX = (512 / T) < 128 ? (512 / T) : 128;
  static constexpr int Q = G::nreal + 3 * G::ncomplex;    // B planes
  static constexpr int A_PLANE_BYTES = BM * ROWB;
  static constexpr int A_BYTES = T * A_PLANE_BYTES;
  static constexpr int B_BYTES = Q * BC_MAX * ROWB;       // plane stride is BC * ROWB at run time
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_FIT = (220 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static_assert(STAGES >= 2, "two stages must fit");
  static constexpr int NBAR = 2 * STAGES + 2;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + NBAR * 8 + 16 + 1024;
  static constexpr int TMEM_COLS = T * BC_MAX <= 256 ? 256 : 512;
  static constexpr int THREADS = 288;
  static constexpr int PF_STAGES = 8;                     // L2 prefetch distance (stages)
};

struct Params {
  int64_t N;
  int Cp, Dp;
  int BC;                 // input channels per tile (multiple of 16)
  int n_dt, n_ct;         // d tiles, c tiles
  int64_t chunk;          // tokens per split (multiple of BKN)
  float* part;            // [splits][T][Dp][Cp]
  float* dbpart;          // [splits][Dp]
  int* err;
  uint32_t wait_limit;
  uint32_t ab_fmt;
};

__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, uint32_t limit,
                                      volatile int* abort_flag) {
  uint64_t t0 = 0;
  for (uint32_t i = 0; i < limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 15u) {
      if (*abort_flag) return false;
      const uint64_t t = globaltimer_ns();
      if (t0 == 0) t0 = t;
      else if (t - t0 > kWaitTimeNs) return false;
    }
  }
  return false;
}

__device__ __forceinline__ bool wwait(uint64_t* bar, uint32_t parity, uint32_t limit,
                                      volatile int* abort_flag) {
  return __all_sync(0xffffffffu, bwait(bar, parity, limit, abort_flag));
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* err) {
  *abort_flag = 1;
  atomicCAS(err, DEV_OK, DEV_TIMEOUT);
}

// Load the T group values of one channel of one token (T*2 bytes, one vector load).
template <int T, typename E>
__device__ __forceinline__ void load_group(const E* p, float* v) {
  if constexpr (T == 8) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const E* e = reinterpret_cast<const E*>(&u);
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] = Elem<E>::to_f(e[t]);
  } else if constexpr (T == 4) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    const E* e = reinterpret_cast<const E*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) v[t] = Elem<E>::to_f(e[t]);
  } else if constexpr (T == 2) {
    const unsigned u = __ldg(reinterpret_cast<const unsigned*>(p));
    const E* e = reinterpret_cast<const E*>(&u);
    v[0] = Elem<E>::to_f(e[0]);
    v[1] = Elem<E>::to_f(e[1]);
  } else {
    const unsigned short u = __ldg(reinterpret_cast<const unsigned short*>(p));
    v[0] = Elem<E>::to_f(*reinterpret_cast<const E*>(&u));
  }
}

template <typename E>
__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  E* e = reinterpret_cast<E*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) e[i] = Elem<E>::from_f(f[i]);
  return u;
}

// Byte offset of the 16-byte chunk j (8 tokens) of row r in a 64B-swizzled K-major plane.
__device__ __forceinline__ uint32_t kmajor_off(int r, int j) {
  return (uint32_t)(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

template <int T, typename E>
__global__ void __launch_bounds__(Cfg<T>::THREADS, 1)
tc_dw_kernel(const E* __restrict__ x, const E* __restrict__ gy, const __grid_constant__ CUtensorMap map_x,
             const __grid_constant__ CUtensorMap map_gy, Params p) {
  using C = Cfg<T>;
  using G = Group<T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* a_buf = smem;
  uint8_t* b_buf = a_buf + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_buf + C::STAGES * C::B_BYTES);
  uint64_t* op_full = bars;                       // 8 transform warps arrive
  uint64_t* op_empty = op_full + C::STAGES;       // MMA commit
  uint64_t* acc_full = op_empty + C::STAGES;
  uint64_t* drain_bar = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tiles = p.n_dt * p.n_ct;
  const int tile = blockIdx.x % tiles, z = blockIdx.x / tiles;
  const int d0 = (tile / p.n_ct) * C::BM, c0 = (tile % p.n_ct) * p.BC;
  const int64_t nbeg = (int64_t)z * p.chunk;
  const int64_t nend = (nbeg + p.chunk < p.N) ? nbeg + p.chunk : p.N;
  const int nst = (int)((nend - nbeg + C::BKN - 1) / C::BKN);
  const uint32_t limit = p.wait_limit;
  const int BC = p.BC;
  const uint32_t b_plane = (uint32_t)BC * C::ROWB;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) { mbar_init(&op_full[i], 8); mbar_init(&op_empty[i], 1); }
    mbar_init(acc_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 8) {
    // --------------------------------------------------- transform warps
    const bool is_a = warp < 4;
    const int r = (warp & 3) * 32 + lane;                 // operand row: d (A) or c (B)
    const int ch = is_a ? d0 + r : c0 + r;                // channel index in the tensor
    const int nch = is_a ? p.Dp : p.Cp;
    const bool active = is_a || r < BC;
    const bool valid = active && ch < nch;
    const E* src = (is_a ? gy : x) + (int64_t)(valid ? ch : 0) * T;
    const int64_t pitch = (int64_t)nch * T;
    constexpr int W = packed::Words<T>::n;                // 32-bit words per token and channel
    constexpr int TOK = C::BKN;
    float dbacc = 0.f;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;

    // Raw words of one stage: one vector load per token, issued ahead of use.
    auto load_stage = [&](uint32_t (&buf)[TOK][W], int st) {
      const int64_t n_st = nbeg + (int64_t)st * TOK;
#pragma unroll
      for (int j = 0; j < TOK; ++j) {
        const int64_t n = n_st + j;
        if (valid && st < nst && n < nend) {
          packed::load_words<T>(src + n * pitch, buf[j]);
        } else {
#pragma unroll
          for (int w = 0; w < W; ++w) buf[j][w] = 0u;
        }
      }
    };

    // Write the plane words of one group of 8 tokens (g) into the stage slot.
    auto store_group = [&](uint32_t (&Pw)[T][4], int g, uint8_t* a_st, uint8_t* b_st) {
      const uint32_t off = kmajor_off(r, g);
      if (is_a) {
#pragma unroll
        for (int q = 0; q < T; ++q)
          *reinterpret_cast<uint4*>(a_st + q * C::A_PLANE_BYTES + off) =
              make_uint4(Pw[q][0], Pw[q][1], Pw[q][2], Pw[q][3]);
      } else {
#pragma unroll
        for (int f = 0; f < G::nreal; ++f)
          *reinterpret_cast<uint4*>(b_st + f * b_plane + off) =
              make_uint4(Pw[f][0], Pw[f][1], Pw[f][2], Pw[f][3]);
#pragma unroll
        for (int k = 1; k <= G::ncomplex; ++k) {
          const int pr = G::nreal + 2 * (k - 1);
          const int q = G::nreal + 3 * (k - 1);
          const uint32_t* re = Pw[pr];
          const uint32_t* im = Pw[pr + 1];
          *reinterpret_cast<uint4*>(b_st + (q + 0) * b_plane + off) = make_uint4(im[0], im[1], im[2], im[3]);
          *reinterpret_cast<uint4*>(b_st + (q + 1) * b_plane + off) = make_uint4(re[0], re[1], re[2], re[3]);
          *reinterpret_cast<uint4*>(b_st + (q + 2) * b_plane + off) =
              make_uint4(packed::neg2(im[0]), packed::neg2(im[1]), packed::neg2(im[2]), packed::neg2(im[3]));
        }
      }
    };

    // One stage: wait for the slot, transform the buffered tokens, publish.
    auto run_stage = [&](const uint32_t (&buf)[TOK][W]) -> bool {
      if (!wwait(&op_empty[s], ph ^ 1, limit, abort_flag)) return false;
      if (active) {
        uint8_t* a_st = a_buf + s * C::A_BYTES;
        uint8_t* b_st = b_buf + s * C::B_BYTES;
#pragma unroll
        for (int g = 0; g < TOK / 8; ++g) {
          uint32_t Pw[T][4];
          if constexpr (T <= 4) {
#pragma unroll
            for (int pr = 0; pr < 4; ++pr) {
              uint32_t P[T];
              packed::dft_pair<T, E>(buf[g * 8 + 2 * pr], buf[g * 8 + 2 * pr + 1], P);
#pragma unroll
              for (int q = 0; q < T; ++q) Pw[q][pr] = P[q];
              if (is_a) {
                const float2 f = packed::Pair<E>::to_f2(P[0]);
                dbacc += f.x + f.y;
              }
            }
          }
          store_group(Pw, g, a_st, b_st);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&op_full[s]);
      if (++s == C::STAGES) { s = 0; ph ^= 1; }
      return true;
    };

    if constexpr (T <= 4) {
      // double-buffered: the next stage's loads are in flight while this one is transformed
      uint32_t bufA[TOK][W], bufB[TOK][W];
      load_stage(bufA, 0);
      for (int st = 0; st < nst; st += 2) {
        load_stage(bufB, st + 1);
        if (!run_stage(bufA)) { ok = false; break; }
        if (st + 1 >= nst) break;
        load_stage(bufA, st + 2);
        if (!run_stage(bufB)) { ok = false; break; }
      }
    } else {
      // T = 8: FP32 butterflies with the sqrt(2)/2 twiddles; loads per group of 8 tokens
      for (int st = 0; st < nst; ++st) {
        if (!wwait(&op_empty[s], ph ^ 1, limit, abort_flag)) { ok = false; break; }
        if (active) {
          uint8_t* a_st = a_buf + s * C::A_BYTES;
          uint8_t* b_st = b_buf + s * C::B_BYTES;
          const int64_t n_st = nbeg + (int64_t)st * TOK;
#pragma unroll 1
          for (int g = 0; g < TOK / 8; ++g) {
            uint32_t raw[8][W];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int64_t n = n_st + g * 8 + j;
              if (valid && n < nend) {
                packed::load_words<T>(src + n * pitch, raw[j]);
              } else {
#pragma unroll
                for (int w = 0; w < W; ++w) raw[j][w] = 0u;
              }
            }
            float Pf[T][8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const E* e = reinterpret_cast<const E*>(raw[j]);
              float v[T], Pj[T];
#pragma unroll
              for (int t = 0; t < T; ++t) v[t] = Elem<E>::to_f(e[t]);
              G::dft(v, Pj);
#pragma unroll
              for (int q = 0; q < T; ++q) Pf[q][j] = Pj[q];
              dbacc += Pj[0];
            }
            uint32_t Pw[T][4];
#pragma unroll
            for (int q = 0; q < T; ++q) {
              const uint4 u = pack8<E>(Pf[q]);
              Pw[q][0] = u.x; Pw[q][1] = u.y; Pw[q][2] = u.z; Pw[q][3] = u.w;
            }
            store_group(Pw, g, a_st, b_st);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&op_full[s]);
        if (++s == C::STAGES) { s = 0; ph ^= 1; }
      }
    }
    if (!ok) raise_abort(abort_flag, p.err);

    if (is_a) {
      // ------------------------------------------------------- epilogue
      const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
      bool got = ok && wwait(acc_full, 0, limit, abort_flag);
      if (!got && ok) raise_abort(abort_flag, p.err);
      if (got) {
        tc_fence_after();
        const bool row_ok = d0 + r < p.Dp;
        const int64_t plane = (int64_t)p.Cp * p.Dp;
        float* base = p.part + (int64_t)z * T * plane + (int64_t)(d0 + r) * p.Cp;
#pragma unroll 1
        for (int cc = 0; cc < BC; cc += 8) {
          uint32_t rg[T][8];
#pragma unroll
          for (int f = 0; f < G::nreal; ++f) tmem_ld_32x32b_x8(tmem_base + lane_addr + f * BC + cc, rg[f]);
#pragma unroll
          for (int k = 1; k <= G::ncomplex; ++k) {
            const uint32_t col = tmem_base + lane_addr + G::nreal * BC + (k - 1) * 2 * BC + cc;
            tmem_ld_32x32b_x8(col, rg[G::nreal + 2 * (k - 1)]);
            tmem_ld_32x32b_x8(col + BC, rg[G::nreal + 2 * (k - 1) + 1]);
          }
          tmem_wait_ld();
          const int c = c0 + cc;
          if (row_ok && c < p.Cp) {
#pragma unroll
            for (int q = 0; q < T; ++q) {
              float* dst = base + q * plane + c;
              if (c + 8 <= p.Cp) {
                reinterpret_cast<float4*>(dst)[0] =
                    make_float4(__uint_as_float(rg[q][0]), __uint_as_float(rg[q][1]),
                                __uint_as_float(rg[q][2]), __uint_as_float(rg[q][3]));
                reinterpret_cast<float4*>(dst)[1] =
                    make_float4(__uint_as_float(rg[q][4]), __uint_as_float(rg[q][5]),
                                __uint_as_float(rg[q][6]), __uint_as_float(rg[q][7]));
              } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  if (c + i < p.Cp) dst[i] = __uint_as_float(rg[q][i]);
              }
            }
          }
        }
        if (c0 == 0 && row_ok) p.dbpart[(int64_t)z * p.Dp + d0 + r] = dbacc;
      }
    }
  } else if (lane == 0) {
    // -------------------------------------------------------------- MMA
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    const uint32_t id_real = idesc_f16(p.ab_fmt, (uint32_t)BC);
    const uint32_t id_cplx = idesc_f16(p.ab_fmt, (uint32_t)(2 * BC));
    // L2 prefetch of the gy and x rows of stage `ps` (this CTA's d and c range)
    auto prefetch = [&](int ps) {
      if (ps >= nst) return;
      const int n = (int)(nbeg + (int64_t)ps * C::BKN);
      for (int xb = 0; xb < C::BM * T; xb += 256) tma_prefetch_2d(&map_gy, d0 * T + xb, n);
      for (int xb = 0; xb < BC * T; xb += 256) tma_prefetch_2d(&map_x, c0 * T + xb, n);
    };
    for (int i = 0; i < C::PF_STAGES; ++i) prefetch(i);
    for (int st = 0; st < nst; ++st) {
      prefetch(st + C::PF_STAGES);
      if (!bwait(&op_full[s], ph, limit, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t a_st = smem_u32(a_buf + s * C::A_BYTES);
      const uint32_t b_st = smem_u32(b_buf + s * C::B_BYTES);
#pragma unroll
      for (int ks = 0; ks < C::BKN / 16; ++ks) {
        const uint32_t koff = ks * 32;
        const uint32_t first = (st > 0 || ks > 0) ? 1u : 0u;
#pragma unroll
        for (int f = 0; f < G::nreal; ++f)
          mma_f16_ss(tmem_base + f * BC, smem_desc(a_st + f * C::A_PLANE_BYTES + koff, C::ROWB),
                     smem_desc(b_st + f * b_plane + koff, C::ROWB), id_real, first);
#pragma unroll
        for (int k = 1; k <= G::ncomplex; ++k) {
          const int pr = G::nreal + 2 * (k - 1);
          const int q = G::nreal + 3 * (k - 1);
          const uint32_t col = tmem_base + G::nreal * BC + (k - 1) * 2 * BC;
          // [Re | Im] += Re G [Re X ; -Im X]
          mma_f16_ss(col, smem_desc(a_st + pr * C::A_PLANE_BYTES + koff, C::ROWB),
                     smem_desc(b_st + (q + 1) * b_plane + koff, C::ROWB), id_cplx, first);
          // [Re | Im] += Im G [Im X ; Re X]
          mma_f16_ss(col, smem_desc(a_st + (pr + 1) * C::A_PLANE_BYTES + koff, C::ROWB),
                     smem_desc(b_st + q * b_plane + koff, C::ROWB), id_cplx, 1u);
        }
      }
      mma_commit(&op_empty[s]);
      if (++s == C::STAGES) { s = 0; ph ^= 1; }
    }
    if (ok) mma_commit(acc_full);
    else raise_abort(abort_flag, p.err);
    mma_commit(drain_bar);
    mbar_wait(drain_bar, 0, kDefaultWaitLimit);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

struct Plan {
  int BC, n_dt, n_ct, splits;
  int64_t chunk;
};

template <int T>
static Plan plan(int64_t Cp, int64_t Dp, int64_t N, int sm_count) {
  using C = Cfg<T>;
  Plan pl;
  const int64_t nct = (Cp + C::BC_MAX - 1) / C::BC_MAX;
  pl.BC = (int)(((Cp + nct - 1) / nct + 15) / 16 * 16);
  pl.n_ct = (int)((Cp + pl.BC - 1) / pl.BC);
  pl.n_dt = (int)((Dp + C::BM - 1) / C::BM);
  const int tiles = pl.n_dt * pl.n_ct;
  int s = sm_count / tiles;
  if (s < 1) s = 1;
  const int64_t max_by_n = (N + C::BKN - 1) / C::BKN;
  if (s > max_by_n) s = (int)max_by_n;
  pl.chunk = ((N + s - 1) / s + C::BKN - 1) / C::BKN * C::BKN;
  pl.splits = (int)((N + pl.chunk - 1) / pl.chunk);
  return pl;
}

template <int T>
size_t workspace_bytes(int64_t Cp, int64_t Dp, int sm_count) {
  const Plan pl = plan<T>(Cp, Dp, INT64_C(1) << 40, sm_count);
  return (size_t)pl.splits * ((size_t)T * Cp * Dp + Dp) * sizeof(float);
}

template <int T, typename E>
static cudaError_t launch_t(const Handle& h, const void* x, const void* gy, float* dW, float* db,
                            int64_t N, cudaStream_t st) {
  using C = Cfg<T>;
  const Plan pl = plan<T>(h.Cp, h.Dp, N, h.sm_count);
  const size_t need = (size_t)pl.splits * ((size_t)T * h.Cp * h.Dp + h.Dp) * sizeof(float);
  if (need > h.ws_bytes) return cudaErrorInvalidValue;
  Params p;
  p.N = N;
  p.Cp = (int)h.Cp;
  p.Dp = (int)h.Dp;
  p.BC = pl.BC;
  p.n_dt = pl.n_dt;
  p.n_ct = pl.n_ct;
  p.chunk = pl.chunk;
  p.part = h.ws;
  p.dbpart = h.ws + (int64_t)pl.splits * T * h.Cp * h.Dp;
  p.err = h.err;
  p.wait_limit = h.wait_limit ? h.wait_limit : kDefaultWaitLimit;
  p.ab_fmt = std::is_same<E, __half>::value ? 0u : 1u;
  // tensor maps used only for L2 prefetches of the token chunks
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!enc) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return cudaErrorNotSupported;
    enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  const CUtensorMapDataType dt = std::is_same<E, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap map_x, map_gy;
  const void* srcs[2] = {x, gy};
  const int64_t widths[2] = {h.Cp * T, h.Dp * T};
  CUtensorMap* maps[2] = {&map_x, &map_gy};
  for (int i = 0; i < 2; ++i) {
    cuuint64_t dims[2] = {(cuuint64_t)widths[i], (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)widths[i] * 2};
    cuuint32_t box[2] = {(cuuint32_t)(widths[i] < 256 ? widths[i] : 256), (cuuint32_t)C::BKN};
    cuuint32_t es[2] = {1, 1};
    if (enc(maps[i], dt, 2, const_cast<void*>(srcs[i]), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(tc_dw_kernel<T, E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const unsigned grid = (unsigned)(pl.n_dt * pl.n_ct * pl.splits);
  tc_dw_kernel<T, E><<<grid, C::THREADS, C::SMEM_BYTES, st>>>((const E*)x, (const E*)gy, map_x, map_gy, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  count_launches(1);
  return launch_dw_reduce(h, pl.splits, p.part, p.dbpart, dW, db, st);
}

template <typename E>
static cudaError_t launch_e(const Handle& h, const void* x, const void* gy, float* dW, float* db,
                            int64_t N, cudaStream_t st) {
  switch (h.T) {
    case 1: return launch_t<1, E>(h, x, gy, dW, db, N, st);
    case 2: return launch_t<2, E>(h, x, gy, dW, db, N, st);
    case 4: return launch_t<4, E>(h, x, gy, dW, db, N, st);
    case 8: return launch_t<8, E>(h, x, gy, dW, db, N, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tcdw

bool tc_dw_supported(const Handle& h) {
  return (h.dtype == EQLIN_F16 || h.dtype == EQLIN_BF16) &&
         (h.T == 1 || h.T == 2 || h.T == 4 || h.T == 8);
}

size_t tc_dw_workspace_bytes(int T, int64_t Cp, int64_t Dp, int sm_count) {
  switch (T) {
    case 1: return tcdw::workspace_bytes<1>(Cp, Dp, sm_count);
    case 2: return tcdw::workspace_bytes<2>(Cp, Dp, sm_count);
    case 4: return tcdw::workspace_bytes<4>(Cp, Dp, sm_count);
    case 8: return tcdw::workspace_bytes<8>(Cp, Dp, sm_count);
  }
  return 0;
}

cudaError_t launch_tc_dw(const Handle& h, const void* x, const void* gy, float* dW, float* db,
                         int64_t N, cudaStream_t st) {
  if (h.dtype == EQLIN_F16) return tcdw::launch_e<__half>(h, x, gy, dW, db, N, st);
  if (h.dtype == EQLIN_BF16) return tcdw::launch_e<__nv_bfloat16>(h, x, gy, dW, db, N, st);
  return cudaErrorNotSupported;
}

}  // namespace eqlin
