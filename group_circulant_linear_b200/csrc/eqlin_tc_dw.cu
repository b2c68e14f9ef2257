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
// contiguous chunk of tokens, in stages of 16 tokens.  Roles:
//   warp 8     (producer)  TMA: the stage's gy rows of the 128 d channels and
//              x rows of the BC c channels into shared memory, and L2
//              prefetches of later stages
//   warps 0-3  (one thread per d)  read the channel's T group values of the 16
//              tokens, take the group DFT (packed token pairs for T <= 4, FP32
//              for T = 8), keep sum_n G_0 in FP32 for db and write the K-major
//              (token-contiguous) A planes; after the main loop they read the
//              accumulators out of TMEM
//   warps 4-7  (one thread per c)  the same for x, writing the B planes
//              (real frequencies, then Im X, Re X, -Im X per complex one)
//   warp 9     allocates TMEM; one thread issues the MMAs
// The per-chunk partial planes go to the handle's workspace as
// [chunk][plane][c][d]; a second kernel sums the chunks in a fixed order and
// applies the inverse DFT (deterministic, no atomics).  All waits are bounded
// as in eqlin_tc.cu.
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
  static constexpr int BKN = 16;                          // tokens per stage (one MMA K step)
  static constexpr int ROWB = BKN * 2;                    // 32-byte K-major rows, 32B swizzle
  static constexpr int BC_MAX = (512 / T) < 128 ? (512 / T) : 128;
  static constexpr int Q = G::nreal + 3 * G::ncomplex;    // B planes
  static constexpr int A_PLANE_BYTES = BM * ROWB;
  static constexpr int A_BYTES = T * A_PLANE_BYTES;
  static constexpr int B_BYTES = Q * BC_MAX * ROWB;       // plane stride is BC * ROWB at run time
  // raw tiles of a stage (TMA, row-major): gy [16 tokens][128 d x T], x [16 tokens][BC x T]
  static constexpr int GY_ROWB = BM * T * 2;
  static constexpr int X_ROWB_MAX = BC_MAX * T * 2;
  static constexpr int RAW_BYTES = BKN * (GY_ROWB + X_ROWB_MAX);
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + RAW_BYTES;
  static constexpr int STAGES_FIT = (220 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static_assert(STAGES >= 2, "two stages must fit");
  static constexpr int NBAR = 4 * STAGES + 2;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + NBAR * 8 + 16 + 1024;
  static constexpr int TMEM_COLS = T * BC_MAX <= 256 ? 256 : 512;
  static constexpr int PRODUCER = 8, MMA_WARP = 9;
  static constexpr int THREADS = 320;
  static constexpr int PF_STAGES = 12;                    // L2 prefetch distance (stages)
  static constexpr int GY_BOX = BM * T <= 256 ? BM * T : 256;   // gy TMA box width (elements)
  static constexpr int W = packed::Words<T>::n;
};

struct Params {
  int64_t N;
  int Cp, Dp;
  int BC;                 // input channels per tile (multiple of 16)
  int n_dt, n_ct;         // d tiles, c tiles
  int64_t chunk;          // tokens per split (multiple of BKN)
  int x_box;              // x TMA box width (elements), divides BC * T
  float* part;            // [splits][T][Cp][Dp]
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

// every lane waits (readers of TMA-written data); the warp agrees on the outcome
__device__ __forceinline__ bool wwait_all(uint64_t* bar, uint32_t parity, uint32_t limit,
                                          volatile int* abort_flag) {
  return __all_sync(0xffffffffu, bwait(bar, parity, limit, abort_flag));
}

// lane 0 waits, the warp follows (slot reuse)
__device__ __forceinline__ bool wwait(uint64_t* bar, uint32_t parity, uint32_t limit,
                                      volatile int* abort_flag, int lane) {
  int ok = 0;
  if (lane == 0) ok = bwait(bar, parity, limit, abort_flag) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* err) {
  *abort_flag = 1;
  atomicCAS(err, DEV_OK, DEV_TIMEOUT);
}

template <typename E>
__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  E* e = reinterpret_cast<E*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) e[i] = Elem<E>::from_f(f[i]);
  return u;
}

// Byte offset of the 16-byte chunk j (8 tokens) of row r in a 32B-swizzled K-major plane.
__device__ __forceinline__ uint32_t kmajor_off(int r, int j) {
  return (uint32_t)(r * 32 + ((j ^ ((r >> 2) & 1)) << 4));
}

template <int T, typename E>
__global__ void __launch_bounds__(Cfg<T>::THREADS, 1)
tc_dw_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_gy, Params p) {
  using C = Cfg<T>;
  using G = Group<T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* a_buf = smem;
  uint8_t* b_buf = a_buf + C::STAGES * C::A_BYTES;
  uint8_t* raw_buf = b_buf + C::STAGES * C::B_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(raw_buf + C::STAGES * C::RAW_BYTES);
  uint64_t* raw_full = bars;                      // TMA
  uint64_t* raw_empty = raw_full + C::STAGES;     // 8 transform warps
  uint64_t* op_full = raw_empty + C::STAGES;      // 8 transform warps
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
  const int x_rowb = BC * T * 2;                  // raw x row bytes of this tile

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], 8);
      mbar_init(&op_full[i], 8);
      mbar_init(&op_empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&map_x);
    prefetch_tensormap(&map_gy);
  }
  if (warp == C::MMA_WARP) {
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
    const bool active = is_a || r < BC;
    // this thread's channel in the raw tile rows
    const uint32_t raw_col = is_a ? (uint32_t)((r / (C::GY_BOX / T)) * C::BKN * C::GY_BOX * 2 +
                                               (r % (C::GY_BOX / T)) * T * 2)
                                  : (uint32_t)((r * T / p.x_box) * C::BKN * p.x_box * 2 +
                                               ((r * T) % p.x_box) * 2);
    const uint32_t raw_rowb = is_a ? (uint32_t)(C::GY_BOX * 2) : (uint32_t)(p.x_box * 2);
    const uint32_t raw_base = is_a ? 0u : (uint32_t)(C::BKN * C::GY_ROWB);
    float dbacc = 0.f;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int st = 0; st < nst; ++st) {
      if (!wwait_all(&raw_full[s], ph, limit, abort_flag) ||
          !wwait(&op_empty[s], ph ^ 1, limit, abort_flag, lane)) {
        ok = false;
        break;
      }
      if (active) {
        const uint8_t* raw = raw_buf + s * C::RAW_BYTES + raw_base + raw_col;
        uint8_t* a_st = a_buf + s * C::A_BYTES;
        uint8_t* b_st = b_buf + s * C::B_BYTES;
#pragma unroll
        for (int g = 0; g < C::BKN / 8; ++g) {
          uint32_t wv[8][C::W];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint8_t* src = raw + (g * 8 + j) * raw_rowb;
            if constexpr (C::W == 4) {
              const uint4 u = *reinterpret_cast<const uint4*>(src);
              wv[j][0] = u.x; wv[j][1] = u.y; wv[j][2] = u.z; wv[j][3] = u.w;
            } else if constexpr (C::W == 2) {
              const uint2 u = *reinterpret_cast<const uint2*>(src);
              wv[j][0] = u.x; wv[j][1] = u.y;
            } else if constexpr (T == 2) {
              wv[j][0] = *reinterpret_cast<const uint32_t*>(src);
            } else {
              wv[j][0] = *reinterpret_cast<const unsigned short*>(src);
            }
          }
          uint32_t Pw[T][4];
          if constexpr (T <= 4) {
#pragma unroll
            for (int pr = 0; pr < 4; ++pr) {
              uint32_t P[T];
              packed::dft_pair<T, E>(wv[2 * pr], wv[2 * pr + 1], P);
#pragma unroll
              for (int q = 0; q < T; ++q) Pw[q][pr] = P[q];
              if (is_a) {
                const float2 f = packed::Pair<E>::to_f2(P[0]);
                dbacc += f.x + f.y;
              }
            }
          } else {
            // T = 8: FP32 butterflies (sqrt(2)/2 twiddles), one rounding per value
#pragma unroll
            for (int pr = 0; pr < 4; ++pr) {
              float Pa[T], Pb[T], va[T], vb[T];
              const E* ea = reinterpret_cast<const E*>(wv[2 * pr]);
              const E* eb = reinterpret_cast<const E*>(wv[2 * pr + 1]);
#pragma unroll
              for (int t = 0; t < T; ++t) { va[t] = Elem<E>::to_f(ea[t]); vb[t] = Elem<E>::to_f(eb[t]); }
              G::dft(va, Pa);
              G::dft(vb, Pb);
              dbacc += Pa[0] + Pb[0];
#pragma unroll
              for (int q = 0; q < T; ++q) {
                E two[2] = {Elem<E>::from_f(Pa[q]), Elem<E>::from_f(Pb[q])};
                Pw[q][pr] = *reinterpret_cast<const uint32_t*>(two);
              }
            }
          }
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
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&raw_empty[s]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&op_full[s]);
      if (++s == C::STAGES) { s = 0; ph ^= 1; }
    }
    if (!ok) raise_abort(abort_flag, p.err);

    if (is_a) {
      // ------------------------------------------------------- epilogue
      // partial planes [z][T][Cp][Dp]: a warp stores 32 consecutive d of one c
      const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
      bool got = ok && wwait_all(acc_full, 0, limit, abort_flag);
      if (!got && ok) raise_abort(abort_flag, p.err);
      if (got) {
        tc_fence_after();
        const int d = d0 + r;
        const bool row_ok = d < p.Dp;
        const int64_t plane = (int64_t)p.Cp * p.Dp;
        float* base = p.part + (int64_t)z * T * plane + d;
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
          if (row_ok) {
#pragma unroll
            for (int q = 0; q < T; ++q)
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int c = c0 + cc + i;
                if (c < p.Cp) base[q * plane + (int64_t)c * p.Dp] = __uint_as_float(rg[q][i]);
              }
          }
        }
        if (c0 == 0 && row_ok) p.dbpart[(int64_t)z * p.Dp + d] = dbacc;
      }
    }
  } else if (warp == C::PRODUCER) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t n_raw = 0;
      bool ok = true;
      const uint32_t tx = (uint32_t)(C::BKN * (C::GY_ROWB + x_rowb));
      auto prefetch = [&](int ps) {
        if (ps >= nst) return;
        const int n = (int)(nbeg + (int64_t)ps * C::BKN);
        for (int xb = 0; xb < C::BM * T; xb += C::GY_BOX) tma_prefetch_2d(&map_gy, d0 * T + xb, n);
        for (int xb = 0; xb < BC * T; xb += p.x_box) tma_prefetch_2d(&map_x, c0 * T + xb, n);
      };
      for (int i = 0; i < C::PF_STAGES; ++i) prefetch(i);
      for (int st = 0; st < nst; ++st) {
        prefetch(st + C::PF_STAGES);
        if (!bwait(&raw_empty[s], ph ^ 1, limit, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&raw_full[s], tx);
        const int n = (int)(nbeg + (int64_t)st * C::BKN);
        uint8_t* dst = raw_buf + s * C::RAW_BYTES;
        for (int b = 0; b < C::BM * T / C::GY_BOX; ++b)
          tma_load_2d(dst + b * C::BKN * C::GY_BOX * 2, &map_gy, d0 * T + b * C::GY_BOX, n, &raw_full[s]);
        dst += C::BKN * C::GY_ROWB;
        for (int b = 0; b < BC * T / p.x_box; ++b)
          tma_load_2d(dst + b * C::BKN * p.x_box * 2, &map_x, c0 * T + b * p.x_box, n, &raw_full[s]);
        ++n_raw;
        if (++s == C::STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      for (int i = 0; i < C::STAGES; ++i)
        if (n_raw > i) mbar_wait(&raw_full[i], (uint32_t)(((n_raw - 1 - i) / C::STAGES) & 1), kDefaultWaitLimit);
    }
  } else if (lane == 0) {
    // -------------------------------------------------------------- MMA
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    const uint32_t id_real = idesc_f16(p.ab_fmt, (uint32_t)BC);
    const uint32_t id_cplx = idesc_f16(p.ab_fmt, (uint32_t)(2 * BC));
    for (int st = 0; st < nst; ++st) {
      if (!bwait(&op_full[s], ph, limit, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t a_st = smem_u32(a_buf + s * C::A_BYTES);
      const uint32_t b_st = smem_u32(b_buf + s * C::B_BYTES);
      const uint32_t first = st > 0 ? 1u : 0u;
#pragma unroll
      for (int f = 0; f < G::nreal; ++f)
        mma_f16_ss(tmem_base + f * BC, smem_desc(a_st + f * C::A_PLANE_BYTES, C::ROWB),
                   smem_desc(b_st + f * b_plane, C::ROWB), id_real, first);
#pragma unroll
      for (int k = 1; k <= G::ncomplex; ++k) {
        const int pr = G::nreal + 2 * (k - 1);
        const int q = G::nreal + 3 * (k - 1);
        const uint32_t col = tmem_base + G::nreal * BC + (k - 1) * 2 * BC;
        // [Re | Im] += Re G [Re X ; -Im X]
        mma_f16_ss(col, smem_desc(a_st + pr * C::A_PLANE_BYTES, C::ROWB),
                   smem_desc(b_st + (q + 1) * b_plane, C::ROWB), id_cplx, first);
        // [Re | Im] += Im G [Im X ; Re X]
        mma_f16_ss(col, smem_desc(a_st + (pr + 1) * C::A_PLANE_BYTES, C::ROWB),
                   smem_desc(b_st + q * b_plane, C::ROWB), id_cplx, 1u);
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
  if (warp == C::MMA_WARP) {
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
  // x box: the largest power-of-two width <= 256 elements that divides BC * T
  int x_box = 256;
  while ((pl.BC * T) % x_box) x_box >>= 1;
  CUtensorMap map_x, map_gy;
  const void* srcs[2] = {x, gy};
  const int64_t widths[2] = {h.Cp * T, h.Dp * T};
  const int boxes[2] = {x_box, C::GY_BOX};
  CUtensorMap* maps[2] = {&map_x, &map_gy};
  for (int i = 0; i < 2; ++i) {
    cuuint64_t dims[2] = {(cuuint64_t)widths[i], (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)widths[i] * 2};
    cuuint32_t box[2] = {(cuuint32_t)boxes[i], (cuuint32_t)C::BKN};
    cuuint32_t es[2] = {1, 1};
    if (enc(maps[i], dt, 2, const_cast<void*>(srcs[i]), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  p.x_box = x_box;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(tc_dw_kernel<T, E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const unsigned grid = (unsigned)(pl.n_dt * pl.n_ct * pl.splits);
  tc_dw_kernel<T, E><<<grid, C::THREADS, C::SMEM_BYTES, st>>>(map_x, map_gy, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  count_launches(1);
  return launch_dw_reduce(h, pl.splits, p.part, p.dbpart, dW, db, /*cd_layout=*/true, st);
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
