// eqlin_tc_dws.cu -- the weight gradient dW, db from stashed spectra.
//
// The stash forms of the forward and the input gradient write the group DFT
// of their inputs, X = DFT(x) and G = DFT(gy) (eqlin_tc.cu), as planes
// [T][channels][tokens] with tokens contiguous.  In the Fourier domain the
// weight gradient of each frequency is then a plain channel GEMM reducing
// over tokens (derived from the layer's definition; the pages print no
// backward formula):
//
//   dW_hat_k[d, c] = sum_n G_k[n, d] * conj(X_k[n, c])
//     real k:     dW_hat_k = sum_n G_k X_k
//     complex k:  Re = sum_n (Gr Xr + Gi Xi),   Im = sum_n (Gi Xr - Gr Xi)
//   db[d] = sum_n G_0[n, d]
//
// so this kernel has no transform at all: TMA brings 32-token slices of the
// spectra straight into a ring of K-major (token-contiguous), 64B-swizzled
// operand tiles, and one thread issues R(T) tcgen05 MMAs per 16 tokens -- for
// p4 six, two per real frequency and four for the complex one, the product
// with -Gr Xi taken with the instruction's negate-B bit so that no negated
// plane has to be stored.  ("Flash EQ-Linear", technical summary, sections
// "Abordagem Algoritmica" (per-frequency GEMMs on the half spectrum) and
// "Implementacao" (fused data flow: the spectra formed once, by the kernels
// that already need them).)
//
// Work unit of one CTA: 128 M channels x BC N channels x one contiguous chunk
// of tokens.  The M side is d or c, whichever pads less to a multiple of 128
// (M = d: A from G, B from X; M = c: A from X, B from G).  Roles:
//   warps 0-3   MMA issuers: lane 0 of warp i issues the MMAs of the
//               accumulator planes it owns (plane q belongs to issuer q mod 4;
//               one thread issues at most about one MMA per 160 cycles whatever
//               its size, and these MMAs are small); warp 0 allocates TMEM
//   warp 8      lane 0 issues the TMA loads of each stage (T A planes, T B planes)
//   warps 4-7   during the main loop, on the CTAs that own db for their d
//               channels, each thread sums the k = 0 plane of G along tokens for
//               one channel; after it, the accumulators out of TMEM (one warp per
//               lane quarter) into the per-chunk partial planes
// The partials [chunk][plane][N channel][M channel] are then summed over the
// chunks in a fixed order with the inverse DFT applied (dw_reduce_kernel;
// deterministic, no atomics).  Every wait is bounded as in eqlin_tc.cu.
#include <cudaTypedefs.h>

#include <type_traits>

#include "eqlin_internal.cuh"
#include "eqlin_ptx.cuh"
#include "eqlin_wait.cuh"

namespace eqlin {
namespace tcdws {

using namespace ptx;
using namespace waits;

template <int T>
struct Cfg {
  using G = Group<T>;
  static constexpr int BM = 128;                             // M channels per tile (MMA M)
  static constexpr int BKN = 32;                             // tokens per stage: two K = 16 MMA steps
  static constexpr int ROWB = BKN * 2;                       // 64-byte K-major rows, 64B swizzle
  static constexpr int BC_MAX = (512 / T) < 256 ? (512 / T) : 256;   // T*BC TMEM columns, MMA N <= 256
  static constexpr int A_PLANE = BM * ROWB;                  // 8 KB
  static constexpr int A_BYTES = T * A_PLANE;
  static constexpr int STAGE_BYTES = A_BYTES + T * BC_MAX * ROWB;   // slot stride (B planes BC * ROWB apart)
  static constexpr int BUDGET = 200 * 1024;
  static constexpr int STAGES = (BUDGET / STAGE_BYTES) > 6 ? 6 : (BUDGET / STAGE_BYTES);
  static_assert(STAGES >= 2, "two stages must fit");
  static constexpr int NBAR = 2 * STAGES + 1;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + NBAR * 8 + 16 + 1024;
  static constexpr int TMEM_COLS = T * BC_MAX <= 256 ? 256 : 512;
  static constexpr int NMMA = T < 4 ? T : 4;            // MMA issuers (warps 0 .. NMMA-1)
  static constexpr int MMA_WARP = 0, EPI0 = 4, EPI_WARPS = 4, PRODUCER = 8;
  static constexpr int THREADS = (PRODUCER + 1) * 32;
};

struct Params {
  int64_t N;
  int Cp, Dp;
  int mdim;               // M-side channels (Dp, or Cp when swapped)
  int BC;                 // N-side channels per tile (multiple of 16, <= BC_MAX)
  int n_mt, n_nt;         // M tiles, N tiles
  int swap;               // 0: M = d (A = G, B = X); 1: M = c (A = X, B = G)
  int64_t chunk;          // tokens per split (multiple of BKN)
  float* part;            // [splits][T][N channels][M channels]
  float* dbpart;          // [splits][Dp]
  int* err;
  uint32_t wait_limit;
  uint32_t ab_fmt;
};

// Sum of the eight 16-bit values of a 16-byte chunk, in FP32.
template <typename E>
__device__ __forceinline__ float sum8(uint4 u) {
  const E* e = reinterpret_cast<const E*>(&u);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += Elem<E>::to_f(e[i]);
  return s;
}

template <int T, typename E>
__global__ void __launch_bounds__(Cfg<T>::THREADS, 1)
tc_dws_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b, Params p) {
  using C = Cfg<T>;
  using G = Group<T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                     // TMA bytes of the stage landed
  uint64_t* empty = full + C::STAGES;        // MMA commit (+ one arrival per db warp)
  uint64_t* acc_full = empty + C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tiles = p.n_mt * p.n_nt;
  const int tile = blockIdx.x % tiles, z = blockIdx.x / tiles;
  const int mt = tile / p.n_nt, nt = tile % p.n_nt;
  const int m0 = mt * C::BM, n0 = nt * p.BC;
  const int64_t nbeg = (int64_t)z * p.chunk;
  const int64_t nend = (nbeg + p.chunk < p.N) ? nbeg + p.chunk : p.N;
  const int nst = (int)((nend - nbeg + C::BKN - 1) / C::BKN);
  const uint32_t limit = p.wait_limit;
  const int BC = p.BC;
  const uint32_t b_plane = (uint32_t)BC * C::ROWB;
  const bool swap = p.swap != 0;
  // The CTAs of the first tile on the other side own db of their d channels
  // for this chunk: the A rows (M = d) or the B rows (M = c) of plane 0.
  const bool sums_db = swap ? (mt == 0) : (nt == 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::NMMA + (sums_db ? C::EPI_WARPS : 0));
    }
    mbar_init(acc_full, C::NMMA);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();   // the previous kernel's writes are visible from here on

  if (warp == C::PRODUCER) {
    // --------------------------------------------------------- producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t n_issued = 0;
      bool ok = true;
      const uint32_t tx = (uint32_t)C::A_BYTES + (uint32_t)T * b_plane;
      for (int st = 0; st < nst; ++st) {
        if (!bwait(&empty[s], ph ^ 1, limit, abort_flag, p.err, site(K_DWS, 1, 2), (uint32_t)st)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[s], tx);
        const int n = (int)(nbeg + (int64_t)st * C::BKN);
        uint8_t* a = smem + s * C::STAGE_BYTES;
        uint8_t* b = a + C::A_BYTES;
#pragma unroll
        for (int q = 0; q < T; ++q) tma_load_3d(a + q * C::A_PLANE, &map_a, n, m0, q, &full[s]);
#pragma unroll
        for (int q = 0; q < T; ++q) tma_load_3d(b + q * b_plane, &map_b, n, n0, q, &full[s]);
        ++n_issued;
        if (++s == C::STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      // every issued copy lands before the CTA exits
      for (int i = 0; i < C::STAGES; ++i)
        if (n_issued > i)
          mbar_wait(&full[i], (uint32_t)(((n_issued - 1 - i) / C::STAGES) & 1), kDefaultWaitLimit);
    }
    __syncwarp();
    grid_dep_launch();
  } else if (warp < C::MMA_WARP + C::NMMA) {
    // -------------------------------------------------------------- MMA
    // Issuer mi owns the accumulator planes q with q % NMMA == mi.
    const int mi = warp - C::MMA_WARP;
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      const uint32_t id = idesc_f16(p.ab_fmt, (uint32_t)BC);
      const uint32_t id_neg = id | (1u << 14);     // D += A * (-B)
      const uint64_t desc0 = smem_desc(smem_u32(smem), C::ROWB);
      const uint32_t ap = C::A_PLANE >> 4, bp = b_plane >> 4;
      for (int st = 0; st < nst; ++st) {
        if (!bwait(&full[s], ph, limit, abort_flag, p.err, site(K_DWS, 2, 1), (uint32_t)st)) { ok = false; break; }
        tc_fence_after();
        const uint64_t a_d = desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
        const uint64_t b_d = a_d + (uint64_t)(C::A_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < C::BKN / 16; ++kk) {
          // 16 tokens = 32 bytes further along the swizzled rows
          const uint64_t ka = a_d + (uint64_t)(kk * 2), kb = b_d + (uint64_t)(kk * 2);
          const uint32_t acc = (st > 0 || kk > 0) ? 1u : 0u;
#pragma unroll
          for (int f = 0; f < G::nreal; ++f)
            if (f % C::NMMA == mi) mma_f16_ss(tmem_base + f * BC, ka + f * ap, kb + f * bp, id, acc);
#pragma unroll
          for (int k = 1; k <= G::ncomplex; ++k) {
            const int pr = G::nreal + 2 * (k - 1), pi = pr + 1;
            if (pr % C::NMMA == mi) {
              // Re += Ar Br + Ai Bi (both orientations)
              const uint32_t re = tmem_base + pr * BC;
              mma_f16_ss(re, ka + pr * ap, kb + pr * bp, id, acc);
              mma_f16_ss(re, ka + pi * ap, kb + pi * bp, id, 1u);
            }
            if (pi % C::NMMA == mi) {
              const uint32_t im = tmem_base + pi * BC;
              if (!swap) {
                // M = d (A = G, B = X): Im += Gi Xr - Gr Xi
                mma_f16_ss(im, ka + pi * ap, kb + pr * bp, id, acc);
                mma_f16_ss(im, ka + pr * ap, kb + pi * bp, id_neg, 1u);
              } else {
                // M = c (A = X, B = G): Im += Xr Gi - Xi Gr
                mma_f16_ss(im, ka + pr * ap, kb + pi * bp, id, acc);
                mma_f16_ss(im, ka + pi * ap, kb + pr * bp, id_neg, 1u);
              }
            }
          }
        }
        mma_commit(&empty[s]);
        if (++s == C::STAGES) { s = 0; ph ^= 1; }
      }
      if (ok) mma_commit(acc_full);
      else raise_abort(abort_flag, p.err);
      // The last commit of each slot fires on the completion the epilogue
      // waits for, and nothing else waits for it: an arrival after the CTA
      // has left would land in another kernel's shared memory.
      for (int i = 0; i < C::STAGES; ++i)
        if (nst > i)
          mbar_wait(&empty[i], (uint32_t)(((nst - 1 - i) / C::STAGES) & 1), kDefaultWaitLimit);
    }
    __syncwarp();
    grid_dep_launch();
  } else if (warp >= C::EPI0) {
    // -------------------------------------------- db sums, then epilogue
    const int r = (warp - C::EPI0) * 32 + lane;              // TMEM lane = M channel of the tile
    const int db_rows = swap ? BC : C::BM;
    float dbacc = 0.f;
    bool ok = true;
    if (sums_db) {
      int s = 0;
      uint32_t ph = 0;
      for (int st = 0; st < nst; ++st) {
        if (!wwait_all(&full[s], ph, limit, abort_flag, p.err, site(K_DWS, 3, 1), (uint32_t)st)) { ok = false; break; }
        if (r < db_rows) {
          // row r of plane 0 of G: 32 tokens in four 16-byte chunks (the
          // 64B swizzle permutes the chunks within the row; the sum is over all)
          const uint8_t* row = smem + s * C::STAGE_BYTES + (swap ? C::A_BYTES : 0) + r * C::ROWB;
          float a = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) a += sum8<E>(*reinterpret_cast<const uint4*>(row + 16 * j));
          dbacc += a;
        }
        // these generic reads precede the slot's next TMA write
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (++s == C::STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) raise_abort(abort_flag, p.err);
    }
    // The next kernel (the split reduction) may be scheduled once every role
    // of every CTA is past its main loop; earlier, its waiting CTAs would sit
    // on these SMs through the loop.
    grid_dep_launch();
    const bool got = ok && wwait_all(acc_full, 0, limit, abort_flag, p.err, site(K_DWS, 3, 3), 0u);
    if (ok && !got) raise_abort(abort_flag, p.err);
    if (got) {
      tc_fence_after();
      const uint32_t lane_addr = (uint32_t)((warp - C::EPI0) * 32) << 16;
      const int m = m0 + r;
      const bool row_ok = m < p.mdim;
      const int ndim = swap ? p.Dp : p.Cp;
      const int64_t plane = (int64_t)p.Cp * p.Dp;
      float* base = p.part + (int64_t)z * T * plane + m;
#pragma unroll 1
      for (int cc = 0; cc < BC; cc += 8) {
        uint32_t rg[T][8];
#pragma unroll
        for (int q = 0; q < T; ++q) tmem_ld_32x32b_x8(tmem_base + lane_addr + q * BC + cc, rg[q]);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int q = 0; q < T; ++q)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int n = n0 + cc + i;
              if (n < ndim) base[q * plane + (int64_t)n * p.mdim] = __uint_as_float(rg[q][i]);
            }
        }
      }
      if (sums_db && r < db_rows) {
        const int d = (swap ? n0 : m0) + r;
        if (d < p.Dp) p.dbpart[(int64_t)z * p.Dp + d] = dbacc;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
  if (warp >= C::MMA_WARP + C::NMMA && warp < C::EPI0) grid_dep_launch();   // idle warps
}

struct Plan {
  int BC, n_mt, n_nt, splits;
  bool swap;
  int64_t chunk;
};

// M side: d, unless c pads less to a multiple of 128.  N side: tiles of BC
// channels (a multiple of 16, at most BC_MAX) that split it evenly.  Token
// chunks: about one CTA per SM over all tiles.
template <int T>
static Plan plan(int64_t Cp, int64_t Dp, int64_t N, int sm_count) {
  using C = Cfg<T>;
  Plan pl;
  const int64_t pad_d = (Dp + C::BM - 1) / C::BM * C::BM - Dp;
  const int64_t pad_c = (Cp + C::BM - 1) / C::BM * C::BM - Cp;
  pl.swap = pad_c < pad_d;
  const int64_t mdim = pl.swap ? Cp : Dp, ndim = pl.swap ? Dp : Cp;
  const int64_t nnt = (ndim + C::BC_MAX - 1) / C::BC_MAX;
  pl.BC = (int)(((ndim + nnt - 1) / nnt + 15) / 16 * 16);
  pl.n_nt = (int)((ndim + pl.BC - 1) / pl.BC);
  pl.n_mt = (int)((mdim + C::BM - 1) / C::BM);
  const int tiles = pl.n_mt * pl.n_nt;
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
static cudaError_t launch_t(const Handle& h, const void* xs, const void* gs, float* dW, float* db, int64_t N,
                            cudaStream_t st) {
  using C = Cfg<T>;
  const Plan pl = plan<T>(h.Cp, h.Dp, N, h.sm_count);
  const size_t need = (size_t)pl.splits * ((size_t)T * h.Cp * h.Dp + h.Dp) * sizeof(float);
  if (need > h.ws_bytes) return cudaErrorInvalidValue;
  const auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return cudaErrorNotSupported;
  Params p;
  p.N = N;
  p.Cp = (int)h.Cp;
  p.Dp = (int)h.Dp;
  p.mdim = (int)(pl.swap ? h.Cp : h.Dp);
  p.BC = pl.BC;
  p.n_mt = pl.n_mt;
  p.n_nt = pl.n_nt;
  p.swap = pl.swap ? 1 : 0;
  p.chunk = pl.chunk;
  p.part = h.ws;
  p.dbpart = h.ws + (int64_t)pl.splits * T * h.Cp * h.Dp;
  p.err = h.err;
  p.wait_limit = h.wait_limit ? h.wait_limit : kDefaultWaitLimit;
  p.ab_fmt = std::is_same<E, __half>::value ? 0u : 1u;
  const CUtensorMapDataType dt = std::is_same<E, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // spectra [T][channels][ld]: boxes of 32 tokens x rows x 1 plane, 64B swizzle
  const int64_t ld = spectra_ld(N);
  CUtensorMap map_a, map_b;
  const void* srcs[2] = {pl.swap ? xs : gs, pl.swap ? gs : xs};
  const int64_t chans[2] = {pl.swap ? h.Cp : h.Dp, pl.swap ? h.Dp : h.Cp};
  const int rows[2] = {C::BM, pl.BC};
  CUtensorMap* maps[2] = {&map_a, &map_b};
  for (int i = 0; i < 2; ++i) {
    cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)chans[i], (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)chans[i] * ld * 2};
    cuuint32_t box[3] = {(cuuint32_t)C::BKN, (cuuint32_t)rows[i], 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(maps[i], dt, 3, const_cast<void*>(srcs[i]), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(tc_dws_kernel<T, E>), C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  const unsigned grid = (unsigned)(pl.n_mt * pl.n_nt * pl.splits);
  cudaError_t e = launch_pdl(tc_dws_kernel<T, E>, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st, map_a, map_b, p);
  if (e != cudaSuccess) return e;
  count_launches(1);
  // partials are [N channel][M channel]: c-major over d when M = d
  return launch_dw_reduce(h, pl.splits, p.part, p.dbpart, dW, db, /*cd_layout=*/!pl.swap, st);
}

template <typename E>
static cudaError_t launch_e(const Handle& h, const void* xs, const void* gs, float* dW, float* db, int64_t N,
                            cudaStream_t st) {
  switch (h.T) {
    case 1: return launch_t<1, E>(h, xs, gs, dW, db, N, st);
    case 2: return launch_t<2, E>(h, xs, gs, dW, db, N, st);
    case 4: return launch_t<4, E>(h, xs, gs, dW, db, N, st);
    case 8: return launch_t<8, E>(h, xs, gs, dW, db, N, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tcdws

size_t tc_dws_workspace_bytes(int T, int64_t Cp, int64_t Dp, int sm_count) {
  switch (T) {
    case 1: return tcdws::workspace_bytes<1>(Cp, Dp, sm_count);
    case 2: return tcdws::workspace_bytes<2>(Cp, Dp, sm_count);
    case 4: return tcdws::workspace_bytes<4>(Cp, Dp, sm_count);
    case 8: return tcdws::workspace_bytes<8>(Cp, Dp, sm_count);
  }
  return 0;
}

cudaError_t launch_tc_dw_spectra(const Handle& h, const void* xs, const void* gs, float* dW, float* db, int64_t N,
                                 cudaStream_t st) {
  if (h.dtype == EQLIN_F16) return tcdws::launch_e<__half>(h, xs, gs, dW, db, N, st);
  if (h.dtype == EQLIN_BF16) return tcdws::launch_e<__nv_bfloat16>(h, xs, gs, dW, db, N, st);
  return cudaErrorNotSupported;
}

}  // namespace eqlin
