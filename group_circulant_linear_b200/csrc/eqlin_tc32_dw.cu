// eqlin_tc32_dw.cu -- FP32 weight gradient dW, db on the tensor cores, 3xTF32.
//
// The same Fourier-domain reduction over tokens as the f16/bf16 kernel
// (eqlin_tc_dw.cu; derived from the layer's definition, the pages print no
// backward formula):
//
//   dW_hat_k[d, c] = sum_n G_k[n, d] * conj(X_k[n, c]),   db[d] = sum_n G_0[n, d]
//
// with every real product split as in the forward (eqlin_tc32.cu): each
// transformed value v becomes hi = tf32(v) and lo = tf32(v - hi), and a
// product a*b is taken as hi(a)hi(b) + hi(a)lo(b) + lo(a)hi(b), three
// kind::tf32 MMAs into one FP32 accumulator.
//
// The tensor core adds each MMA's products into the accumulator with a
// rounding of its own, whose error grows with the number of MMAs that feed
// one accumulator (measured: about 1.5e-8 to 1.9e-8 relative error per MMA).
// So one accumulator takes at most 256 MMAs, as in the forward: 672 tokens
// for T = 1, 680 for T = 2 (three MMAs per 8 tokens), 336 for T = 4 (six into
// a complex accumulator).  A token range longer than
// (splits x that) runs as more waves of CTAs, each split with its own partial
// slot, up to four per SM and tile; beyond that as several launches
// ("passes") over consecutive token ranges, the first writing the per-split
// partial planes and the later ones adding to them in IEEE FP32 (each split's
// slot belongs to one CTA per pass, so the sums are deterministic).  The
// fixed-order reduction over splits and the inverse DFT then follow
// (launch_dw_reduce).
//
// Work unit of one CTA: 128 M channels (d, or c when that pads less) x BC
// N channels (BC <= 256 for T = 1, 2, <= 128 for T = 4) x one chunk of
// tokens, in stages of 16 tokens for T = 1 (two TF32 K steps, 64-byte K-major
// rows with the 64B swizzle; a stage's fixed costs -- barrier waits, commits,
// proxy fences -- then cover twice the work) and 8 for T = 2, 4 (one K step,
// 32-byte rows with the 32B swizzle; their 16-token stages would not fit
// twice in shared memory):
//   warp 16    (producer)  TMA of the stage's raw rows (M side, N side) into
//              the raw ring, L2 prefetches ahead
//   warps 0-15 (transform) two groups of eight warps on alternate stages, so
//              two stages are in flight; in a group 4 A warps (one M channel
//              per thread) and 4 B warps (one or two N channels per thread): the
//              channel's T values of the stage's 8 tokens, the group DFT in
//              FP32, db sums of G_0 on the gy side, the hi/lo split, two
//              16-byte chunks per plane; after the loop the A warps read the
//              accumulators out of TMEM into the partial planes
//   warp 17(+18) MMA issue, an accumulator group per issuer as in the
//              f16/bf16 kernel; for a complex frequency the block products
//   M = d:  [Re | Im] = Re G [Re X ; -Im X] + Im G [Im X ; Re X]   (B planes Im X, Re X, -Im X)
//   M = c:  [Re | Im] = Re X [Re G ; Im G] + Im X [Im G ; -Re G]   (B planes Re G, Im G, -Re G)
// All waits are bounded as in the other tensor-core kernels.
#include <cudaTypedefs.h>

#include "eqlin_internal.cuh"
#include "eqlin_ptx.cuh"
#include "eqlin_wait.cuh"

namespace eqlin {
namespace tc32dw {

using namespace ptx;
using namespace waits;

template <int T>
struct Cfg {
  using G = Group<T>;
  static_assert(T == 1 || T == 2 || T == 4, "3xTF32 tiles for T in {1, 2, 4}");
  static constexpr int BM = 128;                          // M channels per tile (MMA M)
  // N channels per tile: 256 for T = 1, 2 (T * 256 <= 512 TMEM columns), 128
  // for T = 4 (its complex block products are N = 2 * BC MMAs).  Wide N keeps
  // the operand reads per FLOP down: an N = 128 TF32 MMA already reads its
  // operands at the SM's shared-memory rate.
  static constexpr int BC_MAX = T <= 2 ? 256 : 128;
  static constexpr int NRB = BC_MAX / 128;                // N channels per B-side transform thread
  // tokens per stage: 16 for T = 1 (two TF32 K steps), 8 otherwise (the
  // operands of a 16-token stage would not fit twice beside the raw ring)
  static constexpr int BKN = T == 1 ? 16 : 8;
  static constexpr int KSTEPS = BKN / 8;
  static constexpr int ROWB = BKN * 4;                    // K-major rows of 64 or 32 bytes
  static constexpr int Q = G::nreal + 3 * G::ncomplex;    // B planes per part (hi / lo)
  static constexpr int A_PLANE_BYTES = BM * ROWB;
  static constexpr int A_BYTES = 2 * T * A_PLANE_BYTES;   // hi planes 0..T-1, lo planes T..2T-1
  static constexpr int B_BYTES = 2 * Q * BC_MAX * ROWB;   // plane stride BC * ROWB at run time
  static constexpr int OP_BYTES = A_BYTES + B_BYTES;
  // M-side TMA box width (f32 elements): whole channels, at most 256
  static constexpr int MA_BOX = BM * T <= 256 ? BM * T : 256;
  static_assert((BM * T) % MA_BOX == 0 && MA_BOX % T == 0, "whole channels per box, whole boxes per tile");
  static constexpr int MA_ROWB = BM * T * 4;
  static constexpr int NB_ROWB_MAX = BC_MAX * T * 4;
  static constexpr int RAW_BYTES = BKN * (MA_ROWB + NB_ROWB_MAX);
  static constexpr int BUDGET = 220 * 1024;
  static constexpr int OP_STAGES = (BUDGET - 3 * OP_BYTES) / RAW_BYTES >= 4 ? 3 : 2;
  static constexpr int RAW_FIT = (BUDGET - OP_STAGES * OP_BYTES) / RAW_BYTES;
  // even: the transform groups take alternate stages, and both uses of a raw
  // slot k and k + RAW_STAGES then belong to the same group, which consumes
  // them in order (an mbarrier parity wait cannot tell a phase from the one
  // two ahead)
  static constexpr int RAW_STAGES = (RAW_FIT > 6 ? 6 : RAW_FIT) & ~1;
  static_assert(RAW_STAGES >= 2, "two raw stages must fit");
  static constexpr int GRP_WARPS = 8;                     // warps per transform group
  static constexpr int NMMA = (T == 1) ? 1 : 2;
  static constexpr int MMAS = G::nreal + 2 * G::ncomplex;
  __host__ __device__ static constexpr int own_real(int f) { return (NMMA == 1 || 2 * f < MMAS) ? 0 : 1; }
  __host__ __device__ static constexpr int own_cplx(int k) {
    return (NMMA == 1 || 2 * (G::nreal + 2 * (k - 1)) < MMAS) ? 0 : 1;
  }
  static constexpr int NBAR = 2 * RAW_STAGES + 2 * OP_STAGES + 1 + NMMA;
  static constexpr int SMEM_BYTES = OP_STAGES * OP_BYTES + RAW_STAGES * RAW_BYTES + NBAR * 8 + 16 + BC_MAX * 4 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
  static constexpr int TMEM_COLS = T * BC_MAX <= 256 ? 256 : 512;
  static constexpr int TR_WARPS = 16;
  static constexpr int PRODUCER = TR_WARPS, MMA_WARP = TR_WARPS + 1;
  static constexpr int THREADS = (TR_WARPS + 1 + NMMA) * 32;
  static constexpr int PF_STAGES = 16;
  // tokens one accumulator takes: at most 256 MMAs (three, or six into a
  // complex accumulator, per 8-token K step), whole stages
  static constexpr int CHUNK_MAX = 256 / (3 * (G::ncomplex > 0 ? 2 : 1)) * 8 / BKN * BKN;
};

struct Params {
  int64_t N;              // tokens in total
  int64_t n_beg;          // first token of this pass
  int Cp, Dp;
  int mdim;               // M-side channels (Dp, or Cp when swapped)
  int BC;                 // N-side channels per tile (multiple of 16)
  int n_mt, n_nt;
  int swap;               // 0: M = d (A from gy, B from x); 1: M = c (A from x, B from gy)
  int accumulate;         // 0: write the partial planes; 1: add to them
  int64_t chunk;          // tokens per split (multiple of 8, at most Cfg::CHUNK_MAX)
  int nb_box;             // N-side TMA box width (elements), divides BC * T
  float* part;            // [splits][T][N channels][M channels]
  float* dbpart;          // [splits][Dp]
  int* err;
  uint32_t wait_limit;
};

// 16-byte chunk j (4 tokens) of row r in a K-major plane with ROWB-byte rows:
// 32B swizzle (chunk bit 0 XOR row bit 2) for 32-byte rows, 64B swizzle
// (chunk bits 0-1 XOR row bits 1-2) for 64-byte rows
template <int ROWB>
__device__ __forceinline__ uint32_t kmajor_off(int r, int j) {
  if constexpr (ROWB == 32) return (uint32_t)(r * 32 + ((j ^ ((r >> 2) & 1)) << 4));
  else return (uint32_t)(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

template <int N_>
__device__ __forceinline__ void load_group(const uint8_t* src, float (&v)[N_]) {
  static_assert(N_ == 1 || N_ == 2 || N_ == 4, "a channel's T values");
  if constexpr (N_ == 4) {
    const float4 u = *reinterpret_cast<const float4*>(src);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  } else if constexpr (N_ == 2) {
    const float2 u = *reinterpret_cast<const float2*>(src);
    v[0] = u.x; v[1] = u.y;
  } else {
    v[0] = *reinterpret_cast<const float*>(src);
  }
}

template <int T>
__global__ void __launch_bounds__(Cfg<T>::THREADS, 1)
tc32_dw_kernel(const __grid_constant__ CUtensorMap map_m, const __grid_constant__ CUtensorMap map_n, Params p) {
  using C = Cfg<T>;
  using G = Group<T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* op_buf = smem;                                         // [OP_STAGES][A | B]
  uint8_t* raw_buf = op_buf + C::OP_STAGES * C::OP_BYTES;        // [RAW_STAGES][M side | N side]
  uint64_t* bars = reinterpret_cast<uint64_t*>(raw_buf + C::RAW_STAGES * C::RAW_BYTES);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + C::RAW_STAGES;
  uint64_t* op_full = raw_empty + C::RAW_STAGES;
  uint64_t* op_empty = op_full + C::OP_STAGES;
  uint64_t* acc_full = op_empty + C::OP_STAGES;
  uint64_t* drain_bar = acc_full + 1;           // [NMMA]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + C::NMMA);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* db_half = reinterpret_cast<float*>(tmem_slot + 4);       // [BC_MAX] group 1's db sums

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tiles = p.n_mt * p.n_nt;
  const int tile = blockIdx.x % tiles, z = blockIdx.x / tiles;
  const int mt = tile / p.n_nt, nt = tile % p.n_nt;
  const int m0 = mt * C::BM, n0 = nt * p.BC;
  const int64_t nbeg = p.n_beg + (int64_t)z * p.chunk;
  const int64_t nend = (nbeg + p.chunk < p.N) ? nbeg + p.chunk : p.N;
  const int nst = nend > nbeg ? (int)((nend - nbeg + C::BKN - 1) / C::BKN) : 0;
  const uint32_t limit = p.wait_limit;
  const int BC = p.BC;
  const uint32_t b_plane = (uint32_t)BC * C::ROWB;
  const int nb_rowb = BC * T * 4;
  const bool swap = p.swap != 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::RAW_STAGES; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], C::GRP_WARPS);
    }
    for (int i = 0; i < C::OP_STAGES; ++i) {
      mbar_init(&op_full[i], C::GRP_WARPS);
      mbar_init(&op_empty[i], C::NMMA);
    }
    mbar_init(acc_full, C::NMMA);
    for (int i = 0; i < C::NMMA; ++i) mbar_init(&drain_bar[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&map_m);
    prefetch_tensormap(&map_n);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();

  if (warp < C::TR_WARPS) {
    // --------------------------------------------------- transform warps
    const int grp = warp >> 3;                             // stages grp, grp + 2, ...
    const bool is_a = (warp & 7) < 4;
    const int r = (warp & 3) * 32 + lane;                  // first operand row: M channel (A) or N channel (B)
    const int nrows = is_a ? 1 : C::NRB;                   // rows r, r + 128, ... of this thread
    const bool sums_db = is_a != swap;                     // the side that holds gy
    const uint32_t raw_rowb = is_a ? (uint32_t)(C::MA_BOX * 4) : (uint32_t)(p.nb_box * 4);
    // this thread's channels in the raw tile rows
    uint32_t raw_base[C::NRB];
#pragma unroll
    for (int i = 0; i < C::NRB; ++i) {
      const int rr = r + 128 * i;
      raw_base[i] = is_a ? (uint32_t)((rr / (C::MA_BOX / T)) * C::BKN * C::MA_BOX * 4 + (rr % (C::MA_BOX / T)) * T * 4)
                         : (uint32_t)(C::BKN * C::MA_ROWB + (rr * T / p.nb_box) * C::BKN * p.nb_box * 4 +
                                      ((rr * T) % p.nb_box) * 4);
    }
    float dbacc[C::NRB];
#pragma unroll
    for (int i = 0; i < C::NRB; ++i) dbacc[i] = 0.f;
    int rs = grp % C::RAW_STAGES, os = grp % C::OP_STAGES;
    uint32_t rph = 0, oph = 0;
    bool ok = true;
    for (int st = grp; st < nst; st += 2) {
      if (!wwait_all(&raw_full[rs], rph, limit, abort_flag, p.err, site(K_DW, 1, 1), (uint32_t)st)) { ok = false; break; }
      if (!wwait(&op_empty[os], oph ^ 1, limit, abort_flag, lane, p.err, site(K_DW, 1, 4), (uint32_t)st)) { ok = false; break; }
      uint8_t* a_st = op_buf + os * C::OP_BYTES;
      uint8_t* b_st = a_st + C::A_BYTES;
#pragma unroll
      for (int i = 0; i < C::NRB; ++i) {
        const int rr = r + 128 * i;
        if (i >= nrows || (!is_a && rr >= BC)) continue;
        const uint8_t* raw = raw_buf + rs * C::RAW_BYTES + raw_base[i];
        // the stage's tokens as 16-byte chunks of 4 tokens per plane row
#pragma unroll
        for (int c4 = 0; c4 < C::BKN / 4; ++c4) {
          uint32_t hi[T][4], lo[T][4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float v[T], P[T];
            load_group<T>(raw + (4 * c4 + j) * raw_rowb, v);
            G::dft(v, P);
            if (sums_db) dbacc[i] += P[0];
#pragma unroll
            for (int q = 0; q < T; ++q) {
              hi[q][j] = f32_to_tf32(P[q]);
              lo[q][j] = f32_to_tf32(P[q] - __uint_as_float(hi[q][j]));
            }
          }
          const uint32_t off = kmajor_off<C::ROWB>(rr, c4);
          auto put = [&](uint8_t* plane_base, const uint32_t (&w)[4], uint32_t sign) {
            *reinterpret_cast<uint4*>(plane_base + off) =
                make_uint4(w[0] ^ sign, w[1] ^ sign, w[2] ^ sign, w[3] ^ sign);
          };
          if (is_a) {
#pragma unroll
            for (int q = 0; q < T; ++q) {
              put(a_st + q * C::A_PLANE_BYTES, hi[q], 0u);
              put(a_st + (T + q) * C::A_PLANE_BYTES, lo[q], 0u);
            }
          } else {
#pragma unroll
            for (int f = 0; f < G::nreal; ++f) {
              put(b_st + f * b_plane, hi[f], 0u);
              put(b_st + (C::Q + f) * b_plane, lo[f], 0u);
            }
#pragma unroll
            for (int k = 1; k <= G::ncomplex; ++k) {
              const int pr = G::nreal + 2 * (k - 1);
              const int q = G::nreal + 3 * (k - 1);
              // M = d: (Im X, Re X, -Im X);  M = c: (Re G, Im G, -Re G).  The split
              // rounds to nearest (ties away), symmetric in sign: a negated
              // plane is the hi and lo of the plane with their signs flipped.
              const int i0 = swap ? pr : pr + 1, i1 = swap ? pr + 1 : pr;
              put(b_st + (q + 0) * b_plane, hi[i0], 0u);
              put(b_st + (q + 1) * b_plane, hi[i1], 0u);
              put(b_st + (q + 2) * b_plane, hi[i0], 0x80000000u);
              put(b_st + (C::Q + q + 0) * b_plane, lo[i0], 0u);
              put(b_st + (C::Q + q + 1) * b_plane, lo[i1], 0u);
              put(b_st + (C::Q + q + 2) * b_plane, lo[i0], 0x80000000u);
            }
          }
        }
      }
      // orders this stage's reads of the raw slot (before its TMA refill) and
      // its operand writes (before the MMA)
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&raw_empty[rs]);
        mbar_arrive(&op_full[os]);
      }
      rs += 2;
      if (rs >= C::RAW_STAGES) { rs -= C::RAW_STAGES; rph ^= 1; }
      os += 2;
      if (os >= C::OP_STAGES) { os -= C::OP_STAGES; oph ^= 1; }
    }
    if (!ok) raise_abort(abort_flag, p.err);
    grid_dep_launch();

    // db: the side that sums G_0 writes (or adds) its channels' sums; group 1
    // (the odd stages) hands its sums to group 0 through shared memory.  Only
    // the tiles of the other side's first tile write, so each d is written
    // once per chunk.
    const bool db_tile = swap ? (mt == 0) : (nt == 0);
    if (sums_db && db_tile) {
      const int bar_id = is_a ? 1 : 2;
      named_bar_sync(bar_id, 256);
      if (grp == 1)
        for (int i = 0; i < nrows; ++i) db_half[r + 128 * i] = dbacc[i];
      named_bar_sync(bar_id, 256);
      for (int i = 0; i < nrows; ++i) {
        const int rr = r + 128 * i;
        const int d = (swap ? n0 : m0) + rr;
        if (grp == 0 && (is_a || rr < BC) && d < p.Dp) {
          float* dst = p.dbpart + (int64_t)z * p.Dp + d;
          const float v = dbacc[i] + db_half[rr];
          *dst = p.accumulate ? *dst + v : v;
        }
      }
    }

    if (is_a) {
      // ------------------------------------------------------- epilogue
      // Partial planes [z][T][N channel][M channel]: a warp stores 32
      // consecutive M channels of one N channel; transform group g takes the
      // N columns [g * BC/2, (g+1) * BC/2).
      const bool all_ok = named_bar_and(3, 256, ok);
      const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
      bool got = all_ok && wwait_all(acc_full, 0, limit, abort_flag, p.err, site(K_DW, 4, 5), 0u);
      if (!got && all_ok) raise_abort(abort_flag, p.err);
      if (got) {
        tc_fence_after();
        const int m = m0 + r;
        const bool row_ok = m < p.mdim;
        const int ndim = swap ? p.Dp : p.Cp;
        const int64_t plane = (int64_t)p.Cp * p.Dp;
        float* base = p.part + (int64_t)z * T * plane + m;
        const int cbeg = grp * (BC / 2), cend = cbeg + BC / 2;
#pragma unroll 1
        for (int cc = cbeg; cc < cend; cc += 8) {
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
            // a later pass adds to the partials: the chunk's T x 8 loads go out
            // together, before any of its stores, so they wait one memory
            // latency rather than one each
            float add[T][8];
#pragma unroll
            for (int q = 0; q < T; ++q)
#pragma unroll
              for (int i = 0; i < 8; ++i)
                add[q][i] = (p.accumulate && n0 + cc + i < ndim) ? base[q * plane + (int64_t)(n0 + cc + i) * p.mdim]
                                                                 : 0.f;
#pragma unroll
            for (int q = 0; q < T; ++q)
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int n = n0 + cc + i;
                if (n < ndim) base[q * plane + (int64_t)n * p.mdim] = add[q][i] + __uint_as_float(rg[q][i]);
              }
          }
        }
      }
    }
  } else if (warp == C::PRODUCER) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t n_raw = 0;
      bool ok = true;
      const uint32_t tx = (uint32_t)(C::BKN * (C::MA_ROWB + nb_rowb));
      auto prefetch = [&](int ps) {
        if (ps >= nst) return;
        const int n = (int)(nbeg + (int64_t)ps * C::BKN);
        for (int xb = 0; xb < C::BM * T; xb += C::MA_BOX) tma_prefetch_2d(&map_m, m0 * T + xb, n);
        for (int xb = 0; xb < BC * T; xb += p.nb_box) tma_prefetch_2d(&map_n, n0 * T + xb, n);
      };
      for (int i = 0; i < C::PF_STAGES; ++i) prefetch(i);
      for (int st = 0; st < nst; ++st) {
        prefetch(st + C::PF_STAGES);
        if (!bwait(&raw_empty[s], ph ^ 1, limit, abort_flag, p.err, site(K_DW, 2, 2), (uint32_t)st)) { ok = false; break; }
        mbar_arrive_expect_tx(&raw_full[s], tx);
        const int n = (int)(nbeg + (int64_t)st * C::BKN);
        uint8_t* dst = raw_buf + s * C::RAW_BYTES;
        for (int b = 0; b < C::BM * T / C::MA_BOX; ++b)
          tma_load_2d(dst + b * C::BKN * C::MA_BOX * 4, &map_m, m0 * T + b * C::MA_BOX, n, &raw_full[s]);
        dst += C::BKN * C::MA_ROWB;
        for (int b = 0; b < BC * T / p.nb_box; ++b)
          tma_load_2d(dst + b * C::BKN * p.nb_box * 4, &map_n, n0 * T + b * p.nb_box, n, &raw_full[s]);
        ++n_raw;
        if (++s == C::RAW_STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      for (int i = 0; i < C::RAW_STAGES; ++i)
        if (n_raw > i)
          mbar_wait(&raw_full[i], (uint32_t)(((n_raw - 1 - i) / C::RAW_STAGES) & 1), kDefaultWaitLimit);
    }
    __syncwarp();
    grid_dep_launch();
  } else {
    // -------------------------------------------------------------- MMA
    const int mi = warp - C::MMA_WARP;
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      const uint32_t id_real = idesc_tf32((uint32_t)BC);          // both operands K-major
      const uint32_t id_cplx = idesc_tf32((uint32_t)(2 * BC));
      const uint64_t desc0 = smem_desc(smem_u32(op_buf), C::ROWB);
      // window of the first complex product: M = d uses B planes q+1..q+2, M = c planes q..q+1
      const int w1 = swap ? 0 : 1, w2 = swap ? 1 : 0;
      for (int st = 0; st < nst; ++st) {
        if (!bwait(&op_full[s], ph, limit, abort_flag, p.err, site(K_DW, 3, 3), (uint32_t)st)) { ok = false; break; }
        tc_fence_after();
        const uint64_t a_d = desc0 + (uint64_t)((s * C::OP_BYTES) >> 4);
        const uint64_t b_d = a_d + (uint64_t)(C::A_BYTES >> 4);
        const uint32_t bp = b_plane >> 4;
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          // K step kk: 8 tokens = 32 bytes further along the swizzled rows
          const uint64_t ka = a_d + (uint64_t)(kk * 2), kb = b_d + (uint64_t)(kk * 2);
          auto A = [&](int plane) { return ka + (uint64_t)((plane * C::A_PLANE_BYTES) >> 4); };
          auto B = [&](int plane) { return kb + (uint64_t)plane * bp; };
          // a * b = hi(a) hi(b) + hi(a) lo(b) + lo(a) hi(b)
          auto prod3 = [&](uint32_t d, int pa, int pb, uint32_t id, uint32_t acc_first) {
            mma_tf32_ss(d, A(pa), B(pb), id, acc_first);
            mma_tf32_ss(d, A(pa), B(C::Q + pb), id, 1u);
            mma_tf32_ss(d, A(T + pa), B(pb), id, 1u);
          };
          const uint32_t first = (st > 0 || kk > 0) ? 1u : 0u;
#pragma unroll
          for (int f = 0; f < G::nreal; ++f)
            if (C::own_real(f) == mi) prod3(tmem_base + f * BC, f, f, id_real, first);
#pragma unroll
          for (int k = 1; k <= G::ncomplex; ++k) {
            if (C::own_cplx(k) != mi) continue;
            const int pr = G::nreal + 2 * (k - 1);
            const int q = G::nreal + 3 * (k - 1);
            const uint32_t col = tmem_base + G::nreal * BC + (k - 1) * 2 * BC;
            prod3(col, pr, q + w1, id_cplx, first);
            prod3(col, pr + 1, q + w2, id_cplx, 1u);
          }
        }
        mma_commit(&op_empty[s]);
        if (++s == C::OP_STAGES) { s = 0; ph ^= 1; }
      }
      if (ok) mma_commit(acc_full);
      else raise_abort(abort_flag, p.err);
      mma_commit(&drain_bar[mi]);
      mbar_wait(&drain_bar[mi], 0, kDefaultWaitLimit);
      for (int i = 0; i < C::OP_STAGES; ++i)
        if (nst > i) mbar_wait(&op_empty[i], (uint32_t)(((nst - 1 - i) / C::OP_STAGES) & 1), kDefaultWaitLimit);
    }
    __syncwarp();
    grid_dep_launch();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

constexpr int MAX_WAVES = 4;

struct Plan {
  int BC, n_mt, n_nt, splits;   // splits: partial slots (CTAs per tile in a full pass)
  bool swap;
  int64_t chunk;                // tokens per CTA per pass
  int passes;
};

// M side: d, unless c pads less to a multiple of 128.  N side: tiles of BC
// channels (a multiple of 16, at most BC_MAX) that split it evenly.  Splits:
// the SMs per tile, times the waves (at most MAX_WAVES) that keep every chunk
// within CHUNK_MAX; passes: as many more as that still needs.
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
  if (N < 1) N = 1;
  // up to MAX_WAVES waves of CTAs in one launch, each split with a partial
  // slot of its own (the reduction sums them); passes only beyond that
  const int64_t per_wave = (int64_t)s * C::CHUNK_MAX;
  int64_t waves = (N + per_wave - 1) / per_wave;
  if (waves > MAX_WAVES) waves = MAX_WAVES;
  const int64_t sp = s * waves;               // splits per pass
  pl.passes = (int)((N + sp * C::CHUNK_MAX - 1) / (sp * C::CHUNK_MAX));
  const int64_t per_pass = (N + pl.passes - 1) / pl.passes;
  pl.chunk = ((per_pass + sp - 1) / sp + C::BKN - 1) / C::BKN * C::BKN;
  pl.splits = (int)((per_pass + pl.chunk - 1) / pl.chunk);
  return pl;
}

template <int T>
static size_t workspace_bytes(int64_t Cp, int64_t Dp, int sm_count) {
  const Plan pl = plan<T>(Cp, Dp, INT64_C(1) << 40, sm_count);
  return (size_t)pl.splits * ((size_t)T * Cp * Dp + Dp) * sizeof(float);
}

template <int T>
static cudaError_t launch_t(const Handle& h, const void* x, const void* gy, float* dW, float* db, int64_t N,
                            cudaStream_t st) {
  using C = Cfg<T>;
  const Plan pl = plan<T>(h.Cp, h.Dp, N, h.sm_count);
  const size_t need = (size_t)pl.splits * ((size_t)T * h.Cp * h.Dp + h.Dp) * sizeof(float);
  if (need > h.ws_bytes) return cudaErrorInvalidValue;
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
  const auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return cudaErrorNotSupported;
  // N-side box: the largest power of two (elements, at most 256) dividing BC * T
  int nb_box = 256;
  while ((pl.BC * T) % nb_box) nb_box >>= 1;
  CUtensorMap map_m, map_n;
  const void* srcs[2] = {pl.swap ? x : gy, pl.swap ? gy : x};
  const int64_t widths[2] = {(pl.swap ? h.Cp : h.Dp) * T, (pl.swap ? h.Dp : h.Cp) * T};
  const int boxes[2] = {C::MA_BOX, nb_box};
  CUtensorMap* maps[2] = {&map_m, &map_n};
  for (int i = 0; i < 2; ++i) {
    cuuint64_t dims[2] = {(cuuint64_t)widths[i], (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)widths[i] * 4};
    cuuint32_t box[2] = {(cuuint32_t)boxes[i], (cuuint32_t)C::BKN};
    cuuint32_t es[2] = {1, 1};
    if (enc(maps[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(srcs[i]), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  p.nb_box = nb_box;
  {
    const cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(tc32_dw_kernel<T>), C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  // pass i covers tokens [i * per_pass, (i + 1) * per_pass); each of its CTAs
  // has at least one token
  const int64_t per_pass = (int64_t)pl.splits * pl.chunk;
  for (int i = 0; i < pl.passes; ++i) {
    p.n_beg = (int64_t)i * per_pass;
    if (p.n_beg >= N) break;
    p.accumulate = i > 0 ? 1 : 0;
    const int64_t toks = (N - p.n_beg < per_pass) ? N - p.n_beg : per_pass;
    const int64_t zs = (toks + pl.chunk - 1) / pl.chunk;
    const unsigned grid = (unsigned)(pl.n_mt * pl.n_nt * zs);
    const cudaError_t e =
        launch_pdl(tc32_dw_kernel<T>, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st, map_m, map_n, p);
    if (e != cudaSuccess) return e;
    count_launches(1);
  }
  // partials are [N channel][M channel]: c-major over d when M = d
  return launch_dw_reduce(h, pl.splits, p.part, p.dbpart, dW, db, /*cd_layout=*/!pl.swap, st);
}

}  // namespace tc32dw

bool tc32_dw_supported(const Handle& h) { return tc32_supported(h) && h.T != 8; }

size_t tc32_dw_workspace_bytes(int T, int64_t Cp, int64_t Dp, int sm_count) {
  switch (T) {
    case 1: return tc32dw::workspace_bytes<1>(Cp, Dp, sm_count);
    case 2: return tc32dw::workspace_bytes<2>(Cp, Dp, sm_count);
    case 4: return tc32dw::workspace_bytes<4>(Cp, Dp, sm_count);
  }
  return 0;
}

cudaError_t launch_tc32_dw(const Handle& h, const void* x, const void* gy, float* dW, float* db, int64_t N,
                           cudaStream_t st) {
  if (!tc32_dw_supported(h)) return cudaErrorNotSupported;
  switch (h.T) {
    case 1: return tc32dw::launch_t<1>(h, x, gy, dW, db, N, st);
    case 2: return tc32dw::launch_t<2>(h, x, gy, dW, db, N, st);
    case 4: return tc32dw::launch_t<4>(h, x, gy, dW, db, N, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace eqlin
