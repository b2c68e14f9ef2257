// eqlin_tc_dw.cu -- tcgen05 kernel for the weight gradient dW and db.
//
// In the Fourier domain the weight gradient of every frequency k is a channel
// GEMM that reduces over tokens (derived from the layer's definition; the
// pages print no backward formula):
//
//   dW_hat_k[d, c] = sum_n G_k[n, d] * conj(X_k[n, c]),   G = DFT_t(gy), X = DFT_t(x)
//   dW[d, c, tau]  = IDFT_k(dW_hat)[tau]   (with the 1/T),   db[d] = sum_n G_0[n, d]
//
// The MMA's M side (128 rows of TMEM) takes d or c, whichever pads less to a
// multiple of 128; the other side is the N side, BC <= 128 channels.  For a
// complex frequency the two real outputs come from two block products of
// N = 2*BC columns, so p4 again needs six real GEMMs:
//   M = d:  [Re | Im] = Re G [Re X ; -Im X] + Im G [Im X ; Re X]
//           (B planes per complex frequency: Im X, Re X, -Im X)
//   M = c:  [Re | Im] = Re X [Re G ; Im G] + Im X [Im G ; -Re G]
//           (the transposed product conj(X)^T G; B planes: Re G, Im G, -Re G)
//
// Work unit of one CTA: 128 M channels x BC N channels x one contiguous chunk
// of tokens, in stages of 16 tokens.  Roles:
//   warp 16    (producer)  TMA: the stage's rows of the M-side input (gy or x)
//              for the 128 M channels and of the N-side input for the BC N
//              channels into a raw ring, and L2 prefetches of later stages
//   warps 0-15 (transform) two groups of eight warps: on alternate stages
//              (two stages in flight), or in the small-channel configuration
//              on the two halves of every stage's tokens.  In a group, warps
//              0-3 take one M channel each (A planes) and warps 4-7 one N
//              channel each (B planes): read the channel's T group values of
//              its tokens, 8 at a time, take the group DFT (packed token
//              pairs for T <= 4, FP32 for T = 3, 6, 8), keep sum_n G_0 in FP32
//              for db on the side that holds gy, and write K-major
//              (token-contiguous) operand planes.  After the
//              main loop the A warps of both groups read the accumulators out
//              of TMEM, each group half of the N columns
//   warp 17    allocates TMEM; the warp runs the MMA loop and one lane issues
// The raw ring (filled by TMA, freed once the transform has written the
// stage's operands from it) and the operand ring (filled by the transform,
// freed by the MMA commit) are separate, so loads run ahead of the tensor
// core by the whole raw ring.
// The per-chunk partial planes go to the handle's workspace as
// [chunk][plane][N channel][M channel]; a second kernel sums the chunks in a
// fixed order and applies the inverse DFT (deterministic, no atomics).  All
// waits are bounded as in eqlin_tc.cu.
#include <cudaTypedefs.h>

#include <type_traits>

#include "eqlin_internal.cuh"
#include "eqlin_packed.cuh"
#include "eqlin_ptx.cuh"
#include "eqlin_wait.cuh"

namespace eqlin {
namespace tcdw {

using namespace ptx;
using namespace waits;

// BCM caps the N-side tile width: 128 in general; 32 for small-channel shapes
// (an N side of at most 32 channels, as the EQ-Swin-T stage-1 layers have).
// Those take 32 tokens per stage for T <= 4 (two MMA K steps, 64-byte K-major
// rows with the 64B swizzle): each stage then carries twice the work for the same fixed
// cost of its barriers and commit, which is what bounds a stage whose MMAs
// are this small.
template <int T, int BCM = 128>
struct Cfg {
  using G = Group<T>;
  static constexpr int BM = 128;                          // M channels per tile (MMA M)
  static constexpr int BKN = BCM <= 32 && T <= 4 ? 32 : 16;   // tokens per stage (BKN / 16 MMA K steps)
  // ALT: the two transform groups take alternate stages (two stages in
  // flight); otherwise (the small-channel configuration, where that measured
  // slower) they split each stage's tokens
  static constexpr bool ALT = BCM > 32;
  static constexpr int NSB = ALT ? BKN / 8 : BKN / 16;    // 8-token blocks per transform thread and stage
  static constexpr int ROWB = BKN * 2;                    // K-major rows of 32 or 64 bytes, swizzled as wide
  // T * BC_MAX TMEM columns; tile widths are multiples of 16
  static constexpr int BC_MAX = (512 / T / 16 * 16) < BCM ? (512 / T / 16 * 16) : BCM;
  static constexpr int Q = G::nreal + 3 * G::ncomplex;    // B planes
  static constexpr int A_PLANE_BYTES = BM * ROWB;
  static constexpr int A_BYTES = T * A_PLANE_BYTES;
  static constexpr int B_BYTES = Q * BC_MAX * ROWB;       // plane stride is BC * ROWB at run time
  static constexpr int OP_BYTES = A_BYTES + B_BYTES;
  // raw tiles of a stage (TMA, row-major): M side [16 tokens][128 x T], N side [16 tokens][BC x T]
  static constexpr int MA_ROWB = BM * T * 2;
  static constexpr int NB_ROWB_MAX = BC_MAX * T * 2;
  static constexpr int RAW_BYTES = BKN * (MA_ROWB + NB_ROWB_MAX);
  // three operand slots where three raw slots still fit (the transform writes
  // stage k + 2 while the MMAs of k and k + 1 are in flight), four where four
  // raw slots still fit beside them, else two; the rest of 220 KB for raw
  // slots (memory latency)
  static constexpr int OP_STAGES = ALT ? ((220 * 1024 - 3 * OP_BYTES) / RAW_BYTES >= 4 ? 3 : 2)
                                   : (220 * 1024 - 4 * OP_BYTES) / RAW_BYTES >= 4 ? 4
                                   : (220 * 1024 - 3 * OP_BYTES) / RAW_BYTES >= 3 ? 3
                                                                                  : 2;
  static constexpr int RAW_FIT = (220 * 1024 - OP_STAGES * OP_BYTES) / RAW_BYTES;
  // with alternate stages the depth is even, so both uses of a raw slot k and
  // k + RAW_STAGES belong to the same group (an mbarrier parity wait cannot
  // tell a phase from the one two ahead)
  static constexpr int RAW_STAGES = (RAW_FIT > 6 ? 6 : RAW_FIT) & (ALT ? ~1 : ~0);
  static_assert(RAW_STAGES >= 2, "two raw stages must fit");
  // MMA issuers: an accumulator group (a real frequency's plane, or a
  // complex frequency's [Re | Im] block, two MMAs) belongs to one issuer; in
  // order, groups go to issuer 0 until it holds half of the stage's MMAs.
  static constexpr int NMMA = (T == 1) ? 1 : 2;
  static constexpr int MMAS = G::nreal + 2 * G::ncomplex;
  __host__ __device__ static constexpr int own_real(int f) { return (NMMA == 1 || 2 * f < MMAS) ? 0 : 1; }
  __host__ __device__ static constexpr int own_cplx(int k) {
    return (NMMA == 1 || 2 * (G::nreal + 2 * (k - 1)) < MMAS) ? 0 : 1;
  }
  static constexpr int NBAR = 2 * RAW_STAGES + 2 * OP_STAGES + 1 + NMMA;
  static constexpr int SMEM_BYTES = OP_STAGES * OP_BYTES + RAW_STAGES * RAW_BYTES + NBAR * 8 + 16 +
                                    BM * 4 + 1024;
  static constexpr int TMEM_COLS = T * BC_MAX <= 256 ? 256 : 512;
  static constexpr int TR_WARPS = 16;                     // two groups x (4 A + 4 B warps)
  static constexpr int STAGE_ARRIVALS = ALT ? 8 : 16;     // transform warps that fill one stage
  static constexpr int PRODUCER = TR_WARPS, MMA_WARP = TR_WARPS + 1;   // MMA warps MMA_WARP .. + NMMA - 1
  static constexpr int THREADS = (TR_WARPS + 1 + NMMA) * 32;
  static constexpr int PF_STAGES = 12;                    // L2 prefetch distance (stages)
  // M-side TMA box width (elements): a whole number of channels, at most 256
  static constexpr int MA_BOX = BM * T <= 256 ? BM * T : (T & (T - 1)) == 0 ? 256 : 192;
  static_assert((BM * T) % MA_BOX == 0 && MA_BOX % T == 0, "whole channels per box, whole boxes per tile");
  static constexpr int W = packed::Words<T>::n;
};

struct Params {
  int64_t N;
  int Cp, Dp;
  int mdim;               // M-side channels (Dp, or Cp when swapped)
  int BC;                 // N-side channels per tile (multiple of 16)
  int n_mt, n_nt;         // M tiles, N tiles
  int swap;               // 0: M = d (A from gy, B from x); 1: M = c (A from x, B from gy)
  int64_t chunk;          // tokens per split (multiple of BKN)
  int nb_box;             // N-side TMA box width (elements), divides BC * T
  float* part;            // [splits][T][N channels][M channels]
  float* dbpart;          // [splits][Dp]
  int* err;
  uint32_t wait_limit;
  uint32_t ab_fmt;
};

template <typename E>
__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  E* e = reinterpret_cast<E*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) e[i] = Elem<E>::from_f(f[i]);
  return u;
}

// Byte offset of the 16-byte chunk j (8 tokens) of row r in a K-major plane
// with ROWB-byte rows: 32B swizzle (chunk bit 0 XOR row bit 2) for 32-byte
// rows, 64B swizzle (chunk bits 0-1 XOR row bits 1-2) for 64-byte rows.
template <int ROWB>
__device__ __forceinline__ uint32_t kmajor_off(int r, int j) {
  if constexpr (ROWB == 32) return (uint32_t)(r * 32 + ((j ^ ((r >> 2) & 1)) << 4));
  else return (uint32_t)(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

template <int T, typename E, int BCM>
__global__ void __launch_bounds__(Cfg<T, BCM>::THREADS, 1)
tc_dw_kernel(const __grid_constant__ CUtensorMap map_m, const __grid_constant__ CUtensorMap map_n, Params p) {
  using C = Cfg<T, BCM>;
  using G = Group<T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* op_buf = smem;                                         // [OP_STAGES][A | B]
  uint8_t* raw_buf = op_buf + C::OP_STAGES * C::OP_BYTES;        // [RAW_STAGES][M side | N side]
  uint64_t* bars = reinterpret_cast<uint64_t*>(raw_buf + C::RAW_STAGES * C::RAW_BYTES);
  uint64_t* raw_full = bars;                          // TMA bytes
  uint64_t* raw_empty = raw_full + C::RAW_STAGES;     // the transform warps have read the slot
  uint64_t* op_full = raw_empty + C::RAW_STAGES;      // the transform warps have written the operands
  uint64_t* op_empty = op_full + C::OP_STAGES;        // MMA commit
  uint64_t* acc_full = op_empty + C::OP_STAGES;
  uint64_t* drain_bar = acc_full + 1;           // [NMMA]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + C::NMMA);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* db_half = reinterpret_cast<float*>(tmem_slot + 4);       // [BM] token group 1's db sums

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
  const int nb_rowb = BC * T * 2;                 // raw N-side row bytes of this tile
  const bool swap = p.swap != 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::RAW_STAGES; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], C::STAGE_ARRIVALS);
    }
    for (int i = 0; i < C::OP_STAGES; ++i) {
      mbar_init(&op_full[i], C::STAGE_ARRIVALS);
      mbar_init(&op_empty[i], C::NMMA);   // one commit per MMA issuer
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
  grid_dep_wait();   // the previous kernel's writes are visible from here on

  if (warp < C::TR_WARPS) {
    // --------------------------------------------------- transform warps
    const int grp = warp >> 3;                             // ALT: stages grp, grp + 2, ...; else tokens 8*NSB*grp ..
    const bool is_a = (warp & 7) < 4;
    const int r = (warp & 3) * 32 + lane;                  // operand row: M channel (A) or N channel (B)
    const bool active = is_a || r < BC;
    // the side that holds gy also sums G_0 for db: A when M = d, B when M = c
    const bool sums_db = is_a != swap;
    // this thread's channel in the raw tile rows
    const uint32_t raw_col = is_a ? (uint32_t)((r / (C::MA_BOX / T)) * C::BKN * C::MA_BOX * 2 +
                                               (r % (C::MA_BOX / T)) * T * 2)
                                  : (uint32_t)((r * T / p.nb_box) * C::BKN * p.nb_box * 2 +
                                               ((r * T) % p.nb_box) * 2);
    const uint32_t raw_rowb = is_a ? (uint32_t)(C::MA_BOX * 2) : (uint32_t)(p.nb_box * 2);
    const uint32_t raw_base =
        (is_a ? 0u : (uint32_t)(C::BKN * C::MA_ROWB)) + raw_col + (C::ALT ? 0 : grp * C::NSB * 8 * raw_rowb);
    float dbacc = 0.f;
    constexpr int STEP = C::ALT ? 2 : 1;                   // stages between a group's turns
    int rs = C::ALT ? grp % C::RAW_STAGES : 0, os = C::ALT ? grp % C::OP_STAGES : 0;
    uint32_t rph = 0, oph = 0;
    bool ok = true;
    for (int st = C::ALT ? grp : 0; st < nst; st += STEP) {
      if (!wwait_all(&raw_full[rs], rph, limit, abort_flag, p.err, site(K_DW, 1, 1), (uint32_t)st)) { ok = false; break; }
      // the operand slot must have been consumed by the MMAs issued from it
      if (!wwait(&op_empty[os], oph ^ 1, limit, abort_flag, lane, p.err, site(K_DW, 1, 4), (uint32_t)st)) { ok = false; break; }
      uint8_t* a_st = op_buf + os * C::OP_BYTES;
      uint8_t* b_st = a_st + C::A_BYTES;
#pragma unroll
      for (int sb = 0; sb < C::NSB; ++sb) {
        uint32_t Pw[T][4];
        uint32_t wv[8][C::W];
        const uint8_t* raw = raw_buf + rs * C::RAW_BYTES + raw_base + sb * 8 * raw_rowb;
        if (active && (T == 1 || T == 2 || T == 4 || T == 8)) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint8_t* src = raw + j * raw_rowb;
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
        }
        if (!active) continue;
        if constexpr (T == 1 || T == 2 || T == 4) {
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
            uint32_t P[T];
            packed::dft_pair<T, E>(wv[2 * pr], wv[2 * pr + 1], P);
#pragma unroll
            for (int q = 0; q < T; ++q) Pw[q][pr] = P[q];
            if (sums_db) {
              const float2 f = packed::Pair<E>::to_f2(P[0]);
              dbacc += f.x + f.y;
            }
          }
        } else {
          // T = 3, 6, 8: FP32 butterflies (sqrt(3)/2 or sqrt(2)/2 twiddles), one
          // rounding per value; for T = 3, 6 (6 or 12 bytes per channel) the
          // elements are read one by one
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
            float Pa[T], Pb[T], va[T], vb[T];
            const E* ea = T == 8 ? reinterpret_cast<const E*>(wv[2 * pr])
                                 : reinterpret_cast<const E*>(raw + (2 * pr) * raw_rowb);
            const E* eb = T == 8 ? reinterpret_cast<const E*>(wv[2 * pr + 1])
                                 : reinterpret_cast<const E*>(raw + (2 * pr + 1) * raw_rowb);
#pragma unroll
            for (int t = 0; t < T; ++t) { va[t] = Elem<E>::to_f(ea[t]); vb[t] = Elem<E>::to_f(eb[t]); }
            G::dft(va, Pa);
            G::dft(vb, Pb);
            if (sums_db) dbacc += Pa[0] + Pb[0];
#pragma unroll
            for (int q = 0; q < T; ++q) {
              E two[2] = {Elem<E>::from_f(Pa[q]), Elem<E>::from_f(Pb[q])};
              Pw[q][pr] = *reinterpret_cast<const uint32_t*>(two);
            }
          }
        }
        const uint32_t off = kmajor_off<C::ROWB>(r, (C::ALT ? 0 : grp * C::NSB) + sb);
        if (is_a) {
#pragma unroll
          for (int q = 0; q < T; ++q)
            *reinterpret_cast<uint4*>(a_st + q * C::A_PLANE_BYTES + off) = make_uint4(Pw[q][0], Pw[q][1], Pw[q][2], Pw[q][3]);
        } else {
#pragma unroll
          for (int f = 0; f < G::nreal; ++f)
            *reinterpret_cast<uint4*>(b_st + f * b_plane + off) = make_uint4(Pw[f][0], Pw[f][1], Pw[f][2], Pw[f][3]);
#pragma unroll
          for (int k = 1; k <= G::ncomplex; ++k) {
            const int pr = G::nreal + 2 * (k - 1);
            const int q = G::nreal + 3 * (k - 1);
            // M = d: (Im X, Re X, -Im X);  M = c: (Re G, Im G, -Re G)
            const uint32_t* u0 = swap ? Pw[pr] : Pw[pr + 1];
            const uint32_t* u1 = swap ? Pw[pr + 1] : Pw[pr];
            *reinterpret_cast<uint4*>(b_st + (q + 0) * b_plane + off) = make_uint4(u0[0], u0[1], u0[2], u0[3]);
            *reinterpret_cast<uint4*>(b_st + (q + 1) * b_plane + off) = make_uint4(u1[0], u1[1], u1[2], u1[3]);
            *reinterpret_cast<uint4*>(b_st + (q + 2) * b_plane + off) =
                make_uint4(packed::neg2(u0[0]), packed::neg2(u0[1]), packed::neg2(u0[2]), packed::neg2(u0[3]));
          }
        }
      }
      // one generic->async proxy fence orders both this stage's reads of the
      // raw slot (before its TMA refill) and its operand writes (before the MMA)
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&raw_empty[rs]);
        mbar_arrive(&op_full[os]);
      }
      rs += STEP;
      if (rs >= C::RAW_STAGES) { rs -= C::RAW_STAGES; rph ^= 1; }
      os += STEP;
      if (os >= C::OP_STAGES) { os -= C::OP_STAGES; oph ^= 1; }
    }
    if (!ok) raise_abort(abort_flag, p.err);
    // The next kernel (the split reduction) may be scheduled once every role
    // of every CTA is past its main loop.  Triggered any earlier, its CTAs
    // would wait on these SMs through the whole loop, beside the transform
    // warps whose issue slots bound it.
    grid_dep_launch();

    // db: the side that sums G_0 writes its channels' sums; group 1 hands
    // its sums to group 0 through shared memory.  Only the tiles of the other
    // side's first tile write, so each d is written once per chunk.
    const bool db_tile = swap ? (mt == 0) : (nt == 0);
    if (sums_db && db_tile) {
      const int bar_id = is_a ? 1 : 2;
      named_bar_sync(bar_id, 256);
      if (grp == 1) db_half[r] = dbacc;
      named_bar_sync(bar_id, 256);
      const int d = (swap ? n0 : m0) + r;
      if (grp == 0 && active && d < p.Dp) p.dbpart[(int64_t)z * p.Dp + d] = dbacc + db_half[r];
    }

    if (is_a) {
      // ------------------------------------------------------- epilogue
      // The A warps of both token groups (same TMEM lane quarter, same M
      // channel).  Partial planes [z][T][N channel][M channel]: a warp stores
      // 32 consecutive M channels of one N channel; group g takes the N
      // columns [g * BC/2, (g+1) * BC/2).
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
#pragma unroll
            for (int q = 0; q < T; ++q)
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int n = n0 + cc + i;
                if (n < ndim) base[q * plane + (int64_t)n * p.mdim] = __uint_as_float(rg[q][i]);
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
          tma_load_2d(dst + b * C::BKN * C::MA_BOX * 2, &map_m, m0 * T + b * C::MA_BOX, n, &raw_full[s]);
        dst += C::BKN * C::MA_ROWB;
        for (int b = 0; b < BC * T / p.nb_box; ++b)
          tma_load_2d(dst + b * C::BKN * p.nb_box * 2, &map_n, n0 * T + b * p.nb_box, n, &raw_full[s]);
        ++n_raw;
        if (++s == C::RAW_STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      // every issued TMA copy must land before the CTA exits
      for (int i = 0; i < C::RAW_STAGES; ++i)
        if (n_raw > i)
          mbar_wait(&raw_full[i], (uint32_t)(((n_raw - 1 - i) / C::RAW_STAGES) & 1), kDefaultWaitLimit);
    }
    __syncwarp();
    grid_dep_launch();
  } else {
    // -------------------------------------------------------------- MMA
    // Lane 0 of MMA warp mi issues the MMAs of the accumulator groups it
    // owns and commits them; the operand slot's and the accumulator's
    // barriers take one commit per issuer.
    const int mi = warp - C::MMA_WARP;
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      const uint32_t id_real = idesc_f16(p.ab_fmt, (uint32_t)BC);
      const uint32_t id_cplx = idesc_f16(p.ab_fmt, (uint32_t)(2 * BC));
      // descriptors of slot 0, advanced by byte offset >> 4 (start-address field)
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
        for (int kk = 0; kk < C::BKN / 16; ++kk) {
          // K step kk: 16 tokens = 32 bytes further along the swizzled rows
          const uint64_t ka = a_d + (uint64_t)(kk * 2), kb = b_d + (uint64_t)(kk * 2);
          const uint32_t first = (st > 0 || kk > 0) ? 1u : 0u;
#pragma unroll
          for (int f = 0; f < G::nreal; ++f)
            if (C::own_real(f) == mi)
              mma_f16_ss(tmem_base + f * BC, ka + ((f * C::A_PLANE_BYTES) >> 4), kb + f * bp, id_real, first);
#pragma unroll
          for (int k = 1; k <= G::ncomplex; ++k) {
            if (C::own_cplx(k) != mi) continue;
            const int pr = G::nreal + 2 * (k - 1);
            const int q = G::nreal + 3 * (k - 1);
            const uint32_t col = tmem_base + G::nreal * BC + (k - 1) * 2 * BC;
            // [Re | Im] += (Re plane of A) [first window] + (Im plane of A) [second window]
            mma_f16_ss(col, ka + ((pr * C::A_PLANE_BYTES) >> 4), kb + (q + w1) * bp, id_cplx, first);
            mma_f16_ss(col, ka + (((pr + 1) * C::A_PLANE_BYTES) >> 4), kb + (q + w2) * bp, id_cplx, 1u);
          }
        }
        mma_commit(&op_empty[s]);
        if (++s == C::OP_STAGES) { s = 0; ph ^= 1; }
      }
      if (ok) mma_commit(acc_full);
      else raise_abort(abort_flag, p.err);
      mma_commit(&drain_bar[mi]);
      mbar_wait(&drain_bar[mi], 0, kDefaultWaitLimit);
      // The last commit of each operand slot fires on the same completion as
      // the drain's, and nothing else waits for it: an arrival that lands
      // after the CTA has left would write into the shared memory of whatever
      // the SM runs next.  (On an aborted run, with fewer commits, the
      // wall-time cap ends the wait.)
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

struct Plan {
  int BC, n_mt, n_nt, splits;
  bool swap;
  int64_t chunk;
};

// M side: d, unless c pads less to a multiple of 128.  N side: tiles of BC
// channels (a multiple of 16, at most BC_MAX) that split it evenly.
template <int T, int BCM = 128>
static Plan plan(int64_t Cp, int64_t Dp, int64_t N, int sm_count) {
  using C = Cfg<T, BCM>;
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

template <int T, typename E, int BCM>
static cudaError_t launch_b(const Handle& h, const Plan& pl, const void* x, const void* gy, float* dW, float* db,
                            int64_t N, cudaStream_t st) {
  using C = Cfg<T, BCM>;
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
  p.ab_fmt = std::is_same<E, __half>::value ? 0u : 1u;
  const auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt = std::is_same<E, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // N-side box: whole channels, at most 256 elements, a multiple of 16 bytes,
  // dividing BC * T: the largest power of two for T | 8; for T = 3, 6 the
  // channels of the largest divisor of BC that fits
  int nb_box = 256;
  if ((T & (T - 1)) == 0) {
    while ((pl.BC * T) % nb_box) nb_box >>= 1;
  } else {
    int d = pl.BC;
    while (d > 1 && (pl.BC % d || d * T > 256 || (d * T * 2) % 16)) --d;
    nb_box = d * T;
  }
  CUtensorMap map_m, map_n;
  const void* srcs[2] = {pl.swap ? x : gy, pl.swap ? gy : x};
  const int64_t widths[2] = {(pl.swap ? h.Cp : h.Dp) * T, (pl.swap ? h.Dp : h.Cp) * T};
  const int boxes[2] = {C::MA_BOX, nb_box};
  CUtensorMap* maps[2] = {&map_m, &map_n};
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
  p.nb_box = nb_box;
  {
    const cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(tc_dw_kernel<T, E, BCM>), C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  const unsigned grid = (unsigned)(pl.n_mt * pl.n_nt * pl.splits);
  cudaError_t e = launch_pdl(tc_dw_kernel<T, E, BCM>, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st, map_m, map_n, p);
  if (e != cudaSuccess) return e;
  count_launches(1);
  // partials are [N channel][M channel]: c-major over d when M = d
  return launch_dw_reduce(h, pl.splits, p.part, p.dbpart, dW, db, /*cd_layout=*/!pl.swap, st);
}

// The small-channel configuration serves N-side tiles of at most 32 channels;
// the plan (tile widths, splits) is the same for both.
template <int T, typename E>
static cudaError_t launch_t(const Handle& h, const void* x, const void* gy, float* dW, float* db,
                            int64_t N, cudaStream_t st) {
  const Plan pl = plan<T>(h.Cp, h.Dp, N, h.sm_count);
  if (pl.BC <= Cfg<T, 32>::BC_MAX && Cfg<T, 32>::BC_MAX < Cfg<T>::BC_MAX)
    return launch_b<T, E, 32>(h, plan<T, 32>(h.Cp, h.Dp, N, h.sm_count), x, gy, dW, db, N, st);
  return launch_b<T, E, 128>(h, pl, x, gy, dW, db, N, st);
}

template <typename E>
static cudaError_t launch_e(const Handle& h, const void* x, const void* gy, float* dW, float* db,
                            int64_t N, cudaStream_t st) {
  switch (h.T) {
    case 1: return launch_t<1, E>(h, x, gy, dW, db, N, st);
    case 2: return launch_t<2, E>(h, x, gy, dW, db, N, st);
    case 3: return launch_t<3, E>(h, x, gy, dW, db, N, st);
    case 4: return launch_t<4, E>(h, x, gy, dW, db, N, st);
    case 6: return launch_t<6, E>(h, x, gy, dW, db, N, st);
    case 8: return launch_t<8, E>(h, x, gy, dW, db, N, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tcdw

bool tc_dw_supported(const Handle& h) {
  return h.group == EQLIN_GROUP_CYCLIC && (h.dtype == EQLIN_F16 || h.dtype == EQLIN_BF16) &&
         (h.T == 1 || h.T == 2 || h.T == 3 || h.T == 4 || h.T == 6 || h.T == 8);
}

size_t tc_dw_workspace_bytes(int T, int64_t Cp, int64_t Dp, int sm_count) {
  switch (T) {
    case 1: return tcdw::workspace_bytes<1>(Cp, Dp, sm_count);
    case 2: return tcdw::workspace_bytes<2>(Cp, Dp, sm_count);
    case 3: return tcdw::workspace_bytes<3>(Cp, Dp, sm_count);
    case 4: return tcdw::workspace_bytes<4>(Cp, Dp, sm_count);
    case 6: return tcdw::workspace_bytes<6>(Cp, Dp, sm_count);
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
