// eqlin_tc32.cu -- FP32 forward and input gradient on the tensor cores,
// 3xTF32 (tcgen05 kind::tf32, f32 accumulation in TMEM).
//
// A TF32 operand keeps 11 significant bits of an f32 value.  Each value v
// (the group DFT of the input, and each Fourier weight) is split into
// hi = tf32(v) and lo = tf32(v - hi), and every real product of the
// frequency-domain GEMMs is taken as hi*hi + hi*lo + lo*hi: three kind::tf32
// MMAs into the same accumulator.  The term left out, lo*lo, and the rounding
// of lo are each about 2^-22 of |a*b|, so a product carries about 21
// significant bits instead of 11 -- an FP32-level result at three TF32 MMAs
// per product ("Flash EQ-Linear", technical summary, section "Implementacao":
// forward and backward kernels in FP32 as well as FP16).
//
// Same structure as the f16/bf16 kernel (eqlin_tc.cu): one persistent CTA per
// SM over output tiles of 128 tokens x BO output channels (all T group
// positions); per K stage of 8 input channels (one kind::tf32 K step):
//
//   raw producer     (8)    TMA: the stage's raw f32 input tile [128 tokens x
//                    8*T elements] into the raw ring, L2 prefetches ahead
//   weight producer  (9)    one bulk copy of the stage's 2Q weight planes (hi
//                    then lo, stored pre-swizzled per stage)
//   transform warps  (0-7)  two groups of four warps on alternate stages; one
//                    thread per (input channel, 8 tokens): the channel's T
//                    group values of each token, the group DFT in FP32, the
//                    hi/lo split, and 2T frequency planes written as
//                    token-contiguous (MN-major) operands in the 128-byte
//                    swizzle with 32-byte atoms: an atom is 4 channels x 32
//                    tokens, eight atoms per plane.  T = 8 (one operand slot):
//                    all eight warps on every stage, 4 tokens per thread
//   MMA warps        (10, 11) lane 0 of each issues, for the accumulators it
//                    owns, three MMAs per real product: real frequency f one
//                    M=128, N=BO product; complex frequency k the block
//                    products [Re Y | Im Y] = Re X [Re W ; Im W] + Im X
//                    [-Im W ; Re W], N=2*BO each
//   epilogue warps   (12-19) tcgen05.ld of the frequency planes, inverse DFT
//                    (scales carried by the weight planes), bias, f32 rows of
//                    32 outputs (32/T channels) into a 128B-swizzled staging
//                    tile, TMA store
//
// Tiles are as wide as fit (BO = 256 for T = 1, 2; 128 for T = 4; 32 for
// T = 8): an N = 128 TF32 MMA already reads its operands at the SM's
// shared-memory rate, so narrower MMAs make the stage bandwidth-bound.
//
// Every mbarrier wait is bounded; a wait that runs out records a timeout in
// the handle's error word, raises the CTA's abort flag, and the kernel drains
// its in-flight copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include "eqlin_internal.cuh"
#include "eqlin_ptx.cuh"
#include "eqlin_wait.cuh"

namespace eqlin {
namespace tc32 {

using namespace ptx;
using namespace waits;

template <int T, int BO_>
struct Cfg {
  using G = Group<T>;
  static_assert(T == 1 || T == 2 || T == 4 || T == 8, "3xTF32 tiles for T in {1, 2, 4, 8}");
  // SPLIT (T = 8): the 16 hi/lo A planes of a stage leave room for one
  // operand slot, so all eight transform warps work on every stage (four
  // tokens per thread) instead of two groups on alternate stages; with one
  // slot, alternating groups would wait on phases an mbarrier parity cannot
  // tell apart.
  static constexpr bool SPLIT = (T == 8);
  static constexpr int TOK = SPLIT ? 4 : 8;            // tokens per transform thread and stage
  static constexpr int BM = 128;                       // tokens per tile (MMA M)
  static constexpr int BK = TC32_BK;                   // input channels per stage (one MMA K step)
  static constexpr int BO = BO_;
  static constexpr int ACC_COLS = T * BO;              // f32 accumulator columns of a tile
  static_assert(ACC_COLS <= 512 && BO <= 256 && (G::ncomplex == 0 || 2 * BO <= 256), "TMEM columns, MMA N");
  static constexpr int NACC = (ACC_COLS * 2 <= 512) ? 2 : 1;
  static constexpr int TMEM_COLS = NACC * ACC_COLS <= 256 ? 256 : 512;
  static constexpr int Q = G::nreal + 3 * G::ncomplex; // weight planes per stage and part (hi / lo)
  // raw input tile of a stage: 128 tokens x (8 channels x T) f32, row-major (TMA)
  static constexpr int RAW_ROWB = BK * T * 4;
  static constexpr int RAW_BYTES = BM * RAW_ROWB;
  // A: MN-major, 128-byte swizzle with 32-byte atomicity (the layout MN-major
  // TF32 operands take): a 128-byte row is 32 tokens of one channel, an atom
  // 4 channel rows (512 B) in which 32-byte chunk j of row r sits at j ^ r;
  // the two 4-channel K groups of a stage SBO apart, the 4 blocks of 32
  // tokens LBO apart
  static constexpr int A_LBO = 1024;
  static constexpr int A_SBO = 512;
  static constexpr int A_PLANE_BYTES = BM * BK * 4;    // 4 KB
  static constexpr int A_BYTES = 2 * T * A_PLANE_BYTES;   // hi planes 0..T-1, lo planes T..2T-1
  // B: K-major, 32-byte rows (8 channels), 32B swizzle
  static constexpr int B_ROWB = BK * 4;
  static constexpr int B_PLANE_BYTES = BO * B_ROWB;
  static constexpr int B_BYTES = 2 * Q * B_PLANE_BYTES;   // hi planes 0..Q-1, lo planes Q..2Q-1
  // output: f32 rows of 32 elements (128 bytes, 128B swizzle) per TMA store
  static constexpr int OUT_EL = 32;
  static constexpr int OUT_ROWB = OUT_EL * 4;
  static constexpr int OUT_TILE_BYTES = BM * OUT_ROWB;
  // ring depths within the shared-memory budget: three operand slots where
  // four raw slots still fit beside them, else two; two staging tiles per
  // epilogue half where four raw slots still fit, else one; the rest raw
  // slots (even, as in the f16/bf16 kernel: both uses of a slot belong to
  // the same transform group)
  static constexpr int BIAS_BYTES = 2 * BO * 4;        // per epilogue half, the tile's bias (FP32)
  static constexpr int BUDGET = 225 * 1024 - BIAS_BYTES;
  static constexpr int AB_ST =
      SPLIT ? 1 : (BUDGET - 2 * OUT_TILE_BYTES - 3 * (A_BYTES + B_BYTES)) / RAW_BYTES >= 4 ? 3 : 2;
  static constexpr int NSTG = (BUDGET - 4 * OUT_TILE_BYTES - AB_ST * (A_BYTES + B_BYTES)) / RAW_BYTES >= 4 ? 2 : 1;
  static constexpr int STAGING = 2 * NSTG * OUT_TILE_BYTES;
  static constexpr int RAW_FIT = (BUDGET - STAGING - AB_ST * (A_BYTES + B_BYTES)) / RAW_BYTES;
  static constexpr int RAW_ST = (RAW_FIT > 8 ? 8 : RAW_FIT) & (SPLIT ? ~0 : ~1);
  static_assert(RAW_ST >= 2 && (SPLIT || AB_ST >= 2), "two slots per ring (the transform groups take alternate stages)");
  static_assert((A_BYTES + B_BYTES) % 1024 == 0 && RAW_BYTES % 1024 == 0, "1 KB alignment of the swizzled tiles");
  static constexpr int NMMA = (T == 1) ? 1 : 2;
  static constexpr int MMAS = G::nreal + 2 * G::ncomplex;          // block products per stage
  __host__ __device__ static constexpr int own_real(int f) { return (NMMA == 1 || 2 * f < MMAS) ? 0 : 1; }
  __host__ __device__ static constexpr int own_cplx(int k) {
    return NMMA == 1 ? 0 : (2 * (G::nreal + 2 * (k - 1)) < MMAS) ? 0 : 1;
  }
  static constexpr int NBAR = 2 * RAW_ST + 2 * AB_ST + 2 * NACC + NMMA;
  static constexpr int SMEM_BYTES = RAW_ST * RAW_BYTES + AB_ST * (A_BYTES + B_BYTES) + STAGING + BIAS_BYTES +
                                    NBAR * 8 + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
  static constexpr int CH = OUT_EL / T;                // output channels per store chunk
  static constexpr int SUBCH = CH < 8 ? CH : 8;        // channels per inverse-DFT batch
  static_assert(CH % SUBCH == 0 && (SUBCH * T) % 4 == 0, "whole 16-byte output chunks per batch");
  static constexpr int NCHUNK = BO / CH;
  static_assert(NCHUNK % 2 == 0, "chunks alternate between the two epilogue halves");
  static constexpr int TR_WARPS = 8;
  static constexpr int GRP_WARPS = SPLIT ? TR_WARPS : TR_WARPS / 2;   // transform warps that fill one stage
  static constexpr int RAW_PRODUCER = TR_WARPS, B_PRODUCER = TR_WARPS + 1;
  static constexpr int MMA_WARP = TR_WARPS + 2, EPI0 = MMA_WARP + NMMA;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = (EPI0 + EPI_WARPS) * 32;
  static constexpr int PF_STAGES = 12;                 // L2 prefetch distance of the input tiles
};

struct Params {
  int64_t N;
  int K;           // input channels per group element (C' forward, D' for dx)
  int O;           // output channels per group element
  int n_otiles;
  int n_tb;
  int64_t n_tiles;
  const void* wtiles;  // hi/lo weight tiles of this pass
  const float* bias;   // nullptr: none
  int* err;
  uint32_t wait_limit;
};

// 32 lanes x 32 bits, 4 consecutive columns per thread (the T = 8 epilogue's
// 4-channel chunks).
__device__ __forceinline__ void tmem_ld_32x32b_x4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}

template <int N_>
__device__ __forceinline__ void load_group(const uint8_t* src, float (&v)[N_]) {
  static_assert(N_ == 1 || N_ == 2 || N_ == 4 || N_ == 8, "a channel's T values");
  if constexpr (N_ == 8) {
    const float4 a = *reinterpret_cast<const float4*>(src), b = *reinterpret_cast<const float4*>(src + 16);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else if constexpr (N_ == 4) {
    const float4 u = *reinterpret_cast<const float4*>(src);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  } else if constexpr (N_ == 2) {
    const float2 u = *reinterpret_cast<const float2*>(src);
    v[0] = u.x; v[1] = u.y;
  } else {
    v[0] = *reinterpret_cast<const float*>(src);
  }
}

template <int T, int BO>
__global__ void __launch_bounds__(Cfg<T, BO>::THREADS, 1)
tc32_apply_kernel(const __grid_constant__ CUtensorMap map_in, const __grid_constant__ CUtensorMap map_out, Params p) {
  using C = Cfg<T, BO>;
  using G = Group<T>;
  grid_dep_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* a_buf = smem;                                   // [AB_ST][2T planes]
  uint8_t* b_buf = a_buf + C::AB_ST * C::A_BYTES;          // [AB_ST][2Q planes]
  uint8_t* raw_buf = b_buf + C::AB_ST * C::B_BYTES;        // [RAW_ST][raw tile]
  uint8_t* o_buf = raw_buf + C::RAW_ST * C::RAW_BYTES;     // [2 halves][NSTG] staging tiles
  float* s_bias = reinterpret_cast<float*>(o_buf + C::STAGING);
  uint64_t* bars = reinterpret_cast<uint64_t*>(o_buf + C::STAGING + C::BIAS_BYTES);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + C::RAW_ST;
  uint64_t* ab_full = raw_empty + C::RAW_ST;   // A planes written (4 warps) + weight bytes landed
  uint64_t* ab_empty = ab_full + C::AB_ST;     // MMA commits
  uint64_t* acc_full = ab_empty + C::AB_ST;
  uint64_t* acc_empty = acc_full + C::NACC;
  uint64_t* drain_bar = acc_empty + C::NACC;   // [NMMA]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + C::NMMA);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t limit = p.wait_limit;
  const int nk = (p.K + C::BK - 1) / C::BK;
  // tile t: (token block t / n_otiles, output tile t % n_otiles), so the
  // output tiles of a token block run side by side and share its input in L2
  const int64_t my_tiles = p.n_tiles > blockIdx.x ? (p.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::RAW_ST; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], C::GRP_WARPS);
    }
    for (int i = 0; i < C::AB_ST; ++i) {
      mbar_init(&ab_full[i], C::GRP_WARPS + 1);
      mbar_init(&ab_empty[i], C::NMMA);
    }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(&acc_full[i], C::NMMA);
      mbar_init(&acc_empty[i], C::EPI_WARPS * 32);
    }
    for (int i = 0; i < C::NMMA; ++i) mbar_init(&drain_bar[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&map_in);
    prefetch_tensormap(&map_out);
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
    // ----------------------------------------------------- transform warps
    // Thread: channel c of the stage (8 per stage) and 8 consecutive tokens,
    // one 32-byte chunk of a plane row (SPLIT: 4 tokens, a 16-byte half).
    const int grp = C::SPLIT ? 0 : warp / C::GRP_WARPS;
    const int c = lane & 7;
    const int m = C::SPLIT ? warp * 16 + 4 * (lane >> 3) : (warp % C::GRP_WARPS) * 32 + 8 * (lane >> 3);
    const uint32_t a_off =
        (uint32_t)((m >> 5) * C::A_LBO + (c >> 2) * C::A_SBO + (c & 3) * 128 + ((((m & 31) >> 3) ^ (c & 3)) << 5) +
                   (C::SPLIT ? ((m >> 2) & 1) * 16 : 0));
    const uint32_t raw_off = (uint32_t)(m * C::RAW_ROWB + c * T * 4);
    constexpr int STEP = C::SPLIT ? 1 : 2;               // stages between a thread's turns
    int rs = grp % C::RAW_ST, as = grp % C::AB_ST;
    uint32_t rph = 0, aph = 0;
    bool ok = true;
    for (int64_t it = grp; it < my_tiles * nk; it += STEP) {
      if (!wwait_all(&raw_full[rs], rph, limit, abort_flag, p.err, site(K_APPLY, 1, 1), (uint32_t)it)) { ok = false; break; }
      const uint8_t* raw = raw_buf + rs * C::RAW_BYTES + raw_off;
      float v[C::TOK][T];
#pragma unroll
      for (int j = 0; j < C::TOK; ++j) load_group<T>(raw + j * C::RAW_ROWB, v[j]);
      // generic reads of the slot ordered before its next TMA write
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&raw_empty[rs]);
      // group DFT in FP32, then hi = tf32(P), lo = tf32(P - hi)
      uint32_t hi[T][C::TOK], lo[T][C::TOK];
#pragma unroll
      for (int j = 0; j < C::TOK; ++j) {
        float P[T];
        G::dft(v[j], P);
#pragma unroll
        for (int q = 0; q < T; ++q) {
          hi[q][j] = f32_to_tf32(P[q]);
          lo[q][j] = f32_to_tf32(P[q] - __uint_as_float(hi[q][j]));
        }
      }
      rs += STEP;
      if (rs >= C::RAW_ST) { rs -= C::RAW_ST; rph ^= 1; }
      if (!wwait(&ab_empty[as], aph ^ 1, limit, abort_flag, lane, p.err, site(K_APPLY, 1, 4), (uint32_t)it)) { ok = false; break; }
      uint8_t* a_st = a_buf + as * C::A_BYTES;
      if constexpr (C::SPLIT) {
#pragma unroll
        for (int q = 0; q < T; ++q) {
          *reinterpret_cast<uint4*>(a_st + q * C::A_PLANE_BYTES + a_off) =
              make_uint4(hi[q][0], hi[q][1], hi[q][2], hi[q][3]);
          *reinterpret_cast<uint4*>(a_st + (T + q) * C::A_PLANE_BYTES + a_off) =
              make_uint4(lo[q][0], lo[q][1], lo[q][2], lo[q][3]);
        }
      } else {
        // The 16-byte halves of the 32-byte chunk go in opposite orders for
        // channels c and c + 4: one store instruction then covers all eight
        // 16-byte bank groups of a 128-byte row (the two K groups of a stage
        // sit 512 bytes apart, on the same banks), four wavefronts per warp.
        const bool swap_halves = (c >> 2) != 0;
        auto half = [&](const uint32_t (&w)[8], int b) {
          return make_uint4(w[4 * b], w[4 * b + 1], w[4 * b + 2], w[4 * b + 3]);
        };
#pragma unroll
        for (int q = 0; q < T; ++q) {
          uint8_t* ph = a_st + q * C::A_PLANE_BYTES + a_off;
          uint8_t* pl = a_st + (T + q) * C::A_PLANE_BYTES + a_off;
          const uint4 h0 = half(hi[q], 0), h1 = half(hi[q], 1), l0 = half(lo[q], 0), l1 = half(lo[q], 1);
          *reinterpret_cast<uint4*>(ph + (swap_halves ? 16 : 0)) = swap_halves ? h1 : h0;
          *reinterpret_cast<uint4*>(pl + (swap_halves ? 16 : 0)) = swap_halves ? l1 : l0;
          *reinterpret_cast<uint4*>(ph + (swap_halves ? 0 : 16)) = swap_halves ? h0 : h1;
          *reinterpret_cast<uint4*>(pl + (swap_halves ? 0 : 16)) = swap_halves ? l0 : l1;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ab_full[as]);
      as += STEP;
      if (as >= C::AB_ST) { as -= C::AB_ST; aph ^= 1; }
    }
    if (!ok) raise_abort(abort_flag, p.err);
  } else if (warp == C::RAW_PRODUCER) {
    // -------------------------------------------------------- raw producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t n_raw = 0;
      bool ok = true;
      int64_t pf_ti = 0;
      int pf_kb = 0;
      auto prefetch_next = [&]() {
        if (pf_ti >= my_tiles) return;
        const int64_t tile = blockIdx.x + pf_ti * gridDim.x;
        tma_prefetch_2d(&map_in, pf_kb * C::BK * T, (int)(tile / p.n_otiles) * C::BM);
        if (++pf_kb == nk) { pf_kb = 0; ++pf_ti; }
      };
      for (int i = 0; i < C::PF_STAGES; ++i) prefetch_next();
      for (int64_t ti = 0; ti < my_tiles && ok; ++ti) {
        const int64_t tile = blockIdx.x + ti * gridDim.x;
        const int m0 = (int)(tile / p.n_otiles) * C::BM;
        for (int kb = 0; kb < nk; ++kb) {
          prefetch_next();
          if (!bwait(&raw_empty[s], ph ^ 1, limit, abort_flag, p.err, site(K_APPLY, 2, 2), (uint32_t)n_raw)) { ok = false; break; }
          mbar_arrive_expect_tx(&raw_full[s], C::RAW_BYTES);
          tma_load_2d(raw_buf + s * C::RAW_BYTES, &map_in, kb * C::BK * T, m0, &raw_full[s]);
          ++n_raw;
          if (++s == C::RAW_ST) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      for (int i = 0; i < C::RAW_ST; ++i)
        if (n_raw > i) mbar_wait(&raw_full[i], (uint32_t)(((n_raw - 1 - i) / C::RAW_ST) & 1), kDefaultWaitLimit);
    }
  } else if (warp == C::B_PRODUCER) {
    // ----------------------------------------------------- weight producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t n_b = 0;
      bool ok = true;
      for (int64_t ti = 0; ti < my_tiles && ok; ++ti) {
        const int64_t tile = blockIdx.x + ti * gridDim.x;
        const uint8_t* wt =
            reinterpret_cast<const uint8_t*>(p.wtiles) + (tile % p.n_otiles) * (int64_t)nk * C::B_BYTES;
        for (int kb = 0; kb < nk; ++kb) {
          if (!bwait(&ab_empty[s], ph ^ 1, limit, abort_flag, p.err, site(K_APPLY, 3, 4), (uint32_t)n_b)) { ok = false; break; }
          mbar_arrive_expect_tx(&ab_full[s], C::B_BYTES);
          bulk_load(b_buf + s * C::B_BYTES, wt + (int64_t)kb * C::B_BYTES, C::B_BYTES, &ab_full[s]);
          ++n_b;
          if (++s == C::AB_ST) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      for (int i = 0; i < C::AB_ST; ++i)
        if (n_b > i) mbar_wait(&ab_full[i], (uint32_t)(((n_b - 1 - i) / C::AB_ST) & 1), kDefaultWaitLimit);
    }
  } else if (warp < C::MMA_WARP + C::NMMA) {
    // ------------------------------------------------------------- MMA
    const int mi = warp - C::MMA_WARP;
    if (lane == 0) {
      int s = 0, ab = 0;
      uint32_t ph = 0, acph = 0;
      bool ok = true;
      const uint32_t id_real = idesc_tf32(C::BO) | (1u << 15);       // A MN-major
      const uint32_t id_cplx = idesc_tf32(2 * C::BO) | (1u << 15);
      const uint64_t a_desc0 = smem_desc_mn_tf32(smem_u32(a_buf), C::A_LBO, C::A_SBO);
      const uint64_t b_desc0 = smem_desc(smem_u32(b_buf), C::B_ROWB);
      for (int64_t ti = 0; ti < my_tiles && ok; ++ti) {
        if (!bwait(&acc_empty[ab], acph ^ 1, limit, abort_flag, p.err, site(K_APPLY, 4, 6), (uint32_t)ti)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem_base + ab * C::ACC_COLS;
        for (int kb = 0; kb < nk; ++kb) {
          if (!bwait(&ab_full[s], ph, limit, abort_flag, p.err, site(K_APPLY, 4, 3), (uint32_t)(ti * nk + kb))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a_d = a_desc0 + (uint64_t)((s * C::A_BYTES) >> 4);
          const uint64_t b_d = b_desc0 + (uint64_t)((s * C::B_BYTES) >> 4);
          auto A = [&](int plane) { return a_d + (uint64_t)((plane * C::A_PLANE_BYTES) >> 4); };
          auto B = [&](int plane) { return b_d + (uint64_t)((plane * C::B_PLANE_BYTES) >> 4); };
          // a * w = hi(a) hi(w) + hi(a) lo(w) + lo(a) hi(w)
          auto prod3 = [&](uint32_t d, int pa, int pb, uint32_t id, uint32_t acc_first) {
            mma_tf32_ss(d, A(pa), B(pb), id, acc_first);
            mma_tf32_ss(d, A(pa), B(C::Q + pb), id, 1u);
            mma_tf32_ss(d, A(T + pa), B(pb), id, 1u);
          };
          const uint32_t first = kb > 0 ? 1u : 0u;
#pragma unroll
          for (int f = 0; f < G::nreal; ++f)
            if (C::own_real(f) == mi) prod3(acc + f * C::BO, f, f, id_real, first);
#pragma unroll
          for (int k = 1; k <= G::ncomplex; ++k) {
            if (C::own_cplx(k) != mi) continue;
            const int pr = G::nreal + 2 * (k - 1);
            const int q = G::nreal + 3 * (k - 1);
            const uint32_t col = acc + G::nreal * C::BO + (k - 1) * 2 * C::BO;
            prod3(col, pr, q + 1, id_cplx, first);       // [Re Y | Im Y] += Re X [Re W ; Im W]
            prod3(col, pr + 1, q, id_cplx, 1u);          // [Re Y | Im Y] += Im X [-Im W ; Re W]
          }
          mma_commit(&ab_empty[s]);
          if (++s == C::AB_ST) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[ab]);
        if (++ab == C::NACC) { ab = 0; acph ^= 1; }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      mma_commit(&drain_bar[mi]);
      mbar_wait(&drain_bar[mi], 0, kDefaultWaitLimit);
      // the last commits of the operand slots land with the drain's; wait for
      // them so that none arrives after the CTA has left
      const int64_t n_st = my_tiles * nk;
      for (int i = 0; i < C::AB_ST; ++i)
        if (n_st > i) mbar_wait(&ab_empty[i], (uint32_t)(((n_st - 1 - i) / C::AB_ST) & 1), kDefaultWaitLimit);
    }
  } else {
    // ------------------------------------------------------ epilogue warps
    // Two halves of four warps (one per TMEM lane quarter); half h takes the
    // store chunks h, h+2, ...: 32 f32 outputs (32/T channels) of all 128 rows.
    const int e = warp - C::EPI0;
    const int half = e >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const bool issuer = (e & 3) == 0 && lane == 0;
    int sb = 0;
    int ab = 0;
    uint32_t aph = 0;
    bool ok = true;
    for (int64_t ti = 0; ti < my_tiles; ++ti) {
      const int64_t tile = blockIdx.x + ti * gridDim.x;
      const int ot = (int)(tile % p.n_otiles);
      {
        const int ob = ot * C::BO;
        for (int i = (e & 3) * 32 + lane; i < C::BO; i += 128)
          s_bias[half * C::BO + i] = (p.bias && ob + i < p.O) ? __ldg(p.bias + ob + i) : 0.f;
      }
      const bool got = named_bar_and(
          1 + half, 128, wwait(&acc_full[ab], aph, limit, abort_flag, lane, p.err, site(K_APPLY, 5, 5), (uint32_t)ti));
      if (!got) { ok = false; break; }
      tc_fence_after();
      const int m0 = (int)(tile / p.n_otiles) * C::BM;
      const int o0 = ot * C::BO;
      const uint32_t acc = tmem_base + lane_addr + ab * C::ACC_COLS;
#pragma unroll 1
      for (int ci = half; ci < C::NCHUNK; ci += 2) {
        uint8_t* stage_tile = o_buf + (half * C::NSTG + sb) * C::OUT_TILE_BYTES;
        uint8_t* my_row = stage_tile + r * C::OUT_ROWB;
        // the TMA store issued from this staging tile NSTG chunks ago has read it
        if (issuer) bulk_wait_read<C::NSTG - 1>();
        named_bar_sync(1 + half, 128);
        uint32_t rg[T][C::CH];
#pragma unroll
        for (int q = 0; q < T; ++q) {
          const int k = q < G::nreal ? 0 : 1 + (q - G::nreal) / 2;
          const uint32_t col = acc + ci * C::CH +
                               (q < G::nreal ? q * C::BO
                                             : G::nreal * C::BO + (k - 1) * 2 * C::BO + ((q - G::nreal) & 1) * C::BO);
          if constexpr (C::CH == 4) {
            tmem_ld_32x32b_x4(col, *reinterpret_cast<uint32_t(*)[4]>(&rg[q][0]));
          } else if constexpr (C::CH == 8) {
            tmem_ld_32x32b_x8(col, *reinterpret_cast<uint32_t(*)[8]>(&rg[q][0]));
          } else {
#pragma unroll
            for (int h = 0; h < C::CH / 16; ++h) tmem_ld_32x32b_x16(col + 16 * h, &rg[q][16 * h]);
          }
        }
        tmem_wait_ld();
        if (ci + 2 >= C::NCHUNK) {
          tc_fence_before();
          mbar_arrive(&acc_empty[ab]);
        }
#pragma unroll
        for (int sub = 0; sub < C::CH / C::SUBCH; ++sub) {
          const int oc = ci * C::CH + sub * C::SUBCH;
          float bo8[C::SUBCH];
#pragma unroll
          for (int i4 = 0; i4 < C::SUBCH / 4; ++i4) {
            const float4 b4 = *reinterpret_cast<const float4*>(s_bias + half * C::BO + oc + 4 * i4);
            bo8[4 * i4] = b4.x; bo8[4 * i4 + 1] = b4.y; bo8[4 * i4 + 2] = b4.z; bo8[4 * i4 + 3] = b4.w;
          }
          // SUBCH channels x T outputs = SUBCH*T/4 16-byte chunks of this row's 128 bytes
          float vals[C::SUBCH * T];
#pragma unroll
          for (int cc = 0; cc < C::SUBCH; ++cc) {
            float Pc[T];
#pragma unroll
            for (int q = 0; q < T; ++q) Pc[q] = __uint_as_float(rg[q][sub * C::SUBCH + cc]);
            G::idft_scaled(Pc, bo8[cc], vals + cc * T);
          }
#pragma unroll
          for (int v = 0; v < C::SUBCH * T / 4; ++v) {
            const int j = sub * (C::SUBCH * T / 4) + v;
            *reinterpret_cast<float4*>(my_row + ((j ^ (r & 7)) << 4)) =
                make_float4(vals[4 * v], vals[4 * v + 1], vals[4 * v + 2], vals[4 * v + 3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1 + half, 128);
        if (issuer) {
          tma_store_2d(&map_out, stage_tile, (o0 + ci * C::CH) * T, m0);
          bulk_commit();
        }
        if (++sb == C::NSTG) sb = 0;
      }
      if (++ab == C::NACC) { ab = 0; aph ^= 1; }
    }
    if (!ok) raise_abort(abort_flag, p.err);
    if (issuer) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------- pretransform
// One thread per (image, row, 8 K-consecutive entries): the Fourier weights
// of the 8 entries (FP32 DFT along the group axis, scaled by 1/T for real
// frequencies and 2/T for complex ones; the forward image holds (-Im, Re, Im)
// per complex frequency, the input-gradient image the conjugate (Im, Re,
// -Im)), split into hi = tf32(v) and lo = tf32(v - hi); a plane's 8 entries
// are one 32-byte row of a stage (two 16-byte stores).  Threads [0, nA) build
// the forward image (rows d, K c), the rest the input-gradient image (rows c,
// K d); thread 0 .. D'-1 also copy the bias.  Entries past K are zeros.
template <int T>
__global__ void __launch_bounds__(256)
tc32_pretransform_kernel(const float* __restrict__ W, const float* __restrict__ b, float* __restrict__ wt_fwd,
                         float* __restrict__ wt_bwd, float* __restrict__ bias, int Cp, int Dp, int bo_f, int bo_b) {
  using G = Group<T>;
  grid_dep_launch();
  grid_dep_wait();
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid < Dp) bias[tid] = b ? b[tid] : 0.f;
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
  float P[8][T];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t k = k0 + i;
    float v[T];
    // W[d, c, t]: forward rows d, K c; input gradient rows c, K d
    const int64_t base = fwd ? (row * Cp + k) * T : (k * Cp + row) * T;
#pragma unroll
    for (int t = 0; t < T; ++t) v[t] = k < K ? __ldg(W + base + t) : 0.f;
    G::dft(v, P[i]);
  }
  float* out = fwd ? wt_fwd : wt_bwd;
  const int bo = fwd ? bo_f : bo_b;
  const int64_t nkb = (K + TC32_BK - 1) / TC32_BK;
  const float sr = 1.f / T, sc = 2.f / T;
  auto put = [&](int q, const float (&o)[8]) {
    uint32_t h[8], l[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      h[i] = f32_to_tf32(o[i]);
      l[i] = f32_to_tf32(o[i] - __uint_as_float(h[i]));
    }
    const int Q = G::nreal + 3 * G::ncomplex;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const uint32_t* w = part ? l : h;
#pragma unroll
      for (int c4 = 0; c4 < 2; ++c4)
        *reinterpret_cast<uint4*>(out + wtile32_index(T, bo, nkb, row, k0 + 4 * c4, part * Q + q)) =
            make_uint4(w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
    }
  };
  float o[8];
#pragma unroll
  for (int f = 0; f < G::nreal; ++f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = P[i][f] * sr;
    put(f, o);
  }
#pragma unroll
  for (int k = 1; k <= G::ncomplex; ++k) {
    const int pr = G::nreal + 2 * (k - 1), q = G::nreal + 3 * (k - 1);
    const float s0 = fwd ? -1.f : 1.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = s0 * (P[i][pr + 1] * sc);
    put(q + 0, o);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = P[i][pr] * sc;
    put(q + 1, o);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = -s0 * (P[i][pr + 1] * sc);
    put(q + 2, o);
  }
}

// ------------------------------------------------------------------- host
template <int T, int BO>
static cudaError_t launch_t(const Handle& h, bool backward, const void* in, void* out, int64_t N, cudaStream_t st) {
  using C = Cfg<T, BO>;
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return cudaErrorNotSupported;
  const int K = (int)(backward ? h.Dp : h.Cp);
  const int O = (int)(backward ? h.Cp : h.Dp);
  CUtensorMap map_in;      // raw input tiles: 8 channels x T elements x 128 tokens
  {
    cuuint64_t dims[2] = {(cuuint64_t)K * T, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)K * T * 4};
    cuuint32_t box[2] = {(cuuint32_t)(C::BK * T), (cuuint32_t)C::BM};
    cuuint32_t es[2] = {1, 1};
    if (enc(&map_in, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(in), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  CUtensorMap map_out;     // TMA stores: 32 f32 x 128 rows, 128B swizzle
  {
    cuuint64_t dims[2] = {(cuuint64_t)O * T, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)O * T * 4};
    cuuint32_t box[2] = {(cuuint32_t)C::OUT_EL, (cuuint32_t)C::BM};
    cuuint32_t es[2] = {1, 1};
    if (enc(&map_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, out, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  Params p;
  p.N = N;
  p.K = K;
  p.O = O;
  p.n_otiles = (O + C::BO - 1) / C::BO;
  p.n_tb = (int)((N + C::BM - 1) / C::BM);
  p.n_tiles = (int64_t)p.n_tb * p.n_otiles;
  p.wtiles = backward ? h.wt_bwd : h.wt_fwd;
  p.bias = backward ? nullptr : h.bias;
  p.err = h.err;
  p.wait_limit = h.wait_limit ? h.wait_limit : kDefaultWaitLimit;
  {
    const cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(tc32_apply_kernel<T, BO>), C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  int64_t grid = p.n_tiles < h.sm_count ? p.n_tiles : h.sm_count;
  if (grid < 1) grid = 1;
  const cudaError_t e = launch_pdl(tc32_apply_kernel<T, BO>, dim3((unsigned)grid), dim3(C::THREADS), C::SMEM_BYTES,
                                   st, map_in, map_out, p);
  count_launches(1);
  return e;
}

}  // namespace tc32

bool tc32_supported(const Handle& h) {
  return h.group == EQLIN_GROUP_CYCLIC && h.dtype == EQLIN_F32 && (h.T == 1 || h.T == 2 || h.T == 4 || h.T == 8) &&
         tensor_map_encoder() != nullptr;
}

// The tensor core rounds as it adds each MMA's products into the FP32
// accumulator, and the error of a product sum grows with the number of MMAs
// that feed one accumulator (measured: about 1.5e-8 to 1.9e-8 relative
// Frobenius error per MMA); 256 MMAs keep it near 5e-6, half the 1e-5 bound.
bool tc32_pass_ok(const Handle& h, bool backward) {
  if (!tc32_supported(h)) return false;
  const int64_t K = backward ? h.Dp : h.Cp;
  const int64_t per_stage = h.T % 4 == 0 ? 6 : 3;   // MMAs into one accumulator per 8-channel stage
  return per_stage * ((K + TC32_BK - 1) / TC32_BK) <= 256;
}

cudaError_t launch_tc32_apply(const Handle& h, bool backward, const void* in, void* out, int64_t N,
                              cudaStream_t st) {
  if (!tc32_pass_ok(h, backward) || !h.wt_fwd || !h.wt_bwd) return cudaErrorNotSupported;
  const int bo = backward ? h.bo_bwd : h.bo_fwd;
  switch (h.T) {
    case 1: return bo == 256 ? tc32::launch_t<1, 256>(h, backward, in, out, N, st) : cudaErrorInvalidValue;
    case 2:
      return bo == 256   ? tc32::launch_t<2, 256>(h, backward, in, out, N, st)
             : bo == 128 ? tc32::launch_t<2, 128>(h, backward, in, out, N, st)
                         : cudaErrorInvalidValue;
    case 4:
      return bo == 128  ? tc32::launch_t<4, 128>(h, backward, in, out, N, st)
             : bo == 64 ? tc32::launch_t<4, 64>(h, backward, in, out, N, st)
             : bo == 32 ? tc32::launch_t<4, 32>(h, backward, in, out, N, st)
                        : cudaErrorInvalidValue;
    case 8: return bo == 32 ? tc32::launch_t<8, 32>(h, backward, in, out, N, st) : cudaErrorInvalidValue;
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_tc32_pretransform(const Handle& h, const float* W, const float* b, cudaStream_t st) {
  if (!tc32_supported(h) || !h.wt_fwd || !h.wt_bwd) return cudaErrorNotSupported;
  const int64_t n = h.Dp * ((h.Cp + 7) / 8) + h.Cp * ((h.Dp + 7) / 8);
  const int64_t threads = n > h.Dp ? n : h.Dp;
  const dim3 grid((unsigned)((threads + 255) / 256));
  cudaError_t e = cudaErrorInvalidValue;
  switch (h.T) {
    case 1:
      e = launch_pdl(tc32::tc32_pretransform_kernel<1>, grid, dim3(256), 0, st, W, b, (float*)h.wt_fwd,
                     (float*)h.wt_bwd, h.bias, (int)h.Cp, (int)h.Dp, h.bo_fwd, h.bo_bwd);
      break;
    case 2:
      e = launch_pdl(tc32::tc32_pretransform_kernel<2>, grid, dim3(256), 0, st, W, b, (float*)h.wt_fwd,
                     (float*)h.wt_bwd, h.bias, (int)h.Cp, (int)h.Dp, h.bo_fwd, h.bo_bwd);
      break;
    case 4:
      e = launch_pdl(tc32::tc32_pretransform_kernel<4>, grid, dim3(256), 0, st, W, b, (float*)h.wt_fwd,
                     (float*)h.wt_bwd, h.bias, (int)h.Cp, (int)h.Dp, h.bo_fwd, h.bo_bwd);
      break;
    case 8:
      e = launch_pdl(tc32::tc32_pretransform_kernel<8>, grid, dim3(256), 0, st, W, b, (float*)h.wt_fwd,
                     (float*)h.wt_bwd, h.bias, (int)h.Cp, (int)h.Dp, h.bo_fwd, h.bo_bwd);
      break;
  }
  count_launches(1);
  return e;
}

}  // namespace eqlin
