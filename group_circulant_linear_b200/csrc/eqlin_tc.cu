// eqlin_tc.cu -- the tcgen05 (5th-generation tensor core) kernel for the
// forward pass and the input gradient, f16/bf16 in, f32 accumulation.
//
// One persistent CTA per SM walks output tiles of 128 tokens x BO output
// channels (all T group positions).  Per tile and per K stage of 16 input
// channels:
//
//   raw producer     (8)    TMA: the raw input tile of the stage [128 tokens x
//                    16*T elements] into the raw ring; L2 prefetches of raw
//                    tiles several stages ahead
//   weight producer  (9)    one bulk copy of the stage's Fourier weight planes
//                    (stored pre-swizzled per stage) into the operand ring
//   transform warps  (0-7)  two groups of four warps on alternate stages; one
//                    thread per (input channel, 16 tokens): read the
//                    channel's T group values of its tokens from the raw tile,
//                    take the group DFT (adds/subtracts on packed token pairs
//                    for T <= 4, FP32 with the sqrt(2)/2 twiddles for T = 8)
//                    and write the T frequency planes as token-contiguous
//                    (MN-major, 128B-swizzled) MMA operands; then a
//                    generic->async proxy fence
//   MMA warps        (10, 11) lane 0 of each issues tcgen05.mma into TMEM for
//                    the accumulators it owns: for each real frequency one
//                    M=128, N=BO product; for each complex frequency two
//                    M=128, N=2*BO products that accumulate
//                    [Re Y | Im Y] = Re X [Re W ; Im W] + Im X [-Im W ; Re W]
//                    -- R(T) real GEMMs, six for p4.  Two issuers split the
//                    stage's MMAs (p4: the two real frequencies, and the
//                    complex block product), each with its own waits and
//                    commits; an accumulator is only ever written by one
//                    issuer.
//   epilogue warps   (12-19) tcgen05.ld of the frequency planes, inverse DFT
//                    (the weight planes carry its 1/T and 2/T scales, so this
//                    is additions only), bias, cast into a 128B-swizzled
//                    staging tile, TMA store of 64 output elements x 128 rows
//   stash warp       (20, stash forms only) for the tiles of each token
//                    block's first output tile, TMA stores of the stage's
//                    transformed A planes -- the input's spectrum, X = DFT(x)
//                    for the forward, G = DFT(gy) for the input gradient -- to
//                    a caller-owned buffer [T planes][channels][tokens]; the
//                    weight gradient then reads the spectra instead of
//                    transforming x and gy again.  It starts as soon as the
//                    transform has written the planes (its own barrier), so
//                    the stores read them while the weights load and the MMAs
//                    run; an operand slot is free once both have read it.
//
// The two rings are independent: a raw slot is refilled as soon as the
// transform warps have read it, and an operand slot (the stage's A planes and
// weight planes) once the MMAs that read it have completed; so loads run
// ahead of the tensor core by the whole raw ring.
//
// Tail split: when the last wave of tiles would leave at least half of the
// SMs idle, each of its tiles runs as two units on two SMs, each over part of
// the reduction.  The half that finishes its MMAs first stores its FP32
// accumulator in the handle's workspace and raises a flag; the other adds it
// in TMEM and stores the tile (the epilogue warps, below).
//
// ("Flash EQ-Linear", technical summary, sections "Abordagem Algoritmica",
// "Especializacao para o Grupo de Rotacao p4" and "Implementacao": fused data
// flow, Fourier fragments kept on chip, tensor cores.)  The input gradient
// runs the same kernel with the conjugated, transposed weight planes and no
// bias.
//
// Every mbarrier wait is bounded.  A wait that runs out records a timeout in
// the handle's error word, raises a CTA-wide abort flag, and the kernel
// drains its own in-flight TMA copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <type_traits>

#include "eqlin_internal.cuh"
#include "eqlin_packed.cuh"
#include "eqlin_ptx.cuh"
#include "eqlin_wait.cuh"

namespace eqlin {
namespace tc {

using namespace ptx;
using namespace waits;

// GAUSS_: the three-product form of the complex products (p4 only), for
// comparison with the four-product form the paper counts: per complex
// frequency k1 = (Re X + Im X) Re W, k2 = Re X (Im W - Re W), k3 = Im X (Re W
// + Im W), Re Y = k1 - k3, Im Y = k1 + k2 -- five real GEMMs per p4 stage
// instead of six, each N = BO, into five accumulators; the transform adds a
// Re X + Im X plane.
template <int T, int BO_, bool STASH_ = false, bool GAUSS_ = false>
struct Cfg {
  using G = Group<T>;
  static constexpr bool GAUSS = GAUSS_;
  static_assert(!GAUSS || (T == 4 && !STASH_), "the three-product form is the p4 forward's");
  static constexpr int NCX = GAUSS ? G::ncomplex : 0;      // extra A planes (Re X + Im X)
  static constexpr int BM = 128;                       // tokens per tile (MMA M)
  static constexpr int BK = TC_BK;                     // input channels per stage (one MMA K step)
  // output channels per tile and accumulator buffers: T * BO * NACC <= 512 columns
  static constexpr int BO = BO_;
  static constexpr int ACC_COLS = (GAUSS ? G::nreal + 3 * G::ncomplex : T) * BO;
  static_assert(ACC_COLS <= 512 && (Group<T>::ncomplex == 0 || 2 * BO <= 256), "TMEM columns, MMA N");
  static constexpr int NACC = (ACC_COLS * 2 <= 512) ? 2 : 1;
  static constexpr int TMEM_COLS = NACC * ACC_COLS <= 256 ? 256 : 512;
  static constexpr int Q = G::nreal + 3 * G::ncomplex; // weight planes per stage
  // raw input tile of a stage: 128 tokens x (16 channels x T) elements, row-major (TMA)
  static constexpr int RAW_ROWB = BK * T * 2;
  static constexpr int RAW_BYTES = BM * RAW_ROWB;
  // A: MN-major, 128B swizzle: 64-token blocks (LBO apart) of 8-channel groups (SBO apart)
  static constexpr int A_SBO = 1024;
  static constexpr int A_LBO = (BK / 8) * A_SBO;       // 2048
  static constexpr int A_PLANE_BYTES = BM * BK * 2;    // 4 KB
  static constexpr int A_BYTES = (T + NCX) * A_PLANE_BYTES;
  // B: K-major, 32-byte rows (16 channels), 32B swizzle
  static constexpr int B_ROWB = BK * 2;
  static constexpr int B_PLANE_BYTES = BO * B_ROWB;
  static constexpr int B_BYTES = Q * B_PLANE_BYTES;
  // output staging for the TMA stores: per epilogue half two [128 rows x
  // OUT_EL elements] tiles; 64 elements (128 bytes, 128B swizzle) for T | 8,
  // 48 (96 bytes, unswizzled) for T = 3 and 6
  static constexpr bool POW2 = (T & (T - 1)) == 0;
  static constexpr int OUT_EL = POW2 ? 64 : 48;        // output elements per row per store
  static constexpr int OUT_ROWB = OUT_EL * 2;
  static constexpr int OUT_TILE_BYTES = BM * OUT_ROWB;
  static constexpr int STAGING = 4 * OUT_TILE_BYTES;
  // ring depths: operand slots (the A planes of a stage and its weight
  // planes share one slot and one pair of barriers, so the MMA thread waits
  // and commits once per stage): three where four raw slots still fit (the
  // transform writes stage k + 2 while the MMAs of k and k + 1 are in
  // flight), else two; the rest of the budget for raw slots (memory latency)
  //
  // The raw ring's depth is even.  The two transform groups take alternate
  // stages, and stages k and k + RAW_ST share a slot.  With an odd depth they
  // belong to different groups, so one group could wait on the slot's next
  // phase while the other group's stage k had not yet landed; an mbarrier
  // parity wait cannot tell a phase from the one two ahead, so that wait would
  // return at once, read stale data and complete the slot's release early
  // (a second TMA load into a slot whose first was still in flight).  With an
  // even depth both uses of a slot are the same group's, which consumes them
  // in order.
  static constexpr int BUDGET = 224 * 1024;
  static constexpr int AB_ST = (BUDGET - STAGING - 3 * (A_BYTES + B_BYTES)) / RAW_BYTES >= 4 ? 3 : 2;
  static constexpr int RAW_FIT = (BUDGET - STAGING - AB_ST * (A_BYTES + B_BYTES)) / RAW_BYTES;
  static constexpr int RAW_ST = (RAW_FIT > 8 ? 8 : RAW_FIT) & ~1;
  static_assert(RAW_ST >= 2 && AB_ST >= 2, "two slots per ring (the transform groups take alternate stages)");
  static_assert(RAW_ST % 2 == 0, "both uses of a raw slot belong to one transform group");
  // MMA issuers: a group of accumulators (one per real frequency, one per
  // complex frequency, which takes two MMAs) belongs to one issuer; in order,
  // groups go to issuer 0 until it holds half of the stage's MMAs.
  static constexpr int NMMA = (T == 1) ? 1 : 2;
  static constexpr int MMAS = G::nreal + 2 * G::ncomplex;          // MMAs per stage
  __host__ __device__ static constexpr int own_real(int f) {
    return (NMMA == 1 || GAUSS || 2 * f < MMAS) ? 0 : 1;
  }
  __host__ __device__ static constexpr int own_cplx(int k) {
    return NMMA == 1 ? 0 : GAUSS ? 1 : (2 * (G::nreal + 2 * (k - 1)) < MMAS) ? 0 : 1;
  }
  static constexpr int NBAR = 2 * RAW_ST + 3 * AB_ST + 2 * NACC + NMMA + 2;
  // per epilogue half, the bias of the tile's BO channels (FP32)
  static constexpr int BIAS_BYTES = 2 * BO * 4;
  static constexpr int SMEM_BYTES = RAW_ST * RAW_BYTES + AB_ST * (A_BYTES + B_BYTES) + STAGING +
                                    BIAS_BYTES + NBAR * 8 + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
  static constexpr int CH = OUT_EL / T;                // output channels per store chunk
  static_assert(OUT_EL % T == 0 && CH % 8 == 0, "whole channels per store chunk, 8 at a time");
  static constexpr int NCHUNK = BO / CH;               // store chunks per tile (even)
  static_assert(NCHUNK % 2 == 0, "chunks alternate between the two epilogue halves");
  // roles
  static constexpr int TR_WARPS = 8;                   // transform: two groups of four warps
  static constexpr int GRP_WARPS = TR_WARPS / 2;       // warps per stage (16 tokens x 16 channels per warp-half)
  static constexpr int RAW_PRODUCER = TR_WARPS, B_PRODUCER = TR_WARPS + 1;
  static constexpr int MMA_WARP = TR_WARPS + 2, EPI0 = MMA_WARP + NMMA;
  static constexpr int EPI_WARPS = 8;                  // two per TMEM lane quarter
  static constexpr int STASH_WARP = EPI0 + EPI_WARPS;  // present in the stash forms only
  static constexpr int THREADS = (EPI0 + EPI_WARPS + (STASH_ ? 1 : 0)) * 32;
  static constexpr int W = packed::Words<T>::n;        // 32-bit words per token and channel
  static constexpr int PF_STAGES = 10;                 // L2 prefetch distance of the input tiles
  // split tiles: accumulator columns per round of the merge (a contiguous
  // MERGE_COLS x 128 x 4 bytes of the stored image), bulk-copied into one
  // half of the raw ring while the other half's round is added in
  static constexpr int RAW_HALF = RAW_ST * RAW_BYTES / 2;
  static constexpr int MERGE_COLS = (ACC_COLS % 64 == 0 && 64 * BM * 4 <= RAW_HALF)   ? 64
                                    : (ACC_COLS % 32 == 0 && 32 * BM * 4 <= RAW_HALF) ? 32
                                                                                      : 16;
  static_assert(ACC_COLS % MERGE_COLS == 0 && MERGE_COLS * BM * 4 <= RAW_HALF, "merge rounds fit half the raw ring");
};

struct Params {
  int64_t N;       // tokens
  int K;           // input channels per group element (C' forward, D' for dx)
  int O;           // output channels per group element
  int n_otiles;
  int n_tb;        // 128-token blocks
  int64_t n_tiles;
  const void* in;
  const void* wtiles;  // tensor-core weight tiles (rows O, K) of this pass
  const float* bias;   // nullptr: none
  int* err;
  uint32_t wait_limit;
  uint32_t ab_fmt;     // 0 f16, 1 bf16
  // tail split (tc_split_tiles): the last n_split tiles run as two halves
  int n_split;
  float* split_ws;     // [n_split][ACC_COLS / 4][128 rows][4] FP32 accumulators
  int* split_claim;    // [n_split] halves that have finished their MMAs
  int* split_ready;    // [n_split] 1 once the first half's accumulator is stored
  int* split_done;     // CTAs finished (the last one zeroes the flags)
};

// Eight floats to eight 16-bit values (round to nearest even), two per conversion.
template <typename E>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  if constexpr (std::is_same<E, __half>::value) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}
template <typename E>
__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(pack2<E>(f[0], f[1]), pack2<E>(f[2], f[3]), pack2<E>(f[4], f[5]), pack2<E>(f[6], f[7]));
}

template <int T, int BO, typename E, bool STASH, bool GAUSS = false>
__global__ void __launch_bounds__(Cfg<T, BO, STASH, GAUSS>::THREADS, 1)
tc_apply_kernel(const __grid_constant__ CUtensorMap map_in, const __grid_constant__ CUtensorMap map_out,
                const __grid_constant__ CUtensorMap map_stash, Params p) {
  using C = Cfg<T, BO, STASH, GAUSS>;
  using G = Group<T>;
  grid_dep_launch();
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* a_buf = smem;                                   // [AB_ST][T planes]
  uint8_t* b_buf = a_buf + C::AB_ST * C::A_BYTES;          // [AB_ST][Q planes]
  uint8_t* raw_buf = b_buf + C::AB_ST * C::B_BYTES;        // [RAW_ST][raw tile]
  uint8_t* o_buf = raw_buf + C::RAW_ST * C::RAW_BYTES;     // 4 staging tiles
  float* s_bias = reinterpret_cast<float*>(o_buf + C::STAGING);      // [2][BO]
  uint64_t* bars = reinterpret_cast<uint64_t*>(o_buf + C::STAGING + C::BIAS_BYTES);
  uint64_t* raw_full = bars;                   // TMA bytes landed
  uint64_t* raw_empty = raw_full + C::RAW_ST;  // the 8 transform warps have read the slot
  // ab_full: the 8 transform warps have written the A planes and the weight
  // planes' bulk-copy bytes have landed; ab_empty: MMA commit
  uint64_t* ab_full = raw_empty + C::RAW_ST;
  uint64_t* ab_empty = ab_full + C::AB_ST;
  uint64_t* a_ready = ab_empty + C::AB_ST;     // the transform has written the A planes (stash forms)
  uint64_t* acc_full = a_ready + C::AB_ST;
  uint64_t* acc_empty = acc_full + C::NACC;
  uint64_t* drain_bar = acc_empty + C::NACC;    // [NMMA]
  uint64_t* merge_bar = drain_bar + C::NMMA;    // [2] split tiles: a merge round's bytes landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(merge_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* split_mode = abort_flag + 1;   // the epilogue's role in a split tile

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t limit = p.wait_limit;
  const int nk = (p.K + C::BK - 1) / C::BK;
  // Work units of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...  Tiles
  // are numbered t = token block * n_otiles + output tile.  Tiles t < n_whole
  // are whole units (all nk stages); the last n_split tiles are split in two
  // along the reduction, into units n_whole + 2j (stages [0, mid)) and
  // n_whole + 2j + 1 (stages [mid, nk)) of pair j, mid = 3 nk / 8: the
  // shorter half usually finishes first and hands its accumulator over while
  // the longer one still runs its MMAs.  n_whole is a multiple of
  // the grid, so the halves fill part of the last wave side by side.  Whole
  // units follow the tile numbering, so the output tiles of one token block
  // run side by side and share its input tile in L2.  The stash forms take
  // the same whole tiles output tile by output tile instead: only output
  // tile 0 stores, and in the first order a CTA's tiles b, b + grid, ... all
  // have the same output tile whenever n_otiles divides the grid, so half of
  // the CTAs would do every store.  Both forms split the same tiles, so their
  // outputs are identical.
  struct Unit {
    int tb, ot, kb0, kb1, pair;   // token block, output tile, stages; pair -1: a whole tile
  };
  const int n_whole = (int)p.n_tiles - p.n_split;
  const int n_units = n_whole + 2 * p.n_split;
  const int my_units = n_units > (int)blockIdx.x ? (n_units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto unit = [&](int i) -> Unit {
    const int u = (int)blockIdx.x + i * (int)gridDim.x;
    if (u >= n_whole) {
      const int v = u - n_whole, j = v >> 1, mid = (nk * 3) >> 3, t = n_whole + j;
      return (v & 1) ? Unit{t / p.n_otiles, t % p.n_otiles, mid, nk, j}
                     : Unit{t / p.n_otiles, t % p.n_otiles, 0, mid, j};
    }
    if (!STASH) return Unit{u / p.n_otiles, u % p.n_otiles, 0, nk, -1};
    // output tile ot holds q + (ot < rem) of the whole tiles
    const int q = n_whole / p.n_otiles, rem = n_whole % p.n_otiles;
    if (u < rem * (q + 1)) return Unit{u % (q + 1), u / (q + 1), 0, nk, -1};
    const int k = u - rem * (q + 1);
    return Unit{k % q, rem + k / q, 0, nk, -1};
  };
  // stages of this CTA: nk per whole tile, mid or nk - mid per split half
  int my_stages = 0;
  for (int i = 0; i < my_units; ++i) {
    const Unit un = unit(i);
    my_stages += un.kb1 - un.kb0;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::RAW_ST; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], C::GRP_WARPS);
    }
    for (int i = 0; i < C::AB_ST; ++i) {
      mbar_init(&ab_full[i], C::GRP_WARPS + 1);
      mbar_init(&ab_empty[i], C::NMMA + (STASH ? 1 : 0));   // a commit per MMA issuer (+ the stash warp)
      mbar_init(&a_ready[i], C::GRP_WARPS);
    }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(&acc_full[i], C::NMMA);
      mbar_init(&acc_empty[i], C::EPI_WARPS * 32);
    }
    for (int i = 0; i < C::NMMA; ++i) mbar_init(&drain_bar[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&merge_bar[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&map_in);
    prefetch_tensormap(&map_out);
    if (STASH) prefetch_tensormap(&map_stash);
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
    // ----------------------------------------------------- transform warps
    // Two groups of four warps take alternate stages, so two stages are in
    // flight.  Thread: channel c of the stage (16 per stage) and 16
    // consecutive tokens (two blocks of 8).
    const int grp = warp / C::GRP_WARPS;
    const int c = lane & 15;
    const int m = (warp % C::GRP_WARPS) * 32 + 16 * (lane >> 4);   // first of its 16 tokens
    // MN-major placement of 8 tokens (block b) for K row c of a plane
    uint32_t a_off[2];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int mb = m + 8 * b;
      a_off[b] = (uint32_t)((mb >> 6) * C::A_LBO + (c >> 3) * C::A_SBO + (c & 7) * 128 +
                            ((((mb & 63) >> 3) ^ (c & 7)) << 4));
    }
    const uint32_t raw_off = (uint32_t)(m * C::RAW_ROWB + c * T * 2);
    // ring positions of stage `grp`, then advanced by two stages per step
    int rs = grp % C::RAW_ST, as = grp % C::AB_ST;
    uint32_t rph = 0, aph = 0;
    bool ok = true;
    for (int it = grp; it < my_stages; it += 2) {
      if (!wwait_all(&raw_full[rs], rph, limit, abort_flag, p.err, site(K_APPLY, 1, 1), (uint32_t)it)) { ok = false; break; }
      const uint8_t* raw = raw_buf + rs * C::RAW_BYTES + raw_off;
      uint32_t Pw[2][T][4];
      if constexpr (T == 1 || T == 2 || T == 4) {
        // all 16 tokens' words first, so the raw slot is released early
        uint32_t wv[16][C::W];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint8_t* src = raw + j * C::RAW_ROWB;
          if constexpr (C::W == 2) {
            const uint2 u = *reinterpret_cast<const uint2*>(src);
            wv[j][0] = u.x; wv[j][1] = u.y;
          } else if constexpr (T == 2) {
            wv[j][0] = *reinterpret_cast<const uint32_t*>(src);
          } else {
            wv[j][0] = *reinterpret_cast<const unsigned short*>(src);
          }
        }
        // the raw slot may be refilled by TMA (async proxy) once these generic
        // reads are ordered before it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_empty[rs]);
#pragma unroll
        for (int b = 0; b < 2; ++b)
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
            uint32_t P[T];
            packed::dft_pair<T, E>(wv[8 * b + 2 * pr], wv[8 * b + 2 * pr + 1], P);
#pragma unroll
            for (int q = 0; q < T; ++q) Pw[b][q][pr] = P[q];
          }
      } else if constexpr (T == 8) {
        // T = 8: one block of 8 tokens at a time (registers), FP32 butterflies
        // with the sqrt(2)/2 twiddles, one rounding per value
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          uint32_t wv[8][C::W];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 u = *reinterpret_cast<const uint4*>(raw + (8 * b + j) * C::RAW_ROWB);
            wv[j][0] = u.x; wv[j][1] = u.y; wv[j][2] = u.z; wv[j][3] = u.w;
          }
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
            float Pa[T], Pb[T], va[T], vb[T];
            const E* ea = reinterpret_cast<const E*>(wv[2 * pr]);
            const E* eb = reinterpret_cast<const E*>(wv[2 * pr + 1]);
#pragma unroll
            for (int t = 0; t < T; ++t) { va[t] = Elem<E>::to_f(ea[t]); vb[t] = Elem<E>::to_f(eb[t]); }
            G::dft(va, Pa);
            G::dft(vb, Pb);
#pragma unroll
            for (int q = 0; q < T; ++q) Pw[b][q][pr] = pack2<E>(Pa[q], Pb[q]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_empty[rs]);
      } else {
        // T = 3, 6: a channel's T values are 6 or 12 bytes, read element by
        // element, a pair of tokens at a time; FP32 butterflies with the
        // sqrt(3)/2 twiddles, one rounding per value
#pragma unroll
        for (int b = 0; b < 2; ++b) {
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
            const E* ea = reinterpret_cast<const E*>(raw + (8 * b + 2 * pr) * C::RAW_ROWB);
            const E* eb = reinterpret_cast<const E*>(raw + (8 * b + 2 * pr + 1) * C::RAW_ROWB);
            float Pa[T], Pb[T], va[T], vb[T];
#pragma unroll
            for (int t = 0; t < T; ++t) { va[t] = Elem<E>::to_f(ea[t]); vb[t] = Elem<E>::to_f(eb[t]); }
            G::dft(va, Pa);
            G::dft(vb, Pb);
#pragma unroll
            for (int q = 0; q < T; ++q) Pw[b][q][pr] = pack2<E>(Pa[q], Pb[q]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_empty[rs]);
      }
      rs += 2;
      if (rs >= C::RAW_ST) { rs -= C::RAW_ST; rph ^= 1; }
      // the operand slot must have been consumed by the MMAs issued from it
      if (!wwait(&ab_empty[as], aph ^ 1, limit, abort_flag, lane, p.err, site(K_APPLY, 1, 4), (uint32_t)it)) { ok = false; break; }
      uint8_t* a_st = a_buf + as * C::A_BYTES;
#pragma unroll
      for (int b = 0; b < 2; ++b)
#pragma unroll
        for (int q = 0; q < T; ++q)
          *reinterpret_cast<uint4*>(a_st + q * C::A_PLANE_BYTES + a_off[b]) =
              make_uint4(Pw[b][q][0], Pw[b][q][1], Pw[b][q][2], Pw[b][q][3]);
      if constexpr (C::GAUSS) {
        // Re X + Im X of each complex frequency (packed adds, one rounding)
#pragma unroll
        for (int b = 0; b < 2; ++b)
#pragma unroll
          for (int k = 1; k <= G::ncomplex; ++k) {
            const int pr = G::nreal + 2 * (k - 1);
            uint32_t sw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) sw[i] = packed::Pair<E>::add(Pw[b][pr][i], Pw[b][pr + 1][i]);
            *reinterpret_cast<uint4*>(a_st + (T + k - 1) * C::A_PLANE_BYTES + a_off[b]) =
                make_uint4(sw[0], sw[1], sw[2], sw[3]);
          }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ab_full[as]);
        if (STASH) mbar_arrive(&a_ready[as]);
      }
      as += 2;
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
      // L2 prefetch of the raw input tiles PF_STAGES stages ahead of their loads
      int pf_ti = 0;
      int pf_kb = 0;
      auto prefetch_next = [&]() {
        if (pf_ti >= my_units) return;
        const Unit un = unit(pf_ti);
        if (pf_kb < un.kb0) pf_kb = un.kb0;
        tma_prefetch_2d(&map_in, pf_kb * C::BK * T, un.tb * C::BM);
        if (++pf_kb == un.kb1) { pf_kb = 0; ++pf_ti; }
      };
      for (int i = 0; i < C::PF_STAGES; ++i) prefetch_next();
      for (int ti = 0; ti < my_units && ok; ++ti) {
        const Unit un = unit(ti);
        const int m0 = un.tb * C::BM;
        for (int kb = un.kb0; kb < un.kb1; ++kb) {
          prefetch_next();
          if (!bwait(&raw_empty[s], ph ^ 1, limit, abort_flag, p.err, site(K_APPLY, 2, 2), (uint32_t)n_raw)) { ok = false; break; }
          mbar_arrive_expect_tx(&raw_full[s], C::RAW_BYTES);
          tma_load_2d(raw_buf + s * C::RAW_BYTES, &map_in, kb * C::BK * T, m0, &raw_full[s]);
          ++n_raw;
          if (++s == C::RAW_ST) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      // every issued TMA copy must land before the CTA exits (a no-op on the
      // normal path, where the transform warps already waited for them)
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
      for (int ti = 0; ti < my_units && ok; ++ti) {
        const Unit un = unit(ti);
        const uint8_t* wt = reinterpret_cast<const uint8_t*>(p.wtiles) + (int64_t)un.ot * nk * C::B_BYTES;
        for (int kb = un.kb0; kb < un.kb1; ++kb) {
          if (!bwait(&ab_empty[s], ph ^ 1, limit, abort_flag, p.err, site(K_APPLY, 3, 4), (uint32_t)n_b)) { ok = false; break; }
          // the stage's Q weight planes are one contiguous, pre-swizzled tile
          mbar_arrive_expect_tx(&ab_full[s], C::B_BYTES);
          bulk_load(b_buf + s * C::B_BYTES, wt + (int64_t)kb * C::B_BYTES, C::B_BYTES, &ab_full[s]);
          ++n_b;
          if (++s == C::AB_ST) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      // the weight copies must land before the CTA exits.  A slot's phase
      // completes with its bytes and the transform warps' arrivals; if an
      // aborted run never makes those, the wait gives up after its wall-time
      // cap, long after any copy has landed.
      for (int i = 0; i < C::AB_ST; ++i)
        if (n_b > i) mbar_wait(&ab_full[i], (uint32_t)(((n_b - 1 - i) / C::AB_ST) & 1), kDefaultWaitLimit);
    }
  } else if (warp < C::MMA_WARP + C::NMMA) {
    // ------------------------------------------------------------- MMA
    // Issuer mi (lane 0 of MMA warp mi) issues the MMAs of the accumulators it
    // owns and commits them: every operand slot and accumulator barrier takes
    // one commit per issuer.
    const int mi = warp - C::MMA_WARP;
    if (lane == 0) {
      int s = 0, ab = 0;
      uint32_t ph = 0, acph = 0;
      bool ok = true;
      // A is MN-major (bit 15), B K-major
      const uint32_t id_real = idesc_f16(p.ab_fmt, C::BO) | (1u << 15);
      const uint32_t id_cplx = idesc_f16(p.ab_fmt, 2 * C::BO) | (1u << 15);
      // Descriptors of slot 0; a byte offset d inside shared memory (< 256 KB)
      // moves the 14-bit start-address field by d >> 4 without a carry out.
      const uint64_t a_desc0 = smem_desc_mn(smem_u32(a_buf), C::A_LBO, C::A_SBO);
      const uint64_t b_desc0 = smem_desc(smem_u32(b_buf), C::B_ROWB);
      for (int ti = 0; ti < my_units && ok; ++ti) {
        const Unit un = unit(ti);
        if (!bwait(&acc_empty[ab], acph ^ 1, limit, abort_flag, p.err, site(K_APPLY, 4, 6), (uint32_t)ti)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem_base + ab * C::ACC_COLS;
        for (int kb = un.kb0; kb < un.kb1; ++kb) {
          if (!bwait(&ab_full[s], ph, limit, abort_flag, p.err, site(K_APPLY, 4, 3), (uint32_t)(ti * nk + kb))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a_d = a_desc0 + (uint64_t)((s * C::A_BYTES) >> 4);
          const uint64_t b_d = b_desc0 + (uint64_t)((s * C::B_BYTES) >> 4);
          const uint32_t first = kb > un.kb0 ? 1u : 0u;
#pragma unroll
          for (int f = 0; f < G::nreal; ++f)
            if (C::own_real(f) == mi)
              mma_f16_ss(acc + f * C::BO, a_d + ((f * C::A_PLANE_BYTES) >> 4), b_d + ((f * C::B_PLANE_BYTES) >> 4),
                         id_real, first);
#pragma unroll
          for (int k = 1; k <= G::ncomplex; ++k) {
            if (C::own_cplx(k) != mi) continue;
            const int pr = G::nreal + 2 * (k - 1);
            const int q = G::nreal + 3 * (k - 1);
            if constexpr (C::GAUSS) {
              // k1 = (Re X + Im X) Re W, k2 = Re X (Im W - Re W), k3 = Im X (Re W + Im W)
              const uint32_t kc = acc + (G::nreal + 3 * (k - 1)) * C::BO;
              mma_f16_ss(kc, a_d + (((T + k - 1) * C::A_PLANE_BYTES) >> 4), b_d + ((q * C::B_PLANE_BYTES) >> 4),
                         id_real, first);
              mma_f16_ss(kc + C::BO, a_d + ((pr * C::A_PLANE_BYTES) >> 4),
                         b_d + (((q + 1) * C::B_PLANE_BYTES) >> 4), id_real, first);
              mma_f16_ss(kc + 2 * C::BO, a_d + (((pr + 1) * C::A_PLANE_BYTES) >> 4),
                         b_d + (((q + 2) * C::B_PLANE_BYTES) >> 4), id_real, first);
              continue;
            }
            const uint32_t col = acc + G::nreal * C::BO + (k - 1) * 2 * C::BO;
            // [Re Y | Im Y] += Re X [Re W ; Im W]
            mma_f16_ss(col, a_d + ((pr * C::A_PLANE_BYTES) >> 4), b_d + (((q + 1) * C::B_PLANE_BYTES) >> 4),
                       id_cplx, first);
            // [Re Y | Im Y] += Im X [-Im W ; Re W]
            mma_f16_ss(col, a_d + (((pr + 1) * C::A_PLANE_BYTES) >> 4), b_d + ((q * C::B_PLANE_BYTES) >> 4),
                       id_cplx, 1u);
          }
          mma_commit(&ab_empty[s]);
          if (++s == C::AB_ST) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[ab]);
        if (++ab == C::NACC) { ab = 0; acph ^= 1; }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      mma_commit(&drain_bar[mi]);         // arrives once every MMA this thread issued has completed
      mbar_wait(&drain_bar[mi], 0, kDefaultWaitLimit);
      // The last commit of each operand slot fires on the same completion as
      // the drain's, and nothing else waits for it: an arrival that lands
      // after the CTA has left would write into the shared memory of whatever
      // the SM runs next.  (On an aborted run, with fewer commits, the
      // wall-time cap ends the wait.)
      const int n_st = my_stages;
      for (int i = 0; i < C::AB_ST; ++i)
        if (n_st > i) mbar_wait(&ab_empty[i], (uint32_t)(((n_st - 1 - i) / C::AB_ST) & 1), kDefaultWaitLimit);
    }
  } else if (STASH && warp == C::STASH_WARP) {
    // --------------------------------------------------------- stash warp
    // Per stage, once the transform has written the A planes: the tiles of
    // output tile 0 store the slot's T planes (each two TMA boxes of 64 tokens
    // x 16 channels, the 128B-swizzled image they already have) to the
    // spectra buffer, and release the slot (its last arrival) once the stores
    // have read it; other tiles release at once.
    if (lane == 0) {
      int s = 0, pend = -1;
      uint32_t ph = 0;
      bool ok = true;
      for (int ti = 0; ti < my_units && ok; ++ti) {
        const Unit un = unit(ti);
        const bool store = un.ot == 0;
        const int m0 = un.tb * C::BM;
        for (int kb = un.kb0; kb < un.kb1; ++kb) {
          if (!bwait(&a_ready[s], ph, limit, abort_flag, p.err, site(K_APPLY, 6, 7), (uint32_t)(ti * nk + kb))) {
            ok = false;
            break;
          }
          if (store) {
            const uint8_t* a_st = a_buf + s * C::A_BYTES;
#pragma unroll
            for (int q = 0; q < T; ++q)
#pragma unroll
              for (int b = 0; b < 2; ++b)
                tma_store_3d(&map_stash, a_st + q * C::A_PLANE_BYTES + b * C::A_LBO, m0 + 64 * b, kb * C::BK, q);
            bulk_commit();
            bulk_wait_read<1>();          // the previous stage's stores have read their slot
            if (pend >= 0) mbar_arrive(&ab_empty[pend]);
            pend = s;
          } else {
            if (pend >= 0) {
              bulk_wait_read<0>();
              mbar_arrive(&ab_empty[pend]);
              pend = -1;
            }
            mbar_arrive(&ab_empty[s]);
          }
          if (++s == C::AB_ST) { s = 0; ph ^= 1; }
        }
      }
      if (pend >= 0) {
        bulk_wait_read<0>();
        mbar_arrive(&ab_empty[pend]);
      }
      if (!ok) raise_abort(abort_flag, p.err);
      bulk_wait<0>();                     // the stores have completed before the CTA exits
    }
  } else {
    // ------------------------------------------------------ epilogue warps
    // Two halves of four warps (one per TMEM lane quarter); half h takes the
    // store chunks h, h+2, ...  Each chunk is 64 output elements of all 128
    // rows: TMEM -> registers -> inverse DFT + bias -> 128B-swizzled staging
    // tile -> one TMA store.
    const int e = warp - C::EPI0;
    const int half = e >> 2;
    const int quarter = warp & 3;                    // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const bool issuer = (e & 3) == 0 && lane == 0;
    int sb = 0;                                      // staging buffer of this half (0/1)
    int ab = 0;
    uint32_t aph = 0;
    bool ok = true;
    for (int ti = 0; ti < my_units; ++ti) {
      const Unit un = unit(ti);
      // this half's copy of the tile's bias, loaded while the MMAs run (the
      // half's previous tile has finished reading it)
      {
        const int ob = un.ot * C::BO;
        for (int i = (e & 3) * 32 + lane; i < C::BO; i += 128)
          s_bias[half * C::BO + i] = (p.bias && ob + i < p.O) ? __ldg(p.bias + ob + i) : 0.f;
      }
      // the four warps of a half share named barriers, so they decide together.
      // In a launch with split tiles all eight decide together on every tile:
      // a split tile's hand-over synchronizes both halves (barrier 3), so
      // neither half may have left the loop while the other goes on.
      const bool w = wwait(&acc_full[ab], aph, limit, abort_flag, lane, p.err, site(K_APPLY, 5, 5), (uint32_t)ti);
      const bool got = p.n_split > 0 ? named_bar_and(3, C::EPI_WARPS * 32, w) : named_bar_and(1 + half, 128, w);
      if (!got) { ok = false; break; }
      tc_fence_after();
      if (un.pair >= 0) {
        // Half of a split tile.  The first of the pair to get here (mode 1)
        // stores its FP32 accumulator in the pair's workspace and raises the
        // pair's ready flag; the second (mode 2) waits for that flag and adds
        // the stored accumulator to its own in TMEM, then stores the tile as
        // usual.  Neither waits for a CTA that has not reached this point.
        if (e == 0 && lane == 0) {
          int md = atomicAdd(p.split_claim + un.pair, 1) == 0 ? 1 : 2;
          if (md == 2 && !flag_wait(p.split_ready + un.pair, 1, limit, abort_flag, p.err, site(K_APPLY, 5, 8),
                                    (uint32_t)un.pair))
            md = -1;
          *split_mode = md;
        }
        named_bar_sync(3, C::EPI_WARPS * 32);
        const int mode = *split_mode;
        if (mode < 0) { ok = false; break; }
        // the pair's accumulator image: [ACC_COLS / 4][128 rows][4 columns].
        // Half h takes the 16-column groups h, h + 2, ... of its rows.
        float4* part = reinterpret_cast<float4*>(p.split_ws) + (size_t)un.pair * (C::ACC_COLS / 4) * C::BM + r;
        const uint32_t acc0 = tmem_base + lane_addr + ab * C::ACC_COLS;
        if (mode == 1) {
#pragma unroll 1
          for (int g = half; g < C::ACC_COLS / 16; g += 2) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(acc0 + 16 * g, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j)
              __stcg(part + (4 * g + j) * C::BM, make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                             __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
          }
          tc_fence_before();
          mbar_arrive(&acc_empty[ab]);
          // every thread's stores are ordered before the flag that hands them over
          __threadfence();
          named_bar_sync(3, C::EPI_WARPS * 32);
          if (e == 0 && lane == 0) st_release_gpu(p.split_ready + un.pair, 1);
          if (++ab == C::NACC) { ab = 0; aph ^= 1; }
          continue;                    // the partner stores the tile
        }
        // mode 2: accumulator += the partner's, in place.  The stored image
        // comes in rounds of MERGE_COLS columns, each one bulk copy into one
        // half of the raw ring, so that a round lands while the previous one
        // is added in (TMEM read, add, TMEM write).  The ring is idle: a
        // split half is its CTA's last unit (units n_whole and on lie in the
        // last wave), and once its MMAs are done every load of the CTA has
        // landed and been read.
        constexpr int RC = C::MERGE_COLS;
        constexpr int NR = C::ACC_COLS / RC;
        constexpr int RB = RC * C::BM * 4;
        const uint8_t* src =
            reinterpret_cast<const uint8_t*>(p.split_ws) + (size_t)un.pair * C::ACC_COLS * C::BM * 4;
        const bool lead = e == 0 && lane == 0;
        int issued = 0;
        auto issue = [&](int rd) {
          mbar_arrive_expect_tx(&merge_bar[rd & 1], RB);
          bulk_load(raw_buf + (rd & 1) * RB, src + (size_t)rd * RB, RB, &merge_bar[rd & 1]);
          ++issued;
        };
        if (lead) {
          // the partner's generic-proxy stores, acquired through the flag,
          // are read by the async proxy (bulk copies)
          fence_proxy_async_all();
          issue(0);
          if (NR > 1) issue(1);
        }
        bool mok = true;
#pragma unroll 1
        for (int rd = 0; rd < NR; ++rd) {
          // every thread reads the copied bytes, so every thread waits (acquire)
          const bool w2 = bwait(&merge_bar[rd & 1], (uint32_t)((rd >> 1) & 1), limit, abort_flag, p.err,
                                site(K_APPLY, 5, 9), (uint32_t)rd);
          mok = named_bar_and(3, C::EPI_WARPS * 32, w2);
          if (!mok) break;
          const float4* buf = reinterpret_cast<const float4*>(raw_buf + (rd & 1) * RB);
#pragma unroll 1
          for (int g = half; g < RC / 16; g += 2) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(acc0 + rd * RC + 16 * g, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 a = buf[(4 * g + j) * C::BM + r];
              v[4 * j] = __float_as_uint(__uint_as_float(v[4 * j]) + a.x);
              v[4 * j + 1] = __float_as_uint(__uint_as_float(v[4 * j + 1]) + a.y);
              v[4 * j + 2] = __float_as_uint(__uint_as_float(v[4 * j + 2]) + a.z);
              v[4 * j + 3] = __float_as_uint(__uint_as_float(v[4 * j + 3]) + a.w);
            }
            tmem_st_32x32b_x16(acc0 + rd * RC + 16 * g, v);
          }
          // this buffer's generic reads are done before the next bulk copy into it
          fence_proxy_async_smem();
          named_bar_sync(3, C::EPI_WARPS * 32);
          if (lead && rd + 2 < NR) issue(rd + 2);
        }
        if (!mok) {
          // no copy may land after the CTA has left
          if (lead)
            for (int q = 0; q < 2; ++q)
              if (issued > q) mbar_wait(&merge_bar[q], (uint32_t)(((issued - 1 - q) / 2) & 1), kDefaultWaitLimit);
          ok = false;
          break;
        }
        // both halves' sums are in TMEM before either reads the other's columns
        tmem_wait_st();
        tc_fence_before();
        named_bar_sync(3, C::EPI_WARPS * 32);
        tc_fence_after();
      }
      const int m0 = un.tb * C::BM;
      const int o0 = un.ot * C::BO;
      const uint32_t acc = tmem_base + lane_addr + ab * C::ACC_COLS;
#pragma unroll 1
      for (int ci = half; ci < C::NCHUNK; ci += 2) {
        uint8_t* stage_tile = o_buf + (half * 2 + sb) * C::OUT_TILE_BYTES;
        uint8_t* my_row = stage_tile + r * C::OUT_ROWB;
        // the TMA store issued from this staging tile two chunks ago must have read it
        if (issuer) bulk_wait_read<1>();
        named_bar_sync(1 + half, 128);
        // the chunk's T planes x CH channels (64 values) in one batch of TMEM loads
        uint32_t rg[T][C::CH];
        if constexpr (C::GAUSS) {
          // real planes, then per complex frequency k1 -> Re slot, k2 -> Im slot, k3 aside
          uint32_t k3[G::ncomplex][C::CH];
#pragma unroll
          for (int q = 0; q < T; ++q) {
            const int k = q < G::nreal ? 0 : 1 + (q - G::nreal) / 2;
            const uint32_t col = acc + ci * C::CH +
                                 (q < G::nreal ? q * C::BO : (G::nreal + 3 * (k - 1) + ((q - G::nreal) & 1)) * C::BO);
#pragma unroll
            for (int h = 0; h < C::CH / 16; ++h) tmem_ld_32x32b_x16(col + 16 * h, &rg[q][16 * h]);
          }
#pragma unroll
          for (int k = 1; k <= G::ncomplex; ++k) {
            const uint32_t col = acc + ci * C::CH + (G::nreal + 3 * (k - 1) + 2) * C::BO;
#pragma unroll
            for (int h = 0; h < C::CH / 16; ++h) tmem_ld_32x32b_x16(col + 16 * h, &k3[k - 1][16 * h]);
          }
          tmem_wait_ld();
#pragma unroll
          for (int k = 1; k <= G::ncomplex; ++k) {
            const int pr = G::nreal + 2 * (k - 1);
#pragma unroll
            for (int j = 0; j < C::CH; ++j) {
              const float k1 = __uint_as_float(rg[pr][j]), k2 = __uint_as_float(rg[pr + 1][j]);
              rg[pr][j] = __float_as_uint(k1 - __uint_as_float(k3[k - 1][j]));     // Re Y
              rg[pr + 1][j] = __float_as_uint(k1 + k2);                            // Im Y
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < T; ++q) {
            const int k = q < G::nreal ? 0 : 1 + (q - G::nreal) / 2;
            const uint32_t col = acc + ci * C::CH +
                                 (q < G::nreal ? q * C::BO
                                               : G::nreal * C::BO + (k - 1) * 2 * C::BO + ((q - G::nreal) & 1) * C::BO);
            if constexpr (C::CH == 8) {
              tmem_ld_32x32b_x8(col, *reinterpret_cast<uint32_t(*)[8]>(&rg[q][0]));
            } else {
#pragma unroll
              for (int h = 0; h < C::CH / 16; ++h) tmem_ld_32x32b_x16(col + 16 * h, &rg[q][16 * h]);
            }
          }
          tmem_wait_ld();
        }
        if (ci + 2 >= C::NCHUNK) {
          // last TMEM read of this tile by this thread: release the accumulator
          tc_fence_before();
          mbar_arrive(&acc_empty[ab]);
        }
#pragma unroll
        for (int sub = 0; sub < C::CH / 8; ++sub) {
          const int oc = ci * C::CH + sub * 8;       // channel offset within the tile
          float bo8[8];
          {
            const float4 b0 = *reinterpret_cast<const float4*>(s_bias + half * C::BO + oc);
            const float4 b1 = *reinterpret_cast<const float4*>(s_bias + half * C::BO + oc + 4);
            bo8[0] = b0.x; bo8[1] = b0.y; bo8[2] = b0.z; bo8[3] = b0.w;
            bo8[4] = b1.x; bo8[5] = b1.y; bo8[6] = b1.z; bo8[7] = b1.w;
          }
          if constexpr (C::POW2) {
            // 8 channels x T outputs = T 16-byte chunks of this row's 128 bytes;
            // chunk v holds the outputs of channels v*8/T .. (v+1)*8/T - 1
#pragma unroll
            for (int v = 0; v < T; ++v) {
              float vals[8];
#pragma unroll
              for (int cc = 0; cc < 8 / T; ++cc) {
                const int c = v * (8 / T) + cc;
                float Pc[T];
#pragma unroll
                for (int q = 0; q < T; ++q) Pc[q] = __uint_as_float(rg[q][sub * 8 + c]);
                G::idft_scaled(Pc, bo8[c], vals + cc * T);
              }
              const int j = sub * T + v;
              *reinterpret_cast<uint4*>(my_row + ((j ^ (r & 7)) << 4)) = pack8<E>(vals);
            }
          } else {
            // T = 3, 6: the 8 channels' 8T outputs, then T 16-byte chunks of
            // consecutive outputs (unswizzled rows of 96 bytes)
            float vals[8 * T];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float Pc[T];
#pragma unroll
              for (int q = 0; q < T; ++q) Pc[q] = __uint_as_float(rg[q][sub * 8 + c]);
              G::idft_scaled(Pc, bo8[c], vals + c * T);
            }
#pragma unroll
            for (int v = 0; v < T; ++v)
              *reinterpret_cast<uint4*>(my_row + (sub * T + v) * 16) = pack8<E>(vals + 8 * v);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1 + half, 128);
        if (issuer) {
          tma_store_2d(&map_out, stage_tile, (o0 + ci * C::CH) * T, m0);
          bulk_commit();
        }
        sb ^= 1;
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
  if (p.n_split > 0 && threadIdx.x == 0) {
    // the last CTA to finish (every other one is past its last use of the
    // pairs' flags) zeroes them for the next launch
    __threadfence();
    if (atomicAdd(p.split_done, 1) == (int)gridDim.x - 1) {
      __threadfence();
      for (int j = 0; j < p.n_split; ++j) {
        p.split_claim[j] = 0;
        p.split_ready[j] = 0;
      }
      *p.split_done = 0;
    }
  }
}

// ------------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
}

template <int T, int BO, typename E, bool STASH, bool GAUSS = false>
static cudaError_t launch_t(const Handle& h, bool backward, const void* in, void* out, void* stash, int64_t N,
                            cudaStream_t st) {
  using C = Cfg<T, BO, STASH, GAUSS>;
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const int K = (int)(backward ? h.Dp : h.Cp);
  const int O = (int)(backward ? h.Cp : h.Dp);
  const CUtensorMapDataType dt = std::is_same<E, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap map_in;      // raw input tiles: 16 channels x T elements x 128 tokens
  {
    cuuint64_t dims[2] = {(cuuint64_t)K * T, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)K * T * 2};
    cuuint32_t box[2] = {(cuuint32_t)(C::BK * T), (cuuint32_t)C::BM};
    cuuint32_t es[2] = {1, 1};
    if (enc(&map_in, dt, 2, const_cast<void*>(in), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  CUtensorMap map_out;     // TMA stores of the output tile, 64 elements x 128 rows, 128B swizzle
  {
    cuuint64_t dims[2] = {(cuuint64_t)O * T, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)O * T * 2};
    cuuint32_t box[2] = {(cuuint32_t)C::OUT_EL, (cuuint32_t)C::BM};
    cuuint32_t es[2] = {1, 1};
    if (enc(&map_out, dt, 2, out, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            C::POW2 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // spectra of the stash forms: [T planes][K channels][ld tokens], TMA stores of
  // 64 tokens x 16 channels x 1 plane, 128B swizzle (the A planes' own image);
  // the token extent N clips the last tile's rows
  CUtensorMap map_stash = map_out;
  if (STASH) {
    const int64_t ld = spectra_ld(N);
    cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)K, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)K * ld * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)C::BK, 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&map_stash, dt, 3, stash, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
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
  p.in = in;
  p.wtiles = GAUSS ? h.wt_gauss : backward ? h.wt_bwd : h.wt_fwd;
  p.bias = backward ? nullptr : h.bias;
  p.err = h.err;
  p.wait_limit = h.wait_limit ? h.wait_limit : kDefaultWaitLimit;
  p.ab_fmt = std::is_same<E, __half>::value ? 0u : 1u;
  // the tail split, where the handle holds a workspace for this pass
  const int pass = backward ? 1 : 0;
  p.n_split = 0;
  p.split_ws = nullptr;
  p.split_claim = p.split_ready = p.split_done = nullptr;
  if (h.split_ws[pass] && C::ACC_COLS <= h.split_cols[pass])
    p.n_split = tc_split_tiles(p.n_tiles, h.sm_count, (K + C::BK - 1) / C::BK, h.split_pairs[pass]);
  if (p.n_split > 0) {
    int* f = h.split_flags[pass];
    p.split_ws = h.split_ws[pass];
    p.split_claim = f;
    p.split_ready = f + h.split_pairs[pass];
    p.split_done = f + 2 * h.split_pairs[pass];
  }

  {
    const cudaError_t e =
        set_smem_limit(reinterpret_cast<const void*>(tc_apply_kernel<T, BO, E, STASH, GAUSS>), C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  const int64_t n_units = p.n_tiles + p.n_split;
  if (n_units > 0x7FFFFFFF) return cudaErrorInvalidValue;     // the kernel counts tiles in 32 bits
  int64_t grid = n_units < h.sm_count ? n_units : h.sm_count;
  if (grid < 1) grid = 1;
  const cudaError_t e = launch_pdl(tc_apply_kernel<T, BO, E, STASH, GAUSS>, dim3((unsigned)grid), dim3(C::THREADS),
                                   C::SMEM_BYTES, st, map_in, map_out, map_stash, p);
  count_launches(1);
  return e;
}

template <int T, int BO, typename E>
static cudaError_t launch_s(const Handle& h, bool bwd, const void* in, void* out, void* stash, int64_t N,
                            cudaStream_t st) {
  return stash ? launch_t<T, BO, E, true>(h, bwd, in, out, stash, N, st)
               : launch_t<T, BO, E, false>(h, bwd, in, out, nullptr, N, st);
}

template <typename E>
static cudaError_t launch_e(const Handle& h, bool bwd, const void* in, void* out, void* stash, int64_t N,
                            cudaStream_t st) {
  const int bo = bwd ? h.bo_bwd : h.bo_fwd;
  switch (h.T) {
    case 1: return bo == 256 ? launch_s<1, 256, E>(h, bwd, in, out, stash, N, st) : cudaErrorInvalidValue;
    case 2: return bo == 128 ? launch_s<2, 128, E>(h, bwd, in, out, stash, N, st) : cudaErrorInvalidValue;
    case 4:
      switch (bo) {
        case 128: return launch_s<4, 128, E>(h, bwd, in, out, stash, N, st);
        case 96: return launch_s<4, 96, E>(h, bwd, in, out, stash, N, st);
        case 64: return launch_s<4, 64, E>(h, bwd, in, out, stash, N, st);
        case 32: return launch_s<4, 32, E>(h, bwd, in, out, stash, N, st);
      }
      return cudaErrorInvalidValue;
    case 8: return bo == 32 ? launch_s<8, 32, E>(h, bwd, in, out, stash, N, st) : cudaErrorInvalidValue;
    // T = 3, 6: no stash form
    case 3: return bo == 128 && !stash ? launch_t<3, 128, E, false>(h, bwd, in, out, nullptr, N, st) : cudaErrorInvalidValue;
    case 6: return bo == 64 && !stash ? launch_t<6, 64, E, false>(h, bwd, in, out, nullptr, N, st) : cudaErrorInvalidValue;
  }
  return cudaErrorInvalidValue;
}

}  // namespace tc

bool tc_supported(const Handle& h, bool backward) {
  if (h.group != EQLIN_GROUP_CYCLIC) return false;
  if (h.dtype != EQLIN_F16 && h.dtype != EQLIN_BF16) return false;
  if (h.T != 1 && h.T != 2 && h.T != 3 && h.T != 4 && h.T != 6 && h.T != 8) return false;
  const int64_t K = backward ? h.Dp : h.Cp;
  // TMA row pitch of the weight planes (K * 2 bytes) must be a 16-byte multiple
  if (K % 8) return false;
  if (!tc::encode_fn()) return false;
  return true;
}

// The p4 forward in the three-product form (the handle's Gauss image).
template <typename E>
static cudaError_t launch_gauss_e(const Handle& h, const void* in, void* out, int64_t N, cudaStream_t st) {
  switch (h.bo_gauss) {
    case 96: return tc::launch_t<4, 96, E, false, true>(h, false, in, out, nullptr, N, st);
    case 64: return tc::launch_t<4, 64, E, false, true>(h, false, in, out, nullptr, N, st);
    case 32: return tc::launch_t<4, 32, E, false, true>(h, false, in, out, nullptr, N, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_tc_apply_gauss(const Handle& h, const void* in, void* out, int64_t N, cudaStream_t st) {
  if (h.T != 4 || !h.wt_gauss) return cudaErrorNotSupported;
  if (h.dtype == EQLIN_F16) return launch_gauss_e<__half>(h, in, out, N, st);
  if (h.dtype == EQLIN_BF16) return launch_gauss_e<__nv_bfloat16>(h, in, out, N, st);
  return cudaErrorNotSupported;
}

cudaError_t launch_tc_apply(const Handle& h, bool backward, const void* in, void* out, void* stash,
                            int64_t N, cudaStream_t st) {
  if (h.dtype == EQLIN_F16) return tc::launch_e<__half>(h, backward, in, out, stash, N, st);
  if (h.dtype == EQLIN_BF16) return tc::launch_e<__nv_bfloat16>(h, backward, in, out, stash, N, st);
  return cudaErrorNotSupported;
}

}  // namespace eqlin
