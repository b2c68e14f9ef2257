// eqlin_tc.cu -- the tcgen05 (5th-generation tensor core) kernel for the
// forward pass and the input gradient, f16/bf16 in, f32 accumulation.
//
// One persistent CTA per SM walks output tiles of 128 tokens x BO output
// channels (all T group positions).  Per tile and per K stage of BK input
// channels:
//
//   producer warp     TMA: the raw input tile [128 x BK*T] (128B swizzle) and
//                     the Fourier weight planes of the stage
//   transform warps   one thread per token row: DFT along t of the raw row
//                     (adds/subtracts; +-sqrt(2)/2 for T = 8), one rounding to
//                     the operand dtype, written as T K-major swizzled operand
//                     planes; then a generic->async proxy fence
//   MMA warp          one thread issues tcgen05.mma into TMEM: for each real
//                     frequency one M=128, N=BO product; for each complex
//                     frequency two M=128, N=2*BO products that accumulate
//                     [Re Y | Im Y] = Re X [Re W ; Im W] + Im X [-Im W ; Re W]
//                     -- R(T) real GEMMs, six for p4
//   epilogue warps    tcgen05.ld of the frequency planes, inverse DFT with the
//                     1/T, bias, cast, 16-byte stores of y[n, d*T+s]
//
// ("Flash EQ-Linear", technical summary, sections "Abordagem Algoritmica",
// "Especializacao para o Grupo de Rotacao p4" and "Implementacao": fused data
// flow, Fourier fragments kept on chip, tensor cores.)  The accumulators are
// double-buffered in TMEM so the epilogue of one tile overlaps the main loop
// of the next.  The input gradient uses the same kernel with the conjugated,
// transposed weight planes and no bias.
//
// Every mbarrier wait is bounded.  A wait that runs out records a timeout in
// the handle's error word, raises a CTA-wide abort flag, and the kernel
// drains its own in-flight TMA copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <type_traits>

#include "eqlin_internal.cuh"
#include "eqlin_ptx.cuh"

namespace eqlin {
namespace tc {

using namespace ptx;

template <int T>
struct Cfg {
  using G = Group<T>;
  static constexpr int BM = 128;                       // tokens per tile (MMA M)
  static constexpr int RAW_EL = 128;                   // raw input elements per row per stage
  static constexpr int BK = RAW_EL / T;                // input channels per stage
  static constexpr int ROWB = (BK * 2 >= 128) ? 128 : BK * 2;   // operand row bytes = swizzle span
  static constexpr int KATOMS = BK * 2 / ROWB;         // swizzle atoms along K (2 for T = 1)
  static constexpr int KSTEPS = BK / 16;               // MMA K = 16 steps per stage
  static constexpr int BO = (256 / T) < 128 ? (256 / T) : 128;   // output channels per tile
  static constexpr int Q = G::nreal + 3 * G::ncomplex; // weight planes per stage
  static constexpr int ACC_COLS = T * BO;              // f32 accumulator columns per tile
  static constexpr int NACC = 2;                       // accumulator buffers
  static constexpr int TMEM_COLS = NACC * ACC_COLS <= 256 ? 256 : 512;
  static constexpr int RAW_SLOTS = 2;
  static constexpr int RAW_BOX_BYTES = BM * 128;       // one 64-element box of 128 rows
  static constexpr int RAW_BYTES = 2 * RAW_BOX_BYTES;
  static constexpr int A_PLANE_BYTES = BM * BK * 2;
  static constexpr int A_BYTES = T * A_PLANE_BYTES;
  static constexpr int B_PLANE_BYTES = BO * BK * 2;
  static constexpr int B_BYTES = Q * B_PLANE_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SMEM_BUDGET = 224 * 1024;
  static constexpr int STAGES_FIT = (SMEM_BUDGET - RAW_SLOTS * RAW_BYTES - 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static_assert(STAGES >= 2, "shared memory too small for two stages");
  static constexpr int NBAR = 2 * RAW_SLOTS + 3 * STAGES + 2 * NACC + 1;
  static constexpr int SMEM_BYTES =
      RAW_SLOTS * RAW_BYTES + STAGES * STAGE_BYTES + NBAR * 8 + 16 + 1024 /*alignment slack*/;
  // swizzle: 16-byte chunk j of row r sits at chunk j ^ ((r >> SW_SHIFT) & SW_MASK)
  static constexpr int SW_BITS = ROWB == 128 ? 3 : ROWB == 64 ? 2 : 1;
  static constexpr int SW_SHIFT = 3 - SW_BITS;
  static constexpr int SW_MASK = (1 << SW_BITS) - 1;
  static constexpr int THREADS = 320;                  // producer, MMA, 4 transform, 4 epilogue warps
};

struct Params {
  int64_t N;       // tokens
  int K;           // input channels per group element (C' forward, D' for dx)
  int O;           // output channels per group element
  int n_otiles;
  int64_t n_tiles;
  const float* bias;   // nullptr: none
  void* out;
  int* err;
  uint32_t wait_limit;
  uint32_t ab_fmt;     // 0 f16, 1 bf16
};

// Bounded wait that also gives up as soon as another role raised the abort flag.
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

// Every lane polls (each needs the acquire); the warp agrees on the outcome so
// that no lane leaves a loop that holds warp-synchronous operations.
__device__ __forceinline__ bool wwait(uint64_t* bar, uint32_t parity, uint32_t limit,
                                      volatile int* abort_flag) {
  return __all_sync(0xffffffffu, bwait(bar, parity, limit, abort_flag));
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* err) {
  *abort_flag = 1;
  atomicCAS(err, DEV_OK, DEV_TIMEOUT);
}

template <typename E>
__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const E* e = reinterpret_cast<const E*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = Elem<E>::to_f(e[i]);
}

template <typename E>
__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  E* e = reinterpret_cast<E*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) e[i] = Elem<E>::from_f(f[i]);
  return u;
}

template <int T, typename E>
__global__ void __launch_bounds__(Cfg<T>::THREADS, 1)
tc_apply_kernel(const __grid_constant__ CUtensorMap map_in, const __grid_constant__ CUtensorMap map_w,
                Params p) {
  using C = Cfg<T>;
  using G = Group<T>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128B-swizzled tiles
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* raw_buf = smem;
  uint8_t* a_buf = raw_buf + C::RAW_SLOTS * C::RAW_BYTES;
  uint8_t* b_buf = a_buf + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_buf + C::STAGES * C::B_BYTES);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + C::RAW_SLOTS;
  uint64_t* a_full = raw_empty + C::RAW_SLOTS;
  uint64_t* b_full = a_full + C::STAGES;
  uint64_t* ab_empty = b_full + C::STAGES;
  uint64_t* acc_full = ab_empty + C::STAGES;
  uint64_t* acc_empty = acc_full + C::NACC;
  uint64_t* drain_bar = acc_empty + C::NACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t limit = p.wait_limit;
  const int nk = (p.K + C::BK - 1) / C::BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::RAW_SLOTS; ++i) { mbar_init(&raw_full[i], 1); mbar_init(&raw_empty[i], 4); }
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&a_full[i], 4);
      mbar_init(&b_full[i], 1);
      mbar_init(&ab_empty[i], 1);
    }
    for (int i = 0; i < C::NACC; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 128); }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&map_in);
    prefetch_tensormap(&map_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int rs = 0, s = 0;
      uint32_t rph = 0, ph = 0;
      int64_t n_raw = 0, n_b = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
        const int m0 = (int)(tile / p.n_otiles) * C::BM;
        const int o0 = (int)(tile % p.n_otiles) * C::BO;
        for (int kb = 0; kb < nk; ++kb) {
          if (!bwait(&raw_empty[rs], rph ^ 1, limit, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&raw_full[rs], C::RAW_BYTES);
          uint8_t* dst = raw_buf + rs * C::RAW_BYTES;
          tma_load_2d(dst, &map_in, kb * C::RAW_EL, m0, &raw_full[rs]);
          tma_load_2d(dst + C::RAW_BOX_BYTES, &map_in, kb * C::RAW_EL + 64, m0, &raw_full[rs]);
          ++n_raw;
          if (++rs == C::RAW_SLOTS) { rs = 0; rph ^= 1; }

          if (!bwait(&ab_empty[s], ph ^ 1, limit, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&b_full[s], C::B_BYTES);
          uint8_t* bdst = b_buf + s * C::B_BYTES;
#pragma unroll
          for (int q = 0; q < C::Q; ++q)
#pragma unroll
            for (int a = 0; a < C::KATOMS; ++a)
              tma_load_3d(bdst + q * C::B_PLANE_BYTES + a * (C::BO * 128), &map_w,
                          kb * C::BK + a * 64, o0, q, &b_full[s]);
          ++n_b;
          if (++s == C::STAGES) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      {
        // drain: every issued TMA copy must land before the CTA exits (a
        // no-op on the normal path, where the consumers already waited)
        for (int i = 0; i < C::RAW_SLOTS; ++i)
          if (n_raw > i) mbar_wait(&raw_full[i], (uint32_t)(((n_raw - 1 - i) / C::RAW_SLOTS) & 1), kDefaultWaitLimit);
        for (int i = 0; i < C::STAGES; ++i)
          if (n_b > i) mbar_wait(&b_full[i], (uint32_t)(((n_b - 1 - i) / C::STAGES) & 1), kDefaultWaitLimit);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA
    if (lane == 0) {
      int s = 0, ab = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      const uint32_t id_real = idesc_f16(p.ab_fmt, C::BO);
      const uint32_t id_cplx = idesc_f16(p.ab_fmt, 2 * C::BO);
      for (int64_t tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
        if (!bwait(&acc_empty[ab], aph ^ 1, limit, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc = tmem_base + ab * C::ACC_COLS;
        for (int kb = 0; kb < nk; ++kb) {
          if (!bwait(&a_full[s], ph, limit, abort_flag) || !bwait(&b_full[s], ph, limit, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_st = smem_u32(a_buf + s * C::A_BYTES);
          const uint32_t b_st = smem_u32(b_buf + s * C::B_BYTES);
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            const int atom = (ks * 32) / C::ROWB;
            const uint32_t koff = (ks * 32) % C::ROWB;
            const uint32_t a_k = a_st + atom * (C::BM * 128) + koff;
            const uint32_t b_k = b_st + atom * (C::BO * 128) + koff;
            const uint32_t first = (kb > 0 || ks > 0) ? 1u : 0u;
#pragma unroll
            for (int f = 0; f < G::nreal; ++f)
              mma_f16_ss(acc + f * C::BO, smem_desc(a_k + f * C::A_PLANE_BYTES, C::ROWB),
                         smem_desc(b_k + f * C::B_PLANE_BYTES, C::ROWB), id_real, first);
#pragma unroll
            for (int k = 1; k <= G::ncomplex; ++k) {
              const int pr = G::nreal + 2 * (k - 1);
              const int q = G::nreal + 3 * (k - 1);
              const uint32_t col = acc + G::nreal * C::BO + (k - 1) * 2 * C::BO;
              // [Re Y | Im Y] += Re X [Re W ; Im W]
              mma_f16_ss(col, smem_desc(a_k + pr * C::A_PLANE_BYTES, C::ROWB),
                         smem_desc(b_k + (q + 1) * C::B_PLANE_BYTES, C::ROWB), id_cplx, first);
              // [Re Y | Im Y] += Im X [-Im W ; Re W]
              mma_f16_ss(col, smem_desc(a_k + (pr + 1) * C::A_PLANE_BYTES, C::ROWB),
                         smem_desc(b_k + q * C::B_PLANE_BYTES, C::ROWB), id_cplx, 1u);
            }
          }
          mma_commit(&ab_empty[s]);
          if (++s == C::STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[ab]);
        if (++ab == C::NACC) { ab = 0; aph ^= 1; }
      }
      if (!ok) raise_abort(abort_flag, p.err);
      mma_commit(drain_bar);              // arrives once every issued MMA has completed
      mbar_wait(drain_bar, 0, kDefaultWaitLimit);
    }
  } else if (warp < 6) {
    // ----------------------------------------------------- transform warps
    const int r = (warp - 2) * 32 + lane;            // token row within the tile
    int rs = 0, s = 0;
    uint32_t rph = 0, ph = 0;
    bool ok = true;
    const int swz = (r >> C::SW_SHIFT) & C::SW_MASK;
    for (int64_t tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < nk; ++kb) {
        if (!wwait(&raw_full[rs], rph, limit, abort_flag) || !wwait(&ab_empty[s], ph ^ 1, limit, abort_flag)) {
          ok = false;
          break;
        }
        const uint8_t* rrow = raw_buf + rs * C::RAW_BYTES + r * 128;
        uint8_t* a_st = a_buf + s * C::A_BYTES;
        // 8 channels (one 16-byte operand chunk per plane) at a time
#pragma unroll
        for (int g = 0; g < C::BK / 8; ++g) {
          float v[8 * T];
#pragma unroll
          for (int cch = 0; cch < T; ++cch) {
            const int chunk = g * T + cch;           // 16-byte chunk of the 256-byte raw row
            const int box = chunk >> 3, j = chunk & 7;
            const uint4 u = *reinterpret_cast<const uint4*>(rrow + box * C::RAW_BOX_BYTES + ((j ^ (r & 7)) << 4));
            unpack8<E>(u, v + 8 * cch);
          }
          float P[T][8];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float Pc[T];
            G::dft(v + c * T, Pc);
#pragma unroll
            for (int q = 0; q < T; ++q) P[q][c] = Pc[q];
          }
          const int atom = (g * 16) / C::ROWB;
          const int j = g % (C::ROWB / 16);
#pragma unroll
          for (int q = 0; q < T; ++q) {
            uint8_t* dst = a_st + q * C::A_PLANE_BYTES + atom * (C::BM * 128) + r * C::ROWB +
                           ((j ^ swz) << 4);
            *reinterpret_cast<uint4*>(dst) = pack8<E>(P[q]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&raw_empty[rs]);
          mbar_arrive(&a_full[s]);
        }
        if (++rs == C::RAW_SLOTS) { rs = 0; rph ^= 1; }
        if (++s == C::STAGES) { s = 0; ph ^= 1; }
      }
    }
    if (!ok) raise_abort(abort_flag, p.err);
  } else {
    // ------------------------------------------------------ epilogue warps
    const int quarter = warp & 3;                    // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    int ab = 0;
    uint32_t aph = 0;
    bool ok = true;
    E* out = reinterpret_cast<E*>(p.out);
    for (int64_t tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x) {
      if (!wwait(&acc_full[ab], aph, limit, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const int64_t row = (tile / p.n_otiles) * C::BM + r;
      const int o0 = (int)(tile % p.n_otiles) * C::BO;
      const uint32_t acc = tmem_base + lane_addr + ab * C::ACC_COLS;
#pragma unroll 1
      for (int oc = 0; oc < C::BO; oc += 8) {
        uint32_t rg[T][8];
#pragma unroll
        for (int f = 0; f < G::nreal; ++f) tmem_ld_32x32b_x8(acc + f * C::BO + oc, rg[f]);
#pragma unroll
        for (int k = 1; k <= G::ncomplex; ++k) {
          const uint32_t col = acc + G::nreal * C::BO + (k - 1) * 2 * C::BO + oc;
          tmem_ld_32x32b_x8(col, rg[G::nreal + 2 * (k - 1)]);
          tmem_ld_32x32b_x8(col + C::BO, rg[G::nreal + 2 * (k - 1) + 1]);
        }
        tmem_wait_ld();
        const int o = o0 + oc;
        if (row < p.N && o < p.O) {
          float vals[8 * T];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float Pc[T], yc[T];
#pragma unroll
            for (int q = 0; q < T; ++q) Pc[q] = __uint_as_float(rg[q][c]);
            G::idft(Pc, yc);
            const float bo = (p.bias && o + c < p.O) ? __ldg(p.bias + o + c) : 0.f;
#pragma unroll
            for (int s_ = 0; s_ < T; ++s_) vals[c * T + s_] = yc[s_] + bo;
          }
          E* dst = out + row * (int64_t)p.O * T + (int64_t)o * T;
          if (o + 8 <= p.O) {
#pragma unroll
            for (int v = 0; v < T; ++v)
              reinterpret_cast<uint4*>(dst)[v] = pack8<E>(vals + 8 * v);
          } else {
            const int nvalid = (p.O - o) * T;
#pragma unroll
            for (int i = 0; i < 8 * T; ++i)
              if (i < nvalid) dst[i] = Elem<E>::from_f(vals[i]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
      if (++ab == C::NACC) { ab = 0; aph ^= 1; }
    }
    if (!ok) raise_abort(abort_flag, p.err);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

static CUtensorMapSwizzle swz_enum(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
       : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
}

template <int T, typename E>
static cudaError_t launch_t(const Handle& h, bool backward, const void* in, void* out, int64_t N,
                            cudaStream_t st) {
  using C = Cfg<T>;
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const int K = (int)(backward ? h.Dp : h.Cp);
  const int O = (int)(backward ? h.Cp : h.Dp);
  const CUtensorMapDataType dt = std::is_same<E, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap map_in, map_w;
  {
    cuuint64_t dims[2] = {(cuuint64_t)K * T, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)K * T * 2};
    cuuint32_t box[2] = {64, C::BM};
    cuuint32_t es[2] = {1, 1};
    if (enc(&map_in, dt, 2, const_cast<void*>(in), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)O, (cuuint64_t)C::Q};
    cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)K * O * 2};
    cuuint32_t box[3] = {(cuuint32_t)(C::ROWB / 2), (cuuint32_t)C::BO, 1};
    cuuint32_t es[3] = {1, 1, 1};
    void* wptr = backward ? h.wt_bwd : h.wt_fwd;
    if (enc(&map_w, dt, 3, wptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swz_enum(C::ROWB), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  Params p;
  p.N = N;
  p.K = K;
  p.O = O;
  p.n_otiles = (O + C::BO - 1) / C::BO;
  p.n_tiles = ((N + C::BM - 1) / C::BM) * p.n_otiles;
  p.bias = backward ? nullptr : h.bias;
  p.out = out;
  p.err = h.err;
  p.wait_limit = h.wait_limit ? h.wait_limit : kDefaultWaitLimit;
  p.ab_fmt = std::is_same<E, __half>::value ? 0u : 1u;

  static bool attr_set = false;   // per template instance
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(tc_apply_kernel<T, E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int64_t grid = p.n_tiles < h.sm_count ? p.n_tiles : h.sm_count;
  if (grid < 1) grid = 1;
  tc_apply_kernel<T, E><<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, st>>>(map_in, map_w, p);
  count_launches(1);
  return cudaGetLastError();
}

template <typename E>
static cudaError_t launch_e(const Handle& h, bool bwd, const void* in, void* out, int64_t N,
                            cudaStream_t st) {
  switch (h.T) {
    case 1: return launch_t<1, E>(h, bwd, in, out, N, st);
    case 2: return launch_t<2, E>(h, bwd, in, out, N, st);
    case 4: return launch_t<4, E>(h, bwd, in, out, N, st);
    case 8: return launch_t<8, E>(h, bwd, in, out, N, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tc

bool tc_supported(const Handle& h, bool backward) {
  if (h.dtype != EQLIN_F16 && h.dtype != EQLIN_BF16) return false;
  if (h.T != 1 && h.T != 2 && h.T != 4 && h.T != 8) return false;
  const int64_t K = backward ? h.Dp : h.Cp;
  // TMA row pitch of the weight planes (K * 2 bytes) must be a 16-byte multiple
  if (K % 8) return false;
  if (!tc::encode_fn()) return false;
  return true;
}

cudaError_t launch_tc_apply(const Handle& h, bool backward, const void* in, void* out, int64_t N,
                            cudaStream_t st) {
  if (h.dtype == EQLIN_F16) return tc::launch_e<__half>(h, backward, in, out, N, st);
  if (h.dtype == EQLIN_BF16) return tc::launch_e<__nv_bfloat16>(h, backward, in, out, N, st);
  return cudaErrorNotSupported;
}

}  // namespace eqlin
