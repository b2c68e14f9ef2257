// eqlin_packed.cuh -- group DFT of two tokens at once on packed 16-bit pairs.
//
// A transform thread owns one channel and walks over tokens.  For T in
// {1, 2, 4} the forward real DFT along the group axis needs only additions
// and subtractions ("Flash EQ-Linear", technical summary, section
// "Especializacao para o Grupo de Rotacao p4": dyadic coefficients), so it
// is computed on packed pairs (value of token n, value of token n+1) with
// f16x2 / bf16x2 arithmetic.  The result words are already the pairs of
// consecutive tokens that a token-contiguous (K-major or MN-major) operand
// stores, so a plane of 8 tokens is four words: one 16-byte store.
//
// Each butterfly level rounds to the operand type (p4: X0 and X2 take two
// levels, Re X1 and Im X1 one), where an FP32 transform would round once at
// the end; the extra error is within half an ulp of the operand type per level.
#pragma once

#include "eqlin_internal.cuh"

namespace eqlin {
namespace packed {

template <typename E> struct Pair;
template <> struct Pair<__half> {
  static __device__ __forceinline__ uint32_t add(uint32_t a, uint32_t b) {
    __half2 r = __hadd2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static __device__ __forceinline__ uint32_t sub(uint32_t a, uint32_t b) {
    __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static __device__ __forceinline__ float2 to_f2(uint32_t a) {
    return __half22float2(*reinterpret_cast<const __half2*>(&a));
  }
};
template <> struct Pair<__nv_bfloat16> {
  static __device__ __forceinline__ uint32_t add(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hadd2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                               *reinterpret_cast<const __nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static __device__ __forceinline__ uint32_t sub(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                               *reinterpret_cast<const __nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static __device__ __forceinline__ float2 to_f2(uint32_t a) {
    return make_float2(__uint_as_float(a << 16), __uint_as_float(a & 0xffff0000u));
  }
};

// Flip the sign of both halves (exact negation).
__device__ __forceinline__ uint32_t neg2(uint32_t a) { return a ^ 0x80008000u; }

// (low half of a, low half of b) and (high half of a, high half of b)
__device__ __forceinline__ uint32_t lo_lo(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x5410); }
__device__ __forceinline__ uint32_t hi_hi(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x7632); }

// Number of 32-bit words holding the T group values of one channel of one token.
template <int T> struct Words { static constexpr int n = T >= 2 ? T / 2 : 1; };

// Planes of the real DFT for tokens n (wa) and n+1 (wb), in the plane order of
// Group<T>: T=1 [X0]; T=2 [X0, X1]; T=4 [X0, X2, Re X1, Im X1].
// For T = 1 the single 16-bit value sits in the low half of wa[0] / wb[0].
template <int T, typename E>
__device__ __forceinline__ void dft_pair(const uint32_t* wa, const uint32_t* wb, uint32_t* P) {
  using A = Pair<E>;
  static_assert(T == 1 || T == 2 || T == 4, "packed DFT covers T in {1, 2, 4}");
  if constexpr (T == 1) {
    P[0] = lo_lo(wa[0], wb[0]);
  } else if constexpr (T == 2) {
    const uint32_t v0 = lo_lo(wa[0], wb[0]), v1 = hi_hi(wa[0], wb[0]);
    P[0] = A::add(v0, v1);
    P[1] = A::sub(v0, v1);
  } else {
    const uint32_t v0 = lo_lo(wa[0], wb[0]), v1 = hi_hi(wa[0], wb[0]);
    const uint32_t v2 = lo_lo(wa[1], wb[1]), v3 = hi_hi(wa[1], wb[1]);
    const uint32_t s02 = A::add(v0, v2), s13 = A::add(v1, v3);
    P[0] = A::add(s02, s13);      // X0 = x0 + x1 + x2 + x3
    P[1] = A::sub(s02, s13);      // X2 = x0 - x1 + x2 - x3
    P[2] = A::sub(v0, v2);        // Re X1 = x0 - x2
    P[3] = A::sub(v3, v1);        // Im X1 = x3 - x1
  }
}

// Load the Words<T> words of one channel of one token (a single vector load).
template <int T>
__device__ __forceinline__ void load_words(const void* p, uint32_t* w) {
  if constexpr (T == 8) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
  } else if constexpr (T == 4) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = u.x; w[1] = u.y;
  } else if constexpr (T == 2) {
    w[0] = __ldg(reinterpret_cast<const unsigned int*>(p));
  } else {
    w[0] = __ldg(reinterpret_cast<const unsigned short*>(p));
  }
}

}  // namespace packed
}  // namespace eqlin
