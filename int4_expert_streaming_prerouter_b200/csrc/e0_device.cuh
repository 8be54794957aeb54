// Device-side helpers shared by the kernels of libe0moe.so (sm_100a).
//
// Number formats and the int4 affine group-64 expert format follow the model
// description of "The Other Half of the Memory Wall" (reading guide, "Temel fikirler")
// and the ai.info article "Edge0 serve un MoE da 35B ..." ("La versione da 35B usa 256
// esperti distribuiti su 40 livelli"): w = scale * q + min, q = 0..15, groups of 64
// along K, element 2i in the low nibble of byte i, bf16 scale and min.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace e0 {

// Device error codes latched in the context's error word (bit flags).
enum : int {
  DERR_INDEX = 1,      // an expert index outside [0, E)
  DERR_DUP = 2,        // the same expert twice in one token's selection
  DERR_SLOT = 4,       // a pool slot holds another expert than the slot table promises
  DERR_TIMEOUT = 8,    // a bounded wait gave up
};

// Byte offsets of the nine sections of one expert blob.
struct Blob {
  long long gc, gs, gm, uc, us, um, dc, ds, dm, bytes;
};

__host__ __device__ inline Blob blob_of(int d, int I) {
  Blob b;
  long long o = 0;
  const long long codes_gu = (long long)I * d / 2, sm_gu = (long long)I * (d / 64) * 2;
  const long long codes_dn = (long long)d * I / 2, sm_dn = (long long)d * (I / 64) * 2;
  b.gc = o; o += codes_gu; b.gs = o; o += sm_gu; b.gm = o; o += sm_gu;
  b.uc = o; o += codes_gu; b.us = o; o += sm_gu; b.um = o; o += sm_gu;
  b.dc = o; o += codes_dn; b.ds = o; o += sm_dn; b.dm = o; o += sm_dn;
  b.bytes = o;
  return b;
}

__device__ __forceinline__ float bf(uint32_t bits) { return __uint_as_float(bits << 16); }

__device__ __forceinline__ uint16_t f2bf(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Round a double to the nearest bfloat16 (ties to even) directly, without passing
// through binary32: a bfloat16 keeps 8 significant bits, so for |v| in [2^(e-1), 2^e)
// the spacing is 2^(e-8) (2^-133 below the smallest normal).
// Results in the normal range take the integer form of the same rounding on the double's
// bits: add 2^44 - 1 plus the kept lowest bit (bit 45) and keep the top 16 bits of the
// re-biased exponent and 7 mantissa bits (a mantissa carry moves into the exponent).
__device__ __forceinline__ uint16_t d2bf(double v) {
  unsigned long long b = (unsigned long long)__double_as_longlong(v);
  const int eb = (int)((b >> 52) & 0x7FF) - 1023 + 127;   // binary32 biased exponent
  if (eb >= 1 && eb <= 254) {
    b += (1ull << 44) - 1 + ((b >> 45) & 1ull);
    const int e2 = (int)((b >> 52) & 0x7FF) - 1023 + 127;
    const uint32_t sgn = (uint32_t)(b >> 63) << 15;
    if (e2 >= 255) return (uint16_t)(sgn | 0x7F80u);      // rounds past the largest: infinity
    return (uint16_t)(sgn | ((uint32_t)e2 << 7) | (uint32_t)((b >> 45) & 0x7Full));
  }
  if (v == 0.0) return (uint16_t)((unsigned long long)__double_as_longlong(v) >> 48);
  int e = ilogb(v) + 1;
  if (e < -125) e = -125;
  const double r = scalbn(rint(scalbn(v, 8 - e)), e - 8);
  return (uint16_t)(__float_as_uint((float)r) >> 16);
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over aligned groups of `width` lanes (width a power of two <= 32).
__device__ __forceinline__ float group_sum(float v, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// int4 value q (0..15) as an exact float: 2^23 + q has q in its low mantissa bits.
__device__ __forceinline__ float q2f(uint32_t q) {
  return __uint_as_float(0x4B000000u | q) - 8388608.0f;
}

// One 16-byte chunk of an int4 row (32 consecutive K elements, half a group) dotted
// with 32 fp32 activations: sum_k (s q_k + m) x_k = s * sum_k q_k x_k + m * sum_k x_k.
// Word t of the chunk holds elements 8t..8t+7; its nibble i (bits 4i..4i+3) is element
// 8t+i (byte i/2, low nibble when i is even).
__device__ __forceinline__ float chunk_dot(const uint4 w, const float *__restrict__ x, float s,
                                           float m) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  float qx = 0.f, sx = 0.f;
#pragma unroll
  for (int t = 0; t < 4; t++) {
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float xv = x[8 * t + i];
      qx = fmaf(q2f((ws[t] >> (4 * i)) & 0xFu), xv, qx);
      sx += xv;
    }
  }
  return fmaf(s, qx, m * sx);
}

// Same, with the 32 activations given as bf16 (16 x uint32 pairs, element 2p in the
// low half of pair p).
__device__ __forceinline__ float chunk_dot_bf16x(const uint4 w, const uint32_t *__restrict__ xp,
                                                 float s, float m) {
  float x[32];
#pragma unroll
  for (int p = 0; p < 16; p++) {
    x[2 * p] = __uint_as_float(xp[p] << 16);
    x[2 * p + 1] = __uint_as_float(xp[p] & 0xFFFF0000u);
  }
  return chunk_dot(w, x, s, m);
}

// Packed pairs of fp32 (low word = first element) and the f32x2 arithmetic on them.
__device__ __forceinline__ unsigned long long pk2(float a, float b) {
  return ((unsigned long long)__float_as_uint(b) << 32) | __float_as_uint(a);
}
__device__ __forceinline__ unsigned long long f2fma(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2add(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float f2sum(unsigned long long v) {
  return __uint_as_float((uint32_t)v) + __uint_as_float((uint32_t)(v >> 32));
}

}  // namespace e0
