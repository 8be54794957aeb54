// Prefill path: the experts of one MoE block on many tokens as grouped GEMMs on the
// 5th-generation tensor cores (tcgen05.mma, fp32 accumulators in tensor memory).
//
// Method ([G] "Birleştirilmemiş Adaptör Yürütme"; [A] int4 affine g64 experts, SwiGLU):
//   gate/up:  G = Dq(W_gu) X_e^T  (per expert e, tokens routed to e), a = bf16(silu(g) u),
//             the shared expert adds c * B (A x) to g and u first;
//   down:     Y_e = Dq(W_d) A_e^T, y[t] += w_{t,j} Y_e[:, t]  (w = 1 for the shared expert).
//
// B200 design.  One CTA = one 128-row weight tile of one expert x up to 128 tokens.  Eight
// warps produce each 64-wide K block: two threads per weight row dequantise the int4 tile
// to fp16 (w = s q + m, one group of 64 per row per K block) and the token rows (fp16) are
// gathered beside it, both written into shared memory in the 128-byte-swizzled K-major
// layout the tensor core reads; each thread's global loads for the next K block are
// issued before it works on the current one.  One thread issues four tcgen05.mma (M=128, N=tokens, K=16 each) per K block
// into a TMEM accumulator and commits to an mbarrier that frees the stage; four stages are
// in flight.  The epilogue reads TMEM with tcgen05.ld and applies SwiGLU (gate rows 0..63
// and up rows 64..127 of the tile are the same intermediate units) or the gate-weighted
// combine (fp32 atomics into y).  Each dequantised weight is split into two fp16 values
// (hi = fp16(w), lo = fp16(w - hi)) and both are multiplied into the same accumulator, so
// the weights keep ~22 significant bits (one fp16 alone keeps 11, which leaves a ~2e-3
// relative error at the tail of a 40k-output layer); x and a are bf16 values, exactly
// representable in fp16 in their range.
#pragma once
#include <cuda_fp16.h>
#include "e0_device.cuh"
#include "e0_kernels.cuh"

namespace e0 {

constexpr int kTcThreads = 256;
constexpr int kTcMinTokens = 64;    // contexts with at least this many tokens get the tensor-core path
constexpr int kTcN = 128;           // tokens per tile (TMEM columns per accumulator)
constexpr int kTcRawStages = 8;     // int4 code tiles of a K group (4 KB each) in the ring
constexpr int kTcRawAhead = 7;      //   groups loaded ahead of the one being converted
constexpr int kTcBStages = 4;       // activation tiles (16 KB each)
constexpr int kTcBAhead = 3;
constexpr int kTcMaxGroups = 64;    // K / 64 <= 64 (K <= 4096)

struct TcTile {
  int unit;      // unique expert index (== U: the shared expert)
  int n0;        // first token position within the unit's token list
};

struct TcArgs {
  int mode;                 // 0: gate/up + SwiGLU, 1: down + weighted combine
  int T, d, I, k, r;
  float c;
  ExpertSrc src;
  const uint8_t *shared;
  Blob bl;
  Plan P;
  const TcTile *tiles;      // [ntiles]
  const int *ntiles;
  const uint16_t *xp;       // [T, d] x, bf16, K-permuted within 8-blocks (mode 0)
  const float *xsum;        // [T, d/64] group sums of x (mode 0)
  const uint16_t *ap;       // [T, k+1, I] a, bf16, K-permuted (mode 1 input)
  const float *asum;        // [T, k+1, I/64] group sums of a (mode 1)
  uint16_t *ap_out;         // [T, k+1, I] (mode 0 output)
  const uint16_t *Bg, *Bu;  // [I, r] shared-expert LoRA up (mode 0), or nullptr
  const float *lt;          // [T, 3, r]
  const float *gates;       // [T, k] (mode 1)
  float *yacc;              // [T, d] (mode 1)
  int *err;
  unsigned long long timeout_ns;
};

// Position of natural element e of an 8-block in the K-permuted order of the tensor-core
// operands: the block is stored as elements (0,4,1,5,2,6,3,7), the order in which one
// 32-bit word of int4 codes unpacks into four bf16 pairs.
__host__ __device__ __forceinline__ int kperm_pos(int e) { return (e & ~7) | ((e & 3) << 1) | ((e >> 2) & 1); }

// ---------------------------------------------------------------------------------------
// tcgen05 / TMEM helpers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t tc_smem(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row groups 1024 B
// apart.  Fields: start address >> 4 (bits 0-13), leading byte offset >> 4 (16-29, unused
// for swizzled K-major), stride byte offset >> 4 (32-45), descriptor version 1 (46-47),
// base offset 0 (49-51), layout type 2 = 128-byte swizzle (61-63).
__device__ __forceinline__ unsigned long long tc_desc(uint32_t saddr) {
  return (unsigned long long)((saddr >> 4) & 0x3FFFu) | ((unsigned long long)(16u >> 4) << 16) |
         ((unsigned long long)(1024u >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and B bf16
// (bits 7-9 and 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 (bits 17-22), M >> 4
// (bits 24-28).
__device__ __forceinline__ uint32_t tc_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// 16-byte asynchronous global -> shared copy; src_bytes = 0 fills the 16 bytes with zeros.
__device__ __forceinline__ void tc_cp16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void tc_cp4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// the mbarrier receives one arrival once every cp.async this thread issued so far has landed
__device__ __forceinline__ void tc_cp_arrive(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc_smem(bar)) : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, unsigned long long ad, unsigned long long bd, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(tc_smem(bar))
               : "memory");
}

__device__ __forceinline__ void tc_mbar_init(uint64_t *b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(tc_smem(b)), "r"(count) : "memory");
}

__device__ __forceinline__ bool tc_mbar_test(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(tc_smem(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long tc_now() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// bounded wait on an mbarrier phase; false (and the error word set) when the budget ends
__device__ __forceinline__ bool tc_wait(uint64_t *b, uint32_t parity, const TcArgs &A) {
  unsigned long long t0 = 0;
  while (!tc_mbar_test(b, parity)) {
    const unsigned long long now = tc_now();
    if (!t0) t0 = now;
    else if (now - t0 > A.timeout_ns) {
      atomicOr(A.err, DERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// 32 TMEM columns of this warp's 32 lanes into registers (lane i of the warp reads TMEM
// lane 32*(warp%4) + i).
__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

// byte offset of 16-byte chunk `ch` (0..7) of row `row` in a 128-byte-swizzled K-major tile
__device__ __forceinline__ uint32_t sw128(int row, int ch) {
  return (uint32_t)(row * 128 + ((ch ^ (row & 7)) << 4));
}


// bounded wait of every thread on a cp.async / MMA completion phase; false once the
// budget is spent (error word set)
__device__ __forceinline__ bool tc_wait_all(uint64_t *b, uint32_t parity, unsigned long long budget, int *err) {
  unsigned long long t0 = 0;
  while (!tc_mbar_test(b, parity)) {
    const unsigned long long now = tc_now();
    if (!t0) t0 = now;
    else if (now - t0 > budget) {
      atomicOr(err, DERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------------------------------
// Tile list: every unique routed expert (its token list) and the shared expert (all T
// tokens) cut into tiles of up to kTcN tokens.  One block.
// ---------------------------------------------------------------------------------------
__global__ void k_tc_tiles(Plan P, int T, TcTile *tiles, int *ntiles, int cap) {
  if (threadIdx.x != 0) return;
  const int U = P.U[0];
  int n = 0;
  for (int u = 0; u <= U && n < cap; u++) {
    const int cnt = u < U ? P.ustart[u + 1] - P.ustart[u] : T;
    for (int n0 = 0; n0 < cnt && n < cap; n0 += kTcN) tiles[n++] = TcTile{u, n0};
  }
  *ntiles = n;
}

// ---------------------------------------------------------------------------------------
// The grouped expert GEMM.  One CTA = one 128-row weight tile of one expert x up to kTcN
// tokens; grid = max tiles x M tiles per expert (blocks past the real tile count return).
//
// Per K group g of 64 (the quantisation group), with A = the int4 codes as bf16 (128 + q,
// exact) and B = the tokens' activations (bf16, exact):
//   P_g = sum_{k in g} (128 + q_k) x_k           tcgen05.mma into TMEM buffer g % 2
//   acc += s_g * P_g + (m_g - 128 s_g) * X_g      CUDA cores, X_g = sum_{k in g} x_k
// which is sum_k (s_g q_k + m_g) x_k, the affine dequantisation folded into the
// accumulation; so the weights need no fp32 dequantisation and one MMA per K = 16.
// The MMA of group g overlaps the fold of group g - 1 and the conversion of group g + 1.
// Codes and activations stream into shared memory through cp.async rings whose stages
// complete on mbarriers, so loads run several groups ahead of their use.
// ---------------------------------------------------------------------------------------
struct TcSmem {
  uint8_t a[2][128 * 128];                 // A tiles (bf16, 128-byte swizzled K-major)
  uint8_t b[kTcBStages][kTcN * 128];       // B tiles
  uint8_t raw[kTcRawStages][128 * 32];     // int4 codes of one group, 32 bytes per row
  uint16_t sc[128 * kTcMaxGroups];         // scale of every row and group [row][g]
  uint16_t mn[128 * kTcMaxGroups];         // min
  float xs[kTcMaxGroups * kTcN];           // group sums of the B columns [g][column]
  uint64_t rfull[kTcRawStages], bfull[kTcBStages], pre, mma[2];
  uint32_t tmem;
  int tok[kTcN];       // token of each column
  int dst[kTcN];       // ap row (mode 0) / gate index (mode 1) of each column, -1 = none
};

__global__ void __launch_bounds__(kTcThreads, 1) k_moe_gemm_tc(TcArgs A) {
  extern __shared__ __align__(1024) uint8_t tc_raw[];
  // the swizzled tiles need 1024-byte alignment
  TcSmem &S = *reinterpret_cast<TcSmem *>((reinterpret_cast<uintptr_t>(tc_raw) + 1023) & ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int mtiles = A.mode == 0 ? A.I / 64 : A.d / 128;
  const int tile = blockIdx.x / mtiles, mt = blockIdx.x % mtiles;
  if (tile >= *A.ntiles) return;
  const TcTile tl = A.tiles[tile];
  const int U = A.P.U[0];
  const bool shared = tl.unit == U;
  const int cnt = shared ? A.T : A.P.ustart[tl.unit + 1] - A.P.ustart[tl.unit];
  const int ncol = min(kTcN, cnt - tl.n0);
  const int N = (ncol + 15) & ~15;            // MMA N: multiple of 16
  const uint8_t *base = shared ? A.shared : A.src.base(A.P.uexp[tl.unit]);
  const int K = A.mode == 0 ? A.d : A.I;
  const int G = K / 64;
  const unsigned long long budget = A.timeout_ns;

  // column bookkeeping: token and destination of each column of this tile
  for (int c = tid; c < kTcN; c += kTcThreads) {
    int tok = -1, dst = -1;
    if (c < ncol) {
      if (shared) {
        tok = tl.n0 + c;
        dst = A.mode == 0 ? tok * (A.k + 1) + A.k : -1;
      } else {
        const int asg = A.P.assign[A.P.ustart[tl.unit] + tl.n0 + c];   // t * k + slot
        tok = asg / A.k;
        dst = A.mode == 0 ? tok * (A.k + 1) + asg % A.k : asg;
      }
    }
    S.tok[c] = tok;
    S.dst[c] = dst;
  }
  if (tid == 0) {
    for (int s = 0; s < kTcRawStages; s++) tc_mbar_init(&S.rfull[s], kTcThreads);
    for (int s = 0; s < kTcBStages; s++) tc_mbar_init(&S.bfull[s], kTcThreads);
    tc_mbar_init(&S.pre, kTcThreads);
    tc_mbar_init(&S.mma[0], 1);
    tc_mbar_init(&S.mma[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem(&S.tmem)),
                 "r"(2 * kTcN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = S.tmem;
  const uint32_t idesc = tc_idesc(128, N);

  // this thread's weight row (code loads and conversion): two threads per row, 16 code
  // bytes (32 K elements) each.  mode 0 -> gate rows i0..i0+63 then up rows i0..i0+63
  // (i0 = 64 mt); mode 1 -> down rows 128 mt .. 128 mt + 127
  const int row = tid >> 1, half = tid & 1;
  const uint8_t *codes;
  const uint16_t *scl, *mnv;
  if (A.mode == 0) {
    const int i = mt * 64 + (row & 63);
    const bool up = row >= 64;
    codes = base + (up ? A.bl.uc : A.bl.gc) + (size_t)i * (A.d / 2);
    scl = reinterpret_cast<const uint16_t *>(base + (up ? A.bl.us : A.bl.gs)) + (size_t)i * G;
    mnv = reinterpret_cast<const uint16_t *>(base + (up ? A.bl.um : A.bl.gm)) + (size_t)i * G;
  } else {
    const int n = mt * 128 + row;
    codes = base + A.bl.dc + (size_t)n * (A.I / 2);
    scl = reinterpret_cast<const uint16_t *>(base + A.bl.ds) + (size_t)n * G;
    mnv = reinterpret_cast<const uint16_t *>(base + A.bl.dm) + (size_t)n * G;
  }
  // B role: (column, 16-byte chunk) pairs e = tid + m * kTcThreads
  constexpr int kBPer = kTcN * 8 / kTcThreads;
  const uint16_t *bsrc[kBPer];
#pragma unroll
  for (int m = 0; m < kBPer; m++) {
    const int e = tid + m * kTcThreads, c = e >> 3, ch = e & 7;
    const int tok = S.tok[c];
    bsrc[m] = nullptr;
    if (tok >= 0)
      bsrc[m] = (A.mode == 0 ? A.xp + (size_t)tok * A.d
                             : A.ap + (size_t)(tok * (A.k + 1) + (shared ? A.k : S.dst[c] % A.k)) * A.I) + ch * 8;
  }
  auto load_raw = [&](int g) {
    tc_cp16(tc_smem(S.raw[g % kTcRawStages] + row * 32 + half * 16), codes + g * 32 + half * 16, 16);
    tc_cp_arrive(&S.rfull[g % kTcRawStages]);
  };
  auto load_b = [&](int g) {
    uint8_t *dstb = S.b[g % kTcBStages];
#pragma unroll
    for (int m = 0; m < kBPer; m++) {
      const int e = tid + m * kTcThreads, c = e >> 3, ch = e & 7;
      if (c < N) tc_cp16(tc_smem(dstb + sw128(c, ch)), bsrc[m] ? (const void *)(bsrc[m] + g * 64) : (const void *)A.xsum,
                         bsrc[m] ? 16u : 0u);
    }
    tc_cp_arrive(&S.bfull[g % kTcBStages]);
  };

  // scales, mins and the columns' group sums (staged [column][g] in the A area first);
  // rows of fewer than 16 bytes (K < 512) go in 4-byte copies
  {
    const int rb = G * 2;                       // bytes of a row of scales (or mins)
    if (rb % 16 == 0) {
      for (int q = half; q < rb / 16; q += 2) {
        tc_cp16(tc_smem(S.sc + row * G + q * 8), scl + q * 8, 16);
        tc_cp16(tc_smem(S.mn + row * G + q * 8), mnv + q * 8, 16);
      }
    } else {
      for (int q = half; q < rb / 4; q += 2) {
        tc_cp4(tc_smem(S.sc + row * G + q * 2), scl + q * 2);
        tc_cp4(tc_smem(S.mn + row * G + q * 2), mnv + q * 2);
      }
    }
    const int cb = G * 4;                       // bytes of a column's group sums
    const int csz = cb % 16 == 0 ? 16 : 4;
    const int cpc = cb / csz;
    float *stage = reinterpret_cast<float *>(S.a[0]);
    for (int e = tid; e < kTcN * cpc; e += kTcThreads) {
      const int c = e / cpc, q = e % cpc;
      const int tok = S.tok[c];
      if (tok < 0) continue;                    // never read: the MMA columns there are zero
      const float *src = A.mode == 0 ? A.xsum + (size_t)tok * G
                                     : A.asum + (size_t)(tok * (A.k + 1) + (shared ? A.k : S.dst[c] % A.k)) * G;
      if (csz == 16) tc_cp16(tc_smem(stage + c * G + q * 4), src + q * 4, 16);
      else tc_cp4(tc_smem(stage + c * G + q), src + q);
    }
    tc_cp_arrive(&S.pre);
  }
  for (int g = 0; g < kTcRawAhead && g < G; g++) load_raw(g);
  for (int g = 0; g < kTcBAhead && g < G; g++) load_b(g);
  bool ok = tc_wait_all(&S.pre, 0, budget, A.err);
  ok = !__syncthreads_or(!ok);
  {
    const float *stage = reinterpret_cast<const float *>(S.a[0]);
    for (int e = tid; e < kTcN * G; e += kTcThreads) {
      const int g = e / kTcN, c = e % kTcN;
      S.xs[g * kTcN + c] = stage[c * G + g];
    }
  }
  __syncthreads();

  // fold role: TMEM lane = tile row; warps 0-3 take columns 0..63, warps 4-7 64..127
  const int erow = 32 * (warp & 3) + (tid & 31);
  const int cbeg = (warp >> 2) * (kTcN / 2);
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  unsigned long long acc[kTcN / 4];          // 64 fp32 accumulators as packed pairs
#pragma unroll
  for (int i = 0; i < kTcN / 4; i++) acc[i] = 0ull;
  auto fold = [&](int g) {
    const float s = bf(S.sc[erow * G + g]), m = fmaf(-128.f, s, bf(S.mn[erow * G + g]));
    const unsigned long long s2 = pk2(s, s), m2 = pk2(m, m);
    const float *xg = S.xs + g * kTcN + cbeg;
    const uint32_t taddr = lane_addr + (uint32_t)((g & 1) * kTcN + cbeg);
#pragma unroll
    for (int c0 = 0; c0 < kTcN / 2; c0 += 32) {
      if (cbeg + c0 < N) {
        float v[32];
        tc_ld32(taddr + c0, v);
#pragma unroll
        for (int cc = 0; cc < 32; cc += 4) {
          const float4 x4 = *reinterpret_cast<const float4 *>(xg + c0 + cc);
          unsigned long long &a0 = acc[(c0 + cc) / 2], &a1 = acc[(c0 + cc) / 2 + 1];
          a0 = f2fma(m2, pk2(x4.x, x4.y), f2fma(s2, pk2(v[cc], v[cc + 1]), a0));
          a1 = f2fma(m2, pk2(x4.z, x4.w), f2fma(s2, pk2(v[cc + 2], v[cc + 3]), a1));
        }
      }
    }
  };

  int issued = 0;   // groups whose MMAs were issued
  // `ok` only turns false; the barrier of step (c) makes the exit uniform
#pragma unroll 1
  for (int g = 0; g < G; g++) {
    // (a) this group's codes and activations have landed
    if (ok) ok = tc_wait_all(&S.rfull[g % kTcRawStages], (uint32_t)((g / kTcRawStages) & 1), budget, A.err);
    if (ok) ok = tc_wait_all(&S.bfull[g % kTcBStages], (uint32_t)((g / kTcBStages) & 1), budget, A.err);
    // (b) codes -> A tile: word j of this thread's 16 bytes = K elements 8 (4 half + j) ..
    // + 7 = chunk 4 half + j, unpacked in the permuted order (0,4,1,5,2,6,3,7)
    if (ok) {
      const uint4 w = *reinterpret_cast<const uint4 *>(S.raw[g % kTcRawStages] + row * 32 + half * 16);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      uint8_t *dstA = S.a[g & 1];
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const uint32_t wd = ws[j];
        const uint32_t p0 = (wd & 0x000F000Fu) | 0x43004300u;
        const uint32_t p1 = ((wd >> 4) & 0x000F000Fu) | 0x43004300u;
        const uint32_t p2 = ((wd >> 8) & 0x000F000Fu) | 0x43004300u;
        const uint32_t p3 = ((wd >> 12) & 0x000F000Fu) | 0x43004300u;
        *reinterpret_cast<uint4 *>(dstA + sw128(row, half * 4 + j)) = make_uint4(p0, p1, p2, p3);
      }
    }
    // (c) generic-proxy shared writes (and the landed cp.async data) -> tensor core
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t sa = tc_smem(S.a[g & 1]), sb = tc_smem(S.b[g % kTcBStages]);
      const uint32_t td = tmem + (uint32_t)((g & 1) * kTcN);
#pragma unroll
      for (int kk = 0; kk < 4; kk++)   // K = 16 per instruction: 32 bytes along the swizzled row
        tc_mma(td, tc_desc(sa + kk * 32), tc_desc(sb + kk * 32), idesc, kk ? 1u : 0u);
      tc_commit(&S.mma[g & 1]);
    }
    issued = g + 1;
    // (d) fold the previous group once its MMAs are done
    if (g >= 1) {
      ok = tc_wait_all(&S.mma[(g - 1) & 1], (uint32_t)(((g - 1) >> 1) & 1), budget, A.err);
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if (ok) fold(g - 1);
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    }
    // (e) refill: the code stage of group g + kTcRawAhead was last converted at g - 1;
    // the activation stage of g + kTcBAhead was last read by MMA(g - 1), complete
    if (ok) {
      if (g + kTcRawAhead < G) load_raw(g + kTcRawAhead);
      if (g + kTcBAhead < G) load_b(g + kTcBAhead);
    }
  }
  if (ok) {
    ok = tc_wait_all(&S.mma[(G - 1) & 1], (uint32_t)(((G - 1) >> 1) & 1), budget, A.err);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (ok) fold(G - 1);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  if (__syncthreads_or(!ok)) {
    // drain MMAs still in flight and every outstanding copy before giving TMEM back
    if (issued > 0) tc_wait_all(&S.mma[(issued - 1) & 1], (uint32_t)(((issued - 1) >> 1) & 1), budget, A.err);
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kTcN) : "memory");
    return;
  }

  // ------------------------------- epilogue ------------------------------------------
  float *ex = reinterpret_cast<float *>(S.b[0]);   // 64 x kTcN floats: the up values (mode 0)
  if (A.mode == 0) {
    const int i = mt * 64 + (erow & 63);
    const bool up = erow >= 64;
    const bool lora = shared && A.Bg != nullptr;
    float lb[kMaxR];
    if (lora)
      for (int q = 0; q < A.r; q++) lb[q] = bf((up ? A.Bu : A.Bg)[(size_t)i * A.r + q]);
#pragma unroll
    for (int cp = 0; cp < kTcN / 4; cp++) {
      float v0 = __uint_as_float((uint32_t)acc[cp]), v1 = __uint_as_float((uint32_t)(acc[cp] >> 32));
      const int c = cbeg + 2 * cp;
      if (lora && c < ncol) {
        for (int h2 = 0; h2 < 2; h2++) {
          const int tok = S.tok[c + h2];
          if (tok < 0) continue;
          const float *t = A.lt + (size_t)tok * 3 * A.r + (up ? A.r : 0);
          float la = 0.f;
          for (int q = 0; q < A.r; q++) la = fmaf(lb[q], t[q], la);
          if (h2 == 0) v0 = fmaf(A.c, la, v0);
          else v1 = fmaf(A.c, la, v1);
        }
      }
      if (up) {
        ex[(erow - 64) * kTcN + c] = v0;
        ex[(erow - 64) * kTcN + c + 1] = v1;
      } else {
        acc[cp] = pk2(v0, v1);
      }
    }
    __syncthreads();
    if (!up) {
      const int ipos = kperm_pos(i);
#pragma unroll
      for (int cp = 0; cp < kTcN / 4; cp++) {
#pragma unroll
        for (int h2 = 0; h2 < 2; h2++) {
          const int c = cbeg + 2 * cp + h2;
          const int dst = c < ncol ? S.dst[c] : -1;
          if (dst < 0) continue;
          const float g = __uint_as_float(h2 ? (uint32_t)(acc[cp] >> 32) : (uint32_t)acc[cp]);
          const float u = ex[erow * kTcN + c];
          A.ap_out[(size_t)dst * A.I + ipos] = f2bf(g / (1.0f + expf(-g)) * u);   // bf16 rounding point of a
        }
      }
    }
  } else {
    const int n = mt * 128 + erow;
#pragma unroll
    for (int cp = 0; cp < kTcN / 4; cp++) {
#pragma unroll
      for (int h2 = 0; h2 < 2; h2++) {
        const int c = cbeg + 2 * cp + h2;
        const int tok = c < ncol ? S.tok[c] : -1;
        if (tok < 0) continue;
        const float v = __uint_as_float(h2 ? (uint32_t)(acc[cp] >> 32) : (uint32_t)acc[cp]);
        const float w = shared ? 1.0f : A.gates[S.dst[c]];
        atomicAdd(A.yacc + (size_t)tok * A.d + n, w * v);
      }
    }
  }
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kTcN) : "memory");
}

// ---------------------------------------------------------------------------------------
// Dense bf16 rows on the tensor cores: out[t, col0 + j] = sum_k W[j, k] x[t, k] for the
// router ([A]: fp32 router logits), the prerouter head's linear part ([G] "Ön
// Yönlendirici Başlık Mimarisi") and the shared expert's LoRA A rows ([G]
// "Birleştirilmemiş Adaptör Yürütme").  bf16 x bf16 products are exact and accumulate in
// fp32 in TMEM.  The row list concatenates up to four matrices; one CTA = 128 rows x up to
// kTcN tokens; grid = (row tiles, token tiles).
// ---------------------------------------------------------------------------------------
struct RowSeg {
  const uint16_t *w;   // [rows, ldw] bf16 (the first d columns are used)
  int rows, ldw;
  float *out;          // out[t * ldo + col0 + j]
  int ldo, col0;
};

struct TcRowsArgs {
  const uint16_t *x;   // [T, d] bf16
  int T, d;
  RowSeg seg[4];
  int nseg, total;
  int *err;
  unsigned long long timeout_ns;
};

constexpr int kTrStages = 4;
constexpr int kTrAhead = 3;

struct TcRowsSmem {
  uint8_t a[kTrStages][128 * 128];
  uint8_t b[kTrStages][kTcN * 128];
  uint64_t full[kTrStages], mma[kTrStages];
  uint32_t tmem;
};

__device__ __forceinline__ int rowseg_of(const TcRowsArgs &A, int gr, int &lr) {
  int s = 0;
  lr = gr;
  while (s < A.nseg - 1 && lr >= A.seg[s].rows) lr -= A.seg[s++].rows;
  return s;
}

__global__ void __launch_bounds__(kTcThreads, 1) k_tc_rows(TcRowsArgs A) {
  extern __shared__ __align__(1024) uint8_t tr_raw[];
  TcRowsSmem &S = *reinterpret_cast<TcRowsSmem *>((reinterpret_cast<uintptr_t>(tr_raw) + 1023) & ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * kTcN;
  const int ncol = min(kTcN, A.T - n0);
  const int N = (ncol + 15) & ~15;
  const int G = A.d / 64;
  const unsigned long long budget = A.timeout_ns;
  if (tid == 0) {
    for (int s = 0; s < kTrStages; s++) {
      tc_mbar_init(&S.full[s], kTcThreads);
      tc_mbar_init(&S.mma[s], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem(&S.tmem)),
                 "r"(kTcN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = S.tmem;
  const uint32_t idesc = tc_idesc(128, N);
  // (row or column, 16-byte chunk) pairs of this thread: e = tid + m * kTcThreads
  constexpr int kPer = 128 * 8 / kTcThreads;
  const uint16_t *asrc[kPer], *bsrc[kPer];
#pragma unroll
  for (int m = 0; m < kPer; m++) {
    const int e = tid + m * kTcThreads, rr = e >> 3, ch = e & 7;
    const int gr = m0 + rr;
    asrc[m] = nullptr;
    if (gr < A.total) {
      int lr;
      const int s = rowseg_of(A, gr, lr);
      asrc[m] = A.seg[s].w + (size_t)lr * A.seg[s].ldw + ch * 8;
    }
    bsrc[m] = rr < ncol ? A.x + (size_t)(n0 + rr) * A.d + ch * 8 : nullptr;
  }
  auto load = [&](int g) {
    const int st = g % kTrStages;
#pragma unroll
    for (int m = 0; m < kPer; m++) {
      const int e = tid + m * kTcThreads, rr = e >> 3, ch = e & 7;
      tc_cp16(tc_smem(S.a[st] + sw128(rr, ch)), asrc[m] ? (const void *)(asrc[m] + g * 64) : (const void *)A.x,
              asrc[m] ? 16u : 0u);
      if (rr < N)
        tc_cp16(tc_smem(S.b[st] + sw128(rr, ch)), bsrc[m] ? (const void *)(bsrc[m] + g * 64) : (const void *)A.x,
                bsrc[m] ? 16u : 0u);
    }
    tc_cp_arrive(&S.full[st]);
  };
  for (int g = 0; g < kTrAhead && g < G; g++) load(g);
  bool ok = true;
  int issued = 0;
#pragma unroll 1
  for (int g = 0; g < G; g++) {
    if (ok) ok = tc_wait_all(&S.full[g % kTrStages], (uint32_t)((g / kTrStages) & 1), budget, A.err);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t sa = tc_smem(S.a[g % kTrStages]), sb = tc_smem(S.b[g % kTrStages]);
#pragma unroll
      for (int kk = 0; kk < 4; kk++)
        tc_mma(tmem, tc_desc(sa + kk * 32), tc_desc(sb + kk * 32), idesc, (g | kk) ? 1u : 0u);
      tc_commit(&S.mma[g % kTrStages]);
    }
    issued = g + 1;
    // refill the stage of group g - 1 once its MMAs are done
    if (ok && g + kTrAhead < G) {
      if (g >= 1)
        ok = tc_wait_all(&S.mma[(g - 1) % kTrStages], (uint32_t)(((g - 1) / kTrStages) & 1), budget, A.err);
      if (ok) load(g + kTrAhead);
    }
  }
  if (ok) ok = tc_wait_all(&S.mma[(G - 1) % kTrStages], (uint32_t)(((G - 1) / kTrStages) & 1), budget, A.err);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (__syncthreads_or(!ok)) {
    if (issued > 0)
      tc_wait_all(&S.mma[(issued - 1) % kTrStages], (uint32_t)(((issued - 1) / kTrStages) & 1), budget, A.err);
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcN) : "memory");
    return;
  }
  // epilogue: warp w reads TMEM lanes 32 (w % 4).. (rows), columns split between w < 4 and
  // w >= 4; consecutive lanes write consecutive output columns
  const int erow = 32 * (warp & 3) + (tid & 31);
  const int cbeg = (warp >> 2) * (kTcN / 2);
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  const int gr = m0 + erow;
  int lr = 0;
  const int s = gr < A.total ? rowseg_of(A, gr, lr) : 0;
  float *out = A.seg[s].out;
  const int ldo = A.seg[s].ldo, col = A.seg[s].col0 + lr;
#pragma unroll 1
  for (int c0 = cbeg; c0 < cbeg + kTcN / 2 && c0 < N; c0 += 32) {
    float v[32];
    tc_ld32(lane_addr + c0, v);
    if (gr < A.total)
#pragma unroll
      for (int cc = 0; cc < 32; cc++)
        if (c0 + cc < ncol) out[(size_t)(n0 + c0 + cc) * ldo + col] = v[cc];
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcN) : "memory");
}

// ---------------------------------------------------------------------------------------
// Operand preparation: the K-permuted bf16 copy of x (or nullptr) and the fp32 sum of
// every group of 64 (natural order).  One thread per (row, group).
// ---------------------------------------------------------------------------------------
__global__ void k_perm_sums(const uint16_t *__restrict__ x, long long rows, int K, uint16_t *__restrict__ xp,
                            float *__restrict__ sums) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int G = K / 64;
  if (i >= rows * G) return;
  const long long r = i / G;
  const int g = (int)(i % G);
  const uint4 *src = reinterpret_cast<const uint4 *>(x + r * K + g * 64);
  uint4 *dst = xp ? reinterpret_cast<uint4 *>(xp + r * K + g * 64) : nullptr;
  float s = 0.f;
#pragma unroll
  for (int q = 0; q < 8; q++) {
    const uint4 v = src[q];
    // natural elements 8q .. 8q+7 = (v.x lo, v.x hi, v.y lo, v.y hi, v.z lo, ...)
    s += bf(v.x & 0xFFFFu);
    s += bf(v.x >> 16);
    s += bf(v.y & 0xFFFFu);
    s += bf(v.y >> 16);
    s += bf(v.z & 0xFFFFu);
    s += bf(v.z >> 16);
    s += bf(v.w & 0xFFFFu);
    s += bf(v.w >> 16);
    if (dst)   // permuted block (0,4,1,5,2,6,3,7)
      dst[q] = make_uint4(__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632),
                          __byte_perm(v.y, v.w, 0x5410), __byte_perm(v.y, v.w, 0x7632));
  }
  sums[i] = s;
}

// t_d = Ad a_s from the K-permuted bf16 activations (one warp per token and rank row)
__global__ void k_lora_td(const uint16_t *__restrict__ Ad, const uint16_t *__restrict__ ap, int T, int I, int k,
                          int r, float *__restrict__ lt) {
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= T * r) return;
  const int t = w / r, j = w % r;
  const uint16_t *as = ap + ((size_t)t * (k + 1) + k) * I;
  float acc = 0.f;
  for (int i = lane; i < I; i += 32) acc = fmaf(bf(Ad[(size_t)j * I + i]), bf(as[kperm_pos(i)]), acc);
  acc = warp_sum(acc);
  if (lane == 0) lt[((size_t)t * 3 + 2) * r + j] = acc;
}

// y = yacc + c Bd t_d  -> fp32 and bf16 outputs
__global__ void k_tc_finish(const float *__restrict__ yacc, const uint16_t *__restrict__ Bd,
                            const float *__restrict__ lt, int T, int d, int r, float c, uint16_t *__restrict__ y,
                            float *__restrict__ yf) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)T * d) return;
  const int t = (int)(i / d), n = (int)(i % d);
  float v = yacc[i];
  if (Bd) {
    float lo = 0.f;
    for (int q = 0; q < r; q++) lo = fmaf(bf(Bd[(size_t)n * r + q]), lt[((size_t)t * 3 + 2) * r + q], lo);
    v = fmaf(c, lo, v);
  }
  y[i] = f2bf(v);
  if (yf) yf[i] = v;
}

}  // namespace e0
