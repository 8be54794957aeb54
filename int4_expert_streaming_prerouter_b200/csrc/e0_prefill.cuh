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
#include <cuda.h>
#include <cuda_fp16.h>
#include "e0_device.cuh"
#include "e0_kernels.cuh"

namespace e0 {

constexpr int kTcThreads = 256;     // threads of the dense-rows kernel
constexpr int kTcMinTokens = 64;    // contexts with at least this many tokens get the tensor-core path
constexpr int kTcN = 128;           // tokens per tile (TMEM columns per accumulator)
constexpr int kTcMaxGroups = 64;    // K / 64 <= 64 (K <= 4096)

struct TcTile {
  int unit;      // unique expert index (== U: the shared expert)
  int n0;        // first token position within the unit's token list
};

struct TcArgs {
  // B operands as TMA tensor maps (bf16, K-permuted rows, box 64 x 128, 128-byte swizzle):
  // mode 0: [0] x in expert-grouped row order [T k, d], [1] x in token order [T, d];
  // mode 1: [0] a in grouped order [T k + T, I] (the shared expert's rows last)
  CUtensorMap tmB[2];
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
  const uint16_t *ap;       // [T k + T, I] a, bf16, K-permuted, grouped rows (mode 1 input)
  const float *asum;        // [T k + T, I/64] group sums of a (mode 1)
  uint16_t *ap_out;         // [T k + T, I] (mode 0 output)
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
// L2 policies: the int4 codes stream through once (evict first); the activations are read
// again by every weight tile of the same expert (evict last)
__device__ __forceinline__ unsigned long long tc_policy_first() {
  unsigned long long p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ unsigned long long tc_policy_last() {
  unsigned long long p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void tc_cp16_hint(uint32_t dst, const void *src, uint32_t src_bytes, unsigned long long pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst), "l"(src), "r"(src_bytes),
               "l"(pol)
               : "memory");
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

// 64 TMEM columns of this warp's 32 lanes into registers (one load, one wait)
__device__ __forceinline__ void tc_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; i++) v[i] = __uint_as_float(r[i]);
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
  // one warp: tiles per unit, an exclusive scan over the units in order, then every lane
  // writes its units' tiles
  const int lane = threadIdx.x;
  if (lane >= 32) return;
  const int U = P.U[0];
  int base = 0;
  for (int u0 = 0; u0 <= U; u0 += 32) {
    const int u = u0 + lane;
    const int cnt = u < U ? P.ustart[u + 1] - P.ustart[u] : (u == U ? T : 0);
    const int nt = (cnt + kTcN - 1) / kTcN;
    int incl = nt;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    for (int q = 0; q < nt; q++) {
      const int idx = base + incl - nt + q;
      if (idx < cap) tiles[idx] = TcTile{u, q * kTcN};
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) *ntiles = min(base, cap);
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
//
// Warp-specialised, every hand-off on an mbarrier, so that loads, conversion, MMAs and
// folds of different groups overlap:
//   warp  0    loader: one TMA tile load per group brings the tile's 128 activation rows
//              (stored in expert-grouped order, so a tile's tokens are consecutive rows)
//              as the 128-byte swizzled B tile; the lanes copy the columns' group sums
//   warp  1    TMEM owner; one thread issues the four MMAs of each group
//   warps 2-3  converters: thread t owns weight rows t and t + 64; it streams its own rows'
//              codes kTwRawAhead groups ahead with cp.async (no hand-off needed) and
//              writes 128 + q as bf16 into the A tile ring (kTwAStages stages)
//   warps 4-11 folders: TMEM lane quadrant warp % 4, half of the columns each; they fold
//              every group into registers and run the epilogue (SwiGLU, or the weighted
//              combine into y)
// ---------------------------------------------------------------------------------------
constexpr int kTwThreads = 384;
constexpr int kTwLoadWarps = 1, kTwMmaWarp = 1, kTwConv0 = 2, kTwFold0 = 4;
constexpr int kTwAStages = 3;
constexpr int kTwBStages = 6;
constexpr int kTwRawAhead = 3;      // groups of codes in flight per converter thread
constexpr int kTwTBufs = 4;         // TMEM accumulators (kTcN columns each): MMAs run up to 4 groups ahead of the folds

struct TwSmem {
  uint8_t a[kTwAStages][128 * 128];        // A tiles (bf16, 128-byte swizzled K-major)
  uint8_t b[kTwBStages][kTcN * 128];       // B tiles
  float xs[kTwBStages][kTcN];              // the B columns' group sums
  uint8_t raw[kTwRawAhead][128 * 32];      // int4 codes: converter thread t's row t
  uint16_t sc[128 * kTcMaxGroups];         // scale of every row and group [row][g]
  uint16_t mn[128 * kTcMaxGroups];         // min
  uint64_t bfull[kTwBStages], bempty[kTwBStages], afull[kTwAStages], aempty[kTwAStages];
  uint64_t tfull[kTwTBufs], tempty[kTwTBufs], pre;
  uint32_t tmem;
  volatile int abort;
  int tok[kTcN];       // token of each column
  int dst[kTcN];       // ap row (mode 0) / gate index (mode 1) of each column, -1 = none
  float gw[kTcN];      // combine weight of each column (mode 1)
};

// bounded wait on an mbarrier phase that also gives up once another role has aborted
__device__ __forceinline__ bool tw_wait(uint64_t *b, uint32_t parity, unsigned long long budget, int *err,
                                        volatile int *abort) {
  unsigned long long t0 = 0;
  while (!tc_mbar_test(b, parity)) {
    if (*abort) return false;
    const unsigned long long now = tc_now();
    if (!t0) t0 = now;
    else if (now - t0 > budget) {
      atomicOr(err, DERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void tc_mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc_smem(b)) : "memory");
}

__global__ void __launch_bounds__(kTwThreads, 1) k_moe_gemm_tc(const __grid_constant__ TcArgs A) {
  extern __shared__ __align__(1024) uint8_t tc_raw[];
  // the swizzled tiles need 1024-byte alignment
  TwSmem &S = *reinterpret_cast<TwSmem *>((reinterpret_cast<uintptr_t>(tc_raw) + 1023) & ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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

  // column bookkeeping: token, destination and combine weight of each column of this tile
  for (int c = tid; c < kTcN; c += kTwThreads) {
    int tok = -1, dst = -1;
    float w = 0.f;
    if (c < ncol) {
      if (shared) {
        tok = tl.n0 + c;
        dst = A.mode == 0 ? A.T * A.k + tok : -1;             // grouped row of a
        w = 1.f;
      } else {
        const int asg = A.P.assign[A.P.ustart[tl.unit] + tl.n0 + c];   // t * k + slot
        tok = asg / A.k;
        dst = A.mode == 0 ? A.P.ustart[tl.unit] + tl.n0 + c : asg;   // grouped row of a / gate index
        if (A.mode == 1) w = A.gates[asg];
      }
    }
    S.tok[c] = tok;
    S.dst[c] = dst;
    S.gw[c] = w;
  }
  if (tid == 0) {
    for (int s = 0; s < kTwBStages; s++) {
      tc_mbar_init(&S.bfull[s], 33);   // the TMA's expect_tx arrival + 32 group-sum lanes
      tc_mbar_init(&S.bempty[s], 8);
    }
    for (int s = 0; s < kTwAStages; s++) {
      tc_mbar_init(&S.afull[s], 2);
      tc_mbar_init(&S.aempty[s], 1);
    }
    for (int s = 0; s < kTwTBufs; s++) {
      tc_mbar_init(&S.tfull[s], 1);
      tc_mbar_init(&S.tempty[s], 8);
    }
    tc_mbar_init(&S.pre, 64);
    S.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kTwMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem(&S.tmem)),
                 "r"(kTwTBufs * kTcN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = S.tmem;

  if (warp < kTwLoadWarps) {
    // ---------------- loader: one TMA tile load per group + the columns' group sums -------
    // the tile's tokens are consecutive rows of the grouped operand starting at row0; rows
    // past the tensor's end arrive as zeros (their columns are never used)
    const CUtensorMap *map = (A.mode == 0 && shared) ? &A.tmB[1] : &A.tmB[0];
    const int row0 = shared ? (A.mode == 0 ? tl.n0 : A.T * A.k + tl.n0) : A.P.ustart[tl.unit] + tl.n0;
    #pragma unroll 1
    for (int g = 0; g < G; g++) {
      const int bs = g % kTwBStages;
      if (g >= kTwBStages &&
          !tw_wait(&S.bempty[bs], (uint32_t)(((g / kTwBStages) - 1) & 1), budget, A.err, &S.abort))
        break;
      if (lane == 0) {
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc_smem(&S.bfull[bs])),
                     "r"(kTcN * 128)
                     : "memory");
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
                tc_smem(S.b[bs])),
            "l"(map), "r"(g * 64), "r"(row0), "r"(tc_smem(&S.bfull[bs]))
            : "memory");
      }
      for (int c = lane; c < N; c += 32) {
        const int tok = S.tok[c];
        if (tok < 0) continue;    // padding column: its sum is never used
        const float *src = A.mode == 0 ? A.xsum + (size_t)tok * G : A.asum + (size_t)(row0 + c) * G;
        tc_cp4(tc_smem(&S.xs[bs][c]), src + g);
      }
      tc_cp_arrive(&S.bfull[bs]);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kTwMmaWarp) {
    // ---------------- one thread issues the MMAs ------------------------------------------
    if (lane == 0) {
      const uint32_t idesc = tc_idesc(128, N);
      int issued = 0;
      #pragma unroll 1
      for (int g = 0; g < G; g++) {
        const int as = g % kTwAStages, bs = g % kTwBStages, tb = g % kTwTBufs;
        if (!tw_wait(&S.afull[as], (uint32_t)((g / kTwAStages) & 1), budget, A.err, &S.abort)) break;
        if (!tw_wait(&S.bfull[bs], (uint32_t)((g / kTwBStages) & 1), budget, A.err, &S.abort)) break;
        if (g >= kTwTBufs && !tw_wait(&S.tempty[tb], (uint32_t)(((g / kTwTBufs) - 1) & 1), budget, A.err, &S.abort))
          break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t sa = tc_smem(S.a[as]), sb = tc_smem(S.b[bs]);
        const uint32_t td = tmem + (uint32_t)(tb * kTcN);
#pragma unroll
        for (int kk = 0; kk < 4; kk++)   // K = 16 per instruction: 32 bytes along the swizzled row
          tc_mma(td, tc_desc(sa + kk * 32), tc_desc(sb + kk * 32), idesc, kk ? 1u : 0u);
        tc_commit(&S.tfull[tb]);
        tc_commit(&S.aempty[as]);
        issued = g + 1;
      }
      // after an abort, the MMAs in flight finish before TMEM is given back
      if (issued > 0 && issued < G)
        tc_wait_all(&S.tfull[(issued - 1) % kTwTBufs], (uint32_t)(((issued - 1) / kTwTBufs) & 1), budget, A.err);
    }
    __syncwarp();
  } else if (warp < kTwFold0) {
    // ---------------- converters: thread t owns weight rows t and t + 64 ------------------
    // mode 0 -> gate rows i0..i0+63 then up rows i0..i0+63 (i0 = 64 mt); mode 1 -> down
    // rows 128 mt .. 128 mt + 127
    const int t = tid - kTwConv0 * 32;     // 0..63
    const uint8_t *codes[2];
    const uint16_t *scl[2], *mnv[2];
#pragma unroll
    for (int h = 0; h < 2; h++) {
      const int r = t + 64 * h;
      if (A.mode == 0) {
        const int i = mt * 64 + (r & 63);
        const bool up = r >= 64;
        codes[h] = base + (up ? A.bl.uc : A.bl.gc) + (size_t)i * (A.d / 2);
        scl[h] = reinterpret_cast<const uint16_t *>(base + (up ? A.bl.us : A.bl.gs)) + (size_t)i * G;
        mnv[h] = reinterpret_cast<const uint16_t *>(base + (up ? A.bl.um : A.bl.gm)) + (size_t)i * G;
      } else {
        const int n = mt * 128 + r;
        codes[h] = base + A.bl.dc + (size_t)n * (A.I / 2);
        scl[h] = reinterpret_cast<const uint16_t *>(base + A.bl.ds) + (size_t)n * G;
        mnv[h] = reinterpret_cast<const uint16_t *>(base + A.bl.dm) + (size_t)n * G;
      }
      // the row's scales and mins for the folders (rows of fewer than 16 bytes in 4-byte copies)
      const int rb = G * 2;
      if (rb % 16 == 0) {
        for (int q = 0; q < rb / 16; q++) {
          tc_cp16(tc_smem(S.sc + r * G + q * 8), scl[h] + q * 8, 16);
          tc_cp16(tc_smem(S.mn + r * G + q * 8), mnv[h] + q * 8, 16);
        }
      } else {
        for (int q = 0; q < rb / 4; q++) {
          tc_cp4(tc_smem(S.sc + r * G + q * 2), scl[h] + q * 2);
          tc_cp4(tc_smem(S.mn + r * G + q * 2), mnv[h] + q * 2);
        }
      }
    }
    tc_cp_arrive(&S.pre);
    // the rows' codes, kTwRawAhead groups in flight, one cp.async group per K group
    const unsigned long long pol = tc_policy_first();
    auto load_codes = [&](int g, int rs) {
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int r = t + 64 * h;
        tc_cp16_hint(tc_smem(S.raw[rs] + r * 32), codes[h] + g * 32, 16, pol);
        tc_cp16_hint(tc_smem(S.raw[rs] + r * 32 + 16), codes[h] + g * 32 + 16, 16, pol);
      }
    };
    for (int g = 0; g < kTwRawAhead; g++) {
      if (g < G) load_codes(g, g);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    #pragma unroll 1
    for (int g = 0; g < G; g++) {
      const int as = g % kTwAStages, rs = g % kTwRawAhead;
      asm volatile("cp.async.wait_group %0;" ::"n"(kTwRawAhead - 1) : "memory");   // own codes of g
      if (g >= kTwAStages &&
          !tw_wait(&S.aempty[as], (uint32_t)(((g / kTwAStages) - 1) & 1), budget, A.err, &S.abort))
        break;
      // word j of a row's 32 code bytes = K elements 8 j .. 8 j + 7 = chunk j, unpacked in
      // the permuted order (0,4,1,5,2,6,3,7) as bf16 128 + q
      uint8_t *dstA = S.a[as];
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int r = t + 64 * h;
        const uint4 w0 = *reinterpret_cast<const uint4 *>(S.raw[rs] + r * 32);
        const uint4 w1 = *reinterpret_cast<const uint4 *>(S.raw[rs] + r * 32 + 16);
        const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int j = 0; j < 8; j++) {
          const uint32_t wd = ws[j];
          const uint32_t p0 = (wd & 0x000F000Fu) | 0x43004300u;
          const uint32_t p1 = ((wd >> 4) & 0x000F000Fu) | 0x43004300u;
          const uint32_t p2 = ((wd >> 8) & 0x000F000Fu) | 0x43004300u;
          const uint32_t p3 = ((wd >> 12) & 0x000F000Fu) | 0x43004300u;
          *reinterpret_cast<uint4 *>(dstA + sw128(r, j)) = make_uint4(p0, p1, p2, p3);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) tc_mbar_arrive(&S.afull[as]);
      // refill these rows' slots (their words are consumed above) with group g + kTwRawAhead
      if (g + kTwRawAhead < G) load_codes(g + kTwRawAhead, rs);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else {
    // ---------------- folders: TMEM -> registers, acc += s P + (m - 128 s) X -------------
    const int fw = warp - kTwFold0;                 // 0..7
    const int erow = 32 * (warp & 3) + lane;        // tile row = TMEM lane
    const int cbeg = (fw >> 2) * (kTcN / 2);        // this warp's half of the columns
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    unsigned long long acc[kTcN / 4];               // 64 fp32 accumulators as packed pairs
#pragma unroll
    for (int i = 0; i < kTcN / 4; i++) acc[i] = 0ull;
    bool ok = tw_wait(&S.pre, 0, budget, A.err, &S.abort);
    #pragma unroll 1
    for (int g = 0; g < G && ok; g++) {
      const int tb = g % kTwTBufs, bs = g % kTwBStages;
      ok = tw_wait(&S.tfull[tb], (uint32_t)((g / kTwTBufs) & 1), budget, A.err, &S.abort) &&
           tw_wait(&S.bfull[bs], (uint32_t)((g / kTwBStages) & 1), budget, A.err, &S.abort);
      if (!ok) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const float s = bf(S.sc[erow * G + g]), m = fmaf(-128.f, s, bf(S.mn[erow * G + g]));
      const unsigned long long s2 = pk2(s, s), m2 = pk2(m, m);
      const float *xg = S.xs[bs] + cbeg;
      const uint32_t taddr = lane_addr + (uint32_t)(tb * kTcN + cbeg);
      if (cbeg < N) {
        // this warp's 64 columns in one TMEM load (columns past N hold stale values that
        // only reach accumulators of unused columns)
        float v[64];
        tc_ld64(taddr, v);
#pragma unroll
        for (int cc = 0; cc < 64; cc += 4) {
          const float4 x4 = *reinterpret_cast<const float4 *>(xg + cc);
          unsigned long long &a0 = acc[cc / 2], &a1 = acc[cc / 2 + 1];
          a0 = f2fma(m2, pk2(x4.x, x4.y), f2fma(s2, pk2(v[cc], v[cc + 1]), a0));
          a1 = f2fma(m2, pk2(x4.z, x4.w), f2fma(s2, pk2(v[cc + 2], v[cc + 3]), a1));
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        tc_mbar_arrive(&S.tempty[tb]);
        tc_mbar_arrive(&S.bempty[bs]);
      }
    }
    // every folder agrees before the epilogue (named barrier 1: the 8 folder warps)
    {
      uint32_t bad;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbarrier.red.or.pred q, 1, %2, p;\n\t"
          "selp.u32 %0, 1, 0, q;\n\t}"
          : "=r"(bad)
          : "r"((uint32_t)!ok), "r"(256)
          : "memory");
      ok = bad == 0;
    }
    if (ok) {
      // the tile's results go through shared memory as ex[row][column] with a row stride of
      // kTcN + 1 floats, so that lanes on consecutive rows hit different banks both when
      // writing (lane = row) and when reading (lane = row again, or four rows per lane)
      constexpr int XS = kTcN + 1;
      float *ex = reinterpret_cast<float *>(S.b[0]);   // 128 x XS floats (66 KB of the B ring)
      if (A.mode == 0) {
        // gate rows 0..63 and up rows 64..127 (with the shared expert's LoRA up branch);
        // then all 256 folder threads form a = bf16(silu(g) u), thread t taking unit t % 64
        // of four columns per pass
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
          ex[erow * XS + c] = v0;
          ex[erow * XS + c + 1] = v1;
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        const int ft = tid - kTwFold0 * 32, iu = ft & 63;
        const int ipos = kperm_pos(mt * 64 + iu);
        #pragma unroll 4
        for (int c = ft >> 6; c < ncol; c += 4) {
          const int dst = S.dst[c];
          if (dst < 0) continue;
          const float g = ex[iu * XS + c], u = ex[(64 + iu) * XS + c];
          A.ap_out[(size_t)dst * A.I + ipos] = f2bf(g / (1.0f + expf(-g)) * u);   // bf16 rounding point of a
        }
      } else {
        // gate-weighted values to shared memory, then four consecutive output rows of one
        // column per thread, added into y with one vector reduction
#pragma unroll
        for (int cp = 0; cp < kTcN / 4; cp++) {
          const int c = cbeg + 2 * cp;
          ex[erow * XS + c] = S.gw[c] * __uint_as_float((uint32_t)acc[cp]);
          ex[erow * XS + c + 1] = S.gw[c + 1] * __uint_as_float((uint32_t)(acc[cp] >> 32));
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        const int ft = tid - kTwFold0 * 32;
        for (int it = ft; it < ncol * 32; it += 256) {
          const int c = it >> 5, n4 = it & 31;
          const int tok = S.tok[c];
          if (tok < 0) continue;
          const float y0 = ex[(4 * n4) * XS + c], y1 = ex[(4 * n4 + 1) * XS + c];
          const float y2 = ex[(4 * n4 + 2) * XS + c], y3 = ex[(4 * n4 + 3) * XS + c];
          float *dstp = A.yacc + (size_t)tok * A.d + mt * 128 + 4 * n4;
          asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dstp), "f"(y0), "f"(y1), "f"(y2), "f"(y3)
                       : "memory");
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (warp == kTwMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTwTBufs * kTcN) : "memory");
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

// x rows in expert-grouped order: row p of xg = the permuted x row of the token of
// assignment assign[p] (t * k + slot).  One block per row, one 16-byte chunk per thread.
__global__ void k_group_rows(const uint16_t *__restrict__ xp, const int32_t *__restrict__ assign, int k, int d,
                             uint16_t *__restrict__ xg) {
  const int p = blockIdx.x, t = assign[p] / k;
  const uint4 *src = reinterpret_cast<const uint4 *>(xp + (size_t)t * d);
  uint4 *dst = reinterpret_cast<uint4 *>(xg + (size_t)p * d);
  for (int i = threadIdx.x; i < d / 8; i += blockDim.x) dst[i] = src[i];
}

// t_d = Ad a_s from the K-permuted bf16 activations (one warp per token and rank row); the
// shared expert's a rows are rows T k .. T k + T - 1 of the grouped a
__global__ void k_lora_td(const uint16_t *__restrict__ Ad, const uint16_t *__restrict__ ap, int T, int I, int k,
                          int r, float *__restrict__ lt) {
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= T * r) return;
  const int t = w / r, j = w % r;
  const uint16_t *as = ap + ((size_t)T * k + t) * I;
  float acc = 0.f;
  for (int i = lane; i < I; i += 32) acc = fmaf(bf(Ad[(size_t)j * I + i]), bf(as[kperm_pos(i)]), acc);
  acc = warp_sum(acc);
  if (lane == 0) lt[((size_t)t * 3 + 2) * r + j] = acc;
}

// y = yacc + c Bd t_d  -> fp32 and bf16 outputs.  One block per token: t_d in shared
// memory, each thread a strided set of output rows n with its B_d row in 16-byte loads.
__global__ void k_tc_finish(const float *__restrict__ yacc, const uint16_t *__restrict__ Bd,
                            const float *__restrict__ lt, int T, int d, int r, float c, uint16_t *__restrict__ y,
                            float *__restrict__ yf) {
  const int t = blockIdx.x;
  __shared__ float td[kMaxR];
  if (Bd && threadIdx.x < r) td[threadIdx.x] = lt[((size_t)t * 3 + 2) * r + threadIdx.x];
  __syncthreads();
  for (int n = threadIdx.x; n < d; n += blockDim.x) {
    const size_t i = (size_t)t * d + n;
    float v = yacc[i];
    if (Bd) {
      float lo = 0.f;
      if (r % 8 == 0 && ((uintptr_t)Bd & 15) == 0) {
        for (int q0 = 0; q0 < r; q0 += 8) {
          const uint4 w = *reinterpret_cast<const uint4 *>(Bd + (size_t)n * r + q0);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int j = 0; j < 4; j++) {
            lo = fmaf(bf(ws[j] & 0xFFFFu), td[q0 + 2 * j], lo);
            lo = fmaf(bf(ws[j] >> 16), td[q0 + 2 * j + 1], lo);
          }
        }
      } else {
        for (int q = 0; q < r; q++) lo = fmaf(bf(Bd[(size_t)n * r + q]), td[q], lo);
      }
      v = fmaf(c, lo, v);
    }
    y[i] = f2bf(v);
    if (yf) yf[i] = v;
  }
}

}  // namespace e0
