// Prefill path: the experts of one MoE block on many tokens as grouped GEMMs on the
// 5th-generation tensor cores (tcgen05.mma, fp32 accumulators in tensor memory).
//
// Method ([G] "Birleştirilmemiş Adaptör Yürütme"; [A] int4 affine g64 experts, SwiGLU):
//   gate/up:  G = Dq(W_gu) X_e^T  (per expert e, tokens routed to e), a = bf16(silu(g) u),
//             the shared expert adds c * B (A x) to g and u first;
//   down:     Y_e = Dq(W_d) A_e^T, y[t] += w_{t,j} Y_e[:, t]  (w = 1 for the shared expert).
//
// B200 design.  Each int4 weight s q + m enters the tensor core as two exact fp16 parts,
// s (q & 14) and s (q & 1), formed by half-precision FMAs on the masked code bits, so every
// product with the (fp16-held) bf16 activations is exact and accumulates in fp32 with no
// per-group fold; the min term and the shared expert's LoRA up branch are extra K blocks
// of the same accumulation.  The expanded weights go from registers straight into tensor
// memory, the A operand of tcgen05.mma, so shared memory carries only raw codes and
// activation tiles, both by TMA.  Persistent warp-specialised CTAs overlap code/activation
// loads, conversion, MMAs and the epilogues of consecutive work units (details at
// k_moe_gemm_tc).
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include "e0_device.cuh"
#include "e0_kernels.cuh"

namespace e0 {

constexpr int kTcThreads = 256;     // threads of the dense-rows kernel
constexpr int kTcMinTokens = 64;    // contexts with at least this many tokens get the tensor-core path
constexpr int kTcN = 128;           // tokens per tile of the dense-rows kernel (TMEM columns)
constexpr int kTmN = 80;            // tokens per expert tile of the grouped expert GEMM
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
  // int4 code tiles as 3-D TMA maps over [experts][rows][K/2 bytes] (box 128 bytes x 64 or
  // 128 rows, 128-byte swizzle): mode 0: [0] gate, [1] up of the routed experts, [2] gate,
  // [3] up of the shared expert; mode 1: [0] down of the routed experts, [2] of the shared
  CUtensorMap tmC[4];
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
  float *ypart;             // [k + 1][T, d] (mode 1, fixed-order combine) or nullptr
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

// one test of an mbarrier phase; the thread may sleep in it until the phase completes (at
// most ~1 ms), so waiting warps do not take issue slots from the working ones
__device__ __forceinline__ bool tc_mbar_test(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 1000000;\n\t"
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
// tokens) cut into tiles of up to kTmN tokens.  One block.
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
    const int nt = (cnt + kTmN - 1) / kTmN;
    int incl = nt;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    for (int q = 0; q < nt; q++) {
      const int idx = base + incl - nt + q;
      if (idx < cap) tiles[idx] = TcTile{u, q * kTmN};
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) *ntiles = min(base, cap);
}

// ---------------------------------------------------------------------------------------
// The grouped expert GEMM: persistent CTAs (one per SM) walk the work units (one 128-row
// weight tile of one expert x one tile of up to kTmN of its tokens) in a fixed order,
// unit u = tile * M tiles + M tile, CTA b taking u = b, b + grid, ...
//
// Exact affine int4 product without a per-group fold.  With w = s q + m (s, m the bf16
// scale and min of the row's group g, q in 0..15) and q = (q & 14) + (q & 1):
//   sum_k w_k x_k = sum_k s (q_k & 14) x_k + sum_k s (q_k & 1) x_k + sum_g m_g X_g,
// X_g = sum_{k in g} x_k.  s (q & 14) = 2 s (q >> 1) has at most 8 + 3 significant bits and
// s (q & 1) is 0 or s, so both are exact fp16 values (for 2^-13 <= |s| < 64; the pages'
// scales are ~1e-2), and x (bf16) is an exact fp16 value in its range, so the tensor core
// forms every product exactly and accumulates in fp32.  The min term is one more K = 64
// block per unit: A = the row's mins (exact in fp16) twice, B = each column's group sums
// split as X = hi + lo in fp16 (hi = fp16(X), lo = fp16(X - hi), ~22 significant bits
// together).  The shared expert's unmerged LoRA up branch c B (A x) is one more block on
// gate/up: A = the row's B_g (gate rows) or B_u (up rows) twice, B = c t_g, c t_u (t = A x)
// split hi/lo the same way, so every term of g and u leaves the tensor core in fp32.
//
// A tcgen05.mma blocks its issuing thread ~120 cycles whatever N is (N <= 128), so at the
// ~64 tokens a routed expert receives one issuing thread would leave the tensor core
// idle most of the time.  Two threads issue, one the extra blocks and the even K groups,
// the other the odd K groups, each into its own accumulator (the epilogue adds the two);
// each accumulator is double-buffered across units (4 x kTmN TMEM columns).
//
// The expanded operands go from registers straight into tensor memory (A in TMEM), so
// shared memory carries only raw codes and activations (TMA).  Warp roles, every hand-off
// on an mbarrier:
//   warp 0      producer: per 4 K groups one TMA load of the unit's codes (128 rows x 128
//               bytes, 128-byte swizzle; 3-D map over the expert array), per K group one
//               TMA load of the activation tile (expert-grouped rows: a tile's tokens are
//               consecutive rows)
//   warps 1, 2  the two MMA issuers
//   warp 3      unit warp, two units ahead: column bookkeeping (token, destination,
//               combine weight) and the extra blocks' B tiles
//   warps 4-7   epilogue, TMEM lane quadrant warp % 4: SwiGLU (gate/up), or the
//               gate-weighted combine into y (down); then, two units ahead, each thread
//               its weight row's scales and mins as fp16 in [group][row] order
//   warps 8-15  converters, quadrant warp % 4 (weight row 32 (warp % 4) + lane), half
//               h = (warp - 8) / 4 of each 64-wide K block: per unit the extra blocks' A,
//               then per K group both exact fp16 parts, into a 64-column TMEM stage
// ---------------------------------------------------------------------------------------
constexpr int kTmThreads = 512;
constexpr int kTmProdWarp = 0, kTmMma0 = 1, kTmMma1 = 2, kTmUnitWarp = 3, kTmEpi0 = 4, kTmConv0 = 8;
constexpr int kTmEpiThreads = 128, kTmConvWarps = 8;
constexpr int kTmBStages = 6;      // activation tiles in flight (one K group each; even: stage parity = owner)
static_assert(kTmBStages % 2 == 0, "B stage owners");
constexpr int kTmCStages = 3;      // code tiles in flight (four K groups each)
constexpr int kTmAStages = 3;      // A operand stages in TMEM (64 columns: both fp16 parts of one K block): 2 + 1 per issuer
constexpr int kTmMaxG = 32;        // K <= 2048
constexpr int kTmMaxR = 16;        // LoRA rank of the extra block (4 r <= 64)
constexpr int kTmXRow = 65;        // epilogue exchange row stride in floats (conflict-free scalar access)
constexpr int kTmDRow = 132;       // down combine exchange: floats per column (128 rows + pad, 16-byte rows)
static_assert(32 * kTmDRow <= 2 * 64 * kTmXRow, "down combine exchange fits the gate/up one");
constexpr uint32_t kTmACol = 4 * kTmN, kTmCols = 512;
static_assert(kTmACol + kTmAStages * 64 <= kTmCols, "TMEM budget");
static_assert((kTmN * 128) % 1024 == 0 && kTmN % 16 == 0, "tile rows");

struct TmSmem {
  uint8_t b[kTmBStages][kTmN * 128];   // activation tiles (fp16, 128-byte swizzled K-major)
  uint8_t c[kTmCStages][128 * 128];    // int4 code tiles: 128 rows x 4 groups (128-byte swizzle)
  uint8_t bm[2][kTmN * 128];           // min block B tiles: group sums hi | lo | 0, per unit slot
  uint8_t bl[2][kTmN * 128];           // LoRA block B tiles: c t_g hi | lo | c t_u hi | lo
  uint16_t sc[2][kTmMaxG][128];        // fp16 scales [group][row], per unit slot
  uint16_t mn[2][kTmMaxG][128];        // fp16 mins
  alignas(16) float xch[2][64 * kTmXRow];   // epilogue exchange: gate and up values of 64 columns,
                                            // or (down) 32 columns x 128 rows, [column][row + pad]
  int tok[2][kTmN];                    // token of each column (-1: padding)
  int dst[2][kTmN];                    // a row (gate/up) or gate index (down) of each column
  float gw[2][kTmN];                   // combine weight of each column (down)
  uint64_t bfull[kTmBStages], bempty[kTmBStages], cfull[kTmCStages], cempty[kTmCStages];
  uint64_t afull[kTmAStages], aempty[kTmAStages];
  uint64_t accfull[2], accempty[2], ufull[2], uempty[2], sfull[2], drain[2];
  uint32_t tmem;
  volatile int abort;
};

struct TmUnit {
  int tile, mt, unit, n0, ncol, N;
  bool shared;
};

__device__ __forceinline__ TmUnit tm_unit(const TcArgs &A, int u, int mtiles) {
  TmUnit U;
  U.tile = u / mtiles;
  U.mt = u % mtiles;
  const TcTile tl = A.tiles[U.tile];
  U.unit = tl.unit;
  U.n0 = tl.n0;
  U.shared = tl.unit == A.P.U[0];
  const int cnt = U.shared ? A.T : A.P.ustart[tl.unit + 1] - A.P.ustart[tl.unit];
  U.ncol = min(kTmN, cnt - tl.n0);
  U.N = (U.ncol + 15) & ~15;   // MMA N: a multiple of 16
  return U;
}

// bounded wait on an mbarrier phase that also gives up once another role has aborted
__device__ __forceinline__ bool tm_wait(uint64_t *b, uint32_t parity, unsigned long long budget, int *err,
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

// the same wait, agreed by the whole warp (the warp then runs its .sync.aligned
// tensor-memory instructions together, or leaves together)
__device__ __forceinline__ bool tm_wait_warp(uint64_t *b, uint32_t parity, unsigned long long budget, int *err,
                                             volatile int *abort) {
  return __all_sync(0xffffffffu, tm_wait(b, parity, budget, err, abort));
}

__device__ __forceinline__ void tc_mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc_smem(b)) : "memory");
}

__device__ __forceinline__ void tm_expect(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc_smem(b)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tm_load2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          tc_smem(dst)),
      "l"(map), "r"(x), "r"(y), "r"(tc_smem(bar))
      : "memory");
}

__device__ __forceinline__ void tm_load3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar,
                                          unsigned long long pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
      "%3, %4}], [%5], %6;" ::"r"(tc_smem(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(tc_smem(bar)), "l"(pol)
      : "memory");
}

// Instruction descriptor of kind::f16 with fp16 A and B: fp32 accumulator (bits 4-5 = 1),
// A and B fp16 (bits 7-9, 10-12 = 0), both K-major, N >> 3 (bits 17-22), M >> 4 (24-28).
__device__ __forceinline__ uint32_t tm_idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// MMA with the A operand in tensor memory (M = 128 rows in the 128 lanes, K = 16 as 8
// columns of 16-bit pairs) and B in shared memory
__device__ __forceinline__ void tm_mma(uint32_t tmem_d, uint32_t tmem_a, unsigned long long bd, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bd), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 registers into 16 consecutive TMEM columns of this warp's 32 lanes
__device__ __forceinline__ void tm_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ uint32_t tm_hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// bf16 bits -> fp16 bits (exact for values in the fp16 normal range)
__device__ __forceinline__ uint16_t tm_bf2h(uint32_t b) { return __half_as_ushort(__float2half_rn(bf(b))); }

// fp16 pair (lo, hi) of two fp32 values
__device__ __forceinline__ uint32_t tm_h2(float a, float b) {
  return (uint32_t)__half_as_ushort(__float2half_rn(a)) | ((uint32_t)__half_as_ushort(__float2half_rn(b)) << 16);
}
// the fp16 remainders of two fp32 values after their fp16 roundings
__device__ __forceinline__ uint32_t tm_h2lo(float a, float b) {
  return tm_h2(a - __half2float(__float2half_rn(a)), b - __half2float(__float2half_rn(b)));
}

// Row c of the min block's B tile: 16-bit position k holds hi(X_k) for k < GT and
// lo(X_(k-GT)) for GT <= k < 2 GT (X = the column's GT group sums, src = nullptr: zeros).
template <int GT>
__device__ __forceinline__ void tm_bm_row(uint8_t *tile, int c, const float *src) {
  float xv[GT];
#pragma unroll
  for (int g = 0; g < GT; g++) xv[g] = 0.f;
  if (src) {
    if constexpr (GT % 4 == 0) {
#pragma unroll
      for (int g = 0; g < GT; g += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(src + g);
        xv[g] = v.x; xv[g + 1] = v.y; xv[g + 2] = v.z; xv[g + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int g = 0; g < GT; g += 2) {
        const float2 v = *reinterpret_cast<const float2 *>(src + g);
        xv[g] = v.x; xv[g + 1] = v.y;
      }
    }
  }
  uint32_t wv[32];
#pragma unroll
  for (int j = 0; j < GT / 2; j++) wv[j] = tm_h2(xv[2 * j], xv[2 * j + 1]);
#pragma unroll
  for (int j = 0; j < GT / 2; j++) wv[GT / 2 + j] = tm_h2lo(xv[2 * j], xv[2 * j + 1]);
#pragma unroll
  for (int j = GT; j < 32; j++) wv[j] = 0u;
#pragma unroll
  for (int ch = 0; ch < 8; ch++)
    *reinterpret_cast<uint4 *>(tile + sw128(c, ch)) = make_uint4(wv[4 * ch], wv[4 * ch + 1], wv[4 * ch + 2], wv[4 * ch + 3]);
}
template <int GT>
__device__ __forceinline__ void tm_bm_row_any(int G, uint8_t *tile, int c, const float *src) {
  if (G == GT) tm_bm_row<GT>(tile, c, src);
  else if constexpr (GT > 2) tm_bm_row_any<GT - 2>(G, tile, c, src);
}

// Row c of the LoRA block's B tile (rank RT): 16-bit position k holds hi(c t_g[k]) for
// k < RT, lo(c t_g[k - RT]) for RT <= k < 2 RT, hi(c t_u[k - 2 RT]), lo(c t_u[k - 3 RT])
// up to 4 RT (t = the token's A_g x, A_u x; nullptr: zeros).
template <int RT>
__device__ __forceinline__ void tm_bl_row(uint8_t *tile, int c, const float *t, float cs) {
  float tg[RT], tu[RT];
#pragma unroll
  for (int q = 0; q < RT; q += 2) {
    float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
    if (t) {
      a = *reinterpret_cast<const float2 *>(t + q);
      b = *reinterpret_cast<const float2 *>(t + RT + q);
    }
    tg[q] = cs * a.x; tg[q + 1] = cs * a.y;
    tu[q] = cs * b.x; tu[q + 1] = cs * b.y;
  }
  uint32_t wv[32];
#pragma unroll
  for (int j = 0; j < RT / 2; j++) {
    wv[j] = tm_h2(tg[2 * j], tg[2 * j + 1]);
    wv[RT / 2 + j] = tm_h2lo(tg[2 * j], tg[2 * j + 1]);
    wv[RT + j] = tm_h2(tu[2 * j], tu[2 * j + 1]);
    wv[3 * RT / 2 + j] = tm_h2lo(tu[2 * j], tu[2 * j + 1]);
  }
#pragma unroll
  for (int j = 2 * RT; j < 32; j++) wv[j] = 0u;
#pragma unroll
  for (int ch = 0; ch < 8; ch++)
    *reinterpret_cast<uint4 *>(tile + sw128(c, ch)) = make_uint4(wv[4 * ch], wv[4 * ch + 1], wv[4 * ch + 2], wv[4 * ch + 3]);
}
template <int RT>
__device__ __forceinline__ void tm_bl_row_any(int r, uint8_t *tile, int c, const float *t, float cs) {
  if (r == RT) tm_bl_row<RT>(tile, c, t, cs);
  else if constexpr (RT > 2) tm_bl_row_any<RT - 2>(r, tile, c, t, cs);
}

// this thread's weight row's scales and mins as fp16 into [group][row] (the epilogue
// threads, one per row, two units ahead)
__device__ __forceinline__ void tm_fill_scales(const TcArgs &A, const TmUnit &U, int G, int row, uint16_t (*sc)[128],
                                               uint16_t (*mn)[128]) {
  const uint8_t *base = U.shared ? A.shared : A.src.base(A.P.uexp[U.unit]);
  const uint16_t *scl, *mnv;
  if (A.mode == 0) {
    const int i = 64 * U.mt + (row & 63);
    const bool up = row >= 64;
    scl = reinterpret_cast<const uint16_t *>(base + (up ? A.bl.us : A.bl.gs)) + (size_t)i * G;
    mnv = reinterpret_cast<const uint16_t *>(base + (up ? A.bl.um : A.bl.gm)) + (size_t)i * G;
  } else {
    const int n = 128 * U.mt + row;
    scl = reinterpret_cast<const uint16_t *>(base + A.bl.ds) + (size_t)n * G;
    mnv = reinterpret_cast<const uint16_t *>(base + A.bl.dm) + (size_t)n * G;
  }
  if ((G & 7) == 0) {
    uint4 s8[kTmMaxG / 8], m8[kTmMaxG / 8];
#pragma unroll
    for (int j = 0; j < kTmMaxG / 8; j++)
      if (8 * j < G) {
        s8[j] = *reinterpret_cast<const uint4 *>(scl + 8 * j);
        m8[j] = *reinterpret_cast<const uint4 *>(mnv + 8 * j);
      }
#pragma unroll
    for (int j = 0; j < kTmMaxG / 8; j++)
      if (8 * j < G) {
        const uint32_t sw[4] = {s8[j].x, s8[j].y, s8[j].z, s8[j].w}, mw[4] = {m8[j].x, m8[j].y, m8[j].z, m8[j].w};
#pragma unroll
        for (int e = 0; e < 4; e++) {
          sc[8 * j + 2 * e][row] = tm_bf2h(sw[e] & 0xFFFFu);
          sc[8 * j + 2 * e + 1][row] = tm_bf2h(sw[e] >> 16);
          mn[8 * j + 2 * e][row] = tm_bf2h(mw[e] & 0xFFFFu);
          mn[8 * j + 2 * e + 1][row] = tm_bf2h(mw[e] >> 16);
        }
      }
  } else {
    for (int g = 0; g < G; g++) {
      sc[g][row] = tm_bf2h(scl[g]);
      mn[g][row] = tm_bf2h(mnv[g]);
    }
  }
}

__global__ void __launch_bounds__(kTmThreads, 1) k_moe_gemm_tc(const __grid_constant__ TcArgs A) {
  extern __shared__ __align__(1024) uint8_t tm_raw[];
  // the swizzled tiles need 1024-byte alignment
  TmSmem &S = *reinterpret_cast<TmSmem *>((reinterpret_cast<uintptr_t>(tm_raw) + 1023) & ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mtiles = A.mode == 0 ? A.I / 64 : A.d / 128;
  const int total = *A.ntiles * mtiles;
  const int K = A.mode == 0 ? A.d : A.I;
  const int G = K / 64;
  const unsigned long long budget = A.timeout_ns;
  // the LoRA up block runs on the gate/up units of the shared expert
  const bool lora_blk = A.mode == 0 && A.Bg != nullptr;

  if (tid == 0) {
    for (int s = 0; s < kTmBStages; s++) {
      tc_mbar_init(&S.bfull[s], 1);
      tc_mbar_init(&S.bempty[s], 1);
    }
    for (int s = 0; s < kTmCStages; s++) {
      tc_mbar_init(&S.cfull[s], 1);
      tc_mbar_init(&S.cempty[s], kTmConvWarps);
    }
    for (int s = 0; s < kTmAStages; s++) {
      tc_mbar_init(&S.afull[s], kTmConvWarps);
      tc_mbar_init(&S.aempty[s], 1);
    }
    for (int s = 0; s < 2; s++) {
      tc_mbar_init(&S.accfull[s], 2);
      tc_mbar_init(&S.accempty[s], kTmEpiThreads / 32);
      tc_mbar_init(&S.ufull[s], 32);               // the unit warp's bookkeeping and B tiles
      tc_mbar_init(&S.sfull[s], kTmEpiThreads);    // the rows' scales and mins
      tc_mbar_init(&S.uempty[s], kTmEpiThreads / 32);
      tc_mbar_init(&S.drain[s], 1);
    }
    S.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kTmMma0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem(&S.tmem)),
                 "r"(kTmCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = S.tmem;

  if (warp == kTmProdWarp) {
    // ---------------- producer: code tiles and activation tiles ---------------------------
    if (lane == 0) {
      const unsigned long long pol_first = tc_policy_first();
      const unsigned long long pol_keep = tc_policy_last();
      int rg = 0, cc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        const TmUnit U = tm_unit(A, u, mtiles);
        // routed experts' codes are read by one or two token tiles (evict first); the
        // shared expert's by every token tile of the call (keep)
        const unsigned long long pol = U.shared ? pol_keep : pol_first;
        const int z = U.shared ? 0 : A.P.uexp[U.unit];
        const CUtensorMap *mapB = (A.mode == 0 && U.shared) ? &A.tmB[1] : &A.tmB[0];
        const int brow = U.shared ? (A.mode == 0 ? U.n0 : A.T * A.k + U.n0) : A.P.ustart[U.unit] + U.n0;
        for (int g0 = 0; g0 < G && ok; g0 += 4, cc++) {
          const int cs = cc % kTmCStages;
          if (cc >= kTmCStages &&
              !(ok = tm_wait(&S.cempty[cs], (uint32_t)(((cc / kTmCStages) - 1) & 1), budget, A.err, &S.abort)))
            break;
          tm_expect(&S.cfull[cs], 128 * 128);
          if (A.mode == 0) {
            // gate rows 64 mt .. 64 mt + 63, then the up rows of the same intermediate units
            const CUtensorMap *mg = U.shared ? &A.tmC[2] : &A.tmC[0];
            const CUtensorMap *mu = U.shared ? &A.tmC[3] : &A.tmC[1];
            tm_load3d(S.c[cs], mg, 32 * g0, 64 * U.mt, z, &S.cfull[cs], pol);
            tm_load3d(S.c[cs] + 64 * 128, mu, 32 * g0, 64 * U.mt, z, &S.cfull[cs], pol);
          } else {
            tm_load3d(S.c[cs], U.shared ? &A.tmC[2] : &A.tmC[0], 32 * g0, 128 * U.mt, z, &S.cfull[cs], pol);
          }
          const int ng = min(4, G - g0);
          for (int lg = 0; lg < ng; lg++, rg++) {
            const int bs = rg % kTmBStages;
            if (rg >= kTmBStages &&
                !(ok = tm_wait(&S.bempty[bs], (uint32_t)(((rg / kTmBStages) - 1) & 1), budget, A.err, &S.abort)))
              break;
            tm_expect(&S.bfull[bs], kTmN * 128);
            tm_load2d(S.b[bs], mapB, 64 * (g0 + lg), brow, &S.bfull[bs]);
          }
        }
      }
      if (!ok) {
        // every tile load issued lands before the CTA may exit
        for (int s = 0; s < kTmCStages; s++) {
          const int n = cc / kTmCStages + (s < cc % kTmCStages ? 1 : 0);
          if (n > 0) tc_wait_all(&S.cfull[s], (uint32_t)((n - 1) & 1), budget, A.err);
        }
        for (int s = 0; s < kTmBStages; s++) {
          const int n = rg / kTmBStages + (s < rg % kTmBStages ? 1 : 0);
          if (n > 0) tc_wait_all(&S.bfull[s], (uint32_t)((n - 1) & 1), budget, A.err);
        }
      }
    }
    __syncwarp();
  } else if (warp == kTmMma0 || warp == kTmMma1) {
    // ---------------- the two MMA issuers -------------------------------------------------
    // A-stage entries per unit: group 0 .. G - 1, [min block] [LoRA block].  Issuer 0 takes
    // the even groups and the extra blocks (whose B tiles the unit warp fills while the
    // groups run), issuer 1 the odd groups, each both fp16 parts into its own accumulator.  Every stage has one owner, so an issuer waits on each of
    // its barriers' phases in order: A stages 0, 1 belong to issuer 0 and stage 2 to issuer
    // 1; B stage rg % kTmBStages carries real group rg, owned by issuer rg % 2 (every unit
    // has an even number of K groups, kTmBStages is even).
    if (lane == 0) {
      const int part = warp == kTmMma0 ? 0 : 1;
      int kown = 0, rg = 0, it = 0;
      bool ok = true, any = false;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x, it++) {
        const TmUnit U = tm_unit(A, u, mtiles);
        const uint32_t idesc = tm_idesc_f16(128, U.N);
        const int ab = it & 1, slot = it & 1;
        const uint32_t td = tmem + (uint32_t)((2 * part + ab) * kTmN);
        const int nx = 1 + ((lora_blk && U.shared) ? 1 : 0);   // extra blocks of this unit
        ok = it < 2 || tm_wait(&S.accempty[ab], (uint32_t)(((it >> 1) - 1) & 1), budget, A.err, &S.abort);
        if (!ok) break;
        bool first = true;
        for (int e = 0; e < G + nx; e++) {
          const bool real = e < G;
          const bool mine = real ? (e & 1) == part : part == 0;
          const int bs = rg % kTmBStages;
          if (e == G && part == 0 && !(ok = tm_wait(&S.ufull[slot], (uint32_t)((it >> 1) & 1), budget, A.err, &S.abort)))
            break;
          if (mine) {
            const int as = part == 0 ? (kown & 1) : 2;
            const uint32_t ph = (uint32_t)((part == 0 ? (kown >> 1) : kown) & 1);
            ok = tm_wait(&S.afull[as], ph, budget, A.err, &S.abort) &&
                 (!real || tm_wait(&S.bfull[bs], (uint32_t)((rg / kTmBStages) & 1), budget, A.err, &S.abort));
            if (!ok) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t sb = tc_smem(real ? S.b[bs] : (e == G ? S.bm[slot] : S.bl[slot]));
            const uint32_t ta = tmem + kTmACol + (uint32_t)(64 * as);
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {   // K = 16 per instruction: 8 TMEM columns of A, 32 bytes of B
              tm_mma(td, ta + 8 * kk, tc_desc(sb + kk * 32), idesc, first ? 0u : 1u);   // s (q & 14)
              first = false;
              if (real) tm_mma(td, ta + 32 + 8 * kk, tc_desc(sb + kk * 32), idesc, 1u);  // s (q & 1)
            }
            any = true;
            tc_commit(&S.aempty[as]);
            if (real) tc_commit(&S.bempty[bs]);
            kown++;
          }
          if (real) rg++;
        }
        if (!ok) break;
        tc_commit(&S.accfull[ab]);
      }
      // after an abort, the MMAs in flight finish before TMEM is given back
      if (!ok && any) {
        tc_commit(&S.drain[part]);
        tc_wait_all(&S.drain[part], 0u, budget, A.err);
      }
    }
    __syncwarp();
  } else if (warp == kTmUnitWarp) {
    // ---------------- unit warp: bookkeeping, extra blocks' B tiles, scales ---------------
    bool ok = true;
    for (int u = blockIdx.x, it = 0; u < total && ok; u += gridDim.x, it++) {
      const int slot = it & 1;
      if (it >= 2 && !(ok = tm_wait_warp(&S.uempty[slot], (uint32_t)(((it >> 1) - 1) & 1), budget, A.err, &S.abort)))
        break;
      const TmUnit U = tm_unit(A, u, mtiles);
      const int row0 = U.shared ? (A.mode == 0 ? U.n0 : A.T * A.k + U.n0) : A.P.ustart[U.unit] + U.n0;
      const bool lb = lora_blk && U.shared;
      for (int c = lane; c < kTmN; c += 32) {
        int tok = -1, dst = -1;
        float w = 0.f;
        if (c < U.ncol) {
          if (U.shared) {
            tok = U.n0 + c;
            dst = A.mode == 0 ? A.T * A.k + tok : -1;             // grouped row of a
            w = 1.f;
          } else {
            const int asg = A.P.assign[A.P.ustart[U.unit] + U.n0 + c];   // t * k + slot
            tok = asg / A.k;
            dst = A.mode == 0 ? A.P.ustart[U.unit] + U.n0 + c : asg;     // grouped row of a / gate index
            if (A.mode == 1) w = A.gates[asg];
          }
        }
        S.tok[slot][c] = tok;
        S.dst[slot][c] = dst;
        S.gw[slot][c] = w;
        // row c of the min block's B tile: the column's group sums (x by token for gate/up,
        // a by grouped row for down) split hi | lo
        const float *src = tok < 0 ? nullptr : (A.mode == 0 ? A.xsum + (size_t)tok * G : A.asum + (size_t)(row0 + c) * G);
        tm_bm_row_any<kTmMaxG>(G, S.bm[slot], c, src);
        // row c of the LoRA block's B tile: c t_g and c t_u split hi | lo
        if (lb) tm_bl_row_any<kTmMaxR>(A.r, S.bl[slot], c, tok < 0 ? nullptr : A.lt + (size_t)tok * 3 * A.r, A.c);
      }
      // the extra blocks' B tiles are read by the tensor core (async proxy)
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_mbar_arrive(&S.ufull[slot]);
    }
  } else if (warp < kTmConv0) {
    // ---------------- epilogue: TMEM -> SwiGLU / weighted combine --------------------------
    const int q = warp & 3, row = 32 * q + lane, et = tid - kTmEpi0 * 32;   // et 0..127
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    // the rows' scales and mins of a unit, two units ahead (this thread: weight row `row`)
    auto fill = [&](int it2) {
      const int u2 = blockIdx.x + it2 * gridDim.x;
      if (u2 >= total) return;
      const TmUnit U2 = tm_unit(A, u2, mtiles);
      tm_fill_scales(A, U2, G, row, S.sc[it2 & 1], S.mn[it2 & 1]);
      tc_mbar_arrive(&S.sfull[it2 & 1]);
    };
    fill(0);
    fill(1);
    bool ok = true;
    for (int u = blockIdx.x, it = 0; u < total && ok; u += gridDim.x, it++) {
      const int ab = it & 1, slot = it & 1;
      ok = tm_wait_warp(&S.accfull[ab], (uint32_t)((it >> 1) & 1), budget, A.err, &S.abort) &&
           tm_wait_warp(&S.ufull[slot], (uint32_t)((it >> 1) & 1), budget, A.err, &S.abort);
      {
        // the four epilogue warps agree (named barrier 1) before any of them uses the
        // exchange barriers below, so that none is left waiting for a warp that gave up
        uint32_t bad;
        asm volatile(
            "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbarrier.red.or.pred q, 1, %2, p;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(bad)
            : "r"((uint32_t)!ok), "r"(kTmEpiThreads)
            : "memory");
        if (bad) break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const TmUnit U = tm_unit(A, u, mtiles);
      const uint32_t t0 = tmem + tl + (uint32_t)(ab * kTmN), t1 = tmem + tl + (uint32_t)((2 + ab) * kTmN);
      if (A.mode == 0) {
        // rows 0..63 gate, 64..127 up of intermediate units i = 64 mt + (row & 63)
        const bool up = row >= 64;
        for (int h64 = 0; h64 < U.N; h64 += 64) {
          asm volatile("bar.sync 1, 128;" ::: "memory");   // the previous exchange has been read
#pragma unroll
          for (int ch = 0; ch < 2; ch++) {
            const int c0 = h64 + 32 * ch;
            if (c0 < U.N) {
              float v[32], w[32];
              tc_ld32(t0 + c0, v);
              tc_ld32(t1 + c0, w);
              float *xr = S.xch[up ? 1 : 0] + (row & 63) * kTmXRow + 32 * ch;
#pragma unroll
              for (int j = 0; j < 32; j++) xr[j] = v[j] + w[j];
            }
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
          // a = bf16(silu(g) u): thread et takes unit et % 64 of every other column
          const int iu = et & 63, ipos = kperm_pos(64 * U.mt + iu);
          for (int j = et >> 6; j < 64; j += 2) {
            const int c = h64 + j;
            if (c >= U.ncol) break;
            const int dst = S.dst[slot][c];
            if (dst < 0) continue;
            const float g = S.xch[0][iu * kTmXRow + j], uu = S.xch[1][iu * kTmXRow + j];
            // the bf16 rounding point of a, stored as the same value in fp16 (the down
            // GEMM's operand type)
            const float av = __bfloat162float(__float2bfloat16_rn(g / (1.0f + expf(-g)) * uu));
            A.ap_out[(size_t)dst * A.I + ipos] = __half_as_ushort(__float2half_rn(av));
          }
        }
      } else {
        // the gate-weighted combine into y: per chunk of 32 columns the 128 x 32 values go
        // through shared memory ([column][row], rows padded to kTmDRow), so that each thread
        // adds four consecutive rows of one token with one vector reduction (a quarter of
        // the L2 atomic operations of per-element reductions)
        float *xb = &S.xch[0][0];
        for (int ch = 0; ch < (kTmN + 31) / 32; ch++) {
          const int c0 = 32 * ch;
          if (c0 >= U.N) break;                             // block-uniform
          asm volatile("bar.sync 1, 128;" ::: "memory");   // the previous chunk has been read
          {
            float v[32], w[32];
            tc_ld32(t0 + c0, v);                           // (columns past N are read, never used)
            tc_ld32(t1 + c0, w);
#pragma unroll
            for (int j = 0; j < 32; j++) xb[j * kTmDRow + row] = v[j] + w[j];
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll 2
          for (int i = et; i < 32 * 32; i += 128) {
            const int j = i >> 5, r4 = 4 * (i & 31), c = c0 + j;
            if (c >= U.ncol) continue;
            const int tok = S.tok[slot][c];
            if (tok < 0) continue;
            const float g = S.gw[slot][c];
            const float4 val = *reinterpret_cast<const float4 *>(xb + j * kTmDRow + r4);
            if (A.ypart) {
              // fixed-order combine: this (slot, token) contribution stored once, in its own
              // plane (routed slot = assignment mod k, the shared expert's plane k)
              const int dst = S.dst[slot][c], sp = dst >= 0 ? dst % A.k : A.k;
              *reinterpret_cast<float4 *>(A.ypart + ((size_t)sp * A.T + tok) * A.d + 128 * U.mt + r4) =
                  make_float4(g * val.x, g * val.y, g * val.z, g * val.w);
            } else {
              asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(A.yacc + (size_t)tok * A.d + 128 * U.mt + r4),
                           "f"(g * val.x), "f"(g * val.y), "f"(g * val.z), "f"(g * val.w)
                           : "memory");
            }
          }
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        tc_mbar_arrive(&S.accempty[ab]);
        tc_mbar_arrive(&S.uempty[slot]);
      }
      // every MMA of this unit has completed (accfull), so every converter is done with
      // this slot's scales and mins
      fill(it + 2);
    }
  } else {
    // ---------------- converters: codes -> exact fp16 parts in TMEM ----------------------
    const int q = warp & 3, h = (warp - kTmConv0) >> 2;
    const int row = 32 * q + lane;              // weight row of the tile = TMEM lane
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    int gg = 0, cc = 0;
    bool ok = true;
    // one A-stage entry: this thread's 16 columns of part 0 (and of part 1 for a K group),
    // into the next stage of the entry's issuer (stages 0, 1: issuer 0; stage 2: issuer 1)
    int k0 = 0, k1 = 0;
    auto put = [&](const uint32_t (&p1)[16], const uint32_t (&p2)[16], bool two, int owner) -> bool {
      const int as = owner == 0 ? (k0 & 1) : 2;
      const int n = owner == 0 ? (k0 >> 1) : k1;   // earlier uses of this stage
      if (n > 0 && !tm_wait_warp(&S.aempty[as], (uint32_t)((n - 1) & 1), budget, A.err, &S.abort)) return false;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t ta = tmem + tl + kTmACol + (uint32_t)(64 * as + 16 * h);
      tm_st16(ta, p1);
      if (two) tm_st16(ta + 32, p2);
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) tc_mbar_arrive(&S.afull[as]);
      if (owner == 0) k0++;
      else k1++;
      gg++;
      return true;
    };
    for (int u = blockIdx.x, it = 0; u < total && ok; u += gridDim.x, it++) {
      const int slot = it & 1;
      if (!(ok = tm_wait_warp(&S.sfull[slot], (uint32_t)((it >> 1) & 1), budget, A.err, &S.abort))) break;
      const TmUnit U = tm_unit(A, u, mtiles);
      uint32_t p1[16], p2[16];
      for (int g0 = 0; g0 < G && ok; g0 += 4, cc++) {
        const int cs = cc % kTmCStages, ng = min(4, G - g0);
        if (!(ok = tm_wait_warp(&S.cfull[cs], (uint32_t)((cc / kTmCStages) & 1), budget, A.err, &S.abort))) break;
#pragma unroll
        for (int lg = 0; lg < 4; lg++) {
          if (lg >= ng) break;
          // half h of group g0 + lg of this row: 16 bytes = 32 codes
          const uint4 w = *reinterpret_cast<const uint4 *>(S.c[cs] + sw128(row, 2 * lg + h));
          if (lg == ng - 1) {
            __syncwarp();
            if (lane == 0) tc_mbar_arrive(&S.cempty[cs]);
          }
          const uint32_t sh = S.sc[slot][g0 + lg][row];
          const uint32_t s2 = sh | (sh << 16);
          const uint32_t c2 = tm_hfma2(s2, 0xE400E400u, 0u);    // -1024 s, exact
          const uint32_t s16 = tm_hfma2(s2, 0x2C002C00u, 0u);   // s / 16, exact for |s| >= 2^-13
          const uint32_t c16 = tm_hfma2(s2, 0xD400D400u, 0u);   // -64 s, exact
          // word j holds K elements 8 j .. 8 j + 7; nibbles n and n + 4 form the fp16 pair
          // of TMEM column 4 j + n (the K-permuted order of the activation operand).  A
          // nibble in bits 0-3 of its half gives 1024 + (q & 14) and 1024 + (q & 1) as fp16,
          // then (1024 + v) s - 1024 s = v s; one in bits 4-7 is masked in place, giving
          // 1024 + 16 v, then (1024 + 16 v)(s / 16) - 64 s = v s (one rounding, exact as
          // before); nibbles 2 and 3 are those of the word shifted right by 8
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int j = 0; j < 4; j++) {
#pragma unroll
            for (int hb = 0; hb < 2; hb++) {
              const uint32_t sv = hb ? ws[j] >> 8 : ws[j];
              const int n = 2 * hb;
              p1[4 * j + n] = tm_hfma2((sv & 0x000E000Eu) | 0x64006400u, s2, c2);
              p2[4 * j + n] = tm_hfma2((sv & 0x00010001u) | 0x64006400u, s2, c2);
              p1[4 * j + n + 1] = tm_hfma2((sv & 0x00E000E0u) | 0x64006400u, s16, c16);
              p2[4 * j + n + 1] = tm_hfma2((sv & 0x00100010u) | 0x64006400u, s16, c16);
            }
          }
          if (!(ok = put(p1, p2, true, (g0 + lg) & 1))) break;
        }
      }
      // the extra blocks last (issuer 0 takes them after its groups)
      // min block: element k of the row = m_(k mod G) for k < 2 G, else 0 (this thread's
      // elements 32 h .. 32 h + 31)
#pragma unroll
      for (int j = 0; j < 16; j++) {
        const int k0 = 32 * h + 2 * j, k1 = k0 + 1;
        const uint32_t v0 = k0 < 2 * G ? S.mn[slot][k0 < G ? k0 : k0 - G][row] : 0u;
        const uint32_t v1 = k1 < 2 * G ? S.mn[slot][k1 < G ? k1 : k1 - G][row] : 0u;
        p1[j] = v0 | (v1 << 16);
      }
      if (!ok || !(ok = put(p1, p2, false, 0))) break;
      if (lora_blk && U.shared) {
        // LoRA block: gate row i: B_g[i] at k < r and again at r <= k < 2 r; up row: B_u[i]
        // at 2 r <= k < 3 r and again at 3 r <= k < 4 r
        const int i = 64 * U.mt + (row & 63);
        const bool up = row >= 64;
        const uint16_t *Bm = (up ? A.Bu : A.Bg) + (size_t)i * A.r;
        const int k0 = up ? 2 * A.r : 0;
#pragma unroll
        for (int j = 0; j < 16; j++) {
          const int ka = 32 * h + 2 * j, kb = ka + 1;
          const int qa = ka - k0, qb = kb - k0;   // index into the doubled B row
          const uint32_t va = (qa >= 0 && qa < 2 * A.r) ? tm_bf2h(Bm[qa < A.r ? qa : qa - A.r]) : 0u;
          const uint32_t vb = (qb >= 0 && qb < 2 * A.r) ? tm_bf2h(Bm[qb < A.r ? qb : qb - A.r]) : 0u;
          p1[j] = va | (vb << 16);
        }
        if (!(ok = put(p1, p2, false, 0))) break;
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (warp == kTmMma0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmCols) : "memory");
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
// every group of 64 (natural order).  Eight threads per (row, group), one 16-byte word
// each (a warp reads four whole groups), the group sum reduced over the eight.  With `pos`
// (x rows only), each permuted word also goes to the expert-grouped rows of the row's
// k assignments (xg row pos[r k + j]), so that each routed expert's tokens are consecutive.
// ---------------------------------------------------------------------------------------
__global__ void k_perm_sums(const uint16_t *__restrict__ x, long long rows, int K, uint16_t *__restrict__ xp,
                            float *__restrict__ sums, int in_f16, const int32_t *__restrict__ pos, int k,
                            uint16_t *__restrict__ xg) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int G = K / 64;
  const long long rg = i >> 3;            // (row, group)
  const int q = (int)(i & 7);             // this thread's word of the group
  const bool live = rg < rows * G;        // whole octets are live or not (blockDim % 8 == 0)
  const long long r = live ? rg / G : 0;
  const int g = live ? (int)(rg % G) : 0;
  // 16-bit element -> fp32 (bf16 or fp16 input), and a bf16 element as the same fp16 value
  auto val = [&](uint32_t b) { return in_f16 ? __half2float(__ushort_as_half((uint16_t)b)) : bf(b); };
  auto h16 = [&](uint32_t b) { return (uint32_t)__half_as_ushort(__float2half_rn(bf(b))); };
  float s = 0.f;
  if (live) {
    const uint4 v = reinterpret_cast<const uint4 *>(x + r * K + g * 64)[q];
    // natural elements 8q .. 8q+7 = (v.x lo, v.x hi, v.y lo, v.y hi, v.z lo, ...)
    s += val(v.x & 0xFFFFu);
    s += val(v.x >> 16);
    s += val(v.y & 0xFFFFu);
    s += val(v.y >> 16);
    s += val(v.z & 0xFFFFu);
    s += val(v.z >> 16);
    s += val(v.w & 0xFFFFu);
    s += val(v.w >> 16);
    if (xp) {   // bf16 input -> the fp16 tensor-core operand, permuted block (0,4,1,5,2,6,3,7)
      const uint32_t e0 = h16(v.x & 0xFFFFu), e1 = h16(v.x >> 16), e2 = h16(v.y & 0xFFFFu), e3 = h16(v.y >> 16);
      const uint32_t e4 = h16(v.z & 0xFFFFu), e5 = h16(v.z >> 16), e6 = h16(v.w & 0xFFFFu), e7 = h16(v.w >> 16);
      const uint4 pw = make_uint4(e0 | (e4 << 16), e1 | (e5 << 16), e2 | (e6 << 16), e3 | (e7 << 16));
      reinterpret_cast<uint4 *>(xp + r * K + g * 64)[q] = pw;
      if (pos)
        for (int j = 0; j < k; j++) {
          const int p = pos[r * k + j];
          if (p >= 0) reinterpret_cast<uint4 *>(xg + (size_t)p * K + g * 64)[q] = pw;
        }
    }
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (live && q == 0) sums[rg] = s;
}

// t_d = Ad a_s from the K-permuted activations (fp16 holding the bf16 values of a; one warp
// per token and rank row); the shared expert's a rows are rows T k .. T k + T - 1 of the
// grouped a
__global__ void k_lora_td(const uint16_t *__restrict__ Ad, const uint16_t *__restrict__ ap, int T, int I, int k,
                          int r, float *__restrict__ lt) {
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= T * r) return;
  const int t = w / r, j = w % r;
  const uint16_t *as = ap + ((size_t)T * k + t) * I;
  const uint16_t *ad = Ad + (size_t)j * I;
  float acc = 0.f;
  if (I % 8 == 0 && ((uintptr_t)ad & 15) == 0) {
    // one 8-block per lane and step: a (fp16 holding its bf16 values) is stored in the
    // block order (0,4,1,5,2,6,3,7), A_d in natural order
    for (int b = lane; b < I / 8; b += 32) {
      const uint4 aw = *reinterpret_cast<const uint4 *>(as + 8 * b), dw = *reinterpret_cast<const uint4 *>(ad + 8 * b);
      const uint32_t av[4] = {aw.x, aw.y, aw.z, aw.w}, dv[4] = {dw.x, dw.y, dw.z, dw.w};
#pragma unroll
      for (int m = 0; m < 4; m++) {
        // a word m holds elements m (low) and m + 4 (high); A_d word m / 2 holds 2 (m/2)..
        const uint32_t d_lo = (m & 1) ? dv[m >> 1] >> 16 : dv[m >> 1] & 0xFFFFu;        // element m
        const uint32_t d_hi = (m & 1) ? dv[2 + (m >> 1)] >> 16 : dv[2 + (m >> 1)] & 0xFFFFu;   // element m + 4
        acc = fmaf(bf(d_lo), __half2float(__ushort_as_half((uint16_t)(av[m] & 0xFFFFu))), acc);
        acc = fmaf(bf(d_hi), __half2float(__ushort_as_half((uint16_t)(av[m] >> 16))), acc);
      }
    }
  } else {
    for (int i = lane; i < I; i += 32) acc = fmaf(bf(ad[i]), __half2float(__ushort_as_half(as[kperm_pos(i)])), acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) lt[((size_t)t * 3 + 2) * r + j] = acc;
}

// y = yacc + c Bd t_d  -> fp32 and bf16 outputs; with ypart (the fixed-order combine), the
// accumulated value is instead the sum of the token's nslot planes in plane order.  One
// block per token: t_d in shared memory, each thread a strided set of output rows n with
// its B_d row in 16-byte loads.
__global__ void k_tc_finish(const float *__restrict__ yacc, const float *__restrict__ ypart, int nslot,
                            const uint16_t *__restrict__ Bd, const float *__restrict__ lt, int T, int d, int r,
                            float c, uint16_t *__restrict__ y, float *__restrict__ yf) {
  const int t = blockIdx.x;
  __shared__ float td[kMaxR];
  if (Bd && threadIdx.x < r) td[threadIdx.x] = lt[((size_t)t * 3 + 2) * r + threadIdx.x];
  __syncthreads();
  for (int n = threadIdx.x; n < d; n += blockDim.x) {
    const size_t i = (size_t)t * d + n;
    float v;
    if (ypart) {
      v = 0.f;
      for (int j = 0; j < nslot; j++) v += ypart[((size_t)j * T + t) * d + n];
    } else {
      v = yacc[i];
    }
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
