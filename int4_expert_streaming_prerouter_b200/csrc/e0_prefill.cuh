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
constexpr int kTcN = 128;           // tokens per tile (TMEM columns)
constexpr int kTcStages = 4;
constexpr int kTcStageA = 128 * 128;      // 128 rows x 64 fp16
constexpr int kTcStageB = kTcN * 128;     // 128 tokens x 64 fp16

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
  const __half *x16;        // [T, d] (mode 0)
  const __half *a16;        // [T, k+1, I] (mode 1 input)
  __half *a16_out;          // [T, k+1, I] (mode 0 output)
  const uint16_t *Bg, *Bu;  // [I, r] shared-expert LoRA up (mode 0), or nullptr
  const float *lt;          // [T, 3, r]
  const float *gates;       // [T, k] (mode 1)
  float *yacc;              // [T, d] (mode 1)
  int *err;
  unsigned long long timeout_ns;
};

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

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and B fp16
// (bits 7-9, 10-12 = 0), both K-major (bits 15, 16 = 0), N >> 3 (bits 17-22), M >> 4
// (bits 24-28).
__device__ __forceinline__ uint32_t tc_idesc(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
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
// The grouped GEMM.  grid = max tiles x M tiles per expert; blocks past the real tile
// count return at once.
// ---------------------------------------------------------------------------------------
struct TcSmem {
  uint8_t a[kTcStages][kTcStageA];      // fp16(w)
  uint8_t alo[kTcStages][kTcStageA];    // fp16(w - fp16(w))
  uint8_t b[kTcStages][kTcStageB];
  uint64_t done[kTcStages];
  uint64_t fin;
  uint32_t tmem;
  int tok[kTcN];       // token of each column
  int dst[kTcN];       // a16 row (mode 0) / gate index (mode 1) of each column, -1 = none
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
  const int nkb = K / 64;

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
    for (int s = 0; s < kTcStages; s++) tc_mbar_init(&S.done[s], 1);
    tc_mbar_init(&S.fin, 1);
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
  bool ok = true;

  // A producer role: two threads per weight row, each 32 of the 64 K elements of a block.
  // mode 0 -> gate rows i0..i0+63 then up rows i0..i0+63 (i0 = 64 mt); mode 1 -> down
  // rows 128 mt .. 128 mt + 127
  const int row = tid >> 1, half = tid & 1;
  const uint8_t *codes;
  const uint16_t *scl, *mnv;
  if (A.mode == 0) {
    const int i = mt * 64 + (row & 63);
    const bool up = row >= 64;
    codes = base + (up ? A.bl.uc : A.bl.gc) + (size_t)i * (A.d / 2);
    scl = reinterpret_cast<const uint16_t *>(base + (up ? A.bl.us : A.bl.gs)) + (size_t)i * (A.d / 64);
    mnv = reinterpret_cast<const uint16_t *>(base + (up ? A.bl.um : A.bl.gm)) + (size_t)i * (A.d / 64);
  } else {
    const int n = mt * 128 + row;
    codes = base + A.bl.dc + (size_t)n * (A.I / 2);
    scl = reinterpret_cast<const uint16_t *>(base + A.bl.ds) + (size_t)n * (A.I / 64);
    mnv = reinterpret_cast<const uint16_t *>(base + A.bl.dm) + (size_t)n * (A.I / 64);
  }
  // B producer role: (column, chunk) pairs e = tid + m * kTcThreads, m < kBPer
  constexpr int kBPer = kTcN * 8 / kTcThreads;
  const __half *bsrc[kBPer];
#pragma unroll
  for (int m = 0; m < kBPer; m++) {
    const int e = tid + m * kTcThreads, c = e >> 3, ch = e & 7;
    const int tok = c < N ? S.tok[c] : -1;
    bsrc[m] = nullptr;
    if (tok >= 0)
      bsrc[m] = (A.mode == 0 ? A.x16 + (size_t)tok * A.d
                             : A.a16 + (size_t)(tok * (A.k + 1) + (shared ? A.k : S.dst[c] % A.k)) * A.I) + ch * 8;
  }
  // loads of one K block into registers (issued one block ahead of their use)
  uint4 qa, qb[kBPer];
  float sc = 0.f, mn = 0.f;
  auto load_block = [&](int kb) {
    qa = __ldg(reinterpret_cast<const uint4 *>(codes + kb * 32 + half * 16));
    sc = bf(__ldg(scl + kb));
    mn = bf(__ldg(mnv + kb));
#pragma unroll
    for (int m = 0; m < kBPer; m++)
      qb[m] = bsrc[m] ? __ldg(reinterpret_cast<const uint4 *>(bsrc[m] + kb * 64)) : make_uint4(0u, 0u, 0u, 0u);
  };
  load_block(0);

  int issued = 0;   // K blocks whose MMAs were issued (uniform across the block)
#pragma unroll 1
  for (int kb = 0; kb < nkb && ok; kb++) {
    const int s = kb % kTcStages;
    // this block's data, then start the next block's loads
    const uint4 ca = qa;
    const float csc = sc, cmn = mn;
    uint4 cb[kBPer];
#pragma unroll
    for (int m = 0; m < kBPer; m++) cb[m] = qb[m];
    if (kb + 1 < nkb) load_block(kb + 1);
    if (kb >= kTcStages) ok = tc_wait(&S.done[s], (uint32_t)(((kb / kTcStages) - 1) & 1), A);
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    // A: 32 weights -> fp16 hi + lo (about 22 significant bits together), swizzled
    {
      const uint32_t w[4] = {ca.x, ca.y, ca.z, ca.w};
      uint8_t *dstA = S.a[s], *dstL = S.alo[s];
#pragma unroll
      for (int j = 0; j < 4; j++) {
        // code word j of this half = K elements 8 (4 half + j) .. + 7 = chunk 4 half + j
        const uint32_t wd = w[j];
        __half2 h[4], l[4];
#pragma unroll
        for (int p = 0; p < 4; p++) {
          const float w0 = fmaf(csc, (float)((wd >> (8 * p)) & 0xFu), cmn);
          const float w1 = fmaf(csc, (float)((wd >> (8 * p + 4)) & 0xFu), cmn);
          h[p] = __floats2half2_rn(w0, w1);
          const float2 hf = __half22float2(h[p]);
          l[p] = __floats2half2_rn(w0 - hf.x, w1 - hf.y);
        }
        const uint32_t off = sw128(row, half * 4 + j);
        *reinterpret_cast<uint4 *>(dstA + off) =
            make_uint4(*reinterpret_cast<uint32_t *>(&h[0]), *reinterpret_cast<uint32_t *>(&h[1]),
                       *reinterpret_cast<uint32_t *>(&h[2]), *reinterpret_cast<uint32_t *>(&h[3]));
        *reinterpret_cast<uint4 *>(dstL + off) =
            make_uint4(*reinterpret_cast<uint32_t *>(&l[0]), *reinterpret_cast<uint32_t *>(&l[1]),
                       *reinterpret_cast<uint32_t *>(&l[2]), *reinterpret_cast<uint32_t *>(&l[3]));
      }
    }
    // B: token rows of this K block (zero for padding columns), swizzled
#pragma unroll
    for (int m = 0; m < kBPer; m++) {
      const int e = tid + m * kTcThreads, c = e >> 3, ch = e & 7;
      if (c < N) *reinterpret_cast<uint4 *>(S.b[s] + sw128(c, ch)) = cb[m];
    }
    // generic-proxy smem writes -> visible to the tensor core (async proxy)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t sa = tc_smem(S.a[s]), sl = tc_smem(S.alo[s]), sb = tc_smem(S.b[s]);
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {   // K = 16 per instruction: advance 32 bytes in the swizzled row
        tc_mma(tmem, tc_desc(sa + kk * 32), tc_desc(sb + kk * 32), idesc, (kb | kk) ? 1u : 0u);
        tc_mma(tmem, tc_desc(sl + kk * 32), tc_desc(sb + kk * 32), idesc, 1u);
      }
      tc_commit(&S.done[s]);
    }
    issued = kb + 1;
  }
  if (tid == 0 && ok) tc_commit(&S.fin);
  if (ok) ok = tc_wait(&S.fin, 0, A);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (__syncthreads_or(!ok)) {
    // drain any MMA still in flight on the stages before giving TMEM back
    for (int s = 0; s < kTcStages; s++) {
      const int uses = (issued - s + kTcStages - 1) / kTcStages;
      if (uses > 0) tc_wait(&S.done[s], (uint32_t)((uses - 1) & 1), A);
    }
    __syncthreads();
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcN) : "memory");
    return;
  }

  // ------------------------------- epilogue ------------------------------------------
  // warp w reads TMEM lanes 32 (w % 4) .. + 31 (tile row = that lane); warps 0-3 take the
  // first half of the columns, warps 4-7 the second
  const int erow = 32 * (warp & 3) + (tid & 31);
  const int cbeg = (warp >> 2) * (kTcN / 2);
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  float *ex = reinterpret_cast<float *>(S.b[0]);   // 64 x kTcN floats: the up values (mode 0)
  if (A.mode == 0) {
    const int i = mt * 64 + (erow & 63);
    const bool up = erow >= 64;
    float lb[kMaxR];
    const bool lora = shared && A.Bg != nullptr;
    if (lora)
      for (int q = 0; q < A.r; q++) lb[q] = bf((up ? A.Bu : A.Bg)[(size_t)i * A.r + q]);
#pragma unroll 1
    for (int c0 = cbeg; c0 < cbeg + kTcN / 2; c0 += 32) {
      float v[32];
      const bool live = c0 < N;
      if (live) tc_ld32(lane_addr + c0, v);
      if (live && lora)
        for (int cc = 0; cc < 32; cc++) {
          const int tok = S.tok[c0 + cc];
          if (tok < 0) continue;
          const float *t = A.lt + (size_t)tok * 3 * A.r + (up ? A.r : 0);
          float acc = 0.f;
          for (int q = 0; q < A.r; q++) acc = fmaf(lb[q], t[q], acc);
          v[cc] = fmaf(A.c, acc, v[cc]);
        }
      if (live && up)
        for (int cc = 0; cc < 32; cc++) ex[(erow - 64) * kTcN + c0 + cc] = v[cc];
      __syncthreads();
      if (live && !up)
        for (int cc = 0; cc < 32; cc++) {
          const int dst = S.dst[c0 + cc];
          if (dst < 0) continue;
          const float g = v[cc], u = ex[erow * kTcN + c0 + cc];
          const float act = bf(f2bf(g / (1.0f + expf(-g)) * u));   // bf16 rounding point of a
          A.a16_out[(size_t)dst * A.I + i] = __float2half_rn(act);
        }
      __syncthreads();
    }
  } else {
    const int n = mt * 128 + erow;
#pragma unroll 1
    for (int c0 = cbeg; c0 < cbeg + kTcN / 2 && c0 < N; c0 += 32) {
      float v[32];
      tc_ld32(lane_addr + c0, v);
      for (int cc = 0; cc < 32; cc++) {
        const int tok = S.tok[c0 + cc];
        if (tok < 0) continue;
        const float w = shared ? 1.0f : A.gates[S.dst[c0 + cc]];
        atomicAdd(A.yacc + (size_t)tok * A.d + n, w * v[cc]);
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcN) : "memory");
}

// bf16 activations -> fp16 (exact for |x| in the fp16 normal range)
__global__ void k_bf16_to_f16(const uint16_t *__restrict__ x, __half *__restrict__ y, size_t n) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = __float2half_rn(bf(x[i]));
}

// t_d = Ad a_s from the fp16 activations (one warp per token and rank row)
__global__ void k_lora_t16(const uint16_t *__restrict__ Ad, const __half *__restrict__ a, int T, int I, int k,
                           int r, float *__restrict__ lt) {
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= T * r) return;
  const int t = w / r, j = w % r;
  const __half *as = a + ((size_t)t * (k + 1) + k) * I;
  float acc = 0.f;
  for (int i = lane; i < I; i += 32) acc = fmaf(bf(Ad[(size_t)j * I + i]), __half2float(as[i]), acc);
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
