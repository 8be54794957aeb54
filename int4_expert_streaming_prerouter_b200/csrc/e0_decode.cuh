// Persistent decode kernel: one launch runs one decode step of one stream through every
// layer of the stack.
//
// Method (pages: "The Other Half of the Memory Wall" reading guide, "Temel fikirler",
// "Ön Yönlendirici Başlık Mimarisi", "Birleştirilmemiş Adaptör Yürütme", "Sorular"; the
// ai.info article "Edge0 serve un MoE da 35B ..."): per layer, x = bf16(RMSNorm(h)); the
// routing is the previous layer's head prediction made one token earlier, or the layer's
// own router top-k; y = sum_j w_j E_j(x) + E_shared(x) (+ unmerged LoRA); the layer's
// head predicts the next layer's routing for the next token.
//
// B200 design:
//   * One CTA per SM, launched cooperatively (co-residency guaranteed).  Warp 0 is the
//     producer: it streams each task's weight bytes (expert rows, router/head/LoRA rows,
//     norm gamma, the layer input) into a shared-memory ring with 1-D TMA bulk copies
//     (cp.async.bulk, mbarrier completion).  Because the routing of a predicted layer is
//     known a whole token ahead, the producer runs ahead of the data dependencies and keeps
//     HBM busy while the consumers wait for other CTAs.
//   * Consumers (12 warps) compute warp-per-row int4 dot products with fp32 accumulation
//     (packed f32x2 FMA), the SwiGLU, the LoRA branch and the weighted combine.
//   * CTAs exchange results (a, y, LoRA intermediates, logits) through global memory as
//     64-bit words {32-bit tag, payload} written with one relaxed store; a reader polls the
//     data itself until every tag matches, so there is no separate barrier round trip.
//     Tags are unique per (launch, layer).  Every wait is bounded by a %globaltimer budget;
//     on expiry the kernel latches DERR_TIMEOUT, drains its copies and returns.
//   * Work per layer is split into contiguous, balanced ranges per CTA: the (k+1)*I
//     intermediate rows of the gate/up phase and the d output rows of the down phase.
#pragma once
#include "e0_device.cuh"
#include "e0_kernels.cuh"

namespace e0 {

constexpr int kDecThreads = 416;          // 1 producer warp + 12 consumer warps
constexpr int kDecConsumers = 384;
constexpr int kDecCW = 12;
constexpr int kRingBytes = 142 * 1024;
constexpr int kDecMaxK = 4;               // routed experts per token on this path
constexpr int kNSlot = 8;                 // tasks in flight
constexpr int kMaxSeg = 96;               // bulk-copy segments per task

struct DecLayer {
  const uint8_t *experts;
  const uint8_t *shared;
  const uint16_t *Ag, *Bg, *Au, *Bu, *Ad, *Bd;
  const uint16_t *router;
  const uint16_t *gamma;
  const uint16_t *head;   // nullptr: no head
};

struct DecodeParams {
  const DecLayer *layers;
  int L, E, k, r, ldh, onehot, G;
  float eps, c;
  const uint16_t *h;        // [L][D]
  uint16_t *y;              // [L][D]
  float *yf;                // [L][D] or nullptr
  int chained;
  // 0: layers run in order, each layer's first stage waiting for the previous layer's
  // output; > 0 (unchained inputs only): the stages of different layers overlap, the down
  // stage of a layer running `lag` layers behind its gate/up stage
  int lag;
  uint32_t epoch;
  int step0;                // 1: every layer routes with its own router
  const int32_t *pred_in;   // [L+1][maxT][k]: routing predicted for layer l (previous step)
  int32_t *pred_out;        // [L+1][maxT][k]
  int32_t *hist_out;        // [L][maxT][k]: routing used this step
  const int32_t *hist_prev; // [L][maxT][k] or nullptr (previous step's routing)
  int maxT;
  unsigned long long *t_y, *t_rlog, *t_hlog;
  // per layer one block of tagged words produced by the gate/up stage and read by the
  // down stage: [a of the routed slots (k*I) | shared raw g,u (2I) | t_g,t_u (2r) |
  // selected router logits (k)]; `blk` words per layer
  unsigned long long *t_blk;
  int blk;
  int *err;
  unsigned long long timeout_ns;
  int stall_cta;            // test hook: this CTA waits on a tag nobody writes (-1: none)
  unsigned long long *trace;  // optional [G][L][16] %globaltimer stamps (profiling), or nullptr
};

// Timeline stamps of the optional trace (one row of 16 per CTA and layer).
enum : int {
  TR_LAYER = 0, TR_NORM = 1, TR_ROUTE = 2, TR_GU_FULL = 3, TR_GU_DONE = 4, TR_A_POLL = 5,
  TR_TD_POLL = 6, TR_DN_FULL = 7, TR_DN_DONE = 8, TR_P_GU = 9, TR_P_DN = 10, TR_P_R = 11,
  TR_P_GU_START = 12, TR_P_DN_START = 13, TR_GU_ROWS = 14, TR_DN_DOTS = 15
};

// ---------------------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void stamp(const DecodeParams &P, int l, int ev) {
  if (P.trace) P.trace[((size_t)blockIdx.x * P.L + l) * 16 + ev] = gtimer();
}
__device__ __forceinline__ unsigned long long ld_tag(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_tag(unsigned long long *p, uint32_t tag, uint32_t payload) {
  const unsigned long long v = ((unsigned long long)payload << 32) | tag;
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// consumer-only barrier (named barrier 1) that also ORs a predicate across the consumers
__device__ __forceinline__ bool cbar_or(bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbarrier.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(kDecConsumers)
      : "memory");
  return out != 0;
}
__device__ __forceinline__ void cbar() {
  asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumers) : "memory");
}
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

// Balanced contiguous split of N items over G parts (N * G < 2^31 here).
__host__ __device__ __forceinline__ void split_range(int N, int G, int c, int &a, int &b) {
  a = (int)((unsigned)(N * c) / (unsigned)G);
  b = (int)((unsigned)(N * (c + 1)) / (unsigned)G);
}

// nibble i of a 32-bit code word is placed in the mantissa of 2^23 + q * 2^p(i) without
// shifting (i < 5) or after one shift by 12 (i >= 5); the matching activation is
// pre-scaled by 2^-p(i) so that the product is exactly q * x.
__host__ __device__ constexpr float nib_scale(int i) {
  return i == 0 ? 1.f : i == 1 ? 1.f / 16 : (i == 2 || i == 5) ? 1.f / 256 : (i == 3 || i == 6) ? 1.f / 4096 : 1.f / 65536;
}

// sum_k q_k x'_k over one 16-byte chunk (32 nibbles) with the 32 pre-scaled activations
// held in registers.  Exact products (q * 2^p times x * 2^-p), fp32 pairwise accumulation
// with packed f32x2 instructions.
__device__ __forceinline__ float chunk_qdot(const uint4 w, const float (&xr)[32]) {
  const unsigned long long kMagic = pk2(-8388608.f, -8388608.f);
  unsigned long long acc0 = 0ull, acc1 = 0ull;
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int t = 0; t < 4; t++) {
    const uint32_t a = ws[t], b = a >> 12;
    const uint32_t v0 = (a & 0x0000000Fu) | 0x4B000000u, v1 = (a & 0x000000F0u) | 0x4B000000u;
    const uint32_t v2 = (a & 0x00000F00u) | 0x4B000000u, v3 = (a & 0x0000F000u) | 0x4B000000u;
    const uint32_t v4 = (a & 0x000F0000u) | 0x4B000000u, v5 = (b & 0x00000F00u) | 0x4B000000u;
    const uint32_t v6 = (b & 0x0000F000u) | 0x4B000000u, v7 = (b & 0x000F0000u) | 0x4B000000u;
    const unsigned long long q01 = f2add(((unsigned long long)v1 << 32) | v0, kMagic);
    const unsigned long long q23 = f2add(((unsigned long long)v3 << 32) | v2, kMagic);
    const unsigned long long q45 = f2add(((unsigned long long)v5 << 32) | v4, kMagic);
    const unsigned long long q67 = f2add(((unsigned long long)v7 << 32) | v6, kMagic);
    acc0 = f2fma(q01, pk2(xr[8 * t + 0], xr[8 * t + 1]), acc0);
    acc1 = f2fma(q23, pk2(xr[8 * t + 2], xr[8 * t + 3]), acc1);
    acc0 = f2fma(q45, pk2(xr[8 * t + 4], xr[8 * t + 5]), acc0);
    acc1 = f2fma(q67, pk2(xr[8 * t + 6], xr[8 * t + 7]), acc1);
  }
  return f2sum(acc0) + f2sum(acc1);
}

// Activations live in shared memory "chunk-transposed": element e of a row of n16 chunks
// (32 elements each) sits at float index (((e & 31) >> 2) * n16 + (e >> 5)) * 4 + (e & 3),
// so the lanes of a warp, each owning one chunk, read their 32 values with eight
// conflict-free 16-byte loads.
__host__ __device__ __forceinline__ int xt_index(int e, int n16) {
  return ((((e & 31) >> 2) * n16) + (e >> 5)) * 4 + (e & 3);
}
__device__ __forceinline__ void load_chunk(const float *xt, int n16, int ch, float (&xr)[32]) {
#pragma unroll
  for (int q = 0; q < 8; q++) {
    const float4 v = *reinterpret_cast<const float4 *>(xt + (q * n16 + ch) * 4);
    xr[4 * q] = v.x;
    xr[4 * q + 1] = v.y;
    xr[4 * q + 2] = v.z;
    xr[4 * q + 3] = v.w;
  }
}

// Round a double to bf16 (nearest, ties to even) on its bit pattern: keep 7 of the 52
// fraction bits.  Exact for every value in the normal bf16 range; the result is then a
// binary32 value, whose top half is the bf16.
__device__ __forceinline__ uint16_t d2bf_bits(double v) {
  unsigned long long b = (unsigned long long)__double_as_longlong(v);
  b += 0x00000FFFFFFFFFFFull + ((b >> 45) & 1ull);
  b &= ~0x00001FFFFFFFFFFFull;
  return (uint16_t)(__float_as_uint((float)__longlong_as_double((long long)b)) >> 16);
}

// ---------------------------------------------------------------------------------------
// Task layout shared by the producer (which copies) and the consumers (which read).
// ---------------------------------------------------------------------------------------
struct Seg {
  const uint8_t *src;
  uint32_t bytes;
};

struct TaskBuf {
  int n;
  int overflow;
  Seg s[kMaxSeg];
  __device__ __forceinline__ void add(const void *p, size_t bytes) {
    if (n < kMaxSeg) s[n++] = Seg{(const uint8_t *)p, (uint32_t)bytes};
    else overflow = 1;
  }
};

enum : int { TK_ROUTER = 0, TK_GU = 1, TK_DN = 2 };

// Items of a launch's schedule, the same sequence for the producer and the consumers:
//   IT_R   router rows of a reactive layer (producer task),
//   IT_TK  top-k of a reactive layer over every CTA's router logits (consumers only),
//   IT_GU  gate/up stage (producer task), IT_DN  down + combine stage (producer task).
enum : int { IT_R = 0, IT_TK = 1, IT_GU = 2, IT_DN = 3 };
constexpr int kMaxSched = 4 * 64;

// GU range of a CTA split into per-slot pieces.
struct GuPiece {
  int slot, i0, i1;
};

template <int D, int I>
__device__ __forceinline__ int gu_pieces(int k, int G, int c, GuPiece *out) {
  int a, b;
  split_range((k + 1) * I, G, c, a, b);
  int n = 0;
  while (a < b) {
    const int slot = a / I, end = min(b, (slot + 1) * I);
    out[n++] = GuPiece{slot, a - slot * I, end - slot * I};
    a = end;
  }
  return n;
}

// Segment indices of each task kind (a segment may be empty):
//   router task: [0] gamma, [1] h, [2] this CTA's router rows
//   gate/up task: [0] gamma, [1] h, [2] A_g rows, [3] A_u rows, [4, 4+kMaxK) selected
//     router rows, [4+kMaxK] head rows, then per piece p (up to kMaxPieces) 6 segments:
//     gate codes, gate scale, gate min, up codes, up scale, up min
//   down task: [3j .. 3j+2] down codes/scale/min of slot j (j = 0..k), then B_d rows, B_g,
//     B_u, A_d (LoRA matrices of the shared expert, whole)
constexpr int kMaxPieces = 4;
constexpr int kGuHead = 4 + kMaxK;
constexpr int kGuPiece0 = 5 + kMaxK;
__device__ __forceinline__ int dn_bd(int k) { return 3 * (k + 1); }

// Build the segment list of task (kind, layer) for CTA c.  `sel` are the layer's routed
// experts.  The consumer code reads the segments back by the indices above.
template <int D, int I>
__device__ __noinline__ void build_task(const DecodeParams &P, const DecLayer &Y, int kind, int l, int c, bool predicted,
                           const int *sel, TaskBuf &T) {
  const Blob bl = blob_of(D, I);
  T.n = 0;
  T.overflow = 0;
  if (kind == TK_ROUTER) {
    T.add(Y.gamma, D * 2);
    T.add(P.h + (size_t)l * D, D * 2);
    int a, b;
    split_range(P.E, P.G, c, a, b);
    T.add(Y.router + (size_t)a * D, (size_t)(b - a) * D * 2);
  } else if (kind == TK_GU) {
    T.add(Y.gamma, D * 2);
    T.add(P.h + (size_t)l * D, D * 2);
    int a = 0, b = 0;
    if (Y.Ag) split_range(2 * P.r, P.G, c, a, b);
    const int ga = min(a, P.r), gb = min(b, P.r), ua = max(a, P.r) - P.r, ub = max(b, P.r) - P.r;
    T.add(Y.Ag + (size_t)ga * D, (size_t)(gb - ga) * D * 2);
    T.add(Y.Au + (size_t)ua * D, (size_t)(ub - ua) * D * 2);
    a = b = 0;
    if (predicted) split_range(P.k, P.G, (c + P.G - min(2 * P.r, P.G - 1)) % P.G, a, b);
    #pragma unroll 1
    for (int q = 0; q < kMaxK; q++) {
      const bool on = a + q < b;
      T.add(Y.router + (size_t)(on ? sel[a + q] : 0) * D, on ? D * 2 : 0);
    }
    int ha = 0, hb = 0;
    if (Y.head) split_range(P.E, P.G, c, ha, hb);
    T.add(Y.head + (size_t)ha * P.ldh, (size_t)(hb - ha) * P.ldh * 2);
    GuPiece pc[kMaxPieces];
    const int np = gu_pieces<D, I>(P.k, P.G, c, pc);
    #pragma unroll 1
    for (int p = 0; p < np; p++) {
      const uint8_t *base = pc[p].slot < P.k ? Y.experts + (size_t)sel[pc[p].slot] * bl.bytes : Y.shared;
      const int R = pc[p].i1 - pc[p].i0, i0 = pc[p].i0;
      T.add(base + bl.gc + (size_t)i0 * (D / 2), (size_t)R * (D / 2));
      T.add(base + bl.gs + (size_t)i0 * (D / 64) * 2, (size_t)R * (D / 64) * 2);
      T.add(base + bl.gm + (size_t)i0 * (D / 64) * 2, (size_t)R * (D / 64) * 2);
      T.add(base + bl.uc + (size_t)i0 * (D / 2), (size_t)R * (D / 2));
      T.add(base + bl.us + (size_t)i0 * (D / 64) * 2, (size_t)R * (D / 64) * 2);
      T.add(base + bl.um + (size_t)i0 * (D / 64) * 2, (size_t)R * (D / 64) * 2);
    }
  } else {
    int a, b;
    split_range(D, P.G, c, a, b);
    const int R = b - a;
    #pragma unroll 1
    for (int j = 0; j <= P.k; j++) {
      const uint8_t *base = j < P.k ? Y.experts + (size_t)sel[j] * bl.bytes : Y.shared;
      T.add(base + bl.dc + (size_t)a * (I / 2), (size_t)R * (I / 2));
      T.add(base + bl.ds + (size_t)a * (I / 64) * 2, (size_t)R * (I / 64) * 2);
      T.add(base + bl.dm + (size_t)a * (I / 64) * 2, (size_t)R * (I / 64) * 2);
    }
    T.add(Y.Bd + (size_t)a * P.r, Y.Bd ? (size_t)R * P.r * 2 : 0);
    const size_t lb = Y.Bg ? (size_t)I * P.r * 2 : 0;
    T.add(Y.Bg, lb);
    T.add(Y.Bu, lb);
    T.add(Y.Ad, lb);
  }
}

// ---------------------------------------------------------------------------------------
// Shared-memory layout
// ---------------------------------------------------------------------------------------
template <int D, int I>
struct DecSmem {
  uint8_t ring[kRingBytes];
  float x[D];                        // x (natural order): router, head and LoRA rows
  float xt[D];                       // x pre-scaled per nibble position, chunk-transposed
  float yprev[D];                    // previous layer's y (fp32)
  float at[(kDecMaxK + 1) * I];      // a of every slot, pre-scaled, chunk-transposed per slot
  uint32_t stg[kDecMaxK * I];        // routed a payloads as polled
  float asraw[I];                    // the shared expert's a (natural order, for t_d)
  float gus[2 * I];                  // the shared expert's raw g and u (interleaved per row)
  float ydot[64 * (kMaxK + 1)];
  double dred[16];
  float gates[kMaxK];
  float tl[2 * kMaxR];               // t_g, t_u
  float td[kMaxR];                   // t_d
  float rl[kMaxE];                   // router logits (reactive) / selected logits / head logits
  int sel_all[64][kMaxK];            // routing of every layer this step
  float rlsel[64][kMaxK];            // a reactive layer's router logits of its chosen experts
  volatile int sel_ok[64];           // 1 once a reactive layer's top-k is in sel_all
  uint16_t sched[kMaxSched];         // this launch's items: kind << 8 | layer
  int nsched;
  DecLayer lay[64];                  // the layer table
  TaskBuf tb;                        // the producer's task being issued
  int tb_off[kMaxSeg];
  uint32_t seg_off[kNSlot][kMaxSeg]; // ring byte offset of each segment's first wanted byte
  uint64_t full[kNSlot], empty[kNSlot];
  volatile int abort;
};

static_assert(sizeof(DecSmem<2048, 512>) <= 232448, "decode kernel shared memory exceeds 227 KB");

template <int D, int I>
__device__ __forceinline__ bool is_predicted(const DecodeParams &P, const DecSmem<D, I> &S, int l) {
  return !P.step0 && l > 0 && S.lay[l - 1].head != nullptr;
}

__device__ __forceinline__ uint32_t dtag(const DecodeParams &P, int l) { return P.epoch * 64u + (uint32_t)l; }

__device__ __forceinline__ bool timed_out(unsigned long long &t0, unsigned long long budget) {
  const unsigned long long now = gtimer();
  if (!t0) {
    t0 = now;
    return false;
  }
  return now - t0 > budget;
}

// ---------------------------------------------------------------------------------------
// The launch's schedule (one thread).  In order (lag 0): per layer [R, TK] GU DN.  With a
// lag (unchained inputs: no layer reads another layer's output within the step): the
// layers are taken predicted first, then reactive; the router rows of every reactive
// layer come first, a reactive layer's top-k two layers before its gate/up stage (so the
// producer can fetch its experts early), and each down stage `lag` layers after its
// gate/up stage, so that the exchange between the two stages overlaps other layers' work.
// ---------------------------------------------------------------------------------------
template <int D, int I>
__device__ __noinline__ void build_schedule(const DecodeParams &P, DecSmem<D, I> &S) {
  int n = 0;
  if (P.lag == 0) {
    #pragma unroll 1
    for (int l = 0; l < P.L; l++) {
      if (!is_predicted(P, S, l)) {
        S.sched[n++] = (uint16_t)((IT_R << 8) | l);
        S.sched[n++] = (uint16_t)((IT_TK << 8) | l);
      }
      S.sched[n++] = (uint16_t)((IT_GU << 8) | l);
      S.sched[n++] = (uint16_t)((IT_DN << 8) | l);
    }
  } else {
    constexpr int PF = 2;
    uint8_t ord[64];
    int no = 0;
    #pragma unroll 1
    for (int pass = 0; pass < 2; pass++)
      #pragma unroll 1
      for (int l = 0; l < P.L; l++)
        if (is_predicted(P, S, l) == (pass == 0)) ord[no++] = (uint8_t)l;
    #pragma unroll 1
    for (int j = 0; j < no; j++)
      if (!is_predicted(P, S, ord[j])) S.sched[n++] = (uint16_t)((IT_R << 8) | ord[j]);
    #pragma unroll 1
    for (int j = 0; j < PF && j < no; j++)
      if (!is_predicted(P, S, ord[j])) S.sched[n++] = (uint16_t)((IT_TK << 8) | ord[j]);
    #pragma unroll 1
    for (int j = 0; j < no + P.lag; j++) {
      if (j + PF < no && !is_predicted(P, S, ord[j + PF])) S.sched[n++] = (uint16_t)((IT_TK << 8) | ord[j + PF]);
      if (j < no) S.sched[n++] = (uint16_t)((IT_GU << 8) | ord[j]);
      if (j >= P.lag && j - P.lag < no) S.sched[n++] = (uint16_t)((IT_DN << 8) | ord[j - P.lag]);
    }
  }
  S.nsched = n;
}

// ---------------------------------------------------------------------------------------
// Producer (warp 0): walk this CTA's task list and stream it through the ring.  Lane 0
// builds each task's segment list in shared memory and owns the ring bookkeeping; all 32
// lanes issue the bulk copies.
// ---------------------------------------------------------------------------------------
template <int D, int I>
__device__ void producer(const DecodeParams &P, DecSmem<D, I> &S) {
  const int c = blockIdx.x, lane = threadIdx.x & 31;
  int q = 0, head = 0, oldest = 0;
  int qs[kNSlot];
  int sel[kMaxK];
  bool ok = true;

  #pragma unroll 1
  for (int it = 0; it < S.nsched && ok; it++) {
    const int item = S.sched[it] >> 8, l = S.sched[it] & 255;
    if (item == IT_TK) continue;
    const bool pred = is_predicted(P, S, l);
    const int kind = item == IT_R ? TK_ROUTER : item == IT_GU ? TK_GU : TK_DN;
    {
      if (kind != TK_ROUTER) {
        if (!pred) {
          // the consumers publish a reactive layer's own top-k (its TK item) first
          unsigned long long t0 = 0;
          while (S.sel_ok[l & 63] == 0) {
            if (S.abort) { ok = false; break; }
            if (timed_out(t0, P.timeout_ns)) {
              if (lane == 0) atomicOr(P.err, DERR_TIMEOUT);
              S.abort = 1;
              ok = false;
              break;
            }
            __nanosleep(32);
          }
          if (!ok) break;
        }
        #pragma unroll 1
        for (int j = 0; j < P.k; j++) {
          sel[j] = S.sel_all[l & 63][j];
          if (sel[j] < 0 || sel[j] >= P.E) {
            if (lane == 0 && kind == TK_GU) atomicOr(P.err, DERR_INDEX);
            sel[j] = 0;
          }
        }
      }
      if (kind == TK_GU) stamp(P, l, TR_P_GU_START);
      if (kind == TK_DN) stamp(P, l, TR_P_DN_START);
      if (lane == 0) build_task<D, I>(P, S.lay[l], kind, l, c, pred, sel, S.tb);   // out of line
      __syncwarp();
      const int n = S.tb.n;
      if (S.tb.overflow) {
        if (lane == 0) atomicOr(P.err, DERR_TIMEOUT);
        S.abort = 1;
        ok = false;
        break;
      }
      // each lane sizes its segments (rounded out to 16 bytes); warp prefix sum -> offsets
      int mine[3] = {0, 0, 0}, my_sum = 0;
#pragma unroll
      for (int m = 0; m < 3; m++) {
        const int i = lane * 3 + m;
        if (i < n) {
          const uintptr_t lo = (uintptr_t)S.tb.s[i].src & ~(uintptr_t)15;
          const uintptr_t hi = ((uintptr_t)S.tb.s[i].src + S.tb.s[i].bytes + 15) & ~(uintptr_t)15;
          mine[m] = (int)(hi - lo);
          my_sum += mine[m];
        }
      }
      int incl = my_sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int need = __shfl_sync(0xffffffffu, incl, 31);
      const int excl = incl - my_sum;
      if (need > kRingBytes) {
        if (lane == 0) atomicOr(P.err, DERR_TIMEOUT);
        S.abort = 1;
        ok = false;
        break;
      }
      // lane 0: allocate [start, start+need), releasing the oldest tasks as required.  The
      // in-flight bytes are [tail, head) or wrapped [tail, end) + [0, head); a gap of at
      // least one byte keeps head == tail meaning "empty".
      int start = -1;
      if (lane == 0) {
        while (ok) {
          if (q - oldest < kNSlot) {
            if (q == oldest) {
              head = 0;
              start = 0;
              break;
            }
            const int tail = qs[oldest % kNSlot];
            if (head > tail) {
              if (head + need <= kRingBytes) { start = head; break; }
              if (need < tail) { start = 0; break; }
            } else if (head < tail && head + need < tail) {
              start = head;
              break;
            }
          }
          // wait until the consumers have released task `oldest`
          const int slot = oldest % kNSlot;
          const uint32_t par = (uint32_t)((oldest / kNSlot) & 1);
          unsigned long long t0 = 0;
          while (!mbar_test(&S.empty[slot], par)) {
            if (S.abort) { ok = false; break; }
            if (timed_out(t0, P.timeout_ns)) {
              atomicOr(P.err, DERR_TIMEOUT);
              S.abort = 1;
              ok = false;
              break;
            }
          }
          if (ok) oldest++;
        }
      }
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      if (!ok) break;
      start = __shfl_sync(0xffffffffu, start, 0);
      const int slot = q % kNSlot;
      {
        int off = start + excl;
#pragma unroll
        for (int m = 0; m < 3; m++) {
          const int i = lane * 3 + m;
          if (i < n) {
            const uintptr_t lo = (uintptr_t)S.tb.s[i].src & ~(uintptr_t)15;
            S.seg_off[slot][i] = (uint32_t)(off + ((uintptr_t)S.tb.s[i].src - lo));
            S.tb_off[i] = off;
            off += mine[m];
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_expect_tx(&S.full[slot], (uint32_t)need);
      __syncwarp();
#pragma unroll
      for (int m = 0; m < 3; m++) {
        const int i = lane * 3 + m;
        if (i < n && mine[m] > 0) {
          const uintptr_t lo = (uintptr_t)S.tb.s[i].src & ~(uintptr_t)15;
          bulk_g2s(S.ring + S.tb_off[i], (const void *)lo, (uint32_t)mine[m], &S.full[slot]);
        }
      }
      __syncwarp();
      if (lane == 0) {
        qs[slot] = start;
        head = start + need;
      }
      q++;
      if (lane == 0) stamp(P, l, kind == TK_GU ? TR_P_GU : kind == TK_DN ? TR_P_DN : TR_P_R);
    }
  }
  // drain: every issued copy must have landed before the CTA exits
  if (lane == 0) {
    #pragma unroll 1
    for (int s = oldest; s < q; s++) {
      const int slot = s % kNSlot;
      const uint32_t par = (uint32_t)((s / kNSlot) & 1);
      unsigned long long t0 = 0;
      while (!mbar_test(&S.full[slot], par)) {
        if (timed_out(t0, P.timeout_ns)) {
          atomicOr(P.err, DERR_TIMEOUT);
          break;
        }
      }
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------------------
// Consumer helpers
// ---------------------------------------------------------------------------------------
struct Ctl {
  unsigned long long timeout;
  int *err;
  volatile int *abort;
};


// A source range of tagged words and where its 32-bit payloads go (shared memory).
struct Range {
  const unsigned long long *src;
  uint32_t *dst;
  int n;
};

// Poll the concatenation of up to four ranges (all consumer threads call it together):
// every thread issues its up-to-8 loads of a batch before checking any, so a batch costs
// one L2 round trip; a word whose tag is stale is re-polled on the slow path.  Out of line
// so that one copy of this code serves every call site.
__device__ __noinline__ bool poll_ranges(const Range *rg, int nr, uint32_t tag, int tid, const Ctl &C) {
  constexpr int W = 8;
  int total = 0;
#pragma unroll 1
  for (int q = 0; q < nr; q++) total += rg[q].n;
#pragma unroll 1
  for (int base = 0; base < total; base += W * kDecConsumers) {
    const unsigned long long *ad[W];
    uint32_t *dd[W];
    unsigned pending = 0;
#pragma unroll
    for (int m = 0; m < W; m++) {
      int i = base + tid + m * kDecConsumers;
      ad[m] = nullptr;
      dd[m] = nullptr;
      if (i < total) {
        int q = 0;
        while (i >= rg[q].n) i -= rg[q++].n;
        ad[m] = rg[q].src + i;
        dd[m] = rg[q].dst + i;
        pending |= 1u << m;
      }
    }
    // every still-stale word of the batch is re-read together, so each wave of arrivals
    // costs one L2 round trip
    unsigned long long t0 = 0;
    while (pending) {
      unsigned long long v[W];
#pragma unroll
      for (int m = 0; m < W; m++) v[m] = ((pending >> m) & 1u) ? ld_tag(ad[m]) : 0ull;
#pragma unroll
      for (int m = 0; m < W; m++)
        if (((pending >> m) & 1u) && (uint32_t)v[m] == tag) {
          *dd[m] = (uint32_t)(v[m] >> 32);
          pending &= ~(1u << m);
        }
      if (!pending) break;
      if (*C.abort) return false;
      if (timed_out(t0, C.timeout)) {
        atomicOr(C.err, DERR_TIMEOUT);
        *C.abort = 1;
        return false;
      }
      __nanosleep(20);
    }
  }
  return true;
}

// One-range convenience wrapper.
__device__ __forceinline__ bool poll_to(const unsigned long long *src, uint32_t *dst, int n, uint32_t tag, int tid,
                                        const Ctl &C) {
  const Range rg{src, dst, n};
  return poll_ranges(&rg, 1, tag, tid, C);
}

__device__ __forceinline__ bool wait_full(uint64_t *bar, uint32_t par, const Ctl &C) {
  unsigned long long t0 = 0;
  while (!mbar_test(bar, par)) {
    if (*C.abort) return false;
    if (timed_out(t0, C.timeout)) {
      atomicOr(C.err, DERR_TIMEOUT);
      *C.abort = 1;
      return false;
    }
  }
  return true;
}

// bf16 row (D elements in shared memory) dotted with x (fp32, shared memory): one warp.
template <int D>
__device__ __noinline__ float bf16_row_x(const uint16_t *w, const float *x, int lane) {
  float acc = 0.f;
#pragma unroll 2
  for (int ch = lane; ch < D / 8; ch += 32) {
    const uint4 v = *reinterpret_cast<const uint4 *>(w + ch * 8);
    const float4 a = *reinterpret_cast<const float4 *>(x + ch * 8);
    const float4 b = *reinterpret_cast<const float4 *>(x + ch * 8 + 4);
    acc = fmaf(bf(v.x & 0xFFFFu), a.x, acc);
    acc = fmaf(bf(v.x >> 16), a.y, acc);
    acc = fmaf(bf(v.y & 0xFFFFu), a.z, acc);
    acc = fmaf(bf(v.y >> 16), a.w, acc);
    acc = fmaf(bf(v.z & 0xFFFFu), b.x, acc);
    acc = fmaf(bf(v.z >> 16), b.y, acc);
    acc = fmaf(bf(v.w & 0xFFFFu), b.z, acc);
    acc = fmaf(bf(v.w >> 16), b.w, acc);
  }
  return warp_sum(acc);
}

__device__ __noinline__ void warp_topk_ool(const float *v, int E, int k, int lane, int *out) {
  warp_topk(v, E, k, lane, out);
}

// sum of the 32 raw values of a chunk whose registers hold them pre-scaled per nibble
// position (multiplying by 2^p undoes the scaling exactly)
__device__ __forceinline__ float chunk_raw_sum(const float (&xr)[32]) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    s0 = fmaf(xr[i], 1.0f / nib_scale(i & 7), s0);
    s1 = fmaf(xr[i + 1], 1.0f / nib_scale((i + 1) & 7), s1);
  }
  return s0 + s1;
}

// ---------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------
template <int D, int I>
__global__ void __launch_bounds__(kDecThreads, 1) k_decode(DecodeParams P) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecSmem<D, I> &S = *reinterpret_cast<DecSmem<D, I> *>(smem_raw);
  const int tid = threadIdx.x;
  // layer table and the predicted routing of every layer into shared memory
  #pragma unroll 1
  for (int i = tid; i < P.L * (int)(sizeof(DecLayer) / 8); i += kDecThreads)
    reinterpret_cast<unsigned long long *>(S.lay)[i] = reinterpret_cast<const unsigned long long *>(P.layers)[i];
  if (!P.step0)
    #pragma unroll 1
    for (int i = tid; i < P.L * P.k; i += kDecThreads)
      S.sel_all[(i / P.k) & 63][i % P.k] = P.pred_in[((size_t)(i / P.k) * P.maxT) * P.k + i % P.k];
  if (tid < 64) S.sel_ok[tid] = 0;
  __syncthreads();
  if (tid == 0) {
    #pragma unroll 1
    for (int s = 0; s < kNSlot; s++) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kDecCW);
    }
    S.abort = 0;
    build_schedule<D, I>(P, S);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (tid < 32) {
    producer<D, I>(P, S);
    return;
  }
  // ------------------------------- consumers -------------------------------------------
  constexpr int NCH = D / 32;                  // 16-byte code chunks per gate/up row
  constexpr int NCI = I / 32;                  // 16-byte code chunks per down row
  const int ct = tid - 32, warp = ct >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = P.G, k = P.k, r = P.r;
  Ctl C{P.timeout_ns, P.err, &S.abort};
  int q = 0;
  bool ab = false;

  if (c == P.stall_cta) {
    // test hook: wait for a word that is never written, so that the timeout path runs
    ab |= !poll_to(P.t_y, reinterpret_cast<uint32_t *>(S.yprev), 1, 0xFFFFFFFFu, ct, C);
  }

  #pragma unroll 1
  for (int it = 0; it < S.nsched; it++) {
    const int kind = S.sched[it] >> 8, l = S.sched[it] & 255;
    const DecLayer &Y = S.lay[l];
    const bool pred = is_predicted(P, S, l);
    const bool lora = Y.Bg != nullptr;
    const uint32_t tag = dtag(P, l);
    if (kind == IT_TK) {
      // ---- a reactive layer's top-k over every CTA's router logits
      ab |= !poll_to(P.t_rlog + (size_t)l * P.E, reinterpret_cast<uint32_t *>(S.rl), P.E, tag, ct, C);
      if (cbar_or(ab)) break;
      if (warp == 0) {
        int s8[kMaxK];
        warp_topk_ool(S.rl, P.E, k, lane, s8);
        if (lane == 0) {
          #pragma unroll 1
          for (int j = 0; j < k; j++) {
            S.sel_all[l & 63][j] = s8[j];
            S.rlsel[l & 63][j] = (s8[j] >= 0 && s8[j] < P.E) ? S.rl[s8[j]] : 0.f;
          }
          __threadfence_block();
          S.sel_ok[l & 63] = 1;
        }
      }
      cbar();
      if (ct == 0) stamp(P, l, TR_ROUTE);
      continue;
    }
    // ---- in order: a layer's first item waits for the previous layer's output (its data
    // in chained mode)
    if (P.lag == 0 && l > 0 && (kind == IT_R || (kind == IT_GU && pred))) {
      ab |= !poll_to(P.t_y + (size_t)(l - 1) * D, reinterpret_cast<uint32_t *>(S.yprev), D, dtag(P, l - 1), ct, C);
    }
    if (cbar_or(ab)) break;
    if (ct == 0 && kind != IT_DN) stamp(P, l, TR_LAYER);

    const int slot = q % kNSlot;
    const uint32_t par = (uint32_t)((q / kNSlot) & 1);
    ab |= !wait_full(&S.full[slot], par, C);
    if (cbar_or(ab)) break;
    if (kind != IT_DN) {
      // ---- the norm: gamma and h are the first two segments of router and gate/up tasks
      const uint16_t *gam = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][0]);
      const uint16_t *hin = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][1]);
      const bool chain = P.chained && l > 0;
      constexpr int PER = (D + kDecConsumers - 1) / kDecConsumers;
      double hv[PER];
      double ss = 0.0;
#pragma unroll
      for (int m = 0; m < PER; m++) {
        const int i = ct + m * kDecConsumers;
        double v = 0.0;
        if (i < D) {
          v = (double)bf(hin[i]);
          if (chain) v = (double)bf(d2bf_bits(v + (double)S.yprev[i]));
        }
        hv[m] = v;
        ss += v * v;
      }
      ss = warp_sum(ss);
      if (lane == 0) S.dred[warp] = ss;
      cbar();
      double tot = 0.0;
      #pragma unroll 1
      for (int w = 0; w < kDecCW; w++) tot += S.dred[w];
      const double rinv = 1.0 / sqrt(tot / D + (double)P.eps);
#pragma unroll
      for (int m = 0; m < PER; m++) {
        const int i = ct + m * kDecConsumers;
        if (i < D) {
          const float xv = bf(d2bf_bits(hv[m] * (double)bf(gam[i]) * rinv));
          S.x[i] = xv;
          S.xt[xt_index(i, NCH)] = xv * nib_scale(i & 7);
        }
      }
      cbar();
    }
    if (ct == 0 && kind != IT_DN) stamp(P, l, TR_NORM);
    if (kind == IT_R) {
      // ---- a reactive layer's router rows of this CTA
      int a, b;
      split_range(P.E, G, c, a, b);
      const uint16_t *rw = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][2]);
      #pragma unroll 1
      for (int row = a + warp; row < b; row += kDecCW) {
        const float v = bf16_row_x<D>(rw + (size_t)(row - a) * D, S.x, lane);
        if (lane == 0) st_tag(P.t_rlog + (size_t)l * P.E + row, tag, __float_as_uint(v));
      }
    } else if (kind == IT_GU) {
      // ---- gate/up stage ------------------------------------------------------------
      if (ct == 0) stamp(P, l, TR_GU_FULL);
      // LoRA A rows of the shared expert (t_g, t_u), published for the down phase
      int a = 0, b = 0;
      if (lora) split_range(2 * r, G, c, a, b);
      #pragma unroll 1
      for (int qq = a; qq < b; qq++) {
        if (warp == (qq - a) % kDecCW) {
          const uint16_t *row = qq < r ? reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][2]) + (size_t)(qq - a) * D
                                       : reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][3]) +
                                             (size_t)(qq - max(a, r)) * D;
          const float v = bf16_row_x<D>(row, S.x, lane);
          if (lane == 0) st_tag(P.t_blk + (size_t)l * P.blk + (k + 2) * I + qq, tag, __float_as_uint(v));
        }
      }
      // router logits of the predicted experts (their gate weights)
      a = b = 0;
      if (pred) split_range(k, G, (c + G - min(2 * r, G - 1)) % G, a, b);
      #pragma unroll 1
      for (int qq = a; qq < b; qq++) {
        if (warp == kDecCW - 1 - (qq - a) % kDecCW) {
          const float v = bf16_row_x<D>(reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][4 + qq - a]), S.x, lane);
          if (lane == 0) st_tag(P.t_blk + (size_t)l * P.blk + (k + 2) * I + 2 * r + qq, tag, __float_as_uint(v));
        }
      }
      // this CTA's rows of the layer's prerouter head on x
      if (Y.head) {
        int ha, hb;
        split_range(P.E, G, c, ha, hb);
        const uint16_t *hw = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][kGuHead]);
        #pragma unroll 1
        for (int row = ha; row < hb; row++) {
          if (warp == (4 + row - ha) % kDecCW) {
            const float v = bf16_row_x<D>(hw + (size_t)(row - ha) * P.ldh, S.x, lane);
            if (lane == 0) st_tag(P.t_hlog + (size_t)l * P.E + row, tag, __float_as_uint(v));
          }
        }
      }
      // this lane's activation chunks stay in registers for every row of the phase
      constexpr int LPR = NCH < 32 ? NCH : 32;    // lanes per row
      constexpr int RPW = 32 / LPR;               // rows per warp pass
      constexpr int CPL = NCH / LPR;              // chunks per lane
      const int sub = lane / LPR, sl = lane % LPR;
      float xr[CPL][32];
      float xsr[CPL];
#pragma unroll
      for (int cc = 0; cc < CPL; cc++) {
        load_chunk(S.xt, NCH, sl + cc * LPR, xr[cc]);
        xsr[cc] = chunk_raw_sum(xr[cc]);
      }
      GuPiece pc[kMaxPieces];
      const int np = gu_pieces<D, I>(k, G, c, pc);
      float *gu_g = S.ydot;            // raw g and u of every row of this CTA's pieces
      int roff = 0;
      #pragma unroll 1
      for (int p = 0; p < np; p++) {
        const int R = pc[p].i1 - pc[p].i0, sg = kGuPiece0 + 6 * p;
        const uint8_t *gc = S.ring + S.seg_off[slot][sg + 0];
        const uint16_t *gs = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 1]);
        const uint16_t *gm = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 2]);
        const uint8_t *uc = S.ring + S.seg_off[slot][sg + 3];
        const uint16_t *us = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 4]);
        const uint16_t *um = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 5]);
        #pragma unroll 1
        for (int base = warp * RPW; base < 2 * R; base += kDecCW * RPW) {
          const int item = base + sub;
          const bool valid = item < 2 * R;
          float acc = 0.f;
          if (valid) {
            const int row = item >> 1, up = item & 1;
            const uint8_t *cw = (up ? uc : gc) + (size_t)row * (D / 2);
            const uint16_t *sc = (up ? us : gs) + (size_t)row * (D / 64);
            const uint16_t *mn = (up ? um : gm) + (size_t)row * (D / 64);
#pragma unroll
            for (int cc = 0; cc < CPL; cc++) {
              const int ch = sl + cc * LPR;
              const uint4 w = *reinterpret_cast<const uint4 *>(cw + ch * 16);
              const float qd = chunk_qdot(w, xr[cc]);
              acc = fmaf(bf(sc[ch >> 1]), qd, fmaf(bf(mn[ch >> 1]), xsr[cc], acc));
            }
          }
          acc = group_sum(acc, LPR);
          if (valid && sl == 0) gu_g[2 * roff + item] = acc;
        }
        roff += R;
      }
      cbar();
      if (ct == 0) stamp(P, l, TR_GU_ROWS);
      // publish: routed rows as a = bf16(silu(g) u); shared rows as raw (g, u)
      roff = 0;
      #pragma unroll 1
      for (int p = 0; p < np; p++) {
        const int R = pc[p].i1 - pc[p].i0;
        const bool shared = pc[p].slot == k;
        #pragma unroll 1
        for (int row = ct; row < R; row += kDecConsumers) {
          const float g = gu_g[2 * (roff + row)], u = gu_g[2 * (roff + row) + 1];
          const int i = pc[p].i0 + row;
          unsigned long long *blk = P.t_blk + (size_t)l * P.blk;
          if (shared) {
            st_tag(blk + k * I + 2 * i, tag, __float_as_uint(g));
            st_tag(blk + k * I + 2 * i + 1, tag, __float_as_uint(u));
          } else {
            st_tag(blk + pc[p].slot * I + i, tag, f2bf(g / (1.0f + expf(-g)) * u));
          }
        }
        roff += R;
      }
      // routing used by this layer (one CTA records it for the host)
      if (c == 0 && ct < k) P.hist_out[((size_t)l * P.maxT) * k + ct] = S.sel_all[l & 63][ct];
      if (ct == 0) stamp(P, l, TR_GU_DONE);
    } else {
      // ---- down + combine stage -----------------------------------------------------
      // one batched poll over the layer's block: a of the routed slots, the shared
      // expert's raw g/u, t_g/t_u (with LoRA) and the selected router logits (predicted)
      float *at = S.at, *gus = S.gus;
      {
        const unsigned long long *blk = P.t_blk + (size_t)l * P.blk;
        Range rg[4];
        int nr = 0;
        rg[nr++] = Range{blk, S.stg, k * I};
        rg[nr++] = Range{blk + k * I, reinterpret_cast<uint32_t *>(S.gus), 2 * I};
        if (lora) rg[nr++] = Range{blk + (k + 2) * I, reinterpret_cast<uint32_t *>(S.tl), 2 * r};
        if (pred) rg[nr++] = Range{blk + (k + 2) * I + 2 * r, reinterpret_cast<uint32_t *>(S.rl), k};
        ab |= !poll_ranges(rg, nr, tag, ct, C);
      }
      if (cbar_or(ab)) break;
      // routed a values: bf16 payloads -> pre-scaled, chunk-transposed fp32
#pragma unroll 1
      for (int i = ct; i < k * I; i += kDecConsumers) {
        const int j = i / I, e = i - j * I;
        at[j * I + xt_index(e, NCI)] = bf(S.stg[i] & 0xFFFFu) * nib_scale(e & 7);
      }
      if (ct == 0) stamp(P, l, TR_A_POLL);
      if (ct == 0) stamp(P, l, TR_DN_FULL);
      const int sbd = dn_bd(k);
      const uint16_t *bgm = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sbd + 1]);
      const uint16_t *bum = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sbd + 2]);
      const uint16_t *adm = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sbd + 3]);
      // the shared expert's activation with its LoRA up branch (every CTA, same order)
      #pragma unroll 1
      for (int i = ct; i < I; i += kDecConsumers) {
        float g = gus[2 * i], u = gus[2 * i + 1];
        if (lora) {
          float lg = 0.f, lu = 0.f;
          #pragma unroll 1
          for (int j = 0; j < r; j += 8) {
            const uint4 wg = *reinterpret_cast<const uint4 *>(bgm + i * r + j);
            const uint4 wu = *reinterpret_cast<const uint4 *>(bum + i * r + j);
            const uint32_t gw[4] = {wg.x, wg.y, wg.z, wg.w}, uw[4] = {wu.x, wu.y, wu.z, wu.w};
#pragma unroll
            for (int q = 0; q < 4; q++) {
              lg = fmaf(bf(gw[q] & 0xFFFFu), S.tl[j + 2 * q], lg);
              lg = fmaf(bf(gw[q] >> 16), S.tl[j + 2 * q + 1], lg);
              lu = fmaf(bf(uw[q] & 0xFFFFu), S.tl[r + j + 2 * q], lu);
              lu = fmaf(bf(uw[q] >> 16), S.tl[r + j + 2 * q + 1], lu);
            }
          }
          g = fmaf(P.c, lg, g);
          u = fmaf(P.c, lu, u);
        }
        const float av = bf(f2bf(g / (1.0f + expf(-g)) * u));
        S.asraw[i] = av;
        at[k * I + xt_index(i, NCI)] = av * nib_scale(i & 7);
      }
      if (ct == 0) {
        float lg[kMaxK], mx = -INFINITY, sum = 0.f;
        #pragma unroll 1
        for (int j = 0; j < k; j++) {
          lg[j] = pred ? S.rl[j] : S.rlsel[l & 63][j];
          mx = fmaxf(mx, lg[j]);
        }
        #pragma unroll 1
        for (int j = 0; j < k; j++) {
          lg[j] = expf(lg[j] - mx);
          sum += lg[j];
        }
        #pragma unroll 1
        for (int j = 0; j < k; j++) S.gates[j] = lg[j] / sum;
      }
      cbar();
      // t_d = Ad a_s (LoRA down branch)
      if (lora) {
        #pragma unroll 1
        for (int j = warp; j < r; j += kDecCW) {
          float acc = 0.f;
          #pragma unroll 1
          for (int i = lane; i < I; i += 32) acc = fmaf(bf(adm[j * I + i]), S.asraw[i], acc);
          acc = warp_sum(acc);
          if (lane == 0) S.td[j] = acc;
        }
        cbar();
      }
      if (ct == 0) stamp(P, l, TR_TD_POLL);
      int a, b;
      split_range(D, G, c, a, b);
      const int R = b - a;
      constexpr int LPR = NCI < 32 ? NCI : 32;
      constexpr int RPW = 32 / LPR;
      constexpr int CPL = NCI / LPR;
      const int sub = lane / LPR, sl = lane % LPR;
      float *yd = S.ydot;
      #pragma unroll 1
      for (int j = 0; j <= k; j++) {
        // expert j's activation chunks in registers, then its rows
        float ar[CPL][32];
        float asr[CPL];
#pragma unroll
        for (int cc = 0; cc < CPL; cc++) {
          load_chunk(S.at + j * I, NCI, sl + cc * LPR, ar[cc]);
          asr[cc] = chunk_raw_sum(ar[cc]);
        }
        const uint8_t *cb = S.ring + S.seg_off[slot][3 * j];
        const uint16_t *sb = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][3 * j + 1]);
        const uint16_t *mb = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][3 * j + 2]);
        #pragma unroll 1
        for (int base = warp * RPW; base < R; base += kDecCW * RPW) {
          const int row = base + sub;
          const bool valid = row < R;
          float acc = 0.f;
          if (valid) {
            const uint8_t *cw = cb + (size_t)row * (I / 2);
            const uint16_t *sc = sb + (size_t)row * (I / 64);
            const uint16_t *mn = mb + (size_t)row * (I / 64);
#pragma unroll
            for (int cc = 0; cc < CPL; cc++) {
              const int ch = sl + cc * LPR;
              const uint4 w = *reinterpret_cast<const uint4 *>(cw + ch * 16);
              const float qd = chunk_qdot(w, ar[cc]);
              acc = fmaf(bf(sc[ch >> 1]), qd, fmaf(bf(mn[ch >> 1]), asr[cc], acc));
            }
          }
          acc = group_sum(acc, LPR);
          if (valid && sl == 0) yd[row * (k + 1) + j] = acc;
        }
      }
      if (ct == 0) stamp(P, l, TR_DN_DOTS);
      cbar();
      const uint16_t *bd = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sbd]);
      #pragma unroll 1
      for (int row = ct; row < R; row += kDecConsumers) {
        float y = 0.f;
        #pragma unroll 1
        for (int j = 0; j < k; j++) y = fmaf(S.gates[j], yd[row * (k + 1) + j], y);
        y += yd[row * (k + 1) + k];
        if (lora) {
          float lo = 0.f;
          #pragma unroll 1
          for (int j = 0; j < r; j++) lo = fmaf(bf(bd[row * r + j]), S.td[j], lo);
          y = fmaf(P.c, lo, y);
        }
        const int n = a + row;
        st_tag(P.t_y + (size_t)l * D + n, tag, __float_as_uint(y));
        P.y[(size_t)l * D + n] = f2bf(y);
        if (P.yf) P.yf[(size_t)l * D + n] = y;
      }
      if (ct == 0) stamp(P, l, TR_DN_DONE);
    }
    // release the item's ring space
    cbar();
    if (lane == 0) mbar_arrive(&S.empty[slot]);
    q++;
  }
  if (ab) return;
  // ---- head top-k: CTA c handles layer c's head; its logits are complete by now ------
  #pragma unroll 1
  for (int l = c; l < P.L; l += G) {
    const DecLayer &Y = S.lay[l];
    if (!Y.head) continue;
    const uint32_t tag = dtag(P, l);
    bool bad = !poll_to(P.t_hlog + (size_t)l * P.E, reinterpret_cast<uint32_t *>(S.rl), P.E, tag, ct, C);
    if (cbar_or(bad)) return;
    if (P.onehot) {
      // one-hot columns of this layer's routing now and at the previous token
      #pragma unroll 1
      for (int e = ct; e < P.E; e += kDecConsumers) {
        const uint16_t *wr = Y.head + (size_t)e * P.ldh + D;
        float v = S.rl[e];
        #pragma unroll 1
        for (int j = 0; j < k; j++) {
          const int s = S.sel_all[l & 63][j];
          if (s >= 0 && s < P.E) v += bf(wr[s]);
          if (P.hist_prev) {
            const int pv = P.hist_prev[((size_t)l * P.maxT) * k + j];
            if (pv >= 0 && pv < P.E) v += bf(wr[P.E + pv]);
          }
        }
        S.rl[e] = v;
      }
      cbar();
    }
    if (warp == 0) {
      int s8[kMaxK];
      warp_topk_ool(S.rl, P.E, k, lane, s8);
      if (lane < k) {
        int mine = 0;
        #pragma unroll 1
        for (int j = 0; j < k; j++)
          if (j == lane) mine = s8[j];
        P.pred_out[((size_t)(l + 1) * P.maxT) * k + lane] = mine;
      }
    }
    cbar();
  }
}

}  // namespace e0
