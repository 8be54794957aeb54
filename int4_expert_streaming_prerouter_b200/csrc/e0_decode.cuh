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
//   * Consumers (11 warps) compute the int4 dot products on the tensor cores as row pairs
//     that share one activation vector (mma.sync m16n8k16 fp16 with the codes masked in
//     place as fp16 subnormals and the group scale/min folded per group of 64), the SwiGLU, the LoRA branch
//     and the weighted combine.
//   * CTAs exchange results (a, y, LoRA intermediates, logits) through global memory as
//     64-bit words {32-bit tag, payload} written with one relaxed store; a reader polls the
//     data itself until every tag matches, so there is no separate barrier round trip.
//     Tags are unique per (launch, layer).  Every wait is bounded by a %globaltimer budget;
//     on expiry the kernel latches DERR_TIMEOUT, drains its copies and returns.
//   * The work is a host-built list of items per CTA: in layer order for chained inputs,
//     otherwise (flat) each phase's units over all layers cut into contiguous,
//     cost-balanced shares (router rows, x rows, gate/up units, down rows).
#pragma once
#include <algorithm>
#include <vector>
#include "e0_device.cuh"
#include "e0_kernels.cuh"

namespace e0 {

constexpr int kDecCW = 11;                // consumer warps (three warps per SM sub-partition with the producer: 168 registers each)
constexpr int kDecConsumers = 32 * kDecCW;
constexpr int kDecThreads = 32 + kDecConsumers;   // + 1 producer warp
constexpr int kRingBytes = 174 * 1024;
constexpr int kDecMaxK = 4;               // routed experts per token on this path
constexpr int kNSlot = 8;                 // tasks in flight

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
  // 0: layers in order (each layer's first x item waits for the previous layer's output);
  // 1 (unchained inputs only): the flat schedule, every phase's work over all layers
  // cut into cost-balanced contiguous shares across the CTAs
  int flat;
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
  const unsigned long long *sched;  // [G][kMaxItems] item lists (pack_item), built on the host
  const int *sched_n;               // [G] items per CTA
};

// Error bit of this kernel alone (beside the DERR_ bits): an activation outside the range of
// the fp16 tensor-core operand; the step's outputs are then not valid.
constexpr int kDerrRange = 16;

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
// Balanced contiguous split of N items over G parts (N * G < 2^31 here).
__host__ __device__ __forceinline__ void split_range(int N, int G, int c, int &a, int &b) {
  a = (int)((unsigned)(N * c) / (unsigned)G);
  b = (int)((unsigned)(N * (c + 1)) / (unsigned)G);
}


// ---------------------------------------------------------------------------------------
// Tensor-core dot products of int4 rows with one activation vector (gate/up and down).
//
// A warp takes two rows r0, r1 that share the activation vector v and walks their K in
// steps of 512 (eight groups of 64).  In a step, lane (g, t) (g = lane / 4, t = lane % 4)
// holds code words 8 g + 2 t and 8 g + 2 t + 1 of the step of both rows (16 codes of
// group g each).  Word nibbles n0..n7 (elements 8 w .. 8 w + 7) become the fp16 pairs
// {n_j, n_(j+4)}, j = 0..3, masked in place (subnormals q 2^-24 for even j, q 2^-20 for
// odd j; one shift per word brings j = 2, 3 down), exact.  In the m16n8k16 MMA, row g is
// r0 restricted to group g, row g + 8 is r1 restricted to group g, and column g is v
// restricted to group g, paired in the same element order, with v's odd elements held
// as v / 16, so the diagonal entries D[g][g] and D[g + 8][g] are P = 2^-24 sum q v over
// group g of r0 and of r1 (the other entries are not used).  Four MMAs cover a step.  The
// lane that holds the diagonal (t = g / 2) folds the group's affine weights w = s q + m
// into its partial sum as s 2^24 P + m V, V = sum v over the group; a warp sum finishes
// each row.  (The gate/up loop rotates the column groups from step to step so that the
// diagonals, and with them the folds, spread over all four lanes of a group row.)
//
// v lives in shared memory as fp16 pairs in the same order: word w of v is the uint4
// {v0|v4, v1|v5, v2|v6, v3|v7} of elements 8 w .. 8 w + 7 (low half first), odd elements
// divided by 16 (act_f16).
// ---------------------------------------------------------------------------------------
__host__ __device__ __forceinline__ int pair_index(int e) {   // uint16 index of element e
  return (e >> 3) * 8 + (e & 3) * 2 + ((e >> 2) & 1);
}
// uint16 index of element e of an N-element activation vector in the decode kernel's
// tables: elements in pair_index order within each 8-element word, and within each
// 512-element step of n words (64, or what is left) word w stored at (w & 1) n / 2 + (w >> 1),
// so that the two B-fragment words of a row-pair step (w = 8 g + 2 t and 8 g + 2 t + 1) are
// two lane-ordered 16-byte loads without bank conflicts
__device__ __forceinline__ int pair_slot(int e, int N) {
  const int w = e >> 3, s = w >> 6, wl = w & 63;
  const int n = min(64, N / 8 - 64 * s);
  return ((64 * s + (wl & 1) * (n >> 1) + (wl >> 1)) << 3) + (e & 3) * 2 + ((e >> 2) & 1);
}
// Code word w (elements 8 w .. 8 w + 7, element 8 w + j in bits 4 j .. 4 j + 3) -> the four
// fp16 operand pairs {j, j + 4}, masked in place: a nibble pair at bits 0-3 / 16-19 reads as
// the fp16 subnormals q 2^-24, one at bits 4-7 / 20-23 as q 2^-20, both exact.  Five integer
// instructions per word, no offset to remove afterwards.
__device__ __forceinline__ void nib_f16(uint32_t w, uint32_t &e0, uint32_t &e1, uint32_t &e2, uint32_t &e3) {
  const uint32_t h = w >> 8;
  e0 = w & 0x000F000Fu;   // elements 0, 4: q 2^-24
  e1 = w & 0x00F000F0u;   // elements 1, 5: q 2^-20
  e2 = h & 0x000F000Fu;   // elements 2, 6: q 2^-24
  e3 = h & 0x00F000F0u;   // elements 3, 7: q 2^-20
}
// bf16 form (the phased kernels): word nibbles j, j + 4 -> the exact bf16 pair {128 + q_j, 128 + q_(j+4)}
__device__ __forceinline__ uint32_t nib_pair_bf16(uint32_t w, int j) {
  return ((w >> (4 * j)) & 0x000F000Fu) | 0x43004300u;
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// The fp16 operand of activation element e (v a bf16 value): v for even e, v / 16 for odd e,
// so that with the codes above every product is q v 2^-24.  Exact for 2^-13 <= |v| < 65520
// (even e) or 16 * 65520 (odd e); below 2^-13 fp16 keeps v to 2^-20 absolute.  `bad` is set
// when a finite v overflows.
__device__ __forceinline__ uint16_t act_f16(float v, int e, bool &bad) {
  const uint16_t b = __half_as_ushort(__float2half_rn((e & 1) ? v * 0.0625f : v));
  bad |= (b & 0x7FFFu) == 0x7C00u && fabsf(v) <= 3.0e38f;
  return b;
}
// one 512-wide step: c0, c1 the two code words of rows r0, r1; va, vb the activation
// words 8 g + 2 t and 8 g + 2 t + 1 of the step (fp16 operands as act_f16 forms them);
// the diagonal entries come out as 2^-24 sum q v over the lane's group
__device__ __forceinline__ void pair_step(float (&d)[4], uint2 c0, uint2 c1, uint4 va, uint4 vb) {
  d[0] = d[1] = d[2] = d[3] = 0.f;
  uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
  nib_f16(c0.x, a0, a1, a2, a3);
  nib_f16(c1.x, b0, b1, b2, b3);
  mma_f16_16816(d, a0, b0, a1, b1, va.x, va.y);
  mma_f16_16816(d, a2, b2, a3, b3, va.z, va.w);
  nib_f16(c0.y, a0, a1, a2, a3);
  nib_f16(c1.y, b0, b1, b2, b3);
  mma_f16_16816(d, a0, b0, a1, b1, vb.x, vb.y);
  mma_f16_16816(d, a2, b2, a3, b3, vb.z, vb.w);
}
// Sums over the warp of four per-lane values at once (a transposing butterfly, six
// shuffles): lanes 0-7 return the sum of v0, lanes 8-15 of v1, 16-23 of v2, 24-31 of v3.
__device__ __forceinline__ float warp_sum4(float v0, float v1, float v2, float v3, int lane) {
  const bool hi = lane & 16;
  float a = hi ? v2 : v0, b = hi ? v3 : v1;
  a += __shfl_xor_sync(0xffffffffu, hi ? v0 : v2, 16);
  b += __shfl_xor_sync(0xffffffffu, hi ? v1 : v3, 16);
  const bool b8 = lane & 8;
  float c = b8 ? b : a;
  c += __shfl_xor_sync(0xffffffffu, b8 ? a : b, 8);
  c += __shfl_xor_sync(0xffffffffu, c, 4);
  c += __shfl_xor_sync(0xffffffffu, c, 2);
  c += __shfl_xor_sync(0xffffffffu, c, 1);
  return c;
}
// the diagonal lane's affine fold of group G of one row: s 2^24 P + m V (P = 2^-24 sum q v)
__device__ __forceinline__ float group_fold(float P, const uint16_t *sc, const uint16_t *mn, int G, float V) {
  return fmaf(bf(sc[G]) * 16777216.f, P, bf(mn[G]) * V);
}
__device__ __forceinline__ uint2 ld_code2(const uint8_t *p) { return *reinterpret_cast<const uint2 *>(p); }

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
// Work items.  A launch runs a list of items, the same sequence for the producer (which
// streams each item's bytes into the ring) and the consumers (which compute it).  An item
// is one kind of work on a contiguous range [a, a + n) of one layer's units:
//   IT_R   router rows of a reactive layer                         (units: the E experts)
//   IT_TK  top-k of a reactive layer over all its router logits   (consumers only)
//   IT_XR  the other rows dotted with x: the layer's head rows (E, if it has a head),
//          then the shared expert's A_g rows and A_u rows (r each, with LoRA), then the
//          router rows of the predicted experts (k, predicted layers)
//   IT_GU  expert gate/up: unit u = slot u / I (k routed, then the shared expert) and
//          intermediate index u % I, i.e. one gate row and one up row
//   IT_DN  output rows of the down projection and the weighted combine
// The flag bit: on R, XR and GU items, compute the layer's RMSNorm first (the
// previous x item had another layer); on DN items, this is the CTA's first down item of
// the layer, which assembles the shared expert's a_s (with the LoRA up branch) and
// t_d = A_d a_s from the whole LoRA matrices that its task carries, kept for the layer's
// later down items.  The flags are decided when the list is built, so that producer and
// consumers agree on what each task holds.
// ---------------------------------------------------------------------------------------
enum : int { IT_R = 0, IT_TK = 1, IT_XR = 2, IT_GU = 3, IT_DN = 4 };
constexpr int kMaxItems = 320;

struct Item {
  int kind, l, a, n;
  bool first;
};
__host__ __device__ __forceinline__ unsigned long long pack_item(int kind, int l, int a, int n, bool first) {
  return (unsigned long long)kind | ((unsigned long long)first << 4) | ((unsigned long long)l << 8) |
         ((unsigned long long)a << 16) | ((unsigned long long)n << 40);
}
__host__ __device__ __forceinline__ Item unpack_item(unsigned long long v) {
  return Item{(int)(v & 15ull), (int)((v >> 8) & 255ull), (int)((v >> 16) & 0xFFFFFFull), (int)(v >> 40),
              ((v >> 4) & 1ull) != 0};
}

// A range of gate/up units touches consecutive slots ("pieces"): at most kMaxPieces.
constexpr int kMaxPieces = 4;
constexpr int kDnMaxRows = 64;   // down rows per item (register accumulators per warp)
static_assert(kMaxR <= 32, "the down items' LoRA terms take one lane each");

// [s0, s1) = the part of [a, a + n) inside [lo, hi), relative to lo (empty: s0 = s1 = 0)
__device__ __forceinline__ void sub_range(int a, int n, int lo, int hi, int &s0, int &s1) {
  s0 = max(a, lo) - lo;
  s1 = min(a + n, hi) - lo;
  if (s1 <= s0) s0 = s1 = 0;
}

// Segment indices of each task (a segment may be empty):
//   R:  [0] gamma, [1] h (when the item computes the norm), [2] router rows
//   XR: [0] gamma, [1] h, [2] head rows, [3] A_g rows, [4] A_u rows, [5, 5 + kMaxK) the
//       selected router rows
//   GU: [0] gamma, [1] h, then per piece p (up to kMaxPieces) 6 segments from 2 + 6 p:
//       gate codes, gate scale, gate min, up codes, up scale, up min
//   DN: [3j .. 3j+2] down codes/scale/min of slot j (j = 0..k), then B_d rows, and on a
//       layer's first down item B_g, B_u, A_d (the shared expert's LoRA matrices, whole)
constexpr int kXrHead = 2, kXrAg = 3, kXrAu = 4, kXrSel = 5;
constexpr int kGuPiece0 = 2;
__device__ __forceinline__ int dn_bd(int k) { return 3 * (k + 1); }

// Segment i (one per producer lane) of item `it` on the rows of layer Y: its source and
// byte count (0 = empty).  `sel` are the layer's routed experts.  The consumer code reads
// the segments back by the indices above.
constexpr int kMaxItemSegs = 32;
template <int D, int I>
__device__ __forceinline__ void item_seg(const DecodeParams &P, const DecLayer &Y, const Item &it, bool predicted,
                                         const int (&sel)[kMaxK], int i, const uint8_t *&src, uint32_t &bytes) {
  const Blob bl = blob_of(D, I);
  const int l = it.l, a = it.a, n = it.n;
  src = nullptr;
  bytes = 0;
  auto pick = [&](const void *p, size_t b) {
    src = (const uint8_t *)p;
    bytes = (uint32_t)b;
  };
  if (it.kind != IT_DN && i < 2) {
    if (it.first) pick(i == 0 ? (const void *)Y.gamma : (const void *)(P.h + (size_t)l * D), D * 2);
    return;
  }
  if (it.kind == IT_R) {
    if (i == 2) pick(Y.router + (size_t)a * D, (size_t)n * D * 2);
  } else if (it.kind == IT_XR) {
    const int nh = Y.head ? P.E : 0, nl = Y.Ag ? P.r : 0, ns = predicted ? P.k : 0;
    int s0, s1;
    if (i == kXrHead) {
      sub_range(a, n, 0, nh, s0, s1);
      pick(Y.head + (size_t)s0 * P.ldh, (size_t)(s1 - s0) * P.ldh * 2);
    } else if (i == kXrAg) {
      sub_range(a, n, nh, nh + nl, s0, s1);
      pick(Y.Ag + (size_t)s0 * D, (size_t)(s1 - s0) * D * 2);
    } else if (i == kXrAu) {
      sub_range(a, n, nh + nl, nh + 2 * nl, s0, s1);
      pick(Y.Au + (size_t)s0 * D, (size_t)(s1 - s0) * D * 2);
    } else if (i < kXrSel + kMaxK) {
      sub_range(a, n, nh + 2 * nl, nh + 2 * nl + ns, s0, s1);
      const int q = i - kXrSel;
      if (s0 + q < s1) {
        int e = 0;
#pragma unroll
        for (int j = 0; j < kMaxK; j++)
          if (j == s0 + q) e = sel[j];
        pick(Y.router + (size_t)e * D, D * 2);
      }
    }
  } else if (it.kind == IT_GU) {
    // piece p = the p-th slot touched by units [a, a + n): slot a / I + p
    const int p = (i - kGuPiece0) / 6, f = (i - kGuPiece0) % 6;
    const int slot = a / I + p;
    const int i0 = p == 0 ? a % I : 0, i1 = min(a + n - slot * I, I);
    if (i >= kGuPiece0 && i1 > i0) {
      int e = 0;
#pragma unroll
      for (int j = 0; j < kMaxK; j++)
        if (j == slot) e = sel[j];
      const uint8_t *base = slot < P.k ? Y.experts + (size_t)e * bl.bytes : Y.shared;
      const bool codes = f == 0 || f == 3;
      const size_t off = f == 0 ? bl.gc : f == 1 ? bl.gs : f == 2 ? bl.gm : f == 3 ? bl.uc : f == 4 ? bl.us : bl.um;
      const size_t rb = codes ? D / 2 : (D / 64) * 2;
      pick(base + off + (size_t)i0 * rb, (size_t)(i1 - i0) * rb);
    }
  } else if (it.kind == IT_DN) {
    const int nd = 3 * (P.k + 1);
    if (i < nd) {
      const int j = i / 3, f = i % 3;
      int e = 0;
#pragma unroll
      for (int q = 0; q < kMaxK; q++)
        if (q == j) e = sel[q];
      const uint8_t *base = j < P.k ? Y.experts + (size_t)e * bl.bytes : Y.shared;
      const size_t off = f == 0 ? bl.dc : f == 1 ? bl.ds : bl.dm;
      const size_t rb = f == 0 ? I / 2 : (I / 64) * 2;
      pick(base + off + (size_t)a * rb, (size_t)n * rb);
    } else if (i == nd) {
      if (Y.Bd) pick(Y.Bd + (size_t)a * P.r, (size_t)n * P.r * 2);
    } else if (i <= nd + 3) {
      if (Y.Bg && it.first)
        pick(i == nd + 1 ? (const void *)Y.Bg : i == nd + 2 ? (const void *)Y.Bu : (const void *)Y.Ad,
             (size_t)I * P.r * 2);
    }
  }
}

// ---------------------------------------------------------------------------------------
// Shared-memory layout
// ---------------------------------------------------------------------------------------
template <int D, int I>
struct DecSmem {
  uint8_t ring[kRingBytes];
  alignas(16) uint16_t xn[D];        // x as bf16, natural order (for the bf16 rows)
  union {                            // used by different items, never at the same time:
    float yprev[D];                  //   the previous layer's y (fp32), in order + chained
    uint32_t stg[kDecMaxK * I];      //   routed a payloads as polled (a layer's first down item)
  };
  alignas(16) uint16_t ap[(kDecMaxK + 1) * I];   // a of every slot, bf16 pairs (pair_slot order)
  alignas(16) uint16_t xp[D];        // x as bf16 pairs (pair_slot order)
  float asraw[I];                    // the shared expert's a (natural order, for t_d)
  float xg[D / 64];                  // sum of x over each group of 64
  float ag[(kDecMaxK + 1) * (I / 64)];     // sum of each slot's a over each group of 64
  float gus[2 * I];                  // the shared expert's raw g and u (interleaved per row)
  double dred[16];
  float gates[kMaxK];
  float tl[2 * kMaxR];               // t_g, t_u
  float td[kMaxR];                   // t_d
  float rl[kMaxE];                   // router logits (reactive) / selected logits / head logits
  int sel_all[64][kMaxK];            // routing of every layer this step
  float rlsel[64][kMaxK];            // a reactive layer's router logits of its chosen experts
  volatile int sel_ok[64];           // 1 once a reactive layer's top-k is in sel_all
  unsigned long long items[kMaxItems];   // this CTA's item list (pack_item)
  int nitems;
  DecLayer lay[64];                  // the layer table
  int ring_start[kNSlot];            // the producer's ring offset of each slot's task
  uint32_t seg_off[kNSlot][kMaxItemSegs]; // ring byte offset of each segment's first wanted byte
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
// The item lists, one per CTA, built on the host.
//
// In order (chained inputs, or for comparison): per layer [R, TK] XR GU DN, each x item
// and the down item over this CTA's balanced share of the layer's units.
//
// Flat (unchained inputs: no layer reads another layer's output within the step, so the
// layers are independent apart from the predictions that cross to the next token): each
// phase's units over all layers form one list, cut into contiguous cost-balanced shares
// across the CTAs (balanced_cuts), so that a CTA streams long runs of rows of one or two
// layers instead of a sliver
// of every layer.  Phases: R (reactive layers' routers), XR, TK (the reactive layers this
// CTA needs), GU, DN.  Items are cut to at most about 58 KB of weight bytes (three fit the
// ring).  A CTA then computes a handful of norms per step, polls other CTAs' results a
// handful of times, and waits on other CTAs only where a phase needs the previous one
// (R -> TK, GU -> DN).
//
// A list depends only on the model's shape, on which layers carry a head or LoRA, on the
// schedule and on whether the step is a sequence's first (no predictions yet), so the host
// builds each combination once and a CTA copies its own list at launch.
// ---------------------------------------------------------------------------------------
struct SchedShape {
  int L, G, E, k, r, ldh, D, I;
  bool head[64], lora[64];
};

inline bool sched_predicted(const SchedShape &Z, bool step0, int l) {
  return !step0 && l > 0 && Z.head[l - 1];
}
inline int sched_xrows(const SchedShape &Z, bool step0, int l) {
  return (Z.head[l] ? Z.E : 0) + (Z.lora[l] ? 2 * Z.r : 0) + (sched_predicted(Z, step0, l) ? Z.k : 0);
}

// Cuts of one phase's unit list (the units of every layer, in layer order) into G
// contiguous shares of about equal cost: a share costs `per_unit` for each unit plus
// `per_seg` (and extra[l]) for each layer it touches (a norm, a top-k, the shared-expert
// inputs of a layer's first down item: work a CTA does once per layer it touches).  The
// smallest share bound that the greedy cut fits into G shares, found by bisection; share
// c also carries start[c], the cost of what its CTA does before this phase (nullptr: 0).
// cuts[0] = 0, cuts[G] = the phase's unit count.
inline void balanced_cuts(const int *units, const double *extra, int L, int G, double per_unit, double per_seg,
                          const double *start, long long *cuts) {
  long long tot = 0;
  for (int l = 0; l < L; l++) tot += units[l];
  // greedy: each share takes as many units as fit under the bound; true if G shares hold
  // every unit (when writing, the last share takes whatever is left)
  auto greedy = [&](double bound, bool write) {
    long long pos = 0;
    for (int c = 0; c < G; c++) {
      if (write) cuts[c] = pos;
      if (pos >= tot) continue;
      if (write && c == G - 1) { pos = tot; break; }
      double rem = bound - (start ? start[c] : 0.0);
      long long base = 0;
      int l = 0;
      while (l < L && base + units[l] <= pos) base += units[l++];
      while (l < L && pos < tot) {
        if (units[l] == 0) { l++; continue; }
        rem -= per_seg + (extra ? extra[l] : 0.0);
        if (rem < per_unit) break;
        const long long left = base + units[l] - pos;
        const long long take = std::min(left, (long long)(rem / per_unit));
        pos += take;
        rem -= take * per_unit;
        if (take < left) break;
        base += units[l++];
      }
    }
    if (write) cuts[G] = tot;
    return pos >= tot;
  };
  double lo = 0.0, hi = tot * per_unit + (L + 1) * per_seg + 1.0;
  if (extra)
    for (int l = 0; l < L; l++) hi += extra[l];
  if (start)
    for (int c = 0; c < G; c++) hi = std::max(hi, start[c] + tot * per_unit + (L + 1) * per_seg + 1.0);
  for (int it = 0; it < 60; it++) {
    const double mid = 0.5 * (lo + hi);
    if (greedy(mid, false)) hi = mid;
    else lo = mid;
  }
  greedy(hi, true);
}

// The cost of units [lo, hi) of a phase under the same model.
inline double share_cost(const int *units, const double *extra, int L, double per_unit, double per_seg, long long lo,
                         long long hi) {
  double cost = 0.0;
  long long base = 0;
  for (int l = 0; l < L; l++) {
    const long long s0 = std::max(lo, base), s1 = std::min(hi, base + units[l]);
    if (s1 > s0) cost += (s1 - s0) * per_unit + per_seg + (extra ? extra[l] : 0.0);
    base += units[l];
  }
  return cost;
}

// CTA c's items into out[0, kMaxItems); returns their count, or -1 if they do not fit.
inline int build_items(const SchedShape &Z, bool flat, bool step0, int c, unsigned long long *out) {
  const int G = Z.G, L = Z.L, k = Z.k, D = Z.D, I = Z.I;
  int n = 0;
  bool over = false;
  auto put = [&](int kind, int l, int a, int cnt) {
    if (n < kMaxItems) out[n++] = pack_item(kind, l, a, cnt, false);
    else over = true;
  };
  if (!flat) {
    for (int l = 0; l < L; l++) {
      int a, b;
      if (!sched_predicted(Z, step0, l)) {
        split_range(Z.E, G, c, a, b);
        if (b > a) put(IT_R, l, a, b - a);
        put(IT_TK, l, 0, 0);
      }
      split_range(sched_xrows(Z, step0, l), G, c, a, b);
      if (b > a) put(IT_XR, l, a, b - a);
      split_range((k + 1) * I, G, c, a, b);
      if (b > a) put(IT_GU, l, a, b - a);
      split_range(D, G, c, a, b);
      if (b > a) put(IT_DN, l, a, b - a);
    }
  } else {
    constexpr int kItemBytes = 58 * 1024;
    // gate/up items in whole consumer passes where the byte budget allows (a pass covers
    // two units per row group of each consumer warp); down items take the full budget,
    // since fewer, longer down items beat whole passes there
    const int gu_pass = 2 * kDecCW * (32 / (D / 32 < 32 ? D / 32 : 32));
    int gu_chunk = std::min(kItemBytes / (2 * (D / 2 + D / 16)), 288);
    const int dn_chunk = std::min(kItemBytes / ((k + 1) * (I / 2 + I / 16) + 2 * Z.r), kDnMaxRows);
    const int xr_chunk = std::max(kItemBytes / (2 * Z.ldh), 1);
    if (gu_chunk >= gu_pass) gu_chunk -= gu_chunk % gu_pass;
    auto units = [&](int which, int l) {
      return which == 0 ? (sched_predicted(Z, step0, l) ? 0 : Z.E)
           : which == 1 ? sched_xrows(Z, step0, l) : which == 2 ? (k + 1) * I : D;
    };
    // each phase: units(l) per layer over every layer with units, this CTA's share of a
    // cost-balanced cut.  Costs in microseconds on B200: a unit's bytes at the consumers'
    // rate, and the work done once per layer a share touches (the norm for x phases, the
    // top-k of a reactive layer before the gate/up phase, the down inputs of a layer).
    // The gate/up cut also balances what each CTA does before it (its router and x-row
    // shares), so that the CTAs finish the gate/up phase, which the down phase waits
    // for, together.
    struct PhaseCost { int kind, chunk, which; double per_unit, per_seg; bool tk; };
    const PhaseCost ph[4] = {{IT_R, 9, 0, 0.10, 2.0, false},
                             {IT_XR, xr_chunk, 1, 0.15, 2.2, false},
                             {IT_GU, gu_chunk, 2, 0.09, 2.6, true},
                             {IT_DN, dn_chunk, 3, 0.095, 10.0, false}};
    std::vector<double> before(G, 0.0);
    std::vector<long long> cuts(G + 1);
    int n_before_tk = 0;
    for (int f = 0; f < 4; f++) {
      int u_l[64];
      double e_l[64];
      for (int l = 0; l < L; l++) {
        u_l[l] = units(ph[f].which, l);
        e_l[l] = ph[f].tk && !sched_predicted(Z, step0, l) ? 2.7 : 0.0;
      }
      balanced_cuts(u_l, e_l, L, G, ph[f].per_unit, ph[f].per_seg, ph[f].kind == IT_GU ? before.data() : nullptr,
                    cuts.data());
      if (ph[f].kind == IT_R || ph[f].kind == IT_XR)
        for (int cc = 0; cc < G; cc++)
          before[cc] += share_cost(u_l, e_l, L, ph[f].per_unit, ph[f].per_seg, cuts[cc], cuts[cc + 1]);
      if (ph[f].kind == IT_GU) n_before_tk = n;
      const long long lo = cuts[c], hi = cuts[c + 1];
      long long base = 0;
      for (int l = 0; l < L; l++) {
        const int u = u_l[l];
        const long long s0 = std::max(lo, base), s1 = std::min(hi, base + u);
        for (long long a = s0; a < s1; a += ph[f].chunk)
          put(ph[f].kind, l, (int)(a - base), (int)std::min((long long)ph[f].chunk, s1 - a));
        base += u;
      }
    }
    // the top-k items go before the gate/up phase: the reactive layers that this CTA's
    // gate/up or down items touch
    bool need[64] = {};
    for (int q = n_before_tk; q < n; q++) {
      const Item it = unpack_item(out[q]);
      if (!sched_predicted(Z, step0, it.l)) need[it.l] = true;
    }
    int ntk = 0;
    for (int l = 0; l < L; l++) ntk += need[l];
    if (n + ntk > kMaxItems) return -1;
    for (int q = n - 1; q >= n_before_tk; q--) out[q + ntk] = out[q];
    int w = n_before_tk;
    for (int l = 0; l < L; l++)
      if (need[l]) out[w++] = pack_item(IT_TK, l, 0, 0, false);
    n += ntk;
  }
  if (over) return -1;
  // flags: x items compute the norm when the previous x item had another layer; the
  // first down item of each layer assembles the layer's shared-expert inputs
  int lastx = -1, lastd = -1;
  for (int q = 0; q < n; q++) {
    const Item it = unpack_item(out[q]);
    bool f = false;
    if (it.kind == IT_R || it.kind == IT_XR || it.kind == IT_GU) {
      f = it.l != lastx;
      lastx = it.l;
    } else if (it.kind == IT_DN) {
      f = it.l != lastd;
      lastd = it.l;
    }
    out[q] = pack_item(it.kind, it.l, it.a, it.n, f);
  }
  return n;
}

// ---------------------------------------------------------------------------------------
// Producer (warp 0): walk this CTA's task list and stream it through the ring.  Lane 0
// builds each task's segment list in shared memory and owns the ring bookkeeping; all 32
// lanes issue the bulk copies.
// ---------------------------------------------------------------------------------------
template <int D, int I>
__device__ void producer(const DecodeParams &P, DecSmem<D, I> &S) {
  const int lane = threadIdx.x & 31;
  int q = 0, head = 0, oldest = 0;
  int sel[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; j++) sel[j] = 0;
  bool ok = true;

  #pragma unroll 1
  for (int q_it = 0; q_it < S.nitems && ok; q_it++) {
    const Item it = unpack_item(S.items[q_it]);
    if (it.kind == IT_TK) continue;
    const int l = it.l;
    const bool pred = is_predicted(P, S, l);
    if (it.kind == IT_GU || it.kind == IT_DN || (it.kind == IT_XR && pred)) {
      if (!pred) {
        // a reactive layer's experts are known once the consumers ran its TK item
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
#pragma unroll
      for (int j = 0; j < kMaxK; j++) {
        int e = j < P.k ? S.sel_all[l & 63][j] : 0;
        if (e < 0 || e >= P.E) {
          if (lane == 0 && it.kind == IT_GU) atomicOr(P.err, DERR_INDEX);
          e = 0;
        }
        sel[j] = e;
      }
    }
    if (it.kind == IT_GU) stamp(P, l, TR_P_GU_START);
    if (it.kind == IT_DN) stamp(P, l, TR_P_DN_START);
    // each lane builds its own segment (rounded out to 16 bytes); warp prefix sum -> offsets
    const uint8_t *src;
    uint32_t bytes;
    item_seg<D, I>(P, S.lay[l], it, pred, sel, lane, src, bytes);
    const uintptr_t lo = (uintptr_t)src & ~(uintptr_t)15;
    const int mine = bytes ? (int)((((uintptr_t)src + bytes + 15) & ~(uintptr_t)15) - lo) : 0;
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int need = __shfl_sync(0xffffffffu, incl, 31);
    const int excl = incl - mine;
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
          const int tail = S.ring_start[oldest % kNSlot];
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
    const int off = start + excl;
    S.seg_off[slot][lane] = (uint32_t)(off + ((uintptr_t)src - lo));
    __syncwarp();
    if (lane == 0) mbar_expect_tx(&S.full[slot], (uint32_t)need);
    __syncwarp();
    if (mine > 0) bulk_g2s(S.ring + off, (const void *)lo, (uint32_t)mine, &S.full[slot]);
    __syncwarp();
    if (lane == 0) {
      S.ring_start[slot] = start;
      head = start + need;
    }
    q++;
    if (lane == 0) stamp(P, l, it.kind == IT_GU ? TR_P_GU : it.kind == IT_DN ? TR_P_DN : TR_P_R);
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
  constexpr int W = 10;   // a layer's down inputs (about 3,100 words at d = 2048) in one batch
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

// Two bf16 rows r0, r1 (D elements each, in shared memory) dotted with x (bf16, natural
// order), on the tensor cores: one warp.  Per MMA, lane (g, t) holds elements
// 128 s + 16 g + 4 t .. + 3 of both rows and of x, so that MMA row g (g + 8) is row r0 (r1)
// restricted to chunk g of the 128 and column g is x restricted to it; the diagonal
// entries accumulate each row's chunk sums over the steps, and the lanes that hold them
// (t = g / 2) are summed at the end.  No scale folds: the rows are plain bf16.
template <int D>
__device__ __noinline__ float2 bf16_pair_x(const uint16_t *r0, const uint16_t *r1, const uint16_t *xn, int lane) {
  const int g8 = lane >> 2, t4 = lane & 3;
  float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int s = 0; s < D / 128; s++) {
    const int k0 = 128 * s + 16 * g8 + 4 * t4;
    const uint2 a = *reinterpret_cast<const uint2 *>(r0 + k0);
    const uint2 b = *reinterpret_cast<const uint2 *>(r1 + k0);
    const uint2 x = *reinterpret_cast<const uint2 *>(xn + k0);
    mma_bf16_16816(d, a.x, b.x, a.y, b.y, x.x, x.y);
  }
  const bool own = t4 == (g8 >> 1);
  return make_float2(warp_sum(own ? ((g8 & 1) ? d[1] : d[0]) : 0.f), warp_sum(own ? ((g8 & 1) ? d[3] : d[2]) : 0.f));
}

__device__ __noinline__ void warp_topk_ool(const float *v, int E, int k, int lane, int *out) {
  warp_topk(v, E, k, lane, out);
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
    S.nitems = min(max(P.sched_n[blockIdx.x], 0), kMaxItems);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  #pragma unroll 1
  for (int i = tid; i < min(max(P.sched_n[blockIdx.x], 0), kMaxItems); i += kDecThreads)
    S.items[i] = P.sched[(size_t)blockIdx.x * kMaxItems + i];
  __syncthreads();
  if (tid < 32) {
    producer<D, I>(P, S);
    return;
  }
  // ------------------------------- consumers -------------------------------------------
  const int ct = tid - 32, warp = ct >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = P.G, k = P.k, r = P.r;
  Ctl C{P.timeout_ns, P.err, &S.abort};
  int q = 0;
  bool ab = false;
  bool range_bad = false;   // an activation outside the fp16 operand range (act_f16)

  if (c == P.stall_cta) {
    // test hook: wait for a word that is never written, so that the timeout path runs
    ab |= !poll_to(P.t_y, reinterpret_cast<uint32_t *>(S.yprev), 1, 0xFFFFFFFFu, ct, C);
  }

  // Items run without a consumer-wide barrier: every warp waits for the item's bytes on
  // its mbarrier, processes its own rows, publishes them and releases its claim on the
  // ring slot; warps that finish early go on to the next item.  Only items that replace
  // shared state (a layer's norm, a layer's first down item, a top-k) start with a
  // barrier.  After a failed wait a warp keeps walking the list without doing work, so
  // that every consumer thread passes the same barriers.
  #pragma unroll 1
  for (int q_it = 0; q_it < S.nitems; q_it++) {
    const Item it = unpack_item(S.items[q_it]);
    const int l = it.l, ia = it.a, in = it.n;
    const DecLayer &Y = S.lay[l];
    const bool pred = is_predicted(P, S, l);
    const bool lora = Y.Bg != nullptr;
    const uint32_t tag = dtag(P, l);
    unsigned long long *blk = P.t_blk + (size_t)l * P.blk;
    if (it.kind == IT_TK) {
      // ---- a reactive layer's top-k over every CTA's router logits
      ab = cbar_or(ab);
      if (!ab) ab |= !poll_to(P.t_rlog + (size_t)l * P.E, reinterpret_cast<uint32_t *>(S.rl), P.E, tag, ct, C);
      ab = cbar_or(ab);
      if (!ab && warp == 0) {
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
    const bool xitem = it.kind != IT_DN;
    const bool shared_state = it.first;        // norm (x items) or down inputs (down items)
    const int slot = q % kNSlot;
    const uint32_t par = (uint32_t)((q / kNSlot) & 1);
    q++;
    if (shared_state) {
      ab = cbar_or(ab);
      // in order: a layer's norm waits for the previous layer's output (its data when
      // chained)
      if (!ab && !P.flat && xitem && l > 0)
        ab |= !poll_to(P.t_y + (size_t)(l - 1) * D, reinterpret_cast<uint32_t *>(S.yprev), D, dtag(P, l - 1), ct, C);
      if (ct == 0 && xitem) stamp(P, l, TR_LAYER);
      if (!ab) ab |= !wait_full(&S.full[slot], par, C);
      ab = cbar_or(ab);
    } else {
      if (!ab) ab |= !wait_full(&S.full[slot], par, C);
      ab = __any_sync(0xffffffffu, ab);
    }
    if (xitem && shared_state) {
      // ---- the norm: gamma and h are the first two segments of the task
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
        if (i < D && !ab) {
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
        if (i < D && !ab) {
          const uint16_t xb = d2bf_bits(hv[m] * (double)bf(gam[i]) * rinv);
          S.xn[i] = xb;
          S.xp[pair_slot(i, D)] = act_f16(bf(xb), i, range_bad);
        }
      }
      cbar();
      // the group sums that every gate/up row of the layer uses with its minima
      #pragma unroll 1
      for (int G = warp; G < D / 64 && !ab; G += kDecCW) {
        const float v = warp_sum(bf(S.xn[64 * G + lane]) + bf(S.xn[64 * G + 32 + lane]));
        if (lane == 0) S.xg[G] = v;
      }
      cbar();
      if (ct == 0) stamp(P, l, TR_NORM);
    }
    if (ab) {
      // nothing more for this item (the barriers above are the same for every thread)
    } else if (it.kind == IT_R) {
      // ---- router rows of a reactive layer, two rows per warp
      const uint16_t *rw = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][2]);
      #pragma unroll 1
      for (int q2 = 2 * warp; q2 < in; q2 += 2 * kDecCW) {
        const bool two = q2 + 1 < in;                  // warp-uniform
        const float2 v = bf16_pair_x<D>(rw + (size_t)q2 * D, rw + (size_t)(two ? q2 + 1 : q2) * D, S.xn, lane);
        if (lane == 0) {
          st_tag(P.t_rlog + (size_t)l * P.E + ia + q2, tag, __float_as_uint(v.x));
          if (two) st_tag(P.t_rlog + (size_t)l * P.E + ia + q2 + 1, tag, __float_as_uint(v.y));
        }
      }
    } else if (it.kind == IT_XR) {
      // ---- head rows, LoRA A rows and the predicted experts' router rows on x, two rows
      // per warp
      const int nh = Y.head ? P.E : 0, nl = lora ? r : 0;
      auto xr_row = [&](int q2, const uint16_t *&row, unsigned long long *&dst) {
        const int u = ia + q2;
        if (u < nh) {
          row = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][kXrHead]) + (size_t)(u - ia) * P.ldh;
          dst = P.t_hlog + (size_t)l * P.E + u;
        } else if (u < nh + nl) {
          row = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][kXrAg]) + (size_t)(u - max(ia, nh)) * D;
          dst = blk + (k + 2) * I + (u - nh);
        } else if (u < nh + 2 * nl) {
          row = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][kXrAu]) +
                (size_t)(u - max(ia, nh + nl)) * D;
          dst = blk + (k + 2) * I + r + (u - nh - nl);
        } else {
          row = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][kXrSel + u - max(ia, nh + 2 * nl)]);
          dst = blk + (k + 2) * I + 2 * r + (u - nh - 2 * nl);
        }
      };
      #pragma unroll 1
      for (int q2 = 2 * warp; q2 < in; q2 += 2 * kDecCW) {
        const bool two = q2 + 1 < in;                  // warp-uniform
        const uint16_t *row0, *row1;
        unsigned long long *dst0, *dst1;
        xr_row(q2, row0, dst0);
        xr_row(two ? q2 + 1 : q2, row1, dst1);
        const float2 v = bf16_pair_x<D>(row0, row1, S.xn, lane);
        if (lane == 0) {
          st_tag(dst0, tag, __float_as_uint(v.x));
          if (two) st_tag(dst1, tag, __float_as_uint(v.y));
        }
      }
    } else if (it.kind == IT_GU) {
      // ---- gate/up: a unit is the gate row and the up row of one intermediate index, a
      // tensor-core row pair (they share x); a warp takes units u and u + kDecCW of each
      // pass, applies the SwiGLU and publishes
      if (ct == 0) stamp(P, l, TR_GU_FULL);
      constexpr int NG = D / 64, NS = (NG + 7) / 8;   // groups per row, 512-wide steps
      const int g8 = lane >> 2, t4 = lane & 3;
      // Rotated columns: in step st the B column n carries the activation of group
      // pg(n) = 2 (((n >> 1) - st) & 3) + (n & 1) of the step (parity kept, so the loads
      // stay free of bank conflicts), which puts row g's diagonal in lane (g, t) exactly
      // when st % 4 == sown = (t - g / 2) % 4: every lane holds one useful gate and one
      // useful up sum per four steps and folds them once, instead of every lane folding
      // every step for the eight lanes that hold a diagonal.
      const int sown = (t4 - (g8 >> 1)) & 3;
      const int slot0 = ia / I;
      // unit u = global unit ia + u: slot es = (ia + u) / I, index i = (ia + u) % I; its
      // piece p is the slot's order among the item's slots, its row the index minus the
      // piece's first index
      struct UnitRows {
        const uint8_t *gc, *uc;
        const uint16_t *gs, *gm, *us, *um;
      };
      auto unit_rows = [&](int u) {
        const int gidx = ia + u, es = gidx / I, p = es - slot0;
        const int i = gidx - es * I, row = i - (p == 0 ? ia - slot0 * I : 0), sg = kGuPiece0 + 6 * p;
        UnitRows R;
        R.gc = S.ring + S.seg_off[slot][sg + 0] + (size_t)row * (D / 2);
        R.gs = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 1]) + (size_t)row * NG;
        R.gm = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 2]) + (size_t)row * NG;
        R.uc = S.ring + S.seg_off[slot][sg + 3] + (size_t)row * (D / 2);
        R.us = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 4]) + (size_t)row * NG;
        R.um = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 5]) + (size_t)row * NG;
        return R;
      };
      auto publish = [&](int u, float ag, float au) {
        const int gidx = ia + u, es = gidx / I, i = gidx - es * I;
        if (es == k) {
          st_tag(blk + k * I + 2 * i, tag, __float_as_uint(ag));
          st_tag(blk + k * I + 2 * i + 1, tag, __float_as_uint(au));
        } else {
          st_tag(blk + es * I + i, tag, f2bf(ag / (1.0f + expf(-ag)) * au));
        }
      };
      const uint4 *xw = reinterpret_cast<const uint4 *>(S.xp);
      #pragma unroll 1
      for (int u0 = warp; u0 < in; u0 += 2 * kDecCW) {
        const int u1 = u0 + kDecCW;
        const bool two = u1 < in;                      // warp-uniform
        const UnitRows A = unit_rows(u0), B = unit_rows(two ? u1 : u0);
        float ag0 = 0.f, au0 = 0.f, ag1 = 0.f, au1 = 0.f;   // folded sums
        float kg0 = 0.f, ku0 = 0.f, kg1 = 0.f, ku1 = 0.f;   // this lane's diagonal of the chunk
#pragma unroll
        for (int st = 0; st < NS; st++) {
          // every lane takes part in the MMAs; lanes past the row's last group (rows
          // shorter than a step) feed zeros, and so do column lanes past it
          const bool gv = 8 * st + g8 < NG;
          const int pg = 2 * (((g8 >> 1) - st) & 3) + (g8 & 1);   // group of this lane's B column
          const bool bv = 8 * st + pg < NG;
          const int wi = 64 * st + 8 * g8 + 2 * t4;  // code word of this lane (natural order)
          const int nw = min(64, D / 8 - 64 * st);   // activation words of this step
          const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
          const uint2 z2 = make_uint2(0u, 0u);
          const uint4 va = bv ? xw[64 * st + 4 * pg + t4] : z4, vb = bv ? xw[64 * st + nw / 2 + 4 * pg + t4] : z4;
          const bool mine = (st & 3) == sown;
          float d[4];
          pair_step(d, gv ? ld_code2(A.gc + 4 * wi) : z2, gv ? ld_code2(A.uc + 4 * wi) : z2, va, vb);
          kg0 = mine ? ((g8 & 1) ? d[1] : d[0]) : kg0;
          ku0 = mine ? ((g8 & 1) ? d[3] : d[2]) : ku0;
          if (two) {
            pair_step(d, gv ? ld_code2(B.gc + 4 * wi) : z2, gv ? ld_code2(B.uc + 4 * wi) : z2, va, vb);
            kg1 = mine ? ((g8 & 1) ? d[1] : d[0]) : kg1;
            ku1 = mine ? ((g8 & 1) ? d[3] : d[2]) : ku1;
          }
          if ((st & 3) == 3 || st == NS - 1) {
            // end of a chunk of four steps: fold this lane's group of the chunk
            const int G = 8 * ((st & ~3) + sown) + g8;
            if (G < NG) {
              const float V = S.xg[G];
              ag0 += group_fold(kg0, A.gs, A.gm, G, V);
              au0 += group_fold(ku0, A.us, A.um, G, V);
              if (two) {
                ag1 += group_fold(kg1, B.gs, B.gm, G, V);
                au1 += group_fold(ku1, B.us, B.um, G, V);
              }
            }
            kg0 = ku0 = kg1 = ku1 = 0.f;
          }
        }
        // the four row sums at once: lane 0 gets u0's gate and up sums, lane 16 u1's
        const float v = warp_sum4(ag0, au0, ag1, au1, lane);
        const float vu = __shfl_down_sync(0xffffffffu, v, 8);
        if (lane == 0) publish(u0, v, vu);
        if (lane == 16 && two) publish(u1, v, vu);
      }
      if (ct == 0) stamp(P, l, TR_GU_DONE);
    } else {
      // ---- down + combine ---------------------------------------------------------------
      constexpr int NGI = I / 64, NSI = (NGI + 7) / 8;   // groups per down row, 512-wide steps
      float *gus = S.gus;
      if (shared_state) {
        // the layer's first down item here: one batched poll over the layer's block (a of
        // the routed slots, the shared expert's raw g/u, t_g/t_u with LoRA, the selected
        // router logits of a predicted layer), then a_s, the gates and t_d, kept for the
        // layer's later down items
        {
          Range rg[4];
          int nr = 0;
          rg[nr++] = Range{blk, S.stg, k * I};
          rg[nr++] = Range{blk + k * I, reinterpret_cast<uint32_t *>(S.gus), 2 * I};
          if (lora) rg[nr++] = Range{blk + (k + 2) * I, reinterpret_cast<uint32_t *>(S.tl), 2 * r};
          if (pred) rg[nr++] = Range{blk + (k + 2) * I + 2 * r, reinterpret_cast<uint32_t *>(S.rl), k};
          ab |= !poll_ranges(rg, nr, tag, ct, C);
        }
        ab = cbar_or(ab);
        if (!ab) {
          // routed a values: bf16 payloads -> bf16 pairs per slot
#pragma unroll 1
          for (int i = ct; i < k * I; i += kDecConsumers) {
            const int j = i / I, e = i - j * I;
            S.ap[j * I + pair_slot(e, I)] = act_f16(bf(S.stg[i] & 0xFFFFu), e, range_bad);
          }
          if (ct == 0) stamp(P, l, TR_A_POLL);
          const int sbd = dn_bd(k);
          const uint16_t *bgm = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sbd + 1]);
          const uint16_t *bum = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sbd + 2]);
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
                for (int q2 = 0; q2 < 4; q2++) {
                  lg = fmaf(bf(gw[q2] & 0xFFFFu), S.tl[j + 2 * q2], lg);
                  lg = fmaf(bf(gw[q2] >> 16), S.tl[j + 2 * q2 + 1], lg);
                  lu = fmaf(bf(uw[q2] & 0xFFFFu), S.tl[r + j + 2 * q2], lu);
                  lu = fmaf(bf(uw[q2] >> 16), S.tl[r + j + 2 * q2 + 1], lu);
                }
              }
              g = fmaf(P.c, lg, g);
              u = fmaf(P.c, lu, u);
            }
            const uint16_t a16 = f2bf(g / (1.0f + expf(-g)) * u);
            S.asraw[i] = bf(a16);
            S.ap[k * I + pair_slot(i, I)] = act_f16(bf(a16), i, range_bad);
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
        }
        cbar();
        // the group sums that every down row of the layer uses with its minima
        #pragma unroll 1
        for (int G = warp; G < (k + 1) * NGI && !ab; G += kDecCW) {
          // from the natural-order values: the routed slots' bf16 payloads, then a_s
          const int j = G / NGI, e0 = (G % NGI) * 64 + lane;
          const float v = warp_sum(j < k ? bf(S.stg[j * I + e0] & 0xFFFFu) + bf(S.stg[j * I + e0 + 32] & 0xFFFFu)
                                         : S.asraw[e0] + S.asraw[e0 + 32]);
          if (lane == 0) S.ag[G] = v;
        }
        if (!ab && lora) {
          // t_d = Ad a_s (LoRA down branch)
          const uint16_t *adm = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][dn_bd(k) + 3]);
          // one half-warp per row (r is a multiple of 8, so a warp's two rows are both in or
          // both out), four independent partial sums per lane
          const int hw = ct >> 4, h16 = ct & 15;
          #pragma unroll 1
          for (int j = hw; j < r; j += 2 * kDecCW) {
            float acc4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int i = h16; i < I; i += 16) acc4[(i >> 4) & 3] = fmaf(bf(adm[j * I + i]), S.asraw[i], acc4[(i >> 4) & 3]);
            const float acc = group_sum((acc4[0] + acc4[1]) + (acc4[2] + acc4[3]), 16);
            if (h16 == 0) S.td[j] = acc;
          }
        }
        cbar();
        if (ct == 0) stamp(P, l, TR_TD_POLL);
      }
      if (!ab) {
        // a warp takes rows 4 w .. 4 w + 3 of each pass as two tensor-core row pairs and
        // owns them across every expert slot: per slot one step per 512 columns, its fold
        // accumulated per lane in the combine order (routed experts with their gates, then
        // the shared expert); the rows' lanes are summed once at the end
        const int g8 = lane >> 2, t4 = lane & 3;
        const bool own = t4 == (g8 >> 1);
        const uint4 *aw = reinterpret_cast<const uint4 *>(S.ap);
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        const uint2 z2 = make_uint2(0u, 0u);
        #pragma unroll 1
        for (int r0 = 4 * warp; r0 < in; r0 += 4 * kDecCW) {
          const bool pair2 = r0 + 2 < in;             // warp-uniform
          bool rv[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; q4++) rv[q4] = r0 + q4 < in;
          float y4[4] = {0.f, 0.f, 0.f, 0.f};
          #pragma unroll 1
          for (int j = 0; j <= k; j++) {
            const float gj = j < k ? S.gates[j] : 1.f;
            const uint8_t *cb = S.ring + S.seg_off[slot][3 * j];
            const uint16_t *sb = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][3 * j + 1]);
            const uint16_t *mb = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][3 * j + 2]);
            float f4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int st = 0; st < NSI; st++) {
              // every lane takes part in the MMAs; lanes past the row's last group feed
              // zeros and fold nothing
              const int G = 8 * st + g8;
              const bool gv = G < NGI;
              const int wi = 64 * st + 8 * g8 + 2 * t4;
              const int nw = min(64, I / 8 - 64 * st);
              const uint4 va = gv ? aw[j * (I / 8) + 64 * st + lane] : z4;
              const uint4 vb = gv ? aw[j * (I / 8) + 64 * st + nw / 2 + lane] : z4;
              const float V = gv ? S.ag[j * NGI + G] : 0.f;
              float d[4];
#pragma unroll
              for (int h = 0; h < 2; h++) {
                if (h == 1 && !pair2) break;
                const int ra = r0 + 2 * h, rb = ra + 1;
                const bool va_ok = gv && rv[2 * h], vb_ok = gv && rv[2 * h + 1];
                pair_step(d, va_ok ? ld_code2(cb + (size_t)ra * (I / 2) + 4 * wi) : z2,
                          vb_ok ? ld_code2(cb + (size_t)rb * (I / 2) + 4 * wi) : z2, va, vb);
                if (va_ok) f4[2 * h] += group_fold((g8 & 1) ? d[1] : d[0], sb + (size_t)ra * NGI, mb + (size_t)ra * NGI, G, V);
                if (vb_ok) f4[2 * h + 1] += group_fold((g8 & 1) ? d[3] : d[2], sb + (size_t)rb * NGI, mb + (size_t)rb * NGI, G, V);
              }
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; q4++) y4[q4] = j < k ? fmaf(gj, f4[q4], y4[q4]) : y4[q4] + f4[q4];
          }
          // the shared expert's LoRA down branch c * (Bd t_d) of each row, its r terms
          // spread over the lanes; then the four row sums at once (lane 8 q4 gets row
          // r0 + q4), stored by four lanes
          const uint16_t *bd = lora ? reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][dn_bd(k)]) : nullptr;
          float v4[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; q4++) {
            float v = own && rv[q4] ? y4[q4] : 0.f;
            if (lora && rv[q4] && lane < r)    // r <= kMaxR <= 32: one term per lane
              v = fmaf(P.c, bf(bd[(r0 + q4) * r + lane]) * S.td[lane], v);
            v4[q4] = v;
          }
          const float v = warp_sum4(v4[0], v4[1], v4[2], v4[3], lane);
          const int q4 = lane >> 3;
          if ((lane & 7) == 0 && r0 + q4 < in) {
            const int n = ia + r0 + q4;
            st_tag(P.t_y + (size_t)l * D + n, tag, __float_as_uint(v));
            P.y[(size_t)l * D + n] = f2bf(v);
            if (P.yf) P.yf[(size_t)l * D + n] = v;
          }
        }
      }
      if (ct == 0) stamp(P, l, TR_DN_DONE);
    }
    // this warp is done with the item's bytes
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[slot]);
  }
  if (range_bad) atomicOr(P.err, kDerrRange);
  ab = cbar_or(ab);
  if (ab) return;
  // ---- end of step: CTA c records layer c's routing and runs layer c's head top-k; every
  // logit is complete by now --------------------------------------------------------------
  #pragma unroll 1
  for (int l = c; l < P.L; l += G) {
    const DecLayer &Y = S.lay[l];
    const uint32_t tag = dtag(P, l);
    if (!is_predicted(P, S, l) && S.sel_ok[l & 63] == 0) {
      // this CTA did not need the layer's own top-k during the step: take it now
      bool bad = !poll_to(P.t_rlog + (size_t)l * P.E, reinterpret_cast<uint32_t *>(S.rl), P.E, tag, ct, C);
      if (cbar_or(bad)) return;
      if (warp == 0) {
        int s8[kMaxK];
        warp_topk_ool(S.rl, P.E, k, lane, s8);
        if (lane == 0) {
          #pragma unroll 1
          for (int j = 0; j < k; j++) S.sel_all[l & 63][j] = s8[j];
        }
      }
      cbar();
    }
    if (ct < k) P.hist_out[((size_t)l * P.maxT) * k + ct] = S.sel_all[l & 63][ct];
    if (!Y.head) continue;
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
