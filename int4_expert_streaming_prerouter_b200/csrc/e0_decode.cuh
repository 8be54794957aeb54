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
constexpr int kRingBytes = 160 * 1024;
constexpr int kTdpMax = 1024;             // t_d partials a CTA may gather (CTAs x rank)
constexpr int kNSlot = 8;                 // tasks in flight
constexpr int kMaxSeg = 64;               // bulk-copy segments per task

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
  uint32_t epoch;
  int step0;                // 1: every layer routes with its own router
  const int32_t *pred_in;   // [L+1][maxT][k]: routing predicted for layer l (previous step)
  int32_t *pred_out;        // [L+1][maxT][k]
  int32_t *hist_out;        // [L][maxT][k]: routing used this step
  const int32_t *hist_prev; // [L][maxT][k] or nullptr (previous step's routing)
  int maxT;
  unsigned long long *t_y, *t_a, *t_lora, *t_tdp, *t_rsel, *t_rlog, *t_hlog;
  int *err;
  unsigned long long timeout_ns;
  int stall_cta;            // test hook: this CTA waits on a tag nobody writes (-1: none)
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

__host__ __device__ __forceinline__ void split_range(int N, int G, int c, int &a, int &b) {
  a = (int)((long long)N * c / G);
  b = (int)((long long)N * (c + 1) / G);
}

// nibble i of a 32-bit code word is placed in the mantissa of 2^23 + q * 2^p(i) without
// shifting (i < 5) or after one shift by 12 (i >= 5); the matching activation is
// pre-scaled by 2^-p(i) so that the product is exactly q * x.
__host__ __device__ constexpr float nib_scale(int i) {
  return i == 0 ? 1.f : i == 1 ? 1.f / 16 : (i == 2 || i == 5) ? 1.f / 256 : (i == 3 || i == 6) ? 1.f / 4096 : 1.f / 65536;
}

// sum_k q_k x'_k over one 16-byte chunk (32 nibbles), x' pre-scaled as above (fp32 x32 in
// shared memory, 16-byte aligned).  Exact products, fp32 pairwise accumulation.
__device__ __forceinline__ float chunk_qdot(const uint4 w, const float *xp) {
  const unsigned long long kMagic = pk2(-8388608.f, -8388608.f);
  unsigned long long acc0 = 0ull, acc1 = 0ull;
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int t = 0; t < 4; t++) {
    const uint32_t a = ws[t], b = a >> 12;
    const float4 x0 = *reinterpret_cast<const float4 *>(xp + 8 * t);
    const float4 x1 = *reinterpret_cast<const float4 *>(xp + 8 * t + 4);
    const uint32_t v0 = (a & 0x0000000Fu) | 0x4B000000u, v1 = (a & 0x000000F0u) | 0x4B000000u;
    const uint32_t v2 = (a & 0x00000F00u) | 0x4B000000u, v3 = (a & 0x0000F000u) | 0x4B000000u;
    const uint32_t v4 = (a & 0x000F0000u) | 0x4B000000u, v5 = (b & 0x00000F00u) | 0x4B000000u;
    const uint32_t v6 = (b & 0x0000F000u) | 0x4B000000u, v7 = (b & 0x000F0000u) | 0x4B000000u;
    const unsigned long long q01 = f2add(((unsigned long long)v1 << 32) | v0, kMagic);
    const unsigned long long q23 = f2add(((unsigned long long)v3 << 32) | v2, kMagic);
    const unsigned long long q45 = f2add(((unsigned long long)v5 << 32) | v4, kMagic);
    const unsigned long long q67 = f2add(((unsigned long long)v7 << 32) | v6, kMagic);
    acc0 = f2fma(q01, pk2(x0.x, x0.y), acc0);
    acc1 = f2fma(q23, pk2(x0.z, x0.w), acc1);
    acc0 = f2fma(q45, pk2(x1.x, x1.y), acc0);
    acc1 = f2fma(q67, pk2(x1.z, x1.w), acc1);
  }
  return f2sum(acc0) + f2sum(acc1);
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
  Seg s[kMaxSeg];
  __device__ __forceinline__ void add(const void *p, size_t bytes) {
    if (n < kMaxSeg) s[n++] = Seg{(const uint8_t *)p, (uint32_t)bytes};
  }
};

enum : int { TK_ROUTER = 0, TK_GU = 1, TK_DN = 2 };

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

// Build the segment list of task (kind, layer) for CTA c.  `sel` are the layer's routed
// experts.  The consumer code reads the segments back in exactly this order.
template <int D, int I>
__device__ void build_task(const DecodeParams &P, int kind, int l, int c, bool predicted, const int *sel,
                           TaskBuf &T) {
  const DecLayer &Y = P.layers[l];
  const Blob bl = blob_of(D, I);
  T.n = 0;
  if (kind == TK_ROUTER) {
    T.add(Y.gamma, D * 2);
    T.add(P.h + (size_t)l * D, D * 2);
    int a, b;
    split_range(P.E, P.G, c, a, b);
    if (b > a) T.add(Y.router + (size_t)a * D, (size_t)(b - a) * D * 2);
  } else if (kind == TK_GU) {
    if (predicted) {
      T.add(Y.gamma, D * 2);
      T.add(P.h + (size_t)l * D, D * 2);
    }
    int a, b;
    if (Y.Ag) {
      split_range(2 * P.r, P.G, c, a, b);
      for (int q = a; q < b; q++) T.add((q < P.r ? Y.Ag + (size_t)q * D : Y.Au + (size_t)(q - P.r) * D), D * 2);
    }
    if (predicted) {
      split_range(P.k, P.G, (c + P.G - min(2 * P.r, P.G - 1)) % P.G, a, b);
      for (int q = a; q < b; q++) T.add(Y.router + (size_t)sel[q] * D, D * 2);
    }
    GuPiece pc[4];
    const int np = gu_pieces<D, I>(P.k, P.G, c, pc);
    for (int p = 0; p < np; p++) {
      const uint8_t *base = pc[p].slot < P.k ? Y.experts + (size_t)sel[pc[p].slot] * bl.bytes : Y.shared;
      const int R = pc[p].i1 - pc[p].i0, i0 = pc[p].i0;
      T.add(base + bl.gc + (size_t)i0 * (D / 2), (size_t)R * (D / 2));
      T.add(base + bl.gs + (size_t)i0 * (D / 64) * 2, (size_t)R * (D / 64) * 2);
      T.add(base + bl.gm + (size_t)i0 * (D / 64) * 2, (size_t)R * (D / 64) * 2);
      T.add(base + bl.uc + (size_t)i0 * (D / 2), (size_t)R * (D / 2));
      T.add(base + bl.us + (size_t)i0 * (D / 64) * 2, (size_t)R * (D / 64) * 2);
      T.add(base + bl.um + (size_t)i0 * (D / 64) * 2, (size_t)R * (D / 64) * 2);
      if (pc[p].slot == P.k && Y.Bg) {
        T.add(Y.Bg + (size_t)i0 * P.r, (size_t)R * P.r * 2);
        T.add(Y.Bu + (size_t)i0 * P.r, (size_t)R * P.r * 2);
        for (int q = 0; q < P.r; q++) T.add(Y.Ad + (size_t)q * I + i0, (size_t)R * 2);
      }
    }
  } else {
    int a, b;
    split_range(D, P.G, c, a, b);
    const int R = b - a;
    if (R > 0) {
      for (int j = 0; j <= P.k; j++) {
        const uint8_t *base = j < P.k ? Y.experts + (size_t)sel[j] * bl.bytes : Y.shared;
        T.add(base + bl.dc + (size_t)a * (I / 2), (size_t)R * (I / 2));
        T.add(base + bl.ds + (size_t)a * (I / 64) * 2, (size_t)R * (I / 64) * 2);
        T.add(base + bl.dm + (size_t)a * (I / 64) * 2, (size_t)R * (I / 64) * 2);
      }
      if (Y.Bd) T.add(Y.Bd + (size_t)a * P.r, (size_t)R * P.r * 2);
    }
    if (Y.head) {
      split_range(P.E, P.G, c, a, b);
      if (b > a) T.add(Y.head + (size_t)a * P.ldh, (size_t)(b - a) * P.ldh * 2);
    }
  }
}

// ---------------------------------------------------------------------------------------
// Shared-memory layout
// ---------------------------------------------------------------------------------------
template <int D, int I>
struct DecSmem {
  uint8_t ring[kRingBytes];
  float x[D], xp[D], yprev[D];
  float xs32[D / 32];
  float ap[(kMaxK + 1) * I];
  float as32[(kMaxK + 1) * I / 32];
  float ydot[64 * (kMaxK + 1)];
  float red[64];
  double dred[16];
  float gates[kMaxK];
  float tl[2 * kMaxR];      // t_g, t_u
  float td[kMaxR];          // t_d
  float rl[kMaxE];          // router logits (reactive layers)
  float tdp[kTdpMax];       // gathered t_d partials
  int sel[kMaxK];
  int sel_all[64][kMaxK];   // routing of every layer this step (for the head's one-hot)
  uint32_t seg_off[kNSlot][kMaxSeg];   // smem byte offset of each segment's first wanted byte
  uint64_t full[kNSlot], empty[kNSlot];
  volatile int sel_ready;   // layer whose `sel` the consumers have published (reactive)
  volatile int abort;
};

__device__ __forceinline__ bool is_predicted(const DecodeParams &P, int l) {
  return !P.step0 && l > 0 && P.layers[l - 1].head != nullptr;
}

__device__ __forceinline__ uint32_t dtag(const DecodeParams &P, int l) { return P.epoch * 64u + (uint32_t)l; }

// ---------------------------------------------------------------------------------------
// Producer: walk this CTA's task list and stream it through the ring.
// ---------------------------------------------------------------------------------------
template <int D, int I>
__device__ void producer(const DecodeParams &P, DecSmem<D, I> &S) {
  const int c = blockIdx.x;
  TaskBuf T;
  int q = 0;                       // task sequence number
  int head = 0;                    // next free byte of the ring
  int qs[kNSlot];                  // in-flight tasks: start byte (FIFO by q)
  int oldest = 0;                  // sequence number of the oldest in-flight task
  int sel[kMaxK];
  const unsigned long long t_start = gtimer();
  bool ok = true;

  auto wait_empty = [&](int seq) -> bool {
    // wait until the consumers have released task `seq`
    const int slot = seq % kNSlot;
    const uint32_t par = (uint32_t)((seq / kNSlot) & 1);
    unsigned long long t0 = 0;
    while (!mbar_test(&S.empty[slot], par)) {
      if (S.abort) return false;
      if (!t0) t0 = gtimer();
      else if (gtimer() - t0 > P.timeout_ns) {
        atomicOr(P.err, DERR_TIMEOUT);
        S.abort = 1;
        return false;
      }
    }
    return true;
  };

  for (int l = 0; l < P.L && ok; l++) {
    const bool pred = is_predicted(P, l);
    for (int kind = pred ? TK_GU : TK_ROUTER; kind <= TK_DN && ok; kind++) {
      if (kind == TK_GU) {
        if (pred) {
          for (int j = 0; j < P.k; j++) sel[j] = P.pred_in[((size_t)l * P.maxT) * P.k + j];
        } else {
          // the consumers publish the layer's own top-k once its router has run
          unsigned long long t0 = gtimer();
          while (S.sel_ready != l) {
            if (S.abort) { ok = false; break; }
            if (gtimer() - t0 > P.timeout_ns) {
              atomicOr(P.err, DERR_TIMEOUT);
              S.abort = 1;
              ok = false;
              break;
            }
            __nanosleep(32);
          }
          if (!ok) break;
          for (int j = 0; j < P.k; j++) sel[j] = S.sel[j];
        }
        for (int j = 0; j < P.k; j++)
          if (sel[j] < 0 || sel[j] >= P.E) {
            atomicOr(P.err, DERR_INDEX);
            sel[j] = 0;
          }
      }
      build_task<D, I>(P, kind, l, c, pred, sel, T);
      // bytes of this task, each segment rounded out to 16-byte boundaries
      int need = 0;
      for (int i = 0; i < T.n; i++) {
        const uintptr_t lo = (uintptr_t)T.s[i].src & ~(uintptr_t)15;
        const uintptr_t hi = ((uintptr_t)T.s[i].src + T.s[i].bytes + 15) & ~(uintptr_t)15;
        need += (int)(hi - lo);
      }
      if (need > kRingBytes) {
        atomicOr(P.err, DERR_TIMEOUT);
        S.abort = 1;
        ok = false;
        break;
      }
      // allocate [start, start+need) in the ring, releasing the oldest tasks as required.
      // In-flight bytes are [tail, head) (or wrapped: [tail, end) + [0, head)); a gap of at
      // least one byte is kept so that head == tail only when nothing is in flight.
      int start = -1;
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
        ok = wait_empty(oldest);
        oldest++;
      }
      if (!ok) break;
      const int slot = q % kNSlot;
      int off = start;
      for (int i = 0; i < T.n; i++) {
        const uintptr_t lo = (uintptr_t)T.s[i].src & ~(uintptr_t)15;
        const uintptr_t hi = ((uintptr_t)T.s[i].src + T.s[i].bytes + 15) & ~(uintptr_t)15;
        S.seg_off[slot][i] = (uint32_t)(off + ((uintptr_t)T.s[i].src - lo));
        off += (int)(hi - lo);
      }
      mbar_expect_tx(&S.full[slot], (uint32_t)need);
      off = start;
      for (int i = 0; i < T.n; i++) {
        const uintptr_t lo = (uintptr_t)T.s[i].src & ~(uintptr_t)15;
        const uintptr_t hi = ((uintptr_t)T.s[i].src + T.s[i].bytes + 15) & ~(uintptr_t)15;
        bulk_g2s(S.ring + off, (const void *)lo, (uint32_t)(hi - lo), &S.full[slot]);
        off += (int)(hi - lo);
      }
      qs[slot] = start;
      head = start + need;
      q++;
    }
  }
  (void)t_start;
  // drain: every issued copy must have landed before the CTA exits
  for (int s = oldest; s < q; s++) {
    const int slot = s % kNSlot;
    const uint32_t par = (uint32_t)((s / kNSlot) & 1);
    const unsigned long long t0 = gtimer();
    while (!mbar_test(&S.full[slot], par)) {
      if (gtimer() - t0 > P.timeout_ns) {
        atomicOr(P.err, DERR_TIMEOUT);
        break;
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// Consumer helpers
// ---------------------------------------------------------------------------------------
struct Ctl {
  unsigned long long timeout;
  int *err;
  volatile int *abort;
};

// Poll `n` tagged words; returns false on timeout/abort.  Payloads go through `sink`.
template <typename Sink>
__device__ __forceinline__ bool poll_words(const unsigned long long *p, int n, uint32_t tag, int tid, int nthr,
                                           const Ctl &C, Sink sink) {
  for (int i = tid; i < n; i += nthr) {
    unsigned long long v = ld_tag(p + i);
    if ((uint32_t)v != tag) {
      const unsigned long long t0 = gtimer();
      do {
        __nanosleep(20);
        v = ld_tag(p + i);
        if ((uint32_t)v == tag) break;
        if (*C.abort) return false;
        if (gtimer() - t0 > C.timeout) {
          atomicOr(C.err, DERR_TIMEOUT);
          *C.abort = 1;
          return false;
        }
      } while (true);
    }
    sink(i, (uint32_t)(v >> 32));
  }
  return true;
}

__device__ __forceinline__ bool wait_full(uint64_t *bar, uint32_t par, const Ctl &C) {
  if (mbar_test(bar, par)) return true;
  const unsigned long long t0 = gtimer();
  while (!mbar_test(bar, par)) {
    if (*C.abort) return false;
    if (gtimer() - t0 > C.timeout) {
      atomicOr(C.err, DERR_TIMEOUT);
      *C.abort = 1;
      return false;
    }
  }
  return true;
}

// bf16 row (D elements in shared memory) dotted with x (fp32, shared memory): one warp.
template <int D>
__device__ __forceinline__ float bf16_row_x(const uint16_t *w, const float *x, int lane) {
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

// ---------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------
template <int D, int I>
__global__ void __launch_bounds__(kDecThreads, 1) k_decode(DecodeParams P) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecSmem<D, I> &S = *reinterpret_cast<DecSmem<D, I> *>(smem_raw);
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < kNSlot; s++) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kDecCW);
    }
    S.sel_ready = -1;
    S.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (tid < 32) {
    if (tid == 0) producer<D, I>(P, S);
    return;
  }
  // ------------------------------- consumers -------------------------------------------
  const int ct = tid - 32, warp = ct >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = P.G, k = P.k, r = P.r;
  Ctl C{P.timeout_ns, P.err, &S.abort};
  int q = 0;
  bool ab = false;
  // CTAs whose gate/up range holds shared-expert rows (they publish partials of t_d)
  int sh_lo = G, sh_hi = -1;
  for (int cc = 0; cc < G; cc++) {
    int a0, b0;
    split_range((k + 1) * I, G, cc, a0, b0);
    if (b0 > a0 && b0 > k * I) {
      sh_lo = min(sh_lo, cc);
      sh_hi = cc;
    }
  }

  if (c == P.stall_cta) {
    // test hook: wait for a word that is never written, so that the timeout path runs
    ab |= !poll_words(P.t_y, 1, 0xFFFFFFFFu, ct, 1, C, [](int, uint32_t) {});
  }

  for (int l = 0; l < P.L; l++) {
    const DecLayer &Y = P.layers[l];
    const bool pred = is_predicted(P, l);
    const uint32_t tag = dtag(P, l);
    // ---- wait for the previous layer's output (data in chained mode, order otherwise)
    if (l > 0) {
      const uint32_t ptag = dtag(P, l - 1);
      float *yp = S.yprev;
      ab |= !poll_words(P.t_y + (size_t)(l - 1) * D, D, ptag, ct, kDecConsumers, C,
                        [&](int i, uint32_t v) { yp[i] = __uint_as_float(v); });
    }
    if (cbar_or(ab)) break;

    int slot = q % kNSlot;
    uint32_t par = (uint32_t)((q / kNSlot) & 1);
    // ---- the norm: gamma and h are the first two segments of the layer's first task
    ab |= !wait_full(&S.full[slot], par, C);
    if (cbar_or(ab)) break;
    {
      const uint16_t *gam = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][0]);
      const uint16_t *hin = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][1]);
      const bool chain = P.chained && l > 0;
      double ss = 0.0;
      for (int i = ct; i < D; i += kDecConsumers) {
        double v = (double)bf(hin[i]);
        if (chain) v = (double)bf(d2bf(v + (double)S.yprev[i]));
        ss += v * v;
      }
      ss = warp_sum(ss);
      if (lane == 0) S.dred[warp] = ss;
      cbar();
      double tot = 0.0;
      for (int w = 0; w < kDecCW; w++) tot += S.dred[w];
      const double rinv = 1.0 / sqrt(tot / D + (double)P.eps);
      for (int i = ct; i < D; i += kDecConsumers) {
        double v = (double)bf(hin[i]);
        if (chain) v = (double)bf(d2bf(v + (double)S.yprev[i]));
        const float xv = bf(d2bf(v * (double)bf(gam[i]) * rinv));
        S.x[i] = xv;
        S.xp[i] = xv * nib_scale(i & 7);
      }
      cbar();
      for (int ch = ct; ch < D / 32; ch += kDecConsumers) {
        float s = 0.f;
        for (int i = 0; i < 32; i++) s += S.x[ch * 32 + i];
        S.xs32[ch] = s;
      }
    }
    // ---- reactive layer: own router rows, then everyone's logits, then top-k
    if (!pred) {
      int a, b;
      split_range(P.E, G, c, a, b);
      const uint16_t *rw = reinterpret_cast<const uint16_t *>(S.ring + (b > a ? S.seg_off[slot][2] : 0));
      for (int row = a + warp; row < b; row += kDecCW) {
        const float v = bf16_row_x<D>(rw + (size_t)(row - a) * D, S.x, lane);
        if (lane == 0) st_tag(P.t_rlog + (size_t)l * P.E + row, tag, __float_as_uint(v));
      }
      cbar();
      if (lane == 0) mbar_arrive(&S.empty[slot]);
      q++;
      float *rl = S.rl;
      ab |= !poll_words(P.t_rlog + (size_t)l * P.E, P.E, tag, ct, kDecConsumers, C,
                        [&](int i, uint32_t v) { rl[i] = __uint_as_float(v); });
      if (cbar_or(ab)) break;
      if (warp == 0) {
        int s8[kMaxK];
        warp_topk(S.rl, P.E, k, lane, s8);
        if (lane == 0) {
          for (int j = 0; j < k; j++) S.sel[j] = s8[j];
          __threadfence_block();
          S.sel_ready = l;
        }
      }
      cbar();
      slot = q % kNSlot;
      par = (uint32_t)((q / kNSlot) & 1);
      ab |= !wait_full(&S.full[slot], par, C);
      if (cbar_or(ab)) break;
    } else {
      if (ct < k) S.sel[ct] = P.pred_in[((size_t)l * P.maxT) * k + ct];
      cbar();
    }
    // ---- gate/up phase --------------------------------------------------------------
    {
      int sg = pred ? 2 : 0;   // segment cursor
      int a, b;
      if (Y.Ag) {
        split_range(2 * r, G, c, a, b);
        for (int qq = a; qq < b; qq++, sg++) {
          if (warp == (qq - a) % kDecCW) {
            const float v = bf16_row_x<D>(reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg]), S.x, lane);
            if (lane == 0) st_tag(P.t_lora + (size_t)l * 2 * r + qq, tag, __float_as_uint(v));
          }
        }
      }
      if (pred) {
        split_range(k, G, (c + G - min(2 * r, G - 1)) % G, a, b);
        for (int qq = a; qq < b; qq++, sg++) {
          if (warp == (kDecCW - 1 - (qq - a) % kDecCW)) {
            const float v = bf16_row_x<D>(reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg]), S.x, lane);
            if (lane == 0) st_tag(P.t_rsel + (size_t)l * k + qq, tag, __float_as_uint(v));
          }
        }
      }
      GuPiece pc[4];
      const int np = gu_pieces<D, I>(k, G, c, pc);
      constexpr int NCH = D / 32;                 // 16-byte chunks per row
      constexpr int LPR = NCH < 32 ? NCH : 32;    // lanes per row
      constexpr int RPW = 32 / LPR;               // rows per warp pass
      constexpr int CPL = NCH / LPR;              // chunks per lane
      const int sub = lane / LPR, sl = lane % LPR;
      for (int p = 0; p < np; p++) {
        const int R = pc[p].i1 - pc[p].i0;
        const uint8_t *gc = S.ring + S.seg_off[slot][sg + 0];
        const uint16_t *gs = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 1]);
        const uint16_t *gm = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 2]);
        const uint8_t *uc = S.ring + S.seg_off[slot][sg + 3];
        const uint16_t *us = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 4]);
        const uint16_t *um = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 5]);
        const bool shared = pc[p].slot == k;
        const bool lora = shared && Y.Bg != nullptr;
        float *gu_g = S.ydot;          // scratch: raw g and u of this piece (shared expert)
        // warp-per-(row, gate|up) dot products
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
              const float qd = chunk_qdot(w, S.xp + ch * 32);
              acc = fmaf(bf(sc[ch >> 1]), qd, fmaf(bf(mn[ch >> 1]), S.xs32[ch], acc));
            }
          }
          acc = group_sum(acc, LPR);
          if (valid && sl == 0) gu_g[item] = acc;
        }
        cbar();
        if (lora) {
          // t_g, t_u from the CTAs that own the LoRA A rows
          float *tl = S.tl;
          ab |= !poll_words(P.t_lora + (size_t)l * 2 * r, 2 * r, tag, ct, kDecConsumers, C,
                            [&](int i, uint32_t v) { tl[i] = __uint_as_float(v); });
        }
        if (cbar_or(ab)) break;
        // SwiGLU (+ LoRA up) and the tagged store of a; two a values per word
        const uint16_t *bg = lora ? reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 6]) : nullptr;
        const uint16_t *bu = lora ? reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 7]) : nullptr;
        float *ahere = S.ap;           // a values of this piece (fp32 copy of the bf16)
        for (int row = ct; row < R; row += kDecConsumers) {
          float g = gu_g[2 * row], u = gu_g[2 * row + 1];
          if (lora) {
            float lg = 0.f, lu = 0.f;
            for (int j = 0; j < r; j++) {
              lg = fmaf(bf(bg[row * r + j]), S.tl[j], lg);
              lu = fmaf(bf(bu[row * r + j]), S.tl[r + j], lu);
            }
            g = fmaf(P.c, lg, g);
            u = fmaf(P.c, lu, u);
          }
          ahere[row] = bf(f2bf(g / (1.0f + expf(-g)) * u));
        }
        cbar();
        {
          const int i0 = pc[p].i0, gbase = pc[p].slot * I;
          // one tagged word per a value (bf16 bits in the payload)
          for (int i = ct; i < R; i += kDecConsumers) {
            const int gi = gbase + i0 + i;
            const uint32_t bits = __float_as_uint(ahere[i]) >> 16;
            st_tag(P.t_a + (size_t)l * (k + 1) * I + gi, tag, bits);
          }
        }
        if (lora) {
          // partial t_d = Ad[:, rows] a_s[rows] of this CTA, stored per CTA (fixed order sum)
          for (int j = warp; j < r; j += kDecCW) {
            const uint16_t *ad = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][sg + 8 + j]);
            float acc = 0.f;
            for (int i = lane; i < R; i += 32) acc = fmaf(bf(ad[i]), ahere[i], acc);
            acc = warp_sum(acc);
            if (lane == 0) st_tag(P.t_tdp + ((size_t)l * G + c) * r + j, tag, __float_as_uint(acc));
          }
        }
        cbar();
        sg += 6 + (lora ? 2 + r : 0);
      }
      if (cbar_or(ab)) break;
      if (lane == 0) mbar_arrive(&S.empty[slot]);
      q++;
    }
    // ---- down + combine phase ----------------------------------------------------------
    slot = q % kNSlot;
    par = (uint32_t)((q / kNSlot) & 1);
    {
      // a of every slot, gates, t_d
      float *ap = S.ap;
      ab |= !poll_words(P.t_a + (size_t)l * (k + 1) * I, (k + 1) * I, tag, ct, kDecConsumers, C,
                        [&](int i, uint32_t v) { ap[i] = bf(v & 0xFFFFu) * nib_scale(i & 7); });
      float *rl = S.rl;
      if (pred)
        ab |= !poll_words(P.t_rsel + (size_t)l * k, k, tag, ct, kDecConsumers, C,
                          [&](int i, uint32_t v) { rl[i] = __uint_as_float(v); });
      if (Y.Bd) {
        // CTAs whose gate/up range holds shared-expert rows wrote a partial t_d each
        const int ncta = sh_hi - sh_lo + 1, clo = sh_lo;
        float *tdp = S.tdp;    // [ncta][r]; the host checks ncta * r <= kTdpMax
        if (ncta > 0)
          ab |= !poll_words(P.t_tdp + ((size_t)l * G + clo) * r, ncta * r, tag, ct, kDecConsumers, C,
                            [&](int i, uint32_t v) { tdp[i] = __uint_as_float(v); });
        if (cbar_or(ab)) break;
        if (ct < r) {
          float s = 0.f;
          for (int cc = 0; cc < ncta; cc++) s += tdp[cc * r + ct];
          S.td[ct] = s;
        }
      }
      if (cbar_or(ab)) break;
      // chunk sums of a (unscaled) and the gates
      for (int ch = ct; ch < (k + 1) * I / 32; ch += kDecConsumers) {
        float s = 0.f;
        for (int i = 0; i < 32; i++) s += S.ap[ch * 32 + i] / nib_scale(i & 7);
        S.as32[ch] = s;
      }
      if (ct == 0) {
        float lg[kMaxK], mx = -INFINITY, sum = 0.f;
        for (int j = 0; j < k; j++) {
          lg[j] = pred ? S.rl[j] : S.rl[S.sel[j]];
          mx = fmaxf(mx, lg[j]);
        }
        for (int j = 0; j < k; j++) {
          lg[j] = expf(lg[j] - mx);
          sum += lg[j];
        }
        for (int j = 0; j < k; j++) S.gates[j] = lg[j] / sum;
      }
      ab |= !wait_full(&S.full[slot], par, C);
      if (cbar_or(ab)) break;
      int a, b;
      split_range(D, G, c, a, b);
      const int R = b - a;
      constexpr int NCH = I / 32;
      constexpr int LPR = NCH < 32 ? NCH : 32;
      constexpr int RPW = 32 / LPR;
      constexpr int CPL = NCH / LPR;
      const int sub = lane / LPR, sl = lane % LPR;
      float *yd = S.ydot;
      for (int base = warp * RPW; base < R * (k + 1); base += kDecCW * RPW) {
        const int item = base + sub;
        const bool valid = item < R * (k + 1);
        float acc = 0.f;
        if (valid) {
          const int row = item / (k + 1), j = item % (k + 1);
          const uint8_t *cw = S.ring + S.seg_off[slot][3 * j] + (size_t)row * (I / 2);
          const uint16_t *sc = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][3 * j + 1]) + (size_t)row * (I / 64);
          const uint16_t *mn = reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][3 * j + 2]) + (size_t)row * (I / 64);
          const float *aj = S.ap + j * I;
          const float *asj = S.as32 + j * (I / 32);
#pragma unroll
          for (int cc = 0; cc < CPL; cc++) {
            const int ch = sl + cc * LPR;
            const uint4 w = *reinterpret_cast<const uint4 *>(cw + ch * 16);
            const float qd = chunk_qdot(w, aj + ch * 32);
            acc = fmaf(bf(sc[ch >> 1]), qd, fmaf(bf(mn[ch >> 1]), asj[ch], acc));
          }
        }
        acc = group_sum(acc, LPR);
        if (valid && sl == 0) yd[item] = acc;
      }
      // head rows (this layer's prerouter head on x) while the dots above drain
      int sgh = R > 0 ? 3 * (k + 1) + (Y.Bd ? 1 : 0) : 0;
      if (Y.head) {
        int ha, hb;
        split_range(P.E, G, c, ha, hb);
        const uint16_t *hw = reinterpret_cast<const uint16_t *>(S.ring + (hb > ha ? S.seg_off[slot][sgh] : 0));
        for (int row = ha + warp; row < hb; row += kDecCW) {
          const float v = bf16_row_x<D>(hw + (size_t)(row - ha) * P.ldh, S.x, lane);
          if (lane == 0) st_tag(P.t_hlog + (size_t)l * P.E + row, tag, __float_as_uint(v));
        }
      }
      cbar();
      const uint16_t *bd = (Y.Bd && R > 0) ? reinterpret_cast<const uint16_t *>(S.ring + S.seg_off[slot][3 * (k + 1)]) : nullptr;
      for (int row = ct; row < R; row += kDecConsumers) {
        float y = 0.f;
        for (int j = 0; j < k; j++) y = fmaf(S.gates[j], yd[row * (k + 1) + j], y);
        y += yd[row * (k + 1) + k];
        if (bd) {
          float lo = 0.f;
          for (int j = 0; j < r; j++) lo = fmaf(bf(bd[row * r + j]), S.td[j], lo);
          y = fmaf(P.c, lo, y);
        }
        const int n = a + row;
        st_tag(P.t_y + (size_t)l * D + n, tag, __float_as_uint(y));
        P.y[(size_t)l * D + n] = f2bf(y);
        if (P.yf) P.yf[(size_t)l * D + n] = y;
      }
      cbar();
      if (lane == 0) mbar_arrive(&S.empty[slot]);
      q++;
    }
    // routing used by this layer (kept locally; one CTA records it for the host)
    if (ct < k) {
      S.sel_all[l & 63][ct] = S.sel[ct];
      if (c == 0) P.hist_out[((size_t)l * P.maxT) * k + ct] = S.sel[ct];
    }
  }
  if (ab) return;
  // ---- head top-k: CTA c handles layer c's head; its logits are complete by now ------
  for (int l = c; l < P.L; l += G) {
    const DecLayer &Y = P.layers[l];
    if (!Y.head) continue;
    const uint32_t tag = dtag(P, l);
    float *rl = S.rl;
    bool bad = !poll_words(P.t_hlog + (size_t)l * P.E, P.E, tag, ct, kDecConsumers, C,
                           [&](int i, uint32_t v) { rl[i] = __uint_as_float(v); });
    if (cbar_or(bad)) return;
    if (P.onehot) {
      // one-hot columns of this layer's routing now and at the previous token
      for (int e = ct; e < P.E; e += kDecConsumers) {
        const uint16_t *wr = Y.head + (size_t)e * P.ldh + D;
        float v = S.rl[e];
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
      warp_topk(S.rl, P.E, k, lane, s8);
      if (lane < k) {
        int mine = 0;
        for (int j = 0; j < k; j++)
          if (j == lane) mine = s8[j];
        P.pred_out[((size_t)(l + 1) * P.maxT) * k + lane] = mine;
      }
    }
    cbar();
  }
}

}  // namespace e0
