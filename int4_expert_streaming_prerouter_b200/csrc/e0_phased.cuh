// Phased decode: one decode step of up to 8 streams through every layer of the stack as
// six short kernels, for steps whose layer inputs are given (none reads another layer's
// output within the step).
//
// Method (pages: "The Other Half of the Memory Wall" reading guide, "Temel fikirler",
// "Ön Yönlendirici Başlık Mimarisi", "Birleştirilmemiş Adaptör Yürütme", "Sorular"; the
// ai.info article "Edge0 serve un MoE da 35B ..."): per layer x = bf16(RMSNorm(h)); the
// routing is the previous layer's head prediction made one token earlier, or the layer's
// own router top-k; w = softmax of the router logits over the selection;
// y = sum_j w_j E_j(x) + E_shared(x) with the shared expert's unmerged LoRA; the layer's
// head (linear l(u), optionally + fc2(gelu_erf(fc1 u + b1)) + b2 over u = [x; onehot(cur);
// onehot(prev)]) predicts the next layer's routing for the next token.
//
// B200 design:
//   * Six kernels per step, each over every layer at once: norm -> bf16 rows (routers,
//     heads, LoRA A, the full head's fc1) -> routing, gates, expert plan and the heads'
//     top-k -> int4 gate/up + SwiGLU -> activation group sums and the LoRA t_d -> int4
//     down + weighted combine.  The later five are launched with programmatic dependent
//     launch: every kernel lets the next one launch at its start, and each CTA issues the
//     loads that depend on nothing of this step (weight rows of layers whose routing was
//     predicted one token earlier) before it waits for the previous kernel, so the weight
//     stream of one phase starts under the tail of the previous one.
//   * Many small CTAs (one per 8 intermediate indices of one expert, one per 16 output
//     rows of one layer, one per 16 bf16 rows), several resident per SM, each warp
//     issuing all of its weight loads at once: the HBM stream is kept busy by the number
//     of loads in flight, not by a software pipeline.
//   * int4 dot products on the tensor cores with the tokens on the MMA's N dimension:
//     mma.sync m16n8k16 bf16, A = 16 weight rows restricted to 16 K values of one
//     quantisation group, expanded exactly to bf16 128 + q (one mask and one OR per two
//     codes), B = the activations of up to 8 tokens on the same K values, fp32
//     accumulators; after the group's four MMAs the affine weights are folded in once per
//     (row, group, token): acc += s P + (m - 128 s) X, X = the group's activation sum.
//     Each lane's D entries are whole dot products of its rows and tokens: no warp
//     reductions.  K is split across the warps of a CTA and the partial sums are added
//     in a fixed order, so results are reproducible run to run.
#pragma once
#include <algorithm>
#include <vector>
#include "e0_device.cuh"
#include "e0_kernels.cuh"
#include "e0_decode.cuh"

namespace e0 {

constexpr int kPhMaxB = 8;                       // tokens per pass of the kernels (the MMA's N)
constexpr int kPhGroups = 8;                     // passes per step: up to 64 streams
constexpr int kPhMaxU = kPhMaxB * kMaxK + 1;     // distinct routed experts + the shared one
constexpr int kPhMaxH = 512;                     // full-head hidden width on this path
constexpr int kPhBatch = 3;                      // experts whose down rows a warp loads at once
constexpr int kPlanInts = 1 + kPhMaxU;           // U, then the expert list

struct PhLayer {
  const uint8_t *experts, *shared;
  const uint16_t *router, *gamma, *head, *fc1, *fc1_b, *fc2, *fc2_b;
  const uint16_t *Ag, *Bg, *Au, *Bu, *Ad, *Bd;
};

// Work of the bf16-rows kernel: 16 rows of one layer.
enum : int { PR_ROUTER = 0, PR_SEL = 1, PR_HEAD = 2, PR_LORA = 3, PR_FC1 = 4 };
struct PhBlock {
  int l, kind, row0, nrows;
};

struct PhParams {
  const PhLayer *layers;
  int L, B, E, k, r, H, ldh, onehot, step0, maxT;
  float eps, c;
  // the caller's step input and outputs [L][hB][D]; this launch serves tokens
  // tok0 .. tok0 + B - 1 of them (the routing tables are offset to the same tokens)
  const uint16_t *h;
  uint16_t *y;
  float *yf;                    // or nullptr
  int hB, tok0;
  // workspace, token stride kPhMaxB
  uint16_t *x16, *xp;           // [L][8][D] x (natural order) and x in pair order
  float *xs;                    // [L][8][D/64] group sums of x
  float *rlog, *rsel, *hlog;    // [L][8][E] router logits, [L][8][k] selected, [L][8][E] head
  float *lt;                    // [L][8][3][r] t_g = Ag x, t_u = Au x, t_d = Ad a_s
  float *h1;                    // [L][8][H] fc1 x-part
  float *gates;                 // [L][8][k]
  // expert plans, one per layer: U, the U distinct routed experts in first-seen order,
  // and for each of them the slot in which each token routed to it (-1: not routed).
  // plan_cur: this step's (for a predicted layer written by the previous step's routing
  // kernel, which made the prediction; for a reactive layer by this step's);
  // plan_next: the next step's predicted layers, written by this step's heads.
  int *plan_cur, *plan_next;          // [L][kPlanInts]
  int8_t *slot_cur, *slot_next;       // [L][kPhMaxU][kPhMaxB]
  uint16_t *a;                  // [L][8][k+1][I] activations in pair order
  float *gus;                   // [L][8][2][I] the shared expert's g and u before its LoRA
  float *asum;                  // [L][8][k+1][I/64]
  const int32_t *pred_in;       // [L+1][maxT][k] routing predicted for layer l (prev step)
  int32_t *pred_out;            // [L+1][maxT][k]
  int32_t *hist_out;            // [L][maxT][k] routing used
  const int32_t *hist_prev;     // [L][maxT][k] or nullptr
  const PhBlock *blocks;
  int nblocks;
  int *err;
};

// ---------------------------------------------------------------------------------------
// helpers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void ph_launch_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void ph_wait_prev() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint2 ldg_nc64(const void *p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ldg_nc128(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint16_t ldg_nc16(const void *p) {
  unsigned short v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ bool ph_predicted(const PhParams &P, int l) {
  return !P.step0 && l > 0 && P.layers[l - 1].head != nullptr;
}
__device__ __forceinline__ int ph_clamp_e(int e, int E) { return e < 0 ? 0 : (e >= E ? E - 1 : e); }

// The expert plan of one layer from its routing rows idx[n * ld + j] (n < B, j < k), built
// by one warp: the distinct experts in first-seen order (tokens, then rank) and each
// token's slot for each of them.  Entry i = n k + j; lane l handles entries l and l + 32.
__device__ inline void ph_build_plan(const int32_t *idx, int ld, int B, int k, int E, int *plan, int8_t *slots,
                                     int lane) {
  const int n = B * k;
  int e_[2], first[2];
#pragma unroll
  for (int h = 0; h < 2; h++) {
    const int i = lane + 32 * h;
    e_[h] = i < n ? ph_clamp_e(idx[(size_t)(i / k) * ld + i % k], E) : -1;
    first[h] = i;               // first entry with the same expert
    if (i < n)
      for (int j = 0; j < i; j++)
        if (ph_clamp_e(idx[(size_t)(j / k) * ld + j % k], E) == e_[h]) { first[h] = j; break; }
  }
  const unsigned b0 = __ballot_sync(0xffffffffu, lane < n && first[0] == lane);
  const unsigned b1 = __ballot_sync(0xffffffffu, 32 + lane < n && first[1] == 32 + lane);
  const int U = __popc(b0) + __popc(b1);
  // position in the list of entry f (a first occurrence)
  auto pos = [&](int f) {
    return f < 32 ? __popc(b0 & ((1u << f) - 1u)) : __popc(b0) + __popc(b1 & ((1u << (f - 32)) - 1u));
  };
  for (int q = lane; q < U * kPhMaxB; q += 32) slots[q] = -1;
  __syncwarp();
#pragma unroll
  for (int h = 0; h < 2; h++) {
    const int i = lane + 32 * h;
    if (i < n) {
      const int u = pos(first[h]);
      if (first[h] == i) plan[1 + u] = e_[h];
      slots[u * kPhMaxB + i / k] = (int8_t)(i % k);
    }
  }
  if (lane == 0) plan[0] = U;
  __syncwarp();
}

// Fold of one group into two accumulators: acc += s P + (m - 128 s) X.
__device__ __forceinline__ float ph_fold(float acc, float s, float mprime, float Pv, float X) {
  return fmaf(s, Pv, fmaf(mprime, X, acc));
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------------------------------
// K0: RMSNorm of every (layer, token): x in natural order and in pair order, and the
// activation sums of every group of 64.  One CTA per (layer, token).  As in the per-layer
// kernels the norm is evaluated in double and rounded once to bf16.
// ---------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) k_ph_norm(PhParams P) {
  ph_launch_next();
  const int l = blockIdx.x / P.B, n = blockIdx.x % P.B;
  const uint16_t *hr = P.h + ((size_t)l * P.hB + P.tok0 + n) * D;
  const uint16_t *gm = P.layers[l].gamma;
  __shared__ double red[8];
  __shared__ uint16_t xs16[D];
  double ss = 0.0;
  for (int i = threadIdx.x; i < D; i += 256) {
    const double v = (double)bf(hr[i]);
    ss += v * v;
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  double tot = 0.0;
#pragma unroll
  for (int w = 0; w < 8; w++) tot += red[w];
  const double rinv = 1.0 / sqrt(tot / D + (double)P.eps);
  const size_t o = ((size_t)l * kPhMaxB + n) * D;
  for (int i = threadIdx.x; i < D; i += 256) {
    const uint16_t b = d2bf((double)bf(hr[i]) * (double)bf(gm[i]) * rinv);
    xs16[i] = b;
    P.x16[o + i] = b;
    P.xp[o + pair_index(i)] = b;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int G = warp; G < D / 64; G += 8) {
    const float v = warp_sum(bf(xs16[64 * G + lane]) + bf(xs16[64 * G + 32 + lane]));
    if (lane == 0) P.xs[((size_t)l * kPhMaxB + n) * (D / 64) + G] = v;
  }
}

// ---------------------------------------------------------------------------------------
// KA: bf16 rows dotted with x (router rows, selected router rows of predicted layers,
// head rows, LoRA A rows, fc1 rows of the full head).  One CTA per block of 16 rows of one
// layer; warp w takes K chunks [w * CPW, (w + 1) * CPW) of 64.  Per chunk, lane (g, t)
// holds elements 16 t .. 16 t + 15 of rows g and g + 8 (eight bf16 pairs each) and of x of
// token g; MMA m takes pairs 2m, 2m + 1 of each, so that every K value meets its x.
// ---------------------------------------------------------------------------------------
template <int D>
struct PhRowsCfg {
  static constexpr int NCH = D / 64;
  static constexpr int NW = NCH < 16 ? NCH : 16;
  static constexpr int CPW = NCH / NW;
};

template <int D>
__global__ void __launch_bounds__(32 * PhRowsCfg<D>::NW) k_ph_rows(PhParams P) {
  using Cfg = PhRowsCfg<D>;
  constexpr int NW = Cfg::NW, CPW = Cfg::CPW;
  ph_launch_next();
  const PhBlock bk = P.blocks[blockIdx.x];
  const int l = bk.l;
  const PhLayer &Y = P.layers[l];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  __shared__ int s_rows[16];
  __shared__ float part[NW][32][4];
  if (threadIdx.x < 16) {
    const int q = threadIdx.x;
    if (bk.kind == PR_SEL) {
      // the predicted layer's distinct experts: the plan the previous step's heads made
      const int *pl = P.plan_cur + (size_t)l * kPlanInts;
      s_rows[q] = bk.row0 + q < pl[0] ? pl[1 + bk.row0 + q] : -1;
    } else {
      s_rows[q] = q < bk.nrows ? bk.row0 + q : -1;
    }
  }
  __syncthreads();
  // row pointers of MMA rows g and g + 8
  auto row_ptr = [&](int q) -> const uint16_t * {
    const int rw = s_rows[q];
    if (rw < 0) return nullptr;
    switch (bk.kind) {
      case PR_ROUTER:
      case PR_SEL: return Y.router + (size_t)ph_clamp_e(rw, P.E) * D;
      case PR_HEAD: return Y.head + (size_t)rw * P.ldh;
      case PR_LORA: return rw < P.r ? Y.Ag + (size_t)rw * D : Y.Au + (size_t)(rw - P.r) * D;
      default: return Y.fc1 + (size_t)rw * P.ldh;
    }
  };
  const uint16_t *r0 = row_ptr(g), *r1 = row_ptr(g + 8);
  uint4 w0[CPW][2], w1[CPW][2];
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int c = 0; c < CPW; c++) {
    const int k0 = 64 * (warp * CPW + c) + 16 * t;
    w0[c][0] = r0 ? ldg_nc128(r0 + k0) : z4;
    w0[c][1] = r0 ? ldg_nc128(r0 + k0 + 8) : z4;
    w1[c][0] = r1 ? ldg_nc128(r1 + k0) : z4;
    w1[c][1] = r1 ? ldg_nc128(r1 + k0 + 8) : z4;
  }
  ph_wait_prev();
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  const uint16_t *xr = P.x16 + ((size_t)l * kPhMaxB + g) * D;
#pragma unroll
  for (int c = 0; c < CPW; c++) {
    const int k0 = 64 * (warp * CPW + c) + 16 * t;
    uint4 xa = z4, xb = z4;
    if (g < P.B) {
      xa = *reinterpret_cast<const uint4 *>(xr + k0);
      xb = *reinterpret_cast<const uint4 *>(xr + k0 + 8);
    }
    mma_bf16_16816(d, w0[c][0].x, w1[c][0].x, w0[c][0].y, w1[c][0].y, xa.x, xa.y);
    mma_bf16_16816(d, w0[c][0].z, w1[c][0].z, w0[c][0].w, w1[c][0].w, xa.z, xa.w);
    mma_bf16_16816(d, w0[c][1].x, w1[c][1].x, w0[c][1].y, w1[c][1].y, xb.x, xb.y);
    mma_bf16_16816(d, w0[c][1].z, w1[c][1].z, w0[c][1].w, w1[c][1].w, xb.z, xb.w);
  }
#pragma unroll
  for (int q = 0; q < 4; q++) part[warp][lane][q] = d[q];
  __syncthreads();
  // one thread per (row, token): sum the warps' partials in order and store
  for (int tid = threadIdx.x; tid < 16 * P.B; tid += blockDim.x) {
    const int rho = tid % 16, n = tid / 16;
    const int src = 4 * (rho & 7) + n / 2, q = (rho >= 8 ? 2 : 0) + (n & 1);
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; w++) v += part[w][src][q];
    const int rw = s_rows[rho];
    if (rw >= 0) {
      const size_t tn = (size_t)l * kPhMaxB + n;
      switch (bk.kind) {
        case PR_ROUTER: P.rlog[tn * P.E + rw] = v; break;
        case PR_SEL: {
          const int j = P.slot_cur[((size_t)l * kPhMaxU + bk.row0 + rho) * kPhMaxB + n];
          if (j >= 0) P.rsel[tn * P.k + j] = v;
          break;
        }
        case PR_HEAD: P.hlog[tn * P.E + rw] = v; break;
        case PR_LORA: P.lt[(tn * 3 + (rw < P.r ? 0 : 1)) * P.r + (rw < P.r ? rw : rw - P.r)] = v; break;
        default: P.h1[tn * P.H + rw] = v; break;
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// KB: per layer, the routing of every token (the prediction made one token earlier, or
// the own router's top-k), its gate weights, the layer's distinct experts, and the head's
// prediction of the next layer's routing for the next token.  One CTA per layer.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_ph_route(PhParams P) {
  ph_launch_next();
  ph_wait_prev();
  const int l = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PhLayer &Y = P.layers[l];
  const bool pred = ph_predicted(P, l);
  const int k = P.k, E = P.E, B = P.B;
  __shared__ int s_idx[kPhMaxB][kMaxK];
  __shared__ float z[kPhMaxB][kMaxE];
  __shared__ float h1s[kPhMaxB][kPhMaxH];
  if (warp < B) {
    const int n = warp;
    const size_t tn = (size_t)l * kPhMaxB + n;
    int sel[kMaxK];
    if (pred) {
#pragma unroll
      for (int j = 0; j < kMaxK; j++) sel[j] = j < k ? P.pred_in[((size_t)l * P.maxT + n) * k + j] : 0;
    } else {
      warp_topk(P.rlog + tn * E, E, k, lane, sel);
    }
    float lg[kMaxK], mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMaxK; j++) {
      if (j >= k) break;
      if (sel[j] < 0 || sel[j] >= E) {
        if (lane == 0) atomicOr(P.err, DERR_INDEX);
        sel[j] = 0;
      }
      lg[j] = pred ? P.rsel[tn * k + j] : P.rlog[tn * E + sel[j]];
      mx = fmaxf(mx, lg[j]);
    }
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; j++) {
      if (j >= k) break;
      for (int q = j + 1; q < k; q++)
        if (sel[q] == sel[j] && lane == 0) atomicOr(P.err, DERR_DUP);
      lg[j] = expf(lg[j] - mx);
      sum += lg[j];
    }
    if (lane < k) {
      int e = 0;
      float gw = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxK; j++)
        if (j == lane) {
          e = sel[j];
          gw = lg[j] / sum;
        }
      s_idx[n][lane] = e;
      P.hist_out[((size_t)l * P.maxT + n) * k + lane] = e;
      P.gates[tn * k + lane] = gw;
    }
  }
  __syncthreads();
  // a reactive layer's plan for this step's expert kernels (a predicted layer's was made
  // by the previous step's heads)
  if (!pred && warp == 0)
    ph_build_plan(&s_idx[0][0], kMaxK, B, k, E, P.plan_cur + (size_t)l * kPlanInts,
                  P.slot_cur + (size_t)l * kPhMaxU * kPhMaxB, lane);
  if (!Y.head) return;
  // ---- head: z = l(u) [+ fc2(gelu_erf(fc1 u + b1)) + b2], u = [x; onehot(cur); onehot(prev)]
  const int D = P.ldh - (P.onehot ? 2 * E : 0);
  if (P.H > 0) {
    for (int i = threadIdx.x; i < B * P.H; i += blockDim.x) {
      const int n = i / P.H, q = i % P.H;
      float v = P.h1[((size_t)l * kPhMaxB + n) * P.H + q] + bf(Y.fc1_b[q]);
      if (P.onehot) {
        const uint16_t *w = Y.fc1 + (size_t)q * P.ldh + D;
        for (int j = 0; j < k; j++) {
          v += bf(w[s_idx[n][j]]);
          if (P.hist_prev) {
            const int pv = P.hist_prev[((size_t)l * P.maxT + n) * k + j];
            if (pv >= 0 && pv < E) v += bf(w[E + pv]);
          }
        }
      }
      h1s[n][q] = 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
    }
    __syncthreads();
  }
  for (int i = threadIdx.x; i < B * E; i += blockDim.x) {
    const int n = i / E, e = i % E;
    float v = P.hlog[((size_t)l * kPhMaxB + n) * E + e];
    if (P.onehot) {
      const uint16_t *w = Y.head + (size_t)e * P.ldh + D;
      for (int j = 0; j < k; j++) {
        v += bf(w[s_idx[n][j]]);
        if (P.hist_prev) {
          const int pv = P.hist_prev[((size_t)l * P.maxT + n) * k + j];
          if (pv >= 0 && pv < E) v += bf(w[E + pv]);
        }
      }
    }
    if (P.H > 0) {
      const uint16_t *w2 = Y.fc2 + (size_t)e * P.H;
      float acc = 0.f;
      for (int q = 0; q < P.H; q += 8) {
        const uint4 wv = *reinterpret_cast<const uint4 *>(w2 + q);
        acc = fmaf(bf_lo(wv.x), h1s[n][q], acc);
        acc = fmaf(bf_hi(wv.x), h1s[n][q + 1], acc);
        acc = fmaf(bf_lo(wv.y), h1s[n][q + 2], acc);
        acc = fmaf(bf_hi(wv.y), h1s[n][q + 3], acc);
        acc = fmaf(bf_lo(wv.z), h1s[n][q + 4], acc);
        acc = fmaf(bf_hi(wv.z), h1s[n][q + 5], acc);
        acc = fmaf(bf_lo(wv.w), h1s[n][q + 6], acc);
        acc = fmaf(bf_hi(wv.w), h1s[n][q + 7], acc);
      }
      v += acc + bf(Y.fc2_b[e]);
    }
    z[n][e] = v;
  }
  __syncthreads();
  __shared__ int s_pred[kPhMaxB][kMaxK];
  if (warp < B) {
    int p[kMaxK];
    warp_topk(z[warp], E, k, lane, p);
    if (lane < k) {
      int mine = 0;
#pragma unroll
      for (int j = 0; j < kMaxK; j++)
        if (j == lane) mine = p[j];
      P.pred_out[((size_t)(l + 1) * P.maxT + warp) * k + lane] = mine;
      s_pred[warp][lane] = mine;
    }
  }
  __syncthreads();
  // the next step's plan of the layer this head predicts
  if (l + 1 < P.L && warp == 0)
    ph_build_plan(&s_pred[0][0], kMaxK, B, k, E, P.plan_next + (size_t)(l + 1) * kPlanInts,
                  P.slot_next + (size_t)(l + 1) * kPhMaxU * kPhMaxB, lane);
}

// ---------------------------------------------------------------------------------------
// KC: gate/up + SwiGLU.  One CTA per (layer, expert of the layer's plan or the shared
// expert, kPhGuBlocks blocks of 8 intermediate indices): while a block's products are
// formed, the next block's weights are already in flight.  MMA row g is the gate row
// i0 + g, row g + 8 the up row i0 + g; warp w takes groups 4w .. 4w + 3 of K.  Lane (g, t)
// holds bytes 8 t .. 8 t + 7 of each of its rows' groups (16 codes: nibbles j and j + 4 of a
// word form the bf16 pair {128 + q_j, 128 + q_(j+4)}) and the same 16 activations of token
// g in pair order.  The warps' partial sums are added in order.  The shared expert's g and
// u go out before its LoRA and activation, which the next kernel applies.
// ---------------------------------------------------------------------------------------
constexpr int kPhGuBlocks = 8;   // blocks of 8 intermediate indices per gate/up CTA
template <int D, int I>
__global__ void __launch_bounds__(32 * (D / 256)) k_ph_gateup(PhParams P) {
  constexpr int NG = D / 64, NW = NG / 4, O = I / 8, OC = O / kPhGuBlocks;
  static_assert(NG % 4 == 0, "D must be a multiple of 256");
  static_assert(O % kPhGuBlocks == 0, "I / 8 must be a multiple of the blocks per CTA");
  ph_launch_next();
  const int Umax = min(P.B * P.k, P.E) + 1;
  const int oc = blockIdx.x % OC, u = (blockIdx.x / OC) % Umax, l = blockIdx.x / (OC * Umax);
  const PhLayer &Y = P.layers[l];
  const bool pred = ph_predicted(P, l);
  const int k = P.k, E = P.E;
  __shared__ int s_e;
  __shared__ int s_slot[kPhMaxB];
  __shared__ float part[2][NW][32][4];
  if (!pred) ph_wait_prev();
  if (threadIdx.x < kPhMaxB) {
    // this CTA's expert and, per token, the slot it was routed to the expert in
    const int *pl = P.plan_cur + (size_t)l * kPlanInts;
    const int U = pl[0], n = threadIdx.x;
    const int e = u < U ? pl[1 + u] : (u == U ? E : -1);
    if (n == 0) s_e = e;
    s_slot[n] = n >= P.B || e < 0 ? -1 : (e == E ? k : P.slot_cur[((size_t)l * kPhMaxU + u) * kPhMaxB + n]);
  }
  __syncthreads();
  const int e = s_e;
  if (e < 0) return;
  const Blob bl = blob_of(D, I);
  const uint8_t *base = e == E ? Y.shared : Y.experts + (size_t)ph_clamp_e(e, E) * bl.bytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int G0 = warp * 4;
  // one block's weights of this lane: codes of its gate and up rows, their scales and minima
  struct W {
    uint2 cg[4], cu[4], sg, mg, su, mu;
  };
  auto load = [&](int o, W &w) {
    const int i = o * 8 + g;
#pragma unroll
    for (int q = 0; q < 4; q++) {
      w.cg[q] = ldg_nc64(base + bl.gc + (size_t)i * (D / 2) + 32 * (G0 + q) + 8 * t);
      w.cu[q] = ldg_nc64(base + bl.uc + (size_t)i * (D / 2) + 32 * (G0 + q) + 8 * t);
    }
    w.sg = ldg_nc64(base + bl.gs + ((size_t)i * NG + G0) * 2);
    w.mg = ldg_nc64(base + bl.gm + ((size_t)i * NG + G0) * 2);
    w.su = ldg_nc64(base + bl.us + ((size_t)i * NG + G0) * 2);
    w.mu = ldg_nc64(base + bl.um + ((size_t)i * NG + G0) * 2);
  };
  W cur, nxt;
  load(oc * kPhGuBlocks, cur);
  if (pred) ph_wait_prev();
  const size_t tg = (size_t)l * kPhMaxB;
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int ob = 0; ob < kPhGuBlocks; ob++) {
    const int o = oc * kPhGuBlocks + ob;
    if (ob + 1 < kPhGuBlocks) load(o + 1, nxt);
    float ag0 = 0.f, ag1 = 0.f, au0 = 0.f, au1 = 0.f;
#pragma unroll
    for (int q = 0; q < 4; q++) {
      const int G = G0 + q;
      uint4 xa = z4, xb = z4;
      if (g < P.B) {
        const uint16_t *xr = P.xp + (tg + g) * D + 64 * G + 16 * t;
        xa = *reinterpret_cast<const uint4 *>(xr);
        xb = *reinterpret_cast<const uint4 *>(xr + 8);
      }
      const float X0 = 2 * t < P.B ? P.xs[(tg + 2 * t) * NG + G] : 0.f;
      const float X1 = 2 * t + 1 < P.B ? P.xs[(tg + 2 * t + 1) * NG + G] : 0.f;
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      mma_bf16_16816(d, nib_pair_bf16(cur.cg[q].x, 0), nib_pair_bf16(cur.cu[q].x, 0), nib_pair_bf16(cur.cg[q].x, 1),
                     nib_pair_bf16(cur.cu[q].x, 1), xa.x, xa.y);
      mma_bf16_16816(d, nib_pair_bf16(cur.cg[q].x, 2), nib_pair_bf16(cur.cu[q].x, 2), nib_pair_bf16(cur.cg[q].x, 3),
                     nib_pair_bf16(cur.cu[q].x, 3), xa.z, xa.w);
      mma_bf16_16816(d, nib_pair_bf16(cur.cg[q].y, 0), nib_pair_bf16(cur.cu[q].y, 0), nib_pair_bf16(cur.cg[q].y, 1),
                     nib_pair_bf16(cur.cu[q].y, 1), xb.x, xb.y);
      mma_bf16_16816(d, nib_pair_bf16(cur.cg[q].y, 2), nib_pair_bf16(cur.cu[q].y, 2), nib_pair_bf16(cur.cg[q].y, 3),
                     nib_pair_bf16(cur.cu[q].y, 3), xb.z, xb.w);
      const uint32_t wsg = q < 2 ? cur.sg.x : cur.sg.y, wmg = q < 2 ? cur.mg.x : cur.mg.y;
      const uint32_t wsu = q < 2 ? cur.su.x : cur.su.y, wmu = q < 2 ? cur.mu.x : cur.mu.y;
      const float s_g = (q & 1) ? bf_hi(wsg) : bf_lo(wsg), m_g = (q & 1) ? bf_hi(wmg) : bf_lo(wmg);
      const float s_u = (q & 1) ? bf_hi(wsu) : bf_lo(wsu), m_u = (q & 1) ? bf_hi(wmu) : bf_lo(wmu);
      const float mp_g = fmaf(-128.f, s_g, m_g), mp_u = fmaf(-128.f, s_u, m_u);
      ag0 = ph_fold(ag0, s_g, mp_g, d[0], X0);
      ag1 = ph_fold(ag1, s_g, mp_g, d[1], X1);
      au0 = ph_fold(au0, s_u, mp_u, d[2], X0);
      au1 = ph_fold(au1, s_u, mp_u, d[3], X1);
    }
    // partial sums double-buffered: the reduction of block ob - 1 (same buffer two blocks
    // back) finished before this block's barrier
    float (*pt)[32][4] = part[ob & 1];
    pt[warp][lane][0] = ag0;
    pt[warp][lane][1] = ag1;
    pt[warp][lane][2] = au0;
    pt[warp][lane][3] = au1;
    __syncthreads();
    for (int tid = threadIdx.x; tid < 8 * P.B; tid += blockDim.x) {
      const int ii = tid % 8, n = tid / 8;
      const int src = 4 * ii + n / 2, hh = n & 1;
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int w = 0; w < NW; w++) {
        gs += pt[w][src][hh];
        us += pt[w][src][2 + hh];
      }
      const int iidx = o * 8 + ii;
      const size_t tn = tg + n;
      if (e == E) {
        P.gus[tn * 2 * I + iidx] = gs;
        P.gus[tn * 2 * I + I + iidx] = us;
      } else {
        const int sl = s_slot[n];
        if (sl >= 0) P.a[(tn * (k + 1) + sl) * I + pair_index(iidx)] = f2bf(gs / (1.0f + expf(-gs)) * us);
      }
    }
    if (ob + 1 < kPhGuBlocks) cur = nxt;
  }
}

// ---------------------------------------------------------------------------------------
// KT: per (layer, token): the group sums of every slot's activations (the down fold's X)
// and the LoRA down input t_d = Ad a_s of the shared expert.
// ---------------------------------------------------------------------------------------
template <int I>
__global__ void __launch_bounds__(256) k_ph_tdsum(PhParams P) {
  constexpr int NGI = I / 64;
  ph_launch_next();
  ph_wait_prev();
  const int l = blockIdx.x / P.B, n = blockIdx.x % P.B, k = P.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t tn = (size_t)l * kPhMaxB + n;
  uint16_t *a = P.a + tn * (k + 1) * I;
  const PhLayer &Y = P.layers[l];
  {
    // the shared expert's activation: its unmerged LoRA up branch added to g and u
    // (g += c Bg t_g, u += c Bu t_u), then a_s = bf16(silu(g) u)
    const float *gu = P.gus + tn * 2 * I;
    const float *tl = P.lt + tn * 3 * P.r;
    for (int i = threadIdx.x; i < I; i += blockDim.x) {
      float gs = gu[i], us = gu[I + i];
      if (Y.Bg) {
        float lg = 0.f, lu = 0.f;
        for (int q = 0; q < P.r; q++) {
          lg = fmaf(bf(Y.Bg[(size_t)i * P.r + q]), tl[q], lg);
          lu = fmaf(bf(Y.Bu[(size_t)i * P.r + q]), tl[P.r + q], lu);
        }
        gs = fmaf(P.c, lg, gs);
        us = fmaf(P.c, lu, us);
      }
      a[(size_t)k * I + pair_index(i)] = f2bf(gs / (1.0f + expf(-gs)) * us);
    }
  }
  __syncthreads();
  for (int q = warp; q < (k + 1) * NGI; q += 8) {
    const int j = q / NGI, G = q % NGI;
    const uint16_t *ag = a + (size_t)j * I + 64 * G;    // a group of 64 is 64 consecutive pair-order entries
    const float v = warp_sum(bf(ag[lane]) + bf(ag[32 + lane]));
    if (lane == 0) P.asum[tn * (k + 1) * NGI + q] = v;
  }
  if (!Y.Ad) return;
  const uint16_t *as = a + (size_t)k * I;
  for (int q = warp; q < P.r; q += 8) {
    float acc = 0.f;
    for (int i = lane; i < I; i += 32) acc = fmaf(bf(Y.Ad[(size_t)q * I + i]), bf(as[pair_index(i)]), acc);
    acc = warp_sum(acc);
    if (lane == 0) P.lt[(tn * 3 + 2) * P.r + q] = acc;
  }
}

// ---------------------------------------------------------------------------------------
// KD: down projection and weighted combine.  One CTA per (layer, 16 output rows); warp w
// takes group w of the I/64 groups of K, for every expert of the layer's plan and then the
// shared expert.  MMA rows g and g + 8 are output rows n0 + g and n0 + g + 8; column n is
// token n: the activations of token n in the slot where it routed to the expert (zero if
// it did not), so that lane (g, t) accumulates rows g, g + 8 of tokens 2t, 2t + 1 across
// experts with the gate weights, in the plan's order.  Dynamic shared memory: the layer's
// activations [B][k+1][I] (pair order) and their group sums.
// ---------------------------------------------------------------------------------------
template <int D, int I>
__host__ __device__ inline size_t ph_dn_smem(int B, int k) {
  return (size_t)B * (k + 1) * I * 2 + (size_t)B * (k + 1) * (I / 64) * 4;
}

template <int D, int I>
__global__ void __launch_bounds__(32 * (I / 64)) k_ph_down(PhParams P) {
  constexpr int NGI = I / 64, NW = NGI, HX = D / 16;
  ph_launch_next();
  extern __shared__ __align__(16) uint8_t ph_smem[];
  const int B = P.B, k = P.k, E = P.E;
  uint16_t *s_a = reinterpret_cast<uint16_t *>(ph_smem);                       // [B][k+1][I]
  float *s_asum = reinterpret_cast<float *>(s_a + (size_t)B * (k + 1) * I);     // [B][k+1][NGI]
  const int h16 = blockIdx.x % HX, l = blockIdx.x / HX;
  const PhLayer &Y = P.layers[l];
  const bool pred = ph_predicted(P, l);
  __shared__ int s_list[kPhMaxU];
  __shared__ int s_U;
  __shared__ int8_t s_slot[kPhMaxU][kPhMaxB];
  __shared__ float s_gate[kPhMaxB][kMaxK];
  __shared__ float part[NW][32][4];
  if (!pred) ph_wait_prev();
  {
    const int *pl = P.plan_cur + (size_t)l * kPlanInts;
    const int8_t *sl = P.slot_cur + (size_t)l * kPhMaxU * kPhMaxB;
    const int U0 = pl[0];
    if (threadIdx.x == 0) s_U = U0;
    for (int i = threadIdx.x; i < U0; i += blockDim.x) s_list[i] = pl[1 + i];
    for (int i = threadIdx.x; i < U0 * kPhMaxB; i += blockDim.x) (&s_slot[0][0])[i] = sl[i];
  }
  __syncthreads();
  const int U = s_U, total = U + 1;
  const Blob bl = blob_of(D, I);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3, G = warp;
  const int n0 = 16 * h16 + g, n1 = n0 + 8;
  const size_t tg = (size_t)l * kPhMaxB;
  float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
  for (int u0 = 0; u0 < total; u0 += kPhBatch) {
    uint2 c0[kPhBatch], c1[kPhBatch];
    uint16_t sv0[kPhBatch], mv0[kPhBatch], sv1[kPhBatch], mv1[kPhBatch];
#pragma unroll
    for (int b = 0; b < kPhBatch; b++) {
      const int u = u0 + b;
      if (u < total) {
        const uint8_t *base = u < U ? Y.experts + (size_t)ph_clamp_e(s_list[u], E) * bl.bytes : Y.shared;
        c0[b] = ldg_nc64(base + bl.dc + (size_t)n0 * (I / 2) + 32 * G + 8 * t);
        c1[b] = ldg_nc64(base + bl.dc + (size_t)n1 * (I / 2) + 32 * G + 8 * t);
        sv0[b] = ldg_nc16(base + bl.ds + ((size_t)n0 * NGI + G) * 2);
        mv0[b] = ldg_nc16(base + bl.dm + ((size_t)n0 * NGI + G) * 2);
        sv1[b] = ldg_nc16(base + bl.ds + ((size_t)n1 * NGI + G) * 2);
        mv1[b] = ldg_nc16(base + bl.dm + ((size_t)n1 * NGI + G) * 2);
      } else {
        c0[b] = c1[b] = make_uint2(0u, 0u);
        sv0[b] = mv0[b] = sv1[b] = mv1[b] = 0;
      }
    }
    if (u0 == 0) {
      // the activations, their sums and the gates of the layer's tokens
      if (pred) ph_wait_prev();
      const uint4 *src = reinterpret_cast<const uint4 *>(P.a + tg * (k + 1) * I);
      uint4 *dst = reinterpret_cast<uint4 *>(s_a);
      for (int i = threadIdx.x; i < B * (k + 1) * I / 8; i += blockDim.x) dst[i] = src[i];
      for (int i = threadIdx.x; i < B * (k + 1) * NGI; i += blockDim.x) s_asum[i] = P.asum[tg * (k + 1) * NGI + i];
      for (int i = threadIdx.x; i < B * k; i += blockDim.x) s_gate[i / k][i % k] = P.gates[(tg + i / k) * k + i % k];
      __syncthreads();
    }
#pragma unroll
    for (int b = 0; b < kPhBatch; b++) {
      const int u = u0 + b;
      if (u >= total) break;
      const bool sh = u == U;
      // slot of token g (B operand column g) and of tokens 2t, 2t + 1 (gates, sums)
      auto slot_of = [&](int n) -> int { return n >= B ? -1 : (sh ? k : (int)s_slot[u][n]); };
      const int sg = slot_of(g), s0 = slot_of(2 * t), s1 = slot_of(2 * t + 1);
      uint4 xa = make_uint4(0u, 0u, 0u, 0u), xb = xa;
      if (sg >= 0) {
        const uint16_t *ar = s_a + ((size_t)g * (k + 1) + sg) * I + 64 * G + 16 * t;
        xa = *reinterpret_cast<const uint4 *>(ar);
        xb = *reinterpret_cast<const uint4 *>(ar + 8);
      }
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      mma_bf16_16816(d, nib_pair_bf16(c0[b].x, 0), nib_pair_bf16(c1[b].x, 0), nib_pair_bf16(c0[b].x, 1),
                     nib_pair_bf16(c1[b].x, 1), xa.x, xa.y);
      mma_bf16_16816(d, nib_pair_bf16(c0[b].x, 2), nib_pair_bf16(c1[b].x, 2), nib_pair_bf16(c0[b].x, 3),
                     nib_pair_bf16(c1[b].x, 3), xa.z, xa.w);
      mma_bf16_16816(d, nib_pair_bf16(c0[b].y, 0), nib_pair_bf16(c1[b].y, 0), nib_pair_bf16(c0[b].y, 1),
                     nib_pair_bf16(c1[b].y, 1), xb.x, xb.y);
      mma_bf16_16816(d, nib_pair_bf16(c0[b].y, 2), nib_pair_bf16(c1[b].y, 2), nib_pair_bf16(c0[b].y, 3),
                     nib_pair_bf16(c1[b].y, 3), xb.z, xb.w);
      const float gw0 = s0 < 0 ? 0.f : (sh ? 1.f : s_gate[2 * t][s0]);
      const float gw1 = s1 < 0 ? 0.f : (sh ? 1.f : s_gate[2 * t + 1][s1]);
      const float A0 = s0 < 0 ? 0.f : s_asum[((size_t)(2 * t) * (k + 1) + s0) * NGI + G];
      const float A1 = s1 < 0 ? 0.f : s_asum[((size_t)(2 * t + 1) * (k + 1) + s1) * NGI + G];
      const float s_0 = bf(sv0[b]), s_1 = bf(sv1[b]);
      const float mp0 = fmaf(-128.f, s_0, bf(mv0[b])), mp1 = fmaf(-128.f, s_1, bf(mv1[b]));
      y00 = fmaf(gw0, ph_fold(0.f, s_0, mp0, d[0], A0), y00);
      y01 = fmaf(gw1, ph_fold(0.f, s_0, mp0, d[1], A1), y01);
      y10 = fmaf(gw0, ph_fold(0.f, s_1, mp1, d[2], A0), y10);
      y11 = fmaf(gw1, ph_fold(0.f, s_1, mp1, d[3], A1), y11);
    }
  }
  part[warp][lane][0] = y00;
  part[warp][lane][1] = y01;
  part[warp][lane][2] = y10;
  part[warp][lane][3] = y11;
  __syncthreads();
  for (int tid = threadIdx.x; tid < 16 * B; tid += blockDim.x) {
    const int rho = tid % 16, n = tid / 16;
    const int src = 4 * (rho & 7) + n / 2, q = (rho >= 8 ? 2 : 0) + (n & 1);
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; w++) v += part[w][src][q];
    const int row = 16 * h16 + rho;
    if (Y.Bd) {
      // the shared expert's LoRA down branch c Bd t_d
      const float *td = P.lt + ((tg + n) * 3 + 2) * P.r;
      float lo = 0.f;
      for (int q2 = 0; q2 < P.r; q2++) lo = fmaf(bf(Y.Bd[(size_t)row * P.r + q2]), td[q2], lo);
      v = fmaf(P.c, lo, v);
    }
    const size_t oi = ((size_t)l * P.hB + P.tok0 + n) * D + row;
    P.y[oi] = f2bf(v);
    if (P.yf) P.yf[oi] = v;
  }
}

// ---------------------------------------------------------------------------------------
// Host side: the bf16-rows work list of one step shape (tokens, first step or not).
// ---------------------------------------------------------------------------------------
struct PhShape {
  int L, E, k, r, H, B;
  bool head[64], lora[64];
};

inline std::vector<PhBlock> ph_blocks(const PhShape &Z, bool step0) {
  std::vector<PhBlock> out;
  for (int l = 0; l < Z.L; l++) {
    const bool pred = !step0 && l > 0 && Z.head[l - 1];
    if (pred) {
      const int n = std::min(Z.B * Z.k, Z.E);
      for (int b = 0; b < n; b += 16) out.push_back(PhBlock{l, PR_SEL, b, std::min(16, n - b)});
    } else {
      for (int b = 0; b < Z.E; b += 16) out.push_back(PhBlock{l, PR_ROUTER, b, std::min(16, Z.E - b)});
    }
    if (Z.head[l]) {
      for (int b = 0; b < Z.E; b += 16) out.push_back(PhBlock{l, PR_HEAD, b, std::min(16, Z.E - b)});
      for (int b = 0; b < Z.H; b += 16) out.push_back(PhBlock{l, PR_FC1, b, std::min(16, Z.H - b)});
    }
    if (Z.lora[l])
      for (int b = 0; b < 2 * Z.r; b += 16) out.push_back(PhBlock{l, PR_LORA, b, std::min(16, 2 * Z.r - b)});
  }
  return out;
}

}  // namespace e0

namespace e0 {
// The plans of the predicted layers from the previous step's predictions, for a step whose
// previous step did not run the phased kernels (which write them).  One warp per layer.
__global__ void __launch_bounds__(32) k_ph_plan_pred(PhParams P) {
  const int l = blockIdx.x;
  if (!ph_predicted(P, l)) return;
  ph_build_plan(P.pred_in + (size_t)l * P.maxT * P.k, P.k, P.B, P.k, P.E, P.plan_cur + (size_t)l * kPlanInts,
                P.slot_cur + (size_t)l * kPhMaxU * kPhMaxB, threadIdx.x);
}
}  // namespace e0
