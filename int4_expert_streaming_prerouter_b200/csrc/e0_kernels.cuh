// General-T kernels of the MoE block: RMSNorm, bf16 GEMV rows (router, prerouter head,
// LoRA A), warp top-k + gates, expert grouping, int4 gate/up + SwiGLU, int4 down +
// weighted combine.  Any T works here; the decode stack has its own persistent kernel
// and prefill its own tensor-core kernels.
//
// What each kernel computes is stated against the pages by title and section:
//   [G] "The Other Half of the Memory Wall" reading guide; [A] the ai.info article
//   "Edge0 serve un MoE da 35B a 20 token al secondo in 3 GiB".
#pragma once
#include "e0_device.cuh"

namespace e0 {

constexpr int kMaxE = 256;
constexpr int kMaxK = 8;
constexpr int kMaxR = 32;

// Where a layer's routed experts live: resident [E][blob] or the streaming pool, whose
// slot table maps expert id -> slot (or -1) and tags each slot with its expert id.
struct ExpertSrc {
  const uint8_t *resident;    // [E][blob] or nullptr
  long long stride;           // blob bytes
  const uint8_t *pool;        // [slots][blob] of this layer's slot set, or nullptr
  const int32_t *slot_of;     // [E] expert -> slot (pool mode)
  const int32_t *slot_tag;    // [slots] expert held by each slot (pool mode)
  int *err;

  __device__ __forceinline__ const uint8_t *base(int e) const {
    if (pool == nullptr) return resident + (long long)e * stride;
    const int s = slot_of[e];
    if (s < 0 || slot_tag[s] != e) {
      atomicOr(err, DERR_SLOT);
      return pool;  // read a valid slot; the result is flagged as wrong
    }
    return pool + (long long)s * stride;
  }
};

// ---------------------------------------------------------------------------------------
// RMSNorm ([G] "Ön Yönlendirici Başlık Mimarisi": the post-attention layer norm that the
// router, the head and the experts read).  x = bf16(h * gamma / sqrt(mean(h^2) + eps)),
// evaluated in double and rounded once, so that the bf16 decision is taken in the same
// precision as the float64 definition.  With `chain`, h is first replaced by
// bf16(h + chain) (the previous layer's fp32 output).  One block per token.
// ---------------------------------------------------------------------------------------
__global__ void k_norm(const uint16_t *__restrict__ h, const float *__restrict__ chain,
                       const uint16_t *__restrict__ gamma, int d, float eps,
                       uint16_t *__restrict__ xb, float *__restrict__ xf) {
  const int t = blockIdx.x;
  const uint16_t *hr = h + (size_t)t * d;
  const float *cr = chain ? chain + (size_t)t * d : nullptr;
  __shared__ double red[32];
  // the layer input (h, or bf16(h + chain)) of element i, in double
  auto in = [&](int i, uint32_t hb) {
    double v = (double)bf(hb);
    if (cr) v = (double)bf(d2bf(v + (double)cr[i]));
    return v;
  };
  // fast path: 8 consecutive elements per thread held in registers (one read of h, 16-byte
  // accesses); otherwise a strided pass per element
  const bool vec = d % 8 == 0 && d / 8 <= (int)blockDim.x;
  const int c8 = threadIdx.x;                   // this thread's 8-element chunk (fast path)
  double v8[8];
  double ss = 0.0;
  if (vec) {
    if (c8 < d / 8) {
      const uint4 w = *reinterpret_cast<const uint4 *>(hr + 8 * c8);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; j++) {
        v8[2 * j] = in(8 * c8 + 2 * j, ws[j] & 0xFFFFu);
        v8[2 * j + 1] = in(8 * c8 + 2 * j + 1, ws[j] >> 16);
      }
#pragma unroll
      for (int j = 0; j < 8; j++) ss += v8[j] * v8[j];
    }
  } else {
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      const double v = in(i, hr[i]);
      ss += v * v;
    }
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const double rinv = 1.0 / sqrt(red[0] / d + (double)eps);
  if (vec) {
    if (c8 < d / 8) {
      const uint4 gw = *reinterpret_cast<const uint4 *>(gamma + 8 * c8);
      const uint32_t gs[4] = {gw.x, gw.y, gw.z, gw.w};
      uint32_t ob[4];
      float of[8];
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const uint16_t b0 = d2bf(v8[2 * j] * (double)bf(gs[j] & 0xFFFFu) * rinv);
        const uint16_t b1 = d2bf(v8[2 * j + 1] * (double)bf(gs[j] >> 16) * rinv);
        ob[j] = (uint32_t)b0 | ((uint32_t)b1 << 16);
        of[2 * j] = bf(b0);
        of[2 * j + 1] = bf(b1);
      }
      *reinterpret_cast<uint4 *>(xb + (size_t)t * d + 8 * c8) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
      if (xf) {
        float4 *fo = reinterpret_cast<float4 *>(xf + (size_t)t * d + 8 * c8);
        fo[0] = make_float4(of[0], of[1], of[2], of[3]);
        fo[1] = make_float4(of[4], of[5], of[6], of[7]);
      }
    }
  } else {
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      const uint16_t b = d2bf(in(i, hr[i]) * (double)bf(gamma[i]) * rinv);
      xb[(size_t)t * d + i] = b;
      if (xf) xf[(size_t)t * d + i] = bf(b);
    }
  }
}

// ---------------------------------------------------------------------------------------
// bf16 GEMV rows: router logits (all E rows, or only the k routed rows of a token whose
// routing is given), prerouter-head rows ([G] head: the linear path l(x); one-hot columns
// are added in k_route) and the LoRA A rows of the shared expert (t_g = Ag x, t_u = Au x,
// [G] "Birleştirilmemiş Adaptör Yürütme").  One warp per (row, tile of 8 tokens); fp32
// accumulation; results rounded to fp32 by the store.
// ---------------------------------------------------------------------------------------
struct RowsArgs {
  const float *xf;
  int T, d, E, k;
  const uint16_t *Wr;      // router [E, d]
  float *logits;           // [T, E]
  const int32_t *route;    // [T, k] or nullptr
  int full_mode;           // 0: every token routed by `route`; 1: all own router; 2: per token
  const uint16_t *Wh;      // head linear [E, ldh] or nullptr
  int ldh;
  float *hlog;             // [T, E]
  int hacc;                // 1: add the head rows to hlog instead of overwriting it
  const uint16_t *Ag, *Au; // [r, d] or nullptr
  int r;
  float *lt;               // [T, 3, r]
  int *err;
};

constexpr int kRowTile = 8;

__device__ __forceinline__ void bf16_row_dot(const uint16_t *__restrict__ w, const float *__restrict__ xf,
                                             int d, int t0, int nt, int lane, float *acc) {
  for (int c = lane; c < d / 8; c += 32) {
    const uint4 wv = __ldg(reinterpret_cast<const uint4 *>(w + c * 8));
    const float wf[8] = {bf(wv.x & 0xFFFFu), bf(wv.x >> 16), bf(wv.y & 0xFFFFu), bf(wv.y >> 16),
                         bf(wv.z & 0xFFFFu), bf(wv.z >> 16), bf(wv.w & 0xFFFFu), bf(wv.w >> 16)};
#pragma unroll
    for (int tt = 0; tt < kRowTile; tt++) {
      if (tt < nt) {
        const float4 *xp = reinterpret_cast<const float4 *>(xf + (size_t)(t0 + tt) * d + c * 8);
        const float4 a = __ldg(xp), b = __ldg(xp + 1);
        acc[tt] = fmaf(wf[0], a.x, fmaf(wf[1], a.y, fmaf(wf[2], a.z, fmaf(wf[3], a.w, acc[tt]))));
        acc[tt] = fmaf(wf[4], b.x, fmaf(wf[5], b.y, fmaf(wf[6], b.z, fmaf(wf[7], b.w, acc[tt]))));
      }
    }
  }
#pragma unroll
  for (int tt = 0; tt < kRowTile; tt++) acc[tt] = warp_sum(acc[tt]);
}

__device__ __forceinline__ bool needs_full(const RowsArgs &A, int t) {
  if (A.full_mode == 1 || A.route == nullptr) return true;
  if (A.full_mode == 0) return false;
  return A.route[(size_t)t * A.k] < 0;
}

__global__ void k_rows(RowsArgs A) {
  const int lane = threadIdx.x & 31;
  const int nTT = (A.T + kRowTile - 1) / kRowTile;
  const int J_full = (A.Wr && (A.full_mode != 0 || A.route == nullptr)) ? A.E * nTT : 0;
  const int J_sel = (A.Wr && A.route != nullptr && A.full_mode != 1) ? A.T * A.k : 0;
  const int J_head = A.Wh ? A.E * nTT : 0;
  const int J_lora = A.Ag ? 2 * A.r * nTT : 0;
  const int J = J_full + J_sel + J_head + J_lora;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); j < J; j += warps) {
    float acc[kRowTile];
#pragma unroll
    for (int i = 0; i < kRowTile; i++) acc[i] = 0.f;
    if (j < J_full) {
      const int row = j / nTT, t0 = (j % nTT) * kRowTile, nt = min(kRowTile, A.T - t0);
      bf16_row_dot(A.Wr + (size_t)row * A.d, A.xf, A.d, t0, nt, lane, acc);
      if (lane == 0)
        for (int tt = 0; tt < nt; tt++)
          if (needs_full(A, t0 + tt)) A.logits[(size_t)(t0 + tt) * A.E + row] = acc[tt];
    } else if (j < J_full + J_sel) {
      const int q = j - J_full, t = q / A.k;
      if (needs_full(A, t)) continue;
      const int row = A.route[q];
      if (row < 0 || row >= A.E) {
        if (lane == 0) atomicOr(A.err, DERR_INDEX);
        continue;
      }
      bf16_row_dot(A.Wr + (size_t)row * A.d, A.xf, A.d, t, 1, lane, acc);
      if (lane == 0) A.logits[(size_t)t * A.E + row] = acc[0];
    } else if (j < J_full + J_sel + J_head) {
      const int q = j - J_full - J_sel;
      const int row = q / nTT, t0 = (q % nTT) * kRowTile, nt = min(kRowTile, A.T - t0);
      bf16_row_dot(A.Wh + (size_t)row * A.ldh, A.xf, A.d, t0, nt, lane, acc);
      if (lane == 0)
        for (int tt = 0; tt < nt; tt++) {
          float *o = A.hlog + (size_t)(t0 + tt) * A.E + row;
          *o = A.hacc ? *o + acc[tt] : acc[tt];
        }
    } else {
      const int q = j - J_full - J_sel - J_head;
      const int row = q / nTT, t0 = (q % nTT) * kRowTile, nt = min(kRowTile, A.T - t0);
      const int which = row / A.r, rr = row % A.r;
      bf16_row_dot((which ? A.Au : A.Ag) + (size_t)rr * A.d, A.xf, A.d, t0, nt, lane, acc);
      if (lane == 0)
        for (int tt = 0; tt < nt; tt++) A.lt[((size_t)(t0 + tt) * 3 + which) * A.r + rr] = acc[tt];
    }
  }
}

// ---------------------------------------------------------------------------------------
// Warp top-k over E <= 256 fp32 values: descending value, equal values by lower index.
// Every lane returns the same k indices.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void warp_topk(const float *v, int E, int k, int lane, int *out) {
  float vals[kMaxE / 32];
#pragma unroll
  for (int i = 0; i < kMaxE / 32; i++) {
    const int e = lane + 32 * i;
    vals[i] = e < E ? v[e] : -INFINITY;
  }
  unsigned taken = 0;
  for (int s = 0; s < k; s++) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kMaxE / 32; i++) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (vals[i] > bv || (vals[i] == bv && e < be))) {
        bv = vals[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    out[s] = be;
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
  }
}

// ---------------------------------------------------------------------------------------
// Routing: own-router top-k or the given routing ("prediction as routing", [G] "Temel
// fikirler"), gate weights = softmax of the router logits renormalised over the
// selection, and (when the layer has a head) the head's top-k: the routing of the next
// layer at the next token ([G] "Ön Yönlendirici Başlık Mimarisi").  One warp per token.
// ---------------------------------------------------------------------------------------
struct RouteArgs {
  const float *logits;
  int T, E, k;
  const int32_t *route;
  int full_mode;
  int32_t *idx;            // [T, k]
  float *gates;            // [T, k]
  int32_t *hist;           // [T, k] copy of idx kept for the next step's one-hot, or nullptr
  const float *hlog;       // [T, E] or nullptr
  const uint16_t *Wh;      // head linear [E, ldh] (one-hot columns at d.. and d+E..)
  int ldh, d, onehot;
  const int32_t *prev;     // [T, k] routing of this layer at the previous token, or nullptr
  int32_t *pred;           // [T, k]
  float *hz_out;           // [T, E] final head logits, or nullptr
  const int32_t *cur;      // head-only mode (logits == nullptr): this token's routing, or nullptr
  int *err;
};

__global__ void k_route(RouteArgs A) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= A.T) return;
  int sel[kMaxK];
  if (A.logits == nullptr) {
    // head-only mode: the one-hot "current routing" comes from `cur` (all -1 when absent)
    for (int j = 0; j < A.k; j++) sel[j] = A.cur ? A.cur[(size_t)t * A.k + j] : -1;
  } else {
  const float *lg = A.logits + (size_t)t * A.E;
  bool full = A.full_mode == 1 || A.route == nullptr || (A.full_mode == 2 && A.route[(size_t)t * A.k] < 0);
  if (full) {
    warp_topk(lg, A.E, A.k, lane, sel);
  } else {
    for (int j = 0; j < A.k; j++) {
      int e = A.route[(size_t)t * A.k + j];
      if (e < 0 || e >= A.E) {
        if (lane == 0) atomicOr(A.err, DERR_INDEX);
        e = 0;
      }
      sel[j] = e;
    }
    for (int j = 0; j < A.k; j++)
      for (int q = j + 1; q < A.k; q++)
        if (sel[j] == sel[q] && lane == 0) atomicOr(A.err, DERR_DUP);
  }
  float mx = -INFINITY;
  for (int j = 0; j < A.k; j++) mx = fmaxf(mx, lg[sel[j]]);
  float ex[kMaxK], sum = 0.f;
  for (int j = 0; j < A.k; j++) {
    ex[j] = expf(lg[sel[j]] - mx);
    sum += ex[j];
  }
  if (lane < A.k) {
    float mine = 0.f;
    int mysel = 0;
    for (int j = 0; j < A.k; j++)
      if (j == lane) {
        mine = ex[j];
        mysel = sel[j];
      }
    A.idx[(size_t)t * A.k + lane] = mysel;
    A.gates[(size_t)t * A.k + lane] = mine / sum;
    if (A.hist) A.hist[(size_t)t * A.k + lane] = mysel;
  }
  }
  if (A.hlog == nullptr) return;
  // head logits (+ one-hot columns of this token's routing and the previous token's)
  float z[kMaxE / 32];
  for (int i = 0; i < kMaxE / 32; i++) {
    const int e = lane + 32 * i;
    if (e >= A.E) {
      z[i] = -INFINITY;
      continue;
    }
    float v = A.hlog[(size_t)t * A.E + e];
    if (A.onehot) {
      const uint16_t *wr = A.Wh + (size_t)e * A.ldh + A.d;
      for (int j = 0; j < A.k; j++)
        if (sel[j] >= 0 && sel[j] < A.E) v += bf(wr[sel[j]]);
      if (A.prev)
        for (int j = 0; j < A.k; j++) {
          const int p = A.prev[(size_t)t * A.k + j];
          if (p >= 0 && p < A.E) v += bf(wr[A.E + p]);
        }
    }
    z[i] = v;
    if (A.hz_out) A.hz_out[(size_t)t * A.E + e] = v;
  }
  __shared__ float zs[8][kMaxE];
  float *zw = zs[(threadIdx.x >> 5) & 7];
  for (int i = 0; i < kMaxE / 32; i++) {
    const int e = lane + 32 * i;
    if (e < A.E) zw[e] = z[i];
  }
  __syncwarp();
  int p[kMaxK];
  warp_topk(zw, A.E, A.k, lane, p);
  if (lane < A.k) {
    int mine = 0;
    for (int j = 0; j < A.k; j++)
      if (j == lane) mine = p[j];
    A.pred[(size_t)t * A.k + lane] = mine;
  }
}

// ---------------------------------------------------------------------------------------
// Group the T*k (token, slot) assignments by expert: unique experts in increasing id,
// their start offsets, and each expert's assignments in (token, slot) order.  One block.
// ---------------------------------------------------------------------------------------
struct Plan {
  int32_t *U;       // [1]
  int32_t *uexp;    // [E]
  int32_t *ustart;  // [E + 1]
  int32_t *assign;  // [T * k]  entries t * k + j
  int32_t *pos;     // [T * k]  grouped position of entry t * k + j (-1: invalid expert), or nullptr
};

// Counting sort by expert, stable in (token, slot) order: each of the 32 warps owns a
// contiguous chunk of the assignments; per-warp histograms give every (warp, expert) its
// output offset, and inside a batch of 32 the lanes holding the same expert rank
// themselves with a match mask.  One block of 1024 threads.
__global__ void __launch_bounds__(1024) k_plan(const int32_t *__restrict__ idx, int n, int E, Plan P) {
  __shared__ int cnt[32][kMaxE];      // per-warp counts, then per-warp output offsets
  __shared__ int tot[kMaxE];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 32 * kMaxE; i += blockDim.x) (&cnt[0][0])[i] = 0;
  __syncthreads();
  const int chunk = (n + 31) / 32, a0 = warp * chunk, a1 = min(n, a0 + chunk);
  for (int a = a0 + lane; a < a1; a += 32) {
    const int e = idx[a];
    if (e >= 0 && e < E) atomicAdd(&cnt[warp][e], 1);
  }
  __syncthreads();
  // expert totals, then the exclusive scan over experts (one warp)
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int t = 0;
    for (int w = 0; w < 32; w++) t += cnt[w][e];
    tot[e] = t;
  }
  __syncthreads();
  if (warp == 0) {
    int run = 0, u = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int c = e < E ? tot[e] : 0;
      int incl = c;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned nz = __ballot_sync(0xffffffffu, c > 0);
      if (c > 0) {
        const int ui = u + __popc(nz & ((1u << lane) - 1u));
        P.uexp[ui] = e;
        P.ustart[ui] = run + incl - c;
      }
      if (e < E) tot[e] = run + incl - c;    // expert start
      run += __shfl_sync(0xffffffffu, incl, 31);
      u += __popc(nz);
    }
    if (lane == 0) {
      P.ustart[u] = run;
      P.U[0] = u;
    }
  }
  __syncthreads();
  // per-(warp, expert) offsets: expert start + the counts of the earlier warps
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int off = tot[e];
    for (int w = 0; w < 32; w++) {
      const int c = cnt[w][e];
      cnt[w][e] = off;
      off += c;
    }
  }
  __syncthreads();
  for (int base = a0; base < a1; base += 32) {
    const int a = base + lane;
    const int e = a < a1 ? idx[a] : -1;
    const bool ok = e >= 0 && e < E;
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
    if (ok) {
      const int rank = __popc(peers & ((1u << lane) - 1u));
      P.assign[cnt[warp][e] + rank] = a;
      if (P.pos) P.pos[a] = cnt[warp][e] + rank;
    } else if (P.pos && a < a1) {
      P.pos[a] = -1;
    }
    __syncwarp();
    // the lowest lane of each peer group advances its expert's offset
    if (ok && (peers & ((1u << lane) - 1u)) == 0) cnt[warp][e] += __popc(peers);
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------------------
// Expert gate/up + SwiGLU ([A]: experts with int4 affine g64 weights; activation SwiGLU):
//   g = Dq(Wg) x, u = Dq(Wu) x, a = bf16(silu(g) * u).
// The shared expert (item u == U) adds its unmerged LoRA before the activation:
//   g += c Bg t_g, u += c Bu t_u  ([G] "Birleştirilmemiş Adaptör Yürütme").
// One warp per (expert, intermediate row); the row's int4 codes are loaded once and
// reused for every token routed to that expert.
// ---------------------------------------------------------------------------------------
struct GateUpArgs {
  const float *xf;
  int T, d, I, k, r;
  float c;
  ExpertSrc src;
  const uint8_t *shared;
  Blob bl;
  Plan P;
  const uint16_t *Bg, *Bu;  // [I, r] or nullptr
  const float *lt;          // [T, 3, r]
  uint16_t *a;              // [T, k+1, I]
};

constexpr int kMaxCPL = 4;   // 16-byte code chunks per lane: d <= 4096

__global__ void k_gateup(GateUpArgs A) {
  const int lane = threadIdx.x & 31;
  const int U = A.P.U[0];
  const int items = (U + 1) * A.I;
  const int nch = A.d / 32;          // 16-byte chunks per row
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int it = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); it < items; it += warps) {
    const int u = it / A.I, i = it % A.I;
    const bool sh = (u == U);
    const uint8_t *base = sh ? A.shared : A.src.base(A.P.uexp[u]);
    const uint8_t *gc = base + A.bl.gc + (size_t)i * (A.d / 2);
    const uint8_t *uc = base + A.bl.uc + (size_t)i * (A.d / 2);
    const uint16_t *gs = reinterpret_cast<const uint16_t *>(base + A.bl.gs) + (size_t)i * (A.d / 64);
    const uint16_t *gm = reinterpret_cast<const uint16_t *>(base + A.bl.gm) + (size_t)i * (A.d / 64);
    const uint16_t *us = reinterpret_cast<const uint16_t *>(base + A.bl.us) + (size_t)i * (A.d / 64);
    const uint16_t *um = reinterpret_cast<const uint16_t *>(base + A.bl.um) + (size_t)i * (A.d / 64);
    uint4 gw[kMaxCPL], uw[kMaxCPL];
    float gsv[kMaxCPL], gmv[kMaxCPL], usv[kMaxCPL], umv[kMaxCPL];
#pragma unroll
    for (int q = 0; q < kMaxCPL; q++) {
      const int ch = lane + 32 * q;
      if (ch < nch) {
        gw[q] = __ldg(reinterpret_cast<const uint4 *>(gc + ch * 16));
        uw[q] = __ldg(reinterpret_cast<const uint4 *>(uc + ch * 16));
        gsv[q] = bf(gs[ch >> 1]);
        gmv[q] = bf(gm[ch >> 1]);
        usv[q] = bf(us[ch >> 1]);
        umv[q] = bf(um[ch >> 1]);
      }
    }
    const int n_tok = sh ? A.T : A.P.ustart[u + 1] - A.P.ustart[u];
    for (int q2 = 0; q2 < n_tok; q2++) {
      int t, slot;
      if (sh) {
        t = q2;
        slot = A.k;
      } else {
        const int asg = A.P.assign[A.P.ustart[u] + q2];
        t = asg / A.k;
        slot = asg % A.k;
      }
      const float *x = A.xf + (size_t)t * A.d;
      float g = 0.f, v = 0.f;
#pragma unroll
      for (int q = 0; q < kMaxCPL; q++) {
        const int ch = lane + 32 * q;
        if (ch < nch) {
          g += chunk_dot(gw[q], x + ch * 32, gsv[q], gmv[q]);
          v += chunk_dot(uw[q], x + ch * 32, usv[q], umv[q]);
        }
      }
      g = warp_sum(g);
      v = warp_sum(v);
      if (sh && A.Bg != nullptr) {
        const float *tg = A.lt + (size_t)t * 3 * A.r;
        float lg = 0.f, lu = 0.f;
        if (lane < A.r) {
          lg = bf(A.Bg[(size_t)i * A.r + lane]) * tg[lane];
          lu = bf(A.Bu[(size_t)i * A.r + lane]) * tg[A.r + lane];
        }
        g = fmaf(A.c, warp_sum(lg), g);
        v = fmaf(A.c, warp_sum(lu), v);
      }
      if (lane == 0) {
        const float act = g / (1.0f + expf(-g)) * v;
        A.a[((size_t)t * (A.k + 1) + slot) * A.I + i] = f2bf(act);
      }
    }
  }
}

// t_d = Ad a_s for the shared expert's LoRA down branch.  One warp per (token, rank row).
__global__ void k_lora_t(const uint16_t *__restrict__ Ad, const uint16_t *__restrict__ a, int T,
                         int I, int k, int r, float *__restrict__ lt) {
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= T * r) return;
  const int t = w / r, j = w % r;
  const uint16_t *as = a + ((size_t)t * (k + 1) + k) * I;
  float acc = 0.f;
  for (int i = lane; i < I; i += 32) acc = fmaf(bf(Ad[(size_t)j * I + i]), bf(as[i]), acc);
  acc = warp_sum(acc);
  if (lane == 0) lt[((size_t)t * 3 + 2) * r + j] = acc;
}

// ---------------------------------------------------------------------------------------
// Expert down + weighted combine:  y = sum_j w_j Dq(Wd_{S_j}) a_j + Dq(Wd_s) a_s
//                                      + c Bd t_d   ([G] "Birleştirilmemiş Adaptör Yürütme")
// One warp per (token, output row); the (expert, chunk) terms are spread over the lanes
// in a fixed order, so the sum is reproducible run to run.
// ---------------------------------------------------------------------------------------
struct DownArgs {
  int T, d, I, k, r;
  float c;
  ExpertSrc src;
  const uint8_t *shared;
  Blob bl;
  const int32_t *idx;
  const float *gates;
  const uint16_t *a;
  const uint16_t *Bd;     // [d, r] or nullptr
  const float *lt;
  uint16_t *y;            // [T, d]
  float *yf;              // [T, d] or nullptr
};

__global__ void k_down(DownArgs A) {
  const int lane = threadIdx.x & 31;
  const int items = A.T * A.d;
  const int nch = A.I / 32;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int it = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); it < items; it += warps) {
    const int t = it / A.d, n = it % A.d;
    float acc = 0.f;
    for (int p = lane; p < (A.k + 1) * nch; p += 32) {
      const int j = p / nch, ch = p % nch;
      const uint8_t *base;
      float w;
      if (j < A.k) {
        base = A.src.base(A.idx[(size_t)t * A.k + j]);
        w = A.gates[(size_t)t * A.k + j];
      } else {
        base = A.shared;
        w = 1.0f;
      }
      const uint4 cw = __ldg(reinterpret_cast<const uint4 *>(base + A.bl.dc + (size_t)n * (A.I / 2) + ch * 16));
      const uint16_t *ds = reinterpret_cast<const uint16_t *>(base + A.bl.ds) + (size_t)n * (A.I / 64);
      const uint16_t *dm = reinterpret_cast<const uint16_t *>(base + A.bl.dm) + (size_t)n * (A.I / 64);
      const uint32_t *ap = reinterpret_cast<const uint32_t *>(A.a + ((size_t)t * (A.k + 1) + j) * A.I + ch * 32);
      uint32_t xp[16];
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(ap) + q);
        xp[4 * q] = v.x; xp[4 * q + 1] = v.y; xp[4 * q + 2] = v.z; xp[4 * q + 3] = v.w;
      }
      acc = fmaf(w, chunk_dot_bf16x(cw, xp, bf(ds[ch >> 1]), bf(dm[ch >> 1])), acc);
    }
    acc = warp_sum(acc);
    if (A.Bd != nullptr) {
      float l = 0.f;
      if (lane < A.r) l = bf(A.Bd[(size_t)n * A.r + lane]) * A.lt[((size_t)t * 3 + 2) * A.r + lane];
      acc = fmaf(A.c, warp_sum(l), acc);
    }
    if (lane == 0) {
      A.y[(size_t)t * A.d + n] = f2bf(acc);
      if (A.yf) A.yf[(size_t)t * A.d + n] = acc;
    }
  }
}

// ---------------------------------------------------------------------------------------
// Generic bf16 matrix rows on fp32 inputs: out[t][row] = W[row, 0:K] . X[t, 0:K] (+ bias).
// Used by the full prerouter head: fc1 on x and fc2 on the hidden layer.
// ---------------------------------------------------------------------------------------
struct MatRowsArgs {
  const uint16_t *W;
  int ldw, rows, K;
  const float *X;
  int ldx, T;
  const uint16_t *bias;   // [rows] bf16 or nullptr
  float *out;
  int ldo;
};

__global__ void k_mat_rows(MatRowsArgs A) {
  const int lane = threadIdx.x & 31;
  const int nTT = (A.T + kRowTile - 1) / kRowTile;
  const int J = A.rows * nTT;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); j < J; j += warps) {
    const int row = j / nTT, t0 = (j % nTT) * kRowTile, nt = min(kRowTile, A.T - t0);
    float acc[kRowTile];
#pragma unroll
    for (int i = 0; i < kRowTile; i++) acc[i] = 0.f;
    const uint16_t *w = A.W + (size_t)row * A.ldw;
    for (int c = lane; c < A.K / 8; c += 32) {
      const uint4 wv = __ldg(reinterpret_cast<const uint4 *>(w + c * 8));
      const float wf[8] = {bf(wv.x & 0xFFFFu), bf(wv.x >> 16), bf(wv.y & 0xFFFFu), bf(wv.y >> 16),
                           bf(wv.z & 0xFFFFu), bf(wv.z >> 16), bf(wv.w & 0xFFFFu), bf(wv.w >> 16)};
#pragma unroll
      for (int tt = 0; tt < kRowTile; tt++)
        if (tt < nt) {
          const float *xp = A.X + (size_t)(t0 + tt) * A.ldx + c * 8;
#pragma unroll
          for (int q = 0; q < 8; q++) acc[tt] = fmaf(wf[q], xp[q], acc[tt]);
        }
    }
#pragma unroll
    for (int tt = 0; tt < kRowTile; tt++) acc[tt] = warp_sum(acc[tt]);
    if (lane == 0)
      for (int tt = 0; tt < nt; tt++)
        A.out[(size_t)(t0 + tt) * A.ldo + row] = acc[tt] + (A.bias ? bf(A.bias[row]) : 0.f);
  }
}

// Hidden layer of the full head: h1 = gelu_erf(fc1 u + b1), u = [x; onehot(cur); onehot(prev)].
// `pre` holds fc1[:, :d] x; the one-hot columns are gathered here.  One thread per (t, j).
__global__ void k_head_hidden(const float *__restrict__ pre, const uint16_t *__restrict__ fc1,
                              const uint16_t *__restrict__ b1, int T, int H, int ld1, int d, int E,
                              int k, int onehot, const int32_t *__restrict__ cur,
                              const int32_t *__restrict__ prev, float *__restrict__ h1) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * H) return;
  const int t = i / H, j = i % H;
  float v = pre[i] + bf(b1[j]);
  if (onehot) {
    const uint16_t *w = fc1 + (size_t)j * ld1 + d;
    for (int q = 0; q < k; q++) {
      const int c = cur ? cur[(size_t)t * k + q] : -1;
      if (c >= 0 && c < E) v += bf(w[c]);
      const int p = prev ? prev[(size_t)t * k + q] : -1;
      if (p >= 0 && p < E) v += bf(w[E + p]);
    }
  }
  h1[i] = 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

constexpr int kMaxSlots = 256;
struct SlotList {
  int n;
  int e[kMaxSlots];
};

}  // namespace e0
