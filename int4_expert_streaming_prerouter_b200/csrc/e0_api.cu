// C ABI of libe0moe.so: context, weight registration, argument checks, launches of the
// MoE-block kernels, the decode loop with prediction-as-routing, and the streaming tier
// (pinned host store -> HBM slot pool on a side stream).  Declarations and the meaning
// of every argument are in include/e0moe.h.
#include "e0moe.h"
#include "e0_kernels.cuh"
#include "e0_decode.cuh"
#include "e0_phased.cuh"
#include "e0_prefill.cuh"

#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

using namespace e0;

static thread_local std::string g_err;

static int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define CK(call)                                                                         \
  do {                                                                                   \
    cudaError_t e_ = (call);                                                             \
    if (e_ != cudaSuccess) return fail(E0_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

#define CKL(what)                                                                        \
  do {                                                                                   \
    C->stats.kernel_launches++;                                                          \
    cudaError_t e_ = cudaGetLastError();                                                 \
    if (e_ != cudaSuccess) return fail(E0_ERR_CUDA, "launch %s: %s", what, cudaGetErrorString(e_)); \
  } while (0)

// ---------------------------------------------------------------------------------------
// Context
// ---------------------------------------------------------------------------------------
struct StreamPool {
  uint8_t *mem = nullptr;            // [pool_layers][slots][blob]
  int nsets = 0, slots = 0;
  size_t bytes = 0;
  const uint8_t *host = nullptr;     // pinned [L][E][blob]
  int32_t *slot_of = nullptr;        // [nsets][E]
  int32_t *slot_tag = nullptr;       // [nsets][slots]
  cudaStream_t side = nullptr;
  std::vector<cudaEvent_t> ready, freed;   // per pool set
  // event quadruples (copy start/end on the side stream, wait start/end on the compute
  // stream), one per staging round, reused round-robin and accounted on reuse
  struct Rec { cudaEvent_t c0, c1, w0, w1; int state; };
  std::vector<Rec> ring;
  int ring_pos = 0;
  std::vector<int> set_rec;                // per pool set: ring entry of its current round
  int fail_after = -1;                     // host-side fault injection for tests
  int corrupt_set = -1, corrupt_slot = 0, corrupt_tag = 0;  // one-shot wrong slot tag
  // persistent sets (one per layer, kept across steps): the host mirror of every slot's
  // expert (-1: empty) and the staging round that last needed it, for the sticky-slot /
  // least-recently-used replacement
  bool persist = false;
  std::vector<int> tag_h;
  std::vector<long long> use_h;
  long long round = 0;
  int reactive = 0;                        // 1: every layer routes itself and stages on demand
  int32_t *log = nullptr;                  // debug: [L][slots] slot tags each layer computed with
};

// Persistent decode kernel state: device copy of the layer table, tagged exchange buffers
// and the launch epoch (tags are unique per launch and layer).
struct DecodeState {
  bool ready = false;
  DecLayer *d_layers = nullptr;
  unsigned long long *tbuf = nullptr;   // one allocation for every tagged buffer
  unsigned long long *t_y = nullptr, *t_blk = nullptr, *t_rlog = nullptr, *t_hlog = nullptr;
  int blk = 0;
  uint32_t epoch = 0;
  int G = 0;
  size_t smem = 0;
  int stall_cta = -1;
  int flat = 1;                          // unchained steps: the flat schedule
  unsigned long long timeout_ns = 2000000000ull;
  unsigned long long *trace = nullptr;   // profiling timeline (caller-owned), or nullptr
  // item lists of the four schedules (flat or in order) x (first step or not):
  // [4][G][kMaxItems] items and [4][G] counts, schedule index 2 * flat + step0
  unsigned long long *sched = nullptr;
  int *sched_n = nullptr;
};

static void decode_free(DecodeState &S) {
  if (S.d_layers) cudaFree(S.d_layers);
  if (S.tbuf) cudaFree(S.tbuf);
  if (S.sched) cudaFree(S.sched);
  if (S.sched_n) cudaFree(S.sched_n);
  S = DecodeState{};
}

// Phased decode state: the device layer table, the workspace (token stride kPhMaxB) and
// the bf16-rows work lists, one per (batch, first step or not).
struct PhState {
  bool ready = false;
  PhLayer *d_layers = nullptr;
  void *mem = nullptr;                   // one allocation for the whole workspace
  uint16_t *x16 = nullptr, *xp = nullptr, *a = nullptr;
  float *xs = nullptr, *rlog = nullptr, *rsel = nullptr, *hlog = nullptr, *lt = nullptr, *h1 = nullptr,
        *gates = nullptr, *asum = nullptr, *gus = nullptr;
  // expert plans by (step parity, group of kPhMaxB streams, layer)
  int *plan = nullptr;                   // [2][kPhGroups][L][kPlanInts]
  int8_t *slot = nullptr;                // [2][kPhGroups][L][kPhMaxU][kPhMaxB]
  int last_step = -1;                    // the last step that ran the phased kernels
  PhBlock *blocks[2 * (kPhMaxB + 1)] = {};
  int nblocks[2 * (kPhMaxB + 1)] = {};
  // profiling: kernels launched one after another with an event before each and after the
  // last (7 per step), accounted by e0_debug_phase_times
  bool timing = false;
  std::vector<std::vector<cudaEvent_t>> pending;
  double ms[6] = {};
  unsigned long long steps_timed = 0;
};

static void phased_free(PhState &S) {
  for (auto &v : S.pending)
    for (auto e : v) cudaEventDestroy(e);
  if (S.d_layers) cudaFree(S.d_layers);
  if (S.mem) cudaFree(S.mem);
  for (auto *b : S.blocks)
    if (b) cudaFree(b);
  S = PhState{};
}

// One captured decode step (the per-layer kernel sequence of every layer) and its key.
struct DecodeGraph {
  cudaGraphExec_t exec = nullptr;
  int B = 0, parity = -1, step0 = -1, chained = -1, has_f32 = -1;
  unsigned long long launches = 0;
};

struct e0_ctx {
  e0_dims dims{};
  int L = 0, maxT = 0, dev = 0, nsm = 0;
  Blob bl{};
  std::vector<e0_layer> layers;
  std::vector<e0_head> heads;
  bool registered = false;
  // workspaces (device)
  uint16_t *xb = nullptr;
  float *xf = nullptr, *logits = nullptr, *hlog = nullptr, *lt = nullptr, *gates = nullptr;
  int32_t *idx = nullptr;
  uint16_t *a = nullptr;
  int32_t *plan_mem = nullptr;
  Plan plan{};
  float *yscratch = nullptr;         // [2][maxT][d] fp32 outputs for chained decode
  float *h1pre = nullptr, *h1 = nullptr;  // [maxT][H] full-head hidden layer
  int32_t *pred_tab = nullptr;       // [2][L+1][maxT][k]  routing predicted for layer l
  int32_t *hist_tab = nullptr;       // [2][L][maxT][k]    routing used by layer l
  int *err = nullptr;
  int32_t *host_idx = nullptr;       // pinned scratch for routing read-backs
  cudaStream_t last = nullptr;
  int last_step = -1, last_B = 0;
  bool force_general = false;        // route decode through the general per-layer kernels
  int prefill_path = 0;              // 0: tensor cores from kTcMinTokens tokens, 1: CUDA cores, 2: tensor cores
  int decode_mode = 0;               // 0 auto, 1 one-launch kernel, 2 graph of per-layer kernels, 3 eager
  DecodeGraph graphs[6];
  int graph_next = 0;
  cudaStream_t cap = nullptr;        // private stream the decode graphs are captured on
  uint16_t *g_h = nullptr, *g_y = nullptr;   // [L][maxT][d] graph input / output
  float *g_yf = nullptr;                     // [L][maxT][d]
  // tensor-core prefill workspaces: K-permuted bf16 operands and their group-of-64 sums
  uint16_t *xp = nullptr, *ap = nullptr, *xg = nullptr;
  float *xsum = nullptr, *asum = nullptr;
  float *yacc = nullptr;
  float *ypart = nullptr;            // fixed-order prefill combine: [k + 1][maxT][d] (on request)
  bool pf_det = false;
  TcTile *tiles = nullptr;
  int *ntiles = nullptr;
  int tile_cap = 0;
  int32_t *pf_buf = nullptr;         // prefill: [2][maxT+1][k] head predictions, row 0 = -1
  int32_t *pf_idx = nullptr;         // prefill: [maxT+1][k] routing scratch, row 0 = -1
  DecodeState dec{};
  PhState ph{};
  StreamPool pool;
  e0_stats stats{};
  bool time_gemm = false;                          // profiling: event pairs around the GEMMs
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> gemm_ev;
  // decode steps and prefill chunks with host buffers (e0_moe_stack_decode_host,
  // e0_moe_prefill_stack_host): one copy stream for inputs and one for outputs (so that an
  // input copy never queues behind the previous output copy, which waits for its kernels),
  // and two alternating device staging buffers each, ordered with the compute by events
  struct HostIO {
    cudaStream_t cs = nullptr, ds = nullptr;   // host -> device, device -> host
    cudaEvent_t in[2] = {}, out[2] = {}, done[2] = {}, tail = nullptr, tail2 = nullptr;
    uint16_t *h[2] = {}, *y[2] = {};
    float *yf[2] = {};
    bool used[2] = {};
    long long calls = 0;
    // prefill chunks: per-layer staging (maxT x d each)
    cudaEvent_t pin[2] = {}, pout[2] = {}, pdone[2] = {};
    uint16_t *ph[2] = {}, *py[2] = {};
    float *pyf[2] = {};
    bool pused[2] = {};
  } io;
};

extern "C" const char *e0_last_error(void) { return g_err.c_str(); }

static bool supported(const e0_dims &D) {
  return D.d_model > 0 && D.d_model % 256 == 0 && D.d_model <= 4096 && D.d_ff > 0 &&
         D.d_ff % 128 == 0 && D.d_ff <= 4096 && D.top_k >= 1 && D.top_k <= kMaxK &&
         D.n_experts >= D.top_k && D.n_experts <= kMaxE && D.group == 64 && D.lora_rank >= 0 &&
         D.lora_rank <= kMaxR && D.head_hidden >= 0 && D.head_hidden % 8 == 0 && D.head_hidden <= 16384 &&
         (D.head_onehot == 0 || (D.head_onehot == 1 && D.n_experts % 4 == 0));
}

template <typename T>
static int dalloc(T **p, size_t n) {
  const cudaError_t e = cudaMalloc((void **)p, n * sizeof(T) + 16);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(e == cudaErrorMemoryAllocation ? E0_ERR_OOM : E0_ERR_CUDA, "cudaMalloc of %zu bytes failed: %s",
                n * sizeof(T), cudaGetErrorString(e));
  }
  return E0_OK;
}

extern "C" int e0_destroy(e0_ctx *C) {
  if (!C) return E0_OK;
  cudaDeviceSynchronize();
  for (auto &e : C->gemm_ev) {
    cudaEventDestroy(e.first);
    cudaEventDestroy(e.second);
  }
  void *bufs[] = {C->xb, C->xf, C->logits, C->hlog, C->lt, C->gates, C->idx, C->a, C->plan_mem,
                  C->yscratch, C->pred_tab, C->hist_tab, C->err, C->h1pre, C->h1, C->pool.mem, C->pool.slot_of,
                  C->pool.slot_tag, C->xp, C->ap, C->xg, C->xsum, C->asum, C->yacc, C->ypart, C->tiles, C->ntiles, C->pf_buf, C->pf_idx};
  for (void *b : bufs)
    if (b) cudaFree(b);
  decode_free(C->dec);
  phased_free(C->ph);
  for (auto &g : C->graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  if (C->cap) cudaStreamDestroy(C->cap);
  for (void *b : {(void *)C->g_h, (void *)C->g_y, (void *)C->g_yf})
    if (b) cudaFree(b);
  if (C->host_idx) cudaFreeHost(C->host_idx);
  for (auto *v : {&C->pool.ready, &C->pool.freed})
    for (auto e : *v) cudaEventDestroy(e);
  for (auto &r : C->pool.ring)
    for (auto e : {r.c0, r.c1, r.w0, r.w1}) cudaEventDestroy(e);
  if (C->pool.side) cudaStreamDestroy(C->pool.side);
  for (int b = 0; b < 2; b++) {
    for (cudaEvent_t e : {C->io.in[b], C->io.out[b], C->io.done[b], C->io.pin[b], C->io.pout[b], C->io.pdone[b]})
      if (e) cudaEventDestroy(e);
    for (void *m : {(void *)C->io.h[b], (void *)C->io.y[b], (void *)C->io.yf[b], (void *)C->io.ph[b],
                    (void *)C->io.py[b], (void *)C->io.pyf[b]})
      if (m) cudaFree(m);
  }
  for (cudaEvent_t e : {C->io.tail, C->io.tail2})
    if (e) cudaEventDestroy(e);
  for (cudaStream_t st : {C->io.cs, C->io.ds})
    if (st) cudaStreamDestroy(st);
  delete C;
  return E0_OK;
}

extern "C" int e0_create(const e0_dims *dims, int n_layers, int max_tokens, e0_ctx **out) {
  if (!dims || !out || n_layers < 1 || max_tokens < 1 || max_tokens > (1 << 16))
    return fail(E0_ERR_INVALID_ARG, "e0_create: bad arguments");
  if (!supported(*dims))
    return fail(E0_ERR_INVALID_ARG,
                "e0_create: unsupported dims (need d%%256==0, I%%128==0, k<=8, k<=E<=256, r<=32, group 64)");
  *out = nullptr;
  e0_ctx *C = new e0_ctx();
  C->dims = *dims;
  C->L = n_layers;
  C->maxT = max_tokens;
  cudaGetDevice(&C->dev);
  cudaDeviceGetAttribute(&C->nsm, cudaDevAttrMultiProcessorCount, C->dev);
  C->bl = blob_of(dims->d_model, dims->d_ff);
  const size_t T = max_tokens, d = dims->d_model, E = dims->n_experts, I = dims->d_ff,
               k = dims->top_k, r = dims->lora_rank > 0 ? dims->lora_rank : 1;
  int rc = E0_OK;
  if ((rc = dalloc(&C->xb, T * d)) || (rc = dalloc(&C->xf, T * d)) || (rc = dalloc(&C->logits, T * E)) ||
      (rc = dalloc(&C->hlog, T * E)) || (rc = dalloc(&C->lt, T * 3 * r)) || (rc = dalloc(&C->gates, T * k)) ||
      (rc = dalloc(&C->idx, T * k)) || (rc = dalloc(&C->a, T * (k + 1) * I)) ||
      (rc = dalloc(&C->plan_mem, 1 + E + E + 1 + 2 * T * k)) || (rc = dalloc(&C->yscratch, 2 * T * d)) ||
      (rc = dalloc(&C->pred_tab, 2 * (n_layers + 1) * T * k)) ||
      (rc = dalloc(&C->hist_tab, 2 * n_layers * T * k)) || (rc = dalloc(&C->err, 4)) ||
      (dims->head_hidden > 0 && ((rc = dalloc(&C->h1pre, T * dims->head_hidden)) ||
                                 (rc = dalloc(&C->h1, T * dims->head_hidden))))) {
    e0_destroy(C);
    return rc;
  }
  if ((rc = dalloc(&C->pf_buf, 2 * (T + 1) * k)) || (rc = dalloc(&C->pf_idx, (T + 1) * k))) {
    e0_destroy(C);
    return rc;
  }
  cudaMemset(C->pf_buf, 0xFF, 2 * (T + 1) * k * sizeof(int32_t));
  cudaMemset(C->pf_idx, 0xFF, (T + 1) * k * sizeof(int32_t));
  if (T >= kTcMinTokens) {
    C->tile_cap = (int)((T * k + kTmN - 1) / kTmN + std::min(E, T * k) + (T + kTmN - 1) / kTmN + 1);
    if ((rc = dalloc(&C->xp, T * d)) || (rc = dalloc(&C->ap, T * (k + 1) * I)) || (rc = dalloc(&C->xg, T * k * d)) ||
        (rc = dalloc(&C->xsum, T * (d / 64 + 1))) || (rc = dalloc(&C->asum, T * (k + 1) * (I / 64 + 1))) ||
        (rc = dalloc(&C->yacc, T * d)) ||
        (rc = dalloc(&C->tiles, (size_t)C->tile_cap)) || (rc = dalloc(&C->ntiles, 1))) {
      e0_destroy(C);
      return rc;
    }
    // the large dynamic shared memory of the tensor-core kernels is an attribute of the
    // function on the current device: opt in here, for this context's device, so that
    // contexts on several devices of one process each have it
    if (cudaFuncSetAttribute(k_tc_rows, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(TcRowsSmem) + 1024) != cudaSuccess ||
        cudaFuncSetAttribute(k_moe_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(TmSmem) + 1024) != cudaSuccess) {
      cudaGetLastError();
      e0_destroy(C);
      return fail(E0_ERR_CUDA, "e0_create: shared-memory opt-in of the tensor-core kernels failed");
    }
  }
  C->plan.U = C->plan_mem;
  C->plan.uexp = C->plan_mem + 1;
  C->plan.ustart = C->plan_mem + 1 + E;
  C->plan.assign = C->plan_mem + 2 + 2 * E;
  C->plan.pos = C->plan.assign + T * k;
  cudaMemset(C->pred_tab, 0xFF, 2 * (n_layers + 1) * T * k * sizeof(int32_t));
  cudaMemset(C->hist_tab, 0xFF, 2 * n_layers * T * k * sizeof(int32_t));
  cudaMemset(C->err, 0, 16);
  if (cudaMallocHost((void **)&C->host_idx, (n_layers + 2) * T * k * sizeof(int32_t)) != cudaSuccess) {
    e0_destroy(C);
    return fail(E0_ERR_OOM, "pinned scratch allocation failed");
  }
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    e0_destroy(C);
    return fail(E0_ERR_CUDA, "e0_create: %s", cudaGetErrorString(e));
  }
  *out = C;
  return E0_OK;
}

extern "C" int e0_register_model(e0_ctx *C, const e0_layer *layers, const e0_head *heads) {
  if (!C || !layers) return fail(E0_ERR_INVALID_ARG, "e0_register_model: NULL argument");
  for (int l = 0; l < C->L; l++) {
    const e0_layer &Y = layers[l];
    if (!Y.shared || !Y.router_w || !Y.norm_w)
      return fail(E0_ERR_INVALID_ARG, "layer %d: shared, router_w and norm_w are required", l);
    const bool any = Y.lora_Ag || Y.lora_Bg || Y.lora_Au || Y.lora_Bu || Y.lora_Ad || Y.lora_Bd;
    const bool all = Y.lora_Ag && Y.lora_Bg && Y.lora_Au && Y.lora_Bu && Y.lora_Ad && Y.lora_Bd;
    if (any && (!all || C->dims.lora_rank < 1))
      return fail(E0_ERR_INVALID_ARG, "layer %d: LoRA needs all six matrices and lora_rank >= 1", l);
    if (((uintptr_t)Y.shared | (uintptr_t)Y.experts | (uintptr_t)Y.router_w | (uintptr_t)Y.lora_Ag |
         (uintptr_t)Y.lora_Au) & 15)
      return fail(E0_ERR_INVALID_ARG, "layer %d: weight pointers must be 16-byte aligned", l);
    if (heads && heads[l].w_lin) {
      if (C->dims.head_hidden > 0 && !(heads[l].fc1_w && heads[l].fc1_b && heads[l].fc2_w && heads[l].fc2_b))
        return fail(E0_ERR_INVALID_ARG, "layer %d: head_hidden > 0 needs fc1/fc2 weights", l);
      if (((uintptr_t)heads[l].w_lin | (uintptr_t)heads[l].fc1_w | (uintptr_t)heads[l].fc2_w) & 15)
        return fail(E0_ERR_INVALID_ARG, "layer %d: head weights must be 16-byte aligned", l);
    }
  }
  C->layers.assign(layers, layers + C->L);
  C->heads.assign(C->L, e0_head{});
  if (heads) C->heads.assign(heads, heads + C->L);
  C->registered = true;
  C->dec.ready = false;
  C->ph.ready = false;
  for (auto &g : C->graphs) {   // captured pointers belong to the previous registration
    if (g.exec) cudaGraphExecDestroy(g.exec);
    g = DecodeGraph{};
  }
  return E0_OK;
}

// ---------------------------------------------------------------------------------------
// One layer, split in two halves so that the streaming tier can stage experts between
// the routing decision and the expert kernels.
// ---------------------------------------------------------------------------------------
struct LayerCall {
  int l, T;
  const uint16_t *h;
  const float *chain;
  const int32_t *route;
  int full_mode;
  int32_t *idx;            // [T,k] routing (written by k_route)
  float *gates;
  int32_t *hist;           // copy of idx for the next step's one-hot, or nullptr
  bool head;
  const int32_t *prev;     // [T,k] or nullptr
  int32_t *pred;           // [T,k]
  uint16_t *y;
  float *yf;
};

static inline int grid_for(int warps_needed, int cap) {
  int b = (warps_needed + 7) / 8;
  return b < 1 ? 1 : (b > cap ? cap : b);
}

// TMA descriptor of a row-major 16-bit matrix [rows, K] (bf16, or fp16 when f16) read in
// boxes of 64 columns x kTmN rows with the 128-byte swizzle of the tensor-core operand
// tiles (zeros past the end).
// The encoder comes from the driver through the runtime's entry-point query.
static int tmap_bf16_rows(CUtensorMap *m, const void *base, int K, long long rows, bool f16 = false) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return fail(E0_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
  }
  if (((uintptr_t)base & 15) || K % 64 || rows < 1)
    return fail(E0_ERR_INVALID_ARG, "tensor map: base, K or rows not supported");
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kTmN};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = encode(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                            const_cast<void *>(base), dims, strides, box, es,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(E0_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return E0_OK;
}

// TMA descriptor of the int4 codes of one projection of every expert: a 3-D byte tensor
// [count][rows][row_bytes] whose experts lie `stride` bytes apart, read in boxes of 128
// bytes x box_rows rows with the 128-byte swizzle (zeros past the end of a row).
static int tmap_codes(CUtensorMap *m, const void *base, int row_bytes, int rows, int count, long long stride,
                      int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return fail(E0_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
  }
  if (((uintptr_t)base & 15) || row_bytes % 16 || stride % 16 || rows < box_rows || count < 1)
    return fail(E0_ERR_INVALID_ARG, "code tensor map: base, row length, stride or rows not supported");
  const cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)rows, (cuuint64_t)count};
  const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)stride};
  const cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, es,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(E0_ERR_CUDA, "cuTensorMapEncodeTiled (codes) failed (%d)", (int)r);
  return E0_OK;
}

// The tensor-core kernels serve calls of at least kTcMinTokens tokens (or any size when
// selected), in contexts created with the workspaces for them.
static bool use_tc(e0_ctx *C, int T) {
  const e0_dims &D = C->dims;
  return C->xp && D.d_model % 128 == 0 && D.d_model <= 64 * kTmMaxG && D.d_ff % 128 == 0 &&
         (D.lora_rank <= kTmMaxR && D.lora_rank % 2 == 0) &&
         D.d_ff <= 64 * kTmMaxG && (C->prefill_path == 2 || (C->prefill_path == 0 && T >= kTcMinTokens));
}

static int layer_pre(e0_ctx *C, const LayerCall &K, cudaStream_t s) {
  const e0_dims &D = C->dims;
  const e0_layer &Y = C->layers[K.l];
  const e0_head &H = C->heads[K.l];
  k_norm<<<K.T, 256, 0, s>>>(K.h, K.chain, (const uint16_t *)Y.norm_w, D.d_model, D.rms_eps, C->xb, C->xf);
  CKL("k_norm");
  RowsArgs R{};
  R.xf = C->xf; R.T = K.T; R.d = D.d_model; R.E = D.n_experts; R.k = D.top_k;
  R.Wr = (const uint16_t *)Y.router_w; R.logits = C->logits; R.route = K.route; R.full_mode = K.full_mode;
  R.Wh = (K.head && H.w_lin) ? (const uint16_t *)H.w_lin : nullptr;
  R.ldh = D.d_model + (D.head_onehot ? 2 * D.n_experts : 0);
  R.hlog = C->hlog;
  R.Ag = (const uint16_t *)Y.lora_Ag; R.Au = (const uint16_t *)Y.lora_Au; R.r = D.lora_rank; R.lt = C->lt;
  R.err = C->err;
  if (use_tc(C, K.T)) {
    // every row on the tensor cores: full router logits for every token, head, LoRA A
    TcRowsArgs W{};
    W.x = C->xb; W.T = K.T; W.d = D.d_model; W.err = C->err; W.timeout_ns = 2000000000ull;
    W.seg[W.nseg++] = RowSeg{R.Wr, D.n_experts, D.d_model, C->logits, D.n_experts, 0};
    if (R.Wh) W.seg[W.nseg++] = RowSeg{R.Wh, D.n_experts, R.ldh, C->hlog, D.n_experts, 0};
    if (R.Ag) {
      W.seg[W.nseg++] = RowSeg{R.Ag, D.lora_rank, D.d_model, C->lt, 3 * D.lora_rank, 0};
      W.seg[W.nseg++] = RowSeg{R.Au, D.lora_rank, D.d_model, C->lt, 3 * D.lora_rank, D.lora_rank};
    }
    for (int q = 0; q < W.nseg; q++) W.total += W.seg[q].rows;
    const int smem = (int)sizeof(TcRowsSmem) + 1024;   // opted in at e0_create on this context's device
    k_tc_rows<<<dim3((W.total + 127) / 128, (K.T + kTcN - 1) / kTcN), kTcThreads, smem, s>>>(W);
    CKL("k_tc_rows");
  } else {
    const int nTT = (K.T + kRowTile - 1) / kRowTile;
    const int J = D.n_experts * nTT + K.T * D.top_k + (R.Wh ? D.n_experts * nTT : 0) + (R.Ag ? 2 * D.lora_rank * nTT : 0);
    k_rows<<<grid_for(J, 8 * C->nsm), 256, 0, s>>>(R);
    CKL("k_rows");
  }
  RouteArgs A{};
  A.logits = C->logits; A.T = K.T; A.E = D.n_experts; A.k = D.top_k; A.route = K.route; A.full_mode = K.full_mode;
  A.idx = K.idx; A.gates = K.gates; A.hist = K.hist;
  A.hlog = R.Wh ? C->hlog : nullptr; A.Wh = R.Wh; A.ldh = R.ldh; A.d = D.d_model; A.onehot = D.head_onehot;
  A.prev = K.prev; A.pred = K.pred; A.err = C->err;
  k_route<<<(K.T + 7) / 8, 256, 0, s>>>(A);
  CKL("k_route");
  return E0_OK;
}

// The experts of one layer on the tensor cores (grouped tcgen05 GEMMs); used for prefill.
static int layer_post_tc(e0_ctx *C, const LayerCall &K, const ExpertSrc &src, cudaStream_t s) {
  const e0_dims &D = C->dims;
  const e0_layer &Y = C->layers[K.l];
  const size_t nx = (size_t)K.T * D.d_model;
  const long long xg = (long long)K.T * (D.d_model / 64);
  // the permuted x rows, their group sums, and the routed tokens' rows in expert-grouped
  // order (each tile's tokens consecutive)
  k_perm_sums<<<(unsigned)((8 * xg + 255) / 256), 256, 0, s>>>(C->xb, K.T, D.d_model, C->xp, C->xsum, 0,
                                                          C->plan.pos, D.top_k, C->xg);
  CKL("k_perm_sums(x)");
  k_tc_tiles<<<1, 32, 0, s>>>(C->plan, K.T, C->tiles, C->ntiles, C->tile_cap);
  CKL("k_tc_tiles");
  TcArgs A{};
  int rc;
  if ((rc = tmap_bf16_rows(&A.tmB[0], C->xg, D.d_model, (long long)K.T * D.top_k, true)) ||
      (rc = tmap_bf16_rows(&A.tmB[1], C->xp, D.d_model, K.T, true)))
    return rc;
  A.mode = 0; A.T = K.T; A.d = D.d_model; A.I = D.d_ff; A.k = D.top_k; A.r = D.lora_rank; A.c = D.lora_scale;
  A.src = src; A.shared = (const uint8_t *)Y.shared; A.bl = C->bl; A.P = C->plan; A.tiles = C->tiles;
  A.ntiles = C->ntiles; A.xp = C->xp; A.xsum = C->xsum; A.ap = C->ap; A.asum = C->asum; A.ap_out = C->ap;
  A.Bg = (const uint16_t *)Y.lora_Bg; A.Bu = (const uint16_t *)Y.lora_Bu; A.lt = C->lt; A.gates = K.gates;
  A.yacc = C->yacc; A.err = C->err; A.timeout_ns = 2000000000ull;
  const int tc_smem_bytes = (int)sizeof(TmSmem) + 1024;   // opted in at e0_create on this context's device
  const int tmax = std::min(C->tile_cap, (K.T * D.top_k + kTmN - 1) / kTmN + std::min(D.n_experts, K.T * D.top_k) +
                                              (K.T + kTmN - 1) / kTmN);
  const uint8_t *ex = (const uint8_t *)src.resident, *sh = (const uint8_t *)Y.shared;
  const long long bb = C->bl.bytes;
  if ((rc = tmap_codes(&A.tmC[0], ex + C->bl.gc, D.d_model / 2, D.d_ff, D.n_experts, bb, 64)) ||
      (rc = tmap_codes(&A.tmC[1], ex + C->bl.uc, D.d_model / 2, D.d_ff, D.n_experts, bb, 64)) ||
      (rc = tmap_codes(&A.tmC[2], sh + C->bl.gc, D.d_model / 2, D.d_ff, 1, bb, 64)) ||
      (rc = tmap_codes(&A.tmC[3], sh + C->bl.uc, D.d_model / 2, D.d_ff, 1, bb, 64)))
    return rc;
  cudaEvent_t g0 = nullptr, g1 = nullptr;
  if (C->time_gemm && cudaEventCreate(&g0) == cudaSuccess && cudaEventCreate(&g1) == cudaSuccess)
    cudaEventRecord(g0, s);
  k_moe_gemm_tc<<<std::min(C->nsm, tmax * (D.d_ff / 64)), kTmThreads, tc_smem_bytes, s>>>(A);
  CKL("k_moe_gemm_tc(gate/up)");
  if (g1) {
    cudaEventRecord(g1, s);
    C->gemm_ev.push_back({g0, g1});
    g0 = g1 = nullptr;
  }
  const long long ag = (long long)K.T * (D.top_k + 1) * (D.d_ff / 64);
  k_perm_sums<<<(unsigned)((8 * ag + 255) / 256), 256, 0, s>>>(C->ap, (long long)K.T * (D.top_k + 1), D.d_ff, nullptr,
                                                          C->asum, 1, nullptr, 0, nullptr);
  CKL("k_perm_sums(a)");
  if (Y.lora_Ad) {
    k_lora_td<<<(K.T * D.lora_rank + 7) / 8, 256, 0, s>>>((const uint16_t *)Y.lora_Ad, C->ap, K.T, D.d_ff,
                                                           D.top_k, D.lora_rank, C->lt);
    CKL("k_lora_td");
  }
  if (!C->pf_det) CK(cudaMemsetAsync(C->yacc, 0, nx * sizeof(float), s));
  A.ypart = C->pf_det ? C->ypart : nullptr;   // every (slot, token, row) is written once
  A.mode = 1;
  if ((rc = tmap_bf16_rows(&A.tmB[0], C->ap, D.d_ff, (long long)K.T * (D.top_k + 1), true)) ||
      (rc = tmap_codes(&A.tmC[0], ex + C->bl.dc, D.d_ff / 2, D.d_model, D.n_experts, bb, 128)) ||
      (rc = tmap_codes(&A.tmC[2], sh + C->bl.dc, D.d_ff / 2, D.d_model, 1, bb, 128)))
    return rc;
  A.tmB[1] = A.tmB[0];
  A.tmC[1] = A.tmC[0];
  A.tmC[3] = A.tmC[2];
  if (C->time_gemm && cudaEventCreate(&g0) == cudaSuccess && cudaEventCreate(&g1) == cudaSuccess)
    cudaEventRecord(g0, s);
  k_moe_gemm_tc<<<std::min(C->nsm, tmax * (D.d_model / 128)), kTmThreads, tc_smem_bytes, s>>>(A);
  CKL("k_moe_gemm_tc(down)");
  if (g1) {
    cudaEventRecord(g1, s);
    C->gemm_ev.push_back({g0, g1});
  }
  k_tc_finish<<<K.T, 256, 0, s>>>(C->yacc, A.ypart, D.top_k + 1, (const uint16_t *)Y.lora_Bd, C->lt, K.T,
                                  D.d_model, D.lora_rank, D.lora_scale, K.y, K.yf);
  CKL("k_tc_finish");
  return E0_OK;
}

static int layer_post(e0_ctx *C, const LayerCall &K, const ExpertSrc &src, cudaStream_t s) {
  const e0_dims &D = C->dims;
  const e0_layer &Y = C->layers[K.l];
  k_plan<<<1, 1024, 0, s>>>(K.idx, K.T * D.top_k, D.n_experts, C->plan);
  CKL("k_plan");
  const bool tc = src.pool == nullptr && use_tc(C, K.T);
  if (tc) return layer_post_tc(C, K, src, s);
  GateUpArgs G{};
  G.xf = C->xf; G.T = K.T; G.d = D.d_model; G.I = D.d_ff; G.k = D.top_k; G.r = D.lora_rank; G.c = D.lora_scale;
  G.src = src; G.shared = (const uint8_t *)Y.shared; G.bl = C->bl; G.P = C->plan;
  G.Bg = (const uint16_t *)Y.lora_Bg; G.Bu = (const uint16_t *)Y.lora_Bu; G.lt = C->lt; G.a = C->a;
  const int items = (std::min(D.n_experts, K.T * D.top_k) + 1) * D.d_ff;
  k_gateup<<<grid_for(items, 4 * C->nsm), 256, 0, s>>>(G);
  CKL("k_gateup");
  if (Y.lora_Ad) {
    k_lora_t<<<(K.T * D.lora_rank + 7) / 8, 256, 0, s>>>((const uint16_t *)Y.lora_Ad, C->a, K.T, D.d_ff,
                                                          D.top_k, D.lora_rank, C->lt);
    CKL("k_lora_t");
  }
  DownArgs W{};
  W.T = K.T; W.d = D.d_model; W.I = D.d_ff; W.k = D.top_k; W.r = D.lora_rank; W.c = D.lora_scale;
  W.src = src; W.shared = (const uint8_t *)Y.shared; W.bl = C->bl; W.idx = K.idx; W.gates = K.gates; W.a = C->a;
  W.Bd = (const uint16_t *)Y.lora_Bd; W.lt = C->lt; W.y = K.y; W.yf = K.yf;
  k_down<<<grid_for(K.T * D.d_model, 4 * C->nsm), 256, 0, s>>>(W);
  CKL("k_down");
  return E0_OK;
}

static ExpertSrc resident_src(e0_ctx *C, int l) {
  ExpertSrc s{};
  s.resident = (const uint8_t *)C->layers[l].experts;
  s.stride = C->bl.bytes;
  s.err = C->err;
  return s;
}

static ExpertSrc pool_src(e0_ctx *C, int l) {
  ExpertSrc s{};
  const int p = l % C->pool.nsets;
  s.pool = C->pool.mem + (size_t)p * C->pool.slots * C->bl.bytes;
  s.stride = C->bl.bytes;
  s.slot_of = C->pool.slot_of + (size_t)p * C->dims.n_experts;
  s.slot_tag = C->pool.slot_tag + (size_t)p * C->pool.slots;
  s.err = C->err;
  return s;
}

extern "C" int e0_moe_layer_forward(e0_ctx *C, int layer, const void *h, int T, const int32_t *route_idx,
                                    void *y_bf16, float *y_f32, int32_t *idx_out, float *gate_out,
                                    void *stream) {
  if (!C || !C->registered) return fail(E0_ERR_INVALID_ARG, "context missing or model not registered");
  if (layer < 0 || layer >= C->L || T < 1 || T > C->maxT || !h || !y_bf16)
    return fail(E0_ERR_INVALID_ARG, "e0_moe_layer_forward: bad layer/T/pointers (T=%d, max %d)", T, C->maxT);
  if (!C->layers[layer].experts)
    return fail(E0_ERR_INVALID_ARG, "layer %d has no resident experts", layer);
  cudaStream_t s = (cudaStream_t)stream;
  C->last = s;
  LayerCall K{};
  K.l = layer; K.T = T; K.h = (const uint16_t *)h; K.route = route_idx;
  K.full_mode = route_idx ? 2 : 1;
  K.idx = idx_out ? idx_out : C->idx;
  K.gates = gate_out ? gate_out : C->gates;
  K.y = (uint16_t *)y_bf16; K.yf = y_f32;
  int rc = layer_pre(C, K, s);
  if (rc) return rc;
  return layer_post(C, K, resident_src(C, layer), s);
}

// The prerouter head of `layer` on C->xf ([G] "Ön Yönlendirici Başlık Mimarisi"):
// z = l(u) (+ fc2(gelu_erf(fc1 u + b1)) + b2), pred = top-k(z).
static int run_head(e0_ctx *C, int layer, int T, const int32_t *cur, const int32_t *prev, int32_t *pred,
                    float *logits_out, cudaStream_t s) {
  const e0_dims &D = C->dims;
  const e0_head &H = C->heads[layer];
  const int in = D.d_model + (D.head_onehot ? 2 * D.n_experts : 0);
  if (D.head_hidden > 0) {
    MatRowsArgs M{};
    M.W = (const uint16_t *)H.fc1_w; M.ldw = in; M.rows = D.head_hidden; M.K = D.d_model;
    M.X = C->xf; M.ldx = D.d_model; M.T = T; M.out = C->h1pre; M.ldo = D.head_hidden;
    k_mat_rows<<<grid_for(D.head_hidden * ((T + kRowTile - 1) / kRowTile), 8 * C->nsm), 256, 0, s>>>(M);
    CKL("k_mat_rows(fc1)");
    const int n = T * D.head_hidden;
    k_head_hidden<<<(n + 255) / 256, 256, 0, s>>>(C->h1pre, (const uint16_t *)H.fc1_w, (const uint16_t *)H.fc1_b, T,
                                                  D.head_hidden, in, D.d_model, D.n_experts, D.top_k,
                                                  D.head_onehot, cur, prev, C->h1);
    CKL("k_head_hidden");
    MatRowsArgs F{};
    F.W = (const uint16_t *)H.fc2_w; F.ldw = D.head_hidden; F.rows = D.n_experts; F.K = D.head_hidden;
    F.X = C->h1; F.ldx = D.head_hidden; F.T = T; F.bias = (const uint16_t *)H.fc2_b; F.out = C->hlog;
    F.ldo = D.n_experts;
    k_mat_rows<<<grid_for(D.n_experts * ((T + kRowTile - 1) / kRowTile), 8 * C->nsm), 256, 0, s>>>(F);
    CKL("k_mat_rows(fc2)");
  }
  RowsArgs R{};
  R.xf = C->xf; R.T = T; R.d = D.d_model; R.E = D.n_experts; R.k = D.top_k;
  R.Wr = nullptr; R.Wh = (const uint16_t *)H.w_lin; R.ldh = in;
  R.hlog = C->hlog; R.hacc = D.head_hidden > 0; R.err = C->err;
  k_rows<<<grid_for(D.n_experts * ((T + kRowTile - 1) / kRowTile), 8 * C->nsm), 256, 0, s>>>(R);
  CKL("k_rows(head)");
  RouteArgs A{};
  A.logits = nullptr; A.T = T; A.E = D.n_experts; A.k = D.top_k;
  A.hlog = C->hlog; A.Wh = R.Wh; A.ldh = in; A.d = D.d_model; A.onehot = D.head_onehot;
  A.prev = prev; A.cur = cur; A.pred = pred; A.hz_out = logits_out; A.err = C->err;
  k_route<<<(T + 7) / 8, 256, 0, s>>>(A);
  CKL("k_route(head)");
  return E0_OK;
}

__global__ void k_bf16_to_f32(const uint16_t *__restrict__ x, float *__restrict__ y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = bf(x[i]);
}

extern "C" int e0_prerouter_predict(e0_ctx *C, int layer, const void *x, int T, const int32_t *cur_idx,
                                    const int32_t *prev_idx, int32_t *pred_idx, float *logits_out,
                                    void *stream) {
  if (!C || !C->registered) return fail(E0_ERR_INVALID_ARG, "context missing or model not registered");
  if (layer < 0 || layer >= C->L || T < 1 || T > C->maxT || !x || !pred_idx)
    return fail(E0_ERR_INVALID_ARG, "e0_prerouter_predict: bad layer/T/pointers");
  const e0_head &H = C->heads[layer];
  if (!H.w_lin) return fail(E0_ERR_INVALID_ARG, "layer %d has no prerouter head", layer);
  const e0_dims &D = C->dims;
  cudaStream_t s = (cudaStream_t)stream;
  C->last = s;
  const int n = T * D.d_model;
  k_bf16_to_f32<<<(n + 255) / 256, 256, 0, s>>>((const uint16_t *)x, C->xf, n);
  CKL("k_bf16_to_f32");
  return run_head(C, layer, T, cur_idx, prev_idx, pred_idx, logits_out, s);
}

// ---------------------------------------------------------------------------------------
// Streaming tier
// ---------------------------------------------------------------------------------------
extern "C" int e0_stream_register(e0_ctx *C, const void *host_blob, size_t expert_bytes, int pool_layers,
                                  int slots_per_layer) {
  if (!C || !host_blob) return fail(E0_ERR_INVALID_ARG, "e0_stream_register: NULL argument");
  if (expert_bytes != (size_t)C->bl.bytes)
    return fail(E0_ERR_INVALID_ARG, "expert_bytes %zu != blob size %lld", expert_bytes, C->bl.bytes);
  if (pool_layers < 2 || pool_layers > std::max(C->L, 2) || slots_per_layer < C->dims.top_k ||
      slots_per_layer > C->dims.n_experts)
    return fail(E0_ERR_INVALID_ARG, "pool needs 2 <= layer sets <= n_layers and k <= slots <= E");
  if ((uintptr_t)host_blob & 15) return fail(E0_ERR_INVALID_ARG, "host store must be 16-byte aligned");
  StreamPool &P = C->pool;
  if (P.mem) return fail(E0_ERR_INVALID_ARG, "a host store is already registered");
  int rc;
  if ((rc = dalloc(&P.mem, (size_t)pool_layers * slots_per_layer * expert_bytes)) ||
      (rc = dalloc(&P.slot_of, (size_t)pool_layers * C->dims.n_experts)) ||
      (rc = dalloc(&P.slot_tag, (size_t)pool_layers * slots_per_layer)))
    return rc;
  CK(cudaMemset(P.slot_of, 0xFF, (size_t)pool_layers * C->dims.n_experts * 4));
  CK(cudaMemset(P.slot_tag, 0xFF, (size_t)pool_layers * slots_per_layer * 4));
  P.nsets = pool_layers;
  P.slots = slots_per_layer;
  P.bytes = expert_bytes;
  P.persist = pool_layers == C->L;
  P.tag_h.assign((size_t)pool_layers * slots_per_layer, -1);
  P.use_h.assign((size_t)pool_layers * slots_per_layer, -1);
  P.round = 0;
  P.host = (const uint8_t *)host_blob;
  CK(cudaStreamCreateWithFlags(&P.side, cudaStreamNonBlocking));
  for (auto *v : {&P.ready, &P.freed}) {
    v->resize(pool_layers);
    for (auto &e : *v) CK(cudaEventCreate(&e));
  }
  P.ring.resize(4 * (size_t)C->L + 8);
  for (auto &r : P.ring) {
    for (auto *e : {&r.c0, &r.c1, &r.w0, &r.w1}) CK(cudaEventCreate(e));
    r.state = 0;
  }
  P.set_rec.assign(pool_layers, -1);
  CK(cudaDeviceSynchronize());
  return E0_OK;
}

// Write a slot set's table: slot s holds expert L.e[s]; slot_of maps expert -> slot.
// (bad_slot, bad_tag) is a host-armed corruption used by the fault tests (-1: none).
__global__ void k_set_slots(int32_t *slot_of, int32_t *slot_tag, int E, int slots, SlotList L, int bad_slot,
                            int bad_tag) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) slot_of[e] = -1;
  __syncthreads();
  for (int s = threadIdx.x; s < slots; s += blockDim.x) {
    const int e = s < L.n ? L.e[s] : -1;
    slot_tag[s] = (s == bad_slot) ? bad_tag : e;
    if (e >= 0) slot_of[e] = s;
  }
}

// Add one staging round's copy time and compute-stream wait time to the stats.
static void account_rec(e0_ctx *C, StreamPool::Rec &r) {
  if (!r.state) return;
  float ms = 0.f;
  cudaEventSynchronize(r.c1);
  if (cudaEventElapsedTime(&ms, r.c0, r.c1) == cudaSuccess) C->stats.stage_ms += ms;
  if (r.state == 2) {
    cudaEventSynchronize(r.w1);
    if (cudaEventElapsedTime(&ms, r.w0, r.w1) == cudaSuccess) C->stats.exposed_wait_ms += ms;
  }
  cudaGetLastError();
  r.state = 0;
}

// Stage the distinct experts of host_idx[0..n) into the slot set of `layer`.
//   Shared sets (fewer sets than layers: the staged-decode double buffer of [G] "Temel
//   terimler"): the set is rewritten, slot s receives the s-th distinct expert.
//   Persistent sets (one per layer, kept across steps: the incremental sticky-slot stack
//   `incr_stack` of [G] "Temel terimler"): an expert already in the set stays in its slot
//   and costs nothing; each missing expert, in first-seen order, replaces the least
//   recently needed slot among those not needed now (empty slots first, then the oldest
//   staging round, ties to the lower slot).  With as many slots as the step routes to,
//   that is "only the changed slots are rewritten"; with more, the set is a least-
//   recently-used expert cache in HBM in front of the host store.
static int stage_impl(e0_ctx *C, int layer, const int32_t *host_idx, int n, cudaStream_t compute,
                      bool prefetch) {
  StreamPool &P = C->pool;
  if (!P.mem) return fail(E0_ERR_INVALID_ARG, "no host store registered");
  if (layer < 0 || layer >= C->L || n < 1 || !host_idx) return fail(E0_ERR_INVALID_ARG, "stage: bad arguments");
  SlotList need{};
  for (int i = 0; i < n; i++) {
    const int e = host_idx[i];
    if (e < 0 || e >= C->dims.n_experts) return fail(E0_ERR_INVALID_ARG, "stage: expert %d out of range", e);
    bool dup = false;
    for (int q = 0; q < need.n; q++) dup |= need.e[q] == e;
    if (dup) continue;
    if (need.n >= P.slots || need.n >= kMaxSlots)
      return fail(E0_ERR_INVALID_ARG, "stage: more distinct experts than pool slots (%d)", P.slots);
    need.e[need.n++] = e;
  }
  const int p = layer % P.nsets;
  // copies[q] = (slot, expert); lst = the set's content after this round (slot -> expert)
  std::vector<std::pair<int, int>> copies;
  SlotList lst{};
  int hits = 0;
  if (!P.persist) {
    lst = need;
    for (int s = 0; s < need.n; s++) copies.push_back({s, need.e[s]});
  } else {
    int *tag = P.tag_h.data() + (size_t)p * P.slots;
    long long *use = P.use_h.data() + (size_t)p * P.slots;
    const long long rnd = ++P.round;
    std::vector<char> held(P.slots, 0);
    std::vector<int> miss;
    for (int q = 0; q < need.n; q++) {
      int at = -1;
      for (int s = 0; s < P.slots; s++)
        if (tag[s] == need.e[q]) at = s;
      if (at >= 0) {
        held[at] = 1;
        use[at] = rnd;
        hits++;
      } else {
        miss.push_back(need.e[q]);
      }
    }
    std::vector<int> victims;
    for (int s = 0; s < P.slots; s++)
      if (!held[s]) victims.push_back(s);
    std::stable_sort(victims.begin(), victims.end(), [&](int a, int b) { return use[a] < use[b]; });
    for (size_t q = 0; q < miss.size(); q++) {
      const int s = victims[q];            // need.n <= slots, so there are enough victims
      copies.push_back({s, miss[q]});
      tag[s] = miss[q];
      use[s] = rnd;
    }
    lst.n = P.slots;
    for (int s = 0; s < P.slots; s++) lst.e[s] = tag[s];
  }
  C->stats.hit_experts += hits;
  int bad_slot = -1, bad_tag = 0;
  if (P.corrupt_set == p) {
    bad_slot = P.corrupt_slot;
    bad_tag = P.corrupt_tag;
    P.corrupt_set = -1;
  }
  if (copies.empty() && bad_slot < 0) {
    // every expert is already in its slot: nothing to copy, the slot table is unchanged
    P.set_rec[p] = -1;
    return E0_OK;
  }
  StreamPool::Rec &rec = P.ring[P.ring_pos];
  account_rec(C, rec);
  P.set_rec[p] = P.ring_pos;
  P.ring_pos = (P.ring_pos + 1) % (int)P.ring.size();
  // the previous user of this slot set must be done (event recorded after its kernels)
  CK(cudaStreamWaitEvent(P.side, P.freed[p], 0));
  CK(cudaEventRecord(rec.c0, P.side));
  uint8_t *dst = P.mem + (size_t)p * P.slots * P.bytes;
  for (const auto &cp : copies) {
    const uint8_t *src = P.host + ((size_t)layer * C->dims.n_experts + cp.second) * P.bytes;
    if (P.fail_after == 0) {
      P.fail_after = -1;
      if (P.persist) P.tag_h[(size_t)p * P.slots + cp.first] = -1;   // the slot's content is now unknown
      return fail(E0_ERR_STAGING, "staging copy of layer %d expert %d refused (injected)", layer, cp.second);
    }
    if (P.fail_after > 0) P.fail_after--;
    cudaError_t e = cudaMemcpyAsync(dst + (size_t)cp.first * P.bytes, src, P.bytes, cudaMemcpyHostToDevice, P.side);
    if (e != cudaSuccess) {
      if (P.persist) P.tag_h[(size_t)p * P.slots + cp.first] = -1;
      return fail(E0_ERR_STAGING, "staging copy of layer %d expert %d: %s", layer, cp.second, cudaGetErrorString(e));
    }
  }
  k_set_slots<<<1, 256, 0, P.side>>>(P.slot_of + (size_t)p * C->dims.n_experts, P.slot_tag + (size_t)p * P.slots,
                                     C->dims.n_experts, P.slots, lst, bad_slot, bad_tag);
  CKL("k_set_slots");
  CK(cudaEventRecord(rec.c1, P.side));
  CK(cudaEventRecord(P.ready[p], P.side));
  rec.state = 1;
  C->stats.staged_experts += copies.size();
  C->stats.staged_bytes += (uint64_t)copies.size() * P.bytes;
  (prefetch ? C->stats.prefetched_experts : C->stats.ondemand_experts) += copies.size();
  (void)compute;
  return E0_OK;
}

extern "C" int e0_stage_experts(e0_ctx *C, int layer, const int32_t *host_idx, int n, void *compute_stream) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  return stage_impl(C, layer, host_idx, n, (cudaStream_t)compute_stream, true);
}

// The compute stream waits for a layer's staged experts; the wait is bracketed by events
// so that the exposed (stalled) time can be accounted.
static int wait_ready(e0_ctx *C, int layer, cudaStream_t s) {
  StreamPool &P = C->pool;
  const int p = layer % P.nsets;
  if (P.set_rec[p] >= 0) {
    StreamPool::Rec &rec = P.ring[P.set_rec[p]];
    CK(cudaEventRecord(rec.w0, s));
    CK(cudaStreamWaitEvent(s, P.ready[p], 0));
    CK(cudaEventRecord(rec.w1, s));
    if (rec.state == 1) rec.state = 2;
  } else if (!P.persist) {
    return fail(E0_ERR_STAGING, "layer %d was never staged", layer);
  } else {
    // a persistent set that needed no copy: its previous round's copies completed before
    // the previous reader of the set ran; order after them all the same
    CK(cudaStreamWaitEvent(s, P.ready[p], 0));
  }
  if (P.log)
    CK(cudaMemcpyAsync(P.log + (size_t)layer * P.slots, P.slot_tag + (size_t)p * P.slots, (size_t)P.slots * 4,
                       cudaMemcpyDeviceToDevice, s));
  return E0_OK;
}

static int release_set(e0_ctx *C, int layer, cudaStream_t s) {
  CK(cudaEventRecord(C->pool.freed[layer % C->pool.nsets], s));
  return E0_OK;
}

// ---------------------------------------------------------------------------------------
// Decode over the stack
// ---------------------------------------------------------------------------------------
static inline int32_t *pred_at(e0_ctx *C, int parity, int layer) {
  return C->pred_tab + ((size_t)parity * (C->L + 1) + layer) * C->maxT * C->dims.top_k;
}
static inline int32_t *hist_at(e0_ctx *C, int parity, int layer) {
  return C->hist_tab + ((size_t)parity * C->L + layer) * C->maxT * C->dims.top_k;
}

static int host_read_idx(e0_ctx *C, int32_t *host, const int32_t *dev, int n, cudaStream_t s) {
  CK(cudaMemcpyAsync(host, dev, n * sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  return E0_OK;
}

static int unique_list(const int32_t *v, int n, int32_t *out) {
  int m = 0;
  for (int i = 0; i < n; i++) {
    bool seen = false;
    for (int q = 0; q < m; q++) seen |= out[q] == v[i];
    if (!seen) out[m++] = v[i];
  }
  return m;
}

static int stack_decode_general(e0_ctx *C, const uint16_t *h_in, int B, int step, uint16_t *y_out,
                                float *y_f32, int streaming, int chained, cudaStream_t s) {
  const e0_dims &D = C->dims;
  const int k = D.top_k, L = C->L;
  const size_t ld = (size_t)B * D.d_model;
  const int cur = step & 1, prv = cur ^ 1;
  std::vector<int32_t> uniq(B * k);
  // streaming in the reactive mode: no prediction, every layer routes itself and its
  // experts are staged on demand after its router ran (the comparison point of [G]
  // "Sonuçlar": prefetch against fully reactive on-demand loading); no head runs
  const bool reactive = streaming && C->pool.reactive;
  if (reactive)
    CK(cudaMemsetAsync(pred_at(C, cur, 0), 0xFF, (size_t)(L + 1) * C->maxT * k * sizeof(int32_t), s));
  for (int l = 0; l < L; l++) {
    const bool predicted = !reactive && step > 0 && l > 0 && C->heads[l - 1].w_lin != nullptr;
    LayerCall K{};
    K.l = l; K.T = B; K.h = h_in + l * ld;
    float *yf_l = y_f32 ? y_f32 + l * ld : C->yscratch + (size_t)(l & 1) * C->maxT * D.d_model;
    K.chain = (chained && l > 0) ? (y_f32 ? y_f32 + (l - 1) * ld : C->yscratch + (size_t)((l - 1) & 1) * C->maxT * D.d_model)
                                 : nullptr;
    K.route = predicted ? pred_at(C, prv, l) : nullptr;
    K.full_mode = predicted ? 0 : 1;
    K.idx = hist_at(C, cur, l);
    K.gates = C->gates;
    K.hist = nullptr;
    const bool has_head = !reactive && C->heads[l].w_lin != nullptr;
    K.head = has_head && D.head_hidden == 0;   // the linear head is fused into the routing kernel
    K.prev = step > 0 ? hist_at(C, prv, l) : nullptr;
    K.pred = pred_at(C, cur, l + 1);
    K.y = y_out + l * ld;
    K.yf = yf_l;
    if (streaming) {
      if (predicted) {
        // the prediction made one token earlier is already on the host: stage now
        const int n = unique_list(C->host_idx + (size_t)l * C->maxT * k, B * k, uniq.data());
        int rc = stage_impl(C, l, uniq.data(), n, s, true);
        if (rc) return rc;
      }
      int rc = layer_pre(C, K, s);
      if (rc) return rc;
      if (has_head && !K.head && (rc = run_head(C, l, B, K.idx, K.prev, K.pred, nullptr, s))) return rc;
      if (!predicted) {
        // reactive layer: the routing exists only now; read it back and stage on demand
        int32_t *scratch = C->host_idx + (size_t)(L + 1) * C->maxT * k;
        if ((rc = host_read_idx(C, scratch, K.idx, B * k, s))) return rc;
        const int n = unique_list(scratch, B * k, uniq.data());
        if ((rc = stage_impl(C, l, uniq.data(), n, s, false))) return rc;
      }
      if ((rc = wait_ready(C, l, s))) return rc;
      if ((rc = layer_post(C, K, pool_src(C, l), s))) return rc;
      if ((rc = release_set(C, l, s))) return rc;
    } else {
      int rc = layer_pre(C, K, s);
      if (rc) return rc;
      if (has_head && !K.head && (rc = run_head(C, l, B, K.idx, K.prev, K.pred, nullptr, s))) return rc;
      if ((rc = layer_post(C, K, resident_src(C, l), s))) return rc;
    }
  }
  if (streaming && !reactive) {
    // next step's predicted routing, for the staging decisions of the next call
    int rc = host_read_idx(C, C->host_idx, pred_at(C, cur, 0), (L + 1) * C->maxT * k, s);
    if (rc) return rc;
  }
  return E0_OK;
}

// ---------------------------------------------------------------------------------------
// Persistent decode path (one stream, resident experts, linear heads)
// ---------------------------------------------------------------------------------------
template <int D, int I>
static size_t dec_smem() { return sizeof(DecSmem<D, I>); }

static bool decode_geometry(const e0_dims &Dm, int *which) {
  if (Dm.d_model == 2048 && Dm.d_ff == 512) *which = 0;
  else if (Dm.d_model == 256 && Dm.d_ff == 128) *which = 1;
  else return false;
  return true;
}

static bool decode_supported(e0_ctx *C, int B) {
  const e0_dims &D = C->dims;
  int which;
  if (B != 1 || D.head_hidden != 0 || !decode_geometry(D, &which) || C->L > 64 || D.lora_rank % 8 != 0 ||
      D.top_k > kDecMaxK)
    return false;
  for (int l = 0; l < C->L; l++)
    if (!C->layers[l].experts) return false;
  // in order, a CTA's share of a layer's gate/up units must fit the task's pieces and its
  // share of the down rows the per-warp accumulators
  const int G = C->nsm;
  const int gu_units = ((D.top_k + 1) * D.d_ff + G - 1) / G, dn_rows = (D.d_model + G - 1) / G;
  return dn_rows <= kDnMaxRows && gu_units <= 2 * D.d_ff && kGuPiece0 + 6 * kMaxPieces <= kMaxItemSegs &&
         3 * (D.top_k + 1) + 4 <= kMaxItemSegs;
}

static int decode_prepare(e0_ctx *C) {
  DecodeState &S = C->dec;
  if (S.ready) return E0_OK;
  const e0_dims &D = C->dims;
  const int L = C->L, E = D.n_experts, k = D.top_k, r = std::max(D.lora_rank, 1);
  S.G = C->nsm;
  std::vector<DecLayer> h(L);
  for (int l = 0; l < L; l++) {
    const e0_layer &Y = C->layers[l];
    h[l] = DecLayer{(const uint8_t *)Y.experts, (const uint8_t *)Y.shared,
                    (const uint16_t *)Y.lora_Ag, (const uint16_t *)Y.lora_Bg, (const uint16_t *)Y.lora_Au,
                    (const uint16_t *)Y.lora_Bu, (const uint16_t *)Y.lora_Ad, (const uint16_t *)Y.lora_Bd,
                    (const uint16_t *)Y.router_w, (const uint16_t *)Y.norm_w,
                    (const uint16_t *)C->heads[l].w_lin};
  }
  if (!S.d_layers) {
    int rc = dalloc(&S.d_layers, L);
    if (rc) return rc;
  }
  CK(cudaMemcpy(S.d_layers, h.data(), L * sizeof(DecLayer), cudaMemcpyHostToDevice));
  if (!S.tbuf) {
    S.blk = ((k + 2) * D.d_ff + 2 * r + k + 7) / 8 * 8;
    const size_t n_y = (size_t)L * D.d_model, n_b = (size_t)L * S.blk, n_r = (size_t)L * E, n_h = (size_t)L * E;
    const size_t tot = n_y + n_b + n_r + n_h;
    int rc = dalloc(&S.tbuf, tot);
    if (rc) return rc;
    CK(cudaMemset(S.tbuf, 0, tot * 8));
    unsigned long long *p = S.tbuf;
    S.t_y = p; p += n_y;
    S.t_blk = p; p += n_b;
    S.t_rlog = p; p += n_r;
    S.t_hlog = p;
  }
  // the item lists of every schedule, built once for this model
  {
    SchedShape Z{};
    Z.L = L; Z.G = S.G; Z.E = E; Z.k = k; Z.r = D.lora_rank; Z.D = D.d_model; Z.I = D.d_ff;
    Z.ldh = D.d_model + (D.head_onehot ? 2 * E : 0);
    for (int l = 0; l < L; l++) {
      Z.head[l] = C->heads[l].w_lin != nullptr;
      Z.lora[l] = C->layers[l].lora_Ag != nullptr;
    }
    const size_t per = (size_t)S.G * kMaxItems;
    std::vector<unsigned long long> items(4 * per, 0ull);
    std::vector<int> counts(4 * (size_t)S.G, 0);
    for (int v = 0; v < 4; v++)
      for (int c = 0; c < S.G; c++) {
        const int n = build_items(Z, (v >> 1) != 0, (v & 1) != 0, c, items.data() + v * per + (size_t)c * kMaxItems);
        if (n < 0) return fail(E0_ERR_INVALID_ARG, "decode schedule: more than %d items for one CTA", kMaxItems);
        counts[(size_t)v * S.G + c] = n;
      }
    int rc;
    if (!S.sched && (rc = dalloc(&S.sched, 4 * per))) return rc;
    if (!S.sched_n && (rc = dalloc(&S.sched_n, 4 * (size_t)S.G))) return rc;
    CK(cudaMemcpy(S.sched, items.data(), items.size() * sizeof(unsigned long long), cudaMemcpyHostToDevice));
    CK(cudaMemcpy(S.sched_n, counts.data(), counts.size() * sizeof(int), cudaMemcpyHostToDevice));
  }
  int which;
  decode_geometry(D, &which);
  const void *fn = which == 0 ? (const void *)k_decode<2048, 512> : (const void *)k_decode<256, 128>;
  S.smem = which == 0 ? dec_smem<2048, 512>() : dec_smem<256, 128>();
  CK(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S.smem));
  int per_sm = 0;
  CK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kDecThreads, S.smem));
  if (per_sm < 1) return fail(E0_ERR_CUDA, "decode kernel does not fit on an SM (%zu B smem)", S.smem);
  S.ready = true;
  return E0_OK;
}

static int decode_persistent(e0_ctx *C, const uint16_t *h, int step, uint16_t *y, float *yf, int chained,
                             cudaStream_t s) {
  int rc = decode_prepare(C);
  if (rc) return rc;
  DecodeState &S = C->dec;
  const e0_dims &D = C->dims;
  const int cur = step & 1, prv = cur ^ 1;
  DecodeParams P{};
  P.layers = S.d_layers;
  P.L = C->L; P.E = D.n_experts; P.k = D.top_k; P.r = D.lora_rank;
  P.ldh = D.d_model + (D.head_onehot ? 2 * D.n_experts : 0);
  P.onehot = D.head_onehot; P.G = S.G;
  P.eps = D.rms_eps; P.c = D.lora_scale;
  P.h = h; P.y = y; P.yf = yf; P.chained = chained;
  P.flat = chained ? 0 : S.flat;
  P.epoch = ++S.epoch;
  P.step0 = step == 0;
  P.pred_in = step > 0 ? pred_at(C, prv, 0) : nullptr;
  P.pred_out = pred_at(C, cur, 0);
  P.hist_out = hist_at(C, cur, 0);
  P.hist_prev = step > 0 ? hist_at(C, prv, 0) : nullptr;
  P.maxT = C->maxT;
  P.t_y = S.t_y; P.t_blk = S.t_blk; P.blk = S.blk; P.t_rlog = S.t_rlog; P.t_hlog = S.t_hlog;
  P.err = C->err;
  P.timeout_ns = S.timeout_ns;
  P.stall_cta = S.stall_cta;
  P.trace = S.trace;
  {
    const int v = 2 * (P.flat ? 1 : 0) + (P.step0 ? 1 : 0);
    P.sched = S.sched + (size_t)v * S.G * kMaxItems;
    P.sched_n = S.sched_n + (size_t)v * S.G;
  }
  S.stall_cta = -1;
  int which;
  decode_geometry(D, &which);
  const void *fn = which == 0 ? (const void *)k_decode<2048, 512> : (const void *)k_decode<256, 128>;
  void *args[] = {&P};
  CK(cudaLaunchCooperativeKernel(fn, dim3(S.G), dim3(kDecThreads), args, S.smem, s));
  C->stats.kernel_launches++;
  return E0_OK;
}

// ---------------------------------------------------------------------------------------
// Phased decode path (unchained steps of up to kPhMaxB streams, resident experts)
// ---------------------------------------------------------------------------------------
static bool phased_geometry(const e0_dims &Dm, int *which) {
  if (Dm.d_model == 2048 && Dm.d_ff == 512) *which = 0;
  else if (Dm.d_model == 256 && Dm.d_ff == 128) *which = 1;
  else return false;
  return true;
}

static bool phased_supported(e0_ctx *C, int B) {
  const e0_dims &D = C->dims;
  int which;
  if (B < 1 || B > kPhMaxB * kPhGroups || !phased_geometry(D, &which) || C->L > 64 || D.head_hidden > kPhMaxH ||
      D.head_hidden % 16 != 0)
    return false;
  for (int l = 0; l < C->L; l++)
    if (!C->layers[l].experts) return false;
  return true;
}

static int phased_prepare(e0_ctx *C) {
  PhState &S = C->ph;
  if (S.ready) return E0_OK;
  const e0_dims &D = C->dims;
  const int L = C->L;
  std::vector<PhLayer> h(L);
  for (int l = 0; l < L; l++) {
    const e0_layer &Y = C->layers[l];
    const e0_head &H = C->heads[l];
    h[l] = PhLayer{(const uint8_t *)Y.experts, (const uint8_t *)Y.shared, (const uint16_t *)Y.router_w,
                   (const uint16_t *)Y.norm_w, (const uint16_t *)H.w_lin, (const uint16_t *)H.fc1_w,
                   (const uint16_t *)H.fc1_b, (const uint16_t *)H.fc2_w, (const uint16_t *)H.fc2_b,
                   (const uint16_t *)Y.lora_Ag, (const uint16_t *)Y.lora_Bg, (const uint16_t *)Y.lora_Au,
                   (const uint16_t *)Y.lora_Bu, (const uint16_t *)Y.lora_Ad, (const uint16_t *)Y.lora_Bd};
  }
  int rc;
  if (!S.d_layers && (rc = dalloc(&S.d_layers, L))) return rc;
  CK(cudaMemcpy(S.d_layers, h.data(), L * sizeof(PhLayer), cudaMemcpyHostToDevice));
  if (!S.mem) {
    const size_t T = (size_t)L * kPhMaxB, d = D.d_model, E = D.n_experts, I = D.d_ff, k = D.top_k;
    const size_t r = std::max(D.lora_rank, 1), H = std::max(D.head_hidden, 1);
    // sizes in 4-byte words, each region rounded to 16 bytes
    auto w4 = [](size_t bytes) { return (bytes + 15) / 16 * 4; };
    const size_t n_x16 = w4(T * d * 2), n_xp = w4(T * d * 2), n_a = w4(T * (k + 1) * I * 2), n_xs = w4(T * (d / 64) * 4),
                 n_rl = w4(T * E * 4), n_rs = w4(T * k * 4), n_hl = w4(T * E * 4), n_lt = w4(T * 3 * r * 4),
                 n_h1 = w4(T * H * 4), n_g = w4(T * k * 4), n_as = w4(T * (k + 1) * (I / 64) * 4),
                 n_pl = w4((size_t)2 * kPhGroups * L * kPlanInts * 4),
                 n_sl = w4((size_t)2 * kPhGroups * L * kPhMaxU * kPhMaxB),
                 n_gus = w4(T * 2 * I * 4);
    const size_t tot = n_x16 + n_xp + n_a + n_xs + n_rl + n_rs + n_hl + n_lt + n_h1 + n_g + n_as + n_pl + n_sl + n_gus;
    uint32_t *p = nullptr;
    if ((rc = dalloc(&p, tot))) return rc;
    CK(cudaMemset(p, 0, tot * 4));
    S.mem = p;
    S.x16 = (uint16_t *)p; p += n_x16;
    S.xp = (uint16_t *)p; p += n_xp;
    S.a = (uint16_t *)p; p += n_a;
    S.xs = (float *)p; p += n_xs;
    S.rlog = (float *)p; p += n_rl;
    S.rsel = (float *)p; p += n_rs;
    S.hlog = (float *)p; p += n_hl;
    S.lt = (float *)p; p += n_lt;
    S.h1 = (float *)p; p += n_h1;
    S.gates = (float *)p; p += n_g;
    S.asum = (float *)p; p += n_as;
    S.plan = (int *)p; p += n_pl;
    S.slot = (int8_t *)p; p += n_sl;
    S.gus = (float *)p;
  }
  int which;
  phased_geometry(D, &which);
  // the down kernel's dynamic shared memory at the largest batch
  const size_t dn_max = which == 0 ? ph_dn_smem<2048, 512>(kPhMaxB, D.top_k) : ph_dn_smem<256, 128>(kPhMaxB, D.top_k);
  const void *dn = which == 0 ? (const void *)k_ph_down<2048, 512> : (const void *)k_ph_down<256, 128>;
  CK(cudaFuncSetAttribute(dn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dn_max));
  S.ready = true;
  return E0_OK;
}

// The bf16-rows work list for batch B, first step or not (built once per shape).
static int phased_blocks(e0_ctx *C, int B, bool step0, const PhBlock **out, int *n) {
  PhState &S = C->ph;
  const int v = 2 * B + (step0 ? 1 : 0);
  if (!S.blocks[v]) {
    PhShape Z{};
    Z.L = C->L; Z.E = C->dims.n_experts; Z.k = C->dims.top_k; Z.r = C->dims.lora_rank; Z.H = C->dims.head_hidden;
    Z.B = B;
    for (int l = 0; l < C->L; l++) {
      Z.head[l] = C->heads[l].w_lin != nullptr;
      Z.lora[l] = C->layers[l].lora_Ag != nullptr;
    }
    const std::vector<PhBlock> bl = ph_blocks(Z, step0);
    int rc;
    if ((rc = dalloc(&S.blocks[v], bl.size()))) return rc;
    CK(cudaMemcpy(S.blocks[v], bl.data(), bl.size() * sizeof(PhBlock), cudaMemcpyHostToDevice));
    S.nblocks[v] = (int)bl.size();
  }
  *out = S.blocks[v];
  *n = S.nblocks[v];
  return E0_OK;
}

// Launch one kernel of the phased step; pdl = it may start while the previous kernel on the
// stream is still running (it waits with griddepcontrol.wait before reading its outputs).
template <typename Kern>
static cudaError_t ph_launch(Kern kernel, unsigned grid, unsigned block, size_t smem, cudaStream_t s, bool pdl,
                             const PhParams &P) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? at : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, P);
}

template <int D, int I>
static int phased_launch(e0_ctx *C, const PhParams &P, cudaStream_t s) {
  const int L = P.L, B = P.B;
  const int Umax = std::min(B * P.k, P.E) + 1;
  PhState &S = C->ph;
  // profiling: no overlap between the kernels, an event before each and after the last
  const bool tm = S.timing;
  std::vector<cudaEvent_t> ev;
  if (tm) {
    ev.resize(7);
    for (auto &e : ev) CK(cudaEventCreate(&e));
  }
  int q = 0;
#define PHL(call, what)                                                                     \
  do {                                                                                     \
    if (tm) CK(cudaEventRecord(ev[q++], s));                                               \
    C->stats.kernel_launches++;                                                            \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess) return fail(E0_ERR_CUDA, "launch %s: %s", what, cudaGetErrorString(e_)); \
  } while (0)
  const bool pdl = !tm;
  // the first kernel waits for the previous step in full (stream order): whatever the later
  // kernels read before their wait (weights, the previous step's predictions) is complete
  PHL(ph_launch(k_ph_norm<D>, L * B, 256, 0, s, false, P), "k_ph_norm");
  PHL(ph_launch(k_ph_rows<D>, P.nblocks, 32 * PhRowsCfg<D>::NW, 0, s, pdl, P), "k_ph_rows");
  PHL(ph_launch(k_ph_route, L, 256, 0, s, pdl, P), "k_ph_route");
  PHL(ph_launch(k_ph_gateup<D, I>, L * Umax * (I / 8 / kPhGuBlocks), 32 * (D / 256), 0, s, pdl, P), "k_ph_gateup");
  PHL(ph_launch(k_ph_tdsum<I>, L * B, 256, 0, s, pdl, P), "k_ph_tdsum");
  PHL(ph_launch(k_ph_down<D, I>, L * (D / 16), 32 * (I / 64), ph_dn_smem<D, I>(B, P.k), s, pdl, P), "k_ph_down");
#undef PHL
  if (tm) {
    CK(cudaEventRecord(ev[6], s));
    S.pending.push_back(ev);
  }
  return E0_OK;
}

// One phased decode step of B streams: one pass of the six kernels per group of up to
// kPhMaxB streams (each group with its own routing-table offset and expert plans).
static int decode_phased(e0_ctx *C, const uint16_t *h, int B, int step, uint16_t *y, float *yf, cudaStream_t s) {
  int rc = phased_prepare(C);
  if (rc) return rc;
  PhState &S = C->ph;
  const e0_dims &D = C->dims;
  const int cur = step & 1, prv = cur ^ 1, k = D.top_k;
  const bool fix_plans = step > 0 && S.last_step != step - 1;
  S.last_step = -1;
  for (int grp = 0; grp * kPhMaxB < B; grp++) {
    const int tok0 = grp * kPhMaxB, Bg = std::min(kPhMaxB, B - tok0);
    PhParams P{};
    P.layers = S.d_layers;
    P.L = C->L; P.B = Bg; P.E = D.n_experts; P.k = k; P.r = D.lora_rank; P.H = D.head_hidden;
    P.ldh = D.d_model + (D.head_onehot ? 2 * D.n_experts : 0);
    P.onehot = D.head_onehot; P.step0 = step == 0; P.maxT = C->maxT;
    P.eps = D.rms_eps; P.c = D.lora_scale;
    P.h = h; P.y = y; P.yf = yf; P.hB = B; P.tok0 = tok0;
    P.x16 = S.x16; P.xp = S.xp; P.xs = S.xs; P.rlog = S.rlog; P.rsel = S.rsel; P.hlog = S.hlog; P.lt = S.lt;
    P.h1 = S.h1; P.gates = S.gates; P.a = S.a; P.asum = S.asum; P.gus = S.gus;
    P.plan_cur = S.plan + ((size_t)cur * kPhGroups + grp) * C->L * kPlanInts;
    P.plan_next = S.plan + ((size_t)prv * kPhGroups + grp) * C->L * kPlanInts;
    P.slot_cur = S.slot + ((size_t)cur * kPhGroups + grp) * C->L * kPhMaxU * kPhMaxB;
    P.slot_next = S.slot + ((size_t)prv * kPhGroups + grp) * C->L * kPhMaxU * kPhMaxB;
    P.pred_in = step > 0 ? pred_at(C, prv, 0) + (size_t)tok0 * k : nullptr;
    P.pred_out = pred_at(C, cur, 0) + (size_t)tok0 * k;
    P.hist_out = hist_at(C, cur, 0) + (size_t)tok0 * k;
    P.hist_prev = step > 0 ? hist_at(C, prv, 0) + (size_t)tok0 * k : nullptr;
    P.err = C->err;
    if ((rc = phased_blocks(C, Bg, step == 0, &P.blocks, &P.nblocks))) return rc;
    if (fix_plans) {
      // the previous step ran another path: the predicted layers' plans come from its predictions
      k_ph_plan_pred<<<C->L, 32, 0, s>>>(P);
      CKL("k_ph_plan_pred");
    }
    int which;
    phased_geometry(D, &which);
    rc = which == 0 ? phased_launch<2048, 512>(C, P, s) : phased_launch<256, 128>(C, P, s);
    if (rc) return rc;
  }
  S.last_step = step;
  return E0_OK;
}

// Test hook: make CTA `cta` of the next persistent decode launch wait on a word nobody
// writes, with a wait budget of `timeout_ns`; the launch must come back with TIMEOUT.
extern "C" int e0_debug_decode_stall(e0_ctx *C, int cta, unsigned long long timeout_ns) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  C->dec.stall_cta = cta;
  C->dec.timeout_ns = timeout_ns ? timeout_ns : 2000000000ull;
  return E0_OK;
}

// The decode step as a replay of a captured CUDA graph of the per-layer kernels: the
// caller's inputs are copied into fixed buffers, the graph runs on the caller's stream and
// the outputs are copied back.  One graph per (B, step parity, first step, chained, fp32
// output) is captured on first use.
static int decode_graph(e0_ctx *C, const uint16_t *h_in, int B, int step, uint16_t *y_out, float *y_f32, int chained,
                        cudaStream_t s) {
  const e0_dims &D = C->dims;
  const size_t full = (size_t)C->L * C->maxT * D.d_model;
  if (!C->g_h) {
    int rc;
    if ((rc = dalloc(&C->g_h, full)) || (rc = dalloc(&C->g_y, full)) || (rc = dalloc(&C->g_yf, full))) return rc;
    CK(cudaStreamCreateWithFlags(&C->cap, cudaStreamNonBlocking));
  }
  const int parity = step & 1, step0 = step == 0, has_f32 = y_f32 != nullptr;
  DecodeGraph *G = nullptr;
  for (auto &g : C->graphs)
    if (g.exec && g.B == B && g.parity == parity && g.step0 == step0 && g.chained == chained && g.has_f32 == has_f32)
      G = &g;
  if (!G) {
    G = &C->graphs[C->graph_next];
    C->graph_next = (C->graph_next + 1) % (int)(sizeof(C->graphs) / sizeof(C->graphs[0]));
    if (G->exec) cudaGraphExecDestroy(G->exec);
    *G = DecodeGraph{};
    const unsigned long long l0 = C->stats.kernel_launches;
    CK(cudaStreamBeginCapture(C->cap, cudaStreamCaptureModeThreadLocal));
    int rc = stack_decode_general(C, C->g_h, B, step, C->g_y, has_f32 ? C->g_yf : nullptr, 0, chained, C->cap);
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamEndCapture(C->cap, &graph);
    if (rc || e != cudaSuccess) {
      if (graph) cudaGraphDestroy(graph);
      C->stats.kernel_launches = l0;
      return rc ? rc : fail(E0_ERR_CUDA, "decode graph capture: %s", cudaGetErrorString(e));
    }
    e = cudaGraphInstantiate(&G->exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) return fail(E0_ERR_CUDA, "decode graph instantiate: %s", cudaGetErrorString(e));
    G->B = B; G->parity = parity; G->step0 = step0; G->chained = chained; G->has_f32 = has_f32;
    G->launches = C->stats.kernel_launches - l0;
    C->stats.kernel_launches = l0;
  }
  // the graph reads and writes packed [L][B][d] buffers of its own
  const size_t n = (size_t)C->L * B * D.d_model;
  CK(cudaMemcpyAsync(C->g_h, h_in, n * 2, cudaMemcpyDeviceToDevice, s));
  CK(cudaGraphLaunch(G->exec, s));
  C->stats.kernel_launches += G->launches;
  CK(cudaMemcpyAsync(y_out, C->g_y, n * 2, cudaMemcpyDeviceToDevice, s));
  if (y_f32) CK(cudaMemcpyAsync(y_f32, C->g_yf, n * 4, cudaMemcpyDeviceToDevice, s));
  return E0_OK;
}

extern "C" int e0_moe_stack_decode(e0_ctx *C, const void *h_in, int B, int step, void *y_out, float *y_f32,
                                   int streaming, int chained, void *stream) {
  if (!C || !C->registered) return fail(E0_ERR_INVALID_ARG, "context missing or model not registered");
  if (!h_in || !y_out || B < 1 || B > C->maxT || step < 0)
    return fail(E0_ERR_INVALID_ARG, "e0_moe_stack_decode: bad arguments (B=%d, max %d)", B, C->maxT);
  if (step > 0 && (C->last_step != step - 1 || C->last_B != B))
    return fail(E0_ERR_INVALID_ARG, "step %d does not follow step %d with the same B", step, C->last_step);
  if (streaming && !C->pool.mem) return fail(E0_ERR_INVALID_ARG, "streaming decode needs e0_stream_register");
  if (streaming && C->pool.slots < std::min(B * C->dims.top_k, C->dims.n_experts))
    return fail(E0_ERR_INVALID_ARG, "pool has %d slots per layer, a step may route to %d experts", C->pool.slots,
                std::min(B * C->dims.top_k, C->dims.n_experts));
  if (!streaming)
    for (int l = 0; l < C->L; l++)
      if (!C->layers[l].experts) return fail(E0_ERR_INVALID_ARG, "layer %d has no resident experts", l);
  cudaStream_t s = (cudaStream_t)stream;
  C->last = s;
  int rc;
  const bool one_launch = decode_supported(C, B);
  const bool phased = !chained && phased_supported(C, B);
  int mode = C->force_general ? 3 : C->decode_mode;
  // default: the measured fastest per batch: at one stream the one-launch kernel, up to
  // kPhMaxB x kPhGroups streams the phased kernels, beyond that the per-layer kernels
  if (mode == 0) mode = one_launch ? 1 : phased ? 4 : 3;
  if (mode == 4 && !phased) mode = one_launch ? 1 : 3;
  if (mode == 1 && !one_launch) mode = 2;
  if (streaming) mode = 3;                                  // host decisions between layers
  if (mode == 4)
    rc = decode_phased(C, (const uint16_t *)h_in, B, step, (uint16_t *)y_out, y_f32, s);
  else if (mode == 1)
    rc = decode_persistent(C, (const uint16_t *)h_in, step, (uint16_t *)y_out, y_f32, chained, s);
  else if (mode == 2)
    rc = decode_graph(C, (const uint16_t *)h_in, B, step, (uint16_t *)y_out, y_f32, chained, s);
  else
    rc = stack_decode_general(C, (const uint16_t *)h_in, B, step, (uint16_t *)y_out, y_f32, streaming, chained, s);
  if (rc) return rc;
  C->last_step = step;
  C->last_B = B;
  C->stats.steps++;
  return E0_OK;
}

// The two copy streams and their tail events (created on first use).
static int host_io_streams(e0_ctx *C) {
  auto &io = C->io;
  if (io.cs) return E0_OK;
  CK(cudaStreamCreateWithFlags(&io.cs, cudaStreamNonBlocking));
  CK(cudaStreamCreateWithFlags(&io.ds, cudaStreamNonBlocking));
  CK(cudaEventCreateWithFlags(&io.tail, cudaEventDisableTiming));
  CK(cudaEventCreateWithFlags(&io.tail2, cudaEventDisableTiming));
  return E0_OK;
}

// A decode step with the input and output in (pinned) host memory.  Step n uses staging
// buffer n % 2: its input copy (copy stream) waits until step n-2's kernels have read the
// buffer, the step (caller's stream) waits for the input copy and for step n-2's output
// copy out of the buffer, and its output copy (copy stream) waits for the step.  So the
// input copy of step n+1 and the output copy of step n run while the kernels of the
// neighbouring steps do.
extern "C" int e0_moe_stack_decode_host(e0_ctx *C, const void *h_host, int B, int step, void *y_host,
                                        float *y_f32_host, int streaming, int chained, void *stream) {
  if (!C || !C->registered) return fail(E0_ERR_INVALID_ARG, "context missing or model not registered");
  if (!h_host || !y_host || B < 1 || B > C->maxT || step < 0)
    return fail(E0_ERR_INVALID_ARG, "e0_moe_stack_decode_host: bad arguments (B=%d, max %d)", B, C->maxT);
  auto &io = C->io;
  const size_t n = (size_t)C->L * C->maxT * C->dims.d_model, used = (size_t)C->L * B * C->dims.d_model;
  int rc0;
  if ((rc0 = host_io_streams(C))) return rc0;
  if (!io.h[0]) {
    for (int b = 0; b < 2; b++) {
      CK(cudaEventCreateWithFlags(&io.in[b], cudaEventDisableTiming));
      CK(cudaEventCreateWithFlags(&io.out[b], cudaEventDisableTiming));
      CK(cudaEventCreateWithFlags(&io.done[b], cudaEventDisableTiming));
      int rc;
      if ((rc = dalloc(&io.h[b], n)) || (rc = dalloc(&io.y[b], n))) return rc;
    }
  }
  if (y_f32_host && !io.yf[0]) {
    int rc;
    if ((rc = dalloc(&io.yf[0], n)) || (rc = dalloc(&io.yf[1], n))) return rc;
  }
  cudaStream_t s = (cudaStream_t)stream;
  const int b = (int)(io.calls & 1);
  if (io.used[b]) {
    CK(cudaStreamWaitEvent(io.cs, io.out[b], 0));   // step n-2 has read h[b]
    CK(cudaStreamWaitEvent(s, io.done[b], 0));      // y[b] of step n-2 has been copied out
  }
  CK(cudaMemcpyAsync(io.h[b], h_host, used * 2, cudaMemcpyHostToDevice, io.cs));
  CK(cudaEventRecord(io.in[b], io.cs));
  CK(cudaStreamWaitEvent(s, io.in[b], 0));
  const int rc = e0_moe_stack_decode(C, io.h[b], B, step, io.y[b], y_f32_host ? io.yf[b] : nullptr, streaming,
                                     chained, stream);
  io.used[b] = true;
  io.calls++;
  CK(cudaEventRecord(io.out[b], s));
  if (rc) {
    CK(cudaEventRecord(io.done[b], io.ds));
    return rc;
  }
  CK(cudaStreamWaitEvent(io.ds, io.out[b], 0));
  CK(cudaMemcpyAsync(y_host, io.y[b], used * 2, cudaMemcpyDeviceToHost, io.ds));
  if (y_f32_host) CK(cudaMemcpyAsync(y_f32_host, io.yf[b], used * 4, cudaMemcpyDeviceToHost, io.ds));
  CK(cudaEventRecord(io.done[b], io.ds));
  return E0_OK;
}

// Make `stream` wait for every copy that the host-buffer decode and prefill calls have
// issued.
extern "C" int e0_host_io_wait(e0_ctx *C, void *stream) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  if (!C->io.cs) return E0_OK;
  CK(cudaEventRecord(C->io.tail, C->io.cs));
  CK(cudaEventRecord(C->io.tail2, C->io.ds));
  CK(cudaStreamWaitEvent((cudaStream_t)stream, C->io.tail, 0));
  CK(cudaStreamWaitEvent((cudaStream_t)stream, C->io.tail2, 0));
  return E0_OK;
}

// One layer of a prefill chunk (see e0_moe_prefill_stack): h_l, y_l [T, d], yf_l [T, d]
// or NULL, idx_l [T, k] or NULL.  Layer l reads the predictions layer l-1 made in the same
// chunk (alternating buffers).
static int prefill_layer(e0_ctx *C, int l, const uint16_t *h_l, int T, uint16_t *y_l, float *yf_l, int32_t *idx_l,
                         cudaStream_t s) {
  const int k = C->dims.top_k;
  const bool predicted = l > 0 && C->heads[l - 1].w_lin != nullptr;
  int32_t *pin = C->pf_buf + (size_t)((l + 1) & 1) * (C->maxT + 1) * k;   // written by layer l-1's head
  int32_t *pout = C->pf_buf + (size_t)(l & 1) * (C->maxT + 1) * k;
  LayerCall K{};
  K.l = l; K.T = T; K.h = h_l;
  K.route = predicted ? pin : nullptr;          // row t = prediction made on token t-1
  K.full_mode = predicted ? 2 : 1;              // row 0 is -1: token 0 uses its own router
  K.idx = idx_l ? idx_l : C->pf_idx + k;
  K.gates = C->gates;
  K.head = C->heads[l].w_lin != nullptr;
  K.prev = nullptr;
  K.pred = pout + k;                             // prediction of token t -> row t+1
  K.y = y_l;
  K.yf = yf_l;
  int rc = layer_pre(C, K, s);
  if (rc) return rc;
  return layer_post(C, K, resident_src(C, l), s);
}

static int prefill_check(e0_ctx *C, const void *h, int T, const void *y) {
  if (!C || !C->registered) return fail(E0_ERR_INVALID_ARG, "context missing or model not registered");
  if (!h || !y || T < 1 || T > C->maxT)
    return fail(E0_ERR_INVALID_ARG, "prefill stack: bad arguments (T=%d, max %d)", T, C->maxT);
  if (C->dims.head_hidden > 0 || C->dims.head_onehot)
    return fail(E0_ERR_INVALID_ARG, "prefill stack supports the linear head without one-hot inputs");
  for (int l = 0; l < C->L; l++)
    if (!C->layers[l].experts) return fail(E0_ERR_INVALID_ARG, "layer %d has no resident experts", l);
  return E0_OK;
}

// One prefill chunk through every layer.  Layer N+1's routing of token t is the head of
// layer N on token t-1 (prediction as routing, one token ahead); token 0, and layers after
// a layer without a head, route with their own router.  Linear heads without one-hot
// inputs (the workloads' form).
extern "C" int e0_moe_prefill_stack(e0_ctx *C, const void *h_in, int T, void *y_out, float *y_f32, int32_t *idx_out,
                                    void *stream) {
  int rc0;
  if ((rc0 = prefill_check(C, h_in, T, y_out))) return rc0;
  cudaStream_t s = (cudaStream_t)stream;
  C->last = s;
  const size_t ld = (size_t)T * C->dims.d_model;
  for (int l = 0; l < C->L; l++) {
    int rc = prefill_layer(C, l, (const uint16_t *)h_in + l * ld, T, (uint16_t *)y_out + l * ld,
                           y_f32 ? y_f32 + l * ld : nullptr, idx_out ? idx_out + (size_t)l * T * C->dims.top_k : nullptr, s);
    if (rc) return rc;
  }
  return E0_OK;
}

// A prefill chunk with the input and output in (pinned) host memory: layer l's input is
// copied in (input copy stream) while layer l-1 computes, and its output copied out
// (output copy stream) while layer l+1 computes; two alternating device staging buffers,
// ordered by events (the layers' inputs are independent, so the copies of every layer but
// the first and the last hide behind the kernels).
extern "C" int e0_moe_prefill_stack_host(e0_ctx *C, const void *h_host, int T, void *y_host, float *y_f32_host,
                                         int32_t *idx_out, void *stream) {
  int rc;
  if ((rc = prefill_check(C, h_host, T, y_host))) return rc;
  if ((rc = host_io_streams(C))) return rc;
  auto &io = C->io;
  const size_t cap = (size_t)C->maxT * C->dims.d_model, ld = (size_t)T * C->dims.d_model;
  if (!io.ph[0]) {
    for (int b = 0; b < 2; b++) {
      CK(cudaEventCreateWithFlags(&io.pin[b], cudaEventDisableTiming));
      CK(cudaEventCreateWithFlags(&io.pout[b], cudaEventDisableTiming));
      CK(cudaEventCreateWithFlags(&io.pdone[b], cudaEventDisableTiming));
      if ((rc = dalloc(&io.ph[b], cap)) || (rc = dalloc(&io.py[b], cap))) return rc;
    }
  }
  if (y_f32_host && !io.pyf[0])
    for (int b = 0; b < 2; b++)
      if ((rc = dalloc(&io.pyf[b], cap))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  C->last = s;
  for (int l = 0; l < C->L; l++) {
    const int b = l & 1;
    if (io.pused[b]) {
      CK(cudaStreamWaitEvent(io.cs, io.pout[b], 0));   // the layer two back has read ph[b]
      CK(cudaStreamWaitEvent(s, io.pdone[b], 0));      // py[b] of the layer two back is out
    }
    CK(cudaMemcpyAsync(io.ph[b], (const uint16_t *)h_host + l * ld, ld * 2, cudaMemcpyHostToDevice, io.cs));
    CK(cudaEventRecord(io.pin[b], io.cs));
    CK(cudaStreamWaitEvent(s, io.pin[b], 0));
    rc = prefill_layer(C, l, io.ph[b], T, io.py[b], y_f32_host ? io.pyf[b] : nullptr,
                       idx_out ? idx_out + (size_t)l * T * C->dims.top_k : nullptr, s);
    io.pused[b] = true;
    CK(cudaEventRecord(io.pout[b], s));
    if (rc) {
      CK(cudaEventRecord(io.pdone[b], io.ds));
      return rc;
    }
    CK(cudaStreamWaitEvent(io.ds, io.pout[b], 0));
    CK(cudaMemcpyAsync((uint16_t *)y_host + l * ld, io.py[b], ld * 2, cudaMemcpyDeviceToHost, io.ds));
    if (y_f32_host)
      CK(cudaMemcpyAsync(y_f32_host + l * ld, io.pyf[b], ld * 4, cudaMemcpyDeviceToHost, io.ds));
    CK(cudaEventRecord(io.pdone[b], io.ds));
  }
  return E0_OK;
}

extern "C" int e0_get_routing(e0_ctx *C, int B, int32_t *idx_host, int32_t *pred_host) {
  if (!C || C->last_step < 0 || B != C->last_B) return fail(E0_ERR_INVALID_ARG, "no decode step with this B");
  CK(cudaStreamSynchronize(C->last));
  const int k = C->dims.top_k, cur = C->last_step & 1;
  for (int l = 0; l < C->L; l++) {
    if (idx_host) CK(cudaMemcpy(idx_host + (size_t)l * B * k, hist_at(C, cur, l), (size_t)B * k * 4, cudaMemcpyDeviceToHost));
    if (pred_host) {
      if (C->heads[l].w_lin)
        CK(cudaMemcpy(pred_host + (size_t)l * B * k, pred_at(C, cur, l + 1), (size_t)B * k * 4, cudaMemcpyDeviceToHost));
      else
        for (int i = 0; i < B * k; i++) pred_host[(size_t)l * B * k + i] = -1;
    }
  }
  return E0_OK;
}

extern "C" int e0_get_stats(e0_ctx *C, e0_stats *out) {
  if (!C || !out) return fail(E0_ERR_INVALID_ARG, "NULL argument");
  if (C->pool.mem) {
    cudaStreamSynchronize(C->pool.side);
    if (C->last) cudaStreamSynchronize(C->last);
    for (auto &r : C->pool.ring) account_rec(C, r);
  }
  for (auto &e : C->gemm_ev) {
    float ms = 0.f;
    if (cudaEventSynchronize(e.second) == cudaSuccess && cudaEventElapsedTime(&ms, e.first, e.second) == cudaSuccess) {
      C->stats.gemm_timed++;
      C->stats.gemm_ms += ms;
    }
    cudaEventDestroy(e.first);
    cudaEventDestroy(e.second);
  }
  C->gemm_ev.clear();
  *out = C->stats;
  return E0_OK;
}

// Profiling: time every expert-GEMM launch with an event pair (see e0_get_stats).
extern "C" int e0_debug_time_gemm(e0_ctx *C, int on) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  C->time_gemm = on != 0;
  return E0_OK;
}

extern "C" int e0_sync_status(e0_ctx *C) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  if (C->last) CK(cudaStreamSynchronize(C->last));
  if (C->pool.side) CK(cudaStreamSynchronize(C->pool.side));
  int err = 0;
  CK(cudaMemcpy(&err, C->err, sizeof(int), cudaMemcpyDeviceToHost));
  CK(cudaMemset(C->err, 0, sizeof(int)));
  if (err & DERR_SLOT) return fail(E0_ERR_SLOT_MISMATCH, "a kernel found a pool slot holding another expert");
  if (err & DERR_TIMEOUT) return fail(E0_ERR_TIMEOUT, "a bounded device wait gave up");
  if (err & (DERR_INDEX | DERR_DUP))
    return fail(E0_ERR_DEVICE, "routing rejected on the device (%s)",
                (err & DERR_INDEX) ? "expert index out of range" : "duplicate expert in a token");
  if (err & kDerrRange)
    return fail(E0_ERR_DEVICE, "one-launch decode: an activation beyond the fp16 operand range (|v| >= 65520); "
                               "e0_debug_force_general(ctx, 1) runs such steps on the per-layer kernels");
  return E0_OK;
}

// Host-side fault injection for the staging tests: the n-th next staging copy fails.
extern "C" int e0_debug_fail_staging_after(e0_ctx *C, int n) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  C->pool.fail_after = n;
  return E0_OK;
}

// Profiling: the next persistent decode launches write %globaltimer stamps into `buf`
// ([grid][L][16] uint64, caller-owned device memory; NULL turns it off).  Returns the grid.
extern "C" int e0_debug_decode_trace(e0_ctx *C, unsigned long long *buf) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  C->dec.trace = buf;
  return C->nsm;
}

// Select the expert path of e0_moe_layer_forward: 0 = tensor cores from kTcMinTokens
// tokens (default), 1 = CUDA-core kernels, 2 = tensor cores whenever the context has them.
extern "C" int e0_prefill_fixed_order(e0_ctx *C, int on) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  if (on && !C->ypart) {
    const size_t n = (size_t)(C->dims.top_k + 1) * C->maxT * C->dims.d_model;
    int rc = dalloc(&C->ypart, n);
    if (rc) return rc;
  }
  C->pf_det = on != 0;
  return E0_OK;
}

extern "C" int e0_debug_prefill_path(e0_ctx *C, int mode) {
  if (!C || mode < 0 || mode > 2) return fail(E0_ERR_INVALID_ARG, "bad prefill path");
  C->prefill_path = mode;
  return E0_OK;
}

// Decode implementation: 0 = default, 1 = one-launch kernel (B = 1), 2 = CUDA-graph replay
// of the per-layer kernels, 3 = per-layer kernels launched one by one, 4 = phased kernels.
extern "C" int e0_debug_decode_mode(e0_ctx *C, int mode) {
  if (!C || mode < 0 || mode > 4) return fail(E0_ERR_INVALID_ARG, "bad decode mode");
  C->decode_mode = mode;
  return E0_OK;
}

// Profiling of the phased decode path: on = 1 launches its six kernels one after another
// (no programmatic overlap) with an event before each; e0_debug_phase_times adds up the
// kernels' durations over the timed steps.
extern "C" int e0_debug_phase_timing(e0_ctx *C, int on) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  C->ph.timing = on != 0;
  return E0_OK;
}

extern "C" int e0_debug_phase_times(e0_ctx *C, double *ms6, unsigned long long *steps) {
  if (!C || !ms6 || !steps) return fail(E0_ERR_INVALID_ARG, "NULL argument");
  PhState &S = C->ph;
  for (auto &v : S.pending) {
    CK(cudaEventSynchronize(v[6]));
    for (int q = 0; q < 6; q++) {
      float ms = 0.f;
      CK(cudaEventElapsedTime(&ms, v[q], v[q + 1]));
      S.ms[q] += ms;
    }
    S.steps_timed++;
    for (auto e : v) cudaEventDestroy(e);
  }
  S.pending.clear();
  for (int q = 0; q < 6; q++) ms6[q] = S.ms[q];
  *steps = S.steps_timed;
  return E0_OK;
}

// Schedule of the one-launch decode kernel on unchained steps: 1 = flat (default), 0 =
// layers in order.
extern "C" int e0_debug_decode_flat(e0_ctx *C, int on) {
  if (!C || on < 0 || on > 1) return fail(E0_ERR_INVALID_ARG, "bad decode schedule");
  C->dec.flat = on;
  return E0_OK;
}

// The one-launch decode kernel's item list of one CTA, built by the same host function
// that the context uses (no device call).
extern "C" int e0_decode_items(const e0_dims *dims, int n_layers, const uint8_t *has_head, const uint8_t *has_lora,
                               int n_ctas, int flat, int step0, int cta, uint64_t *items_out, int cap, int *n_out) {
  if (!dims || !has_head || !has_lora || !items_out || !n_out || n_layers < 1 || n_layers > 64 || n_ctas < 1 ||
      cta < 0 || cta >= n_ctas || cap < 0 || dims->d_model < 64 || dims->d_model % 64 || dims->d_ff < 64 ||
      dims->d_ff % 64 || dims->n_experts < 1 || dims->top_k < 1 || dims->top_k > kMaxK || dims->lora_rank < 0)
    return fail(E0_ERR_INVALID_ARG, "e0_decode_items: bad arguments");
  SchedShape Z{};
  Z.L = n_layers; Z.G = n_ctas; Z.E = dims->n_experts; Z.k = dims->top_k; Z.r = dims->lora_rank;
  Z.D = dims->d_model; Z.I = dims->d_ff;
  Z.ldh = dims->d_model + (dims->head_onehot ? 2 * dims->n_experts : 0);
  for (int l = 0; l < n_layers; l++) {
    Z.head[l] = has_head[l] != 0;
    Z.lora[l] = has_lora[l] != 0;
  }
  std::vector<unsigned long long> buf(kMaxItems);
  const int n = build_items(Z, flat != 0, step0 != 0, cta, buf.data());
  if (n < 0) return fail(E0_ERR_INVALID_ARG, "e0_decode_items: more than %d items for one CTA", kMaxItems);
  if (n > cap) return fail(E0_ERR_INVALID_ARG, "e0_decode_items: %d items, capacity %d", n, cap);
  for (int i = 0; i < n; i++) items_out[i] = buf[i];
  *n_out = n;
  return E0_OK;
}

// Select the decode implementation: 1 = general per-layer kernels only (comparisons).
extern "C" int e0_debug_force_general(e0_ctx *C, int on) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  C->force_general = on != 0;
  return E0_OK;
}

// Arm a one-shot wrong tag: the next staging into `pool_set` tags `slot` with `expert`
// (tests: the kernels must report the mismatch instead of reading the wrong blob).
extern "C" int e0_debug_set_slot_tag(e0_ctx *C, int pool_set, int slot, int expert) {
  if (!C || !C->pool.mem || pool_set < 0 || pool_set >= C->pool.nsets || slot < 0 || slot >= C->pool.slots)
    return fail(E0_ERR_INVALID_ARG, "bad slot");
  C->pool.corrupt_set = pool_set;
  C->pool.corrupt_slot = slot;
  C->pool.corrupt_tag = expert;
  return E0_OK;
}

// Streaming mode: 0 = prefetch from the head predictions made one token earlier
// (prediction as routing; layers without a predictor on demand), 1 = fully reactive:
// every layer routes with its own router and stages on demand after it ran.
extern "C" int e0_stream_mode(e0_ctx *C, int reactive) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  if (reactive != 0 && reactive != 1) return fail(E0_ERR_INVALID_ARG, "stream mode must be 0 or 1");
  if (C->pool.reactive != reactive) C->last_step = -1;      // the routing tables of the two modes differ: a new sequence starts
  C->pool.reactive = reactive;
  return E0_OK;
}

// Debug: record, for every streamed layer, the slot tags of its pool set at the point where
// its expert kernels read them (one cudaMemcpyAsync on the compute stream after the wait
// for the staging copies) into log[layer * slots + s]; NULL stops it.
extern "C" int e0_debug_stream_log(e0_ctx *C, int32_t *log) {
  if (!C) return fail(E0_ERR_INVALID_ARG, "NULL context");
  if (!C->pool.mem) return fail(E0_ERR_INVALID_ARG, "no host store registered");
  C->pool.log = log;
  return E0_OK;
}

// Debug: the device address of slot `slot` of pool set `set` (read its blob to check the
// staged bytes); E0_ERR_INVALID_ARG outside the pool.
extern "C" int e0_debug_pool_slot(e0_ctx *C, int set, int slot, void **out) {
  if (!C || !out) return fail(E0_ERR_INVALID_ARG, "NULL argument");
  const StreamPool &P = C->pool;
  if (!P.mem || set < 0 || set >= P.nsets || slot < 0 || slot >= P.slots)
    return fail(E0_ERR_INVALID_ARG, "no such pool slot");
  *out = P.mem + ((size_t)set * P.slots + slot) * P.bytes;
  return E0_OK;
}

// ---------------------------------------------------------------------------------------
// One MoE block without any allocation.
//
// Some callers cannot call cudaMalloc: a serving runtime that fixes its whole memory plan at
// start-up and forbids allocation afterwards, code that runs while another component owns
// the device allocator, or code that must not trigger the implicit device synchronisation
// an allocation can cause.  This entry point needs no context and allocates nothing: its
// intermediates live in one file-scope device array of fixed size, which every GPU that
// loads this library holds until the process exits.
// ---------------------------------------------------------------------------------------
static constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;   // 4 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
// The device address of g_noalloc_scratch belongs to the library's module as loaded in one
// CUDA context: the host-side symbol is not an address a kernel may use, and a device
// reset or another (non-primary) context on the same device loads the module again at
// another address.  So the address is looked up once per context, keyed by the context's
// process-unique id (cuCtxGetId; a handle value can be reused after a reset), and kept in
// a small table that a mutex guards against concurrent first calls from several host
// threads.
static constexpr int kNoAllocMaxContexts = 64;
struct NoAllocEntry {
  unsigned long long ctx_id;
  unsigned char *base;
  int nsm;
};
static NoAllocEntry g_noalloc_tab[kNoAllocMaxContexts];
static int g_noalloc_n = 0;
static std::mutex g_noalloc_mu;

// The scratch array's address and the SM count for the calling thread's current context.
static int noalloc_scratch(unsigned char **base, int *nsm) {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!get_cur || !get_id) {
    void *f1 = nullptr, *f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || !f1 ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess || !f2)
      return fail(E0_ERR_CUDA, "noalloc forward: cuCtxGetCurrent / cuCtxGetId are not available");
    get_cur = (PFN_cuCtxGetCurrent_v4000)f1;
    get_id = (PFN_cuCtxGetId_v12000)f2;
  }
  int dev = 0;
  CK(cudaGetDevice(&dev));
  CUcontext cur = nullptr;
  unsigned long long id = 0;
  if (get_cur(&cur) != CUDA_SUCCESS || !cur) {
    // no context current on this thread yet: the symbol lookup below makes the runtime's
    // primary context current
    void *p = nullptr;
    CK(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    if (get_cur(&cur) != CUDA_SUCCESS || !cur) return fail(E0_ERR_CUDA, "noalloc forward: no current CUDA context");
  }
  if (get_id(cur, &id) != CUDA_SUCCESS) return fail(E0_ERR_CUDA, "noalloc forward: cuCtxGetId failed");
  for (int i = 0; i < g_noalloc_n; i++)
    if (g_noalloc_tab[i].ctx_id == id) {
      *base = g_noalloc_tab[i].base;
      *nsm = g_noalloc_tab[i].nsm;
      return E0_OK;
    }
  // first call in this context: look the address up (must not run inside a stream capture)
  void *p = nullptr;
  CK(cudaGetSymbolAddress(&p, g_noalloc_scratch));
  int n_sm = 0;
  CK(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
  NoAllocEntry &slot = g_noalloc_tab[g_noalloc_n < kNoAllocMaxContexts ? g_noalloc_n++ : (int)(id % kNoAllocMaxContexts)];
  slot = NoAllocEntry{id, (unsigned char *)p, n_sm};
  *base = slot.base;
  *nsm = slot.nsm;
  return E0_OK;
}

static size_t noalloc_align(size_t v) { return (v + 255) & ~(size_t)255; }

extern "C" int e0_moe_layer_forward_noalloc(const e0_dims *dims, const e0_layer *layer, const void *h, int T,
                                            const int32_t *route_idx, void *y_bf16, float *y_f32,
                                            int32_t *idx_out, float *gate_out, int *dev_status, void *stream) {
  if (!dims || !layer || !h || !y_bf16 || T < 1) return fail(E0_ERR_INVALID_ARG, "noalloc forward: bad arguments");
  if (!supported(*dims) || dims->head_hidden < 0)
    return fail(E0_ERR_INVALID_ARG, "noalloc forward: unsupported dims");
  const e0_layer &Y = *layer;
  if (!Y.experts || !Y.shared || !Y.router_w || !Y.norm_w)
    return fail(E0_ERR_INVALID_ARG, "noalloc forward: experts, shared, router_w and norm_w are required");
  const bool any = Y.lora_Ag || Y.lora_Bg || Y.lora_Au || Y.lora_Bu || Y.lora_Ad || Y.lora_Bd;
  const bool all = Y.lora_Ag && Y.lora_Bg && Y.lora_Au && Y.lora_Bu && Y.lora_Ad && Y.lora_Bd;
  if (any && (!all || dims->lora_rank < 1))
    return fail(E0_ERR_INVALID_ARG, "noalloc forward: LoRA needs all six matrices and lora_rank >= 1");
  const e0_dims &D = *dims;
  const size_t d = D.d_model, E = D.n_experts, I = D.d_ff, k = D.top_k, r = D.lora_rank > 0 ? D.lora_rank : 1;
  // scratch layout (each region 256-byte aligned)
  size_t off = 0;
  const size_t o_err = off;    off += noalloc_align(sizeof(int));
  const size_t o_xb = off;     off += noalloc_align((size_t)T * d * 2);
  const size_t o_xf = off;     off += noalloc_align((size_t)T * d * 4);
  const size_t o_log = off;    off += noalloc_align((size_t)T * E * 4);
  const size_t o_lt = off;     off += noalloc_align((size_t)T * 3 * r * 4);
  const size_t o_idx = off;    off += noalloc_align((size_t)T * k * 4);
  const size_t o_gate = off;   off += noalloc_align((size_t)T * k * 4);
  const size_t o_a = off;      off += noalloc_align((size_t)T * (k + 1) * I * 2);
  const size_t o_plan = off;   off += noalloc_align((1 + 2 * E + 1 + (size_t)T * k) * 4);
  if (off > kNoAllocScratchBytes)
    return fail(E0_ERR_INVALID_ARG,
                "noalloc forward: T=%d needs %zu bytes of scratch, the fixed maximum is %zu bytes", T, off,
                kNoAllocScratchBytes);
  unsigned char *base = nullptr;
  int nsm = 0;
  if (int rc = noalloc_scratch(&base, &nsm)) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  int *err = dev_status ? dev_status : (int *)(base + o_err);
  if (!dev_status) CK(cudaMemsetAsync(err, 0, sizeof(int), s));
  uint16_t *xb = (uint16_t *)(base + o_xb);
  float *xf = (float *)(base + o_xf), *logits = (float *)(base + o_log), *lt = (float *)(base + o_lt);
  int32_t *idx = idx_out ? idx_out : (int32_t *)(base + o_idx);
  float *gates = gate_out ? gate_out : (float *)(base + o_gate);
  uint16_t *a = (uint16_t *)(base + o_a);
  int32_t *pm = (int32_t *)(base + o_plan);
  Plan plan{pm, pm + 1, pm + 1 + E, pm + 2 + 2 * E};
  const int full_mode = route_idx ? 2 : 1;
#define NOALLOC_CKL(what)                                                                    \
  do {                                                                                     \
    cudaError_t e_ = cudaGetLastError();                                                   \
    if (e_ != cudaSuccess) return fail(E0_ERR_CUDA, "launch %s: %s", what, cudaGetErrorString(e_)); \
  } while (0)
  k_norm<<<T, 256, 0, s>>>((const uint16_t *)h, nullptr, (const uint16_t *)Y.norm_w, D.d_model, D.rms_eps, xb, xf);
  NOALLOC_CKL("k_norm");
  RowsArgs R{};
  R.xf = xf; R.T = T; R.d = D.d_model; R.E = D.n_experts; R.k = D.top_k;
  R.Wr = (const uint16_t *)Y.router_w; R.logits = logits; R.route = route_idx; R.full_mode = full_mode;
  R.Wh = nullptr; R.hlog = nullptr;
  R.Ag = (const uint16_t *)Y.lora_Ag; R.Au = (const uint16_t *)Y.lora_Au; R.r = D.lora_rank; R.lt = lt; R.err = err;
  const int nTT = (T + kRowTile - 1) / kRowTile;
  const int J = D.n_experts * nTT + T * D.top_k + (R.Ag ? 2 * D.lora_rank * nTT : 0);
  k_rows<<<grid_for(J, 8 * nsm), 256, 0, s>>>(R);
  NOALLOC_CKL("k_rows");
  RouteArgs A{};
  A.logits = logits; A.T = T; A.E = D.n_experts; A.k = D.top_k; A.route = route_idx; A.full_mode = full_mode;
  A.idx = idx; A.gates = gates; A.err = err;
  k_route<<<(T + 7) / 8, 256, 0, s>>>(A);
  NOALLOC_CKL("k_route");
  k_plan<<<1, 1024, 0, s>>>(idx, T * D.top_k, D.n_experts, plan);
  NOALLOC_CKL("k_plan");
  ExpertSrc src{};
  src.resident = (const uint8_t *)Y.experts;
  src.stride = blob_of(D.d_model, D.d_ff).bytes;
  src.err = err;
  GateUpArgs G{};
  G.xf = xf; G.T = T; G.d = D.d_model; G.I = D.d_ff; G.k = D.top_k; G.r = D.lora_rank; G.c = D.lora_scale;
  G.src = src; G.shared = (const uint8_t *)Y.shared; G.bl = blob_of(D.d_model, D.d_ff); G.P = plan;
  G.Bg = (const uint16_t *)Y.lora_Bg; G.Bu = (const uint16_t *)Y.lora_Bu; G.lt = lt; G.a = a;
  const int items = (std::min(D.n_experts, T * D.top_k) + 1) * D.d_ff;
  k_gateup<<<grid_for(items, 4 * nsm), 256, 0, s>>>(G);
  NOALLOC_CKL("k_gateup");
  if (Y.lora_Ad) {
    k_lora_t<<<(T * D.lora_rank + 7) / 8, 256, 0, s>>>((const uint16_t *)Y.lora_Ad, a, T, D.d_ff, D.top_k,
                                                        D.lora_rank, lt);
    NOALLOC_CKL("k_lora_t");
  }
  DownArgs W{};
  W.T = T; W.d = D.d_model; W.I = D.d_ff; W.k = D.top_k; W.r = D.lora_rank; W.c = D.lora_scale;
  W.src = src; W.shared = (const uint8_t *)Y.shared; W.bl = blob_of(D.d_model, D.d_ff); W.idx = idx; W.gates = gates;
  W.a = a; W.Bd = (const uint16_t *)Y.lora_Bd; W.lt = lt; W.y = (uint16_t *)y_bf16; W.yf = y_f32;
  k_down<<<grid_for(T * D.d_model, 4 * nsm), 256, 0, s>>>(W);
  NOALLOC_CKL("k_down");
#undef NOALLOC_CKL
  return E0_OK;
}
