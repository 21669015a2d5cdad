// Host side of the MoE decode library: layer object, launch plans,
// programmatic-dependent-launch chaining, the shared-expert side stream and
// the C ABI declared in include/moe_decode.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <utility>

#include "../../include/moe_decode.h"
#include "gemv.cuh"
#include "kernels.cuh"
#include "mma_grouped.cuh"
#include "mx_umma.cuh"
#include "dense_umma.cuh"
#include "persistent.cuh"

using namespace moe;

namespace {

constexpr int kSmemBudget = 227 * 1024;  // dynamic shared memory per CTA (1 CTA per SM)
constexpr int kMaxStages = kMaxStagesDev;
constexpr int kXBudget = 64 * 1024;       // staged activation vectors
constexpr int kPrefetchBytes = 64 * 1024; // stages kept in flight ahead of the consumers
constexpr int kRouterBucketBytes = kBucketScratchBytes + kTopkCandBytes;  // routing finish scratch

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

enum Kind { K_ROUTER = 0, K_SGU = 1, K_SDN = 2, K_GU = 3, K_DN = 4, K_DNC = 5, K_SGU_MX = 6, K_SDN_MX = 7,
            K_NUM = 8 };

// Fixed per weight stream: weight format, epilogue, activation type, output
// rows per warp row, warps per item, and how many of those warps split K
// (item rows = rpw * wpi / ks).
struct KindTraits { int wf, epi, xk, rpw, wpi, ks; };
#ifndef MOE_DENSE_KSPLIT
#define MOE_DENSE_KSPLIT 4
#endif
#ifndef MOE_GU_RPW
#define MOE_GU_RPW 1
#endif
#ifndef MOE_GU_WPI
#define MOE_GU_WPI 4
#endif
#ifndef MOE_DN_RPW
#define MOE_DN_RPW 4
#endif
#ifndef MOE_DN_WPI
#define MOE_DN_WPI 4
#endif
constexpr KindTraits kTraits[K_NUM] = {
    // router: 2 rows (28 KB) per item, K split over 4 warps
    {W_BF16, EPI_ROUTER, X_BF16, 2, MOE_DENSE_KSPLIT, MOE_DENSE_KSPLIT},
    // shared gate/up: 1 output row (2 x 14 KB), K split over 4 warps
    {W_BF16, EPI_SWIGLU, X_BF16, 1, MOE_DENSE_KSPLIT, MOE_DENSE_KSPLIT},
    {W_BF16, EPI_STORE, X_F32, 2, 4, 1},          // shared down: 8 rows (32 KB)
    {W_MXFP4, EPI_SWIGLU, X_BF16, MOE_GU_RPW, MOE_GU_WPI, 1},       // routed gate/up: 4 output rows (2 x 14 KB)
    {W_MXFP4, EPI_STORE, X_F32, MOE_DN_RPW, MOE_DN_WPI, 1},         // routed down: 16 rows (16 KB)
    {W_MXFP4, EPI_DOWN_COMBINE, X_F32, MOE_DN_RPW, MOE_DN_WPI, 1},  // routed down + combine
    // MXFP4 shared expert: the routed instances in dense mode (every token, one group)
    {W_MXFP4, EPI_SWIGLU, X_BF16, MOE_GU_RPW, MOE_GU_WPI, 1},
    {W_MXFP4, EPI_STORE, X_F32, MOE_DN_RPW, MOE_DN_WPI, 1},
};

struct GemvPlan {
  bool ok = false;
  int K = 0, out_rows = 0, R = 0, ncw = 0, wpi = 0, n_stages = 0, stage_bytes = 0, stage_offset = 0, x_offset = 0;
  int xcap = 0, scales_global = 0, threads = 0, smem = 0, ksplit = 1;
  bool fast = false;  // run the shape-specialised one-token instance
};

// Work decomposition of one weight stream.  `slots_needed` = activation
// vectors the stream can address (B, or B*k for the down projection),
// `max_groups` = most groups (experts) the stream can have active,
// `tok_per_group` = most activation vectors one group uses.
// Row quarters of the split-K (one-token MXFP4) instances: an item is
// kSplitKRows / (2 for SwiGLU) rows per warp times this many warp rows, each
// spread over the K slices.  Gate/up: 4 gate + 4 up rows (2 x 14 KB codes);
// down: 32 rows (32 KB).
#ifndef MOE_SPLITK_GU
#define MOE_SPLITK_GU 0  // gate/up: 0 = whole rows per warp (faster there), 1 = split-K
#endif
#ifndef MOE_SPLITK_GU_RQ
#define MOE_SPLITK_GU_RQ 1
#endif
#ifndef MOE_SPLITK_DN_RQ
#define MOE_SPLITK_DN_RQ 4
#endif

GemvPlan make_plan(Kind kind, int K, int out_rows, int slots_needed, int max_groups, int tok_per_group,
                   long long s_gstride, int num_sms, bool fast = false, bool splitk_ok = true) {
  GemvPlan p;
  KindTraits t = kTraits[kind];
  const bool mx = t.wf == W_MXFP4;
  const bool swiglu = t.epi == EPI_SWIGLU;
  const bool splitk = splitk_ok && fast && mx && (!swiglu || MOE_SPLITK_GU);  // warps = row quarters x K slices
  if (splitk) {
    const int ks = (K / 32 + 31) / 32;
    const int rq = swiglu ? MOE_SPLITK_GU_RQ : MOE_SPLITK_DN_RQ;
    t.rpw = swiglu ? kSplitKRows / 2 : kSplitKRows;
    t.wpi = rq * ks;
  }
  // bf16 K split: only where the 16-byte chunks divide evenly over the slices
  if (t.ks > 1 && (K / 8) % t.ks != 0) {
    t.wpi /= t.ks;
    t.ks = 1;
  }
  const int R = t.rpw * t.wpi / (splitk ? (K / 32 + 31) / 32 : t.ks);
  if (K <= 0 || K % 32 || out_rows <= 0 || out_rows % R) return p;
  const int rowbytes = mx ? K / 2 : K * 2;
  const int sbytes = mx ? K / 32 : 0;
  const int rows = swiglu ? 2 * R : R;
  // scale rows go through TMA only when every copy is 16-byte aligned and sized
  // (the split-K instances read them from the stage: no other way)
  const bool sg = mx && (((long long)R * sbytes) % 16 != 0 || s_gstride % 16 != 0);
  if (splitk && sg) return p;
  const int stage = (int)align_up((size_t)rows * (rowbytes + (mx && !sg ? sbytes : 0)), 128);
  // activation slots: a CTA's contiguous item range spans at most
  // ceil(items per CTA / items per group) + 1 groups
  const int n_rt = out_rows / R;
  const long long items_per_cta = ((long long)max_groups * n_rt + num_sms - 1) / num_sms;
  const int groups_per_cta = (int)std::min<long long>(max_groups, (items_per_cta + n_rt - 1) / n_rt + 1);
  const int xrow = x_row_bytes(t.wf, t.xk, K);
  int xcap = std::min(slots_needed, groups_per_cta * tok_per_group);
  xcap = std::min(std::min(xcap, kMaxSlots), std::max(1, kXBudget / xrow));
  const int hdr = (int)align_up(16 * 64 + sizeof(PhaseTable) + (kMaxSlots + 2 + kMaxStagesDev + kMaxStageUnits + kMaxWarpsAny * kPubInts + kRedFloats) * 4, 128);
  const int x_off = hdr;
  const int st_off = (int)align_up((size_t)x_off + (size_t)xcap * xrow, 128);
  int ns = std::min(kMaxStages, (kSmemBudget - st_off) / stage);
  if (ns < 2) return p;
  const int pf = std::max(1, (kPrefetchBytes + stage - 1) / stage);
  // consumer warps: whole groups of wpi, at most ns - pf groups consuming at once.
  // Items go to the groups round robin, so the ring holds a multiple of the
  // group count: every stage is then always consumed by the same group, in
  // item order, and a group never waits on a stage whose previous phase
  // another group has not finished.
  const int max_warps = splitk ? kMaxSplitKWarps : consumer_warps_for(t.wf, t.epi);
  if (t.wpi > max_warps || t.wpi < kMinItemWarps) return p;
  int groups = std::max(1, std::min(std::min(max_warps / t.wpi, kMaxItemGroups), std::max(1, ns - pf)));
  while (groups > 1 && (ns / groups) * groups - groups < pf) --groups;
  ns = (ns / groups) * groups;
  p.ok = true;
  p.K = K;
  p.out_rows = out_rows;
  p.R = R;
  p.wpi = t.wpi;
  p.ncw = groups * t.wpi;
  p.n_stages = ns;
  p.stage_bytes = stage;
  p.stage_offset = st_off;
  p.x_offset = x_off;
  p.xcap = xcap;
  p.scales_global = sg ? 1 : 0;
  p.threads = (p.ncw + 1) * 32;
  p.smem = st_off + ns * stage;
  // the router kernel's last CTA builds the buckets in its idle stage ring
  if (kind == K_ROUTER) p.smem = std::max(p.smem, st_off + kRouterBucketBytes);
  if (p.smem > kSmemBudget) return GemvPlan{};
  p.fast = fast;
  p.ksplit = splitk ? 1 : t.ks;
  return p;
}

typedef void (*GemvFn)(const GemvArgs);

// Reduction lengths with shape-specialised instances (the full-size layer).
constexpr int kFastH = 7168;
constexpr int kFastI = 2048;

template <int TMAX, int KH, int KI, bool kSplitDn = true>
GemvFn pick_fn(Kind k) {
  switch (k) {
    case K_ROUTER: return gemv_kernel<W_BF16, EPI_ROUTER, X_BF16, TMAX, 2, KH>;
    case K_SGU: return gemv_kernel<W_BF16, EPI_SWIGLU, X_BF16, TMAX, 1, KH>;
    case K_SDN: return gemv_kernel<W_BF16, EPI_STORE, X_F32, TMAX, 2, KI>;
    // instances with a compile-time K and one token are the split-K ones
    case K_GU:
    case K_SGU_MX:
      return gemv_kernel<W_MXFP4, EPI_SWIGLU, X_BF16, TMAX, (KH && TMAX == 1 && MOE_SPLITK_GU) ? kSplitKRows / 2 : MOE_GU_RPW, KH>;
    case K_DN:
    case K_SDN_MX:
      return gemv_kernel<W_MXFP4, EPI_STORE, X_F32, TMAX, (KI && TMAX == 1 && kSplitDn) ? kSplitKRows : MOE_DN_RPW, KI>;
    case K_DNC:
      return gemv_kernel<W_MXFP4, EPI_DOWN_COMBINE, X_F32, TMAX,
                         (KI && TMAX == 1 && kSplitDn) ? kSplitKRows : MOE_DN_RPW, KI>;
    default: return nullptr;
  }
}

// fast = the shape-specialised one-token instance (K must be kFastI for the
// down projections, kFastH for the others)
// small = the one-token-per-pass plans of batches 2..kSmallBatch (no split-K:
// those instances take exactly one token per item)
GemvFn gemv_fn(Kind k, int tmax, bool fast = false, bool small = false) {
  if (tmax == 1) {
    if (!fast) return pick_fn<1, 0, 0>(k);
    return small ? pick_fn<1, kFastH, kFastI, false>(k) : pick_fn<1, kFastH, kFastI>(k);
  }
  return pick_fn<2, 0, 0>(k);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The dynamic shared-memory limit of a kernel instance is a per-device
// property shared by every layer (and the allocation-free router): it is
// raised to what a plan needs and never lowered, so that creating a layer
// whose plans need less cannot make the launches of an earlier layer fail.
std::mutex g_smem_mu;
std::map<std::pair<int, const void*>, int> g_smem_limit;

cudaError_t raise_smem_limit(const void* fn, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_smem_mu);
  int& cur = g_smem_limit[std::make_pair(dev, fn)];
  if (bytes <= cur) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) cur = bytes;
  return e;
}

}  // namespace

// ---------------------------------------------------------------------------
// Allocation-free router/top-k: its only scratch (the fp32 logits, the top-k
// kernel's CTA counter and an error word) lives in this file-scope device
// array.  Host code must not use the array's name as a device address; the
// address comes from cudaGetSymbolAddress, once per device.
namespace {
constexpr int kNoAllocMaxLogits = kMaxBatch * kMaxExperts;  // 65536 floats (B * E)
struct NoAllocScratch {
  float logits[kNoAllocMaxLogits];
  int done_counter;
  int err;
};
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};
int g_noalloc_sms[kNoAllocMaxDevices] = {};
}  // namespace
static __device__ __align__(256) unsigned char g_noalloc_scratch[sizeof(NoAllocScratch)];

struct moe_layer {
  moe_layer_config cfg{};
  moe_layer_weights w{};
  int device = 0;
  int num_sms = 0;
  bool pdl = true;
  bool side_stream = false;
  bool prefetch = true;
  bool sigmoid = false;  // router scoring (MOE_FLAG_ROUTER_SIGMOID)
  bool shared_mx = false; // the shared expert's weights are MXFP4
  int persist = 0;        // persistent batch-1 kernel: 0 off, 1 generic instance, 2 shape-specialised
  int* grid_bar = nullptr;
  char* arena = nullptr;
  uint16_t* wr_t = nullptr;  // router matrix, expert-major [E][H]
  float* logits = nullptr;
  moe_routing plan{};
  float* h = nullptr;
  float* y = nullptr;
  float* hs = nullptr;
  float* ys = nullptr;
  int* router_cnt = nullptr;
  int* pub_cnt = nullptr;     // [2]: router CTAs with outputs published, shared-down CTAs past the wait
  int* tile_cnt = nullptr;
  __half* xh = nullptr;       // grouped path: f16 copy of the activations of one projection
  int* xe = nullptr;          // ... and its per-row exponents
  int mma_stages[2] = {0, 0};  // grouped path ring depth: [gate/up, down] (0 = not usable)
  bool grouped = false;
  // tcgen05 block-scaled expert path: tensor maps over the weights and over
  // the activation-term buffers, and the buffers themselves
  bool mx = false;         // the shapes allow it and its scale copies exist
  bool mx_forced = false;  // MOE_FLAG_MX_EXPERTS: at every batch size
  bool mx_default = false; // above batch 1 unless MOE_FLAG_NO_GROUPED / MOE_FLAG_WARP_MMA
  CUtensorMap tm_agu{}, tm_adn{}, tm_bx{}, tm_bh{}, tm_bx8{}, tm_bh8{}, tm_bx128{}, tm_bh128{};
  bool swap = false;        // both projections take the swapped-operand kernels (H a multiple of 256)
  float* sw_ws = nullptr;   // their stream-K partial sums [num_sms][2][16 x 256]
  int* sw_cnt = nullptr;    // ... and per-unit part counters [(E + B*k/16 + 1) * max(I/128, H/256)]
  uint8_t* aqx = nullptr;   // E2M1 terms of x per pair position [MB*k*T][H/2]
  uint8_t* bsfx = nullptr;  // ... their scales, chunk layout [MB*k][H/128][512]
  uint8_t* aqh = nullptr;   // E2M1 terms of h [MB*k*T][I/2]
  uint8_t* bsfh = nullptr;  // ... their scales, chunk layout [MB*k][I/128][512]
  // dense bf16 streams on tcgen05 above batch 1 (router + shared expert)
  bool dense = false;
  CUtensorMap tm_wr{}, tm_sgu{}, tm_sdn{}, tm_ht{};
  uint16_t* hterms = nullptr;  // bf16 terms of h_s [MB * kDnHTerms][I_s]
  float* dws1 = nullptr;       // stream-K partials of the router + shared gate/up launch
  float* dws2 = nullptr;       // ... of the shared down launch
  int dparts1 = 0, dparts2 = 0;
  int* dtile_cnt = nullptr;    // [tiles of both launches]
  char* dense_mem = nullptr;
  char* mx_mem = nullptr;   // the weight scales in chunk layout (copied at create):
  uint8_t* wsf_gu = nullptr;  // gate/up [E * 2I/128][H/128][512]
  uint8_t* wsf_dn = nullptr;  // down [E * H/128][I/128][512]
  int* err = nullptr;
  uint16_t* x_stage = nullptr;
  uint16_t* res_stage = nullptr;
  uint16_t* out_stage = nullptr;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  cudaEvent_t probe_start = nullptr, probe_stop = nullptr;
  GemvPlan plans[K_NUM][3];  // [kind][plan slot: 0 batch 1, 1 two tokens per pass, 2 small batches]
};

namespace {

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Batches 2..kSmallBatch take one token per pass (most of their experts see
// one token) on the compile-time-K instances; larger ones two per pass.
// The dense bf16 streams keep two tokens per pass there.
constexpr int kSmallBatch = 8;
bool routed_kind(Kind k) { return k == K_GU || k == K_DN || k == K_DNC; }
// The routed down projection at batch 1 takes the one-token plans of the
// small batches (whole rows per warp): measured faster there than the
// split-K instance, whose cross-warp reduction stalls on barriers.
int slot_for(Kind k, int B) {
  if (B == 1 && (k == K_DN || k == K_DNC)) return 2;
  return B == 1 ? 0 : ((B <= kSmallBatch && routed_kind(k)) ? 2 : 1);
}
int tmax_of_slot(int t) { return t == 1 ? 2 : 1; }
int tmax_for(int B) { return B == 1 ? 1 : 2; }  // dense streams

template <typename... Args>
cudaError_t launch_ex(void (*kern)(Args...), dim3 grid, int block, int smem, cudaStream_t st, bool pdl,
                      Args... args) {
  cudaLaunchConfig_t c = {};
  c.gridDim = grid;
  c.blockDim = dim3(block);
  c.dynamicSmemBytes = (size_t)smem;
  c.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  c.attrs = attr;
  c.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&c, kern, args...);
}

GemvArgs base_args(const moe_layer* L, const GemvPlan& p) {
  GemvArgs a;
  std::memset(&a, 0, sizeof(a));
  a.K = p.K;
  a.out_rows = p.out_rows;
  a.R = p.R;
  a.ncw = p.ncw;
  a.wpi = p.wpi;
  a.n_stages = p.n_stages;
  a.stage_bytes = p.stage_bytes;
  a.stage_offset = p.stage_offset;
  a.x_offset = p.x_offset;
  a.xcap = p.xcap;
  a.scales_global = p.scales_global;
  a.ksplit = p.ksplit;
  a.top_k = L->cfg.top_k;
  a.n_experts = L->cfg.n_experts;
  a.err = L->err;
  return a;
}

cudaError_t run_gemv(moe_layer* L, Kind k, int B, const GemvArgs& a, cudaStream_t st, bool pdl, int grid = 0) {
  const int sl = slot_for(k, B);
  const GemvPlan& p = L->plans[k][sl];
  return launch_ex(gemv_fn(k, tmax_of_slot(sl), p.fast, sl == 2), grid > 0 ? grid : L->num_sms, p.threads, p.smem,
                   st, pdl, a);
}

const GemvPlan& plan_of(const moe_layer* L, Kind k, int B) { return L->plans[k][slot_for(k, B)]; }

bool routing_ok(const moe_routing* r) {
  return r && r->topk_idx && r->topk_w && r->counts && r->offsets && r->pair_ids && r->active && r->n_active;
}

// Router GEMV (logits, fp32) whose last CTA selects the top-k, computes the
// weights and builds the buckets.  with_shared: the shared expert's bf16
// gate/up rows ride along as extra items (same activation x), so the
// routing finish overlaps the shared expert's weight stream; h_s lands in
// L->hs.
GemvArgs router_args(const moe_layer* L, const void* x, int B, const moe_routing& r, bool with_shared) {
  const GemvPlan& p = plan_of(L, K_ROUTER, B);
  GemvArgs a = base_args(L, p);
  a.w = reinterpret_cast<const uint8_t*>(L->wr_t);
  a.act = x;
  a.routed = 0;
  a.n_tokens = B;
  a.out = L->logits;
  a.bias = L->sigmoid ? nullptr : L->w.router_bias;  // sigmoid scoring: the bias steers selection only
  a.scoring = L->sigmoid ? 1 : 0;
  a.sel_bias = L->sigmoid ? L->w.router_bias : nullptr;
  a.topk_w = r.topk_w;
  a.topk_idx = r.topk_idx;
  a.counts = r.counts;
  a.offsets_out = r.offsets;
  a.pair_ids_out = r.pair_ids;
  a.active_out = r.active;
  a.n_active_out = r.n_active;
  a.done_counter = L->router_cnt;
  if (with_shared) {
    a.w2 = reinterpret_cast<const uint8_t*>(L->w.shared_gate_up);
    a.out2 = L->hs;
    a.n_items2 = L->cfg.shared_inter;
    a.up_off2 = L->cfg.shared_inter;
  }
  return a;
}

cudaError_t launch_router(moe_layer* L, const void* x, int B, const moe_routing& r, cudaStream_t st,
                          bool with_shared = false) {
  GemvArgs a = router_args(L, x, B, r, with_shared);
  // the shared down projection launched next starts on this count (see launch_shared)
  if (with_shared && L->pdl) a.pub_counter = L->pub_cnt;
  return run_gemv(L, K_ROUTER, B, a, st, L->pdl);
}

GemvArgs shared_down_args(const moe_layer* L, int B, float* ys) {
  const bool mx = L->shared_mx;
  const GemvPlan& p = plan_of(L, mx ? K_SDN_MX : K_SDN, B);
  GemvArgs a = base_args(L, p);
  a.w = mx ? L->w.shared_mx_down : reinterpret_cast<const uint8_t*>(L->w.shared_down);
  a.sc = mx ? L->w.shared_mx_s_down : nullptr;
  a.act = L->hs;
  a.n_tokens = B;
  a.out = ys;
  return a;
}

// Shared expert: gate/up + SwiGLU, then down.  late: the gate/up kernel may
// read x before its predecessor completes (see GemvArgs::pdl_late).
// after_router: the down projection follows the router kernel that computed
// h_s; it starts once every router CTA has published (pub_cnt), overlapping
// the router's routing finish, and completes only after the router grid.
cudaError_t launch_shared(moe_layer* L, const void* x, int B, float* ys, cudaStream_t st, bool pdl,
                          bool late = false, bool down_only = false, bool after_router = false) {
  const int H = L->cfg.hidden, Is = L->cfg.shared_inter;
  const bool mx = L->shared_mx;
  const Kind kgu = mx ? K_SGU_MX : K_SGU, kdn = mx ? K_SDN_MX : K_SDN;
  if (!down_only) {
    const GemvPlan& p = plan_of(L, kgu, B);
    GemvArgs a = base_args(L, p);
    a.w = mx ? L->w.shared_mx_gate_up : reinterpret_cast<const uint8_t*>(L->w.shared_gate_up);
    a.sc = mx ? L->w.shared_mx_s_gate_up : nullptr;
    a.up_off = Is;
    a.act = x;
    a.n_tokens = B;
    a.out = L->hs;
    a.pdl_late = late && pdl ? 1 : 0;
    cudaError_t e = run_gemv(L, kgu, B, a, st, pdl);
    if (e != cudaSuccess) return e;
  }
  (void)H;
  GemvArgs d = shared_down_args(L, B, ys);
  if (after_router && pdl && L->num_sms > 1) {
    d.dep_counter = L->pub_cnt;
    d.dep_target = L->num_sms;  // the router's grid
    d.dep_pass = L->pub_cnt + 1;
    d.pdl_late = 1;
    // one CTA fewer than SMs: the router's last CTA keeps its SM for the
    // routing finish, and no CTA of this stream waits for that SM to free
    return run_gemv(L, kdn, B, d, st, pdl, L->num_sms - 1);
  }
  return run_gemv(L, kdn, B, d, st, pdl);
}

GemvArgs routed_args(const moe_layer* L, const GemvPlan& p, const moe_routing& r, int B) {
  GemvArgs a = base_args(L, p);
  a.routed = 1;
  a.n_pairs = B * L->cfg.top_k;
  a.n_active = r.n_active;
  a.active = r.active;
  a.offsets = r.offsets;
  a.pair_ids = r.pair_ids;
  return a;
}

// Batches above this size use the grouped tensor-core expert kernels (at or
// below it most experts see one token and the GEMV kernels are faster).
#ifndef MOE_GROUPED_MIN_BATCH
#define MOE_GROUPED_MIN_BATCH 8
#endif
constexpr int kGroupedMinBatch = MOE_GROUPED_MIN_BATCH;

cudaError_t launch_grouped(moe_layer* L, bool gate_up, int B, const moe_routing& r, const void* act, float* out,
                           cudaStream_t st);

cudaError_t launch_gate_up_streams(moe_layer* L, const void* x, int B, const moe_routing& r, cudaStream_t st);

// ---- tcgen05 block-scaled expert path -------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library); null if unavailable
EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2-D tiled map over a row-major matrix: `inner` elements per row, `rows`
// rows `row_bytes` apart; box = box_inner x box_rows; 128-byte swizzle
bool encode_map(CUtensorMap* m, CUtensorMapDataType t, const void* base, uint64_t inner, uint64_t rows,
                uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, t, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

struct MxPlan {
  int n_max, stage_bytes, n_stages, smem, off_up, off_b, off_sfa, off_sfb;
};

// B columns of one pass: the same for both projections of a call (the
// gate/up epilogue writes the down projection's scale chunks per pass)
int mx_n_max(int B) { return std::min(kMxNMax, (B * kMxTerms + 15) & ~15); }

// shared-memory ring of one projection: a stage holds the A tile(s), the B
// rows of one pass and the scale-factor chunks (two per operand)
MxPlan mx_plan(bool gate_up, int B) {
  MxPlan p;
  p.n_max = mx_n_max(B);
  p.off_up = gate_up ? kMxATile : 0;
  p.off_b = (gate_up ? 2 : 1) * kMxATile;
  p.off_sfa = p.off_b + (int)align_up((size_t)p.n_max * 128, 1024);
  p.off_sfb = p.off_sfa + (gate_up ? 4 : 2) * kMxChunkBytes;
  p.stage_bytes = (int)align_up((size_t)p.off_sfb + 2 * kMxChunkBytes, 1024);
  p.n_stages = std::min(gate_up ? kMxMaxStagesGU : kMxMaxStagesDn,
                        (kSmemBudget - 2 * kMxHeaderBytes) / p.stage_bytes);
  p.smem = 2 * kMxHeaderBytes + p.n_stages * p.stage_bytes;
  return p;
}

MxArgs mx_args(const moe_layer* L, bool gate_up, int B, const moe_routing& r, const MxPlan& p, float* out) {
  const int H = L->cfg.hidden, I = L->cfg.inter, k = L->cfg.top_k;
  MxArgs a;
  std::memset(&a, 0, sizeof(a));
  a.wsf = gate_up ? L->wsf_gu : L->wsf_dn;
  a.a_tiles = (gate_up ? 2 * I : H) / kMxRows;
  a.up_tile = gate_up ? I / kMxRows : 0;
  a.K = gate_up ? H : I;
  a.out_rows = gate_up ? I : H;
  a.top_k = k;
  a.n_pairs = B * k;
  a.n_experts = L->cfg.n_experts;
  a.n_active = r.n_active;
  a.active = r.active;
  a.offsets = r.offsets;
  a.pair_ids = r.pair_ids;
  a.bsf = gate_up ? L->bsfx : L->bsfh;
  a.n_max = p.n_max;
  a.out_f32 = out;
  a.next_aq = gate_up ? L->aqh : nullptr;
  a.next_bsf = gate_up ? L->bsfh : nullptr;
  a.next_rpp = L->swap ? kSwRowsPerTok : kMxTerms;
  a.n_stages = p.n_stages;
  a.stage_bytes = p.stage_bytes;
  a.off_up = p.off_up;
  a.off_b = p.off_b;
  a.off_sfa = p.off_sfa;
  a.off_sfb = p.off_sfb;
  a.err = L->err;
  return a;
}

// tokens per pass of the swapped kernels: every expert's (at most B) tokens
// below batch 16, 16 from there
int sw_tokens_per_pass(int B) { return std::min(B, kSwTokMax); }

// arguments of a swapped-operand projection, without its outputs; the stage
// ring holds the pass's activation rows, the two weight tiles and the scale
// chunks (two per operand tile)
SwArgs sw_args(const moe_layer* L, bool gate_up, int B, const moe_routing& r) {
  const int H = L->cfg.hidden, I = L->cfg.inter, k = L->cfg.top_k;
  SwArgs a;
  std::memset(&a, 0, sizeof(a));
  a.wsf = gate_up ? L->wsf_gu : L->wsf_dn;
  a.a_tiles = (gate_up ? 2 * I : H) / kMxRows;
  a.tile2 = gate_up ? I / kMxRows : 1;
  a.K = gate_up ? H : I;
  a.out_rows = gate_up ? I : H;
  a.n_rt = gate_up ? I / kMxRows : H / kSwN;
  a.top_k = k;
  a.n_pairs = B * k;
  a.n_experts = L->cfg.n_experts;
  a.n_active = r.n_active;
  a.active = r.active;
  a.offsets = r.offsets;
  a.pair_ids = r.pair_ids;
  a.asf = gate_up ? L->bsfx : L->bsfh;
  a.tpp = sw_tokens_per_pass(B);
  a.one_pass = B <= a.tpp ? 1 : 0;  // an expert holds at most B tokens
  a.off_w = (int)align_up((size_t)a.tpp * kSwRowsPerTok * 128, 1024);
  a.off_sfa = a.off_w + 2 * kMxATile;
  a.off_sfw = a.off_sfa + 2 * kMxChunkBytes;
  a.stage_bytes = (int)align_up((size_t)a.off_sfw + 4 * kMxChunkBytes, 1024);
  a.n_stages = std::min(kSwMaxStages, (kSmemBudget - 2 * kMxHeaderBytes - kSwTableBytes) / a.stage_bytes);
  a.ws = L->sw_ws;
  a.item_cnt = L->sw_cnt;
  a.err = L->err;
  return a;
}

int sw_smem(const SwArgs& a) { return 2 * kMxHeaderBytes + kSwTableBytes + a.n_stages * a.stage_bytes; }

// gate/up on the tensor cores: x -> E2M1 terms per pair position, then the
// block-scaled MMA kernel (h fp32 into `h`, and h's terms for the down kernel)
cudaError_t launch_mx_gate_up(moe_layer* L, const void* x, int B, const moe_routing& r, float* h, cudaStream_t st,
                              cudaEvent_t ev0, cudaEvent_t ev1) {
  const int H = L->cfg.hidden, k = L->cfg.top_k;
  // batch 1: every position holds the same token, whose terms are made once
  const int by_token = B == 1 ? 1 : 0;
  const dim3 grid(B, (H / 32 + 31) / 32);
  const int rpp = L->swap ? kSwRowsPerTok : kMxTerms;
  const int tpp = L->swap ? sw_tokens_per_pass(B) : mx_n_max(B) / kMxTerms;
  cudaError_t e = launch_ex(mx_x_terms_kernel<kMxTerms>, grid, 256, 0, st, L->pdl, static_cast<const uint16_t*>(x),
                            H, k, B * k, L->cfg.n_experts, tpp, rpp,
                            static_cast<const int*>(r.pair_ids), static_cast<const int*>(r.topk_idx),
                            static_cast<const int*>(r.offsets), by_token, L->aqx, L->bsfx, L->err);
  if (e != cudaSuccess) return e;
  if (L->swap) {
    // gate/up writes h in fp32 (L->h); a small kernel then makes its terms
    // for the down projection (the conversion costs far more CUDA-core time
    // in the gate/up epilogue, beside the running copies and MMAs)
    SwArgs a = sw_args(L, true, B, r);
    a.a_by_token = by_token;
    a.h = L->h;
    a.h_only = 1;
    (void)h;
    a.next_aq = L->aqh;
    a.next_bsf = L->bsfh;
    if (ev0 && (e = cudaEventRecord(ev0, st)) != cudaSuccess) return e;
    e = launch_ex(mx_swap_kernel<true, kMxTerms>, L->num_sms, kMxThreads, sw_smem(a), st, L->pdl, L->tm_agu,
                  L->tm_bx8, L->tm_bx128, a);
    if (e == cudaSuccess && ev1) e = cudaEventRecord(ev1, st);
    if (e != cudaSuccess) return e;
    const int I = L->cfg.inter;
    const long long n_thr = (long long)B * k * (I / 32) * 8;
    return launch_ex(mx_h_terms_kernel<kMxTerms>, (int)((n_thr + 255) / 256), 256, 0, st, L->pdl,
                     static_cast<const float*>(L->h), I, k, B * k, L->cfg.n_experts, sw_tokens_per_pass(B),
                     kSwRowsPerTok, static_cast<const int*>(r.pair_ids), static_cast<const int*>(r.topk_idx),
                     static_cast<const int*>(r.offsets), L->aqh, L->bsfh, L->err);
  }
  const MxPlan p = mx_plan(true, B);
  MxArgs a = mx_args(L, true, B, r, p, h);
  a.b_by_token = by_token;
  if (ev0 && (e = cudaEventRecord(ev0, st)) != cudaSuccess) return e;
  e = launch_ex(mx_expert_kernel<true, kMxTerms>, L->num_sms, kMxThreads, p.smem, st, L->pdl, L->tm_agu, L->tm_bx,
                a);
  if (e == cudaSuccess && ev1) e = cudaEventRecord(ev1, st);
  return e;
}

// down projection with the operands swapped; with `residual` non-null fused
// with the combine (and the next layer's L2 prefetch)
cudaError_t launch_mx_down_swap(moe_layer* L, int B, const moe_routing& r, float* y, cudaStream_t st,
                                const void* residual, void* out, const float* ys, const moe_layer* next) {
  SwArgs a = sw_args(L, false, B, r);
  a.y = y;
  if (residual) {
    a.comb_w = r.topk_w;
    a.y_shared = ys;
    a.residual = static_cast<const uint16_t*>(residual);
    a.out_bf16 = static_cast<uint16_t*>(out);
    a.batch = B;
    a.tile_counter = L->tile_cnt;
  }
  if (next && L->prefetch) {
    a.pf_ptr[0] = reinterpret_cast<const uint8_t*>(next->wr_t);
    a.pf_bytes[0] = (long long)next->cfg.n_experts * next->cfg.hidden * 2;
    if (next->cfg.shared_inter > 0) {
      a.pf_ptr[1] = reinterpret_cast<const uint8_t*>(next->w.shared_gate_up);
      a.pf_bytes[1] = (long long)2 * next->cfg.shared_inter * next->cfg.hidden * 2;
    }
  }
  return launch_ex(mx_swap_kernel<false, kMxTerms>, L->num_sms, kMxThreads, sw_smem(a), st, L->pdl, L->tm_adn,
                   L->tm_bh8, L->tm_bh128, a);
}

// down projection on the tensor cores; with `residual` non-null fused with
// the combine (and the next layer's L2 prefetch)
cudaError_t launch_mx_down(moe_layer* L, int B, const moe_routing& r, float* y, cudaStream_t st,
                           const void* residual = nullptr, void* out = nullptr, const float* ys = nullptr,
                           const moe_layer* next = nullptr) {
  if (L->swap) return launch_mx_down_swap(L, B, r, y, st, residual, out, ys, next);
  const MxPlan p = mx_plan(false, B);
  MxArgs a = mx_args(L, false, B, r, p, y);
  if (residual) {
    a.comb_w = r.topk_w;
    a.y_shared = ys;
    a.residual = static_cast<const uint16_t*>(residual);
    a.out_bf16 = static_cast<uint16_t*>(out);
    a.batch = B;
    a.tile_counter = L->tile_cnt;
    if (next && L->prefetch) {
      a.pf_ptr[0] = reinterpret_cast<const uint8_t*>(next->wr_t);
      a.pf_bytes[0] = (long long)next->cfg.n_experts * next->cfg.hidden * 2;
      if (next->cfg.shared_inter > 0) {
        a.pf_ptr[1] = reinterpret_cast<const uint8_t*>(next->w.shared_gate_up);
        a.pf_bytes[1] = (long long)2 * next->cfg.shared_inter * next->cfg.hidden * 2;
      }
    }
  }
  return launch_ex(mx_expert_kernel<false, kMxTerms>, L->num_sms, kMxThreads, p.smem, st, L->pdl, L->tm_adn,
                   L->tm_bh, a);
}

// Kernels of a call's routed experts: the tcgen05 kernels where forced, and
// by default above batch 1 (at batch 1 the CUDA-core GEMVs are as fast);
// else the grouped warp-MMA kernels above kGroupedMinBatch, else the GEMVs.
int expert_path(const moe_layer* L, int B) {
  if (L->mx && (L->mx_forced || (B > 1 && L->mx_default))) return MOE_PATH_TCGEN05;
  if (B > kGroupedMinBatch && L->grouped) return MOE_PATH_GROUPED;
  return MOE_PATH_GEMV;
}

// ---- dense bf16 streams on tcgen05 (batches above 1) ----------------------
// Above batch 1, where the routed experts run on the tcgen05 kernels and no
// side stream is used: the router and the bf16 shared expert's gate/up in one
// launch, the shared down projection in a second, then the routing finish.
bool dense_for(const moe_layer* L, int B) {
  return L->dense && B > 1 && !L->side_stream && expert_path(L, B) == MOE_PATH_TCGEN05;
}

int dn_tiles_k1(const moe_layer* L) {
  const int E = L->cfg.n_experts, Is = L->cfg.shared_inter;
  return (E + kDnRows - 1) / kDnRows + ((Is > 0 && !L->shared_mx) ? Is / kDnRows : 0);
}

void dn_fill_plan(DenseArgs& a) {
  const bool glu = a.n_streams > 1 ? (a.st[0].up_rows || a.st[1].up_rows) : a.st[0].up_rows != 0;
  a.off_up = glu ? kDnATile : 0;
  a.off_b = (glu ? 2 : 1) * kDnATile;
  a.stage_bytes = (int)align_up((size_t)a.off_b + (size_t)a.n * 128, 1024);
  a.n_stages = std::min(kDnMaxStages, (kSmemBudget - 2 * kDnHeaderBytes) / a.stage_bytes);
}

int dn_smem(const DenseArgs& a) { return 2 * kDnHeaderBytes + a.n_stages * a.stage_bytes; }

// the router's tiles (stream 0), then the bf16 shared expert's gate/up tiles
// (stream 1); skip_mask: the streams left out (the staged entry points),
// with the same split of the rest as the fused launch, so the same sums
enum { kDnSkipRouter = 1, kDnSkipShared = 2 };
DenseArgs dn_args_k1(const moe_layer* L, int B, int skip_mask = 0) {
  DenseArgs a;
  std::memset(&a, 0, sizeof(a));
  const int E = L->cfg.n_experts, Is = L->cfg.shared_inter;
  a.st[0].n_tiles = (E + kDnRows - 1) / kDnRows;
  a.st[0].out_rows = E;
  a.st[0].out = L->logits;
  a.st[0].bias = L->sigmoid ? nullptr : L->w.router_bias;  // sigmoid scoring: the bias steers selection only
  a.n_streams = 1;
  if (Is > 0 && !L->shared_mx) {
    DenseStream& g = a.st[1];
    g.n_tiles = Is / kDnRows;
    g.up_rows = Is;
    g.out_rows = Is;
    g.out = L->hs;
    g.next_terms = L->hterms;
    a.n_streams = 2;
  }
  a.skip_mask = skip_mask & ((1 << a.n_streams) - 1);
  a.K = L->cfg.hidden;
  a.B = B;
  a.terms = 1;
  a.n = (B + 15) & ~15;
  a.ws = L->dws1;
  a.ws_parts = L->dparts1;
  a.tile_cnt = L->dtile_cnt;
  a.err = L->err;
  dn_fill_plan(a);
  return a;
}

DenseArgs dn_args_sdn(const moe_layer* L, int B, float* ys) {
  DenseArgs a;
  std::memset(&a, 0, sizeof(a));
  const int H = L->cfg.hidden;
  a.st[0].n_tiles = H / kDnRows;
  a.st[0].out_rows = H;
  a.st[0].out = ys;
  a.n_streams = 1;
  a.K = L->cfg.shared_inter;
  a.B = B;
  a.terms = kDnHTerms;
  a.n = (B * kDnHTerms + 15) & ~15;
  a.ws = L->dws2;
  a.ws_parts = L->dparts2;
  a.tile_cnt = L->dtile_cnt + dn_tiles_k1(L);
  a.err = L->err;
  dn_fill_plan(a);
  return a;
}

// the most parts any tile of a launch is cut into, on a grid of G CTAs
int dn_max_parts(const DenseArgs& a, int G) {
  const DnSplit d = dn_split(a, G);
  long long m = 1;
  for (long long t = 0; t < d.T0 + d.T1; ++t) m = std::max(m, d.owner((t + 1) * d.S - 1) - d.owner(t * d.S) + 1);
  return (int)m;
}

cudaError_t launch_dense_k1(moe_layer* L, const void* x, int B, cudaStream_t st, int skip_mask = 0) {
  const int H = L->cfg.hidden;
  // the activations: a tensor map over this call's x (B rows; rows past B read as zero)
  CUtensorMap tmx;
  if (!encode_map(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)H, (uint64_t)B, (uint64_t)H * 2, kDnKBox,
                  kDnBBox))
    return cudaErrorInvalidValue;
  const DenseArgs a = dn_args_k1(L, B, skip_mask);
  return launch_ex(dense_bf16_kernel, L->num_sms, kDnThreads, dn_smem(a), st, L->pdl, L->tm_wr,
                   a.n_streams > 1 ? L->tm_sgu : L->tm_wr, tmx, a);
}

// the shared down projection leaves kSdnFreeSms SMs to the routing finish
// and the activation terms, which run beside it in the fused forward
constexpr int kSdnFreeSms = 16;
int sdn_grid(const moe_layer* L) { return std::max(1, L->num_sms - kSdnFreeSms); }

cudaError_t launch_dense_sdn(moe_layer* L, int B, float* ys, cudaStream_t st, bool pdl = true) {
  const DenseArgs a = dn_args_sdn(L, B, ys);
  return launch_ex(dense_bf16_kernel, sdn_grid(L), kDnThreads, dn_smem(a), st, L->pdl && pdl, L->tm_sdn, L->tm_sdn,
                   L->tm_ht, a);
}

cudaError_t launch_routing_finish(moe_layer* L, const void* x, int B, const moe_routing& r, cudaStream_t st) {
  const GemvArgs a = router_args(L, x, B, r, false);
  return launch_ex(routing_finish_kernel, B, 256, kBucketScratchBytes + kTopkCandBytes, st, L->pdl, a);
}

cudaError_t launch_gate_up(moe_layer* L, const void* x, int B, const moe_routing& r, cudaStream_t st,
                           cudaEvent_t ev0 = nullptr, cudaEvent_t ev1 = nullptr) {
  if (expert_path(L, B) == MOE_PATH_TCGEN05) return launch_mx_gate_up(L, x, B, r, L->h, st, ev0, ev1);
  if (ev0) {
    const cudaError_t e = cudaEventRecord(ev0, st);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = launch_gate_up_streams(L, x, B, r, st);
  if (e == cudaSuccess && ev1) e = cudaEventRecord(ev1, st);
  return e;
}

GemvArgs gate_up_args(const moe_layer* L, const void* x, int B, const moe_routing& r) {
  const int H = L->cfg.hidden, I = L->cfg.inter;
  const GemvPlan& p = plan_of(L, K_GU, B);
  GemvArgs a = routed_args(L, p, r, B);
  a.w = L->w.w_gate_up;
  a.sc = L->w.s_gate_up;
  a.w_gstride = (long long)2 * I * (H / 2);
  a.s_gstride = (long long)2 * I * (H / 32);
  a.up_off = I;
  a.act = x;
  a.act_by_pair = 0;
  a.out = L->h;
  return a;
}

cudaError_t launch_gate_up_streams(moe_layer* L, const void* x, int B, const moe_routing& r, cudaStream_t st) {
  if (expert_path(L, B) == MOE_PATH_GROUPED) return launch_grouped(L, true, B, r, x, L->h, st);
  return run_gemv(L, K_GU, B, gate_up_args(L, x, B, r), st, L->pdl);
}

// Grouped tensor-core projection (batch > 1): f16 copy of the activation
// rows, then the MMA kernel.  gate/up: x rows -> h; down: h rows -> y.
cudaError_t launch_grouped(moe_layer* L, bool gate_up, int B, const moe_routing& r, const void* act, float* out,
                           cudaStream_t st) {
  const int H = L->cfg.hidden, I = L->cfg.inter, k = L->cfg.top_k;
  const int K = gate_up ? H : I;
  const int rows = gate_up ? B : B * k;
  cudaError_t e = gate_up ? launch_ex(act_to_f16_kernel<false>, rows, 256, 0, st, L->pdl, act, K, L->xh, L->xe)
                          : launch_ex(act_to_f16_kernel<true>, rows, 256, 0, st, L->pdl, act, K, L->xh, L->xe);
  if (e != cudaSuccess) return e;
  MmaArgs m;
  std::memset(&m, 0, sizeof(m));
  m.w = gate_up ? L->w.w_gate_up : L->w.w_down;
  m.sc = gate_up ? L->w.s_gate_up : L->w.s_down;
  m.w_gstride = gate_up ? (long long)2 * I * (H / 2) : (long long)H * (I / 2);
  m.s_gstride = gate_up ? (long long)2 * I * (H / 32) : (long long)H * (I / 32);
  m.K = K;
  m.out_rows = gate_up ? I : H;
  m.up_off = gate_up ? I : 0;
  m.xh = L->xh;
  m.xe = L->xe;
  m.act_by_pair = gate_up ? 0 : 1;
  m.top_k = k;
  m.n_pairs = B * k;
  m.n_experts = L->cfg.n_experts;
  m.n_active = r.n_active;
  m.active = r.active;
  m.offsets = r.offsets;
  m.pair_ids = r.pair_ids;
  m.out = out;
  m.n_stages = L->mma_stages[gate_up ? 0 : 1];
  m.stage_bytes = (int)align_up((size_t)kMmaRows * (K / 2 + K / 32), 128);
  m.err = L->err;
  const int smem = kMmaHeaderBytes + m.n_stages * m.stage_bytes;
  return gate_up ? launch_ex(grouped_mma_kernel<true>, L->num_sms, (kMmaWarps + 1) * 32, smem, st, L->pdl, m)
                 : launch_ex(grouped_mma_kernel<false>, L->num_sms, (kMmaWarps + 1) * 32, smem, st, L->pdl, m);
}

cudaError_t launch_combine(moe_layer* L, int B, const moe_routing& r, const float* y, const float* ys,
                           const void* residual, void* out, cudaStream_t st);
constexpr int kMxFusedCombineMaxB = 2;  // tensor-core down projection: combine inside up to this batch
GemvArgs down_args(const moe_layer* L, int B, const moe_routing& r, float* y, bool fused, const void* residual,
                   void* out, const float* ys, const moe_layer* next);

cudaError_t launch_down(moe_layer* L, int B, const moe_routing& r, float* y, bool fused, const void* residual,
                        void* out, const float* ys, moe_layer* next, cudaStream_t st, bool pdl) {
  const int path = expert_path(L, B);
  if (path == MOE_PATH_TCGEN05) {
    (void)pdl;
    if (!fused) return launch_mx_down(L, B, r, y, st);
    if (B <= kMxFusedCombineMaxB) return launch_mx_down(L, B, r, y, st, residual, out, ys, next);
    // larger batches: the combine runs over every SM after the projection
    // (in the projection kernel the last expert of a row tile would combine
    // the tile's rows for all B tokens alone)
    cudaError_t e = launch_mx_down(L, B, r, y, st, nullptr, nullptr, nullptr, next);
    if (e == cudaSuccess) e = launch_combine(L, B, r, y, ys, residual, out, st);
    return e;
  }
  if (path == MOE_PATH_GROUPED) {
    // tensor-core projection into y, then the fixed-order combine
    cudaError_t e = launch_grouped(L, false, B, r, L->h, y, st);
    if (e == cudaSuccess && fused) e = launch_combine(L, B, r, y, ys, residual, out, st);
    (void)next;
    (void)pdl;
    return e;
  }
  const Kind k = fused ? K_DNC : K_DN;
  return run_gemv(L, k, B, down_args(L, B, r, y, fused, residual, out, ys, next), st, pdl);
}

GemvArgs down_args(const moe_layer* L, int B, const moe_routing& r, float* y, bool fused, const void* residual,
                   void* out, const float* ys, const moe_layer* next) {
  const int H = L->cfg.hidden, I = L->cfg.inter;
  const Kind k = fused ? K_DNC : K_DN;
  const GemvPlan& p = plan_of(L, k, B);
  GemvArgs a = routed_args(L, p, r, B);
  a.w = L->w.w_down;
  a.sc = L->w.s_down;
  a.w_gstride = (long long)H * (I / 2);
  a.s_gstride = (long long)H * (I / 32);
  a.act = L->h;
  a.act_by_pair = 1;
  a.out = y;
  if (fused) {
    a.comb_w = r.topk_w;
    a.y_shared = ys;
    a.residual = static_cast<const uint16_t*>(residual);
    a.out_bf16 = static_cast<uint16_t*>(out);
    a.batch = B;
    a.tile_counter = L->tile_cnt;
    if (next && L->prefetch) {
      a.pf_ptr[0] = reinterpret_cast<const uint8_t*>(next->wr_t);
      a.pf_bytes[0] = (long long)next->cfg.n_experts * next->cfg.hidden * 2;
      if (next->cfg.shared_inter > 0) {
        a.pf_ptr[1] = reinterpret_cast<const uint8_t*>(next->w.shared_gate_up);
        a.pf_bytes[1] = (long long)2 * next->cfg.shared_inter * next->cfg.hidden * 2;
      }
    }
  }
  return a;
}

// the persistent kernel's instances: the streams of the batch-1 chain
// (shape-specialised: compile-time K, split-K down; generic: runtime K)
#define PERSIST_FAST persistent_b1_kernel<kFastH, kFastI, MOE_SPLITK_GU ? kSplitKRows / 2 : MOE_GU_RPW, MOE_DN_RPW>
#define PERSIST_GENERIC persistent_b1_kernel<0, 0, MOE_GU_RPW, MOE_DN_RPW>

// The whole batch-1 step as one cooperative kernel (MOE_FLAG_PERSISTENT).
cudaError_t launch_persistent(moe_layer* L, moe_layer* next, const void* x, const void* residual, void* out,
                              cudaStream_t st) {
  PersistArgs p;
  std::memset(&p, 0, sizeof(p));
  const bool has_shared = L->cfg.shared_inter > 0;
  p.router = router_args(L, x, 1, L->plan, has_shared);
  if (has_shared) {
    p.sdown = shared_down_args(L, 1, L->ys);
    p.has_sdown = 1;
  }
  p.gu = gate_up_args(L, x, 1, L->plan);
  p.dnc = down_args(L, 1, L->plan, L->y, true, residual, out, has_shared ? L->ys : nullptr, next);
  p.grid_bar = L->grid_bar;
  p.err = L->err;
  int threads = 0, smem = 0;
  const Kind kinds[4] = {K_ROUTER, K_SDN, K_GU, K_DNC};
  for (Kind kk : kinds) {
    if (kk == K_SDN && !has_shared) continue;
    threads = std::max(threads, plan_of(L, kk, 1).threads);
    smem = std::max(smem, plan_of(L, kk, 1).smem);
  }
  cudaError_t e = cudaMemsetAsync(L->grid_bar, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(L->num_sms);
  c.blockDim = dim3(threads);
  c.dynamicSmemBytes = (size_t)smem;
  c.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  c.attrs = attr;
  c.numAttrs = 1;
  return L->persist == 2 ? cudaLaunchKernelEx(&c, PERSIST_FAST, p) : cudaLaunchKernelEx(&c, PERSIST_GENERIC, p);
}

cudaError_t launch_combine(moe_layer* L, int B, const moe_routing& r, const float* y, const float* ys,
                           const void* residual, void* out, cudaStream_t st) {
  GemvArgs a;
  std::memset(&a, 0, sizeof(a));
  a.out_rows = L->cfg.hidden;
  a.top_k = L->cfg.top_k;
  a.comb_w = r.topk_w;
  a.y_shared = ys;
  a.residual = static_cast<const uint16_t*>(residual);
  a.out_bf16 = static_cast<uint16_t*>(out);
  a.batch = B;
  const long long n = (long long)B * L->cfg.hidden;
  const int grid = (int)std::min<long long>((n + 255) / 256, (long long)L->num_sms * 8);
  return launch_ex(combine_kernel, grid, 256, 0, st, L->pdl, a, y);
}

moe_status_t check_call(const moe_layer* L, int B) {
  if (!L) return MOE_ERR_INVALID_ARG;
  if (B < 1 || B > L->cfg.max_batch) return MOE_ERR_INVALID_ARG;
  // the layer's pointers belong to the device current at its creation
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != L->device) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// Makes a layer's device current for a call that may come with another
// device current (destroy, the error readout) and restores the caller's.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      prev = -1;
      return;
    }
    ok = prev == dev || cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    if (ok && prev >= 0) cudaSetDevice(prev);
  }
};

// Failure-path self-test: a wait on an mbarrier that nothing will complete
// (phase 0 of a fresh barrier) gives up after `limit` cycles and records the
// timeout, exactly as the layer's kernels do.
__global__ void selftest_wait_kernel(int* err, long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (!mbar_wait_bounded(&bar, 0u, limit) && threadIdx.x == 0) atomicExch(err, kErrTimeout);
}

std::atomic<bool> g_fail_next_alloc{false};  // MOE_SELFTEST_FAIL_NEXT_ALLOC

}  // namespace

extern "C" {

moe_status_t moe_selftest(int what, void* stream) {
  if (what == MOE_SELFTEST_FAIL_NEXT_ALLOC) {
    g_fail_next_alloc.store(true);
    return MOE_OK;
  }
  if (what != MOE_SELFTEST_WAIT_TIMEOUT) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  int* d = nullptr;
  if (cudaMalloc(&d, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_OOM;
  }
  int h = -1;
  cudaError_t e = cudaMemsetAsync(d, 0, sizeof(int), st);
  if (e == cudaSuccess) {
    selftest_wait_kernel<<<1, 32, 0, st>>>(d, 1ll << 20);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(&h, d, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaFree(d);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return h == kErrTimeout ? MOE_ERR_TIMEOUT : (h == 0 ? MOE_OK : MOE_ERR_CUDA);
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or device";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_OOM: return "out of device memory";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

moe_status_t moe_layer_create(const moe_layer_config* cfg, const moe_layer_weights* w, moe_layer_t* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg || !w) return MOE_ERR_INVALID_ARG;
  const moe_layer_config c = *cfg;
  if (c.hidden <= 0 || c.hidden % 32 || c.inter <= 0 || c.inter % 32 || c.shared_inter < 0 ||
      c.shared_inter % 32 || c.n_experts < 1 || c.n_experts > kMaxExperts || c.top_k < 1 ||
      c.top_k > kMaxTopK || c.top_k > c.n_experts || c.max_batch < 1 || c.max_batch > kMaxBatch)
    return MOE_ERR_INVALID_ARG;
  if (!w->router_w || !w->w_gate_up || !w->s_gate_up || !w->w_down || !w->s_down) return MOE_ERR_INVALID_ARG;
  const bool smx = w->shared_mx_gate_up != nullptr;
  if (smx && (!w->shared_mx_s_gate_up || !w->shared_mx_down || !w->shared_mx_s_down || w->shared_gate_up ||
              w->shared_down || c.shared_inter <= 0))
    return MOE_ERR_INVALID_ARG;
  if (c.shared_inter > 0 && !smx && (!w->shared_gate_up || !w->shared_down)) return MOE_ERR_INVALID_ARG;
  if (smx) {
    const void* sp[] = {w->shared_mx_gate_up, w->shared_mx_s_gate_up, w->shared_mx_down, w->shared_mx_s_down};
    for (const void* p : sp)
      if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  }
  const void* ptrs[] = {w->router_w, w->w_gate_up, w->s_gate_up, w->w_down, w->s_down};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (c.shared_inter > 0 && !smx && (!aligned16(w->shared_gate_up) || !aligned16(w->shared_down)))
    return MOE_ERR_INVALID_ARG;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10) return MOE_ERR_UNSUPPORTED;

  moe_layer* L = new (std::nothrow) moe_layer();
  if (!L) return MOE_ERR_OOM;
  L->cfg = c;
  L->w = *w;
  L->device = dev;
  L->num_sms = sms;
  L->pdl = !(c.flags & MOE_FLAG_NO_PDL);
  L->side_stream = (c.flags & MOE_FLAG_SIDE_STREAM) != 0;
  L->prefetch = !(c.flags & MOE_FLAG_NO_PREFETCH);
  L->sigmoid = (c.flags & MOE_FLAG_ROUTER_SIGMOID) != 0;
  L->shared_mx = smx;

  const int H = c.hidden, E = c.n_experts, k = c.top_k, I = c.inter, Is = c.shared_inter, MB = c.max_batch;
  // plans: [0] for B = 1 (one token per pass), [1] for B > 1 (two per pass)
  for (int t = 0; t < 3; ++t) {
    const int nb = t == 0 ? 1 : (t == 2 ? std::min(MB, kSmallBatch) : MB);
    const int maxg = std::min(E, nb * k);  // experts one call can activate
    const bool one = t != 1;            // one token per pass
    const bool fh = one && H == kFastH, fi = one && I == kFastI, fis = one && Is == kFastI;
    const bool sk = t == 0;             // split-K down projection: batch 1 only
    if (t == 2) {  // routed kinds only
      L->plans[K_GU][t] = make_plan(K_GU, H, I, nb, maxg, nb, (long long)2 * I * (H / 32), sms, fh);
      L->plans[K_DN][t] = make_plan(K_DN, I, H, nb * k, maxg, nb, (long long)H * (I / 32), sms, fi, false);
      L->plans[K_DNC][t] = make_plan(K_DNC, I, H, nb * k, maxg, nb, (long long)H * (I / 32), sms, fi, false);
      if (!(L->plans[K_GU][t].ok && L->plans[K_DN][t].ok && L->plans[K_DNC][t].ok)) {
        delete L;
        return MOE_ERR_UNSUPPORTED;
      }
      continue;
    }
    L->plans[K_ROUTER][t] = make_plan(K_ROUTER, H, E, nb, 1, nb, 0, sms, fh);
    L->plans[K_GU][t] = make_plan(K_GU, H, I, nb, maxg, nb, (long long)2 * I * (H / 32), sms, fh);
    L->plans[K_DN][t] = make_plan(K_DN, I, H, nb * k, maxg, nb, (long long)H * (I / 32), sms, fi, sk);
    L->plans[K_DNC][t] = make_plan(K_DNC, I, H, nb * k, maxg, nb, (long long)H * (I / 32), sms, fi, sk);
    const Kind kgu = smx ? K_SGU_MX : K_SGU, kdn = smx ? K_SDN_MX : K_SDN;
    if (Is > 0) {
      L->plans[kgu][t] = make_plan(kgu, H, Is, nb, 1, nb, smx ? (long long)2 * Is * (H / 32) : 0, sms, fh);
      L->plans[kdn][t] = make_plan(kdn, Is, H, nb, 1, nb, smx ? (long long)H * (Is / 32) : 0, sms, fis, sk);
    }
    bool ok = L->plans[K_ROUTER][t].ok && L->plans[K_GU][t].ok && L->plans[K_DN][t].ok && L->plans[K_DNC][t].ok;
    if (Is > 0) ok = ok && L->plans[kgu][t].ok && L->plans[kdn][t].ok;
    if (!ok) {
      delete L;
      return MOE_ERR_UNSUPPORTED;
    }
  }

  // scratch arena
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t o_wr = take((size_t)E * H * 2);
  const size_t o_lg = take((size_t)MB * E * 4);
  const size_t o_ti = take((size_t)MB * k * 4);
  const size_t o_tw = take((size_t)MB * k * 4);
  const size_t o_cn = take((size_t)E * 4);
  const size_t o_of = take((size_t)(E + 1) * 4);
  const size_t o_pi = take((size_t)MB * k * 4);
  const size_t o_ac = take((size_t)E * 4);
  const size_t o_na = take(4);
  const size_t o_h = take((size_t)MB * k * I * 4);
  const size_t o_y = take((size_t)MB * k * H * 4);
  const size_t o_hs = take((size_t)MB * std::max(Is, 1) * 4);
  const size_t o_ys = take((size_t)MB * H * 4);
  const size_t o_rc = take(4);
  const size_t o_pc = take(8);
  const size_t o_tc = take((size_t)H * 4);  // one counter per down-projection row tile (<= H)
  const size_t o_er = take(4);
  const size_t o_gb = take(4);
  const size_t o_xh = take((size_t)MB * std::max(H, k * I) * 2);
  const size_t o_xe = take((size_t)MB * k * 4);
  const size_t o_xs = take((size_t)MB * H * 2);
  const size_t o_rs = take((size_t)MB * H * 2);
  const size_t o_os = take((size_t)MB * H * 2);
  const size_t o_aqx = take((size_t)MB * k * kSwRowsPerTok * (H / 2));  // 8 rows per position (>= kMxTerms)
  const size_t o_sfx = take((size_t)MB * k * ((H + kMxKChunk - 1) / kMxKChunk) * kMxChunkBytes);
  const size_t o_aqh = take((size_t)MB * k * kSwRowsPerTok * (I / 2));  // 8 rows per position (>= kMxTerms)
  const size_t o_sfh = take((size_t)MB * k * ((I + kMxKChunk - 1) / kMxKChunk) * kMxChunkBytes);
  const size_t o_sww = take((size_t)sms * 2 * kSwSlotFloats * 4);
  // units of the swapped kernels: passes over all groups (<= E + B*k/16) x items per expert
  const size_t o_swc = take((size_t)(E + MB * k / kSwTokMax + 1) * std::max(I / kMxRows, H / kSwN + 1) * 4);
  if (g_fail_next_alloc.exchange(false) || cudaMalloc(&L->arena, off) != cudaSuccess) {
    cudaGetLastError();
    delete L;
    return MOE_ERR_OOM;
  }
  char* A = L->arena;
  L->wr_t = reinterpret_cast<uint16_t*>(A + o_wr);
  L->logits = reinterpret_cast<float*>(A + o_lg);
  L->plan.topk_idx = reinterpret_cast<int32_t*>(A + o_ti);
  L->plan.topk_w = reinterpret_cast<float*>(A + o_tw);
  L->plan.counts = reinterpret_cast<int32_t*>(A + o_cn);
  L->plan.offsets = reinterpret_cast<int32_t*>(A + o_of);
  L->plan.pair_ids = reinterpret_cast<int32_t*>(A + o_pi);
  L->plan.active = reinterpret_cast<int32_t*>(A + o_ac);
  L->plan.n_active = reinterpret_cast<int32_t*>(A + o_na);
  L->h = reinterpret_cast<float*>(A + o_h);
  L->y = reinterpret_cast<float*>(A + o_y);
  L->hs = reinterpret_cast<float*>(A + o_hs);
  L->ys = reinterpret_cast<float*>(A + o_ys);
  L->router_cnt = reinterpret_cast<int*>(A + o_rc);
  L->pub_cnt = reinterpret_cast<int*>(A + o_pc);
  L->tile_cnt = reinterpret_cast<int*>(A + o_tc);
  L->err = reinterpret_cast<int*>(A + o_er);
  L->grid_bar = reinterpret_cast<int*>(A + o_gb);
  L->xh = reinterpret_cast<__half*>(A + o_xh);
  L->xe = reinterpret_cast<int*>(A + o_xe);
  L->x_stage = reinterpret_cast<uint16_t*>(A + o_xs);
  L->res_stage = reinterpret_cast<uint16_t*>(A + o_rs);
  L->out_stage = reinterpret_cast<uint16_t*>(A + o_os);
  L->aqx = reinterpret_cast<uint8_t*>(A + o_aqx);
  L->bsfx = reinterpret_cast<uint8_t*>(A + o_sfx);
  L->aqh = reinterpret_cast<uint8_t*>(A + o_aqh);
  L->bsfh = reinterpret_cast<uint8_t*>(A + o_sfh);
  L->sw_ws = reinterpret_cast<float*>(A + o_sww);
  L->sw_cnt = reinterpret_cast<int*>(A + o_swc);

  cudaError_t e = cudaMemset(L->arena, 0, off);
  if (e == cudaSuccess) {
    dim3 blk(32, 8), grd((E + 31) / 32, (H + 31) / 32);
    transpose_u16_kernel<<<grd, blk>>>(static_cast<const uint16_t*>(w->router_w), L->wr_t, H, E);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&L->side, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->ev_fork, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->ev_join, cudaEventDisableTiming);
  // The small kernels run under the same shared-memory carve-out as the
  // streaming ones: an SM cannot change its carve-out while a CTA is resident,
  // so a small CTA under a smaller carve-out would keep a streaming CTA (of
  // the next kernel, launched early) off its SM until it exits.
  // grouped tensor-core path (batch > 1): ring depth per projection
  if (!(c.flags & MOE_FLAG_NO_GROUPED) && MB > kGroupedMinBatch) {
    const int Ks[2] = {H, I};
    bool ok = true;
    for (int q = 0; q < 2; ++q) {
      const int K = Ks[q];
      if (K % (32 * kMmaWarps) != 0) { ok = false; break; }
      const int stage = (int)align_up((size_t)kMmaRows * (K / 2 + K / 32), 128);
      const int ns = std::min(kMmaMaxStages, (kSmemBudget - kMmaHeaderBytes) / stage);
      if (ns < 2) { ok = false; break; }
      L->mma_stages[q] = ns;
    }
    if (ok && (I % (kMmaRows / 2)) == 0 && (H % kMmaRows) == 0) L->grouped = true;
  }
  // tcgen05 block-scaled path: K and output rows in whole 128-tiles, tensor
  // maps encodable (packed E2M1 rows as bytes: 128 per copy), and room for the
  // weight scales in chunk layout, which are copied here once
  if (e == cudaSuccess && H % kMxKChunk == 0 && I % kMxKChunk == 0) {
    const uint64_t mxr = (uint64_t)MB * k * kMxTerms;
    L->mx = encode_map(&L->tm_agu, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->w_gate_up, (uint64_t)H / 2,
                       (uint64_t)E * 2 * I, (uint64_t)H / 2, 128, kMxRows) &&
            encode_map(&L->tm_adn, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->w_down, (uint64_t)I / 2, (uint64_t)E * H,
                       (uint64_t)I / 2, 128, kMxRows) &&
            encode_map(&L->tm_bx, CU_TENSOR_MAP_DATA_TYPE_UINT8, L->aqx, (uint64_t)H / 2, mxr, (uint64_t)H / 2, 128,
                       kMxBBox) &&
            encode_map(&L->tm_bh, CU_TENSOR_MAP_DATA_TYPE_UINT8, L->aqh, (uint64_t)I / 2, mxr, (uint64_t)I / 2, 128,
                       kMxBBox);
    // the swapped kernels read x's and h's terms 8 rows per position (box 8 rows)
    L->swap = L->mx && H % kSwN == 0 &&
              encode_map(&L->tm_bx8, CU_TENSOR_MAP_DATA_TYPE_UINT8, L->aqx, (uint64_t)H / 2,
                         (uint64_t)MB * k * kSwRowsPerTok, (uint64_t)H / 2, 128, kSwRowsPerTok) &&
              encode_map(&L->tm_bh8, CU_TENSOR_MAP_DATA_TYPE_UINT8, L->aqh, (uint64_t)I / 2,
                         (uint64_t)MB * k * kSwRowsPerTok, (uint64_t)I / 2, 128, kSwRowsPerTok) &&
              // a whole pass of 16 tokens in one copy (128 rows)
              encode_map(&L->tm_bx128, CU_TENSOR_MAP_DATA_TYPE_UINT8, L->aqx, (uint64_t)H / 2,
                         (uint64_t)MB * k * kSwRowsPerTok, (uint64_t)H / 2, 128, kMxRows) &&
              encode_map(&L->tm_bh128, CU_TENSOR_MAP_DATA_TYPE_UINT8, L->aqh, (uint64_t)I / 2,
                         (uint64_t)MB * k * kSwRowsPerTok, (uint64_t)I / 2, 128, kMxRows);
    if (L->mx) {
      // the scale arrays hold one byte per 32 weights: the chunk copies are the same size
      const size_t gu_bytes = (size_t)E * 2 * I * (H / 32), dn_bytes = (size_t)E * H * (I / 32);
      if (cudaMalloc(&L->mx_mem, gu_bytes + dn_bytes) != cudaSuccess) {
        cudaGetLastError();
        L->mx = false;
        if (c.flags & MOE_FLAG_MX_EXPERTS) {
          moe_layer_destroy(L);
          return MOE_ERR_OOM;
        }
      } else {
        L->wsf_gu = reinterpret_cast<uint8_t*>(L->mx_mem);
        L->wsf_dn = L->wsf_gu + gu_bytes;
        const long long tiles_gu = (long long)E * 2 * I / kMxRows, tiles_dn = (long long)E * H / kMxRows;
        mx_pack_scales_kernel<<<4 * L->num_sms, 256>>>(w->s_gate_up, tiles_gu, H, L->wsf_gu);
        mx_pack_scales_kernel<<<4 * L->num_sms, 256>>>(w->s_down, tiles_dn, I, L->wsf_dn);
        e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
      }
    }
    L->mx_forced = (c.flags & MOE_FLAG_MX_EXPERTS) != 0;
    L->mx_default = !(c.flags & (MOE_FLAG_NO_GROUPED | MOE_FLAG_WARP_MMA));
  }
  // dense bf16 streams on tcgen05 above batch 1: tensor maps over the router
  // copy and the bf16 shared expert, the h_s terms buffer, the stream-K
  // workspaces (sized for the most parts any tile is cut into) and counters
  if (e == cudaSuccess && L->mx && MB > 1 && H % kDnRows == 0 && (Is == 0 || smx || Is % kDnRows == 0)) {
    const bool sh = Is > 0 && !smx;
    CUtensorMap probe;  // a map of two rows with a 16-row box, as the activations of batch 2 take
    bool ok = encode_map(&L->tm_wr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L->wr_t, (uint64_t)H, (uint64_t)E,
                         (uint64_t)H * 2, kDnKBox, kDnRows) &&
              encode_map(&probe, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L->x_stage, (uint64_t)H, 2, (uint64_t)H * 2,
                         kDnKBox, kDnBBox);
    if (ok && sh)
      ok = encode_map(&L->tm_sgu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->shared_gate_up, (uint64_t)H,
                      (uint64_t)2 * Is, (uint64_t)H * 2, kDnKBox, kDnRows) &&
           encode_map(&L->tm_sdn, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->shared_down, (uint64_t)Is, (uint64_t)H,
                      (uint64_t)Is * 2, kDnKBox, kDnRows);
    if (ok) {
      const int t1 = dn_tiles_k1(L), t2 = sh ? H / kDnRows : 0;
      L->dparts1 = dn_max_parts(dn_args_k1(L, 2), L->num_sms);
      L->dparts2 = sh ? std::max(dn_max_parts(dn_args_sdn(L, 2, L->ys), L->num_sms),
                                 dn_max_parts(dn_args_sdn(L, 2, L->ys), sdn_grid(L)))
                      : 1;
      const size_t part = (size_t)2 * kDnNMax * kDnRows * sizeof(float);
      const size_t b_ht = align_up((size_t)MB * kDnHTerms * std::max(Is, 1) * 2, 256);
      const size_t b_w1 = (size_t)t1 * L->dparts1 * part, b_w2 = (size_t)std::max(t2, 1) * L->dparts2 * part;
      const size_t b_tc = (size_t)(t1 + t2) * sizeof(int);
      if (cudaMalloc(&L->dense_mem, b_ht + b_w1 + b_w2 + b_tc) != cudaSuccess) {
        cudaGetLastError();
        ok = false;
      } else {
        L->hterms = reinterpret_cast<uint16_t*>(L->dense_mem);
        L->dws1 = reinterpret_cast<float*>(L->dense_mem + b_ht);
        L->dws2 = reinterpret_cast<float*>(L->dense_mem + b_ht + b_w1);
        L->dtile_cnt = reinterpret_cast<int*>(L->dense_mem + b_ht + b_w1 + b_w2);
        e = cudaMemset(L->dense_mem, 0, b_ht + b_w1 + b_w2 + b_tc);
        if (e == cudaSuccess && sh)
          ok = encode_map(&L->tm_ht, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L->hterms, (uint64_t)Is,
                          (uint64_t)MB * kDnHTerms, (uint64_t)Is * 2, kDnKBox, kDnBBox);
      }
    }
    if (e == cudaSuccess && ok) {
      e = raise_smem_limit(reinterpret_cast<const void*>(dense_bf16_kernel), kSmemBudget);
      if (e == cudaSuccess)
        e = raise_smem_limit(reinterpret_cast<const void*>(routing_finish_kernel), kBucketScratchBytes + kTopkCandBytes);
    }
    L->dense = ok && e == cudaSuccess;
  }
  if (e == cudaSuccess && L->mx) {
    e = raise_smem_limit(reinterpret_cast<const void*>(mx_expert_kernel<true, kMxTerms>), kSmemBudget);
    if (e == cudaSuccess)
      e = raise_smem_limit(reinterpret_cast<const void*>(mx_expert_kernel<false, kMxTerms>), kSmemBudget);
    if (e == cudaSuccess)
      e = raise_smem_limit(reinterpret_cast<const void*>(mx_swap_kernel<false, kMxTerms>), kSmemBudget);
    if (e == cudaSuccess)
      e = raise_smem_limit(reinterpret_cast<const void*>(mx_swap_kernel<true, kMxTerms>), kSmemBudget);
  }
  // persistent batch-1 kernel: needs the bf16 (or no) shared expert, no side
  // stream, and one shape-specialised or one generic instance for all streams
  if (e == cudaSuccess && (c.flags & MOE_FLAG_PERSISTENT)) {
    const bool fast = H == kFastH && I == kFastI && (Is == 0 || Is == kFastI);
    const bool generic = H != kFastH && I != kFastI && Is != kFastI;
    if (L->shared_mx || L->side_stream || !(fast || generic)) {
      moe_layer_destroy(L);
      return MOE_ERR_UNSUPPORTED;
    }
    int threads = 0, smem = 0;
    for (Kind kk : {K_ROUTER, K_SDN, K_GU, K_DNC}) {
      if (kk == K_SDN && Is == 0) continue;
      threads = std::max(threads, plan_of(L, kk, 1).threads);
      smem = std::max(smem, plan_of(L, kk, 1).smem);
    }
    const void* fn = fast ? reinterpret_cast<const void*>(PERSIST_FAST) : reinterpret_cast<const void*>(PERSIST_GENERIC);
    e = raise_smem_limit(fn, smem);
    int per_sm = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem);
    if (e == cudaSuccess && per_sm < 1) {
      moe_layer_destroy(L);
      return MOE_ERR_UNSUPPORTED;
    }
    L->persist = fast ? 2 : 1;
  }
  if ((c.flags & MOE_FLAG_MX_EXPERTS) && !L->mx && e == cudaSuccess) {
    moe_layer_destroy(L);
    return MOE_ERR_UNSUPPORTED;
  }
  if (e == cudaSuccess && L->grouped) {
    e = raise_smem_limit(reinterpret_cast<const void*>(grouped_mma_kernel<true>), kSmemBudget);
    if (e == cudaSuccess) e = raise_smem_limit(reinterpret_cast<const void*>(grouped_mma_kernel<false>), kSmemBudget);
  }
  const void* small_kernels[] = {reinterpret_cast<const void*>(mx_x_terms_kernel<kMxTerms>),
                                 reinterpret_cast<const void*>(mx_h_terms_kernel<kMxTerms>),
                                 reinterpret_cast<const void*>(act_to_f16_kernel<false>),
                                 reinterpret_cast<const void*>(act_to_f16_kernel<true>),
                                 reinterpret_cast<const void*>(combine_kernel)};
  for (const void* f : small_kernels)
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  for (int kk = 0; kk < K_NUM && e == cudaSuccess; ++kk)
    for (int t = 0; t < 3 && e == cudaSuccess; ++t) {
      const GemvPlan& p = L->plans[kk][t];
      if (!p.ok) continue;
      e = raise_smem_limit(reinterpret_cast<const void*>(gemv_fn((Kind)kk, tmax_of_slot(t), p.fast, t == 2)), p.smem);
    }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    moe_layer_destroy(L);
    return MOE_ERR_CUDA;
  }
  *out = L;
  return MOE_OK;
}

moe_status_t moe_layer_destroy(moe_layer_t L) {
  if (!L) return MOE_OK;
  DeviceGuard guard(L->device);
  if (L->side) cudaStreamSynchronize(L->side);
  cudaDeviceSynchronize();
  if (L->ev_fork) cudaEventDestroy(L->ev_fork);
  if (L->ev_join) cudaEventDestroy(L->ev_join);
  if (L->side) cudaStreamDestroy(L->side);
  if (L->arena) cudaFree(L->arena);
  if (L->mx_mem) cudaFree(L->mx_mem);
  if (L->dense_mem) cudaFree(L->dense_mem);
  delete L;
  return MOE_OK;
}

int moe_layer_expert_path(moe_layer_t L, int B) {
  if (!L || B < 1 || B > L->cfg.max_batch) return -1;
  return expert_path(L, B);
}

moe_status_t moe_layer_routing(moe_layer_t L, moe_routing* out) {
  if (!L || !out) return MOE_ERR_INVALID_ARG;
  *out = L->plan;
  return MOE_OK;
}

moe_status_t moe_router_topk(moe_layer_t L, const void* x, int B, const moe_routing* r, void* stream) {
  moe_status_t s = check_call(L, B);
  if (s != MOE_OK) return s;
  if (!x || !aligned16(x)) return MOE_ERR_INVALID_ARG;
  if (r && !routing_ok(r)) return MOE_ERR_INVALID_ARG;
  const moe_routing& rr = r ? *r : L->plan;
  if (dense_for(L, B)) {
    // the router on the dense tensor-core kernel (same split as the fused
    // forward's router launch, so the same logits), then the routing finish
    cudaError_t e = launch_dense_k1(L, x, B, (cudaStream_t)stream, kDnSkipShared);
    if (e == cudaSuccess) e = launch_routing_finish(L, x, B, rr, (cudaStream_t)stream);
    return cuda_status(e);
  }
  return cuda_status(launch_router(L, x, B, rr, (cudaStream_t)stream));
}

moe_status_t moe_experts_mxfp4(moe_layer_t L, const void* x, int B, const moe_routing* r, float* y_routed,
                               float* y_shared, void* stream) {
  moe_status_t s = check_call(L, B);
  if (s != MOE_OK) return s;
  if (!x || !aligned16(x) || !y_routed || !aligned16(y_routed)) return MOE_ERR_INVALID_ARG;
  if (L->cfg.shared_inter > 0 && (!y_shared || !aligned16(y_shared))) return MOE_ERR_INVALID_ARG;
  if (r && !routing_ok(r)) return MOE_ERR_INVALID_ARG;
  const moe_routing& rr = r ? *r : L->plan;
  cudaStream_t st = (cudaStream_t)stream;
  const bool has_shared = L->cfg.shared_inter > 0;
  // as in moe_layer_forward: a bf16 shared expert above batch 1 on the
  // tensor-core path runs the dense kernels whatever the side-stream flag
  const bool fork = has_shared && L->side_stream && !(dense_for(L, B) && !L->shared_mx);
  cudaError_t e = cudaSuccess;
  if (fork) {
    e = cudaEventRecord(L->ev_fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(L->side, L->ev_fork, 0);
    if (e == cudaSuccess) e = launch_shared(L, x, B, y_shared, L->side, false);
    if (e == cudaSuccess) e = cudaEventRecord(L->ev_join, L->side);
  }
  if (e == cudaSuccess) e = launch_gate_up(L, x, B, rr, st);
  if (e == cudaSuccess) e = launch_down(L, B, rr, y_routed, false, nullptr, nullptr, nullptr, nullptr, st, L->pdl);
  if (e == cudaSuccess && has_shared && !fork) {
    if (dense_for(L, B) && !L->shared_mx) {
      // the bf16 shared expert on the dense tensor-core kernels, as in moe_layer_forward
      e = launch_dense_k1(L, x, B, st, kDnSkipRouter);
      if (e == cudaSuccess) e = launch_dense_sdn(L, B, y_shared, st);
    } else {
      e = launch_shared(L, x, B, y_shared, st, L->pdl);
    }
  }
  if (e == cudaSuccess && fork) e = cudaStreamWaitEvent(st, L->ev_join, 0);
  return cuda_status(e);
}

moe_status_t moe_combine_residual(moe_layer_t L, int B, const moe_routing* r, const float* y_routed,
                                  const float* y_shared, const void* residual, void* out, void* stream) {
  moe_status_t s = check_call(L, B);
  if (s != MOE_OK) return s;
  if (!y_routed || !residual || !out || !aligned16(y_routed) || !aligned16(residual) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (r && !routing_ok(r)) return MOE_ERR_INVALID_ARG;
  const moe_routing& rr = r ? *r : L->plan;
  return cuda_status(launch_combine(L, B, rr, y_routed, y_shared, residual, out, (cudaStream_t)stream));
}

moe_status_t moe_layer_forward(moe_layer_t L, moe_layer_t next, const void* x, const void* residual, void* out,
                               int B, void* stream) {
  moe_status_t s = check_call(L, B);
  if (s != MOE_OK) return s;
  if (!x || !residual || !out || !aligned16(x) || !aligned16(residual) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (next && next->device != L->device) return MOE_ERR_INVALID_ARG;  // prefetch reads local memory only
  cudaStream_t st = (cudaStream_t)stream;
  const bool has_shared = L->cfg.shared_inter > 0;
  // above batch 1 on the tensor-core path a bf16 shared expert's down
  // projection takes the side stream anyway (below)
  const bool dense = dense_for(L, B);
  const bool fork = has_shared && L->side_stream && !(dense && !L->shared_mx);
  cudaError_t e = cudaSuccess;
  if (fork) {
    e = cudaEventRecord(L->ev_fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(L->side, L->ev_fork, 0);
    if (e == cudaSuccess) e = launch_shared(L, x, B, L->ys, L->side, false);
    if (e == cudaSuccess) e = cudaEventRecord(L->ev_join, L->side);
  }
  if (B == 1 && L->persist && !fork) return cuda_status(launch_persistent(L, next, x, residual, out, st));
  if (dense) {
    // router (+ shared gate/up), then the shared down projection on the side
    // stream beside the routing finish, the activation terms and the routed
    // experts (its grid leaves SMs free for the first two); the combine waits
    // for it
    if (e == cudaSuccess) e = launch_dense_k1(L, x, B, st);
    bool join = fork;  // an MXFP4 shared expert forked above
    if (e == cudaSuccess && has_shared && !fork) {
      if (L->shared_mx) {
        e = launch_shared(L, x, B, L->ys, st, L->pdl);
      } else {
        e = cudaEventRecord(L->ev_fork, st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(L->side, L->ev_fork, 0);
        if (e == cudaSuccess) e = launch_dense_sdn(L, B, L->ys, L->side, false);
        if (e == cudaSuccess) e = cudaEventRecord(L->ev_join, L->side);
        join = true;
      }
    }
    if (e == cudaSuccess) e = launch_routing_finish(L, x, B, L->plan, st);
    if (e == cudaSuccess) e = launch_gate_up(L, x, B, L->plan, st, L->probe_start, L->probe_stop);
    if (e == cudaSuccess && join) e = cudaStreamWaitEvent(st, L->ev_join, 0);
    if (e == cudaSuccess)
      e = launch_down(L, B, L->plan, L->y, true, residual, out, has_shared ? L->ys : nullptr, next, st, L->pdl);
    return cuda_status(e);
  }
  // the bf16 shared expert's gate/up rows stream inside the router kernel
  const bool fuse_sgu = has_shared && !fork && !L->shared_mx;
  if (e == cudaSuccess) e = launch_router(L, x, B, L->plan, st, fuse_sgu);
  if (e == cudaSuccess && has_shared && !fork)
    e = launch_shared(L, x, B, L->ys, st, L->pdl, true, /*down_only*/ fuse_sgu, /*after_router*/ fuse_sgu);
  if (e == cudaSuccess) e = launch_gate_up(L, x, B, L->plan, st, L->probe_start, L->probe_stop);
  if (e == cudaSuccess && fork) e = cudaStreamWaitEvent(st, L->ev_join, 0);
  if (e == cudaSuccess)
    e = launch_down(L, B, L->plan, L->y, true, residual, out, has_shared ? L->ys : nullptr, next, st,
                    L->pdl && !fork);
  return cuda_status(e);
}

moe_status_t moe_layer_forward_host(moe_layer_t L, const void* x_host, const void* residual_host, void* out_host,
                                    int B, void* stream) {
  moe_status_t s = check_call(L, B);
  if (s != MOE_OK) return s;
  if (!x_host || !residual_host || !out_host) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t bytes = (size_t)B * L->cfg.hidden * 2;
  cudaError_t e = cudaMemcpyAsync(L->x_stage, x_host, bytes, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(L->res_stage, residual_host, bytes, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  s = moe_layer_forward(L, nullptr, L->x_stage, L->res_stage, L->out_stage, B, stream);
  if (s != MOE_OK) return s;
  return cuda_status(cudaMemcpyAsync(out_host, L->out_stage, bytes, cudaMemcpyDeviceToHost, st));
}

moe_status_t moe_layer_last_device_error(moe_layer_t L) {
  if (!L) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(L->device);
  if (!guard.ok) return MOE_ERR_CUDA;
  // the layer may run on a non-blocking stream, which a copy on the legacy
  // stream would not wait for: wait for all of the device's work first
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, L->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v == 0) return MOE_OK;
  // clear the word and the completion counters a cut-short launch may have
  // left behind, and finish before the caller's next launch on any stream
  cudaError_t e = cudaMemset(L->err, 0, sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(L->router_cnt, 0, sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(L->pub_cnt, 0, 2 * sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(L->tile_cnt, 0, sizeof(int) * L->cfg.hidden);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return v == kErrTimeout ? MOE_ERR_TIMEOUT : MOE_ERR_INVALID_ARG;
}

moe_status_t moe_router_topk_noalloc(const void* router_w_em, const float* router_bias, int hidden, int n_experts,
                                     int top_k, const void* x, int B, const moe_routing* r, void* stream) {
  if (!router_w_em || !x || !aligned16(router_w_em) || !aligned16(x) || !routing_ok(r)) return MOE_ERR_INVALID_ARG;
  // n_experts even: the router's work items are pairs of expert rows
  if (hidden <= 0 || hidden % 32 || hidden > 32 * 32 * 16 || n_experts < 2 || n_experts > kMaxExperts ||
      n_experts % 2 || top_k < 1 || top_k > kMaxTopK || top_k > n_experts || B < 1 || B > kMaxBatch ||
      (long long)B * n_experts > kNoAllocMaxLogits)
    return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_UNSUPPORTED;
  void* base = nullptr;
  int sms = 0;
  {
    // first call on this device: resolve the array's device address (with the
    // device current) and raise the kernels' shared-memory limits
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      int major = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&g_noalloc_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (major != 10) return MOE_ERR_UNSUPPORTED;
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MOE_ERR_CUDA;
      // the largest dynamic shared memory any router plan asks for
      if (raise_smem_limit(reinterpret_cast<const void*>(gemv_fn(K_ROUTER, 1)), kSmemBudget) != cudaSuccess ||
          raise_smem_limit(reinterpret_cast<const void*>(gemv_fn(K_ROUTER, 2)), kSmemBudget) != cudaSuccess)
        return MOE_ERR_CUDA;
      g_noalloc_ptr[dev] = ptr;
    }
    base = g_noalloc_ptr[dev];
    sms = g_noalloc_sms[dev];
  }
  NoAllocScratch* sc = static_cast<NoAllocScratch*>(base);
  const GemvPlan p = make_plan(K_ROUTER, hidden, n_experts, B, 1, B, 0, sms);
  if (!p.ok) return MOE_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  // the counter must start at zero (a call cut short could leave it set)
  cudaError_t e = cudaMemsetAsync(&sc->done_counter, 0, sizeof(int), st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  GemvArgs a;
  std::memset(&a, 0, sizeof(a));
  a.K = p.K;
  a.out_rows = p.out_rows;
  a.R = p.R;
  a.ncw = p.ncw;
  a.wpi = p.wpi;
  a.n_stages = p.n_stages;
  a.stage_bytes = p.stage_bytes;
  a.stage_offset = p.stage_offset;
  a.x_offset = p.x_offset;
  a.xcap = p.xcap;
  a.ksplit = p.ksplit;
  a.top_k = top_k;
  a.n_experts = n_experts;
  a.err = &sc->err;
  a.w = static_cast<const uint8_t*>(router_w_em);
  a.act = x;
  a.n_tokens = B;
  a.out = sc->logits;
  a.bias = router_bias;
  a.topk_w = r->topk_w;
  a.topk_idx = r->topk_idx;
  a.counts = r->counts;
  a.offsets_out = r->offsets;
  a.pair_ids_out = r->pair_ids;
  a.active_out = r->active;
  a.n_active_out = r->n_active;
  a.done_counter = &sc->done_counter;
  const int tm = tmax_for(B);
  return cuda_status(launch_ex(gemv_fn(K_ROUTER, tm), sms, p.threads, p.smem, st, false, a));
}

moe_status_t moe_router_topk_noalloc_last_error(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_UNSUPPORTED;
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    base = g_noalloc_ptr[dev];
  }
  if (!base) return MOE_OK;  // no allocation-free call on this device yet
  // the calls may run on non-blocking streams: wait for all of the device's work
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  NoAllocScratch* sc = static_cast<NoAllocScratch*>(base);
  int v = 0;
  if (cudaMemcpy(&v, &sc->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v == 0) return MOE_OK;
  // clear the word and the top-k completion counter a cut-short call may have
  // left set (every call also clears the counter on its stream before use)
  if (cudaMemset(&sc->err, 0, sizeof(int)) != cudaSuccess ||
      cudaMemset(&sc->done_counter, 0, sizeof(int)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
    return MOE_ERR_CUDA;
  return v == kErrTimeout ? MOE_ERR_TIMEOUT : MOE_ERR_INVALID_ARG;
}

moe_status_t moe_layer_set_probe(moe_layer_t L, void* start, void* stop) {
  if (!L || ((start == nullptr) != (stop == nullptr))) return MOE_ERR_INVALID_ARG;
  L->probe_start = (cudaEvent_t)start;
  L->probe_stop = (cudaEvent_t)stop;
  return MOE_OK;
}

}  // extern "C"
