// Device code of the MoE decode layer (sm_100a).
//
// One streaming-GEMV kernel template covers the four weight streams of the
// layer: the router (bf16, dense), the shared expert's gate/up and down
// (bf16, dense) and the routed experts' gate/up and down (MXFP4, one group
// per active expert).  Decode at batch <= 64 is a weight stream: every byte
// of an active weight matrix is read once and used for a handful of tokens,
// so the kernel is built to keep HBM busy:
//
//  * persistent CTAs (one per SM), each owning a contiguous range of work
//    items; an item is R consecutive output rows of one group;
//  * one producer warp moves each item's weight tile (codes and scales, all
//    rows contiguous in memory) into a ring of shared-memory stages with 1-D
//    TMA bulk copies, completion counted on mbarriers, with an L2
//    evict-first policy for the single-use routed weights;
//  * consumer warps are split into row groups; inside a row group each
//    thread owns one 32-element K chunk (= one MXFP4 scale block), keeps
//    the activations of that chunk in registers across rows, decodes the
//    weights in registers (cvt e2m1x2 -> f16x2 -> fp32, or bf16 -> fp32)
//    and accumulates in fp32; a fixed butterfly + ordered cross-warp sum
//    reduces the chunk partials (bitwise reproducible);
//  * epilogues: store, SwiGLU, router logits (+ bias, then the last CTA
//    runs top-k, softmax and bucketing), and down projection fused with the
//    routing-weight combine and the residual add (last CTA to finish a row
//    tile sums that tile in ascending expert order).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace moe {

enum WFmt : int { W_MXFP4 = 0, W_BF16 = 1 };
enum Epi : int { EPI_STORE = 0, EPI_SWIGLU = 1, EPI_ROUTER = 2, EPI_DOWN_COMBINE = 3 };

constexpr int kErrTimeout = 5;
constexpr int kErrBadPlan = 6;

__device__ __forceinline__ int clamp_group(int g, int n, int* err) {
  if (g < 0 || g >= n) {
    if (err) atomicExch(err, kErrBadPlan);
    return g < 0 ? 0 : n - 1;
  }
  return g;
}
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 1024;
constexpr int kMaxBatch = 64;

struct GemvArgs {
  // weights: group g's tile of output rows [r0, r0+R) starts at
  //   w  + g*w_gstride + r0*w_rowbytes            (and + up_off*w_rowbytes for SwiGLU up rows)
  //   sc + g*s_gstride + r0*(K/32)                 (MXFP4 only)
  const uint8_t* w;
  const uint8_t* sc;
  long long w_gstride;
  long long s_gstride;
  int K;
  int out_rows;   // output rows per group
  int up_off;     // SwiGLU: rows between a gate row and its up row (= out_rows)
  int R;          // output rows per item
  int G;          // row groups per CTA
  int wpr;        // warps per row group
  int n_stages;
  int stage_bytes;
  // activations: row-major [*][K], bf16 or fp32
  const void* act;
  // token lists
  int routed;       // 1: one group per active expert; 0: a single dense group
  int n_tokens;     // dense group size (B)
  int top_k;
  int n_pairs;      // routed: B * top_k (pair ids are < n_pairs)
  int act_by_pair;  // routed: activation row = pair (1) or pair / top_k (0)
  const int* n_active;
  const int* active;
  const int* offsets;
  const int* pair_ids;
  // outputs: out[orow][out_rows], orow = pair (routed) or token (dense)
  float* out;
  // router extras
  const float* bias;
  float* topk_w;
  int* topk_idx;
  int* counts;
  int* offsets_out;
  int* pair_ids_out;
  int* active_out;
  int* n_active_out;
  int n_experts;
  int* done_counter;
  // combine extras (EPI_DOWN_COMBINE)
  const float* comb_w;      // topk_w [B][k]
  const float* y_shared;    // [B][H] or null
  const uint16_t* residual; // bf16 [B][H]
  uint16_t* out_bf16;       // bf16 [B][H]
  int batch;
  int* tile_counter;        // [out_rows / R]
  // L2 prefetch of the next layer's weights (issued by CTAs when their items are done)
  const uint8_t* pf_ptr[2];
  long long pf_bytes[2];
  int* err;
};

// ---------------------------------------------------------------------------
// warp reduction of V values (V a power of two <= 32): afterwards lane l
// holds the full warp sum of value index l / (32 / V).
template <int V>
__device__ __forceinline__ float warp_reduce_multi(float (&v)[V], int lane) {
  constexpr int kStages = (V >= 32) ? 5 : (V >= 16) ? 4 : (V >= 8) ? 3 : (V >= 4) ? 2 : (V >= 2) ? 1 : 0;
  // transposing stages: offsets 16, 8, ... halve the number of live values
#pragma unroll
  for (int s = 0; s < kStages; ++s) {
    const int off = 16 >> s;
    const int n = V >> s;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float keep = upper ? v[i + n / 2] : v[i];
      const float send = upper ? v[i] : v[i + n / 2];
      v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
    }
  }
  float r = v[0];
#pragma unroll
  for (int s = kStages; s < 5; ++s) r += __shfl_xor_sync(0xFFFFFFFFu, r, 16 >> s);
  return r;
}

template <int T>
struct NextPow2 {
  static constexpr int value = T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : T <= 8 ? 8 : T <= 16 ? 16 : 32;
};

// dot products of one 32-element chunk of NW weight rows with T activation chunks
// (tokens t >= T of the TMAX-wide arrays are left untouched)
template <int WF, int NW, int T, int TMAX>
__device__ __forceinline__ void chunk_dots(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scl,
                                           const int (&row)[NW], int rowbytes, int sblocks, int c,
                                           const float (&x)[TMAX][32], float (&acc)[NW][TMAX]) {
#pragma unroll
  for (int r = 0; r < NW; ++r) {
    float d[T];
#pragma unroll
    for (int t = 0; t < T; ++t) d[t] = 0.f;
    if constexpr (WF == W_MXFP4) {
      const uint4 q = lds128(codes + (size_t)row[r] * rowbytes + c * 16);
      const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t h2[4];
        e2m1x8_to_f16x2(qw[i], h2);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2[j]));
#pragma unroll
          for (int t = 0; t < T; ++t) {
            d[t] = fmaf(f.x, x[t][8 * i + 2 * j], d[t]);
            d[t] = fmaf(f.y, x[t][8 * i + 2 * j + 1], d[t]);
          }
        }
      }
      const float s = e8m0_to_f32(scl[(size_t)row[r] * sblocks + c]);
#pragma unroll
      for (int t = 0; t < T; ++t) acc[r][t] = d[t] * s;
    } else {
      const uint8_t* base = codes + (size_t)row[r] * rowbytes + c * 64;
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        const uint4 q = lds128(base + 16 * v4);
        const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = bf16lo_to_f32(qw[i]), hi = bf16hi_to_f32(qw[i]);
#pragma unroll
          for (int t = 0; t < T; ++t) {
            d[t] = fmaf(lo, x[t][8 * v4 + 2 * i], d[t]);
            d[t] = fmaf(hi, x[t][8 * v4 + 2 * i + 1], d[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < T; ++t) acc[r][t] = d[t];
    }
  }
}

template <bool ACT_F32>
__device__ __forceinline__ void load_act_chunk(const void* act, int arow, int K, int c, float (&x)[32]) {
  if constexpr (ACT_F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(act) + (size_t)arow * K + c * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 v = __ldg(p + i);
      x[4 * i] = v.x;
      x[4 * i + 1] = v.y;
      x[4 * i + 2] = v.z;
      x[4 * i + 3] = v.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(act) + (size_t)arow * K + c * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = __ldg(p + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[8 * i + 2 * j] = bf16lo_to_f32(w[j]);
        x[8 * i + 2 * j + 1] = bf16hi_to_f32(w[j]);
      }
    }
  }
}

// Fixed-order combine of one output element: residual + y_shared + sum_j w_j y_j
// (fp32, fused multiply-adds in ascending j = ascending expert id), bf16 once.
__device__ __forceinline__ uint16_t combine_one(const GemvArgs& a, const float* __restrict__ y, int H, int b,
                                                int r) {
  float acc = __uint_as_float((uint32_t)a.residual[(size_t)b * H + r] << 16);
  if (a.y_shared) acc += __ldcg(a.y_shared + (size_t)b * H + r);
  const int k = a.top_k;
  for (int j = 0; j < k; ++j) acc = fmaf(__ldcg(a.comb_w + b * k + j), __ldcg(y + ((size_t)b * k + j) * H + r), acc);
  return f32_to_bf16_rne(acc);
}

// ---------------------------------------------------------------------------
// Router finish: top-k (warp per token), softmax over the selected logits and
// bucketing, by the last CTA of the router grid.  logits [B][E] fp32.
__device__ void router_finish(const GemvArgs& a, unsigned char* smem) {
  const int E = a.n_experts, k = a.top_k, B = a.n_tokens;
  const int nthreads = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = nthreads >> 5;
  const int PL = (E + 31) / 32;  // experts per lane, lane l holds [l*PL, (l+1)*PL)
  int* s_idx = reinterpret_cast<int*>(smem);                               // [B*k]
  unsigned long long* s_mask = reinterpret_cast<unsigned long long*>(smem + 8 * 1024);  // [E]
  int* s_off = reinterpret_cast<int*>(smem + 8 * 1024 + 8 * kMaxExperts);               // [E+1]
  const float* logits = a.out;

  for (int b = warp; b < B; b += nwarps) {
    uint32_t key[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = lane * PL + i;
      uint32_t kk = 0u;  // below every real key
      if (i < PL && e < E) {
        const uint32_t u = __float_as_uint(__ldcg(logits + (size_t)b * E + e));
        kk = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // order-preserving map
        if (kk == 0u) kk = 1u;                              // keep 0 for "empty"
      }
      key[i] = kk;
    }
    uint32_t sel = 0u;
    for (int r = 0; r < k; ++r) {
      uint32_t best = 0u;
      int bslot = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const bool live = !((sel >> i) & 1u);
        if (live && key[i] > best) {
          best = key[i];
          bslot = i;
        }
      }
      const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, best);
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, best == m);
      const int win = __ffs(bal) - 1;  // lowest lane = lowest expert ids among equals
      if (lane == win) sel |= 1u << bslot;
    }
    // ascending expert id: lanes in order, slots in order within a lane
    const int nsel = __popc(sel);
    int pre = nsel;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, pre, o);
      if (lane >= o) pre += t;
    }
    pre -= nsel;
    // softmax over the selected logits in fp32: m = largest selected logit
    float lmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if ((sel >> i) & 1u) lmax = fmaxf(lmax, __ldcg(logits + (size_t)b * E + lane * PL + i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xFFFFFFFFu, lmax, o));
    float ex[32];
    float zl = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      ex[i] = 0.f;
      if ((sel >> i) & 1u) {
        ex[i] = expf(__ldcg(logits + (size_t)b * E + lane * PL + i) - lmax);
      }
    }
    // z = sum over selected in ascending expert order (lane order, then slot order)
#pragma unroll
    for (int i = 0; i < 32; ++i) zl += ex[i];
    float z = 0.f;
    for (int l = 0; l < 32; ++l) z += __shfl_sync(0xFFFFFFFFu, zl, l);
    int pos = pre;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((sel >> i) & 1u) {
        const int e = lane * PL + i;
        a.topk_idx[b * k + pos] = e;
        a.topk_w[b * k + pos] = ex[i] / z;
        s_idx[b * k + pos] = e;
        ++pos;
      }
    }
  }
  __syncthreads();
  // bucketing: token bitmask per expert (B <= 64), counts = popcount,
  // offsets = exclusive scan, pair position = offset + number of earlier tokens
  for (int e = tid; e < E; e += nthreads) s_mask[e] = 0ull;
  __syncthreads();
  for (int p = tid; p < B * k; p += nthreads) atomicOr(&s_mask[s_idx[p]], 1ull << (p / k));
  __syncthreads();
  if (warp == 0) {
    int cnt_l = 0, act_l = 0;
    for (int i = 0; i < PL; ++i) {
      const int e = lane * PL + i;
      if (e < E) {
        const int c = __popcll(s_mask[e]);
        cnt_l += c;
        act_l += c > 0;
      }
    }
    int cpre = cnt_l, apre = act_l;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t1 = __shfl_up_sync(0xFFFFFFFFu, cpre, o);
      const int t2 = __shfl_up_sync(0xFFFFFFFFu, apre, o);
      if (lane >= o) {
        cpre += t1;
        apre += t2;
      }
    }
    cpre -= cnt_l;
    apre -= act_l;
    for (int i = 0; i < PL; ++i) {
      const int e = lane * PL + i;
      if (e < E) {
        const int c = __popcll(s_mask[e]);
        s_off[e] = cpre;
        a.offsets_out[e] = cpre;
        a.counts[e] = c;
        if (c > 0) a.active_out[apre++] = e;
        cpre += c;
      }
    }
    if (lane == 31) {
      s_off[E] = cpre;
      a.offsets_out[E] = cpre;
      *a.n_active_out = apre;
    }
  }
  __syncthreads();
  for (int p = tid; p < B * k; p += nthreads) {
    const int e = s_idx[p];
    const int b = p / k;
    const unsigned long long below = (b == 0) ? 0ull : (s_mask[e] & ((1ull << b) - 1ull));
    a.pair_ids_out[s_off[e] + __popcll(below)] = p;
  }
}

// ---------------------------------------------------------------------------
template <int WF, int EPI, bool ACT_F32, int RPG, int TMAX, int MAXT>
__global__ void __launch_bounds__(MAXT, 1) stream_gemv_kernel(const GemvArgs a) {
  constexpr bool kSwiglu = (EPI == EPI_SWIGLU);
  constexpr int NW = kSwiglu ? 2 * RPG : RPG;  // weight rows per thread per item
  extern __shared__ __align__(128) unsigned char smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ncw = a.G * a.wpr;  // consumer warps
  const int nct = ncw * 32;
  const int K = a.K;
  const int C = K >> 5;
  const int rowbytes = (WF == W_MXFP4) ? (K >> 1) : (K << 1);
  const int sblocks = K >> 5;
  const int rows_per_item = kSwiglu ? 2 * a.R : a.R;
  const int codes_bytes = rows_per_item * rowbytes;

  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty_bar = full_bar + a.n_stages;
  float* red = reinterpret_cast<float*>(empty_bar + a.n_stages);       // [2][G][wpr][32]
  volatile int* s_flags = reinterpret_cast<volatile int*>(red + 2 * a.G * a.wpr * 32);  // [4]
  unsigned char* stages = smem + ((((size_t)2 * a.n_stages * 8 + (size_t)2 * a.G * a.wpr * 32 * 4 + 16) + 127) & ~(size_t)127);

  if (tid == 0) {
    for (int s = 0; s < a.n_stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], ncw);
    }
    s_flags[0] = 0;  // abort
    s_flags[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // Dense weight streams may start before the previous grid finishes (weights
  // are static); anything produced upstream (routing plan, activations) is
  // only read after pdl_wait().
  const bool producer = (warp == ncw);
  if (a.routed || !producer) pdl_wait();

  // A routing plan from elsewhere is validated, never trusted: groups and
  // token counts are clamped into range (and flagged) before they address memory.
  int n_groups = a.routed ? *a.n_active : 1;
  if (n_groups < 0 || n_groups > a.n_experts) {
    if (tid == 0) atomicExch(a.err, kErrBadPlan);
    n_groups = n_groups < 0 ? 0 : a.n_experts;
  }
  const int n_rt = a.out_rows / a.R;
  const long long n_items = (long long)n_groups * n_rt;
  const long long it0 = n_items * blockIdx.x / gridDim.x;
  const long long it1 = n_items * (blockIdx.x + 1) / gridDim.x;

  if (producer) {
    if (lane == 0) {
      // every weight byte is used once per step: do not let it displace
      // activations, scratch or prefetched next-layer weights in L2
      const uint64_t pol = l2_policy_evict_first();
      int s = 0;
      uint32_t ph = 0;
      for (long long it = it0; it < it1; ++it) {
        if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u)) {
          atomicExch(a.err, kErrTimeout);
          s_flags[0] = 1;
          break;
        }
        if (s_flags[0]) break;
        const int g = (int)(it / n_rt);
        const int rt = (int)(it - (long long)g * n_rt);
        const int grp = a.routed ? clamp_group(a.active[g], a.n_experts, a.err) : 0;
        const int r0 = rt * a.R;
        unsigned char* st = stages + (size_t)s * a.stage_bytes;
        const uint32_t cb = (uint32_t)(a.R * rowbytes);
        const uint32_t sb = (WF == W_MXFP4) ? (uint32_t)(a.R * sblocks) : 0u;
        const uint32_t total = (kSwiglu ? 2u : 1u) * (cb + sb);
        mbar_arrive_expect_tx(&full_bar[s], total);
        const uint8_t* wg = a.w + (long long)grp * a.w_gstride;
        bulk_g2s(st, wg + (size_t)r0 * rowbytes, cb, &full_bar[s], pol);
        if (kSwiglu) bulk_g2s(st + cb, wg + (size_t)(r0 + a.up_off) * rowbytes, cb, &full_bar[s], pol);
        if (WF == W_MXFP4) {
          const uint8_t* sg = a.sc + (long long)grp * a.s_gstride;
          bulk_g2s(st + codes_bytes, sg + (size_t)r0 * sblocks, sb, &full_bar[s], pol);
          if (kSwiglu) bulk_g2s(st + codes_bytes + sb, sg + (size_t)(r0 + a.up_off) * sblocks, sb, &full_bar[s], pol);
        }
        if (++s == a.n_stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (s_flags[0]) {
        // aborting: let copies already issued land before the CTA exits
        for (int q = 0; q < a.n_stages; ++q) (void)mbar_wait_bounded(&full_bar[q], 0u, 1ll << 24),
                                              (void)mbar_wait_bounded(&full_bar[q], 1u, 1ll << 24);
      }
    }
  } else {
    // ------------------------------ consumers ------------------------------
    const int rg = warp / a.wpr;           // row group
    const int wig = warp - rg * a.wpr;     // warp in group
    const int c = wig * 32 + lane;         // K chunk owned by this thread
    const bool has_chunk = c < C;
    const int gtid = wig * 32 + lane;      // thread index inside the row group
    float x[TMAX][32];
    int cached_group = -1;
    int s = 0;
    uint32_t ph = 0;
    int buf = 0;
    for (long long it = it0; it < it1; ++it) {
      const int g = (int)(it / n_rt);
      const int rt = (int)(it - (long long)g * n_rt);
      const int grp = a.routed ? clamp_group(a.active[g], a.n_experts, nullptr) : 0;
      int tok0 = a.routed ? a.offsets[grp] : 0;
      int ntok = a.routed ? (a.offsets[grp + 1] - tok0) : a.n_tokens;
      if (a.routed && (tok0 < 0 || ntok < 1 || tok0 + ntok > a.n_pairs)) {
        if (lane == 0) atomicExch(a.err, kErrBadPlan);
        tok0 = 0;
        ntok = 1;
      }

      if (!mbar_wait_bounded(&full_bar[s], ph)) {
        atomicExch(a.err, kErrTimeout);
        s_flags[0] = 1;
      }
      if (s_flags[0]) break;
      const unsigned char* st = stages + (size_t)s * a.stage_bytes;

      int rowsel[NW];
#pragma unroll
      for (int r = 0; r < NW; ++r) rowsel[r] = (r < RPG) ? (rg * RPG + r) : (a.R + rg * RPG + (r - RPG));

      for (int tb = 0; tb < ntok; tb += TMAX) {
        const int T = min(TMAX, ntok - tb);
        int arow[TMAX], orow[TMAX];
#pragma unroll
        for (int t = 0; t < TMAX; ++t) {
          const int tt = min(tb + t, ntok - 1);
          if (a.routed) {
            int p = a.pair_ids[tok0 + tt];
            if (p < 0 || p >= a.n_pairs) p = 0;
            arow[t] = a.act_by_pair ? p : p / a.top_k;
            orow[t] = p;
          } else {
            arow[t] = tt;
            orow[t] = tt;
          }
        }
        const bool reuse = (ntok <= TMAX) && (cached_group == (a.routed ? grp : 0));
        if (!reuse && has_chunk) {
#pragma unroll
          for (int t = 0; t < TMAX; ++t)
            if (t < T) load_act_chunk<ACT_F32>(a.act, arow[t], K, c, x[t]);
        }
        cached_group = (ntok <= TMAX) ? (a.routed ? grp : 0) : -1;

        float acc[NW][TMAX];
#pragma unroll
        for (int r = 0; r < NW; ++r)
#pragma unroll
          for (int t = 0; t < TMAX; ++t) acc[r][t] = 0.f;
        if (has_chunk) {
          if (T == TMAX) {
            chunk_dots<WF, NW, TMAX, TMAX>(st, st + codes_bytes, rowsel, rowbytes, sblocks, c, x, acc);
          } else if constexpr (TMAX > 1) {
            if (T == 1) chunk_dots<WF, NW, 1, TMAX>(st, st + codes_bytes, rowsel, rowbytes, sblocks, c, x, acc);
            else if (T == 2) chunk_dots<WF, NW, (TMAX > 2 ? 2 : 1), TMAX>(st, st + codes_bytes, rowsel, rowbytes, sblocks, c, x, acc);
            else chunk_dots<WF, NW, (TMAX > 3 ? 3 : 1), TMAX>(st, st + codes_bytes, rowsel, rowbytes, sblocks, c, x, acc);
          }
        }
        if (tb + TMAX >= ntok) {
          // stage no longer needed: hand it back to the producer
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty_bar[s]);
        }
        // --- reduce over the row group ---
        constexpr int V = NextPow2<NW * TMAX>::value;
        float v[V];
#pragma unroll
        for (int i = 0; i < V; ++i) v[i] = 0.f;
#pragma unroll
        for (int r = 0; r < NW; ++r)
#pragma unroll
          for (int t = 0; t < TMAX; ++t) v[r * TMAX + t] = acc[r][t];
        const float tot = warp_reduce_multi<V>(v, lane);
        float* rb = red + ((size_t)(buf * a.G + rg) * a.wpr) * 32;
        if ((lane & (32 / V - 1)) == 0) rb[wig * 32 + lane / (32 / V)] = tot;
        named_bar_sync(1, nct);
        // --- epilogue ---
        const int nout = (kSwiglu ? RPG : NW) * TMAX;
        if (gtid < nout) {
          const int rr = gtid / TMAX, t = gtid - (gtid / TMAX) * TMAX;
          if (t < T) {
            float s0 = 0.f;
            for (int w2 = 0; w2 < a.wpr; ++w2) s0 += rb[w2 * 32 + rr * TMAX + t];
            const int orow_out = rt * a.R + rg * RPG + rr;
            float val = s0;
            if constexpr (kSwiglu) {
              float s1 = 0.f;
              for (int w2 = 0; w2 < a.wpr; ++w2) s1 += rb[w2 * 32 + (RPG + rr) * TMAX + t];
              val = s0 / (1.0f + expf(-s0)) * s1;
            }
            if constexpr (EPI == EPI_ROUTER) {
              if (a.bias) val += a.bias[orow_out];
            }
            int orow_t = orow[0];
#pragma unroll
            for (int q = 1; q < TMAX; ++q)
              if (t == q) orow_t = orow[q];
            a.out[(size_t)orow_t * a.out_rows + orow_out] = val;
          }
        }
        buf ^= 1;
      }
      if constexpr (EPI == EPI_DOWN_COMBINE) {
        // last CTA to finish row tile rt (over all active experts) combines it
        __threadfence();
        named_bar_sync(1, nct);
        if (tid == 0) {
          const int old = atomicAdd(&a.tile_counter[rt], 1);
          s_flags[1] = (old == n_groups - 1);
        }
        named_bar_sync(1, nct);
        if (s_flags[1]) {
          __threadfence();
          const int H = a.out_rows;
          for (int i = tid; i < a.batch * a.R; i += nct) {
            const int b = i / a.R, r = rt * a.R + (i - (i / a.R) * a.R);
            a.out_bf16[(size_t)b * H + r] = combine_one(a, a.out, H, b, r);
          }
          if (tid == 0) a.tile_counter[rt] = 0;
        }
      }
      if (++s == a.n_stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  }

  // Let the next kernel in the stream start its prologue.
  pdl_launch_dependents();

  if constexpr (EPI == EPI_DOWN_COMBINE) {
    // tail: warm L2 with the next layer's static weights (one slice per CTA)
    if (tid == 32 * ncw && !s_flags[0]) {
      for (int q = 0; q < 2; ++q) {
        if (!a.pf_ptr[q] || a.pf_bytes[q] <= 0) continue;
        const long long per = ((a.pf_bytes[q] / gridDim.x) + 15) & ~15ll;
        const long long beg = per * blockIdx.x;
        long long end = beg + per;
        if (end > a.pf_bytes[q]) end = a.pf_bytes[q];
        for (long long o = beg; o < end; o += 65536) {
          const long long n = (end - o) < 65536 ? (end - o) : 65536;
          if (n >= 16) prefetch_l2(a.pf_ptr[q] + o, (uint32_t)(n & ~15ll));
        }
      }
    }
  }

  if constexpr (EPI == EPI_ROUTER) {
    __syncthreads();
    __threadfence();
    if (tid == 0) {
      const int old = atomicAdd(a.done_counter, 1);
      s_flags[1] = (old == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (s_flags[1]) {
      __threadfence();
      router_finish(a, stages);
      if (tid == 0) *a.done_counter = 0;
    }
  }
}

// Staged combine: out = bf16(residual + y_shared + sum_j w_j y_j), one thread per element.
__global__ void combine_kernel(const GemvArgs a, const float* __restrict__ y) {
  pdl_wait();
  const int H = a.out_rows;
  const long long n = (long long)a.batch * H;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int b = (int)(i / H), r = (int)(i - (long long)b * H);
    a.out_bf16[i] = combine_one(a, y, H, b, r);
  }
  pdl_launch_dependents();
}

// [H][E] -> [E][H] copy of the router matrix (bf16 as u16), tiled through shared memory.
__global__ void transpose_u16_kernel(const uint16_t* __restrict__ in, uint16_t* __restrict__ out, int rows, int cols) {
  __shared__ uint16_t tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = in[(size_t)r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[(size_t)c * rows + r] = tile[threadIdx.x][i];
  }
}

}  // namespace moe
