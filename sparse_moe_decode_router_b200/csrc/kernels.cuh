// Device code shared by the MoE decode kernels (sm_100a): kernel arguments,
// the multi-value warp reduction, the router's top-k / softmax / bucketing
// finish, the fixed-order combine, and the router-matrix transpose.  The
// streaming GEMV kernel itself is in gemv.cuh.
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
  int ncw;        // consumer warps per CTA (one more warp produces)
  int wpi;        // warps sharing one item (R = rows per warp * wpi)
  int n_stages;   // shared-memory stages in the ring
  int stage_bytes;
  int stage_offset;   // byte offset of the stage ring in dynamic shared memory
  int x_offset;       // byte offset of the staged activation vectors
  int xcap;           // activation vectors staged at a time
  int scales_global;  // 1: MXFP4 scale rows are read from global memory (rows too short for TMA)
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
  int* done_counter;       // top-k kernel: CTAs done (the last one buckets and resets it)
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
  int ksplit;       // bf16 streams: warps of a group that split K (partial sums meet in shared memory)
  int pdl_late;     // dense stream whose activations are final at launch: no wait before
                   // reading them; every thread waits for the preceding grid at exit instead
  int scoring;      // top-k: 0 = softmax over the selected logits (bias already in the
                    // logits); 1 = sigmoid scores, selection by score + sel_bias, weights
                    // score / sum of the selected scores
  const float* sel_bias;  // sigmoid scoring: the selection bias [E] (or null)
  // router kernel: the shared expert's gate/up rows as extra items (same
  // activation, same bf16 format): gate row i at w2 + i*rowbytes, up row at
  // w2 + (i + up_off2)*rowbytes, h_s = silu(gate . x) * (up . x) into out2 [B][n_items2]
  const uint8_t* w2;
  float* out2;
  int n_items2;
  int up_off2;
  // router kernel: every CTA adds 1 to *pub_counter once its outputs (logits,
  // h_s) are written, then lets the next grid launch, before the routing
  // finish.  A dense stream that reads only those outputs (the shared down
  // projection) waits for *dep_counter to reach dep_target (the router's
  // grid) instead of the whole router grid; the last of its CTAs to get past
  // resets *dep_counter and *dep_pass.  It runs with pdl_late, so it still
  // completes only after the router grid.
  int* pub_counter;
  int* dep_counter;
  int dep_target;
  int* dep_pass;
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

// Fixed-order combine of one output element: residual + y_shared + sum_j w_j y_j
// (fp32, fused multiply-adds in ascending j = ascending expert id), bf16 once.
// The loads of up to sixteen pairs go out together, ahead of their ordered sums.
__device__ __forceinline__ uint16_t combine_elem(const uint16_t* __restrict__ residual, const float* y_shared,
                                                 const float* comb_w, int k, const float* y, int H, int b, int r) {
  float acc = __uint_as_float((uint32_t)residual[(size_t)b * H + r] << 16);
  if (y_shared) acc += __ldcg(y_shared + (size_t)b * H + r);
  for (int j0 = 0; j0 < k; j0 += 16) {
    float wv[16], yv[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      wv[j] = 0.f;
      yv[j] = 0.f;
      if (j0 + j < k) {
        wv[j] = __ldcg(comb_w + b * k + j0 + j);
        yv[j] = __ldcg(y + ((size_t)b * k + j0 + j) * H + r);
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j0 + j < k) acc = fmaf(wv[j], yv[j], acc);
  }
  return f32_to_bf16_rne(acc);
}

__device__ __forceinline__ uint16_t combine_one(const GemvArgs& a, const float* __restrict__ y, int H, int b,
                                                int r) {
  return combine_elem(a.residual, a.y_shared, a.comb_w, a.top_k, y, H, b, r);
}

// ---------------------------------------------------------------------------
// Top-k, softmax and bucketing (one CTA per token, 8 warps).
//
// Order-preserving key of an fp32 logit (larger logit -> larger key; 0 is
// reserved for "no expert").
__device__ __forceinline__ uint32_t logit_key(float f) {
  const uint32_t u = __float_as_uint(f);
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return k ? k : 1u;
}

// One warp selects the k largest keys among n candidates held in a blocked
// layout (lane l owns candidates [l*PL, l*PL + PL)), whose ids ascend with the
// candidate index; equal keys go to the lower id.  Returns the selection as a
// per-lane slot bitmask.
template <int PL>
__device__ __forceinline__ uint32_t warp_select_topk(const uint32_t (&key)[PL], int k, int lane) {
  uint32_t sel = 0u;
  for (int r = 0; r < k; ++r) {
    uint32_t best = 0u;
    int bslot = 0;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const bool live = !((sel >> i) & 1u);
      if (live && key[i] > best) {
        best = key[i];
        bslot = i;
      }
    }
    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, best);
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, best == m && m != 0u);
    if (lane == __ffs(bal) - 1) sel |= 1u << bslot;
  }
  return sel;
}

// Weights of token b's selection and its output, ascending expert id, in one
// fixed order: lane j < k of the warp holds the j-th selected expert (id and
// logit, or sigmoid score); the softmax max and the normaliser are warp
// reductions over the lanes in position order (every top-k path uses this,
// so they give the same bits).
__device__ __forceinline__ void topk_emit(const GemvArgs& a, int b, float v, int id, int lane) {
  const int k = a.top_k;
  const bool on = lane < k;
  float m = on ? v : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  const float e = on ? (a.scoring == 1 ? v : expf(v - m)) : 0.f;
  float z = e;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
  if (on) {
    a.topk_idx[b * k + lane] = id;
    a.topk_w[b * k + lane] = e / z;
  }
}

// The warp-selected candidates (PL per lane, ids ascending with lane*PL +
// slot; `sel` marks the selection) in position order through `scratch`
// (k floats + k ints of this warp), then topk_emit.
template <int PL>
__device__ __forceinline__ void topk_write(const GemvArgs& a, int b, uint32_t sel, const float (&val)[PL],
                                           const int (&id)[PL], int lane, float* sv, int* si) {
  const int ns = __popc(sel);
  int pre = ns;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, pre, o);
    if (lane >= o) pre += t;
  }
  pre -= ns;
  __syncwarp();
  int pos = pre;
#pragma unroll
  for (int i = 0; i < PL; ++i)
    if ((sel >> i) & 1u) {
      sv[pos] = val[i];
      si[pos] = id[i];
      ++pos;
    }
  __syncwarp();
  const bool on = lane < a.top_k;
  topk_emit(a, b, on ? sv[lane] : 0.f, on ? si[lane] : 0, lane);
}

// Selection keys and values of experts [lo, hi) of token b (hi - lo <= 32*PL),
// lane l owning [lo + l*PL, lo + l*PL + PL)
template <int PL>
__device__ __forceinline__ void topk_load(const GemvArgs& a, const float* __restrict__ lg, int b, int lo, int hi,
                                          int lane, uint32_t (&key)[PL], float (&val)[PL], int (&id)[PL]) {
  const int E = a.n_experts;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lo + lane * PL + i;
    const bool ok = e < hi;
    float v = ok ? __ldcg(lg + (size_t)b * E + e) : 0.f;
    if (a.scoring == 1) {
      v = 1.0f / (1.0f + expf(-v));
      key[i] = ok ? logit_key(v + (a.sel_bias ? __ldg(a.sel_bias + e) : 0.f)) : 0u;
    } else {
      key[i] = ok ? logit_key(v) : 0u;
    }
    val[i] = v;
    id[i] = e;
  }
}

// ---------------------------------------------------------------------------
// Routing finish inside the router kernel (its last CTA, nthreads threads
// meeting on named barrier `bar`): per token the k largest scores of all E
// experts, equal scores going to the lower id; then the weights (softmax
// over the selected logits, or the selected sigmoid scores normalised),
// written in ascending expert id.
//
// Two levels, every warp of the CTA busy: the experts are cut into slices of
// at most 128 (4 per lane, in registers); a warp takes a (token, slice) pair
// and writes the slice's top-k to shared memory, ids ascending within and
// across slices; then one warp per token selects the top-k of those
// candidates (at most 8 per lane).  Every member of the overall top-k is in
// its slice's top-k (at most k-1 experts of the slice precede it in the
// order score desc, id asc), so the result equals a scan of all E experts.
// Tokens go in rounds of as many as the scratch holds.
constexpr int kBucketScratchBytes = 8 * kMaxExperts + 4 * kMaxExperts + 4 * 64;  // s_mask, s_off, s_wsum
constexpr int kTopkSlice = 128;
constexpr int kTopkCandBytes = 48 * 1024;  // scratch: candidates (key, value, id) of one round

__device__ void topk_tail(const GemvArgs& a, const float* __restrict__ lg, int tid, int nthreads, int bar,
                          unsigned char* scratch) {
  const int B = a.n_tokens, E = a.n_experts, k = a.top_k;
  const int nw = nthreads >> 5, warp = tid >> 5, lane = tid & 31;
  const int n_sl = (E + kTopkSlice - 1) / kTopkSlice;  // <= 8: at most 8*k <= 256 candidates per token
  const int per_tok = n_sl * k;
  const int tb = max(1, min(B, kTopkCandBytes / (12 * per_tok)));  // tokens per round
  uint32_t* ck = reinterpret_cast<uint32_t*>(scratch);
  float* cv = reinterpret_cast<float*>(scratch + 4 * (kTopkCandBytes / 12));
  int* ci = reinterpret_cast<int*>(scratch + 8 * (kTopkCandBytes / 12));
  for (int b0 = 0; b0 < B; b0 += tb) {
    const int nb = min(tb, B - b0);
    for (int job = warp; job < nb * n_sl; job += nw) {
      const int bl = job / n_sl, sl = job - bl * n_sl;
      const int lo = sl * kTopkSlice, hi = min(E, lo + kTopkSlice);
      uint32_t key[4];
      float val[4];
      int id[4];
      topk_load<4>(a, lg, b0 + bl, lo, hi, lane, key, val, id);
      const uint32_t sel = warp_select_topk<4>(key, k, lane);
      const int ns = __popc(sel);
      int pre = ns;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, pre, o);
        if (lane >= o) pre += t;
      }
      const int total = __shfl_sync(0xFFFFFFFFu, pre, 31);  // min(k, slice size)
      pre -= ns;
      const int base = job * k;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if ((sel >> i) & 1u) {
          ck[base + pre] = key[i];
          cv[base + pre] = val[i];
          ci[base + pre] = id[i];
          ++pre;
        }
      for (int j = total + lane; j < k; j += 32) ck[base + j] = 0u;  // empty slots (key 0: no expert)
    }
    named_bar_sync(bar, nthreads);
    for (int bl = warp; bl < nb; bl += nw) {
      const int PL = (per_tok + 31) / 32;  // <= 8
      uint32_t key[8];
      float val[8];
      int id[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = lane * PL + i;
        const bool ok = i < PL && c < per_tok;
        key[i] = ok ? ck[bl * per_tok + c] : 0u;
        val[i] = ok ? cv[bl * per_tok + c] : 0.f;
        id[i] = ok ? ci[bl * per_tok + c] : 0;
      }
      const uint32_t sel = warp_select_topk<8>(key, k, lane);
      // this token's candidate slots are free once the warp has them in registers
      topk_write<8>(a, b0 + bl, sel, val, id, lane, cv + bl * per_tok, ci + bl * per_tok);
    }
    named_bar_sync(bar, nthreads);  // the next round reuses the scratch
  }
}

// Buckets of the B*k pairs from topk_idx (global, written by this block
// before a barrier): counts, exclusive offsets, pair ids sorted by
// (expert, b, j), the active list.  nt threads (a multiple of 32, at most
// 32 warps) meeting on named barrier `bar`, each owning ceil(E/nt) experts;
// scratch: s_mask [E] u64, s_off [E] int, s_wsum [2*32] int.
__device__ void bucket_block(const GemvArgs& a, int B, int tid, int nt, int bar, unsigned long long* s_mask,
                             int* s_off, int* s_wsum) {
  const int E = a.n_experts, k = a.top_k;
  const int lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += nt) s_mask[e] = 0ull;
  named_bar_sync(bar, nt);
  for (int p = tid; p < B * k; p += nt) atomicOr(&s_mask[__ldcg(a.topk_idx + p)], 1ull << (p / k));
  named_bar_sync(bar, nt);
  // thread t owns the experts [t*per, (t+1)*per): counts, then block scans
  // of the pair counts and of the active flags
  const int per = (E + nt - 1) / nt;
  const int e_lo = min(E, tid * per), e_hi = min(E, e_lo + per);
  int tc = 0, ta = 0;
  for (int e = e_lo; e < e_hi; ++e) {
    const int c = __popcll(s_mask[e]);
    tc += c;
    ta += c > 0;
  }
  int ic = tc, ia = ta;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t1 = __shfl_up_sync(0xFFFFFFFFu, ic, o);
    const int t2 = __shfl_up_sync(0xFFFFFFFFu, ia, o);
    if (lane >= o) {
      ic += t1;
      ia += t2;
    }
  }
  if (lane == 31) {
    s_wsum[2 * warp] = ic;
    s_wsum[2 * warp + 1] = ia;
  }
  named_bar_sync(bar, nt);
  int wc = 0, wa = 0;
  for (int w = 0; w < warp; ++w) {
    wc += s_wsum[2 * w];
    wa += s_wsum[2 * w + 1];
  }
  int off = wc + ic - tc, act = wa + ia - ta;
  for (int e = e_lo; e < e_hi; ++e) {
    const int c = __popcll(s_mask[e]);
    s_off[e] = off;
    a.offsets_out[e] = off;
    a.counts[e] = c;
    if (c > 0) a.active_out[act++] = e;
    off += c;
  }
  if (e_lo < E && e_hi == E) {  // the thread owning the last expert
    a.offsets_out[E] = off;
    *a.n_active_out = act;
  }
  named_bar_sync(bar, nt);
  for (int p = tid; p < B * k; p += nt) {
    const int e = __ldcg(a.topk_idx + p);
    const int bb = p / k;
    const unsigned long long below = (bb == 0) ? 0ull : (s_mask[e] & ((1ull << bb) - 1ull));
    a.pair_ids_out[s_off[e] + __popcll(below)] = p;
  }
}

// Top-k of one token with a whole block (nt threads: 2 to 32 warps).  The
// order is (key descending, id ascending): the pages' tie rule as the rest of
// the library applies it.  Warp w takes the ids [w*S, (w+1)*S), S = E / nw
// rounded up, PL of them per lane (id = lo + lane + 32*i); each lane sorts
// its own in registers, then the warp takes its k best by k rounds of "the
// best lane head wins and pops" (one max-reduction and one ballot per round;
// a second reduction only when keys tie).  Warp 0 merges the nw sorted lists
// the same way, orders the k winners by id and writes them through
// topk_emit.  With bucket_b1 (a batch of one token) the routing plan is
// written here too: the active list is the selection, offsets count the
// selected ids below each expert, the pairs are in order.
constexpr int kTopkBlockScratch = 12 * 32 * kMaxTopK + 8 * 2 * kMaxTopK + 64;

struct TopkHead {
  uint32_t hi, lo;  // key (0: none) and ~id
  float v;
};

__device__ __forceinline__ bool topk_before(const TopkHead& a, const TopkHead& b) {
  return a.hi > b.hi || (a.hi == b.hi && a.lo > b.lo);
}

// the lane whose head is first in the order among all lanes (-1: every head empty)
__device__ __forceinline__ int topk_round_winner(const TopkHead& h) {
  const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, h.hi);
  if (m == 0u) return -1;
  unsigned bal = __ballot_sync(0xFFFFFFFFu, h.hi == m);
  if (__popc(bal) > 1) {
    const uint32_t ml = __reduce_max_sync(0xFFFFFFFFu, h.hi == m ? h.lo : 0u);
    bal = __ballot_sync(0xFFFFFFFFu, h.hi == m && h.lo == ml);
  }
  return __ffs(bal) - 1;
}

template <int PLM>
__device__ void topk_token_block_pl(const GemvArgs& a, const float* __restrict__ lg, int b, int tid, int nt, int bar,
                                    bool bucket_b1, unsigned char* scratch) {
  const int E = a.n_experts, k = a.top_k;
  const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
  const int S = (E + nw - 1) / nw, lo = warp * S, hi = min(E, lo + S);
  uint32_t* c_hi = reinterpret_cast<uint32_t*>(scratch);  // [nw][k] each warp's list, in order
  uint32_t* c_lo = c_hi + 32 * kMaxTopK;
  float* c_v = reinterpret_cast<float*>(c_lo + 32 * kMaxTopK);
  int* s_id = reinterpret_cast<int*>(c_v + 32 * kMaxTopK);  // the selection, ascending id
  float* s_v = reinterpret_cast<float*>(s_id + kMaxTopK);
  TopkHead h[PLM];
#pragma unroll
  for (int i = 0; i < PLM; ++i) {
    const int e = lo + lane + 32 * i;
    const bool ok = e < hi;
    float v = ok ? __ldcg(lg + e) : 0.f;
    uint32_t key;
    if (a.scoring == 1) {
      v = 1.0f / (1.0f + expf(-v));
      key = ok ? logit_key(v + (a.sel_bias ? __ldg(a.sel_bias + e) : 0.f)) : 0u;
    } else {
      key = ok ? logit_key(v) : 0u;
    }
    h[i].hi = key;
    h[i].lo = ~(uint32_t)e;
    h[i].v = v;
  }
  // lane-local sort, first in the order at h[0] (odd-even transposition)
#pragma unroll
  for (int pass = 0; pass < PLM; ++pass) {
#pragma unroll
    for (int i = pass & 1; i + 1 < PLM; i += 2) {
      if (topk_before(h[i + 1], h[i])) {
        const TopkHead t = h[i];
        h[i] = h[i + 1];
        h[i + 1] = t;
      }
    }
  }
  if (lane < k) c_hi[warp * k + lane] = 0u;
  __syncwarp();
  for (int r = 0; r < k; ++r) {
    const int w = topk_round_winner(h[0]);
    if (w < 0) break;
    if (lane == w) {
      c_hi[warp * k + r] = h[0].hi;
      c_lo[warp * k + r] = h[0].lo;
      c_v[warp * k + r] = h[0].v;
#pragma unroll
      for (int i = 0; i + 1 < PLM; ++i) h[i] = h[i + 1];
      h[PLM - 1].hi = 0u;
    }
  }
  named_bar_sync(bar, nt);
  if (warp == 0) {
    // merge: lane l < nw walks list l
    int ptr = 0;
    TopkHead cur;
    cur.hi = lane < nw ? c_hi[lane * k] : 0u;
    cur.lo = lane < nw ? c_lo[lane * k] : 0u;
    cur.v = lane < nw ? c_v[lane * k] : 0.f;
    int my_id = 0;
    float my_v = 0.f;
    for (int r = 0; r < k; ++r) {
      const int w = topk_round_winner(cur);
      const uint32_t wl = __shfl_sync(0xFFFFFFFFu, cur.lo, w < 0 ? 0 : w);
      const float wv = __shfl_sync(0xFFFFFFFFu, cur.v, w < 0 ? 0 : w);
      if (lane == r) {
        my_id = (int)~wl;
        my_v = wv;
      }
      if (lane == w) {
        ++ptr;
        const bool more = ptr < k;
        cur.hi = more ? c_hi[lane * k + ptr] : 0u;
        cur.lo = more ? c_lo[lane * k + ptr] : 0u;
        cur.v = more ? c_v[lane * k + ptr] : 0.f;
      }
    }
    // ascending id: lane r's rank among the k winners
    int rank = 0;
    for (int i = 0; i < k; ++i) {
      const int oi = __shfl_sync(0xFFFFFFFFu, my_id, i);
      rank += (lane < k && oi < my_id) ? 1 : 0;
    }
    if (lane < k) {
      s_id[rank] = my_id;
      s_v[rank] = my_v;
    }
    __syncwarp();
    const bool on = lane < k;
    const int id = on ? s_id[lane] : 0;
    topk_emit(a, b, on ? s_v[lane] : 0.f, id, lane);
    if (bucket_b1) {
      if (on) {
        a.active_out[lane] = id;
        a.pair_ids_out[lane] = lane;
      }
      if (lane == 0) {
        a.offsets_out[E] = k;
        *a.n_active_out = k;
      }
    }
  }
  if (bucket_b1) {
    named_bar_sync(bar, nt);  // the selection, ascending, in s_id
    for (int e = tid; e < E; e += nt) {
      int below = 0;
      bool on = false;
      for (int i = 0; i < k; ++i) {
        const int si = s_id[i];
        below += si < e ? 1 : 0;
        on = on || si == e;
      }
      a.offsets_out[e] = below;
      a.counts[e] = on ? 1 : 0;
    }
  }
}

__device__ void topk_token_block(const GemvArgs& a, const float* __restrict__ lg, int b, int tid, int nt, int bar,
                                 bool bucket_b1, unsigned char* scratch) {
  const int nw = nt >> 5, E = a.n_experts;
  const int per_lane = ((E + nw - 1) / nw + 31) / 32;
  if (nw < 2 || nw > 32 || a.top_k < 1 || a.top_k > kMaxTopK || a.top_k > E || per_lane > 16) {
    if (tid == 0) atomicExch(a.err, kErrBadPlan);
    return;
  }
  if (per_lane <= 4) topk_token_block_pl<4>(a, lg, b, tid, nt, bar, bucket_b1, scratch);
  else topk_token_block_pl<16>(a, lg, b, tid, nt, bar, bucket_b1, scratch);
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
