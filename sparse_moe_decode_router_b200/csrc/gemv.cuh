// Warp-item streaming GEMV for the MoE decode layer (sm_100a).
//
// Decode at batch <= 64 streams each active weight matrix from HBM once per
// step and multiplies it with a handful of activation vectors.  The kernel:
//
//  * persistent CTAs, one per SM; each owns a contiguous range of work items
//    (an item = R consecutive output rows of one group: one active expert,
//    or the single dense group of the router / shared expert), sized so that
//    each TMA copy moves 14-32 KB;
//  * one producer lane moves every item's weight rows (codes, and for MXFP4
//    the E8M0 scale rows) into a ring of shared-memory stages with 1-D TMA
//    bulk copies (evict-first L2 policy: weights are read once per step);
//    completion is counted on per-stage mbarriers;
//  * an item is taken by a group of warps.  By default each warp owns whole
//    rows and its lanes split K, so a row's dot product needs only an in-warp
//    butterfly and the stage is handed back with one mbarrier arrive per
//    warp.  The bf16 router and shared gate/up split K over the group's
//    warps, and the one-token MXFP4 down projection ("split-K" instances)
//    gives each lane one 32-element block of a warp-wide K slice; there the
//    warps' partial sums meet in shared memory behind a group barrier and
//    are added in ascending slice order by one warp;
//  * the activation vectors an item needs sit in shared memory, staged once
//    per "phase" (a run of groups whose tokens fit): MXFP4 streams keep them
//    as f16 scaled by a per-vector power of two (exact for bf16 inputs,
//    11-bit rounding for fp32 ones) in a lane-interleaved layout that makes
//    every 16-byte read conflict-free; bf16 streams keep bf16 or fp32 as is;
//  * MXFP4 weights are decoded in registers (cvt e2m1x2 -> f16x2); products
//    and partial sums over eight products are packed f16 (fma.rn.f16x2), the
//    block's partial sums are added in fp32 and scaled by its E8M0 value, and
//    blocks accumulate in fp32; bf16 weights use mixed fp32 FMAs;
//  * epilogues: store, SwiGLU, router logits (+ bias; top-k follows in its own
//    kernel), and the down projection fused with the routing-weight combine
//    and residual add (the warp group that completes a row tile over all
//    active experts combines it in ascending expert order).
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

enum XKind : int { X_BF16 = 0, X_F32 = 1 };

// 16 consumer warps: four 4-warp groups per SM (measured faster than 12 on the
// one-token down projection; 20 spills its registers)
#ifndef MOE_MAX_CONSUMER_WARPS
#define MOE_MAX_CONSUMER_WARPS 16
#endif
constexpr int kMaxConsumerWarps = MOE_MAX_CONSUMER_WARPS;
// the MXFP4 gate/up streams (two weight rows per output, K = hidden) keep 12:
// measured faster there (the 16-warp launch bound cuts their registers to 96)
#ifndef MOE_GU_CONSUMER_WARPS
#define MOE_GU_CONSUMER_WARPS 12
#endif
// consumer warps of a whole-row (not split-K) instance: its launch bound and its plans
__host__ __device__ constexpr int consumer_warps_for(int wf, int epi) {
  return (wf == W_MXFP4 && epi == EPI_SWIGLU && MOE_GU_CONSUMER_WARPS < kMaxConsumerWarps) ? MOE_GU_CONSUMER_WARPS
                                                                                        : kMaxConsumerWarps;
}
// Split-K instances (one token, MXFP4, compile-time K): more, lighter warps.
#ifndef MOE_MAX_SPLITK_WARPS
#define MOE_MAX_SPLITK_WARPS 16
#endif
constexpr int kMaxSplitKWarps = MOE_MAX_SPLITK_WARPS;
constexpr int kMaxWarpsAny = kMaxSplitKWarps > kMaxConsumerWarps ? kMaxSplitKWarps : kMaxConsumerWarps;
constexpr int kSplitKRows = 8;  // weight rows per warp in the split-K instances
// cross-warp partial sums of the split-K instances: two item buffers per group
constexpr int kRedFloats = 2 * kMaxSplitKWarps * kSplitKRows;
constexpr int kMaxStagesDev = 24;     // stage ring slots the shared-memory header reserves
constexpr int kMaxStageUnits = 64;    // (vector, segment) units of one staging pass
constexpr int kMaxPhases = 32;
constexpr int kMaxSlots = 32;

struct PhaseDesc {
  int g0, g1;    // groups [g0, g1) (indices into the active list; 0..1 for dense)
  int t0, t1;    // token range inside each group's token list (split groups only; else 0, INT_MAX)
  int nslots;    // activation vectors staged for this phase
  int first_item, last_item;  // CTA-local item range [first, last) of this phase
};

struct PhaseTable {
  int n;
  int bad;
  PhaseDesc ph[kMaxPhases];
  int slot_src[kMaxPhases][kMaxSlots];  // source row of each slot (token or pair)
};

// ---------------------------------------------------------------------------
// packed f16x2 multiply-adds (one rounding each) and the f16x2 -> fp32 sum
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ float h2_sum_f32(uint32_t v) {
  float lo, hi;
  asm("{\n\t.reg .f16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.f32.f16 %0, l;\n\t"
      "cvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(v));
  return lo + hi;
}

// mixed-precision FMAs: fp32 accumulator, two bf16 products from packed pairs
__device__ __forceinline__ float fma2_bf16(uint32_t w2, uint32_t x2, float acc) {
  asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %1;\n\t"
      "mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.bf16 %0, a0, b0, %0;\n\t"
      "fma.rn.f32.bf16 %0, a1, b1, %0;\n\t}"
      : "+f"(acc)
      : "r"(w2), "r"(x2));
  return acc;
}

// 32-element MXFP4 chunk (16 code bytes = 16 f16x2 after decode, element pair
// j in w[j]) dotted with a 32-element f16 activation chunk (4 x 16 bytes,
// lane-interleaved).  Products and the two partial sums are packed f16x2: the
// even pairs go to one accumulator, the odd pairs to the other, so each f16
// lane sums eight products, each with one rounding (the products themselves
// are exact for bf16 activations: 2 + 8 significant bits).  The activations
// are staged with max|x| in [2^8, 2^9), so a partial sum stays below
// 8 * 6 * 2^9 = 24576 < 65504.  The four partial sums are added in fp32.
__device__ __forceinline__ float dot32_h2(const uint32_t (&w)[16], const uint4 (&xv)[4]) {
  uint32_t a0 = hmul2(w[0], xv[0].x), a1 = hmul2(w[1], xv[0].y);
  a0 = hfma2(w[2], xv[0].z, a0);
  a1 = hfma2(w[3], xv[0].w, a1);
#pragma unroll
  for (int q = 1; q < 4; ++q) {
    a0 = hfma2(w[4 * q + 0], xv[q].x, a0);
    a1 = hfma2(w[4 * q + 1], xv[q].y, a1);
    a0 = hfma2(w[4 * q + 2], xv[q].z, a0);
    a1 = hfma2(w[4 * q + 3], xv[q].w, a1);
  }
  return h2_sum_f32(a0) + h2_sum_f32(a1);
}

__device__ __forceinline__ void decode_chunk(const uint4 q, uint32_t (&w)[16]) {
  uint32_t t[4];
  e2m1x8_to_f16x2(q.x, t);
  w[0] = t[0]; w[1] = t[1]; w[2] = t[2]; w[3] = t[3];
  e2m1x8_to_f16x2(q.y, t);
  w[4] = t[0]; w[5] = t[1]; w[6] = t[2]; w[7] = t[3];
  e2m1x8_to_f16x2(q.z, t);
  w[8] = t[0]; w[9] = t[1]; w[10] = t[2]; w[11] = t[3];
  e2m1x8_to_f16x2(q.w, t);
  w[12] = t[0]; w[13] = t[1]; w[14] = t[2]; w[15] = t[3];
}

// f16 activation layout in shared memory: element k of a K-vector, k = 32*b + 8*q + j
// (chunk b = 32*i + l), lives at half index ((i*4 + q)*32 + l)*8 + j.  Lane l's q-th
// 16-byte read of chunk b is then contiguous across the warp.
__device__ __forceinline__ int xperm_index(int k) {
  const int b = k >> 5, q = (k >> 3) & 3, j = k & 7;
  const int i = b >> 5, l = b & 31;
  return (((i * 4 + q) * 32 + l) << 3) + j;
}

// ---------------------------------------------------------------------------
// Phase table: runs of groups whose activation vectors fit in `xcap` slots.
// Built by one thread; `lo`/`hi` = the CTA's item range.
__device__ void build_phases(const GemvArgs& a, long long lo, long long hi, int n_rt, int xcap,
                             PhaseTable& pt) {
  pt.n = 0;
  pt.bad = 0;
  if (lo >= hi) return;
  if (!a.routed) {
    // dense: token chunks of xcap, each over the whole item range
    for (int t0 = 0; t0 < a.n_tokens; t0 += xcap) {
      if (pt.n == kMaxPhases) { pt.bad = 1; return; }
      PhaseDesc& p = pt.ph[pt.n];
      p.g0 = 0; p.g1 = 1;
      p.t0 = t0; p.t1 = min(a.n_tokens, t0 + xcap);
      p.nslots = p.t1 - p.t0;
      for (int s = 0; s < p.nslots; ++s) pt.slot_src[pt.n][s] = t0 + s;
      p.first_item = 0;
      p.last_item = (int)(hi - lo);
      ++pt.n;
    }
    return;
  }
  const int gfirst = (int)(lo / n_rt), glast = (int)((hi - 1) / n_rt);
  int cur = -1;  // open phase index
  for (int g = gfirst; g <= glast; ++g) {
    const int e = clamp_group(a.active[g], a.n_experts, nullptr);
    const int b0 = a.offsets[e], cnt = a.offsets[e + 1] - b0;
    const long long ilo = max(lo, (long long)g * n_rt), ihi = min(hi, (long long)(g + 1) * n_rt);
    // activation rows this group needs
    int need[kMaxSlots];
    int nneed = 0;
    bool split = false;
    for (int t = 0; t < cnt; ++t) {
      int p = a.pair_ids[b0 + t];
      if (p < 0 || p >= a.n_pairs) p = 0;
      const int src = a.act_by_pair ? p : p / a.top_k;
      bool dup = false;
      for (int u = 0; u < nneed; ++u) dup |= (need[u] == src);
      if (!dup) {
        if (nneed == xcap || nneed == kMaxSlots) { split = true; break; }
        need[nneed++] = src;
      }
    }
    if (split) {
      // a group with more activation rows than slots: own phases, token chunks of xcap
      cur = -1;
      for (int t0 = 0; t0 < cnt; t0 += xcap) {
        if (pt.n == kMaxPhases) { pt.bad = 1; return; }
        PhaseDesc& p = pt.ph[pt.n];
        p.g0 = g; p.g1 = g + 1;
        p.t0 = t0; p.t1 = min(cnt, t0 + xcap);
        p.nslots = 0;
        for (int t = p.t0; t < p.t1; ++t) {
          int pr = a.pair_ids[b0 + t];
          if (pr < 0 || pr >= a.n_pairs) pr = 0;
          pt.slot_src[pt.n][p.nslots++] = a.act_by_pair ? pr : pr / a.top_k;  // duplicates allowed
        }
        p.first_item = (int)(ilo - lo);
        p.last_item = (int)(ihi - lo);
        ++pt.n;
      }
      continue;
    }
    // try to extend the open phase with this group's new rows
    if (cur >= 0) {
      PhaseDesc& p = pt.ph[cur];
      int add = 0;
      for (int u = 0; u < nneed; ++u) {
        bool have = false;
        for (int s = 0; s < p.nslots; ++s) have |= (pt.slot_src[cur][s] == need[u]);
        add += !have;
      }
      if (p.nslots + add <= xcap) {
        for (int u = 0; u < nneed; ++u) {
          bool have = false;
          for (int s = 0; s < p.nslots; ++s) have |= (pt.slot_src[cur][s] == need[u]);
          if (!have) pt.slot_src[cur][p.nslots++] = need[u];
        }
        p.g1 = g + 1;
        p.last_item = (int)(ihi - lo);
        continue;
      }
    }
    if (pt.n == kMaxPhases) { pt.bad = 1; return; }
    cur = pt.n++;
    PhaseDesc& p = pt.ph[cur];
    p.g0 = g; p.g1 = g + 1;
    p.t0 = 0; p.t1 = 1 << 30;
    p.nslots = nneed;
    for (int u = 0; u < nneed; ++u) pt.slot_src[cur][u] = need[u];
    p.first_item = (int)(ilo - lo);
    p.last_item = (int)(ihi - lo);
  }
}

// 2^e as an exact fp32 (e clamped to the normal range).
__device__ __forceinline__ float pow2f(int e) {
  e = max(-126, min(127, e));
  return __uint_as_float((uint32_t)(e + 127) << 23);
}

// Staging of activation vectors into shared memory.  Activations come from
// the preceding kernel, which under programmatic dependent launch may still
// be writing them while this grid starts: they are read through L2 only
// (ld.global.cg), never through the non-coherent read-only path, which is
// reserved for weights that no kernel writes.  MXFP4 streams: f16 of
// x * 2^-e in the lane-interleaved layout, e chosen from max|x| so that the
// largest element sits in [2^8, 2^9) (exact for bf16 inputs down to 2^-25 of
// the largest element, one rounding for fp32 ones); the headroom above keeps
// the f16 partial sums of dot32_h2 finite.  bf16 streams: a plain copy of the bf16 or fp32 row.
// Work is split into (vector, segment) units over all consumer warps; all
// loads are 16-byte vectors with several in flight.

// max |x| over 8-element groups [g0, g1) of row `row`
template <int XK>
__device__ float segment_amax(const void* src_base, int row, int K, int g0, int g1, int lane) {
  float amax = 0.f;
  if constexpr (XK == X_F32) {
    const float4* s = reinterpret_cast<const float4*>(static_cast<const float*>(src_base) + (size_t)row * K);
#pragma unroll 4
    for (int g = g0 + lane; g < g1; g += 32) {
      const float4 v0 = __ldcg(s + 2 * g), v1 = __ldcg(s + 2 * g + 1);
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v0.x), fabsf(v0.y)), fmaxf(fabsf(v0.z), fabsf(v0.w))));
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v1.x), fabsf(v1.y)), fmaxf(fabsf(v1.z), fabsf(v1.w))));
    }
  } else {
    const uint4* s = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src_base) + (size_t)row * K);
#pragma unroll 4
    for (int g = g0 + lane; g < g1; g += 32) {
      const uint4 v = __ldcg(s + g);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fmaxf(fabsf(bf16lo_to_f32(w[j])), fabsf(bf16hi_to_f32(w[j]))));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  return amax;
}

// 8-element groups [g0, g1) of row `row` -> f16 * 2^-e, interleaved layout
template <int XK>
__device__ void segment_to_f16(const void* src_base, int row, int K, int g0, int g1, float scale, unsigned char* dst,
                               int lane) {
#pragma unroll 4
  for (int g = g0 + lane; g < g1; g += 32) {
    float v[8];
    if constexpr (XK == X_F32) {
      const float4* s = reinterpret_cast<const float4*>(static_cast<const float*>(src_base) + (size_t)row * K);
      const float4 v0 = __ldcg(s + 2 * g), v1 = __ldcg(s + 2 * g + 1);
      v[0] = v0.x; v[1] = v0.y; v[2] = v0.z; v[3] = v0.w; v[4] = v1.x; v[5] = v1.y; v[6] = v1.z; v[7] = v1.w;
    } else {
      const uint4* s = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src_base) + (size_t)row * K);
      const uint4 u = __ldcg(s + g);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] = bf16lo_to_f32(w[j]);
        v[2 * j + 1] = bf16hi_to_f32(w[j]);
      }
    }
    uint32_t hv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 h2 = __floats2half2_rn(v[2 * j] * scale, v[2 * j + 1] * scale);
      hv[j] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    // 8 consecutive elements k = 8g .. 8g+7 stay contiguous in the interleaved layout
    *reinterpret_cast<uint4*>(dst + 2 * xperm_index(8 * g)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
  }
}

__device__ __forceinline__ int shift_for_amax(float amax) {
  int e = 0;
  if (amax > 0.f && amax < INFINITY) {
    const int ef = (int)((__float_as_uint(amax) >> 23) & 0xFF);
    e = (ef > 0 ? ef - 127 : -127) - 8;  // floor(log2(amax)) - 8
    e = max(-126, min(127, e));
  }
  return e;
}

template <int WF, int XK>
__device__ void stage_phase(const void* src, const int* slot_src, int nslots, int K, unsigned char* xbuf,
                            int xrow_bytes, int* slot_e, float* s_amax, int warp, int ncw, int lane, int nct) {
  if (nslots <= 0) return;
  const int ngrp = K >> 3;
  int nseg = max(1, ncw / nslots);
  nseg = min(nseg, max(1, kMaxStageUnits / nslots));
  const int seglen = (ngrp + nseg - 1) / nseg;
  const int units = nslots * nseg;
  if constexpr (WF == W_MXFP4) {
    for (int u = warp; u < units; u += ncw) {
      const int sl = u / nseg, q = u - sl * nseg;
      const float m = segment_amax<XK>(src, slot_src[sl], K, q * seglen, min(ngrp, (q + 1) * seglen), lane);
      if (lane == 0) s_amax[u] = m;
    }
    named_bar_sync(1, nct);
    for (int u = warp; u < units; u += ncw) {
      const int sl = u / nseg, q = u - sl * nseg;
      float m = 0.f;
      for (int i = 0; i < nseg; ++i) m = fmaxf(m, s_amax[sl * nseg + i]);
      const int e = shift_for_amax(m);
      if (lane == 0 && q == 0) slot_e[sl] = e;
      segment_to_f16<XK>(src, slot_src[sl], K, q * seglen, min(ngrp, (q + 1) * seglen), pow2f(-e),
                         xbuf + (size_t)sl * xrow_bytes, lane);
    }
  } else {
    const int esz = (XK == X_F32) ? 4 : 2;
    const int n16 = K * esz / 16;
    const int seg16 = (n16 + nseg - 1) / nseg;
    for (int u = warp; u < units; u += ncw) {
      const int sl = u / nseg, q = u - sl * nseg;
      const uint4* s = reinterpret_cast<const uint4*>(static_cast<const unsigned char*>(src) +
                                                      (size_t)slot_src[sl] * K * esz);
      uint4* d = reinterpret_cast<uint4*>(xbuf + (size_t)sl * xrow_bytes);
      const int i1 = min(n16, (q + 1) * seg16);
#pragma unroll 4
      for (int i = q * seg16 + lane; i < i1; i += 32) d[i] = __ldcg(s + i);
      if (lane == 0 && q == 0) slot_e[sl] = 0;
    }
  }
}

// Bytes of one staged activation vector (MXFP4 streams: whole groups of 32
// chunks in the interleaved f16 layout).
__host__ __device__ constexpr int x_row_bytes(int wf, int xk, int K) {
  return wf == W_MXFP4 ? ((K / 32 + 31) / 32) * 2048 : K * (xk == X_F32 ? 4 : 2);
}

// ---------------------------------------------------------------------------
// Fused combine bookkeeping.  A warp group writes the unweighted expert
// outputs y of its items to the scratch; every kPubBatch items all warps of
// the group meet in publish_round().  After a group barrier (the group's y
// stores are then ordered before the leader's fence) the leader warp issues
// one gpu-scope fence and one tile-counter atomic per item (lanes in
// parallel).  The atomics' results are examined one round later, so their
// latency hides behind the next batch: the row tiles whose count reached the
// number of active experts are listed in shared memory, and after a second
// group barrier every warp of the group combines them, one output element per
// lane, in ascending expert order.
constexpr int kPubBatch = 8;


constexpr int kPubInts = kPubBatch + 1;  // per group: [0] = tiles to combine, [1..] = their row tiles

__device__ __forceinline__ void group_bar(int q0, int wpi) {
  named_bar_sync(3 + q0, wpi * 32);
}

__device__ void publish_round(const GemvArgs& a, const int* pend_rt, int npend, int& prev_cnt, int& prev_rt,
                              int& nprev, int n_groups, int wi, int q0, int lane, int* s_pub) {
  group_bar(q0, a.wpi);  // every warp of the group has written its y rows of the pending items
  if (wi == 0) {
    // results of the previous round first (their atomics completed long ago)
    const bool rdy = lane < nprev && prev_cnt == n_groups - 1;
    const unsigned m = __ballot_sync(0xFFFFFFFFu, rdy);
    if (rdy) {
      s_pub[1 + __popc(m & ((1u << lane) - 1u))] = prev_rt;
      a.tile_counter[prev_rt] = 0;  // every contribution has arrived: ready for the next launch
    }
    if (lane == 0) s_pub[0] = __popc(m);
    if (m) fence_acq_rel_gpu();  // acquire: the other contributors' y stores before our loads
    if (npend > 0) {
      fence_acq_rel_gpu();  // release: this group's y stores (ordered by the group barrier) before its counts
      int rt = 0;
#pragma unroll
      for (int i = 0; i < kPubBatch; ++i)
        if (lane == i) rt = pend_rt[i];
      prev_rt = rt;
      prev_cnt = (lane < npend) ? atomicAdd(&a.tile_counter[rt], 1) : -1;
    }
  }
  nprev = npend;
  group_bar(q0, a.wpi);
  const int nready = s_pub[0];
  if (nready == 0) return;
  const int H = a.out_rows, per_tile = a.batch * a.R;
  for (int o = wi * 32 + lane; o < nready * per_tile; o += a.wpi * 32) {
    const int ti = o / per_tile, q = o - ti * per_tile;
    const int b = q / a.R, r = s_pub[1 + ti] * a.R + (q - (q / a.R) * a.R);
    a.out_bf16[(size_t)b * H + r] = combine_one(a, a.out, H, b, r);
  }
}

// ---------------------------------------------------------------------------
// Per-item token list: up to TMAX (slot, output row, exponent) per pass.
struct TokenPass {
  int n;
  int slot[4];
  int orow[4];
  int e[4];
};

// RPW = output rows per warp (SwiGLU: one gate row and one up row per output row).
// An item (R = RPW * wpi output rows, one stage) is shared by a group of wpi warps.
// KT: the reduction length as a compile-time constant (0 = taken from the
// arguments).  Specialised instances unroll the chunk loop with constant
// addressing and, for MXFP4, read the E8M0 scale bytes from global memory with
// loads issued ahead of the stage wait (the stage then holds codes only).
//
// The body runs as a device function so that the persistent single-launch
// layer can run several streams back to back in one kernel; a block may then
// have more threads than this stream's plan uses: the extra warps leave at
// once, and every barrier below counts only the plan's (ncw + 1) warps.
constexpr int kBarAll = 15;  // named barrier over all of a stream's warps
// named barriers: 1 (consumers), 2 (phase table), 3 + group (item groups), kBarAll
constexpr int kMaxItemGroups = kBarAll - 3;
// warps per item that keep ncw / wpi <= kMaxItemGroups for any ncw <= kMaxWarpsAny
constexpr int kMinItemWarps = (kMaxWarpsAny + kMaxItemGroups - 1) / kMaxItemGroups;

template <int WF, int EPI, int XK, int TMAX, int RPW, int KT>
__device__ __forceinline__ void gemv_body(const GemvArgs& a, unsigned char* smem) {
  constexpr bool kSwiglu = (EPI == EPI_SWIGLU);
  // router: expert rows, then (optionally) the shared expert's gate/up rows as
  // extra items, then the top-k / weights / buckets in the last CTA
  constexpr bool kRouter = (EPI == EPI_ROUTER);
  constexpr int NWR = kSwiglu ? 2 * RPW : RPW;  // weight rows per warp
  static_assert(NWR % 2 == 0, "rows are processed in pairs");
  // kFast: the split-K instance.  Lanes own one 32-element chunk each, a
  // warp covers 32 chunks (a K slice) of NWR rows, and an item's KS slices go
  // to KS warps of the group (times R / RPW row quarters).
  constexpr bool kOneTokMx = (KT != 0) && (WF == W_MXFP4) && (TMAX == 1);
  constexpr bool kFast = kOneTokMx && NWR == kSplitKRows;
  // kUnroll: one token, compile-time K, whole rows per warp (lane-strided
  // chunks, fully unrolled, constant shared-memory offsets)
  constexpr bool kUnroll = kOneTokMx && !kFast;
  constexpr int KS = KT ? ((KT / 32) + 31) / 32 : 1;  // K slices of 32 chunks (= chunks per lane when unrolled)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ncw = a.ncw;
  if (warp > ncw) return;  // beyond this stream's plan (persistent layer only)
  const int K = KT ? KT : a.K;
  const bool sglobal = a.scales_global != 0;
  const int C = K >> 5;                                   // 32-element chunks per row
  const int rowbytes = (WF == W_MXFP4) ? (K >> 1) : (K << 1);
  const int sblocks = K >> 5;
  const int rows_per_item = kSwiglu ? 2 * a.R : a.R;
  const int codes_bytes = rows_per_item * rowbytes;
  const int xrow_bytes = x_row_bytes(WF, XK, K);

  // shared memory: [barriers][phase table][slot exponents][x slots][stages]
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty_bar = full_bar + a.n_stages;
  PhaseTable* pt = reinterpret_cast<PhaseTable*>(smem + 16 * 64);
  int* slot_e = reinterpret_cast<int*>(smem + 16 * 64 + sizeof(PhaseTable));
  volatile int* s_flag = slot_e + kMaxSlots;
  int* s_item_cnt = slot_e + kMaxSlots + 2;  // [n_stages] warps done with the item in that stage
  float* s_amax = reinterpret_cast<float*>(s_item_cnt + kMaxStagesDev);  // [kMaxStageUnits] staging partial maxima
  int* s_pub = reinterpret_cast<int*>(s_amax + kMaxStageUnits);          // [kMaxWarpsAny][kPubInts] combine lists
  float* s_red = reinterpret_cast<float*>(s_pub + kMaxWarpsAny * kPubInts);  // [kRedFloats] split-K partials
  unsigned char* xbuf = smem + a.x_offset;
  unsigned char* stages = smem + a.stage_offset;

  if (tid == 0) {
    for (int s = 0; s < a.n_stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], a.wpi);
    }
    s_flag[0] = 0;  // abort: set by any wait that gives up; every loop then drains without work
    s_flag[1] = 0;
    for (int q = 0; q < a.n_stages; ++q) s_item_cnt[q] = 0;
    fence_barrier_init();
  }
  const bool producer = (warp == ncw);
  // Routed streams depend on the routing plan: everyone waits for the previous
  // grid first.  Dense streams only need it for their activations, so their
  // producer starts on the (static) weights right away.
  if (a.routed) pdl_wait();

  int n_groups = a.routed ? *a.n_active : 1;
  if (n_groups < 0 || n_groups > a.n_experts) {
    if (tid == 0) atomicExch(a.err, kErrBadPlan);
    n_groups = n_groups < 0 ? 0 : a.n_experts;
  }
  const int n_router = a.out_rows / a.R;                   // router: items of expert rows
  const int n_rt = n_router + (kRouter ? a.n_items2 : 0);  // ... then shared gate/up items
  const long long n_items = (long long)n_groups * n_rt;
  const long long lo = n_items * blockIdx.x / gridDim.x;
  const long long hi = n_items * (blockIdx.x + 1) / gridDim.x;

  const int nthreads_all = (ncw + 1) * 32;
  named_bar_sync(kBarAll, nthreads_all);  // barriers initialised
  // plan invariants (see the host planner): stages are a multiple of the warp
  // groups, and an item's rows are exactly what the group's warps cover
  const int kq_plan = kFast ? KS : ((WF == W_BF16 && a.ksplit > 1) ? a.ksplit : 1);
  if ((a.ncw % a.wpi) != 0 || (a.n_stages % (a.ncw / a.wpi)) != 0 || (a.wpi % kq_plan) != 0 ||
      a.R != RPW * (a.wpi / kq_plan) || a.ncw > kMaxWarpsAny || a.wpi < kMinItemWarps) {
    if (tid == 0) atomicExch(a.err, kErrBadPlan);
    return;
  }
  // The producer lane builds the phase table and starts streaming at once; the
  // consumers wait for the table on named barrier 2 (the producer only arrives).
  if (producer) {
    if (lane == 0) {
      build_phases(a, lo, hi, n_rt, a.xcap, *pt);
      if (pt->bad) atomicExch(a.err, kErrBadPlan);
    }
    __syncwarp();
    asm volatile("bar.arrive 2, %0;" ::"r"(nthreads_all) : "memory");
  } else {
    if (!a.routed && !a.pdl_late) pdl_wait();
    if (a.dep_counter && tid == 0) {
      // the preceding kernel's outputs this stream reads are published (bounded wait)
      const long long t0 = clock64();
      bool ok = true;
      while (true) {
        int v;
        asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(a.dep_counter) : "memory");
        if (v >= a.dep_target) break;
        if (clock64() - t0 > (1ll << 31)) { ok = false; break; }
        __nanosleep(64);
      }
      if (!ok) {
        atomicExch(a.err, kErrTimeout);
        s_flag[0] = 1;
      }
      fence_acq_rel_gpu();
      if (atomicAdd(a.dep_pass, 1) == (int)gridDim.x - 1) {  // every CTA of this grid is past the wait
        *a.dep_counter = 0;
        *a.dep_pass = 0;
      }
    }
    named_bar_sync(2, nthreads_all);
  }

  if (producer) {
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int pg = -1, pgrp = 0;  // cached group -> expert lookup
      for (int p = 0; p < pt->n && ok; ++p) {
        const int jbeg = pt->ph[p].first_item, jend = pt->ph[p].last_item;
        int g = (int)((lo + jbeg) / n_rt);
        int rt = (int)((lo + jbeg) - (long long)g * n_rt);
        for (int j = jbeg; j < jend; ++j, (++rt == n_rt ? (rt = 0, ++g) : 0)) {
          if (s_flag[0] || !mbar_wait_bounded(&empty_bar[s], ph ^ 1u)) {
            if (!s_flag[0]) atomicExch(a.err, kErrTimeout);
            s_flag[0] = 1;
            ok = false;
            break;
          }
          if (g != pg) {
            pg = g;
            pgrp = a.routed ? clamp_group(a.active[g], a.n_experts, a.err) : 0;
          }
          const int grp = pgrp;
          const int r0 = rt * a.R;
          unsigned char* st = stages + (size_t)s * a.stage_bytes;
          const uint32_t cb = (uint32_t)(a.R * rowbytes);
          const uint32_t sb = (WF == W_MXFP4 && !sglobal) ? (uint32_t)(a.R * sblocks) : 0u;
          mbar_arrive_expect_tx(&full_bar[s], (kSwiglu ? 2u : 1u) * (cb + sb));
          const uint8_t* wg = a.w + (long long)grp * a.w_gstride;
          if (kRouter && rt >= n_router) {
            // shared gate/up item: its gate row and up row (R = 2 rows of stage)
            const int j2 = rt - n_router;
            bulk_g2s(st, a.w2 + (size_t)j2 * rowbytes, (uint32_t)rowbytes, &full_bar[s], pol);
            bulk_g2s(st + rowbytes, a.w2 + (size_t)(j2 + a.up_off2) * rowbytes, (uint32_t)rowbytes, &full_bar[s], pol);
          } else {
            bulk_g2s(st, wg + (size_t)r0 * rowbytes, cb, &full_bar[s], pol);
          }
          if (kSwiglu) bulk_g2s(st + cb, wg + (size_t)(r0 + a.up_off) * rowbytes, cb, &full_bar[s], pol);
          if (WF == W_MXFP4 && !sglobal) {
            const uint8_t* sg = a.sc + (long long)grp * a.s_gstride;
            bulk_g2s(st + codes_bytes, sg + (size_t)r0 * sblocks, sb, &full_bar[s], pol);
            if (kSwiglu)
              bulk_g2s(st + codes_bytes + sb, sg + (size_t)(r0 + a.up_off) * sblocks, sb, &full_bar[s], pol);
          }
          if (++s == a.n_stages) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        // let copies already in flight land before the CTA can exit
        for (int q = 0; q < a.n_stages; ++q) {
          (void)mbar_wait_bounded(&full_bar[q], 0u, 1ll << 24);
          (void)mbar_wait_bounded(&full_bar[q], 1u, 1ll << 24);
        }
      }
    }
  } else {
    // ------------------------------ consumers ------------------------------
    const int nct = ncw * 32;
    int jglob = 0;  // CTA-local item counter across phases (stage ring position)
    for (int p = 0; p < pt->n; ++p) {
      const PhaseDesc ph = pt->ph[p];
      // stage this phase's activation vectors, each split over several warps
      named_bar_sync(1, nct);
      stage_phase<WF, XK>(a.act, &pt->slot_src[p][0], ph.nslots, K, xbuf, xrow_bytes, slot_e, s_amax, warp, ncw,
                          lane, nct);
      named_bar_sync(1, nct);
      const int nit = ph.last_item - ph.first_item;
      int c_g = -1, c_grp = 0, c_tok0 = 0, c_ntok = 1, c_tp_tb = -1;
      int nred = 0;  // K-split reduction rounds of this warp (buffer parity)
      int pend_rt[kPubBatch], npend = 0;  // fused combine: items written, not yet published
      int prev_cnt = 0, prev_rt = 0, nprev = 0;  // last published batch: atomic result per lane
      (void)pend_rt; (void)npend; (void)prev_cnt; (void)prev_rt; (void)nprev;
      TokenPass tp;
      tp.n = 0;
      const int ng = ncw / a.wpi;          // warp groups, one item each at a time
      const int q0 = warp / a.wpi;         // this warp's group
      const int wi = warp - q0 * a.wpi;    // this warp's share of the item
      int g = (int)((lo + ph.first_item + q0) / n_rt);
      int rt = (int)((lo + ph.first_item + q0) - (long long)g * n_rt);
      // ring position of this group's first item; each step moves ng stages on
      int s = (jglob + q0) % a.n_stages;
      uint32_t par = (uint32_t)(((jglob + q0) / a.n_stages) & 1);
      for (int jj = q0; jj < nit; jj += ng) {
        if (jj != q0) {  // advance (g, rt) and the ring position by ng items
          rt += ng;
          while (rt >= n_rt) { rt -= n_rt; ++g; }
          s += ng;
          if (s >= a.n_stages) { s -= a.n_stages; par ^= 1u; }
        }
        const bool skip = s_flag[0] != 0;  // aborting: no work, but every barrier is still met
        // group and token list: looked up once per group change, kept in registers
        if (g != c_g) {
          c_g = g;
          c_grp = a.routed ? clamp_group(a.active[g], a.n_experts, nullptr) : 0;
          c_tok0 = 0;
          c_ntok = a.n_tokens;
          if (a.routed) {
            c_tok0 = a.offsets[c_grp];
            c_ntok = a.offsets[c_grp + 1] - c_tok0;
            if (c_tok0 < 0 || c_ntok < 1 || c_tok0 + c_ntok > a.n_pairs) {
              if (lane == 0) atomicExch(a.err, kErrBadPlan);
              c_tok0 = 0;
              c_ntok = 1;
            }
          }
          c_tp_tb = -1;
        }
        const int grp = c_grp, tok0 = c_tok0, ntok = c_ntok;
        const int tlo = a.routed ? max(0, ph.t0) : ph.t0;
        const int thi = a.routed ? min(ntok, ph.t1) : ph.t1;

        bool have = !skip;
        if (have && !mbar_wait_bounded(&full_bar[s], par)) {
          if (lane == 0) atomicExch(a.err, kErrTimeout);
          s_flag[0] = 1;
          have = false;
        }
        const unsigned char* st = stages + (size_t)s * a.stage_bytes;
        if constexpr (kFast) {
          // ---- split-K item (one token): this warp's K slice of its NWR rows ----
          // The group barrier below is met on every item, with or without work,
          // so that an aborting warp can never leave the others waiting.
          const bool work = have && tlo < thi;
          if (work && tlo != c_tp_tb) {
            c_tp_tb = tlo;
            int src = tlo, orow = tlo;
            if (a.routed) {
              int pr = a.pair_ids[tok0 + tlo];
              if (pr < 0 || pr >= a.n_pairs) pr = 0;
              src = a.act_by_pair ? pr : pr / a.top_k;
              orow = pr;
            }
            int sl = 0;
            for (int u = 0; u < ph.nslots; ++u)
              if (pt->slot_src[p][u] == src) sl = u;
            tp.n = 1;
            tp.slot[0] = sl;
            tp.orow[0] = orow;
            tp.e[0] = slot_e[sl];
          }
          const int ks = wi % KS, rq = wi / KS;  // K slice, row quarter
          const int b = ks * 32 + lane;          // this lane's chunk
          const bool bok = work && b < C;
          int srow[NWR];
#pragma unroll
          for (int r = 0; r < NWR; ++r)
            srow[r] = kSwiglu ? (r < RPW ? rq * RPW + r : a.R + rq * RPW + (r - RPW)) : rq * RPW + r;
          // everything this warp needs from the stage, then hand it back at once
          uint4 xv[4], cv[NWR];
          uint32_t sv[NWR];
          const uint32_t xs_s =
              smem_addr(xbuf) + (uint32_t)(tp.slot[0] * xrow_bytes) + (uint32_t)(ks * 2048 + 16 * lane);
          const uint32_t st_s = smem_addr(st) + 16u * (uint32_t)b;
          const unsigned char* scl = st + codes_bytes;
#pragma unroll
          for (int q = 0; q < 4; ++q) xv[q] = bok ? lds128_s(xs_s + 512u * q) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int r = 0; r < NWR; ++r) {
            cv[r] = bok ? lds128_s(st_s + (uint32_t)(srow[r] * rowbytes)) : make_uint4(0u, 0u, 0u, 0u);
            sv[r] = bok ? lds_u8(scl + srow[r] * sblocks + b) : 127u;
          }
          if (have) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[s]);
          }
          float v[NWR];
#pragma unroll
          for (int r = 0; r < NWR; ++r) {
            uint32_t w[16];
            decode_chunk(cv[r], w);
            v[r] = dot32_h2(w, xv) * e8m0_to_f32(sv[r]);
          }
          // across the warp (lane L ends with row L / (32 / NWR)), then across the
          // KS slices in ascending order, by the item's finishing warp
          const float tot = warp_reduce_multi<NWR>(v, lane);
          const int nit_g = jj / ng;  // this group's item counter
          float* red = s_red + (size_t)(q0 * a.wpi) * 2 * NWR + (size_t)(nit_g & 1) * a.wpi * NWR;
          if ((lane & (32 / NWR - 1)) == 0) red[wi * NWR + lane / (32 / NWR)] = tot;
          group_bar(q0, a.wpi);
          if (work && wi == nit_g % a.wpi) {
            const int nrq = a.wpi / KS;
            const int o = lane;  // output row of the item handled by this lane
            if (o < nrq * RPW) {
              const int orq = o / RPW, orr = o - orq * RPW;
              float gsum = 0.f, usum = 0.f;
#pragma unroll
              for (int k2 = 0; k2 < KS; ++k2) {
                gsum += red[(orq * KS + k2) * NWR + orr];
                if constexpr (kSwiglu) usum += red[(orq * KS + k2) * NWR + RPW + orr];
              }
              const int row = rt * a.R + o;
              float val;
              if constexpr (kSwiglu) {
                const float gg = gsum * pow2f(tp.e[0]), uu = usum * pow2f(tp.e[0]);
                val = gg / (1.0f + expf(-gg)) * uu;
              } else {
                val = gsum * pow2f(tp.e[0]);
              }
              a.out[(size_t)tp.orow[0] * a.out_rows + row] = val;
            }
          }
        } else {
        // bf16 streams may split K over the group's warps: warp wi takes K slice
        // wi % kq of the rows of warp-row wi / kq; partial sums meet in s_red
        const int kq = (WF == W_BF16 && a.ksplit > 1) ? a.ksplit : 1;
        const int ksl = wi % kq, wr = wi / kq;
        // with K split, every warp of the group runs the same token passes (the
        // group barrier inside is met even by a warp that is aborting)
        for (int tb = tlo; (have || kq > 1) && tb < thi; tb += TMAX) {
          if (tb != c_tp_tb) {
          c_tp_tb = tb;
          tp.n = min(TMAX, thi - tb);
#pragma unroll
          for (int t = 0; t < TMAX; ++t) {
            const int tt = min(tb + t, thi - 1);
            int src, orow;
            if (a.routed) {
              int pr = a.pair_ids[tok0 + tt];
              if (pr < 0 || pr >= a.n_pairs) pr = 0;
              src = a.act_by_pair ? pr : pr / a.top_k;
              orow = pr;
            } else {
              src = tt;
              orow = tt;
            }
            int sl = 0;
            for (int u = 0; u < ph.nslots; ++u)
              if (pt->slot_src[p][u] == src) sl = u;
            tp.slot[t] = sl;
            tp.orow[t] = orow;
            tp.e[t] = slot_e[sl];
          }
          }
          float acc[NWR][TMAX];
#pragma unroll
          for (int r = 0; r < NWR; ++r)
#pragma unroll
            for (int t = 0; t < TMAX; ++t) acc[r][t] = 0.f;

          // stage rows handled by this warp
          int srow[NWR];
#pragma unroll
          for (int r = 0; r < NWR; ++r)
            srow[r] = kSwiglu ? (r < RPW ? wr * RPW + r : a.R + wr * RPW + (r - RPW)) : wr * RPW + r;
          if constexpr (kUnroll) {
            const unsigned char* scl = st + codes_bytes;
            float sreg[NWR][KS];
#pragma unroll
            for (int r = 0; r < NWR; ++r)
#pragma unroll
              for (int ci = 0; ci < KS; ++ci)
                sreg[r][ci] = sglobal ? 1.f
                                      : e8m0_to_f32(lane + 32 * ci < C ? lds_u8(scl + srow[r] * sblocks + lane + 32 * ci)
                                                                       : 127u);
            const uint8_t* sgl = a.sc + (long long)grp * a.s_gstride;
            if (sglobal) {
              const int r0 = rt * a.R;
#pragma unroll
              for (int r = 0; r < NWR; ++r) {
                const int gr = kSwiglu && srow[r] >= a.R ? r0 + a.up_off + srow[r] - a.R : r0 + srow[r];
#pragma unroll
                for (int ci = 0; ci < KS; ++ci)
                  if (lane + 32 * ci < C) sreg[r][ci] = e8m0_to_f32(__ldg(sgl + (size_t)gr * sblocks + lane + 32 * ci));
              }
            }
            const uint32_t xs_s = smem_addr(xbuf) + (uint32_t)(tp.slot[0] * xrow_bytes) + 16u * lane;
            uint32_t rb_s[NWR];
#pragma unroll
            for (int r = 0; r < NWR; ++r) rb_s[r] = smem_addr(st) + (uint32_t)(srow[r] * rowbytes) + 16u * lane;
#pragma unroll
            for (int ci = 0; ci < KS; ++ci) {
              if (lane + 32 * ci < C) {
                uint4 xv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) xv[q] = lds128_s(xs_s + (uint32_t)((ci * 4 + q) * 512));
#pragma unroll
                for (int r = 0; r < NWR; ++r) {
                  uint32_t w[16];
                  decode_chunk(lds128_s(rb_s[r] + 512u * ci), w);
                  acc[r][0] = fmaf(dot32_h2(w, xv), sreg[r][ci], acc[r][0]);
                }
              }
            }
          } else if constexpr (WF == W_MXFP4) {
            // scale rows: in the stage after the codes, or (short rows) straight from global
            const uint8_t* scl = st + codes_bytes;
            const uint8_t* sgl = a.sc + (long long)grp * a.s_gstride;
            const int r0 = rt * a.R;
            int gsrow[NWR];  // global row of each stage row (scales read from global)
#pragma unroll
            for (int r = 0; r < NWR; ++r)
              gsrow[r] = kSwiglu && srow[r] >= a.R ? r0 + a.up_off + srow[r] - a.R : r0 + srow[r];
            if (TMAX == 1 && NWR >= 4) {
              // one activation vector, several rows: each chunk's loads (activations,
              // every row's codes and scale bytes) go out together, then the rows
              const unsigned char* xs = xbuf + (size_t)tp.slot[0] * xrow_bytes;
              for (int b = lane; b < C; b += 32) {
                const int ii = b >> 5;
                uint4 xv[4], cv[NWR];
                uint32_t sv[NWR];
#pragma unroll
                for (int q = 0; q < 4; ++q) xv[q] = lds128(xs + ((((ii * 4 + q) * 32) + lane) << 4));
#pragma unroll
                for (int r = 0; r < NWR; ++r) {
                  cv[r] = lds128(st + (size_t)srow[r] * rowbytes + 16 * b);
                  sv[r] = sglobal ? (uint32_t)__ldg(sgl + (size_t)gsrow[r] * sblocks + b)
                                          : lds_u8(scl + srow[r] * sblocks + b);
                }
#pragma unroll
                for (int r = 0; r < NWR; ++r) {
                  uint32_t w[16];
                  decode_chunk(cv[r], w);
                  acc[r][0] = fmaf(dot32_h2(w, xv), e8m0_to_f32(sv[r]), acc[r][0]);
                }
              }
            } else
            for (int b = lane; b < C; b += 32) {
              const int i = b >> 5;
#pragma unroll
              for (int t = 0; t < TMAX; ++t) {
                if (t < tp.n) {
                  // the activation chunk once, then every row of this warp one at a time
                  const unsigned char* xs = xbuf + (size_t)tp.slot[t] * xrow_bytes;
                  uint4 xv[4];
#pragma unroll
                  for (int q = 0; q < 4; ++q) xv[q] = lds128(xs + ((((i * 4 + q) * 32) + lane) << 4));
#pragma unroll
                  for (int r = 0; r < NWR; ++r) {
                    uint32_t w[16];
                    decode_chunk(lds128(st + (size_t)srow[r] * rowbytes + 16 * b), w);
                    const float sc = sglobal ? e8m0_to_f32(__ldg(sgl + (size_t)gsrow[r] * sblocks + b))
                                                     : e8m0_to_f32(lds_u8(scl + srow[r] * sblocks + b));
                    acc[r][t] = fmaf(dot32_h2(w, xv), sc, acc[r][t]);
                  }
                }
              }
            }
          } else {
            // bf16 weights: lane owns 8-element (16-byte) chunks, contiguous across the warp
            const int c8 = K >> 3;
            const int per = c8 / kq, b8_hi = (ksl == kq - 1) ? c8 : (ksl + 1) * per;
            for (int b8 = ksl * per + lane; have && b8 < b8_hi; b8 += 32) {
#pragma unroll
              for (int rp = 0; rp < NWR; rp += 2) {
                const uint4 qa = lds128(st + (size_t)srow[rp] * rowbytes + 16 * b8);
                const uint4 qb = lds128(st + (size_t)srow[rp + 1] * rowbytes + 16 * b8);
#pragma unroll
                for (int t = 0; t < TMAX; ++t) {
                  if (t < tp.n) {
                    const unsigned char* xs = xbuf + (size_t)tp.slot[t] * xrow_bytes;
                    if constexpr (XK == X_BF16) {
                      const uint4 xv = lds128(xs + 16 * b8);
                      float pa = 0.f, pb = 0.f;
                      pa = fma2_bf16(qa.x, xv.x, pa); pb = fma2_bf16(qb.x, xv.x, pb);
                      pa = fma2_bf16(qa.y, xv.y, pa); pb = fma2_bf16(qb.y, xv.y, pb);
                      pa = fma2_bf16(qa.z, xv.z, pa); pb = fma2_bf16(qb.z, xv.z, pb);
                      pa = fma2_bf16(qa.w, xv.w, pa); pb = fma2_bf16(qb.w, xv.w, pb);
                      acc[rp][t] += pa;
                      acc[rp + 1][t] += pb;
                    } else {
                      const uint4 x0 = lds128(xs + 32 * b8), x1 = lds128(xs + 32 * b8 + 16);
                      const float xf[8] = {__uint_as_float(x0.x), __uint_as_float(x0.y), __uint_as_float(x0.z),
                                           __uint_as_float(x0.w), __uint_as_float(x1.x), __uint_as_float(x1.y),
                                           __uint_as_float(x1.z), __uint_as_float(x1.w)};
                      const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w}, wb[4] = {qb.x, qb.y, qb.z, qb.w};
                      float pa = 0.f, pb = 0.f;
#pragma unroll
                      for (int j = 0; j < 4; ++j) {
                        pa = fmaf(bf16lo_to_f32(wa[j]), xf[2 * j], pa);
                        pa = fmaf(bf16hi_to_f32(wa[j]), xf[2 * j + 1], pa);
                        pb = fmaf(bf16lo_to_f32(wb[j]), xf[2 * j], pb);
                        pb = fmaf(bf16hi_to_f32(wb[j]), xf[2 * j + 1], pb);
                      }
                      acc[rp][t] += pa;
                      acc[rp + 1][t] += pb;
                    }
                  }
                }
              }
            }
          }
          if (have && tb + TMAX >= thi) {
            // the stage is no longer read: hand it back to the producer
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[s]);
          }
          // --- reduce across the warp ---
          constexpr int V = NextPow2<NWR * TMAX>::value;
          float v[V];
#pragma unroll
          for (int q = 0; q < V; ++q) v[q] = 0.f;
#pragma unroll
          for (int r = 0; r < NWR; ++r)
#pragma unroll
            for (int t = 0; t < TMAX; ++t) v[r * TMAX + t] = acc[r][t];
          const float tot = warp_reduce_multi<V>(v, lane);
          // lane L holds value L / (32 / V); gather what the epilogue lanes need
          const int vi = lane / (32 / V);
          float mine = tot;
          if (kq > 1) {
            // K slices: partial sums through shared memory (two buffers, one per
            // alternate pass), summed in ascending slice order by slice 0's warp
            float* red = s_red + ((size_t)q0 * 2 + (nred & 1)) * a.wpi * V;
            ++nred;
            if ((lane & (32 / V - 1)) == 0) red[wi * V + vi] = tot;
            group_bar(q0, a.wpi);
            if (ksl != 0 || !have) continue;
            mine = 0.f;
            for (int k2 = 0; k2 < kq; ++k2) mine += red[(wr * kq + k2) * V + vi];
          }
          // --- epilogue: lanes 0 .. (outputs-1) ---
          const int nout = RPW * TMAX;
          const int oi = lane;  // output index handled by this lane
          const int rr = oi / TMAX, t = oi - (oi / TMAX) * TMAX;
          const float g_or_y = __shfl_sync(0xFFFFFFFFu, mine, (rr * TMAX + t) * (32 / V) & 31);
          const float up = __shfl_sync(0xFFFFFFFFu, mine, ((RPW + rr) * TMAX + t) * (32 / V) & 31);
          (void)vi;
          if (kRouter && rt >= n_router) {
            // shared gate/up item: stage row 0 is the gate row, row 1 the up row
            const float second = __shfl_sync(0xFFFFFFFFu, mine, (TMAX + t) * (32 / V) & 31);
            if (oi < TMAX && t < tp.n) {
              const int orow_t = (t == 0) ? tp.orow[0] : tp.orow[TMAX - 1];
              a.out2[(size_t)orow_t * a.n_items2 + (rt - n_router)] = g_or_y / (1.0f + expf(-g_or_y)) * second;
            }
          } else if (oi < nout && t < tp.n) {
            int et = tp.e[0], orow_t = tp.orow[0];
#pragma unroll
            for (int q = 1; q < TMAX; ++q)
              if (t == q) { et = tp.e[q]; orow_t = tp.orow[q]; }
            const int row = rt * a.R + wr * RPW + rr;
            float val;
            if constexpr (kSwiglu) {
              const float gg = (WF == W_MXFP4) ? g_or_y * pow2f(et) : g_or_y;
              const float uu = (WF == W_MXFP4) ? up * pow2f(et) : up;
              val = gg / (1.0f + expf(-gg)) * uu;
            } else {
              val = (WF == W_MXFP4) ? g_or_y * pow2f(et) : g_or_y;
              if constexpr (EPI == EPI_ROUTER) {
                if (a.bias) val += a.bias[row];
              }
            }
            a.out[(size_t)orow_t * a.out_rows + row] = val;
          }
        }
        }  // generic item
        if constexpr (EPI == EPI_DOWN_COMBINE) {
          // publish in batches: see publish_round().  A group whose tokens are
          // split over several phases (more activation rows than slots) runs
          // each of its items once per phase: the item counts once, with the
          // phase that holds the group's last tokens (the earlier phases' y
          // stores are ordered before it by the phase barrier).
          if (thi >= ntok) pend_rt[npend++] = rt;
          if (npend == kPubBatch) {
            publish_round(a, pend_rt, npend, prev_cnt, prev_rt, nprev, n_groups, wi, q0, lane, s_pub + q0 * kPubInts);
            npend = 0;
          }
        }
      }
      if constexpr (EPI == EPI_DOWN_COMBINE) {
        // end of phase: publish what is left, then settle the last results
        // (npend and nprev are the same in every warp of the group)
        if (npend > 0) publish_round(a, pend_rt, npend, prev_cnt, prev_rt, nprev, n_groups, wi, q0, lane, s_pub + q0 * kPubInts);
        npend = 0;
        if (nprev > 0) publish_round(a, pend_rt, 0, prev_cnt, prev_rt, nprev, n_groups, wi, q0, lane, s_pub + q0 * kPubInts);
        nprev = 0;
      }
      jglob += nit;
    }
  }

  if constexpr (kRouter) {
    if (a.topk_idx) {
      // every CTA's logits are written: the last CTA to get here selects the
      // top-k of every token, then builds the buckets
      named_bar_sync(kBarAll, nthreads_all);  // this CTA's logit stores, performed CTA-wide
      if (tid == 0) {
        fence_acq_rel_gpu();  // release: ... and at gpu scope, before the count
        if (a.pub_counter) atomicAdd(a.pub_counter, 1);
        const bool last = atomicAdd(a.done_counter, 1) == (int)gridDim.x - 1;
        if (last) fence_acq_rel_gpu();  // acquire: every CTA's logits before the reads below
        s_flag[1] = last ? 1 : 0;
      }
      named_bar_sync(kBarAll, nthreads_all);
      // the next kernel may launch now: what it may read before its own wait
      // (h_s, behind pub_counter) is published; the routing finish follows
      pdl_launch_dependents();
      if (s_flag[1]) {
        // the stage ring is idle now: top-k scratch, then bucket scratch
        if (a.n_tokens == 1) {
          // one token: the whole CTA selects it and writes the plan as it goes
          topk_token_block(a, a.out, 0, tid, nthreads_all, kBarAll, true, stages);
        } else {
          topk_tail(a, a.out, tid, nthreads_all, kBarAll, stages + kBucketScratchBytes);
          named_bar_sync(kBarAll, nthreads_all);  // topk_idx stores performed CTA-wide
          unsigned long long* s_mask = reinterpret_cast<unsigned long long*>(stages);
          int* s_off = reinterpret_cast<int*>(stages + 8 * kMaxExperts);
          int* s_wsum = s_off + kMaxExperts;
          bucket_block(a, a.n_tokens, tid, nthreads_all, kBarAll, s_mask, s_off, s_wsum);
        }
        if (tid == 0) *a.done_counter = 0;
      }
    }
  }

  // Let the next kernel in the stream start its prologue.
  pdl_launch_dependents();
  // A stream that skipped the wait still completes only after its predecessor,
  // so the kernels behind it inherit that dependency.
  if (a.pdl_late) pdl_wait();

  if constexpr (EPI == EPI_DOWN_COMBINE) {
    // tail: warm L2 with the next layer's static weights (one slice per CTA)
    if (tid == 32 * ncw) {
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

}

template <int WF, int EPI, int XK, int TMAX, int RPW, int KT>
__global__ void __launch_bounds__(((KT != 0 && WF == W_MXFP4 && TMAX == 1 &&
                                    (EPI == EPI_SWIGLU ? 2 * RPW : RPW) == kSplitKRows)
                                       ? kMaxSplitKWarps
                                       : consumer_warps_for(WF, EPI)) * 32 + 32,
                                  1) gemv_kernel(const GemvArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  gemv_body<WF, EPI, XK, TMAX, RPW, KT>(a, smem);
}

}  // namespace moe
