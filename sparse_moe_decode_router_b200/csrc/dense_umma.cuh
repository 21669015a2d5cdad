// Dense bf16 projections on the 5th-generation tensor cores (tcgen05.mma
// kind::f16, sm_100a) for batches above 1: the router (logits), the shared
// expert's gate/up (SwiGLU) and its down projection.
//
// At one token the CUDA-core streams read each weight once and spend a few
// instructions per weight.  With B tokens they must hold all B activation
// rows next to the weights; shared memory takes four 7168-element rows, so
// the weights would stream once per four tokens.  Here the weights are the A
// operand (M = 128 rows per MMA, K-major bf16, TMA tiles of 128 rows x 64
// elements under the 128-byte swizzle) and the tokens the B operand (one
// column per token, or per term), so every weight is read from HBM once
// whatever the batch:
//
//  * work is split along K as well as rows ("stream-K"): the (tile, stage)
//    pairs of all of a launch's tiles form one list, weighted by the A tiles a
//    stage moves (gate + up = 2), and every CTA takes a contiguous stretch of
//    equal weight; a stretch covers the end of one tile, whole tiles and the
//    start of another.  Each piece ("part") of a tile accumulates its K range
//    in tensor memory and writes it to a workspace; the last part to arrive
//    (a counter per tile) adds the parts in ascending K order (so the result
//    does not depend on which part finishes last) and runs the epilogue;
//  * the producer starts on the weights before waiting for the preceding
//    kernel (they are static); the activations follow the wait;
//  * epilogues: logits (+ bias); h_s = silu(g) * u as fp32 and as two bf16
//    terms (the value rounded, then the rounding error rounded) that are the
//    B operand of the shared down projection; y_s.
//
// Warp roles (192 threads, one CTA per SM): warp 0 TMA producer, warp 1
// tensor memory + MMA issuer, warps 2..5 epilogue (TMEM lanes 32*(w%4)..).
// Every wait is bounded; a wait that gives up records MOE_ERR_TIMEOUT.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "mx_umma.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kDnRows = 128;                      // M
constexpr int kDnKBox = 64;                       // K elements per stage (128 bytes of bf16 per row)
constexpr int kDnATile = kDnRows * kDnKBox * 2;   // 16 KB
constexpr int kDnBBox = 16;                       // B rows per TMA copy (2 KB)
constexpr int kDnNMax = 128;                      // B columns
constexpr int kDnThreads = 192;
constexpr int kDnTmemCols = 256;                  // two accumulator buffers: [gate | up] <= 128 columns
constexpr int kDnMaxStages = 16;
constexpr int kDnHTerms = 2;                      // bf16 terms of h_s (B columns per token of the shared down)
constexpr int kDnHeaderBytes = 1024;
constexpr int kDnRedUnits = 4;                    // last part of a tile: units (4 rows x 1 token) per thread ...
constexpr int kDnRedParts = 4;                    // ... and parts whose loads are in flight together
static_assert(8 * (2 * kDnMaxStages + 6) + 32 <= kDnHeaderBytes, "header");

struct DenseStream {
  int n_tiles;          // 128-row output tiles
  int a_row0;           // first weight row in this stream's A tensor map
  int up_rows;          // SwiGLU: rows from a gate row to its up row (0: plain projection)
  int out_rows;         // valid output rows (the last tile may be partial)
  float* out;           // [B][out_rows] fp32
  const float* bias;    // per output row (plain streams), or null
  uint16_t* next_terms; // SwiGLU: bf16 terms of the output [B * kDnHTerms][out_rows], or null
};

struct DenseArgs {
  DenseStream st[2];
  int n_streams;     // 1 or 2 (both over the same K and the same activations)
  int skip_mask;     // bit s: stream s is part of the partition but not computed (the
                     // staged entry points compute one stream with the fused launch's split)
  int K;             // multiple of 64
  int B;             // tokens
  int terms;         // B columns per token: 1 (x) or kDnHTerms (h_s terms)
  int n;             // B columns, multiple of 16, >= B * terms, <= kDnNMax
  int n_stages, stage_bytes, off_up, off_b;
  float* ws;         // partials: [tile][part][gate/up][column][row] fp32
  int ws_parts;      // parts per tile the workspace holds
  int* tile_cnt;     // [all tiles], zero between launches
  int* err;
};

// stream-K partition: stage i of the launch's list (tiles of stream 0, then
// stream 1; S stages per tile) weighs 2, or 3 for a SwiGLU stream.  CTA c of
// the first G owns stages [first(c), first(c + 1)); G is at most half the
// stages, so every such range holds at least one stage (a range's weight is
// at least 4) and the parts of a tile are the ranges of consecutive CTAs.
// CTAs from G on have no work.
struct DnSplit {
  long long S, T0, T1, w0, w1, W0, W, G;
  __host__ __device__ long long first(long long c) const {
    if (c >= G) return (T0 + T1) * S;
    const long long wt = c * W / G;
    if (wt <= W0) return (wt + w0 - 1) / w0;
    return T0 * S + (wt - W0 + w1 - 1) / w1;
  }
  // the CTA whose range holds stage i
  __host__ __device__ long long owner(long long i) const {
    long long lo = 0, hi = G - 1;
    while (lo < hi) {
      const long long mid = (lo + hi + 1) / 2;
      if (first(mid) <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
};

__host__ __device__ inline DnSplit dn_split(const DenseArgs& a, int G) {
  DnSplit d;
  d.S = a.K / kDnKBox;
  d.T0 = a.st[0].n_tiles;
  d.T1 = a.n_streams > 1 ? a.st[1].n_tiles : 0;
  // a stage's cost: its A tiles' bytes plus a fixed part per stage (the
  // barrier round trip, the copies' and MMAs' issue): one tile weighs 2, a
  // gate/up pair 3 (measured: a one-tile stage takes ~0.68 of a pair's time)
  d.w0 = a.st[0].up_rows ? 3 : 2;
  d.w1 = (a.n_streams > 1 && a.st[1].up_rows) ? 3 : 2;
  d.W0 = d.T0 * d.S * d.w0;
  d.W = d.W0 + d.T1 * d.S * d.w1;
  const long long half = (d.T0 + d.T1) * d.S / 2;
  d.G = half < 1 ? 1 : (half < G ? half : G);
  return d;
}

// a run: the stretch of one CTA's range inside one tile
struct DnRun {
  int tile;    // tile index over both streams
  int s;       // stream
  int lt;      // tile within the stream
  int k0, nk;  // first stage and stages of the run
  int part, nparts;
};

struct DnWalk {
  const DnSplit& d;
  long long it, hi;
  __device__ DnWalk(const DnSplit& sp, long long lo, long long hi_) : d(sp), it(lo), hi(hi_) {}
  __device__ bool valid() const { return it < hi; }
  __device__ DnRun run() const {
    DnRun r;
    const long long ti = it / d.S;
    const long long end = min(hi, (ti + 1) * d.S);
    r.tile = (int)ti;
    r.s = ti < d.T0 ? 0 : 1;
    r.lt = (int)(ti < d.T0 ? ti : ti - d.T0);
    r.k0 = (int)(it - ti * d.S);
    r.nk = (int)(end - it);
    const long long c0 = d.owner(ti * d.S);
    r.part = (int)(d.owner(it) - c0);
    r.nparts = (int)(d.owner((ti + 1) * d.S - 1) - c0 + 1);
    return r;
  }
  __device__ void next() {
    const long long ti = it / d.S;
    it = min(hi, (ti + 1) * d.S);
  }
};

__device__ __forceinline__ void tc_mma_f16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

// instruction descriptor, kind::f16: A and B bf16, K-major, fp32 accumulate, M = 128, N columns
__host__ __device__ constexpr uint32_t dn_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kDnRows >> 4) << 24);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  uint16_t h;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(f));
  return h;
}

__global__ void __launch_bounds__(kDnThreads, 1)
    dense_bf16_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                      const __grid_constant__ CUtensorMap tmB, const DenseArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t raw = smem_addr(smem_raw);
  unsigned char* hdr = smem_raw;
  unsigned char* ring = smem_raw + (((raw + kDnHeaderBytes + 1023u) & ~1023u) - raw);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(hdr);
  uint64_t* empty_bar = full_bar + kDnMaxStages;
  uint64_t* acc_full = empty_bar + kDnMaxStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done_bar = acc_empty + 2;
  uint64_t* epi_bar = done_bar + 1;
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(hdr + 8 * (2 * kDnMaxStages + 6));
  volatile int* s_abort = reinterpret_cast<volatile int*>(hdr + 8 * (2 * kDnMaxStages + 6) + 16);
  volatile int* s_last = s_abort + 1;

  const int ns = a.n_stages;
  if (tid == 0) {
    for (int s = 0; s < kDnMaxStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(done_bar, 1);
    mbar_init(epi_bar, 4);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr((const void*)s_tmem)),
                 "r"(kDnTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    if (a.n_streams > 1) tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  const bool plan_ok = ns >= 1 && ns <= kDnMaxStages && (a.K % kDnKBox) == 0 && a.n >= 16 && a.n <= kDnNMax &&
                       (a.n % 16) == 0 && a.B * a.terms <= a.n && a.n_streams >= 1 && a.n_streams <= 2;
  if (!plan_ok && tid == 0) atomicExch(a.err, kErrBadPlan);
  const DnSplit d = dn_split(a, gridDim.x);
  const long long lo = d.first(blockIdx.x), hi = d.first(blockIdx.x + 1);
  const long long lim_long = 1ll << 31, lim_short = 1ll << 20;
  const int nbox = a.n / kDnBBox;

  if (plan_ok && warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      // the weights of the first stages go out before the wait for the
      // preceding kernel (static data); the activations after it
      const long long npf = min((long long)ns, hi - lo);
      {
        int s = 0;
        long long done = 0;
        for (DnWalk w(d, lo, hi); w.valid() && done < npf; w.next()) {
          const DnRun r = w.run();
          if ((a.skip_mask >> r.s) & 1) continue;
          const DenseStream& S = a.st[r.s];
          const CUtensorMap* tm = r.s ? &tmA1 : &tmA0;
          const int arow = S.a_row0 + r.lt * kDnRows;
          for (int k = 0; k < r.nk && done < npf; ++k, ++done, ++s) {
            const uint32_t sa = smem_addr(ring + (size_t)s * a.stage_bytes);
            mbar_arrive_expect_tx(&full_bar[s], (S.up_rows ? 2u : 1u) * kDnATile + (uint32_t)nbox * kDnBBox * 128u);
            tma_load_2d(sa, tm, (r.k0 + k) * kDnKBox, arow, &full_bar[s], pol);
            if (S.up_rows) tma_load_2d(sa + a.off_up, tm, (r.k0 + k) * kDnKBox, arow + S.up_rows, &full_bar[s], pol);
          }
        }
      }
      pdl_wait();
      int s = 0;
      uint32_t ph = 0;
      long long q = 0;  // stage counter of this CTA
      for (DnWalk w(d, lo, hi); w.valid() && !*s_abort; w.next()) {
        const DnRun r = w.run();
        if ((a.skip_mask >> r.s) & 1) continue;
        const DenseStream& S = a.st[r.s];
        const CUtensorMap* tm = r.s ? &tmA1 : &tmA0;
        const int arow = S.a_row0 + r.lt * kDnRows;
        for (int k = 0; k < r.nk; ++k, ++q) {
          const int kk = r.k0 + k;
          const uint32_t sa = smem_addr(ring + (size_t)s * a.stage_bytes);
          if (q >= npf) {
            if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, *s_abort ? lim_short : lim_long)) {
              atomicExch(a.err, kErrTimeout);
              *s_abort = 1;
              break;
            }
            mbar_arrive_expect_tx(&full_bar[s], (S.up_rows ? 2u : 1u) * kDnATile + (uint32_t)nbox * kDnBBox * 128u);
            tma_load_2d(sa, tm, kk * kDnKBox, arow, &full_bar[s], pol);
            if (S.up_rows) tma_load_2d(sa + a.off_up, tm, kk * kDnKBox, arow + S.up_rows, &full_bar[s], pol);
          }
          for (int j = 0; j < nbox; ++j)
            tma_load_2d_nohint(sa + a.off_b + j * kDnBBox * 128, &tmB, kk * kDnKBox, kDnBBox * j, &full_bar[s]);
          if (++s == ns) { s = 0; ph ^= 1u; }
        }
      }
      if (*s_abort) {
        for (int qq = 0; qq < ns; ++qq) {
          (void)mbar_wait_bounded(&full_bar[qq], 0u, lim_short);
          (void)mbar_wait_bounded(&full_bar[qq], 1u, lim_short);
        }
      }
    }
    // every copy of this CTA is issued: the next grid may start its prologue
    // on SMs as they free up (it waits for this grid before reading its outputs)
    __syncwarp();
    pdl_launch_dependents();
  } else {
    // activations (B operand) and the workspace come from the preceding kernels
    pdl_wait();
  }

  if (plan_ok && warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      int s = 0, uc = 0;
      uint32_t ph = 0;
      const uint32_t idesc = dn_idesc(a.n);
      for (DnWalk w(d, lo, hi); w.valid() && !*s_abort; w.next()) {
        const DnRun r = w.run();
        if ((a.skip_mask >> r.s) & 1) continue;
        const bool glu = a.st[r.s].up_rows != 0;
        const int b = uc & 1;
        if (!mbar_wait_bounded(&acc_empty[b], (((uint32_t)uc >> 1) & 1u) ^ 1u, lim_long)) {
          atomicExch(a.err, kErrTimeout);
          *s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_g = tmem + (uint32_t)(b * kDnNMax);
        const uint32_t d_u = d_g + (uint32_t)(kDnNMax / 2);
        bool ok = true;
        for (int k = 0; k < r.nk; ++k) {
          if (!mbar_wait_bounded(&full_bar[s], ph, *s_abort ? lim_short : lim_long)) {
            atomicExch(a.err, kErrTimeout);
            *s_abort = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_addr(ring + (size_t)s * a.stage_bytes);
          const uint64_t ad = desc_sw128(st), bd = desc_sw128(st + a.off_b);
          const uint64_t ud = desc_sw128(st + a.off_up);
#pragma unroll
          for (int j = 0; j < kDnKBox / 16; ++j) {  // K = 16 per MMA: +32 bytes per swizzled row
            const uint32_t acc = (k > 0 || j > 0) ? 1u : 0u;
            tc_mma_f16(d_g, ad + 2u * j, bd + 2u * j, idesc, acc);
            if (glu) tc_mma_f16(d_u, ud + 2u * j, bd + 2u * j, idesc, acc);
          }
          tc_commit(&empty_bar[s]);
          if (++s == ns) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&acc_full[b]);
        ++uc;
      }
      tc_commit(done_bar);
      if (!mbar_wait_bounded(done_bar, 0u, lim_long)) atomicExch(a.err, kErrTimeout);
    }
    __syncwarp();
  } else if (plan_ok && warp >= 2) {
    // ------------------------------ epilogue ----------------------------------
    const int q = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    const int rloc = 32 * q + lane;  // row of the tile held by this lane
    const int et = (warp - 2) * 32 + lane;  // 0..127 over the four epilogue warps
    int uc = 0;
    uint32_t epi_ph = 0;
    auto epi_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_bar);
      bool ok = mbar_wait_bounded(epi_bar, epi_ph, *s_abort ? lim_short : lim_long);
      ok = __all_sync(0xFFFFFFFFu, ok);
      epi_ph ^= 1u;
      if (!ok) {
        if (lane == 0) atomicExch(a.err, kErrTimeout);
        *s_abort = 1;
      }
      return ok;
    };
    const int ncol = a.n;
    for (DnWalk w(d, lo, hi); w.valid(); w.next()) {
      const DnRun r = w.run();
      if ((a.skip_mask >> r.s) & 1) continue;
      const DenseStream& S = a.st[r.s];
      const bool glu = S.up_rows != 0;
      const int b = uc & 1;
      bool ok = !*s_abort && mbar_wait_bounded(&acc_full[b], ((uint32_t)uc >> 1) & 1u, lim_long);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (lane == 0 && !*s_abort) atomicExch(a.err, kErrTimeout);
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      // this part of the tile -> the workspace, column-major (one 512-byte row per column)
      const bool in_ws = r.part < a.ws_parts;
      float* wp = a.ws + (((size_t)r.tile * a.ws_parts + (in_ws ? r.part : 0)) * 2) * kDnNMax * kDnRows;
      for (int c = 0; c < ncol; c += 16) {
        float v[16];
        tc_ld16(lane_base + (uint32_t)(b * kDnNMax + c), v);
        float u[16];
        if (glu) tc_ld16(lane_base + (uint32_t)(b * kDnNMax + kDnNMax / 2 + c), u);
        tc_wait_ld();
        if (in_ws) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            wp[(size_t)(c + i) * kDnRows + rloc] = v[i];
            if (glu) wp[(size_t)(kDnNMax + c + i) * kDnRows + rloc] = u[i];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
      if (!in_ws && lane == 0) atomicExch(a.err, kErrBadPlan);
      // count the part; the last of the tile's parts finishes the tile
      if (!epi_sync()) break;
      if (warp == 2 && lane == 0) {
        fence_acq_rel_gpu();
        const int prev = atomicAdd(&a.tile_cnt[r.tile], 1);
        const bool last = prev == r.nparts - 1;
        if (last) {
          fence_acq_rel_gpu();
          a.tile_cnt[r.tile] = 0;
        }
        *s_last = last ? 1 : 0;
      }
      if (!epi_sync()) break;
      if (*s_last) {
        // the tile's parts, added in ascending K order.  A unit is four rows
        // of one token (a float4 of each part's column); thread et takes the
        // units et, et + 128, ... (a warp reads 512 contiguous bytes per
        // load), kDnRedUnits units and kDnRedParts parts at a time
        const float* w0 = a.ws + ((size_t)r.tile * a.ws_parts * 2) * kDnNMax * kDnRows;
        const int np = min(r.nparts, a.ws_parts);
        const size_t pstr = (size_t)2 * kDnNMax * kDnRows;
        const int n_units = a.B * (kDnRows / 4);
        const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int u0 = et; u0 < n_units; u0 += kDnRedUnits * 128) {
          float4 g[kDnRedUnits], uu[kDnRedUnits];
#pragma unroll
          for (int j = 0; j < kDnRedUnits; ++j) g[j] = uu[j] = zero4;
          for (int t = 0; t < a.terms; ++t) {
            float4 sg[kDnRedUnits], su[kDnRedUnits];
#pragma unroll
            for (int j = 0; j < kDnRedUnits; ++j) sg[j] = su[j] = zero4;
            for (int p0 = 0; p0 < np; p0 += kDnRedParts) {
              float4 vg[kDnRedParts][kDnRedUnits], vu[kDnRedParts][kDnRedUnits];
#pragma unroll
              for (int i = 0; i < kDnRedParts; ++i) {
#pragma unroll
                for (int j = 0; j < kDnRedUnits; ++j) {
                  const int u = u0 + 128 * j;
                  const bool on = p0 + i < np && u < n_units;
                  const float* src = w0 + (size_t)(p0 + i) * pstr +
                                     (size_t)((u >> 5) * a.terms + t) * kDnRows + 4 * (u & 31);
                  vg[i][j] = on ? __ldcg(reinterpret_cast<const float4*>(src)) : zero4;
                  vu[i][j] = (on && glu) ? __ldcg(reinterpret_cast<const float4*>(src + kDnNMax * kDnRows)) : zero4;
                }
              }
#pragma unroll
              for (int i = 0; i < kDnRedParts; ++i) {
                if (p0 + i >= np) break;
#pragma unroll
                for (int j = 0; j < kDnRedUnits; ++j) {
                  add4(sg[j], vg[i][j]);
                  add4(su[j], vu[i][j]);
                }
              }
            }
#pragma unroll
            for (int j = 0; j < kDnRedUnits; ++j) {
              add4(g[j], sg[j]);
              add4(uu[j], su[j]);
            }
          }
#pragma unroll
          for (int j = 0; j < kDnRedUnits; ++j) {
            const int u = u0 + 128 * j;
            if (u >= n_units) break;
            const int bt = u >> 5, row0 = r.lt * kDnRows + 4 * (u & 31);
            const float gv[4] = {g[j].x, g[j].y, g[j].z, g[j].w};
            const float uv[4] = {uu[j].x, uu[j].y, uu[j].z, uu[j].w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int row = row0 + c;
              if (row >= S.out_rows) break;
              if (glu) {
                const float h = gv[c] / (1.0f + expf(-gv[c])) * uv[c];
                S.out[(size_t)bt * S.out_rows + row] = h;
                if (S.next_terms) {
                  const uint16_t t0 = f32_to_bf16_bits(h);
                  const uint16_t t1 = f32_to_bf16_bits(h - __uint_as_float((uint32_t)t0 << 16));
                  S.next_terms[((size_t)bt * kDnHTerms) * S.out_rows + row] = t0;
                  S.next_terms[((size_t)bt * kDnHTerms + 1) * S.out_rows + row] = t1;
                }
              } else {
                S.out[(size_t)bt * S.out_rows + row] = gv[c] + (S.bias ? S.bias[row] : 0.f);
              }
            }
          }
        }
      }
      if (!epi_sync()) break;  // s_last is read before the next run overwrites it
      ++uc;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kDnTmemCols) : "memory");
  }
  pdl_launch_dependents();
}

// Routing finish of batches above 1, after a router stream without one:
// CTA b selects token b's top-k (topk_token_block), the last
// CTA to finish builds the buckets.  Dynamic shared memory: kBucketScratchBytes
// + kTopkCandBytes.
__global__ void __launch_bounds__(256) routing_finish_kernel(const GemvArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_last;
  pdl_wait();
  pdl_launch_dependents();  // the activation terms read the plan after their own wait
  const int tid = threadIdx.x, b = blockIdx.x;
  const int E = a.n_experts;
  topk_token_block(a, a.out + (size_t)b * E, b, tid, blockDim.x, 1, false, smem + kBucketScratchBytes);
  __syncthreads();  // this CTA's topk stores, performed CTA-wide
  if (tid == 0) {
    fence_acq_rel_gpu();
    const bool last = atomicAdd(a.done_counter, 1) == (int)gridDim.x - 1;
    if (last) fence_acq_rel_gpu();
    s_last = last ? 1 : 0;
  }
  __syncthreads();
  if (s_last) {
    unsigned long long* s_mask = reinterpret_cast<unsigned long long*>(smem);
    int* s_off = reinterpret_cast<int*>(smem + 8 * kMaxExperts);
    int* s_wsum = s_off + kMaxExperts;
    bucket_block(a, a.n_tokens, tid, blockDim.x, 1, s_mask, s_off, s_wsum);
    if (tid == 0) *a.done_counter = 0;
  }
  pdl_launch_dependents();
}

}  // namespace moe
