// Grouped MXFP4 expert projections on the tensor cores (batch > 1).
//
// Each expert's weight rows are streamed once (TMA bulk copies into a
// shared-memory ring, one producer lane) and multiplied with every token routed
// to that expert: E2M1 codes are decoded once per weight, straight into the A
// fragments of warp-level `mma.sync.m16n8k16` (f16 inputs, fp32 accumulate);
// the tokens form the N dimension in tiles of 8.  The E8M0 scale of each
// 32-element block is applied in fp32 to that block's two MMAs, so any scale
// is exact.  Activations are read from an f16 copy (each row scaled by a power
// of two, see act_to_f16_kernel) through L2.
//
// Work unit ("item"): 16 weight rows of one active expert -- 8 gate + 8 up
// rows for gate/up (the SwiGLU pair meets in one lane's accumulators), 16
// rows for down -- over the full K.  One group of kMmaWarps consumer warps
// takes every item; warp w covers K slice w, and the slices' partial sums
// meet in shared memory, added in ascending slice order by the item's
// finishing warp.  Items are dealt to the CTAs in contiguous ranges.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kMmaWarps = 8;       // consumer warps (K slices)
constexpr int kMmaRows = 16;       // weight rows per item
constexpr int kMmaNTiles = 4;      // token tiles of 8 handled per pass (32 tokens)
constexpr int kMmaMaxStages = 8;
constexpr int kMmaPf = 4;  // blocks of activation fragments fetched ahead
// dynamic shared memory ahead of the ring: barriers, abort flag, partial sums
constexpr int kMmaHeaderBytes = 256 + 2 * 8 * 4 * 32 * 4 * 4;

struct MmaArgs {
  const uint8_t* w;    // E2M1 codes, expert-major: group g's row r at w + g*w_gstride + r*(K/2)
  const uint8_t* sc;   // E8M0 scales: sc + g*s_gstride + r*(K/32)
  long long w_gstride;
  long long s_gstride;
  int K;               // multiple of 32 * kMmaWarps
  int out_rows;        // output rows per expert (I for gate/up, H for down)
  int up_off;          // gate/up: rows between a gate row and its up row
  const __half* xh;    // activations in f16, [rows][K], row scaled by 2^-xe[row]
  const int* xe;       // per-row exponents
  int act_by_pair;     // activation row = pair id (1) or pair / top_k (0)
  int top_k;
  int n_pairs;
  int n_experts;
  const int* n_active;
  const int* active;
  const int* offsets;
  const int* pair_ids;
  float* out;          // [pair][out_rows] fp32
  int n_stages;
  int stage_bytes;
  int* err;
};

// f16 copy of activation rows: row r of `src` (bf16 or fp32, K elements) is
// scaled by 2^-e, e chosen from max|x| so that the largest element sits in
// [2^14, 2^15) (exact for bf16, one rounding for fp32); one CTA per row.
// Within each 32-element block the elements are stored in the order the MMA's
// B fragments want them: thread tq of a quad takes elements {2tq, 2tq+1,
// 2tq+8, 2tq+9, 2tq+16, 2tq+17, 2tq+24, 2tq+25} as one 16-byte vector.
template <bool kF32>
__global__ void __launch_bounds__(256) act_to_f16_kernel(const void* __restrict__ src, int K, __half* __restrict__ dst,
                                                         int* __restrict__ exps) {
  __shared__ float s_max[8];
  __shared__ int s_e;
  const int r = blockIdx.x, tid = threadIdx.x;
  pdl_wait();
  float m = 0.f;
  for (int i = tid; i < K; i += 256) {
    const float v = kF32 ? __ldcg(static_cast<const float*>(src) + (size_t)r * K + i)
                         : bf16lo_to_f32(static_cast<const uint16_t*>(src)[(size_t)r * K + i]);
    m = fmaxf(m, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((tid & 31) == 0) s_max[tid >> 5] = m;
  __syncthreads();
  if (tid == 0) {
    float mm = 0.f;
    for (int w = 0; w < 8; ++w) mm = fmaxf(mm, s_max[w]);
    int e = 0;
    if (mm > 0.f && mm < INFINITY) {
      const int ef = (int)((__float_as_uint(mm) >> 23) & 0xFF);
      e = (ef > 0 ? ef - 127 : -127) - 14;
      e = max(-126, min(127, e));
    }
    s_e = e;
    exps[r] = e;
  }
  __syncthreads();
  const float sc = __uint_as_float((uint32_t)(max(-126, min(127, -s_e)) + 127) << 23);
  for (int i = tid; i < K; i += 256) {
    const float v = kF32 ? __ldcg(static_cast<const float*>(src) + (size_t)r * K + i)
                         : bf16lo_to_f32(static_cast<const uint16_t*>(src)[(size_t)r * K + i]);
    const int p = i & 31;
    const int pos = ((i >> 5) * 4 + ((p >> 1) & 3)) * 8 + (((p >> 4) * 2 + ((p >> 3) & 1)) * 2) + (p & 1);
    dst[(size_t)r * K + pos] = __float2half_rn(v * sc);
  }
  pdl_launch_dependents();
}

// byte `sh/8` of w, E2M1 pair -> f16x2
__device__ __forceinline__ uint32_t e2m1_byte_to_f16x2(uint32_t w, uint32_t sh) {
  uint32_t d;
  asm("{\n\t.reg .b8 b, b1, b2, b3;\n\t.reg .b32 t;\n\t"
      "shr.b32 t, %1, %2;\n\t"
      "mov.b32 {b, b1, b2, b3}, t;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
      : "=r"(d)
      : "r"(w), "r"(sh));
  return d;
}

// D = A(16x16, f16, row) * B(16x8, f16, col) + C, fp32
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                          const float (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
        "f"(c[3]));
}

__device__ __forceinline__ uint4 ldg128_cg(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

template <bool kSwiglu>
__global__ void __launch_bounds__((kMmaWarps + 1) * 32, 1) grouped_mma_kernel(const MmaArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = a.K;
  const int rowbytes = K >> 1, sblocks = K >> 5;
  const int R = kSwiglu ? kMmaRows / 2 : kMmaRows;  // output rows per item
  const uint32_t codes_bytes = (uint32_t)(kMmaRows * rowbytes);

  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty_bar = full_bar + kMmaMaxStages;
  uint64_t* group_bar_m = empty_bar + kMmaMaxStages;  // consumer-warp barrier (bounded waits)
  volatile int* s_flag = reinterpret_cast<volatile int*>(smem + 16 * kMmaMaxStages + 16);
  // partial sums: [2 buffers][warp][n tile][lane][4]
  float* s_red = reinterpret_cast<float*>(smem + 256);
  static_assert(kMmaHeaderBytes == 256 + 2 * kMmaWarps * kMmaNTiles * 32 * 4 * (int)sizeof(float), "header");
  unsigned char* stages = smem + kMmaHeaderBytes;

  if (tid == 0) {
    for (int s = 0; s < a.n_stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kMmaWarps);
    }
    mbar_init(group_bar_m, kMmaWarps);
    s_flag[0] = 0;
    fence_barrier_init();
  }
  pdl_wait();  // routing plan and activations come from the preceding kernels
  int n_groups = *a.n_active;
  if (n_groups < 0 || n_groups > a.n_experts) {
    if (tid == 0) atomicExch(a.err, kErrBadPlan);
    n_groups = n_groups < 0 ? 0 : a.n_experts;
  }
  const int n_rt = a.out_rows / R;
  const long long n_items = (long long)n_groups * n_rt;
  const long long lo = n_items * blockIdx.x / gridDim.x;
  const long long hi = n_items * (blockIdx.x + 1) / gridDim.x;
  __syncthreads();
  if (a.n_stages < 1 || a.n_stages > kMmaMaxStages || (K % (32 * kMmaWarps)) != 0 || (a.out_rows % R) != 0) {
    if (tid == 0) atomicExch(a.err, kErrBadPlan);
    return;
  }

  if (warp == kMmaWarps) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int s = 0;
      uint32_t ph = 0;
      int pg = -1, pgrp = 0;
      const uint32_t cb = (uint32_t)(R * rowbytes), sb = (uint32_t)(R * sblocks);
      for (long long it = lo; it < hi; ++it) {
        if (s_flag[0] || !mbar_wait_bounded(&empty_bar[s], ph ^ 1u)) {
          if (!s_flag[0]) atomicExch(a.err, kErrTimeout);
          s_flag[0] = 1;
          break;
        }
        const int g = (int)(it / n_rt), r0 = (int)(it - (long long)g * n_rt) * R;
        if (g != pg) {
          pg = g;
          pgrp = clamp_group(a.active[g], a.n_experts, a.err);
        }
        unsigned char* st = stages + (size_t)s * a.stage_bytes;
        const uint8_t* wg = a.w + (long long)pgrp * a.w_gstride;
        const uint8_t* sg = a.sc + (long long)pgrp * a.s_gstride;
        mbar_arrive_expect_tx(&full_bar[s], (kSwiglu ? 2u : 1u) * (cb + sb));
        bulk_g2s(st, wg + (size_t)r0 * rowbytes, cb, &full_bar[s], pol);
        bulk_g2s(st + codes_bytes, sg + (size_t)r0 * sblocks, sb, &full_bar[s], pol);
        if (kSwiglu) {
          bulk_g2s(st + cb, wg + (size_t)(r0 + a.up_off) * rowbytes, cb, &full_bar[s], pol);
          bulk_g2s(st + codes_bytes + sb, sg + (size_t)(r0 + a.up_off) * sblocks, sb, &full_bar[s], pol);
        }
        if (++s == a.n_stages) { s = 0; ph ^= 1u; }
      }
      if (s_flag[0]) {
        for (int q = 0; q < a.n_stages; ++q) {
          (void)mbar_wait_bounded(&full_bar[q], 0u, 1ll << 24);
          (void)mbar_wait_bounded(&full_bar[q], 1u, 1ll << 24);
        }
      }
    }
    pdl_launch_dependents();
    return;
  }

  // ------------------------------ consumers ------------------------------
  const int gq = lane >> 2, tq = lane & 3;  // mma group id / thread in group
  const uint32_t sh = 8u * (uint32_t)tq;
  const int nblk = sblocks / kMmaWarps;      // 32-element blocks in this warp's K slice
  const int kb0 = warp * nblk;
  int s = 0;
  uint32_t par = 0;
  int cg = -1, tok0 = 0, ntok = 0;
  int nit = 0, npass_done = 0;  // items and token passes of this CTA so far
  uint32_t gph = 0;              // phase of the consumer-warp barrier
  for (long long it = lo; it < hi; ++it, ++nit) {
    const int g = (int)(it / n_rt), r0 = (int)(it - (long long)g * n_rt) * R;
    if (g != cg) {
      cg = g;
      const int grp = clamp_group(a.active[g], a.n_experts, nullptr);
      tok0 = a.offsets[grp];
      ntok = a.offsets[grp + 1] - tok0;
      if (tok0 < 0 || ntok < 0 || tok0 + ntok > a.n_pairs) {
        if (lane == 0) atomicExch(a.err, kErrBadPlan);
        tok0 = 0;
        ntok = 0;
      }
    }
    bool have = s_flag[0] == 0;
    if (have && !mbar_wait_bounded(&full_bar[s], par)) {
      if (lane == 0) atomicExch(a.err, kErrTimeout);
      s_flag[0] = 1;
      have = false;
    }
    have = __all_sync(0xFFFFFFFFu, have);  // the MMAs below need the whole warp
    const unsigned char* st = stages + (size_t)s * a.stage_bytes;
    // token passes of up to 8 * kMmaNTiles tokens; every warp runs the same passes
    for (int t0 = 0; t0 < max(ntok, 1); t0 += 8 * kMmaNTiles) {
      const int npass = min(ntok - t0, 8 * kMmaNTiles);
      // this lane's activation rows (token column gq of each n tile)
      const __half* xrow[kMmaNTiles];
#pragma unroll
      for (int nt = 0; nt < kMmaNTiles; ++nt) {
        const int c = nt * 8 + gq;
        xrow[nt] = nullptr;
        if (have && c < npass) {
          int pr = a.pair_ids[tok0 + t0 + c];
          if (pr < 0 || pr >= a.n_pairs) pr = 0;
          const int src = a.act_by_pair ? pr : pr / a.top_k;
          xrow[nt] = a.xh + (size_t)src * K;
        }
      }
      float acc[kMmaNTiles][4];
#pragma unroll
      for (int nt = 0; nt < kMmaNTiles; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[nt][q] = 0.f;
      const float zero[4] = {0.f, 0.f, 0.f, 0.f};
      if (have && npass > 0) {
        const int ntiles = (npass + 7) >> 3;
        const unsigned char* rowA = st + (size_t)gq * rowbytes;
        const unsigned char* rowB = st + (size_t)(gq + 8) * rowbytes;
        const unsigned char* scl = st + codes_bytes;
        // Token tiles two at a time; their activation fragments (one 16-byte
        // load per block, tile and lane) are fetched kMmaPf blocks ahead.  The
        // MMAs are warp-collective: whether a tile is computed depends only on
        // warp-uniform values; a lane without a token in a tile feeds zeros.
#pragma unroll
        for (int pp = 0; pp < kMmaNTiles / 2; ++pp) {
          if (2 * pp < ntiles) {
            const bool two = 2 * pp + 1 < ntiles;  // warp-uniform
            const uint4* xp0 = reinterpret_cast<const uint4*>(xrow[2 * pp]);
            const uint4* xp1 = two ? reinterpret_cast<const uint4*>(xrow[2 * pp + 1]) : nullptr;
            uint4 xq[kMmaPf][2];
#pragma unroll
            for (int j = 0; j < kMmaPf; ++j) {
              const int kb = kb0 + j;
              xq[j][0] = (xp0 && j < nblk) ? ldg128_cg(xp0 + kb * 4 + tq) : make_uint4(0u, 0u, 0u, 0u);
              xq[j][1] = (xp1 && j < nblk) ? ldg128_cg(xp1 + kb * 4 + tq) : make_uint4(0u, 0u, 0u, 0u);
            }
            for (int i = 0; i < nblk; i += kMmaPf) {
#pragma unroll
              for (int j = 0; j < kMmaPf; ++j) {
                const int ib = i + j;
                if (ib < nblk) {  // warp-uniform
                  const int kb = kb0 + ib;
                  const uint4 wa = lds128(rowA + 16 * kb), wb = lds128(rowB + 16 * kb);
                  const float sa = e8m0_to_f32(lds_u8(scl + gq * sblocks + kb));
                  const float sbv = e8m0_to_f32(lds_u8(scl + (gq + 8) * sblocks + kb));
                  uint32_t a0[4], a1[4];
                  a0[0] = e2m1_byte_to_f16x2(wa.x, sh);
                  a0[1] = e2m1_byte_to_f16x2(wb.x, sh);
                  a0[2] = e2m1_byte_to_f16x2(wa.y, sh);
                  a0[3] = e2m1_byte_to_f16x2(wb.y, sh);
                  a1[0] = e2m1_byte_to_f16x2(wa.z, sh);
                  a1[1] = e2m1_byte_to_f16x2(wb.z, sh);
                  a1[2] = e2m1_byte_to_f16x2(wa.w, sh);
                  a1[3] = e2m1_byte_to_f16x2(wb.w, sh);
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    if (h == 0 || two) {  // warp-uniform
                      float d[4];
                      mma_16816(d, a0, xq[j][h].x, xq[j][h].y, zero);
                      mma_16816(d, a1, xq[j][h].z, xq[j][h].w, d);
                      float(&ac)[4] = acc[2 * pp + h];
                      ac[0] = fmaf(d[0], sa, ac[0]);
                      ac[1] = fmaf(d[1], sa, ac[1]);
                      ac[2] = fmaf(d[2], sbv, ac[2]);
                      ac[3] = fmaf(d[3], sbv, ac[3]);
                    }
                  }
                  const int nb = ib + kMmaPf;
                  if (nb < nblk) {
                    if (xp0) xq[j][0] = ldg128_cg(xp0 + (kb0 + nb) * 4 + tq);
                    if (xp1) xq[j][1] = ldg128_cg(xp1 + (kb0 + nb) * 4 + tq);
                  }
                }
              }
            }
          }
        }
      }
      // partial sums of this K slice, then the item's finishing warp adds the
      // slices in ascending order and writes the outputs
      // buffers alternate pass by pass: a warp writes a buffer again only after
      // the next pass's barrier, which the finisher reaches after its reads
      float* red = s_red + (size_t)(npass_done & 1) * kMmaWarps * kMmaNTiles * 128;
#pragma unroll
      for (int nt = 0; nt < kMmaNTiles; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) red[((warp * kMmaNTiles + nt) * 32 + lane) * 4 + q] = acc[nt][q];
      if (t0 + 8 * kMmaNTiles >= ntok && have) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);
      }
      // all consumer warps meet here (an mbarrier, so the wait is bounded: a
      // warp that gives up records the timeout and the item's outputs are void)
      __syncwarp();
      if (lane == 0) mbar_arrive(group_bar_m);
      // (once aborting, waits are short so that a broken pipeline ends quickly)
      if (!mbar_wait_bounded(group_bar_m, gph, s_flag[0] ? (1ll << 20) : (1ll << 31))) {
        if (lane == 0) atomicExch(a.err, kErrTimeout);
        s_flag[0] = 1;
        have = false;
      }
      have = __all_sync(0xFFFFFFFFu, have);
      gph ^= 1u;
      if (have && warp == (int)(npass_done % kMmaWarps) && npass > 0) {
#pragma unroll
        for (int nt = 0; nt < kMmaNTiles; ++nt) {
          float v[4] = {0.f, 0.f, 0.f, 0.f};
          for (int w = 0; w < kMmaWarps; ++w)
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] += red[((w * kMmaNTiles + nt) * 32 + lane) * 4 + q];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = nt * 8 + 2 * tq + cc;  // token column of accumulator pair cc
            if (c < npass) {
              const int pr = a.pair_ids[tok0 + t0 + c];
              if (pr >= 0 && pr < a.n_pairs) {
                const int src = a.act_by_pair ? pr : pr / a.top_k;
                const float e = __uint_as_float((uint32_t)(max(-126, min(127, a.xe[src])) + 127) << 23);
                float* o = a.out + (size_t)pr * a.out_rows;
                if (kSwiglu) {
                  const float gg = v[cc] * e, uu = v[2 + cc] * e;
                  o[r0 + gq] = gg / (1.0f + expf(-gg)) * uu;
                } else {
                  o[r0 + gq] = v[cc] * e;
                  o[r0 + gq + 8] = v[2 + cc] * e;
                }
              }
            }
          }
        }
      }
      ++npass_done;
    }
    if (++s == a.n_stages) { s = 0; par ^= 1u; }
  }
  pdl_launch_dependents();
}

}  // namespace moe
