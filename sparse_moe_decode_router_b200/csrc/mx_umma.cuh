// Routed MXFP4 expert projections on the 5th-generation tensor cores
// (tcgen05 block-scaled MMA, sm_100a).
//
// The decode-path pages use batch-specialised expert kernels (smzdm, section on
// the four-step rework, first step); here one kernel design serves every batch
// size by leaving all per-weight work to the TMA unit and the tensor cores:
//
//  * weights (A operand, M = 128 rows of one expert per MMA) are E2M1 codes
//    copied by tiled TMA with the 16U4_ALIGN16B element type, which expands
//    each 16 packed 4-bit values into a 16-byte shared-memory chunk (8 bytes
//    of data, 8 of gap) -- the layout `tcgen05.mma.kind::mxf8f6f4` reads for a
//    4-bit operand -- under the 128-byte swizzle.  No CUDA-core instruction
//    touches a weight;
//  * the weights' E8M0 block scales (one per row and 32 K elements) are
//    gathered by one warp into the scale-factor chunk layout (128 rows x 4
//    K-blocks in 512 bytes: row r = r0 + 32*r1 at byte 16*r0 + 4*r1 + block)
//    and copied into tensor memory with `tcgen05.cp.32x128b.warpx4`;
//  * activations (B operand) are MX values too: each token's activation row
//    is split into kTerms E4M3 terms (the value, then what the first term
//    missed, ...), each with its own E8M0 scale per 32 elements chosen so the
//    block maximum fits E4M3's 448 without clipping.  A token's terms are
//    separate B columns; the epilogue adds them.  Three terms carry about 12
//    significant bits, more than the 11 of the f16 the CUDA-core kernels use;
//  * B columns are rows of a buffer ordered like the routing plan's pair list
//    (position q of pair_ids, term t -> row q*kTerms + t), so an expert's
//    tokens are one contiguous run of rows: one tiled TMA per 8 rows;
//  * the accumulators live in tensor memory (fp32, M = 128 lanes x N
//    columns, two buffers so the epilogue of one item overlaps the MMAs of
//    the next) and are read back with `tcgen05.ld.32x32b`.
//
// Warp roles (256 threads, one CTA per SM): warp 0 issues the TMA copies,
// warp 1 owns the tensor memory and one of its lanes issues the MMAs, warp 2
// builds the scale-factor chunks, warps 4..7 are the epilogue (warp w reads
// TMEM lanes 32*(w%4) .. +31).  Every wait is bounded: a wait that gives up
// records MOE_ERR_TIMEOUT in the error word and the CTA drains without work.
//
// Epilogues: gate/up -> h = silu(g) * u per (row, token), written as fp32
// (optional) and as the down projection's E4M3 terms; down -> y fp32 per
// (pair, row).  An item is 128 output rows of one active expert (gate/up:
// 128 gate rows and the matching 128 up rows as two MMAs into two
// accumulators), all K, for up to kMxNMax / kTerms tokens per pass; experts
// with more tokens take several passes over the same weights.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kMxRows = 128;       // M: weight rows per MMA (one TMEM lane each)
constexpr int kMxKTile = 128;      // K elements per pipeline stage (one 128-byte swizzle row)
constexpr int kMxNMax = 64;        // B columns per pass (tokens x terms, padded to 16)
constexpr int kMxMaxStages = 12;   // TMEM: scale chunks of 12 stages fit below column 432
constexpr int kMxThreads = 256;
constexpr int kMxTmemCols = 512;
constexpr int kMxAccCols = 128;    // per accumulator buffer: gate [0, 64), up [64, 128)
constexpr int kMxSfaCol0 = 256;    // per stage 8 columns: gate chunk, up chunk (256 + 8*12 <= 384)
constexpr int kMxSfbCol0 = 384;    // per stage 4 columns (384 + 4*12 <= 512)
static_assert(kMxSfaCol0 + 8 * kMxMaxStages <= kMxSfbCol0 && kMxSfbCol0 + 4 * kMxMaxStages <= kMxTmemCols,
              "scale-factor columns");
constexpr int kMxHeaderBytes = 1024;
static_assert(8 * (2 * kMxMaxStages + 6) + 32 <= kMxHeaderBytes, "header");
constexpr int kMxABytes = kMxRows * kMxKTile;  // one A tile in shared memory (16 KB, expanded)
constexpr uint32_t kMxATx = kMxRows * kMxKTile / 2;  // bytes one A tile moves (packed)

struct MxArgs {
  const uint8_t* sc;        // weight E8M0 scales [E][rows][K/32]
  long long s_gstride;      // bytes per expert in sc
  int a_rows;               // weight rows per expert in the A tensor map (2I or H)
  int K;                    // reduction length, multiple of 128
  int out_rows;             // output rows per expert (I or H), multiple of 128
  int up_off;               // gate/up: rows from a gate row to its up row (= I); 0 for down
  int top_k;
  int n_pairs;              // B * top_k of this call
  int n_experts;
  const int* n_active;
  const int* active;
  const int* offsets;
  const int* pair_ids;
  const uint8_t* asf;       // activation term scales [act_rows][K/32]
  int act_rows;             // rows of the activation-term buffers (capacity)
  int n_max;                // B columns one pass may use (multiple of 16, <= kMxNMax)
  float* out_f32;           // gate/up: h [pair][I] (may be null); down: y [pair][H]
  uint8_t* next_aq;         // gate/up: the down projection's E4M3 terms [act_rows][I]
  uint8_t* next_asf;        // ... and their scales [act_rows][I/32]
  int n_stages;
  int stage_bytes;          // multiple of 1024
  int off_up, off_b, off_sfa, off_sfb;  // byte offsets inside a stage
  // down projection fused with the combine (comb_w non-null): per 128-row
  // tile of H the last item to finish (a counter per tile reaching the
  // number of active experts) writes out[b][r] = bf16(residual + y_shared +
  // sum_j w[b][j] y[b*k+j][r]) for every token, ascending j
  const float* comb_w;      // topk_w [B][k]
  const float* y_shared;    // [B][H] or null
  const uint16_t* residual; // bf16 [B][H]
  uint16_t* out_bf16;       // bf16 [B][H]
  int batch;
  int* tile_counter;        // [H / 128], zero between launches
  // L2 prefetch of the next layer's static weights, issued at the end
  const uint8_t* pf_ptr[2];
  long long pf_bytes[2];
  int* err;
};

// ---------------------------------------------------------------------------
// tcgen05 / TMA helpers (inline PTX, ISA 8.7)
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem], block-scaled: A scales at sfa, B scales at sfb
__device__ __forceinline__ void tc_mma_mx(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                          uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// 32 TMEM lanes x 128 bits from shared memory, broadcast to all four lane quadrants
__device__ __forceinline__ void tc_cp_32x128_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// shared-memory matrix descriptor, K-major with the 128-byte swizzle: rows of
// 128 bytes, 8-row groups 1024 bytes apart (SBO), version 1 (sm_100)
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// descriptor of a scale-factor chunk: no swizzle, 8-row x 16-byte core
// matrices stored contiguously (128 bytes apart)
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(128 >> 4) << 32) |
         ((uint64_t)1 << 46);
}

// instruction descriptor, kind::mxf8f6f4 block-scaled: A E2M1, B E4M3, both
// K-major, E8M0 scale factors, M = 128, N columns; the K-block of each scale
// vector is set per MMA (bits 29-30 for A, 4-5 for B)
__host__ __device__ constexpr uint32_t mx_idesc(int n) {
  return (5u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | ((uint32_t)(kMxRows >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, "
      "%4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d_nohint(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// MX activation terms.  A term of a 32-element block: scale 2^e with e the
// smallest integer that keeps max|v| * 2^-e <= 448 (E4M3's largest finite
// value), then each element rounded to nearest even E4M3 (saturating).
__device__ __forceinline__ int mx_scale_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  const uint32_t u = __float_as_uint(amax);
  const int ef = (int)((u >> 23) & 0xFFu);
  const int E = ef ? ef - 127 : -127;
  const int e = E - 8 + ((u & 0x7FFFFFu) > 0x600000u ? 1 : 0);  // 448 = 1.75 * 2^8
  return max(-127, min(127, e));
}

// 2^e as an exact fp32 for e in [-127, 127] (2^-127 is subnormal)
__device__ __forceinline__ float pow2_exact(int e) {
  return __uint_as_float(e >= -126 ? (uint32_t)(e + 127) << 23 : 0x00400000u);
}

__device__ __forceinline__ uint32_t f32_to_e4m3(float v) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(d) : "f"(v));
  return d & 0xFFu;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  uint32_t h2;
  const uint16_t in = (uint16_t)(b | (b << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// x (bf16 [B][K]) -> terms of the gate/up activations, one CTA per position
// q of the pair list: rows q*kTerms + t of aq [.][K] and asf [.][K/32].
template <int kTerms>
__global__ void __launch_bounds__(256) mx_x_terms_kernel(const uint16_t* __restrict__ x, int K, int top_k, int n_pairs,
                                                         const int* __restrict__ pair_ids, uint8_t* __restrict__ aq,
                                                         uint8_t* __restrict__ asf, int* err) {
  pdl_wait();
  const int q = blockIdx.x;
  int p = pair_ids[q];
  if (p < 0 || p >= n_pairs) {
    if (threadIdx.x == 0) atomicExch(err, kErrBadPlan);
    p = 0;
  }
  const int b = p / top_k;
  const int nblk = K >> 5;
  for (int blk = threadIdx.x; blk < nblk; blk += blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)b * K + 32 * blk);
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 u = __ldcg(src + i);  // written by a preceding kernel: coherent path
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * i + 2 * j] = bf16lo_to_f32(w[j]);
        v[8 * i + 2 * j + 1] = bf16hi_to_f32(w[j]);
      }
    }
#pragma unroll
    for (int t = 0; t < kTerms; ++t) {
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
      const int e = mx_scale_exp(amax);
      const float inv = pow2_exact(-e), sc = pow2_exact(e);
      uint32_t packed[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) packed[i] = 0u;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint32_t c = f32_to_e4m3(v[i] * inv);
        packed[i >> 2] |= c << (8 * (i & 3));
        v[i] -= e4m3_to_f32(c) * sc;
      }
      uint4* dst = reinterpret_cast<uint4*>(aq + ((size_t)q * kTerms + t) * K + 32 * blk);
      dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      asf[((size_t)q * kTerms + t) * nblk + blk] = (uint8_t)(e + 127);
    }
  }
  pdl_launch_dependents();
}

// ---------------------------------------------------------------------------
// Per-CTA item walk shared by every role: items are (active group, 128-row
// tile), contiguous ranges per CTA; each item runs one pass per kMxNMax /
// kTerms tokens of its expert.
struct MxUnit {
  int e;      // expert
  int rt;     // row tile
  int tok;    // first position of this pass in the pair list
  int ntok;   // tokens in this pass
  int n;      // B columns (multiple of 16: M = 128 MMAs take N in steps of 16)
};

template <int kTerms>
struct MxWalk {
  const MxArgs& a;
  long long it, hi;
  int n_rt, pass, npass, e, tok0, cnt;
  bool bad;
  __device__ MxWalk(const MxArgs& args, long long lo, long long hi_, int nrt)
      : a(args), it(lo), hi(hi_), n_rt(nrt), pass(0), npass(0), e(0), tok0(0), cnt(0), bad(false) {
    if (it < hi) load();
  }
  __device__ void load() {
    const int g = (int)(it / n_rt);
    e = a.active[g];
    if (e < 0 || e >= a.n_experts) { bad = true; e = 0; }
    tok0 = a.offsets[e];
    cnt = a.offsets[e + 1] - tok0;
    if (tok0 < 0 || cnt < 1 || tok0 + cnt > a.n_pairs) { bad = true; tok0 = 0; cnt = 1; }
    const int tpp = a.n_max / kTerms;
    npass = (cnt + tpp - 1) / tpp;
    pass = 0;
  }
  __device__ bool valid() const { return it < hi; }
  __device__ MxUnit unit() const {
    const int tpp = a.n_max / kTerms;
    MxUnit u;
    u.e = e;
    u.rt = (int)(it % n_rt);
    u.tok = tok0 + pass * tpp;
    u.ntok = min(tpp, cnt - pass * tpp);
    u.n = (u.ntok * kTerms + 15) & ~15;
    return u;
  }
  __device__ void next() {
    if (++pass < npass) return;
    if (++it < hi) load();
  }
};

template <int kTerms>
__device__ __forceinline__ float warp_amax(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

template <bool kSwiglu, int kTerms>
__global__ void __launch_bounds__(kMxThreads, 1)
    mx_expert_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const MxArgs a) {
  static_assert(kMxNMax % 16 == 0 && kTerms >= 1 && kTerms <= 3, "terms");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // header: barriers and flags; the stage ring starts at the next 1024-byte boundary
  const uint32_t raw = smem_addr(smem_raw);
  unsigned char* hdr = smem_raw;
  unsigned char* ring = smem_raw + (((raw + kMxHeaderBytes + 1023u) & ~1023u) - raw);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(hdr);
  uint64_t* empty_bar = full_bar + kMxMaxStages;
  uint64_t* acc_full = empty_bar + kMxMaxStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done_bar = acc_empty + 2;
  uint64_t* epi_bar = done_bar + 1;  // the four epilogue warps meet here (fused combine)
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(hdr + 8 * (2 * kMxMaxStages + 6));
  volatile int* s_abort = reinterpret_cast<volatile int*>(hdr + 8 * (2 * kMxMaxStages + 6) + 16);
  volatile int* s_last = s_abort + 1;

  const int K = a.K, KT = K / kMxKTile, sblk = K / 32;
  const int ns = a.n_stages;
  if (tid == 0) {
    for (int s = 0; s < kMxMaxStages; ++s) {
      mbar_init(&full_bar[s], 2);    // the TMA thread's expect-tx arrive + the scale-factor warp
      mbar_init(&empty_bar[s], 1);   // tcgen05.commit after the stage's MMAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);    // tcgen05.commit after an item's last MMA
      mbar_init(&acc_empty[b], 4);   // one arrive per epilogue warp
    }
    mbar_init(done_bar, 1);
    mbar_init(epi_bar, 4);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    // the whole tensor memory of the SM: one CTA per SM (shared memory use)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr((const void*)s_tmem)),
                 "r"(kMxTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  // the routing plan and the activation terms come from the preceding kernels
  pdl_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  int n_groups = *a.n_active;
  if (n_groups < 0 || n_groups > a.n_experts) {
    if (tid == 0) atomicExch(a.err, kErrBadPlan);
    n_groups = n_groups < 0 ? 0 : a.n_experts;
  }
  const int n_rt = a.out_rows / kMxRows;
  const long long n_items = (long long)n_groups * n_rt;
  const long long lo = n_items * blockIdx.x / gridDim.x;
  const long long hi = n_items * (blockIdx.x + 1) / gridDim.x;
  const bool plan_ok = ns >= 1 && ns <= kMxMaxStages && (K % kMxKTile) == 0 && (a.out_rows % kMxRows) == 0 &&
                       a.n_max >= 16 && a.n_max <= kMxNMax && (a.n_max % 16) == 0;
  if (!plan_ok) {
    if (tid == 0) atomicExch(a.err, kErrBadPlan);
  }
  const long long lim_long = 1ll << 31, lim_short = 1ll << 20;

  if (plan_ok && warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int s = 0;
      uint32_t ph = 0;
      for (MxWalk<kTerms> w(a, lo, hi, n_rt); w.valid() && !*s_abort; w.next()) {
        const MxUnit u = w.unit();
        const int arow = u.e * a.a_rows + u.rt * kMxRows;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, *s_abort ? lim_short : lim_long)) {
            atomicExch(a.err, kErrTimeout);
            *s_abort = 1;
            break;
          }
          const uint32_t st = smem_addr(ring + (size_t)s * a.stage_bytes);
          mbar_arrive_expect_tx(&full_bar[s], (kSwiglu ? 2u : 1u) * kMxATx + (uint32_t)u.n * 128u);
          tma_load_2d(st, &tmA, kt * kMxKTile, arow, &full_bar[s], pol);
          if (kSwiglu) tma_load_2d(st + a.off_up, &tmA, kt * kMxKTile, arow + a.up_off, &full_bar[s], pol);
          for (int j = 0; j < u.n / 8; ++j)
            tma_load_2d_nohint(st + a.off_b + 1024 * j, &tmB, kt * kMxKTile, u.tok * kTerms + 8 * j, &full_bar[s]);
          if (++s == ns) { s = 0; ph ^= 1u; }
        }
      }
      if (*s_abort) {
        // let copies already in flight land before the CTA can exit
        for (int q = 0; q < ns; ++q) {
          (void)mbar_wait_bounded(&full_bar[q], 0u, lim_short);
          (void)mbar_wait_bounded(&full_bar[q], 1u, lim_short);
        }
      }
      // warm L2 with the next layer's static weights (one slice per CTA)
      for (int qq = 0; qq < 2; ++qq) {
        if (!a.pf_ptr[qq] || a.pf_bytes[qq] <= 0) continue;
        const long long per = ((a.pf_bytes[qq] / gridDim.x) + 15) & ~15ll;
        const long long beg = per * blockIdx.x;
        const long long end = min(beg + per, a.pf_bytes[qq]);
        for (long long o = beg; o < end; o += 65536) {
          const long long nb = min(end - o, 65536ll);
          if (nb >= 16) prefetch_l2(a.pf_ptr[qq] + o, (uint32_t)(nb & ~15ll));
        }
      }
    }
  } else if (plan_ok && warp == 2) {
    // ------------------------- scale-factor chunks ----------------------------
    // Weight scales are static (read-only path); the activation scales come
    // from the preceding kernel and are read through L2 (coherent path).
    // Lane l covers rows l + 32*m (m = 0..3) of the A tile(s) and B columns
    // l + 32*m (m = 0..1).  Where a scale row is a multiple of 16 bytes long,
    // one 16-byte load per row fetches four stages' scale bytes, and the next
    // group of four is requested before the current one is stored, so the
    // loads' latency overlaps the stages.
    const bool wide = (sblk % 16) == 0;
    int s = 0;
    uint32_t ph = 0;
    for (MxWalk<kTerms> w(a, lo, hi, n_rt); w.valid() && !*s_abort; w.next()) {
      const MxUnit u = w.unit();
      const uint8_t* sg = a.sc + (long long)u.e * a.s_gstride;
      const int r0 = u.rt * kMxRows;
      // 16-byte groups (4 K-tiles) of this lane's rows: A gate, A up, B
      auto load_group = [&](int kg, uint4 (&ga)[4], uint4 (&ua)[4], uint4 (&bb)[2]) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          ga[m] = __ldg(reinterpret_cast<const uint4*>(sg + (size_t)(r0 + lane + 32 * m) * sblk + 4 * kg));
          if (kSwiglu)
            ua[m] = __ldg(reinterpret_cast<const uint4*>(sg + (size_t)(r0 + a.up_off + lane + 32 * m) * sblk + 4 * kg));
        }
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const int n = lane + 32 * m, row = u.tok * kTerms + n;
          bb[m] = (n < u.n && row < a.act_rows)
                      ? __ldcg(reinterpret_cast<const uint4*>(a.asf + (size_t)row * sblk + 4 * kg))
                      : make_uint4(0u, 0u, 0u, 0u);
        }
      };
      uint4 cg[4], cu[4], cb[2], ng[4], nu[4], nb[2];
      if (wide) load_group(0, cg, cu, cb);
      bool stop = false;
      for (int kg = 0; kg < KT && !stop; kg += 4) {
        if (wide && kg + 4 < KT) load_group(kg + 4, ng, nu, nb);
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          const int kt = kg + j4;
          if (kt >= KT) break;
          bool ok = mbar_wait_bounded(&empty_bar[s], ph ^ 1u, *s_abort ? lim_short : lim_long);
          ok = __all_sync(0xFFFFFFFFu, ok);
          if (!ok) {
            if (lane == 0) atomicExch(a.err, kErrTimeout);
            *s_abort = 1;
            stop = true;
            break;
          }
          uint32_t vg[4], vu[4], vb[4];
          if (wide) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              vg[m] = j4 == 0 ? cg[m].x : j4 == 1 ? cg[m].y : j4 == 2 ? cg[m].z : cg[m].w;
              vu[m] = j4 == 0 ? cu[m].x : j4 == 1 ? cu[m].y : j4 == 2 ? cu[m].z : cu[m].w;
            }
#pragma unroll
            for (int m = 0; m < 2; ++m)
              vb[m] = j4 == 0 ? cb[m].x : j4 == 1 ? cb[m].y : j4 == 2 ? cb[m].z : cb[m].w;
          } else {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              vg[m] = __ldg(reinterpret_cast<const uint32_t*>(sg + (size_t)(r0 + lane + 32 * m) * sblk + 4 * kt));
              vu[m] = kSwiglu ? __ldg(reinterpret_cast<const uint32_t*>(sg + (size_t)(r0 + a.up_off + lane + 32 * m) *
                                                                                 sblk + 4 * kt))
                              : 0u;
            }
#pragma unroll
            for (int m = 0; m < 2; ++m) {
              const int n = lane + 32 * m, row = u.tok * kTerms + n;
              vb[m] = (n < u.n && row < a.act_rows)
                          ? __ldcg(reinterpret_cast<const uint32_t*>(a.asf + (size_t)row * sblk + 4 * kt))
                          : 0u;
            }
          }
          vb[2] = vb[3] = 0u;  // B columns 64..127 (beyond kMxNMax)
          unsigned char* st = ring + (size_t)s * a.stage_bytes;
          *reinterpret_cast<uint4*>(st + a.off_sfa + 16 * lane) = make_uint4(vg[0], vg[1], vg[2], vg[3]);
          if (kSwiglu)
            *reinterpret_cast<uint4*>(st + a.off_sfa + 512 + 16 * lane) = make_uint4(vu[0], vu[1], vu[2], vu[3]);
          *reinterpret_cast<uint4*>(st + a.off_sfb + 16 * lane) = make_uint4(vb[0], vb[1], vb[2], vb[3]);
          // generic-proxy stores -> visible to tcgen05.cp (async proxy)
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) mbar_arrive(&full_bar[s]);
          if (++s == ns) { s = 0; ph ^= 1u; }
        }
        if (wide) {
#pragma unroll
          for (int m = 0; m < 4; ++m) { cg[m] = ng[m]; cu[m] = nu[m]; }
#pragma unroll
          for (int m = 0; m < 2; ++m) cb[m] = nb[m];
        }
      }
    }
  } else if (plan_ok && warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      int s = 0, uc = 0;
      uint32_t ph = 0;
      for (MxWalk<kTerms> w(a, lo, hi, n_rt); w.valid() && !*s_abort; w.next(), ++uc) {
        const MxUnit u = w.unit();
        const int b = uc & 1;
        if (!mbar_wait_bounded(&acc_empty[b], (((uint32_t)uc >> 1) & 1u) ^ 1u, lim_long)) {
          atomicExch(a.err, kErrTimeout);
          *s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_g = tmem + (uint32_t)(b * kMxAccCols);
        const uint32_t d_u = d_g + (uint32_t)(kMxAccCols / 2);
        const uint32_t idesc = mx_idesc(u.n);
        bool ok = true;
        for (int kt = 0; kt < KT && ok; ++kt) {
          if (!mbar_wait_bounded(&full_bar[s], ph, *s_abort ? lim_short : lim_long)) {
            atomicExch(a.err, kErrTimeout);
            *s_abort = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_addr(ring + (size_t)s * a.stage_bytes);
          const uint32_t sfa_g = tmem + (uint32_t)(kMxSfaCol0 + 8 * s), sfa_u = sfa_g + 4u;
          const uint32_t sfb = tmem + (uint32_t)(kMxSfbCol0 + 4 * s);
          tc_cp_32x128_x4(sfa_g, desc_sf(st + a.off_sfa));
          if (kSwiglu) tc_cp_32x128_x4(sfa_u, desc_sf(st + a.off_sfa + 512));
          tc_cp_32x128_x4(sfb, desc_sf(st + a.off_sfb));
          const uint64_t ad = desc_sw128(st), bd = desc_sw128(st + a.off_b);
          const uint64_t ud = kSwiglu ? desc_sw128(st + a.off_up) : 0ull;
#pragma unroll
          for (int j = 0; j < kMxKTile / 32; ++j) {
            // K-block j of the stage: +32 bytes in every swizzled row; scale byte j
            const uint32_t id = idesc | ((uint32_t)j << 29) | ((uint32_t)j << 4);
            const uint32_t acc = (kt > 0 || j > 0) ? 1u : 0u;
            const uint32_t sel = (uint32_t)j << 30;
            tc_mma_mx(d_g, ad + 2u * j, bd + 2u * j, id, sfa_g | sel, sfb | sel, acc);
            if (kSwiglu) tc_mma_mx(d_u, ud + 2u * j, bd + 2u * j, id, sfa_u | sel, sfb | sel, acc);
          }
          tc_commit(&empty_bar[s]);  // the stage is free once these MMAs have read it
          if (++s == ns) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&acc_full[b]);
      }
      // every MMA issued by this thread has completed before the TMEM is freed
      tc_commit(done_bar);
      if (!mbar_wait_bounded(done_bar, 0u, lim_long)) atomicExch(a.err, kErrTimeout);
    }
    __syncwarp();
  } else if (plan_ok && warp >= 4) {
    // ------------------------------ epilogue ----------------------------------
    const int q = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    int uc = 0;
    uint32_t epi_ph = 0;
    // bounded meeting of the four epilogue warps (a warp that gives up
    // records the timeout and stops; the others then time out too)
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
    for (MxWalk<kTerms> w(a, lo, hi, n_rt); w.valid(); w.next(), ++uc) {
      const MxUnit u = w.unit();
      const int b = uc & 1;
      bool ok = !*s_abort && mbar_wait_bounded(&acc_full[b], ((uint32_t)uc >> 1) & 1u, lim_long);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (lane == 0 && !*s_abort) atomicExch(a.err, kErrTimeout);
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      float g[kMxNMax], up[kSwiglu ? kMxNMax : 1];
#pragma unroll
      for (int c = 0; c < kMxNMax / 16; ++c) {
        if (16 * c < u.n) {  // warp-uniform
          float t16[16];
          tc_ld16(lane_base + (uint32_t)(b * kMxAccCols + 16 * c), t16);
#pragma unroll
          for (int i = 0; i < 16; ++i) g[16 * c + i] = t16[i];
          if (kSwiglu) {
            tc_ld16(lane_base + (uint32_t)(b * kMxAccCols + kMxAccCols / 2 + 16 * c), t16);
#pragma unroll
            for (int i = 0; i < 16; ++i) up[16 * c + i] = t16[i];
          }
        }
      }
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
      const int row = u.rt * kMxRows + 32 * q + lane;  // output row of this lane
#pragma unroll
      for (int i = 0; i < kMxNMax / kTerms; ++i) {
        if (i < u.ntok) {  // warp-uniform
          float gs = 0.f, us = 0.f;
#pragma unroll
          for (int t = 0; t < kTerms; ++t) {
            gs += g[i * kTerms + t];
            if (kSwiglu) us += up[i * kTerms + t];
          }
          const int pos = u.tok + i;
          int pr = a.pair_ids[pos];
          if (pr < 0 || pr >= a.n_pairs) pr = 0;
          if (kSwiglu) {
            const float hv = gs / (1.0f + expf(-gs)) * us;
            if (a.out_f32) a.out_f32[(size_t)pr * a.out_rows + row] = hv;
            // the down projection's terms: this warp's 32 rows are one 32-element block of h
            float r = hv;
            const int blk = row >> 5;
#pragma unroll
            for (int t = 0; t < kTerms; ++t) {
              const int e = mx_scale_exp(warp_amax<kTerms>(fabsf(r)));
              const uint32_t c = f32_to_e4m3(r * pow2_exact(-e));
              r -= e4m3_to_f32(c) * pow2_exact(e);
              const size_t drow = (size_t)pos * kTerms + t;
              a.next_aq[drow * a.out_rows + row] = (uint8_t)c;
              if (lane == 0) a.next_asf[drow * (a.out_rows / 32) + blk] = (uint8_t)(e + 127);
            }
          } else {
            a.out_f32[(size_t)pr * a.out_rows + row] = gs;
          }
        }
      }
      if (!kSwiglu && a.comb_w && w.pass == w.npass - 1) {
        // the item is complete: count it for its row tile; the last expert to
        // arrive combines the tile's rows for every token
        __threadfence();         // this thread's y stores, visible at gpu scope
        if (!epi_sync()) break;  // the four epilogue warps' y stores are done
        if (warp == 4 && lane == 0) {
          const int prev = atomicAdd(&a.tile_counter[u.rt], 1);
          const bool last = prev == n_groups - 1;
          if (last) a.tile_counter[u.rt] = 0;  // every contribution is in: ready for the next launch
          *s_last = last ? 1 : 0;
        }
        if (!epi_sync()) break;
        if (*s_last) {
          __threadfence();
          const int H = a.out_rows;
          for (int bb = 0; bb < a.batch; ++bb)
            a.out_bf16[(size_t)bb * H + row] =
                combine_elem(a.residual, a.y_shared, a.comb_w, a.top_k, a.out_f32, H, bb, row);
        }
        if (!epi_sync()) break;  // s_last is read before the next item overwrites it
      }
    }
  }
  // all roles done: free the tensor memory (warp 1 owns it)
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kMxTmemCols) : "memory");
  }
  pdl_launch_dependents();
}

}  // namespace moe
