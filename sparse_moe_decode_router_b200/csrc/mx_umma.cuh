// Routed MXFP4 expert projections on the 5th-generation tensor cores
// (tcgen05 block-scaled MMA, kind::mxf4, sm_100a).
//
// The decode-path pages use batch-specialised expert kernels (smzdm, section on
// the four-step rework, first step); here one kernel design serves every batch
// size by leaving all per-weight work to the TMA unit and the tensor cores:
//
//  * weights (A operand, M = 128 rows of one expert per MMA) stay in their
//    packed E2M1 form from HBM to the tensor core: a tiled TMA copies 128 rows
//    x 128 bytes (256 K elements) per stage under the 128-byte swizzle, which
//    is the K-major layout `tcgen05.mma.kind::mxf4` reads.  Shared memory holds
//    exactly the bytes that HBM delivers, and every row segment a copy reads is
//    one full 128-byte line;
//  * the weights' E8M0 block scales (one per row and 32 K elements) are copied
//    once, when the layer is created, into the scale-factor chunk layout that
//    `tcgen05.cp.32x128b.warpx4` takes (128 rows x 4 K-blocks in 512 bytes: row
//    r = r0 + 32*r1 at byte 16*r0 + 4*r1 + block), chunks of one row tile
//    consecutive along K.  A stage's scales are then one 1-D bulk copy;
//  * activations (B operand) are MX values too: each activation row is split
//    into kTerms E2M1 terms (the value, then what the first term missed, ...),
//    each with its own E8M0 scale per 32 elements chosen so the block maximum
//    fits E2M1's 6 without clipping.  A token's terms are separate B columns;
//    the epilogue adds them.  Five terms keep the block's error below about
//    2^-14 of its largest element, finer than the f16 activations of the
//    CUDA-core kernels;
//  * B columns are rows of a buffer ordered like the routing plan's pair list
//    (position q of pair_ids, term t -> row q*kTerms + t), so an expert's
//    tokens are one contiguous run of rows (tiled TMA, 16 rows per copy).  The
//    producer of the terms writes their scales straight into chunks keyed by
//    the first position of the pass that reads them, so B's scales are a bulk
//    copy as well;
//  * the accumulators live in tensor memory (fp32, M = 128 lanes x N
//    columns, two buffers so the epilogue of one item overlaps the MMAs of
//    the next) and are read back with `tcgen05.ld.32x32b`.
//
// Warp roles (192 threads, one CTA per SM): warp 0 issues every copy (TMA
// tiles and bulk scale chunks), warp 1 owns the tensor memory and one of its
// lanes issues the scale copies into tensor memory and the MMAs, warps 2..5
// are the epilogue (warp w reads TMEM lanes 32*(w%4) .. +31).  Every wait is
// bounded: a wait that gives up records MOE_ERR_TIMEOUT in the error word and
// the CTA drains without work.
//
// Epilogues: gate/up -> h = silu(g) * u per (row, token), written as fp32
// (optional) and as the down projection's E2M1 terms; down -> y fp32 per
// (pair, row).  An item is 128 output rows of one active expert (gate/up:
// 128 gate rows and the matching 128 up rows as two MMAs into two
// accumulators), all K, for up to n_max / kTerms tokens per pass; experts
// with more tokens take several passes over the same weights.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kMxRows = 128;        // M: weight rows per MMA (one TMEM lane each)
constexpr int kMxKStage = 256;      // K elements per pipeline stage (one 128-byte swizzle row)
constexpr int kMxKChunk = 128;      // K elements per scale-factor chunk (4 blocks of 32)
constexpr int kMxChunkBytes = 512;  // one chunk: 128 rows (or B columns) x 4 E8M0 bytes
constexpr int kMxATile = kMxRows * kMxKStage / 2;  // one A tile (16 KB, packed)
constexpr int kMxBBox = 16;         // B rows per TMA copy (2 KB)
constexpr int kMxTerms = 5;         // E2M1 terms per activation value
constexpr int kMxNMax = 80;         // B columns per pass: 16 tokens x 5 terms
constexpr int kMxTokMax = kMxNMax / kMxTerms;
constexpr int kMxThreads = 192;
constexpr int kMxTmemCols = 512;
constexpr int kMxAccCols = 2 * kMxNMax;   // per accumulator buffer: gate [0, 80), up [80, 160)
constexpr int kMxSfCol0 = 2 * kMxAccCols; // scale factors after the two buffers (column 320)
constexpr int kMxSfColsGU = 24;           // per stage: gate, up and B, two chunks of 4 columns each
constexpr int kMxSfColsDn = 16;           // per stage: A and B
constexpr int kMxMaxStagesGU = (kMxTmemCols - kMxSfCol0) / kMxSfColsGU;  // 8
constexpr int kMxMaxStagesDn = (kMxTmemCols - kMxSfCol0) / kMxSfColsDn;  // 12
constexpr int kMxMaxStages = kMxMaxStagesDn;
static_assert(kMxNMax % 16 == 0 && kMxNMax <= 128, "B columns: multiples of 16, one scale chunk");
static_assert(kMxSfCol0 + kMxMaxStagesGU * kMxSfColsGU <= kMxTmemCols, "tensor memory");
constexpr int kMxHeaderBytes = 1024;
static_assert(8 * (2 * kMxMaxStages + 6) + 32 <= kMxHeaderBytes, "header");

struct MxArgs {
  const uint8_t* wsf;       // weight scales, chunk layout [E * a_tiles][K/128][512]
  int a_tiles;              // 128-row tiles per expert in the A matrix (2I/128 or H/128)
  int up_tile;              // gate/up: tiles from a gate tile to its up tile (I/128); 0 for down
  int K;                    // reduction length, multiple of 128
  int out_rows;             // output rows per expert (I or H), multiple of 128
  int top_k;
  int n_pairs;              // B * top_k of this call
  int n_experts;
  const int* n_active;
  const int* active;
  const int* offsets;
  const int* pair_ids;
  const uint8_t* bsf;       // activation scales, chunk layout [pass-start position][K/128][512]
  int b_by_token;           // batch 1 gate/up: every pass reads B rows 0.. and chunk 0 (the token's terms)
  int n_max;                // B columns one pass may use (multiple of 16, <= kMxNMax)
  float* out_f32;           // gate/up: h [pair][I] (may be null); down: y [pair][H]
  uint8_t* next_aq;         // gate/up: the down projection's E2M1 terms [pos*next_rpp + t][I/2]
  uint8_t* next_bsf;        // ... and their scale chunks [pos][I/128][512] (pass row i*next_rpp + t)
  int next_rpp;             // rows per pair position of those terms (kTerms, or 8 for the swapped down)
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

// D[tmem] (+)= A[smem] * B[smem], both packed E2M1, K = 64, block-scaled by
// E8M0 factors (two per row and column: 32-element blocks) at sfa and sfb
__device__ __forceinline__ void tc_mma_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                            uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
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

// instruction descriptor, kind::mxf4 block-scaled: A and B E2M1, both
// K-major, E8M0 scale factors, M = 128, N columns, K = 64; the byte of each
// scale word that the MMA starts at (0 or 2: two 32-element blocks per MMA)
// is set per MMA (bits 29-30 for A, 4-5 for B)
__host__ __device__ constexpr uint32_t mx_idesc(int n) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | ((uint32_t)(kMxRows >> 4) << 24);
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
// smallest integer that keeps max|v| * 2^-e <= 6 (E2M1's largest value), then
// each element rounded to the nearest E2M1 value, ties to the even code.
__device__ __forceinline__ int mx_scale_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  const uint32_t u = __float_as_uint(amax);
  const int ef = (int)((u >> 23) & 0xFFu);
  const int E = ef ? ef - 127 : -127;
  const int e = E - 2 + ((u & 0x7FFFFFu) > 0x400000u ? 1 : 0);  // 6 = 1.5 * 2^2
  return max(-127, min(127, e));
}

// 2^e as an exact fp32 for e in [-127, 127] (2^-127 is subnormal)
__device__ __forceinline__ float pow2_exact(int e) {
  return __uint_as_float(e >= -126 ? (uint32_t)(e + 127) << 23 : 0x00400000u);
}

// E2M1 code (sign bit 3) of v, round to nearest even, saturating at 6.  The
// value is converted into both halves of the byte, so the nibble order of
// the packed conversion does not matter.
__device__ __forceinline__ uint32_t f32_to_e2m1(float v) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %1;\n\tmov.b32 %0, {t, t, t, t};\n\t}"
      : "=r"(r)
      : "f"(v));
  return r & 0xFu;
}

// value of an E2M1 code: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
  const uint32_t m = c & 7u;
  const float mag = m < 2u ? 0.5f * (float)m
                           : __uint_as_float(((m >> 1) + 126u) << 23) * (1.0f + 0.5f * (float)(m & 1u));
  return (c & 8u) ? -mag : mag;
}

__device__ __forceinline__ void add4(float4& s, const float4& v) {
  s.x += v.x;
  s.y += v.y;
  s.z += v.z;
  s.w += v.w;
}

__device__ __forceinline__ float warp_amax(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// byte of a B column's scale in its chunk: column n = r0 + 32*r1, K-block kb
__device__ __forceinline__ int sf_chunk_byte(int n, int kb) { return 16 * (n & 31) + 4 * (n >> 5) + kb; }

// x (bf16 [B][K]) -> terms of the gate/up activations: row q*rpp + t of
// aq [.][K/2] (packed E2M1, even element in the low nibble) and the scales
// into the chunks of q's pass, for every pair position q of the token.
// Grid (B, ceil(K/1024)), 256 threads: eight lanes of CTA (b, g) take one
// 32-element block of token b (four elements each; the block's maximum is a
// three-step exchange within the eight lanes), make its terms once and write
// them to the token's top_k positions (found by a scan of pair_ids).
// With by_token (batch 1) row 0 is the token itself, which every position
// reads, and its chunk is chunk 0 (columns = terms).
template <int kTerms>
__global__ void __launch_bounds__(256) mx_x_terms_kernel(const uint16_t* __restrict__ x, int K, int top_k, int n_pairs,
                                                         int n_experts, int tpp, int rpp,
                                                         const int* __restrict__ pair_ids,
                                                         const int* __restrict__ topk_idx,
                                                         const int* __restrict__ offsets, int by_token,
                                                         uint8_t* __restrict__ aq, uint8_t* __restrict__ bsf, int* err) {
  __shared__ int s_q[kMaxTopK], s_p0[kMaxTopK], s_e[kMaxTopK];
  pdl_wait();
  // the next kernel (the gate/up projection) may start its prologue and
  // static-weight copies now; it reads these outputs after its own wait
  pdl_launch_dependents();
  const int b = blockIdx.x, tid = threadIdx.x;
  const int l8 = tid & 7, blk = blockIdx.y * (blockDim.x >> 3) + (tid >> 3);
  const int nq = by_token ? 1 : top_k;
  if (nq < 1 || nq > kMaxTopK || rpp < kTerms || tpp * rpp > kMxRows) {
    if (tid == 0) atomicExch(err, kErrBadPlan);
    pdl_launch_dependents();
    return;
  }
  // written by preceding kernels: coherent loads, all issued before the first wait
  const bool has_blk = blk < (K >> 5);  // uniform over a block's eight lanes
  uint2 xr = make_uint2(0u, 0u);
  if (has_blk) xr = __ldcg(reinterpret_cast<const uint2*>(x + (size_t)b * K + 32 * blk + 4 * l8));
  if (tid < nq) {
    s_q[tid] = by_token ? 0 : -1;
    s_e[tid] = by_token ? 0 : __ldcg(topk_idx + b * top_k + tid);
  }
  __syncthreads();
  if (!by_token) {
    // the token's pairs b*top_k + j sit at the positions q with pair_ids[q] = that pair
    const int pb = b * top_k;
    for (int q = tid; q < n_pairs; q += blockDim.x) {
      const int p = __ldcg(pair_ids + q);
      if (p >= pb && p < pb + top_k) s_q[p - pb] = q;
    }
    __syncthreads();
  }
  bool bad = false;
  if (tid < nq) {
    // the first position of the pass that holds q: passes of tpp tokens from the expert's offset
    const int q = s_q[tid], e = s_e[tid];
    int p0 = 0;
    if (!by_token) {
      p0 = -1;
      if (q >= 0 && e >= 0 && e < n_experts) {
        const int off = __ldcg(offsets + e), end = __ldcg(offsets + e + 1);
        if (off >= 0 && q >= off && q < end) p0 = off + (q - off) / tpp * tpp;
      }
    }
    s_p0[tid] = p0;
    bad = p0 < 0;
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) atomicExch(err, kErrBadPlan);
    pdl_launch_dependents();
    return;
  }
  // every lane takes part in the exchanges (lanes of a block past K hold zeros)
  float v[4] = {__uint_as_float(xr.x << 16), __uint_as_float(xr.x & 0xFFFF0000u), __uint_as_float(xr.y << 16),
                __uint_as_float(xr.y & 0xFFFF0000u)};
  uint32_t w[kTerms];
  int ex[kTerms];
#pragma unroll
  for (int t = 0; t < kTerms; ++t) {
    float am = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
    const int e = mx_scale_exp(am);
    const float down = pow2_exact(-e), up = pow2_exact(e);
    uint32_t pk = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t c = f32_to_e2m1(v[j] * down);
      v[j] -= e2m1_to_f32(c) * up;
      pk |= c << (4 * j);  // element 2m in the low nibble of byte m
    }
    w[t] = pk;
    ex[t] = e;
  }
  if (has_blk) {
    for (int j = 0; j < nq; ++j) {
      const int q = s_q[j], p0 = s_p0[j];
      const int n0 = (q - p0) * rpp;  // this position's first row (column) in its pass's scale chunks
      uint8_t* chunk = bsf + ((size_t)p0 * (K / kMxKChunk) + (blk >> 2)) * kMxChunkBytes;
#pragma unroll
      for (int t = 0; t < kTerms; ++t) {
        *reinterpret_cast<uint16_t*>(aq + ((size_t)q * rpp + t) * (K / 2) + 16 * blk + 2 * l8) = (uint16_t)w[t];
        if (l8 == 0) chunk[sf_chunk_byte(n0 + t, blk & 3)] = (uint8_t)(ex[t] + 127);
      }
    }
  }
  pdl_launch_dependents();
}

// h (fp32 [pair][I], written by the gate/up kernel) -> the down projection's
// E2M1 terms: row q*rpp + t of aq [.][I/2] and the scales into the chunks of
// q's pass (passes of tpp tokens from the expert's offset), for every pair
// position q.  Eight lanes per (position, 32-element block), four elements
// each; grid (ceil(n_pairs * I/32 * 8 / 256)).
template <int kTerms>
__global__ void __launch_bounds__(256) mx_h_terms_kernel(const float* __restrict__ h, int I, int top_k, int n_pairs,
                                                         int n_experts, int tpp, int rpp,
                                                         const int* __restrict__ pair_ids,
                                                         const int* __restrict__ topk_idx,
                                                         const int* __restrict__ offsets, uint8_t* __restrict__ aq,
                                                         uint8_t* __restrict__ bsf, int* err) {
  pdl_wait();
  pdl_launch_dependents();  // as in mx_x_terms_kernel: the down projection's prologue may start
  const int nb = I >> 5;  // blocks per row
  const long long gi = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long gb = gi >> 3;  // (position, block); a block's eight lanes share it
  const int l8 = threadIdx.x & 7;
  const bool on = gb < (long long)n_pairs * nb && rpp >= kTerms && tpp * rpp <= kMxRows;
  int q = 0, blk = 0, p = 0, p0 = -1;
  if (on) {
    q = (int)(gb / nb);
    blk = (int)(gb - (long long)q * nb);
    // the pair at position q, its expert and the first position of q's pass
    p = __ldcg(pair_ids + q);
    const int e = (p >= 0 && p < n_pairs) ? __ldcg(topk_idx + p) : -1;
    if (e >= 0 && e < n_experts) {
      const int off = __ldcg(offsets + e), end = __ldcg(offsets + e + 1);
      if (off >= 0 && q >= off && q < end) p0 = off + (q - off) / tpp * tpp;
    }
    if (p0 < 0 && l8 == 0) atomicExch(err, kErrBadPlan);
  }
  const bool ok = on && p0 >= 0;  // uniform over a block's eight lanes
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  if (ok) {
    const float4 f = __ldcg(reinterpret_cast<const float4*>(h + (size_t)p * I + 32 * blk + 4 * l8));
    v[0] = f.x;
    v[1] = f.y;
    v[2] = f.z;
    v[3] = f.w;
  }
  const int n0 = (q - p0) * rpp;
  uint8_t* chunk = bsf + ((size_t)max(p0, 0) * (I / kMxKChunk) + (blk >> 2)) * kMxChunkBytes;
#pragma unroll
  for (int t = 0; t < kTerms; ++t) {
    float am = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
    const int ex = mx_scale_exp(am);
    const float down = pow2_exact(-ex), up = pow2_exact(ex);
    uint32_t pk = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t c = f32_to_e2m1(v[j] * down);
      v[j] -= e2m1_to_f32(c) * up;
      pk |= c << (4 * j);
    }
    if (ok) {
      *reinterpret_cast<uint16_t*>(aq + ((size_t)q * rpp + t) * (I / 2) + 16 * blk + 2 * l8) = (uint16_t)pk;
      if (l8 == 0) chunk[sf_chunk_byte(n0 + t, blk & 3)] = (uint8_t)(ex + 127);
    }
  }
  pdl_launch_dependents();
}

// Weight scales [n_tiles * 128 rows][K/32] -> chunk layout [n_tiles][K/128][512]
// (layer creation, once per projection)
__global__ void mx_pack_scales_kernel(const uint8_t* __restrict__ sc, long long n_tiles, int K,
                                      uint8_t* __restrict__ out) {
  const int sblk = K / 32, KC = K / kMxKChunk;
  const long long n = n_tiles * KC * 32;  // one thread per (chunk, r0)
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int r0 = (int)(i & 31);
    const long long c = i >> 5;
    const int kc = (int)(c % KC);
    const long long tile = c / KC;
    uint32_t w[4];
#pragma unroll
    for (int r1 = 0; r1 < 4; ++r1) {
      const uint8_t* s = sc + (tile * kMxRows + r0 + 32 * r1) * sblk + 4 * kc;
      w[r1] = (uint32_t)s[0] | ((uint32_t)s[1] << 8) | ((uint32_t)s[2] << 16) | ((uint32_t)s[3] << 24);
    }
    *reinterpret_cast<uint4*>(out + c * kMxChunkBytes + 16 * r0) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ---------------------------------------------------------------------------
// Per-CTA item walk shared by every role: items are (active group, 128-row
// tile), contiguous ranges per CTA; each item runs one pass per n_max /
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
  __device__ MxWalk(const MxArgs& args, long long lo, long long hi_, int nrt)
      : a(args), it(lo), hi(hi_), n_rt(nrt), pass(0), npass(0), e(0), tok0(0), cnt(0) {
    if (it < hi) load();
  }
  __device__ void load() {
    const int g = (int)(it / n_rt);
    e = __ldcg(a.active + g);
    if (e < 0 || e >= a.n_experts) e = 0;
    tok0 = __ldcg(a.offsets + e);
    cnt = __ldcg(a.offsets + e + 1) - tok0;
    if (tok0 < 0 || cnt < 1 || tok0 + cnt > a.n_pairs) { tok0 = 0; cnt = 1; }
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

template <bool kSwiglu, int kTerms>
__global__ void __launch_bounds__(kMxThreads, 1)
    mx_expert_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const MxArgs a) {
  static_assert(kTerms >= 1 && kTerms * kMxTokMax <= kMxNMax, "terms");
  constexpr int kSfCols = kSwiglu ? kMxSfColsGU : kMxSfColsDn;
  constexpr int kMaxNs = kSwiglu ? kMxMaxStagesGU : kMxMaxStagesDn;
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

  const int K = a.K, KC = K / kMxKChunk, KS = (KC + 1) / 2;
  const int ns = a.n_stages;
  if (tid == 0) {
    for (int s = 0; s < kMxMaxStages; ++s) {
      mbar_init(&full_bar[s], 1);    // the TMA thread's expect-tx arrive
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

  int n_groups = __ldcg(a.n_active);
  if (n_groups < 0 || n_groups > a.n_experts) {
    if (tid == 0) atomicExch(a.err, kErrBadPlan);
    n_groups = n_groups < 0 ? 0 : a.n_experts;
  }
  const int n_rt = a.out_rows / kMxRows;
  const long long n_items = (long long)n_groups * n_rt;
  const long long lo = n_items * blockIdx.x / gridDim.x;
  const long long hi = n_items * (blockIdx.x + 1) / gridDim.x;
  const bool plan_ok = ns >= 1 && ns <= kMaxNs && (K % kMxKChunk) == 0 && (a.out_rows % kMxRows) == 0 &&
                       a.n_max >= 16 && a.n_max <= kMxNMax && (a.n_max % 16) == 0 && a.n_max >= kTerms;
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
        const long long tile = (long long)u.e * a.a_tiles + u.rt;  // the gate (or only) 128-row tile
        const int arow = (int)(tile * kMxRows);
        const uint8_t* sfa_g = a.wsf + tile * KC * kMxChunkBytes;
        const uint8_t* sfa_u = a.wsf + (tile + a.up_tile) * KC * kMxChunkBytes;
        const int bpos = a.b_by_token ? 0 : u.tok;  // B rows bpos*kTerms.. and scale chunk bpos
        const uint8_t* sfb = a.bsf + (size_t)bpos * KC * kMxChunkBytes;
        const int nbox = u.n / kMxBBox;
        for (int kt = 0; kt < KS; ++kt) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, *s_abort ? lim_short : lim_long)) {
            atomicExch(a.err, kErrTimeout);
            *s_abort = 1;
            break;
          }
          const int nck = min(2, KC - 2 * kt);  // scale chunks of this stage (1 in a last half stage)
          const uint32_t cb = (uint32_t)(nck * kMxChunkBytes);
          unsigned char* st = ring + (size_t)s * a.stage_bytes;
          const uint32_t sa = smem_addr(st);
          mbar_arrive_expect_tx(&full_bar[s], (kSwiglu ? 2u : 1u) * ((uint32_t)kMxATile + cb) +
                                                  (uint32_t)nbox * (kMxBBox * 128u) + cb);
          tma_load_2d(sa, &tmA, kt * 128, arow, &full_bar[s], pol);
          if (kSwiglu) tma_load_2d(sa + a.off_up, &tmA, kt * 128, arow + a.up_tile * kMxRows, &full_bar[s], pol);
          for (int j = 0; j < nbox; ++j)
            tma_load_2d_nohint(sa + a.off_b + j * kMxBBox * 128, &tmB, kt * 128, bpos * kTerms + kMxBBox * j,
                               &full_bar[s]);
          const size_t ck = (size_t)2 * kt * kMxChunkBytes;
          bulk_g2s(st + a.off_sfa, sfa_g + ck, cb, &full_bar[s], pol);
          if (kSwiglu) bulk_g2s(st + a.off_sfa + 2 * kMxChunkBytes, sfa_u + ck, cb, &full_bar[s], pol);
          bulk_g2s_nohint(st + a.off_sfb, sfb + ck, cb, &full_bar[s]);
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
        const uint32_t d_u = d_g + (uint32_t)kMxNMax;
        const uint32_t idesc = mx_idesc(u.n);
        bool ok = true;
        for (int kt = 0; kt < KS && ok; ++kt) {
          if (!mbar_wait_bounded(&full_bar[s], ph, *s_abort ? lim_short : lim_long)) {
            atomicExch(a.err, kErrTimeout);
            *s_abort = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const int nck = min(2, KC - 2 * kt);
          const uint32_t st = smem_addr(ring + (size_t)s * a.stage_bytes);
          const uint32_t sf = tmem + (uint32_t)(kMxSfCol0 + kSfCols * s);
          const uint32_t sfa_g = sf, sfa_u = sf + 8u, sfb = sf + (kSwiglu ? 16u : 8u);
          for (int c = 0; c < nck; ++c) {
            tc_cp_32x128_x4(sfa_g + 4u * c, desc_sf(st + a.off_sfa + c * kMxChunkBytes));
            if (kSwiglu) tc_cp_32x128_x4(sfa_u + 4u * c, desc_sf(st + a.off_sfa + (2 + c) * kMxChunkBytes));
            tc_cp_32x128_x4(sfb + 4u * c, desc_sf(st + a.off_sfb + c * kMxChunkBytes));
          }
          const uint64_t ad = desc_sw128(st), bd = desc_sw128(st + a.off_b);
          const uint64_t ud = kSwiglu ? desc_sw128(st + a.off_up) : 0ull;
          for (int j = 0; j < 2 * nck; ++j) {
            // MMA j of the stage: +32 bytes in every swizzled row; its two
            // scale bytes start at byte 2*(j%2) of chunk j/2's words
            const uint32_t sb = 2u * (uint32_t)(j & 1), col = 4u * (uint32_t)(j >> 1);
            const uint32_t id = idesc | (sb << 29) | (sb << 4);
            const uint32_t acc = (kt > 0 || j > 0) ? 1u : 0u;
            const uint32_t tag = sb << 30;
            tc_mma_mxf4(d_g, ad + 2u * j, bd + 2u * j, id, (sfa_g + col) | tag, (sfb + col) | tag, acc);
            if (kSwiglu) tc_mma_mxf4(d_u, ud + 2u * j, bd + 2u * j, id, (sfa_u + col) | tag, (sfb + col) | tag, acc);
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
  } else if (plan_ok && warp >= 2) {
    // ------------------------------ epilogue ----------------------------------
    const int q = warp & 3;  // TMEM lane quadrant of this warp
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
    const int KCn = a.out_rows / kMxKChunk;  // gate/up: chunks per row of the down projection's B
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
      // per token: the sum of its kTerms columns, ascending
      float gs[kMxTokMax], us[kMxTokMax];
#pragma unroll
      for (int i = 0; i < kMxTokMax; ++i) gs[i] = us[i] = 0.f;
#pragma unroll
      for (int c = 0; c < kMxNMax / 16; ++c) {
        if (16 * c < u.n) {  // warp-uniform
          float g16[16], u16[16];
          tc_ld16(lane_base + (uint32_t)(b * kMxAccCols + 16 * c), g16);
          if (kSwiglu) tc_ld16(lane_base + (uint32_t)(b * kMxAccCols + kMxNMax + 16 * c), u16);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            gs[(16 * c + i) / kTerms] += g16[i];
            if (kSwiglu) us[(16 * c + i) / kTerms] += u16[i];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
      const int row = u.rt * kMxRows + 32 * q + lane;  // output row of this lane
#pragma unroll
      for (int i = 0; i < kMxTokMax; ++i) {
        if (i < u.ntok) {  // warp-uniform
          const int pos = u.tok + i;
          int pr = __ldcg(a.pair_ids + pos);
          if (pr < 0 || pr >= a.n_pairs) pr = 0;
          if (kSwiglu) {
            const float hv = gs[i] / (1.0f + expf(-gs[i])) * us[i];
            if (a.out_f32) a.out_f32[(size_t)pr * a.out_rows + row] = hv;
            // the down projection's terms: this warp's 32 rows are one
            // 32-element block of h; lanes 8m .. 8m+7 make one 32-bit word
            float r = hv;
            uint8_t* chunk = a.next_bsf + ((size_t)u.tok * KCn + u.rt) * kMxChunkBytes;
#pragma unroll
            for (int t = 0; t < kTerms; ++t) {
              const int e = mx_scale_exp(warp_amax(fabsf(r)));
              const uint32_t c = f32_to_e2m1(r * pow2_exact(-e));
              r -= e2m1_to_f32(c) * pow2_exact(e);
              uint32_t v = c << (4 * (lane & 7));
#pragma unroll
              for (int o = 1; o < 8; o <<= 1) v |= __shfl_xor_sync(0xFFFFFFFFu, v, o);
              const size_t drow = (size_t)pos * a.next_rpp + t;
              if ((lane & 7) == 0)
                *reinterpret_cast<uint32_t*>(a.next_aq + drow * (a.out_rows / 2) + (u.rt * kMxRows + 32 * q) / 2 +
                                             (lane >> 3) * 4) = v;
              if (lane == 0) chunk[sf_chunk_byte(i * a.next_rpp + t, q)] = (uint8_t)(e + 127);
            }
          } else {
            a.out_f32[(size_t)pr * a.out_rows + row] = gs[i];
          }
        }
      }
      if (!kSwiglu && a.comb_w && w.pass == w.npass - 1) {
        // the item is complete: count it for its row tile; the last expert to
        // arrive combines the tile's rows for every token
        if (!epi_sync()) break;  // the four epilogue warps' y stores, performed CTA-wide
        if (warp == 2 && lane == 0) {
          fence_acq_rel_gpu();  // release: ... and at gpu scope, before the count
          const int prev = atomicAdd(&a.tile_counter[u.rt], 1);
          const bool last = prev == n_groups - 1;
          if (last) {
            fence_acq_rel_gpu();  // acquire: the other experts' y rows before the combine's loads
            a.tile_counter[u.rt] = 0;  // every contribution is in: ready for the next launch
          }
          *s_last = last ? 1 : 0;
        }
        if (!epi_sync()) break;
        if (*s_last) {
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

// ---------------------------------------------------------------------------
// Expert projections with the operands swapped: the activation terms are
// the A operand (M = 128 rows: row 8*i + t = token i of the pass, term t;
// rows with t >= kTerms and beyond the pass are padding whose results are
// dropped) and the weights the B operand (N = 256: two 128-row weight tiles
// side by side).  An item is (active expert, 256 weight rows): for gate/up
// the gate tile and the up tile of the same 128 rows of h, for the down
// projection two consecutive 128-row tiles of W_down.  One MMA covers 256
// weight rows x 64 K, so a stage of 32 KB of weights takes 4 MMAs and 6
// scale copies.  The accumulator (128 x 256 fp32) takes half of tensor
// memory, so there is one buffer: the epilogue frees it as soon as it has
// read it.
//
// Work split.  When every expert's tokens fit one pass (batch <= 16) the
// launch's (item, K stage) list is cut into equal stretches, one per CTA
// ("stream-K"): every SM streams the same number of weight bytes.  A
// stretch holds the end of one item, whole items and the start of another;
// the pieces ("parts") of a split item write their term-summed partial sums
// to a workspace slot of their CTA, and the last part to arrive (a counter
// per item) adds the parts in ascending K order and runs the epilogue.
// Larger batches cut the item list into equal runs of whole items (each
// expert's passes of 16 tokens stay in one CTA).
//
// Epilogue.  Warp w reads TMEM lanes 32*(w%4).. = tokens 4*(w%4) .. +3 of
// the pass, 8 lanes (terms) each.  The terms of a token are summed across
// its 8 lanes by recursive halving: after three exchange steps lane l of
// the group holds the sums of columns 32c + 4l .. 32c + 4l + 3 of each
// 32-column chunk c.  Gate/up then forms h = silu(g) * u for those rows and
// splits h into the down projection's E2M1 terms (32-row blocks: the max
// over the group's 8 lanes); the down projection stores y and, for the last
// expert of a 256-row tile, runs the fused combine.
constexpr int kSwRowsPerTok = 8;                    // A rows per token (kTerms used)
constexpr int kSwTokMax = kMxRows / kSwRowsPerTok;  // 16 tokens per pass
constexpr int kSwN = 256;                           // weight rows per MMA (two tiles)
constexpr int kSwSfColsStage = 24;                  // activations 2 chunks x 4 + weights 2 chunks x 8
constexpr int kSwMaxStages = (kMxTmemCols - kSwN) / kSwSfColsStage;  // 10
constexpr int kSwSlotFloats = kSwTokMax * kSwN;     // one workspace slot: a part's sums for a pass
constexpr int kSwGrpMax = 64;                       // groups a CTA keeps in its table
constexpr int kSwPrefBytes = 2 * (kMaxExperts + 8);  // pass prefix (16-bit: at most E + B*k/16 passes)
constexpr int kSwStageOut = 4 * kMxTerms * 64;       // gate/up epilogue warp: 4 tokens x terms x 64 bytes of h
constexpr int kSwTableBytes = kSwPrefBytes + 16 * kSwGrpMax + 4 * kSwStageOut;
static_assert(kMxHeaderBytes >= 8 * (2 * kSwMaxStages + 6) + 32, "header");

struct SwArgs {
  const uint8_t* wsf;       // weight scales, chunk layout [weight tiles][K/128][512]
  int a_tiles;              // 128-row weight tiles per expert (gate/up: 2I/128, down: H/128)
  int tile2;                // tiles from an item's first weight tile to its second (gate/up: I/128, down: 1)
  int K;                    // gate/up H, down I; multiple of 128
  int out_rows;             // gate/up I, down H: rows of the projection's output per pair
  int n_rt;                 // items per expert (gate/up I/128, down H/256)
  int top_k, n_pairs, n_experts;
  const int* n_active;
  const int* active;
  const int* offsets;
  const int* pair_ids;
  const uint8_t* asf;       // activation scale chunks [pass-start position][K/128][512], row m = 8*i + t
  int a_by_token;           // batch-1 gate/up: every position reads row set 0 and chunk 0 (the token)
  int tpp;                  // tokens per pass (<= kSwTokMax)
  int one_pass;             // 1: every expert's tokens fit one pass (batch <= tpp): no pass prefix
  int n_stages, stage_bytes, off_w, off_sfa, off_sfw;  // the activation rows sit at offset 0 of a stage
  float* ws;                // stream-K partial sums: [grid][2 slots][kSwSlotFloats]
  int* item_cnt;            // per unit: pieces arrived, zero between launches
  // gate/up
  float* h;                 // h fp32 [pair][I], or null
  int h_only;               // 1: h fp32 only; its terms come from mx_h_terms_kernel
  uint8_t* next_aq;         // h's E2M1 terms [pos*8 + t][I/2]
  uint8_t* next_bsf;        // their scale chunks [pass-start position][I/128][512], row 8*i + t
  // down
  float* y;                 // [pair][H]
  const float* comb_w;      // fused combine (topk_w [B][k]) or null
  const float* y_shared;
  const uint16_t* residual;
  uint16_t* out_bf16;
  int batch;
  int* tile_counter;        // [H / 256], zero between launches
  const uint8_t* pf_ptr[2];
  long long pf_bytes[2];
  int* err;
};

// (expert, first position, tokens) of active group g, checked against the plan
template <typename Args>
__device__ __forceinline__ int3 sw_group_entry(const Args& a, int g) {
  int e = __ldcg(a.active + g);
  if (e < 0 || e >= a.n_experts) e = 0;
  int tok0 = __ldcg(a.offsets + e);
  int cnt = __ldcg(a.offsets + e + 1) - tok0;
  if (tok0 < 0 || cnt < 1 || tok0 + cnt > a.n_pairs) {
    tok0 = 0;
    cnt = 1;
  }
  return make_int3(e, tok0, cnt);
}

// the group whose passes hold global pass gp: the largest g with pref[g] <= gp
__device__ __forceinline__ int sw_group_of_pass(const uint16_t* pref, int n_groups, int gp) {
  int lo = 0, hi = n_groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pref[mid] <= gp) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// the launch's work list in K-stage units: stage it of unit it / KS
struct SwSplit {
  long long T, G;  // stages of the list; CTAs that take a stretch (the others have none)
  __device__ long long first(long long c) const { return c >= G ? T : c * T / G; }
  // the CTA whose stretch holds stage s: the largest c with first(c) <= s
  __device__ long long owner(long long s) const { return ((s + 1) * G + T - 1) / T - 1; }
};

struct SwRun {
  int e, rt, tok, ntok;  // expert, item within the expert, first position and tokens of the pass
  long long unit;        // unit index in the launch's list
  int k0, nk;            // first K stage and stages of the run
  int part, nparts;      // this run's piece of the unit (stream-K), and the unit's pieces
};

// The launch's units are (active group, pass of tpp tokens, item): unit
// gp*n_rt + rt for the gp-th pass over all groups (a group's passes are
// consecutive).  pref[g] is the first pass of group g (null when every group
// has one pass); a CTA keeps (expert, first position, tokens) of the groups
// its stretch touches in shared memory (grp, from group g_first), so the
// walk makes no global loads.
struct SwWalk {
  const SwArgs& a;
  const SwSplit& sp;
  const uint16_t* pref;
  const int4* grp;
  long long it, hi, unit;
  int KS, n_groups, g_first, n_tab, pass, e, tok0, cnt;
  __device__ SwWalk(const SwArgs& args, const SwSplit& split, const uint16_t* pref_, const int4* grp_, int n_groups_,
                    int g_first_, int n_tab_, long long lo, long long hi_, int ks)
      : a(args), sp(split), pref(pref_), grp(grp_), it(lo), hi(hi_), unit(0), KS(ks), n_groups(n_groups_),
        g_first(g_first_), n_tab(n_tab_), pass(0), e(0), tok0(0), cnt(0) {
    if (it < hi) load();
  }
  __device__ void load() {
    unit = it / KS;
    const int gp = (int)(unit / a.n_rt);
    int g = gp;
    if (pref) g = sw_group_of_pass(pref, n_groups, gp);
    pass = pref ? gp - pref[g] : 0;
    const int j = g - g_first;
    if (j >= 0 && j < n_tab) {
      const int4 t = grp[j];
      e = t.x;
      tok0 = t.y;
      cnt = t.z;
    } else {
      const int3 t = sw_group_entry(a, g);
      e = t.x;
      tok0 = t.y;
      cnt = t.z;
    }
  }
  __device__ bool valid() const { return it < hi; }
  __device__ SwRun run() const {
    SwRun r;
    r.e = e;
    r.unit = unit;
    r.rt = (int)(unit % a.n_rt);
    r.tok = tok0 + pass * a.tpp;
    r.ntok = max(1, min(a.tpp, cnt - pass * a.tpp));
    r.k0 = (int)(it - unit * KS);
    r.nk = (int)(min(hi, (unit + 1) * KS) - it);
    const long long c0 = sp.owner(unit * KS);
    r.part = (int)(sp.owner(it) - c0);
    r.nparts = (int)(sp.owner((unit + 1) * KS - 1) - c0 + 1);
    return r;
  }
  __device__ void next() {
    it = min(hi, (unit + 1) * KS);
    if (it < hi) load();
  }
};

// a pass of more than 4 tokens takes its activation rows as one 128-row copy
// (rows beyond the pass are padding; it needs the whole 16 KB A tile in the
// stage), fewer tokens one 8-row copy each
__device__ __forceinline__ bool sw_act_whole(const SwArgs& a, const SwRun& r) {
  return !a.a_by_token && r.ntok > 4 && a.off_w >= kMxRows * 128;
}
__device__ __forceinline__ uint32_t sw_act_bytes(const SwArgs& a, const SwRun& r) {
  return sw_act_whole(a, r) ? (uint32_t)kMxRows * 128u : (uint32_t)r.ntok * (kSwRowsPerTok * 128u);
}

__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// sum of 32 columns over the 8 lanes of a group (xor 4, 2, 1 exchanges);
// lane l8 of the group returns columns 4*l8 .. 4*l8 + 3
__device__ __forceinline__ float4 group_reduce_scatter(const float (&v)[32], int l8) {
  const bool k2 = (l8 & 4) != 0, k1 = (l8 & 2) != 0, k0 = (l8 & 1) != 0;
  float w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float mine = k2 ? v[16 + i] : v[i], send = k2 ? v[i] : v[16 + i];
    w[i] = mine + __shfl_xor_sync(0xFFFFFFFFu, send, 4);
  }
  float x[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float mine = k1 ? w[8 + i] : w[i], send = k1 ? w[i] : w[8 + i];
    x[i] = mine + __shfl_xor_sync(0xFFFFFFFFu, send, 2);
  }
  float y[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float mine = k0 ? x[4 + i] : x[i], send = k0 ? x[i] : x[4 + i];
    y[i] = mine + __shfl_xor_sync(0xFFFFFFFFu, send, 1);
  }
  return make_float4(y[0], y[1], y[2], y[3]);
}

__device__ __forceinline__ float group_amax(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, 1));
  v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, 2));
  return fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, 4));
}

template <bool kGU, int kTerms>
__global__ void __launch_bounds__(kMxThreads, 1)
    mx_swap_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmA16, const SwArgs a) {
  static_assert(kTerms >= 1 && kTerms <= kSwRowsPerTok, "terms");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t raw = smem_addr(smem_raw);
  unsigned char* hdr = smem_raw;
  unsigned char* ring = smem_raw + (((raw + kMxHeaderBytes + kSwTableBytes + 1023u) & ~1023u) - raw);
  uint16_t* s_pref = reinterpret_cast<uint16_t*>(hdr + kMxHeaderBytes);              // [n_groups + 1]
  int4* s_grp = reinterpret_cast<int4*>(hdr + kMxHeaderBytes + kSwPrefBytes);          // [kSwGrpMax]
  unsigned char* s_out = hdr + kMxHeaderBytes + kSwPrefBytes + 16 * kSwGrpMax;        // [4 warps][kSwStageOut]
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(hdr);
  uint64_t* empty_bar = full_bar + kSwMaxStages;
  uint64_t* acc_full = empty_bar + kSwMaxStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* done_bar = acc_empty + 1;
  uint64_t* epi_bar = done_bar + 1;
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(hdr + 8 * (2 * kSwMaxStages + 6));
  volatile int* s_abort = reinterpret_cast<volatile int*>(hdr + 8 * (2 * kSwMaxStages + 6) + 16);
  volatile int* s_last = s_abort + 1;

  const int K = a.K, KC = K / kMxKChunk, KS = (KC + 1) / 2;
  const int ns = a.n_stages;
  if (tid == 0) {
    for (int s = 0; s < kSwMaxStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_init(done_bar, 1);
    mbar_init(epi_bar, 4);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr((const void*)s_tmem)),
                 "r"(kMxTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmA16);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  // The routing plan is complete before this grid starts: the kernel before
  // (the activation terms, or gate/up for the down projection) waited for its
  // producer before letting this grid launch.  So the plan, the partition and
  // the first stages' weights (static) are read before the wait for the
  // preceding kernel; the activations and every output follow it.
  int n_groups = __ldcg(a.n_active);
  if (n_groups < 0 || n_groups > a.n_experts) {
    if (tid == 0) atomicExch(a.err, kErrBadPlan);
    n_groups = n_groups < 0 ? 0 : a.n_experts;
  }
  // passes of the groups: prefix over the active list (one block scan), unless
  // every group has one pass
  const uint16_t* pref = nullptr;
  int n_gp = n_groups;  // passes over all groups
  if (!a.one_pass && n_groups > 0) {
    const int nt = blockDim.x, per = (n_groups + nt - 1) / nt;
    const int g0 = min(n_groups, tid * per), g1 = min(n_groups, g0 + per);
    int c = 0;
    for (int g = g0; g < g1; ++g) {
      const int np = (sw_group_entry(a, g).z + a.tpp - 1) / a.tpp;
      s_pref[g] = (uint16_t)np;  // this thread's own entries: passes, then their prefix below
      c += np;
    }
    int inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
      if (lane >= o) inc += v;
    }
    int* s_wsum = reinterpret_cast<int*>(s_grp);  // scratch until the table is written
    if (lane == 31) s_wsum[warp] = inc;
    __syncthreads();
    int base = 0;
    for (int w2 = 0; w2 < warp; ++w2) base += s_wsum[w2];
    int run = base + inc - c;
    for (int g = g0; g < g1; ++g) {
      const int np = s_pref[g];
      s_pref[g] = (uint16_t)run;
      run += np;
    }
    if (g0 < n_groups && g1 == n_groups) s_pref[n_groups] = (uint16_t)run;
    __syncthreads();
    n_gp = s_pref[n_groups];
    pref = s_pref;
  }
  const long long n_units = (long long)n_gp * a.n_rt;
  SwSplit sp;
  sp.T = n_units * KS;
  sp.G = max(1ll, min((long long)gridDim.x, sp.T / 2));
  const long long lo = sp.first(blockIdx.x), hi = sp.first(blockIdx.x + 1);
  // the groups of this CTA's stretch, in shared memory
  int g_first = 0, n_tab = 0;
  if (lo < hi) {
    const int gp0 = (int)(lo / KS / a.n_rt), gp1 = (int)((hi - 1) / KS / a.n_rt);
    g_first = pref ? sw_group_of_pass(pref, n_groups, gp0) : gp0;
    const int g_last = pref ? sw_group_of_pass(pref, n_groups, gp1) : gp1;
    n_tab = min(kSwGrpMax, g_last - g_first + 1);
    for (int j = tid; j < n_tab; j += blockDim.x) {
      const int3 t = sw_group_entry(a, g_first + j);
      s_grp[j] = make_int4(t.x, t.y, t.z, 0);
    }
  }
  __syncthreads();
  const bool plan_ok = ns >= 1 && ns <= kSwMaxStages && (K % kMxKChunk) == 0 && a.n_rt >= 1 && a.tpp >= 1 &&
                       a.tpp <= kSwTokMax && a.off_w >= a.tpp * kSwRowsPerTok * 128 &&
                       a.off_w + 2 * kMxATile >= kMxRows * 128;
  if (!plan_ok && tid == 0) atomicExch(a.err, kErrBadPlan);
  const long long lim_long = 1ll << 31, lim_short = 1ll << 20;
  const int step = kGU ? 1 : 2;  // weight tiles per item along the expert's rows

  if (plan_ok && warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      // the first stages' weight tiles and scales before the wait
      const long long npf = min((long long)ns, hi - lo);
      {
        int s = 0;
        long long q = 0;
        for (SwWalk w(a, sp, pref, s_grp, n_groups, g_first, n_tab, lo, hi, KS); w.valid() && q < npf; w.next()) {
          const SwRun r = w.run();
          const long long tile0 = (long long)r.e * a.a_tiles + (long long)step * r.rt;
          const long long tile1 = tile0 + a.tile2;
          for (int kt = r.k0; kt < r.k0 + r.nk && q < npf; ++kt, ++q, ++s) {
            const int nck = min(2, KC - 2 * kt);
            const uint32_t cb = (uint32_t)(nck * kMxChunkBytes);
            unsigned char* st = ring + (size_t)s * a.stage_bytes;
            const uint32_t sa = smem_addr(st);
            mbar_arrive_expect_tx(&full_bar[s], sw_act_bytes(a, r) + 2u * kMxATile + 3u * cb);
            tma_load_2d(sa + a.off_w, &tmW, kt * 128, (int)(tile0 * kMxRows), &full_bar[s], pol);
            tma_load_2d(sa + a.off_w + kMxATile, &tmW, kt * 128, (int)(tile1 * kMxRows), &full_bar[s], pol);
            const size_t ck = (size_t)2 * kt * kMxChunkBytes;
            bulk_g2s(st + a.off_sfw, a.wsf + tile0 * KC * kMxChunkBytes + ck, cb, &full_bar[s], pol);
            bulk_g2s(st + a.off_sfw + 2 * kMxChunkBytes, a.wsf + tile1 * KC * kMxChunkBytes + ck, cb, &full_bar[s],
                     pol);
          }
        }
      }
      pdl_wait();
      int s = 0;
      uint32_t ph = 0;
      long long q = 0;  // stage counter of this CTA
      for (SwWalk w(a, sp, pref, s_grp, n_groups, g_first, n_tab, lo, hi, KS); w.valid() && !*s_abort; w.next()) {
        const SwRun r = w.run();
        const long long tile0 = (long long)r.e * a.a_tiles + (long long)step * r.rt;
        const long long tile1 = tile0 + a.tile2;
        const uint8_t* sfw0 = a.wsf + tile0 * KC * kMxChunkBytes;
        const uint8_t* sfw1 = a.wsf + tile1 * KC * kMxChunkBytes;
        const int arow = a.a_by_token ? 0 : r.tok;
        const uint8_t* sfa = a.asf + (size_t)arow * KC * kMxChunkBytes;
        for (int kt = r.k0; kt < r.k0 + r.nk; ++kt, ++q) {
          const int nck = min(2, KC - 2 * kt);
          const uint32_t cb = (uint32_t)(nck * kMxChunkBytes);
          unsigned char* st = ring + (size_t)s * a.stage_bytes;
          const uint32_t sa = smem_addr(st);
          const size_t ck = (size_t)2 * kt * kMxChunkBytes;
          if (q >= npf) {
            if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, *s_abort ? lim_short : lim_long)) {
              atomicExch(a.err, kErrTimeout);
              *s_abort = 1;
              break;
            }
            mbar_arrive_expect_tx(&full_bar[s], sw_act_bytes(a, r) + 2u * kMxATile + 3u * cb);
            tma_load_2d(sa + a.off_w, &tmW, kt * 128, (int)(tile0 * kMxRows), &full_bar[s], pol);
            tma_load_2d(sa + a.off_w + kMxATile, &tmW, kt * 128, (int)(tile1 * kMxRows), &full_bar[s], pol);
            bulk_g2s(st + a.off_sfw, sfw0 + ck, cb, &full_bar[s], pol);
            bulk_g2s(st + a.off_sfw + 2 * kMxChunkBytes, sfw1 + ck, cb, &full_bar[s], pol);
          }
          // the activation rows and their scales: written by the preceding kernel
          if (sw_act_whole(a, r)) {
            tma_load_2d_nohint(sa, &tmA16, kt * 128, r.tok * kSwRowsPerTok, &full_bar[s]);
          } else {
            for (int i = 0; i < r.ntok; ++i)
              tma_load_2d_nohint(sa + i * kSwRowsPerTok * 128, &tmA, kt * 128,
                                 (a.a_by_token ? 0 : r.tok + i) * kSwRowsPerTok, &full_bar[s]);
          }
          bulk_g2s_nohint(st + a.off_sfa, sfa + ck, cb, &full_bar[s]);
          if (++s == ns) { s = 0; ph ^= 1u; }
        }
      }
      if (*s_abort) {
        for (int q = 0; q < ns; ++q) {
          (void)mbar_wait_bounded(&full_bar[q], 0u, lim_short);
          (void)mbar_wait_bounded(&full_bar[q], 1u, lim_short);
        }
      }
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
    // every copy of this CTA is issued: the next grid may start its prologue
    // on SMs as they free up (it waits for this grid before reading its outputs)
    __syncwarp();
    pdl_launch_dependents();
  } else if (plan_ok && warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    pdl_wait();
    if (lane == 0) {
      int s = 0, uc = 0;
      uint32_t ph = 0;
      const uint32_t idesc = mx_idesc(kSwN);
      for (SwWalk w(a, sp, pref, s_grp, n_groups, g_first, n_tab, lo, hi, KS); w.valid() && !*s_abort; w.next(), ++uc) {
        const SwRun r = w.run();
        if (!mbar_wait_bounded(acc_empty, ((uint32_t)uc & 1u) ^ 1u, lim_long)) {
          atomicExch(a.err, kErrTimeout);
          *s_abort = 1;
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kt = r.k0; kt < r.k0 + r.nk; ++kt) {
          if (!mbar_wait_bounded(&full_bar[s], ph, *s_abort ? lim_short : lim_long)) {
            atomicExch(a.err, kErrTimeout);
            *s_abort = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const int nck = min(2, KC - 2 * kt);
          const uint32_t st = smem_addr(ring + (size_t)s * a.stage_bytes);
          const uint32_t sfa = tmem + (uint32_t)(kSwN + kSwSfColsStage * s), sfw = sfa + 8u;
          for (int c = 0; c < nck; ++c) {
            tc_cp_32x128_x4(sfa + 4u * c, desc_sf(st + a.off_sfa + c * kMxChunkBytes));
            // the first weight tile -> columns 0..3 of the chunk's pair, the second -> 4..7
            tc_cp_32x128_x4(sfw + 8u * c, desc_sf(st + a.off_sfw + c * kMxChunkBytes));
            tc_cp_32x128_x4(sfw + 8u * c + 4u, desc_sf(st + a.off_sfw + (2 + c) * kMxChunkBytes));
          }
          const uint64_t ad = desc_sw128(st), bd = desc_sw128(st + a.off_w);
          for (int j = 0; j < 2 * nck; ++j) {
            const uint32_t sb = 2u * (uint32_t)(j & 1), cj = (uint32_t)(j >> 1);
            const uint32_t id = idesc | (sb << 29) | (sb << 4);
            const uint32_t acc = (kt > r.k0 || j > 0) ? 1u : 0u;
            const uint32_t tag = sb << 30;
            tc_mma_mxf4(tmem, ad + 2u * j, bd + 2u * j, id, (sfa + 4u * cj) | tag, (sfw + 8u * cj) | tag, acc);
          }
          tc_commit(&empty_bar[s]);
          if (++s == ns) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      tc_commit(done_bar);
      if (!mbar_wait_bounded(done_bar, 0u, lim_long)) atomicExch(a.err, kErrTimeout);
    }
    __syncwarp();
  } else if (plan_ok && warp >= 2) {
    // ------------------------------ epilogue ----------------------------------
    pdl_wait();  // outputs (and the workspace) are written after the preceding kernel
    const int q = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    const int l8 = lane & 7, ti = 4 * q + (lane >> 3);  // term (and column quarter), token of the pass
    const int et = (warp - 2) * 32 + lane;              // 0..127 over the four epilogue warps
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
    for (SwWalk w(a, sp, pref, s_grp, n_groups, g_first, n_tab, lo, hi, KS); w.valid(); w.next(), ++uc) {
      const SwRun r = w.run();
      // the lane's pair, loaded while the MMAs run
      int pr = 0;
      if (ti < r.ntok) pr = __ldcg(a.pair_ids + r.tok + ti);
      bool ok = !*s_abort && mbar_wait_bounded(acc_full, (uint32_t)uc & 1u, lim_long);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (lane == 0 && !*s_abort) atomicExch(a.err, kErrTimeout);
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      const bool quad = 4 * q < r.ntok;  // warp-uniform: the quadrant holds tokens of the pass
      const bool mine = ti < r.ntok;
      float4 res[kSwN / 32];
      if (quad) {
        // a rolled loop (the epilogue shares the SM with the other roles'
        // code); the results shift down so every index stays static
        float v[32];
        tc_ld32(lane_base, v);
#pragma unroll 1
        for (int c = 0; c < kSwN / 32; ++c) {
          tc_wait_ld();
          float cur[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) cur[i] = l8 < kTerms ? v[i] : 0.f;
          if (c + 1 < kSwN / 32) tc_ld32(lane_base + (uint32_t)(32 * (c + 1)), v);
          const float4 r4 = group_reduce_scatter(cur, l8);
#pragma unroll
          for (int j = 0; j + 1 < kSwN / 32; ++j) res[j] = res[j + 1];
          res[kSwN / 32 - 1] = r4;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);  // the accumulator is free for the next run
      bool fin = true;
      if (r.nparts > 1) {
        // a piece of a split item: its sums to the CTA's slot, then the count
        const long long c_me = blockIdx.x;
        const int my_slot = (int)(2 * c_me + (sp.first(c_me) >= r.unit * KS ? 0 : 1));
        if (quad && mine) {
          float4* dst = reinterpret_cast<float4*>(a.ws + (size_t)my_slot * kSwSlotFloats + (size_t)ti * kSwN + 4 * l8);
#pragma unroll
          for (int c = 0; c < kSwN / 32; ++c) dst[8 * c] = res[c];
        }
        if (!epi_sync()) break;
        if (warp == 2 && lane == 0) {
          fence_acq_rel_gpu();
          const int prev = atomicAdd(&a.item_cnt[r.unit], 1);
          const bool last = prev == r.nparts - 1;
          if (last) {
            fence_acq_rel_gpu();
            a.item_cnt[r.unit] = 0;
          }
          *s_last = last ? 1 : 0;
        }
        if (!epi_sync()) break;
        fin = *s_last != 0;
        if (fin && quad) {
          // every piece, ascending K order
          const long long c0 = sp.owner(r.unit * KS);
#pragma unroll
          for (int c = 0; c < kSwN / 32; ++c) res[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int p = 0; p < r.nparts; ++p) {
            const long long cp = c0 + p;
            const int slot = (int)(2 * cp + (sp.first(cp) >= r.unit * KS ? 0 : 1));
            const float4* src =
                reinterpret_cast<const float4*>(a.ws + (size_t)slot * kSwSlotFloats + (size_t)ti * kSwN + 4 * l8);
            float4 pv[kSwN / 32];
#pragma unroll
            for (int c = 0; c < kSwN / 32; ++c) pv[c] = mine ? __ldcg(src + 8 * c) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int c = 0; c < kSwN / 32; ++c) add4(res[c], pv[c]);
          }
        }
      }
      if (fin && quad) {
        if (pr < 0 || pr >= a.n_pairs) pr = 0;
        if (kGU && a.h_only) {
          // h rows rt*128 + 32c + 4*l8 .. +3 in fp32 (gate in chunk c, up in chunk c + 4)
          if (mine) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float4 g4 = res[c], u4 = res[c + 4];
              *reinterpret_cast<float4*>(a.h + (size_t)pr * a.out_rows + r.rt * kMxRows + 32 * c + 4 * l8) =
                  make_float4(g4.x / (1.0f + expf(-g4.x)) * u4.x, g4.y / (1.0f + expf(-g4.y)) * u4.y,
                              g4.z / (1.0f + expf(-g4.z)) * u4.z, g4.w / (1.0f + expf(-g4.w)) * u4.w);
            }
          }
        } else if (kGU) {
          // h rows rt*128 + 32c + 4*l8 .. +3: gate in chunk c, up in chunk c + 4.
          // The packed terms go through this warp's staging bytes ([token of
          // the warp][term][64 bytes = the item's 128 rows]) and out as
          // 16-byte stores; the four block scales of a (token, term) are one
          // 32-bit word of the pass's chunk.
          unsigned char* stg = s_out + (warp - 2) * kSwStageOut;
          const int lg = lane >> 3;
          uint32_t sfw[kTerms];
#pragma unroll
          for (int t = 0; t < kTerms; ++t) sfw[t] = 0u;
          // h for the four 32-row blocks, then the terms block by block with the
          // four blocks' (independent) reductions interleaved
          // (lanes of absent tokens hold whatever the padding rows produced,
          // possibly Inf or NaN: zeros keep them off the division's slow path)
          float hv[4][4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 g4 = mine ? res[c] : z4, u4 = mine ? res[c + 4] : z4;
            hv[c][0] = g4.x / (1.0f + expf(-g4.x)) * u4.x;
            hv[c][1] = g4.y / (1.0f + expf(-g4.y)) * u4.y;
            hv[c][2] = g4.z / (1.0f + expf(-g4.z)) * u4.z;
            hv[c][3] = g4.w / (1.0f + expf(-g4.w)) * u4.w;
            if (mine && a.h)
              *reinterpret_cast<float4*>(a.h + (size_t)pr * a.out_rows + r.rt * kMxRows + 32 * c + 4 * l8) =
                  make_float4(hv[c][0], hv[c][1], hv[c][2], hv[c][3]);
          }
#pragma unroll
          for (int t = 0; t < kTerms; ++t) {
            float am[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
              am[c] = fmaxf(fmaxf(fabsf(hv[c][0]), fabsf(hv[c][1])), fmaxf(fabsf(hv[c][2]), fabsf(hv[c][3])));
#pragma unroll
            for (int o = 1; o < 8; o <<= 1)
#pragma unroll
              for (int c = 0; c < 4; ++c) am[c] = fmaxf(am[c], __shfl_xor_sync(0xFFFFFFFFu, am[c], o));
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int e = mx_scale_exp(am[c]);
              uint32_t packed = 0;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t cd = f32_to_e2m1(hv[c][j] * pow2_exact(-e));
                hv[c][j] -= e2m1_to_f32(cd) * pow2_exact(e);
                packed |= cd << (4 * j);
              }
              *reinterpret_cast<uint16_t*>(stg + (lg * kTerms + t) * 64 + 16 * c + 2 * l8) = (uint16_t)packed;
              sfw[t] |= (uint32_t)(e + 127) << (8 * c);
            }
          }
          __syncwarp();
          const int KCn = a.out_rows / kMxKChunk;
          if (mine && l8 == 0) {
            uint8_t* chunk = a.next_bsf + ((size_t)r.tok * KCn + r.rt) * kMxChunkBytes;
#pragma unroll
            for (int t = 0; t < kTerms; ++t)
              *reinterpret_cast<uint32_t*>(chunk + sf_chunk_byte(ti * kSwRowsPerTok + t, 0)) = sfw[t];
          }
          for (int idx = lane; idx < 4 * kTerms * 4; idx += 32) {
            const int tg = idx / (kTerms * 4), t = (idx >> 2) % kTerms, part = idx & 3;
            const int tok_i = 4 * q + tg;  // token of the pass
            if (tok_i < r.ntok) {
              const uint4 v = *reinterpret_cast<const uint4*>(stg + (tg * kTerms + t) * 64 + 16 * part);
              const size_t pos = (size_t)r.tok + tok_i;
              *reinterpret_cast<uint4*>(a.next_aq + (pos * kSwRowsPerTok + t) * (a.out_rows / 2) + r.rt * 64 +
                                        16 * part) = v;
            }
          }
          __syncwarp();  // the staging bytes are rewritten by the next run
        } else if (mine) {
          float4* dst = reinterpret_cast<float4*>(a.y + (size_t)pr * a.out_rows + r.rt * kSwN + 4 * l8);
#pragma unroll
          for (int c = 0; c < kSwN / 32; ++c) dst[8 * c] = res[c];
        }
      }
      if (!kGU && fin && a.comb_w) {
        // the unit is complete: count it for its row tile; the last unit (of
        // all groups and passes) to arrive combines the tile's rows
        if (!epi_sync()) break;  // the four epilogue warps' y stores, performed CTA-wide
        if (warp == 2 && lane == 0) {
          fence_acq_rel_gpu();
          const int prev = atomicAdd(&a.tile_counter[r.rt], 1);
          const bool last = prev == n_gp - 1;
          if (last) {
            fence_acq_rel_gpu();
            a.tile_counter[r.rt] = 0;
          }
          *s_last = last ? 1 : 0;
        }
        if (!epi_sync()) break;
        if (*s_last) {
          const int H = a.out_rows, row0 = r.rt * kSwN;
          for (int bb = 0; bb < a.batch; ++bb) {
            a.out_bf16[(size_t)bb * H + row0 + et] =
                combine_elem(a.residual, a.y_shared, a.comb_w, a.top_k, a.y, H, bb, row0 + et);
            a.out_bf16[(size_t)bb * H + row0 + 128 + et] =
                combine_elem(a.residual, a.y_shared, a.comb_w, a.top_k, a.y, H, bb, row0 + 128 + et);
          }
        }
      }
      if (r.nparts > 1 || (!kGU && fin && a.comb_w))
        if (!epi_sync()) break;  // s_last is rewritten by the next run
    }
  }
  if (!plan_ok) pdl_wait();  // no role ran: still complete only after the preceding grid
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
