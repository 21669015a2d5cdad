// Device side of the seeded synthetic-input generator (see synth/__init__.py
// for the recipe).  Inputs only: no part of the MoE layer's arithmetic lives
// here.  Philox4x32-10 follows Salmon et al., "Parallel random numbers: as
// easy as 1, 2, 3" (SC'11).  Every value is produced with integer operations
// and single round-to-nearest fp32 multiplies (__fmul_rn, compiled with
// -fmad=false), so the bits equal the numpy generator's.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

struct U4 { uint32_t x, y, z, w; };

__device__ __forceinline__ U4 philox4x32_10(U4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = U4{hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0};
  }
  return c;
}

// Centred Irwin-Hall(4) sums for elements 2q and 2q+1 of a substream.
__device__ __forceinline__ void ih_pair(uint64_t q, uint32_t sub0, uint32_t sub1,
                                        uint32_t k0, uint32_t k1, int& s_even, int& s_odd) {
  U4 o = philox4x32_10(U4{(uint32_t)q, (uint32_t)(q >> 32), sub0, sub1}, k0, k1);
  s_even = (int)(o.x & 0xFFFF) + (int)(o.x >> 16) + (int)(o.y & 0xFFFF) + (int)(o.y >> 16) - 2 * 65535;
  s_odd  = (int)(o.z & 0xFFFF) + (int)(o.z >> 16) + (int)(o.w & 0xFFFF) + (int)(o.w >> 16) - 2 * 65535;
}

__device__ __forceinline__ uint16_t bf16_rne_bits(float v) {
  const uint32_t u = __float_as_uint(v);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

__global__ void fill_bf16_kernel(uint16_t* out, int64_t n, uint32_t k0, uint32_t k1,
                                 uint32_t sub0, uint32_t sub1, float c) {
  const int64_t npair = (n + 1) / 2;
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < npair;
       q += (int64_t)gridDim.x * blockDim.x) {
    int se, so;
    ih_pair((uint64_t)q, sub0, sub1, k0, k1, se, so);
    out[2 * q] = bf16_rne_bits(__fmul_rn((float)se, c));
    if (2 * q + 1 < n) out[2 * q + 1] = bf16_rne_bits(__fmul_rn((float)so, c));
  }
}

__device__ __forceinline__ int floor_log2_pos(float a) {
  const uint32_t u = __float_as_uint(a);
  const int ef = (int)((u >> 23) & 0xFF);
  if (ef > 0) return ef - 127;
  const uint32_t m = u & 0x7FFFFFu;
  return (32 - __clz(m)) - 150;
}

__device__ __forceinline__ uint32_t e2m1_round(float a) {
  // round to nearest even onto {0, .5, 1, 1.5, 2, 3, 4, 6}, saturating at 6
  if (a <= 0.25f) return 0;
  if (a < 0.75f) return 1;
  if (a <= 1.25f) return 2;
  if (a < 1.75f) return 3;
  if (a <= 2.5f) return 4;
  if (a < 3.5f) return 5;
  if (a <= 5.0f) return 6;
  return 7;
}

// One thread per 32-element block of one row of one expert.
__global__ void fill_mxfp4_kernel(uint8_t* codes, uint8_t* scales, int64_t n_experts,
                                  int64_t rows, int64_t K, uint32_t k0, uint32_t k1,
                                  uint32_t expert0, float c) {
  const int64_t kb = K / 32;
  const int64_t per_expert = rows * kb;
  const int64_t total = n_experts * per_expert;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t slot = t / per_expert;
    const int64_t rb = t - slot * per_expert;        // row * kb + block
    const int64_t row = rb / kb, blk = rb - row * kb;
    const uint64_t n0 = (uint64_t)(row * K + blk * 32);   // first element index in the expert
    float v[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      int se, so;
      ih_pair((n0 >> 1) + i, expert0 + (uint32_t)slot, 0u, k0, k1, se, so);
      v[2 * i] = __fmul_rn((float)se, c);
      v[2 * i + 1] = __fmul_rn((float)so, c);
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    int s = 0;
    if (amax > 0.f) s = floor_log2_pos(amax) - 2 + 127;
    s = s < 0 ? 0 : (s > 254 ? 254 : s);
    const uint32_t eb = (uint32_t)(254 - s);
    const float inv = __uint_as_float(eb > 0 ? (eb << 23) : 0x00400000u);
    uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      uint32_t code = e2m1_round(__fmul_rn(fabsf(v[i]), inv));
      if (__float_as_uint(v[i]) >> 31) code |= 8u;
      w[i >> 3] |= code << (4 * (i & 7));
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + slot * rows * (K / 2) + row * (K / 2) + blk * 16);
    *dst = make_uint4(w[0], w[1], w[2], w[3]);
    scales[slot * rows * kb + row * kb + blk] = (uint8_t)s;
  }
}

int grid_for(int64_t work) {
  int64_t g = (work + 255) / 256;
  if (g > 148 * 64) g = 148 * 64;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

extern "C" int synth_fill_bf16(void* out, int64_t n, uint32_t k0, uint32_t k1, uint32_t sub0,
                               uint32_t sub1, float c, void* stream) {
  if (!out || n <= 0) return 1;
  fill_bf16_kernel<<<grid_for((n + 1) / 2), 256, 0, (cudaStream_t)stream>>>(
      (uint16_t*)out, n, k0, k1, sub0, sub1, c);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

extern "C" int synth_fill_mxfp4(void* codes, void* scales, int64_t n_experts, int64_t rows,
                                int64_t K, uint32_t k0, uint32_t k1, uint32_t expert0, float c,
                                void* stream) {
  if (!codes || !scales || n_experts <= 0 || rows <= 0 || K <= 0 || K % 32) return 1;
  if (((uintptr_t)codes) % 16) return 1;
  fill_mxfp4_kernel<<<grid_for(n_experts * rows * (K / 32)), 256, 0, (cudaStream_t)stream>>>(
      (uint8_t*)codes, (uint8_t*)scales, n_experts, rows, K, k0, k1, expert0, c);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
