// Persistent single-launch batch-1 layer: the whole decode step in one
// cooperative kernel (the pages' persistent kernels under a CUDA graph:
// yeyulingfeng, section 02).  Each CTA (one per SM, all co-resident) runs the
// streams of the chained path back to back, with an in-kernel grid barrier
// only where the data needs one:
//
//   router (+ the bf16 shared expert's gate/up rows; the last CTA finishes
//   the routing)  | grid barrier: routing plan and h_s complete |
//   shared down   -> routed gate/up (no barrier: independent) |
//   grid barrier: h and y_s complete | routed down + combine + residual
//
// so a CTA that finishes the shared expert's rows moves straight on to the
// routed experts, and there are no launch gaps.  The arithmetic of every
// stream is that of the chained kernels, so the results are the same bit for
// bit.  Barrier waits are bounded: one that gives up records MOE_ERR_TIMEOUT.
#pragma once
#include "gemv.cuh"

namespace moe {

struct PersistArgs {
  GemvArgs router, sdown, gu, dnc;
  int has_sdown;
  int* grid_bar;  // zero at launch; counts CTA arrivals over both barriers
  int* err;
};

__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// end of one stream: every thread is done with shared memory, and the
// stream's mbarriers are invalidated before the next stream initialises its
// own in the same bytes
__device__ __forceinline__ void stream_end(unsigned char* smem, int n_stages) {
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    for (int i = 0; i < 2 * n_stages; ++i) mbar_inval(&bars[i]);
  }
  __syncthreads();
}

// all CTAs of the grid meet: arrival `target` of the counter ends the wait
__device__ void grid_barrier(int* bar, int target, int* err) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(bar, 1);
    const long long t0 = clock64();
    while (true) {
      int v;
      asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
      if (v >= target) break;
      if (clock64() - t0 > (1ll << 31)) {
        atomicExch(err, kErrTimeout);
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
  }
  __syncthreads();
}

// KH, KI: the shape-specialised reduction lengths (hidden, intermediate) or
// 0; GU_RPW, DN_RPW: output rows per warp of the routed gate/up and down
// streams (the instances the chained path launches at batch 1)
template <int KH, int KI, int GU_RPW, int DN_RPW>
__global__ void __launch_bounds__(kMaxSplitKWarps * 32 + 32, 1) persistent_b1_kernel(const PersistArgs p) {
  extern __shared__ __align__(128) unsigned char smem[];
  gemv_body<W_BF16, EPI_ROUTER, X_BF16, 1, 2, KH>(p.router, smem);
  stream_end(smem, p.router.n_stages);
  grid_barrier(p.grid_bar, (int)gridDim.x, p.err);
  if (p.has_sdown) {
    gemv_body<W_BF16, EPI_STORE, X_F32, 1, 2, KI>(p.sdown, smem);
    stream_end(smem, p.sdown.n_stages);
  }
  gemv_body<W_MXFP4, EPI_SWIGLU, X_BF16, 1, GU_RPW, KH>(p.gu, smem);
  stream_end(smem, p.gu.n_stages);
  grid_barrier(p.grid_bar, 2 * (int)gridDim.x, p.err);
  gemv_body<W_MXFP4, EPI_DOWN_COMBINE, X_F32, 1, DN_RPW, KI>(p.dnc, smem);
}

}  // namespace moe
