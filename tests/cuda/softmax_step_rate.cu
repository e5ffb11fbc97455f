// The flash kernel's softmax step on its own: per iteration each warp loads
// 128 score columns of its tensor-memory lane quarter, applies the library's
// exponential block (flash.cuh, flash_exp_block: MUFU ex2 for some pairs, the
// FMA-pipe polynomial for NPOLY of every 8) with a running max read from
// shared memory, and stores the 64 packed 16-bit weights over the scores.
// No barriers, no MMAs, no row max: the rate the step can reach when nothing
// else in the kernel holds it up, at 1, 2 or 3 warps per SM scheduler.
#include "flash.cuh"

namespace {

template <int NPOLY>
__global__ void __launch_bounds__(384, 1) softmax_step_kernel(unsigned long long* cycles, const uint32_t* scores,
                                                              int iters) {
  __shared__ uint32_t taddr;
  __shared__ float running_max[2];
  constexpr int BN = 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    sdattn::tmem_alloc(&taddr, 512);
    sdattn::tmem_relinquish();
  }
  if (threadIdx.x < 2) running_max[threadIdx.x] = 1.0f + threadIdx.x;
  sdattn::tc_fence_before();
  __syncthreads();
  sdattn::tc_fence_after();
  // warp w: lane quarter w % 4, columns 128 (w / 4) .. + 127 (at most 12 warps: 384 columns)
  const uint32_t base = taddr + (static_cast<uint32_t>((warp & 3) * 32) << 16) + (warp >> 2) * 128;
  {
    uint32_t v[64];
    for (int half = 0; half < 2; ++half) {
#pragma unroll
      for (int k = 0; k < 64; ++k) v[k] = scores[(threadIdx.x * BN + half * 64 + k) & 4095];
      sdattn::tmem_st_x64(base + half * 64, v);
    }
    sdattn::tmem_wait_st();
  }
  const uint64_t c2 = sdattn::f2_pack(0.228f, 0.228f);
  __syncthreads();
  const unsigned long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
    const float m = *reinterpret_cast<volatile float*>(&running_max[it & 1]);
    uint32_t v[BN];
    sdattn::tmem_ld_x128(base, v);
    sdattn::tmem_wait_ld();
    sdattn::reg_fence<BN>(v);
    uint32_t pk[BN / 2];
    sdattn::flash_exp_block<BN, false, NPOLY>(v, c2, sdattn::f2_pack(-m, -m), pk);
    sdattn::tmem_st_x64(base, pk);
    sdattn::tmem_wait_st();
  }
  const unsigned long long t1 = clock64();
  if (lane == 0) cycles[blockIdx.x * 12 + warp] = t1 - t0;
  sdattn::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    sdattn::tc_fence_after();
    sdattn::tmem_dealloc(taddr, 512);
  }
}

template <int NPOLY>
int run(int blocks, int warps, int iters, unsigned long long* cycles, const uint32_t* scores) {
  // 120 KB of dynamic shared memory keeps one CTA per SM, so the 512-column
  // allocation never waits for another CTA's
  auto kern = softmax_step_kernel<NPOLY>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 120 * 1024) != cudaSuccess) return 2;
  kern<<<blocks, warps * 32, 120 * 1024>>>(cycles, scores, iters);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

}  // namespace

// cycles: device buffer of blocks * 12 counters (per warp, clock cycles over
// all iterations); scores: 4096 fp32 values on the device.  warps in 1..12.
extern "C" int softmax_step_rate_run(int npoly, int blocks, int warps, int iters, unsigned long long* cycles,
                                     const uint32_t* scores) {
  if (warps < 1 || warps > 12 || blocks < 1 || iters < 1) return 1;
  switch (npoly) {
    case 0: return run<0>(blocks, warps, iters, cycles, scores);
    case 3: return run<3>(blocks, warps, iters, cycles, scores);
    case 4: return run<4>(blocks, warps, iters, cycles, scores);
    default: return 1;
  }
}
