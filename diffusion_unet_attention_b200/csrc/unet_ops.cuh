// unet_ops.cuh -- the two specialised UNet kernels beside attention.
//
// "Speed Is All You Need" (news summary, section on the three optimisations,
// specialised-kernels paragraphs):
//   * group normalisation, used throughout the UNet: the channels of a feature
//     map are split into groups and each group is normalised on its own; the
//     paper runs it as a single GPU command without intermediate tensors;
//   * GELU (the Gaussian error function and the arithmetic around it) fused
//     with the split and the multiplication that accompany it, one command.
//
// B200 design.  Both are HBM-bound: every input byte is read once and every
// output byte written once, with 16-byte coalesced accesses.
//   group_norm  one thread-block cluster of K CTAs (K = 1 .. 8) per (batch,
//               group).  In NCHW a group's C/G channels x H x W values are
//               contiguous; each CTA of the cluster loads its share of them
//               into registers (up to 8 chunks of 8 values per thread), then
//               the cluster reduces the sum, and then the sum of squared
//               deviations from the mean (two passes over registers, no
//               cancellation): warp shuffles, one shared-memory exchange per
//               CTA, and the CTA totals read across the cluster through
//               distributed shared memory in rank order.  It writes
//               y = (x - mean) * a_c + beta_c with a_c = gamma_c / sqrt(var + eps).
//   geglu       a grid-stride stream over the output: each thread reads 8
//               values of h and the matching 8 of the gate g from the same
//               input row and writes 8 of h * g/2 (1 + erf(g / sqrt 2)), erf
//               by a published rational approximation (gelu_erf).
#pragma once

#include "sm100.cuh"

namespace sdattn {

struct GNParams {
  const void* X;
  void* Y;
  const float* gamma;
  const float* beta;
  int G;          // groups
  int cpg;        // channels per group
  int HW;         // spatial size of a channel (a multiple of 8)
  int gsize;      // values per group, cpg * HW
  int cpc;        // 16-byte chunks of a group per CTA of its cluster
  float eps;
};

constexpr int kGNThreads = 512;   // 128 registers per thread: up to 8 chunks held
constexpr int kGNMaxCluster = 8;

template <bool BF16>
__device__ __forceinline__ void unpack8(const uint4& w, float* f) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t;
    if constexpr (BF16) {
      t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i]));
    } else {
      t = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
    }
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

template <bool BF16>
__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(pack2<BF16>(f[0], f[1]), pack2<BF16>(f[2], f[3]), pack2<BF16>(f[4], f[5]),
                    pack2<BF16>(f[6], f[7]));
}

// Sum over the CTA; every thread gets the total.  `red` holds 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();                  // red may still be read by a previous reduction
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = lane < nw ? red[lane] : 0.f;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
  return t;
}

// Sum over the cluster: every CTA publishes its CTA total in `slot`, and every
// thread adds the cluster's totals in rank order (the same result everywhere).
__device__ __forceinline__ float cluster_sum(float cta_total, float* slot, uint32_t k) {
  if (threadIdx.x == 0) *slot = cta_total;
  cluster_sync();
  float t = 0.f;
  for (uint32_t r = 0; r < k; ++r) t += ld_cluster_f32(slot, r);
  return t;
}

// One group per cluster of K CTAs (K = 1 .. 8, the launch's cluster size); CTA
// r of the cluster holds chunks [r * cpc, (r + 1) * cpc) of the group.
template <int U, bool BF16>
__global__ void __launch_bounds__(kGNThreads) group_norm_kernel(const GNParams p) {
  __shared__ float red[32];
  __shared__ float part[2];
  const uint32_t k = cluster_size(), rank = cluster_rank();
  const int64_t grp = blockIdx.x / k;   // b * G + g
  const int g = static_cast<int>(grp % p.G);
  const uint4* xs = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.X) + grp * p.gsize);
  uint4* ys = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.Y) + grp * p.gsize);
  const int c0 = static_cast<int>(rank) * p.cpc;
  const int c1 = min(p.gsize / 8, c0 + p.cpc);
  const int hw8 = p.HW / 8;   // chunks per channel
  grid_dependency_wait();
  grid_launch_dependents();
  uint4 r[U];
  float sum = 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int i = c0 + threadIdx.x + u * blockDim.x;
    r[u] = i < c1 ? __ldcs(xs + i) : make_uint4(0, 0, 0, 0);   // zeros add nothing to the sum
    float f[8];
    unpack8<BF16>(r[u], f);
#pragma unroll
    for (int e = 0; e < 8; ++e) sum += f[e];
  }
  const float inv_n = 1.f / static_cast<float>(p.gsize);
  const float mean = cluster_sum(block_sum(sum, red), &part[0], k) * inv_n;
  float sq = 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int i = c0 + threadIdx.x + u * blockDim.x;
    if (i < c1) {
      float f[8];
      unpack8<BF16>(r[u], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float dv = f[e] - mean;
        sq = fmaf(dv, dv, sq);
      }
    }
  }
  const float var = cluster_sum(block_sum(sq, red), &part[1], k) * inv_n;
  const float rstd = 1.f / sqrtf(var + p.eps);
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int i = c0 + threadIdx.x + u * blockDim.x;
    if (i < c1) {
      const int c = g * p.cpg + i / hw8;   // a chunk lies inside one channel
      const float a = rstd * __ldg(p.gamma + c);
      const float b = __ldg(p.beta + c);
      float f[8];
      unpack8<BF16>(r[u], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = fmaf(f[e] - mean, a, b);
      __stcs(ys + i, pack8<BF16>(f));
    }
  }
  cluster_sync();   // no CTA leaves while another may still read its partial sums
}

// GELU(g) = g/2 (1 + erf(g / sqrt 2)) with erf from Abramowitz and Stegun,
// Handbook of Mathematical Functions (1964), formula 7.1.26: for x >= 0,
//   erfc(x) ~ t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-x^2),
//   t = 1 / (1 + p x),
// with absolute error at most 1.5e-7; erf(-x) = -erf(x) covers g < 0.  The
// reciprocal and the exponential run on the MUFU unit, the rest is five FMAs.
__device__ __forceinline__ float gelu_erf(float g) {
  constexpr float kP = 0.3275911f, kA1 = 0.254829592f, kA2 = -0.284496736f, kA3 = 1.421413741f,
                  kA4 = -1.453152027f, kA5 = 1.061405429f;
  constexpr float kRsqrt2 = 0.7071067811865476f, kL2E = 1.4426950408889634f;
  const float x = fabsf(g) * kRsqrt2;
  float t;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(kP, x, 1.f)));
  const float poly = t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, kA5, kA4), kA3), kA2), kA1);
  const float erfc_x = poly * ex2_approx(-x * x * kL2E);   // erfc(|g| / sqrt 2)
  // 1 + erf(g / sqrt 2) is 2 - erfc for g >= 0 and erfc for g < 0
  return 0.5f * g * (g >= 0.f ? 2.f - erfc_x : erfc_x);
}

struct GegluParams {
  const void* X;   // [T][2F]
  void* Y;         // [T][F]
  int64_t T;
  int F;           // a multiple of 8
};

template <bool BF16>
__global__ void __launch_bounds__(256) geglu_kernel(const GegluParams p) {
  const int64_t fc = p.F / 8;   // 16-byte chunks per output row
  const int64_t n = p.T * fc;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const uint16_t* X = static_cast<const uint16_t*>(p.X);
  uint16_t* Y = static_cast<uint16_t*>(p.Y);
  grid_dependency_wait();
  grid_launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += 2 * stride) {
    // two chunks per iteration: four 16-byte loads in flight per thread
    uint4 hw[2], gw[2];
    int64_t t[2], c[2];
    bool ok[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t j = i + k * stride;
      ok[k] = j < n;
      t[k] = ok[k] ? j / fc : 0;
      c[k] = ok[k] ? j - t[k] * fc : 0;
      const uint16_t* row = X + t[k] * 2 * p.F + c[k] * 8;
      hw[k] = ok[k] ? __ldcs(reinterpret_cast<const uint4*>(row)) : make_uint4(0, 0, 0, 0);
      gw[k] = ok[k] ? __ldcs(reinterpret_cast<const uint4*>(row + p.F)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (!ok[k]) continue;
      float h[8], g[8], y[8];
      unpack8<BF16>(hw[k], h);
      unpack8<BF16>(gw[k], g);
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = h[e] * gelu_erf(g[e]);
      __stcs(reinterpret_cast<uint4*>(Y + t[k] * p.F + c[k] * 8), pack8<BF16>(y));
    }
  }
}

}  // namespace sdattn
