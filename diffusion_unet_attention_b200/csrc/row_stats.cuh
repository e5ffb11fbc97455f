// row_stats.cuh -- the stand-alone form of the partially fused softmax's
// reduction: a kernel that reads a materialised score matrix A and reduces
// each row to (L_i, S_i) = (max_j A_ij, sum_j exp(A_ij - L_i)).
//
// "Speed Is All You Need" (news summary, section on the three optimisations,
// partially fused softmax paragraph): a GPU shader maps the large matrix A to
// the vectors L and S; because that map has far fewer outputs than inputs, A
// is grouped into blocks, each block is reduced, and the partial results are
// reduced again to the final ones, each part in a single GPU command.
//
// B200 design.  Memory-bound: A is read once with coalesced 16-byte loads.
//   - one warp reduces one (row, column split) item; lane l reads 16-byte
//     groups l, l + 32, l + 64, ... of the row segment, eight loads in flight,
//     so each warp instruction moves 512 contiguous bytes;
//   - a lane keeps a running (m, s) pair, updated once per eight loaded
//     groups (the group max first, then sum of exp(a - m) on the MUFU unit);
//   - the 32 lane pairs merge by warp shuffles (butterfly, five steps);
//   - when a row is split over several warps (few rows, long rows), each
//     split writes its pair to the workspace and bumps the row's arrival
//     counter; the split that arrives last merges all of them in split order
//     and writes LS, then clears what it read, so a completed call leaves the
//     workspace zero.  No warp ever waits for another.
// The work is one launch; the grid is persistent (a multiple of the SM count)
// and its warps stride over the items.
#pragma once

#include "sm100.cuh"

namespace sdattn {

struct RowStatsParams {
  const void* A;
  int64_t lda;        // row stride of A in elements (16-byte rows)
  int64_t rows;       // B * H * N
  int M;              // valid columns per row
  int nsplit;         // column splits per row
  int split_cols;     // columns per split (a multiple of 8)
  float* LS;          // [rows][2]
  uint32_t* tickets;  // [rows] when nsplit > 1
  float2* part;       // [rows][nsplit] when nsplit > 1
};

constexpr int kRowStatsWarps = 16;   // warps per CTA
constexpr int kRowStatsUnroll = 8;   // 16-byte loads in flight per lane

// (m, s) of the union of two column sets, natural-base sums, base-2 exponent.
__device__ __forceinline__ void rs_merge(float& m, float& s, float m2, float s2) {
  constexpr float L2E = 1.4426950408889634f;
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;   // both empty
  s = s * ex2_approx((m - mm) * L2E) + s2 * ex2_approx((m2 - mm) * L2E);
  m = mm;
}

// 8 values of A from one 16-byte group: fp32 (two groups per call, 4 + 4) or fp16 (one group).
template <typename AT>
struct RowGroup;

template <>
struct RowGroup<float> {
  static constexpr int PER = 4;   // elements per 16-byte group
};

template <>
struct RowGroup<__half> {
  static constexpr int PER = 8;
};

template <typename AT>
__device__ __forceinline__ void unpack_group(const uint4& g, float* out) {
  if constexpr (sizeof(AT) == 4) {
    out[0] = __uint_as_float(g.x);
    out[1] = __uint_as_float(g.y);
    out[2] = __uint_as_float(g.z);
    out[3] = __uint_as_float(g.w);
  } else {
    const uint32_t w[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
}

template <typename AT>
__global__ void __launch_bounds__(kRowStatsWarps * 32)
    row_stats_kernel(const RowStatsParams p) {
  constexpr float L2E = 1.4426950408889634f;
  constexpr int PER = RowGroup<AT>::PER;
  constexpr int U = kRowStatsUnroll;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = static_cast<int64_t>(blockIdx.x) * kRowStatsWarps + (threadIdx.x >> 5);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kRowStatsWarps;
  const int64_t items = p.rows * p.nsplit;
  grid_dependency_wait();
  grid_launch_dependents();
  for (int64_t it = warp0; it < items; it += nwarps) {
    const int64_t row = it / p.nsplit;
    const int sp = static_cast<int>(it - row * p.nsplit);
    const int c0 = sp * p.split_cols;
    const int c1 = min(p.M, c0 + p.split_cols);
    const uint8_t* base = reinterpret_cast<const uint8_t*>(p.A) + (row * p.lda + c0) * sizeof(AT);
    const int ngroups = (c1 - c0 + PER - 1) / PER;   // 16-byte groups holding valid columns
    float m = -INFINITY, s = 0.f;
    for (int g0 = 0; g0 < ngroups; g0 += 32 * U) {
      uint4 g[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int gi = g0 + u * 32 + lane;
        g[u] = gi < ngroups ? __ldcs(reinterpret_cast<const uint4*>(base) + gi) : make_uint4(0, 0, 0, 0);
      }
      float v[U * PER];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        unpack_group<AT>(g[u], v + u * PER);
        const int col = c0 + (g0 + u * 32 + lane) * PER;   // column of v[u * PER]
#pragma unroll
        for (int e = 0; e < PER; ++e)
          if (col + e >= c1) v[u * PER + e] = -INFINITY;
      }
      // batch max, then rescale the running sum once, then the exponentials
      float bm = v[0];
#pragma unroll
      for (int i = 1; i < U * PER; ++i) bm = fmaxf(bm, v[i]);
      if (bm > m) {
        s = (m == -INFINITY) ? 0.f : s * ex2_approx((m - bm) * L2E);
        m = bm;
      }
      if (m != -INFINITY) {
        const float nm = -m * L2E;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < U * PER; ++i) acc[i & 3] += ex2_approx(fmaf(v[i], L2E, nm));
        s += (acc[0] + acc[1]) + (acc[2] + acc[3]);
      }
    }
    // butterfly merge of the 32 lane pairs: every lane ends with the warp's pair
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
      const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
      rs_merge(m, s, m2, s2);
    }
    if (p.nsplit == 1) {
      if (lane == 0) *reinterpret_cast<float2*>(p.LS + 2 * row) = make_float2(m, s);
      continue;
    }
    // split combine: publish this split's pair, the last split to arrive merges
    uint32_t last = 0;
    if (lane == 0) {
      __stcg(p.part + row * p.nsplit + sp, make_float2(m, s));
      last = atomic_add_acq_rel_gpu(p.tickets + row, 1u) == static_cast<uint32_t>(p.nsplit - 1) ? 1u : 0u;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) continue;
    float mm = -INFINITY, ss = 0.f;
    for (int k = lane; k < p.nsplit; k += 32) {
      const float2 q = __ldcg(p.part + row * p.nsplit + k);
      rs_merge(mm, ss, q.x, q.y);
      __stcg(p.part + row * p.nsplit + k, make_float2(0.f, 0.f));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, mm, off);
      const float s2 = __shfl_xor_sync(0xffffffffu, ss, off);
      rs_merge(mm, ss, m2, s2);
    }
    if (lane == 0) {
      *reinterpret_cast<float2*>(p.LS + 2 * row) = make_float2(mm, ss);
      p.tickets[row] = 0u;
    }
  }
}

}  // namespace sdattn
