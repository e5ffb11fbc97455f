// winograd.cuh -- the UNet's 3x3 convolution (stride 1, zero padding 1) by
// Winograd's minimal filtering F(4x4, 3x3): 4x4 output tiles from 6x6 input
// tiles, 36 multiplications per tile and channel pair instead of 144.
//
// "Speed Is All You Need" (news summary, section on the three optimisations,
// Winograd paragraphs): the 3x3 convolutions run as Winograd convolutions, a
// 4x4 tile being named the best balance of compute efficiency and memory.
// The transforms are those of Lavin and Gray, "Fast Algorithms for
// Convolutional Neural Networks" (2016), F(4, 3) with interpolation points
// 0, 1, -1, 2, -2 and infinity, applied along both axes:
//   Y = A^T [ (G g G^T) (.) (B^T d B) ] A       (.) elementwise, per 6x6 tile
// summed over input channels, which on B200 is a batched matrix product: for
// each of the 36 transformed positions xi,
//   M[xi] (K x T) = U[xi] (K x C) V[xi]^T (C x T)
// over T = N * ceil(H/4) * ceil(W/4) tiles, run on the tensor cores.
//
// Four kernels, layouts of the caller's workspace:
//   wino_filter_kernel  w [K][C][3][3]  -> U [36][K][C]   (once per filter; dtype)
//   wino_input_kernel   x [N][C][H][W]  -> V [36][T][C]   (dtype)
//   wino_gemm_kernel    U, V            -> M [36][K][ldm] (fp32, ldm = T rounded up to 4)
//   wino_output_kernel  M, bias         -> y [N][K][H][W] (dtype)
// The transforms run in fp32; U and V are rounded to the input's 16-bit type
// (the tensor cores' operands), M and the output transform stay fp32.
#pragma once

#include "sm100.cuh"

namespace sdattn {

struct WinoGeom {
  int N, C, K, H, W;
  int TH, TW;   // tiles down and across: ceil(H / 4), ceil(W / 4)
  int T;        // N * TH * TW
  int ldm;      // row stride of M in floats (T rounded up to 4)
  int CB;       // input kernel: channels per CTA
};

template <bool BF16>
__device__ __forceinline__ float ld16(const uint16_t* p) {
  const uint16_t b = *p;
  if constexpr (BF16) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  } else {
    return __half2float(__ushort_as_half(b));
  }
}

template <bool BF16>
__device__ __forceinline__ uint16_t to16(float f) {
  if constexpr (BF16) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
  } else {
    return __half_as_ushort(__float2half_rn(f));
  }
}

// u = G g for one column of a 3x3 filter (stride s), G the 6x3 filter transform.
__device__ __forceinline__ void wino_g3(const float* g, int s, float* u, int us) {
  const float g0 = g[0], g1 = g[s], g2 = g[2 * s];
  constexpr float k6 = 1.f / 6.f, k12 = 1.f / 12.f, k24 = 1.f / 24.f;
  u[0] = 0.25f * g0;
  u[us] = -k6 * (g0 + g1 + g2);
  u[2 * us] = -k6 * (g0 - g1 + g2);
  u[3 * us] = fmaf(k24, g0, fmaf(k12, g1, k6 * g2));
  u[4 * us] = fmaf(k24, g0, fmaf(-k12, g1, k6 * g2));
  u[5 * us] = g2;
}

// y = A^T m for one column of a 6x6 product tile (stride s), A^T the 4x6 output transform.
__device__ __forceinline__ void wino_at4(const float* m, int s, float* y, int ys) {
  const float m0 = m[0], m1 = m[s], m2 = m[2 * s], m3 = m[3 * s], m4 = m[4 * s], m5 = m[5 * s];
  const float a = m1 + m2, b = m1 - m2, c = m3 + m4, e = m3 - m4;
  y[0] = m0 + a + c;
  y[ys] = fmaf(2.f, e, b);
  y[2 * ys] = fmaf(4.f, c, a);
  y[3 * ys] = fmaf(8.f, e, b) + m5;
}

// One thread per (k, c): U[xi][k][c] = (G g G^T)[xi], xi = 6 a + b.
template <bool BF16>
__global__ void __launch_bounds__(256) wino_filter_kernel(const uint16_t* __restrict__ w, uint16_t* __restrict__ U,
                                                          int K, int C) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;   // k * C + c
  if (i >= static_cast<int64_t>(K) * C) return;
  float g[9], t[18], u[36];
#pragma unroll
  for (int j = 0; j < 9; ++j) g[j] = ld16<BF16>(w + i * 9 + j);
#pragma unroll
  for (int col = 0; col < 3; ++col) wino_g3(g + col, 3, t + col, 3);    // t = G g      (6 x 3)
#pragma unroll
  for (int row = 0; row < 6; ++row) wino_g3(t + 3 * row, 1, u + 6 * row, 1);   // u = t G^T (6 x 6)
  const int64_t plane = static_cast<int64_t>(K) * C;
#pragma unroll
  for (int xi = 0; xi < 36; ++xi) U[xi * plane + i] = to16<BF16>(u[xi]);
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// t = B^T d for one column of a 6x6 input tile (stride s between its entries),
// B^T the 6x6 input transform, on packed pairs: two channels at once, one
// f32x2 instruction per step.
__device__ __forceinline__ void wino_bt6x2(const uint64_t* d, int s, uint64_t* t, int ts) {
  const uint64_t d0 = d[0], d1 = d[s], d2 = d[2 * s], d3 = d[3 * s], d4 = d[4 * s], d5 = d[5 * s];
  const uint64_t c4 = f2_pack(4.f, 4.f), cm4 = f2_pack(-4.f, -4.f), cm5 = f2_pack(-5.f, -5.f);
  const uint64_t c2 = f2_pack(2.f, 2.f);
  const uint64_t d42 = f2_sub(d4, d2);
  t[0] = f2_fma(c4, d0, f2_fma(cm5, d2, d4));
  t[ts] = f2_fma(cm4, f2_add(d1, d2), f2_add(d3, d4));
  t[2 * ts] = f2_fma(c4, f2_sub(d1, d2), f2_sub(d4, d3));
  t[3 * ts] = f2_fma(c2, f2_sub(d3, d1), d42);
  t[4 * ts] = f2_fma(c2, f2_sub(d1, d3), d42);
  t[5 * ts] = f2_fma(c4, d1, f2_fma(cm5, d3, d5));
}

template <bool BF16>
__device__ __forceinline__ uint64_t unpack_pair(uint32_t v) {
  float2 f;
  if constexpr (BF16) {
    f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v));
  } else {
    f = __half22float2(*reinterpret_cast<const __half2*>(&v));
  }
  return f2_pack(f.x, f.y);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack_pair(uint64_t v) {
  float lo, hi;
  f2_unpack(v, lo, hi);
  return pack2<BF16>(lo, hi);
}

// Shared-memory rows of the input kernel, per pair of channels (c, c + 1)
// interleaved as 32-bit words (low half c): six input rows, each holding x's
// W columns from word 8 on and zeros around them (word 7 is w = -1); a pair's
// block is padded to an odd number of words so that lanes on consecutive
// pairs read distinct banks.
struct WinoRows {
  int Wp;   // words per row: 4 TW + 16
  int PS;   // words per channel pair: 6 Wp + 1
  __host__ __device__ static WinoRows of(int TW) {
    WinoRows r;
    r.Wp = 4 * TW + 16;
    r.PS = 6 * r.Wp + 1;
    return r;
  }
};

// A CTA takes one row of tiles (batch n, tile row th) and CB channels (an
// even number): the six input rows of each channel pair are staged in shared
// memory with the zero border (16-byte loads of both channels' rows, two of
// each in flight per thread, interleaved into words, when W is a multiple of
// 8), then each thread transforms one (channel pair, tile) at a time on packed
// fp32 pairs, consecutive threads taking consecutive pairs so that V's rows
// are written contiguously, 4 bytes (two channels) per thread.
template <bool BF16>
__global__ void __launch_bounds__(256) wino_input_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ V,
                                                         const WinoGeom g) {
  extern __shared__ __align__(16) uint32_t sw[];   // [CB / 2][PS]
  const WinoRows L = WinoRows::of(g.TW);
  const int n = blockIdx.x / g.TH, th = blockIdx.x % g.TH;
  const int c0 = blockIdx.y * g.CB;
  const int P = g.CB / 2;
  grid_dependency_wait();
  grid_launch_dependents();
  // zeros: the border words of every row (0..7 and W+8 .. Wp-1), and whole
  // rows outside 0..H-1 or past the last channel
  for (int r = threadIdx.x; r < P * 6; r += blockDim.x) {
    const int pp = r / 6, i = r - pp * 6;
    const int h = th * 4 - 1 + i, c = c0 + 2 * pp;
    uint32_t* row = sw + pp * L.PS + i * L.Wp;
    if (h >= 0 && h < g.H && c < g.C) {
      for (int j = 0; j < 8; ++j) row[j] = 0u;
      for (int j = 8 + g.W; j < L.Wp; ++j) row[j] = 0u;
    } else {
      for (int j = 0; j < L.Wp; ++j) row[j] = 0u;
    }
  }
  const uint16_t* xn = x + static_cast<int64_t>(n) * g.C * g.H * g.W;
  if ((g.W & 7) == 0) {
    const int chunks = g.W / 8;                  // 16-byte pieces per row
    const int items = P * 6 * chunks;
    for (int base = threadIdx.x; base < items; base += 2 * blockDim.x) {
      uint4 ra[2], rb[2];
      int dst[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int it = base + u * blockDim.x;
        const int pp = it / (6 * chunks), rem = it - pp * 6 * chunks, i = rem / chunks, ch = rem - i * chunks;
        const int c = c0 + 2 * pp, h = th * 4 - 1 + i;
        const bool ok = it < items && c < g.C && h >= 0 && h < g.H;   // C is even: c + 1 < C too
        dst[u] = ok ? pp * L.PS + i * L.Wp + 8 + ch * 8 : -1;
        const uint4* ra_p = reinterpret_cast<const uint4*>(xn + (static_cast<int64_t>(c) * g.H + h) * g.W) + ch;
        const uint4* rb_p = reinterpret_cast<const uint4*>(xn + (static_cast<int64_t>(c + 1) * g.H + h) * g.W) + ch;
        ra[u] = ok ? __ldcs(ra_p) : make_uint4(0, 0, 0, 0);
        rb[u] = ok ? __ldcs(rb_p) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (dst[u] < 0) continue;
        const uint32_t a[4] = {ra[u].x, ra[u].y, ra[u].z, ra[u].w}, b[4] = {rb[u].x, rb[u].y, rb[u].z, rb[u].w};
        uint32_t* d = sw + dst[u];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          d[2 * k] = __byte_perm(a[k], b[k], 0x5410);       // (c, c+1) of column 2k
          d[2 * k + 1] = __byte_perm(a[k], b[k], 0x7632);   // (c, c+1) of column 2k + 1
        }
      }
    }
  } else {
    const int items = P * 6 * g.W;
    for (int base = threadIdx.x; base < items; base += 4 * blockDim.x) {
      uint32_t r[4];
      int dst[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int it = base + u * blockDim.x;
        const int pp = it / (6 * g.W), rem = it - pp * 6 * g.W, i = rem / g.W, wc = rem - i * g.W;
        const int c = c0 + 2 * pp, h = th * 4 - 1 + i;
        const bool ok = it < items && c < g.C && h >= 0 && h < g.H;
        dst[u] = ok ? pp * L.PS + i * L.Wp + 8 + wc : -1;
        r[u] = ok ? uint32_t(xn[(static_cast<int64_t>(c) * g.H + h) * g.W + wc]) |
                        (uint32_t(xn[(static_cast<int64_t>(c + 1) * g.H + h) * g.W + wc]) << 16)
                  : 0u;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (dst[u] >= 0) sw[dst[u]] = r[u];
    }
  }
  __syncthreads();
  const int64_t plane = static_cast<int64_t>(g.T) * g.C;
  const int64_t tile0 = (static_cast<int64_t>(n) * g.TH + th) * g.TW;
  for (int it = threadIdx.x; it < P * g.TW; it += blockDim.x) {
    const int pp = it % P, tw = it / P;
    const int c = c0 + 2 * pp;
    if (c >= g.C) continue;
    uint64_t d[36], t[36];
    const uint32_t* src = sw + pp * L.PS + 7 + tw * 4;   // word 7 is w = -1
#pragma unroll
    for (int i = 0; i < 6; ++i)
#pragma unroll
      for (int j = 0; j < 6; ++j) d[6 * i + j] = unpack_pair<BF16>(src[i * L.Wp + j]);
#pragma unroll
    for (int col = 0; col < 6; ++col) wino_bt6x2(d + col, 6, t + col, 6);     // t = B^T d
#pragma unroll
    for (int row = 0; row < 6; ++row) wino_bt6x2(t + 6 * row, 1, d + 6 * row, 1);   // v = t B (into d)
    uint32_t* out = reinterpret_cast<uint32_t*>(V + (tile0 + tw) * g.C + c);
#pragma unroll
    for (int xi = 0; xi < 36; ++xi) out[xi * (plane / 2)] = pack_pair<BF16>(d[xi]);
  }
}

// One thread per (k, tile), consecutive threads taking consecutive tiles:
// y = A^T m A + bias over the tile's 36 products, stored where inside H x W.
template <bool BF16>
__global__ void __launch_bounds__(256) wino_output_kernel(const float* __restrict__ M, const float* __restrict__ bias,
                                                          uint16_t* __restrict__ y, const WinoGeom g) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(g.K) * g.T) return;
  const int k = static_cast<int>(i / g.T), tile = static_cast<int>(i - static_cast<int64_t>(k) * g.T);
  const int64_t plane = static_cast<int64_t>(g.K) * g.ldm;
  float m[36], s[24], o[16];
#pragma unroll
  for (int xi = 0; xi < 36; ++xi) m[xi] = __ldcs(M + xi * plane + static_cast<int64_t>(k) * g.ldm + tile);
#pragma unroll
  for (int col = 0; col < 6; ++col) wino_at4(m + col, 6, s + col, 6);      // s = A^T m   (4 x 6)
#pragma unroll
  for (int row = 0; row < 4; ++row) wino_at4(s + 6 * row, 1, o + 4 * row, 1);   // o = s A  (4 x 4)
  const float b = bias != nullptr ? __ldg(bias + k) : 0.f;
  const int tpi = g.TH * g.TW;
  const int n = tile / tpi, rem = tile - n * tpi, th = rem / g.TW, tw = rem - th * g.TW;
  uint16_t* out = y + (static_cast<int64_t>(n) * g.K + k) * g.H * g.W;
  const bool whole = (g.W & 3) == 0;   // a tile row is 8 aligned bytes of y
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int h = th * 4 + p;
    if (h >= g.H) break;
    uint16_t* orow = out + static_cast<int64_t>(h) * g.W + tw * 4;
    if (whole) {
      const uint32_t lo = uint32_t(to16<BF16>(o[4 * p] + b)) | (uint32_t(to16<BF16>(o[4 * p + 1] + b)) << 16);
      const uint32_t hi = uint32_t(to16<BF16>(o[4 * p + 2] + b)) | (uint32_t(to16<BF16>(o[4 * p + 3] + b)) << 16);
      *reinterpret_cast<uint2*>(orow) = make_uint2(lo, hi);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (tw * 4 + q < g.W) orow[q] = to16<BF16>(o[4 * p + q] + b);
    }
  }
}

// ---------------------------------------------------------------------------
// Batched product over the 36 transformed positions:
//   M[xi][k][t] = sum_c U[xi][k][c] V[xi][t][c]
// A unit is (xi, block of 128 k, block of 128 t), both operands K-major
// (c contiguous) 128-row x 64-column tiles, 128-byte swizzled, no multicast.
// Roles: warp 0 TMA (a ring of U/V stage pairs), warp 1 MMA (tcgen05 SS,
// 128 x 128 x 16, fp32 accumulators in two tensor-memory buffers so that a
// unit's epilogue overlaps the next unit's products), warps 4..7 epilogue
// (one accumulator row, i.e. one k, per thread): each warp stages 32 k x 32 t
// pieces of M in shared memory (128-byte swizzled, two buffers per warp) and
// stores them with TMA, which also clips them at M's edges.
// ---------------------------------------------------------------------------
struct WinoGemmCfg {
  static constexpr int BK = 64;                 // c per stage
  static constexpr int TILE = 128 * 128;        // bytes of a 128-row x 64-column 16-bit tile
  static constexpr int STAGE = 2 * TILE;        // U tile, V tile
  static constexpr int STAGES = 5;
  static constexpr int STG = 4096;              // one 32 x 32 fp32 piece of M
  static constexpr int OFF_STG = STAGES * STAGE;   // [4 warps][2][STG]
  static constexpr int OFF_BAR = OFF_STG + 4 * 2 * STG;
  static constexpr int NBAR = 2 * STAGES + 4 + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static constexpr int NTHREADS = 256;
  static constexpr uint32_t TMEM_COLS = 256;
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct WinoGemmParams {
  float* M;
  int K, T, ldm;
  int kbs, tbs;    // blocks of 128 along k and t
  int units;       // 36 * kbs * tbs
  int ksteps;      // ceil(C / 64)
};

template <bool BF16>
__global__ void __launch_bounds__(WinoGemmCfg::NTHREADS, 1)
    wino_gemm_kernel(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmM, const WinoGemmParams p) {
  using C = WinoGemmCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                     // [STAGES] TMA -> MMA
  uint64_t* empty = full + C::STAGES;        // [STAGES] MMA -> TMA
  uint64_t* acc_full = empty + C::STAGES;    // [2] MMA -> epilogue
  uint64_t* acc_empty = acc_full + 2;        // [2] epilogue -> MMA
  uint64_t* drain_bar = acc_empty + 2;
  uint32_t* misc = reinterpret_cast<uint32_t*>(drain_bar + 1);   // [0] tensor memory, [1] abort
  volatile uint32_t* abort_flag = misc + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain_bar, 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmM);
  }
  if (warp == 1) {
    tmem_alloc(&misc[0], C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  grid_dependency_wait();
  grid_launch_dependents();

  const int per_xi = p.kbs * p.tbs;
  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      uint32_t c = 0;
      bool live = true;
      for (int u = blockIdx.x; u < p.units && live; u += gridDim.x) {
        const int xi = u / per_xi, r = u - xi * per_xi, kb = r / p.tbs, tb = r - kb * p.tbs;
        for (int ks = 0; ks < p.ksteps; ++ks, ++c) {
          const uint32_t st = c % C::STAGES, n = c / C::STAGES;
          if (!mbar_wait(&empty[st], (n & 1) ^ 1, kSiteKEmpty, abort_flag)) { live = false; break; }
          uint8_t* s = smem + st * C::STAGE;
          mbar_arrive_expect_tx(&full[st], C::STAGE);
          tma_load_3d(s, &tmU, ks * C::BK, kb * 128, xi, &full[st]);
          tma_load_3d(s + C::TILE, &tmV, ks * C::BK, tb * 128, xi, &full[st]);
        }
      }
      // every load this thread issued lands before the CTA can exit
      volatile uint32_t never = 0;
      for (uint32_t st = 0; st < C::STAGES && st < c; ++st) {
        const uint32_t uses = (c - st + C::STAGES - 1) / C::STAGES;
        mbar_wait(&full[st], (uses - 1) & 1, kSiteKFull, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    constexpr uint32_t idesc = idesc_f16(128, 128, BF16, false, false);
    const uint32_t base = smem_u32(smem);
    uint32_t c = 0, ui = 0;
    bool live = true;
    for (int u = blockIdx.x; u < p.units && live; u += gridDim.x, ++ui) {
      const uint32_t ab = ui & 1, na = ui >> 1;
      if (!mbar_wait_warp(&acc_empty[ab], (na & 1) ^ 1, kSiteAccEmpty, abort_flag)) { live = false; break; }
      tc_fence_after();
      for (int ks = 0; ks < p.ksteps; ++ks, ++c) {
        const uint32_t st = c % C::STAGES, n = c / C::STAGES;
        if (!mbar_wait_warp(&full[st], n & 1, kSiteKFull, abort_flag)) { live = false; break; }
        tc_fence_after();
        const uint32_t s = base + st * C::STAGE;
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk)
          mma_ss(tmem + ab * 128, sdesc_sw128(s + kk * 32, 16, 1024), sdesc_sw128(s + C::TILE + kk * 32, 16, 1024),
                 idesc, (ks > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[st]);
      }
      if (live) mma_commit(&acc_full[ab]);
    }
    volatile uint32_t never = 0;
    mma_commit(drain_bar);
    mbar_wait_warp(drain_bar, 0, kSiteAccFull, &never);
  } else if (warp >= 4) {
    // ------------------------------ epilogue ----------------------------------
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* stg = smem + C::OFF_STG + (warp - 4) * 2 * C::STG;
    uint32_t ui = 0, sc = 0;
    bool live = true;
    for (int u = blockIdx.x; u < p.units && live; u += gridDim.x, ++ui) {
      const int xi = u / per_xi, r = u - xi * per_xi, kb = r / p.tbs, tb = r - kb * p.tbs;
      const uint32_t ab = ui & 1, na = ui >> 1;
      live = __all_sync(0xffffffffu, mbar_wait(&acc_full[ab], na & 1, kSiteAccFull, abort_flag));
      if (!live) break;
      tc_fence_after();
#pragma unroll 1
      for (int c32 = 0; c32 < 4; ++c32) {
        const int t0 = tb * 128 + c32 * 32;
        // stores start inside M (rows past K, columns past ldm are not issued;
        // a piece that runs over an edge is clipped by TMA)
        if (t0 >= p.ldm || kb * 128 + quarter * 32 >= p.K) break;
        uint32_t v[32];
        tmem_ld_x32(tmem + ab * 128 + c32 * 32 + lane_off, v);
        tmem_wait_ld();
        reg_fence<32>(v);
        uint8_t* buf = stg + (sc & 1) * C::STG;
        if (lane == 0) bulk_wait_read<1>();   // this buffer's previous store has read it
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
              make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmM, buf, t0, kb * 128 + quarter * 32, xi);
          bulk_commit();
        }
        ++sc;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sdattn
