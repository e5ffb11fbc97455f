// flash_tf32.cuh -- the FlashAttention form for fp32 inputs: Q, K and V are
// read as fp32 and multiplied on the tensor cores as tf32 (kind::tf32), O is
// written in fp32.
//
// "Speed Is All You Need" (news summary, section on the three optimisations,
// FlashAttention paragraph): exact attention computed block by block in one
// kernel without writing the score matrix to memory.  This form serves
// callers whose activations are fp32 (the small fp32 configuration) without
// rounding them to 16 bits first: Q, K, V and P are rounded to tf32 (10-bit
// mantissas, to nearest) on chip before the tensor-core products (the
// tensor core would otherwise drop the low bits, a bias toward zero that
// alone costs about 1e-3 of relative error in O), and every sum accumulates
// in fp32.
//
// Layout in shared memory: 32-column fp32 slabs of 128-byte rows, 128-byte
// swizzled (the same swizzle as the 16-bit kernels' 64-column slabs).
//   Q tile   DSL slabs x 128 rows          (d = 40, 80, 160: 2, 3, 5 slabs)
//   K tile   DSL slabs x BN rows (keys)     S = Q K^T: M = 128, N = BN, K = 8 per MMA
//   V tile   DSL slabs x BN rows            as loaded (d contiguous)
//   V^T tile BN / 32 slabs x PVN rows       P V: M = 128, N = PVN, K = 8 per MMA
// The tensor core takes a 32-bit operand with its N dimension contiguous only
// in a 32-byte-atom swizzle; rather than that layout, two warps transpose
// each V tile in shared memory into V^T with the keys contiguous (the same
// K-major layout as the S product's operands).  PVN = d + 1 rounded up to 16:
// row d of V^T holds ones, so column d of O accumulates the row sum; rows
// d .. PVN - 1 are written once.
// One 128-row query tile per CTA, persistent over the (b*H + h, row tile)
// units; roles: warp 0 TMA, warp 1 MMA, warps 2, 3, 8, 9 operand preparation (Q
// and K rounded to tf32 in place, V transposed and rounded), warps 4..7
// softmax (one row per thread), with S, P (fp32, BN columns) and O in tensor
// memory.
#pragma once

#include "flash.cuh"

namespace sdattn {

__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn, bool b_mn) {
  // D fp32 (bits 4-5 = 1), A and B tf32 (format 2 in bits 7-9 and 10-12), majors, N / 8, M / 16
  return (1u << 4) | (2u << 7) | (2u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]   (A: 128 lanes x K fp32 values, one per column)
__device__ __forceinline__ void mma_ts_tf32(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t round_tf32(float f) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(f));
  return r;
}

template <int D>
struct FlashTF32Cfg {
  static constexpr int BN = D == 160 ? 32 : 64;            // keys per K / V tile
  static constexpr int DSL = (D + 31) / 32;                // slabs of Q and K
  static constexpr int PVN = (D + 1 + 15) / 16 * 16;       // P V width: d and the row-sum column
  static constexpr int KSTEPS = D / 8;                     // K = 8 per tf32 MMA
  static constexpr int Q_SLAB = 128 * 128;
  static constexpr int KV_SLAB = BN * 128;
  static constexpr int Q_BYTES = DSL * Q_SLAB;
  static constexpr int K_BYTES = DSL * KV_SLAB;
  static constexpr int V_BYTES = DSL * KV_SLAB;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int VT_SLAB = PVN * 128;                // 32 keys of PVN rows
  static constexpr int VT_STAGE = (BN / 32) * VT_SLAB;
  // as many K / V / V^T stages as fit (at most 4): loads run that many key
  // tiles ahead of the preparation, products and softmax
  static constexpr int STAGES_FIT = (232448 - Q_BYTES - 1024 - 16 - 8 * (8 + 5 * 4)) / (STAGE + VT_STAGE);
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static_assert(STAGES >= 2, "key / value ring too shallow");
  static constexpr uint32_t TM_S = 0, TM_P = BN, TM_O = 2 * BN;
  static constexpr uint32_t TMEM_COLS = TM_O + PVN <= 256 ? 256 : 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = Q_BYTES;
  static constexpr int OFF_VT = OFF_KV + STAGES * STAGE;
  static constexpr int OFF_BAR = OFF_VT + STAGES * VT_STAGE;
  static constexpr int NBAR = 3 + 5 * STAGES + 5;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  // preparation warps 2, 3, 8, 9: measured at 64x64, 2 -> 4 warps took the
  // call from 440 to 336 us; 6 or 8 gave nothing more
  static constexpr int NPREP = 4;
  static constexpr int NTHREADS = 256 + 32 * (NPREP - 2);
  static_assert(D % 8 == 0 && BN % 32 == 0, "whole MMA K steps, whole V^T slabs");
  static_assert(TM_O + PVN <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(KV_SLAB % 1024 == 0 && VT_SLAB % 1024 == 0, "swizzle atoms");
};

struct FlashTF32Params {
  int N, M, BH;
  int tph;      // 128-row query tiles per (b, h)
  int nkv;      // key tiles of BN
  int units;    // BH * tph
  float c;      // scale * log2(e)
  float scale;
  float* O;     // [BH][N][D] fp32
  float* LS;    // optional [BH][N][2]
};

template <int D>
__global__ void __launch_bounds__(FlashTF32Cfg<D>::NTHREADS, 1)
    flash_tf32_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const FlashTF32Params p) {
  using C = FlashTF32Cfg<D>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sKV = smem + C::OFF_KV;
  uint8_t* sVT = smem + C::OFF_VT;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;                     // TMA -> MMA
  uint64_t* q_empty = q_full + 1;              // MMA -> TMA: the unit's products no longer read Q
  uint64_t* q_ready = q_empty + 1;             // preparation -> MMA: Q rounded
  uint64_t* k_full = q_ready + 1;              // [STAGES]
  uint64_t* v_full = k_full + C::STAGES;       // [STAGES]
  uint64_t* kv_empty = v_full + C::STAGES;     // [STAGES]
  uint64_t* vt_full = kv_empty + C::STAGES;    // [STAGES] preparation -> MMA: V^T written
  uint64_t* k_ready = vt_full + C::STAGES;     // [STAGES] preparation -> MMA: K rounded
  uint64_t* s_full = k_ready + C::STAGES;      // MMA -> softmax: S ready
  uint64_t* s_free = s_full + 1;               // softmax -> MMA: S loaded
  uint64_t* p_full = s_free + 1;               // softmax -> MMA: P written (O rescaled)
  uint64_t* pv_done = p_full + 1;              // MMA -> softmax: P V done
  uint64_t* drain_bar = pv_done + 1;
  uint32_t* misc = reinterpret_cast<uint32_t*>(drain_bar + 1);   // [0] tensor memory, [1] abort
  volatile uint32_t* abort_flag = misc + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(q_ready, C::NPREP);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&vt_full[i], C::NPREP);
      mbar_init(&k_ready[i], C::NPREP);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(drain_bar, 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  // V^T rows D .. PVN - 1, for good: row D ones (the row sum), the rest zeros
  for (int i = threadIdx.x; i < C::STAGES * (BN / 32) * (C::PVN - D); i += blockDim.x) {
    const int row = D + i % (C::PVN - D), slab = i / (C::PVN - D);
    uint4* dst = reinterpret_cast<uint4*>(sVT + slab * C::VT_SLAB + row * 128);
    const uint32_t w = row == D ? 0x3F800000u : 0u;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) dst[ch] = make_uint4(w, w, w, w);
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
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

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      uint32_t kvc = 0, ui = 0;
      bool live = true;
      for (int u = blockIdx.x; u < p.units && live; u += gridDim.x, ++ui) {
        const int bh = u / p.tph, qt = u % p.tph;
        if (!mbar_wait(q_empty, (ui & 1) ^ 1, kSiteQEmpty, abort_flag)) { live = false; break; }
        mbar_arrive_expect_tx(q_full, C::Q_BYTES);
        for (int s = 0; s < C::DSL; ++s) tma_load_3d(sQ + s * C::Q_SLAB, &tmQ, 32 * s, qt * 128, bh, q_full);
        for (int j = 0; j < p.nkv; ++j, ++kvc) {
          const uint32_t st = kvc % C::STAGES, n = kvc / C::STAGES;
          if (!mbar_wait(&kv_empty[st], (n & 1) ^ 1, kSiteKEmpty, abort_flag)) { live = false; break; }
          uint8_t* sK = sKV + st * C::STAGE;
          uint8_t* sV = sK + C::K_BYTES;
          mbar_arrive_expect_tx(&k_full[st], C::K_BYTES);
          for (int s = 0; s < C::DSL; ++s) tma_load_3d(sK + s * C::KV_SLAB, &tmK, 32 * s, j * BN, bh, &k_full[st]);
          mbar_arrive_expect_tx(&v_full[st], C::V_BYTES);
          for (int s = 0; s < C::DSL; ++s) tma_load_3d(sV + s * C::KV_SLAB, &tmV, 32 * s, j * BN, bh, &v_full[st]);
        }
      }
      volatile uint32_t never = 0;
      if (ui > 0) mbar_wait(q_full, (ui - 1) & 1, kSiteQFull, &never);
      for (uint32_t st = 0; st < C::STAGES && st < kvc; ++st) {
        const uint32_t uses = (kvc - st + C::STAGES - 1) / C::STAGES;
        mbar_wait(&k_full[st], (uses - 1) & 1, kSiteKFull, &never);
        mbar_wait(&v_full[st], (uses - 1) & 1, kSiteVFull, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    // Per key tile j: S_j (once the softmax has loaded S_{j-1}), then P V for
    // tile j - 1 (once P_{j-1} is written).
    constexpr uint32_t idesc_s = idesc_tf32(128, BN, false, false);
    constexpr uint32_t idesc_pv = idesc_tf32(128, C::PVN, false, false);   // V^T: keys contiguous
    const uint32_t q_base = smem_u32(sQ), kv_base = smem_u32(sKV);
    const uint32_t s_tm = tmem + C::TM_S, p_tm = tmem + C::TM_P, o_tm = tmem + C::TM_O;
    uint32_t t = 0, kvc = 0, ui = 0;
    bool live = true;
    for (int u = blockIdx.x; u < p.units && live; u += gridDim.x, ++ui) {
      if (!mbar_wait_warp(q_ready, ui & 1, kSiteQFull, abort_flag)) { live = false; break; }
      for (int j = 0; j <= p.nkv; ++j) {
        if (j < p.nkv) {
          const uint32_t kv = kvc + j, st = kv % C::STAGES, n = kv / C::STAGES;
          if (!mbar_wait_warp(&k_ready[st], n & 1, kSiteKFull, abort_flag)) { live = false; break; }
          if (t + j >= 1 && !mbar_wait_warp(s_free, (t + j - 1) & 1, kSiteSFull, abort_flag)) { live = false; break; }
          tc_fence_after();
          const uint32_t kb = kv_base + st * C::STAGE;
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {   // K = 8 per step: four steps per 32-column slab
            const uint32_t off = (kk & 3) * 32;
            mma_ss_tf32(s_tm, sdesc_sw128(q_base + (kk >> 2) * C::Q_SLAB + off, 16, 1024),
                        sdesc_sw128(kb + (kk >> 2) * C::KV_SLAB + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(s_full);
          if (j == p.nkv - 1) mma_commit(q_empty);   // the unit's last read of Q
        }
        if (j >= 1) {
          const uint32_t kv = kvc + j - 1, st = kv % C::STAGES, n = kv / C::STAGES;
          if (!mbar_wait_warp(&vt_full[st], n & 1, kSiteVFull, abort_flag)) { live = false; break; }
          if (!mbar_wait_warp(p_full, (t + j - 1) & 1, kSitePFull, abort_flag)) { live = false; break; }
          tc_fence_after();
          const uint32_t vt = smem_u32(sVT) + st * C::VT_STAGE;
#pragma unroll
          for (int kk = 0; kk < BN / 8; ++kk)   // K = 8 keys per step: four steps per 32-key slab
            mma_ts_tf32(o_tm, p_tm + kk * 8, sdesc_sw128(vt + (kk >> 2) * C::VT_SLAB + (kk & 3) * 32, 16, 1024),
                        idesc_pv, (j > 1 || kk > 0) ? 1u : 0u);
          mma_commit(pv_done);
          mma_commit(&kv_empty[st]);
        }
      }
      t += p.nkv;
      kvc += p.nkv;
    }
    volatile uint32_t never = 0;
    mma_commit(drain_bar);
    mbar_wait_warp(drain_bar, 0, kSitePvDone, &never);
  } else if (warp == 2 || warp == 3 || warp >= 8) {
    // ------------------------- operand preparation --------------------------
    // Q and K rounded to tf32 in place; V [key r][column c] (as loaded:
    // 32-column slabs, 128-byte swizzled) -> V^T [row c][key r] (32-key slabs,
    // 128-byte swizzled), rows 0 .. D - 1, rounded to tf32.
    const int tid = warp >= 8 ? static_cast<int>(threadIdx.x) - 192 : static_cast<int>(threadIdx.x) - 64;
    constexpr int kPrepThreads = 32 * C::NPREP;
    // 16 bytes per access (the swizzle moves whole 16-byte chunks, so the
    // rounding does not care where a word sits)
    auto round_in_place = [&](uint8_t* base, int words) {
      uint4* w = reinterpret_cast<uint4*>(base);
#pragma unroll 4
      for (int i = tid; i < words / 4; i += kPrepThreads) {
        uint4 x = w[i];
        x.x = round_tf32(__uint_as_float(x.x));
        x.y = round_tf32(__uint_as_float(x.y));
        x.z = round_tf32(__uint_as_float(x.z));
        x.w = round_tf32(__uint_as_float(x.w));
        w[i] = x;
      }
    };
    auto publish = [&](uint64_t* bar) {
      fence_proxy_async_smem();   // generic-proxy writes before the tensor core reads them
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    uint32_t kvc = 0, ui = 0;
    bool live = true;
    for (int u = blockIdx.x; u < p.units && live; u += gridDim.x, ++ui) {
      live = __all_sync(0xffffffffu, mbar_wait(q_full, ui & 1, kSiteQFull, abort_flag));
      if (!live) break;
      round_in_place(sQ, C::Q_BYTES / 4);
      publish(q_ready);
      for (int j = 0; j < p.nkv; ++j, ++kvc) {
        const uint32_t st = kvc % C::STAGES, n = kvc / C::STAGES;
        uint8_t* sK = sKV + st * C::STAGE;
        live = __all_sync(0xffffffffu, mbar_wait(&k_full[st], n & 1, kSiteKFull, abort_flag));
        if (!live) break;
        round_in_place(sK, C::K_BYTES / 4);
        publish(&k_ready[st]);
        live = __all_sync(0xffffffffu, mbar_wait(&v_full[st], n & 1, kSiteVFull, abort_flag));
        if (!live) break;
        const uint8_t* sV = sK + C::K_BYTES;
        uint8_t* vt = sVT + st * C::VT_STAGE;
        // one item = key r, columns c4 .. c4 + 3: a 16-byte chunk of V's row
        // (consecutive lanes take consecutive keys: eight lanes cover the
        // eight chunk positions of the swizzle, no bank conflicts), four
        // rounded words into four rows of V^T
#pragma unroll 2
        for (int idx = tid; idx < (D / 4) * BN; idx += kPrepThreads) {
          const int c4 = (idx / BN) * 4, r = idx - (idx / BN) * BN;
          const uint4 x = *reinterpret_cast<const uint4*>(sV + (c4 >> 5) * C::KV_SLAB + r * 128 +
                                                          ((((c4 & 31) >> 2) ^ (r & 7)) << 4));
          const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
          uint8_t* vrow = vt + (r >> 5) * C::VT_SLAB + (r & 3) * 4;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = c4 + i;
            *reinterpret_cast<uint32_t*>(vrow + c * 128 + ((((r & 31) >> 2) ^ (c & 7)) << 4)) =
                round_tf32(__uint_as_float(xv[i]));
          }
        }
        publish(&vt_full[st]);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------------------- softmax, one row per thread -----------------------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_tmem = tmem + C::TM_S + lane_off, p_tmem = tmem + C::TM_P + lane_off;
    const uint32_t o_tmem = tmem + C::TM_O + lane_off;
    const float c = p.c;
    uint32_t t = 0;
    bool live = true;
    for (int u = blockIdx.x; u < p.units && live; u += gridDim.x) {
      const int bh = u / p.tph, qt = u % p.tph;
      const int row = qt * 128 + r;
      float m_used = -INFINITY, rawmax = -INFINITY;
      for (int j = 0; j < p.nkv; ++j, ++t) {
        live = __all_sync(0xffffffffu, mbar_wait(s_full, t & 1, kSiteSFull, abort_flag));
        if (!live) break;
        tc_fence_after();
        uint32_t v[BN];
        if constexpr (BN == 64) {
          tmem_ld_x64(s_tmem, v);
        } else {
          tmem_ld_x32(s_tmem, v);
        }
        tmem_wait_ld();
        reg_fence<BN>(v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        const int valid = p.M - j * BN;
        float mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < BN; ++k) {
          if (k >= valid) v[k] = __float_as_uint(-INFINITY);
          mx = fmaxf(mx, __uint_as_float(v[k]));
        }
        rawmax = fmaxf(rawmax, mx);
        const float mt = mx * c;
        float alpha = 1.f;
        bool rescale = false;
        if (mt > m_used + 8.f) {   // the lazy rule of flash.cuh
          alpha = ex2_approx(m_used - mt);
          m_used = mt;
          rescale = j > 0;
        }
#pragma unroll
        for (int k = 0; k < BN; ++k) v[k] = round_tf32(ex2_approx(fmaf(__uint_as_float(v[k]), c, -m_used)));
        if (j > 0) {
          // P V of the previous tile must be done: P is reused and O may be rescaled
          live = __all_sync(0xffffffffu, mbar_wait(pv_done, (t - 1) & 1, kSitePvDone, abort_flag));
          if (!live) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
            for (int cc = 0; cc < C::PVN; cc += 16) {
              uint32_t o[16];
              tmem_ld_x16(o_tmem + cc, o);
              tmem_wait_ld();
              reg_fence<16>(o);
#pragma unroll
              for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st_x16(o_tmem + cc, o);
            }
          }
        }
#pragma unroll
        for (int cc = 0; cc < BN; cc += 16) tmem_st_x16(p_tmem + cc, v + cc);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!live) break;
      // ---- epilogue: O / l, with l = column D of O ----
      live = __all_sync(0xffffffffu, mbar_wait(pv_done, (t - 1) & 1, kSitePvDone, abort_flag));
      if (!live) break;
      tc_fence_after();
      float l;
      {
        uint32_t o8[8];
        tmem_ld_x8(o_tmem + (D / 8) * 8, o8);   // column D is element D % 8 of its group of 8
        tmem_wait_ld();
        reg_fence<8>(o8);
        l = __uint_as_float(o8[D % 8]);
      }
      const float inv = 1.f / l;
      float* orow = p.O + (static_cast<int64_t>(bh) * p.N + row) * D;
#pragma unroll
      for (int c8 = 0; c8 < D / 8; ++c8) {
        uint32_t o[8];
        tmem_ld_x8(o_tmem + c8 * 8, o);
        tmem_wait_ld();
        reg_fence<8>(o);
        if (row < p.N) {
          reinterpret_cast<float4*>(orow)[2 * c8] = make_float4(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv,
                                                                __uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
          reinterpret_cast<float4*>(orow)[2 * c8 + 1] = make_float4(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv,
                                                                    __uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
        }
      }
      if (p.LS != nullptr && row < p.N) {
        *reinterpret_cast<float2*>(p.LS + 2 * (static_cast<int64_t>(bh) * p.N + row)) =
            make_float2(rawmax * p.scale, l * ex2_approx(m_used - rawmax * c));
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sdattn
