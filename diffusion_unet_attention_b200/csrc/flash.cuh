// flash.cuh -- FlashAttention form: exact attention in one kernel, tiled over
// keys with an online softmax; the score matrix never reaches memory.
//
// "Speed Is All You Need" (news summary, section on the three optimisations,
// FlashAttention paragraph): an IO-aware exact attention that computes block
// by block (tiling) and fuses all attention operations into one kernel,
// cutting high-bandwidth-memory traffic; the summary notes the kernel is
// register-intensive.
//
// B200 design.  One persistent CTA per SM walks (b*H + h, group of NQ
// 128-row query tiles) units.  Roles:
//   warp 0            TMA producer: the unit's NQ Q tiles, then a ring of
//                     (K tile, V tile) stages, 128-byte swizzled, no multicast;
//   warp 1            tcgen05 MMA issuer: S = Q K^T into tensor memory; once
//                     the softmax has written P (16-bit, aliasing S in tensor
//                     memory) O += P V with O accumulated in tensor memory;
//   warps 4+4q..7+4q  softmax for query tile q, one row per thread: row max,
//                     p = 2^(s*scale*log2e - m), row sum, P packed to 16 bits,
//                     and the rescale of O when the running max grows.
// With NQ = 2 the two tiles ping-pong: while one tile's softmax runs, the
// tensor core computes the other's scores.  With NQ = 1 the S buffer is
// doubled instead, so the next tile's scores are ready when the softmax is.
// The running max is only raised when a tile's max exceeds it by more than
// 2^8 (in the base-2 exponent), so O is rescaled rarely; p stays below 256,
// which 16-bit P and the fp32 accumulators absorb exactly as the true max would.
#pragma once

#include "sm100.cuh"

namespace sdattn {

struct FlashParams {
  int N, M, BH;
  int tph;     // units per (b, h): query-tile groups of NQ x 128 rows
  int nkv;     // key tiles of BN
  int units;   // BH * tph
  float c;     // scale * log2(e)
  float scale;
  void* O;
  float* LS;   // optional
};

template <int D, int NQ, int BN>
struct FlashCfg {
  static constexpr int DSLABS = (D + 63) / 64;
  static constexpr int KSTEPS = (D + 15) / 16;
  static constexpr int PVN = DSLABS * 64;
  static constexpr int SBUF = NQ == 1 ? 2 : 1;     // S/P buffers per query tile
  static constexpr int Q_TILE = DSLABS * 128 * 128;
  static constexpr int KV_SLAB = BN * 128;
  static constexpr int K_BYTES = DSLABS * KV_SLAB;
  static constexpr int V_BYTES = DSLABS * KV_SLAB;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int STAGES_FIT = (226 * 1024 - NQ * Q_TILE) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static constexpr int QCOLS = SBUF * BN + PVN;     // tensor-memory columns per query tile
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = NQ * Q_TILE;
  static constexpr int OFF_BAR = OFF_KV + STAGES * STAGE;
  static constexpr int NBAR = 2 + 3 * STAGES + NQ * SBUF + 2 * NQ + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static constexpr int NTHREADS = 128 + 128 * NQ;
  // With two S buffers the MMA issuer runs one tile further ahead, so the
  // ring needs a third stage to keep loads overlapped with compute.
  static_assert(STAGES >= 2 + (SBUF - 1), "key/value ring too shallow");
  static_assert(NQ * QCOLS <= 512, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 128, "key tile");
};

template <int D, int NQ, int BN, bool BF16, int NPOLY>
__global__ void __launch_bounds__(FlashCfg<D, NQ, BN>::NTHREADS, 1)
    flash_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const FlashParams p) {
  using C = FlashCfg<D, NQ, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sKV = smem + C::OFF_KV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* v_full = k_full + C::STAGES;
  uint64_t* kv_empty = v_full + C::STAGES;
  uint64_t* s_full = kv_empty + C::STAGES;          // [NQ][SBUF]
  uint64_t* p_full = s_full + NQ * C::SBUF;         // [NQ]
  uint64_t* pv_done = p_full + NQ;                  // [NQ]
  uint64_t* drain_bar = pv_done + NQ;
  uint32_t* misc = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile uint32_t* abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < NQ * C::SBUF; ++i) mbar_init(&s_full[i], 1);
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain_bar, 1);
    misc[1] = 0;
    fence_mbar_init();
  }
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

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if constexpr (NQ == 2) regs_dec<120>();
    if (lane == 0) {
      uint32_t kvc = 0, nq = 0;
      bool live = true;
      for (int u = blockIdx.x; u < p.units && live; u += gridDim.x) {
        const int bh = u / p.tph, qg = u % p.tph;
        if (!mbar_wait(q_empty, (nq & 1) ^ 1, kSiteQEmpty, abort_flag)) { live = false; break; }
        ++nq;
        mbar_arrive_expect_tx(q_full, NQ * C::Q_TILE);
        for (int q = 0; q < NQ; ++q)
          for (int s = 0; s < C::DSLABS; ++s)
            tma_load_3d(sQ + q * C::Q_TILE + s * 16384, &tmQ, 64 * s, (qg * NQ + q) * 128, bh, q_full);
        for (int j = 0; j < p.nkv; ++j, ++kvc) {
          const uint32_t st = kvc % C::STAGES, n = kvc / C::STAGES;
          if (!mbar_wait(&kv_empty[st], (n & 1) ^ 1, kSiteKEmpty, abort_flag)) { live = false; break; }
          uint8_t* sK = sKV + st * C::STAGE;
          uint8_t* sV = sK + C::K_BYTES;
          mbar_arrive_expect_tx(&k_full[st], C::K_BYTES);
          for (int s = 0; s < C::DSLABS; ++s) tma_load_3d(sK + s * C::KV_SLAB, &tmK, 64 * s, j * BN, bh, &k_full[st]);
          mbar_arrive_expect_tx(&v_full[st], C::V_BYTES);
          for (int s = 0; s < C::DSLABS; ++s) tma_load_3d(sV + s * C::KV_SLAB, &tmV, 64 * s, j * BN, bh, &v_full[st]);
        }
      }
      volatile uint32_t never = 0;
      if (nq > 0) mbar_wait(q_full, (nq - 1) & 1, kSiteQFull, &never);
      for (uint32_t st = 0; st < C::STAGES && st < kvc; ++st) {
        const uint32_t uses = (kvc - st + C::STAGES - 1) / C::STAGES;
        mbar_wait(&k_full[st], (uses - 1) & 1, kSiteKFull, &never);
        mbar_wait(&v_full[st], (uses - 1) & 1, kSiteVFull, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    if constexpr (NQ == 2) regs_dec<120>();
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f16(128, BN, BF16, false, false);
      constexpr uint32_t idesc_pv = idesc_f16(128, C::PVN, BF16, false, true);
      const uint32_t q_base = smem_u32(sQ), kv_base_addr = smem_u32(sKV);
      uint32_t t_base = 0, kv_base = 0, ui = 0;
      bool live = true;

      auto issue_pv = [&](int q, int jj) -> bool {
        const uint32_t kv = kv_base + jj;
        const uint32_t st = kv % C::STAGES, n = kv / C::STAGES;
        const uint32_t t = t_base + jj;
        if (q == 0 && !mbar_wait(&v_full[st], n & 1, kSiteVFull, abort_flag)) return false;
        if (!mbar_wait(&p_full[q], t & 1, kSitePFull, abort_flag)) return false;
        tc_fence_after();
        const uint32_t p_tmem = tmem + q * C::QCOLS + (t % C::SBUF) * BN;
        const uint32_t o_tmem = tmem + q * C::QCOLS + C::SBUF * BN;
        const uint32_t v_addr = kv_base_addr + st * C::STAGE + C::K_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(v_addr + kk * 2048, C::KV_SLAB, 1024);
          mma_ts(o_tmem, p_tmem + kk * 8, bd, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&pv_done[q]);
        return true;
      };

      for (int u = blockIdx.x; u < p.units && live; u += gridDim.x, ++ui) {
        if (!mbar_wait(q_full, ui & 1, kSiteQFull, abort_flag)) { live = false; break; }
        tc_fence_after();
        for (int j = 0; j < p.nkv && live; ++j) {
          const uint32_t kv = kv_base + j;
          const uint32_t st = kv % C::STAGES, n = kv / C::STAGES;
          const uint32_t t = t_base + j;
          if (C::SBUF == 2 && j >= 2) {
            // release tile j-2's stage before waiting for tile j's keys
            for (int q = 0; q < NQ && live; ++q)
              if (!issue_pv(q, j - 2)) live = false;
            if (!live) break;
            mma_commit(&kv_empty[(kv - 2) % C::STAGES]);
          }
          for (int q = 0; q < NQ && live; ++q) {
            if (C::SBUF == 1 && j >= 1 && !issue_pv(q, j - 1)) { live = false; break; }
            if (q == 0) {
              if (!mbar_wait(&k_full[st], n & 1, kSiteKFull, abort_flag)) { live = false; break; }
              tc_fence_after();
            }
            const uint32_t s_tmem = tmem + q * C::QCOLS + (t % C::SBUF) * BN;
            const uint32_t k_addr = kv_base_addr + st * C::STAGE;
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS; ++kk) {
              const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
              const uint32_t koff = (kk >> 2) * C::KV_SLAB + (kk & 3) * 32;
              const uint64_t ad = sdesc_sw128(q_base + q * C::Q_TILE + off, 16, 1024);
              const uint64_t bd = sdesc_sw128(k_addr + koff, 16, 1024);
              mma_ss(s_tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
            }
            mma_commit(&s_full[q * C::SBUF + (t % C::SBUF)]);
          }
          if (C::SBUF == 1 && live && j >= 1) mma_commit(&kv_empty[(kv - 1) % C::STAGES]);
        }
        const int j0 = p.nkv > C::SBUF ? p.nkv - C::SBUF : 0;
        for (int jj = j0; jj < p.nkv && live; ++jj) {
          for (int q = 0; q < NQ && live; ++q)
            if (!issue_pv(q, jj)) live = false;
          if (live) mma_commit(&kv_empty[(kv_base + jj) % C::STAGES]);
        }
        if (live) mma_commit(q_empty);
        t_base += p.nkv;
        kv_base += p.nkv;
      }
      volatile uint32_t never = 0;
      mma_commit(drain_bar);
      mbar_wait(drain_bar, 0, kSitePvDone, &never);
    }
  } else if (warp >= 4) {
    // ---------------------------- softmax, tile q -----------------------------
    if constexpr (NQ == 2) regs_inc<192>();
    const int q = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t o_tmem = tmem + q * C::QCOLS + C::SBUF * BN + lane_off;
    const float c = p.c;
    // V's padding column D is set to 1 in every tile, so column D of O
    // accumulates the row sum of P in fp32 on the tensor core.
    constexpr int TAIL = D - 64 * (C::DSLABS - 1);           // columns of V's last slab
    const uint32_t one16 = BF16 ? 0x3F80u : 0x3C00u;
    uint32_t t = 0;        // tiles seen by this query-tile slot (all units)
    uint32_t kvt = 0;      // key tiles seen (stage index)
    bool live = true;
    for (int u = blockIdx.x; u < p.units && live; u += gridDim.x) {
      const int bh = u / p.tph, qg = u % p.tph;
      const int row = (qg * NQ + q) * 128 + r;
      float m_used = -INFINITY, rawmax = -INFINITY;
      for (int j = 0; j < p.nkv; ++j, ++t, ++kvt) {
        const uint32_t slot = t % C::SBUF, n = t / C::SBUF;
        if (q == 0) {
          // ones column of this tile's V rows (after the tile has landed)
          const uint32_t st = kvt % C::STAGES, ns = kvt / C::STAGES;
          live = __all_sync(0xffffffffu, mbar_wait(&v_full[st], ns & 1, kSiteVFull, abort_flag));
          if (!live) break;
          if (r < BN) {
            uint8_t* vrow = sKV + st * C::STAGE + C::K_BYTES + (C::DSLABS - 1) * C::KV_SLAB + r * 128;
            *reinterpret_cast<uint4*>(vrow + (((TAIL / 8) ^ (r & 7)) << 4)) = make_uint4(one16, 0u, 0u, 0u);
            fence_proxy_async_smem();
          }
        }
        live = __all_sync(0xffffffffu, mbar_wait(&s_full[q * C::SBUF + slot], n & 1, kSiteSFull, abort_flag));
        if (!live) break;
        tc_fence_after();
        const uint32_t s_tmem = tmem + q * C::QCOLS + slot * BN + lane_off;
        uint32_t v[BN];
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) tmem_ld_x32(s_tmem + cc * 32, v + cc * 32);
        tmem_wait_ld();
        reg_fence<BN>(v);
        const int valid = p.M - j * BN;
        if (valid < BN) {
#pragma unroll
          for (int k = 0; k < BN; ++k)
            if (k >= valid) v[k] = __float_as_uint(-INFINITY);
        }
        // row max: eight independent three-input chains, then a small tree
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __uint_as_float(v[i]);
        int k0 = 8;
#pragma unroll
        for (; k0 + 16 <= BN; k0 += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[i] = fmax3(acc[i], __uint_as_float(v[k0 + i]), __uint_as_float(v[k0 + 8 + i]));
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (k0 + i < BN) acc[i] = fmaxf(acc[i], __uint_as_float(v[k0 + i]));
        const float mx = fmaxf(fmax3(acc[0], acc[1], acc[2]), fmax3(acc[3], acc[4], fmax3(acc[5], acc[6], acc[7])));
        rawmax = fmaxf(rawmax, mx);
        const float mt = mx * c;
        float alpha = 1.f;
        bool rescale = false;
        if (mt > m_used + 8.f) {
          alpha = ex2_approx(m_used - mt);
          m_used = mt;
          rescale = (j > 0);
        }
        // p = 2^(s*c - m): NPOLY of every 8 pairs on the FMA pipe, the rest on MUFU
        const uint64_t c2 = f2_pack(c, c);
        const uint64_t nm2 = f2_pack(-m_used, -m_used);
        uint32_t pk[BN / 2];
#pragma unroll
        for (int k = 0; k < BN / 2; ++k) {
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1])), c2, nm2);
          float x0, x1, e0, e1;
          f2_unpack(x2, x0, x1);
          if ((k & 7) < NPOLY) {
            exp2_poly2(x0, x1, e0, e1);
          } else {
            e0 = ex2_approx(x0);
            e1 = ex2_approx(x1);
          }
          pk[k] = pack2<BF16>(e0, e1);
        }
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) tmem_st_x16(s_tmem + cc * 16, pk + cc * 16);
        if (j > 0) {
          // P V of the previous tile must be done before O is touched
          live = __all_sync(0xffffffffu, mbar_wait(&pv_done[q], (t - 1) & 1, kSitePvDone, abort_flag));
          if (!live) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
            for (int cc = 0; cc < C::PVN / 32; ++cc) {
              uint32_t o[32];
              tmem_ld_x32(o_tmem + cc * 32, o);
              tmem_wait_ld();
              reg_fence<32>(o);
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st_x16(o_tmem + cc * 32, o);
              tmem_st_x16(o_tmem + cc * 32 + 16, o + 16);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[q]);
      }
      if (!live) break;
      // ---- epilogue: O / l, with l = column D of O ----
      live = __all_sync(0xffffffffu, mbar_wait(&pv_done[q], (t - 1) & 1, kSitePvDone, abort_flag));
      if (!live) break;
      tc_fence_after();
      float l;
      {
        uint32_t o[8];
        tmem_ld_x8(o_tmem + D, o);
        tmem_wait_ld();
        reg_fence<8>(o);
        l = __uint_as_float(o[0]);
      }
      const float inv = 1.f / l;
      uint8_t* orow = reinterpret_cast<uint8_t*>(p.O) + (static_cast<int64_t>(bh) * p.N + row) * D * 2;
#pragma unroll
      for (int c8 = 0; c8 < D / 8; ++c8) {
        uint32_t o[8];
        tmem_ld_x8(o_tmem + c8 * 8, o);
        tmem_wait_ld();
        reg_fence<8>(o);
        uint4 w;
        w.x = pack2<BF16>(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
        w.y = pack2<BF16>(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
        w.z = pack2<BF16>(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
        w.w = pack2<BF16>(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
        if (row < p.N) *reinterpret_cast<uint4*>(orow + c8 * 16) = w;
      }
      if (p.LS != nullptr && row < p.N) {
        const float L = rawmax * p.scale;
        const float S = l * ex2_approx(m_used - rawmax * c);
        *reinterpret_cast<float2*>(p.LS + 2 * (static_cast<int64_t>(bh) * p.N + row)) = make_float2(L, S);
      }
      tc_fence_before();
    }
  } else {
    // idle warps of the first warp group
    if constexpr (NQ == 2) regs_dec<120>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sdattn
