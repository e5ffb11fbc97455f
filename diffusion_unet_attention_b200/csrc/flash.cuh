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
// S, P and O have separate tensor-memory buffers per query tile.  The softmax
// releases S as soon as it has loaded it into registers, so the tensor core
// computes the next tile's scores while this tile's exponentials run; P is
// released when P V completes.  With NQ = 2 two query tiles share the key
// and value stages and their softmax phases overlap on the SM.
// The running max is only raised when a tile's max exceeds it by more than
// 2^8 (in the base-2 exponent), so O is rescaled rarely; p stays below 256,
// which 16-bit P and the fp32 accumulators absorb exactly as the true max would.
// The row sum l comes from the tensor core: V's padding column D holds 1 in
// every stage (written once; the V tile loads never cover it), so column D of
// O accumulates sum_j p_j from the same 16-bit P that multiplies V.
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
  int inject_stall;   // test hook: the MMA warp first waits on a barrier nothing completes
};

template <int D, int NQ, int BN>
struct FlashCfg {
  static constexpr int DSLABS = (D + 63) / 64;
  static constexpr int KSTEPS = (D + 15) / 16;
  static constexpr int PVN = DSLABS * 64;          // P V width: D padded to 64, column D = row sum
  static constexpr int TAIL = D - 64 * (DSLABS - 1);  // V columns loaded into its last slab
  static constexpr int Q_TILE = DSLABS * 128 * 128;
  static constexpr int KV_SLAB = BN * 128;
  static constexpr int K_BYTES = DSLABS * KV_SLAB;
  static constexpr int V_BYTES = DSLABS * KV_SLAB;
  static constexpr int V_TX = (DSLABS - 1) * KV_SLAB + TAIL * 2 * BN;   // bytes the V loads deliver
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int QBUF = 2;                  // Q tiles double-buffered across work units
  // 227 KB per CTA, less alignment slack, barriers and the tensor-memory word
  static constexpr int STAGES_FIT = (232448 - 1024 - 16 - 8 * 32 - QBUF * NQ * Q_TILE) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  // tensor memory per query tile: S (BN fp32), P (BN/2 columns of 16-bit pairs), O (PVN fp32)
  static constexpr uint32_t TM_S = 0;
  static constexpr uint32_t TM_P = BN;
  static constexpr uint32_t TM_O = BN + BN / 2;
  static constexpr int QCOLS = BN + BN / 2 + PVN;
  static constexpr uint32_t TMEM_COLS = NQ * QCOLS <= 256 ? 256 : 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = QBUF * NQ * Q_TILE;
  static constexpr int OFF_BAR = OFF_KV + STAGES * STAGE;
  static constexpr int NBAR = 2 * QBUF + 3 * STAGES + 5 * NQ + 2;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static constexpr int NTHREADS = 128 + 128 * NQ;
  static_assert(STAGES >= 2, "key/value ring too shallow");
  static_assert(NQ * QCOLS <= 512, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 128, "key tile");
  static_assert(TAIL % 8 == 0 && TAIL < 64, "room for the ones column in V's last slab");
};

template <int D, int NQ, int BN, bool BF16, int NPOLY>
__global__ void __launch_bounds__(FlashCfg<D, NQ, BN>::NTHREADS, 1)
    flash_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmVt,
                 const FlashParams p) {
  using C = FlashCfg<D, NQ, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sKV = smem + C::OFF_KV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;                  // [QBUF]
  uint64_t* q_empty = q_full + C::QBUF;     // [QBUF] released by every query tile's MMA warp
  uint64_t* k_full = q_empty + C::QBUF;
  uint64_t* v_full = k_full + C::STAGES;
  uint64_t* kv_empty = v_full + C::STAGES;
  // Each query tile has its own MMA-issuing warp and its own handshakes; the
  // tiles share only the Q load and the key/value stages.
  uint64_t* s_full = kv_empty + C::STAGES;   // [NQ] MMA -> softmax: S ready
  uint64_t* s_free = s_full + NQ;            // [NQ] softmax -> MMA: S loaded, buffer free
  uint64_t* p_full = s_free + NQ;            // [NQ] softmax -> MMA: P written (O rescaled)
  uint64_t* pv_done = p_full + NQ;           // [NQ] MMA -> softmax: P V done, P free
  uint64_t* drain_bar = pv_done + NQ;        // [NQ]
  uint64_t* stall_bar = drain_bar + NQ;      // never completed: target of the stall test hook
  uint64_t* stagger = stall_bar + 1;         // query tile 0 -> 1, once: start half a tile apart
  uint32_t* misc = reinterpret_cast<uint32_t*>(stall_bar + 1);
  volatile uint32_t* abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::QBUF; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], NQ);
    }
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], NQ);
    }
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
      mbar_init(&drain_bar[i], 1);
    }
    mbar_init(stall_bar, 1);
    mbar_init(stagger, 4);
    misc[1] = 0;
    fence_mbar_init();
  }
  // V's last slab: the loads cover its first TAIL columns; column D (chunk
  // TAIL/8 of each 128-byte row, element 0) holds 1 and the rest 0, for good.
  {
    const uint32_t one16 = BF16 ? 0x3F80u : 0x3C00u;
    for (int i = threadIdx.x; i < C::STAGES * BN; i += blockDim.x) {
      const int st = i / BN, r = i % BN;
      uint8_t* row = sKV + st * C::STAGE + C::K_BYTES + (C::DSLABS - 1) * C::KV_SLAB + r * 128;
#pragma unroll
      for (int ch = C::TAIL / 8; ch < 8; ++ch)
        *reinterpret_cast<uint4*>(row + ((ch ^ (r & 7)) << 4)) =
            make_uint4(ch == C::TAIL / 8 ? one16 : 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmVt);
  }
  if (warp == 1) {
    tmem_alloc(&misc[0], C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  // Everything above touched only this CTA's own resources; global inputs and
  // outputs are used only once the previous kernel of the stream is complete.
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if constexpr (NQ == 2) regs_dec<120>();
    if (lane == 0) {
      uint32_t kvc = 0, nq = 0;
      bool live = true;
      for (int u = blockIdx.x; u < p.units && live; u += gridDim.x) {
        const int bh = u / p.tph, qg = u % p.tph;
        const uint32_t qb = nq % C::QBUF, qn = nq / C::QBUF;
        if (!mbar_wait(&q_empty[qb], (qn & 1) ^ 1, kSiteQEmpty, abort_flag)) { live = false; break; }
        ++nq;
        mbar_arrive_expect_tx(&q_full[qb], NQ * C::Q_TILE);
        for (int q = 0; q < NQ; ++q)
          for (int s = 0; s < C::DSLABS; ++s)
            tma_load_3d(sQ + (qb * NQ + q) * C::Q_TILE + s * 16384, &tmQ, 64 * s, (qg * NQ + q) * 128, bh,
                        &q_full[qb]);
        for (int j = 0; j < p.nkv; ++j, ++kvc) {
          const uint32_t st = kvc % C::STAGES, n = kvc / C::STAGES;
          if (!mbar_wait(&kv_empty[st], (n & 1) ^ 1, kSiteKEmpty, abort_flag)) { live = false; break; }
          uint8_t* sK = sKV + st * C::STAGE;
          uint8_t* sV = sK + C::K_BYTES;
          mbar_arrive_expect_tx(&k_full[st], C::K_BYTES);
          for (int s = 0; s < C::DSLABS; ++s) tma_load_3d(sK + s * C::KV_SLAB, &tmK, 64 * s, j * BN, bh, &k_full[st]);
          mbar_arrive_expect_tx(&v_full[st], C::V_TX);
          for (int s = 0; s + 1 < C::DSLABS; ++s)
            tma_load_3d(sV + s * C::KV_SLAB, &tmV, 64 * s, j * BN, bh, &v_full[st]);
          tma_load_3d(sV + (C::DSLABS - 1) * C::KV_SLAB, &tmVt, 64 * (C::DSLABS - 1), j * BN, bh, &v_full[st]);
        }
      }
      volatile uint32_t never = 0;
      for (uint32_t qb = 0; qb < C::QBUF && qb < nq; ++qb) {
        const uint32_t uses = (nq - qb + C::QBUF - 1) / C::QBUF;
        mbar_wait(&q_full[qb], (uses - 1) & 1, kSiteQFull, &never);
      }
      for (uint32_t st = 0; st < C::STAGES && st < kvc; ++st) {
        const uint32_t uses = (kvc - st + C::STAGES - 1) / C::STAGES;
        mbar_wait(&k_full[st], (uses - 1) & 1, kSiteKFull, &never);
        mbar_wait(&v_full[st], (uses - 1) & 1, kSiteVFull, &never);
      }
    }
  } else if (warp >= 1 && warp <= NQ) {
    // --------------------------- MMA issuer, tile q ---------------------------
    // The whole warp runs the loop; one elected lane issues.  Per key tile j:
    // S_j (once the softmax has loaded S_{j-1}), then P V for tile j-1 (once
    // P_{j-1} is written).  Warp 1 + q serves query tile q only.
    if constexpr (NQ == 2) regs_dec<120>();
    const int q = warp - 1;
    constexpr uint32_t idesc_s = idesc_f16(128, BN, BF16, false, false);
    constexpr uint32_t idesc_pv = idesc_f16(128, C::PVN, BF16, false, true);
    // descriptors of this tile's first Q slab and of stage 0's K and V; others by address offset
    const uint64_t q_desc00 = sdesc_sw128(smem_u32(sQ) + q * C::Q_TILE, 16, 1024);
    const uint64_t k_desc0 = sdesc_sw128(smem_u32(sKV), 16, 1024);
    const uint64_t v_desc0 = sdesc_sw128(smem_u32(sKV) + C::K_BYTES, C::KV_SLAB, 1024);
    const uint32_t s_tm = tmem + q * C::QCOLS + C::TM_S;
    const uint32_t p_tm = tmem + q * C::QCOLS + C::TM_P;
    const uint32_t o_tm = tmem + q * C::QCOLS + C::TM_O;
    uint32_t t_base = 0, kv_base = 0, ui = 0;
    bool live = true;
    if (p.inject_stall) live = mbar_wait_warp(stall_bar, 0, kSiteInjected, abort_flag);   // runs out
    for (int u = blockIdx.x; u < p.units && live; u += gridDim.x, ++ui) {
      const uint32_t qb = ui % C::QBUF, qn = ui / C::QBUF;
      if (!mbar_wait_warp(&q_full[qb], qn & 1, kSiteQFull, abort_flag)) { live = false; break; }
      const uint64_t q_desc0 = q_desc00 + ((qb * NQ * C::Q_TILE) >> 4);
      for (int j = 0; j <= p.nkv; ++j) {
        if (j < p.nkv) {
          const uint32_t kv = kv_base + j, t = t_base + j;
          const uint32_t st = kv % C::STAGES, n = kv / C::STAGES;
          if (!mbar_wait_warp(&k_full[st], n & 1, kSiteKFull, abort_flag)) { live = false; break; }
          if (t >= 1 && !mbar_wait_warp(&s_free[q], (t - 1) & 1, kSiteSFull, abort_flag)) { live = false; break; }
          tc_fence_after();
          const uint64_t kd = k_desc0 + ((st * C::STAGE) >> 4);
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk)
            mma_ss(s_tm, q_desc0 + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                   kd + (((kk >> 2) * C::KV_SLAB + (kk & 3) * 32) >> 4), idesc_s, kk > 0 ? 1u : 0u);
          mma_commit(&s_full[q]);
        }
        if (j >= 1) {
          const uint32_t kv = kv_base + j - 1, t = t_base + j - 1;
          const uint32_t st = kv % C::STAGES, n = kv / C::STAGES;
          if (!mbar_wait_warp(&v_full[st], n & 1, kSiteVFull, abort_flag)) { live = false; break; }
          if (!mbar_wait_warp(&p_full[q], t & 1, kSitePFull, abort_flag)) { live = false; break; }
          tc_fence_after();
          const uint64_t vd = v_desc0 + ((st * C::STAGE) >> 4);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_ts(o_tm, p_tm + kk * 8, vd + ((kk * 2048) >> 4), idesc_pv, (j > 1 || kk > 0) ? 1u : 0u);
          mma_commit(&pv_done[q]);
          mma_commit(&kv_empty[st]);
        }
      }
      if (live) mma_commit(&q_empty[qb]);
      t_base += p.nkv;
      kv_base += p.nkv;
    }
    volatile uint32_t never = 0;
    mma_commit(&drain_bar[q]);
    mbar_wait_warp(&drain_bar[q], 0, kSitePvDone, &never);
  } else if (warp >= 4) {
    // ---------------------------- softmax, tile q -----------------------------
    if constexpr (NQ == 2) regs_inc<192>();
    const int q = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_tmem = tmem + q * C::QCOLS + C::TM_S + lane_off;
    const uint32_t p_tmem = tmem + q * C::QCOLS + C::TM_P + lane_off;
    const uint32_t o_tmem = tmem + q * C::QCOLS + C::TM_O + lane_off;
    const float c = p.c;
    uint32_t t = 0;        // tiles seen by this query-tile slot (all units)
    bool live = true;
    // The two query tiles run independently (own MMA warp, own handshakes,
    // Q double-buffered); started half a tile apart, their softmax phases
    // interleave on the SM instead of contending for the exponential unit.
    if (NQ == 2 && q == 1) live = __all_sync(0xffffffffu, mbar_wait(stagger, 0, kSiteSFull, abort_flag));
    for (int u = blockIdx.x; u < p.units && live; u += gridDim.x) {
      const int bh = u / p.tph, qg = u % p.tph;
      const int row = (qg * NQ + q) * 128 + r;
      float m_used = -INFINITY, rawmax = -INFINITY;
      for (int j = 0; j < p.nkv; ++j, ++t) {
        live = __all_sync(0xffffffffu, mbar_wait(&s_full[q], t & 1, kSiteSFull, abort_flag));
        if (!live) break;
        tc_fence_after();
        uint32_t v[BN];
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) tmem_ld_x32(s_tmem + cc * 32, v + cc * 32);
        tmem_wait_ld();
        reg_fence<BN>(v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[q]);
        const int valid = p.M - j * BN;
        if (valid < BN) {
#pragma unroll
          for (int k = 0; k < BN; ++k)
            if (k >= valid) v[k] = __float_as_uint(-INFINITY);
        }
        // row max: MAXCH independent three-input chains, then a small tree
        constexpr int MAXCH = 16;
        float acc[MAXCH];
#pragma unroll
        for (int i = 0; i < MAXCH; ++i) acc[i] = __uint_as_float(v[i]);
        int k0 = MAXCH;
#pragma unroll
        for (; k0 + 2 * MAXCH <= BN; k0 += 2 * MAXCH)
#pragma unroll
          for (int i = 0; i < MAXCH; ++i)
            acc[i] = fmax3(acc[i], __uint_as_float(v[k0 + i]), __uint_as_float(v[k0 + MAXCH + i]));
#pragma unroll
        for (int i = 0; i < MAXCH; ++i)
          if (k0 + i < BN) acc[i] = fmaxf(acc[i], __uint_as_float(v[k0 + i]));
#pragma unroll
        for (int w = MAXCH; w > 1; w /= 2)
#pragma unroll
          for (int i = 0; i < w / 2; ++i) acc[i] = fmaxf(acc[i], acc[i + w / 2]);
        const float mx = acc[0];
        rawmax = fmaxf(rawmax, mx);
        if (NQ == 2 && q == 0 && t == 0) {
          __syncwarp();
          if (lane == 0) mbar_arrive(stagger);
        }
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
        if (j > 0) {
          // P V of the previous tile must be done: P is reused and O may be rescaled
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
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) tmem_st_x16(p_tmem + cc * 16, pk + cc * 16);
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
