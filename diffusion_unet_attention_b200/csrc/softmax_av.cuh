// softmax_av.cuh -- partially fused softmax, second kernel: the softmax
// normalisation fused with the multiplication by V,
//   O_i = (sum_j exp(A_ij - L_i) V_j) / S_i.
//
// "Speed Is All You Need" (news summary, section on the three optimisations,
// partially fused softmax paragraph): once L and S are known, the softmax is
// fused with the matrix multiplication by V, so no normalised probability
// matrix is ever written.
//
// B200 design.  One persistent CTA per SM walks (b*H + h, 128-row tile) units.
//   warp 0      TMA producer: a ring of (A block 128 x 64, fp32 or fp16, and V
//               block 64 x d) stages, 128-byte swizzled;
//   warps 2..   RG groups of four row warps, one query row per thread;
//               group g takes the CTA's key blocks c with c % RG == g: reads
//               its 64 scores of the block from shared memory, computes
//               p = exp(a - L_i) in registers, packs p to 16 bits and writes
//               it to tensor memory (P buffer g);
//   warp 1      tcgen05 MMA issuer: O += P V with P taken from tensor memory
//               and V from shared memory, O accumulated in tensor memory
//               (accumulators rotating over row tiles, so one tile's
//               epilogue overlaps the next tile's products).
// Several row warps per scheduler keep the exponentials and shared-memory
// reads of one block in flight while another block's tensor-memory store
// and hand-offs complete.  Group (tile index % RG) runs a tile's epilogue:
// it scales O by 1/S_i and stores it, each warp's 32 consecutive rows through
// its own shared-memory slice as consecutive 16-byte chunks.  Every barrier
// that a group waits on (its stages of the ring, its P buffer, the O
// accumulators whose epilogues it runs) is used by that group alone, in
// order, so no wait can match the parity of an earlier phase.
// Since L_i is final, no rescaling is ever needed.
//
// Small grids (row tiles filling under half the SMs): a thread-block cluster
// of k CTAs shares each row tile, CTA r taking key blocks [r nkb / k,
// (r + 1) nkb / k).  Since L_i and S_i are final, the k partial products
// sum_j exp(A_ij - L_i) V_j simply add: each CTA leaves its fp32 partial rows
// in its own shared memory, and after a cluster barrier CTA r sums rows
// [r 128 / k, (r + 1) 128 / k) of all k partials (read through distributed
// shared memory, in rank order, so the result does not depend on timing),
// scales them by 1/S_i and stores them.
#pragma once

#include "sm100.cuh"

namespace sdattn {

struct AVParams {
  int N, M, BH;
  int nrt;    // 128-row tiles per (b, h)
  int nkb;    // 64-key blocks
  int units;  // BH * nrt
  int ksplit; // CTAs of a cluster sharing one row tile's key blocks (1: persistent grid, whole tiles)
  const float* LS;
  void* O;
};

template <int D, bool AF16 = false>
struct AVCfg {
  static constexpr int DSLABS = (D + 63) / 64;
  static constexpr int PVN = DSLABS * 64;              // MMA N (head width padded to 64)
  static constexpr int BK = 64;                        // keys per block
  static constexpr int A_BYTES = 128 * BK * (AF16 ? 2 : 4);   // fp32: two 16 KB boxes of 32 columns; fp16: one of 64
  static constexpr int V_SLAB = BK * 128;              // 8 KB: 64 keys x 64 elements
  static constexpr int V_BYTES = DSLABS * V_SLAB;
  static constexpr int STAGE_BYTES = A_BYTES + V_BYTES;
  // Row-warp groups: group g takes the key blocks c with c % RG == g.  The
  // ring's stage c % STAGES is then refilled for one group only (STAGES is a
  // multiple of RG), so a group waits on a stage at most one load ahead of
  // what it consumed there itself.  Were consecutive loads of a stage taken by
  // different groups, a group could wait for the load after next while the
  // next is still in flight, and the phase parity it waits for would match
  // the phase already completed.
  // The O accumulators rotate over row tiles the same way: tile ui uses
  // accumulator ui % NOB and group ui % RG runs its epilogue, so NOB is a
  // multiple of RG and an accumulator's epilogues are always one group's.
  // Measured at 64x64: with fp32 A two groups keep four stages in flight,
  // three only three stages (slower); fp16 A fits six stages either way and
  // gains from the third group (d = 160 has no tensor memory for a third O).
  static constexpr int RG = (AF16 && D <= 80) ? 3 : 2;
  static constexpr int NPB = RG == 1 ? 2 : RG;       // P buffers in tensor memory (group g uses buffer g)
  static constexpr int NOB = RG == 1 ? 2 : RG;       // O accumulators
  static constexpr int NTHREADS = 64 + 128 * RG;
  static constexpr int OCW = (D <= 80 || RG > 2) ? 40 : 80;    // O columns per coalesced store pass
  static constexpr int STG_BYTES = 4 * RG * RowStage<OCW>::BYTES;   // one store slice per row warp
  static constexpr int FIXED = STG_BYTES + (4 * 6 + 2 * NPB + 2 * NOB + 1) * 8 + 16 + 1024;
  static constexpr int STAGES_FIT = (232448 - FIXED) / STAGE_BYTES;
  static constexpr int STAGES = (STAGES_FIT < 6 ? STAGES_FIT : 6) / RG * RG;
  static_assert(STAGES >= 2 && STAGES % RG == 0, "each ring stage serves one row group");
  static constexpr int OFF_A = 0;
  static constexpr int OFF_V = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_STG = OFF_V + STAGES * V_BYTES;
  // key split: 128 partial rows of D fp32 (padded: eight lanes writing one
  // 16-byte chunk of eight rows hit eight bank groups) over the stage buffers
  static constexpr int PPITCH = D + 4;
  static_assert(128 * PPITCH * 4 <= OFF_STG, "partial rows fit in the stage buffers");
  static constexpr int OFF_BAR = OFF_STG + STG_BYTES;
  static constexpr int NBAR = 4 * STAGES + 2 * NPB + 2 * NOB + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static constexpr uint32_t TM_P = 0;      // NPB P buffers of 32 columns (128 x 64 16-bit)
  static constexpr uint32_t TM_O = (32 * NPB + 63) / 64 * 64;   // NOB O accumulators, PVN columns each
  static constexpr uint32_t TMEM_COLS = TM_O + NOB * PVN <= 256 ? 256 : 512;
  static_assert(TM_O + NOB * PVN <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
};

template <int D, bool BF16, bool AF16>
__global__ void __launch_bounds__(AVCfg<D, AF16>::NTHREADS, 1)
    softmax_av_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmV,
                      const AVParams p) {
  using C = AVCfg<D, AF16>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* a_full = bars;
  uint64_t* a_empty = a_full + C::STAGES;
  uint64_t* v_full = a_empty + C::STAGES;
  uint64_t* v_empty = v_full + C::STAGES;
  uint64_t* p_full = v_empty + C::STAGES;   // [NPB] per P buffer
  uint64_t* p_empty = p_full + C::NPB;
  uint64_t* o_full = p_empty + C::NPB;      // [NOB] per O accumulator
  uint64_t* o_empty = o_full + C::NOB;      // [NOB] the accumulator's epilogue has read it
  uint64_t* drain_bar = o_empty + C::NOB;
  uint32_t* misc = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile uint32_t* abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 4);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < C::NPB; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&p_empty[i], 1);
    }
    for (int i = 0; i < C::NOB; ++i) {
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 4);
    }
    mbar_init(drain_bar, 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmA);
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
  // Everything above touched only this CTA's own resources; global inputs and
  // outputs are used only once the previous kernel of the stream is complete.
  grid_dependency_wait();
  grid_launch_dependents();

  // work: whole row tiles over a persistent grid, or (ksplit > 1) one row
  // tile per cluster, CTA `rank` taking its share of the key blocks
  const bool split = p.ksplit > 1;
  const int u_first = split ? static_cast<int>(blockIdx.x) / p.ksplit : static_cast<int>(blockIdx.x);
  const int u_step = split ? p.units : static_cast<int>(gridDim.x);
  const int kb0 = split ? static_cast<int>(cluster_rank()) * p.nkb / p.ksplit : 0;
  const int kb1 = split ? (static_cast<int>(cluster_rank()) + 1) * p.nkb / p.ksplit : p.nkb;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      uint32_t c = 0;
      bool live = true;
      for (int u = u_first; u < p.units && live; u += u_step) {
        const int bh = u / p.nrt, rt = u % p.nrt;
        for (int kb = kb0; kb < kb1; ++kb, ++c) {
          const uint32_t st = c % C::STAGES, n = c / C::STAGES;
          if (!mbar_wait(&a_empty[st], (n & 1) ^ 1, kSiteAEmpty, abort_flag)) { live = false; break; }
          if (!mbar_wait(&v_empty[st], (n & 1) ^ 1, kSiteVEmpty, abort_flag)) { live = false; break; }
          mbar_arrive_expect_tx(&a_full[st], C::A_BYTES);
          tma_load_3d(sA + st * C::A_BYTES, &tmA, kb * C::BK, rt * 128, bh, &a_full[st]);
          if constexpr (!AF16)
            tma_load_3d(sA + st * C::A_BYTES + C::A_BYTES / 2, &tmA, kb * C::BK + 32, rt * 128, bh, &a_full[st]);
          mbar_arrive_expect_tx(&v_full[st], C::V_BYTES);
          for (int s = 0; s < C::DSLABS; ++s)
            tma_load_3d(sV + st * C::V_BYTES + s * C::V_SLAB, &tmV, 64 * s, kb * C::BK, bh, &v_full[st]);
        }
      }
      volatile uint32_t never = 0;
      for (uint32_t st = 0; st < C::STAGES && st < c; ++st) {
        const uint32_t uses = (c - st + C::STAGES - 1) / C::STAGES;
        mbar_wait(&a_full[st], (uses - 1) & 1, kSiteAFull, &never);
        mbar_wait(&v_full[st], (uses - 1) & 1, kSiteVFull, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    {   // the whole warp runs the loop; one elected lane issues
      constexpr uint32_t idesc = idesc_f16(128, C::PVN, BF16, false, true);
      const uint32_t v_base = smem_u32(sV);
      uint32_t c = 0, pc = 0, ui = 0;
      bool live = true;
      for (int u = u_first; u < p.units && live; u += u_step, ++ui) {
        const uint32_t ob = ui % C::NOB;
        // the epilogue of tile ui - NOB must have read this accumulator
        if (ui >= C::NOB && !mbar_wait_warp(&o_empty[ob], (ui / C::NOB - 1) & 1, kSiteOFull, abort_flag)) {
          live = false;
          break;
        }
        const uint32_t o_tm = tmem + C::TM_O + ob * C::PVN;
        for (int kb = kb0; kb < kb1; ++kb, ++c, ++pc) {
          const uint32_t st = c % C::STAGES, n = c / C::STAGES;
          const uint32_t pb = pc % C::NPB, np = pc / C::NPB;
          if (!mbar_wait_warp(&v_full[st], n & 1, kSiteVFull, abort_flag)) { live = false; break; }
          if (!mbar_wait_warp(&p_full[pb], np & 1, kSitePFull, abort_flag)) { live = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            // V block, MN-major: 16 keys = two 8-row groups (SBO 1024 B apart);
            // 64-element column slabs C::V_SLAB bytes apart (LBO).
            const uint64_t bd = sdesc_sw128(v_base + st * C::V_BYTES + kk * 2048, C::V_SLAB, 1024);
            mma_ts(o_tm, tmem + C::TM_P + pb * 32 + kk * 8, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&v_empty[st]);
          mma_commit(&p_empty[pb]);
        }
        if (live) mma_commit(&o_full[ob]);
      }
      volatile uint32_t never = 0;
      mma_commit(drain_bar);
      mbar_wait_warp(drain_bar, 0, kSiteOFull, &never);
    }
  } else {
    // --------------------- softmax rows and epilogue --------------------------
    constexpr float L2E = 1.4426950408889634f;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                // row of the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t g = static_cast<uint32_t>(warp - 2) >> 2;   // row group: key blocks c with c % RG == g
    uint32_t c = 0, pc = 0, ui = 0;
    bool live = true;
    for (int u = u_first; u < p.units && live; u += u_step, ++ui) {
      const int bh = u / p.nrt, rt = u % p.nrt;
      const int row = rt * 128 + r;
      float Lr = 0.f, Sr = 1.f;
      if (row < p.N) {
        const float2 ls = *reinterpret_cast<const float2*>(p.LS + 2 * (static_cast<int64_t>(bh) * p.N + row));
        Lr = ls.x;
        Sr = ls.y;
      }
      const float nl = -Lr * L2E;
      for (int kb = kb0; kb < kb1; ++kb, ++c, ++pc) {
        if (c % C::RG != g) continue;   // another group's block
        const uint32_t st = c % C::STAGES, n = c / C::STAGES;
        live = __all_sync(0xffffffffu, mbar_wait(&a_full[st], n & 1, kSiteAFull, abort_flag));
        if (!live) break;
        // this row's 64 scores, 128-byte swizzled rows: two 32-column fp32
        // boxes, or one 64-column fp16 box
        uint32_t pk[32];
        const int valid = p.M - kb * C::BK;           // columns of this block inside [0, M)
        if constexpr (AF16) {
          const uint8_t* rowp = sA + st * C::A_BYTES + r * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 h = *reinterpret_cast<const uint4*>(rowp + ((j ^ (r & 7)) << 4));
            const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
              const int k = 8 * j + 2 * i;
              float e0 = ex2_approx(fmaf(a.x, L2E, nl));
              float e1 = ex2_approx(fmaf(a.y, L2E, nl));
              if (valid < C::BK) {
                e0 = (k + 0 < valid) ? e0 : 0.f;
                e1 = (k + 1 < valid) ? e1 : 0.f;
              }
              pk[k / 2] = pack2<BF16>(e0, e1);
            }
          }
        } else {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint8_t* rowp = sA + st * C::A_BYTES + h * (C::A_BYTES / 2) + r * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 a = *reinterpret_cast<const float4*>(rowp + ((j ^ (r & 7)) << 4));
              const int k = h * 32 + 4 * j;
              float e0 = ex2_approx(fmaf(a.x, L2E, nl));
              float e1 = ex2_approx(fmaf(a.y, L2E, nl));
              float e2 = ex2_approx(fmaf(a.z, L2E, nl));
              float e3 = ex2_approx(fmaf(a.w, L2E, nl));
              if (valid < C::BK) {
                e0 = (k + 0 < valid) ? e0 : 0.f;
                e1 = (k + 1 < valid) ? e1 : 0.f;
                e2 = (k + 2 < valid) ? e2 : 0.f;
                e3 = (k + 3 < valid) ? e3 : 0.f;
              }
              pk[k / 2 + 0] = pack2<BF16>(e0, e1);
              pk[k / 2 + 1] = pack2<BF16>(e2, e3);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_empty[st]);
        const uint32_t pb = pc % C::NPB, np = pc / C::NPB;
        live = __all_sync(0xffffffffu, mbar_wait(&p_empty[pb], (np & 1) ^ 1, kSitePEmpty, abort_flag));
        if (!live) break;
        tc_fence_after();
        tmem_st_x16(tmem + C::TM_P + pb * 32 + lane_off, pk);
        tmem_st_x16(tmem + C::TM_P + pb * 32 + 16 + lane_off, pk + 16);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[pb]);
      }
      if (!live) break;
      // ---- epilogue: O_i / S_i, by group ui % RG ----
      if (ui % C::RG != g) continue;
      const uint32_t ob = ui % C::NOB;
      const uint32_t o_tm = tmem + C::TM_O + ob * C::PVN + lane_off;
      live = __all_sync(0xffffffffu, mbar_wait(&o_full[ob], (ui / C::NOB) & 1, kSiteOFull, abort_flag));
      if (!live) break;
      tc_fence_after();
      if (p.ksplit > 1) {
        // this CTA's share of the key range: unnormalised fp32 rows into shared
        // memory (the stage buffers are idle now), summed by the cluster below
        float* prow = reinterpret_cast<float*>(smem) + r * C::PPITCH;
#pragma unroll
        for (int c8 = 0; c8 < D / 8; ++c8) {
          uint32_t o[8];
          tmem_ld_x8(o_tm + c8 * 8, o);
          tmem_wait_ld();
          reg_fence<8>(o);
          *reinterpret_cast<uint4*>(prow + c8 * 8) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(prow + c8 * 8 + 4) = make_uint4(o[4], o[5], o[6], o[7]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_empty[ob]);
        continue;
      }
      const float inv = 1.f / Sr;
      const int row_w = row - lane;   // the warp's first row
      uint8_t* owarp = reinterpret_cast<uint8_t*>(p.O) + (static_cast<int64_t>(bh) * p.N + row_w) * D * 2;
      // each row warp has a slice of its own: with one key block per tile the
      // groups finish consecutive tiles at the same time
      uint8_t* slice = smem + C::OFF_STG + (warp - 2) * RowStage<C::OCW>::BYTES;
#pragma unroll
      for (int pass = 0; pass < D / C::OCW; ++pass) {
        uint32_t o[C::OCW];
#pragma unroll
        for (int c8 = 0; c8 < C::OCW / 8; ++c8) tmem_ld_x8(o_tm + pass * C::OCW + c8 * 8, o + c8 * 8);
        tmem_wait_ld();
        reg_fence<C::OCW>(o);
        if (pass == D / C::OCW - 1) {
          // the accumulator is read: tile ui + NOB may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_empty[ob]);
        }
#pragma unroll
        for (int c8 = 0; c8 < C::OCW / 8; ++c8) {
          const uint32_t* oc = o + c8 * 8;
          uint4 w;
          w.x = pack2<BF16>(__uint_as_float(oc[0]) * inv, __uint_as_float(oc[1]) * inv);
          w.y = pack2<BF16>(__uint_as_float(oc[2]) * inv, __uint_as_float(oc[3]) * inv);
          w.z = pack2<BF16>(__uint_as_float(oc[4]) * inv, __uint_as_float(oc[5]) * inv);
          w.w = pack2<BF16>(__uint_as_float(oc[6]) * inv, __uint_as_float(oc[7]) * inv);
          stage_put<C::OCW>(slice, lane, c8, w);
        }
        stage_flush<C::OCW>(slice, lane, owarp + pass * C::OCW * 2, D * 2, p.N - row_w);
      }
      tc_fence_before();
    }
  }

  if (p.ksplit > 1) {
    // every thread of every CTA of the cluster passes both barriers, also
    // after a wait ran out (the results are then wrong, and the error word says so)
    const uint32_t k = static_cast<uint32_t>(p.ksplit);
    const uint32_t rank = cluster_rank();
    const int bh = u_first / p.nrt, rt = u_first % p.nrt;
    __syncwarp();
    cluster_sync();
    if (warp >= 2) {
      const int r0 = static_cast<int>(rank) * 128 / static_cast<int>(k);
      const int r1 = static_cast<int>(rank + 1) * 128 / static_cast<int>(k);
      const float* part0 = reinterpret_cast<const float*>(smem);
      for (int it = threadIdx.x - 64; it < (r1 - r0) * (D / 8); it += 128 * C::RG) {
        const int rr = r0 + it / (D / 8), c8 = it % (D / 8);
        const int row = rt * 128 + rr;
        if (row >= p.N) continue;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (uint32_t j = 0; j < k; ++j) {
          const float4 a = ld_cluster_f32x4(part0 + rr * C::PPITCH + c8 * 8, j);
          const float4 b = ld_cluster_f32x4(part0 + rr * C::PPITCH + c8 * 8 + 4, j);
          acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
          acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
        }
        const int64_t grow = static_cast<int64_t>(bh) * p.N + row;
        const float inv = 1.f / p.LS[2 * grow + 1];
        uint4 w;
        w.x = pack2<BF16>(acc[0] * inv, acc[1] * inv);
        w.y = pack2<BF16>(acc[2] * inv, acc[3] * inv);
        w.z = pack2<BF16>(acc[4] * inv, acc[5] * inv);
        w.w = pack2<BF16>(acc[6] * inv, acc[7] * inv);
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.O) + grow * D * 2 + c8 * 16) = w;
      }
    }
    __syncwarp();
    cluster_sync();   // no CTA leaves while another may still read its partial rows
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sdattn
