// qk_stats.cuh -- partially fused softmax, first kernel:
//   A = scale * Q K^T (fp32, stored), and per-row statistics (L_i, S_i).
//
// "Speed Is All You Need" (news summary, section on the three optimisations,
// partially fused softmax paragraph): a kernel maps the large matrix A to the
// vectors L and S (an N x 2 tensor) so that no full softmax runs over A; since
// that map has far fewer outputs than inputs, A is grouped into blocks, each
// block is reduced, and the partial results are reduced to the final ones.
//
// B200 design.  One persistent CTA per SM walks work units
// (b*H + h, 128-row tile, column split).  Inside a CTA:
//   warp 0      TMA producer: the unit's Q tile once, then a ring of K tiles;
//   warp 1      tcgen05 MMA issuer: S = Q K^T for one 128x128 block into one
//               of two TMEM accumulators (double-buffered);
//   warps 2..5  epilogue, one TMEM lane (= one query row) per thread: scales
//               the block, reduces it to a partial (m_b, s_b) pair, merges it
//               into the row's running pair, and streams the fp32 block to HBM
//               through swizzled shared-memory staging and TMA stores.
// When a row's columns are split over several units, each unit writes its
// merged pair to the workspace and bumps an arrival counter; the unit that
// arrives last merges all splits into LS, then zeroes the partials it read and
// the counter (no spinning), so a completed call leaves the workspace zero.
// When every unit has its own CTA and a row tile is split over at most 8 of
// them (small calls), the splits of a tile form a thread-block cluster
// instead: each leaves its merged pairs in its shared memory and, after a
// cluster barrier, CTA `rank` merges rows [rank 128 / k, (rank + 1) 128 / k)
// of all k splits in split order, read through distributed shared memory;
// no workspace is used.
//
// Store modes (template parameter AMODE):
//   kAF32Stats  A in fp32 and the row statistics (the partially fused form);
//   kAF32Only   A in fp32 only: the first pass of the three-pass form, whose
//               statistics come from a separate kernel that reads A back
//               (row_stats.cuh);
//   kAF16Stats  A rounded to fp16 (half the bytes of A written and read), the
//               statistics taken from the rounded values, so that the second
//               kernel's exp(A_ij - L_i) sum to exactly S_i's terms.
#pragma once

#include "sm100.cuh"

namespace sdattn {

enum QKMode : int { kAF32Stats = 0, kAF32Only = 1, kAF16Stats = 2 };

struct QKParams {
  int N, M, BH;
  int nrt;      // 128-row tiles per (b, h)
  int nb;       // 128-column blocks per row
  int nsplit;   // column splits per row tile
  int cbs;      // column blocks per split
  int units;    // BH * nrt * nsplit
  float scale;
  int cmerge;         // splits of a row tile merged across a cluster (one unit per CTA)
  float* LS;          // [BH][N][2]
  float2* part;       // [BH * nrt][128][nsplit]
  uint32_t* tickets;  // [BH * nrt]
};

template <int D>
struct QKCfg {
  static constexpr int DSLABS = (D + 63) / 64;    // 64-element (128 B) column slabs of Q / K
  static constexpr int KSTEPS = (D + 15) / 16;    // K=16 MMA steps (zero-padded past D)
  static constexpr int SLAB = 128 * 128;          // one slab of a 128-row tile, bytes
  static constexpr int KSTAGES = DSLABS == 1 ? 3 : 2;
  static constexpr int QBUF = 2;                  // Q double-buffered: the next unit's Q loads early
  static constexpr int EPI = DSLABS == 3 ? 1 : 2;   // epilogue warp groups (alternate 128-column blocks)
  static constexpr int NSTG = DSLABS == 1 ? 4 : 2;   // 4 KB staging buffers per epilogue warp
  static constexpr int STG = 4096;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBUF * DSLABS * SLAB;
  static constexpr int OFF_STG = OFF_K + KSTAGES * DSLABS * SLAB;
  static constexpr int OFF_MRG = OFF_STG + 4 * EPI * NSTG * STG;   // [2 slots][128 rows] float2
  static constexpr int OFF_CP = OFF_MRG + (EPI == 2 ? 2 * 128 * 8 : 0);   // [128 rows] float2: cluster merge
  static constexpr int OFF_BAR = OFF_CP + 128 * 8;
  static constexpr int NBAR = 2 * QBUF + 2 * KSTAGES + 4 + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;   // + misc words + alignment slack
  static constexpr int NTHREADS = 64 + 128 * EPI;
  static constexpr uint32_t TMEM_COLS = 256;
  static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ void qk_decode(const QKParams& p, int u, int& bh, int& rt, int& sp, int& cb0,
                                          int& cb1) {
  sp = u % p.nsplit;
  const int t = u / p.nsplit;
  rt = t % p.nrt;
  bh = t / p.nrt;
  cb0 = sp * p.cbs;
  cb1 = min(p.nb, cb0 + p.cbs);
}

// Merge of two (max, sum-of-exp) pairs: the pair of the union of their columns.
__device__ __forceinline__ void ms_merge(float& m, float& s, float m2, float s2) {
  constexpr float L2E = 1.4426950408889634f;
  if (m2 > m) {
    s = s * ex2_approx((m - m2) * L2E) + s2;
    m = m2;
  } else {
    s = s + s2 * ex2_approx((m2 - m) * L2E);
  }
}

template <int D, bool BF16, int AMODE>
__global__ void __launch_bounds__(QKCfg<D>::NTHREADS, 1)
    qk_stats_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmA, const QKParams p) {
  using C = QKCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sStg = smem + C::OFF_STG;
  float2* sMrg = reinterpret_cast<float2*>(smem + C::OFF_MRG);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;                // [QBUF]
  uint64_t* q_empty = q_full + C::QBUF;   // [QBUF]
  uint64_t* k_full = q_empty + C::QBUF;
  uint64_t* k_empty = k_full + C::KSTAGES;
  uint64_t* acc_full = k_empty + C::KSTAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain_bar = acc_empty + 2;
  uint32_t* misc = reinterpret_cast<uint32_t*>(drain_bar + 1);   // [0] tmem base, [1] abort, [2] last-split flag
  volatile uint32_t* abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::QBUF; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < C::KSTAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain_bar, 1);
    misc[1] = 0;
    misc[2] = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmA);
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
    if (lane == 0) {
      uint32_t kc = 0, nq = 0;   // K tiles and Q tiles issued
      bool live = true;
      for (int u = blockIdx.x; u < p.units && live; u += gridDim.x) {
        int bh, rt, sp, cb0, cb1;
        qk_decode(p, u, bh, rt, sp, cb0, cb1);
        const uint32_t qb = nq % C::QBUF, qn = nq / C::QBUF;
        if (!mbar_wait(&q_empty[qb], (qn & 1) ^ 1, kSiteQEmpty, abort_flag)) { live = false; break; }
        ++nq;
        mbar_arrive_expect_tx(&q_full[qb], C::DSLABS * C::SLAB);
        for (int s = 0; s < C::DSLABS; ++s)
          tma_load_3d(sQ + (qb * C::DSLABS + s) * C::SLAB, &tmQ, 64 * s, rt * 128, bh, &q_full[qb]);
        for (int cb = cb0; cb < cb1; ++cb, ++kc) {
          const uint32_t st = kc % C::KSTAGES, n = kc / C::KSTAGES;
          if (!mbar_wait(&k_empty[st], (n & 1) ^ 1, kSiteKEmpty, abort_flag)) { live = false; break; }
          mbar_arrive_expect_tx(&k_full[st], C::DSLABS * C::SLAB);
          for (int s = 0; s < C::DSLABS; ++s)
            tma_load_3d(sK + (st * C::DSLABS + s) * C::SLAB, &tmK, 64 * s, cb * 128, bh, &k_full[st]);
        }
      }
      // Let every load this thread issued land before the CTA can exit.
      volatile uint32_t never = 0;
      for (uint32_t qb = 0; qb < C::QBUF && qb < nq; ++qb) {
        const uint32_t uses = (nq - qb + C::QBUF - 1) / C::QBUF;
        mbar_wait(&q_full[qb], (uses - 1) & 1, kSiteQFull, &never);
      }
      for (uint32_t st = 0; st < C::KSTAGES && st < kc; ++st) {
        const uint32_t uses = (kc - st + C::KSTAGES - 1) / C::KSTAGES;
        mbar_wait(&k_full[st], (uses - 1) & 1, kSiteKFull, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    {   // the whole warp runs the loop; one elected lane issues
      constexpr uint32_t idesc = idesc_f16(128, 128, BF16, false, false);
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK);
      uint32_t kc = 0, ac = 0, ui = 0;
      bool live = true;
      for (int u = blockIdx.x; u < p.units && live; u += gridDim.x, ++ui) {
        int bh, rt, sp, cb0, cb1;
        qk_decode(p, u, bh, rt, sp, cb0, cb1);
        const uint32_t qb = ui % C::QBUF, qn = ui / C::QBUF;
        if (!mbar_wait_warp(&q_full[qb], qn & 1, kSiteQFull, abort_flag)) { live = false; break; }
        tc_fence_after();
        for (int cb = cb0; cb < cb1; ++cb, ++kc, ++ac) {
          const uint32_t st = kc % C::KSTAGES, n = kc / C::KSTAGES;
          const uint32_t ab = ac & 1, na = ac >> 1;
          if (!mbar_wait_warp(&k_full[st], n & 1, kSiteKFull, abort_flag)) { live = false; break; }
          if (!mbar_wait_warp(&acc_empty[ab], (na & 1) ^ 1, kSiteAccEmpty, abort_flag)) { live = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem + ab * 128;
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const uint32_t off = (kk >> 2) * C::SLAB + (kk & 3) * 32;
            const uint64_t ad = sdesc_sw128(q_base + qb * C::DSLABS * C::SLAB + off, 16, 1024);
            const uint64_t bd = sdesc_sw128(k_base + st * C::DSLABS * C::SLAB + off, 16, 1024);
            mma_ss(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&k_empty[st]);
          mma_commit(&acc_full[ab]);
        }
        if (live) mma_commit(&q_empty[qb]);
      }
      // Wait until every MMA this thread issued has finished.
      volatile uint32_t never = 0;
      mma_commit(drain_bar);
      mbar_wait_warp(drain_bar, 0, kSiteAccFull, &never);
    }
  } else {
    // ------------------------------ epilogue ----------------------------------
    constexpr float L2E = 1.4426950408889634f;
    const int quarter = warp & 3;                 // TMEM lanes quarter*32 .. +31
    const int row_local = quarter * 32 + lane;    // row of the 128-row tile
    const int e = (warp - 2) >> 2;                // epilogue group: with two, group e takes accumulator e
    uint8_t* stg = sStg + (warp - 2) * C::NSTG * C::STG;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t ac = 0, sc = 0, ui = 0;
    bool live = true;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++ui) {
      int bh, rt, sp, cb0, cb1;
      qk_decode(p, u, bh, rt, sp, cb0, cb1);
      float m_run = -INFINITY, s_run = 0.f;
      for (int cb = cb0; cb < cb1 && live; ++cb, ++ac) {
        const uint32_t ab = ac & 1, na = ac >> 1;
        if (C::EPI == 2 && static_cast<int>(ab) != e) continue;
        live = __all_sync(0xffffffffu, mbar_wait(&acc_full[ab], na & 1, kSiteAccFull, abort_flag));
        if (!live) break;
        tc_fence_after();
        const int col0 = cb * 128;
        const int valid = min(128, p.M - col0);
        // One half (64 columns) of the block: scale (and round, for fp16 A),
        // reduce to a partial (m, s) over its valid columns and merge it into
        // the row's running pair, then stream it to A in 128-byte chunks per
        // row (32 fp32 or 64 fp16 columns per chunk).
        auto half = [&](const uint32_t* hv, int h) {
          // scale, two columns per instruction (f32x2: each product rounded as alone)
          float a[64];
          const uint64_t sc2 = f2_pack(p.scale, p.scale);
#pragma unroll
          for (int k = 0; k < 64; k += 2)
            f2_unpack(f2_mul(f2_pack(__uint_as_float(hv[k]), __uint_as_float(hv[k + 1])), sc2), a[k], a[k + 1]);
          if constexpr (AMODE == kAF16Stats) {
            // A is stored in fp16: the statistics are taken from the stored values
#pragma unroll
            for (int k = 0; k < 64; k += 2) {
              const float2 r = __half22float2(__floats2half2_rn(a[k], a[k + 1]));
              a[k] = r.x;
              a[k + 1] = r.y;
            }
          }
          const int hvalid = valid - 64 * h;   // valid columns of this half (may be <= 0)
          if constexpr (AMODE != kAF32Only) {
            if (hvalid > 0) {
              // eight independent chains for the max and for the sum, then a tree
              float mx8[8], sm8[8];
              if (hvalid >= 64) {
#pragma unroll
                for (int i = 0; i < 8; ++i) mx8[i] = fmax3(a[i], a[8 + i], a[16 + i]);
#pragma unroll
                for (int k = 24; k < 64; k += 16)
#pragma unroll
                  for (int i = 0; i < 8; ++i) mx8[i] = fmax3(mx8[i], a[k + i], (k + 8 + i < 64) ? a[k + 8 + i] : a[k + i]);
              } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
                for (int k = 0; k < 64; ++k) mx8[k & 7] = (k < hvalid) ? fmaxf(mx8[k & 7], a[k]) : mx8[k & 7];
              }
              const float mb =
                  fmaxf(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], fmax3(mx8[5], mx8[6], mx8[7])));
              const float nmb = -mb * L2E;
#pragma unroll
              for (int i = 0; i < 8; ++i) sm8[i] = 0.f;
              if (hvalid >= 64) {
                // column k adds into sum k % 8 in column order, as the scalar
                // form below, two columns per f32x2 step
                const uint64_t l2e2 = f2_pack(L2E, L2E), nmb2 = f2_pack(nmb, nmb);
                uint64_t s2[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) s2[i] = f2_pack(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < 64; k += 2) {
                  float x0, x1;
                  f2_unpack(f2_fma(f2_pack(a[k], a[k + 1]), l2e2, nmb2), x0, x1);
                  s2[(k >> 1) & 3] = f2_add(s2[(k >> 1) & 3], f2_pack(ex2_approx(x0), ex2_approx(x1)));
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) f2_unpack(s2[i], sm8[2 * i], sm8[2 * i + 1]);
              } else {
#pragma unroll
                for (int k = 0; k < 64; ++k) sm8[k & 7] += (k < hvalid) ? ex2_approx(fmaf(a[k], L2E, nmb)) : 0.f;
              }
              const float sb = ((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) + ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7]));
              ms_merge(m_run, s_run, mb, sb);
            }
          }
          constexpr int CC = AMODE == kAF16Stats ? 64 : 32;   // columns per chunk
#pragma unroll
          for (int c = 0; c < 64 / CC; ++c) {
            const int col = col0 + 64 * h + CC * c;
            if (col >= p.M) break;
            uint8_t* buf = stg + (sc % C::NSTG) * C::STG;
            if (lane == 0) bulk_wait_read<C::NSTG - 1>();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              uint4 w;
              if constexpr (AMODE == kAF16Stats) {
                const float* s8 = a + CC * c + 8 * j;   // already fp16 values: packing is exact
                w = make_uint4(pack2<false>(s8[0], s8[1]), pack2<false>(s8[2], s8[3]), pack2<false>(s8[4], s8[5]),
                               pack2<false>(s8[6], s8[7]));
              } else {
                const float* s4 = a + CC * c + 4 * j;
                w = make_uint4(__float_as_uint(s4[0]), __float_as_uint(s4[1]), __float_as_uint(s4[2]),
                               __float_as_uint(s4[3]));
              }
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) = w;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tmA, buf, col, rt * 128 + quarter * 32, bh);
              bulk_commit();
            }
            ++sc;
          }
        };
        // The accumulator in two 64-column loads: the second lands while the
        // first half is reduced and staged.
        uint32_t v0[64], v1[64];
        tmem_ld_x64(tmem + ab * 128 + lane_off, v0);
        tmem_wait_ld();
        reg_fence<64>(v0);
        tmem_ld_x64(tmem + ab * 128 + 64 + lane_off, v1);
        half(v0, 0);
        tmem_wait_ld();
        reg_fence<64>(v1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        half(v1, 1);
      }
      if constexpr (AMODE == kAF32Only) continue;   // no statistics to finish
      // ---- the two groups' pairs merge; group 0 finishes the unit ----
      if (C::EPI == 2) {
        float2* slot = sMrg + (ui & 1) * 128;
        if (e == 1) slot[row_local] = make_float2(m_run, s_run);
        named_bar_sync(1, 256);
        if (e == 1) continue;
        const float2 o = slot[row_local];
        ms_merge(m_run, s_run, o.x, o.y);
      }
      // ---- unit result: the merged pair of this split ----
      const int row = rt * 128 + row_local;
      if (p.cmerge) {
        reinterpret_cast<float2*>(smem + C::OFF_CP)[row_local] = make_float2(m_run, s_run);
      } else if (p.nsplit == 1) {
        if (live && row < p.N)
          *reinterpret_cast<float2*>(p.LS + 2 * (static_cast<int64_t>(bh) * p.N + row)) = make_float2(m_run, s_run);
      } else {
        const int64_t tile = static_cast<int64_t>(bh) * p.nrt + rt;
        if (live) p.part[(tile * 128 + row_local) * p.nsplit + sp] = make_float2(m_run, s_run);
        named_bar_sync(2, 128);
        if (threadIdx.x == 64) {
          uint32_t last = 0;
          if (live) {
            __threadfence();
            last = (atomicAdd(&p.tickets[tile], 1u) == static_cast<uint32_t>(p.nsplit - 1)) ? 1u : 0u;
          }
          misc[2] = last;
        }
        named_bar_sync(2, 128);
        if (misc[2]) {
          __threadfence();
          float m = -INFINITY, s = 0.f;
          const float2* pr = p.part + (tile * 128 + row_local) * p.nsplit;
          for (int k = 0; k < p.nsplit; ++k) {
            const float2 q = __ldcg(pr + k);
            ms_merge(m, s, q.x, q.y);
          }
          // leave the workspace all-zero for the next call, whatever its shape
          for (int k = 0; k < p.nsplit; ++k) __stcg(const_cast<float2*>(pr) + k, make_float2(0.f, 0.f));
          if (row < p.N)
            *reinterpret_cast<float2*>(p.LS + 2 * (static_cast<int64_t>(bh) * p.N + row)) = make_float2(m, s);
          if (threadIdx.x == 64) p.tickets[tile] = 0u;
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  if (p.cmerge) {
    // every thread of every CTA of the cluster passes both barriers, also
    // after a wait ran out (the results are then wrong, and the error word says so)
    __syncwarp();
    cluster_sync();
    if (warp >= 2 && warp < 6) {   // the first epilogue group merges this CTA's share of the rows
      int bh, rt, sp, cb0, cb1;
      qk_decode(p, blockIdx.x, bh, rt, sp, cb0, cb1);
      const uint32_t k = static_cast<uint32_t>(p.nsplit), rank = cluster_rank();
      const int r0 = static_cast<int>(rank) * 128 / p.nsplit, r1 = static_cast<int>(rank + 1) * 128 / p.nsplit;
      const float* cp = reinterpret_cast<const float*>(smem + C::OFF_CP);
      for (int rr = r0 + static_cast<int>(threadIdx.x) - 64; rr < r1; rr += 128) {
        const int row = rt * 128 + rr;
        if (row >= p.N) continue;
        float m = -INFINITY, sum = 0.f;
        for (uint32_t j = 0; j < k; ++j) ms_merge(m, sum, ld_cluster_f32(cp + 2 * rr, j), ld_cluster_f32(cp + 2 * rr + 1, j));
        *reinterpret_cast<float2*>(p.LS + 2 * (static_cast<int64_t>(bh) * p.N + row)) = make_float2(m, sum);
      }
    }
    __syncwarp();
    cluster_sync();   // no CTA leaves while another may still read its pairs
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sdattn
