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
// 128-row query tiles) units, whole, or, when the units do not fill the last
// wave, as equal shares of all (unit, key tile) pairs; a unit cut between two
// CTAs is merged by one of its halves (flash_cut_epilogue).  Roles:
//   warp 0            TMA producer: the unit's NQ Q tiles, then a ring of
//                     (K tile, V tile) stages, 128-byte swizzled, no multicast;
//   warp 1 + q        tcgen05 MMA issuer for query tile q: S = Q K^T into
//                     tensor memory; once the softmax has written P (16-bit,
//                     its own tensor-memory buffer) O += P V, with O
//                     accumulated in tensor memory;
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
//
// Precise variant (template flag PREC; two query tiles per CTA only with
// 96-key tiles, which leave room in tensor memory for both tiles' S, P, P's
// residual and O): P is carried
// as a 16-bit high part plus the 16-bit rounding of its residual, P V runs as
// two MMAs into the same accumulator, and O is written in fp32.  Both parts
// have the input's type, so with bf16 inputs (8-bit mantissas) the weights
// keep about 16 bits and the result meets the fp16 accuracy bar; a bf16 O
// alone would round each output by up to 2^-9 of its value.
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
  // Split schedule (split != 0): CTA b of G = gridDim.x takes the contiguous
  // range [b W / G, (b + 1) W / G) of the W = units * nkv (unit, key tile)
  // pairs in unit-major order.  The host splits only when W / G >= nkv, so a
  // unit is cut at most once, between two neighbouring CTAs: the head half
  // (its first key tiles) ends CTA b's range, the tail half starts CTA b+1's.
  // One of the two halves merges them, settled on a counter in `tickets`,
  // from the other's partial rows in `part` (flash_cut_epilogue).  Without
  // the split CTA b takes the whole units b, b + G, b + 2G, ...
  int split;
  uint32_t* tickets;   // [G * NQ], all zero on entry and on exit
  float* part;         // [G * NQ][2][ROWF / 4][128 rows][4]: column quads, rows contiguous
  // Small grids (ksplit > 1, one query tile per CTA): a thread-block cluster
  // of ksplit CTAs shares unit blockIdx.x / ksplit, CTA `rank` taking key
  // tiles [rank nkv / ksplit, (rank + 1) nkv / ksplit); the partial rows are
  // merged across the cluster through distributed shared memory.
  int ksplit;
};

// The work of one CTA as a list of segments: key tiles [j0, j1) of unit u.
// Split schedule: a range [u_first:j_first, u_last:j_last) is walked as the
// head half of unit u_last (its key tiles [0, j_last), when there is one)
// first, then units u_first .. u_last - 1, the first from key tile j_first.
// With the cut units first, both halves of a cut unit finish early in their
// CTAs' runs and every CTA ends on a whole unit: the merge of two halves is
// never the last thing a CTA does.
// KS: the kernel may run cluster-split units (one query tile per CTA only);
// the check is compiled out of the two-tile kernel.
template <bool KS>
struct FlashSegments {
  int u, j0, j1;
  int u_first, j_first, u_last;
  __device__ __forceinline__ explicit FlashSegments(const FlashParams& p) {
    if (KS && p.ksplit > 1) {
      const int rank = static_cast<int>(cluster_rank());
      u = static_cast<int>(blockIdx.x) / p.ksplit;
      j0 = rank * p.nkv / p.ksplit;
      j1 = (rank + 1) * p.nkv / p.ksplit;
    } else if (p.split) {
      const int64_t w = static_cast<int64_t>(p.units) * p.nkv;
      const int64_t b = w * blockIdx.x / gridDim.x, e = w * (blockIdx.x + 1) / gridDim.x;
      u_first = static_cast<int>(b / p.nkv);
      j_first = static_cast<int>(b - static_cast<int64_t>(u_first) * p.nkv);
      u_last = static_cast<int>(e / p.nkv);
      const int j_last = static_cast<int>(e - static_cast<int64_t>(u_last) * p.nkv);
      if (j_last > 0) {
        u = u_last;
        j0 = 0;
        j1 = j_last;
      } else {
        first_whole(p);
      }
    } else {
      u = blockIdx.x;
      j0 = 0;
      j1 = p.nkv;
    }
  }
  __device__ __forceinline__ void first_whole(const FlashParams& p) {
    u = u_first;
    j0 = j_first;
    j1 = u_first < u_last ? p.nkv : j0;
  }
  __device__ __forceinline__ bool valid(const FlashParams& p) const { return j0 < j1 && u < p.units; }
  __device__ __forceinline__ void next(const FlashParams& p) {
    if (KS && p.ksplit > 1) {
      u = p.units;   // one segment per CTA
    } else if (p.split) {
      if (u == u_last) {
        first_whole(p);
      } else {
        ++u;
        j0 = 0;
        j1 = u < u_last ? p.nkv : 0;
      }
    } else {
      u += gridDim.x;
    }
  }
  __device__ __forceinline__ bool cut(const FlashParams& p) const { return j0 > 0 || j1 < p.nkv; }
};

template <int D, int NQ, int BN, bool PREC = false>
struct FlashCfg {
  static constexpr int DSLABS = (D + 63) / 64;
  static constexpr int KSTEPS = (D + 15) / 16;
  // P V width: D and the row-sum column D, rounded up to the MMA's multiple of
  // 16 (48 at d = 40); tensor memory keeps D padded to 64 per query tile
  static constexpr int PVN = (D + 1 + 15) / 16 * 16;
  static constexpr int PV_COLS = DSLABS * 64;
  static constexpr int TAIL = D - 64 * (DSLABS - 1);  // V columns loaded into its last slab
  static constexpr int Q_TILE = DSLABS * 128 * 128;
  static constexpr int KV_SLAB = BN * 128;
  static constexpr int K_BYTES = DSLABS * KV_SLAB;
  static constexpr int V_BYTES = DSLABS * KV_SLAB;
  static constexpr int V_TX = (DSLABS - 1) * KV_SLAB + TAIL * 2 * BN;   // bytes the V loads deliver
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int QBUF = 2;                  // Q tiles double-buffered across work units
  // O store passes, in 16-bit columns (an fp32 O column counts as two)
  static constexpr int OCW = PREC ? 80 : (D <= 80 ? D : 80);
  static constexpr int OPASS = (PREC ? 2 * D : D) / OCW;
  static constexpr int STG_BYTES = 4 * NQ * RowStage<OCW>::BYTES;   // one slice per softmax warp
  // 227 KB per CTA, less alignment slack, barriers and the tensor-memory word
  static constexpr int STAGES_FIT = (232448 - 1024 - 16 - 8 * 32 - QBUF * NQ * Q_TILE - STG_BYTES) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  // tensor memory per query tile: S (BN fp32), P (BN/2 columns of 16-bit
  // pairs; with PREC a second such buffer holds P's residual), O (PV_COLS fp32)
  static constexpr uint32_t TM_S = 0;
  static constexpr uint32_t TM_P = BN;
  static constexpr uint32_t TM_PL = BN + BN / 2;
  static constexpr uint32_t TM_O = BN + (PREC ? BN : BN / 2);
  static constexpr int QCOLS = TM_O + PV_COLS;
  static constexpr uint32_t TMEM_COLS = NQ * QCOLS <= 256 ? 256 : 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = QBUF * NQ * Q_TILE;
  static constexpr int OFF_STG = OFF_KV + STAGES * STAGE;
  static constexpr int OFF_BAR = OFF_STG + STG_BYTES;
  static constexpr int NBAR = 2 * QBUF + 3 * STAGES + 5 * NQ + 2;
  static constexpr int MISC = 4 + 4 * NQ;   // words after the barriers
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + MISC * 4 + 1024;
  static constexpr int NTHREADS = 128 + 128 * NQ;
  static constexpr bool KS = NQ == 1 && !PREC;   // units may be split over a cluster
  // a partial row of a cut unit: D unnormalised O columns, then (m, l, raw max), padded to 16 bytes
  static constexpr int ROWF = (D + 3 + 3) / 4 * 4;
  static_assert(STAGES >= 2, "key/value ring too shallow");
  static_assert(NQ * QCOLS <= 512, "tensor memory budget");
  static_assert(NQ >= 1 && NQ <= 3, "MMA warps 1..NQ share the first warp group with the TMA warp");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 128, "key tile");
  static_assert(TAIL % 8 == 0 && TAIL < 64, "room for the ones column in V's last slab");
  static_assert((PREC ? 2 * D : D) % OCW == 0, "whole store passes");
  // the precise variant never cuts a unit (it runs without the split schedule)
  static_assert(NQ > 1 || 128 * (D + 4) * 4 <= STAGES * STAGE, "cluster partial rows fit in the key/value stages");
};

// A unit whose key range is cut between two CTAs (split schedule) is
// finished by whichever half can see the other's results: each half has its
// unnormalised rows O, running max m (base 2, scaled), row sum l and raw
// score max, and the merge always combines head (h) then tail (t):
//   m = max(m_h, m_t),  O = (O_h 2^(m_h-m) + O_t 2^(m_t-m)) / (l_h 2^(m_h-m) + l_t 2^(m_t-m)).
// A half that cannot merge leaves its rows in the workspace, stored as quads
// of columns with the 128 rows of a quad contiguous (32 consecutive rows
// read or write 512 contiguous bytes):
//   part[slot][half][ROWF / 4][128][4],  quad D / 4 = (m, l, raw max, 0).
// Who merges is settled on one counter per (cut, query tile), by atomic adds
// with acquire-release semantics:
//   head: writes its rows, then adds 1;
//   tail: adds 2 first; if the head's 1 is there it merges at once, without
//         writing its rows; otherwise it writes them and adds 4;
// the add that completes {1, 4} merges (the head, seeing 4; or the tail's
// second add, seeing 1).  Exactly one side merges, from the other's rows in
// the workspace and its own in tensor memory.  With each CTA's head half
// scheduled first, the tail normally finds the head done.
// A unit shared by a cluster (ksplit > 1): every CTA leaves, per row r of the
// tile, its unnormalised O row, running max m (base 2, scaled), row sum l and
// raw score max in shared memory at the start of its (now idle) key/value
// stages, rows CPITCH floats apart; after a cluster barrier CTA `rank` merges
// rows [rank 128 / k, (rank + 1) 128 / k) over the k CTAs in rank order:
//   m = max m_j,  O = sum_j O_j 2^(m_j - m) / sum_j l_j 2^(m_j - m).
template <int D>
struct ClusterRows {
  static constexpr int CPITCH = D + 4;   // D columns, then (m, l, raw max, 0); 16-byte rows
};

template <int ROWF>
__device__ __forceinline__ float4* partial_rows(float* part, int64_t slot, int half) {
  return reinterpret_cast<float4*>(part) + (slot * 2 + half) * (ROWF / 4) * 128;
}

// p = 2^(s*c - m) for one row's key tile, packed to 16-bit pairs: NPOLY of
// every 8 pairs on the FMA pipe (exp2_poly2), the rest on MUFU.
template <int BN, bool BF16, int NPOLY, bool PREC = false>
__device__ __forceinline__ void flash_exp_block(const uint32_t (&v)[BN], uint64_t c2, uint64_t nm2,
                                                uint32_t (&pk)[BN / 2], uint32_t* pl = nullptr) {
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
    if constexpr (PREC) {
      // the residual of the 16-bit rounding, itself rounded to 16 bits
      float h0, h1;
      if constexpr (BF16) {
        const float2 h = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[k]));
        h0 = h.x;
        h1 = h.y;
      } else {
        const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&pk[k]));
        h0 = h.x;
        h1 = h.y;
      }
      pl[k] = pack2<BF16>(e0 - h0, e1 - h1);
    }
  }
}

// named barrier of query tile q's four softmax warps (ids 1 + q, fixed at compile time)
__device__ __forceinline__ void softmax_bar_sync(int q) {
  if (q == 0)
    named_bar_sync(1, 128);
  else if (q == 1)
    named_bar_sync(2, 128);
  else
    named_bar_sync(3, 128);
}

// One counter update for the tile: thread r == 0 adds v (acquire-release),
// the old value reaches every thread of the tile through `flag`.
__device__ __forceinline__ uint32_t tile_count(uint32_t* ticket, uint32_t v, int q, int r, volatile uint32_t* flag) {
  if (r == 0) *flag = atomic_add_acq_rel_gpu(ticket, v);
  softmax_bar_sync(q);
  return *flag;
}

// Epilogue of a cut unit for the tile's 128 softmax threads (one row each).
// flags: two words, used once each.  Out of line: it runs at most twice per
// CTA, and inlined it would weigh on the register allocation of the softmax
// loop (the softmax warps hold more registers than any callee may use).
template <int D, int OCW, bool BF16, int ROWF>
__device__ __noinline__ void flash_cut_epilogue(float* part, uint32_t* tickets, float* LS, int N, float scale,
                                                float c, uint32_t o_tmem, int side, int64_t slot, int q, int r,
                                                int bh, int row, float m_used, float l, float rawmax,
                                                volatile uint32_t* flags, uint8_t* slice, uint8_t* owarp,
                                                int ovalid) {
  float4* mine = partial_rows<ROWF>(part, slot, side) + r;
  const float4* theirs = partial_rows<ROWF>(part, slot, side ^ 1) + r;
  constexpr int G = D / 8 < 5 ? D / 8 : 5;   // chunks of 8 columns per tensor-memory wait
  static_assert((D / 8) % G == 0, "column groups");
  auto write_mine = [&]() {
#pragma unroll
    for (int g0 = 0; g0 < D / 8; g0 += G) {
      uint32_t o[8 * G];
#pragma unroll
      for (int i = 0; i < G; ++i) tmem_ld_x8(o_tmem + (g0 + i) * 8, o + 8 * i);
      tmem_wait_ld();
      reg_fence<8 * G>(o);
#pragma unroll
      for (int i = 0; i < 2 * G; ++i)
        __stcg(mine + (g0 * 2 + i) * 128, make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                                     __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3])));
    }
    __stcg(mine + (D / 4) * 128, make_float4(m_used, l, rawmax, 0.f));
    softmax_bar_sync(q);   // the tile's rows before the count that publishes them
  };
  bool merge, wrote = true;
  if (side == 0) {
    write_mine();
    merge = (tile_count(&tickets[slot], 1u, q, r, &flags[0]) & 4u) != 0u;
  } else {
    merge = (tile_count(&tickets[slot], 2u, q, r, &flags[0]) & 1u) != 0u;
    wrote = !merge;
    if (!merge) {
      write_mine();
      merge = (tile_count(&tickets[slot], 4u, q, r, &flags[1]) & 1u) != 0u;
    }
  }
  if (!merge) return;
  const float4 t2 = __ldcg(theirs + (D / 4) * 128);
  const float m_h = side ? t2.x : m_used, m_t = side ? m_used : t2.x;
  const float l_h = side ? t2.y : l, l_t = side ? l : t2.y;
  const float m = fmaxf(m_h, m_t);
  const float a_h = ex2_approx(m_h - m), a_t = ex2_approx(m_t - m);
  const float a_mine = side ? a_t : a_h, a_theirs = side ? a_h : a_t;
  const float lsum = fmaf(l_h, a_h, l_t * a_t);
  const float inv = 1.f / lsum;
  const int lane = r & 31;
  static_assert((OCW / 8) % G == 0, "column groups per store pass");
#pragma unroll
  for (int g0 = 0; g0 < D / 8; g0 += G) {
    uint32_t o[8 * G];
    float4 u[2 * G];
#pragma unroll
    for (int i = 0; i < G; ++i) tmem_ld_x8(o_tmem + (g0 + i) * 8, o + 8 * i);
#pragma unroll
    for (int i = 0; i < 2 * G; ++i) u[i] = __ldcg(theirs + (g0 * 2 + i) * 128);
    tmem_wait_ld();
    reg_fence<8 * G>(o);
#pragma unroll
    for (int i = 0; i < G; ++i) {
      const float g[8] = {u[2 * i].x, u[2 * i].y, u[2 * i].z, u[2 * i].w,
                          u[2 * i + 1].x, u[2 * i + 1].y, u[2 * i + 1].z, u[2 * i + 1].w};
      float f[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float ov = __uint_as_float(o[8 * i + k]);
        f[k] = (side ? fmaf(g[k], a_h, ov * a_mine) : fmaf(ov, a_h, g[k] * a_theirs)) * inv;
      }
      uint4 w;
      w.x = pack2<BF16>(f[0], f[1]);
      w.y = pack2<BF16>(f[2], f[3]);
      w.z = pack2<BF16>(f[4], f[5]);
      w.w = pack2<BF16>(f[6], f[7]);
      stage_put<OCW>(slice, lane, (g0 + i) % (OCW / 8), w);
    }
    if ((g0 + G) % (OCW / 8) == 0)   // a store pass is complete
      stage_flush<OCW>(slice, lane, owarp + ((g0 + G) / (OCW / 8) - 1) * OCW * 2, D * 2, ovalid);
  }
  if (LS != nullptr && row < N) {
    const float raw = fmaxf(rawmax, t2.z);
    *reinterpret_cast<float2*>(LS + 2 * (static_cast<int64_t>(bh) * N + row)) =
        make_float2(raw * scale, lsum * ex2_approx(m - raw * c));
  }
  // leave the workspace all zero for the next call
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int k = 0; k < ROWF / 4; ++k) {
    if (wrote) __stcg(mine + k * 128, z);
    __stcg(const_cast<float4*>(theirs) + k * 128, z);
  }
  if (r == 0) tickets[slot] = 0u;
}

template <int D, int NQ, int BN, bool BF16, int NPOLY, bool PREC = false>
__global__ void __launch_bounds__(FlashCfg<D, NQ, BN, PREC>::NTHREADS, 1)
    flash_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmVt,
                 const FlashParams p) {
  using C = FlashCfg<D, NQ, BN, PREC>;
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
  // [0] tensor memory, [1] abort, [4 + 4q + 2k ..]: tile q's two count words for its k-th cut unit
  uint32_t* misc = reinterpret_cast<uint32_t*>(stagger + 1);
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
      for (FlashSegments<C::KS> sg(p); sg.valid(p) && live; sg.next(p)) {
        const int bh = sg.u / p.tph, qg = sg.u % p.tph;
        const uint32_t qb = nq % C::QBUF, qn = nq / C::QBUF;
        if (!mbar_wait(&q_empty[qb], (qn & 1) ^ 1, kSiteQEmpty, abort_flag)) { live = false; break; }
        ++nq;
        mbar_arrive_expect_tx(&q_full[qb], NQ * C::Q_TILE);
        for (int q = 0; q < NQ; ++q)
          for (int s = 0; s < C::DSLABS; ++s)
            tma_load_3d(sQ + (qb * NQ + q) * C::Q_TILE + s * 16384, &tmQ, 64 * s, (qg * NQ + q) * 128, bh,
                        &q_full[qb]);
        for (int j = sg.j0; j < sg.j1; ++j, ++kvc) {
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
    const uint32_t pl_tm = tmem + q * C::QCOLS + C::TM_PL;
    const uint32_t o_tm = tmem + q * C::QCOLS + C::TM_O;
    uint32_t t_base = 0, kv_base = 0, ui = 0;
    bool live = true;
    if (p.inject_stall) live = mbar_wait_warp(stall_bar, 0, kSiteInjected, abort_flag);   // runs out
    for (FlashSegments<C::KS> sg(p); sg.valid(p) && live; sg.next(p), ++ui) {
      const uint32_t qb = ui % C::QBUF, qn = ui / C::QBUF;
      if (!mbar_wait_warp(&q_full[qb], qn & 1, kSiteQFull, abort_flag)) { live = false; break; }
      const uint64_t q_desc0 = q_desc00 + ((qb * NQ * C::Q_TILE) >> 4);
      const int len = sg.j1 - sg.j0;
      for (int j = 0; j <= len; ++j) {
        if (j < len) {
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
          if constexpr (PREC) {
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) mma_ts(o_tm, pl_tm + kk * 8, vd + ((kk * 2048) >> 4), idesc_pv, 1u);
          }
          mma_commit(&pv_done[q]);
          mma_commit(&kv_empty[st]);
        }
      }
      if (live) mma_commit(&q_empty[qb]);
      t_base += len;
      kv_base += len;
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
    const uint32_t pl_tmem = tmem + q * C::QCOLS + C::TM_PL + lane_off;
    const uint32_t o_tmem = tmem + q * C::QCOLS + C::TM_O + lane_off;
    const float c = p.c;
    uint32_t t = 0;        // tiles seen by this query-tile slot (all units)
    bool live = true;
    // The two query tiles run independently (own MMA warp, own handshakes,
    // Q double-buffered); started half a tile apart, their softmax phases
    // interleave on the SM instead of contending for the exponential unit.
    if (NQ == 2 && q == 1) live = __all_sync(0xffffffffu, mbar_wait(stagger, 0, kSiteSFull, abort_flag));
    int kcut = 0;          // cut units seen (at most two)
    for (FlashSegments<C::KS> sg(p); sg.valid(p) && live; sg.next(p)) {
      const int bh = sg.u / p.tph, qg = sg.u % p.tph;
      const int row = (qg * NQ + q) * 128 + r;
      float m_used = -INFINITY, rawmax = -INFINITY;
      for (int j = sg.j0; j < sg.j1; ++j, ++t) {
        live = __all_sync(0xffffffffu, mbar_wait(&s_full[q], t & 1, kSiteSFull, abort_flag));
        if (!live) break;
        tc_fence_after();
        uint32_t v[BN];
        if constexpr (BN == 128) {
          tmem_ld_x128(s_tmem, v);
        } else {
#pragma unroll
          for (int cc = 0; cc < BN / 32; ++cc) tmem_ld_x32(s_tmem + cc * 32, v + cc * 32);
        }
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
        const float mt = mx * c;
        const uint64_t c2 = f2_pack(c, c);
        float alpha = 1.f;
        bool rescale = false;
        uint32_t pk[BN / 2];
        uint32_t pl[PREC ? BN / 2 : 1];
        if (NQ == 2 && q == 0 && t == 0) {
          __syncwarp();
          if (lane == 0) mbar_arrive(stagger);
        }
        if (mt > m_used + 8.f) {
          alpha = ex2_approx(m_used - mt);
          m_used = mt;
          rescale = (j > sg.j0);
        }
        flash_exp_block<BN, BF16, NPOLY, PREC>(v, c2, f2_pack(-m_used, -m_used), pk, pl);
        if (j > sg.j0) {
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
            if constexpr (C::PVN % 32 != 0) {
              constexpr int c0 = C::PVN / 32 * 32;
              uint32_t o[16];
              tmem_ld_x16(o_tmem + c0, o);
              tmem_wait_ld();
              reg_fence<16>(o);
#pragma unroll
              for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st_x16(o_tmem + c0, o);
            }
          }
        }
        if constexpr (BN == 128) {
          tmem_st_x64(p_tmem, pk);
          if constexpr (PREC) tmem_st_x64(pl_tmem, pl);
        } else {
#pragma unroll
          for (int cc = 0; cc < BN / 32; ++cc) tmem_st_x16(p_tmem + cc * 16, pk + cc * 16);
          if constexpr (PREC) {
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc) tmem_st_x16(pl_tmem + cc * 16, pl + cc * 16);
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
      // this warp's 32 rows of O: consecutive rows, stored through its shared-memory slice
      constexpr int EB = PREC ? 4 : 2;   // bytes per O element
      const int row_w = row - lane;
      uint8_t* owarp = reinterpret_cast<uint8_t*>(p.O) + (static_cast<int64_t>(bh) * p.N + row_w) * D * EB;
      const int ovalid = p.N - row_w;
      uint8_t* slice = smem + C::OFF_STG + (warp - 4) * RowStage<C::OCW>::BYTES;
      if constexpr (NQ == 1 && !PREC) {
        if (p.ksplit > 1) {
          // this CTA's share of the key range: unnormalised row, m, l, raw max
          float* prow = reinterpret_cast<float*>(sKV) + r * ClusterRows<D>::CPITCH;
          float l = 0.f;
#pragma unroll
          for (int c8 = 0; c8 <= D / 8; ++c8) {
            uint32_t o[8];
            tmem_ld_x8(o_tmem + c8 * 8, o);
            tmem_wait_ld();
            reg_fence<8>(o);
            if (c8 < D / 8) {
              *reinterpret_cast<uint4*>(prow + c8 * 8) = make_uint4(o[0], o[1], o[2], o[3]);
              *reinterpret_cast<uint4*>(prow + c8 * 8 + 4) = make_uint4(o[4], o[5], o[6], o[7]);
            } else {
              l = __uint_as_float(o[0]);
            }
          }
          *reinterpret_cast<float4*>(prow + D) = make_float4(m_used, l, rawmax, 0.f);
          tc_fence_before();
          continue;
        }
      }
      if (!(p.split && sg.cut(p))) {
        // O in store passes of PC columns; the first pass also brings the row
        // sum l (column D) when it fits beside them, all behind one wait
        constexpr int NPASS = C::OPASS;
        constexpr int PC = C::OCW * 2 / EB;        // O columns per pass
        constexpr int XL = NPASS == 1 ? 8 : 0;     // column D loaded with the only pass
        float l = 0.f, inv = 0.f;
        if constexpr (NPASS > 1) {
          uint32_t t8[8];
          tmem_ld_x8(o_tmem + D, t8);
          tmem_wait_ld();
          reg_fence<8>(t8);
          l = __uint_as_float(t8[0]);
          inv = 1.f / l;
        }
#pragma unroll
        for (int ps = 0; ps < NPASS; ++ps) {
          uint32_t o[PC + XL];
#pragma unroll
          for (int c8 = 0; c8 < (PC + XL) / 8; ++c8) tmem_ld_x8(o_tmem + ps * PC + c8 * 8, o + c8 * 8);
          tmem_wait_ld();
          reg_fence<PC + XL>(o);
          if constexpr (NPASS == 1) {
            l = __uint_as_float(o[D]);
            inv = 1.f / l;
          }
#pragma unroll
          for (int ch = 0; ch < C::OCW / 8; ++ch) {   // 16-byte chunks of the pass
            uint4 w;
            if constexpr (PREC) {
              const uint32_t* oc = o + ch * 4;
              w = make_uint4(__float_as_uint(__uint_as_float(oc[0]) * inv), __float_as_uint(__uint_as_float(oc[1]) * inv),
                             __float_as_uint(__uint_as_float(oc[2]) * inv), __float_as_uint(__uint_as_float(oc[3]) * inv));
            } else {
              const uint32_t* oc = o + ch * 8;
              w.x = pack2<BF16>(__uint_as_float(oc[0]) * inv, __uint_as_float(oc[1]) * inv);
              w.y = pack2<BF16>(__uint_as_float(oc[2]) * inv, __uint_as_float(oc[3]) * inv);
              w.z = pack2<BF16>(__uint_as_float(oc[4]) * inv, __uint_as_float(oc[5]) * inv);
              w.w = pack2<BF16>(__uint_as_float(oc[6]) * inv, __uint_as_float(oc[7]) * inv);
            }
            stage_put<C::OCW>(slice, lane, ch, w);
          }
          stage_flush<C::OCW>(slice, lane, owarp + ps * C::OCW * 2, D * EB, ovalid);
        }
        if (p.LS != nullptr && row < p.N) {
          const float L = rawmax * p.scale;
          const float S = l * ex2_approx(m_used - rawmax * c);
          *reinterpret_cast<float2*>(p.LS + 2 * (static_cast<int64_t>(bh) * p.N + row)) = make_float2(L, S);
        }
      } else if constexpr (!PREC) {
        if (kcut < 2) {
          float l;
          {
            uint32_t o[8];
            tmem_ld_x8(o_tmem + D, o);
            tmem_wait_ld();
            reg_fence<8>(o);
            l = __uint_as_float(o[0]);
          }
          const int side = sg.j0 > 0 ? 1 : 0;   // 0: head half, 1: tail half
          flash_cut_epilogue<D, C::OCW, BF16, C::ROWF>(p.part, p.tickets, p.LS, p.N, p.scale, c, o_tmem, side,
                                                      static_cast<int64_t>(blockIdx.x - side) * NQ + q, q, r, bh, row,
                                                      m_used, l, rawmax, misc + 4 + 4 * q + 2 * kcut, slice, owarp,
                                                      ovalid);
          ++kcut;
        }
      }
      tc_fence_before();
    }
  } else {
    // idle warps of the first warp group
    if constexpr (NQ == 2) regs_dec<120>();
  }

  if constexpr (NQ == 1 && !PREC) {
    if (p.ksplit > 1) {
      // every thread of every CTA of the cluster passes both barriers, also
      // after a wait ran out (the results are then wrong, and the error word says so)
      constexpr int CP = ClusterRows<D>::CPITCH;
      const uint32_t k = static_cast<uint32_t>(p.ksplit);
      const uint32_t rank = cluster_rank();
      const int u = static_cast<int>(blockIdx.x) / p.ksplit;
      const int bh = u / p.tph, row0 = (u % p.tph) * 128;
      __syncwarp();
      cluster_sync();
      if (warp >= 4) {
        const int r0 = static_cast<int>(rank) * 128 / static_cast<int>(k);
        const int r1 = static_cast<int>(rank + 1) * 128 / static_cast<int>(k);
        const float* part0 = reinterpret_cast<const float*>(sKV);
        for (int it = threadIdx.x - 128; it < (r1 - r0) * (D / 8); it += 128) {
          const int rr = r0 + it / (D / 8), c8 = it % (D / 8);
          const int row = row0 + rr;
          if (row >= p.N) continue;
          float m = -INFINITY;
          for (uint32_t j = 0; j < k; ++j) m = fmaxf(m, ld_cluster_f32(part0 + rr * CP + D, j));
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          float lsum = 0.f, raw = -INFINITY;
          for (uint32_t j = 0; j < k; ++j) {
            const float4 st = ld_cluster_f32x4(part0 + rr * CP + D, j);   // (m_j, l_j, raw max_j, 0)
            const float a = ex2_approx(st.x - m);
            lsum = fmaf(st.y, a, lsum);
            raw = fmaxf(raw, st.z);
            const float4 x0 = ld_cluster_f32x4(part0 + rr * CP + c8 * 8, j);
            const float4 x1 = ld_cluster_f32x4(part0 + rr * CP + c8 * 8 + 4, j);
            acc[0] = fmaf(x0.x, a, acc[0]); acc[1] = fmaf(x0.y, a, acc[1]);
            acc[2] = fmaf(x0.z, a, acc[2]); acc[3] = fmaf(x0.w, a, acc[3]);
            acc[4] = fmaf(x1.x, a, acc[4]); acc[5] = fmaf(x1.y, a, acc[5]);
            acc[6] = fmaf(x1.z, a, acc[6]); acc[7] = fmaf(x1.w, a, acc[7]);
          }
          const float inv = 1.f / lsum;
          const int64_t grow = static_cast<int64_t>(bh) * p.N + row;
          uint4 w;
          w.x = pack2<BF16>(acc[0] * inv, acc[1] * inv);
          w.y = pack2<BF16>(acc[2] * inv, acc[3] * inv);
          w.z = pack2<BF16>(acc[4] * inv, acc[5] * inv);
          w.w = pack2<BF16>(acc[6] * inv, acc[7] * inv);
          *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.O) + grow * D * 2 + c8 * 16) = w;
          if (c8 == 0 && p.LS != nullptr)
            *reinterpret_cast<float2*>(p.LS + 2 * grow) = make_float2(raw * p.scale, lsum * ex2_approx(m - raw * p.c));
        }
      }
      __syncwarp();
      cluster_sync();   // no CTA leaves while another may still read its partial rows
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
