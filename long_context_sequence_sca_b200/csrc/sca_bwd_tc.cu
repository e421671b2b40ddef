// Sliding Chunk Attention backward on 5th-generation tensor cores (sm_100a).
//
// Gradients of O_s = softmax(Q_s [K_{s-1}; K_s]^T) [V_{s-1}; V_s] (Gecko
// digest, paper.rainbus.top, method step details, step 3; scale 1, causal
// inside the current chunk, no previous chunk for chunk 1).  With the
// forward's row log-sum-exp l_t and delta_t = rowsum(dO_t * O_t):
//     P = exp(S - l),  dP = dO V^T,  dS = P * (dP - delta),
//     dV = P^T dO,  dK = dS^T Q,  dQ = dS K.
// The pages print no backward; this is the chain rule of the forward.
//
// Two kernels of one template, each one CTA per 128-row tile of one (b, h):
//   kDQ = false  rows are keys: S^T = K Q_i^T and dP^T = V dO_i^T into TMEM
//                for every query tile i that sees the key tile (the rest of
//                its chunk from the diagonal on, and the whole next chunk);
//                P^T and dS^T go back to TMEM as bf16; dV += P^T dO_i and
//                dK += dS^T Q_i read them from TMEM (TS form).
//   kDQ = true   rows are queries: S = Q K_j^T and dP = dO V_j^T for the key
//                tiles of the window; dQ += dS K_j.
// Roles (576 threads): warp 0 TMA producer (the CTA's two fixed tiles once,
// then a ring of two-tile stages for the loop operands, with the loop rows'
// statistics for kDQ = false), warp 1 TMEM allocator and MMA issuer, warps
// 2-17 four element-wise warpgroups, each owning 32 of the 128 loop columns
// (warpgroup w writes its packed bf16 results over the S columns it has
// consumed, at column 32 w, and the TS MMAs read each 16-column K step from
// where its warpgroup put it).  Four warps per sub-partition, one 32-column
// TMEM round trip each, keep the TMEM latency of the element-wise pass
// hidden (with two warpgroups of 64 columns it took 2.4x its SFU time).
// Only the diagonal tile is masked.
//
// Requires bf16, d in {64, 128}, c % 128 == 0.  Every wait is bounded; on a
// timeout the CTA drains its copies and MMAs, frees TMEM and returns with
// the status word set.
#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

constexpr int kRows = 128;          // rows per tile (keys or queries)
// Element-wise warpgroups per kernel (measured: 4 for dK/dV, 2 for dQ).
#ifndef GECKO_BWD_EW
#define GECKO_BWD_EW 4
#endif
#ifndef GECKO_BWD_EW_DQ
#define GECKO_BWD_EW_DQ 2
#endif
template <bool kDQ>
struct EwLayout {
  static constexpr int n = kDQ ? GECKO_BWD_EW_DQ : GECKO_BWD_EW;   // warpgroups
  static constexpr int cw = kRows / n;                             // loop columns per warpgroup
  static constexpr int threads = 64 + 128 * n;
  static_assert(cw % 32 == 0, "whole 32-column TMEM loads per warpgroup");
};
// Of every 8 exponential pairs of P, GECKO_BWD_SFU_PAIRS go to the SFU and the
// rest to the FMA pipe (exp2_poly2).  Measured on B200 (bench workload):
// 8/8 on the SFU is fastest (dK/dV 5.80 ms against 7.06 ms at 6/8, where the
// polynomial's registers push the 96-register budget into spills), so 8 is
// the default and other splits remain a compile-time option.
#ifndef GECKO_BWD_SFU_PAIRS
#define GECKO_BWD_SFU_PAIRS 8
#endif
constexpr int kBwdSfuPairs = GECKO_BWD_SFU_PAIRS;

template <int D>
struct BwdCfg {
  static constexpr int kTileBytes = kRows * D * 2;
  static constexpr int kBoxBytes = kRows * 64 * 2;
  static constexpr int kStages = D == 64 ? 4 : 2;
  // a stage: two operand tiles, then -log2(e) l and delta of its 128 rows
  static constexpr int kStageBytes = 2 * kTileBytes + 1024;
  static constexpr int kFixOff = 0;
  static constexpr int kStageOff = 2 * kTileBytes;
  static constexpr int kBarOff = kStageOff + kStages * kStageBytes;
  // fix_full, ld_full[NS], ld_empty[NS], s_ready, dp_ready, p_done, ds_done, acc_full, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 6;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kStageBytes % 1024 == 0 && kStageOff % 1024 == 0, "1024-byte aligned operand tiles");
  static_assert(kAlloc <= 232448, "dynamic shared memory above the sm_100 per-block limit");
  static constexpr uint32_t kTmemCols = 512;
  // S (then P, packed), dP (then dS, packed; dK/dV kernel), accumulators A
  // and B, and (dQ kernel) two buffers for packed dS in the spare columns
  static constexpr uint32_t kColS = 0, kColP = 128, kColA = 256, kColB = 256 + D;
  static constexpr uint32_t kColF = 384;   // + 64 * (step % 2), 64 packed columns each
  // the dK/dV kernel uses accumulators A and B, the dQ kernel A and the dS buffers
  static_assert(kColF + 128 <= kTmemCols && kColA + D <= kColF && kColB + D <= kTmemCols, "TMEM columns");
};

// Tile coordinates of CTA `bid`.  CTAs of one (b, h, chunk) are adjacent
// (they share the loop tiles of that window in L2), the most expensive first.
struct BwdTile {
  int64_t bh;
  int row;             // row tile (128 rows)
  int beg, end;        // loop tiles [beg, end)
};

__device__ __forceinline__ BwdTile bwd_tile(int bid, int T, int c, bool dq) {
  const int n_tiles = T / kRows, tpc = c / kRows, S = T / c;
  const int g = bid / tpc, o = bid % tpc;
  BwdTile t;
  t.bh = g / S;
  const int ch = g % S;
  if (!dq) {
    // key tile: queries from the diagonal to the end of the next chunk
    t.row = ch * tpc + o;
    t.beg = t.row;
    t.end = (ch + 2) * tpc < n_tiles ? (ch + 2) * tpc : n_tiles;
  } else {
    // query tile: keys from the previous chunk's start to the diagonal
    t.row = ch * tpc + (tpc - 1 - o);
    t.beg = ch >= 1 ? (ch - 1) * tpc : 0;
    t.end = t.row + 1;
  }
  return t;
}

template <int D, bool kDQ>
__global__ void __launch_bounds__(EwLayout<kDQ>::threads, 1)
sca_bwd_tc_kernel(const __grid_constant__ CUtensorMap map_fix0, const __grid_constant__ CUtensorMap map_fix1,
                  const __grid_constant__ CUtensorMap map_st0, const __grid_constant__ CUtensorMap map_st1,
                  const float* __restrict__ nlse2, const float* __restrict__ delta,
                  const float* __restrict__ dv_add, __nv_bfloat16* __restrict__ out_a,
                  __nv_bfloat16* __restrict__ out_b, int T, int c, int* status) {
  using Cfg = BwdCfg<D>;
  constexpr int NS = Cfg::kStages;
  constexpr int kEW = EwLayout<kDQ>::n, kCW = EwLayout<kDQ>::cw;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sFix = smem + Cfg::kFixOff;
  uint8_t* sStage = smem + Cfg::kStageOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* fix_full = bars;
  uint64_t* ld_full = bars + 1;
  uint64_t* ld_empty = ld_full + NS;
  // S and dP are committed separately, so the exponentials of P overlap the
  // dP product and the previous step's dK product; P (dK/dV kernel) and dS
  // are handed back separately for the same reason.
  uint64_t* s_ready = ld_empty + NS;
  uint64_t* dp_ready = s_ready + 1;
  uint64_t* p_done = dp_ready + 1;
  uint64_t* ds_done = p_done + 1;
  uint64_t* acc_full = ds_done + 1;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x % 32;
  const BwdTile tile = bwd_tile(blockIdx.x, T, c, kDQ);
  const int N = tile.end - tile.beg;
  const int64_t rowbase = tile.bh * (int64_t)T;

  if (threadIdx.x == 0) {
    mbar_init(fix_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(ld_full + s, 1);
      mbar_init(ld_empty + s, 1);
    }
    mbar_init(s_ready, 1);
    mbar_init(dp_ready, 1);
    mbar_init(p_done, 128 * kEW);
    mbar_init(ds_done, 128 * kEW);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_fix0);
    tma_prefetch_desc(&map_fix1);
    tma_prefetch_desc(&map_st0);
    tma_prefetch_desc(&map_st1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      bool ok = true;
      const int frow = (int)(rowbase + (int64_t)tile.row * kRows);
      mbar_arrive_expect_tx(fix_full, 2 * Cfg::kTileBytes);
      for (int b = 0; b < D / 64; ++b) {
        tma_load_2d(sFix + b * Cfg::kBoxBytes, &map_fix0, fix_full, b * 64, frow);
        tma_load_2d(sFix + Cfg::kTileBytes + b * Cfg::kBoxBytes, &map_fix1, fix_full, b * 64, frow);
      }
      int n = 0;
      for (; n < N; ++n) {
        const int st = n % NS;
        if (n >= NS && !(ok = mbar_wait(ld_empty + st, (uint32_t)(n / NS - 1) & 1, abort_flag, status))) break;
        uint8_t* sb = sStage + st * Cfg::kStageBytes;
        const int64_t lrow = rowbase + (int64_t)(tile.beg + n) * kRows;
        mbar_arrive_expect_tx(ld_full + st, 2 * Cfg::kTileBytes + (kDQ ? 0 : 1024));
        for (int b = 0; b < D / 64; ++b) {
          tma_load_2d(sb + b * Cfg::kBoxBytes, &map_st0, ld_full + st, b * 64, (int)lrow);
          tma_load_2d(sb + Cfg::kTileBytes + b * Cfg::kBoxBytes, &map_st1, ld_full + st, b * 64, (int)lrow);
        }
        if (!kDQ) {
          bulk_load_1d(sb + 2 * Cfg::kTileBytes, nlse2 + lrow, 512, ld_full + st);
          bulk_load_1d(sb + 2 * Cfg::kTileBytes + 512, delta + lrow, 512, ld_full + st);
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA exits
        for (int m = n - NS > 0 ? n - NS : 0; m < n; ++m) mbar_wait_drain(ld_full + m % NS, (uint32_t)(m / NS) & 1);
        mbar_wait_drain(fix_full, 0);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc_ss = idesc_bf16_f32(kRows, kRows, false, false);
      constexpr uint32_t idesc_ts = idesc_bf16_f32(kRows, D, false, true);
      const uint32_t fa = smem_u32(sFix), sa = smem_u32(sStage);
      bool ok = mbar_wait(fix_full, 0, abort_flag, status);
      tc_fence_after();
      const SDesc a0 = sdesc_sw128_split(fa, 16, 1024), a1 = sdesc_sw128_split(fa + Cfg::kTileBytes, 16, 1024);
      // Per step n the order is: the P-side product of step n - 1 (dV; dQ's
      // only product), S(n), the dS-side product of step n - 1 (dK), dP(n).
      // Each product overwrites a TMEM region only after the product that
      // read it was issued (the tensor pipe runs them in order).
      auto ts_products = [&](int m, bool p_side) {
        const uint32_t pb = sa + (m % NS) * Cfg::kStageBytes;
        const SDesc b0 = sdesc_sw128_split(pb, Cfg::kBoxBytes, 1024);                     // st0, MN-major
        const SDesc b1 = sdesc_sw128_split(pb + Cfg::kTileBytes, Cfg::kBoxBytes, 1024);   // st1, MN-major
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk) {
          // K step kk covers loop columns 16 kk .. 16 kk + 15, packed by
          // warpgroup (16 kk) / kCW at its own column offset
          const uint32_t acol = (uint32_t)((16 * kk / kCW) * kCW + (16 * kk % kCW) / 2);
          const uint32_t acc = (m > 0 || kk > 0) ? 1u : 0u;
          if (kDQ)
            // dS buffers are packed compactly: loop column q at column q / 2
            umma_ts(tmem + Cfg::kColA, tmem + Cfg::kColF + 64 * (m % 2) + 8 * kk, sdesc_at(b0, kk * 2048), idesc_ts,
                    acc);  // dQ += dS K
          else if (p_side)
            umma_ts(tmem + Cfg::kColA, tmem + Cfg::kColS + acol, sdesc_at(b1, kk * 2048), idesc_ts, acc);  // dV += P^T dO
          else
            umma_ts(tmem + Cfg::kColB, tmem + Cfg::kColP + acol, sdesc_at(b0, kk * 2048), idesc_ts, acc);  // dK += dS^T Q
        }
      };
      auto ss_product = [&](int m, uint32_t col, const SDesc& a, int tile) {
        const SDesc bq = sdesc_sw128_split(sa + (m % NS) * Cfg::kStageBytes + tile * Cfg::kTileBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t kbyte = (kk / 4) * Cfg::kBoxBytes + (kk % 4) * 32;
          umma_ss(tmem + col, sdesc_at(a, kbyte), sdesc_at(bq, kbyte), idesc_ss, kk > 0 ? 1u : 0u);
        }
      };
      for (int n = 0; n <= N && ok; ++n) {
        if (kDQ) {
          // dQ kernel: S(n) as soon as P(n - 1) has been read out of S, so
          // the exponentials of step n overlap dQ(n - 1) and dP(n); dS lives
          // in its own double buffer
          if (n < N) {
            if (n > 0 && !(ok = mbar_wait(p_done, (uint32_t)(n - 1) & 1, abort_flag, status))) break;
            if (!(ok = mbar_wait(ld_full + n % NS, (uint32_t)(n / NS) & 1, abort_flag, status))) break;
            tc_fence_after();
            ss_product(n, Cfg::kColS, a0, 0);   // S = fix0 st0^T
            umma_commit(s_ready);
          }
          if (n > 0) {
            if (!(ok = mbar_wait(ds_done, (uint32_t)(n - 1) & 1, abort_flag, status))) break;
            tc_fence_after();
            ts_products(n - 1, true);
            umma_commit(ld_empty + (n - 1) % NS);
          }
          if (n < N) {
            ss_product(n, Cfg::kColP, a1, 1);   // dP = fix1 st1^T
            umma_commit(dp_ready);
          }
          continue;
        }
        if (n > 0) {
          if (!(ok = mbar_wait(p_done, (uint32_t)(n - 1) & 1, abort_flag, status))) break;
          tc_fence_after();
          ts_products(n - 1, true);
        }
        if (n < N) {
          if (!(ok = mbar_wait(ld_full + n % NS, (uint32_t)(n / NS) & 1, abort_flag, status))) break;
          tc_fence_after();
          ss_product(n, Cfg::kColS, a0, 0);   // S = fix0 st0^T
          umma_commit(s_ready);
        }
        if (n > 0) {
          if (!(ok = mbar_wait(ds_done, (uint32_t)(n - 1) & 1, abort_flag, status))) break;
          tc_fence_after();
          ts_products(n - 1, false);
          umma_commit(ld_empty + (n - 1) % NS);
        }
        if (n < N) {
          ss_product(n, Cfg::kColP, a1, 1);   // dP = fix1 st1^T
          umma_commit(dp_ready);
        }
      }
      if (ok) umma_commit(acc_full);
      // all issued MMAs complete before TMEM is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- element-wise warpgroups --
    const int w = (warp - 2) / 4;             // loop columns kCW w .. kCW w + kCW - 1
    const int r = (warp % 4) * 32 + lane;     // row within the tile = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const uint64_t l2e2 = pack2(kLog2e, kLog2e);
    float my_nl = 0.f, my_dl = 0.f;
    if (kDQ) {
      my_nl = nlse2[rowbase + (int64_t)tile.row * kRows + r];
      my_dl = delta[rowbase + (int64_t)tile.row * kRows + r];
    }
    bool ok = true;
    for (int n = 0; n < N; ++n) {
      ok = __all_sync(0xffffffffu, mbar_wait(s_ready, (uint32_t)n & 1, abort_flag, status));
      if (!ok) break;
      if (!kDQ) {
        // the loop rows' statistics came with the stage's copies
        ok = __all_sync(0xffffffffu, mbar_wait(ld_full + n % NS, (uint32_t)(n / NS) & 1, abort_flag, status));
        if (!ok) break;
      }
      tc_fence_after();
      const bool diag = tile.beg + n == tile.row;
      const float* st_nl = reinterpret_cast<const float*>(sStage + (n % NS) * Cfg::kStageBytes + 2 * Cfg::kTileBytes);
      const float* st_dl = st_nl + kRows;
      // P = 2^(S log2 e - log2(e) l), kept in fp32 for dS; the dK/dV kernel
      // also hands P (bf16) to the dV product
      float pf[kCW];
#pragma unroll
      for (int cb = 0; cb < kCW / 32; ++cb) {
        const int col0 = kCW * w + 32 * cb;
        uint32_t sv[32];
        tmem_ld32p(lane_addr + Cfg::kColS + col0, sv);
        tmem_wait_ld();
        uint32_t pkP[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int cc = col0 + 2 * x;
          uint64_t nl2;
          if (kDQ) {
            nl2 = pack2(my_nl, my_nl);
          } else {
            const float2 a = reinterpret_cast<const float2*>(st_nl)[cc / 2];
            nl2 = pack2(a.x, a.y);
          }
          const uint64_t a2 = ffma2(pack2(__uint_as_float(sv[2 * x]), __uint_as_float(sv[2 * x + 1])), l2e2, nl2);
          float p0, p1;
          if (x % 8 < kBwdSfuPairs) {
            float a0, a1;
            unpack2(a2, a0, a1);
            p0 = ex2(a0);
            p1 = ex2(a1);
          } else {
            unpack2(exp2_poly2(a2), p0, p1);
          }
          if (diag) {
            // dK/dV: rows are keys, a query before the key sees nothing;
            // dQ: rows are queries, keys after the query are masked
            if (kDQ ? (cc > r) : (cc < r)) p0 = 0.f;
            if (kDQ ? (cc + 1 > r) : (cc + 1 < r)) p1 = 0.f;
          }
          pf[32 * cb + 2 * x] = p0;
          pf[32 * cb + 2 * x + 1] = p1;
          pkP[x] = pack_bf16x2(p0, p1);
        }
        if (!kDQ) tmem_st16(lane_addr + Cfg::kColS + kCW * w + 16 * cb, pkP);
      }
      // S has been read (and, for dK/dV, P written): the MMA thread may go on
      if (!kDQ) tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_done);
      // dS = P (dP - delta)
      ok = __all_sync(0xffffffffu, mbar_wait(dp_ready, (uint32_t)n & 1, abort_flag, status));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < kCW / 32; ++cb) {
        const int col0 = kCW * w + 32 * cb;
        uint32_t pkD[16];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {   // 16 columns of dP at a time (register budget)
          uint32_t pv[16];
          tmem_ld16p(lane_addr + Cfg::kColP + col0 + 16 * hh, pv);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const int cc = col0 + 16 * hh + 2 * x;
            uint64_t dl2;
            if (kDQ) {
              dl2 = pack2(-my_dl, -my_dl);
            } else {
              const float2 b = reinterpret_cast<const float2*>(st_dl)[cc / 2];
              dl2 = pack2(-b.x, -b.y);
            }
            const int pi = 32 * cb + 16 * hh + 2 * x;
            float d0, d1;
            unpack2(fmul2(pack2(pf[pi], pf[pi + 1]),
                          fadd2(pack2(__uint_as_float(pv[2 * x]), __uint_as_float(pv[2 * x + 1])), dl2)),
                    d0, d1);
            pkD[8 * hh + x] = pack_bf16x2(d0, d1);
          }
        }
        tmem_st16(lane_addr + (kDQ ? Cfg::kColF + 64 * (n % 2) + (kCW / 2) * w : Cfg::kColP + kCW * w) + 16 * cb,
                  pkD);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_done);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, status));
    if (ok) {
      tc_fence_after();
      const int64_t grow = rowbase + (int64_t)tile.row * kRows + r;
      // dK/dV: the 2D output columns of a row (dV, with the AWM part added,
      // then dK) split evenly over the warpgroups; dQ: 32 columns per
      // warpgroup (those past D have none).  `active` is warp-uniform.
      constexpr int OW = kDQ ? (D / kEW > 32 ? D / kEW : 32) : 2 * D / kEW;
      static_assert(OW % 32 == 0, "whole 32-column TMEM loads in the epilogue");
      const int c0 = w * OW;
      const bool active = !kDQ || c0 < D;
      const bool is_dk = !kDQ && c0 >= D;
      const int cc0 = is_dk ? c0 - D : c0;
      const uint32_t col = (is_dk ? Cfg::kColB : Cfg::kColA) + (uint32_t)cc0;
      __nv_bfloat16* orow = (is_dk ? out_b : out_a) + grow * D + cc0;
      const float* add = (!kDQ && !is_dk && dv_add) ? dv_add + grow * D + cc0 : nullptr;
#pragma unroll 1
      for (int cb = 0; cb < (active ? OW / 32 : 0); ++cb) {
        uint32_t o[32];
        tmem_ld32(lane_addr + col + cb * 32, o);
        tmem_wait_ld();
        float f[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) f[x] = __uint_as_float(o[x]);
        if (add) {
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const float4 a4 = reinterpret_cast<const float4*>(add + cb * 32)[x];
            f[4 * x] += a4.x;
            f[4 * x + 1] += a4.y;
            f[4 * x + 2] += a4.z;
            f[4 * x + 3] += a4.w;
          }
        }
        uint4 v4[4];
        uint32_t* vp = reinterpret_cast<uint32_t*>(v4);
#pragma unroll
        for (int x = 0; x < 16; ++x) vp[x] = pack_bf16x2(f[2 * x], f[2 * x + 1]);
        uint4* dst = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
        for (int x = 0; x < 4; ++x) dst[x] = v4[x];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// --------------------------------------------------------------- host --

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn bwd_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [rows, d] bf16 row-major as a 2D tensor; box 128 rows x 64 columns,
// 128-byte swizzle (the K-major / MN-major UMMA operand layout).
cudaError_t bwd_map(CUtensorMap* m, const void* base, int64_t rows, int d) {
  EncodeTiledFn fn = bwd_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_sca_bwd_tc_impl(const BwdProblem& b, const BwdWorkspace& w, cudaStream_t st, int part) {
  using Cfg = BwdCfg<D>;
  const Problem& p = b.f;
  const int64_t rows = p.B * p.H * p.T;
  CUtensorMap mq, mk, mv, mdo;
  cudaError_t e;
  if ((e = bwd_map(&mq, p.q, rows, D)) != cudaSuccess) return e;
  if ((e = bwd_map(&mk, p.k, rows, D)) != cudaSuccess) return e;
  if ((e = bwd_map(&mv, p.v, rows, D)) != cudaSuccess) return e;
  if ((e = bwd_map(&mdo, b.dout_sca, rows, D)) != cudaSuccess) return e;
  const unsigned grid = (unsigned)(p.B * p.H * (p.T / kRows));
  const int T = (int)p.T, c = (int)p.c;
  if ((e = cudaFuncSetAttribute(sca_bwd_tc_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg::kAlloc)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(sca_bwd_tc_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg::kAlloc)) != cudaSuccess)
    return e;
  if (part == 0)
    // dK, dV (the AWM part of dV is added in the epilogue)
    sca_bwd_tc_kernel<D, false><<<grid, EwLayout<false>::threads, Cfg::kAlloc, st>>>(
        mk, mv, mq, mdo, w.nlse2, w.delta, w.dv_awm, static_cast<__nv_bfloat16*>(b.dv),
        static_cast<__nv_bfloat16*>(b.dk), T, c, p.status);
  else
    sca_bwd_tc_kernel<D, true><<<grid, EwLayout<true>::threads, Cfg::kAlloc, st>>>(
        mq, mdo, mk, mv, w.nlse2, w.delta, nullptr, static_cast<__nv_bfloat16*>(b.dq), nullptr, T, c, p.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sca_bwd_tc(const BwdProblem& b, const BwdWorkspace& w, cudaStream_t st, int part) {
  return b.f.d == 64 ? launch_sca_bwd_tc_impl<64>(b, w, st, part) : launch_sca_bwd_tc_impl<128>(b, w, st, part);
}

}  // namespace gecko
