// Adaptive Working Memory kernels on 5th-generation tensor cores (sm_100a).
//
// The AWM of the Gecko digest (paper.rainbus.top, core method and method
// step details, steps 4-5) needs, per (b, h) and chunk s, the online-softmax
// kernel Phi_s = exp(Km_s - log z^s) and the feature softmax Psi_s.  Since
// Phi_s = rho_s (.) Phi~_s with the chunk-local Phi~_s = exp(Km_s - lse_s)
// (values in (0, 1], columns summing to 1) and rho_s = exp(lse_s - log z^s),
// the chunk kernel computes
//   Bm_s = Phi~_s^T V_s,   Cm_s = Phi~_s^T Psi_s        (d x d, fp32)
// independently of the prefix over chunks, and the carry applies the row
// scales: M'_{s+1} = r_s (.) M'_s + rho_s (.) (Bm_s - Cm_s M'_s).  The
// readout is O_m,s = psi(Qm_s) M'_{s-1}.  Phi~, Psi and psi take fp32
// exponentials on the SFU (packed f16 ones give the same number of results
// per clock on B200 and cost conversions) and enter the tensor core as bf16.
//
// awm_chunk_tc_kernel: one CTA per (chunk, bh), two per SM.  The chunk is
// streamed in tiles of 64 tokens; V and K_m tiles arrive by TMA; 128 threads
// (two per token) compute Phi and Psi in fp32 and store them as bf16 next
// to V in one 128-byte-swizzled, MN-major stage [V | Psi | Phi], so a single
// tcgen05.mma with M = d, N = 2d accumulates [Phi^T V | Phi^T Psi] in TMEM.
// In the forward (one CTA per chunk) the kernel also computes each chunk's
// per-feature log-sum-exp lse_s: it exponentiates against a per-feature
// reference (the first tile's column maximum; a chunk whose keys climb too
// far above it is redone with a running maximum raised lazily with a
// rescale of the accumulated rows), reads the column sums of those
// exponentials off the Cm block (every row of Psi sums to 1) and
// normalises Bm and Cm in the epilogue, so K_m is read once.
//
// awm_carry_tc_kernel (d = 128): the sequential carry, one CTA per (b, h),
// the product Cm_s M'_s as bf16 hi + lo MMAs; it also writes M'_s as the
// readout's bf16 operand image.
//
// awm_readout_tc_kernel: persistent, a contiguous range of 128-row tiles per
// CTA; Q_m tiles by TMA into a 4-stage ring, psi numerators formed in place
// (K-major A operand), the operand image of M'_{s-1} by one bulk copy per
// chunk, the output tile staged in the freed stage and stored by TMA.
#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

// ------------------------------------------------------------ chunk GEMMs --


// What a chunk-kernel launch computes.
//   kChunkFwd    Bm = Phi~^T V, Cm = Phi~^T Psi with bf16 operands:
//                stage [V | Psi | Phi].
//   kChunkSplit  the same products with each computed operand carried as two
//                bf16 parts (hi + lo, fp32 exponentials), for a backward whose
//                softmax gradients keep only the small differences between
//                the rows of M': stage [V | Psi_hi | Psi_lo | Phi_hi | Phi_lo];
//                D += Phi_hi^T [V | Psi_hi] + Phi_lo^T [V | Psi_hi], Cm += Phi_hi^T Psi_lo.
//   kChunkE      E = psi(Q_m)^T dO_m for the backward (Q_m arrives in the
//                K_m slot, dO_m in the V slot): stage [dO | psi_hi | psi_lo].
//   kChunkFwdStats  kChunkFwd with the chunk's per-feature log-sum-exp
//                computed in the same pass: Phi^ = exp(Km - m_f)
//                with a lazily raised per-feature reference m_f, the column
//                sums read off the Cm block (rows of Psi sum to 1), and
//                Bm, Cm normalised in the epilogue, which also writes lse.
//                Given a flag array, only the chunks flagged there run (the
//                fix-up pass of kChunkFwdStatsFirst).
//   kChunkFwdStatsFirst  the same statistics with the reference m_f fixed at
//                the first tile's column maximum, so the later tiles need no
//                column maxima and no barriers; a chunk whose exponent
//                arguments climb more than kRefSlack above that reference
//                is flagged (its results are then unusable) and redone by
//                kChunkFwdStats.
enum ChunkMode { kChunkFwd = 0, kChunkSplit = 1, kChunkE = 2, kChunkFwdStats = 3, kChunkFwdStatsFirst = 4 };

// Growth (log2 units) that kChunkFwdStatsFirst allows the exponentials above
// the first tile's reference: Phi^ <= 2^32, so the sums over a chunk of up
// to 2^31 tokens stay below 2^63, and their products with values |V| < 2^64
// inside the fp32 range.
constexpr float kRefSlack = 32.f;

// Compute threads of the chunk kernel: two per token row of a 64-token
// tile.  (Eight compute warps, four threads per row, measured slower: 0.228
// against 0.219-0.224 ms at the bench workload; so did hinting the next 2-8
// tiles into L2 ahead of the two-stage ring: no change.)
constexpr int kChunkCompute = 128;
template <int D, int Mode = kChunkFwd>
struct ChunkCfg {
  // Tokens per tile and stages.  32-token tiles through 4 stages (three
  // loads in flight instead of one) measured slower for the forward mode
  // (0.210 against 0.183 ms at the bench workload), so every mode streams
  // 64-token tiles through 2 stages.
  static constexpr int kKT = 64;
  static constexpr int kStages = 2;
  static constexpr int kTPR = kChunkCompute / kKT;        // compute threads per token row
  static constexpr int kBox = kKT * 128;                 // one [kKT x 64] bf16 box
  static constexpr int kOperand = (D / 64) * kBox;       // a [kKT x D] operand
  static constexpr int kSlots = Mode == kChunkSplit ? 5 : 3;
  static constexpr int kStage = kSlots * kOperand;
  static constexpr int kBarOff = kStages * kStage;
  // v_full[kStages], op_full[kStages], stage_empty[kStages], acc_full
  static constexpr int kNumBars = 3 * kStages + 1;
  // D floats: -log2(e) times each feature's reference (16-byte aligned for
  // vector loads)
  static constexpr int kLzOff = (kBarOff + kNumBars * 8 + 15) / 16 * 16;
  static_assert(kLzOff % 16 == 0, "vector loads of the references");
  static constexpr int kMiscOff = kLzOff + D * 4;
  // fused statistics: per-tile column maxima of K_m from 8 groups of 8 rows
  // ([8][D] bf16, stored 16 bytes at a time)
  static constexpr int kPartOff = (kMiscOff + 16 + 15) / 16 * 16;
  static_assert(kPartOff % 16 == 0, "16-byte stores of the column maxima");
  // [kChunkCompute / (D / 8) row groups][D] bf16 = 2 KB
  static constexpr int kBytes = kPartOff + (Mode == kChunkFwdStats || Mode == kChunkFwdStatsFirst ? 2048 : 0);
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = Mode == kChunkE ? D : (D == 128 ? 256 : 128);
};

// Warps 0-3 compute, warp 4 = TMA producer, warp 5 = MMA issuer; two CTAs
// per SM.
constexpr int kChunkThreads = kChunkCompute + 64;
constexpr int kChunkTmaWarp = kChunkCompute / 32, kChunkMmaWarp = kChunkTmaWarp + 1;
template <int D, int Mode = kChunkFwd>
__global__ void __launch_bounds__(kChunkThreads, 2) awm_chunk_tc_kernel(const __grid_constant__ CUtensorMap map_v,
                                                           const __grid_constant__ CUtensorMap map_km,
                                                           float* __restrict__ lse, float* __restrict__ Bm,
                                                           float* __restrict__ Cm, uint16_t* __restrict__ Cimg,
                                                           int T, int c, int koff, int parts, int* flags,
                                                           int* status) {
  using Cfg = ChunkCfg<D, Mode>;
  // kChunkFwdStats / kChunkFwdStatsFirst: the forward products with the
  // chunk's statistics computed here: it writes lse instead of reading it
  constexpr bool kFirstRef = Mode == kChunkFwdStatsFirst;
  constexpr bool kStats = Mode == kChunkFwdStats || kFirstRef;
  constexpr bool kFwd = Mode == kChunkFwd || kStats;
  // fused statistics: the column maxima of a tile come from kRG groups of
  // kKT / kRG rows, one thread per (row group, 8 features)
  constexpr int kFG = D / 8, kRG = kChunkCompute / kFG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int NS = Cfg::kStages, kKT = Cfg::kKT;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* v_full = bars;          // [NS] TMA -> MMA
  uint64_t* op_full = bars + NS;    // [NS] compute -> MMA (128 arrivals)
  uint64_t* st_empty = bars + 2 * NS;   // [NS] MMA -> TMA, compute
  uint64_t* acc_full = bars + 3 * NS;
  // -log2(e) * (the reference of each feature): lse_s, or m_f with the fused statistics
  float* nref2 = reinterpret_cast<float*>(smem + Cfg::kLzOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);
  // kChunkFwdStatsFirst: set when an exponent argument exceeded kRefSlack
  volatile int* outgrown = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 8);

  // `parts` CTAs share a chunk (forward mode only): CTA part p takes tiles
  // [p n / parts, (p + 1) n / parts) and adds its products into Bm, Cm
  // (zeroed by the host) with vector reductions
  const int s = blockIdx.x / parts, part = blockIdx.x % parts, S = gridDim.x / parts;
  const int64_t bh = blockIdx.y;
  // the readouts of chunks 1 and 2 read a zero state: their E is never used
  if (Mode == kChunkE && s < 2) return;
  // the fix-up pass redoes only the chunks that the first-tile pass flagged
  if (Mode == kChunkFwdStats && flags != nullptr && flags[bh * S + s] == 0) return;
  const int warp = warp_id_uniform(), lane = threadIdx.x % 32;
  const int t0 = part * (c / kKT) / parts;
  const int n_tiles = (part + 1) * (c / kKT) / parts - t0;
  const int64_t row0 = bh * (int64_t)T + (int64_t)s * c + (int64_t)t0 * kKT;
  // v carries koff extra leading rows per (b, h) when a sequence is continued
  const int64_t vrow0 = bh * (int64_t)(T + koff) + koff + (int64_t)s * c + (int64_t)t0 * kKT;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(v_full + i, 1);
      mbar_init(op_full + i, kChunkCompute);
      mbar_init(st_empty + i, 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    *outgrown = 0;
    fence_mbar_init();
  }
  if (Mode != kChunkE && !kStats)
    for (int f = threadIdx.x; f < D; f += blockDim.x) nref2[f] = -lse[(bh * S + s) * D + f] * kLog2e;
  if (warp == kChunkMmaWarp) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kChunkTmaWarp) {
    // ------------------------------------------------ V and K_m by TMA --
    // V into the V slot, K_m into the Psi slot (where it is turned into Psi
    // in place), both on v_full.
    if (lane == 0) {
      tma_prefetch_desc(&map_v);
      tma_prefetch_desc(&map_km);
      int issued = 0;
      for (int kt = 0; kt < n_tiles; ++kt) {
        const int st = kt % NS;
        if (!mbar_wait(st_empty + st, ((kt / NS) & 1) ^ 1, abort_flag, status)) break;
        mbar_arrive_expect_tx(v_full + st, 2 * Cfg::kOperand);
        ++issued;
        for (int b = 0; b < D / 64; ++b) {
          tma_load_2d(smem + st * Cfg::kStage + b * Cfg::kBox, &map_v, v_full + st, b * 64,
                      (int)(vrow0 + (int64_t)kt * kKT));
          tma_load_2d(smem + st * Cfg::kStage + Cfg::kOperand + b * Cfg::kBox, &map_km, v_full + st, b * 64,
                      (int)(row0 + (int64_t)kt * kKT));
        }
      }
      if (*abort_flag) {
        // the copies issued land before the CTA exits
        for (int t = issued > NS ? issued - NS : 0; t < issued; ++t) mbar_wait_drain(v_full + t % NS, (t / NS) & 1);
      }
    }
    __syncwarp();
  } else if (warp == kChunkMmaWarp) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(D, 2 * D, true, true);
      constexpr uint32_t idesc1 = idesc_bf16_f32(D, D, true, true);
      const uint32_t base = smem_u32(smem);
      bool ok = true;
      for (int kt = 0; kt < n_tiles && ok; ++kt) {
        const int st = kt % NS;
        const uint32_t ph = (kt / NS) & 1;
        if (!(ok = mbar_wait(v_full + st, ph, abort_flag, status))) break;
        if (!(ok = mbar_wait(op_full + st, ph, abort_flag, status))) break;
        tc_fence_after();
        const uint32_t sb = base + st * Cfg::kStage;
        auto desc = [&](int slot, int kk) { return sdesc_sw128(sb + slot * Cfg::kOperand + kk * 2048, Cfg::kBox, 1024); };
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk) {
          const uint32_t acc = (kt > 0 || kk > 0) ? 1u : 0u;
          if (kFwd) {
            // A = Phi^T (M = D features, MN-major), B = [V | Psi] (N = 2D, MN-major)
            umma_ss(tmem, desc(2, kk), desc(0, kk), idesc, acc);
          } else if (Mode == kChunkSplit) {
            umma_ss(tmem, desc(3, kk), desc(0, kk), idesc, acc);        // Phi_hi^T [V | Psi_hi]
            umma_ss(tmem, desc(4, kk), desc(0, kk), idesc, 1u);         // Phi_lo^T [V | Psi_hi]
            umma_ss(tmem + D, desc(3, kk), desc(2, kk), idesc1, 1u);    // Phi_hi^T Psi_lo
          } else {
            umma_ss(tmem, desc(1, kk), desc(0, kk), idesc1, acc);       // psi_hi^T dO
            umma_ss(tmem, desc(2, kk), desc(0, kk), idesc1, 1u);        // psi_lo^T dO
          }
        }
        umma_commit(st_empty + st);
      }
      umma_commit(acc_full);
      mbar_wait_drain(acc_full, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------ Phi / Psi, then epilogue --
    constexpr int TPR = Cfg::kTPR;        // threads per token row
    const int r = threadIdx.x / TPR;      // token row within the tile
    const int h = threadIdx.x % TPR;      // which part of the features
    constexpr int HF = D / TPR;           // features per thread
    bool ok = true;
    // fused statistics: this thread's feature f = threadIdx.x (TMEM lane f
    // of the accumulator) and its reference m_f (log2 units)
    float m_f = 0.f;
    // kChunkFwdStatsFirst: the largest exponent argument of this thread
    float umax = -INFINITY;
    for (int kt = 0; kt < n_tiles; ++kt) {
      const int st = kt % NS;
      // column maxima (and the barriers around them) on every tile, or on
      // the first one only
      const bool colmax = kStats && (!kFirstRef || kt == 0);
      // V and K_m of this tile have landed (the copy also waited for the
      // MMAs of tile kt - NS to release the stage)
      if (colmax) {
        // the compute warps leave the loop together (they meet at named
        // barriers below)
        ok = bar_and(1, kChunkCompute, mbar_wait(v_full + st, (kt / NS) & 1, abort_flag, status));
      } else {
        ok = __all_sync(0xffffffffu, mbar_wait(v_full + st, (kt / NS) & 1, abort_flag, status));
      }
      if (!ok) break;
      uint8_t* stg = smem + st * Cfg::kStage;
      if (colmax) {
        // Column maxima of the K_m tile: thread (rg, g) takes the kKT / kRG
        // rows of group rg for features 8 g .. 8 g + 7, then the thread of
        // feature f combines the kRG row groups.  The thread of feature f
        // is the one whose TMEM lane holds accumulator row f: lane f for
        // M = 128, lane 16 w + (f % 16) of warp w = f / 16 for M = 64.
        __nv_bfloat162* part = reinterpret_cast<__nv_bfloat162*>(smem + Cfg::kPartOff);
        {
          constexpr int kRPG = kKT / kRG;
          const int g = threadIdx.x % kFG, rg = threadIdx.x / kFG;
          uint4 mx = *reinterpret_cast<const uint4*>(stg + Cfg::kOperand + sw128_off(kRPG * rg, 8 * g, kKT));
          __nv_bfloat162* m2 = reinterpret_cast<__nv_bfloat162*>(&mx);
#pragma unroll
          for (int rr = 1; rr < kRPG; ++rr) {
            uint4 v = *reinterpret_cast<const uint4*>(stg + Cfg::kOperand + sw128_off(kRPG * rg + rr, 8 * g, kKT));
            const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
            for (int j = 0; j < 4; ++j) m2[j] = __hmax2(m2[j], v2[j]);
          }
          *reinterpret_cast<uint4*>(part + rg * (D / 2) + 4 * g) = mx;
        }
        const bool feat = D == 128 ? threadIdx.x < D : lane < 16;
        named_bar_sync(1, kChunkCompute);
        const int f = feat ? (D == 128 ? (int)threadIdx.x : warp * 16 + lane) : 0;
        const __nv_bfloat16* ph = reinterpret_cast<const __nv_bfloat16*>(part);
        float mt = __bfloat162float(ph[f]);
#pragma unroll
        for (int q = 1; q < kRG; ++q) mt = fmaxf(mt, __bfloat162float(ph[q * D + f]));
        const float mt2 = feat ? mt * kLog2e : 0.f;
        // The reference is raised lazily, only when the tile's maximum
        // exceeds it by more than 8 (every exponential stays <= 2^8), and
        // the accumulated rows of feature f are then scaled to the new one.
        const bool grow = feat && kt > 0 && mt2 > m_f + 8.f;
        if (kt == 0) m_f = mt2;
        bool rok = true;
        if (__any_sync(0xffffffffu, grow)) {
          // TMEM rows are scaled with warp-collective loads and stores once
          // the MMAs of tile kt - 1 are done
          rok = __all_sync(0xffffffffu, mbar_wait(st_empty + (kt - 1) % NS, ((kt - 1) / NS) & 1, abort_flag, status));
          if (rok) {
            tc_fence_after();
            const float scale = grow ? ex2(m_f - mt2) : 1.f;
            const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
            for (int cb = 0; cb < 2 * D / 32; ++cb) {
              uint32_t v[32];
              tmem_ld32(taddr + cb * 32, v);
              tmem_wait_ld();
#pragma unroll
              for (int x = 0; x < 32; ++x) v[x] = __float_as_uint(__uint_as_float(v[x]) * scale);
              tmem_st32(taddr + cb * 32, v);
            }
            tmem_wait_st();
          }
        }
        if (grow) m_f = mt2;
        if (feat) nref2[f] = -m_f;
        // every reference is in place and every column maximum was read
        // before K_m is overwritten by Psi below
        ok = bar_and(1, kChunkCompute, rok);
        if (!ok) break;
      }
      float x[HF];
#pragma unroll
      for (int i = 0; i < HF / 8; ++i) {
        const uint4 raw = *reinterpret_cast<const uint4*>(stg + Cfg::kOperand + sw128_off(r, h * HF + 8 * i, kKT));
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f2 = __bfloat1622float2(p2[j]);
          x[8 * i + 2 * j] = f2.x;
          x[8 * i + 2 * j + 1] = f2.y;
        }
      }
      // row maximum over this thread's features (four 3-input chains)
      float m4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
      for (int i = 4; i + 8 <= HF; i += 8)
#pragma unroll
        for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], x[i + q], x[i + 4 + q]);
#pragma unroll
      for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], x[HF - 4 + q]);
      float mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
#pragma unroll
      for (int o = 1; o < TPR; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mx2 = mx * kLog2e;
      float e[HF], sum = 0.f;
      if (kFwd) {
        // fp32 exponentials on the SFU (the packed f16 form gives the same
        // number of results per clock and costs conversions); arguments by
        // packed FMA
        const uint64_t l2e2 = pack2(kLog2e, kLog2e), nmx2 = pack2(-mx2, -mx2);
        uint64_t sum2 = pack2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < HF / 8; ++i) {
          const int col = h * HF + 8 * i;
          const float4 za = *reinterpret_cast<const float4*>(nref2 + col);
          const float4 zb = *reinterpret_cast<const float4*>(nref2 + col + 4);
          const uint64_t nz[4] = {pack2(za.x, za.y), pack2(za.z, za.w), pack2(zb.x, zb.y), pack2(zb.z, zb.w)};
          uint4 pf;
          uint32_t* qq = reinterpret_cast<uint32_t*>(&pf);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int a = 8 * i + 2 * j;
            const uint64_t x2 = pack2(x[a], x[a + 1]);
            float u0, u1, v0, v1;
            unpack2(ffma2(x2, l2e2, nz[j]), u0, u1);
            if (kFirstRef) umax = fmax3(umax, u0, u1);
            qq[j] = pack_bf16x2(ex2(u0), ex2(u1));
            unpack2(ffma2(x2, l2e2, nmx2), v0, v1);
            e[a] = ex2(v0);
            e[a + 1] = ex2(v1);
            sum2 = fadd2(sum2, pack2(e[a], e[a + 1]));
          }
          *reinterpret_cast<uint4*>(stg + 2 * Cfg::kOperand + sw128_off(r, col, kKT)) = pf;
        }
        float s0, s1;
        unpack2(sum2, s0, s1);
        sum = s0 + s1;
      } else {
        // fp32 exponentials; Phi (split mode only) as bf16 hi and lo parts
#pragma unroll
        for (int i = 0; i < HF / 8; ++i) {
          const int col = h * HF + 8 * i;
          uint4 fh, fl;
          uint32_t* fhp = reinterpret_cast<uint32_t*>(&fh);
          uint32_t* flp = reinterpret_cast<uint32_t*>(&fl);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int a = 8 * i + 2 * j;
            if (Mode == kChunkSplit) {
              const float p0 = ex2(fmaf(x[a], kLog2e, nref2[col + 2 * j]));
              const float p1 = ex2(fmaf(x[a + 1], kLog2e, nref2[col + 2 * j + 1]));
              fhp[j] = pack_bf16x2(p0, p1);
              const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&fhp[j]));
              flp[j] = pack_bf16x2(p0 - hi.x, p1 - hi.y);
            }
            e[a] = ex2(fmaf(x[a], kLog2e, -mx2));
            e[a + 1] = ex2(fmaf(x[a + 1], kLog2e, -mx2));
            sum += e[a] + e[a + 1];
          }
          if (Mode == kChunkSplit) {
            *reinterpret_cast<uint4*>(stg + 3 * Cfg::kOperand + sw128_off(r, col, kKT)) = fh;
            *reinterpret_cast<uint4*>(stg + 4 * Cfg::kOperand + sw128_off(r, col, kKT)) = fl;
          }
        }
      }
#pragma unroll
      for (int o = 1; o < TPR; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float inv = 1.f / sum;
#pragma unroll
      for (int i = 0; i < HF / 8; ++i) {
        const int col = h * HF + 8 * i;
        uint4 ps, pl;
        uint32_t* pp = reinterpret_cast<uint32_t*>(&ps);
        uint32_t* plp = reinterpret_cast<uint32_t*>(&pl);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float a0, a1;
          unpack2(fmul2(pack2(e[8 * i + 2 * j], e[8 * i + 2 * j + 1]), pack2(inv, inv)), a0, a1);
          pp[j] = pack_bf16x2(a0, a1);
          if (!kFwd) {
            const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pp[j]));
            plp[j] = pack_bf16x2(a0 - hi.x, a1 - hi.y);
          }
        }
        *reinterpret_cast<uint4*>(stg + Cfg::kOperand + sw128_off(r, col, kKT)) = ps;
        if (!kFwd) *reinterpret_cast<uint4*>(stg + 2 * Cfg::kOperand + sw128_off(r, col, kKT)) = pl;
      }
      // generic-proxy writes must be visible to the tensor core (async proxy)
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      if (kStats) tc_fence_before();   // orders the TMEM rescale before the next MMA
      mbar_arrive(op_full + st);
    }
    if (kFirstRef && umax > kRefSlack) *outgrown = 1;
    // epilogue (warps 0-3): accumulator row f = TMEM lane; columns [0, D) = Bm, [D, 2D) = Cm
    if (warp >= 4) ok = false;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, status));
    if (ok) {
      tc_fence_after();
      // M = 128: row f lives in lane f.  M = 64: rows 16w..16w+15 live in
      // lanes 32w..32w+15 of warp w.
      const bool valid = D == 128 || lane < 16;
      const int f = D == 128 ? warp * 32 + lane : warp * 16 + lane;
      const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
      const int64_t o = (bh * S + s) * (int64_t)D * D + (int64_t)f * D;
      // fused statistics: the column sum of Phi^ over the chunk is the row
      // sum of the Cm block (every row of Psi sums to 1); Bm and Cm rows are
      // divided by it and lse_f = ln(sum) + m_f ln 2
      float inv = 1.f;
      if (kStats) {
        float sum = 0.f;
#pragma unroll 1
        for (int cb = D / 32; cb < 2 * D / 32; ++cb) {
          uint32_t v[32];
          tmem_ld32(taddr + cb * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) sum += __uint_as_float(v[x]);
        }
        inv = 1.f / sum;
        if (valid) lse[(bh * S + s) * D + f] = (m_f + log2f(sum)) * kLn2;
      }
#pragma unroll 1
      for (int cb = 0; cb < (Mode == kChunkE ? D : 2 * D) / 32; ++cb) {
        uint32_t v[32];
        tmem_ld32(taddr + cb * 32, v);
        tmem_wait_ld();
        if (kStats) {
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = __float_as_uint(__uint_as_float(v[x]) * inv);
        }
        if (valid) {
          float* dst = (cb * 32 < D) ? (Bm + o + cb * 32) : (Cm + o + cb * 32 - D);
          if (Mode == kChunkFwd && parts > 1) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              red_add_v4(dst + 4 * i, __uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                         __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              reinterpret_cast<float4*>(dst)[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                              __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
          if (kFwd && D == 128 && Cimg && parts == 1 && cb * 32 >= D) {
            // Cm row f as the tensor-core carry's bf16 A operand (K-major)
            uint8_t* img = reinterpret_cast<uint8_t*>(Cimg + (bh * S + s) * (int64_t)D * D);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              *reinterpret_cast<uint4*>(img + sw128_off(f, cb * 32 - D + 8 * i, 128)) =
                  make_uint4(pack_bf16x2(__uint_as_float(v[8 * i]), __uint_as_float(v[8 * i + 1])),
                             pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                             pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                             pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kChunkMmaWarp) tmem_dealloc(tmem, Cfg::kTmemCols);
  // every chunk's flag is written, so the array needs no clearing
  if (kFirstRef && threadIdx.x == 0) flags[bh * S + s] = *outgrown;
}

// Cm_s rounded to bf16 in the carry's K-major 128-byte-swizzled operand
// layout (the image the forward chunk kernel writes itself when one CTA owns
// the chunk), from the fp32 Cm that several CTAs accumulated.  grid B*H*S,
// one thread per row.
__global__ void __launch_bounds__(128) awm_cimg_kernel(const float* __restrict__ Cm, uint16_t* __restrict__ Cimg) {
  const int64_t m = blockIdx.x;
  const int f = threadIdx.x;
  const float* row = Cm + m * 128 * 128 + (int64_t)f * 128;
  uint8_t* img = reinterpret_cast<uint8_t*>(Cimg + m * 128 * 128);
#pragma unroll 4
  for (int cb = 0; cb < 128; cb += 8) {
    const float4 a = *reinterpret_cast<const float4*>(row + cb);
    const float4 b = *reinterpret_cast<const float4*>(row + cb + 4);
    *reinterpret_cast<uint4*>(img + sw128_off(f, cb, 128)) =
        make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
  }
}

// --------------------------------------------------------------- readout --

template <int D>
struct ReadoutCfg {
  static constexpr int kTile = 128 * D * 2;      // a 128-row tile, bf16, D / 64 swizzled boxes of 16 KB
  static constexpr int kBox = 128 * 128;         // one [128 rows x 64] box
  // Q_m tile ring; each stage returns to the producer once the tile's MMA
  // has read it
  // One M' image buffer and four input stages measured slightly faster than
  // two image buffers and three stages (0.1218 against 0.1236 ms at the
  // bench workload): the image of the next chunk then waits for the last
  // MMA of the current one, about once per 32 tiles.
  static constexpr int kImgBufs = 1;
  static constexpr int kStages = 4;
  static constexpr int kImg = D * D * 2;         // one M' operand image
  static constexpr int kImgOff = kStages * kTile;
  static constexpr int kOutOff = kImgOff + kImgBufs * kImg;   // two output staging tiles
  static constexpr int kBarOff = kOutOff + 2 * kTile;
  // q_full, op_full, st_empty [kStages]; img_full, img_empty, acc_full,
  // acc_empty, out_ready, out_free [2]; drain
  static constexpr int kNumBars = 3 * kStages + 12 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory above the per-block limit");
  static constexpr uint32_t kTmemCols = 2 * D;   // two accumulators
  // psi warps (4: one thread per row; 8: two per row, measured 0.129 against
  // 0.135 ms at the bench workload); then 4 epilogue warps, the TMA warp
  // and the MMA warp
#ifndef GECKO_READOUT_PSI_WARPS
#define GECKO_READOUT_PSI_WARPS 8
#endif
  static constexpr int kPsiWarps = GECKO_READOUT_PSI_WARPS;
  static constexpr int kTPR = kPsiWarps / 4;     // psi threads per row
  static constexpr int kEpiWarp0 = kPsiWarps, kTmaWarp = kPsiWarps + 4, kMmaWarp = kPsiWarps + 5;
  static constexpr int kThreads = (kPsiWarps + 6) * 32;
};

// The readout O_m,s = psi(Qm_s) M'_{s-1} (Gecko digest, method step details,
// step 5).  Persistent: CTA b takes a contiguous range of the 128-row tiles
// ordered by (b, h), chunk, tile, balanced by weight (a tile of chunks 1
// and 2 of a fresh sequence only writes zeros: weight 1; every other tile
// reads Q_m and writes out_mem: weight 2).  448 threads:
//   warps 0-7  psi: two threads per row turn it (Q_m tile by TMA, K-major A
//              operand layout) into psi = exp(q - max) / sum in place, bf16;
//   warps 8-11 epilogue: accumulator rows from TMEM to bf16 in one of two
//              output staging tiles, stored by one TMA store; zero tiles
//              are written directly;
//   warp 12    TMA producer: Q_m tiles into a 4-stage ring (a stage is free
//              again once its tile's MMA has read it), and the operand
//              image of M'_{s-1} (bf16, written by the carry in the MN-major
//              B layout) by one bulk copy whenever the chunk changes
//              (one image buffer);
//   warp 13    TMEM allocation and the MMAs (one thread), two accumulators.
template <int D>
__global__ void __launch_bounds__(ReadoutCfg<D>::kThreads, 1)
awm_readout_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_o,
                      const uint16_t* __restrict__ Mimg, __nv_bfloat16* __restrict__ out, int T, int c, int S,
                      int BH, int fresh, int* status) {
  using Cfg = ReadoutCfg<D>;
  constexpr int NS = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* q_full = bars;                // TMA -> psi warps
  uint64_t* op_full = q_full + NS;        // psi warps -> MMA
  uint64_t* st_empty = op_full + NS;      // the tile's MMA read the stage -> TMA
  uint64_t* img_full = st_empty + NS;     // [2] image copy -> MMA
  uint64_t* img_empty = img_full + 2;     // [2] last MMA of the image's chunk -> TMA
  uint64_t* acc_full = img_empty + 2;     // [2] MMA -> epilogue
  uint64_t* acc_empty = acc_full + 2;     // [2] epilogue (128) -> MMA
  uint64_t* out_ready = acc_empty + 2;    // [2] epilogue (128) wrote the output tile -> storing thread
  uint64_t* out_free = out_ready + 2;     // [2] the store of that tile finished reading it -> epilogue
  uint64_t* drain = out_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);

  const int warp = warp_id_uniform(), lane = threadIdx.x % 32;
  const int nt = c / 128;                        // tiles per chunk
  const int zc = fresh ? (S < 2 ? S : 2) : 0;   // leading zero chunks per (b, h)
  // weighted split: per (b, h) the zero tiles weigh 1, the others 2
  const int64_t wbh = (int64_t)zc * nt + 2 * (int64_t)(S - zc) * nt;
  const int64_t W = wbh * BH;
  auto tile_at = [&](int64_t x) -> int64_t {   // first tile whose cumulative weight reaches x
    const int64_t bh = x / wbh, r = x % wbh, z = (int64_t)zc * nt;
    return bh * (int64_t)S * nt + (r < z ? r : z + (r - z + 1) / 2);
  };
  const int64_t u0 = tile_at(W * blockIdx.x / gridDim.x);
  const int64_t u1 = blockIdx.x + 1 == gridDim.x ? (int64_t)BH * S * nt : tile_at(W * (blockIdx.x + 1) / gridDim.x);
  const int m = (int)(u1 - u0);   // tiles of this CTA
  // the CTA's tiles are walked with counters (no 64-bit division per tile)
  struct TileIt {
    int bh, s, kt;
  };
  const TileIt first{(int)(u0 / ((int64_t)S * nt)), (int)((u0 / nt) % S), (int)(u0 % nt)};
  auto next = [&](TileIt& t) {
    if (++t.kt == nt) {
      t.kt = 0;
      if (++t.s == S) {
        t.s = 0;
        ++t.bh;
      }
    }
  };
  auto is_zero = [&](const TileIt& t) { return t.s < zc; };
  auto row_of = [&](const TileIt& t) { return (int64_t)t.bh * T + (int64_t)t.s * c + t.kt * 128; };
  auto img_of = [&](const TileIt& t) { return (int64_t)t.bh * (S + 1) + t.s; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(op_full + i, Cfg::kPsiWarps * 32);
      mbar_init(st_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(img_full + i, 1);
      mbar_init(img_empty + i, 1);
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 128);
      mbar_init(out_ready + i, 128);
      mbar_init(out_free + i, 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == Cfg::kMmaWarp) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == Cfg::kTmaWarp) {
    // --------------------------------------------------- TMA producer --
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      int n = 0, k = -1;
      int64_t cur = -1;
      bool ok = true;
      TileIt t = first;
      for (int i = 0; i < m && ok; ++i, next(t)) {
        if (is_zero(t)) continue;
        const int64_t im = img_of(t);
        if (im != cur) {
          cur = im;
          ++k;
          constexpr int IB = Cfg::kImgBufs;
          if (k >= IB && !(ok = mbar_wait(img_empty + k % IB, ((k / IB) - 1) & 1, abort_flag, status))) break;
          mbar_arrive_expect_tx(img_full + k % IB, Cfg::kImg);
          bulk_load_1d(smem + Cfg::kImgOff + (k % IB) * Cfg::kImg, Mimg + im * (int64_t)D * D, Cfg::kImg,
                       img_full + k % IB);
        }
        const int st = n % NS;
        if (n >= NS && !(ok = mbar_wait(st_empty + st, ((n / NS) - 1) & 1, abort_flag, status))) break;
        mbar_arrive_expect_tx(q_full + st, Cfg::kTile);
        for (int b = 0; b < D / 64; ++b)
          tma_load_2d(smem + st * Cfg::kTile + b * Cfg::kBox, &map_q, q_full + st, b * 64, (int)row_of(t));
        ++n;
      }
      if (!ok) {
        // copies already issued land before the CTA exits
        for (int t = n > NS ? n - NS : 0; t < n; ++t) mbar_wait_drain(q_full + t % NS, (t / NS) & 1);
        for (int t = k >= Cfg::kImgBufs ? k - Cfg::kImgBufs + 1 : 0; t <= k; ++t)
          mbar_wait_drain(img_full + t % Cfg::kImgBufs, (t / Cfg::kImgBufs) & 1);
      }
    }
    __syncwarp();
  } else if (warp == Cfg::kMmaWarp) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
      const uint32_t base = smem_u32(smem);
      int n = 0, k = -1;
      int64_t cur = -1;
      bool ok = true;
      TileIt t = first;
      for (int i = 0; i < m && ok; ++i, next(t)) {
        if (is_zero(t)) continue;
        const int64_t im = img_of(t);
        if (im != cur) {
          cur = im;
          ++k;
          if (!(ok = mbar_wait(img_full + k % Cfg::kImgBufs, (k / Cfg::kImgBufs) & 1, abort_flag, status))) break;
        }
        const int st = n % NS, a = n & 1;
        if (!(ok = mbar_wait(op_full + st, (n / NS) & 1, abort_flag, status))) break;
        if (!(ok = mbar_wait(acc_empty + a, ((n >> 1) & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        const SDesc ad = sdesc_sw128_split(base + st * Cfg::kTile, 16, 1024);
        const SDesc bd = sdesc_sw128_split(base + Cfg::kImgOff + (k % Cfg::kImgBufs) * Cfg::kImg, D * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk / 4) * Cfg::kBox + (kk % 4) * 32;
          umma_ss(tmem + a * D, sdesc_at(ad, koff), sdesc_at(bd, kk * 16 * 128), idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(acc_full + a);
        umma_commit(st_empty + st);   // the psi operand has been read
        // the image is released after the last tile of its chunk in this
        // range (tiles of one chunk are consecutive; the next chunk's tiles,
        // if any, are never zero tiles of the same image)
        if (i + 1 == m || t.kt + 1 == nt) umma_commit(img_empty + k % Cfg::kImgBufs);
        ++n;
      }
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else if (warp < Cfg::kPsiWarps) {
    // -------------------------------------------------- psi numerators --
    constexpr int TPR = Cfg::kTPR, CPT = D / TPR;   // threads per row, columns per thread
    const int r = threadIdx.x / TPR;                // row of the tile
    const int c0 = (threadIdx.x % TPR) * CPT;
    int n = 0;
    bool ok = true;
    TileIt t = first;
    for (int i = 0; i < m; ++i, next(t)) {
      if (is_zero(t)) continue;
      const int st = n % NS;
      ok = __all_sync(0xffffffffu, mbar_wait(q_full + st, (n / NS) & 1, abort_flag, status));
      if (!ok) break;
      uint8_t* tile = smem + st * Cfg::kTile;
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < CPT / 8; ++i) {
        const uint4 q = *reinterpret_cast<const uint4*>(tile + sw128_off(r, c0 + 8 * i, 128));
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f2 = __bfloat1622float2(p2[j]);
          mx = fmax3(mx, f2.x, f2.y);
        }
      }
      if (TPR == 2) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      const float mx2 = mx * kLog2e;
      // fp32 exponentials on the SFU, arguments by packed FMA; psi is
      // normalised before it is rounded to bf16, so the MMA gives the
      // readout rows directly
      const uint64_t l2e2 = pack2(kLog2e, kLog2e), nmx2 = pack2(-mx2, -mx2);
      uint64_t sum2 = pack2(0.f, 0.f);
      float e[CPT];
#pragma unroll
      for (int i = 0; i < CPT / 8; ++i) {
        const uint4 q = *reinterpret_cast<const uint4*>(tile + sw128_off(r, c0 + 8 * i, 128));
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f2 = __bfloat1622float2(p2[j]);
          float u0, u1;
          unpack2(ffma2(pack2(f2.x, f2.y), l2e2, nmx2), u0, u1);
          e[8 * i + 2 * j] = ex2(u0);
          e[8 * i + 2 * j + 1] = ex2(u1);
          sum2 = fadd2(sum2, pack2(e[8 * i + 2 * j], e[8 * i + 2 * j + 1]));
        }
      }
      float sum, s1;
      unpack2(sum2, sum, s1);
      sum += s1;
      if (TPR == 2) sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      const uint64_t inv2 = pack2(1.f / sum, 1.f / sum);
#pragma unroll
      for (int i = 0; i < CPT / 8; ++i) {
        uint4 pv;
        uint32_t* pp = reinterpret_cast<uint32_t*>(&pv);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float a0, a1;
          unpack2(fmul2(pack2(e[8 * i + 2 * j], e[8 * i + 2 * j + 1]), inv2), a0, a1);
          pp[j] = pack_bf16x2(a0, a1);
        }
        *reinterpret_cast<uint4*>(tile + sw128_off(r, c0 + 8 * i, 128)) = pv;
      }
      fence_proxy_async_smem();   // the numerators are read by the tensor core (async proxy)
      mbar_arrive(op_full + st);
      ++n;
    }
  } else {
    // --------------------------------------------------------- epilogue --
    const int q4 = warp % 4;                       // TMEM lane quarter
    const int r = q4 * 32 + lane;                  // row of the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
    const bool leader = warp == Cfg::kEpiWarp0 && lane == 0;   // issues the stores
    int n = 0;
    bool ok = true;
    TileIt t = first;
    for (int i = 0; i < m && ok; ++i, next(t)) {
      if (is_zero(t)) {
        const uint4 z = make_uint4(0, 0, 0, 0);
        uint4* dst = reinterpret_cast<uint4*>(out + (row_of(t) + r) * D);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) dst[i] = z;
        continue;
      }
      const int a = n & 1;   // accumulator and output staging tile
      ok = __all_sync(0xffffffffu, mbar_wait(acc_full + a, (n >> 1) & 1, abort_flag, status));
      if (!ok) break;
      // the store of tile n - 2 has finished reading this staging tile
      if (n >= 2) ok = __all_sync(0xffffffffu, mbar_wait(out_free + a, ((n >> 1) - 1) & 1, abort_flag, status));
      if (!ok) break;
      tc_fence_after();
      uint8_t* tile = smem + Cfg::kOutOff + a * Cfg::kTile;
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t v[32];
        tmem_ld32(lane_addr + a * D + cb * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * x + 0]), __uint_as_float(v[8 * x + 1]));
          w.y = pack_bf16x2(__uint_as_float(v[8 * x + 2]), __uint_as_float(v[8 * x + 3]));
          w.z = pack_bf16x2(__uint_as_float(v[8 * x + 4]), __uint_as_float(v[8 * x + 5]));
          w.w = pack_bf16x2(__uint_as_float(v[8 * x + 6]), __uint_as_float(v[8 * x + 7]));
          *reinterpret_cast<uint4*>(tile + sw128_off(r, cb * 32 + 8 * x, 128)) = w;
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty + a);
      fence_proxy_async_smem();   // the tile is read by the TMA store (async proxy)
      mbar_arrive(out_ready + a);
      if (leader) {
        if (!(ok = mbar_wait(out_ready + a, (n >> 1) & 1, abort_flag, status))) break;
        for (int b = 0; b < D / 64; ++b) tma_store_2d(&map_o, tile + b * Cfg::kBox, b * 64, (int)row_of(t));
        bulk_commit();
        // the previous tile's store has finished reading its staging tile
        bulk_wait_read<1>();
        if (n > 0) mbar_arrive(out_free + (a ^ 1));
      }
      ++n;
    }
    if (leader) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == Cfg::kMmaWarp) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// ------------------------------------------------------------------ carry --

// The sequential carry on the tensor cores, d = 128 (Gecko digest, method
// step details, step 4, with the row scales factored out as in the SIMT
// carry):
//   M'_{s+1} = r_s (.) M'_s + rho_s (.) (Bm_s - Cm_s M'_s).
// Columns of M' evolve independently, so two CTAs share a (b, h), each
// owning 64 columns: 128 threads, thread f holding row f of its columns in
// fp32 registers (the master copy) and TMEM lane f of the product.  Per step
// the product Cm_s M'_s[:, cols] runs as two bf16 MMAs (M = 128, N = 64),
// Cm M_hi + Cm M_lo, with M' split into hi + lo parts and Cm rounded to bf16
// once by the chunk kernel (emulated over 128 chunks of 512 tokens the state
// stays within 2e-5 of fp64); fp32 accumulation.  Cm_s (the chunk kernel's
// bf16 operand image, one bulk copy) and Bm_s[:, cols] (TMA, 128-byte
// swizzled so each thread reads its row without bank conflicts) arrive two
// steps ahead in double buffers.  The hi part of M'_s's B operand is also the
// readout's operand image of M'_s (64 columns = one box of it) and leaves by
// one bulk store.  Only the states the forward reads later are written in
// fp32: Mst[0] = M'_1, and Mst[S-1], Mst[S] (the exported state).
struct CarryTcCfg {
  static constexpr int kD = 128, kN = 64;         // d, columns per CTA
  static constexpr int kA = kD * kD * 2;          // Cm_s, bf16 K-major (two 64-column boxes of 128 rows)
  static constexpr int kBox = 128 * 128;          // one bf16 box [128 rows x 64]
  static constexpr int kOp = kD * kN * 2;         // one B operand: [128 K rows x 64 N] bf16, one box
  static constexpr int kBm = kD * kN * 4;         // Bm_s[:, cols] fp32: two boxes [128 rows x 32]
  static constexpr int kFBox = 128 * 128;         // one fp32 box [128 rows x 32]
  static constexpr int kAOff = 0;                 // [2] A buffers
  static constexpr int kBmOff = kAOff + 2 * kA;   // [2] Bm buffers
  static constexpr int kBhiOff = kBmOff + 2 * kBm, kBloOff = kBhiOff + kOp;
  static constexpr int kBarOff = kBloOff + kOp;   // in_full[2], m_done, drain
  static constexpr int kMiscOff = kBarOff + 32;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

__global__ void __launch_bounds__(128, 1)
awm_carry_tc_kernel(const __grid_constant__ CUtensorMap map_b, const uint16_t* __restrict__ Cimg,
                    const float* __restrict__ ratio, const float* __restrict__ rho, float* __restrict__ Mst, int S,
                    const float* __restrict__ M0, int64_t sd, uint16_t* __restrict__ Mimg,
                    const float* __restrict__ Mprev0, int* status) {
  using Cfg = CarryTcCfg;
  constexpr int D = Cfg::kD, N = Cfg::kN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* in_full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);   // [2] A and Bm of a step
  uint64_t* m_done = in_full + 2;
  uint64_t* drain = in_full + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);
  const int64_t bh = blockIdx.x / 2;
  const int half = blockIdx.x % 2, j0 = half * N;
  const int f = threadIdx.x, warp = f / 32;
  const int64_t mat = (int64_t)D * D;
  float* mout = Mst + bh * (int64_t)(S + 1) * mat;
  uint16_t* iout = Mimg ? Mimg + bh * (int64_t)(S + 1) * mat : nullptr;
  int loads = 0;   // steps whose inputs have been requested (thread 0)
  auto load_step = [&](int s) {   // thread 0: Cm_s and Bm_s[:, cols] into buffer s & 1
    uint64_t* bar = in_full + (s & 1);
    mbar_arrive_expect_tx(bar, Cfg::kA + Cfg::kBm);
    bulk_load_1d(smem + Cfg::kAOff + (s & 1) * Cfg::kA, Cimg + (bh * S + s) * mat, Cfg::kA, bar);
    for (int b = 0; b < N / 32; ++b)
      tma_load_2d(smem + Cfg::kBmOff + (s & 1) * Cfg::kBm + b * Cfg::kFBox, &map_b, bar, j0 + b * 32,
                  (int)((bh * S + s) * D));
    ++loads;
  };

  if (f == 0) {
    mbar_init(in_full, 1);
    mbar_init(in_full + 1, 1);
    mbar_init(m_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_b);
    for (int s = 0; s < 2 && s < S; ++s) load_step(s);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, N);
    tmem_relinquish();
  }
  // M'_1: zero, or the carried M'_cur of a continued sequence
  float m[N];
#pragma unroll
  for (int j = 0; j < N; j += 4) {
    const float4 v =
        M0 ? *reinterpret_cast<const float4*>(M0 + bh * sd + (int64_t)f * D + j0 + j) : make_float4(0, 0, 0, 0);
    m[j] = v.x; m[j + 1] = v.y; m[j + 2] = v.z; m[j + 3] = v.w;
    *reinterpret_cast<float4*>(mout + (int64_t)f * D + j0 + j) = v;
  }
  if (iout && Mprev0) {
    // image 0: the carried M'_prev, read by a continued sequence's first chunk
    uint8_t* img = reinterpret_cast<uint8_t*>(iout);
#pragma unroll 4
    for (int j = 0; j < N; j += 8) {
      const float4 a = *reinterpret_cast<const float4*>(Mprev0 + bh * sd + (int64_t)f * D + j0 + j);
      const float4 b = *reinterpret_cast<const float4*>(Mprev0 + bh * sd + (int64_t)f * D + j0 + j + 4);
      *reinterpret_cast<uint4*>(img + sw128_off(f, j0 + j, D)) =
          make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
  const uint32_t base = smem_u32(smem);
  constexpr uint32_t idesc = idesc_bf16_f32(128, N, false, true);
  float rf = 0.f, pf = 0.f;   // r_s and rho_s of this thread's row, read one step ahead
  if (S > 0) {
    rf = ratio[bh * S * D + f];
    pf = rho[bh * S * D + f];
  }

  // Every exit from the loop follows a block barrier and tests the CTA's
  // abort flag, so all warps leave together; a wait that gives up only
  // raises the flag.
  for (int s = 0; s < S; ++s) {
    const int buf = s & 1;
    // the previous image store has finished reading B_hi before it is rewritten
    if (f == 0) bulk_wait_read<0>();
    __syncthreads();
    if (*abort_flag) break;
    // B = M'_s[:, cols] as hi + lo (row f = K index f, MN-major, one box)
#pragma unroll
    for (int j = 0; j < N; j += 8) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        hi[t] = pack_bf16x2(m[j + 2 * t], m[j + 2 * t + 1]);
        const float2 h2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi[t]));
        lo[t] = pack_bf16x2(m[j + 2 * t] - h2.x, m[j + 2 * t + 1] - h2.y);
      }
      const uint32_t o = sw128_off(f, j, D);
      *reinterpret_cast<uint4*>(smem + Cfg::kBhiOff + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(smem + Cfg::kBloOff + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    fence_proxy_async_smem();   // the operands are read by the tensor core and the bulk store
    __syncthreads();
    if (f == 0) {
      // B_hi is the readout's image of M'_s[:, cols] (box `half` of Mst[s]'s image), read by chunk s + 1
      if (iout && s + 1 < S) {
        bulk_store_1d(reinterpret_cast<uint8_t*>(iout + (int64_t)(s + 1) * mat) + half * Cfg::kBox,
                      smem + Cfg::kBhiOff, Cfg::kOp);
        bulk_commit();
      }
      if (mbar_wait(in_full + buf, (s >> 1) & 1, abort_flag, status)) {
        tc_fence_after();
        const SDesc ad = sdesc_sw128_split(base + Cfg::kAOff + buf * Cfg::kA, 16, 1024);
        const SDesc bh_ = sdesc_sw128_split(base + Cfg::kBhiOff, N * 128, 1024);
        const SDesc bl = sdesc_sw128_split(base + Cfg::kBloOff, N * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (kk / 4) * Cfg::kBox + (kk % 4) * 32, kb = kk * 16 * 128;
          umma_ss(tmem, sdesc_at(ad, ka), sdesc_at(bh_, kb), idesc, kk > 0 ? 1u : 0u);
          umma_ss(tmem, sdesc_at(ad, ka), sdesc_at(bl, kb), idesc, 1u);
        }
        umma_commit(m_done);
      }
    }
    float rn = 0.f, pn = 0.f;
    if (s + 1 < S) {
      rn = ratio[(bh * S + s + 1) * D + f];
      pn = rho[(bh * S + s + 1) * D + f];
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait(m_done, s & 1, abort_flag, status) &&
                                                mbar_wait(in_full + buf, (s >> 1) & 1, abort_flag, status));
    tc_fence_after();
    if (ok) {
#pragma unroll
      for (int cb = 0; cb < N / 32; ++cb) {
        uint32_t acc[32];
        tmem_ld32(lane_addr + cb * 32, acc);
        float bv[32];
        const uint8_t* bbox = smem + Cfg::kBmOff + buf * Cfg::kBm + cb * Cfg::kFBox + f * 128;
#pragma unroll
        for (int t = 0; t < 8; ++t) {   // fp32 box: 16-byte chunk t of row f sits at chunk t ^ (f & 7)
          const float4 v = *reinterpret_cast<const float4*>(bbox + ((t ^ (f & 7)) << 4));
          bv[4 * t] = v.x; bv[4 * t + 1] = v.y; bv[4 * t + 2] = v.z; bv[4 * t + 3] = v.w;
        }
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t)
          m[cb * 32 + t] = fmaf(rf, m[cb * 32 + t], pf * (bv[t] - __uint_as_float(acc[t])));
      }
      if (s + 2 >= S) {
        // Mst[s + 1] is one of the last two states: the exported state
        float* row = mout + (int64_t)(s + 1) * mat + (int64_t)f * D + j0;
#pragma unroll
        for (int j = 0; j < N; j += 4) *reinterpret_cast<float4*>(row + j) = make_float4(m[j], m[j + 1], m[j + 2], m[j + 3]);
      }
    }
    rf = rn;
    pf = pn;
    tc_fence_before();
    __syncthreads();   // buffer `buf` is free: step s + 2's inputs may land there
    if (f == 0 && s + 2 < S && !*abort_flag) load_step(s + 2);
  }
  if (f == 0) {
    bulk_wait_all();
    if (*abort_flag) {
      // no MMA may still write TMEM and no copy still land when the CTA
      // exits: the input copies issued complete phases of in_full[t & 1]
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
      for (int t = loads > 2 ? loads - 2 : 0; t < loads; ++t) mbar_wait_drain(in_full + (t & 1), (t >> 1) & 1);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, N);
}

// ------------------------------------------------------------------ host --

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

template <int D, int Mode>
cudaError_t chunk_impl(const Problem& p, const void* vsrc, const void* ksrc, float* lse, float* out0,
                       float* out1, cudaStream_t st, uint16_t* cimg = nullptr, int parts = 1,
                       int* flags = nullptr) {
  using Cfg = ChunkCfg<D, Mode>;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  // V and K_m as [rows, D], boxes of [64 rows x 64] bf16, 128B swizzle (V
  // carries koff extra leading rows per (b, h) for a continued sequence)
  auto map = [&](CUtensorMap* m, const void* base, int64_t rows) {
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)Cfg::kKT};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  const int64_t koff = Mode == kChunkE ? 0 : p.koff;
  CUtensorMap mv, mkm;
  if (!map(&mv, vsrc, p.B * p.H * (p.T + koff)) || !map(&mkm, ksrc, p.B * p.H * p.T)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(awm_chunk_tc_kernel<D, Mode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg::kAlloc);
  if (e != cudaSuccess) return e;
  awm_chunk_tc_kernel<D, Mode><<<dim3(p.S * parts, p.B * p.H), kChunkThreads, Cfg::kAlloc, st>>>(
      mv, mkm, lse, out0, out1, cimg, (int)p.T, (int)p.c, (int)koff, parts, flags, p.status);
  return cudaGetLastError();
}

template <int D>
cudaError_t readout_impl(const Problem& p, const Workspace& w, cudaStream_t st) {
  using Cfg = ReadoutCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(awm_readout_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg::kAlloc);
  if (e != cudaSuccess) return e;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  // Q_m (load) and out_mem (store) as [B H T rows, D], boxes of [128 rows x 64] bf16, 128B swizzle
  auto map = [&](CUtensorMap* m, const void* base) {
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(p.B * p.H * p.T)};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  CUtensorMap mq, mo;
  if (!map(&mq, p.qm) || !map(&mo, p.out_mem)) return cudaErrorInvalidValue;
  const int64_t tiles = p.B * p.H * p.S * (p.c / 128);
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  awm_readout_tc_kernel<D><<<grid, Cfg::kThreads, Cfg::kAlloc, st>>>(
      mq, mo, w.Mimg, static_cast<__nv_bfloat16*>(p.out_mem), (int)p.T, (int)p.c, p.S, (int)(p.B * p.H),
      p.state0 == nullptr ? 1 : 0, p.status);
  return cudaGetLastError();
}

cudaError_t carry_tc_impl(const Problem& p, const Workspace& w, cudaStream_t st, bool images) {
  using Cfg = CarryTcCfg;
  cudaError_t e = cudaFuncSetAttribute(awm_carry_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kAlloc);
  if (e != cudaSuccess) return e;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  // Bm as [BH S d rows, d] fp32, boxes of [128 rows x 32] with 128B swizzle
  CUtensorMap mb;
  cuuint64_t dims[2] = {128, (cuuint64_t)(p.B * p.H * p.S * 128)};
  cuuint64_t strides[1] = {128 * 4};
  cuuint32_t box[2] = {32, 128};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, w.Bm, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
      CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  awm_carry_tc_kernel<<<(unsigned)(2 * p.B * p.H), 128, Cfg::kAlloc, st>>>(
      mb, w.Cimg, w.ratio, w.rho, w.Mst, p.S, p.state0 ? p.state0 + 128 * 128 : nullptr, state_floats(128),
      images ? w.Mimg : nullptr, p.state0, p.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_awm_carry_tc(const Problem& p, const Workspace& w, cudaStream_t st, bool images) {
  return carry_tc_impl(p, w, st, images);
}

cudaError_t launch_awm_chunk_tc(const Problem& p, const Workspace& w, cudaStream_t st, int parts) {
  if (parts < 1 || parts > (int)(p.c / 64)) return cudaErrorInvalidValue;
  if (parts > 1) {
    // the CTAs of a chunk add into zeroed products
    const size_t bytes = sizeof(float) * p.B * p.H * p.S * p.d * p.d;
    cudaError_t e;
    if ((e = cudaMemsetAsync(w.Bm, 0, bytes, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(w.Cm, 0, bytes, st)) != cudaSuccess) return e;
  }
  cudaError_t e = p.d == 64 ? chunk_impl<64, kChunkFwd>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st, nullptr, parts)
                            : chunk_impl<128, kChunkFwd>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st, w.Cimg, parts);
  if (e != cudaSuccess || parts == 1 || p.d != 128) return e;
  awm_cimg_kernel<<<(unsigned)(p.B * p.H * p.S), 128, 0, st>>>(w.Cm, w.Cimg);
  return cudaGetLastError();
}

// Reference of the fused statistics: taken from each chunk's first tile,
// with the running-reference kernel redoing the chunks that outgrow it (1),
// or the running reference for every chunk (0).
#ifndef GECKO_CHUNK_FIRST_REF
#define GECKO_CHUNK_FIRST_REF 1
#endif

cudaError_t launch_awm_chunk_tc_stats(const Problem& p, const Workspace& w, cudaStream_t st) {
  uint16_t* cimg = p.d == 128 ? w.Cimg : nullptr;
  if (!GECKO_CHUNK_FIRST_REF)
    return p.d == 64 ? chunk_impl<64, kChunkFwdStats>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st)
                     : chunk_impl<128, kChunkFwdStats>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st, cimg);
  cudaError_t e =
      p.d == 64 ? chunk_impl<64, kChunkFwdStatsFirst>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st, cimg, 1, w.flags)
                : chunk_impl<128, kChunkFwdStatsFirst>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st, cimg, 1, w.flags);
  if (e != cudaSuccess) return e;
  // the fix-up pass: its CTAs of unflagged chunks return at once
  return p.d == 64 ? chunk_impl<64, kChunkFwdStats>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st, cimg, 1, w.flags)
                   : chunk_impl<128, kChunkFwdStats>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st, cimg, 1, w.flags);
}

cudaError_t launch_awm_chunk_tc_split(const Problem& p, const Workspace& w, cudaStream_t st) {
  return p.d == 64 ? chunk_impl<64, kChunkSplit>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st)
                   : chunk_impl<128, kChunkSplit>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st);
}

cudaError_t launch_awm_bwd_e_tc(const Problem& p, const void* dout_mem, float* E, cudaStream_t st) {
  return p.d == 64 ? chunk_impl<64, kChunkE>(p, dout_mem, p.qm, nullptr, E, nullptr, st)
                   : chunk_impl<128, kChunkE>(p, dout_mem, p.qm, nullptr, E, nullptr, st);
}

cudaError_t launch_awm_readout_tc(const Problem& p, const Workspace& w, cudaStream_t st) {
  return p.d == 64 ? readout_impl<64>(p, w, st) : readout_impl<128>(p, w, st);
}

}  // namespace gecko
