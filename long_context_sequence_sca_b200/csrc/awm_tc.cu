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
// readout is O_m,s = psi(Qm_s) M'_{s-1}.  Phi~, Psi and psi take their
// exponentials in packed f16 (two per SFU op); they enter the tensor core as
// bf16, whose 8-bit mantissa is coarser than f16's.
//
// awm_chunk_tc_kernel: one CTA per (chunk, bh).  The chunk is streamed in
// tiles of 64 tokens.  V tiles arrive by TMA; 128 threads (two per token)
// compute Phi and Psi in fp32 and store them as bf16 next to V in one
// 128-byte-swizzled, MN-major stage [V | Psi | Phi], so a single
// tcgen05.mma with M = d, N = 2d accumulates [Phi^T V | Phi^T Psi] in TMEM.
//
// awm_readout_tc_kernel: one CTA per (chunk, bh).  M'_{s-1} is converted to
// bf16 once into shared memory (MN-major B operand); every 128-row tile of
// Qm_s is turned into psi rows (K-major A operand) by 128 threads, one row
// each, and multiplied on the tensor core; the epilogue writes bf16 rows.
#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

// Byte offset of element (row, col) in a 128-byte-swizzled tile made of
// 64-column boxes of `rows` rows each (the TMA SWIZZLE_128B layout).
__device__ __forceinline__ uint32_t sw128_off(int row, int col, int rows) {
  const int box = col >> 6, cc = col & 63;
  return box * rows * 128 + row * 128 + ((((cc >> 3) ^ (row & 7)) << 4)) + ((cc & 7) << 1);
}

// ------------------------------------------------------------ chunk GEMMs --

constexpr int kKT = 64;  // tokens per tile

// What a chunk-kernel launch computes.
//   kChunkFwd    Bm = Phi~^T V, Cm = Phi~^T Psi with bf16 operands (f16
//                exponentials): stage [V | Psi | Phi].
//   kChunkSplit  the same products with each computed operand carried as two
//                bf16 parts (hi + lo, fp32 exponentials), for a backward whose
//                softmax gradients keep only the small differences between
//                the rows of M': stage [V | Psi_hi | Psi_lo | Phi_hi | Phi_lo];
//                D += Phi_hi^T [V | Psi_hi] + Phi_lo^T [V | Psi_hi], Cm += Phi_hi^T Psi_lo.
//   kChunkE      E = psi(Q_m)^T dO_m for the backward (Q_m arrives in the
//                K_m slot, dO_m in the V slot): stage [dO | psi_hi | psi_lo].
enum ChunkMode { kChunkFwd = 0, kChunkSplit = 1, kChunkE = 2 };

template <int D, int Mode = kChunkFwd>
struct ChunkCfg {
  static constexpr int kBox = kKT * 128;                 // one [64 x 64] bf16 box
  static constexpr int kOperand = (D / 64) * kBox;       // a [64 x D] operand
  static constexpr int kSlots = Mode == kChunkSplit ? 5 : 3;
  static constexpr int kStage = kSlots * kOperand;
  static constexpr int kStages = 2;
  static constexpr int kBarOff = kStages * kStage;
  // v_full[2], op_full[2], stage_empty[2], acc_full
  static constexpr int kNumBars = 7;
  static constexpr int kLzOff = kBarOff + kNumBars * 8;  // D floats: log2(e) * log z^s
  static constexpr int kMiscOff = kLzOff + D * 4;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = Mode == kChunkE ? D : (D == 128 ? 256 : 128);
};

// 128 compute threads (warps 0-3), warp 4 = TMA producer, warp 5 = MMA issuer.
template <int D, int Mode = kChunkFwd>
__global__ void __launch_bounds__(192, 2) awm_chunk_tc_kernel(const __grid_constant__ CUtensorMap map_v,
                                                           const __grid_constant__ CUtensorMap map_km,
                                                           const float* __restrict__ lse, float* __restrict__ Bm,
                                                           float* __restrict__ Cm, int T, int c, int koff,
                                                           int* status) {
  using Cfg = ChunkCfg<D, Mode>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* v_full = bars;          // [2] TMA -> MMA
  uint64_t* op_full = bars + 2;     // [2] compute -> MMA (128 arrivals)
  uint64_t* st_empty = bars + 4;    // [2] MMA -> TMA, compute
  uint64_t* acc_full = bars + 6;
  float* lz2 = reinterpret_cast<float*>(smem + Cfg::kLzOff);  // log2(e) * lse_s
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);

  const int s = blockIdx.x, S = gridDim.x;
  const int64_t bh = blockIdx.y;
  // the readouts of chunks 1 and 2 read a zero state: their E is never used
  if (Mode == kChunkE && s < 2) return;
  const int warp = warp_id_uniform(), lane = threadIdx.x % 32;
  const int n_tiles = c / kKT;
  const int64_t row0 = bh * (int64_t)T + (int64_t)s * c;
  // v carries koff extra leading rows per (b, h) when a sequence is continued
  const int64_t vrow0 = bh * (int64_t)(T + koff) + koff + (int64_t)s * c;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(v_full + i, 1);
      mbar_init(op_full + i, 128);
      mbar_init(st_empty + i, 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (Mode != kChunkE)
    for (int f = threadIdx.x; f < D; f += blockDim.x) lz2[f] = lse[(bh * S + s) * D + f] * kLog2e;
  if (warp == 5) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------ V and K_m by TMA --
    // V into the V slot, K_m into the Psi slot (where it is turned into Psi
    // in place), both on v_full.
    if (lane == 0) {
      tma_prefetch_desc(&map_v);
      tma_prefetch_desc(&map_km);
      for (int kt = 0; kt < n_tiles; ++kt) {
        const int st = kt & 1;
        if (!mbar_wait(st_empty + st, ((kt >> 1) & 1) ^ 1, abort_flag, status)) break;
        mbar_arrive_expect_tx(v_full + st, 2 * Cfg::kOperand);
        for (int b = 0; b < D / 64; ++b) {
          tma_load_2d(smem + st * Cfg::kStage + b * Cfg::kBox, &map_v, v_full + st, b * 64,
                      (int)(vrow0 + (int64_t)kt * kKT));
          tma_load_2d(smem + st * Cfg::kStage + Cfg::kOperand + b * Cfg::kBox, &map_km, v_full + st, b * 64,
                      (int)(row0 + (int64_t)kt * kKT));
        }
      }
      if (*abort_flag) {
        for (int st = 0; st < 2; ++st) mbar_wait_drain(v_full + st, ((n_tiles - 1 - st) >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(D, 2 * D, true, true);
      constexpr uint32_t idesc1 = idesc_bf16_f32(D, D, true, true);
      const uint32_t base = smem_u32(smem);
      bool ok = true;
      for (int kt = 0; kt < n_tiles && ok; ++kt) {
        const int st = kt & 1;
        const uint32_t ph = (kt >> 1) & 1;
        if (!(ok = mbar_wait(v_full + st, ph, abort_flag, status))) break;
        if (!(ok = mbar_wait(op_full + st, ph, abort_flag, status))) break;
        tc_fence_after();
        const uint32_t sb = base + st * Cfg::kStage;
        auto desc = [&](int slot, int kk) { return sdesc_sw128(sb + slot * Cfg::kOperand + kk * 2048, Cfg::kBox, 1024); };
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk) {
          const uint32_t acc = (kt > 0 || kk > 0) ? 1u : 0u;
          if (Mode == kChunkFwd) {
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
    const int r = threadIdx.x >> 1;       // token row within the tile
    const int h = threadIdx.x & 1;        // which half of the features
    constexpr int HF = D / 2;             // features per thread
    bool ok = true;
    for (int kt = 0; kt < n_tiles; ++kt) {
      const int st = kt & 1;
      // V and K_m of this tile have landed (the copy also waited for the
      // MMAs of tile kt - 2 to release the stage)
      ok = __all_sync(0xffffffffu, mbar_wait(v_full + st, (kt >> 1) & 1, abort_flag, status));
      if (!ok) break;
      uint8_t* stg = smem + st * Cfg::kStage;
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
      float mx = x[0];
#pragma unroll
      for (int i = 1; i < HF; ++i) mx = fmaxf(mx, x[i]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      const float mx2 = mx * kLog2e;
      float e[HF], sum = 0.f;
      if (Mode == kChunkFwd) {
#pragma unroll
        for (int i = 0; i < HF / 8; ++i) {
          const int col = h * HF + 8 * i;
          uint4 pf;
          uint32_t* qq = reinterpret_cast<uint32_t*>(&pf);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int a = 8 * i + 2 * j;
            float p0, p1;
            ex2_h2(fmaf(x[a], kLog2e, -lz2[col + 2 * j]), fmaf(x[a + 1], kLog2e, -lz2[col + 2 * j + 1]), p0, p1);
            qq[j] = pack_bf16x2(p0, p1);
            ex2_h2(fmaf(x[a], kLog2e, -mx2), fmaf(x[a + 1], kLog2e, -mx2), e[a], e[a + 1]);
            sum += e[a] + e[a + 1];
          }
          *reinterpret_cast<uint4*>(stg + 2 * Cfg::kOperand + sw128_off(r, col, kKT)) = pf;
        }
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
              const float p0 = ex2(fmaf(x[a], kLog2e, -lz2[col + 2 * j]));
              const float p1 = ex2(fmaf(x[a + 1], kLog2e, -lz2[col + 2 * j + 1]));
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
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      const float inv = 1.f / sum;
#pragma unroll
      for (int i = 0; i < HF / 8; ++i) {
        const int col = h * HF + 8 * i;
        uint4 ps, pl;
        uint32_t* pp = reinterpret_cast<uint32_t*>(&ps);
        uint32_t* plp = reinterpret_cast<uint32_t*>(&pl);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float a0 = e[8 * i + 2 * j] * inv, a1 = e[8 * i + 2 * j + 1] * inv;
          pp[j] = pack_bf16x2(a0, a1);
          if (Mode != kChunkFwd) {
            const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pp[j]));
            plp[j] = pack_bf16x2(a0 - hi.x, a1 - hi.y);
          }
        }
        *reinterpret_cast<uint4*>(stg + Cfg::kOperand + sw128_off(r, col, kKT)) = ps;
        if (Mode != kChunkFwd) *reinterpret_cast<uint4*>(stg + 2 * Cfg::kOperand + sw128_off(r, col, kKT)) = pl;
      }
      // generic-proxy writes must be visible to the tensor core (async proxy)
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(op_full + st);
    }
    // epilogue: accumulator row f = TMEM lane; columns [0, D) = Bm, [D, 2D) = Cm
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, status));
    if (ok) {
      tc_fence_after();
      // M = 128: row f lives in lane f.  M = 64: rows 16w..16w+15 live in
      // lanes 32w..32w+15 of warp w.
      const bool valid = D == 128 || lane < 16;
      const int f = D == 128 ? warp * 32 + lane : warp * 16 + lane;
      const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
      const int64_t o = (bh * S + s) * (int64_t)D * D + (int64_t)f * D;
#pragma unroll 1
      for (int cb = 0; cb < (Mode == kChunkE ? D : 2 * D) / 32; ++cb) {
        uint32_t v[32];
        tmem_ld32(taddr + cb * 32, v);
        tmem_wait_ld();
        if (valid) {
          float* dst = (cb * 32 < D) ? (Bm + o + cb * 32) : (Cm + o + cb * 32 - D);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(dst)[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                            __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// --------------------------------------------------------------- readout --

template <int D>
struct ReadoutCfg {
  static constexpr int kBox = 128 * 128;        // one [128 rows x 64] bf16 box, 128B-swizzled
  static constexpr int kA = 128 * D * 2;       // a Q_m tile = the psi operand (K-major, D/64 boxes)
  static constexpr int kB = D * D * 2;         // M' bf16, MN-major, D/64 boxes of [D x 64]
  static constexpr int kAOff = 0;              // two tiles
  static constexpr int kBOff = 2 * kA;
  static constexpr int kBarOff = kBOff + kB;
  static constexpr int kNumBars = 5;           // q_full[2], acc_full[2], drain
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 2 * D;   // two accumulators
};

// 128 threads: one row each; thread 0 also issues the TMA copies and the
// MMAs.  grid (S, BH, G): CTA g of a chunk takes its 128-row tiles g,
// g + G, ...  Each Q_m tile arrives by TMA in the 128B-swizzled K-major
// layout of the MMA's A operand; every thread turns its row into the
// unnormalised numerators exp(q - max) in place (bf16, packed f16
// exponentials), and the epilogue scales row t by 1 / sum_t.  Two tile
// buffers and two accumulators: the next tile's copy is issued as soon as
// the MMA that read its buffer has completed, and a tile's MMA overlaps the
// previous tile's epilogue.
template <int D>
__global__ void __launch_bounds__(128) awm_readout_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                                                             const float* __restrict__ Mst,
                                                             __nv_bfloat16* __restrict__ out, int T, int c,
                                                             const float* __restrict__ Mprev0, int64_t sd,
                                                             int* status) {
  using Cfg = ReadoutCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);  // [2] TMA -> threads
  uint64_t* acc_full = q_full + 2;                                        // [2] MMA -> threads, TMA
  uint64_t* drain = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);

  const int s = blockIdx.x, S = gridDim.x;
  const int64_t bh = blockIdx.y;
  const int g = blockIdx.z, G = gridDim.z;
  const int warp = warp_id_uniform();
  const int r = threadIdx.x;
  const int n_tiles = c / 128;
  const int m = n_tiles > g ? (n_tiles - g + G - 1) / G : 0;  // tiles of this CTA
  const int64_t row0 = bh * (int64_t)T + (int64_t)s * c;

  if (s < 2 && Mprev0 == nullptr) {
    // a fresh sequence: chunks 1 and 2 read M'_0 = M'_1 = 0
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int idx = 0; idx < m; ++idx) {
      uint4* dst = reinterpret_cast<uint4*>(out + (row0 + (int64_t)(g + idx * G) * 128) * D);
      for (int i = threadIdx.x; i < 128 * D / 8; i += blockDim.x) dst[i] = z;
    }
    return;
  }
  if (m == 0) return;
  auto load_tile = [&](int idx) {   // thread 0: tile idx into buffer idx & 1
    const int buf = idx & 1;
    mbar_arrive_expect_tx(q_full + buf, Cfg::kA);
    for (int b = 0; b < D / 64; ++b)
      tma_load_2d(smem + Cfg::kAOff + buf * Cfg::kA + b * Cfg::kBox, &map_q, q_full + buf, b * 64,
                  (int)(row0 + (int64_t)(g + idx * G) * 128));
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(acc_full + i, 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_q);
    load_tile(0);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  // B operand: M'_{s-1} (0-based chunk s reads Mst[s-1]; a continued
  // sequence's first chunk reads the carried M'_prev) as bf16, rows = key
  // feature f (K), columns = value dim j (N, contiguous): MN-major.
  const float* M = s == 0 ? Mprev0 + bh * sd : Mst + (bh * (S + 1) + (s - 1)) * (int64_t)D * D;
  for (int i = threadIdx.x; i < D * D / 8; i += blockDim.x) {
    const int f = (i * 8) / D, j = (i * 8) % D;
    const float4 a = reinterpret_cast<const float4*>(M + f * D + j)[0];
    const float4 b = reinterpret_cast<const float4*>(M + f * D + j)[1];
    uint4 p;
    p.x = pack_bf16x2(a.x, a.y);
    p.y = pack_bf16x2(a.z, a.w);
    p.z = pack_bf16x2(b.x, b.y);
    p.w = pack_bf16x2(b.z, b.w);
    *reinterpret_cast<uint4*>(smem + Cfg::kBOff + sw128_off(f, j, D)) = p;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t base = smem_u32(smem);
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
  const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
  const SDesc bdesc = sdesc_sw128_split(base + Cfg::kBOff, D * 128, 1024);
  bool ok = true;

  auto store_tile = [&](int kt, int buf, uint32_t parity, float inv) -> bool {
    if (!__all_sync(0xffffffffu, mbar_wait(acc_full + buf, parity, abort_flag, status))) return false;
    tc_fence_after();
    __nv_bfloat16* orow = out + (row0 + (int64_t)kt * 128 + r) * D;
#pragma unroll 1
    for (int cb = 0; cb < D / 32; ++cb) {
      uint32_t v[32];
      tmem_ld32(lane_addr + buf * D + cb * 32, v);
      tmem_wait_ld();
      uint4 w[4];
      uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        wp[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv, __uint_as_float(v[2 * i + 1]) * inv);
      uint4* dst = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = w[i];
    }
    tc_fence_before();
    return true;
  };

  float inv_prev = 0.f;
  int issued = 1;   // tiles whose copy has been issued (thread 0)
  for (int idx = 0; idx < m && ok; ++idx) {
    const int kt = g + idx * G, buf = idx & 1;
    ok = __all_sync(0xffffffffu, mbar_wait(q_full + buf, (idx >> 1) & 1, abort_flag, status));
    if (!ok) break;
    // psi numerators exp(q - max) of row r, written over the row in place
    uint8_t* a = smem + Cfg::kAOff + buf * Cfg::kA;
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      const uint4 q = *reinterpret_cast<const uint4*>(a + sw128_off(r, 8 * i, 128));
      const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f2 = __bfloat1622float2(p2[j]);
        mx = fmax3(mx, f2.x, f2.y);
      }
    }
    const float mx2 = mx * kLog2e;
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      uint4* qa = reinterpret_cast<uint4*>(a + sw128_off(r, 8 * i, 128));
      const uint4 q = *qa;
      const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&q);
      uint4 p;
      uint32_t* pp = reinterpret_cast<uint32_t*>(&p);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f2 = __bfloat1622float2(p2[j]);
        float e0, e1;
        ex2_h2(fmaf(f2.x, kLog2e, -mx2), fmaf(f2.y, kLog2e, -mx2), e0, e1);
        sum += e0 + e1;
        pp[j] = pack_bf16x2(e0, e1);
      }
      *qa = p;
    }
    const float inv = 1.f / sum;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) {
      const SDesc ad = sdesc_sw128_split(base + Cfg::kAOff + buf * Cfg::kA, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (kk / 4) * (128 * 128) + (kk % 4) * 32;
        umma_ss(tmem + buf * D, sdesc_at(ad, koff), sdesc_at(bdesc, kk * 16 * 128), idesc, kk > 0 ? 1u : 0u);
      }
      umma_commit(acc_full + buf);
      // refill the other buffer once the MMA that read it (tile idx - 1) is done
      if (idx + 1 < m) {
        if (idx == 0 || mbar_wait(acc_full + (buf ^ 1), ((idx - 1) >> 1) & 1, abort_flag, status)) {
          load_tile(idx + 1);
          ++issued;
        }
      }
    }
    // epilogue of the previous tile overlaps this tile's MMA
    if (idx > 0) ok = store_tile(kt - G, buf ^ 1, ((idx - 1) >> 1) & 1, inv_prev);
    inv_prev = inv;
  }
  if (ok) ok = store_tile(g + (m - 1) * G, (m - 1) & 1, ((m - 1) >> 1) & 1, inv_prev);
  if (!ok && threadIdx.x == 0) {
    // no MMA may still write TMEM, and no copy still write shared memory,
    // when the CTA exits
    umma_commit(drain);
    mbar_wait_drain(drain, 0);
    for (int t = issued > 2 ? issued - 2 : 0; t < issued; ++t) mbar_wait_drain(q_full + (t & 1), (t >> 1) & 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, Cfg::kTmemCols);
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
cudaError_t chunk_impl(const Problem& p, const void* vsrc, const void* ksrc, const float* lse, float* out0,
                       float* out1, cudaStream_t st) {
  using Cfg = ChunkCfg<D, Mode>;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  // V and K_m as [rows, D], boxes of [64 rows x 64] bf16, 128B swizzle (V
  // carries koff extra leading rows per (b, h) for a continued sequence)
  auto map = [&](CUtensorMap* m, const void* base, int64_t rows) {
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kKT};
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
  awm_chunk_tc_kernel<D, Mode><<<dim3(p.S, p.B * p.H), 192, Cfg::kAlloc, st>>>(
      mv, mkm, lse, out0, out1, (int)p.T, (int)p.c, (int)koff, p.status);
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
  CUtensorMap mq;   // Q_m as [B H T rows, D], boxes of [128 rows x 64] bf16, 128B swizzle
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(p.B * p.H * p.T)};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p.qm), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // split each chunk's 128-row tiles over G CTAs (up to 8 tiles per CTA)
  const int n_tiles = (int)(p.c / 128);
  const int G = n_tiles > 8 ? (n_tiles + 7) / 8 : 1;
  awm_readout_tc_kernel<D><<<dim3(p.S, p.B * p.H, G), 128, Cfg::kAlloc, st>>>(
      mq, w.Mst, static_cast<__nv_bfloat16*>(p.out_mem), (int)p.T, (int)p.c, p.state0, state_floats(D), p.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_awm_chunk_tc(const Problem& p, const Workspace& w, cudaStream_t st) {
  return p.d == 64 ? chunk_impl<64, kChunkFwd>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st)
                   : chunk_impl<128, kChunkFwd>(p, p.v, p.km, w.lse, w.Bm, w.Cm, st);
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
