// Gradients of the Adaptive Working Memory's per-chunk terms on 5th-generation
// tensor cores (sm_100a), for K_m and V (the AWM recurrence of the Gecko
// digest, paper.rainbus.top, core method and method step details, step 4;
// the pages print no backward, this is the chain rule of that update).
//
// For chunk s (1-based), with G = dLoss/dM'_{s+1}, M = M'_s and per row i of
// the chunk Phi_i = exp(Km_i - L_s), Psi_i = softmax(Km_i):
//     dR_i   = Phi_i G                       (the AWM part of dV_i)
//     dPhi_i = (V_i - Psi_i M) G^T = V_i G^T - Psi_i W,     W = M G^T
//     dPsi_i = -dR_i M^T = -Phi_i W^T
//     dKm_i  = dPhi_i * Phi_i + Psi_i * (dPsi_i - <dPsi_i, Psi_i>) + dl_s * Phi~_i
// where Phi~ = Phi / rho_s and dl_s is the log-sum gradient (awm_bwd_dl).
// W (d x d per chunk, fp32) comes from awm_bwd_w_kernel, so every row needs
// only products with constant d x d matrices: five tensor-core products per
// 128-row tile, all of whose operands exist before the first is issued.
//
// The rows of M are within a few percent of one another (each is a running
// average of V), and the softmax term keeps only the differences of dPsi
// across features; so the operand of dPsi carries W in two bf16 parts
// (hi + lo), the others one.
//
// awm_bwd_chunk_tc_kernel: grid (S, BH, G); CTA g of a chunk takes the
// chunk's 128-row tiles g, g + G, ...  160 threads: warps 0-3 one row each
// (TMEM lane = row), warp 4 TMEM allocator, TMA producer and MMA issuer.
// Per tile: K_m and V by TMA (K-major, 128B swizzle); the row threads write
// Phi and Psi as packed bf16 into TMEM; then
//     acc_R   = Phi G                (TS, G MN-major)
//     acc_Phi = V G^T + Psi (-W)     (SS with G K-major, then TS)
//     acc_Psi = Phi (-W)^T hi + lo   (TS, W K-major)
// and the row threads finish dKm and dV in fp32.
#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

__device__ __forceinline__ uint32_t bsw128_off(int row, int col, int rows) {
  const int box = col >> 6, cc = col & 63;
  return box * rows * 128 + row * 128 + ((((cc >> 3) ^ (row & 7)) << 4)) + ((cc & 7) << 1);
}

// W_s = M'_s G_{s+1}^T, fp32, for every chunk.  grid (S, BH), 256 threads,
// each an 8 x 8 block (D = 128) or 4 x 4 block (D = 64); both operands staged
// transposed in shared memory so the inner loop reads contiguous columns.
template <int D>
__global__ void __launch_bounds__(256) awm_bwd_w_kernel(const float* __restrict__ Mst, const float* __restrict__ Gst,
                                                        float* __restrict__ Wout) {
  constexpr int TB = D / 16;  // outputs per thread per dimension
  constexpr int LD = D + 4;
  extern __shared__ float smem_w[];
  float* Mt = smem_w;          // [j][a] = M[a][j]
  float* Gt = Mt + D * LD;     // [j][b] = G[b][j]
  const int z = blockIdx.x, S = gridDim.x;
  const int64_t bh = blockIdx.y;
  const int64_t mat = (int64_t)D * D;
  const float* M = Mst + (bh * (S + 1) + z) * mat;       // M'_s, s = z + 1
  const float* G = Gst + (bh * (S + 1) + z + 1) * mat;   // G_{s+1}
  for (int i = threadIdx.x; i < D * D; i += 256) {
    const int a = i / D, j = i % D;
    Mt[j * LD + a] = M[i];
    Gt[j * LD + a] = G[i];
  }
  __syncthreads();
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  float acc[TB][TB];
#pragma unroll
  for (int i = 0; i < TB; ++i)
#pragma unroll
    for (int k = 0; k < TB; ++k) acc[i][k] = 0.f;
#pragma unroll 4
  for (int j = 0; j < D; ++j) {
    float m[TB], g[TB];
#pragma unroll
    for (int i = 0; i < TB; ++i) {
      m[i] = Mt[j * LD + ty * TB + i];
      g[i] = Gt[j * LD + tx * TB + i];
    }
#pragma unroll
    for (int i = 0; i < TB; ++i)
#pragma unroll
      for (int k = 0; k < TB; ++k) acc[i][k] = fmaf(m[i], g[k], acc[i][k]);
  }
  float* W = Wout + (bh * S + z) * mat;
#pragma unroll
  for (int i = 0; i < TB; ++i)
#pragma unroll
    for (int k = 0; k < TB; ++k) W[(ty * TB + i) * D + tx * TB + k] = acc[i][k];
}

template <int D>
struct ChunkBwdCfg {
  static constexpr int kTile = 128 * D * 2;        // a [128 x D] bf16 tile (D/64 boxes of 128 rows)
  static constexpr int kMat = D * D * 2;           // a [D x D] bf16 matrix (D/64 boxes of D rows)
  static constexpr int kKmOff = 0;
  static constexpr int kVOff = kTile;
  static constexpr int kGOff = 2 * kTile;
  static constexpr int kWhiOff = kGOff + kMat;
  static constexpr int kWloOff = kWhiOff + kMat;
  static constexpr int kVecOff = kWloOff + kMat;   // 3 D floats: log2(e) L_s, 1 / rho_s, dl_s
  static constexpr int kBarOff = kVecOff + 3 * D * 4;
  // ld_full, op_full, acc_full, tile_done, drain
  static constexpr int kNumBars = 5;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "dynamic shared memory above the sm_100 per-block limit");
  static constexpr uint32_t kTmemCols = D == 128 ? 512 : 256;
  static constexpr uint32_t kColR = 0, kColPhiAcc = D, kColPsiAcc = 2 * D, kColPhi = 3 * D,
                            kColPsi = 3 * D + D / 2;
};

template <int D>
__global__ void __launch_bounds__(160, 1) awm_bwd_chunk_tc_kernel(
    const __grid_constant__ CUtensorMap map_km, const __grid_constant__ CUtensorMap map_v,
    const float* __restrict__ Gst, const float* __restrict__ Wst, const float* __restrict__ logz,
    const float* __restrict__ rho, const float* __restrict__ dl, __nv_bfloat16* __restrict__ dkm,
    float* __restrict__ dv_awm, int T, int c, int* status) {
  using Cfg = ChunkBwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* ld_full = bars;
  uint64_t* op_full = bars + 1;
  uint64_t* acc_full = bars + 2;
  uint64_t* tile_done = bars + 3;
  uint64_t* drain = bars + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);
  float* vL2 = reinterpret_cast<float*>(smem + Cfg::kVecOff);
  float* vInvRho = vL2 + D;
  float* vDl = vInvRho + D;

  const int z = blockIdx.x, S = gridDim.x;
  const int64_t bh = blockIdx.y;
  const int g = blockIdx.z, GG = gridDim.z;
  const int warp = warp_id_uniform(), lane = threadIdx.x % 32;
  const int n_tiles = c / 128;
  const int m = n_tiles > g ? (n_tiles - g + GG - 1) / GG : 0;
  if (m == 0) return;
  const int64_t row0 = bh * (int64_t)T + (int64_t)z * c;
  const int64_t mat = (int64_t)D * D;

  if (threadIdx.x == 0) {
    mbar_init(ld_full, 1);
    mbar_init(op_full, 128);
    mbar_init(acc_full, 1);
    mbar_init(tile_done, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  // B operands: G_{s+1} as bf16; -W_s as bf16 hi and lo parts
  {
    const float* Gm = Gst + (bh * (S + 1) + z + 1) * mat;
    const float* Wm = Wst + (bh * S + z) * mat;
    for (int i = threadIdx.x; i < D * D / 8; i += blockDim.x) {
      const int f = (i * 8) / D, j = (i * 8) % D;
      const float4 ga = reinterpret_cast<const float4*>(Gm + f * D + j)[0];
      const float4 gb = reinterpret_cast<const float4*>(Gm + f * D + j)[1];
      const float4 wa = reinterpret_cast<const float4*>(Wm + f * D + j)[0];
      const float4 wb = reinterpret_cast<const float4*>(Wm + f * D + j)[1];
      const float gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
      const float wv[8] = {-wa.x, -wa.y, -wa.z, -wa.w, -wb.x, -wb.y, -wb.z, -wb.w};
      uint4 pg, ph, pl;
      uint32_t* pgp = reinterpret_cast<uint32_t*>(&pg);
      uint32_t* php = reinterpret_cast<uint32_t*>(&ph);
      uint32_t* plp = reinterpret_cast<uint32_t*>(&pl);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        pgp[q] = pack_bf16x2(gv[2 * q], gv[2 * q + 1]);
        php[q] = pack_bf16x2(wv[2 * q], wv[2 * q + 1]);
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&php[q]));
        plp[q] = pack_bf16x2(wv[2 * q] - hi.x, wv[2 * q + 1] - hi.y);
      }
      const uint32_t o = bsw128_off(f, j, D);
      *reinterpret_cast<uint4*>(smem + Cfg::kGOff + o) = pg;
      *reinterpret_cast<uint4*>(smem + Cfg::kWhiOff + o) = ph;
      *reinterpret_cast<uint4*>(smem + Cfg::kWloOff + o) = pl;
    }
    for (int f = threadIdx.x; f < D; f += blockDim.x) {
      const int64_t zi = (bh * S + z) * D + f;
      vL2[f] = logz[zi] * kLog2e;
      vInvRho[f] = 1.f / rho[zi];
      vDl[f] = dl[zi];
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t base = smem_u32(smem);

  if (warp == 4) {
    // ------------------------------------------------- TMA and MMA issue --
    if (lane == 0) {
      tma_prefetch_desc(&map_km);
      tma_prefetch_desc(&map_v);
      constexpr uint32_t idesc_mn = idesc_bf16_f32(128, D, false, true);   // B MN-major
      constexpr uint32_t idesc_k = idesc_bf16_f32(128, D, false, false);   // B K-major
      constexpr int kBox = 128 * 128;   // one 64-column box of a 128-row tile
      const SDesc g_mn = sdesc_sw128_split(base + Cfg::kGOff, D * 128, 1024);
      const SDesc w_mn = sdesc_sw128_split(base + Cfg::kWhiOff, D * 128, 1024);
      const SDesc g_k = sdesc_sw128_split(base + Cfg::kGOff, 16, 1024);
      const SDesc whi_k = sdesc_sw128_split(base + Cfg::kWhiOff, 16, 1024);
      const SDesc wlo_k = sdesc_sw128_split(base + Cfg::kWloOff, 16, 1024);
      const SDesc v_a = sdesc_sw128_split(base + Cfg::kVOff, 16, 1024);
      bool ok = true;
      int issued = -1;   // last tile whose copies were issued
      for (int idx = 0; idx < m && ok; ++idx) {
        const int kt = g + idx * GG;
        if (idx > 0 && !(ok = mbar_wait(tile_done, (uint32_t)(idx - 1) & 1, abort_flag, status))) break;
        issued = idx;
        mbar_arrive_expect_tx(ld_full, 2 * Cfg::kTile);
        for (int b = 0; b < D / 64; ++b) {
          tma_load_2d(smem + Cfg::kKmOff + b * kBox, &map_km, ld_full, b * 64, (int)(row0 + (int64_t)kt * 128));
          tma_load_2d(smem + Cfg::kVOff + b * kBox, &map_v, ld_full, b * 64, (int)(row0 + (int64_t)kt * 128));
        }
        if (!(ok = mbar_wait(op_full, (uint32_t)idx & 1, abort_flag, status))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t acc = kk > 0 ? 1u : 0u;
          const uint32_t mn_off = kk * 16 * 128;                       // 16 K rows of an MN-major operand
          const uint32_t kb_mat = (kk / 4) * (D * 128) + (kk % 4) * 32;  // K step of a K-major D-row matrix
          const uint32_t kb_tile = (kk / 4) * kBox + (kk % 4) * 32;      // K step of a K-major 128-row tile
          umma_ts(tmem + Cfg::kColR, tmem + Cfg::kColPhi + kk * 8, sdesc_at(g_mn, mn_off), idesc_mn, acc);
          umma_ss(tmem + Cfg::kColPhiAcc, sdesc_at(v_a, kb_tile), sdesc_at(g_k, kb_mat), idesc_k, acc);
          umma_ts(tmem + Cfg::kColPsiAcc, tmem + Cfg::kColPhi + kk * 8, sdesc_at(whi_k, kb_mat), idesc_k, acc);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t mn_off = kk * 16 * 128;
          const uint32_t kb_mat = (kk / 4) * (D * 128) + (kk % 4) * 32;
          umma_ts(tmem + Cfg::kColPhiAcc, tmem + Cfg::kColPsi + kk * 8, sdesc_at(w_mn, mn_off), idesc_mn, 1u);
          umma_ts(tmem + Cfg::kColPsiAcc, tmem + Cfg::kColPhi + kk * 8, sdesc_at(wlo_k, kb_mat), idesc_k, 1u);
        }
        umma_commit(acc_full);
      }
      // nothing in flight when the CTA exits: the last copies have been
      // consumed (or are drained here) and every MMA has completed
      if (!ok && issued >= 0) mbar_wait_drain(ld_full, (uint32_t)issued & 1);
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // --------------------------------------------------- row threads --
    const int r = threadIdx.x;   // row of the tile = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    bool ok = true;
    for (int idx = 0; idx < m; ++idx) {
      const int kt = g + idx * GG;
      ok = __all_sync(0xffffffffu, mbar_wait(ld_full, (uint32_t)idx & 1, abort_flag, status));
      if (!ok) break;
      const uint8_t* km = smem + Cfg::kKmOff;
      auto xval = [&](int col) -> float2 {   // K_m[r][col], K_m[r][col + 1]
        const uint32_t raw = *reinterpret_cast<const uint32_t*>(km + bsw128_off(r, col, 128));
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw));
      };
      float mx = -INFINITY;
#pragma unroll 8
      for (int col = 0; col < D; col += 2) {
        const float2 x = xval(col);
        mx = fmax3(mx, x.x, x.y);
      }
      const float mx2 = mx * kLog2e;
      float sum = 0.f;
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int col = cb * 32 + 2 * q;
          const float2 x = xval(col);
          sum += ex2(fmaf(x.x, kLog2e, -mx2)) + ex2(fmaf(x.y, kLog2e, -mx2));
          pk[q] = pack_bf16x2(ex2(fmaf(x.x, kLog2e, -vL2[col])), ex2(fmaf(x.y, kLog2e, -vL2[col + 1])));
        }
        tmem_st16(lane_addr + Cfg::kColPhi + cb * 16, pk);
      }
      const float inv = 1.f / sum;
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float2 x = xval(cb * 32 + 2 * q);
          pk[q] = pack_bf16x2(ex2(fmaf(x.x, kLog2e, -mx2)) * inv, ex2(fmaf(x.y, kLog2e, -mx2)) * inv);
        }
        tmem_st16(lane_addr + Cfg::kColPsi + cb * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(op_full);
      ok = __all_sync(0xffffffffu, mbar_wait(acc_full, (uint32_t)idx & 1, abort_flag, status));
      if (!ok) break;
      tc_fence_after();
      // <dPsi, Psi>
      float dot = 0.f;
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t a[32];
        tmem_ld32(lane_addr + Cfg::kColPsiAcc + cb * 32, a);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float2 x = xval(cb * 32 + 2 * q);
          dot = fmaf(__uint_as_float(a[2 * q]), ex2(fmaf(x.x, kLog2e, -mx2)), dot);
          dot = fmaf(__uint_as_float(a[2 * q + 1]), ex2(fmaf(x.y, kLog2e, -mx2)), dot);
        }
      }
      dot *= inv;
      const int64_t grow = row0 + (int64_t)kt * 128 + r;
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t aR[32], aPhi[32], aPsi[32], bPhi[16], bPsi[16];
        tmem_ld32(lane_addr + Cfg::kColR + cb * 32, aR);
        tmem_ld32(lane_addr + Cfg::kColPhiAcc + cb * 32, aPhi);
        tmem_ld32(lane_addr + Cfg::kColPsiAcc + cb * 32, aPsi);
        // Phi and Psi of this row as the MMAs used them (bf16): here they only
        // scale terms, so their rounding stays at the output's resolution
        tmem_ld16p(lane_addr + Cfg::kColPhi + cb * 16, bPhi);
        tmem_ld16p(lane_addr + Cfg::kColPsi + cb * 16, bPsi);
        tmem_wait_ld();
        float4* dvp = reinterpret_cast<float4*>(dv_awm + grow * D + cb * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dvp[q] = make_float4(__uint_as_float(aR[4 * q]), __uint_as_float(aR[4 * q + 1]),
                               __uint_as_float(aR[4 * q + 2]), __uint_as_float(aR[4 * q + 3]));
        uint32_t out[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int col = cb * 32 + 2 * q;
          const float2 phi2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bPhi[q]));
          const float2 psi2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bPsi[q]));
          float res[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float phi = e ? phi2.y : phi2.x;
            const float psi = e ? psi2.y : psi2.x;
            res[e] = __uint_as_float(aPhi[2 * q + e]) * phi + psi * (__uint_as_float(aPsi[2 * q + e]) - dot) +
                     vDl[col + e] * phi * vInvRho[col + e];
          }
          out[q] = pack_bf16x2(res[0], res[1]);
        }
        uint4* dst = reinterpret_cast<uint4*>(dkm + grow * D + cb * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
      }
      tc_fence_before();
      mbar_arrive(tile_done);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// ------------------------------------------------------ readout gradient --
//
// O_m,s = psi(Qm_s) M'_{s-1} (digest, method step details, step 5) gives
//     dQm_i = psi_i * (g_i - <g_i, psi_i>),   g_i = dO_m,i M'_{s-1}^T,
// zero for chunks 1 and 2 (they read M'_0 = M'_1 = 0).  g is one tensor-core
// product per 128-row tile with M' in two bf16 parts (the centring keeps
// only the differences between the rows of M').  grid (S, BH, G), 160
// threads: warps 0-3 one row each, warp 4 TMEM, TMA and MMA issue.

template <int D>
struct ReadoutBwdCfg {
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kMat = D * D * 2;
  static constexpr int kDoOff = 0;
  static constexpr int kQmOff = kTile;
  static constexpr int kMhiOff = 2 * kTile;
  static constexpr int kMloOff = kMhiOff + kMat;
  static constexpr int kBarOff = kMloOff + kMat;
  // ld_full, acc_full, tile_done, drain
  static constexpr int kNumBars = 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "dynamic shared memory above the sm_100 per-block limit");
  static constexpr uint32_t kTmemCols = D;
};

template <int D>
__global__ void __launch_bounds__(160, 1) awm_bwd_readout_tc_kernel(
    const __grid_constant__ CUtensorMap map_do, const __grid_constant__ CUtensorMap map_qm,
    const float* __restrict__ Mst, __nv_bfloat16* __restrict__ dqm, int T, int c, int* status) {
  using Cfg = ReadoutBwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* ld_full = bars;
  uint64_t* acc_full = bars + 1;
  uint64_t* tile_done = bars + 2;
  uint64_t* drain = bars + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);

  const int z = blockIdx.x, S = gridDim.x;
  const int64_t bh = blockIdx.y;
  const int g = blockIdx.z, GG = gridDim.z;
  const int warp = warp_id_uniform(), lane = threadIdx.x % 32;
  const int n_tiles = c / 128;
  const int m = n_tiles > g ? (n_tiles - g + GG - 1) / GG : 0;
  const int64_t row0 = bh * (int64_t)T + (int64_t)z * c;
  if (m == 0) return;
  if (z < 2) {
    const uint4 zero = make_uint4(0, 0, 0, 0);
    for (int idx = 0; idx < m; ++idx) {
      uint4* dst = reinterpret_cast<uint4*>(dqm + (row0 + (int64_t)(g + idx * GG) * 128) * D);
      for (int i = threadIdx.x; i < 128 * D / 8; i += blockDim.x) dst[i] = zero;
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(ld_full, 1);
    mbar_init(acc_full, 1);
    mbar_init(tile_done, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  // B operand: M'_{s-1} (0-based chunk z reads Mst[z - 1]) as bf16 hi + lo,
  // stored [f][j]; read K-major (N = f rows, K = j) it is M'^T.
  {
    const float* M = Mst + (bh * (S + 1) + z - 1) * (int64_t)D * D;
    for (int i = threadIdx.x; i < D * D / 8; i += blockDim.x) {
      const int f = (i * 8) / D, j = (i * 8) % D;
      const float4 a = reinterpret_cast<const float4*>(M + f * D + j)[0];
      const float4 b = reinterpret_cast<const float4*>(M + f * D + j)[1];
      const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint4 ph, pl;
      uint32_t* php = reinterpret_cast<uint32_t*>(&ph);
      uint32_t* plp = reinterpret_cast<uint32_t*>(&pl);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        php[q] = pack_bf16x2(v[2 * q], v[2 * q + 1]);
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&php[q]));
        plp[q] = pack_bf16x2(v[2 * q] - hi.x, v[2 * q + 1] - hi.y);
      }
      const uint32_t o = bsw128_off(f, j, D);
      *reinterpret_cast<uint4*>(smem + Cfg::kMhiOff + o) = ph;
      *reinterpret_cast<uint4*>(smem + Cfg::kMloOff + o) = pl;
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t base = smem_u32(smem);

  if (warp == 4) {
    // ------------------------------------------------- TMA and MMA issue --
    if (lane == 0) {
      tma_prefetch_desc(&map_do);
      tma_prefetch_desc(&map_qm);
      constexpr uint32_t idesc_k = idesc_bf16_f32(128, D, false, false);
      constexpr int kBox = 128 * 128;
      const SDesc a_do = sdesc_sw128_split(base + Cfg::kDoOff, 16, 1024);
      const SDesc mhi = sdesc_sw128_split(base + Cfg::kMhiOff, 16, 1024);
      const SDesc mlo = sdesc_sw128_split(base + Cfg::kMloOff, 16, 1024);
      bool ok = true;
      int issued = -1;
      for (int idx = 0; idx < m && ok; ++idx) {
        const int kt = g + idx * GG;
        if (idx > 0 && !(ok = mbar_wait(tile_done, (uint32_t)(idx - 1) & 1, abort_flag, status))) break;
        issued = idx;
        mbar_arrive_expect_tx(ld_full, 2 * Cfg::kTile);
        for (int b = 0; b < D / 64; ++b) {
          tma_load_2d(smem + Cfg::kDoOff + b * kBox, &map_do, ld_full, b * 64, (int)(row0 + (int64_t)kt * 128));
          tma_load_2d(smem + Cfg::kQmOff + b * kBox, &map_qm, ld_full, b * 64, (int)(row0 + (int64_t)kt * 128));
        }
        if (!(ok = mbar_wait(ld_full, (uint32_t)idx & 1, abort_flag, status))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t kb_tile = (kk / 4) * kBox + (kk % 4) * 32;
          const uint32_t kb_mat = (kk / 4) * (D * 128) + (kk % 4) * 32;
          umma_ss(tmem, sdesc_at(a_do, kb_tile), sdesc_at(mhi, kb_mat), idesc_k, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t kb_tile = (kk / 4) * kBox + (kk % 4) * 32;
          const uint32_t kb_mat = (kk / 4) * (D * 128) + (kk % 4) * 32;
          umma_ss(tmem, sdesc_at(a_do, kb_tile), sdesc_at(mlo, kb_mat), idesc_k, 1u);
        }
        umma_commit(acc_full);
      }
      if (!ok && issued >= 0) mbar_wait_drain(ld_full, (uint32_t)issued & 1);
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // --------------------------------------------------- row threads --
    const int r = threadIdx.x;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const uint8_t* qm = smem + Cfg::kQmOff;
    auto xval = [&](int col) -> float2 {
      const uint32_t raw = *reinterpret_cast<const uint32_t*>(qm + bsw128_off(r, col, 128));
      return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw));
    };
    bool ok = true;
    for (int idx = 0; idx < m; ++idx) {
      const int kt = g + idx * GG;
      ok = __all_sync(0xffffffffu, mbar_wait(ld_full, (uint32_t)idx & 1, abort_flag, status));
      if (!ok) break;
      float mx = -INFINITY;
#pragma unroll 8
      for (int col = 0; col < D; col += 2) {
        const float2 x = xval(col);
        mx = fmax3(mx, x.x, x.y);
      }
      const float mx2 = mx * kLog2e;
      float sum = 0.f;
#pragma unroll 8
      for (int col = 0; col < D; col += 2) {
        const float2 x = xval(col);
        sum += ex2(fmaf(x.x, kLog2e, -mx2)) + ex2(fmaf(x.y, kLog2e, -mx2));
      }
      const float inv = 1.f / sum;
      ok = __all_sync(0xffffffffu, mbar_wait(acc_full, (uint32_t)idx & 1, abort_flag, status));
      if (!ok) break;
      tc_fence_after();
      float dot = 0.f;
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t a[32];
        tmem_ld32(lane_addr + cb * 32, a);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float2 x = xval(cb * 32 + 2 * q);
          dot = fmaf(__uint_as_float(a[2 * q]), ex2(fmaf(x.x, kLog2e, -mx2)), dot);
          dot = fmaf(__uint_as_float(a[2 * q + 1]), ex2(fmaf(x.y, kLog2e, -mx2)), dot);
        }
      }
      dot *= inv;
      __nv_bfloat16* orow = dqm + (row0 + (int64_t)kt * 128 + r) * D;
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t a[32];
        tmem_ld32(lane_addr + cb * 32, a);
        tmem_wait_ld();
        uint32_t out[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float2 x = xval(cb * 32 + 2 * q);
          const float p0 = ex2(fmaf(x.x, kLog2e, -mx2)) * inv, p1 = ex2(fmaf(x.y, kLog2e, -mx2)) * inv;
          out[q] = pack_bf16x2(p0 * (__uint_as_float(a[2 * q]) - dot), p1 * (__uint_as_float(a[2 * q + 1]) - dot));
        }
        uint4* dst = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
      }
      tc_fence_before();
      mbar_arrive(tile_done);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// --------------------------------------------------------------- host --

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn awm_bwd_encode_fn() {
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

// [rows, d] bf16 as a 2D tensor; box 128 rows x 64 columns, 128-byte swizzle
cudaError_t awm_bwd_map(CUtensorMap* mp, const void* base, int64_t rows, int d) {
  EncodeTiledFn fn = awm_bwd_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D>
cudaError_t awm_bwd_chunk_tc_impl(const BwdProblem& b, const Workspace& fw, const BwdWorkspace& w, cudaStream_t st) {
  using Cfg = ChunkBwdCfg<D>;
  const Problem& p = b.f;
  const int64_t BH = p.B * p.H;
  const size_t smw = sizeof(float) * 2 * D * (D + 4);
  cudaError_t e = cudaFuncSetAttribute(awm_bwd_w_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smw);
  if (e != cudaSuccess) return e;
  awm_bwd_w_kernel<D><<<dim3(p.S, (unsigned)BH), 256, smw, st>>>(fw.Mst, w.G, w.W);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  CUtensorMap mkm, mv;
  if ((e = awm_bwd_map(&mkm, p.km, BH * p.T, D)) != cudaSuccess) return e;
  if ((e = awm_bwd_map(&mv, p.v, BH * p.T, D)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(awm_bwd_chunk_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg::kAlloc)) != cudaSuccess)
    return e;
  const int n_tiles = (int)(p.c / 128);
  const int G = n_tiles > 8 ? (n_tiles + 7) / 8 : 1;   // up to 8 tiles per CTA
  awm_bwd_chunk_tc_kernel<D><<<dim3(p.S, (unsigned)BH, G), 160, Cfg::kAlloc, st>>>(
      mkm, mv, w.G, w.W, fw.logz, fw.rho, w.dl, static_cast<__nv_bfloat16*>(b.dkm), w.dv_awm, (int)p.T, (int)p.c,
      p.status);
  return cudaGetLastError();
}

template <int D>
cudaError_t awm_bwd_readout_tc_impl(const BwdProblem& b, const Workspace& fw, cudaStream_t st) {
  using Cfg = ReadoutBwdCfg<D>;
  const Problem& p = b.f;
  const int64_t BH = p.B * p.H;
  CUtensorMap mdo, mqm;
  cudaError_t e;
  if ((e = awm_bwd_map(&mdo, b.dout_mem, BH * p.T, D)) != cudaSuccess) return e;
  if ((e = awm_bwd_map(&mqm, p.qm, BH * p.T, D)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(awm_bwd_readout_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg::kAlloc)) != cudaSuccess)
    return e;
  const int n_tiles = (int)(p.c / 128);
  const int G = n_tiles > 8 ? (n_tiles + 7) / 8 : 1;
  awm_bwd_readout_tc_kernel<D><<<dim3(p.S, (unsigned)BH, G), 160, Cfg::kAlloc, st>>>(
      mdo, mqm, fw.Mst, static_cast<__nv_bfloat16*>(b.dqm), (int)p.T, (int)p.c, p.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_awm_bwd_readout_tc(const BwdProblem& b, const Workspace& fw, cudaStream_t st) {
  return b.f.d == 64 ? awm_bwd_readout_tc_impl<64>(b, fw, st) : awm_bwd_readout_tc_impl<128>(b, fw, st);
}

cudaError_t launch_awm_bwd_chunk_tc(const BwdProblem& b, const Workspace& fw, const BwdWorkspace& w,
                                    cudaStream_t st) {
  return b.f.d == 64 ? awm_bwd_chunk_tc_impl<64>(b, fw, w, st) : awm_bwd_chunk_tc_impl<128>(b, fw, w, st);
}

}  // namespace gecko
