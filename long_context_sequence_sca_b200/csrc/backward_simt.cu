// CUDA-core (fp32 FMA) kernels of the Gecko backward: gradients of Sliding
// Chunk Attention and of the Adaptive Working Memory recurrence with respect
// to q, k, v, q_m, k_m.  They serve every dtype and shape; the tensor-core
// SCA backward replaces the two SCA kernels for bf16 where it applies.
//
// The forward being differentiated is the Gecko digest (paper.rainbus.top),
// core method (phi^s, z^s, psi) and method step details, steps 3-5, with the
// paperlayer.ai summary, sections 3.2-3.3 and Appendix A (M'_1 = 0).  The
// pages print no backward; the reverse pass is the chain rule of that
// forward.  Following the summary's appendix B.1 (backward pass), only the
// chunk-boundary states M'_s are kept (recomputed by the forward kernels)
// and everything inside a chunk is rebuilt here.
//
// AWM notation (1-based chunk s, M'_s the state read by chunk s + 1,
// G_s = dLoss/dM'_s, Phi_s = rho_s (.) Phi~_s, L_s = log z^s, l_s = log e_s):
//   G_s   = E_{s+1} + r_s (.) G_{s+1} - Cm_s^T (rho_s (.) G_{s+1}),  G_{S+1} = 0,
//           E_s = psi(Qm_s)^T dO_m,s,  Cm_s = Phi~_s^T Psi_s
//   dR    = Phi_s G_{s+1},  R = V_s - Psi_s M'_s  (dV_s += dR)
//   dK_m  = (R G_{s+1}^T) * Phi_s + Psi_s * (dPsi - <dPsi, Psi_s>) + dl_s Phi~_s,
//           dPsi = -dR M'_s^T
//   dl_s  = rho_s dLbar_s,  dLbar_s = dL_s + r_{s+1} dLbar_{s+1},
//           dL_s = -<G_{s+1}, M'_{s+1}>_row + r_{s+1} <G_{s+2}, M'_{s+1}>_row
//   dQ_m  = psi_q * (dO_m M'_{s-1}^T - <., psi_q>)
// (the two row sums in dL_s collect the log z dependence of Phi_s and of the
// ratios r; Phi_s^T R equals M'_{s+1} - r_s (.) M'_s, which turns the
// column sums of dPhi * Phi into the first row sum).
#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// ------------------------------------------------------------------ SCA --

// delta_t = sum_f dO[t, f] O[t, f] (O = stored output + its rounding
// residual when the forward kept it), and -log2(e) l_t for the exp2 form of
// the tensor-core kernels; one warp per row.
template <typename TIn, int D>
__global__ void __launch_bounds__(256) sca_bwd_delta_kernel(const TIn* __restrict__ out, const TIn* __restrict__ out_lo,
                                                            const TIn* __restrict__ dout,
                                                            const float* __restrict__ lse, float* __restrict__ delta,
                                                            float* __restrict__ nlse2, int64_t rows) {
  const int64_t row = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;  // uniform per warp
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < D / 32; ++i) {
    const int64_t g = row * D + lane + 32 * i;
    const float o = to_f32(out[g]) + (out_lo ? to_f32(out_lo[g]) : 0.f);
    acc = fmaf(o, to_f32(dout[g]), acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) {
    delta[row] = acc;
    nlse2[row] = -kLog2e * lse[row];
  }
}

// dQ: 32 queries per CTA, 4 threads per query (each owns D/4 dims), the
// window's keys and values streamed through shared memory 32 rows at a time.
// p = exp(q.k - lse_t), ds = p (dO.v - delta_t), dq = sum ds k.  grid (T/32, BH).
template <typename TIn, int D>
__global__ void __launch_bounds__(128) sca_bwd_dq_simt_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                                                              const TIn* __restrict__ v, const TIn* __restrict__ dout,
                                                              const float* __restrict__ lse,
                                                              const float* __restrict__ delta, TIn* __restrict__ dq,
                                                              int64_t T, int c) {
  constexpr int QD = D / 4;
  __shared__ float ks[32][D + 4];
  __shared__ float vs[32][D + 4];
  const int64_t bh = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * 32;
  const int tid = threadIdx.x;
  const int qi = tid / 4, part = tid % 4;
  const int64_t t = t0 + qi;
  const int64_t lo = t0 / c >= 1 ? (t0 / c - 1) * c : 0;  // all 32 rows share one chunk
  const int64_t base = bh * T;
  float qv[QD], dov[QD], acc[QD];
#pragma unroll
  for (int i = 0; i < QD; ++i) {
    qv[i] = to_f32(q[(base + t) * D + part * QD + i]);
    dov[i] = to_f32(dout[(base + t) * D + part * QD + i]);
    acc[i] = 0.f;
  }
  const float lt = lse[base + t], dt = delta[base + t];
  for (int64_t k0 = lo; k0 <= t0 + 31; k0 += 32) {
    __syncthreads();
    for (int i = tid; i < 32 * D; i += 128) {
      const int r = i / D, cc = i % D;
      ks[r][cc] = to_f32(k[(base + k0 + r) * D + cc]);
      vs[r][cc] = to_f32(v[(base + k0 + r) * D + cc]);
    }
    __syncthreads();
    for (int j = 0; j < 32; ++j) {
      float sc = 0.f, dp = 0.f;
#pragma unroll
      for (int i = 0; i < QD; ++i) {
        sc = fmaf(qv[i], ks[j][part * QD + i], sc);
        dp = fmaf(dov[i], vs[j][part * QD + i], dp);
      }
      sc += __shfl_xor_sync(0xffffffffu, sc, 1);
      sc += __shfl_xor_sync(0xffffffffu, sc, 2);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      dp += __shfl_xor_sync(0xffffffffu, dp, 2);
      if (k0 + j > t) continue;  // causal inside the current chunk
      const float ds = expf(sc - lt) * (dp - dt);
#pragma unroll
      for (int i = 0; i < QD; ++i) acc[i] = fmaf(ds, ks[j][part * QD + i], acc[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < QD; ++i) dq[(base + t) * D + part * QD + i] = from_f32<TIn>(acc[i]);
}

// dK, dV: 32 keys per CTA, 4 threads per key; the queries that see these keys
// (from the first key to the end of the next chunk) streamed through shared
// memory.  dv = sum p dO (+ the AWM part dv_add, fp32), dk = sum ds q.
// grid (T/32, BH).
template <typename TIn, int D>
__global__ void __launch_bounds__(128) sca_bwd_dkdv_simt_kernel(
    const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v, const TIn* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ delta, const float* __restrict__ dv_add,
    TIn* __restrict__ dk, TIn* __restrict__ dv, int64_t T, int c) {
  constexpr int QD = D / 4;
  __shared__ float qs[32][D + 4];
  __shared__ float os[32][D + 4];
  __shared__ float ls[32], dls[32];
  const int64_t bh = blockIdx.y;
  const int64_t u0 = (int64_t)blockIdx.x * 32;
  const int tid = threadIdx.x;
  const int ki = tid / 4, part = tid % 4;
  const int64_t u = u0 + ki;
  const int64_t base = bh * T;
  const int64_t thi = (u0 / c + 2) * c < T ? (u0 / c + 2) * c : T;  // end of the next chunk
  float kv[QD], vv[QD], dka[QD], dva[QD];
#pragma unroll
  for (int i = 0; i < QD; ++i) {
    kv[i] = to_f32(k[(base + u) * D + part * QD + i]);
    vv[i] = to_f32(v[(base + u) * D + part * QD + i]);
    dka[i] = 0.f;
    dva[i] = 0.f;
  }
  for (int64_t t0 = u0; t0 < thi; t0 += 32) {
    __syncthreads();
    for (int i = tid; i < 32 * D; i += 128) {
      const int r = i / D, cc = i % D;
      qs[r][cc] = to_f32(q[(base + t0 + r) * D + cc]);
      os[r][cc] = to_f32(dout[(base + t0 + r) * D + cc]);
    }
    if (tid < 32) {
      ls[tid] = lse[base + t0 + tid];
      dls[tid] = delta[base + t0 + tid];
    }
    __syncthreads();
    for (int r = 0; r < 32; ++r) {
      float sc = 0.f, dp = 0.f;
#pragma unroll
      for (int i = 0; i < QD; ++i) {
        sc = fmaf(kv[i], qs[r][part * QD + i], sc);
        dp = fmaf(vv[i], os[r][part * QD + i], dp);
      }
      sc += __shfl_xor_sync(0xffffffffu, sc, 1);
      sc += __shfl_xor_sync(0xffffffffu, sc, 2);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      dp += __shfl_xor_sync(0xffffffffu, dp, 2);
      if (t0 + r < u) continue;  // query before the key
      const float p = expf(sc - ls[r]);
      const float ds = p * (dp - dls[r]);
#pragma unroll
      for (int i = 0; i < QD; ++i) {
        dva[i] = fmaf(p, os[r][part * QD + i], dva[i]);
        dka[i] = fmaf(ds, qs[r][part * QD + i], dka[i]);
      }
    }
  }
  const int64_t o = (base + u) * D + part * QD;
#pragma unroll
  for (int i = 0; i < QD; ++i) {
    dk[o + i] = from_f32<TIn>(dka[i]);
    dv[o + i] = from_f32<TIn>(dva[i] + (dv_add ? dv_add[o + i] : 0.f));
  }
}

// ------------------------------------------------------------------ AWM --

// E_s = psi(Qm_s)^T dO_m,s (D x D) for 0-based chunks s >= 2 (chunks 1 and 2
// read a zero state, so their readouts send no gradient into the state).
// grid (S, BH), 256 threads as a 16 x 16 grid of (D/16) x (D/16) tiles.
template <typename TIn, int D>
__global__ void __launch_bounds__(256) awm_bwd_e_simt_kernel(const TIn* __restrict__ qm, const TIn* __restrict__ dout,
                                                             float* __restrict__ E, int64_t T, int c) {
  constexpr int RT = 16;
  constexpr int TM = D / 16;
  const int s = blockIdx.x;
  const int S = gridDim.x;
  if (s < 2) return;
  const int64_t bh = blockIdx.y;
  __shared__ float ps[RT][D];
  __shared__ float os[RT][D];
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  const int warp = tid / 32, lane = tid % 32;
  float acc[TM][TM];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TM; ++j) acc[i][j] = 0.f;
  const int64_t row0 = bh * T + (int64_t)s * c;
  for (int r0 = 0; r0 < c; r0 += RT) {
    for (int rr = warp; rr < RT; rr += 8) {
      const int64_t g = (row0 + r0 + rr) * D;
      float x[D / 32], mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        x[i] = to_f32(qm[g + lane + 32 * i]);
        mx = fmaxf(mx, x[i]);
      }
      mx = warp_max(mx);
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        x[i] = expf(x[i] - mx);
        sum += x[i];
      }
      const float inv = 1.f / warp_sum(sum);
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        ps[rr][lane + 32 * i] = x[i] * inv;
        os[rr][lane + 32 * i] = to_f32(dout[g + lane + 32 * i]);
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < RT; ++t) {
      float a[TM], b[TM];
#pragma unroll
      for (int i = 0; i < TM; ++i) {
        a[i] = ps[t][ty * TM + i];
        b[i] = os[t][tx * TM + i];
      }
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TM; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* Eo = E + (bh * S + s) * (int64_t)D * D;
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TM; ++j) Eo[(ty * TM + i) * D + tx * TM + j] = acc[i][j];
}

// Reverse carry, one slice of JC columns of G per CTA (columns evolve
// independently):  G_s = E_{s+1} + r_s (.) G_{s+1} - Cm_s^T (rho_s (.) G_{s+1})
// for 1-based s = S .. 2, G_{S+1} = 0.  Writes Gst[bh, s - 1] = G_s for
// s = 1 .. S + 1 (G_1 is never read and is written as zero).  Everything the
// next step reads from global memory (Cm_s, the CTA's slice of E_{s+1}, r_s,
// rho_s) is copied into shared memory with 16-byte asynchronous copies while
// this step computes (double buffer).  grid (D/JC, BH), 256 threads.
template <int D, int JC>
struct BwdCarryStage {
  static constexpr int LD = D + 4;
  static constexpr int kC = 0, kE = D * LD, kR = kE + D * JC, kP = kR + D;
  static constexpr int kFloats = kP + D;
};

template <int D, int JC>
__global__ void __launch_bounds__(256) awm_bwd_carry_kernel(const float* __restrict__ E, const float* __restrict__ Cm,
                                                            const float* __restrict__ ratio,
                                                            const float* __restrict__ rho, float* __restrict__ Gst,
                                                            int S) {
  using St = BwdCarryStage<D, JC>;
  constexpr int PER = D * JC / 256;
  static_assert(PER >= 1 && 256 / (JC / PER) == D, "thread layout");
  constexpr int LD = St::LD;
  extern __shared__ float smem_bc[];
  // buffer b at smem_bc + b * St::kFloats (computed, so no pointer array in local memory)
  float* Gs = smem_bc + 2 * St::kFloats;          // [D][JC]
  const int64_t bh = blockIdx.y;
  const int j0 = blockIdx.x * JC;
  const int tid = threadIdx.x;
  const int f = tid / (JC / PER);
  const int jj = (tid % (JC / PER)) * PER;
  const int64_t mat = (int64_t)D * D;
  float* gout = Gst + bh * (int64_t)(S + 1) * mat;
  // step k handles 1-based s = S - k (k = 0 .. S - 2), 0-based chunk z = s - 1
  auto stage = [&](int k, float* dst) {
    const int s = S - k, z = s - 1;
    const float4* C4 = reinterpret_cast<const float4*>(Cm + (bh * S + z) * mat);
    for (int i = tid; i < D * D / 4; i += 256) {
      const int row = (i * 4) / D, col = (i * 4) % D;
      cp_async16(dst + St::kC + row * LD + col, C4 + i);
    }
    if (s <= S - 1) {   // E_{s+1}: 0-based chunk s (none after the last chunk)
      const float* Es = E + (bh * S + s) * mat + j0;
      for (int i = tid; i < D * JC / 4; i += 256) {
        const int row = (i * 4) / JC, col = (i * 4) % JC;
        cp_async16(dst + St::kE + row * JC + col, Es + row * D + col);
      }
    }
    for (int i = tid; i < D / 4; i += 256) {
      cp_async16(dst + St::kR + 4 * i, ratio + (bh * S + z) * D + 4 * i);
      cp_async16(dst + St::kP + 4 * i, rho + (bh * S + z) * D + 4 * i);
    }
    cp_async_commit();
  };
  const int steps = S - 1;   // s = S .. 2
  if (steps > 0) stage(0, smem_bc);
  for (int i = tid; i < D * JC; i += 256) Gs[i] = 0.f;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    gout[(int64_t)S * mat + f * D + j0 + jj + j] = 0.f;  // G_{S+1}
    gout[f * D + j0 + jj + j] = 0.f;                     // G_1
  }
  for (int k = 0; k < steps; ++k) {
    const int s = S - k;
    const float* sb = smem_bc + (k & 1) * St::kFloats;
    if (k + 1 < steps) {
      stage(k + 1, smem_bc + ((k + 1) & 1) * St::kFloats);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const float* Cs = sb + St::kC;
    const float* rz = sb + St::kP;
    const float rf = sb[St::kR + f];
    float acc[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) acc[j] = s <= S - 1 ? sb[St::kE + f * JC + jj + j] : 0.f;
#pragma unroll 4
    for (int g = 0; g < D; ++g) {
      const float cgf = Cs[g * LD + f] * rz[g];
#pragma unroll
      for (int j = 0; j < PER; ++j) acc[j] = fmaf(-cgf, Gs[g * JC + jj + j], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < PER; ++j) acc[j] = fmaf(rf, Gs[f * JC + jj + j], acc[j]);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < PER; ++j) Gs[f * JC + jj + j] = acc[j];
    float* dst = gout + (int64_t)(s - 1) * mat + f * D + j0 + jj;
    if (PER % 4 == 0) {
#pragma unroll
      for (int j = 0; j < PER; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < PER; ++j) dst[j] = acc[j];
    }
  }
}

// Gradient of the per-chunk log exp-sums, one warp per (bh, feature f):
// the reverse of L_s = logaddexp(L_{s-1}, l_s) over s = S .. 1 with the
// log z dependence of Phi_s and r_s collected as two row sums of G (*) M'.
// dl[bh, s-1, f] = dLoss/dl_s[f].
template <int D>
__global__ void __launch_bounds__(256) awm_bwd_dl_kernel(const float* __restrict__ Gst, const float* __restrict__ Mst,
                                                         const float* __restrict__ ratio,
                                                         const float* __restrict__ rho, float* __restrict__ dl, int S,
                                                         int64_t n) {
  const int64_t w = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (w >= n) return;  // uniform per warp
  const int64_t bh = w / D;
  const int f = (int)(w % D);
  const int64_t mat = (int64_t)D * D;
  const float* G = Gst + bh * (S + 1) * mat + f * D;
  const float* M = Mst + bh * (S + 1) * mat + f * D;
  float rb_next = 0.f, lbar_next = 0.f;  // r_{s+1} <G_{s+2}, M'_{s+1}>, r_{s+1} dLbar_{s+1}
  for (int s = S; s >= 1; --s) {
    // G_{s+1} = Gst[s], M'_{s+1} = Mst[s], M'_s = Mst[s-1]
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const int j = lane + 32 * i;
      const float g = G[(int64_t)s * mat + j];
      a = fmaf(g, M[(int64_t)s * mat + j], a);
      b = fmaf(g, M[(int64_t)(s - 1) * mat + j], b);
    }
    a = warp_sum(a);
    b = warp_sum(b);
    const int64_t zi = (bh * S + (s - 1)) * D + f;
    const float lbar = -a + rb_next + lbar_next;
    if (lane == 0) dl[zi] = lbar * rho[zi];
    const float rs = ratio[zi];
    rb_next = rs * b;
    lbar_next = rs * lbar;
  }
}

// Row vector (in the per-warp buffer xr, 4 rows) times a D x D matrix in
// shared memory with row stride D + 1.  Lane owns output columns
// lane + 32 u.  kTrans: out[f] = sum_k x[k] A[f][k], else out[j] = sum_k x[k] A[k][j].
template <int D, bool kTrans>
__device__ __forceinline__ void rows_times(const float* __restrict__ xr, const float* __restrict__ A, int lane,
                                           float (&out)[4][D / 32]) {
  constexpr int U = D / 32;
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int u = 0; u < U; ++u) out[r][u] = 0.f;
#pragma unroll 2
  for (int k4 = 0; k4 < D / 4; ++k4) {
    float4 x[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) x[r] = reinterpret_cast<const float4*>(xr + r * D)[k4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int kx = k4 * 4 + kk;
      float a[U];
#pragma unroll
      for (int u = 0; u < U; ++u) a[u] = kTrans ? A[(lane + 32 * u) * (D + 1) + kx] : A[kx * (D + 1) + lane + 32 * u];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float xv = kk == 0 ? x[r].x : kk == 1 ? x[r].y : kk == 2 ? x[r].z : x[r].w;
#pragma unroll
        for (int u = 0; u < U; ++u) out[r][u] = fmaf(xv, a[u], out[r][u]);
      }
    }
  }
}

template <int D>
__device__ __forceinline__ void put_rows(float* xr, const float (&x)[4][D / 32], int lane) {
  __syncwarp();
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int u = 0; u < D / 32; ++u) xr[r * D + lane + 32 * u] = x[r][u];
  __syncwarp();
}

// Per-chunk AWM gradients of K_m and V (all chunks in parallel once G and dl
// are known).  grid (c / 32, S, BH), 256 threads: 8 warps x 4 rows; lane owns
// the features lane + 32 u.  G_{s+1} and M'_s sit in shared memory (fp32,
// row stride D + 1 so both orientations read without bank conflicts).
template <typename TIn, int D>
__global__ void __launch_bounds__(256) awm_bwd_chunk_simt_kernel(
    const TIn* __restrict__ km, const TIn* __restrict__ v, const float* __restrict__ Gst,
    const float* __restrict__ Mst, const float* __restrict__ lse, const float* __restrict__ logz,
    const float* __restrict__ dl, TIn* __restrict__ dkm, float* __restrict__ dv_awm, int64_t T, int c) {
  constexpr int U = D / 32;
  extern __shared__ float smem_ac[];
  float* Gs = smem_ac;                // [D][D+1]  G_{s+1}
  float* Ms = Gs + D * (D + 1);       // [D][D+1]  M'_s
  float* xb = Ms + D * (D + 1);       // [8][4][D]
  const int z = blockIdx.y;           // 0-based chunk: 1-based s = z + 1
  const int S = gridDim.y;
  const int64_t bh = blockIdx.z;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int64_t mat = (int64_t)D * D;
  const float* G = Gst + (bh * (S + 1) + z + 1) * mat;
  const float* M = Mst + (bh * (S + 1) + z) * mat;
  for (int i = tid; i < D * D; i += 256) {
    Gs[(i / D) * (D + 1) + i % D] = G[i];
    Ms[(i / D) * (D + 1) + i % D] = M[i];
  }
  __syncthreads();
  float* xr = xb + warp * 4 * D;
  const int64_t row0 = bh * T + (int64_t)z * c + (int64_t)blockIdx.x * 32 + warp * 4;
  const int64_t zi = (bh * S + z) * D;
  float Lz[U], lz[U], dlz[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    Lz[u] = logz[zi + lane + 32 * u];
    lz[u] = lse[zi + lane + 32 * u];
    dlz[u] = dl[zi + lane + 32 * u];
  }
  float x[4][U], psi[4][U], phi[4][U], dR[4][U], t[4][U];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      x[r][u] = to_f32(km[(row0 + r) * D + lane + 32 * u]);
      mx = fmaxf(mx, x[r][u]);
    }
    mx = warp_max(mx);
    float sum = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      psi[r][u] = expf(x[r][u] - mx);
      sum += psi[r][u];
      phi[r][u] = expf(x[r][u] - Lz[u]);
    }
    const float inv = 1.f / warp_sum(sum);
#pragma unroll
    for (int u = 0; u < U; ++u) psi[r][u] *= inv;
  }
  // dR = Phi G_{s+1}  (the AWM part of dV)
  put_rows<D>(xr, phi, lane);
  rows_times<D, false>(xr, Gs, lane, dR);
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int u = 0; u < U; ++u) dv_awm[(row0 + r) * D + lane + 32 * u] = dR[r][u];
  // R = V - Psi M'_s
  put_rows<D>(xr, psi, lane);
  rows_times<D, false>(xr, Ms, lane, t);
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int u = 0; u < U; ++u) t[r][u] = to_f32(v[(row0 + r) * D + lane + 32 * u]) - t[r][u];
  // dPhi = R G_{s+1}^T ; the Phi and log-sum terms of dK_m
  put_rows<D>(xr, t, lane);
  rows_times<D, true>(xr, Gs, lane, t);
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int u = 0; u < U; ++u) x[r][u] = t[r][u] * phi[r][u] + dlz[u] * expf(x[r][u] - lz[u]);
  // dPsi = -dR M'_s^T ; the softmax term of dK_m
  put_rows<D>(xr, dR, lane);
  rows_times<D, true>(xr, Ms, lane, t);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    float dot = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) dot = fmaf(-t[r][u], psi[r][u], dot);
    dot = warp_sum(dot);
#pragma unroll
    for (int u = 0; u < U; ++u)
      dkm[(row0 + r) * D + lane + 32 * u] = from_f32<TIn>(x[r][u] + psi[r][u] * (-t[r][u] - dot));
  }
}

// dQ_m = psi_q * (dO_m M'_{s-1}^T - <., psi_q>) for 0-based chunks >= 2; zero
// for the first two chunks.  grid (c / 32, S, BH), 8 warps x 4 rows.
template <typename TIn, int D>
__global__ void __launch_bounds__(256) awm_bwd_readout_simt_kernel(const TIn* __restrict__ qm,
                                                                   const TIn* __restrict__ dout,
                                                                   const float* __restrict__ Mst,
                                                                   TIn* __restrict__ dqm, int64_t T, int c) {
  constexpr int U = D / 32;
  extern __shared__ float smem_ar[];
  float* Ms = smem_ar;             // [D][D+1]  M'_{s-1}
  float* xb = Ms + D * (D + 1);    // [8][4][D]
  const int z = blockIdx.y;
  const int S = gridDim.y;
  const int64_t bh = blockIdx.z;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int64_t row0 = bh * T + (int64_t)z * c + (int64_t)blockIdx.x * 32 + warp * 4;
  if (z < 2) {
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int u = 0; u < U; ++u) dqm[(row0 + r) * D + lane + 32 * u] = from_f32<TIn>(0.f);
    return;
  }
  const int64_t mat = (int64_t)D * D;
  const float* M = Mst + (bh * (S + 1) + z - 1) * mat;  // M'_{s-1} with s = z + 1
  for (int i = tid; i < D * D; i += 256) Ms[(i / D) * (D + 1) + i % D] = M[i];
  __syncthreads();
  float* xr = xb + warp * 4 * D;
  float psi[4][U], g[4][U];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      psi[r][u] = to_f32(qm[(row0 + r) * D + lane + 32 * u]);
      mx = fmaxf(mx, psi[r][u]);
      g[r][u] = to_f32(dout[(row0 + r) * D + lane + 32 * u]);
    }
    mx = warp_max(mx);
    float sum = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      psi[r][u] = expf(psi[r][u] - mx);
      sum += psi[r][u];
    }
    const float inv = 1.f / warp_sum(sum);
#pragma unroll
    for (int u = 0; u < U; ++u) psi[r][u] *= inv;
  }
  put_rows<D>(xr, g, lane);
  rows_times<D, true>(xr, Ms, lane, g);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    float dot = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) dot = fmaf(g[r][u], psi[r][u], dot);
    dot = warp_sum(dot);
#pragma unroll
    for (int u = 0; u < U; ++u) dqm[(row0 + r) * D + lane + 32 * u] = from_f32<TIn>(psi[r][u] * (g[r][u] - dot));
  }
}

// ---------------------------------------------------------------- host --

template <typename TIn, int D>
cudaError_t sca_bwd_delta_impl(const BwdProblem& b, const BwdWorkspace& w, cudaStream_t st) {
  const Problem& p = b.f;
  const int64_t rows = p.B * p.H * p.T;
  sca_bwd_delta_kernel<TIn, D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      static_cast<const TIn*>(b.out_sca), static_cast<const TIn*>(b.out_sca_lo), static_cast<const TIn*>(b.dout_sca),
      b.lse, w.delta, w.nlse2, rows);
  return cudaGetLastError();
}

template <typename TIn, int D>
cudaError_t sca_bwd_simt_impl(const BwdProblem& b, const BwdWorkspace& w, cudaStream_t st, int part) {
  const Problem& p = b.f;
  const dim3 grid((unsigned)(p.T / 32), (unsigned)(p.B * p.H));
  if (part == 0)
    sca_bwd_dkdv_simt_kernel<TIn, D><<<grid, 128, 0, st>>>(
        static_cast<const TIn*>(p.q), static_cast<const TIn*>(p.k), static_cast<const TIn*>(p.v),
        static_cast<const TIn*>(b.dout_sca), b.lse, w.delta, w.dv_awm, static_cast<TIn*>(b.dk),
        static_cast<TIn*>(b.dv), p.T, (int)p.c);
  else
    sca_bwd_dq_simt_kernel<TIn, D><<<grid, 128, 0, st>>>(
        static_cast<const TIn*>(p.q), static_cast<const TIn*>(p.k), static_cast<const TIn*>(p.v),
        static_cast<const TIn*>(b.dout_sca), b.lse, w.delta, static_cast<TIn*>(b.dq), p.T, (int)p.c);
  return cudaGetLastError();
}

template <int D, int JC>
cudaError_t bwd_carry_launch(const Workspace& fw, const BwdWorkspace& w, int64_t BH, int S, cudaStream_t st) {
  const size_t smc = sizeof(float) * (2 * BwdCarryStage<D, JC>::kFloats + D * JC);
  cudaError_t e = cudaFuncSetAttribute(awm_bwd_carry_kernel<D, JC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smc);
  if (e != cudaSuccess) return e;
  awm_bwd_carry_kernel<D, JC><<<dim3(D / JC, (unsigned)BH), 256, smc, st>>>(w.E, fw.Cm, fw.ratio, fw.rho, w.G, S);
  return cudaGetLastError();
}

template <typename TIn, int D>
cudaError_t awm_bwd_impl(const BwdProblem& b, const Workspace& fw, const BwdWorkspace& w, cudaStream_t st,
                         bool tc) {
  const Problem& p = b.f;
  const int64_t BH = p.B * p.H;
  const int S = p.S;
  if (tc) {
    cudaError_t e0 = launch_awm_bwd_e_tc(p, b.dout_mem, w.E, st);
    if (e0 != cudaSuccess) return e0;
  } else {
    awm_bwd_e_simt_kernel<TIn, D><<<dim3(S, (unsigned)BH), 256, 0, st>>>(
        static_cast<const TIn*>(p.qm), static_cast<const TIn*>(b.dout_mem), w.E, p.T, (int)p.c);
  }
  cudaError_t e = carry_slice(BH, D) == 32 ? bwd_carry_launch<D, 32>(fw, w, BH, S, st)
                  : carry_slice(BH, D) == 16 ? bwd_carry_launch<D, 16>(fw, w, BH, S, st)
                                             : bwd_carry_launch<D, 8>(fw, w, BH, S, st);
  if (e != cudaSuccess) return e;
  const int64_t nw = BH * D;
  awm_bwd_dl_kernel<D><<<(unsigned)((nw + 7) / 8), 256, 0, st>>>(w.G, fw.Mst, fw.ratio, fw.rho, w.dl, S, nw);
  const dim3 grid((unsigned)(p.c / 32), (unsigned)S, (unsigned)BH);
  if (tc) {
    if ((e = launch_awm_bwd_chunk_tc(b, fw, w, st)) != cudaSuccess) return e;
  } else {
    const size_t smk = sizeof(float) * (2 * D * (D + 1) + 8 * 4 * D);
    e = cudaFuncSetAttribute(awm_bwd_chunk_simt_kernel<TIn, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smk);
    if (e != cudaSuccess) return e;
    awm_bwd_chunk_simt_kernel<TIn, D><<<grid, 256, smk, st>>>(
        static_cast<const TIn*>(p.km), static_cast<const TIn*>(p.v), w.G, fw.Mst, fw.lse, fw.logz, w.dl,
        static_cast<TIn*>(b.dkm), w.dv_awm, p.T, (int)p.c);
  }
  if (tc) {
    if ((e = launch_awm_bwd_readout_tc(b, fw, st)) != cudaSuccess) return e;
  } else {
    const size_t smr = sizeof(float) * (D * (D + 1) + 8 * 4 * D);
    e = cudaFuncSetAttribute(awm_bwd_readout_simt_kernel<TIn, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smr);
    if (e != cudaSuccess) return e;
    awm_bwd_readout_simt_kernel<TIn, D><<<grid, 256, smr, st>>>(
        static_cast<const TIn*>(p.qm), static_cast<const TIn*>(b.dout_mem), fw.Mst, static_cast<TIn*>(b.dqm), p.T,
        (int)p.c);
  }
  return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(int64_t BH, int64_t T, int64_t c, int64_t d) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int64_t S = T / c;
  return 2 * al(sizeof(float) * BH * T) + 2 * al(sizeof(float) * BH * S * d * d) +
         al(sizeof(float) * BH * (S + 1) * d * d) + al(sizeof(float) * BH * S * d) + al(sizeof(float) * BH * T * d);
}

BwdWorkspace carve_bwd_workspace(void* base, int64_t BH, int64_t T, int64_t c, int64_t d) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int64_t S = T / c;
  char* p = static_cast<char*>(base);
  BwdWorkspace w;
  w.delta = reinterpret_cast<float*>(p);
  p += al(sizeof(float) * BH * T);
  w.nlse2 = reinterpret_cast<float*>(p);
  p += al(sizeof(float) * BH * T);
  w.E = reinterpret_cast<float*>(p);
  p += al(sizeof(float) * BH * S * d * d);
  w.G = reinterpret_cast<float*>(p);
  p += al(sizeof(float) * BH * (S + 1) * d * d);
  w.dl = reinterpret_cast<float*>(p);
  p += al(sizeof(float) * BH * S * d);
  w.dv_awm = reinterpret_cast<float*>(p);
  p += al(sizeof(float) * BH * T * d);
  w.W = reinterpret_cast<float*>(p);
  return w;
}

#define GECKO_BWD_DISPATCH(FN, ...)                                                                 \
  (b.f.dtype == kF32 ? (b.f.d == 64 ? FN<float, 64>(__VA_ARGS__) : FN<float, 128>(__VA_ARGS__))         \
                     : (b.f.d == 64 ? FN<__nv_bfloat16, 64>(__VA_ARGS__) : FN<__nv_bfloat16, 128>(__VA_ARGS__)))

cudaError_t launch_sca_bwd_delta(const BwdProblem& b, const BwdWorkspace& w, cudaStream_t st) {
  return GECKO_BWD_DISPATCH(sca_bwd_delta_impl, b, w, st);
}
cudaError_t launch_sca_bwd_simt(const BwdProblem& b, const BwdWorkspace& w, cudaStream_t st, int part) {
  return GECKO_BWD_DISPATCH(sca_bwd_simt_impl, b, w, st, part);
}
cudaError_t launch_awm_bwd(const BwdProblem& b, const Workspace& fw, const BwdWorkspace& w, cudaStream_t st,
                           bool tc) {
  return GECKO_BWD_DISPATCH(awm_bwd_impl, b, fw, w, st, tc && b.f.dtype == kBF16);
}
#undef GECKO_BWD_DISPATCH

}  // namespace gecko
