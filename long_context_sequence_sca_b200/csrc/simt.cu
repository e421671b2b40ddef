// SIMT (CUDA-core, fp32 FMA) kernels of the Gecko forward.  They serve the
// fp32 dtype (where tensor-core tf32 would miss a 1e-4 error bound) and any
// shape the tensor-core kernels do not cover.  Inputs are float or bf16;
// arithmetic is fp32 throughout.
//
// Definitions follow the Gecko digest (paper.rainbus.top): core method
// (phi^s, z^s, psi) and method step details, steps 3-5 (SCA, the M'_s
// update, the readout); and the paperlayer.ai summary, sections 3.2-3.3 and
// Appendix A (M'_1 = 0).
#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

template <typename T> struct Vec8;  // 8 elements in one or two 16-byte words
template <> struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
};
template <> struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&x)[8]) {
    float4 a = reinterpret_cast<const float4*>(p)[0];
    float4 b = reinterpret_cast<const float4*>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

// ------------------------------------------------------------------------
// Partial statistics of K_m per block of R rows: for each feature f the
// block max m and sum_i exp(km[i, f] - m).  grid (T / R, BH), 256 threads;
// each thread holds 8 features of R / RG rows in registers, takes their max
// and then their exp-sum (one SFU exp2 per element), then the row groups are
// merged in shared memory.
template <typename TIn, int D, int R>
__global__ void __launch_bounds__(256) awm_lse_partial_kernel(const TIn* __restrict__ km, float2* __restrict__ part,
                                                              int64_t T) {
  constexpr int TPR = D / 8;          // threads per row
  constexpr int RG = 256 / TPR;       // rows processed in parallel
  constexpr int NR = R / RG;          // rows per thread
  const int blk = blockIdx.x, nblk = gridDim.x;
  const int64_t bh = blockIdx.y;
  const int lane8 = threadIdx.x % TPR;
  const int rg = threadIdx.x / TPR;
  const TIn* base = km + (bh * T + (int64_t)blk * R) * D + lane8 * 8;
  float x[NR][8];
#pragma unroll
  for (int n = 0; n < NR; ++n) Vec8<TIn>::load(base + (int64_t)(rg + n * RG) * D, x[n]);
  float m[8], acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    m[i] = x[0][i];
#pragma unroll
    for (int n = 1; n < NR; ++n) m[i] = fmaxf(m[i], x[n][i]);
    const float m2 = m[i] * kLog2e;
    acc[i] = 0.f;
#pragma unroll
    for (int n = 0; n < NR; ++n) acc[i] += ex2(fmaf(x[n][i], kLog2e, -m2));
  }
  __shared__ float sm[RG][D + 1];
  __shared__ float ss[RG][D + 1];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    sm[rg][lane8 * 8 + i] = m[i];
    ss[rg][lane8 * 8 + i] = acc[i];
  }
  __syncthreads();
  for (int f = threadIdx.x; f < D; f += 256) {
    float M = -INFINITY;
    for (int g = 0; g < RG; ++g) M = fmaxf(M, sm[g][f]);
    float tot = 0.f;
    for (int g = 0; g < RG; ++g) tot += ss[g][f] * expf(sm[g][f] - M);
    part[(bh * nblk + blk) * D + f] = make_float2(M, tot);
  }
}

// Merge the P partials of each chunk: lse[bh, s, f] = log sum over the
// chunk of exp(km[., f]).  grid (S, BH), D threads.
template <int D>
__global__ void __launch_bounds__(D) awm_lse_combine_kernel(const float2* __restrict__ part,
                                                            float* __restrict__ lse, int P) {
  const int s = blockIdx.x, S = gridDim.x;
  const int64_t bh = blockIdx.y;
  const int f = threadIdx.x;
  const float2* p = part + (bh * (int64_t)S * P + (int64_t)s * P) * D + f;
  float M = -INFINITY;
  for (int i = 0; i < P; ++i) M = fmaxf(M, p[(int64_t)i * D].x);
  float tot = 0.f;
  for (int i = 0; i < P; ++i) {
    const float2 v = p[(int64_t)i * D];
    tot += v.y * expf(v.x - M);
  }
  lse[(bh * S + s) * D + f] = M + logf(tot);
}

// ------------------------------------------------------------------------
// Prefix over chunks: log z^s = logaddexp(log z^{s-1}, lse_s) with the
// running sum in fp64, the row ratio r_s = z^{s-1}/z^s (0 for s = 1) and the
// chunk weight
// rho_s = e_s / z^s = exp(lse_s - log z^s).  A continued sequence seeds the
// prefix with the carried log z (logz0, stride sd per (b, h)).  grid BH, D
// threads.
template <int D>
__global__ void __launch_bounds__(D) awm_prefix_kernel(const float* __restrict__ lse, float* __restrict__ logz,
                                                       float* __restrict__ ratio, float* __restrict__ rho, int S,
                                                       const float* __restrict__ logz0, int64_t sd) {
  const int64_t bh = blockIdx.x;
  const int f = threadIdx.x;
  const bool seeded = logz0 != nullptr;
  double L = seeded ? (double)logz0[bh * sd + f] : 0.0;
  // the chunk log-sum-exps are read 8 chunks ahead of the sequential chain,
  // so their load latency is paid once per 8 steps
  float ahead[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) ahead[k] = k < S ? lse[(bh * S + k) * D + f] : 0.f;
  for (int s = 0; s < S; ++s) {
    const int64_t o = (bh * S + s) * D + f;
    const double e = ahead[s % 8];
    if (s % 8 == 7) {
#pragma unroll
      for (int k = 0; k < 8; ++k) ahead[k] = s + 1 + k < S ? lse[(bh * S + s + 1 + k) * D + f] : 0.f;
    }
    double Ln;
    if (s == 0 && !seeded) {
      Ln = e;
    } else {
      // the running sum stays in fp64; the correction log(1 + e^(lo - hi))
      // lies in [0, ln 2] and is accurate to fp32 rounding
      const double hi = fmax(L, e), lo = fmin(L, e);
      Ln = hi + (double)log1pf(expf((float)(lo - hi)));
    }
    logz[o] = (float)Ln;
    // both exponents are <= 0 (log z is non-decreasing and >= lse)
    ratio[o] = (s == 0 && !seeded) ? 0.f : expf((float)(L - Ln));
    rho[o] = expf((float)(e - Ln));
    L = Ln;
  }
}

// ------------------------------------------------------------------------
// Per-chunk GEMMs of the AWM update, in fp32:
//   Bm_s = Phi~_s^T V_s,   Cm_s = Phi~_s^T Psi_s       (D x D each)
// with the chunk-local kernel Phi~_s = exp(Km_s - lse_s) (columns sum to 1)
// and Psi_s = rowsoftmax(Km_s).  The online-softmax kernel of the update is
// Phi_s = rho_s (.) Phi~_s with rho_s = exp(lse_s - log z^s); the carry
// applies rho_s to the rows of Bm_s and Cm_s.
// grid (S, BH), 256 threads as a 16 x 16 grid of (D/16) x (D/16) tiles.
template <typename TIn, int D>
__global__ void __launch_bounds__(256) awm_chunk_simt_kernel(const TIn* __restrict__ km,
                                                             const TIn* __restrict__ v,
                                                             const float* __restrict__ lse,
                                                             float* __restrict__ Bm, float* __restrict__ Cm,
                                                             int64_t T, int c, int64_t koff) {
  constexpr int RT = 16;       // token rows per step
  constexpr int TM = D / 16;   // outputs per thread per dim
  const int s = blockIdx.x;
  const int S = gridDim.x;
  const int64_t bh = blockIdx.y;
  __shared__ float phi_s[RT][D];
  __shared__ float psi_s[RT][D];
  __shared__ float v_s[RT][D];
  __shared__ float lz[D];
  const int tid = threadIdx.x;
  for (int f = tid; f < D; f += 256) lz[f] = lse[(bh * S + s) * D + f];
  const int ty = tid / 16, tx = tid % 16;
  float accB[TM][TM], accC[TM][TM];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TM; ++j) { accB[i][j] = 0.f; accC[i][j] = 0.f; }
  const int64_t row0 = bh * T + (int64_t)s * c;
  // v carries koff extra leading rows per (b, h) when a sequence is continued
  const int64_t vrow0 = bh * (T + koff) + koff + (int64_t)s * c;
  const int warp = tid / 32, lane = tid % 32;
  __syncthreads();
  for (int r0 = 0; r0 < c; r0 += RT) {
    // each warp prepares RT/8 rows: phi, psi (warp-wide softmax over D), v
    for (int rr = warp; rr < RT; rr += 8) {
      const int64_t g = (row0 + r0 + rr) * D;
      const int64_t gv = (vrow0 + r0 + rr) * D;
      float x[D / 32];
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        x[i] = to_f32(km[g + lane + 32 * i]);
        mx = fmaxf(mx, x[i]);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffff, mx, o));
      float sum = 0.f, e[D / 32];
#pragma unroll
      for (int i = 0; i < D / 32; ++i) { e[i] = expf(x[i] - mx); sum += e[i]; }
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffff, sum, o);
      const float inv = 1.f / sum;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        const int f = lane + 32 * i;
        psi_s[rr][f] = e[i] * inv;
        phi_s[rr][f] = expf(x[i] - lz[f]);
        v_s[rr][f] = to_f32(v[gv + f]);
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < RT; ++t) {
      float a[TM], b[TM], p[TM];
#pragma unroll
      for (int i = 0; i < TM; ++i) {
        a[i] = phi_s[t][ty * TM + i];
        b[i] = v_s[t][tx * TM + i];
        p[i] = psi_s[t][tx * TM + i];
      }
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TM; ++j) {
          accB[i][j] = fmaf(a[i], b[j], accB[i][j]);
          accC[i][j] = fmaf(a[i], p[j], accC[i][j]);
        }
    }
    __syncthreads();
  }
  const int64_t o = (bh * S + s) * (int64_t)D * D;
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TM; ++j) {
      Bm[o + (ty * TM + i) * D + tx * TM + j] = accB[i][j];
      Cm[o + (ty * TM + i) * D + tx * TM + j] = accC[i][j];
    }
}

// ------------------------------------------------------------------------
// The sequential carry, one slice of JC value columns per CTA (columns of M'
// evolve independently):
//   M'_{s+1}[:, J] = r_s (.) M'_s[:, J] + rho_s (.) (Bm_s[:, J] - Cm_s M'_s[:, J])
// (row scales r_s = z^{s-1}/z^s and rho_s = e_s/z^s).  Writes
// Mst[bh, s] = M'_{s+1} for s = 0..S.  M'_1 = 0 for a fresh sequence; a
// continued one starts from the carried M' (M0, stride sd per (b, h)).
// Everything step s + 1 reads from global memory (Cm, the CTA's slice of
// Bm, r, rho) is copied into shared memory with 16-byte asynchronous copies
// while step s computes (double buffer), so a step's critical path holds
// only shared-memory reads and FMAs.  grid (D / JC, BH), 256 threads.
template <int D, int JC>
struct CarryStage {
  static constexpr int LD = D + 4;   // padded row of Cm (keeps 16-byte alignment)
  static constexpr int kC = 0, kB = D * LD, kR = kB + D * JC, kP = kR + D;
  static constexpr int kFloats = kP + D;
};

// The thread's RB x CB block of a d x d matrix as bf16 into a readout
// operand image (128-byte-swizzled MN-major, 64-column boxes of D rows).
template <int D, int RB, int CB>
__device__ __forceinline__ void put_image(uint16_t* img, int f0, int c0, const float (&v)[RB][CB]) {
  uint8_t* base = reinterpret_cast<uint8_t*>(img);
#pragma unroll
  for (int i = 0; i < RB; ++i)
#pragma unroll
    for (int j = 0; j < CB; ++j)
      *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(f0 + i, c0 + j, D)) = __float2bfloat16_rn(v[i][j]);
}

template <int D, int JC>
__global__ void __launch_bounds__(256) awm_carry_kernel(const float* __restrict__ Bm,
                                                        const float* __restrict__ Cm,
                                                        const float* __restrict__ ratio,
                                                        const float* __restrict__ rho,
                                                        float* __restrict__ Mst, int S,
                                                        const float* __restrict__ M0, int64_t sd,
                                                        uint16_t* __restrict__ Mimg,
                                                        const float* __restrict__ Mprev0) {
  using St = CarryStage<D, JC>;
  // each thread owns an RB x CB block of the slice: rows f0 .. f0 + RB - 1,
  // columns c0 .. c0 + CB - 1 (8 column groups, D / RB row groups), so that
  // four steps of the inner product cost RB + 4 shared loads for 4 RB CB FMAs
  constexpr int CB = JC / 8, RB = D / 32;
  static_assert(CB >= 1 && RB * CB * 256 == D * JC, "thread layout");
  constexpr int LD = St::LD;
  extern __shared__ float smem_carry[];
  // buffer b at smem_carry + b * St::kFloats (computed, so no pointer array in local memory)
  float* Ms = smem_carry + 2 * St::kFloats;            // [D][JC]
  const int64_t bh = blockIdx.y;
  const int j0 = blockIdx.x * JC;
  const int tid = threadIdx.x;
  const int f0 = (tid / 8) * RB, c0 = (tid % 8) * CB;
  const int64_t mst_stride = (int64_t)D * D;
  auto stage = [&](int s, float* dst) {
    const float4* C4 = reinterpret_cast<const float4*>(Cm + (bh * S + s) * mst_stride);
    for (int i = tid; i < D * D / 4; i += 256) {
      const int row = (i * 4) / D, col = (i * 4) % D;
      cp_async16(dst + St::kC + row * LD + col, C4 + i);
    }
    const float* Bs = Bm + (bh * S + s) * mst_stride + j0;
    for (int i = tid; i < D * JC / 4; i += 256) {
      const int row = (i * 4) / JC, col = (i * 4) % JC;
      cp_async16(dst + St::kB + row * JC + col, Bs + row * D + col);
    }
    for (int i = tid; i < D / 4; i += 256) {
      cp_async16(dst + St::kR + 4 * i, ratio + (bh * S + s) * D + 4 * i);
      cp_async16(dst + St::kP + 4 * i, rho + (bh * S + s) * D + 4 * i);
    }
    cp_async_commit();
  };
  if (S > 0) stage(0, smem_carry);
  for (int i = tid; i < D * JC; i += 256)
    Ms[i] = M0 ? M0[bh * sd + (i / JC) * D + j0 + i % JC] : 0.f;
  float* mout = Mst + bh * (int64_t)(S + 1) * mst_stride;
  // readout operand images (if requested): image k + 1 holds Mst[k] for
  // k < S, image 0 the carried M'_prev of a continued sequence
  uint16_t* iout = Mimg ? Mimg + bh * (int64_t)(S + 1) * mst_stride : nullptr;
  __syncthreads();
  {
    float m1[RB][CB];
#pragma unroll
    for (int i = 0; i < RB; ++i)
#pragma unroll
      for (int j = 0; j < CB; ++j) {
        m1[i][j] = Ms[(f0 + i) * JC + c0 + j];
        mout[(f0 + i) * D + j0 + c0 + j] = m1[i][j];   // M'_1
      }
    if (iout && S > 1) put_image<D, RB, CB>(iout + mst_stride, f0, j0 + c0, m1);
    if (iout && Mprev0) {
#pragma unroll
      for (int i = 0; i < RB; ++i)
#pragma unroll
        for (int j = 0; j < CB; ++j) m1[i][j] = Mprev0[bh * sd + (f0 + i) * D + j0 + c0 + j];
      put_image<D, RB, CB>(iout, f0, j0 + c0, m1);
    }
  }
  for (int s = 0; s < S; ++s) {
    const float* sb = smem_carry + (s & 1) * St::kFloats;
    if (s + 1 < S) {
      stage(s + 1, smem_carry + ((s + 1) & 1) * St::kFloats);   // its buffer was last read by step s - 1
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const float* Cs = sb + St::kC;
    float acc[RB][CB];
#pragma unroll
    for (int i = 0; i < RB; ++i)
#pragma unroll
      for (int j = 0; j < CB; ++j) acc[i][j] = sb[St::kB + (f0 + i) * JC + c0 + j];
#pragma unroll 2
    for (int g = 0; g < D; g += 4) {
      float4 cr[RB];
#pragma unroll
      for (int i = 0; i < RB; ++i) cr[i] = *reinterpret_cast<const float4*>(Cs + (f0 + i) * LD + g);
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) {
        float m[CB];
#pragma unroll
        for (int j = 0; j < CB; ++j) m[j] = Ms[(g + gg) * JC + c0 + j];
#pragma unroll
        for (int i = 0; i < RB; ++i) {
          const float c = gg == 0 ? cr[i].x : gg == 1 ? cr[i].y : gg == 2 ? cr[i].z : cr[i].w;
#pragma unroll
          for (int j = 0; j < CB; ++j) acc[i][j] = fmaf(-c, m[j], acc[i][j]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < RB; ++i) {
      const float rf = sb[St::kR + f0 + i], pf = sb[St::kP + f0 + i];
#pragma unroll
      for (int j = 0; j < CB; ++j) acc[i][j] = fmaf(rf, Ms[(f0 + i) * JC + c0 + j], pf * acc[i][j]);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < RB; ++i) {
      float* dst = mout + (int64_t)(s + 1) * mst_stride + (f0 + i) * D + j0 + c0;
#pragma unroll
      for (int j = 0; j < CB; ++j) {
        Ms[(f0 + i) * JC + c0 + j] = acc[i][j];
        dst[j] = acc[i][j];
      }
    }
    if (iout && s + 2 < S) put_image<D, RB, CB>(iout + (int64_t)(s + 2) * mst_stride, f0, j0 + c0, acc);
  }
}

// ------------------------------------------------------------------------
// Readout O_m,s = psi(Qm_s) M'_{s-1}.  For a fresh sequence chunks 1 and 2
// read zero; a continued one reads the carried M'_prev (Mprev0, stride sd)
// for its first chunk and the carried M'_cur (= Mst[0]) for its second.
// grid (c / 64, S, BH), 256 threads; 64 rows per CTA.
template <typename TIn, int D>
__global__ void __launch_bounds__(256) awm_readout_simt_kernel(const TIn* __restrict__ qm,
                                                               const float* __restrict__ Mst,
                                                               TIn* __restrict__ out, int64_t T, int c,
                                                               const float* __restrict__ Mprev0, int64_t sd) {
  constexpr int R = 64;
  constexpr int CT = D / 16;  // columns per thread
  extern __shared__ float smem_ro[];
  float* Ms = smem_ro;          // [D][D]
  float* ps = Ms + D * D;       // [R][D + 1]
  const int s = blockIdx.y;     // 0-based chunk
  const int S = gridDim.y;
  const int64_t bh = blockIdx.z;
  const int64_t row0 = bh * T + (int64_t)s * c + (int64_t)blockIdx.x * R;
  const int tid = threadIdx.x;
  if (s < 2 && Mprev0 == nullptr) {
    for (int i = tid; i < R * D; i += 256) out[row0 * D + i] = from_f32<TIn>(0.f);
    return;
  }
  // 0-based chunk s is chunk s+1; it reads M'_s = Mst[s - 1] (M'_prev for s = 0)
  const float* M = s == 0 ? Mprev0 + bh * sd : Mst + (bh * (S + 1) + (s - 1)) * (int64_t)D * D;
  for (int i = tid; i < D * D; i += 256) Ms[i] = M[i];
  const int warp = tid / 32, lane = tid % 32;
  for (int rr = warp; rr < R; rr += 8) {
    float x[D / 32], mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      x[i] = to_f32(qm[(row0 + rr) * D + lane + 32 * i]);
      mx = fmaxf(mx, x[i]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffff, mx, o));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) { x[i] = expf(x[i] - mx); sum += x[i]; }
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffff, sum, o);
    const float inv = 1.f / sum;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) ps[rr * (D + 1) + lane + 32 * i] = x[i] * inv;
  }
  __syncthreads();
  const int ty = tid / 16, tx = tid % 16;  // rows ty*4..+4, cols tx*CT..+CT
  float acc[4][CT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < CT; ++j) acc[i][j] = 0.f;
  for (int f = 0; f < D; ++f) {
    float a[4], b[CT];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = ps[(ty * 4 + i) * (D + 1) + f];
#pragma unroll
    for (int j = 0; j < CT; ++j) b[j] = Ms[f * D + tx * CT + j];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < CT; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < CT; ++j) out[(row0 + ty * 4 + i) * D + tx * CT + j] = from_f32<TIn>(acc[i][j]);
}

// ------------------------------------------------------------------------
// SCA with CUDA cores: 32 queries per CTA, 4 threads per query (each owns
// D/4 dims of q and of the output), keys streamed through shared memory in
// tiles of 32 with an online softmax; writes each row's log-sum-exp to lse
// when it is given.  Scale 1.  k and v hold koff extra
// leading rows per (b, h) (the previous chunk of a continued sequence, so
// chunk 1 then has a previous chunk).  grid (T / 32, BH).
template <typename TIn, int D>
__global__ void __launch_bounds__(128) sca_simt_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                                                       const TIn* __restrict__ v, TIn* __restrict__ out,
                                                       float* __restrict__ lse, TIn* __restrict__ out_lo,
                                                       int64_t T, int c, int64_t koff) {
  constexpr int QD = D / 4;
  __shared__ float ks[32][D + 4];
  __shared__ float vs[32][D + 4];
  const int64_t bh = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * 32;
  const int tid = threadIdx.x;
  const int qi = tid / 4, part = tid % 4;
  const int64_t t = t0 + qi;
  // window start in segment coordinates (negative: rows of the prepended chunk);
  // all 32 rows share one chunk
  const int64_t lo = (t0 / c >= 1 || koff > 0) ? (t0 / c - 1) * c : 0;
  const int64_t kbase = bh * (T + koff) + koff;
  const TIn* qrow = q + (bh * T + t) * D + part * QD;
  float qv[QD], acc[QD];
#pragma unroll
  for (int i = 0; i < QD; ++i) { qv[i] = to_f32(qrow[i]); acc[i] = 0.f; }
  float m = -INFINITY, l = 0.f;
  const int64_t hi = t0 + 31;
  for (int64_t k0 = lo; k0 <= hi; k0 += 32) {
    __syncthreads();
    for (int i = tid; i < 32 * D; i += 128) {
      const int r = i / D, cc = i % D;
      const int64_t g = (kbase + k0 + r) * D + cc;
      ks[r][cc] = to_f32(k[g]);
      vs[r][cc] = to_f32(v[g]);
    }
    __syncthreads();
    for (int j = 0; j < 32; ++j) {
      float sc = 0.f;
#pragma unroll
      for (int i = 0; i < QD; ++i) sc = fmaf(qv[i], ks[j][part * QD + i], sc);
      sc += __shfl_xor_sync(0xffffffff, sc, 1);
      sc += __shfl_xor_sync(0xffffffff, sc, 2);
      if (k0 + j > t) continue;  // causal inside the current chunk
      const float mn = fmaxf(m, sc);
      const float corr = expf(m - mn);
      const float p = expf(sc - mn);
      l = l * corr + p;
#pragma unroll
      for (int i = 0; i < QD; ++i) acc[i] = fmaf(p, vs[j][part * QD + i], acc[i] * corr);
      m = mn;
    }
  }
  const float inv = 1.f / l;
  if (lse && part == 0) lse[bh * T + t] = m + logf(l);
  TIn* orow = out + (bh * T + t) * D + part * QD;
#pragma unroll
  for (int i = 0; i < QD; ++i) orow[i] = from_f32<TIn>(acc[i] * inv);
  if (out_lo) {
    // rounding residual of the stored output (zero for fp32)
    TIn* lrow = out_lo + (bh * T + t) * D + part * QD;
#pragma unroll
    for (int i = 0; i < QD; ++i) {
      const float x = acc[i] * inv;
      lrow[i] = from_f32<TIn>(x - to_f32(from_f32<TIn>(x)));
    }
  }
}

template <typename TIn, int D>
cudaError_t awm_stats_impl(const Problem& p, const Workspace& w, cudaStream_t st) {
  const int64_t BH = p.B * p.H;
  const int R = stats_block_rows(p.c);
  const int P = (int)(p.c / R);
  const dim3 grid((unsigned)(p.T / R), BH);
  if (R == 128)
    awm_lse_partial_kernel<TIn, D, 128><<<grid, 256, 0, st>>>(static_cast<const TIn*>(p.km), w.part, p.T);
  else
    awm_lse_partial_kernel<TIn, D, 64><<<grid, 256, 0, st>>>(static_cast<const TIn*>(p.km), w.part, p.T);
  awm_lse_combine_kernel<D><<<dim3(p.S, BH), D, 0, st>>>(w.part, w.lse, P);
  const int64_t sd = state_floats(D);
  awm_prefix_kernel<D><<<BH, D, 0, st>>>(w.lse, w.logz, w.ratio, w.rho, p.S,
                                         p.state0 ? p.state0 + 2 * D * D : nullptr, sd);
  return cudaGetLastError();
}

template <int D>
cudaError_t awm_prefix_impl(const Problem& p, const Workspace& w, cudaStream_t st) {
  awm_prefix_kernel<D><<<p.B * p.H, D, 0, st>>>(w.lse, w.logz, w.ratio, w.rho, p.S,
                                               p.state0 ? p.state0 + 2 * D * D : nullptr, state_floats(D));
  return cudaGetLastError();
}

template <typename TIn, int D>
cudaError_t awm_chunk_simt_impl(const Problem& p, const Workspace& w, cudaStream_t st) {
  awm_chunk_simt_kernel<TIn, D><<<dim3(p.S, p.B * p.H), 256, 0, st>>>(
      static_cast<const TIn*>(p.km), static_cast<const TIn*>(p.v), w.lse, w.Bm, w.Cm, p.T, (int)p.c, p.koff);
  return cudaGetLastError();
}

template <int D, int JC>
cudaError_t awm_carry_launch(const Problem& p, const Workspace& w, cudaStream_t st, bool images) {
  const size_t smem = sizeof(float) * (2 * CarryStage<D, JC>::kFloats + D * JC);
  cudaError_t e = cudaFuncSetAttribute(awm_carry_kernel<D, JC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  awm_carry_kernel<D, JC><<<dim3(D / JC, p.B * p.H), 256, smem, st>>>(
      w.Bm, w.Cm, w.ratio, w.rho, w.Mst, p.S, p.state0 ? p.state0 + D * D : nullptr, state_floats(D),
      images ? w.Mimg : nullptr, p.state0);
  return cudaGetLastError();
}

template <int D>
cudaError_t awm_carry_impl(const Problem& p, const Workspace& w, cudaStream_t st, bool images) {
  const int jc = carry_slice(p.B * p.H, D);
  return jc == 32 ? awm_carry_launch<D, 32>(p, w, st, images)
                  : jc == 16 ? awm_carry_launch<D, 16>(p, w, st, images) : awm_carry_launch<D, 8>(p, w, st, images);
}

template <typename TIn, int D>
cudaError_t awm_readout_simt_impl(const Problem& p, const Workspace& w, cudaStream_t st) {
  const size_t smem = sizeof(float) * (D * D + 64 * (D + 1));
  cudaError_t e =
      cudaFuncSetAttribute(awm_readout_simt_kernel<TIn, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  awm_readout_simt_kernel<TIn, D><<<dim3(p.c / 64, p.S, p.B * p.H), 256, smem, st>>>(
      static_cast<const TIn*>(p.qm), w.Mst, static_cast<TIn*>(p.out_mem), p.T, (int)p.c, p.state0, state_floats(D));
  return cudaGetLastError();
}

template <typename TIn, int D>
cudaError_t launch_sca_simt_impl(const Problem& p, cudaStream_t st) {
  sca_simt_kernel<TIn, D><<<dim3(p.T / 32, p.B * p.H), 128, 0, st>>>(
      static_cast<const TIn*>(p.q), static_cast<const TIn*>(p.k), static_cast<const TIn*>(p.v),
      static_cast<TIn*>(p.out_sca), p.lse, static_cast<TIn*>(p.out_sca_lo), p.T, (int)p.c, p.koff);
  return cudaGetLastError();
}

}  // namespace

#define GECKO_DISPATCH(FN)                                                              \
  (p.dtype == kF32 ? (p.d == 64 ? FN<float, 64>(p, w, st) : FN<float, 128>(p, w, st))      \
                   : (p.d == 64 ? FN<__nv_bfloat16, 64>(p, w, st) : FN<__nv_bfloat16, 128>(p, w, st)))

cudaError_t launch_awm_stats(const Problem& p, const Workspace& w, cudaStream_t st) {
  return GECKO_DISPATCH(awm_stats_impl);
}
cudaError_t launch_awm_prefix(const Problem& p, const Workspace& w, cudaStream_t st) {
  return p.d == 64 ? awm_prefix_impl<64>(p, w, st) : awm_prefix_impl<128>(p, w, st);
}
cudaError_t launch_awm_chunk_simt(const Problem& p, const Workspace& w, cudaStream_t st) {
  return GECKO_DISPATCH(awm_chunk_simt_impl);
}
cudaError_t launch_awm_carry(const Problem& p, const Workspace& w, cudaStream_t st, bool images) {
  return p.d == 64 ? awm_carry_impl<64>(p, w, st, images) : awm_carry_impl<128>(p, w, st, images);
}
cudaError_t launch_awm_readout_simt(const Problem& p, const Workspace& w, cudaStream_t st) {
  return GECKO_DISPATCH(awm_readout_simt_impl);
}
#undef GECKO_DISPATCH

cudaError_t launch_sca_simt(const Problem& p, cudaStream_t st) {
  if (p.dtype == kF32)
    return p.d == 64 ? launch_sca_simt_impl<float, 64>(p, st) : launch_sca_simt_impl<float, 128>(p, st);
  return p.d == 64 ? launch_sca_simt_impl<__nv_bfloat16, 64>(p, st)
                   : launch_sca_simt_impl<__nv_bfloat16, 128>(p, st);
}

}  // namespace gecko
