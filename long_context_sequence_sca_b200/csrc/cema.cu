// CEMA: complex multi-dimensional damped exponential moving average, the
// recurrence that produces the layer input X' = CEMA(X) (Gecko digest,
// paper.rainbus.top, background section on the exponential moving average;
// paperlayer.ai summary, section 2.1 and Appendix B.1):
//
//   u_t[d, j] = beta[d, j] x_t[d]                       (expansion, h = 16)
//   h_t[d, j] = alpha u_t + q h_{t-1},  q = (1 - alpha delta)(cos theta + i sin theta)
//   y_t[d]    = Re(sum_j eta[d, j] h_t[d, j])            (projection)
//
// with q replaced by 0 at a document start (the state restarts at
// h_t = alpha u_t).  The recurrence is an affine map per step, so it is
// evaluated as a chunked scan (the pages' Appendix B.1 reformulates it as a
// parallel associative scan over (q, p) tuples):
//   1. cema_local_kernel: every 256-token chunk is scanned from a zero state,
//      giving its end state B_c (one thread per (batch, chunk, feature), the
//      16 complex states in registers).
//   2. cema_carry_kernel: per (batch, feature, j), H_{c+1} = A_c H_c + B_c
//      over the chunks, with A_c = q^len (0 if the chunk holds a reset).
//   3. cema_out_kernel: every chunk is rescanned from its incoming H_c and
//      y is written.
// Work is FP32 FMA on the CUDA cores (the recurrence is elementwise, not a
// contraction); loads and stores of x and y are coalesced over features.
#include <cmath>

#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

constexpr int kCemaH = 16;      // hidden dimensions per feature
constexpr int kCemaLC = 256;    // tokens per chunk
constexpr int kCemaThreads = 128;
constexpr int kCemaUnroll = 8;  // tokens whose inputs are loaded ahead

// Per-feature constants: q (re, im) and alpha * beta.
struct CemaCoef {
  float qr[kCemaH], qi[kCemaH], ab[kCemaH];
};

__device__ __forceinline__ void load_coef(CemaCoef& k, const float* alpha, const float* delta, const float* theta,
                                          const float* beta, int d) {
#pragma unroll
  for (int j = 0; j < kCemaH; ++j) {
    const float a = alpha[d * kCemaH + j], m = 1.f - a * delta[d * kCemaH + j];
    float s, c;
    sincosf(theta[d * kCemaH + j], &s, &c);
    k.qr[j] = m * c;
    k.qi[j] = m * s;
    k.ab[j] = a * beta[d * kCemaH + j];
  }
}

// Stage the chunk's reset flags in shared memory (1 = a document starts).
__device__ __forceinline__ void stage_resets(uint8_t* rs, const uint8_t* reset, int64_t b, int64_t L, int64_t t0,
                                             int n) {
  for (int i = threadIdx.x; i < kCemaLC; i += blockDim.x) rs[i] = (reset && i < n) ? reset[b * L + t0 + i] : 0;
  __syncthreads();
}

// 1. Local scan of one chunk from zero, in units of alpha beta:
//    g_t = q g_{t-1} + x_t (g = 0 across a reset), B_c = alpha beta g_end.
//    Writes Bc[b, c, d, j] (complex) and, from block 0, the chunk's reset
//    flag.  grid (ceil(D / 128), C, B).
template <typename TIn>
__global__ void __launch_bounds__(kCemaThreads) cema_local_kernel(const TIn* __restrict__ x, const float* alpha,
                                                                  const float* delta, const float* theta,
                                                                  const float* beta, const uint8_t* reset,
                                                                  float2* __restrict__ Bc,
                                                                  uint8_t* __restrict__ chunk_reset, int64_t L,
                                                                  int64_t D) {
  __shared__ uint8_t rs[kCemaLC];
  const int64_t b = blockIdx.z, c = blockIdx.y;
  const int64_t d = (int64_t)blockIdx.x * kCemaThreads + threadIdx.x;
  const int64_t t0 = c * kCemaLC;
  const int n = (int)(L - t0 < kCemaLC ? L - t0 : kCemaLC);
  stage_resets(rs, reset, b, L, t0, n);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    int any = 0;
    for (int i = 0; i < n; ++i) any |= rs[i];
    chunk_reset[b * gridDim.y + c] = (uint8_t)any;
  }
  if (d >= D) return;
  CemaCoef k;
  load_coef(k, alpha, delta, theta, beta, (int)d);
  float gr[kCemaH], gi[kCemaH];
#pragma unroll
  for (int j = 0; j < kCemaH; ++j) gr[j] = gi[j] = 0.f;
  const TIn* xp = x + (b * L + t0) * D + d;
  for (int s = 0; s < n; s += kCemaUnroll) {
    float xv[kCemaUnroll];
#pragma unroll
    for (int u = 0; u < kCemaUnroll; ++u) xv[u] = s + u < n ? to_f32(xp[(int64_t)(s + u) * D]) : 0.f;
#pragma unroll
    for (int u = 0; u < kCemaUnroll; ++u) {
      if (s + u >= n) break;
      if (rs[s + u]) {
#pragma unroll
        for (int j = 0; j < kCemaH; ++j) gr[j] = gi[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < kCemaH; ++j) {
        const float r = fmaf(k.qr[j], gr[j], fmaf(-k.qi[j], gi[j], xv[u]));
        gi[j] = fmaf(k.qr[j], gi[j], k.qi[j] * gr[j]);
        gr[j] = r;
      }
    }
  }
  float4* out = reinterpret_cast<float4*>(Bc + ((b * gridDim.y + c) * D + d) * kCemaH);
#pragma unroll
  for (int j = 0; j < kCemaH; j += 2)
    out[j / 2] = make_float4(k.ab[j] * gr[j], k.ab[j] * gi[j], k.ab[j + 1] * gr[j + 1], k.ab[j + 1] * gi[j + 1]);
}

// 2. Carry across chunks: H_{c+1} = A_c H_c + B_c, A_c = q^len_c (0 when
//    the chunk holds a reset); Hin[b, c] = H_c.  q^len is taken in fp64
//    (len * theta can be a few thousand radians).  One thread per
//    (b, d, j); grid ceil(B * D * 16 / 256).
__global__ void __launch_bounds__(256) cema_carry_kernel(const float* alpha, const float* delta, const float* theta,
                                                         const float2* __restrict__ Bc,
                                                         const uint8_t* __restrict__ chunk_reset,
                                                         float2* __restrict__ Hin, const float* state_in,
                                                         float* state_out, int64_t B, int64_t L, int64_t D, int C) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * D * kCemaH) return;
  const int64_t j = idx % kCemaH, d = (idx / kCemaH) % D, b = idx / (kCemaH * D);
  const double m = 1.0 - (double)alpha[d * kCemaH + j] * (double)delta[d * kCemaH + j];
  const double th = theta[d * kCemaH + j];
  // full chunks and the last (possibly shorter) chunk
  const int64_t nlast = L - (int64_t)(C - 1) * kCemaLC;
  const double mf = pow(m, (double)kCemaLC), ml = pow(m, (double)nlast);
  const float2 Af = make_float2((float)(mf * cos(kCemaLC * th)), (float)(mf * sin(kCemaLC * th)));
  const float2 Al = make_float2((float)(ml * cos(nlast * th)), (float)(ml * sin(nlast * th)));
  float hr = 0.f, hi = 0.f;
  if (state_in) {
    hr = state_in[2 * idx];
    hi = state_in[2 * idx + 1];
  }
  for (int c = 0; c < C; ++c) {
    const int64_t o = ((b * C + c) * D + d) * kCemaH + j;
    Hin[o] = make_float2(hr, hi);
    const float2 bc = Bc[o];
    if (chunk_reset[b * C + c]) {
      hr = bc.x;
      hi = bc.y;
    } else {
      const float2 A = c == C - 1 ? Al : Af;
      const float r = fmaf(A.x, hr, fmaf(-A.y, hi, bc.x));
      hi = fmaf(A.x, hi, fmaf(A.y, hr, bc.y));
      hr = r;
    }
  }
  if (state_out) {
    state_out[2 * idx] = hr;
    state_out[2 * idx + 1] = hi;
  }
}

// 3. Rescan every chunk from its incoming state and write
//    y_t = Re(sum_j eta_j h_t,j).  grid (ceil(D / 128), C, B).
template <typename TIn>
__global__ void __launch_bounds__(kCemaThreads) cema_out_kernel(const TIn* __restrict__ x, const float* alpha,
                                                                const float* delta, const float* theta,
                                                                const float* beta, const float* eta,
                                                                const uint8_t* reset, const float2* __restrict__ Hin,
                                                                TIn* __restrict__ y, int64_t L, int64_t D) {
  __shared__ uint8_t rs[kCemaLC];
  const int64_t b = blockIdx.z, c = blockIdx.y;
  const int64_t d = (int64_t)blockIdx.x * kCemaThreads + threadIdx.x;
  const int64_t t0 = c * kCemaLC;
  const int n = (int)(L - t0 < kCemaLC ? L - t0 : kCemaLC);
  stage_resets(rs, reset, b, L, t0, n);
  if (d >= D) return;
  CemaCoef k;
  load_coef(k, alpha, delta, theta, beta, (int)d);
  float er[kCemaH], ei[kCemaH], hr[kCemaH], hi[kCemaH];
  const float4* hin = reinterpret_cast<const float4*>(Hin + ((b * gridDim.y + c) * D + d) * kCemaH);
#pragma unroll
  for (int j = 0; j < kCemaH; j += 2) {
    const float4 v = hin[j / 2];
    hr[j] = v.x;
    hi[j] = v.y;
    hr[j + 1] = v.z;
    hi[j + 1] = v.w;
    er[j] = eta[(d * kCemaH + j) * 2];
    ei[j] = eta[(d * kCemaH + j) * 2 + 1];
    er[j + 1] = eta[(d * kCemaH + j + 1) * 2];
    ei[j + 1] = eta[(d * kCemaH + j + 1) * 2 + 1];
  }
  const TIn* xp = x + (b * L + t0) * D + d;
  TIn* yp = y + (b * L + t0) * D + d;
  for (int s = 0; s < n; s += kCemaUnroll) {
    float xv[kCemaUnroll];
#pragma unroll
    for (int u = 0; u < kCemaUnroll; ++u) xv[u] = s + u < n ? to_f32(xp[(int64_t)(s + u) * D]) : 0.f;
#pragma unroll
    for (int u = 0; u < kCemaUnroll; ++u) {
      if (s + u >= n) break;
      if (rs[s + u]) {
#pragma unroll
        for (int j = 0; j < kCemaH; ++j) hr[j] = hi[j] = 0.f;
      }
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int j = 0; j < kCemaH; ++j) {
        const float p = k.ab[j] * xv[u];
        const float r = fmaf(k.qr[j], hr[j], fmaf(-k.qi[j], hi[j], p));
        hi[j] = fmaf(k.qr[j], hi[j], k.qi[j] * hr[j]);
        hr[j] = r;
        if (j & 1)
          acc1 = fmaf(er[j], hr[j], fmaf(-ei[j], hi[j], acc1));
        else
          acc0 = fmaf(er[j], hr[j], fmaf(-ei[j], hi[j], acc0));
      }
      yp[(int64_t)(s + u) * D] = from_f32<TIn>(acc0 + acc1);
    }
  }
}

template <typename TIn>
cudaError_t cema_impl(const CemaProblem& p, const CemaWorkspace& w, cudaStream_t st) {
  const int C = (int)((p.L + kCemaLC - 1) / kCemaLC);
  const dim3 grid((unsigned)((p.D + kCemaThreads - 1) / kCemaThreads), (unsigned)C, (unsigned)p.B);
  cema_local_kernel<TIn><<<grid, kCemaThreads, 0, st>>>(static_cast<const TIn*>(p.x), p.alpha, p.delta, p.theta,
                                                         p.beta, p.reset, w.Bc, w.chunk_reset, p.L, p.D);
  const int64_t nthr = p.B * p.D * kCemaH;
  cema_carry_kernel<<<(unsigned)((nthr + 255) / 256), 256, 0, st>>>(p.alpha, p.delta, p.theta, w.Bc, w.chunk_reset,
                                                                     w.Hin, p.state_in, p.state_out, p.B, p.L, p.D,
                                                                     C);
  cema_out_kernel<TIn><<<grid, kCemaThreads, 0, st>>>(static_cast<const TIn*>(p.x), p.alpha, p.delta, p.theta,
                                                       p.beta, p.eta, p.reset, w.Hin, static_cast<TIn*>(p.y), p.L,
                                                       p.D);
  return cudaGetLastError();
}

}  // namespace

int64_t cema_chunks(int64_t L) { return (L + kCemaLC - 1) / kCemaLC; }

size_t cema_workspace_bytes(int64_t B, int64_t L, int64_t D) {
  const int64_t C = cema_chunks(L);
  return (size_t)(2 * B * C * D * kCemaH) * sizeof(float2) + (size_t)(B * C + 255) / 256 * 256;
}

CemaWorkspace carve_cema_workspace(void* base, int64_t B, int64_t L, int64_t D) {
  const int64_t C = cema_chunks(L);
  CemaWorkspace w;
  w.Bc = static_cast<float2*>(base);
  w.Hin = w.Bc + B * C * D * kCemaH;
  w.chunk_reset = reinterpret_cast<uint8_t*>(w.Hin + B * C * D * kCemaH);
  return w;
}

cudaError_t launch_cema(const CemaProblem& p, const CemaWorkspace& w, cudaStream_t st) {
  return p.dtype == kBF16 ? cema_impl<__nv_bfloat16>(p, w, st) : cema_impl<float>(p, w, st);
}

int cema_hidden() { return kCemaH; }

}  // namespace gecko
