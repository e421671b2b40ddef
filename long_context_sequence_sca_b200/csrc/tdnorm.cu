// Timestep decay normalisation, the normalisation before Gecko's
// projections (Gecko digest, paper.rainbus.top, section on technical
// novelty: m_t = beta1 m_{t-1} + (1 - beta1) mu_t with Adam-style bias
// correction; paperlayer.ai summary, sections 2.2 and 3.1).  Per batch b,
// token t and feature group g (D / G contiguous features):
//
//   mu_t, s2_t = mean and biased variance of x_t over the group
//   m_t = beta1 m_{t-1} + (1 - beta1) mu_t,   v_t = beta2 v_{t-1} + (1 - beta2) s2_t
//   m^_t = m_t / (1 - beta1^t),  v^_t = v_t / (1 - beta2^t)      (t from 1)
//   y_t = (x_t - m^_t) / sqrt(v^_t + eps) * gamma + bias
//
// Three HBM-bound kernels: group statistics (one pass over x), the decayed
// statistics as a block-wide scan per (b, g) over the tokens, and the
// elementwise normalisation (a second pass over x, writing y).
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

// 8 values of a 16-byte vector as floats.
template <typename TIn>
__device__ __forceinline__ void load8(const TIn* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 a = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

template <typename TIn>
__device__ __forceinline__ void store8(TIn* p, const float (&v)[8]);
template <>
__device__ __forceinline__ void store8<float>(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[8]) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

// 1. mu, s2 [B*L, G] for every (token, group): one thread per pair, the
//    group's features read in 16-byte vectors; variance by the shifted
//    one-pass sums (shift = the group's first value) for accuracy.
template <typename TIn>
__global__ void __launch_bounds__(256) tdnorm_stats_kernel(const TIn* __restrict__ x, float2* __restrict__ st,
                                                           int64_t rows, int64_t D, int G) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * G) return;
  const int64_t row = idx / G;
  const int g = (int)(idx % G);
  const int gs = (int)(D / G);
  const TIn* p = x + row * D + (int64_t)g * gs;
  const float k = to_f32(p[0]);
  float s = 0.f, q = 0.f;
  int i = 0;
  for (; i + 32 <= gs; i += 32) {   // four 16-byte loads in flight
    float v[4][8];
#pragma unroll
    for (int u = 0; u < 4; ++u) load8(p + i + 8 * u, v[u]);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float dv = v[u][e] - k;
        s += dv;
        q = fmaf(dv, dv, q);
      }
  }
  for (; i < gs; i += 8) {
    float v[8];
    load8(p + i, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float dv = v[e] - k;
      s += dv;
      q = fmaf(dv, dv, q);
    }
  }
  const float mean_d = s / gs;
  st[idx] = make_float2(k + mean_d, fmaxf(q / gs - mean_d * mean_d, 0.f));
}

// 2. Decayed, bias-corrected statistics -> per (token, group) affine
//    (scale = 1 / sqrt(v^ + eps), shift = -m^ scale).  One block per (b, g);
//    thread i owns tokens [i n, (i + 1) n).  Each thread scans its tokens
//    from zero, the per-thread end values are combined by a block-wide
//    scan of the affine maps z -> beta^n z + e (Hillis-Steele in shared
//    memory), and each thread rescans its tokens from its carry-in.
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) tdnorm_scan_kernel(const float2* __restrict__ st,
                                                                   float2* __restrict__ aff, int64_t L, int G,
                                                                   float beta1, float beta2, float eps) {
  __shared__ float2 s_e[kScanThreads];     // (m, v) end values, then inclusive prefixes
  __shared__ float2 s_a[kScanThreads];     // (beta1^len, beta2^len) of the combined span
  const int b = blockIdx.x / G, g = blockIdx.x % G;
  const int tid = threadIdx.x;
  const int64_t n = (L + kScanThreads - 1) / kScanThreads;
  const int64_t t0 = (int64_t)tid * n < L ? (int64_t)tid * n : L, t1 = t0 + n < L ? t0 + n : L;
  const float2* sp = st + ((int64_t)b * L) * G + g;
  float m = 0.f, v = 0.f;
  for (int64_t t = t0; t < t1; t += 8) {
    float2 mv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) mv[u] = t + u < t1 ? sp[(t + u) * G] : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (t + u < t1) {
        m = fmaf(beta1, m, (1.f - beta1) * mv[u].x);
        v = fmaf(beta2, v, (1.f - beta2) * mv[u].y);
      }
  }
  const int len = (int)(t1 - t0);
  s_e[tid] = make_float2(m, v);
  s_a[tid] = make_float2(powf(beta1, (float)len), powf(beta2, (float)len));
  __syncthreads();
  // inclusive scan of the maps: combine (a_prev, e_prev) then (a, e) -> (a a_prev, a e_prev + e)
  for (int off = 1; off < kScanThreads; off <<= 1) {
    float2 e = s_e[tid], a = s_a[tid];
    if (tid >= off) {
      const float2 ep = s_e[tid - off], ap = s_a[tid - off];
      e = make_float2(fmaf(a.x, ep.x, e.x), fmaf(a.y, ep.y, e.y));
      a = make_float2(a.x * ap.x, a.y * ap.y);
    }
    __syncthreads();
    s_e[tid] = e;
    s_a[tid] = a;
    __syncthreads();
  }
  // carry-in = inclusive prefix of the previous thread
  m = tid > 0 ? s_e[tid - 1].x : 0.f;
  v = tid > 0 ? s_e[tid - 1].y : 0.f;
  // beta^(t+1) as a running fp64 product from the thread's first token, so
  // 1 - beta^(t+1) keeps its digits for small t (beta = 0 gives 1)
  double p1 = pow((double)beta1, (double)(t0 + 1)), p2 = pow((double)beta2, (double)(t0 + 1));
  float2* ap = aff + ((int64_t)b * L) * G + g;
  for (int64_t t = t0; t < t1; t += 8) {
    float2 mv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) mv[u] = t + u < t1 ? sp[(t + u) * G] : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (t + u < t1) {
        m = fmaf(beta1, m, (1.f - beta1) * mv[u].x);
        v = fmaf(beta2, v, (1.f - beta2) * mv[u].y);
        const float c1 = (float)(1.0 - p1), c2 = (float)(1.0 - p2);
        p1 *= beta1;
        p2 *= beta2;
        const float scale = rsqrtf(v / c2 + eps);
        ap[(t + u) * G] = make_float2(scale, -(m / c1) * scale);
      }
  }
}

// 3. y = (x scale + shift) gamma + bias, 8 features (16 bytes) per thread.
template <typename TIn>
__global__ void __launch_bounds__(256) tdnorm_apply_kernel(const TIn* __restrict__ x, TIn* __restrict__ y,
                                                           const float2* __restrict__ aff,
                                                           const float* __restrict__ gamma,
                                                           const float* __restrict__ bias, int64_t rows, int64_t D,
                                                           int G) {
  const int64_t vpr = D / 8;   // vectors per row
  const int gs = (int)(D / G);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * vpr;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / vpr;
    const int f0 = (int)(i % vpr) * 8;
    const float2 a = aff[row * G + f0 / gs];
    float v[8];
    load8(x + row * D + f0, v);
    const float4 g0 = reinterpret_cast<const float4*>(gamma + f0)[0], g1 = reinterpret_cast<const float4*>(gamma + f0)[1];
    const float4 b0 = reinterpret_cast<const float4*>(bias + f0)[0], b1 = reinterpret_cast<const float4*>(bias + f0)[1];
    const float gm[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    const float bs[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = fmaf(fmaf(v[e], a.x, a.y), gm[e], bs[e]);
    store8(y + row * D + f0, v);
  }
}

template <typename TIn>
cudaError_t tdnorm_impl(const NormProblem& p, const NormWorkspace& w, cudaStream_t st) {
  const int64_t rows = p.B * p.L;
  const int64_t pairs = rows * p.G;
  tdnorm_stats_kernel<TIn><<<(unsigned)((pairs + 255) / 256), 256, 0, st>>>(static_cast<const TIn*>(p.x), w.stats,
                                                                              rows, p.D, (int)p.G);
  tdnorm_scan_kernel<<<(unsigned)(p.B * p.G), kScanThreads, 0, st>>>(w.stats, w.affine, p.L, (int)p.G, p.beta1,
                                                                      p.beta2, p.eps);
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  const int64_t vecs = rows * (p.D / 8);
  const int64_t want = (vecs + 255) / 256;
  const unsigned blocks = (unsigned)std::min<int64_t>(want, (int64_t)sms * 8);
  tdnorm_apply_kernel<TIn><<<blocks, 256, 0, st>>>(static_cast<const TIn*>(p.x), static_cast<TIn*>(p.y), w.affine,
                                                    p.gamma, p.bias, rows, p.D, (int)p.G);
  return cudaGetLastError();
}

}  // namespace

size_t tdnorm_workspace_bytes(int64_t B, int64_t L, int64_t G) { return (size_t)(2 * B * L * G) * sizeof(float2); }

NormWorkspace carve_tdnorm_workspace(void* base, int64_t B, int64_t L, int64_t G) {
  NormWorkspace w;
  w.stats = static_cast<float2*>(base);
  w.affine = w.stats + B * L * G;
  return w;
}

cudaError_t launch_tdnorm(const NormProblem& p, const NormWorkspace& w, cudaStream_t st) {
  return p.dtype == kBF16 ? tdnorm_impl<__nv_bfloat16>(p, w, st) : tdnorm_impl<float>(p, w, st);
}

}  // namespace gecko
