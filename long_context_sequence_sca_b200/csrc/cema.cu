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
#include <cstdlib>

#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

bool env_flag(const char* name) {
  const char* e = std::getenv(name);
  return e && e[0] == '1';
}

constexpr int kCemaH = 16;      // hidden dimensions per feature
constexpr int kCemaLC = 256;    // tokens per chunk
constexpr int kCemaThreads = 128;
#ifndef GECKO_CEMA_UNROLL
#define GECKO_CEMA_UNROLL 8
#endif
#ifndef GECKO_CEMA_MINB
#define GECKO_CEMA_MINB 1
#endif
#ifndef GECKO_CEMA_SPLIT
#define GECKO_CEMA_SPLIT 1
#endif
constexpr int kCemaUnroll = GECKO_CEMA_UNROLL;  // tokens per group; the next group's inputs are loaded ahead

static_assert(kCemaUnroll % 8 == 0 && kCemaLC % kCemaUnroll == 0, "token groups of 8k dividing the chunk");
// Threads per feature: each holds kCemaH / kCemaSplit hidden dimensions (as
// packed pairs (j, j + 1)); two per feature halve the registers per thread,
// doubling the warps resident per SM.
constexpr int kCemaSplit = GECKO_CEMA_SPLIT;
constexpr int kCemaFeat = kCemaThreads / kCemaSplit;   // features per block
constexpr int kCemaP = kCemaH / 2 / kCemaSplit;        // packed pairs per thread

// Per-feature constants as packed pairs over (j, j + 1): Re q, Im q, -Im q
// and alpha * beta.  The recurrence then runs on f32x2 FMAs, real parts of
// two hidden dimensions in one register pair and imaginary parts in another.
struct CemaCoef {
  uint64_t qr[kCemaP], qi[kCemaP], nqi[kCemaP], ab[kCemaP];
};

__device__ __forceinline__ void load_coef(CemaCoef& k, const float* alpha, const float* delta, const float* theta,
                                          const float* beta, int d, int j0) {
#pragma unroll
  for (int jp = 0; jp < kCemaP; ++jp) {
    float qr[2], qi[2], ab[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = j0 + 2 * jp + e;
      const float a = alpha[d * kCemaH + j], m = 1.f - a * delta[d * kCemaH + j];
      float s, c;
      sincosf(theta[d * kCemaH + j], &s, &c);
      qr[e] = m * c;
      qi[e] = m * s;
      ab[e] = a * beta[d * kCemaH + j];
    }
    k.qr[jp] = pack2(qr[0], qr[1]);
    k.qi[jp] = pack2(qi[0], qi[1]);
    k.nqi[jp] = pack2(-qi[0], -qi[1]);
    k.ab[jp] = pack2(ab[0], ab[1]);
  }
}

// Inputs of tokens s .. s + kCemaUnroll - 1 of the chunk (0 past its end).
template <typename TIn>
__device__ __forceinline__ void load_group(float (&v)[kCemaUnroll], const TIn* xp, int s, int n, int64_t D) {
#pragma unroll
  for (int u = 0; u < kCemaUnroll; ++u) v[u] = s + u < n ? to_f32(xp[(int64_t)(s + u) * D]) : 0.f;
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
__global__ void __launch_bounds__(kCemaThreads, GECKO_CEMA_MINB) cema_local_kernel(const TIn* __restrict__ x, const float* alpha,
                                                                  const float* delta, const float* theta,
                                                                  const float* beta, const uint8_t* reset,
                                                                  float2* __restrict__ Bc,
                                                                  uint8_t* __restrict__ chunk_reset, int64_t L,
                                                                  int64_t D) {
  __shared__ __align__(8) uint8_t rs[kCemaLC];
  const int64_t b = blockIdx.z, c = blockIdx.y;
  const int64_t d0 = (int64_t)blockIdx.x * kCemaFeat + threadIdx.x / kCemaSplit;
  const bool valid = d0 < D;          // a feature past D computes on feature D - 1 and stores nothing
  const int64_t d = valid ? d0 : D - 1;
  const int j0 = (int)(threadIdx.x % kCemaSplit) * (kCemaH / kCemaSplit);   // first hidden dimension of this thread
  const int64_t t0 = c * kCemaLC;
  const int n = (int)(L - t0 < kCemaLC ? L - t0 : kCemaLC);
  stage_resets(rs, reset, b, L, t0, n);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    int any = 0;
    for (int i = 0; i < n; ++i) any |= rs[i];
    chunk_reset[b * gridDim.y + c] = (uint8_t)any;
  }
  CemaCoef k;
  load_coef(k, alpha, delta, theta, beta, (int)d, j0);
  uint64_t gr[kCemaP], gi[kCemaP];
#pragma unroll
  for (int jp = 0; jp < kCemaP; ++jp) gr[jp] = gi[jp] = pack2(0.f, 0.f);
  const TIn* xp = x + (b * L + t0) * D + d;
  // inputs of the next group of kCemaUnroll tokens are loaded while the
  // current group is computed
  float xa[kCemaUnroll], xb[kCemaUnroll];
  load_group(xa, xp, 0, n, D);
  for (int s = 0; s < n; s += kCemaUnroll) {
    if (s + kCemaUnroll < n) load_group(xb, xp, s + kCemaUnroll, n, D);
    uint64_t rmask = 0;   // resets of this group
#pragma unroll
    for (int g = 0; g < kCemaUnroll / 8; ++g) rmask |= *reinterpret_cast<const uint64_t*>(rs + s + 8 * g);
#pragma unroll
    for (int u = 0; u < kCemaUnroll; ++u) {
      if (s + u >= n) break;
      if (rmask && rs[s + u]) {
#pragma unroll
        for (int jp = 0; jp < kCemaP; ++jp) gr[jp] = gi[jp] = pack2(0.f, 0.f);
      }
      const uint64_t x2 = pack2(xa[u], xa[u]);
#pragma unroll
      for (int jp = 0; jp < kCemaP; ++jp) {
        const uint64_t r = ffma2(k.qr[jp], gr[jp], ffma2(k.nqi[jp], gi[jp], x2));
        gi[jp] = ffma2(k.qr[jp], gi[jp], fmul2(k.qi[jp], gr[jp]));
        gr[jp] = r;
      }
    }
#pragma unroll
    for (int u = 0; u < kCemaUnroll; ++u) xa[u] = xb[u];
  }
  if (!valid) return;
  float4* out = reinterpret_cast<float4*>(Bc + ((b * gridDim.y + c) * D + d) * kCemaH + j0);
#pragma unroll
  for (int jp = 0; jp < kCemaP; ++jp) {
    float r0, r1, i0, i1;
    unpack2(fmul2(k.ab[jp], gr[jp]), r0, r1);
    unpack2(fmul2(k.ab[jp], gi[jp]), i0, i1);
    out[jp] = make_float4(r0, i0, r1, i1);
  }
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
__global__ void __launch_bounds__(kCemaThreads, GECKO_CEMA_MINB) cema_out_kernel(const TIn* __restrict__ x, const float* alpha,
                                                                const float* delta, const float* theta,
                                                                const float* beta, const float* eta,
                                                                const uint8_t* reset, const float2* __restrict__ Hin,
                                                                TIn* __restrict__ y, int64_t L, int64_t D) {
  __shared__ __align__(8) uint8_t rs[kCemaLC];
  const int64_t b = blockIdx.z, c = blockIdx.y;
  const int64_t d0 = (int64_t)blockIdx.x * kCemaFeat + threadIdx.x / kCemaSplit;
  const bool valid = d0 < D;          // a feature past D computes on feature D - 1 and stores nothing
  const int64_t d = valid ? d0 : D - 1;
  const int j0 = (int)(threadIdx.x % kCemaSplit) * (kCemaH / kCemaSplit);   // first hidden dimension of this thread
  const int64_t t0 = c * kCemaLC;
  const int n = (int)(L - t0 < kCemaLC ? L - t0 : kCemaLC);
  stage_resets(rs, reset, b, L, t0, n);
  CemaCoef k;
  load_coef(k, alpha, delta, theta, beta, (int)d, j0);
  uint64_t er[kCemaP], nei[kCemaP], hr[kCemaP], hi[kCemaP];
  const float4* hin = reinterpret_cast<const float4*>(Hin + ((b * gridDim.y + c) * D + d) * kCemaH + j0);
  const float4* et = reinterpret_cast<const float4*>(eta + ((int64_t)d * kCemaH + j0) * 2);
#pragma unroll
  for (int jp = 0; jp < kCemaP; ++jp) {
    const float4 v = hin[jp], e = et[jp];   // (re_j, im_j, re_j+1, im_j+1)
    hr[jp] = pack2(v.x, v.z);
    hi[jp] = pack2(v.y, v.w);
    er[jp] = pack2(e.x, e.z);
    nei[jp] = pack2(-e.y, -e.w);
  }
  const TIn* xp = x + (b * L + t0) * D + d;
  TIn* yp = y + (b * L + t0) * D + d;
  float xa[kCemaUnroll], xb[kCemaUnroll];
  load_group(xa, xp, 0, n, D);
  for (int s = 0; s < n; s += kCemaUnroll) {
    if (s + kCemaUnroll < n) load_group(xb, xp, s + kCemaUnroll, n, D);
    uint64_t rmask = 0;
#pragma unroll
    for (int g = 0; g < kCemaUnroll / 8; ++g) rmask |= *reinterpret_cast<const uint64_t*>(rs + s + 8 * g);
#pragma unroll
    for (int u = 0; u < kCemaUnroll; ++u) {
      if (s + u >= n) break;
      const float xv_u = xa[u];
      if (rmask && rs[s + u]) {
#pragma unroll
        for (int jp = 0; jp < kCemaP; ++jp) hr[jp] = hi[jp] = pack2(0.f, 0.f);
      }
      const uint64_t x2 = pack2(xv_u, xv_u);
      uint64_t acc[2] = {pack2(0.f, 0.f), pack2(0.f, 0.f)};
#pragma unroll
      for (int jp = 0; jp < kCemaP; ++jp) {
        const uint64_t r = ffma2(k.qr[jp], hr[jp], ffma2(k.nqi[jp], hi[jp], fmul2(k.ab[jp], x2)));
        hi[jp] = ffma2(k.qr[jp], hi[jp], fmul2(k.qi[jp], hr[jp]));
        hr[jp] = r;
        acc[jp & 1] = ffma2(er[jp], hr[jp], ffma2(nei[jp], hi[jp], acc[jp & 1]));
      }
      float a0, a1, a2, a3;
      unpack2(acc[0], a0, a1);
      unpack2(acc[1], a2, a3);
      float yv = (a0 + a1) + (a2 + a3);
      if (kCemaSplit == 2) yv += __shfl_xor_sync(0xffffffffu, yv, 1);   // the feature's other half
      if (valid && j0 == 0) yp[(int64_t)(s + u) * D] = from_f32<TIn>(yv);
    }
#pragma unroll
    for (int u = 0; u < kCemaUnroll; ++u) xa[u] = xb[u];
  }
}


#ifndef GECKO_CEMA_PACKED_PAIRS
#define GECKO_CEMA_PACKED_PAIRS 4
#endif
// Pairs (j, j + 1) updated with packed f32x2 FMAs; the others with scalar
// FMAs on the two halves (packed FMAs issue to one of the SM's two FP32 FMA
// pipes only, scalar ones to either, so a mix keeps both busy).
constexpr int kCemaPackedPairs = GECKO_CEMA_PACKED_PAIRS;

// h <- q h + p for a pair: (hr, hi) packed re/im of j, j + 1.
template <bool kPacked>
__device__ __forceinline__ void cstep(uint64_t& hr, uint64_t& hi, uint64_t qr, uint64_t qi, uint64_t nqi,
                                      uint64_t p) {
  if (kPacked) {
    const uint64_t r = ffma2(qr, hr, ffma2(nqi, hi, p));
    hi = ffma2(qr, hi, fmul2(qi, hr));
    hr = r;
  } else {
    float r0, r1, i0, i1, a0, a1, b0, b1, n0, n1, p0, p1;
    unpack2(hr, r0, r1);
    unpack2(hi, i0, i1);
    unpack2(qr, a0, a1);
    unpack2(qi, b0, b1);
    unpack2(nqi, n0, n1);
    unpack2(p, p0, p1);
    hr = pack2(fmaf(a0, r0, fmaf(n0, i0, p0)), fmaf(a1, r1, fmaf(n1, i1, p1)));
    hi = pack2(fmaf(a0, i0, b0 * r0), fmaf(a1, i1, b1 * r1));
  }
}

// acc += Re(eta h) for a pair: er, nei = Re eta, -Im eta.
template <bool kPacked>
__device__ __forceinline__ void cproj(uint64_t& acc, uint64_t er, uint64_t nei, uint64_t hr, uint64_t hi) {
  if (kPacked) {
    acc = ffma2(er, hr, ffma2(nei, hi, acc));
  } else {
    float c0, c1, e0, e1, f0, f1, r0, r1, i0, i1;
    unpack2(acc, c0, c1);
    unpack2(er, e0, e1);
    unpack2(nei, f0, f1);
    unpack2(hr, r0, r1);
    unpack2(hi, i0, i1);
    acc = pack2(fmaf(e0, r0, fmaf(f0, i0, c0)), fmaf(e1, r1, fmaf(f1, i1, c1)));
  }
}

// ---------------------------------------------------- TMA-staged (bf16) --
// With bf16 data and D % 8 == 0 the chunk of x a block scans (128 features
// x 256 tokens, 64 KB) is brought into shared memory by one TMA copy, so the
// scans read shared memory instead of issuing one strided 2-byte global load
// per token; the output kernel writes y over the same tile and stores it
// with one TMA store.  Tensor maps are 3D {D, L, B} so a chunk never crosses
// into another batch's rows (loads past L read zeros, stores past L are
// dropped).
constexpr int kTileBytes = kCemaLC * kCemaThreads * 2;   // 64 KB
constexpr int kTmaSmem = kTileBytes + 128 + 128;          // tile, mbarrier, alignment slack

__device__ __forceinline__ __nv_bfloat16* stage_tile(uint8_t* raw, uint64_t** bar) {
  uint8_t* t = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 127) & ~uintptr_t(127));
  *bar = reinterpret_cast<uint64_t*>(t + kTileBytes);
  return reinterpret_cast<__nv_bfloat16*>(t);
}

__global__ void __launch_bounds__(kCemaThreads) cema_local_tma_kernel(const __grid_constant__ CUtensorMap mx,
                                                                      const float* alpha, const float* delta,
                                                                      const float* theta, const float* beta,
                                                                      const uint8_t* reset, float2* __restrict__ Bc,
                                                                      uint8_t* __restrict__ chunk_reset, int64_t L,
                                                                      int64_t D, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint8_t rs[kCemaLC];
  __shared__ int abort_flag;
  uint64_t* bar;
  const __nv_bfloat16* tile = stage_tile(smem_raw, &bar);
  const int64_t b = blockIdx.z, c = blockIdx.y;
  const int f = threadIdx.x;
  const int64_t d0 = (int64_t)blockIdx.x * kCemaThreads + f;
  const bool valid = d0 < D;
  const int64_t d = valid ? d0 : D - 1;
  const int64_t t0 = c * kCemaLC;
  const int n = (int)(L - t0 < kCemaLC ? L - t0 : kCemaLC);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, kTileBytes);
    tma_load_3d(const_cast<__nv_bfloat16*>(tile), &mx, bar, (int)(blockIdx.x * kCemaThreads), (int)t0, (int)b);
  }
  stage_resets(rs, reset, b, L, t0, n);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    int any = 0;
    for (int i = 0; i < n; ++i) any |= rs[i];
    chunk_reset[b * gridDim.y + c] = (uint8_t)any;
  }
  CemaCoef k;
  load_coef(k, alpha, delta, theta, beta, (int)d, 0);
  if (!mbar_wait(bar, 0, &abort_flag, status)) {
    mbar_wait_drain(bar, 0);
    return;
  }
  uint64_t gr[kCemaP], gi[kCemaP];
#pragma unroll
  for (int jp = 0; jp < kCemaP; ++jp) gr[jp] = gi[jp] = pack2(0.f, 0.f);
  for (int s = 0; s < n; s += 8) {
    const uint64_t rmask = *reinterpret_cast<const uint64_t*>(rs + s);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (s + u >= n) break;
      if (rmask && rs[s + u]) {
#pragma unroll
        for (int jp = 0; jp < kCemaP; ++jp) gr[jp] = gi[jp] = pack2(0.f, 0.f);
      }
      const float xv = __bfloat162float(tile[(s + u) * kCemaThreads + f]);
      const uint64_t x2 = pack2(xv, xv);
#pragma unroll
      for (int jp = 0; jp < kCemaP; ++jp) {
        if (jp < kCemaPackedPairs)
          cstep<true>(gr[jp], gi[jp], k.qr[jp], k.qi[jp], k.nqi[jp], x2);
        else
          cstep<false>(gr[jp], gi[jp], k.qr[jp], k.qi[jp], k.nqi[jp], x2);
      }
    }
  }
  if (!valid) return;
  float4* out = reinterpret_cast<float4*>(Bc + ((b * gridDim.y + c) * D + d) * kCemaH);
#pragma unroll
  for (int jp = 0; jp < kCemaP; ++jp) {
    float r0, r1, i0, i1;
    unpack2(fmul2(k.ab[jp], gr[jp]), r0, r1);
    unpack2(fmul2(k.ab[jp], gi[jp]), i0, i1);
    out[jp] = make_float4(r0, i0, r1, i1);
  }
}

__global__ void __launch_bounds__(kCemaThreads) cema_out_tma_kernel(const __grid_constant__ CUtensorMap mx,
                                                                    const __grid_constant__ CUtensorMap my,
                                                                    const float* alpha, const float* delta,
                                                                    const float* theta, const float* beta,
                                                                    const float* eta, const uint8_t* reset,
                                                                    const float2* __restrict__ Hin, int64_t L,
                                                                    int64_t D, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint8_t rs[kCemaLC];
  __shared__ int abort_flag;
  uint64_t* bar;
  __nv_bfloat16* tile = stage_tile(smem_raw, &bar);
  const int64_t b = blockIdx.z, c = blockIdx.y;
  const int f = threadIdx.x;
  const int64_t d0 = (int64_t)blockIdx.x * kCemaThreads + f;
  const int64_t d = d0 < D ? d0 : D - 1;
  const int64_t t0 = c * kCemaLC;
  const int n = (int)(L - t0 < kCemaLC ? L - t0 : kCemaLC);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, kTileBytes);
    tma_load_3d(tile, &mx, bar, (int)(blockIdx.x * kCemaThreads), (int)t0, (int)b);
  }
  stage_resets(rs, reset, b, L, t0, n);
  CemaCoef k;
  load_coef(k, alpha, delta, theta, beta, (int)d, 0);
  uint64_t er[kCemaP], nei[kCemaP], hr[kCemaP], hi[kCemaP];
  const float4* hin = reinterpret_cast<const float4*>(Hin + ((b * gridDim.y + c) * D + d) * kCemaH);
  const float4* et = reinterpret_cast<const float4*>(eta + (int64_t)d * kCemaH * 2);
#pragma unroll
  for (int jp = 0; jp < kCemaP; ++jp) {
    const float4 v = hin[jp], e = et[jp];
    hr[jp] = pack2(v.x, v.z);
    hi[jp] = pack2(v.y, v.w);
    er[jp] = pack2(e.x, e.z);
    nei[jp] = pack2(-e.y, -e.w);
  }
  const bool ok = mbar_wait(bar, 0, &abort_flag, status);
  if (__syncthreads_or(!ok)) {
    mbar_wait_drain(bar, 0);
    return;
  }
  for (int s = 0; s < n; s += 8) {
    const uint64_t rmask = *reinterpret_cast<const uint64_t*>(rs + s);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (s + u >= n) break;
      if (rmask && rs[s + u]) {
#pragma unroll
        for (int jp = 0; jp < kCemaP; ++jp) hr[jp] = hi[jp] = pack2(0.f, 0.f);
      }
      __nv_bfloat16* xs = tile + (s + u) * kCemaThreads + f;
      const float xv = __bfloat162float(*xs);
      const uint64_t x2 = pack2(xv, xv);
      uint64_t acc[2] = {pack2(0.f, 0.f), pack2(0.f, 0.f)};
#pragma unroll
      for (int jp = 0; jp < kCemaP; ++jp) {
        if (jp < kCemaPackedPairs) {
          cstep<true>(hr[jp], hi[jp], k.qr[jp], k.qi[jp], k.nqi[jp], fmul2(k.ab[jp], x2));
          cproj<true>(acc[jp & 1], er[jp], nei[jp], hr[jp], hi[jp]);
        } else {
          float a0, a1;
          unpack2(k.ab[jp], a0, a1);
          cstep<false>(hr[jp], hi[jp], k.qr[jp], k.qi[jp], k.nqi[jp], pack2(a0 * xv, a1 * xv));
          cproj<false>(acc[jp & 1], er[jp], nei[jp], hr[jp], hi[jp]);
        }
      }
      float a0, a1, a2, a3;
      unpack2(acc[0], a0, a1);
      unpack2(acc[1], a2, a3);
      *xs = __float2bfloat16_rn((a0 + a1) + (a2 + a3));   // y over the consumed x
    }
  }
  // the tile now holds y: hand it to the TMA store (async proxy)
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) {
    tma_store_3d(&my, tile, (int)(blockIdx.x * kCemaThreads), (int)t0, (int)b);
    bulk_commit();
    bulk_wait_read_all();
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn cema_encode_fn() {
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

// x or y [B, L, D] bf16 as a 3D map {D, L, B}, box {128, 256, 1}.
bool cema_map(CUtensorMap* m, const void* base, const CemaProblem& p) {
  EncodeTiledFn fn = cema_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)p.D, (cuuint64_t)p.L, (cuuint64_t)p.B};
  cuuint64_t strides[2] = {(cuuint64_t)p.D * 2, (cuuint64_t)(p.L * p.D * 2)};
  cuuint32_t box[3] = {kCemaThreads, kCemaLC, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t cema_tma_impl(const CemaProblem& p, const CemaWorkspace& w, cudaStream_t st) {
  CUtensorMap mx, my;
  if (!cema_map(&mx, p.x, p) || !cema_map(&my, p.y, p)) return cudaErrorInvalidValue;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(cema_local_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTmaSmem)))
    return e;
  if ((e = cudaFuncSetAttribute(cema_out_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTmaSmem)))
    return e;
  const int C = (int)((p.L + kCemaLC - 1) / kCemaLC);
  const dim3 grid((unsigned)((p.D + kCemaThreads - 1) / kCemaThreads), (unsigned)C, (unsigned)p.B);
  cema_local_tma_kernel<<<grid, kCemaThreads, kTmaSmem, st>>>(mx, p.alpha, p.delta, p.theta, p.beta, p.reset, w.Bc,
                                                              w.chunk_reset, p.L, p.D, p.status);
  const int64_t nthr = p.B * p.D * kCemaH;
  cema_carry_kernel<<<(unsigned)((nthr + 255) / 256), 256, 0, st>>>(p.alpha, p.delta, p.theta, w.Bc, w.chunk_reset,
                                                                     w.Hin, p.state_in, p.state_out, p.B, p.L, p.D,
                                                                     C);
  cema_out_tma_kernel<<<grid, kCemaThreads, kTmaSmem, st>>>(mx, my, p.alpha, p.delta, p.theta, p.beta, p.eta,
                                                            p.reset, w.Hin, p.L, p.D, p.status);
  return cudaGetLastError();
}

template <typename TIn>
cudaError_t cema_impl(const CemaProblem& p, const CemaWorkspace& w, cudaStream_t st) {
  const int C = (int)((p.L + kCemaLC - 1) / kCemaLC);
  const dim3 grid((unsigned)((p.D + kCemaFeat - 1) / kCemaFeat), (unsigned)C, (unsigned)p.B);
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
  if (p.dtype != kBF16) return cema_impl<float>(p, w, st);
  // TMA needs 16-byte row strides (D % 8 == 0) and 32-bit coordinates
  if (p.D % 8 == 0 && p.L < (int64_t(1) << 31) && !env_flag("GECKO_CEMA_PLAIN")) return cema_tma_impl(p, w, st);
  return cema_impl<__nv_bfloat16>(p, w, st);
}

int cema_hidden() { return kCemaH; }

}  // namespace gecko
