// Context parallelism for one long sequence split into P consecutive
// segments (one per rank).  The AWM carry of the Gecko digest
// (paper.rainbus.top, method step details, step 4) is affine in the state:
//     M'_{s+1} = A_s M'_s + b_s,   A_s = diag(r_s) - diag(rho_s) C~_s,
//                                  b_s = rho_s (.) B~_s,
// once log z is known (r_s, rho_s depend on it).  log z itself is a prefix
// of per-chunk exp-sums.  So a rank needs from the ranks before it only
//   (1) the log-exp-sum of all their tokens (its log z offset), and
//   (2) their composed segment maps, which turn M'_in of a segment into its
//       last two states;
// and SCA needs the previous segment's last chunk of K and V.  The kernels
// here compose what the ranks exchanged; the segment maps come from the
// forward's own stats, chunk and carry kernels (gecko_api.cu).
#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

// dst[bh] = I (D x D) for every (b, h); stride in floats between (b, h).
__global__ void set_identity_kernel(float* __restrict__ dst, int64_t stride, int D, int64_t BH) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= BH * D * D) return;
  const int64_t bh = i / ((int64_t)D * D);
  const int e = (int)(i % ((int64_t)D * D));
  dst[bh * stride + e] = (e / D == e % D) ? 1.f : 0.f;
}

// log z at the start of segment `rank`: logsumexp over the segments before
// it of their log-exp-sums (fp64); -inf for the first segment.  lsum is
// [P, BH, D]; out is written with stride `sd` per (b, h).  grid BH, D threads.
__global__ void cp_logz_kernel(const float* __restrict__ lsum, float* __restrict__ out, int rank, int64_t BH,
                               int D, int64_t sd) {
  const int64_t bh = blockIdx.x;
  const int f = threadIdx.x;
  if (f >= D) return;
  double L = -INFINITY;
  for (int j = 0; j < rank; ++j) {
    const double e = lsum[((int64_t)j * BH + bh) * D + f];
    const double hi = fmax(L, e), lo = fmin(L, e);
    L = hi == -INFINITY ? -INFINITY : hi + log1p(exp(lo - hi));
  }
  out[bh * sd + f] = (float)L;
}

// Composition of the segment maps of the ranks before `rank`, one slice of
// JC columns per CTA (columns are independent):
//   M_0 = 0,  M_{j+1} = A_j M_j + b_j          -> M'_in of segment `rank`
//   M'_prev = A'_{rank-1} M_{rank-1} + b'_{rank-1}  (the state before the
//             previous segment's last chunk)
// maps is [P, BH, 4, D, D]: A, b, A', b'.  Writes M'_prev and M'_in of each
// (b, h) at out[bh * sd] and out[bh * sd + D*D].  grid (D/JC, BH), 256 threads.
template <int D, int JC>
__global__ void __launch_bounds__(256) cp_compose_kernel(const float* __restrict__ maps, float* __restrict__ out,
                                                         int rank, int64_t BH, int64_t sd) {
  constexpr int PER = D * JC / 256;
  static_assert(256 / (JC / PER) == D, "thread layout");
  constexpr int LD = D + 4;
  extern __shared__ float smem_cp[];
  float* As = smem_cp;       // [D][LD]
  float* Ms = As + D * LD;   // [D][JC]
  const int64_t bh = blockIdx.y;
  const int j0 = blockIdx.x * JC;
  const int tid = threadIdx.x;
  const int f = tid / (JC / PER);
  const int jj = (tid % (JC / PER)) * PER;
  const int64_t mat = (int64_t)D * D;
  for (int i = tid; i < D * JC; i += 256) Ms[i] = 0.f;
  // one step: acc = X M + y for the matrix pair (X, y) at map index `which`
  auto step = [&](int j, int which, float (&acc)[PER]) {
    const float* X = maps + (((int64_t)j * BH + bh) * 4 + which) * mat;
    const float* y = X + mat;
    __syncthreads();
    for (int i = tid; i < D * D / 4; i += 256) {
      const int row = (i * 4) / D, col = (i * 4) % D;
      *reinterpret_cast<float4*>(As + row * LD + col) = reinterpret_cast<const float4*>(X)[i];
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < PER; ++q) acc[q] = y[f * D + j0 + jj + q];
#pragma unroll 4
    for (int g = 0; g < D; ++g) {
      const float a = As[f * LD + g];
#pragma unroll
      for (int q = 0; q < PER; ++q) acc[q] = fmaf(a, Ms[g * JC + jj + q], acc[q]);
    }
  };
  for (int j = 0; j < rank; ++j) {
    float acc[PER];
    if (j == rank - 1) {
      step(j, 2, acc);   // A', b': the state entering segment j's last chunk
#pragma unroll
      for (int q = 0; q < PER; ++q) out[bh * sd + f * D + j0 + jj + q] = acc[q];
    }
    step(j, 0, acc);     // A, b: the state after segment j
    __syncthreads();
#pragma unroll
    for (int q = 0; q < PER; ++q) Ms[f * JC + jj + q] = acc[q];
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    out[bh * sd + mat + f * D + j0 + jj + q] = Ms[f * JC + jj + q];
    if (rank == 0) out[bh * sd + f * D + j0 + jj + q] = 0.f;
  }
}

template <int D>
cudaError_t compose_impl(const float* maps, float* out, int rank, int64_t BH, int64_t sd, cudaStream_t st) {
  constexpr int JC = 16;
  const size_t smem = sizeof(float) * (D * (D + 4) + D * JC);
  cudaError_t e = cudaFuncSetAttribute(cp_compose_kernel<D, JC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  cp_compose_kernel<D, JC><<<dim3(D / JC, (unsigned)BH), 256, smem, st>>>(maps, out, rank, BH, sd);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_set_identity(float* dst, int64_t stride, int d, int64_t BH, cudaStream_t st) {
  const int64_t n = BH * d * d;
  set_identity_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(dst, stride, d, BH);
  return cudaGetLastError();
}

cudaError_t launch_cp_logz(const float* lsum, float* out, int rank, int64_t BH, int d, int64_t sd, cudaStream_t st) {
  cp_logz_kernel<<<(unsigned)BH, d, 0, st>>>(lsum, out, rank, BH, d, sd);
  return cudaGetLastError();
}

cudaError_t launch_cp_compose(const float* maps, float* out, int rank, int64_t BH, int d, int64_t sd,
                              cudaStream_t st) {
  return d == 64 ? compose_impl<64>(maps, out, rank, BH, sd, st) : compose_impl<128>(maps, out, rank, BH, sd, st);
}

}  // namespace gecko
