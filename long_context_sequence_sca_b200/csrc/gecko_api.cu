// C-ABI host side of the Gecko forward: argument validation, the per-device
// workspace, the launch sequence and the state export.  See include/gecko.h
// for the contract of each entry point.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <array>
#include <atomic>
#include <map>
#include <vector>
#include <mutex>
#include <string>

#include "../../include/gecko.h"
#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {

// The device status word (bit kStatusTimeout: a bounded wait ran out).
__device__ int g_status_word;

// Fixed working memory of gecko_sca_awm_forward_noalloc.  In host code this
// name is only a stand-in: its device address comes from
// cudaGetSymbolAddress, resolved once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GECKO_NOALLOC_SCRATCH_BYTES];

size_t workspace_bytes(int64_t BH, int64_t T, int64_t c, int64_t d) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int64_t S = T / c;
  const size_t part = al(sizeof(float) * 2 * BH * (T / stats_block_rows(c)) * d);
  const size_t vec = al(sizeof(float) * BH * S * d);
  const size_t mat = al(sizeof(float) * BH * S * d * d);
  const size_t mst = al(sizeof(float) * BH * (S + 1) * d * d);
  const size_t img = al(sizeof(uint16_t) * BH * (S + 1) * d * d);
  const size_t cimg = al(sizeof(uint16_t) * BH * S * d * d);
  const size_t flags = al(sizeof(int) * BH * S);
  return part + 4 * vec + 2 * mat + mst + img + cimg + flags;
}

Workspace carve_workspace(void* base, int64_t BH, int64_t T, int64_t c, int64_t d) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  char* p = static_cast<char*>(base);
  Workspace w;
  const int64_t S = T / c;
  const size_t part = al(sizeof(float) * 2 * BH * (T / stats_block_rows(c)) * d);
  const size_t vec = al(sizeof(float) * BH * S * d);
  const size_t mat = al(sizeof(float) * BH * S * d * d);
  w.part = reinterpret_cast<float2*>(p);
  p += part;
  w.lse = reinterpret_cast<float*>(p);
  p += vec;
  w.logz = reinterpret_cast<float*>(p);
  p += vec;
  w.ratio = reinterpret_cast<float*>(p);
  p += vec;
  w.rho = reinterpret_cast<float*>(p);
  p += vec;
  w.Bm = reinterpret_cast<float*>(p);
  p += mat;
  w.Cm = reinterpret_cast<float*>(p);
  p += mat;
  w.Mst = reinterpret_cast<float*>(p);
  p += al(sizeof(float) * BH * (S + 1) * d * d);
  w.Mimg = reinterpret_cast<uint16_t*>(p);
  p += al(sizeof(uint16_t) * BH * (S + 1) * d * d);
  w.Cimg = reinterpret_cast<uint16_t*>(p);
  p += al(sizeof(uint16_t) * BH * S * d * d);
  w.flags = reinterpret_cast<int*>(p);
  return w;
}

namespace {

thread_local std::string t_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_err = buf;
  return code;
}

struct DeviceState {
  void* ws = nullptr;
  size_t ws_bytes = 0;
  int* status = nullptr;  // device address of g_status_word
  bool have_state = false;
  int64_t B = 0, H = 0, d = 0, S = 0, T = 0;
  void* noalloc_scratch = nullptr;  // device address of g_noalloc_scratch
  void* state = nullptr;             // copy of a carried state (continued sequences)
  size_t state_bytes = 0;
  void* cema_ws = nullptr;           // CEMA chunk states
  size_t cema_ws_bytes = 0;
  void* norm_ws = nullptr;           // timestep-norm group statistics
  size_t norm_ws_bytes = 0;
  void* bwd_ws = nullptr;            // backward workspace
  size_t bwd_ws_bytes = 0;
};

std::mutex g_mu;
std::map<int, DeviceState> g_dev;

bool env_is(const char* name, const char* val) {
  const char* e = std::getenv(name);
  return e && std::strcmp(e, val) == 0;
}

int check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return GECKO_OK;
  return fail(GECKO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Per-device set-up: resolve the status word's device address.
int device_state(int dev, DeviceState** out) {
  DeviceState& ds = g_dev[dev];
  if (!ds.status) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return check_cuda(e, "cudaGetSymbolAddress(status word)");
    ds.status = static_cast<int*>(p);
  }
  *out = &ds;
  return GECKO_OK;
}

constexpr int64_t kMaxGridYZ = 65535;

int validate(const void* const* ptrs, int n, int64_t B, int64_t H, int64_t T, int64_t c, int64_t d, int dtype) {
  for (int i = 0; i < n; ++i)
    if (!ptrs[i]) return fail(GECKO_ERR_ARG, "tensor argument %d is NULL", i);
  if (dtype != GECKO_F32 && dtype != GECKO_BF16) return fail(GECKO_ERR_ARG, "unknown dtype %d", dtype);
  if (B < 1 || H < 1 || T < 1 || c < 1 || d < 1)
    return fail(GECKO_ERR_ARG, "sizes must be >= 1 (B=%lld H=%lld T=%lld c=%lld d=%lld)", (long long)B,
                (long long)H, (long long)T, (long long)c, (long long)d);
  if (d != 64 && d != 128) return fail(GECKO_ERR_SHAPE, "d must be 64 or 128 (got %lld)", (long long)d);
  if (c % 64 != 0) return fail(GECKO_ERR_SHAPE, "c must be a multiple of 64 (got %lld)", (long long)c);
  if (T % c != 0) return fail(GECKO_ERR_SHAPE, "T %% c != 0 (T=%lld c=%lld)", (long long)T, (long long)c);
  // element count and byte size must fit comfortably in int64; token
  // indices must fit the 32-bit ranges the kernels use, and (b, h) pairs and
  // chunks index grid dimensions y and z (at most 65535 each)
  const long double elems = (long double)B * H * T * d;
  if (elems * 4 > 4.0e18L) return fail(GECKO_ERR_SHAPE, "tensor size overflows");
  if (T > (int64_t(1) << 31) - 256) return fail(GECKO_ERR_SHAPE, "T exceeds the kernels' index range");
  if (B * H > kMaxGridYZ || T / c > kMaxGridYZ)
    return fail(GECKO_ERR_SHAPE, "B*H = %lld and T/c = %lld must each be at most %d", (long long)(B * H),
                (long long)(T / c), (int)kMaxGridYZ);
  for (int i = 0; i < n; ++i)
    if (reinterpret_cast<uintptr_t>(ptrs[i]) % 16 != 0)
      return fail(GECKO_ERR_ALIGN, "tensor argument %d is not 16-byte aligned", i);
  return GECKO_OK;
}

// Optional per-stage timing with CUDA events recorded on the caller's
// stream around each stage of a forward or backward; accumulated until read.
constexpr int kStages = 5;     // forward: awm stats, awm chunk, awm carry, awm readout, sca
constexpr int kBwdStages = 5;  // backward: awm rebuild, awm backward, sca delta, sca dK/dV, sca dQ
std::atomic<bool> g_timing{false};
std::mutex g_tmu;
std::vector<cudaEvent_t> g_event_pool;

template <int N>
struct StageLog {
  std::vector<std::array<cudaEvent_t, N + 1>> pending;
};
StageLog<kStages> g_fwd_log;
StageLog<kBwdStages> g_bwd_log;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

template <int N>
struct StageEventsT {
  cudaStream_t st;
  bool on;
  StageLog<N>& log;
  std::array<cudaEvent_t, N + 1> ev{};
  StageEventsT(cudaStream_t s, StageLog<N>& l) : st(s), on(g_timing.load()), log(l) {
    if (on) {
      std::lock_guard<std::mutex> lk(g_tmu);
      for (auto& e : ev) e = take_event();
    }
  }
  void mark(int i) {
    if (on) cudaEventRecord(ev[i], st);
  }
  void commit() {
    if (!on) return;
    std::lock_guard<std::mutex> lk(g_tmu);
    log.pending.push_back(ev);
    on = false;
  }
  ~StageEventsT() {
    if (!on) return;  // an error path: recycle the events
    std::lock_guard<std::mutex> lk(g_tmu);
    for (auto& e : ev) g_event_pool.push_back(e);
  }
};

struct StageEvents : StageEventsT<kStages> {
  explicit StageEvents(cudaStream_t s) : StageEventsT<kStages>(s, g_fwd_log) {}
};
struct BwdStageEvents : StageEventsT<kBwdStages> {
  explicit BwdStageEvents(cudaStream_t s) : StageEventsT<kBwdStages>(s, g_bwd_log) {}
};

// Sum of each stage's time over the logged calls; the log is emptied.
template <int N>
int read_stage_log(StageLog<N>& log, float* ms_per_stage, int capacity, int* n_calls) {
  if (!ms_per_stage || !n_calls || capacity < 1) return fail(GECKO_ERR_ARG, "bad timing buffers");
  std::lock_guard<std::mutex> lk(g_tmu);
  double acc[N] = {0};
  for (auto& evs : log.pending) {
    cudaError_t e = cudaEventSynchronize(evs[N]);
    if (e != cudaSuccess) return check_cuda(e, "event synchronize");
    for (int i = 0; i < N; ++i) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, evs[i], evs[i + 1]);
      acc[i] += ms;
    }
    for (auto& x : evs) g_event_pool.push_back(x);
  }
  *n_calls = (int)log.pending.size();
  log.pending.clear();
  for (int i = 0; i < N && i < capacity; ++i) ms_per_stage[i] = (float)acc[i];
  return GECKO_OK;
}

}  // namespace
}  // namespace gecko

using namespace gecko;

namespace gecko {
namespace {

// Grow a per-device buffer with stream-ordered allocation.
int ensure_buffer(void** buf, size_t* have, size_t need, cudaStream_t st, const char* what) {
  if (need <= *have) return GECKO_OK;
  if (*buf) {
    cudaFreeAsync(*buf, st);
    *buf = nullptr;
    *have = 0;
  }
  void* p = nullptr;
  cudaError_t e = cudaMallocAsync(&p, need, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(GECKO_ERR_ALLOC, "%s of %zu bytes: %s", what, need, cudaGetErrorString(e));
  }
  *buf = p;
  *have = need;
  return GECKO_OK;
}

// How a forward computes the AWM statistics and chunk products.
//   parts  CTAs per chunk.  The tensor-core chunk kernel runs two CTAs per SM
//          and one CTA's time is that of a whole chunk, so when the chunks
//          are too few to fill the GPU (small batches, context-parallel
//          segments of a few chunks) several CTAs share each chunk and add
//          their products together.  The count minimises
//          waves x (tiles per CTA + 2); it changes only if that saves a
//          quarter of the time.
//   fused  with one CTA per chunk, the chunk kernel computes each chunk's
//          log-sum-exp itself (read off its Cm block), which saves a
//          second pass over K_m; the prefix over chunks then runs after it.
//          Otherwise a statistics pass precedes the chunk products (several
//          CTAs per chunk need the chunk's lse before they start).
//          GECKO_FUSED_STATS=0 at build time keeps the separate pass.
#ifndef GECKO_FUSED_STATS
#define GECKO_FUSED_STATS 1
#endif
struct AwmPlan {
  bool fused;
  int parts;
};

AwmPlan awm_plan(const Problem& p, bool use_tc) {
  AwmPlan a{false, 1};
  if (use_tc) {
    const int64_t ctas = p.B * p.H * p.S, slots = 2 * (int64_t)sm_count(), n = p.c / 64;
    auto cost = [&](int64_t P) { return (ctas * P + slots - 1) / slots * (n + 2 * P); };   // x P
    int64_t best = 1;
    for (int64_t P = 2; P <= n / 4 && P <= 16; ++P)
      if (cost(P) * best < cost(best) * P) best = P;
    // cost(P) / P against cost(1): switch only for a saving of a quarter
    if (best > 1 && 4 * cost(best) <= 3 * cost(1) * best) a.parts = (int)best;
    // GECKO_CHUNK_PARTS=k forces k CTAs per chunk (tests cover both forms)
    if (const char* f = getenv("GECKO_CHUNK_PARTS")) {
      const long k = strtol(f, nullptr, 10);
      if (k >= 1 && k <= n) a.parts = (int)k;
    }
    a.fused = GECKO_FUSED_STATS && a.parts == 1;
  }
  return a;
}

// The statistics pass, when the plan has one.
int awm_stats_pass(const Problem& p, const Workspace& w, cudaStream_t st, const AwmPlan& a) {
  return a.fused ? GECKO_OK : check_cuda(launch_awm_stats(p, w, st), "awm stats");
}

// The chunk products (and, when fused, the statistics and the prefix).
int awm_chunks(const Problem& p, const Workspace& w, cudaStream_t st, bool use_tc, const AwmPlan& a) {
  int rc;
  if (a.fused) {
    if ((rc = check_cuda(launch_awm_chunk_tc_stats(p, w, st), "awm chunk"))) return rc;
    return check_cuda(launch_awm_prefix(p, w, st), "awm prefix");
  }
  return check_cuda(use_tc ? launch_awm_chunk_tc(p, w, st, a.parts) : launch_awm_chunk_simt(p, w, st), "awm chunk");
}

// The allocating forward, fresh (state_in == nullptr) or continuing a
// sequence (k, v with c prepended rows per (b, h); state_in on the device
// or host).  state_out, if given, receives (M'_S, M'_{S+1}, log z^S).
int run_forward(const void* q, const void* k, const void* v, const void* qm, const void* km, void* out_sca,
                void* out_mem, const float* state_in, float* state_out, int64_t B, int64_t H, int64_t T,
                int64_t c, int64_t d, int dtype, void* stream, float* lse = nullptr,
                void* out_sca_lo = nullptr) {
  const void* ptrs[7] = {q, k, v, qm, km, out_sca, out_mem};
  int rc = validate(ptrs, 7, B, H, T, c, d, dtype);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;

  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* ds = nullptr;
  if ((rc = device_state(dev, &ds))) return rc;

  const int64_t S = T / c;
  const int64_t BH = B * H;
  const int64_t sd = state_floats(d);
  if (env_is("GECKO_FAIL_ALLOC", "1")) return fail(GECKO_ERR_ALLOC, "workspace allocation failed (injected)");
  ds->have_state = false;  // set again once this forward is enqueued
  if ((rc = ensure_buffer(&ds->ws, &ds->ws_bytes, workspace_bytes(BH, T, c, d), st, "workspace"))) return rc;
  Workspace w = carve_workspace(ds->ws, BH, T, c, d);

  Problem p{q, k, v, qm, km, out_sca, out_mem, B, H, T, c, d, (int)S, dtype, ds->status};
  p.lse = lse;
  p.out_sca_lo = out_sca_lo;
  if (state_in) {
    // private copy, so state_out may alias state_in
    if ((rc = ensure_buffer(&ds->state, &ds->state_bytes, sizeof(float) * BH * sd, st, "state copy"))) return rc;
    if ((rc = check_cuda(cudaMemcpyAsync(ds->state, state_in, sizeof(float) * BH * sd, cudaMemcpyDefault, st),
                         "copy state in")))
      return rc;
    p.koff = c;
    p.state0 = static_cast<const float*>(ds->state);
  }
  // GECKO_KERNELS=simt selects the CUDA-core kernels for every dtype (a
  // second, independent GPU implementation used to cross-check the
  // tensor-core path).
  const bool force_simt = env_is("GECKO_KERNELS", "simt");
  const bool use_tc = !force_simt && tc_supported(p);

  cudaGetLastError();  // clear stale errors from the caller
  StageEvents ev(st);
  ev.mark(0);
  const AwmPlan plan = awm_plan(p, use_tc);
  if ((rc = awm_stats_pass(p, w, st, plan))) return rc;
  ev.mark(1);
  if ((rc = awm_chunks(p, w, st, use_tc, plan))) return rc;
  ev.mark(2);
  if ((rc = check_cuda(use_tc && d == 128 ? launch_awm_carry_tc(p, w, st, true) : launch_awm_carry(p, w, st, use_tc),
                       "awm carry")))
    return rc;
  ev.mark(3);
  if ((rc = check_cuda(use_tc ? launch_awm_readout_tc(p, w, st) : launch_awm_readout_simt(p, w, st),
                       "awm readout")))
    return rc;
  ev.mark(4);
  if ((rc = check_cuda(use_tc ? launch_sca_tc(p, st) : launch_sca_simt(p, st), "sca"))) return rc;
  ev.mark(5);
  ev.commit();
  if (state_out) {
    // (M'_S, M'_{S+1}, log z^S) of every (b, h): Mst[S-1], Mst[S], logz[S-1]
    const size_t mat = sizeof(float) * d * d, rec = sizeof(float) * sd;
    if ((rc = check_cuda(cudaMemcpy2DAsync(state_out, rec, w.Mst + (S - 1) * d * d, mat * (S + 1), 2 * mat, BH,
                                           cudaMemcpyDefault, st),
                         "copy state out (M)")))
      return rc;
    if ((rc = check_cuda(cudaMemcpy2DAsync(state_out + 2 * d * d, rec, w.logz + (S - 1) * d, sizeof(float) * d * S,
                                           sizeof(float) * d, BH, cudaMemcpyDefault, st),
                         "copy state out (log z)")))
      return rc;
  }
  ds->have_state = true;
  ds->B = B;
  ds->H = H;
  ds->d = d;
  ds->S = S;
  ds->T = T;
  return GECKO_OK;
}

// The backward: rematerialise the AWM chunk-boundary states with the
// forward kernels, then the AWM reverse pass, then the SCA gradients (whose
// dV kernel adds the AWM part of dV).
int run_backward(const void* q, const void* k, const void* v, const void* qm, const void* km, const void* out_sca,
                 const void* out_sca_lo, const float* lse, const void* dout_sca, const void* dout_mem, void* dq, void* dk, void* dv,
                 void* dqm, void* dkm, int64_t B, int64_t H, int64_t T, int64_t c, int64_t d, int dtype,
                 void* stream) {
  const void* ptrs[14] = {q, k, v, qm, km, out_sca, lse, dout_sca, dout_mem, dq, dk, dv, dqm, dkm};
  int rc = validate(ptrs, 14, B, H, T, c, d, dtype);
  if (rc) return rc;
  if (reinterpret_cast<uintptr_t>(out_sca_lo) % 16 != 0)
    return fail(GECKO_ERR_ALIGN, "out_sca_lo is not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;

  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* ds = nullptr;
  if ((rc = device_state(dev, &ds))) return rc;
  const int64_t S = T / c;
  const int64_t BH = B * H;
  ds->have_state = false;  // set again once the rebuild is enqueued
  if ((rc = ensure_buffer(&ds->ws, &ds->ws_bytes, workspace_bytes(BH, T, c, d), st, "workspace"))) return rc;
  if ((rc = ensure_buffer(&ds->bwd_ws, &ds->bwd_ws_bytes, bwd_workspace_bytes(BH, T, c, d), st,
                          "backward workspace")))
    return rc;
  Workspace w = carve_workspace(ds->ws, BH, T, c, d);
  BwdWorkspace bw = carve_bwd_workspace(ds->bwd_ws, BH, T, c, d);
  BwdProblem b{Problem{q, k, v, qm, km, nullptr, nullptr, B, H, T, c, d, (int)S, dtype, ds->status},
               out_sca, out_sca_lo, lse, dout_sca, dout_mem, dq, dk, dv, dqm, dkm};
  const Problem& p = b.f;

  const bool use_tc = !env_is("GECKO_KERNELS", "simt") && tc_supported(p);
  cudaGetLastError();
  BwdStageEvents ev(st);
  ev.mark(0);
  if ((rc = check_cuda(launch_awm_stats(p, w, st), "awm stats"))) return rc;
  // The chunk products are rebuilt to near fp32 (fp32 on the CUDA cores, or
  // bf16 hi + lo operands on the tensor cores): the rows of M' are close to
  // one another (each is a running average of V), and the softmax gradients
  // keep only their differences, which plain bf16 operands blur.
  if ((rc = check_cuda(use_tc ? launch_awm_chunk_tc_split(p, w, st) : launch_awm_chunk_simt(p, w, st),
                       "awm chunk")))
    return rc;
  if ((rc = check_cuda(launch_awm_carry(p, w, st), "awm carry"))) return rc;
  ev.mark(1);
  if ((rc = check_cuda(launch_awm_bwd(b, w, bw, st, use_tc), "awm backward"))) return rc;
  ev.mark(2);
  if ((rc = check_cuda(launch_sca_bwd_delta(b, bw, st), "sca backward delta"))) return rc;
  ev.mark(3);
  for (int part = 0; part < 2; ++part) {   // dK/dV (with the AWM part of dV), then dQ
    if ((rc = check_cuda(use_tc ? launch_sca_bwd_tc(b, bw, st, part) : launch_sca_bwd_simt(b, bw, st, part),
                         "sca backward")))
      return rc;
    ev.mark(4 + part);
  }
  ev.commit();
  ds->have_state = true;  // the rematerialised states are this sequence's
  ds->B = B;
  ds->H = H;
  ds->d = d;
  ds->S = S;
  ds->T = T;
  return GECKO_OK;
}

}  // namespace
}  // namespace gecko

extern "C" int gecko_sca_awm_forward_train(const void* q, const void* k, const void* v, const void* qm,
                                           const void* km, void* out_sca, void* out_mem, float* lse,
                                           void* out_sca_lo, int64_t B, int64_t H, int64_t T, int64_t c, int64_t d,
                                           int dtype, void* stream) {
  if (!lse) return fail(GECKO_ERR_ARG, "lse is NULL");
  if (reinterpret_cast<uintptr_t>(lse) % 16 != 0) return fail(GECKO_ERR_ALIGN, "lse is not 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(out_sca_lo) % 16 != 0)
    return fail(GECKO_ERR_ALIGN, "out_sca_lo is not 16-byte aligned");
  return run_forward(q, k, v, qm, km, out_sca, out_mem, nullptr, nullptr, B, H, T, c, d, dtype, stream, lse,
                     out_sca_lo);
}

extern "C" int gecko_sca_awm_backward(const void* q, const void* k, const void* v, const void* qm, const void* km,
                                      const void* out_sca, const void* out_sca_lo, const float* lse,
                                      const void* dout_sca, const void* dout_mem, void* dq, void* dk, void* dv,
                                      void* dqm, void* dkm, int64_t B, int64_t H, int64_t T, int64_t c, int64_t d,
                                      int dtype, void* stream) {
  return run_backward(q, k, v, qm, km, out_sca, out_sca_lo, lse, dout_sca, dout_mem, dq, dk, dv, dqm, dkm, B, H, T,
                      c, d, dtype, stream);
}

// ----------------------------------------------------- context parallelism

extern "C" int gecko_awm_segment_logsum(const void* km, float* lsum_out, int64_t B, int64_t H, int64_t T, int64_t c,
                                        int64_t d, int dtype, void* stream) {
  const void* ptrs[2] = {km, lsum_out};
  int rc = validate(ptrs, 2, B, H, T, c, d, dtype);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* ds = nullptr;
  if ((rc = device_state(dev, &ds))) return rc;
  const int64_t S = T / c, BH = B * H;
  ds->have_state = false;  // the forward's workspace is overwritten below
  if ((rc = ensure_buffer(&ds->ws, &ds->ws_bytes, workspace_bytes(BH, T, c, d), st, "workspace"))) return rc;
  Workspace w = carve_workspace(ds->ws, BH, T, c, d);
  Problem p{nullptr, nullptr, nullptr, nullptr, km, nullptr, nullptr, B, H, T, c, d, (int)S, dtype, ds->status};
  cudaGetLastError();
  if ((rc = check_cuda(launch_awm_stats(p, w, st), "awm stats"))) return rc;
  // log z^S of the segment started from zero = the log-sum of all its tokens
  return check_cuda(cudaMemcpy2DAsync(lsum_out, sizeof(float) * d, w.logz + (S - 1) * d, sizeof(float) * d * S,
                                      sizeof(float) * d, BH, cudaMemcpyDeviceToDevice, st),
                    "copy log-sum");
}

extern "C" int gecko_awm_segment_maps(const void* km, const void* v, const float* logz_in, float* maps_out,
                                      int64_t B, int64_t H, int64_t T, int64_t c, int64_t d, int dtype,
                                      void* stream) {
  const void* ptrs[4] = {km, v, logz_in, maps_out};
  int rc = validate(ptrs, 4, B, H, T, c, d, dtype);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* ds = nullptr;
  if ((rc = device_state(dev, &ds))) return rc;
  const int64_t S = T / c, BH = B * H, sd = state_floats(d), mat = d * d;
  ds->have_state = false;  // the forward's workspace is overwritten below
  if ((rc = ensure_buffer(&ds->ws, &ds->ws_bytes, workspace_bytes(BH, T, c, d), st, "workspace"))) return rc;
  if ((rc = ensure_buffer(&ds->state, &ds->state_bytes, sizeof(float) * BH * sd, st, "state"))) return rc;
  Workspace w = carve_workspace(ds->ws, BH, T, c, d);
  float* state = static_cast<float*>(ds->state);
  Problem p{nullptr, nullptr, v, nullptr, km, nullptr, nullptr, B, H, T, c, d, (int)S, dtype, ds->status};
  p.state0 = state;   // log z seed and the carry's starting state; no prepended K/V rows (koff = 0)
  const bool use_tc = !env_is("GECKO_KERNELS", "simt") && tc_supported(p);
  cudaGetLastError();
  if ((rc = check_cuda(cudaMemsetAsync(state, 0, sizeof(float) * BH * sd, st), "clear state"))) return rc;
  if ((rc = check_cuda(cudaMemcpy2DAsync(state + 2 * mat, sizeof(float) * sd, logz_in, sizeof(float) * d,
                                         sizeof(float) * d, BH, cudaMemcpyDeviceToDevice, st),
                       "seed log z")))
    return rc;
  const AwmPlan plan = awm_plan(p, use_tc);
  if ((rc = awm_stats_pass(p, w, st, plan))) return rc;
  if ((rc = awm_chunks(p, w, st, use_tc, plan))) return rc;
  // the tensor-core carry at d = 128 (its C operand image comes from the chunk products)
  auto carry = [&]() {
    return check_cuda(use_tc && d == 128 ? launch_awm_carry_tc(p, w, st, false) : launch_awm_carry(p, w, st),
                      "awm carry");
  };
  // maps_out[bh] = (A, b, A', b'): the carry from M'_in = 0 gives b (after the
  // last chunk) and b' (before it); with the chunk terms zeroed and M'_in = I
  // it gives A and A'.
  auto take = [&](int slot_last, int slot_prev) -> int {
    const size_t m4 = sizeof(float) * mat;
    int r = check_cuda(cudaMemcpy2DAsync(maps_out + slot_last * mat, 4 * m4, w.Mst + S * mat, (S + 1) * m4, m4, BH,
                                         cudaMemcpyDeviceToDevice, st),
                       "copy map");
    if (r) return r;
    return check_cuda(cudaMemcpy2DAsync(maps_out + slot_prev * mat, 4 * m4, w.Mst + (S - 1) * mat, (S + 1) * m4,
                                        m4, BH, cudaMemcpyDeviceToDevice, st),
                      "copy map");
  };
  if ((rc = carry())) return rc;
  if ((rc = take(1, 3))) return rc;
  if ((rc = check_cuda(cudaMemsetAsync(w.Bm, 0, sizeof(float) * BH * S * mat, st), "clear chunk terms"))) return rc;
  if ((rc = check_cuda(launch_set_identity(state + mat, sd, (int)d, BH, st), "identity"))) return rc;
  if ((rc = carry())) return rc;
  return take(0, 2);
}

extern "C" int gecko_awm_cp_logz(const float* lsum_all, int P, int rank, float* logz_out, int64_t B, int64_t H,
                                 int64_t d, void* stream) {
  if (!lsum_all || !logz_out) return fail(GECKO_ERR_ARG, "NULL pointer");
  if (P < 1 || rank < 0 || rank >= P) return fail(GECKO_ERR_ARG, "rank %d of %d", rank, P);
  if (B < 1 || H < 1 || (d != 64 && d != 128)) return fail(GECKO_ERR_SHAPE, "bad B, H or d");
  if (B * H > kMaxGridYZ) return fail(GECKO_ERR_SHAPE, "B*H must be at most %d", (int)kMaxGridYZ);
  cudaGetLastError();
  return check_cuda(launch_cp_logz(lsum_all, logz_out, rank, B * H, (int)d, d, static_cast<cudaStream_t>(stream)),
                    "cp log z");
}

extern "C" int gecko_awm_cp_state(const float* lsum_all, const float* maps_all, int P, int rank, float* state_out,
                                  int64_t B, int64_t H, int64_t d, void* stream) {
  if (!lsum_all || !maps_all || !state_out) return fail(GECKO_ERR_ARG, "NULL pointer");
  if (P < 1 || rank < 0 || rank >= P) return fail(GECKO_ERR_ARG, "rank %d of %d", rank, P);
  if (B < 1 || H < 1 || (d != 64 && d != 128)) return fail(GECKO_ERR_SHAPE, "bad B, H or d");
  if (B * H > kMaxGridYZ) return fail(GECKO_ERR_SHAPE, "B*H must be at most %d", (int)kMaxGridYZ);
  if (reinterpret_cast<uintptr_t>(maps_all) % 16 != 0) return fail(GECKO_ERR_ALIGN, "maps not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t BH = B * H, sd = state_floats(d);
  cudaGetLastError();
  int rc;
  if ((rc = check_cuda(launch_cp_logz(lsum_all, state_out + 2 * d * d, rank, BH, (int)d, sd, st), "cp log z")))
    return rc;
  return check_cuda(launch_cp_compose(maps_all, state_out, rank, BH, (int)d, sd, st), "cp compose");
}

extern "C" int gecko_sca_awm_forward(const void* q, const void* k, const void* v, const void* qm, const void* km,
                                     void* out_sca, void* out_mem, int64_t B, int64_t H, int64_t T, int64_t c,
                                     int64_t d, int dtype, void* stream) {
  return run_forward(q, k, v, qm, km, out_sca, out_mem, nullptr, nullptr, B, H, T, c, d, dtype, stream);
}

extern "C" int gecko_sca_awm_forward_continue(const void* q, const void* k, const void* v, const void* qm,
                                              const void* km, void* out_sca, void* out_mem, const float* state_in,
                                              float* state_out, int64_t B, int64_t H, int64_t T, int64_t c,
                                              int64_t d, int dtype, void* stream) {
  return run_forward(q, k, v, qm, km, out_sca, out_mem, state_in, state_out, B, H, T, c, d, dtype, stream);
}

extern "C" int gecko_awm_state(float* M_out, float* logz_out, int64_t B, int64_t H, int64_t d, void* stream) {
  if (!M_out || !logz_out) return fail(GECKO_ERR_ARG, "NULL output pointer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0, rc;
  if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_dev.find(dev);
  if (it == g_dev.end() || !it->second.have_state || !it->second.ws)
    return fail(GECKO_ERR_NO_STATE, "no forward has run on device %d", dev);
  DeviceState& ds = it->second;
  if (B != ds.B || H != ds.H || d != ds.d)
    return fail(GECKO_ERR_ARG, "state is B=%lld H=%lld d=%lld, asked for B=%lld H=%lld d=%lld", (long long)ds.B,
                (long long)ds.H, (long long)ds.d, (long long)B, (long long)H, (long long)d);
  const int64_t BH = B * H, S = ds.S;
  Workspace w = carve_workspace(ds.ws, BH, ds.T, ds.T / ds.S, d);
  const size_t mat = sizeof(float) * d * d;
  // M'_{S+1} of each (b, h) sits at Mst[bh, S]; log z^S at logz[bh, S-1]
  if ((rc = check_cuda(cudaMemcpy2DAsync(M_out, mat, w.Mst + S * d * d, mat * (S + 1), mat, BH,
                                         cudaMemcpyDefault, st),
                       "copy M")))
    return rc;
  if ((rc = check_cuda(cudaMemcpy2DAsync(logz_out, sizeof(float) * d, w.logz + (S - 1) * d,
                                         sizeof(float) * d * S, sizeof(float) * d, BH, cudaMemcpyDefault, st),
                       "copy log z")))
    return rc;
  if ((rc = check_cuda(cudaStreamSynchronize(st), "synchronize"))) return rc;
  int word = 0;
  if ((rc = check_cuda(cudaMemcpy(&word, ds.status, sizeof(int), cudaMemcpyDeviceToHost), "read status")))
    return rc;
  if (word & kStatusTimeout) return fail(GECKO_ERR_TIMEOUT, "a kernel of the last forward timed out on a wait");
  return GECKO_OK;
}

extern "C" int gecko_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0, rc;
  if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* ds = nullptr;
  if ((rc = device_state(dev, &ds))) return rc;
  if ((rc = check_cuda(cudaStreamSynchronize(st), "synchronize"))) return rc;
  int word = 0;
  if ((rc = check_cuda(cudaMemcpy(&word, ds->status, sizeof(int), cudaMemcpyDeviceToHost), "read status")))
    return rc;
  const int zero = 0;
  if ((rc = check_cuda(cudaMemcpy(ds->status, &zero, sizeof(int), cudaMemcpyHostToDevice), "clear status")))
    return rc;
  if (word & kStatusTimeout) return fail(GECKO_ERR_TIMEOUT, "a kernel gave up on a bounded wait");
  return GECKO_OK;
}

extern "C" const char* gecko_last_error(void) { return t_err.c_str(); }

extern "C" void gecko_release(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto& kv : g_dev) {
    if (kv.second.ws || kv.second.state || kv.second.cema_ws || kv.second.norm_ws || kv.second.bwd_ws) {
      cudaSetDevice(kv.first);
      cudaDeviceSynchronize();
      if (kv.second.ws) cudaFree(kv.second.ws);
      if (kv.second.state) cudaFree(kv.second.state);
      if (kv.second.cema_ws) cudaFree(kv.second.cema_ws);
      if (kv.second.norm_ws) cudaFree(kv.second.norm_ws);
      if (kv.second.bwd_ws) cudaFree(kv.second.bwd_ws);
    }
    kv.second.ws = nullptr;
    kv.second.ws_bytes = 0;
    kv.second.state = nullptr;
    kv.second.state_bytes = 0;
    kv.second.cema_ws = nullptr;
    kv.second.cema_ws_bytes = 0;
    kv.second.norm_ws = nullptr;
    kv.second.norm_ws_bytes = 0;
    kv.second.bwd_ws = nullptr;
    kv.second.bwd_ws_bytes = 0;
    kv.second.have_state = false;
  }
  cudaSetDevice(cur);
}

extern "C" int gecko_timing_enable(int enable) {
  g_timing.store(enable != 0);
  return GECKO_OK;
}

extern "C" int gecko_timing_read(float* ms_per_stage, int capacity, int* n_calls) {
  return read_stage_log(g_fwd_log, ms_per_stage, capacity, n_calls);
}

extern "C" int gecko_timing_read_backward(float* ms_per_stage, int capacity, int* n_calls) {
  return read_stage_log(g_bwd_log, ms_per_stage, capacity, n_calls);
}

extern "C" int gecko_sca_awm_forward_noalloc(const void* q, const void* k, const void* v, const void* qm,
                                             const void* km, void* out_sca, void* out_mem, int64_t B, int64_t H,
                                             int64_t T, int64_t c, int64_t d, int dtype, void* stream) {
  const void* ptrs[7] = {q, k, v, qm, km, out_sca, out_mem};
  int rc = validate(ptrs, 7, B, H, T, c, d, dtype);
  if (rc) return rc;
  const int64_t S = T / c;
  const int64_t BH = B * H;
  const size_t need = workspace_bytes(BH, T, c, d);
  if (need > GECKO_NOALLOC_SCRATCH_BYTES)
    return fail(GECKO_ERR_LIMIT,
                "this problem needs %zu bytes of working memory; the no-allocation entry point has a fixed "
                "scratch of %llu bytes (use gecko_sca_awm_forward)",
                need, (unsigned long long)GECKO_NOALLOC_SCRATCH_BYTES);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;

  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* ds = nullptr;
  if ((rc = device_state(dev, &ds))) return rc;
  if (!ds->noalloc_scratch) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return check_cuda(e, "cudaGetSymbolAddress(no-allocation scratch)");
    ds->noalloc_scratch = p;
  }
  Workspace w = carve_workspace(ds->noalloc_scratch, BH, T, c, d);

  Problem p{q, k, v, qm, km, out_sca, out_mem, B, H, T, c, d, (int)S, dtype, ds->status};
  const bool use_tc = !env_is("GECKO_KERNELS", "simt") && tc_supported(p);
  cudaGetLastError();
  const AwmPlan plan = awm_plan(p, use_tc);
  if ((rc = awm_stats_pass(p, w, st, plan))) return rc;
  if ((rc = awm_chunks(p, w, st, use_tc, plan))) return rc;
  if ((rc = check_cuda(use_tc && d == 128 ? launch_awm_carry_tc(p, w, st, true) : launch_awm_carry(p, w, st, use_tc),
                       "awm carry")))
    return rc;
  if ((rc = check_cuda(use_tc ? launch_awm_readout_tc(p, w, st) : launch_awm_readout_simt(p, w, st),
                       "awm readout")))
    return rc;
  if ((rc = check_cuda(use_tc ? launch_sca_tc(p, st) : launch_sca_simt(p, st), "sca"))) return rc;
  return GECKO_OK;
}

extern "C" int gecko_cema_forward(const void* x, void* y, const float* alpha, const float* delta,
                                  const float* theta, const float* beta, const float* eta, const uint8_t* reset,
                                  const float* state_in, float* state_out, int64_t B, int64_t L, int64_t D,
                                  int64_t h, int dtype, void* stream) {
  const void* ptrs[7] = {x, y, alpha, delta, theta, beta, eta};
  for (int i = 0; i < 7; ++i)
    if (!ptrs[i]) return fail(GECKO_ERR_ARG, "tensor argument %d is NULL", i);
  if (dtype != GECKO_F32 && dtype != GECKO_BF16) return fail(GECKO_ERR_ARG, "unknown dtype %d", dtype);
  if (B < 1 || L < 1 || D < 1 || h < 1)
    return fail(GECKO_ERR_ARG, "sizes must be >= 1 (B=%lld L=%lld D=%lld h=%lld)", (long long)B, (long long)L,
                (long long)D, (long long)h);
  if (h != cema_hidden()) return fail(GECKO_ERR_SHAPE, "h must be %d (got %lld)", cema_hidden(), (long long)h);
  if ((long double)B * L * D * 4 > 4.0e18L) return fail(GECKO_ERR_SHAPE, "tensor size overflows");
  // grid: (ceil(D / 128), chunks, B) within CUDA's y and z limits
  if (cema_chunks(L) > 65535 || B > 65535 || D > (int64_t(1) << 30))
    return fail(GECKO_ERR_SHAPE, "size exceeds kernel index range (B <= 65535, L <= 65535 * 256)");
  const void* all[10] = {x, y, alpha, delta, theta, beta, eta, reset, state_in, state_out};
  for (int i = 0; i < 10; ++i)
    if (reinterpret_cast<uintptr_t>(all[i]) % 16 != 0)
      return fail(GECKO_ERR_ALIGN, "argument %d is not 16-byte aligned", i);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0, rc;
  if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* ds = nullptr;
  if ((rc = device_state(dev, &ds))) return rc;
  if ((rc = ensure_buffer(&ds->cema_ws, &ds->cema_ws_bytes, cema_workspace_bytes(B, L, D), st, "CEMA workspace")))
    return rc;
  CemaProblem p{x, y, alpha, delta, theta, beta, eta, reset, state_in, state_out, B, L, D, dtype, ds->status};
  return check_cuda(launch_cema(p, carve_cema_workspace(ds->cema_ws, B, L, D), st), "CEMA launch");
}

extern "C" int gecko_tdnorm_forward(const void* x, void* y, const float* gamma, const float* bias, int64_t B,
                                    int64_t L, int64_t D, int64_t G, float beta1, float beta2, float eps, int dtype,
                                    void* stream) {
  const void* ptrs[4] = {x, y, gamma, bias};
  for (int i = 0; i < 4; ++i) {
    if (!ptrs[i]) return fail(GECKO_ERR_ARG, "tensor argument %d is NULL", i);
    if (reinterpret_cast<uintptr_t>(ptrs[i]) % 16 != 0)
      return fail(GECKO_ERR_ALIGN, "tensor argument %d is not 16-byte aligned", i);
  }
  if (dtype != GECKO_F32 && dtype != GECKO_BF16) return fail(GECKO_ERR_ARG, "unknown dtype %d", dtype);
  if (B < 1 || L < 1 || D < 1 || G < 1)
    return fail(GECKO_ERR_ARG, "sizes must be >= 1 (B=%lld L=%lld D=%lld G=%lld)", (long long)B, (long long)L,
                (long long)D, (long long)G);
  if (!(beta1 >= 0.f && beta1 < 1.f && beta2 >= 0.f && beta2 < 1.f && eps >= 0.f))
    return fail(GECKO_ERR_ARG, "need 0 <= beta1, beta2 < 1 and eps >= 0");
  if (D % G != 0 || (D / G) % 8 != 0)
    return fail(GECKO_ERR_SHAPE, "D / G must be a whole multiple of 8 (D=%lld G=%lld)", (long long)D, (long long)G);
  if ((long double)B * L * D * 4 > 4.0e18L || B * G > (1 << 30))
    return fail(GECKO_ERR_SHAPE, "size exceeds kernel index range");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0, rc;
  if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* ds = nullptr;
  if ((rc = device_state(dev, &ds))) return rc;
  if ((rc = ensure_buffer(&ds->norm_ws, &ds->norm_ws_bytes, tdnorm_workspace_bytes(B, L, G), st,
                          "normalisation workspace")))
    return rc;
  NormProblem p{x, y, gamma, bias, B, L, D, G, beta1, beta2, eps, dtype};
  return check_cuda(launch_tdnorm(p, carve_tdnorm_workspace(ds->norm_ws, B, L, G), st), "normalisation launch");
}
