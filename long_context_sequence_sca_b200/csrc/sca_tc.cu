// Sliding Chunk Attention forward on 5th-generation tensor cores (sm_100a).
//
// Computes, per (b, h) and chunk s of c tokens (Gecko digest,
// paper.rainbus.top, method step details, step 3; paperlayer.ai summary,
// section 3.2):
//     O_s = softmax(Q_s [K_{s-1}; K_s]^T) [V_{s-1}; V_s]
// with scale 1, a causal mask inside the current chunk, and no previous chunk
// for chunk 1.  Requires bf16, d in {64, 128}, c % 128 == 0.
//
// Design (one persistent CTA per SM, 384 threads in three warpgroups):
//   warp 0      TMA producer: Q tiles once per work unit; K and V tiles of
//               128 keys through rings of shared-memory stages, loads issued
//               in the order of the iterations that free their slots.
//   warps 1-2   MMA issuers, one thread each, one per query tile i (warp 1
//               also allocates TMEM): S_i = Q_i K_j^T (SS form) into TMEM,
//               O_i += P_i V_j with P_i read from TMEM (TS form).
//   warp 3      idle (it completes the first warpgroup, whose registers
//               setmaxnreg hands to the softmax warpgroups).
//   warps 4-7   softmax for query tile 0, warps 8-11 for query tile 1; one
//               thread per query row (TMEM lane quarter = warp % 4); online
//               max/sum in registers; P written back to TMEM as bf16 over the
//               S columns; epilogue O / l.
// A work unit is two adjacent 128-row query tiles of one (b, h); CTAs claim
// units from a global counter in the schedule's order (decode_unit).  The
// two issuers alternate by turns (PV(0), QK(0) then PV(1), QK(1) for each
// key tile) so each softmax warpgroup's exp work overlaps the other tile's
// MMAs.  Only the
// diagonal key tile of each query tile is masked; key tiles entirely above
// the diagonal or before the previous chunk are never loaded.
//
// The running max is updated lazily: O and l are rescaled only when a new
// tile's row max exceeds the reference by more than 8 (log2 units), which
// keeps every exponent <= 2^8 and leaves the final O / l unchanged.
//
// Every wait is bounded (see mbar_wait); on a timeout the CTA drains its
// in-flight copies and MMAs, frees TMEM and returns with the status word set.
#include <cstdio>

#include "common.cuh"
#include "gecko_internal.h"

namespace gecko {
namespace {

constexpr int kBM = 128;   // query rows per tile
constexpr int kBN = 128;   // keys per tile
// Warp layout.  GECKO_SCA_WG3=1 (default): 12 warps in three warpgroups
// (TMA, MMA and two idle warps; softmax of tile 0; softmax of tile 1), and
// setmaxnreg moves registers from the first warpgroup to the softmax
// warpgroups (88 and 2 x 208 per thread).  With 10 warps two SM
// sub-partitions hold three warps each, which caps every thread at 168
// registers; the 12-warp layout measured 2.76-2.77 ms against 2.86-2.90 ms
// per launch on the bench workload.  GECKO_SCA_WG3=0 keeps the 10-warp layout.
#ifndef GECKO_SCA_WG3
#define GECKO_SCA_WG3 1
#endif
constexpr int kThreads = GECKO_SCA_WG3 ? 384 : 320;   // TMA, MMA (+TMEM allocation), [2 idle], 2 x 4 softmax
constexpr int kSoftmaxWarp0 = GECKO_SCA_WG3 ? 4 : 2;  // first softmax warp
// Per-thread registers after setmaxnreg (GECKO_SCA_WG3).  The split must fit
// the registers the block was launched with: 128 x kRegsCtl + 256 x
// kRegsSoftmax <= 384 x 168 = 64512 (a larger sum would leave setmaxnreg.inc
// waiting for registers forever).  96 / 200 measured 2.59-2.60 against
// 2.63-2.67 ms for 88 / 208 (the two MMA issuers live in the first warpgroup).
constexpr int kRegsCtl = 96, kRegsSoftmax = 200;
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= 384 * 168, "setmaxnreg split above the launch registers");
// Of every 8 exponential pairs, GECKO_SFU_PAIRS are evaluated on the SFU
// (ex2.approx) and the rest on the FMA pipe (exp2_poly2).  Measured on B200
// with the bench workload the all-SFU setting is fastest (the polynomial
// costs ~10 issue cycles per element against the SFU's 8-cycle warp rate),
// so 8 is the default; other splits remain available at compile time.
#ifndef GECKO_SFU_PAIRS
#define GECKO_SFU_PAIRS 8
#endif
constexpr int kSfuPairs = GECKO_SFU_PAIRS;
// GECKO_SCA_ONEPASS=1: the softmax reads each S tile from TMEM once into
// registers (row max and exponentials from the same registers) instead of
// streaming it twice (needs the 12-warp layout's registers).  Measured
// slower than two passes (2.81-2.83 against 2.76-2.77 ms), so off by default.
#ifndef GECKO_SCA_ONEPASS
#define GECKO_SCA_ONEPASS 0
#endif
// GECKO_SCA_ISSUERS=2 (default): warps 1 and 2 each issue one query tile's
// MMAs and take strict turns (tile 0's step of iteration j, then tile 1's),
// so the barrier waits, commits and loop work of one issuer overlap the
// other's MMAs on the tensor core (SCA kernel 2.68 against 2.73 ms over
// eight interleaved runs on the bench workload).  Each issuer releases K_j
// and V_{j-1} with its own commit (a commit covers only the committing
// thread's MMAs).  GECKO_SCA_ISSUERS=1 keeps one MMA thread for both tiles.
#ifndef GECKO_SCA_ISSUERS
#define GECKO_SCA_ISSUERS 2
#endif
constexpr int kIssuers = GECKO_SCA_ISSUERS;
// Register budget of the kernel: the default lets the compiler fit 320
// threads on one SM; GECKO_SCA_MAXNREG caps registers per thread instead.
#ifdef GECKO_SCA_MAXNREG
#define SCA_BOUNDS __maxnreg__(GECKO_SCA_MAXNREG)
#else
#define SCA_BOUNDS __launch_bounds__(kThreads, 1)
#endif

// Units are claimed dynamically from a global counter, in the schedule's
// order, by each CTA's TMA thread, which publishes them to the CTA's other
// roles through a ring of kUnitRing slots.  The producer claims at most
// max(kKStages, kVStages) + 1 units ahead of the slowest reader (its K and V
// loads lead the MMAs by at most that many iterations, every unit has at
// least one, and the softmax warps trail the MMA issuers by at most one
// unit), so 8 slots are never overwritten before they are read.
constexpr int kUnitRing = 8;

// Next unit to claim (reset to 0 on the launching stream before each launch;
// forwards on one device are not concurrent).
__device__ unsigned g_unit_counter;

template <int D>
struct ScaCfg {
  static constexpr int kTileBytes = 128 * D * 2;       // 128 rows x D bf16, D/64 swizzled boxes
  static constexpr int kBoxBytes = 128 * 64 * 2;       // one [128 x 64] box
  // Ring depths.  At d = 128 shared memory holds Q (two tiles) and five K/V
  // tiles (224 KB): 2 K and 3 V stages measured ~1 % faster than 3 K and 2 V
  // on the bench workload (2.72-2.76 against 2.76-2.77 ms per launch), and a
  // K ring of 2 alone cost nothing, so V waits were the ones worth shortening.
  // At d = 64 tiles are half the size: 5 K and 4 V stages.
#ifdef GECKO_SCA_KSTAGES
  static constexpr int kKStages = D == 64 ? 5 : GECKO_SCA_KSTAGES;
#else
  static constexpr int kKStages = D == 64 ? 5 : 2;
#endif
#ifdef GECKO_SCA_VSTAGES
  static constexpr int kVStages = D == 64 ? 4 : GECKO_SCA_VSTAGES;
#else
  static constexpr int kVStages = D == 64 ? 4 : 3;
#endif
  // it_done has one slot per K/V iteration in flight: the deeper of the two rings
  static constexpr int kIterRing = kKStages > kVStages ? kKStages : kVStages;
  static_assert(kIterRing + 2 <= kUnitRing, "unit ring too short for the K/V lead");
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
  // q_full, q_empty, k_full[KS], it_done[max(KS, VS)], v_full[VS], s_full[2],
  // p_full[2], o_full[2], o_empty[2], drain, unit_ready[kUnitRing], turn_done[2]
  static constexpr int kNumBars = 2 + kKStages + (kKStages > kVStages ? kKStages : kVStages) + kVStages + 8 + 1 +
                                  kUnitRing + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // tmem address, abort flag, then the unit ring (kUnitRing uint32)
  static constexpr int kBytes = kMiscOff + 8 + 4 * kUnitRing;
  static constexpr int kAlloc = kBytes + 1024;         // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "dynamic shared memory above the sm_100 per-block limit");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
};

struct Unit {
  int64_t bh;
  int q0;        // first query row of tile 0
  int nt;        // tiles in the unit (1 or 2)
  int beg[2];    // first key tile (128-key units) of each query tile
  int end[2];    // one past the last (= diagonal tile + 1)
};

// Map a linear unit index to (bh, pair).  When c % 256 == 0 the units are
// grouped by (bh, chunk): the c / 256 units of one group read the same K/V
// window (previous + current chunk), so running them next to each other
// keeps that window in L2 while the group is in flight (ordering the whole
// grid by cost instead puts ~148 different windows in flight, far more than
// L2 holds, and every K/V tile then comes from DRAM).  Inside a group the
// units go from the most to the least expensive; groups of later chunks
// come first and the cheap chunk-1 groups last, which keeps the tail short.
__device__ __forceinline__ Unit decode_unit(int u, int BH, int T, int c, int koff) {
  const int pairs = (T + 255) / 256;
  Unit U;
  int pair;
  if (c % 256 == 0) {
    const int npc = c / 256;
    const int S = T / c;
    const int g = u / npc;
    const int o = npc - 1 - u % npc;
    const int n_main = (S - 1) * BH;
    int ch;
    if (g < n_main) {
      ch = S - 1 - g / BH;
      U.bh = g % BH;
    } else {
      ch = 0;
      U.bh = g - n_main;
    }
    pair = ch * npc + o;
  } else {
    pair = u / BH;
    U.bh = u % BH;
  }
  (void)pairs;
  U.q0 = pair * 256;
  U.nt = (U.q0 + 128 < T) ? 2 : 1;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r0 = U.q0 + 128 * i;
    const int ch = r0 / c;
    // window start; negative (the prepended previous chunk) when koff > 0
    const int lo = (ch >= 1 || koff > 0) ? (ch - 1) * c : 0;
    U.beg[i] = lo / kBN;
    U.end[i] = r0 / kBN + 1;
    if (i >= U.nt) { U.beg[i] = 0; U.end[i] = 0; }
  }
  return U;
}

// Key-tile range of query tile i of a unit, selected by value so that a
// runtime i does not force the unit into local memory.
__device__ __forceinline__ int ubeg(const Unit& U, int i) { return i ? U.beg[1] : U.beg[0]; }
__device__ __forceinline__ int uend(const Unit& U, int i) { return i ? U.end[1] : U.end[0]; }

// The TMA thread's claims: ordinal n of this CTA's work is unit
// slot[n % kUnitRing]; a claim takes the next unit of the global counter
// (n_units once all are taken, the end marker), writes it to its slot and
// arrives on the slot's barrier.
struct Claims {
  unsigned* counter;
  uint32_t* slot;
  uint64_t* ready;
  int claimed;
  int n_units;

  __device__ __forceinline__ int unit_of(int n) {
    while (claimed <= n) {
      const unsigned u = atomicAdd(counter, 1u);
      const int s = claimed % kUnitRing;
      slot[s] = u < (unsigned)n_units ? u : (unsigned)n_units;
      mbar_arrive(ready + s);   // release: the slot write is visible to its readers
      ++claimed;
    }
    return (int)slot[n % kUnitRing];
  }
};

// Walks the K/V iterations of one CTA in the order the MMA issuers consume
// them: its units in the order claimed, and each unit's key tiles in order.
struct KvWalk {
  int n;            // ordinal of the current unit
  int u;            // current unit (>= n_units: finished)
  int j, je;        // current key tile of the unit, one past its last
  int64_t kvbase;   // first K/V row of the unit's (b, h)
  uint32_t it;      // iterations walked so far
};

__device__ __forceinline__ void kv_walk_enter(KvWalk& w, int n, Claims& cl, int BH, int T, int c, int koff) {
  w.n = n;
  w.u = cl.unit_of(n);
  if (w.u < cl.n_units) {
    const Unit U = decode_unit(w.u, BH, T, c, koff);
    w.j = U.beg[0];
    w.je = U.nt == 2 ? U.end[1] : U.end[0];
    w.kvbase = U.bh * (int64_t)(T + koff) + koff;
  }
}

__device__ __forceinline__ void kv_walk_next(KvWalk& w, Claims& cl, int BH, int T, int c, int koff) {
  ++w.it;
  if (++w.j == w.je) {
    const uint32_t it = w.it;
    kv_walk_enter(w, w.n + 1, cl, BH, T, c, koff);
    w.it = it;
  }
}

// Pass 2 of the softmax of one 128-key S tile for this thread's row: p =
// 2^(s log2e - m_ref) in chunks of 32 columns (the next chunk's TMEM load is
// in flight while this one is computed), P as bf16 written over the
// consumed S columns, and the row sum of p returned.  The argument uses
// packed FMA; on tiles off the diagonal, of every 8 pairs kSfuPairs go to
// the SFU (ex2.approx) and the rest to the FMA pipe (exp2_poly2).  The
// diagonal tile masks keys after the row (r = row in the tile) and takes
// every exponential on the SFU, so masked keys give exactly 0.
template <bool kDiag>
__device__ __forceinline__ float softmax_pass2(uint32_t s_addr, float m_ref, int r) {
  const uint64_t l2e2 = pack2(kLog2e, kLog2e);
  const uint64_t nm2 = pack2(-m_ref, -m_ref);
  uint64_t acc2[2] = {pack2(0.f, 0.f), pack2(0.f, 0.f)};
  uint32_t cur[32], nxt[32];
  tmem_ld32p(s_addr, cur);
#pragma unroll
  for (int cb = 0; cb < kBN / 32; ++cb) {
    tmem_wait_ld();
    if (cb + 1 < kBN / 32) tmem_ld32p(s_addr + (cb + 1) * 32, nxt);
    if (kDiag) {
#pragma unroll
      for (int x = 0; x < 32; ++x)
        if (cb * 32 + x > r) cur[x] = __float_as_uint(-INFINITY);
    }
    uint32_t pk[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const uint64_t a2 = ffma2(pack2(__uint_as_float(cur[2 * x]), __uint_as_float(cur[2 * x + 1])), l2e2, nm2);
      uint64_t p2;
      if (kDiag || x % 8 < kSfuPairs) {
        float a0, a1;
        unpack2(a2, a0, a1);
        p2 = pack2(ex2(a0), ex2(a1));
      } else {
        p2 = exp2_poly2(a2);
      }
      acc2[x & 1] = fadd2(acc2[x & 1], p2);
      float p0, p1;
      unpack2(p2, p0, p1);
      pk[x] = pack_bf16x2(p0, p1);
    }
    tmem_st16(s_addr + cb * 16, pk);
    if (cb + 1 < kBN / 32) {
#pragma unroll
      for (int x = 0; x < 32; ++x) cur[x] = nxt[x];
    }
  }
  tmem_wait_st();
  float a0, a1, b0, b1;
  unpack2(acc2[0], a0, a1);
  unpack2(acc2[1], b0, b1);
  return (a0 + a1) + (b0 + b1);
}

#if GECKO_SCA_ONEPASS
// Max of a 128-column score row held in registers (8 independent chains).
__device__ __forceinline__ float row_max128(const uint32_t* sr) {
  float mp[8];
#pragma unroll
  for (int y = 0; y < 8; ++y) mp[y] = fmax3(__uint_as_float(sr[y]), __uint_as_float(sr[y + 8]), __uint_as_float(sr[y + 16]));
#pragma unroll
  for (int x = 24; x + 16 < 128; x += 16)
#pragma unroll
    for (int y = 0; y < 8; ++y) mp[y] = fmax3(mp[y], __uint_as_float(sr[x + y]), __uint_as_float(sr[x + 8 + y]));
#pragma unroll
  for (int y = 0; y < 8; ++y) mp[y] = fmaxf(mp[y], __uint_as_float(sr[120 + y]));
  return fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
}

// The exponential pass of softmax_pass2 on a row already in registers
// (masked entries set to -inf by the caller): P (bf16) written over the S
// columns 32 scores at a time, the row sum returned.
template <bool kDiag>
__device__ __forceinline__ float softmax_exp_regs(const uint32_t* sr, uint32_t s_addr, float m_ref) {
  const uint64_t l2e2 = pack2(kLog2e, kLog2e);
  const uint64_t nm2 = pack2(-m_ref, -m_ref);
  uint64_t acc2[2] = {pack2(0.f, 0.f), pack2(0.f, 0.f)};
#pragma unroll
  for (int cb = 0; cb < kBN / 32; ++cb) {
    uint32_t pk[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const uint64_t a2 = ffma2(pack2(__uint_as_float(sr[cb * 32 + 2 * x]), __uint_as_float(sr[cb * 32 + 2 * x + 1])),
                                l2e2, nm2);
      uint64_t p2;
      if (kDiag || x % 8 < kSfuPairs) {
        float a0, a1;
        unpack2(a2, a0, a1);
        p2 = pack2(ex2(a0), ex2(a1));
      } else {
        p2 = exp2_poly2(a2);
      }
      acc2[x & 1] = fadd2(acc2[x & 1], p2);
      float p0, p1;
      unpack2(p2, p0, p1);
      pk[x] = pack_bf16x2(p0, p1);
    }
    tmem_st16(s_addr + cb * 16, pk);
  }
  tmem_wait_st();
  float a0, a1, b0, b1;
  unpack2(acc2[0], a0, a1);
  unpack2(acc2[1], b0, b1);
  return (a0 + a1) + (b0 + b1);
}
#endif

template <int D>
__global__ void SCA_BOUNDS
sca_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
              const __grid_constant__ CUtensorMap map_v, __nv_bfloat16* __restrict__ out,
              float* __restrict__ lse, __nv_bfloat16* __restrict__ out_lo, int T, int c, int BH,
              int n_units, int koff, unsigned* unit_counter, int* status) {
  using Cfg = ScaCfg<D>;
  constexpr int KS = Cfg::kKStages, VS = Cfg::kVStages, IR = Cfg::kIterRing;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Cfg::kQOff;
  uint8_t* sK = smem + Cfg::kKOff;
  uint8_t* sV = smem + Cfg::kVOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  // it_done[m % IR] completes when the MMAs of K/V iteration m are done:
  // they were the last readers of K_m and of V_{m-1}
  uint64_t* it_done = k_full + KS;
  uint64_t* v_full = it_done + IR;
  uint64_t* s_full = v_full + VS;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* o_empty = o_full + 2;
  uint64_t* drain = o_empty + 2;
  uint64_t* unit_ready = drain + 1;   // [kUnitRing]
  uint64_t* turn_done = unit_ready + kUnitRing;   // [2] two issuers: issuer i finished its turn
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);
  uint32_t* unit_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff + 8);   // [kUnitRing]

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, kIssuers);
    for (int s = 0; s < KS; ++s) mbar_init(k_full + s, 1);
    for (int s = 0; s < IR; ++s) mbar_init(it_done + s, kIssuers);
    for (int s = 0; s < VS; ++s) mbar_init(v_full + s, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 128);
      mbar_init(o_full + i, 1);
      mbar_init(o_empty + i, 128);
    }
    mbar_init(drain, kIssuers);
    mbar_init(turn_done + 0, 1);
    mbar_init(turn_done + 1, 1);
    for (int r = 0; r < kUnitRing; ++r) mbar_init(unit_ready + r, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_q);
    tma_prefetch_desc(&map_k);
    tma_prefetch_desc(&map_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;


#if GECKO_SCA_WG3
  if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsCtl));
#endif
  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      // Three load streams, each in the order the MMA issuers consume them:
      // Q of every unit, K_m and V_m of every K/V iteration m.  A load
      // first waits until the previous reader of its slot is done: K_m for
      // iteration m - KS, V_m for iteration m + 1 - VS (V_m is read by the
      // PV MMAs of iteration m + 1), Q of a unit for the last QK of the
      // previous unit.  Issuing the loads in the order of those iterations
      // (not unit by unit) lets K run ahead of V by its deeper ring, and
      // every wait is then for an iteration whose own loads were issued
      // earlier, so the producer never waits on itself.
      Claims cl{unit_counter, unit_slot, unit_ready, 0, n_units};
      KvWalk kw{}, vw{};
      kv_walk_enter(kw, 0, cl, BH, T, c, koff);
      vw = kw;
      int qn = 0;
      int qu = cl.unit_of(0);
      uint32_t qit0 = 0;   // first K/V iteration of unit qu
      bool ok = true;
      while (ok) {
        const bool has_k = kw.u < n_units, has_v = vw.u < n_units, has_q = qu < n_units;
        if (!has_k && !has_v && !has_q) break;
        const int64_t tK = has_k ? (int64_t)kw.it - KS : INT64_MAX;
        const int64_t tV = has_v ? (int64_t)vw.it + 1 - VS : INT64_MAX;
        const int64_t tQ = has_q ? (int64_t)qit0 - 1 : INT64_MAX;
        if (tQ <= tK && tQ <= tV) {
          const Unit U = decode_unit(qu, BH, T, c, koff);
          if (qn > 0 && !(ok = mbar_wait(q_empty, (qn - 1) & 1, abort_flag, status))) break;
          mbar_arrive_expect_tx(q_full, U.nt * Cfg::kTileBytes);
          const int64_t rowbase = U.bh * (int64_t)T;
          for (int i = 0; i < U.nt; ++i)
            for (int b = 0; b < D / 64; ++b)
              tma_load_2d(sQ + i * Cfg::kTileBytes + b * Cfg::kBoxBytes, &map_q, q_full, b * 64,
                          (int)(rowbase + U.q0 + 128 * i));
          qit0 += (uint32_t)((U.nt == 2 ? U.end[1] : U.end[0]) - U.beg[0]);
          ++qn;
          qu = cl.unit_of(qn);
        } else if (tV <= tK) {
          if (tV >= 0 && !(ok = mbar_wait(it_done + tV % IR, (uint32_t)(tV / IR) & 1, abort_flag, status))) break;
          const int st = vw.it % VS;
          const int row = (int)(vw.kvbase + (int64_t)vw.j * kBN);
          mbar_arrive_expect_tx(v_full + st, Cfg::kTileBytes);
          for (int b = 0; b < D / 64; ++b)
            tma_load_2d(sV + st * Cfg::kTileBytes + b * Cfg::kBoxBytes, &map_v, v_full + st, b * 64, row);
          kv_walk_next(vw, cl, BH, T, c, koff);
        } else {
          if (tK >= 0 && !(ok = mbar_wait(it_done + tK % IR, (uint32_t)(tK / IR) & 1, abort_flag, status))) break;
          const int st = kw.it % KS;
          const int row = (int)(kw.kvbase + (int64_t)kw.j * kBN);
          mbar_arrive_expect_tx(k_full + st, Cfg::kTileBytes);
          for (int b = 0; b < D / 64; ++b)
            tma_load_2d(sK + st * Cfg::kTileBytes + b * Cfg::kBoxBytes, &map_k, k_full + st, b * 64, row);
          kv_walk_next(kw, cl, BH, T, c, koff);
        }
      }
      if (!ok) {
        // let every copy already issued land before the CTA exits (older
        // copies of a slot landed before its reuse was allowed)
        for (uint32_t idx = kw.it >= (uint32_t)KS ? kw.it - KS : 0; idx < kw.it; ++idx)
          mbar_wait_drain(k_full + idx % KS, (idx / KS) & 1);
        for (uint32_t idx = vw.it >= (uint32_t)VS ? vw.it - VS : 0; idx < vw.it; ++idx)
          mbar_wait_drain(v_full + idx % VS, (idx / VS) & 1);
        if (qn > 0) mbar_wait_drain(q_full, (qn - 1) & 1);
      }
    }
    __syncwarp();
  } else if (kIssuers == 2 && (warp == 1 || warp == 2)) {
    // ------------------------------------------- two MMA issuers, one per tile --
    if (lane == 0) {
      const int i = warp - 1;   // the query tile this thread issues for
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      const uint32_t qa = smem_u32(sQ) + i * Cfg::kTileBytes, ka = smem_u32(sK), va = smem_u32(sV);
      const uint32_t colS = i == 0 ? Cfg::kColS0 : Cfg::kColS1;
      const uint32_t colO = i == 0 ? Cfg::kColO0 : Cfg::kColO1;
      uint32_t kv_it = 0, p_par = 0, o_par = 0, turn = 0;
      bool ok = true;
      for (int n = 0;; ++n) {
        if (!(ok = mbar_wait(unit_ready + n % kUnitRing, (n / kUnitRing) & 1, abort_flag, status))) break;
        const int u = (int)unit_slot[n % kUnitRing];
        if (u >= n_units) break;
        const Unit U = decode_unit(u, BH, T, c, koff);
        if (!(ok = mbar_wait(q_full, n & 1, abort_flag, status))) break;
        tc_fence_after();
        const int jb = U.beg[0], je = U.nt == 2 ? U.end[1] : U.end[0];
        const int bi = i < U.nt ? ubeg(U, i) : 0, ei = i < U.nt ? uend(U, i) : 0;
        for (int j = jb; j <= je && ok; ++j) {
          // turn (j, i): after the other issuer's turn (j, 0) or (j - 1, 1)
          if (!(i == 0 && turn == 0)) {
            const uint32_t q = i == 0 ? turn - 1 : turn;
            if (!(ok = mbar_wait(turn_done + (1 - i), q & 1, abort_flag, status))) break;
          }
          if (j - 1 >= bi && j - 1 < ei) {
            // O_i += P_i V_{j-1} (V_{j-1} was waited for with this tile's QK of iteration j - 1)
            if (j - 1 == bi) {
              if (!(ok = mbar_wait(o_empty + i, (o_par & 1) ^ 1, abort_flag, status))) break;
            }
            if (!(ok = mbar_wait(p_full + i, p_par & 1, abort_flag, status))) break;
            p_par ^= 1u;
            tc_fence_after();
            const SDesc vd = sdesc_sw128_split(va + ((kv_it - 1) % VS) * Cfg::kTileBytes, Cfg::kBoxBytes, 1024);
            umma_ts(tmem + colO, tmem + colS, sdesc_at(vd, 0), idesc_pv, j - 1 > bi ? 1u : 0u);
#pragma unroll
            for (int kk = 1; kk < kBN / 16; ++kk)
              umma_ts(tmem + colO, tmem + colS + kk * 8, sdesc_at(vd, kk * 2048), idesc_pv, 1u);
            if (j - 1 == ei - 1) {
              umma_commit(o_full + i);
              o_par ^= 1u;
            }
          }
          if (j >= bi && j < ei) {
            // S_i = Q_i K_j^T; V_j (read by the PVs of iteration j + 1) is waited for here too
            if (!(ok = mbar_wait(k_full + kv_it % KS, (kv_it / KS) & 1, abort_flag, status))) break;
            if (!(ok = mbar_wait(v_full + kv_it % VS, (kv_it / VS) & 1, abort_flag, status))) break;
            tc_fence_after();
            const SDesc qd = sdesc_sw128_split(qa, 16, 1024);
            const SDesc kd = sdesc_sw128_split(ka + (kv_it % KS) * Cfg::kTileBytes, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t kbyte = (kk / 4) * Cfg::kBoxBytes + (kk % 4) * 32;
              umma_ss(tmem + colS, sdesc_at(qd, kbyte), sdesc_at(kd, kbyte), idesc_qk, kk > 0 ? 1u : 0u);
            }
            umma_commit(s_full + i);
          }
          mbar_arrive(turn_done + i);
          ++turn;
          if (j < je) {
            // this issuer is done with K_j and V_{j-1} once its MMAs so far complete
            umma_commit(it_done + kv_it % IR);
            if (j == je - 1) umma_commit(q_empty);
            ++kv_it;
          }
        }
        if (!ok) break;
      }
      // all issued MMAs complete before TMEM is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK), va = smem_u32(sV);
      // bit i: the phase parity of tile i's p_full and o_empty waits
      uint32_t kv_it = 0, p_par = 0, o_par = 0;
      int n = 0;
      bool ok = true;
      for (;; ++n) {
        if (!(ok = mbar_wait(unit_ready + n % kUnitRing, (n / kUnitRing) & 1, abort_flag, status))) break;
        const int u = (int)unit_slot[n % kUnitRing];
        if (u >= n_units) break;
        const Unit U = decode_unit(u, BH, T, c, koff);
        if (!(ok = mbar_wait(q_full, n & 1, abort_flag, status))) break;
        tc_fence_after();
        const int jb = U.beg[0], je = U.nt == 2 ? U.end[1] : U.end[0];
        for (int j = jb; j <= je && ok; ++j) {
          const uint32_t stK = kv_it % KS;
          // K_j and V_j are waited for together, right before the first QK
          // of iteration j (V_j is first read by the PVs of iteration j + 1).
          // A wait placed right after a group of MMAs overlaps the tensor
          // core's work on that group; at the top of the iteration it would
          // add to the gap before the next PV (SCA kernel 2.68-2.74 against
          // 2.75-2.77 ms on the bench workload).
          bool k_ready = false;
          const uint32_t stV = (kv_it - 1) % VS;   // V_{j-1}, waited for in iteration j - 1
          for (int i = 0; i < U.nt && ok; ++i) {
            const uint32_t colS = i == 0 ? Cfg::kColS0 : Cfg::kColS1;
            const uint32_t colO = i == 0 ? Cfg::kColO0 : Cfg::kColO1;
            if (j - 1 >= ubeg(U, i) && j - 1 < uend(U, i)) {
              // O_i += P_i V_{j-1}
              if (j - 1 == ubeg(U, i)) {
                if (!(ok = mbar_wait(o_empty + i, ((o_par >> i) & 1) ^ 1, abort_flag, status))) break;
              }
              if (!(ok = mbar_wait(p_full + i, (p_par >> i) & 1, abort_flag, status))) break;
              p_par ^= 1u << i;
              tc_fence_after();
              const SDesc vd = sdesc_sw128_split(va + stV * Cfg::kTileBytes, Cfg::kBoxBytes, 1024);
              umma_ts(tmem + colO, tmem + colS, sdesc_at(vd, 0), idesc_pv, j - 1 > ubeg(U, i) ? 1u : 0u);
#pragma unroll
              for (int kk = 1; kk < kBN / 16; ++kk)
                umma_ts(tmem + colO, tmem + colS + kk * 8, sdesc_at(vd, kk * 2048), idesc_pv, 1u);
              if (j - 1 == uend(U, i) - 1) {
                umma_commit(o_full + i);
                o_par ^= 1u << i;
              }
            }
            if (j >= ubeg(U, i) && j < uend(U, i)) {
              if (!k_ready) {
                if (!(ok = mbar_wait(k_full + stK, (kv_it / KS) & 1, abort_flag, status))) break;
                if (!(ok = mbar_wait(v_full + kv_it % VS, (kv_it / VS) & 1, abort_flag, status))) break;
                tc_fence_after();
                k_ready = true;
              }
              // S_i = Q_i K_j^T
              const SDesc qd = sdesc_sw128_split(qa + i * Cfg::kTileBytes, 16, 1024);
              const SDesc kd = sdesc_sw128_split(ka + stK * Cfg::kTileBytes, 16, 1024);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t kbyte = (kk / 4) * Cfg::kBoxBytes + (kk % 4) * 32;
                umma_ss(tmem + colS, sdesc_at(qd, kbyte), sdesc_at(kd, kbyte), idesc_qk, kk > 0 ? 1u : 0u);
              }
              umma_commit(s_full + i);
            }
          }
          if (!ok) break;
          if (j < je) {
            // no commit for it_done: the softmax warpgroup of the iteration's
            // last active tile arrives on it once that tile's S is complete
            if (j == je - 1) umma_commit(q_empty);
            ++kv_it;
          }
        }
        if (!ok) break;
      }
      // all issued MMAs complete before TMEM is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else if (warp >= kSoftmaxWarp0) {
#if GECKO_SCA_WG3
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsSoftmax));
#endif
    // ------------------------------------------------ softmax warpgroups --
    const int i = (warp - kSoftmaxWarp0) / 4;   // query tile handled by this warpgroup
    const int r = (warp % 4) * 32 + lane;   // row within the tile = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const uint32_t colS = i == 0 ? Cfg::kColS0 : Cfg::kColS1;
    const uint32_t colO = i == 0 ? Cfg::kColO0 : Cfg::kColO1;
    uint32_t s_cnt = 0, o_cnt = 0;
    bool ok = true;
    uint32_t it_base = 0;   // K/V iterations of this CTA's earlier units (both warpgroups see every unit)
    for (int n = 0;; ++n) {
      ok = __all_sync(0xffffffffu, mbar_wait(unit_ready + n % kUnitRing, (n / kUnitRing) & 1, abort_flag, status));
      if (!ok) break;
      const int u = (int)unit_slot[n % kUnitRing];
      if (u >= n_units) break;
      const Unit U = decode_unit(u, BH, T, c, koff);
      const int jb = U.beg[0], je = U.nt == 2 ? U.end[1] : U.end[0];
      const uint32_t unit_it0 = it_base;
      it_base += (uint32_t)(je - jb);
      if (i >= U.nt) continue;
      float m_ref = 0.f, l = 0.f;
      for (int j = ubeg(U, i); j < uend(U, i); ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(s_full + i, s_cnt & 1, abort_flag, status));
        if (!ok) break;
        // With one MMA thread, the QK of the iteration's last active tile is
        // its last MMA, so its completion (just observed) means K_j and
        // V_{j-1} are no longer read: one thread of that tile's warpgroup
        // releases them to the producer.  (Two issuers release them with
        // their own commits.)
        if (kIssuers == 1 && (i == 1 || !(U.nt == 2 && j >= U.beg[1])) && warp % 4 == 2 && lane == 0)
          mbar_arrive(it_done + (unit_it0 + (uint32_t)(j - jb)) % IR);
        ++s_cnt;
        tc_fence_after();
        const bool diag = j == uend(U, i) - 1;
#if GECKO_SCA_ONEPASS
        // the whole S row in registers: one TMEM read, one wait
        uint32_t sr[kBN];
#pragma unroll
        for (int h = 0; h < kBN / 32; ++h) tmem_ld32p(lane_addr + colS + h * 32, sr + h * 32);
        tmem_wait_ld();
        if (diag) {
#pragma unroll
          for (int x = 0; x < kBN; ++x)
            if (x > r) sr[x] = __float_as_uint(-INFINITY);
        }
        const float mt = row_max128(sr);
#else
        // pass 1: row max, streaming S out of TMEM 64 columns at a time
        float mt = -INFINITY;
#pragma unroll
        for (int h = 0; h < kBN / 64; ++h) {
          uint32_t sr[64];
          tmem_ld32p(lane_addr + colS + h * 64, sr);
          tmem_ld32p(lane_addr + colS + h * 64 + 32, sr + 32);
          tmem_wait_ld();
          if (diag) {
#pragma unroll
            for (int x = 0; x < 64; ++x)
              if (h * 64 + x > r) sr[x] = __float_as_uint(-INFINITY);
          }
          float mp[8];
#pragma unroll
          for (int y = 0; y < 8; ++y)
            mp[y] = fmax3(__uint_as_float(sr[y]), __uint_as_float(sr[y + 8]), __uint_as_float(sr[y + 16]));
#pragma unroll
          for (int x = 24; x + 16 < 64; x += 16)
#pragma unroll
            for (int y = 0; y < 8; ++y) mp[y] = fmax3(mp[y], __uint_as_float(sr[x + y]), __uint_as_float(sr[x + 8 + y]));
#pragma unroll
          for (int y = 0; y < 8; ++y) mp[y] = fmaxf(mp[y], __uint_as_float(sr[56 + y]));
          mt = fmax3(mt, fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7])), -INFINITY);
        }
#endif
        const float m2 = mt * kLog2e;
        const bool grow = j != ubeg(U, i) && m2 > m_ref + 8.f;
        if (j == ubeg(U, i)) m_ref = m2;
        // O is rescaled with warp-collective TMEM loads and stores, so the
        // whole warp takes this branch when any of its rows needs it (the
        // other rows scale by 1)
        if (__any_sync(0xffffffffu, grow)) {
          const float scale = grow ? ex2(m_ref - m2) : 1.f;
          if (grow) {
            l *= scale;
            m_ref = m2;
          }
#pragma unroll 1
          for (int cb = 0; cb < D / 32; ++cb) {
            uint32_t o[32];
            tmem_ld32(lane_addr + colO + cb * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * scale);
            tmem_st32(lane_addr + colO + cb * 32, o);
          }
        }
        // pass 2: p = 2^(s log2e - m_ref), P (bf16) written over the consumed
        // S columns, row sum into l
#if GECKO_SCA_ONEPASS
        l += diag ? softmax_exp_regs<true>(sr, lane_addr + colS, m_ref) : softmax_exp_regs<false>(sr, lane_addr + colS, m_ref);
#else
        l += diag ? softmax_pass2<true>(lane_addr + colS, m_ref, r) : softmax_pass2<false>(lane_addr + colS, m_ref, r);
#endif
        tc_fence_before();
        mbar_arrive(p_full + i);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 rows
      ok = __all_sync(0xffffffffu, mbar_wait(o_full + i, o_cnt & 1, abort_flag, status));
      if (!ok) break;
      ++o_cnt;
      tc_fence_after();
      const float inv = 1.f / l;
      // row log-sum-exp (natural log) for a backward pass: p = 2^(s log2e - m_ref) / l
      if (lse) lse[U.bh * (int64_t)T + U.q0 + 128 * i + r] = (m_ref + log2f(l)) * kLn2;
      __nv_bfloat16* orow = out + (U.bh * (int64_t)T + U.q0 + 128 * i + r) * D;
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t o[32];
        tmem_ld32(lane_addr + colO + cb * 32, o);
        tmem_wait_ld();
        uint4 w[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int x = 0; x < 16; ++x)
          wp[x] = pack_bf16x2(__uint_as_float(o[2 * x]) * inv, __uint_as_float(o[2 * x + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
        for (int x = 0; x < 4; ++x) dst[x] = w[x];
        if (out_lo) {
          // what the bf16 output dropped, for a backward that needs O more
          // exactly (its row term rowsum(dO * O) cancels at long windows)
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wp[x]));
            wp[x] = pack_bf16x2(__uint_as_float(o[2 * x]) * inv - hi.x, __uint_as_float(o[2 * x + 1]) * inv - hi.y);
          }
          uint4* dlo = reinterpret_cast<uint4*>(out_lo + (orow - out) + cb * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) dlo[x] = w[x];
        }
      }
      tc_fence_before();
      mbar_arrive(o_empty + i);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// --------------------------------------------------------------- host --

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

// [rows, d] bf16 row-major viewed as a 2D tensor; box = 128 rows x 64 columns,
// 128-byte swizzle (the canonical K-major / MN-major UMMA operand layout).
cudaError_t make_map(CUtensorMap* m, const void* base, int64_t rows, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}


template <int D>
cudaError_t launch_sca_tc_impl(const Problem& p, cudaStream_t st) {
  using Cfg = ScaCfg<D>;
  const int64_t rows = p.B * p.H * p.T;
  const int64_t kv_rows = p.B * p.H * (p.T + p.koff);
  CUtensorMap mq, mk, mv;
  cudaError_t e;
  if ((e = make_map(&mq, p.q, rows, D)) != cudaSuccess) return e;
  if ((e = make_map(&mk, p.k, kv_rows, D)) != cudaSuccess) return e;
  if ((e = make_map(&mv, p.v, kv_rows, D)) != cudaSuccess) return e;
  const int BH = (int)(p.B * p.H);
  const int T = (int)p.T;
  const int n_units = BH * ((T + 255) / 256);
  const int grid = n_units < sm_count() ? n_units : sm_count();
  if ((e = cudaFuncSetAttribute(sca_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kAlloc)) !=
      cudaSuccess)
    return e;
#if GECKO_SCA_WG3
  {
    // the setmaxnreg split must fit the registers the kernel is launched with
    static int regs = 0;
    if (!regs) {
      cudaFuncAttributes fa;
      if ((e = cudaFuncGetAttributes(&fa, sca_tc_kernel<D>)) != cudaSuccess) return e;
      regs = fa.numRegs;
    }
    if (128 * kRegsCtl + 256 * kRegsSoftmax > kThreads * regs) return cudaErrorInvalidConfiguration;
  }
#endif
  // the unit counter starts from zero for every launch (stream-ordered)
  unsigned* counter = nullptr;
  if ((e = cudaGetSymbolAddress(reinterpret_cast<void**>(&counter), g_unit_counter)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(counter, 0, sizeof(unsigned), st)) != cudaSuccess) return e;
  sca_tc_kernel<D><<<grid, kThreads, Cfg::kAlloc, st>>>(mq, mk, mv, static_cast<__nv_bfloat16*>(p.out_sca), p.lse,
                                                        static_cast<__nv_bfloat16*>(p.out_sca_lo), T,
                                                        (int)p.c, BH, n_units, (int)p.koff, counter, p.status);
  return cudaGetLastError();
}

}  // namespace

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

bool tc_supported(const Problem& p) {
  if (p.dtype != kBF16 || p.c % 128 != 0) return false;
  // rows addressed through 32-bit TMA coordinates
  if (p.B * p.H * (p.T + p.koff) > (int64_t(1) << 31) - 1) return false;
  int dev = 0, major = 0, minor = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  return major == 10 && minor == 0;
}

cudaError_t launch_sca_tc(const Problem& p, cudaStream_t st) {
  return p.d == 64 ? launch_sca_tc_impl<64>(p, st) : launch_sca_tc_impl<128>(p, st);
}

}  // namespace gecko
