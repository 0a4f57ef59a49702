// BSFA prefill forward kernel for sm_100a.
//
// "Block Sparse Flash Attention" (§4 Method; §4.1 Gating Mechanism; §4.4
// Algorithm and Implementation; App. B.2 FlashAttention-2 tiled computation):
// every score tile S_ij = Q_i K_j^T / sqrt(d) is computed exactly; the block
// maximum s_max(i,j) is compared against the threshold of the head (or of the
// head and query tile, §4.2 "Threshold Calibration"); a block below it is
// skipped: its V tile is never loaded, its PV product is never issued and the
// running statistics (m, l, O) are left untouched. Diagonal blocks bypass the
// gate. N need not be a multiple of the tile sizes: query rows and keys at or
// past N are padding (zero-filled by TMA, masked out of the gate and softmax).
//
// One CTA owns two 128-row query slots that read the same K/V blocks: two query
// heads of one KV group on the same rows (GQA), or two adjacent 128-row tiles of
// one head (MHA, odd group sizes). Each slot holds one query tile when Bq = 128,
// two when Bq = 64. Warp roles (384 threads):
//   warps 0-3   softmax / gate / epilogue of slot 0; warps 4-7 the same for
//               slot 1. Thread r of a warpgroup owns row r of its slot (TMEM
//               lane r) and all of its key columns, so a row maximum never
//               leaves its thread. The two warpgroups run concurrently: while one
//               waits on the tensor core or on its gate barrier, the other
//               computes exponentials.
//   warp 8      TMEM allocation + TMA loads of both Q tiles and every K block;
//   warp 9      tcgen05.mma issue (one thread), both slots in a fixed order, each
//               step released by a named barrier the slot's warpgroup arrives on
//               once its P is stored;
//   warp 10     TMA loads of V, issued only for blocks some slot kept;
//   warp 11     S waiter: all 32 lanes poll each "S is in TMEM" completion and
//               turn it into a named barrier the slot's warpgroup starts its
//               step on.
// TMEM columns: S of slot 0 and 1 ([0,Bk), [Bk,2Bk)), then O of slot 0 and 1
// (D columns each). P is written back as bf16 over the first Bk/2 columns of its
// slot's S and read from there as the A operand of the PV product.
//
// MMA issue order per block j: for each slot, PV_s(j) (if kept) then QK_s(j+1).
// The commit that announces S_s(j+1) therefore also covers PV_s(j): when the
// softmax sees S_s(j+1), O_s is quiescent and may be rescaled in place.
#pragma once

#include "ptx.cuh"

namespace bsfa {

struct FwdParams {
  const float* tau;   // [Hq], or [Hq, tau_tiles] when tau_tiles > 0
  int tau_tiles;      // 0: one threshold per head; else per (head, query tile), the last column reused past its end
  uint16_t* out;      // bf16 [B, N, Hq, D]
  float* lse;         // [B, Hq, N] or null
  uint8_t* mask;      // [B, Hq, N/Bq, N/Bk] or null
  int* status;        // device status word
  // Mask-writing (debug) launches only: [0] V tiles loaded, [1] PV products issued
  // (one per slot and kept block), accumulated over launches.
  unsigned long long* counts;
  int B, Hq, Hkv, N;  // N need not be a multiple of the tile sizes: rows and keys >= N are masked
  // Packed variable-length batch (the kernel's VARLEN variants; null otherwise):
  // sequence e holds rows [cu_seqlens[e], cu_seqlens[e+1]) of the N = total rows,
  // and B is the sequence count.
  const int* cu_seqlens;
  int max_seqlen;     // longest sequence (N for [B, N] inputs): sizes the grid
  int mask_mq, mask_mkv;   // query tiles and key blocks per sequence in the block mask
  int group;          // Hq / Hkv
  int hq_begin, hq_count;   // the query heads this launch computes (all of them unless head-sharded)
  int pair_heads;     // 1: slots are query heads 2p and 2p+1 on the same rows
  // The query rows this launch computes, in row units (128-row tiles when
  // pair_heads, else pairs of adjacent 128-row tiles): [row_unit0, row_unit0 + row_units).
  int row_unit0, row_units;
  int gate_gap;       // 0: the BSFA gate (block maximum against tau); 1: the gap gate, tau holding gamma
                      // (selects the kernel's GAP template argument at launch)
  float scale;        // 1/sqrt(D): the gate compares s_max(raw) * scale against tau
  float scale_log2;   // log2(e)/sqrt(D): exponent scale of the softmax
  // Cycle trace of the first trace_ctas CTAs (kernels built with BSFA_TRACE only;
  // null otherwise): kTraceStride SM-clock stamps per CTA, laid out as below.
  unsigned long long* trace;
  int trace_ctas;
};

// Trace layout per CTA (clock64 stamps; steps past kTraceSteps are not recorded):
//   [0] start, [1] SM id, [2] end, [3 + w] warp w's clock right after the first
//   __syncthreads (the clocks of an SM's sub-partitions need not agree: these
//   give each warp's offset)
//   softmax  kTrSoftmax + (s * kTraceSteps + j) * 8 + e, by the slot's row-0 thread:
//            e = 0 S-ready barrier passed, 1 TMEM fence done, 2 scores loaded, 3 row
//            maxima taken, 4 gate barrier passed, 5 exponentials done, 6 P stored,
//            7 P-ready arrival
//   mma      kTrMma + (s * kTraceSteps + j) * 4 + e: 0 P-ready passed, 1 V ready (kept
//            blocks), 2 PV issued, 3 next QK issued and committed
//   waiter   kTrWait + s * kTraceSteps + j: s_full seen
//   V        kTrV + j * 2 + e: 0 decision seen, 1 load issued (or found not needed)
//   K        kTrK + j: load issued
//   epilogue kTrEpi + s * 2 + e: 0 o_done seen, 1 rows written
constexpr int kTraceSteps = 64;
constexpr int kTrSoftmax = 16;
constexpr int kTrMma = kTrSoftmax + 2 * kTraceSteps * 8;
constexpr int kTrWait = kTrMma + 2 * kTraceSteps * 4;
constexpr int kTrV = kTrWait + 2 * kTraceSteps;
constexpr int kTrK = kTrV + 2 * kTraceSteps;
constexpr int kTrEpi = kTrK + kTraceSteps;
constexpr int kTraceStride = 1920;
static_assert(kTrEpi + 4 <= kTraceStride, "trace layout");

#ifdef BSFA_TRACE
__device__ __forceinline__ void trace_at(const FwdParams& p, int idx) {
  if (p.trace != nullptr && (int)blockIdx.x < p.trace_ctas)
    p.trace[(size_t)blockIdx.x * kTraceStride + idx] = clock64();
}
__device__ __forceinline__ void trace_step(const FwdParams& p, int base, int j, int e, int per) {
  if (j < kTraceSteps) trace_at(p, base + j * per + e);
}
#define BSFA_TRACE_AT(p, idx) trace_at((p), (idx))
#define BSFA_TRACE_STEP(p, base, j, e, per) trace_step((p), (base), (j), (e), (per))
#else
#define BSFA_TRACE_AT(p, idx) ((void)0)
#define BSFA_TRACE_STEP(p, base, j, e, per) ((void)0)
#endif

// O is rescaled only when the running maximum grows by more than 2^8 in the
// exp2 domain; until then P is taken against the stale maximum (values <= 2^8,
// exact in the final O / l ratio).
constexpr float kRescaleThreshold = 8.0f;
// One softmax warpgroup per slot; thread r of a warpgroup owns row r of its slot.
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 32 * (kSoftmaxWarps + 4);
constexpr int kLaunchRegs = 168;      // 65536 / kThreads, rounded down to the allocation granularity
constexpr int kSoftmaxRegs = 216;
constexpr int kProducerRegs = 72;
static_assert(kSoftmaxWarps * 32 * kSoftmaxRegs + 128 * kProducerRegs <= kThreads * kLaunchRegs, "register split");
// Named barriers (0 is __syncthreads):
//   kSReadyBar + s  "S of slot s is in TMEM": the waiter warp joins once s_full
//                   says so, the slot's warpgroup at the start of its step (a
//                   hardware barrier, so the softmax's critical path has no
//                   shared-memory poll of the MMA's completion barrier);
//   kGateBar + s    the gate of slot s: an OR over its warpgroup's comparisons;
//   kPReadyBar + s  P of slot s is stored (or the block was skipped, or the step
//                   abandoned): the warpgroup arrives, the whole MMA warp syncs.
constexpr uint32_t kSReadyBar = 1;
constexpr uint32_t kGateBar = 3;
constexpr uint32_t kPReadyBar = 5;
constexpr uint32_t kSReadyCount = 32 * (4 + 1);
constexpr uint32_t kGateCount = 128;
constexpr uint32_t kPReadyCount = 32 * (4 + 1);

__device__ __forceinline__ void named_barrier_arrive(uint32_t id, uint32_t count) {
  asm volatile("barrier.cta.arrive.aligned %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int D, int BQ, int BK>
struct FwdShape {
  static constexpr int ROWS = 128;
  static constexpr int NSUB = ROWS / BQ;   // query tiles per slot
  static constexpr int DCH = D / 64;       // 128-byte swizzle chunks along D
  static constexpr int KS = 2;             // K ring depth
  static constexpr int VS = 2;             // V ring depth
  static constexpr uint32_t Q_BYTES = ROWS * D * 2;
  static constexpr uint32_t KV_BYTES = BK * D * 2;
  static constexpr uint32_t OFF_Q = 0;                        // two Q tiles
  static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KS * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + VS * KV_BYTES;
  static constexpr uint32_t BAR_BYTES = 8448;                       // barriers and gate decisions
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + BAR_BYTES;        // base is 1024-aligned (checked)
  static constexpr uint32_t TMEM_S0 = 0;
  static constexpr uint32_t TMEM_O0 = 2 * BK;
  static constexpr uint32_t TMEM_COLS = (2 * BK + 2 * D <= 256) ? 256 : 512;
  static_assert(D == 64 || D == 128, "D");
  static_assert(BQ == 64 || BQ == 128, "Bq");
  static_assert(BK == 64 || BK == 128, "Bk");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Gate decisions of every block, one bit per (slot, block): at most this many
// key blocks per sequence.
constexpr int kMaxKeyBlocks = 4096;

template <int KS, int VS>
struct alignas(16) FwdBarriers {
  uint64_t q_full;
  uint64_t k_full[KS], k_empty[KS];
  uint64_t v_full[VS], v_empty[VS];
  uint64_t s_full[2], o_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;                               // any role gave up on a bounded wait
  int sm_abort[2][2];                      // [slot][block parity]: the waiter gave up on that step's S
  alignas(16) uint8_t gate_dec[2][kMaxKeyBlocks];   // 0 undecided, 1 skipped, 2 kept
};

struct FwdUnit {
  int b, kvh;
  int hq[2], q0[2], nblk[2];   // q0: first row of the slot within its sequence
};

// Where a unit's sequence lies among packed sequences (VARLEN variants only).
struct SeqSpan {
  int row0, len;               // the sequence's first row in the N dimension, and its length
  int seq;                     // the sequence's index
};

template <bool VARLEN>
__device__ __forceinline__ FwdUnit decode_unit(const FwdParams& p, int u, bool causal, int bk, SeqSpan& sp) {
  FwdUnit w;
  if (p.pair_heads) {
    // Consecutive units: the head pairs of one row block, a KV group's pairs adjacent.
    const int per = p.B * (p.hq_count / 2);
    const int hp = u % per, t = u / per;
    const int qt = p.row_unit0 + (causal ? p.row_units - 1 - t : t);   // heaviest causal rows first
    w.b = hp / (p.hq_count / 2);
    const int h0 = p.hq_begin + 2 * (hp % (p.hq_count / 2));
    w.hq[0] = h0;
    w.hq[1] = h0 + 1;
    w.q0[0] = w.q0[1] = qt * 128;
  } else {
    const int per = p.B * p.hq_count;
    const int bh = u % per, t = u / per;
    const int qp = p.row_unit0 + (causal ? p.row_units - 1 - t : t);
    w.b = bh / p.hq_count;
    w.hq[0] = w.hq[1] = p.hq_begin + bh % p.hq_count;
    w.q0[0] = 2 * qp * 128;
    w.q0[1] = w.q0[0] + 128;
  }
  w.kvh = w.hq[0] / p.group;
  int len = p.N;
  if (VARLEN) {   // packed sequences: one batch entry of N = total rows
    // Offsets are clamped to [0, N] and lengths to max_seqlen, so no access can
    // leave the caller's buffers whatever the offsets hold.
    sp.seq = w.b;
    sp.row0 = min(max(p.cu_seqlens[w.b], 0), p.N);
    sp.len = len = min(min(max(p.cu_seqlens[w.b + 1], sp.row0), p.N) - sp.row0, p.max_seqlen);
    w.b = 0;
  }
#pragma unroll
  for (int s = 0; s < 2; ++s)
    w.nblk[s] = (w.q0[s] >= len) ? 0 : (causal ? min((w.q0[s] + 128) / bk, (len + bk - 1) / bk) : (len + bk - 1) / bk);
  return w;
}

// The unit's sequence length, first row and index. For [B, N] inputs these are
// compile-time forms of N, 0 and b, and the span is never read.
template <bool VARLEN>
__device__ __forceinline__ int unit_len(const SeqSpan& sp, const FwdParams& p) { return VARLEN ? sp.len : p.N; }
template <bool VARLEN>
__device__ __forceinline__ int unit_row0(const SeqSpan& sp) { return VARLEN ? sp.row0 : 0; }
template <bool VARLEN>
__device__ __forceinline__ int unit_seq(const FwdUnit& w, const SeqSpan& sp) { return VARLEN ? sp.seq : w.b; }

// Bounded wait used when draining in-flight copies/MMAs on the way out: it does
// not give up early on the abort flag, only on the time limit.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  int local = 0;
  return mbar_wait(bar, parity, &local);
}

// ---------------------------------------------------------------------------- K/Q producer (warp 8, one thread)

template <int D, int BQ, int BK, bool VARLEN, typename Bars>
__device__ __forceinline__ void kq_producer(const FwdParams& p, const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                            uint8_t* smem, Bars* bars, const FwdUnit& w, const SeqSpan& sp) {
  using S = FwdShape<D, BQ, BK>;
  volatile int* abort_flag = &bars->abort;
  prefetch_tensormap(tm_q);
  prefetch_tensormap(tm_k);
  const int nq = (w.nblk[0] > 0) + (w.nblk[1] > 0);
  mbar_arrive_expect_tx(&bars->q_full, nq * S::Q_BYTES);
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    if (w.nblk[s] == 0) continue;
#pragma unroll
    for (int c = 0; c < S::DCH; ++c)
      tma_load_4d(smem + S::OFF_Q + s * S::Q_BYTES + c * (S::ROWS * 128), tm_q, &bars->q_full, c * 64, w.hq[s],
                  unit_row0<VARLEN>(sp) + w.q0[s], w.b);
  }
  const int nblk = max(w.nblk[0], w.nblk[1]);
  int issued = 0;
  for (int t = 0; t < nblk; ++t) {
    const int slot = t % S::KS;
    if (!mbar_wait(&bars->k_empty[slot], ((t / S::KS) & 1) ^ 1, abort_flag)) break;
    mbar_arrive_expect_tx(&bars->k_full[slot], S::KV_BYTES);
#pragma unroll
    for (int c = 0; c < S::DCH; ++c)
      tma_load_4d(smem + S::OFF_K + slot * S::KV_BYTES + c * (BK * 128), tm_k, &bars->k_full[slot], c * 64, w.kvh,
                  unit_row0<VARLEN>(sp) + t * BK, w.b);
    BSFA_TRACE_STEP(p, kTrK, t, 0, 1);
    issued = t + 1;
  }
  // Copies still in flight must land before the CTA exits.
  drain_wait(&bars->q_full, 0);
  for (int t = (issued > S::KS ? issued - S::KS : 0); t < issued; ++t)
    drain_wait(&bars->k_full[t % S::KS], (t / S::KS) & 1);
}

// Bounded wait until slot s's gate decision for block j is published. The
// thread sleeps between looks: a tight shared-memory spin would steal the
// bandwidth the QK^T MMAs (both operands in shared memory) depend on.
template <typename Bars>
__device__ __forceinline__ bool wait_decided(Bars* bars, int s, int j) {
  volatile uint8_t* dec = &bars->gate_dec[s][j];
  volatile int* abort_flag = &bars->abort;
  if (*dec != 0) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    __nanosleep(64);
    if (*dec != 0) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitTimeoutNs) {
      *abort_flag = 1;
      return false;
    }
  }
}

// ---------------------------------------------------------------------------- V producer (one thread)

template <int D, int BQ, int BK, bool VARLEN, bool COUNT, typename Bars>
__device__ __forceinline__ void v_producer(const FwdParams& p, const CUtensorMap* tm_v, uint8_t* smem, Bars* bars,
                                           const FwdUnit& w, const SeqSpan& sp) {
  using S = FwdShape<D, BQ, BK>;
  volatile int* abort_flag = &bars->abort;
  prefetch_tensormap(tm_v);
  const int nblk = max(w.nblk[0], w.nblk[1]);
  int v_count = 0;
  bool failed = false;
  for (int j = 0; j < nblk && !failed; ++j) {
    bool loaded = false;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (j >= w.nblk[s] || loaded) continue;   // (once one slot keeps j, V(j) is requested)
      if (!wait_decided(bars, s, j)) { failed = true; break; }
      BSFA_TRACE_STEP(p, kTrV, j, 0, 2);
      const bool keep = ((volatile uint8_t*)bars->gate_dec[s])[j] == 2;
      if (!keep) continue;               // skipped by this slot
      const int slot = v_count % S::VS;
      if (!mbar_wait(&bars->v_empty[slot], ((v_count / S::VS) & 1) ^ 1, abort_flag)) { failed = true; break; }
      mbar_arrive_expect_tx(&bars->v_full[slot], S::KV_BYTES);
#pragma unroll
      for (int c = 0; c < S::DCH; ++c)
        tma_load_4d(smem + S::OFF_V + slot * S::KV_BYTES + c * (BK * 128), tm_v, &bars->v_full[slot], c * 64, w.kvh,
                    unit_row0<VARLEN>(sp) + j * BK, w.b);
      loaded = true;
      if (COUNT) atomicAdd(&p.counts[0], 1ull);
    }
    BSFA_TRACE_STEP(p, kTrV, j, 1, 2);
    if (loaded) ++v_count;
  }
  for (int n = (v_count > S::VS ? v_count - S::VS : 0); n < v_count; ++n)
    drain_wait(&bars->v_full[n % S::VS], (n / S::VS) & 1);
}

// ---------------------------------------------------------------------------- S waiter (warp 11, whole warp)

// Watches s_full for every (slot, block) step in the MMA warp's issue order and
// joins that slot's named barrier once S is in TMEM. All 32 lanes poll, so the
// warp is converged when it reaches the (warp-aligned) barrier and none of its
// lanes can arrive before the poll has seen S. It syncs rather than only
// arriving, so it stays in lockstep with each warpgroup's steps even when its
// waits give up (then it marks the step's abort flag first and joins anyway):
// the softmax warps never wait on a barrier that cannot complete.
template <typename Bars>
__device__ __forceinline__ void s_waiter(const FwdParams& p, Bars* bars, const FwdUnit& w) {
  volatile int* abort_flag = &bars->abort;
  const int lane = threadIdx.x & 31;
  const int nblk = max(w.nblk[0], w.nblk[1]);
  for (int j = 0; j < nblk; ++j) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (j >= w.nblk[s]) continue;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[s], j & 1, abort_flag));
      if (!got && lane == 0) ((volatile int*)bars->sm_abort[s])[j & 1] = 1;
      if (lane == 0) BSFA_TRACE_STEP(p, kTrWait + s * kTraceSteps, j, 0, 1);
      __syncwarp();
      named_barrier_sync(kSReadyBar + s, kSReadyCount);
    }
  }
}

// ---------------------------------------------------------------------------- MMA issuer (warp 9, one thread)

template <int D, int BQ, int BK, bool COUNT, typename Bars>
__device__ __forceinline__ void mma_issuer(const FwdParams& p, uint8_t* smem, Bars* bars, uint32_t tmem,
                                           const FwdUnit& w) {
  using S = FwdShape<D, BQ, BK>;
  constexpr uint32_t IDESC_QK = make_idesc_bf16(128, BK, false);   // B = K tile, K-major
  constexpr uint32_t IDESC_PV = make_idesc_bf16(128, D, true);     // B = V tile, MN-major
  volatile int* abort_flag = &bars->abort;
  const int nblk = max(w.nblk[0], w.nblk[1]);

  auto qk = [&](int s, int kslot) {
    const uint32_t q_addr = smem_u32(smem + S::OFF_Q + s * S::Q_BYTES);
    const uint32_t k_addr = smem_u32(smem + S::OFF_K + kslot * S::KV_BYTES);
    const uint32_t d_tmem = tmem + S::TMEM_S0 + s * BK;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t ch = kk / 4, koff = (kk % 4) * 32;   // 16 bf16 = 32 bytes per K step
      const uint64_t a = make_sdesc_sw128(q_addr + ch * (S::ROWS * 128) + koff, 16, 1024);
      const uint64_t bd = make_sdesc_sw128(k_addr + ch * (BK * 128) + koff, 16, 1024);
      mma_ss(d_tmem, a, bd, IDESC_QK, kk > 0 ? 1u : 0u);
    }
  };
  auto pv = [&](int s, int vslot, bool first) {
    const uint32_t v_addr = smem_u32(smem + S::OFF_V + vslot * S::KV_BYTES);
    const uint32_t p_tmem = tmem + S::TMEM_S0 + s * BK;
    const uint32_t o_tmem = tmem + S::TMEM_O0 + s * D;
#pragma unroll
    for (int kk = 0; kk < BK / 16; ++kk) {
      // 16 keys per K step: 16 rows of 128 bytes in V; 8 packed bf16x2 columns of P.
      const uint64_t bd = make_sdesc_sw128(v_addr + kk * 16 * 128, BK * 128, 1024);
      mma_ts(o_tmem, p_tmem + kk * 8, bd, IDESC_PV, (!first || kk > 0) ? 1u : 0u);
    }
  };

  const bool leader = (threadIdx.x & 31) == 0;
  bool ok = true;
  if (leader) ok = mbar_wait(&bars->q_full, 0, abort_flag) && mbar_wait(&bars->k_full[0], 0, abort_flag);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok && leader) {
    tc_fence_after();
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (w.nblk[s] == 0) continue;
      qk(s, 0);
      tc_commit(&bars->s_full[s]);
    }
    tc_commit(&bars->k_empty[0]);
  }
  int v_count = 0;
  bool pv_started[2] = {false, false};
  // The whole warp syncs on every (slot, block) step's P-ready barrier with the
  // slot's warpgroup, even after a give-up; lane 0 issues.
  for (int j = 0; j < nblk; ++j) {
    bool k_ready = false, v_ready = false;
    int vslot = 0;
    const int kslot = (j + 1) % S::KS;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (j >= w.nblk[s]) continue;
      __syncwarp();                           // the barrier is warp-aligned: lane 0 may still be issuing
      named_barrier_sync(kPReadyBar + s, kPReadyCount);
      if (leader && ok) {
        BSFA_TRACE_STEP(p, kTrMma + s * kTraceSteps * 4, j, 0, 4);
        tc_fence_after();
        if (*abort_flag) ok = false;
        if (ok && ((volatile uint8_t*)bars->gate_dec[s])[j] == 2) {
          if (!v_ready) {
            vslot = v_count % S::VS;
            if (!mbar_wait(&bars->v_full[vslot], (v_count / S::VS) & 1, abort_flag)) ok = false;
            else { tc_fence_after(); v_ready = true; }
          }
          if (ok) {
            BSFA_TRACE_STEP(p, kTrMma + s * kTraceSteps * 4, j, 1, 4);
            pv(s, vslot, !pv_started[s]);
            pv_started[s] = true;
            if (COUNT) atomicAdd(&p.counts[1], 1ull);
            BSFA_TRACE_STEP(p, kTrMma + s * kTraceSteps * 4, j, 2, 4);
          }
        }
        if (ok) {
          if (j + 1 < w.nblk[s]) {
            if (!k_ready) {
              if (!mbar_wait(&bars->k_full[kslot], ((j + 1) / S::KS) & 1, abort_flag)) ok = false;
              else { tc_fence_after(); k_ready = true; }
            }
            if (ok) {
              qk(s, kslot);
              tc_commit(&bars->s_full[s]);
            }
          } else {
            tc_commit(&bars->o_done[s]);
          }
          BSFA_TRACE_STEP(p, kTrMma + s * kTraceSteps * 4, j, 3, 4);
        }
      }
    }
    if (leader) {
      if (v_ready) {
        tc_commit(&bars->v_empty[vslot]);
        ++v_count;
      }
      if (k_ready) tc_commit(&bars->k_empty[kslot]);
    }
    __syncwarp();
  }
  // Every MMA issued above must complete before TMEM is released.
  if (leader) {
    tc_commit(&bars->drain);
    drain_wait(&bars->drain, 0);
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------- softmax / gate / epilogue (warps 0-7)

// Warpgroup s (warps 4s..4s+3) works on slot s alone. Thread r owns row r of the
// slot (TMEM lane r) and every key column of it, so the row maximum is the
// thread's own; the block maximum of a query tile is never formed: the gate
// decision is the OR that the tile's named barrier computes over the threads'
// own comparisons.
struct SoftmaxRow {
  float m = -INFINITY;   // reference maximum of the exponentials, exp2 domain (lazy)
  float l = 0.f;         // running normaliser
  float M = -INFINITY;   // true row maximum over the kept blocks, exp2 domain (gap gate)
};

// One step (slot s, block j). Returns false when the step is abandoned (the
// waiter gave up on S, or an earlier step was abandoned: 'failed'); every thread
// of the warpgroup reads the same abort flag after the same barrier, so they
// agree. An abandoned step still takes the S-ready barrier, so the barrier
// accounting of the warpgroup and the waiter warp agrees.
template <int D, int BQ, int BK, bool CAUSAL, bool WRITE_MASK, bool GAP, bool VARLEN, typename Bars>
__device__ __forceinline__ bool softmax_block(const FwdParams& p, Bars* bars, uint32_t tmem, const FwdUnit& w,
                                              const SeqSpan& sp, int s, int j, float tau, SoftmaxRow& st,
                                              bool failed) {
  using S = FwdShape<D, BQ, BK>;
  const int lane = threadIdx.x & 31;
  const int wq = (threadIdx.x >> 5) & 3;     // warp within the warpgroup: TMEM lane quarter
  const int r = wq * 32 + lane;              // row within the slot, TMEM lane
  const int hq = s ? w.hq[1] : w.hq[0];
  const int q0 = s ? w.q0[1] : w.q0[0];
  const int qrow = q0 + r;
  const int sub = r / BQ;                    // query tile within the slot (Bq = 64: two per slot)
  const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
  const uint32_t s_tmem = tmem + S::TMEM_S0 + s * BK + lane_off;
  const uint32_t o_tmem = tmem + S::TMEM_O0 + s * D + lane_off;
  const int len = unit_len<VARLEN>(sp, p);

  // S(s, j) is in TMEM once the waiter warp has arrived (it watches s_full).
  named_barrier_sync(kSReadyBar + s, kSReadyCount);
  const int tr = kTrSoftmax + s * kTraceSteps * 8;
  (void)tr;
  const bool trace_me = r == 0;
  if (r == 0) BSFA_TRACE_STEP(p, tr, j, 0, 8);
  if (failed || ((volatile int*)bars->sm_abort[s])[j & 1]) {
    named_barrier_arrive(kPReadyBar + s, kPReadyCount);    // the MMA warp takes every step's barrier too
    return false;
  }
  tc_fence_after();
  if (r == 0) BSFA_TRACE_STEP(p, tr, j, 1, 8);
  float sv[BK];
  {
    uint32_t raw[BK];
    if constexpr (BK == 128) tmem_ld_x128(s_tmem, raw);
    else tmem_ld_x64(s_tmem, raw);
#pragma unroll
    for (int c = 0; c < BK; ++c) sv[c] = __uint_as_float(raw[c]);
  }
  if (r == 0) BSFA_TRACE_STEP(p, tr, j, 2, 8);
  // Last valid key of this row: the diagonal (causal) or the sequence end. A
  // causal padding row (qrow >= N) also sees the zero-filled keys up to qrow;
  // it is left out of the gate and never written, and V is zero there.
  const int k0 = j * BK;
  const int klim = CAUSAL ? qrow : len - 1;
  if (k0 + BK - 1 > klim) {                    // this row's columns reach past it
#pragma unroll
    for (int c = 0; c < BK; ++c)
      if (k0 + c > klim) sv[c] = -INFINITY;
  }
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
  for (int c = 0; c < BK; c += 8) {
    m0 = max3(m0, sv[c], sv[c + 1]);
    m1 = max3(m1, sv[c + 2], sv[c + 3]);
    m2 = max3(m2, sv[c + 4], sv[c + 5]);
    m3 = max3(m3, sv[c + 6], sv[c + 7]);
  }
  const float rmax = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
  if (r == 0) BSFA_TRACE_STEP(p, tr, j, 3, 8);
  // Gate: s_max * scale >= tau holds exactly when some row's maximum does, so the
  // barrier's OR over the query tile's threads is the decision. Rows past N are
  // padding. The gap gate (tau = gamma * log2(e)) keeps the block when some row
  // with a valid entry has no kept block yet or reaches its running maximum
  // minus gamma.
  const bool above =
      qrow < len && (GAP ? (rmax > -INFINITY && (st.M == -INFINITY || rmax * p.scale_log2 >= st.M - tau))
                         : (rmax * p.scale >= tau));
  bool any_above[S::NSUB];
  any_above[0] = named_barrier_or(kGateBar + s, kGateCount, above && (S::NSUB == 1 || sub == 0));
  if constexpr (S::NSUB == 2) any_above[1] = named_barrier_or(kGateBar + s, kGateCount, above && sub == 1);
  if (r == 0) BSFA_TRACE_STEP(p, tr, j, 4, 8);
  int code[S::NSUB];
  bool keep_any = false;
#pragma unroll
  for (int t = 0; t < S::NSUB; ++t) {
    // Visible: some (row < N, key <= row) entry. Diagonal: judged on the full-size
    // tile and block (as if the sequence were padded to whole tiles), so the block
    // holding a row's own key is forced even in a last tile of one row.
    const int lo = q0 + t * BQ;
    const int k_lo = j * BK;
    const bool visible = lo < len && (!CAUSAL || k_lo <= min(lo + BQ - 1, len - 1));
    const bool diag = visible && (CAUSAL ? k_lo + BK - 1 > lo : (k_lo < lo + BQ && k_lo + BK > lo));
    code[t] = !visible ? 3 : diag ? 2 : (any_above[t] ? 1 : 0);
    keep_any |= (code[t] == 1 || code[t] == 2);
  }
  if (r == 0) {
    if (WRITE_MASK) {
      const int mq = p.mask_mq, mkv = p.mask_mkv;
#pragma unroll
      for (int t = 0; t < S::NSUB; ++t)
        if (code[t] != 3)
          p.mask[((size_t)(unit_seq<VARLEN>(w, sp) * p.Hq + hq) * mq + (q0 / BQ + t)) * mkv + j] = (uint8_t)code[t];
    }
    // Publish the decision (one byte, no fence) so the V tile, if kept, is fetched
    // right away; the MMA warp reads it after the P-ready barrier, which orders it.
    ((volatile uint8_t*)bars->gate_dec[s])[j] = keep_any ? 2 : 1;
  }
  if (!keep_any) {                 // skipped by every tile of the slot: release S, nothing else
    tc_fence_before();
    __syncwarp();
    named_barrier_arrive(kPReadyBar + s, kPReadyCount);
    if (r == 0) BSFA_TRACE_STEP(p, tr, j, 7, 8);
    return true;
  }

  const int my_code = (S::NSUB == 1 || sub == 0) ? code[0] : code[S::NSUB - 1];
  const bool my_keep = (my_code == 1 || my_code == 2);       // uniform within a warp
  float m = st.m;
  bool need_rescale = false;
  float alpha = 1.f;
  if (my_keep) {
    const float mx = rmax * p.scale_log2;
    if (GAP) st.M = fmaxf(st.M, mx);
    if (mx > m + kRescaleThreshold) {      // also taken on the first finite maximum
      if (m != -INFINITY) {
        alpha = ex2_approx(m - mx);
        need_rescale = true;
      }
      m = mx;
    }
  }
  // P = 2^(s * log2(e)/sqrt(d) - m): 3 of every 4 exponentials on the SFU (ex2),
  // 1 as a polynomial on the FMA pipe, the rest of the arithmetic in f32x2 pairs,
  // in three passes (arguments, exponentials, packing and sums), which schedules
  // the SFU and FMA work better than one fused pass. P (bf16 pairs) goes over S
  // columns this thread has already read.
  const bool live = my_keep && (m != -INFINITY);
  const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
  const float2 nm2 = make_float2(-m, -m);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
  const bool zero_p = __any_sync(0xffffffffu, !live) && !live;   // rows this block does not update: P = 0
  constexpr int H = BK / 4;                  // pairs per half
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[H];
    float2 xv[H];
#pragma unroll
    for (int e = 0; e < H; ++e) xv[e] = __ffma2_rn(make_float2(sv[2 * (h * H + e)], sv[2 * (h * H + e) + 1]), sl2, nm2);
#pragma unroll
    for (int e = 0; e < H; ++e) {
      if ((e & 3) == 3) xv[e] = exp2_poly2(xv[e]);
      else xv[e] = make_float2(ex2_approx(xv[e].x), ex2_approx(xv[e].y));
    }
#pragma unroll
    for (int e = 0; e < H; ++e) {
      pk[e] = zero_p ? 0u : pack_bf16x2(xv[e].x, xv[e].y);
      if (e & 1) acc1 = __fadd2_rn(acc1, xv[e]);
      else acc0 = __fadd2_rn(acc0, xv[e]);
    }
    if constexpr (H == 32) tmem_st_x32(s_tmem + h * H, pk);
    else tmem_st_x16(s_tmem + h * H, pk);
  }
  if (live) st.l = st.l * alpha + ((acc0.x + acc0.y) + (acc1.x + acc1.y));
  if (trace_me) BSFA_TRACE_STEP(p, tr, j, 5, 8);
  tmem_st_wait();
  if (r == 0) BSFA_TRACE_STEP(p, tr, j, 6, 8);

  // O_s is quiescent here: the commit that announced S_s(j) also covered PV_s(j-1).
  if (__any_sync(0xffffffffu, need_rescale)) {
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld_x32(o_tmem + c * 32, o);
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
      tmem_st_x32(o_tmem + c * 32, o);
    }
    tmem_st_wait();
  }
  st.m = m;
  tc_fence_before();
  __syncwarp();
  named_barrier_arrive(kPReadyBar + s, kPReadyCount);
  if (r == 0) BSFA_TRACE_STEP(p, tr, j, 7, 8);
  return true;
}

// Epilogue of slot s: each thread writes its row, O / l as bf16 with 16-byte
// stores; lse is the natural-log logsumexp over the kept set.
template <int D, int BQ, int BK, bool VARLEN, typename Bars>
__device__ __forceinline__ void softmax_epilogue(const FwdParams& p, Bars* bars, uint32_t tmem, const FwdUnit& w,
                                                 const SeqSpan& sp, int s, const SoftmaxRow& st, bool failed) {
  using S = FwdShape<D, BQ, BK>;
  if (failed) return;                        // uniform across the warpgroup
  volatile int* abort_flag = &bars->abort;
  const int lane = threadIdx.x & 31;
  const int wq = (threadIdx.x >> 5) & 3;
  const int r = wq * 32 + lane;
  const int hq = s ? w.hq[1] : w.hq[0];
  const int q0 = s ? w.q0[1] : w.q0[0];
  const int qrow = q0 + r;
  bool ok = true;
  if (lane == 0) ok = mbar_wait(&bars->o_done[s], 0, abort_flag);
  ok = __shfl_sync(0xffffffffu, ok, 0);      // the TMEM loads below are warp-collective
  if (!ok) return;
  if (r == 0) BSFA_TRACE_AT(p, kTrEpi + s * 2);
  tc_fence_after();
  const uint32_t o_tmem = tmem + S::TMEM_O0 + s * D + ((uint32_t)(wq * 32) << 16);
  // Padding rows of a last tile (qrow >= N) take part in the warp's TMEM loads
  // (warp-collective) but store nothing.
  const bool row_ok = qrow < unit_len<VARLEN>(sp, p);
  const float inv_l = 1.f / st.l;     // > 0: every row keeps its diagonal block, which holds its own key
  uint16_t* orow = p.out + ((size_t)(w.b * p.N + unit_row0<VARLEN>(sp) + qrow) * p.Hq + hq) * D;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld_x32(o_tmem + c * 32, o);
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
      pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
    if (row_ok) {
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
    }
  }
  if (row_ok && p.lse != nullptr)
    p.lse[(size_t)(w.b * p.Hq + hq) * p.N + unit_row0<VARLEN>(sp) + qrow] = (st.m + __log2f(st.l)) * 0.69314718055994531f;
  if (r == 0) BSFA_TRACE_AT(p, kTrEpi + s * 2 + 1);
}

template <int D, int BQ, int BK, bool CAUSAL, bool WRITE_MASK, bool GAP, bool VARLEN, typename Bars>
__device__ __forceinline__ void softmax_role(const FwdParams& p, Bars* bars, uint32_t tmem, const FwdUnit& w,
                                             const SeqSpan& sp) {
  const int s = threadIdx.x >> 7;            // this warpgroup's slot
  const int nblk = s ? w.nblk[1] : w.nblk[0];
  if (nblk == 0) return;                     // slot past the end of the sequence
  // This thread's threshold: its query tile's column of the table (clamped to
  // the table's last column), or the head's single value.
  const int sub = ((threadIdx.x >> 5) & 3) * 32 / BQ;
  const int hq = s ? w.hq[1] : w.hq[0];
  const int tile = (s ? w.q0[1] : w.q0[0]) / BQ + sub;
  const float t = p.tau_tiles > 0 ? p.tau[hq * p.tau_tiles + min(tile, p.tau_tiles - 1)] : p.tau[hq];
  const float tau = GAP ? t * 1.4426950408889634f : t;   // gamma in the exp2 domain of the running maximum
  SoftmaxRow st;
  bool failed = false;
  // Every step is taken even after an abort (then without work), in the
  // waiter warp's order.
#pragma unroll 1
  for (int j = 0; j < nblk; ++j)
    failed = !softmax_block<D, BQ, BK, CAUSAL, WRITE_MASK, GAP, VARLEN>(p, bars, tmem, w, sp, s, j, tau, st, failed);
  softmax_epilogue<D, BQ, BK, VARLEN>(p, bars, tmem, w, sp, s, st, failed);
}

// ---------------------------------------------------------------------------- kernel

template <int D, int BQ, int BK, bool CAUSAL, bool WRITE_MASK, bool GAP, bool VARLEN>
__global__ void __launch_bounds__(kThreads, 1)
    bsfa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using S = FwdShape<D, BQ, BK>;
  using Bars = FwdBarriers<S::KS, S::VS>;
  static_assert(sizeof(Bars) <= S::BAR_BYTES, "barrier block");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  Bars* bars = reinterpret_cast<Bars*>(smem + S::OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  SeqSpan sp;
  const FwdUnit w = decode_unit<VARLEN>(p, blockIdx.x, CAUSAL, BK, sp);
  if (VARLEN && w.nblk[0] == 0 && w.nblk[1] == 0) return;   // rows past a short packed sequence's end: no work

  if (threadIdx.x == 0) {
#ifdef BSFA_TRACE
    BSFA_TRACE_AT(p, 0);
    if (p.trace != nullptr && (int)blockIdx.x < p.trace_ctas) {
      unsigned smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      p.trace[(size_t)blockIdx.x * kTraceStride + 1] = smid;
    }
#endif
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < S::KS; ++i) { mbar_init(&bars->k_full[i], 1); mbar_init(&bars->k_empty[i], 1); }
    for (int i = 0; i < S::VS; ++i) { mbar_init(&bars->v_full[i], 1); mbar_init(&bars->v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->o_done[i], 1);
      bars->sm_abort[i][0] = bars->sm_abort[i][1] = 0;
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  // Gate decisions start undecided (0); every thread clears a share.
  for (int i = threadIdx.x; i < 2 * kMaxKeyBlocks / 16; i += kThreads)
    reinterpret_cast<uint4*>(&bars->gate_dec[0][0])[i] = make_uint4(0u, 0u, 0u, 0u);
  // The 128-byte swizzle and the descriptors assume a 1024-byte aligned base.
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(p.status, 2);
    return;
  }
  if (warp == kSoftmaxWarps) {
    tmem_alloc(&bars->tmem_base, S::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  if (lane == 0) BSFA_TRACE_AT(p, 3 + warp);
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < kSoftmaxWarps) {
    regs_increase<kSoftmaxRegs>();
    softmax_role<D, BQ, BK, CAUSAL, WRITE_MASK, GAP, VARLEN>(p, bars, tmem, w, sp);
  } else {
    regs_decrease<kProducerRegs>();
    if (lane == 0) {
      if (warp == kSoftmaxWarps) kq_producer<D, BQ, BK, VARLEN>(p, &tm_q, &tm_k, smem, bars, w, sp);
      else if (warp == kSoftmaxWarps + 2) v_producer<D, BQ, BK, VARLEN, WRITE_MASK>(p, &tm_v, smem, bars, w, sp);
    }
    __syncwarp();
    if (warp == kSoftmaxWarps + 1) mma_issuer<D, BQ, BK, WRITE_MASK>(p, smem, bars, tmem, w);
    if (warp == kSoftmaxWarps + 3) s_waiter(p, bars, w);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kSoftmaxWarps) {
    tc_fence_after();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
  if (threadIdx.x == 0 && ((volatile int*)&bars->abort)[0]) atomicOr(p.status, 1);
  if (threadIdx.x == 0) BSFA_TRACE_AT(p, 2);
}

}  // namespace bsfa
