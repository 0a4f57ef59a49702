// BSFA prefill forward kernel for sm_100a.
//
// "Block Sparse Flash Attention" (§4 Method; §4.1 Gating Mechanism; §4.4
// Algorithm and Implementation; App. B.2 FlashAttention-2 tiled computation):
// every score tile S_ij = Q_i K_j^T / sqrt(d) is computed exactly; the block
// maximum s_max(i,j) is compared against the head's threshold tau; a block below
// tau is skipped: its V tile is never loaded, its PV product is never issued and
// the running statistics (m, l, O) are left untouched. Diagonal blocks bypass the
// gate.
//
// One CTA owns two 128-row query slots that read the same K/V blocks: two query
// heads of one KV group on the same rows (GQA), or two adjacent 128-row tiles of
// one head (MHA, odd group sizes). Each slot holds one query tile when Bq = 128,
// two when Bq = 64. Warp roles (384 threads):
//   warps 0-3, 4-7  softmax / gate / epilogue of slot 0 and slot 1: thread r of
//                   the warpgroup owns row r of its slot (TMEM lane r);
//   warp 8          TMEM allocation + TMA loads of both Q tiles and every K block;
//   warp 9          tcgen05.mma issue (one thread);
//   warp 10         TMA loads of V, issued only for blocks some slot kept;
//   warp 11         idle (completes the producer warpgroup for the register split).
// The two softmax warpgroups run in ping-pong: while one computes its
// exponentials, the tensor core works on the other slot. TMEM columns: S of
// slot 0 and 1 ([0,Bk), [Bk,2Bk)), then O of slot 0 and 1 (D columns each).
// P is written back as bf16 over the first Bk/2 columns of its slot's S and read
// from there as the A operand of the PV product.
//
// MMA issue order per block j: for each slot, PV_s(j) (if kept) then QK_s(j+1).
// The commit that announces S_s(j+1) therefore also covers PV_s(j): when the
// softmax sees S_s(j+1), O_s is quiescent and may be rescaled in place.
#pragma once

#include "ptx.cuh"

namespace bsfa {

struct FwdParams {
  const float* tau;   // [Hq]
  uint16_t* out;      // bf16 [B, N, Hq, D]
  float* lse;         // [B, Hq, N] or null
  uint8_t* mask;      // [B, Hq, N/Bq, N/Bk] or null
  int* status;        // device status word
  int B, Hq, Hkv, N;
  int group;          // Hq / Hkv
  int pair_heads;     // 1: slots are query heads 2p and 2p+1 on the same rows
  float scale;        // 1/sqrt(D): the gate compares s_max(raw) * scale against tau
  float scale_log2;   // log2(e)/sqrt(D): exponent scale of the softmax
};

// O is rescaled only when the running maximum grows by more than 2^8 in the
// exp2 domain; until then P is taken against the stale maximum (values <= 2^8,
// exact in the final O / l ratio).
constexpr float kRescaleThreshold = 8.0f;
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;      // 65536 / 384, rounded down to the allocation granularity
constexpr int kSoftmaxRegs = 216;
constexpr int kProducerRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kProducerRegs <= kThreads * kLaunchRegs, "register split");

template <int D, int BQ, int BK>
struct FwdShape {
  static constexpr int ROWS = 128;
  static constexpr int NSUB = ROWS / BQ;   // query tiles per slot
  static constexpr int DCH = D / 64;       // 128-byte swizzle chunks along D
  static constexpr int KS = 3;             // K ring depth
  static constexpr int VS = 2;             // V ring depth
  static constexpr int GR = 4;             // gate-decision ring depth (per slot)
  static constexpr uint32_t Q_BYTES = ROWS * D * 2;
  static constexpr uint32_t KV_BYTES = BK * D * 2;
  static constexpr uint32_t OFF_Q = 0;                        // two Q tiles
  static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KS * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + VS * KV_BYTES;
  static constexpr uint32_t BAR_BYTES = 1024;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;   // + alignment slack
  static constexpr uint32_t TMEM_S0 = 0;
  static constexpr uint32_t TMEM_O0 = 2 * BK;
  static constexpr uint32_t TMEM_COLS = (2 * BK + 2 * D <= 256) ? 256 : 512;
  static_assert(D == 64 || D == 128, "D");
  static_assert(BQ == 64 || BQ == 128, "Bq");
  static_assert(BK == 64 || BK == 128, "Bk");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <int KS, int VS, int GR>
struct alignas(8) FwdBarriers {
  uint64_t q_full;
  uint64_t k_full[KS], k_empty[KS];
  uint64_t v_full[VS], v_empty[VS];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t gate_full[2][GR], gate_empty[2][GR];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int gate_flag[2][GR];
  int p_keep[2];
  float red[2][2][4];   // [slot][block parity][warp]
};

struct FwdUnit {
  int b, kvh;
  int hq[2], q0[2], nblk[2];
};

__device__ __forceinline__ FwdUnit decode_unit(const FwdParams& p, int u, bool causal, int bk) {
  const int tiles = p.N / 128;
  FwdUnit w;
  if (p.pair_heads) {
    // Consecutive units: the head pairs of one row block, a KV group's pairs adjacent.
    const int per = p.B * (p.Hq / 2);
    const int hp = u % per, t = u / per;
    const int qt = causal ? tiles - 1 - t : t;     // heaviest causal rows first
    w.b = hp / (p.Hq / 2);
    const int h0 = 2 * (hp % (p.Hq / 2));
    w.hq[0] = h0;
    w.hq[1] = h0 + 1;
    w.q0[0] = w.q0[1] = qt * 128;
  } else {
    const int pairs = (tiles + 1) / 2;
    const int per = p.B * p.Hq;
    const int bh = u % per, t = u / per;
    const int qp = causal ? pairs - 1 - t : t;
    w.b = bh / p.Hq;
    w.hq[0] = w.hq[1] = bh % p.Hq;
    w.q0[0] = 2 * qp * 128;
    w.q0[1] = w.q0[0] + 128;
  }
  w.kvh = w.hq[0] / p.group;
#pragma unroll
  for (int s = 0; s < 2; ++s)
    w.nblk[s] = (w.q0[s] >= p.N) ? 0 : (causal ? (w.q0[s] + 128) / bk : p.N / bk);
  return w;
}

// Bounded wait used when draining in-flight copies/MMAs on the way out: it does
// not give up early on the abort flag, only on the time limit.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  int local = 0;
  return mbar_wait(bar, parity, &local);
}

// ---------------------------------------------------------------------------- K/Q producer (warp 8, one thread)

template <int D, int BQ, int BK, typename Bars>
__device__ __forceinline__ void kq_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k, uint8_t* smem,
                                            Bars* bars, const FwdUnit& w) {
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
                  w.q0[s], w.b);
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
                  t * BK, w.b);
    issued = t + 1;
  }
  // Copies still in flight must land before the CTA exits.
  drain_wait(&bars->q_full, 0);
  for (int t = (issued > S::KS ? issued - S::KS : 0); t < issued; ++t)
    drain_wait(&bars->k_full[t % S::KS], (t / S::KS) & 1);
}

// ---------------------------------------------------------------------------- V producer (warp 10, one thread)

template <int D, int BQ, int BK, typename Bars>
__device__ __forceinline__ void v_producer(const CUtensorMap* tm_v, uint8_t* smem, Bars* bars, const FwdUnit& w) {
  using S = FwdShape<D, BQ, BK>;
  volatile int* abort_flag = &bars->abort;
  volatile int* gate_flag = &bars->gate_flag[0][0];
  prefetch_tensormap(tm_v);
  const int nblk = max(w.nblk[0], w.nblk[1]);
  int v_count = 0;
  bool failed = false;
  for (int j = 0; j < nblk && !failed; ++j) {
    const int g = j % S::GR;
    bool loaded = false;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (j >= w.nblk[s]) continue;
      if (!mbar_wait(&bars->gate_full[s][g], (j / S::GR) & 1, abort_flag)) { failed = true; break; }
      const int keep = gate_flag[s * S::GR + g];
      mbar_arrive(&bars->gate_empty[s][g]);
      if (!keep || loaded) continue;     // skipped by this slot (or already requested)
      const int slot = v_count % S::VS;
      if (!mbar_wait(&bars->v_empty[slot], ((v_count / S::VS) & 1) ^ 1, abort_flag)) { failed = true; break; }
      mbar_arrive_expect_tx(&bars->v_full[slot], S::KV_BYTES);
#pragma unroll
      for (int c = 0; c < S::DCH; ++c)
        tma_load_4d(smem + S::OFF_V + slot * S::KV_BYTES + c * (BK * 128), tm_v, &bars->v_full[slot], c * 64, w.kvh,
                    j * BK, w.b);
      loaded = true;
    }
    if (loaded) ++v_count;
  }
  for (int n = (v_count > S::VS ? v_count - S::VS : 0); n < v_count; ++n)
    drain_wait(&bars->v_full[n % S::VS], (n / S::VS) & 1);
}

// ---------------------------------------------------------------------------- MMA issuer (warp 9, one thread)

template <int D, int BQ, int BK, typename Bars>
__device__ __forceinline__ void mma_issuer(uint8_t* smem, Bars* bars, uint32_t tmem, const FwdUnit& w) {
  using S = FwdShape<D, BQ, BK>;
  constexpr uint32_t IDESC_QK = make_idesc_bf16(128, BK, false);   // B = K tile, K-major
  constexpr uint32_t IDESC_PV = make_idesc_bf16(128, D, true);     // B = V tile, MN-major
  volatile int* abort_flag = &bars->abort;
  volatile int* p_keep = bars->p_keep;
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

  bool ok = mbar_wait(&bars->q_full, 0, abort_flag) && mbar_wait(&bars->k_full[0], 0, abort_flag);
  if (ok) {
    tc_fence_after();
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (w.nblk[s] == 0) continue;
      qk(s, 0);
      tc_commit(&bars->s_full[s]);
    }
    tc_commit(&bars->k_empty[0]);
    int v_count = 0;
    bool pv_started[2] = {false, false};
    for (int j = 0; j < nblk && ok; ++j) {
      bool k_ready = false, v_ready = false;
      int vslot = 0;
      const int kslot = (j + 1) % S::KS;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (j >= w.nblk[s]) continue;
        if (!mbar_wait(&bars->p_full[s], j & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (p_keep[s]) {
          if (!v_ready) {
            vslot = v_count % S::VS;
            if (!mbar_wait(&bars->v_full[vslot], (v_count / S::VS) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            v_ready = true;
          }
          pv(s, vslot, !pv_started[s]);
          pv_started[s] = true;
        }
        if (j + 1 < w.nblk[s]) {
          if (!k_ready) {
            if (!mbar_wait(&bars->k_full[kslot], ((j + 1) / S::KS) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            k_ready = true;
          }
          qk(s, kslot);
          tc_commit(&bars->s_full[s]);
        } else {
          tc_commit(&bars->o_done[s]);     // this slot's last block: O is final once this lands
        }
      }
      if (v_ready) {
        tc_commit(&bars->v_empty[vslot]);
        ++v_count;
      }
      if (k_ready) tc_commit(&bars->k_empty[kslot]);
    }
  }
  // Every MMA issued above must complete before TMEM is released.
  tc_commit(&bars->drain);
  drain_wait(&bars->drain, 0);
}

// ---------------------------------------------------------------------------- softmax / gate / epilogue (warps 0-7)

template <int D, int BQ, int BK, bool CAUSAL, bool WRITE_MASK, typename Bars>
__device__ __forceinline__ void softmax_role(const FwdParams& p, Bars* bars, uint32_t tmem, const FwdUnit& w) {
  using S = FwdShape<D, BQ, BK>;
  volatile int* abort_flag = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = warp >> 2;                 // slot
  const int wid = warp & 3;                // warp within the slot's warpgroup
  const int r = wid * 32 + lane;           // row within the slot, TMEM lane
  // (selects rather than runtime indexing keep the unit in registers)
  const int nblk = s ? w.nblk[1] : w.nblk[0];
  if (nblk == 0) return;                   // slot past the end of the sequence
  const int hq = s ? w.hq[1] : w.hq[0];
  const int q0 = s ? w.q0[1] : w.q0[0];
  const int b = w.b;
  const int qrow = q0 + r;
  const int sub = r / BQ;
  const uint32_t lane_off = (uint32_t)(wid * 32) << 16;
  const uint32_t s_tmem = tmem + S::TMEM_S0 + s * BK + lane_off;
  const uint32_t o_tmem = tmem + S::TMEM_O0 + s * D + lane_off;
  const float tau = p.tau[hq];
  const int mq = p.N / BQ, mkv = p.N / BK;

  float m = -INFINITY;   // running maximum, exp2 domain
  float l = 0.f;         // running normaliser
  bool failed = false;

  for (int j = 0; j < nblk; ++j) {
    const int buf = j & 1;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[s], j & 1, abort_flag));
    float sv[BK];
    float rmax = -INFINITY;
    if (ok) {
      tc_fence_after();
      uint32_t raw[BK];
      if constexpr (BK == 128) tmem_ld_x128(s_tmem, raw);
      else tmem_ld_x64(s_tmem, raw);
#pragma unroll
      for (int c = 0; c < BK; ++c) sv[c] = __uint_as_float(raw[c]);
      if (CAUSAL && (j + 1) * BK - 1 > q0) {       // block straddles the causal boundary
#pragma unroll
        for (int c = 0; c < BK; ++c)
          if (j * BK + c > qrow) sv[c] = -INFINITY;
      }
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int c = 0; c < BK; c += 4) {
        m0 = max3(m0, sv[c], sv[c + 1]);
        m1 = max3(m1, sv[c + 2], sv[c + 3]);
      }
      rmax = fmaxf(m0, m1);
    }
    // Block maximum of each query tile: warp reduction, then across the tile's warps.
    const float wmax = warp_max_redux(rmax);
    if (lane == 0) bars->red[s][buf][wid] = wmax;
    if (named_barrier_or(1 + s, 128, failed || !ok || *abort_flag)) {
      failed = true;
      break;
    }
    int code[S::NSUB];
    bool keep_any = false;
#pragma unroll
    for (int t = 0; t < S::NSUB; ++t) {
      float bm = -INFINITY;
#pragma unroll
      for (int u = t * (BQ / 32); u < (t + 1) * (BQ / 32); ++u) bm = fmaxf(bm, bars->red[s][buf][u]);
      const int lo = q0 + t * BQ, hi = lo + BQ - 1;
      const int k_lo = j * BK, k_hi = k_lo + BK - 1;
      const bool visible = !CAUSAL || k_lo <= hi;
      const bool diag = CAUSAL ? (visible && k_hi > lo) : (k_lo <= hi && k_hi >= lo);
      code[t] = !visible ? 3 : diag ? 2 : ((bm * p.scale >= tau) ? 1 : 0);
      keep_any |= (code[t] == 1 || code[t] == 2);
    }
    if (r == 0) {
      if (WRITE_MASK) {
#pragma unroll
        for (int t = 0; t < S::NSUB; ++t)
          if (code[t] != 3)
            p.mask[((size_t)(b * p.Hq + hq) * mq + (q0 / BQ + t)) * mkv + j] = (uint8_t)code[t];
      }
      // Publish the decision so the V tile (if kept) is fetched right away.
      const int g = j % S::GR;
      if (mbar_wait(&bars->gate_empty[s][g], ((j / S::GR) & 1) ^ 1, abort_flag)) {
        ((volatile int*)&bars->gate_flag[s][g])[0] = keep_any ? 1 : 0;
        mbar_arrive(&bars->gate_full[s][g]);
      } else {
        failed = true;
      }
      ((volatile int*)bars->p_keep)[s] = keep_any ? 1 : 0;
    }
    __syncwarp();
    if (!keep_any) {                 // skipped by every tile of the slot: release S, nothing else
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[s]);
      continue;
    }

    const int my_code = (S::NSUB == 1 || sub == 0) ? code[0] : code[S::NSUB - 1];
    const bool my_keep = (my_code == 1 || my_code == 2);       // uniform within a warp
    bool need_rescale = false;
    float alpha = 1.f;
    if (my_keep) {
      const float mx = rmax * p.scale_log2;
      if (mx > m + kRescaleThreshold) {      // also taken on the first finite maximum
        if (m != -INFINITY) {
          alpha = ex2_approx(m - mx);
          need_rescale = true;
        }
        m = mx;
      }
      l *= alpha;
    }
    // P = 2^(s * log2(e)/sqrt(d) - m): half of the exponentials on the SFU (ex2),
    // half as a polynomial on the FMA pipe, all other arithmetic in f32x2 pairs.
    const bool live = my_keep && (m != -INFINITY);
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    const float2 nm2 = make_float2(-m, -m);
    float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
    uint32_t pk[BK / 2];
#pragma unroll
    for (int e = 0; e < BK / 2; e += 2) {
      const float2 xa = __ffma2_rn(make_float2(sv[2 * e], sv[2 * e + 1]), sl2, nm2);
      const float2 xb = __ffma2_rn(make_float2(sv[2 * e + 2], sv[2 * e + 3]), sl2, nm2);
      const float2 pa = make_float2(ex2_approx(xa.x), ex2_approx(xa.y));
      const float2 pb = exp2_poly2(xb);
      acc0 = __fadd2_rn(acc0, pa);
      acc1 = __fadd2_rn(acc1, pb);
      pk[e] = pack_bf16x2(pa.x, pa.y);
      pk[e + 1] = pack_bf16x2(pb.x, pb.y);
    }
    if (__any_sync(0xffffffffu, !live)) {   // rows this block does not update: P = 0
      if (!live) {
#pragma unroll
        for (int e = 0; e < BK / 2; ++e) pk[e] = 0u;
        acc0 = acc1 = make_float2(0.f, 0.f);
      }
    }
    l += (acc0.x + acc0.y) + (acc1.x + acc1.y);
    if constexpr (BK == 128) tmem_st_x64(s_tmem, pk);   // P (bf16 pairs) over the consumed S columns
    else tmem_st_x32(s_tmem, pk);
    tmem_st_wait();

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
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->p_full[s]);
  }

  // Epilogue: O / l -> bf16 rows, lse = ln-sum-exp over the kept set.
  bool ok = !failed;
  if (ok) ok = mbar_wait(&bars->o_done[s], 0, abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
    tc_fence_after();
    const float inv_l = 1.f / l;     // l > 0: every row keeps its diagonal block, which holds its own key
    uint16_t* orow = p.out + ((size_t)(b * p.N + qrow) * p.Hq + hq) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld_x32(o_tmem + c * 32, o);
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
      uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
    }
    if (p.lse != nullptr) p.lse[(size_t)(b * p.Hq + hq) * p.N + qrow] = (m + __log2f(l)) * 0.69314718055994531f;
  }
}

// ---------------------------------------------------------------------------- kernel

template <int D, int BQ, int BK, bool CAUSAL, bool WRITE_MASK>
__global__ void __launch_bounds__(kThreads, 1)
    bsfa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using S = FwdShape<D, BQ, BK>;
  using Bars = FwdBarriers<S::KS, S::VS, S::GR>;
  static_assert(sizeof(Bars) <= S::BAR_BYTES, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + S::OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const FwdUnit w = decode_unit(p, blockIdx.x, CAUSAL, BK);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < S::KS; ++i) { mbar_init(&bars->k_full[i], 1); mbar_init(&bars->k_empty[i], 1); }
    for (int i = 0; i < S::VS; ++i) { mbar_init(&bars->v_full[i], 1); mbar_init(&bars->v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 4);          // one arrival per softmax warp
      mbar_init(&bars->o_done[i], 1);
      for (int g = 0; g < S::GR; ++g) { mbar_init(&bars->gate_full[i][g], 1); mbar_init(&bars->gate_empty[i][g], 1); }
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(&bars->tmem_base, S::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 8) {
    regs_increase<kSoftmaxRegs>();
    softmax_role<D, BQ, BK, CAUSAL, WRITE_MASK>(p, bars, tmem, w);
  } else {
    regs_decrease<kProducerRegs>();
    if (lane == 0) {
      if (warp == 8) kq_producer<D, BQ, BK>(&tm_q, &tm_k, smem, bars, w);
      else if (warp == 9) mma_issuer<D, BQ, BK>(smem, bars, tmem, w);
      else if (warp == 10) v_producer<D, BQ, BK>(&tm_v, smem, bars, w);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
  if (threadIdx.x == 0 && ((volatile int*)&bars->abort)[0]) atomicOr(p.status, 1);
}

}  // namespace bsfa
