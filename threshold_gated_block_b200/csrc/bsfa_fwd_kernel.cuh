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
// One CTA owns 128 query rows of one (batch, query head): one query tile when
// Bq = 128, two when Bq = 64. Warp roles (224 threads):
//   warps 0-3  softmax / gate / epilogue: thread r owns row r (TMEM lane r);
//   warp 4     TMEM allocation + TMA loads of Q (once) and of every K block;
//   warp 5     tcgen05.mma issue (one thread): S = Q K^T into TMEM, O += P V;
//   warp 6     TMA loads of V, issued only for blocks the gate kept.
// TMEM columns: S double buffer [0, 2*Bk), O [2*Bk, 2*Bk + D). P is written
// back as bf16 over the first Bk/2 columns of its S buffer and read from there
// as the A operand of the PV product.
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
  float scale;        // 1/sqrt(D): the gate compares s_max(raw) * scale against tau
  float scale_log2;   // log2(e)/sqrt(D): exponent scale of the softmax
};

// O is rescaled only when the running maximum grows by more than 2^8 in the
// exp2 domain; until then P is taken against the stale maximum (values <= 2^8,
// exact in the final O / l ratio).
constexpr float kRescaleThreshold = 8.0f;
constexpr int kThreads = 224;

template <int D, int BQ, int BK>
struct FwdShape {
  static constexpr int ROWS = 128;
  static constexpr int NSUB = ROWS / BQ;   // query tiles per CTA
  static constexpr int DCH = D / 64;       // 128-byte swizzle chunks along D
  static constexpr int KS = 3;             // K ring depth
  static constexpr int VS = 2;             // V ring depth
  static constexpr int GR = 4;             // gate-decision ring depth
  static constexpr uint32_t Q_BYTES = ROWS * D * 2;
  static constexpr uint32_t KV_BYTES = BK * D * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KS * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + VS * KV_BYTES;
  static constexpr uint32_t BAR_BYTES = 1024;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;   // + alignment slack
  static constexpr uint32_t TMEM_S0 = 0;
  static constexpr uint32_t TMEM_S1 = BK;
  static constexpr uint32_t TMEM_O = 2 * BK;
  static constexpr uint32_t TMEM_COLS = (2 * BK + D <= 256) ? 256 : 512;
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
  uint64_t s_full[2], p_full[2];
  uint64_t o_done;
  uint64_t gate_full[GR], gate_empty[GR];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int gate_flag[GR];
  int p_keep[2];
  float red[2][4];
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Bounded wait used when draining in-flight copies/MMAs on the way out: it does
// not give up early on the abort flag, only on the time limit.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  int local = 0;
  return mbar_wait(bar, parity, &local);
}

// ---------------------------------------------------------------------------- K/Q producer (warp 4, one thread)

template <int D, int BQ, int BK, typename Bars>
__device__ __forceinline__ void kq_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k, uint8_t* smem,
                                            Bars* bars, int b, int hq, int kvh, int q0, int nblk) {
  using S = FwdShape<D, BQ, BK>;
  volatile int* abort_flag = &bars->abort;
  prefetch_tensormap(tm_q);
  prefetch_tensormap(tm_k);
  mbar_arrive_expect_tx(&bars->q_full, S::Q_BYTES);
#pragma unroll
  for (int c = 0; c < S::DCH; ++c)
    tma_load_4d(smem + S::OFF_Q + c * (S::ROWS * 128), tm_q, &bars->q_full, c * 64, hq, q0, b);
  int issued = 0;
  for (int t = 0; t < nblk; ++t) {
    const int slot = t % S::KS;
    if (!mbar_wait(&bars->k_empty[slot], ((t / S::KS) & 1) ^ 1, abort_flag)) break;
    mbar_arrive_expect_tx(&bars->k_full[slot], S::KV_BYTES);
#pragma unroll
    for (int c = 0; c < S::DCH; ++c)
      tma_load_4d(smem + S::OFF_K + slot * S::KV_BYTES + c * (BK * 128), tm_k, &bars->k_full[slot], c * 64, kvh,
                  t * BK, b);
    issued = t + 1;
  }
  // Copies still in flight must land before the CTA exits.
  drain_wait(&bars->q_full, 0);
  for (int t = (issued > S::KS ? issued - S::KS : 0); t < issued; ++t)
    drain_wait(&bars->k_full[t % S::KS], (t / S::KS) & 1);
}

// ---------------------------------------------------------------------------- V producer (warp 6, one thread)

template <int D, int BQ, int BK, typename Bars>
__device__ __forceinline__ void v_producer(const CUtensorMap* tm_v, uint8_t* smem, Bars* bars, int b, int kvh,
                                           int nblk) {
  using S = FwdShape<D, BQ, BK>;
  volatile int* abort_flag = &bars->abort;
  volatile int* gate_flag = bars->gate_flag;
  prefetch_tensormap(tm_v);
  int v_count = 0;
  for (int j = 0; j < nblk; ++j) {
    const int g = j % S::GR;
    if (!mbar_wait(&bars->gate_full[g], (j / S::GR) & 1, abort_flag)) break;
    const int keep = gate_flag[g];
    mbar_arrive(&bars->gate_empty[g]);
    if (!keep) continue;            // skipped block: its values are never loaded
    const int slot = v_count % S::VS;
    if (!mbar_wait(&bars->v_empty[slot], ((v_count / S::VS) & 1) ^ 1, abort_flag)) break;
    mbar_arrive_expect_tx(&bars->v_full[slot], S::KV_BYTES);
#pragma unroll
    for (int c = 0; c < S::DCH; ++c)
      tma_load_4d(smem + S::OFF_V + slot * S::KV_BYTES + c * (BK * 128), tm_v, &bars->v_full[slot], c * 64, kvh,
                  j * BK, b);
    ++v_count;
  }
  for (int n = (v_count > S::VS ? v_count - S::VS : 0); n < v_count; ++n)
    drain_wait(&bars->v_full[n % S::VS], (n / S::VS) & 1);
}

// ---------------------------------------------------------------------------- MMA issuer (warp 5, one thread)

template <int D, int BQ, int BK, typename Bars>
__device__ __forceinline__ void mma_issuer(uint8_t* smem, Bars* bars, uint32_t tmem, int nblk) {
  using S = FwdShape<D, BQ, BK>;
  constexpr uint32_t IDESC_QK = make_idesc_bf16(128, BK, false);   // B = K tile, K-major
  constexpr uint32_t IDESC_PV = make_idesc_bf16(128, D, true);     // B = V tile, MN-major
  volatile int* abort_flag = &bars->abort;
  volatile int* p_keep = bars->p_keep;
  const uint32_t q_addr = smem_u32(smem + S::OFF_Q);

  auto issue_qk = [&](int t) -> bool {
    const int slot = t % S::KS;
    if (!mbar_wait(&bars->k_full[slot], (t / S::KS) & 1, abort_flag)) return false;
    tc_fence_after();
    const uint32_t k_addr = smem_u32(smem + S::OFF_K + slot * S::KV_BYTES);
    const uint32_t d_tmem = tmem + ((t & 1) ? S::TMEM_S1 : S::TMEM_S0);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t ch = kk / 4, koff = (kk % 4) * 32;   // 16 bf16 = 32 bytes per K step
      const uint64_t a = make_sdesc_sw128(q_addr + ch * (S::ROWS * 128) + koff, 16, 1024);
      const uint64_t bd = make_sdesc_sw128(k_addr + ch * (BK * 128) + koff, 16, 1024);
      mma_ss(d_tmem, a, bd, IDESC_QK, kk > 0 ? 1u : 0u);
    }
    tc_commit(&bars->k_empty[slot]);
    tc_commit(&bars->s_full[t & 1]);
    return true;
  };

  if (mbar_wait(&bars->q_full, 0, abort_flag) && issue_qk(0)) {
    int v_count = 0, pv_count = 0;
    for (int j = 0; j < nblk; ++j) {
      if (j + 1 < nblk && !issue_qk(j + 1)) break;
      if (!mbar_wait(&bars->p_full[j & 1], (j >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      if (!p_keep[j & 1]) continue;          // skipped block: no PV product
      const int slot = v_count % S::VS;
      if (!mbar_wait(&bars->v_full[slot], (v_count / S::VS) & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t v_addr = smem_u32(smem + S::OFF_V + slot * S::KV_BYTES);
      const uint32_t p_tmem = tmem + ((j & 1) ? S::TMEM_S1 : S::TMEM_S0);
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        // 16 keys per K step: 16 rows of 128 bytes in V; 8 packed bf16x2 columns of P.
        const uint64_t bd = make_sdesc_sw128(v_addr + kk * 16 * 128, BK * 128, 1024);
        mma_ts(tmem + S::TMEM_O, p_tmem + kk * 8, bd, IDESC_PV, (pv_count > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(&bars->v_empty[slot]);
      tc_commit(&bars->o_done);
      ++v_count;
      ++pv_count;
    }
  }
  // Every MMA issued above must complete before TMEM is released.
  tc_commit(&bars->drain);
  drain_wait(&bars->drain, 0);
}

// ---------------------------------------------------------------------------- softmax / gate / epilogue (warps 0-3)

template <int D, int BQ, int BK, bool CAUSAL, bool WRITE_MASK, typename Bars>
__device__ __forceinline__ void softmax_role(const FwdParams& p, Bars* bars, uint32_t tmem, int b, int hq, int q0,
                                             int nblk) {
  using S = FwdShape<D, BQ, BK>;
  volatile int* abort_flag = &bars->abort;
  const int r = threadIdx.x;
  const int warp = r >> 5, lane = r & 31;
  const int qrow = q0 + r;
  const int sub = r / BQ;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const float tau = p.tau[hq];
  const int mq = p.N / BQ, mkv = p.N / BK;

  float m = -INFINITY;   // running maximum, exp2 domain
  float l = 0.f;         // running normaliser
  int pv_count = 0;      // PV products issued so far (one per block some tile kept)
  bool failed = false;

  for (int j = 0; j < nblk; ++j) {
    const int buf = j & 1;
    const uint32_t s_tmem = tmem + (buf ? S::TMEM_S1 : S::TMEM_S0) + lane_off;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[buf], (j >> 1) & 1, abort_flag));
    float sv[BK];
    float rmax = -INFINITY;
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < BK / 32; ++c) {
        uint32_t t[32];
        tmem_ld_x32(s_tmem + c * 32, t);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(t[e]);
      }
      if (CAUSAL && (j + 1) * BK - 1 > q0) {       // block straddles the causal boundary
#pragma unroll
        for (int c = 0; c < BK; ++c)
          if (j * BK + c > qrow) sv[c] = -INFINITY;
      }
#pragma unroll
      for (int c = 0; c < BK; ++c) rmax = fmaxf(rmax, sv[c]);
    }
    // Block maximum of each query tile: warp shuffle, then across the tile's warps.
    const float wmax = warp_max(rmax);
    if (lane == 0) bars->red[buf][warp] = wmax;
    if (named_barrier_or(1, 128, failed || !ok || *abort_flag)) {
      failed = true;
      break;
    }
    int code[S::NSUB];
    bool keep_any = false;
#pragma unroll
    for (int s = 0; s < S::NSUB; ++s) {
      float bm = -INFINITY;
#pragma unroll
      for (int w = s * (BQ / 32); w < (s + 1) * (BQ / 32); ++w) bm = fmaxf(bm, bars->red[buf][w]);
      const int lo = q0 + s * BQ, hi = lo + BQ - 1;
      const int k_lo = j * BK, k_hi = k_lo + BK - 1;
      const bool visible = !CAUSAL || k_lo <= hi;
      const bool diag = CAUSAL ? (visible && k_hi > lo) : (k_lo <= hi && k_hi >= lo);
      code[s] = !visible ? 3 : diag ? 2 : ((bm * p.scale >= tau) ? 1 : 0);
      keep_any |= (code[s] == 1 || code[s] == 2);
    }
    if (r == 0) {
      if (WRITE_MASK) {
#pragma unroll
        for (int s = 0; s < S::NSUB; ++s)
          if (code[s] != 3)
            p.mask[((size_t)(b * p.Hq + hq) * mq + (q0 / BQ + s)) * mkv + j] = (uint8_t)code[s];
      }
      // Publish the decision so the V tile (if kept) is fetched right away.
      const int g = j % S::GR;
      if (mbar_wait(&bars->gate_empty[g], ((j / S::GR) & 1) ^ 1, abort_flag)) {
        ((volatile int*)bars->gate_flag)[g] = keep_any ? 1 : 0;
        mbar_arrive(&bars->gate_full[g]);
      } else {
        failed = true;
      }
      ((volatile int*)bars->p_keep)[buf] = keep_any ? 1 : 0;
    }
    __syncwarp();
    if (!keep_any) {                 // skipped by every tile: release the S buffer, nothing else
      tc_fence_before();
      mbar_arrive(&bars->p_full[buf]);
      continue;
    }

    const bool my_keep = (code[sub] == 1 || code[sub] == 2);   // uniform within a warp
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
    const bool live = my_keep && (m != -INFINITY);
    const float neg_m = live ? -m : 0.f;
    float lsum = 0.f;
#pragma unroll
    for (int c = 0; c < BK / 32; ++c) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float p0 = 0.f, p1 = 0.f;
        if (live) {
          p0 = ex2_approx(fmaf(sv[c * 32 + 2 * e], p.scale_log2, neg_m));
          p1 = ex2_approx(fmaf(sv[c * 32 + 2 * e + 1], p.scale_log2, neg_m));
        }
        lsum += p0 + p1;
        pk[e] = pack_bf16x2(p0, p1);
      }
      tmem_st_x16(s_tmem + c * 16, pk);       // P (bf16 pairs) over the consumed S columns
    }
    l += lsum;
    tmem_st_wait();

    // The O rescale needs every earlier PV product finished.
    bool ok2 = true;
    if (pv_count > 0) ok2 = mbar_wait(&bars->o_done, (pv_count - 1) & 1, abort_flag);
    ok2 = __all_sync(0xffffffffu, ok2);
    if (!ok2) failed = true;
    if (ok2 && __any_sync(0xffffffffu, need_rescale)) {
      tc_fence_after();
      const uint32_t o_tmem = tmem + S::TMEM_O + lane_off;
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
    ++pv_count;
    tc_fence_before();
    mbar_arrive(&bars->p_full[buf]);
  }

  // Epilogue: O / l -> bf16 rows, lse = ln-sum-exp over the kept set.
  bool ok = !failed;
  if (ok && pv_count > 0) ok = mbar_wait(&bars->o_done, (pv_count - 1) & 1, abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
    tc_fence_after();
    const uint32_t o_tmem = tmem + S::TMEM_O + lane_off;
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

  // Work unit: heaviest causal tiles first; the query heads of one KV group are
  // neighbours in launch order so their K/V blocks are shared through L2.
  const int tiles = p.N / S::ROWS;
  const int bh = blockIdx.x % (p.B * p.Hq);
  const int t_lin = blockIdx.x / (p.B * p.Hq);
  const int qt = CAUSAL ? (tiles - 1 - t_lin) : t_lin;
  const int hq = bh % p.Hq, b = bh / p.Hq;
  const int kvh = hq / p.group;
  const int q0 = qt * S::ROWS;
  const int nblk = CAUSAL ? (q0 + S::ROWS) / BK : p.N / BK;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < S::KS; ++i) { mbar_init(&bars->k_full[i], 1); mbar_init(&bars->k_empty[i], 1); }
    for (int i = 0; i < S::VS; ++i) { mbar_init(&bars->v_full[i], 1); mbar_init(&bars->v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&bars->s_full[i], 1); mbar_init(&bars->p_full[i], 128); }
    mbar_init(&bars->o_done, 1);
    for (int i = 0; i < S::GR; ++i) { mbar_init(&bars->gate_full[i], 1); mbar_init(&bars->gate_empty[i], 1); }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(&bars->tmem_base, S::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
    softmax_role<D, BQ, BK, CAUSAL, WRITE_MASK>(p, bars, tmem, b, hq, q0, nblk);
  } else if (warp == 4) {
    if (lane == 0) kq_producer<D, BQ, BK>(&tm_q, &tm_k, smem, bars, b, hq, kvh, q0, nblk);
    __syncwarp();
  } else if (warp == 5) {
    if (lane == 0) mma_issuer<D, BQ, BK>(smem, bars, tmem, nblk);
    __syncwarp();
  } else {
    if (lane == 0) v_producer<D, BQ, BK>(&tm_v, smem, bars, b, kvh, nblk);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
  if (threadIdx.x == 0 && ((volatile int*)&bars->abort)[0]) atomicOr(p.status, 1);
}

}  // namespace bsfa
