// Kernel instantiation and launch for one head dimension (used by the per-D
// translation units so the 96 kernel variants compile in parallel).
#pragma once

#include <atomic>
#include <cstdint>

#include <cuda_runtime.h>

#include "bsfa_fwd_kernel.cuh"

namespace bsfa {

// Devices (bit per device index, at most 64) on which a kernel variant's
// dynamic shared-memory limit has been raised. The attribute is per device and
// function, so it is set on a variant's first launch on each device only.
template <int D, int BQ, int BK, bool CAUSAL, bool MASK, bool GAP, bool VARLEN>
struct VariantAttr {
  static inline std::atomic<uint64_t> ready{0};
};

template <int D, int BQ, int BK, bool CAUSAL, bool MASK, bool GAP, bool VARLEN = false>
cudaError_t launch_variant(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                           int grid, int dev, cudaStream_t stream) {
  using S = FwdShape<D, BQ, BK>;
  auto kern = bsfa_fwd_kernel<D, BQ, BK, CAUSAL, MASK, GAP, VARLEN>;
  const uint64_t bit = 1ull << (dev & 63);
  auto& ready = VariantAttr<D, BQ, BK, CAUSAL, MASK, GAP, VARLEN>::ready;
  if ((ready.load(std::memory_order_acquire) & bit) == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    ready.fetch_or(bit, std::memory_order_release);
  }
  kern<<<grid, kThreads, S::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                       int Bq, int Bk, bool causal, bool mask, int grid, int dev, cudaStream_t s) {
#define BSFA_CASE(BQ, BK)                                                                          \
  if (Bq == BQ && Bk == BK) {                                                                      \
    if (p.cu_seqlens != nullptr) {     /* packed sequences, threshold gate */                      \
      if (causal)                                                                                  \
        return mask ? launch_variant<D, BQ, BK, true, true, false, true>(tq, tk, tv, p, grid, dev, s)   \
                    : launch_variant<D, BQ, BK, true, false, false, true>(tq, tk, tv, p, grid, dev, s); \
      return mask ? launch_variant<D, BQ, BK, false, true, false, true>(tq, tk, tv, p, grid, dev, s)    \
                  : launch_variant<D, BQ, BK, false, false, false, true>(tq, tk, tv, p, grid, dev, s);  \
    }                                                                                              \
    if (p.gate_gap) {                                                                              \
      if (causal)                                                                                  \
        return mask ? launch_variant<D, BQ, BK, true, true, true>(tq, tk, tv, p, grid, dev, s)          \
                    : launch_variant<D, BQ, BK, true, false, true>(tq, tk, tv, p, grid, dev, s);        \
      return mask ? launch_variant<D, BQ, BK, false, true, true>(tq, tk, tv, p, grid, dev, s)           \
                  : launch_variant<D, BQ, BK, false, false, true>(tq, tk, tv, p, grid, dev, s);         \
    }                                                                                              \
    if (causal)                                                                                    \
      return mask ? launch_variant<D, BQ, BK, true, true, false>(tq, tk, tv, p, grid, dev, s)           \
                  : launch_variant<D, BQ, BK, true, false, false>(tq, tk, tv, p, grid, dev, s);         \
    return mask ? launch_variant<D, BQ, BK, false, true, false>(tq, tk, tv, p, grid, dev, s)            \
                : launch_variant<D, BQ, BK, false, false, false>(tq, tk, tv, p, grid, dev, s);          \
  }
  BSFA_CASE(64, 64)
  BSFA_CASE(64, 128)
  BSFA_CASE(128, 64)
  BSFA_CASE(128, 128)
#undef BSFA_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_d64(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, int, int,
                           bool, bool, int, int, cudaStream_t);
cudaError_t launch_fwd_d128(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, int, int,
                            bool, bool, int, int, cudaStream_t);

}  // namespace bsfa
