// BSFA forward kernels, head dimension 64.
#include "bsfa_launch.cuh"

namespace bsfa {
cudaError_t launch_fwd_d64(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                           int Bq, int Bk, bool causal, bool mask, int grid, int dev, cudaStream_t s) {
  return launch_fwd<64>(tq, tk, tv, p, Bq, Bk, causal, mask, grid, dev, s);
}
}  // namespace bsfa
