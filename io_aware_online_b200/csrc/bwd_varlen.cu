// bwd_varlen.cu -- the attention backward over packed varlen sequences
// (cu_seqlens, section 3.2): the kernels of bwd_kernel.cuh with VARLEN set.
#include "bwd_kernel.cuh"

namespace fa {

cudaError_t launch_bwd_varlen(const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, const CUtensorMap& tdo,
                              const CUtensorMap& tl, const CUtensorMap& td, const BwdParams& p,
                              bool bf16, int d, cudaStream_t stream) {
  return launch_bwd_all<true>(tq, tk, tv, tdo, tl, td, p, bf16, d, stream);
}

}  // namespace fa
