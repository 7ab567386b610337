// bwd.cu -- launcher of the attention backward (kernels in bwd_kernel.cuh):
// dense batches here, packed varlen sequences in bwd_varlen.cu.
#include "bwd_kernel.cuh"

namespace fa {

cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tl, const CUtensorMap& td,
                       const BwdParams& p, bool bf16, int d, cudaStream_t stream) {
  if (p.cu_q != nullptr) return launch_bwd_varlen(tq, tk, tv, tdo, tl, td, p, bf16, d, stream);
  return launch_bwd_all<false>(tq, tk, tv, tdo, tl, td, p, bf16, d, stream);
}

}  // namespace fa
