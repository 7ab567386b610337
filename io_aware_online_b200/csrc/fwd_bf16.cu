// fwd_bf16.cu -- bf16 instantiations of the prefill kernel.
#include "fwd_launch.cuh"

namespace fa {
cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int d, int batch, int rows_q,
                            cudaStream_t stream) {
  return launch_fwd_dtype<true>(tq, tk, tv, p, d, batch, rows_q, stream);
}
}  // namespace fa
