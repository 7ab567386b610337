// fwd_fp8.cu -- E4M3-input instantiations of the prefill kernel (D = 128, bf16
// output): both products on tcgen05.mma kind::f8f6f4.
#include "fwd_launch.cuh"

namespace fa {
cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const FwdParams& p, int d, int batch, int rows_q,
                           cudaStream_t stream) {
  if (d != 128) return cudaErrorInvalidValue;
  const bool sc = p.softcap_log2 > 0.f;
  const bool al = p.alibi != nullptr;
#define FA_FWD8_CASE(SC, AL)                                                               \
  if (sc == SC && al == AL)                                                                \
    return launch_fwd_inst<128, 2, true, SC, AL, 0, true>(tq, tk, tv, p, batch, rows_q, stream);
  FA_FWD8_CASE(false, false)
  FA_FWD8_CASE(true, false)
  FA_FWD8_CASE(false, true)
  FA_FWD8_CASE(true, true)
#undef FA_FWD8_CASE
  return cudaErrorInvalidValue;
}
}  // namespace fa
