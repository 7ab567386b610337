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
  // exponential pairs (of 8) on the FMA pipe: the 8-bit path is bound by the
  // exponentials (its products take half the bf16 time); FA_EXP2_EMU overrides
  const int emu = (sc || al) ? 0 : fp8_exp2_emu_choice();
#define FA_FWD8_CASE(SC, AL, EM)                                                           \
  if (sc == SC && al == AL && emu == EM)                                                   \
    return launch_fwd_inst<128, 2, true, SC, AL, EM, true>(tq, tk, tv, p, batch, rows_q, stream);
  FA_FWD8_CASE(false, false, 0)
  FA_FWD8_CASE(false, false, 2)
  FA_FWD8_CASE(false, false, 3)
  FA_FWD8_CASE(false, false, 4)
  FA_FWD8_CASE(true, false, 0)
  FA_FWD8_CASE(false, true, 0)
  FA_FWD8_CASE(true, true, 0)
#undef FA_FWD8_CASE
  return cudaErrorInvalidValue;
}
}  // namespace fa
