// fwd_launch.cuh -- instantiation and launch of the prefill kernel for one input
// dtype (included by fwd_f16.cu and fwd_bf16.cu so the two compile in parallel).
#pragma once

#include "fwd_kernel.cuh"

namespace fa {

template <int D, bool BF16, bool SOFTCAP, bool ALIBI>
cudaError_t launch_fwd_inst(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int batch, int n_pairs, cudaStream_t stream) {
  auto kern = fwd_kernel<D, BF16, SOFTCAP, ALIBI>;
  constexpr int smem = FwdCfg<D>::kSmemAlloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(p.H), static_cast<unsigned>(batch),
                  static_cast<unsigned>(n_pairs));
  kern<<<grid, kFwdThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <bool BF16>
cudaError_t launch_fwd_dtype(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const FwdParams& p, int d, int batch, int n_pairs,
                             cudaStream_t stream) {
  const bool sc = p.softcap_log2 > 0.f;
  const bool al = p.alibi != nullptr;
#define FA_FWD_CASE(DD, SC, AL)                                                            \
  if (d == DD && sc == SC && al == AL)                                                     \
    return launch_fwd_inst<DD, BF16, SC, AL>(tq, tk, tv, p, batch, n_pairs, stream);
  FA_FWD_CASE(64, false, false)
  FA_FWD_CASE(64, true, false)
  FA_FWD_CASE(64, false, true)
  FA_FWD_CASE(64, true, true)
  FA_FWD_CASE(128, false, false)
  FA_FWD_CASE(128, true, false)
  FA_FWD_CASE(128, false, true)
  FA_FWD_CASE(128, true, true)
#undef FA_FWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fa
