// fwd_launch.cuh -- instantiation and launch of the prefill kernel for one input
// dtype (included by fwd_f16.cu and fwd_bf16.cu so the two compile in parallel).
#pragma once

#include <cstdlib>

#include "fwd_kernel.cuh"

namespace fa {

template <int D, bool BF16, bool SOFTCAP, bool ALIBI, int EMU>
cudaError_t launch_fwd_inst(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int batch, int n_pairs, cudaStream_t stream) {
  auto kern = fwd_kernel<D, BF16, SOFTCAP, ALIBI, EMU>;
  constexpr int smem = FwdCfg<D>::kSmemAlloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(p.H), static_cast<unsigned>(batch),
                  static_cast<unsigned>(n_pairs));
  kern<<<grid, kFwdThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

// Pairs (of every 8) whose exp2 runs on the FMA pipe when neither softcap nor
// ALiBi is on; FA_EXP2_EMU in the environment overrides (0, 2, 3 or 4).
inline int exp2_emu_choice(int d) {
  static const int env = [] {
    const char* e = std::getenv("FA_EXP2_EMU");
    return e ? std::atoi(e) : -1;
  }();
  if (env == 0 || env == 2 || env == 3 || env == 4) return env;
  return d == 64 ? 2 : 0;
}

template <bool BF16>
cudaError_t launch_fwd_dtype(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const FwdParams& p, int d, int batch, int n_pairs,
                             cudaStream_t stream) {
  const bool sc = p.softcap_log2 > 0.f;
  const bool al = p.alibi != nullptr;
  const int emu = (sc || al) ? 0 : exp2_emu_choice(d);
#define FA_FWD_CASE(DD, SC, AL, EM)                                                        \
  if (d == DD && sc == SC && al == AL && emu == EM)                                        \
    return launch_fwd_inst<DD, BF16, SC, AL, EM>(tq, tk, tv, p, batch, n_pairs, stream);
  FA_FWD_CASE(64, false, false, 0)
  FA_FWD_CASE(64, false, false, 2)
  FA_FWD_CASE(64, false, false, 3)
  FA_FWD_CASE(64, false, false, 4)
  FA_FWD_CASE(64, true, false, 0)
  FA_FWD_CASE(64, false, true, 0)
  FA_FWD_CASE(64, true, true, 0)
  FA_FWD_CASE(128, false, false, 0)
  FA_FWD_CASE(128, false, false, 2)
  FA_FWD_CASE(128, false, false, 3)
  FA_FWD_CASE(128, false, false, 4)
  FA_FWD_CASE(128, true, false, 0)
  FA_FWD_CASE(128, false, true, 0)
  FA_FWD_CASE(128, true, true, 0)
#undef FA_FWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fa
