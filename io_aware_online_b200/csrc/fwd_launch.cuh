// fwd_launch.cuh -- instantiation and launch of the prefill kernel for one input
// dtype (included by fwd_f16.cu and fwd_bf16.cu so the two compile in parallel).
#pragma once

#include <algorithm>
#include <cstdlib>

#include "fwd_kernel.cuh"

namespace fa {

template <int D, int T, bool BF16, bool SOFTCAP, bool ALIBI, int EMU, bool FP8 = false,
          bool KV = false>
cudaError_t launch_fwd_inst(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int batch, int rows_q, cudaStream_t stream) {
  using Cfg = FwdCfg<D, T, FP8 ? 1 : 2>;
  auto kern = fwd_kernel<D, T, BF16, SOFTCAP, ALIBI, EMU, FP8, KV>;
  constexpr int smem = Cfg::kSmemAlloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess && T == 1)  // room for two CTAs per SM
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int n_units = (rows_q + T * kBM - 1) / (T * kBM);
  dim3 grid;
  if (p.persistent) {
    // as many CTAs as are resident at once (Cfg::kMinBlocks per SM), or fewer items
    const long n_pi = p.pair ? (n_units + 1) / 2 : n_units;
    const long items = static_cast<long>(batch) * p.H * n_pi;
    const long slots = static_cast<long>(p.sm_count) * Cfg::kMinBlocks;
    grid = dim3(static_cast<unsigned>(std::max(1L, std::min(items, slots))));
  } else {
    grid = p.tile_major ? dim3(static_cast<unsigned>(n_units), static_cast<unsigned>(p.H),
                               static_cast<unsigned>(batch))
                        : dim3(static_cast<unsigned>(p.H), static_cast<unsigned>(batch),
                               static_cast<unsigned>(n_units));
  }
  kern<<<grid, Cfg::kThreads, smem, stream>>>(tq, tk, tv, p);
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

// Query tiles per CTA at D = 64 (D = 128 always takes two); FA_FWD_TILES in the
// environment overrides (1 or 2).
inline int fwd_tiles_choice() {
  static const int env = [] {
    const char* e = std::getenv("FA_FWD_TILES");
    return e ? std::atoi(e) : -1;
  }();
  if (env == 1 || env == 2) return env;
  return 2;
}

// The same choice for the 8-bit path (default 2).
inline int fp8_exp2_emu_choice() {
  static const int env = [] {
    const char* e = std::getenv("FA_EXP2_EMU");
    return e ? std::atoi(e) : -1;
  }();
  if (env == 0 || env == 2 || env == 3 || env == 4) return env;
  return 2;
}

template <bool BF16>
cudaError_t launch_fwd_dtype(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const FwdParams& p, int d, int batch, int rows_q,
                             cudaStream_t stream) {
  const bool sc = p.softcap_log2 > 0.f;
  const bool al = p.alibi != nullptr;
  if (p.kv_mode) {  // KV-cache mode: two tiles, the default exponential split
#define FA_FWD_KV_CASE(DD, SC, AL, EM)                                                     \
  if (d == DD && sc == SC && al == AL)                                                     \
    return launch_fwd_inst<DD, 2, BF16, SC, AL, EM, false, true>(tq, tk, tv, p, batch, rows_q, \
                                                                 stream);
    FA_FWD_KV_CASE(64, false, false, 2)
    FA_FWD_KV_CASE(64, true, false, 0)
    FA_FWD_KV_CASE(64, false, true, 0)
    FA_FWD_KV_CASE(64, true, true, 0)
    FA_FWD_KV_CASE(128, false, false, 0)
    FA_FWD_KV_CASE(128, true, false, 0)
    FA_FWD_KV_CASE(128, false, true, 0)
    FA_FWD_KV_CASE(128, true, true, 0)
#undef FA_FWD_KV_CASE
    return cudaErrorInvalidValue;
  }
  const int emu = (sc || al) ? 0 : exp2_emu_choice(d);
  const int tiles = (d == 64) ? fwd_tiles_choice() : 2;
#define FA_FWD_CASE(DD, TT, SC, AL, EM)                                                    \
  if (d == DD && tiles == TT && sc == SC && al == AL && emu == EM)                         \
    return launch_fwd_inst<DD, TT, BF16, SC, AL, EM>(tq, tk, tv, p, batch, rows_q, stream);
  FA_FWD_CASE(64, 1, false, false, 0)
  FA_FWD_CASE(64, 1, false, false, 2)
  FA_FWD_CASE(64, 1, false, false, 3)
  FA_FWD_CASE(64, 1, false, false, 4)
  FA_FWD_CASE(64, 1, true, false, 0)
  FA_FWD_CASE(64, 1, false, true, 0)
  FA_FWD_CASE(64, 1, true, true, 0)
  FA_FWD_CASE(64, 2, false, false, 0)
  FA_FWD_CASE(64, 2, false, false, 2)
  FA_FWD_CASE(64, 2, false, false, 3)
  FA_FWD_CASE(64, 2, false, false, 4)
  FA_FWD_CASE(64, 2, true, false, 0)
  FA_FWD_CASE(64, 2, false, true, 0)
  FA_FWD_CASE(64, 2, true, true, 0)
  FA_FWD_CASE(128, 2, false, false, 0)
  FA_FWD_CASE(128, 2, false, false, 2)
  FA_FWD_CASE(128, 2, false, false, 3)
  FA_FWD_CASE(128, 2, false, false, 4)
  FA_FWD_CASE(128, 2, true, false, 0)
  FA_FWD_CASE(128, 2, false, true, 0)
  FA_FWD_CASE(128, 2, true, true, 0)
#undef FA_FWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fa
