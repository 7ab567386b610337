// decode.cu -- instantiation and launch of the split-KV decode kernel.
#include <algorithm>

#include "decode_kernel.cuh"

namespace fa {

template <int D, bool BF16, int RMAX>
static cudaError_t launch_decode_inst(const CUtensorMap& tk, const CUtensorMap& tv,
                                      const DecodeParams& p, cudaStream_t stream) {
  auto kern = decode_kernel<D, BF16, RMAX>;
  constexpr int smem = DecCfg<D, RMAX>::kSmemAlloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  // persistent grid: as many CTAs as fit at once, each walking the item list
  const long items = static_cast<long>(p.B) * p.Hkv * p.num_splits;
  const long per_sm = (RMAX <= 4) ? 3 : 1;
  const long ctas = std::min(items, per_sm * std::max(1, p.sm_count));
  if (ctas <= 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(ctas), kDecThreads, smem, stream>>>(tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_decode_prep(const DecodeParams& p, cudaStream_t stream) {
  decode_prep_kernel<<<1, 128, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                          bool bf16, int d, cudaStream_t stream) {
  const int rmax = (p.R <= 4) ? 4 : 16;
#define FA_DEC_CASE(DD, BF, RM) \
  if (d == DD && bf16 == BF && rmax == RM) return launch_decode_inst<DD, BF, RM>(tk, tv, p, stream);
  FA_DEC_CASE(64, false, 4)
  FA_DEC_CASE(64, false, 16)
  FA_DEC_CASE(64, true, 4)
  FA_DEC_CASE(64, true, 16)
  FA_DEC_CASE(128, false, 4)
  FA_DEC_CASE(128, false, 16)
  FA_DEC_CASE(128, true, 4)
  FA_DEC_CASE(128, true, 16)
#undef FA_DEC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fa
