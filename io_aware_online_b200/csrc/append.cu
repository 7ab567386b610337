// append.cu -- in-place KV-cache append: the new keys and values of a decoding or
// chunked-prefill step are written after each sequence's cached keys (tag page
// "flash attention", section 3.3, flash_attn_with_kvcache with k and v given).
//
// Pure data movement, bound by HBM.  A token's row over all KV heads (Hkv * D
// 16-bit values) is contiguous both in k_new / v_new and in the cache, so one warp
// copies one (sequence, token): it resolves the destination once and its lanes
// move the row as 16-byte vectors, several loads in flight each.  The destination
// of position x of sequence b is row x % page of pool block block_table[b, x / page]
// (paged cache) or row x of sequence b (contiguous cache).  Tokens whose position
// or block lies outside the cache are skipped and reported in the device status
// word.
#include <cuda_runtime.h>

#include <cstdint>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

constexpr int kAppendThreads = 256;  // 8 warps = 8 tokens per CTA
constexpr int kAppendUnroll = 4;      // 16-byte vectors per lane per round, K and V each

__global__ void __launch_bounds__(kAppendThreads) kv_append_kernel(const AppendParams p) {
  const int lane = threadIdx.x % 32;
  const int64_t tok = static_cast<int64_t>(blockIdx.x) * (kAppendThreads / 32) + threadIdx.x / 32;
  if (tok >= static_cast<int64_t>(p.B) * p.S_new) return;  // warp-uniform
  const int t = static_cast<int>(tok % p.S_new);
  const int b = static_cast<int>(tok / p.S_new);
  const int pos = p.cache_seqlens[b] + t;
  int64_t dst_tok;  // destination token row, in units of Hkv * D elements
  if (p.block_table != nullptr) {
    if (pos < 0 || pos >= p.max_blocks * p.page_size) {
      if (lane == 0) atomicOr(p.status, kDevBadLength);
      return;
    }
    const int blk = p.block_table[static_cast<int64_t>(b) * p.max_blocks + pos / p.page_size];
    if (blk < 0 || blk >= p.num_blocks) {
      if (lane == 0) atomicOr(p.status, kDevBadBlock);
      return;
    }
    dst_tok = static_cast<int64_t>(blk) * p.page_size + pos % p.page_size;
  } else {
    if (pos < 0 || pos >= p.seqlen_k_max) {
      if (lane == 0) atomicOr(p.status, kDevBadLength);
      return;
    }
    dst_tok = static_cast<int64_t>(b) * p.seqlen_k_max + pos;
  }
  const int nvec = p.Hkv * p.D / 8;  // 16-byte vectors per token row
  const uint4* ks = reinterpret_cast<const uint4*>(p.k_new) + tok * nvec;
  const uint4* vs = reinterpret_cast<const uint4*>(p.v_new) + tok * nvec;
  uint4* kd = reinterpret_cast<uint4*>(p.k_cache) + dst_tok * nvec;
  uint4* vd = reinterpret_cast<uint4*>(p.v_cache) + dst_tok * nvec;
  for (int base = 0; base < nvec; base += 32 * kAppendUnroll) {
    uint4 kr[kAppendUnroll], vr[kAppendUnroll];
#pragma unroll
    for (int u = 0; u < kAppendUnroll; ++u) {
      const int i = base + u * 32 + lane;
      if (i < nvec) {
        kr[u] = ks[i];
        vr[u] = vs[i];
      }
    }
#pragma unroll
    for (int u = 0; u < kAppendUnroll; ++u) {
      const int i = base + u * 32 + lane;
      if (i < nvec) {
        kd[i] = kr[u];
        vd[i] = vr[u];
      }
    }
  }
}

cudaError_t launch_kv_append(const AppendParams& p, cudaStream_t stream) {
  const int64_t tokens = static_cast<int64_t>(p.B) * p.S_new;
  if (tokens == 0) return cudaSuccess;
  const int64_t blocks = (tokens + kAppendThreads / 32 - 1) / (kAppendThreads / 32);
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  kv_append_kernel<<<static_cast<unsigned>(blocks), kAppendThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace fa
