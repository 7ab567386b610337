// append.cu -- in-place KV-cache append: the new keys and values of a decoding or
// chunked-prefill step are written after each sequence's cached keys (tag page
// "flash attention", section 3.3, flash_attn_with_kvcache with k and v given).
//
// Pure data movement, bound by HBM: each new (sequence, token, KV head) row of
// head_dim 16-bit values is copied once for K and once for V with 16-byte loads
// and stores, one thread per 16 bytes.  The destination of position x of sequence
// b is row x % page of pool block block_table[b, x / page] (paged cache) or row x
// of sequence b (contiguous cache).  Rows whose position or block lies outside the
// cache are skipped and reported in the device status word.
#include <cuda_runtime.h>

#include <cstdint>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads) kv_append_kernel(const AppendParams p) {
  const int vec_per_row = p.D / 8;  // 16-byte vectors per row
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * kAppendThreads + threadIdx.x;
  const int64_t rows = static_cast<int64_t>(p.B) * p.S_new * p.Hkv;
  const int64_t row = gid / vec_per_row;
  if (row >= rows) return;
  const int v = static_cast<int>(gid % vec_per_row);
  const int hk = static_cast<int>(row % p.Hkv);
  const int t = static_cast<int>((row / p.Hkv) % p.S_new);
  const int b = static_cast<int>(row / (static_cast<int64_t>(p.Hkv) * p.S_new));
  const int pos = p.cache_seqlens[b] + t;
  int64_t dst_row;  // row index in units of D elements
  if (p.block_table != nullptr) {
    if (pos < 0 || pos >= p.max_blocks * p.page_size) {
      if (v == 0) atomicOr(p.status, kDevBadLength);
      return;
    }
    const int blk = p.block_table[static_cast<int64_t>(b) * p.max_blocks + pos / p.page_size];
    if (blk < 0 || blk >= p.num_blocks) {
      if (v == 0) atomicOr(p.status, kDevBadBlock);
      return;
    }
    dst_row = (static_cast<int64_t>(blk) * p.page_size + pos % p.page_size) * p.Hkv + hk;
  } else {
    if (pos < 0 || pos >= p.seqlen_k_max) {
      if (v == 0) atomicOr(p.status, kDevBadLength);
      return;
    }
    dst_row = (static_cast<int64_t>(b) * p.seqlen_k_max + pos) * p.Hkv + hk;
  }
  const int64_t src = row * vec_per_row + v;  // k_new is [B, S_new, Hkv, D] = rows x D
  const int64_t dst = dst_row * vec_per_row + v;
  reinterpret_cast<uint4*>(p.k_cache)[dst] = reinterpret_cast<const uint4*>(p.k_new)[src];
  reinterpret_cast<uint4*>(p.v_cache)[dst] = reinterpret_cast<const uint4*>(p.v_new)[src];
}

cudaError_t launch_kv_append(const AppendParams& p, cudaStream_t stream) {
  const int64_t threads = static_cast<int64_t>(p.B) * p.S_new * p.Hkv * (p.D / 8);
  if (threads == 0) return cudaSuccess;
  const int64_t blocks = (threads + kAppendThreads - 1) / kAppendThreads;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  kv_append_kernel<<<static_cast<unsigned>(blocks), kAppendThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace fa
