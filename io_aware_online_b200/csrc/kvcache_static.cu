// kvcache_static.cu -- fa_fwd_kvcache_static: the split-KV decode without a
// caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run
// attention: code embedded in a host framework that owns every device allocation
// through its own pool and forbids side allocations, or a latency-critical
// serving loop where a cudaMalloc could synchronise the device.  For them this
// entry point takes its scratch (the decode kernel's work-item counter and the
// fp32 split partials) from one fixed array in device memory that the library
// defines below, instead of from a workspace argument.  It allocates nothing:
// no cudaMalloc, no cudaFree, no allocating library routine.
//
// Costs and rules of the fixed array:
// - it is kFaStaticScratchBytes (24 MiB) on every GPU where the library is
//   loaded, held until the process exits.  That holds the split partials of a
//   64-sequence, 32-head, head-dim-128 decode at up to 23 splits;
// - a call whose scratch need (fa_kvcache_workspace_size) exceeds it is
//   rejected with FA_ERR_WORKSPACE before anything is launched;
// - all calls share the array and it keeps the last call's contents; what must
//   start at zero (the work-item counter) is cleared by each call on its own
//   stream, so calls that overlap on the GPU race with each other and must be
//   serialised by the caller;
// - the first call on each device looks the array's device address up with
//   cudaGetSymbolAddress, with that device current; make that first call before
//   any stream capture.  The address is cached for the life of the process: after
//   a device reset (cudaDeviceReset, or the primary context released and made
//   again) the cached address is stale and this entry point must not be called.
#include <cuda_runtime.h>

#include <climits>
#include <cstdio>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

// 24 MiB, 256-byte aligned: the fixed scratch of fa_fwd_kvcache_static.
static constexpr size_t kFaStaticScratchBytes = size_t(24) << 20;
static __device__ __align__(256) unsigned char g_fa_static_scratch[kFaStaticScratchBytes];

namespace {
constexpr int kMaxDev = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDev] = {};

// Device address of the scratch array on the current device, looked up once per
// device (with that device current) and cached.
int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
    return fa::set_error(FA_ERR_CUDA, "fa_fwd_kvcache_static: no usable current CUDA device");
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (g_static_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_fa_static_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fa::set_error(FA_ERR_CUDA,
                           "fa_fwd_kvcache_static: cudaGetSymbolAddress of the scratch array failed");
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return FA_OK;
}
}  // namespace

extern "C" {

FA_API size_t fa_kvcache_static_scratch_bytes(void) { return kFaStaticScratchBytes; }

FA_API int fa_fwd_kvcache_static(const void* q, const void* k_cache, const void* v_cache,
                                 void* out, float* lse, int dtype, int batch, int seqlen_q,
                                 int num_heads, int num_heads_k, int head_dim,
                                 const int32_t* block_table, int max_blocks_per_seq,
                                 int page_size, int num_blocks, int seqlen_k_max,
                                 const int32_t* cache_seqlens, float softmax_scale, int causal,
                                 int window_left, int window_right, float softcap,
                                 const float* alibi_slopes, int num_splits, void* stream) {
  const bool paged = block_table != nullptr;
  // the arguments the size check reads are validated first, so that a malformed call
  // gets the same FA_ERR_INVALID_ARG as from fa_fwd_kvcache, not a scratch-size error
  const int64_t max_k64 = paged ? static_cast<int64_t>(max_blocks_per_seq) * page_size
                                : static_cast<int64_t>(seqlen_k_max);
  if (max_k64 < 0 || max_k64 > INT_MAX || num_splits < 0 || num_splits > 256)
    return fa::set_error(FA_ERR_INVALID_ARG,
                         "fa_fwd_kvcache_static: cache extent or num_splits out of range");
  const int max_k = static_cast<int>(max_k64);
  const size_t need = fa_kvcache_workspace_size(batch, seqlen_q, num_heads, num_heads_k,
                                                head_dim, max_k, paged ? page_size : 0,
                                                num_splits);
  if (need > kFaStaticScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "fa_fwd_kvcache_static: this call needs %zu bytes of scratch but the fixed array "
             "holds %zu; use fewer splits or fa_fwd_kvcache with a workspace",
             need, kFaStaticScratchBytes);
    return fa::set_error(FA_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  const int rc = static_scratch(&scratch);
  if (rc != FA_OK) return rc;
  return fa_fwd_kvcache(q, k_cache, v_cache, out, lse, dtype, batch, seqlen_q, num_heads,
                        num_heads_k, head_dim, block_table, max_blocks_per_seq, page_size,
                        num_blocks, seqlen_k_max, cache_seqlens, softmax_scale, causal,
                        window_left, window_right, softcap, alibi_slopes, num_splits, scratch,
                        kFaStaticScratchBytes, stream);
}

}  // extern "C"
