// fa_internal.h -- launch parameters and launcher declarations shared by the
// host layer (fa_api.cu) and the kernel translation units.  Not installed.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// ---------------------------------------------------------------- prefill
struct FwdParams {
  void* out;                       // 16-bit output rows
  float* lse;                      // nullable
  int64_t o_sb, o_ss, o_sh;        // output element strides (batch, seq, head)
  const int32_t* cu_q;             // varlen offsets (NULL = dense)
  const int32_t* cu_k;
  int Sq, Sk;                      // dense: per-batch lengths; varlen: unused
  int H, G;                        // query heads, query heads per KV head
  int total_q;                     // varlen: packed query rows (LSE row stride)
  float scale_log2;                // softmax_scale * log2(e)
  float softcap_log2;              // softcap * log2(e)
  float tanh_k;                    // 2 * log2(e) * softmax_scale / softcap
  const float* alibi;              // [H] or NULL
  int causal, wl, wr;              // mask flags; -1 = unbounded window side
  int tile_major;                  // grid x = query tiles (no mask: equal work per tile)
  // persistent schedule (dense calls): CTA c takes items c, c + gridDim.x, ... of the
  // (batch, head, pair) order; pair: an item is units n-1-u and u of one head
  int persistent, pair, B;
  int sm_count;                    // SMs of the device (persistent grid size)
  float v_descale;                 // 8-bit inputs: O is multiplied by it (1 otherwise)
  // KV-cache mode (fa_fwd_kvcache with many query rows): K/V come from a paged pool
  // [num_blocks, page, Hkv, D] through block_table, or from a contiguous cache
  // [B, Sk, Hkv, D], in 64-row boxes; sequence b attends cache_seqlens[b] + k_add keys
  int kv_mode;
  const int32_t* block_table;      // [B, max_blocks] or NULL (contiguous cache)
  const int32_t* cache_seqlens;    // [B] or NULL (= Sk)
  int k_add, page_size, max_blocks, num_blocks;
  unsigned int* status;            // device status word
  uint64_t timeout_ns;             // bounded-wait limit
};

// ---------------------------------------------------------------- decode
struct DecodeParams {
  const void* q;                   // [B, Sq, H, D] contiguous
  void* out;                       // [B, Sq, H, D] (num_splits == 1)
  float* lse;                      // [B, H, Sq] or NULL (num_splits == 1)
  float* ws_o;                     // [splits, B, Sq, H, D] fp32 partials (num_splits > 1)
  float* ws_lse;                   // [splits, B, Sq, H]
  const int32_t* block_table;      // [B, max_blocks] or NULL (contiguous cache)
  const int32_t* cache_seqlens;    // [B] or NULL
  int k_add;                       // keys appended after cache_seqlens[b] by this call
  int B, Sq, H, Hkv, G, R;         // R = G * Sq query rows per KV head
  int max_blocks, page_size, num_blocks, seqlen_k_max;
  int unit;                        // tokens per split unit (page or 64)
  int num_splits;
  float scale_log2, softcap_log2, tanh_k;
  int has_softcap;
  const float* alibi;
  int causal, wl, wr;
  unsigned int* status;
  uint64_t timeout_ns;
  int sm_count;                    // persistent grid: CTAs per SM x sm_count (capped at items)
  unsigned int* item_counter;      // workspace word, zero at launch: next work item to claim
  // longest-first order of the sequences (int16, in the workspace header after the
  // counter), written by the prep kernel when B <= kDecOrderMax; NULL: natural order
  const int16_t* order;
};

// Sequences the decode prep kernel ranks: the order fits the workspace's 256-byte
// header after the counter (bytes 16 .. 255, int16 entries).
constexpr int kDecOrderMax = 120;

cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                          bool bf16, int d, cudaStream_t stream);
// Zeroes the decode's work-item counter and, when p.order is set, writes the
// longest-first order of the sequences (one small CTA, before launch_decode).
cudaError_t launch_decode_prep(const DecodeParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- KV append
struct AppendParams {
  void* k_cache;                   // paged pool [num_blocks, page, Hkv, D] or [B, Sk_max, Hkv, D]
  void* v_cache;
  const void* k_new;               // [B, S_new, Hkv, D] contiguous
  const void* v_new;
  const int32_t* block_table;      // [B, max_blocks] or NULL (contiguous cache)
  const int32_t* cache_seqlens;    // [B]: keys in the cache before the append
  int B, S_new, Hkv, D;
  int max_blocks, page_size, num_blocks, seqlen_k_max;
  unsigned int* status;
};

cudaError_t launch_kv_append(const AppendParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- combine
struct CombineParams {
  const float* op;                 // partial outputs
  const float* lp;                 // partial LSEs
  void* out;                       // [B, S, H, D] contiguous
  float* lse;                      // [B, H, S] or NULL
  int64_t op_s[5];                 // b, s, h, d, split
  int64_t lp_s[4];                 // b, s, h, split
  int B, S, H, D, splits;
  int out_dtype;                   // 0 fp16, 1 bf16, 2 fp32
};

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- backward
struct BwdParams {
  const void* out;                 // forward output O [B, Sq, H, D] (16-bit, contiguous)
  const void* dout;                // dO, same layout
  const float* lse;                // [B, H, Sq] (varlen [H, total_q]) natural-log LSE of the forward
  float* dvec;                     // [B, H, Sq] D = rowsum(dO * O) (workspace)
  float* lse2;                     // [B, H, Sq] LSE * log2(e) (workspace, after dvec)
  int sq_pad;                      // row stride of dvec / lse2: Sq rounded up to 4
  void* dq;                        // [B, Sq, H, D] 16-bit
  void* dk;                        // [B, Sk, Hkv, D] 16-bit
  void* dv;
  int B, Sq, Sk, H, Hkv, G;
  float scale;                     // softmax_scale
  float scale_log2;                // softmax_scale * log2(e)
  float softcap_log2;              // softcap * log2(e) (0: no softcap)
  float tanh_k;                    // 2 * log2(e) * softmax_scale / softcap
  const float* alibi;              // [H] or NULL
  int causal, wl, wr;
  // varlen (both non-NULL): sequence b owns rows cu_q[b] .. cu_q[b+1]-1 of the
  // packed [total_q, H, D] tensors (Sq = total_q, B = number of sequences)
  const int32_t* cu_q;
  const int32_t* cu_k;
  int rows_q, rows_k;              // the grid's per-sequence extents (varlen: max_seqlen)
  unsigned int* status;
  uint64_t timeout_ns;
};

cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tl, const CUtensorMap& td,
                       const BwdParams& p, bool bf16, int d, cudaStream_t stream);
cudaError_t launch_bwd_varlen(const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, const CUtensorMap& tdo,
                              const CUtensorMap& tl, const CUtensorMap& td, const BwdParams& p,
                              bool bf16, int d, cudaStream_t stream);

cudaError_t launch_wait_timeout_selftest(unsigned int* status, uint64_t timeout_ns,
                                         cudaStream_t stream);

// Sets the calling thread's fa_last_error() message; returns `code`.
int set_error(int code, const char* msg);

}  // namespace fa
