// fa_api.cu -- the C ABI declared in include/fa.h: argument validation, TMA tensor
// descriptor encoding and kernel launches on the caller's stream.  No memory is
// allocated here; the only library state is the lazily resolved tensor-map
// encoder, per-device SM counts and the device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "fa.h"
#include "fa_internal.h"

namespace fa {
cudaError_t launch_fwd_f16(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                           const FwdParams&, int, int, int, cudaStream_t);
cudaError_t launch_fwd_bf16(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                            const FwdParams&, int, int, int, cudaStream_t);
cudaError_t launch_fwd_fp8(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                           const FwdParams&, int, int, int, cudaStream_t);
}  // namespace fa

// Device status word: kernels OR FA_DEV_* bits into it; fa_device_status reads it.
__device__ unsigned int g_fa_status_word;

namespace {

constexpr int kMaxDevices = 64;
thread_local std::string g_err;
std::atomic<int> g_timeout_ms{-1};
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
unsigned int* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

uint64_t timeout_ns() {
  int ms = g_timeout_ms.load();
  if (ms < 0) {
    const char* env = std::getenv("FA_WAIT_TIMEOUT_MS");
    ms = (env != nullptr && std::atoi(env) > 0) ? std::atoi(env) : 1000;
    g_timeout_ms.store(ms);
  }
  return static_cast<uint64_t>(ms) * 1000000ull;
}

// Per-device set-up: the status word's device address and the SM count.
int device_state(int* dev_out, unsigned int** status, int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_CUDA, "device ordinal %d too large", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_status_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_fa_status_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    g_sm_count[dev] = n;
    g_status_ptr[dev] = static_cast<unsigned int*>(ptr);
  }
  if (dev_out) *dev_out = dev;
  if (status) *status = g_status_ptr[dev];
  if (sms) *sms = g_sm_count[dev];
  return FA_OK;
}

int sm_count_or_default() {
  int sms = 0;
  if (device_state(nullptr, nullptr, &sms) != FA_OK || sms <= 0) return 148;
  return sms;
}

int get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode != nullptr) return FA_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
    return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return FA_OK;
}

// 4-D tiled map over 16-bit elements, 128-byte swizzle (box inner extent 64).
int encode_4d(CUtensorMap* map, const void* ptr, const uint64_t dims[4],
              const uint64_t strides_bytes[3], const uint32_t box[4], const char* what,
              bool bytes = false) {
  for (int i = 0; i < 3; ++i)
    if (strides_bytes[i] % 16 != 0 || strides_bytes[i] >= (1ull << 40) || strides_bytes[i] == 0)
      return fail(FA_ERR_INVALID_ARG, "%s: stride %d (%llu bytes) must be a positive multiple of 16",
                  what, i, static_cast<unsigned long long>(strides_bytes[i]));
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t gs[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
  cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
  CUresult r = g_encode(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16,
                        4, const_cast<void*>(ptr), gd, gs, bx,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_INVALID_ARG, "%s: tensor map encoding failed (%d)", what, (int)r);
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int resolve_scale(float in, int d, float* out) {
  const float s = std::isnan(in) ? 1.0f / std::sqrt(static_cast<float>(d)) : in;
  if (!(s >= 0.f) || std::isinf(s)) return fail(FA_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0 (or NaN for the default)");
  *out = s;
  return FA_OK;
}

int check_common(int dtype, int head_dim, int H, int Hkv, int wl, int wr, float softcap) {
  if (dtype != FA_FP16 && dtype != FA_BF16)
    return fail(FA_ERR_UNSUPPORTED, "dtype %d: only FA_FP16 and FA_BF16 inputs are supported", dtype);
  if (head_dim != 64 && head_dim != 128)
    return fail(FA_ERR_UNSUPPORTED, "head_dim %d: supported values are 64 and 128", head_dim);
  if (H <= 0 || Hkv <= 0 || H % Hkv != 0)
    return fail(FA_ERR_INVALID_ARG, "num_heads (%d) must be a positive multiple of num_heads_k (%d)", H, Hkv);
  if (wl < -1 || wr < -1)
    return fail(FA_ERR_INVALID_ARG, "window sizes must be >= -1 (got %d, %d)", wl, wr);
  if (!(softcap >= 0.f) || std::isinf(softcap))
    return fail(FA_ERR_INVALID_ARG, "softcap must be finite and >= 0");
  return FA_OK;
}

void fill_score_params(float scale, float softcap, float* scale_log2, float* softcap_log2,
                       float* tanh_k) {
  const float log2e = 1.4426950408889634f;
  // softmax_scale = 0 makes every score 0.  The kernels fold the scale into the
  // exponent and rely on it being positive (-inf * scale must stay -inf), so 0 is
  // evaluated as 1e-30: |score| * 1e-30 stays below 2^-24 for any fp16/bf16
  // input, so every exp2 is exactly 1.0f and the LSE moves by < 1e-18.
  if (scale == 0.f) scale = 1e-30f;
  *scale_log2 = scale * log2e;
  *softcap_log2 = softcap > 0.f ? softcap * log2e : 0.f;
  *tanh_k = softcap > 0.f ? 2.f * log2e * scale / softcap : 0.f;
}

// Largest split count: the combine kernel keeps one weight per split in shared
// memory (kCombineMaxSplits in combine.cu).
constexpr int kMaxSplits = 256;

int resolve_splits(int batch, int Sq, int H, int Hkv, int d, int max_seqlen_k, int unit,
                   int num_splits) {
  (void)Sq; (void)H; (void)d;
  if (batch < 0 || Hkv <= 0 || max_seqlen_k < 0 || unit <= 0 || num_splits < 0 ||
      num_splits > kMaxSplits)
    return -1;
  const int units = std::max(1, (max_seqlen_k + unit - 1) / unit);
  if (num_splits > 0) return std::min(num_splits, units);
  // heuristic: about eight work items per resident decode CTA (three per SM), so the
  // persistent CTAs finish together despite unequal sequence lengths
  const long ctas = std::max(1L, static_cast<long>(batch) * Hkv);
  const long want = 24L * sm_count_or_default();
  long s = (want + ctas - 1) / ctas;
  s = std::min<long>(s, std::min(units, 64));
  return static_cast<int>(std::max(1L, s));
}

}  // namespace

namespace fa {
// Error reporting for entry points defined in other translation units.
int set_error(int code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace fa

extern "C" {

const char* fa_last_error(void) { return g_err.c_str(); }

int fa_version(void) { return 100; }

int fa_set_wait_timeout_ms(int ms) {
  if (ms < 1) return fail(FA_ERR_INVALID_ARG, "timeout must be >= 1 ms");
  g_timeout_ms.store(ms);
  return FA_OK;
}

int fa_device_status(int clear, unsigned int* flags) {
  g_err.clear();
  int rc = device_state(nullptr, nullptr, nullptr);
  if (rc != FA_OK) return rc;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_fa_status_word, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (clear) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_fa_status_word, &z, sizeof(z));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
  }
  if (flags) *flags = v;
  if (v != 0) return fail(FA_ERR_DEVICE, "device status flags 0x%x", v);
  return FA_OK;
}

// fa_fwd's body; fp8: E4M3 q, k, v (head_dim 128), bf16 output, per-tensor descales.
static int fwd_impl(const void* q, const void* k, const void* v, void* out, float* lse, int dtype,
                    int batch, int seqlen_q, int seqlen_k, int num_heads, int num_heads_k,
                    int head_dim, const int64_t* q_strides, const int64_t* k_strides,
                    const int64_t* v_strides, const int64_t* o_strides,
                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int max_seqlen_q,
                    int max_seqlen_k, float softmax_scale, int causal, int window_left,
                    int window_right, float softcap, const float* alibi_slopes, void* stream,
                    bool fp8, float q_descale, float k_descale, float v_descale) {
  int rc = check_common(fp8 ? FA_BF16 : dtype, head_dim, num_heads, num_heads_k, window_left,
                        window_right, softcap);
  if (rc != FA_OK) return rc;
  if (fp8 && head_dim != 128)
    return fail(FA_ERR_UNSUPPORTED, "fa_fwd_fp8: head_dim %d (8-bit inputs need 128)", head_dim);
  if (fp8 && (!(q_descale > 0.f) || !(k_descale > 0.f) || !(v_descale > 0.f) ||
              std::isinf(q_descale) || std::isinf(k_descale) || std::isinf(v_descale)))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd_fp8: descale factors must be finite and > 0");
  const int in_align = fp8 ? 16 : 8;  // elements per 16 bytes of input
  if (!q || !k || !v || !out) return fail(FA_ERR_INVALID_ARG, "fa_fwd: q, k, v and out must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd: q, k, v and out must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd: lse must be 4-byte aligned");
  if (batch < 0 || seqlen_q < 0 || seqlen_k < 0)
    return fail(FA_ERR_INVALID_ARG, "fa_fwd: negative size");
  const bool varlen = cu_seqlens_q != nullptr || cu_seqlens_k != nullptr;
  if (varlen && (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd: varlen needs both cu_seqlens_q and cu_seqlens_k");
  if (varlen && (max_seqlen_q < 0 || max_seqlen_k < 0 || max_seqlen_q > seqlen_q || max_seqlen_k > seqlen_k))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd: max_seqlen must lie in [0, total rows]");
  float scale;
  if ((rc = resolve_scale(softmax_scale, head_dim, &scale)) != FA_OK) return rc;
  const int H = num_heads, Hkv = num_heads_k, d = head_dim;
  const int64_t dq[3] = {static_cast<int64_t>(std::max(seqlen_q, 1)) * H * d, static_cast<int64_t>(H) * d, d};
  const int64_t dk[3] = {static_cast<int64_t>(std::max(seqlen_k, 1)) * Hkv * d, static_cast<int64_t>(Hkv) * d, d};
  const int64_t* qs = q_strides ? q_strides : dq;
  const int64_t* ks = k_strides ? k_strides : dk;
  const int64_t* vs = v_strides ? v_strides : dk;
  const int64_t* os = o_strides ? o_strides : dq;
  for (int i = varlen ? 1 : 0; i < 3; ++i)
    if (qs[i] <= 0 || ks[i] <= 0 || vs[i] <= 0 || os[i] <= 0 || qs[i] % in_align ||
        ks[i] % in_align || vs[i] % in_align || os[i] % 8)
      return fail(FA_ERR_INVALID_ARG, "fa_fwd: strides must be positive multiples of 16 bytes");
  const int rows_q = varlen ? max_seqlen_q : seqlen_q;
  if (batch == 0 || rows_q == 0) return FA_OK;  // nothing to compute
  const int n_tiles = (rows_q + 127) / 128;
  if (batch > 65535 || n_tiles > 65535)
    return fail(FA_ERR_UNSUPPORTED, "fa_fwd: batch (%d) or query tiles (%d) above 65535", batch, n_tiles);
  if ((rc = get_encoder()) != FA_OK) return rc;
  unsigned int* status = nullptr;
  int sms = 0;
  if ((rc = device_state(nullptr, &status, &sms)) != FA_OK) return rc;

  CUtensorMap tq, tk, tv;
  // one 128-byte swizzle atom per row of the box: 64 16-bit or 128 8-bit elements
  const uint32_t box[4] = {fp8 ? 128u : 64u, 128, 1, 1};
  const uint64_t eb = fp8 ? 1 : 2;  // bytes per input element
  const uint64_t nb = varlen ? 1 : static_cast<uint64_t>(batch);
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(d), static_cast<uint64_t>(std::max(seqlen_q, 1)),
                              static_cast<uint64_t>(H), nb};
    const uint64_t st[3] = {static_cast<uint64_t>(qs[1]) * eb, static_cast<uint64_t>(qs[2]) * eb,
                            varlen ? static_cast<uint64_t>(qs[1]) * eb * std::max(seqlen_q, 1)
                                   : static_cast<uint64_t>(qs[0]) * eb};
    if ((rc = encode_4d(&tq, q, dims, st, box, "q", fp8)) != FA_OK) return rc;
  }
  const int64_t* kvs[2] = {ks, vs};
  const void* kvp[2] = {k, v};
  CUtensorMap* kvm[2] = {&tk, &tv};
  for (int t = 0; t < 2; ++t) {
    const uint64_t dims[4] = {static_cast<uint64_t>(d), static_cast<uint64_t>(std::max(seqlen_k, 1)),
                              static_cast<uint64_t>(Hkv), nb};
    const uint64_t st[3] = {static_cast<uint64_t>(kvs[t][1]) * eb, static_cast<uint64_t>(kvs[t][2]) * eb,
                            varlen ? static_cast<uint64_t>(kvs[t][1]) * eb * std::max(seqlen_k, 1)
                                   : static_cast<uint64_t>(kvs[t][0]) * eb};
    if ((rc = encode_4d(kvm[t], kvp[t], dims, st, box, t == 0 ? "k" : "v", fp8)) != FA_OK)
      return rc;
  }

  fa::FwdParams p{};
  p.out = out;
  p.lse = lse;
  p.o_sb = varlen ? 0 : os[0];
  p.o_ss = os[1];
  p.o_sh = os[2];
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.Sq = seqlen_q;
  p.Sk = seqlen_k;
  p.H = H;
  p.G = H / Hkv;
  p.total_q = seqlen_q;
  // 8-bit inputs: the scores carry q_descale * k_descale, folded into the scale
  fill_score_params(fp8 ? scale * q_descale * k_descale : scale, softcap, &p.scale_log2,
                    &p.softcap_log2, &p.tanh_k);
  p.v_descale = fp8 ? v_descale : 1.f;
  p.alibi = alibi_slopes;
  p.causal = causal ? 1 : 0;
  p.wl = window_left;
  p.wr = window_right;
  p.tile_major = (!causal && window_left < 0 && window_right < 0) ? 1 : 0;
  // dense calls run a persistent grid; under a mask the work of a unit grows with
  // its row index, and pairing the heaviest unit with the lightest evens it out
  p.persistent = varlen ? 0 : 1;
  p.pair = (causal || window_left >= 0 || window_right >= 0) ? 1 : 0;
  p.B = batch;
  p.sm_count = sms;
  p.status = status;
  p.timeout_ns = timeout_ns();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = fp8 ? fa::launch_fwd_fp8(tq, tk, tv, p, d, batch, rows_q, st)
                  : (dtype == FA_BF16)
                      ? fa::launch_fwd_bf16(tq, tk, tv, p, d, batch, rows_q, st)
                      : fa::launch_fwd_f16(tq, tk, tv, p, d, batch, rows_q, st);
  if (e != cudaSuccess) return cuda_fail(e, "fa_fwd launch");
  return FA_OK;
}

int fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int dtype,
           int batch, int seqlen_q, int seqlen_k, int num_heads, int num_heads_k, int head_dim,
           const int64_t* q_strides, const int64_t* k_strides, const int64_t* v_strides,
           const int64_t* o_strides, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
           int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal, int window_left,
           int window_right, float softcap, const float* alibi_slopes, void* stream) {
  g_err.clear();
  return fwd_impl(q, k, v, out, lse, dtype, batch, seqlen_q, seqlen_k, num_heads, num_heads_k,
                  head_dim, q_strides, k_strides, v_strides, o_strides, cu_seqlens_q,
                  cu_seqlens_k, max_seqlen_q, max_seqlen_k, softmax_scale, causal, window_left,
                  window_right, softcap, alibi_slopes, stream, false, 1.f, 1.f, 1.f);
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse,
               float q_descale, float k_descale, float v_descale, int batch, int seqlen_q,
               int seqlen_k, int num_heads, int num_heads_k, int head_dim,
               const int64_t* q_strides, const int64_t* k_strides, const int64_t* v_strides,
               const int64_t* o_strides, const int32_t* cu_seqlens_q,
               const int32_t* cu_seqlens_k, int max_seqlen_q, int max_seqlen_k,
               float softmax_scale, int causal, int window_left, int window_right,
               float softcap, const float* alibi_slopes, void* stream) {
  g_err.clear();
  return fwd_impl(q, k, v, out, lse, FA_BF16, batch, seqlen_q, seqlen_k, num_heads, num_heads_k,
                  head_dim, q_strides, k_strides, v_strides, o_strides, cu_seqlens_q,
                  cu_seqlens_k, max_seqlen_q, max_seqlen_k, softmax_scale, causal, window_left,
                  window_right, softcap, alibi_slopes, stream, true, q_descale, k_descale,
                  v_descale);
}

// Query rows per KV head above which fa_fwd_kvcache runs the tensor-core prefill
// kernel over the cache instead of the split-KV decode kernel.
static constexpr int kDecodeMaxRows = 16;

static bool kvcache_uses_prefill(int seqlen_q, int num_heads, int num_heads_k) {
  return num_heads_k > 0 &&
         static_cast<long>(num_heads / num_heads_k) * seqlen_q > kDecodeMaxRows;
}

int fa_kvcache_num_splits(int batch, int seqlen_q, int num_heads, int num_heads_k, int head_dim,
                          int max_seqlen_k, int page_size, int num_splits) {
  if (num_splits < 0 || num_splits > kMaxSplits) return -1;
  if (kvcache_uses_prefill(seqlen_q, num_heads, num_heads_k)) return 1;  // no split partials
  const int unit = page_size > 0 ? page_size : 64;
  return resolve_splits(batch, seqlen_q, num_heads, num_heads_k, head_dim, max_seqlen_k, unit,
                        num_splits);
}

// Workspace layout: a 256-byte header (word 0: the decode kernel's work-item counter,
// zeroed at every call; bytes 16 .. 255: the longest-first order of up to 120
// sequences, int16) followed, when the split count is above 1, by the fp32 partial
// outputs [splits, B, Sq, H, D] and partial LSEs [splits, B, Sq, H].
static constexpr size_t kWsHeader = 256;

size_t fa_kvcache_workspace_size(int batch, int seqlen_q, int num_heads, int num_heads_k,
                                 int head_dim, int max_seqlen_k, int page_size, int num_splits) {
  const int s = fa_kvcache_num_splits(batch, seqlen_q, num_heads, num_heads_k, head_dim,
                                      max_seqlen_k, page_size, num_splits);
  if (s <= 0 || batch <= 0 || seqlen_q <= 0 || num_heads <= 0 || head_dim <= 0) return kWsHeader;
  if (s == 1) return kWsHeader;
  return kWsHeader +
         static_cast<size_t>(s) * batch * seqlen_q * num_heads * (head_dim + 1) * sizeof(float);
}

// fa_fwd_kvcache's body.  `app` (optional) is an append of k_add new keys per
// sequence, launched on the same stream once every argument has been checked.
static int kvcache_impl(const void* q, const void* k_cache, const void* v_cache, void* out,
                        float* lse, int dtype, int batch, int seqlen_q, int num_heads,
                        int num_heads_k, int head_dim, const int32_t* block_table,
                        int max_blocks_per_seq, int page_size, int num_blocks, int seqlen_k_max,
                        const int32_t* cache_seqlens, float softmax_scale, int causal,
                        int window_left, int window_right, float softcap,
                        const float* alibi_slopes, int num_splits, void* workspace,
                        size_t workspace_bytes, void* stream, fa::AppendParams* app) {
  int rc = check_common(dtype, head_dim, num_heads, num_heads_k, window_left, window_right, softcap);
  if (rc != FA_OK) return rc;
  if (!k_cache || !v_cache || ((!q || !out) && batch > 0 && seqlen_q > 0))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd_kvcache: q, k_cache, v_cache and out must be non-NULL");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd_kvcache: q, caches and out must be 16-byte aligned");
  if (batch < 0 || seqlen_q < 0 || num_splits < 0)
    return fail(FA_ERR_INVALID_ARG, "fa_fwd_kvcache: negative size");
  if (num_splits > kMaxSplits)
    return fail(FA_ERR_INVALID_ARG, "fa_fwd_kvcache: num_splits must be in [0, %d]", kMaxSplits);
  const int H = num_heads, Hkv = num_heads_k, d = head_dim, G = H / Hkv;
  const bool use_prefill = kvcache_uses_prefill(seqlen_q, H, Hkv);
  const bool paged = block_table != nullptr;
  int max_k, unit;
  if (paged) {
    if (page_size <= 0 || page_size % 64 != 0)
      return fail(FA_ERR_INVALID_ARG, "fa_fwd_kvcache: page_size must be a positive multiple of 64");
    if (num_blocks <= 0 || max_blocks_per_seq <= 0)
      return fail(FA_ERR_INVALID_ARG, "fa_fwd_kvcache: num_blocks and max_blocks_per_seq must be positive");
    if (cache_seqlens == nullptr)
      return fail(FA_ERR_INVALID_ARG, "fa_fwd_kvcache: a paged cache needs cache_seqlens");
    if (static_cast<int64_t>(max_blocks_per_seq) * page_size > INT_MAX)
      return fail(FA_ERR_INVALID_ARG, "fa_fwd_kvcache: max_blocks_per_seq * page_size overflows int");
    max_k = max_blocks_per_seq * page_size;
    unit = page_size;
  } else {
    if (seqlen_k_max < 0) return fail(FA_ERR_INVALID_ARG, "fa_fwd_kvcache: seqlen_k_max < 0");
    max_k = seqlen_k_max;
    unit = 64;
  }
  float scale;
  if ((rc = resolve_scale(softmax_scale, d, &scale)) != FA_OK) return rc;
  if (batch > 65535 || Hkv > 65535)
    return fail(FA_ERR_UNSUPPORTED, "fa_fwd_kvcache: batch or num_heads_k above 65535");
  if (batch == 0) return FA_OK;
  if (seqlen_q == 0) {  // nothing to attend; an append still happens
    if (app == nullptr) return FA_OK;
    unsigned int* st0 = nullptr;
    if ((rc = device_state(nullptr, &st0, nullptr)) != FA_OK) return rc;
    app->status = st0;
    const cudaError_t e0 = fa::launch_kv_append(*app, static_cast<cudaStream_t>(stream));
    return e0 == cudaSuccess ? FA_OK : cuda_fail(e0, "fa_fwd_kvcache_append append launch");
  }
  const size_t need = fa_kvcache_workspace_size(batch, seqlen_q, H, Hkv, d, max_k,
                                                paged ? page_size : 0, num_splits);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace))
    return fail(FA_ERR_WORKSPACE, "fa_fwd_kvcache: needs %zu bytes of 16-byte aligned workspace (got %zu)",
                need, workspace_bytes);
  if ((rc = get_encoder()) != FA_OK) return rc;
  unsigned int* status = nullptr;
  int sms = 0;
  if ((rc = device_state(nullptr, &status, &sms)) != FA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (app != nullptr) app->status = status;

  if (use_prefill) {
    // many query rows per KV head (chunked prefill against the cache): the tcgen05
    // prefill kernel, K/V read from the cache in 64-row boxes
    if (seqlen_q > 65535 * 128)
      return fail(FA_ERR_UNSUPPORTED, "fa_fwd_kvcache: seqlen_q %d too large", seqlen_q);
    CUtensorMap tq, tk, tv;
    {
      const uint32_t box[4] = {64, 128, 1, 1};
      const uint64_t dims[4] = {static_cast<uint64_t>(d), static_cast<uint64_t>(seqlen_q),
                                static_cast<uint64_t>(H), static_cast<uint64_t>(batch)};
      const uint64_t st[3] = {static_cast<uint64_t>(H) * d * 2, static_cast<uint64_t>(d) * 2,
                              static_cast<uint64_t>(seqlen_q) * H * d * 2};
      if ((rc = encode_4d(&tq, q, dims, st, box, "q")) != FA_OK) return rc;
    }
    {
      const uint32_t box[4] = {64, 64, 1, 1};
      const uint64_t rows = paged ? page_size : std::max(seqlen_k_max, 1);
      const uint64_t dims[4] = {static_cast<uint64_t>(d), rows, static_cast<uint64_t>(Hkv),
                                static_cast<uint64_t>(paged ? num_blocks : batch)};
      const uint64_t st[3] = {static_cast<uint64_t>(Hkv) * d * 2, static_cast<uint64_t>(d) * 2,
                              rows * Hkv * d * 2};
      if ((rc = encode_4d(&tk, k_cache, dims, st, box, "k_cache")) != FA_OK) return rc;
      if ((rc = encode_4d(&tv, v_cache, dims, st, box, "v_cache")) != FA_OK) return rc;
    }
    fa::FwdParams f{};
    f.out = out;
    f.lse = lse;
    f.o_sb = static_cast<int64_t>(seqlen_q) * H * d;
    f.o_ss = static_cast<int64_t>(H) * d;
    f.o_sh = d;
    f.Sq = seqlen_q;
    f.Sk = paged ? 0 : seqlen_k_max;
    f.H = H;
    f.G = G;
    f.total_q = seqlen_q;
    fill_score_params(scale, softcap, &f.scale_log2, &f.softcap_log2, &f.tanh_k);
    f.alibi = alibi_slopes;
    f.causal = causal ? 1 : 0;
    f.wl = window_left;
    f.wr = window_right;
    f.tile_major = (!causal && window_left < 0 && window_right < 0) ? 1 : 0;
    f.status = status;
    f.timeout_ns = timeout_ns();
    f.kv_mode = 1;
    f.block_table = block_table;
    f.cache_seqlens = cache_seqlens;
    f.k_add = app ? app->S_new : 0;
    f.page_size = page_size;
    f.max_blocks = max_blocks_per_seq;
    f.num_blocks = num_blocks;
    cudaError_t e = cudaSuccess;
    if (app != nullptr && (e = fa::launch_kv_append(*app, s)) != cudaSuccess)
      return cuda_fail(e, "fa_fwd_kvcache_append append launch");
    e = (dtype == FA_BF16) ? fa::launch_fwd_bf16(tq, tk, tv, f, d, batch, seqlen_q, s)
                           : fa::launch_fwd_f16(tq, tk, tv, f, d, batch, seqlen_q, s);
    if (e != cudaSuccess) return cuda_fail(e, "fa_fwd_kvcache prefill launch");
    return FA_OK;
  }
  const int splits = resolve_splits(batch, seqlen_q, H, Hkv, d, max_k, unit, num_splits);

  CUtensorMap tk, tv;
  const uint32_t box[4] = {64, 1, 64, 1};
  uint64_t dims[4], st[3];
  dims[0] = d;
  dims[1] = Hkv;
  st[0] = static_cast<uint64_t>(d) * 2;
  st[1] = static_cast<uint64_t>(Hkv) * d * 2;
  if (paged) {
    dims[2] = page_size;
    dims[3] = num_blocks;
    st[2] = static_cast<uint64_t>(page_size) * Hkv * d * 2;
  } else {
    dims[2] = std::max(seqlen_k_max, 1);
    dims[3] = batch;
    st[2] = static_cast<uint64_t>(std::max(seqlen_k_max, 1)) * Hkv * d * 2;
  }
  if ((rc = encode_4d(&tk, k_cache, dims, st, box, "k_cache")) != FA_OK) return rc;
  if ((rc = encode_4d(&tv, v_cache, dims, st, box, "v_cache")) != FA_OK) return rc;

  fa::DecodeParams p{};
  p.q = q;
  p.out = out;
  p.lse = lse;
  float* ws_parts = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWsHeader);
  p.ws_o = splits > 1 ? ws_parts : nullptr;
  p.ws_lse = splits > 1 ? ws_parts + static_cast<size_t>(splits) * batch * seqlen_q * H * d
                        : nullptr;
  p.item_counter = static_cast<unsigned int*>(workspace);
  p.block_table = block_table;
  p.cache_seqlens = cache_seqlens;
  p.k_add = app ? app->S_new : 0;
  p.B = batch;
  p.Sq = seqlen_q;
  p.H = H;
  p.Hkv = Hkv;
  p.G = G;
  p.R = G * seqlen_q;
  p.max_blocks = max_blocks_per_seq;
  p.page_size = page_size;
  p.num_blocks = num_blocks;
  p.seqlen_k_max = seqlen_k_max;
  p.unit = unit;
  p.num_splits = splits;
  fill_score_params(scale, softcap, &p.scale_log2, &p.softcap_log2, &p.tanh_k);
  p.has_softcap = softcap > 0.f ? 1 : 0;
  p.alibi = alibi_slopes;
  p.causal = causal ? 1 : 0;
  p.wl = window_left;
  p.wr = window_right;
  p.status = status;
  p.timeout_ns = timeout_ns();
  p.sm_count = sms;
  cudaError_t e;
  if (app != nullptr) {
    e = fa::launch_kv_append(*app, s);
    if (e != cudaSuccess) return cuda_fail(e, "fa_fwd_kvcache_append append launch");
  }
  // the counter is zeroed and, for batches of up to kDecOrderMax sequences, their
  // longest-first order written after it (one small kernel before the split kernel)
  p.order = (cache_seqlens != nullptr && batch <= fa::kDecOrderMax)
                ? reinterpret_cast<const int16_t*>(static_cast<uint8_t*>(workspace) + 16)
                : nullptr;
  e = fa::launch_decode_prep(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "fa_fwd_kvcache prep launch");
  e = fa::launch_decode(tk, tv, p, dtype == FA_BF16, d, s);
  if (e != cudaSuccess) return cuda_fail(e, "fa_fwd_kvcache split kernel launch");
  if (splits > 1) {
    fa::CombineParams c{};
    c.op = p.ws_o;
    c.lp = p.ws_lse;
    c.out = out;
    c.lse = lse;
    const int64_t rows = static_cast<int64_t>(batch) * seqlen_q * H;
    c.op_s[0] = static_cast<int64_t>(seqlen_q) * H * d;
    c.op_s[1] = static_cast<int64_t>(H) * d;
    c.op_s[2] = d;
    c.op_s[3] = 1;
    c.op_s[4] = rows * d;
    c.lp_s[0] = static_cast<int64_t>(seqlen_q) * H;
    c.lp_s[1] = H;
    c.lp_s[2] = 1;
    c.lp_s[3] = rows;
    c.B = batch;
    c.S = seqlen_q;
    c.H = H;
    c.D = d;
    c.splits = splits;
    c.out_dtype = dtype;
    e = fa::launch_combine(c, s);
    if (e != cudaSuccess) return cuda_fail(e, "fa_fwd_kvcache combine launch");
  }
  return FA_OK;
}

// Backward workspace: D and LSE * log2(e), each [batch * num_heads rows, seqlen_q
// rounded up to 4] fp32 (16-byte rows for the tensor maps that load them).
size_t fa_bwd_workspace_size(int batch, int seqlen_q, int num_heads) {
  if (batch <= 0 || seqlen_q <= 0 || num_heads <= 0) return 256;
  const size_t half = static_cast<size_t>(batch) * num_heads * ((seqlen_q + 3) / 4 * 4) *
                      sizeof(float);
  return (2 * half + 255) / 256 * 256;
}

// 2-D fp32 tensor map over [rows, cols] with a row stride in bytes, box {box_cols, 1}
// (box_cols * 4 a multiple of 16 bytes).
static int encode_vec_rows(CUtensorMap* map, const void* ptr, uint64_t cols, uint64_t rows,
                           uint64_t stride_bytes, uint32_t box_cols, const char* what) {
  cuuint64_t gd[2] = {cols, rows};
  cuuint64_t gs[1] = {stride_bytes};
  cuuint32_t bx[2] = {box_cols, 1};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), gd, gs,
                        bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_INVALID_ARG, "%s: tensor map encoding failed (%d)", what, (int)r);
  return FA_OK;
}

int fa_bwd(const void* dout, const void* q, const void* k, const void* v, const void* out,
           const float* lse, void* dq, void* dk, void* dv, int dtype, int batch, int seqlen_q,
           int seqlen_k, int num_heads, int num_heads_k, int head_dim,
           const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int max_seqlen_q,
           int max_seqlen_k, float softmax_scale, int causal, int window_left, int window_right,
           float softcap, const float* alibi_slopes, void* workspace, size_t workspace_bytes,
           void* stream) {
  g_err.clear();
  int rc = check_common(dtype, head_dim, num_heads, num_heads_k, window_left, window_right, softcap);
  if (rc != FA_OK) return rc;
  const bool varlen = cu_seqlens_q != nullptr || cu_seqlens_k != nullptr;
  if (varlen && (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr))
    return fail(FA_ERR_INVALID_ARG, "fa_bwd: varlen needs both cu_seqlens_q and cu_seqlens_k");
  if (varlen && (max_seqlen_q < 0 || max_seqlen_k < 0 || max_seqlen_q > seqlen_q ||
                 max_seqlen_k > seqlen_k))
    return fail(FA_ERR_INVALID_ARG, "fa_bwd: max_seqlen must lie in [0, total rows]");
  if (!dout || !q || !k || !v || !out || !lse || !dq || !dk || !dv)
    return fail(FA_ERR_INVALID_ARG, "fa_bwd: every tensor argument must be non-NULL");
  if (!aligned16(dout) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(FA_ERR_INVALID_ARG, "fa_bwd: 16-byte aligned tensors (lse 4-byte) required");
  if (batch < 0 || seqlen_q < 0 || seqlen_k < 0)
    return fail(FA_ERR_INVALID_ARG, "fa_bwd: negative size");
  float scale;
  if ((rc = resolve_scale(softmax_scale, head_dim, &scale)) != FA_OK) return rc;
  const int H = num_heads, Hkv = num_heads_k, d = head_dim;
  // tensors, maps and statistics of a varlen call are those of one packed batch entry
  const int bm = varlen ? 1 : batch;
  const size_t need = fa_bwd_workspace_size(bm, seqlen_q, H);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace))
    return fail(FA_ERR_WORKSPACE, "fa_bwd: needs %zu bytes of 16-byte aligned workspace (got %zu)",
                need, workspace_bytes);
  if (batch == 0 || (seqlen_q == 0 && seqlen_k == 0)) return FA_OK;
  if (seqlen_q == 0 || seqlen_k == 0) {  // nothing attends: every gradient is zero
    cudaStream_t s0 = static_cast<cudaStream_t>(stream);
    cudaError_t e0 = cudaSuccess;
    if (seqlen_k > 0) {
      const size_t kv = static_cast<size_t>(bm) * seqlen_k * Hkv * d * 2;
      if ((e0 = cudaMemsetAsync(dk, 0, kv, s0)) == cudaSuccess) e0 = cudaMemsetAsync(dv, 0, kv, s0);
    } else {
      e0 = cudaMemsetAsync(dq, 0, static_cast<size_t>(bm) * seqlen_q * H * d * 2, s0);
    }
    return e0 == cudaSuccess ? FA_OK : cuda_fail(e0, "fa_bwd zero fill");
  }
  const int rows_q = varlen ? max_seqlen_q : seqlen_q;  // per-sequence extents of the grid
  const int rows_k = varlen ? max_seqlen_k : seqlen_k;
  if (batch > 65535 || H > 65535 || (rows_q + 127) / 128 > 65535 || (rows_k + 127) / 128 > 65535)
    return fail(FA_ERR_UNSUPPORTED, "fa_bwd: sizes above the grid limits");
  if ((rc = get_encoder()) != FA_OK) return rc;
  unsigned int* status = nullptr;
  if ((rc = device_state(nullptr, &status, nullptr)) != FA_OK) return rc;
  CUtensorMap tq, tk, tv, tdo;
  const uint32_t box[4] = {64, 128, 1, 1};
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(d), static_cast<uint64_t>(seqlen_q),
                              static_cast<uint64_t>(H), static_cast<uint64_t>(bm)};
    const uint64_t st[3] = {static_cast<uint64_t>(H) * d * 2, static_cast<uint64_t>(d) * 2,
                            static_cast<uint64_t>(seqlen_q) * H * d * 2};
    if ((rc = encode_4d(&tq, q, dims, st, box, "q")) != FA_OK) return rc;
    if ((rc = encode_4d(&tdo, dout, dims, st, box, "dout")) != FA_OK) return rc;
  }
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(d), static_cast<uint64_t>(seqlen_k),
                              static_cast<uint64_t>(Hkv), static_cast<uint64_t>(bm)};
    const uint64_t st[3] = {static_cast<uint64_t>(Hkv) * d * 2, static_cast<uint64_t>(d) * 2,
                            static_cast<uint64_t>(seqlen_k) * Hkv * d * 2};
    if ((rc = encode_4d(&tk, k, dims, st, box, "k")) != FA_OK) return rc;
    if ((rc = encode_4d(&tv, v, dims, st, box, "v")) != FA_OK) return rc;
  }
  const int sq_pad = (seqlen_q + 3) / 4 * 4;
  float* dvec = static_cast<float*>(workspace);
  float* lse2 = dvec + static_cast<size_t>(bm) * H * sq_pad;
  // rows: the true length, so columns past the end load as 0.  Varlen blocks start at
  // any packed row; their copies start at the multiple of 4 below it (a tensor copy's
  // first column must sit on 16 bytes) and are 132 columns wide to cover the block.
  const uint32_t stat_box = varlen ? 132u : 128u;
  CUtensorMap tl, td;
  if ((rc = encode_vec_rows(&tl, lse2, seqlen_q, static_cast<uint64_t>(bm) * H,
                            static_cast<uint64_t>(sq_pad) * 4, stat_box, "lse workspace")) != FA_OK)
    return rc;
  if ((rc = encode_vec_rows(&td, dvec, seqlen_q, static_cast<uint64_t>(bm) * H,
                            static_cast<uint64_t>(sq_pad) * 4, stat_box, "D workspace")) != FA_OK)
    return rc;
  fa::BwdParams p{};
  p.out = out;
  p.dout = dout;
  p.lse = lse;
  p.dvec = dvec;
  p.lse2 = lse2;
  p.sq_pad = sq_pad;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.B = batch;
  p.Sq = seqlen_q;
  p.Sk = seqlen_k;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.scale = scale;
  float softcap_log2 = 0.f, tanh_k = 0.f, scale_log2 = 0.f;
  fill_score_params(scale, softcap, &scale_log2, &softcap_log2, &tanh_k);
  p.scale_log2 = scale_log2;
  p.softcap_log2 = softcap_log2;
  p.tanh_k = tanh_k;
  p.alibi = alibi_slopes;
  p.causal = causal ? 1 : 0;
  p.wl = window_left;
  p.wr = window_right;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.rows_q = rows_q;
  p.rows_k = rows_k;
  p.status = status;
  p.timeout_ns = timeout_ns();
  const cudaError_t e = fa::launch_bwd(tq, tk, tv, tdo, tl, td, p, dtype == FA_BF16, d,
                                       static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "fa_bwd launch");
}

int fa_selftest_wait_timeout(int timeout_ms, void* stream) {
  g_err.clear();
  if (timeout_ms <= 0 || timeout_ms > 10000)
    return fail(FA_ERR_INVALID_ARG, "fa_selftest_wait_timeout: timeout_ms must be in 1..10000");
  unsigned int* status = nullptr;
  int rc = device_state(nullptr, &status, nullptr);
  if (rc != FA_OK) return rc;
  const cudaError_t e = fa::launch_wait_timeout_selftest(
      status, static_cast<uint64_t>(timeout_ms) * 1000000ull, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "fa_selftest_wait_timeout launch");
}

int fa_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache, void* out, float* lse,
                   int dtype, int batch, int seqlen_q, int num_heads, int num_heads_k,
                   int head_dim, const int32_t* block_table, int max_blocks_per_seq,
                   int page_size, int num_blocks, int seqlen_k_max,
                   const int32_t* cache_seqlens, float softmax_scale, int causal,
                   int window_left, int window_right, float softcap,
                   const float* alibi_slopes, int num_splits, void* workspace,
                   size_t workspace_bytes, void* stream) {
  g_err.clear();
  return kvcache_impl(q, k_cache, v_cache, out, lse, dtype, batch, seqlen_q, num_heads,
                      num_heads_k, head_dim, block_table, max_blocks_per_seq, page_size,
                      num_blocks, seqlen_k_max, cache_seqlens, softmax_scale, causal, window_left,
                      window_right, softcap, alibi_slopes, num_splits, workspace, workspace_bytes,
                      stream, nullptr);
}

// Checks the arguments of an append and fills `a` (status left for the caller).
static int append_args(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                       int dtype, int batch, int seqlen_new, int num_heads_k, int head_dim,
                       const int32_t* block_table, int max_blocks_per_seq, int page_size,
                       int num_blocks, int seqlen_k_max, const int32_t* cache_seqlens,
                       fa::AppendParams* a) {
  if (dtype != FA_FP16 && dtype != FA_BF16)
    return fail(FA_ERR_UNSUPPORTED, "kv append: dtype must be FA_FP16 or FA_BF16");
  if (head_dim <= 0 || head_dim > 256 || head_dim % 8)
    return fail(FA_ERR_UNSUPPORTED, "kv append: head_dim %d (a multiple of 8 up to 256)", head_dim);
  if (batch < 0 || seqlen_new < 0 || num_heads_k <= 0)
    return fail(FA_ERR_INVALID_ARG, "kv append: negative size or num_heads_k <= 0");
  if (!k_cache || !v_cache || (seqlen_new > 0 && batch > 0 && (!k_new || !v_new)))
    return fail(FA_ERR_INVALID_ARG, "kv append: caches and new keys/values must be non-NULL");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_new) || !aligned16(v_new))
    return fail(FA_ERR_INVALID_ARG, "kv append: caches and new keys/values must be 16-byte aligned");
  if (cache_seqlens == nullptr)
    return fail(FA_ERR_INVALID_ARG, "kv append: cache_seqlens (keys before the append) is required");
  if (block_table != nullptr) {
    if (page_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
      return fail(FA_ERR_INVALID_ARG, "kv append: page_size, num_blocks and max_blocks_per_seq must be positive");
  } else if (seqlen_k_max < 0) {
    return fail(FA_ERR_INVALID_ARG, "kv append: seqlen_k_max < 0");
  }
  *a = fa::AppendParams{};
  a->k_cache = k_cache;
  a->v_cache = v_cache;
  a->k_new = k_new;
  a->v_new = v_new;
  a->block_table = block_table;
  a->cache_seqlens = cache_seqlens;
  a->B = batch;
  a->S_new = seqlen_new;
  a->Hkv = num_heads_k;
  a->D = head_dim;
  a->max_blocks = max_blocks_per_seq;
  a->page_size = page_size;
  a->num_blocks = num_blocks;
  a->seqlen_k_max = seqlen_k_max;
  return FA_OK;
}

int fa_kvcache_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                      int dtype, int batch, int seqlen_new, int num_heads_k, int head_dim,
                      const int32_t* block_table, int max_blocks_per_seq, int page_size,
                      int num_blocks, int seqlen_k_max, const int32_t* cache_seqlens,
                      void* stream) {
  g_err.clear();
  fa::AppendParams a;
  int rc = append_args(k_cache, v_cache, k_new, v_new, dtype, batch, seqlen_new, num_heads_k,
                       head_dim, block_table, max_blocks_per_seq, page_size, num_blocks,
                       seqlen_k_max, cache_seqlens, &a);
  if (rc != FA_OK) return rc;
  if (batch == 0 || seqlen_new == 0) return FA_OK;
  if ((rc = device_state(nullptr, &a.status, nullptr)) != FA_OK) return rc;
  const cudaError_t e = fa::launch_kv_append(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "fa_kvcache_append launch");
}

int fa_fwd_kvcache_append(const void* q, void* k_cache, void* v_cache, const void* k_new,
                          const void* v_new, int seqlen_new, void* out, float* lse, int dtype,
                          int batch, int seqlen_q, int num_heads, int num_heads_k, int head_dim,
                          const int32_t* block_table, int max_blocks_per_seq, int page_size,
                          int num_blocks, int seqlen_k_max, const int32_t* cache_seqlens,
                          float softmax_scale, int causal, int window_left, int window_right,
                          float softcap, const float* alibi_slopes, int num_splits,
                          void* workspace, size_t workspace_bytes, void* stream) {
  g_err.clear();
  fa::AppendParams a;
  int rc = append_args(k_cache, v_cache, k_new, v_new, dtype, batch, seqlen_new, num_heads_k,
                       head_dim, block_table, max_blocks_per_seq, page_size, num_blocks,
                       seqlen_k_max, cache_seqlens, &a);
  if (rc != FA_OK) return rc;
  return kvcache_impl(q, k_cache, v_cache, out, lse, dtype, batch, seqlen_q, num_heads,
                      num_heads_k, head_dim, block_table, max_blocks_per_seq, page_size,
                      num_blocks, seqlen_k_max, cache_seqlens, softmax_scale, causal, window_left,
                      window_right, softcap, alibi_slopes, num_splits, workspace, workspace_bytes,
                      stream, seqlen_new > 0 ? &a : nullptr);
}

int fa_combine(const float* out_partial, const float* lse_partial, void* out, float* lse,
               int out_dtype, int batch, int seqlen, int num_heads, int head_dim, int num_splits,
               const int64_t* op_strides, const int64_t* lp_strides, void* stream) {
  g_err.clear();
  if (!out_partial || !lse_partial || !out)
    return fail(FA_ERR_INVALID_ARG, "fa_combine: out_partial, lse_partial and out must be non-NULL");
  if (out_dtype != FA_FP16 && out_dtype != FA_BF16 && out_dtype != FA_FP32)
    return fail(FA_ERR_UNSUPPORTED, "fa_combine: out_dtype %d", out_dtype);
  if (batch < 0 || seqlen < 0 || num_heads <= 0 || head_dim <= 0 || head_dim > 256 || head_dim % 4)
    return fail(FA_ERR_INVALID_ARG, "fa_combine: bad sizes (head_dim must be a multiple of 4 up to 256)");
  if (num_splits < 1 || num_splits > 256)
    return fail(FA_ERR_INVALID_ARG, "fa_combine: num_splits must be in [1, 256]");
  if ((reinterpret_cast<uintptr_t>(out_partial) | reinterpret_cast<uintptr_t>(lse_partial)) & 3u)
    return fail(FA_ERR_INVALID_ARG, "fa_combine: partials must be 4-byte aligned");
  fa::CombineParams c{};
  const int64_t S = seqlen, H = num_heads, D = head_dim, SP = num_splits;
  const int64_t dop[5] = {S * H * D * SP, H * D * SP, D * SP, SP, 1};
  const int64_t dlp[4] = {S * H * SP, H * SP, SP, 1};
  for (int i = 0; i < 5; ++i) c.op_s[i] = op_strides ? op_strides[i] : dop[i];
  for (int i = 0; i < 4; ++i) c.lp_s[i] = lp_strides ? lp_strides[i] : dlp[i];
  for (int i = 0; i < 5; ++i)
    if (c.op_s[i] < 0 || (i < 4 && c.lp_s[i] < 0))
      return fail(FA_ERR_INVALID_ARG, "fa_combine: strides must be >= 0");
  c.op = out_partial;
  c.lp = lse_partial;
  c.out = out;
  c.lse = lse;
  c.B = batch;
  c.S = seqlen;
  c.H = num_heads;
  c.D = head_dim;
  c.splits = num_splits;
  c.out_dtype = out_dtype;
  if (batch == 0 || seqlen == 0) return FA_OK;
  int rc = device_state(nullptr, nullptr, nullptr);
  if (rc != FA_OK) return rc;
  cudaError_t e = fa::launch_combine(c, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fa_combine launch");
  return FA_OK;
}

}  // extern "C"
