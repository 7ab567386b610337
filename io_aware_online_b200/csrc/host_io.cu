// host_io.cu -- fa_fwd_host: the dense attention forward on operands that live in
// host memory, with the PCIe transfers pipelined against the kernels.
//
// A caller whose q, k and v sit in host memory would otherwise copy them in, run
// fa_fwd and copy O out, one step after the other, and the transfers dominate: a
// causal B=4, S=4096, H=32, d=64 fp16 prefill moves 268 MB across the bus for a
// kernel of about 0.4 ms.  This entry point cuts the batch into chunks of whole
// sequences and moves them through two device slots of a caller-provided workspace
// on three streams of its own, so that while chunk c is computed, chunk c+1 is
// copied in and chunk c-1 copied out (host-to-device and device-to-host copies use
// separate copy engines and overlap each other and the kernels).  Each chunk is one
// fa_fwd call over its sequences; the kernel computes every (sequence, head) on its
// own, so the results are bit-identical to a single fa_fwd call over the batch.
//
// Ordering: the call's work starts after everything already enqueued on the
// caller's stream and, when that stream reaches the point of the call, all of it
// (the last copy into `out` / `lse` included) has completed.  The internal streams
// and events are created once per device, on that device's first call, and kept
// for the life of the process (after a device reset they are stale and this entry
// point must not be called).  Calls are serialised by a lock while they enqueue.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdio>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace {

constexpr int kPipeMaxDev = 64;
constexpr int kMaxChunks = 4;  // the batch is cut into at most this many chunks
constexpr size_t kAlign = 256;

struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done[3] = {}, in_ev[2] = {}, comp_ev[2] = {}, out_ev[2] = {};
};

std::mutex g_host_mu;
HostPipe g_pipe[kPipeMaxDev];

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Per-chunk byte sizes of the workspace slots.
struct Slot {
  size_t q, kv, lse, total;
};

Slot slot_bytes(int cb, int seqlen_q, int seqlen_k, int num_heads, int num_heads_k,
                int head_dim, bool with_lse) {
  Slot s;
  s.q = align_up(static_cast<size_t>(cb) * seqlen_q * num_heads * head_dim * 2);
  s.kv = align_up(static_cast<size_t>(cb) * seqlen_k * num_heads_k * head_dim * 2);
  s.lse = with_lse ? align_up(static_cast<size_t>(cb) * num_heads * seqlen_q * 4) : 0;
  s.total = 2 * s.q + 2 * s.kv + s.lse;  // q, k, v, out, lse
  return s;
}

int chunk_batch(int batch) {
  const int n = std::min(batch, kMaxChunks);
  return (batch + n - 1) / n;
}

int pipe_of_current_device(HostPipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kPipeMaxDev)
    return fa::set_error(FA_ERR_CUDA, "fa_fwd_host: no usable current CUDA device");
  HostPipe& p = g_pipe[dev];
  if (!p.ready) {
    bool ok = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.comp, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < 3; ++i)
      ok = cudaEventCreateWithFlags(&p.done[i], cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < 2; ++i)
      ok = cudaEventCreateWithFlags(&p.in_ev[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.comp_ev[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.out_ev[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return fa::set_error(FA_ERR_CUDA, "fa_fwd_host: creating streams or events failed");
    p.ready = true;
  }
  *out = &p;
  return FA_OK;
}

}  // namespace

extern "C" {

FA_API size_t fa_fwd_host_workspace_size(int batch, int seqlen_q, int seqlen_k, int num_heads,
                                         int num_heads_k, int head_dim, int with_lse) {
  if (batch <= 0 || seqlen_q <= 0 || seqlen_k <= 0 || num_heads <= 0 || num_heads_k <= 0 ||
      head_dim <= 0)
    return 0;
  const Slot s = slot_bytes(chunk_batch(batch), seqlen_q, seqlen_k, num_heads, num_heads_k,
                            head_dim, with_lse != 0);
  return align_up(static_cast<size_t>(num_heads) * 4) + 2 * s.total;
}

FA_API int fa_fwd_host(const void* q, const void* k, const void* v, void* out, float* lse,
                       int dtype, int batch, int seqlen_q, int seqlen_k, int num_heads,
                       int num_heads_k, int head_dim, float softmax_scale, int causal,
                       int window_left, int window_right, float softcap,
                       const float* alibi_slopes, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr)
    return fa::set_error(FA_ERR_INVALID_ARG, "fa_fwd_host: q, k, v and out are required");
  if (dtype != FA_FP16 && dtype != FA_BF16)
    return fa::set_error(FA_ERR_UNSUPPORTED, "fa_fwd_host: dtype must be FA_FP16 or FA_BF16");
  if (batch < 0 || seqlen_q <= 0 || seqlen_k <= 0 || num_heads <= 0 || num_heads_k <= 0 ||
      num_heads % num_heads_k != 0)
    return fa::set_error(FA_ERR_INVALID_ARG, "fa_fwd_host: bad shape");
  if (head_dim != 64 && head_dim != 128)
    return fa::set_error(FA_ERR_UNSUPPORTED, "fa_fwd_host: head_dim must be 64 or 128");
  if (static_cast<int64_t>(seqlen_q) * num_heads * head_dim > INT_MAX ||
      static_cast<int64_t>(seqlen_k) * num_heads_k * head_dim > INT_MAX)
    return fa::set_error(FA_ERR_UNSUPPORTED, "fa_fwd_host: a sequence exceeds 2^31 elements");
  if (batch == 0) return FA_OK;
  const size_t need = fa_fwd_host_workspace_size(batch, seqlen_q, seqlen_k, num_heads,
                                                 num_heads_k, head_dim, lse != nullptr);
  if (workspace == nullptr || workspace_bytes < need ||
      reinterpret_cast<uintptr_t>(workspace) % kAlign != 0)
    return fa::set_error(FA_ERR_WORKSPACE,
                         "fa_fwd_host: workspace missing, not 256-byte aligned or smaller than "
                         "fa_fwd_host_workspace_size()");

  std::lock_guard<std::mutex> lk(g_host_mu);
  HostPipe* pp = nullptr;
  int rc = pipe_of_current_device(&pp);
  if (rc != FA_OK) return rc;
  HostPipe& P = *pp;
  const cudaStream_t user = static_cast<cudaStream_t>(stream);

  // per-sequence byte counts of the host operands ([B, S, H, d] and [B, H, Sq])
  const size_t q_seq = static_cast<size_t>(seqlen_q) * num_heads * head_dim * 2;
  const size_t kv_seq = static_cast<size_t>(seqlen_k) * num_heads_k * head_dim * 2;
  const size_t lse_seq = static_cast<size_t>(num_heads) * seqlen_q * 4;
  const int cb = chunk_batch(batch);
  const Slot sb = slot_bytes(cb, seqlen_q, seqlen_k, num_heads, num_heads_k, head_dim,
                             lse != nullptr);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* d_alibi = reinterpret_cast<float*>(ws);
  uint8_t* slots = ws + align_up(static_cast<size_t>(num_heads) * 4);

  const char* what = nullptr;  // the failed CUDA step, if any
  auto ck = [&](cudaError_t e, const char* step) {
    if (e != cudaSuccess && what == nullptr) what = step;
    return e == cudaSuccess;
  };
  bool ok = ck(cudaEventRecord(P.start, user), "event record") &&
            ck(cudaStreamWaitEvent(P.in, P.start, 0), "stream wait") &&
            ck(cudaStreamWaitEvent(P.comp, P.start, 0), "stream wait") &&
            ck(cudaStreamWaitEvent(P.out, P.start, 0), "stream wait");
  if (ok && alibi_slopes != nullptr)
    ok = ck(cudaMemcpyAsync(d_alibi, alibi_slopes, static_cast<size_t>(num_heads) * 4,
                            cudaMemcpyDefault, P.comp),
            "ALiBi slope copy");
  const int n_chunks = (batch + cb - 1) / cb;
  for (int c = 0; ok && rc == FA_OK && c < n_chunks; ++c) {
    const int b0 = c * cb, nb = std::min(cb, batch - b0), s = c & 1;
    uint8_t* dq = slots + s * sb.total;
    uint8_t* dk = dq + sb.q;
    uint8_t* dv = dk + sb.kv;
    uint8_t* dout = dv + sb.kv;
    float* dlse = (lse != nullptr) ? reinterpret_cast<float*>(dout + sb.q) : nullptr;
    // the slot is free once the copy-out of chunk c - 2 (which followed its kernel) is done
    if (c >= 2) ok = ck(cudaStreamWaitEvent(P.in, P.out_ev[s], 0), "stream wait");
    ok = ok &&
         ck(cudaMemcpyAsync(dq, static_cast<const uint8_t*>(q) + b0 * q_seq, nb * q_seq,
                            cudaMemcpyDefault, P.in),
            "q copy") &&
         ck(cudaMemcpyAsync(dk, static_cast<const uint8_t*>(k) + b0 * kv_seq, nb * kv_seq,
                            cudaMemcpyDefault, P.in),
            "k copy") &&
         ck(cudaMemcpyAsync(dv, static_cast<const uint8_t*>(v) + b0 * kv_seq, nb * kv_seq,
                            cudaMemcpyDefault, P.in),
            "v copy") &&
         ck(cudaEventRecord(P.in_ev[s], P.in), "event record") &&
         ck(cudaStreamWaitEvent(P.comp, P.in_ev[s], 0), "stream wait");
    if (!ok) break;
    rc = fa_fwd(dq, dk, dv, dout, dlse, dtype, nb, seqlen_q, seqlen_k, num_heads, num_heads_k,
                head_dim, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, 0,
                softmax_scale, causal, window_left, window_right, softcap,
                alibi_slopes != nullptr ? d_alibi : nullptr, P.comp);
    if (rc != FA_OK) break;
    ok = ck(cudaEventRecord(P.comp_ev[s], P.comp), "event record") &&
         ck(cudaStreamWaitEvent(P.out, P.comp_ev[s], 0), "stream wait") &&
         ck(cudaMemcpyAsync(static_cast<uint8_t*>(out) + b0 * q_seq, dout, nb * q_seq,
                            cudaMemcpyDefault, P.out),
            "out copy");
    if (ok && lse != nullptr)
      ok = ck(cudaMemcpyAsync(reinterpret_cast<uint8_t*>(lse) + b0 * lse_seq, dlse, nb * lse_seq,
                              cudaMemcpyDefault, P.out),
              "lse copy");
    ok = ok && ck(cudaEventRecord(P.out_ev[s], P.out), "event record");
  }
  // join: the caller's stream waits for all three streams, whatever happened above,
  // so that nothing enqueued here still runs once the caller sees the stream done
  const cudaStream_t st[3] = {P.in, P.comp, P.out};
  bool joined = true;
  for (int i = 0; i < 3; ++i)
    joined = ck(cudaEventRecord(P.done[i], st[i]), "event record") &&
             ck(cudaStreamWaitEvent(user, P.done[i], 0), "stream wait") && joined;
  if (rc != FA_OK) return rc;  // fa_fwd's own error message stands
  if (!ok || !joined) {
    char msg[160];
    snprintf(msg, sizeof(msg), "fa_fwd_host: CUDA %s failed", what ? what : "call");
    return fa::set_error(FA_ERR_CUDA, msg);
  }
  return FA_OK;
}

}  // extern "C"
