// decode_kernel.cuh -- split-KV attention of a few query rows against a (paged) KV
// cache, sm_100a.  Changelog post: v2.2 split-KV ("flash-decoding": the KV cache
// is cut along the sequence, each block handles one range, an extra kernel
// reduces) and v2.5 paged KV cache (a block_table addresses the pages);
// "FlashAttention common interfaces" section 3.3 for the argument set.
//
// This path is bound by HBM bandwidth (about 2 FMAs per cache byte), so it runs
// on the CUDA cores and spends its effort on the memory stream.
//
// Work item = (sequence b, KV head hk, split s): the keys of pages
// [s*c, min((s+1)*c, pages)) of sequence b (c = ceil(pages / num_splits)), for all
// R = G * Sq query rows that read KV head hk, so each cache byte is read once.
// The kernel is persistent: a fixed grid of CTAs (3 per SM) claims items one at a
// time from a counter (atomicAdd; items differ in length by up to 32x, so a static
// assignment leaves a long tail), and within a CTA the stream of 64-token K/V
// tiles runs on across item boundaries, so no CTA drains its copy pipeline.
// Items are claimed longest sequence first (a prep kernel ranks the sequences by
// cache length before the launch), so the last items to finish are the shortest:
// at 4 splits an item of a 32K-token sequence is 8K tokens, and claimed last it
// would leave most CTAs idle for its whole duration.
//   warps 0-3  consumers: warp w owns tokens [16w, 16w+16) of every tile and runs
//              its own online softmax (max, sum) and P*V over them, with no
//              barrier between warps inside the tile loop; at the end of an item
//              the four partial (m, l, O) merge by the LSE rule and one partial
//              (O_s, lse_s) or, unsplit, the final O and LSE is written
//   warp  4    producer: claims the next item, publishes its index with a bulk
//              copy of its query rows into the staging slot, then
//              streams the item's K and V tiles (TMA, 64
//              tokens of one KV head each, block_table looked up once per tile)
//              into a 2-stage ring
//   Scores: lane (token pair, quarter of the head dim) -> shuffle reduction.
//   P*V:    lane owns D/32 adjacent head-dim columns; the warp's 16 probabilities
//           per row pass through a warp-private shared buffer.
// Keys past cache_seqlens[b] (page tails, possibly garbage) are masked by
// selection and skipped in P*V, so nothing they hold can reach the output.
#pragma once

#include <climits>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

constexpr int kDecTok = 64;       // tokens per tile
constexpr int kDecStages = 2;     // 2-stage ring, three CTAs per SM (~190 KB of reads in flight)
constexpr int kDecConsumers = 128;
constexpr int kDecThreads = kDecConsumers + 32;

template <int D, int RMAX>
struct DecCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kChunkBytes = kDecTok * 128;      // 64 tokens x 128 bytes
  static constexpr int kTileBytes = kDecTok * D * 2;     // one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kPart = D / 4;                    // head-dim elements per quarter
  static constexpr int kQPartStride = kPart + 8;         // padded (bank spread)
  static constexpr int kQRawOff = kDecStages * kStageBytes;
  static constexpr int kQRawBytes = RMAX * D * 2;        // one staging slot (16-bit rows)
  static constexpr int kQOff = kQRawOff + kQRawBytes;
  static constexpr int kQBytes = RMAX * 4 * kQPartStride * 4;
  static constexpr int kPOff = kQOff + kQBytes;
  static constexpr int kPBytes = kDecTok * RMAX * 4;        // [warp][16 tokens][RMAX]
  static constexpr int kRedOff = kPOff + kPBytes;
  static constexpr int kRedBytes = 2 * 4 * RMAX * 4;        // per-warp m and l
  static constexpr int kAccOff = kRedOff + kRedBytes;
  static constexpr int kAccBytes = 2 * RMAX * D * 4;        // O rows of two warps (merge)
  static constexpr int kBarOff = (kAccOff + kAccBytes + 7) & ~7;
  // full[ST], empty[ST], qfull[2], qempty[2]
  static constexpr int kMiscOff = kBarOff + (2 * kDecStages + 4) * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;  // abort flag, item index per slot
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static constexpr int kCols = D / 32;                   // head-dim columns per lane in P*V
};

__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Barrier among `nthreads` threads that also ORs `pred` across them.
__device__ __forceinline__ bool named_sync_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ bool dec_wait_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// Geometry of one work item, computed identically by producer and consumers.
struct DecItem {
  int b, hk, split, L, off, t_lo, n_tiles;
};

__device__ __forceinline__ DecItem dec_item(const DecodeParams& p, int item) {
  DecItem it;
  it.split = item % p.num_splits;
  it.hk = (item / p.num_splits) % p.Hkv;
  it.b = item / (p.num_splits * p.Hkv);
  if (p.order != nullptr) it.b = p.order[it.b];  // longest sequences first
  it.L = ((p.cache_seqlens != nullptr) ? p.cache_seqlens[it.b] : p.seqlen_k_max) + p.k_add;
  {
    // a length the cache cannot hold would read past the block table: clamp it
    // and report (identically in the producer and the consumers)
    const int cap = (p.block_table != nullptr) ? p.max_blocks * p.page_size : p.seqlen_k_max;
    if (it.L < 0 || it.L > cap) {
      atomicOr(p.status, kDevBadLength);
      it.L = min(max(it.L, 0), cap);
    }
  }
  const int n_units = (it.L + p.unit - 1) / p.unit;
  const int per = (n_units + p.num_splits - 1) / p.num_splits;
  const int u_begin = it.split * per;
  const int u_end = min(n_units, u_begin + per);
  const bool has_left = p.wl >= 0;
  const bool has_right = p.causal || p.wr >= 0;
  const int right = p.causal ? 0 : p.wr;
  it.off = it.L - p.Sq;  // query i sits at key position i + off
  int kb_lo = u_begin * p.unit;
  int kb_hi = min(u_end * p.unit, it.L);
  if (has_left) kb_lo = max(kb_lo, it.off - p.wl);                      // row i = 0
  if (has_right) kb_hi = min(kb_hi, p.Sq - 1 + it.off + right + 1);     // row i = Sq-1
  kb_lo = max(kb_lo, 0);
  it.t_lo = kb_lo / kDecTok;
  it.n_tiles = (kb_hi > kb_lo) ? (kb_hi + kDecTok - 1) / kDecTok - it.t_lo : 0;
  return it;
}

// One CTA: zero the work-item counter; rank the sequences by attended length,
// longest first (ties by index), into p.order.  O(B^2 / threads) comparisons for
// B <= kDecOrderMax.
__global__ void __launch_bounds__(128) decode_prep_kernel(const DecodeParams p) {
  if (threadIdx.x == 0) *p.item_counter = 0u;
  if (p.order == nullptr) return;
  int16_t* order = const_cast<int16_t*>(p.order);
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    const int lb = p.cache_seqlens[b];
    int rank = 0;
    for (int c = 0; c < p.B; ++c) {
      const int lc = p.cache_seqlens[c];
      rank += (lc > lb) || (lc == lb && c < b);
    }
    order[rank] = static_cast<int16_t>(b);
  }
}

template <int D, bool BF16, int RMAX>
__global__ void __launch_bounds__(kDecThreads, RMAX <= 4 ? 3 : 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecodeParams p) {
  using Cfg = DecCfg<D, RMAX>;
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.6931471805599453f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* q_raw = smem + Cfg::kQRawOff;
  float* q_s = reinterpret_cast<float*>(smem + Cfg::kQOff);
  float* p_s = reinterpret_cast<float*>(smem + Cfg::kPOff);
  float* red = reinterpret_cast<float*>(smem + Cfg::kRedOff);
  float* accs = reinterpret_cast<float*>(smem + Cfg::kAccOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* empty = full + kDecStages;
  uint64_t* qfull = full + 2 * kDecStages;
  uint64_t* qempty = qfull + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff);
  volatile int* slot_item = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);
  uint8_t* stage0 = smem;

  const int tid = threadIdx.x;
  const int warp = tid / 32, lane = tid % 32;
  const int n_items = p.B * p.Hkv * p.num_splits;

  if (tid == kDecConsumers) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kDecConsumers);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(qfull + s, 1);
      mbar_init(qempty + s, kDecConsumers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtx w{abort_flag, p.status, p.timeout_ns};

  if (warp == kDecConsumers / 32) {
    // ======================================================== producer
    if (lane == 0) {
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      int last[kDecStages], lastq[2];
      for (int s = 0; s < kDecStages; ++s) last[s] = -1;
      lastq[0] = lastq[1] = -1;
      int n = 0, qi = 0;
      bool ok = true;
      for (;; ++qi) {
        const int slot = 0;
        const uint32_t qph = qi & 1;
        if (!(ok = wait_bounded(qempty + slot, qph ^ 1, w))) break;
        const int item = static_cast<int>(atomicAdd(p.item_counter, 1u));
        slot_item[slot] = item;  // published to the consumers by the qfull arrive
        if (item >= n_items) {   // no work left: release the consumers and stop
          mbar_arrive(qfull + slot);
          break;
        }
        const DecItem itm = dec_item(p, item);
        // query rows of the item: Sq runs of G contiguous heads
        const uint32_t run = static_cast<uint32_t>(p.G) * D * 2;
        mbar_arrive_expect_tx(qfull + slot, run * p.Sq);
        for (int i = 0; i < p.Sq; ++i) {
          const uint8_t* src = static_cast<const uint8_t*>(p.q) +
                               ((static_cast<size_t>(itm.b) * p.Sq + i) * p.H +
                                static_cast<size_t>(itm.hk) * p.G) * D * 2;
          bulk_load(q_raw + slot * Cfg::kQRawBytes + i * run, src, run, qfull + slot);
        }
        lastq[slot] = qph;
        for (int t = 0; t < itm.n_tiles; ++t, ++n) {
          const int s = n % kDecStages;
          const uint32_t ph = (n / kDecStages) & 1;
          if (!(ok = wait_bounded(empty + s, ph ^ 1, w))) break;
          const int tok0 = (itm.t_lo + t) * kDecTok;
          int c2, c3;
          if (p.block_table != nullptr) {
            int blk = p.block_table[static_cast<size_t>(itm.b) * p.max_blocks + tok0 / p.page_size];
            if (blk < 0 || blk >= p.num_blocks) {
              atomicOr(p.status, kDevBadBlock);
              blk = 0;  // read a valid page; the status word reports the fault
            }
            c2 = tok0 % p.page_size;
            c3 = blk;
          } else {
            c2 = tok0;
            c3 = itm.b;
          }
          uint8_t* st = stage0 + s * Cfg::kStageBytes;
          mbar_arrive_expect_tx(full + s, Cfg::kStageBytes);
#pragma unroll
          for (int c = 0; c < Cfg::kChunks; ++c) {
            tma_load_4d(st + c * Cfg::kChunkBytes, &tmK, full + s, c * 64, itm.hk, c2, c3);
            tma_load_4d(st + Cfg::kTileBytes + c * Cfg::kChunkBytes, &tmV, full + s, c * 64,
                        itm.hk, c2, c3);
          }
          last[s] = ph;
        }
      }
      if (*abort_flag) {  // let this CTA's own copies land before the smem goes away
        for (int s = 0; s < kDecStages; ++s)
          if (last[s] >= 0) dec_wait_drain(full + s, last[s], p.timeout_ns);
        for (int s = 0; s < 2; ++s)
          if (lastq[s] >= 0) dec_wait_drain(qfull + s, lastq[s], p.timeout_ns);
      }
    }
    __syncwarp();
    return;
  }

  // ========================================================== consumers
  const int tpl = lane / 4, part = lane % 4;   // scores: tokens 16w + tpl and 16w + tpl + 8
  const bool has_left = p.wl >= 0;
  const bool has_right = p.causal || p.wr >= 0;
  const int right = p.causal ? 0 : p.wr;
  float* p_w = p_s + warp * 16 * RMAX;         // this warp's probabilities [16][RMAX]
  int n = 0, qi = 0;
  bool ok = true;
  for (;; ++qi) {
    const int slot = 0;
    ok = wait_bounded(qfull + slot, qi & 1, w);
    if (named_sync_or(1, kDecConsumers, !ok)) break;
    const int item = slot_item[slot];
    if (item >= n_items) break;  // the producer found no more work
    const DecItem itm = dec_item(p, item);
    // ---- query rows: 16-bit staging slot -> fp32 padded quarters
    {
      const uint16_t* raw = reinterpret_cast<const uint16_t*>(q_raw + slot * Cfg::kQRawBytes);
      for (int idx = tid; idx < RMAX * D; idx += kDecConsumers) {
        const int r = idx / D, e = idx % D;
        float qv = 0.f;
        if (r < p.R) {
          const int g = r / p.Sq, i = r % p.Sq;
          const uint16_t bits = raw[(i * p.G + g) * D + e];
          if constexpr (BF16)
            qv = __uint_as_float(static_cast<uint32_t>(bits) << 16);
          else
            qv = __half2float(__ushort_as_half(bits));
        }
        q_s[(r * 4 + e / Cfg::kPart) * Cfg::kQPartStride + e % Cfg::kPart] = qv;
      }
      mbar_arrive(qempty + slot);
      named_sync(1, kDecConsumers);
    }
    int lo_r[RMAX], hi_r[RMAX];
    float slope2[RMAX], cpos[RMAX];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      const int i = (r < p.R) ? r % p.Sq : 0;
      const int c = i + itm.off;
      lo_r[r] = (r < p.R && has_left) ? c - p.wl : INT_MIN / 2;
      hi_r[r] = (r < p.R && has_right) ? min(c + right, itm.L - 1) : itm.L - 1;
      const int h = itm.hk * p.G + ((r < p.R) ? r / p.Sq : 0);
      slope2[r] = (p.alibi != nullptr) ? p.alibi[h] * kLog2e : 0.f;
      cpos[r] = static_cast<float>(c);
    }
    float m_run[RMAX], l_part[RMAX];
    float acc[RMAX][Cfg::kCols];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      m_run[r] = -INFINITY;
      l_part[r] = 0.f;
#pragma unroll
      for (int c = 0; c < Cfg::kCols; ++c) acc[r][c] = 0.f;
    }
    // this lane's head-dim columns in P*V: e0 .. e0 + kCols - 1
    const int e0 = lane * Cfg::kCols;
    const int v_chunk = e0 / 64, v_u16 = (e0 % 64) / 8, v_in = (e0 % 8) * 2;

    for (int t = 0; t < itm.n_tiles; ++t, ++n) {
      const int s = n % kDecStages;
      const uint32_t ph = (n / kDecStages) & 1;
      ok = wait_bounded(full + s, ph, w);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      const uint8_t* sK = stage0 + s * Cfg::kStageBytes;
      const uint8_t* sV = sK + Cfg::kTileBytes;
      const int tok0 = (itm.t_lo + t) * kDecTok;
      const int ta = warp * 16 + tpl, tb = ta + 8;

      // ---- scores for tokens ta and tb (packed fp32 pairs: one FMA per 2 MACs)
      float2 pa[RMAX], pb[RMAX];
#pragma unroll
      for (int r = 0; r < RMAX; ++r) pa[r] = pb[r] = make_float2(0.f, 0.f);
#pragma unroll
      for (int u = 0; u < Cfg::kPart / 8; ++u) {
        const int e = part * Cfg::kPart + u * 8;
        const int chunk = e / 64, u16 = (e % 64) / 8;
        const uint4 ka = *reinterpret_cast<const uint4*>(sK + chunk * Cfg::kChunkBytes +
                                                         ta * 128 + ((u16 ^ (ta & 7)) << 4));
        const uint4 kb = *reinterpret_cast<const uint4*>(sK + chunk * Cfg::kChunkBytes +
                                                         tb * 128 + ((u16 ^ (tb & 7)) << 4));
        const float2 fa0 = unpack2<BF16>(ka.x), fa1 = unpack2<BF16>(ka.y),
                     fa2 = unpack2<BF16>(ka.z), fa3 = unpack2<BF16>(ka.w);
        const float2 fb0 = unpack2<BF16>(kb.x), fb1 = unpack2<BF16>(kb.y),
                     fb2 = unpack2<BF16>(kb.z), fb3 = unpack2<BF16>(kb.w);
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
          const float4* qp =
              reinterpret_cast<const float4*>(q_s + (r * 4 + part) * Cfg::kQPartStride + u * 8);
          const float4 q0 = qp[0], q1 = qp[1];
          const float2 q00 = make_float2(q0.x, q0.y), q01 = make_float2(q0.z, q0.w);
          const float2 q10 = make_float2(q1.x, q1.y), q11 = make_float2(q1.z, q1.w);
          pa[r] = fma2(q00, fa0, pa[r]);
          pa[r] = fma2(q01, fa1, pa[r]);
          pa[r] = fma2(q10, fa2, pa[r]);
          pa[r] = fma2(q11, fa3, pa[r]);
          pb[r] = fma2(q00, fb0, pb[r]);
          pb[r] = fma2(q01, fb1, pb[r]);
          pb[r] = fma2(q10, fb2, pb[r]);
          pb[r] = fma2(q11, fb3, pb[r]);
        }
      }
      // ---- full dot products, transform (base-2 units), mask, warp-local max
      const int ja = tok0 + ta, jb = tok0 + tb;
      float sa[RMAX], sb[RMAX], alpha[RMAX];
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        float xa = pa[r].x + pa[r].y, xb = pb[r].x + pb[r].y;
        xa += __shfl_xor_sync(0xffffffffu, xa, 1);
        xa += __shfl_xor_sync(0xffffffffu, xa, 2);
        xb += __shfl_xor_sync(0xffffffffu, xb, 1);
        xb += __shfl_xor_sync(0xffffffffu, xb, 2);
        if (p.has_softcap) {
          xa = fmaf(-2.f * p.softcap_log2, rcp(ex2(xa * p.tanh_k) + 1.f), p.softcap_log2);
          xb = fmaf(-2.f * p.softcap_log2, rcp(ex2(xb * p.tanh_k) + 1.f), p.softcap_log2);
        } else {
          xa *= p.scale_log2;
          xb *= p.scale_log2;
        }
        xa = fmaf(-slope2[r], fabsf(cpos[r] - static_cast<float>(ja)), xa);
        xb = fmaf(-slope2[r], fabsf(cpos[r] - static_cast<float>(jb)), xb);
        sa[r] = (ja >= lo_r[r] && ja <= hi_r[r]) ? xa : -INFINITY;
        sb[r] = (jb >= lo_r[r] && jb <= hi_r[r]) ? xb : -INFINITY;
        float mx = fmaxf(sa[r], sb[r]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run[r], mx);
        alpha[r] = (m_new == -INFINITY) ? 1.f : ex2(m_run[r] - m_new);
        m_run[r] = m_new;
        const float pa_ = (sa[r] == -INFINITY) ? 0.f : ex2(sa[r] - m_new);
        const float pb_ = (sb[r] == -INFINITY) ? 0.f : ex2(sb[r] - m_new);
        if (part == 0) {
          p_w[tpl * RMAX + r] = pa_;
          p_w[(tpl + 8) * RMAX + r] = pb_;
          l_part[r] = fmaf(l_part[r], alpha[r], pa_ + pb_);
        }
      }
      __syncwarp();
      // ---- P * V over this warp's 16 tokens, kCols columns per lane
#pragma unroll
      for (int r = 0; r < RMAX; ++r)
#pragma unroll
        for (int c = 0; c < Cfg::kCols; ++c) acc[r][c] *= alpha[r];
      const int n_valid = min(16, itm.L - tok0 - warp * 16);  // keys at or past L are skipped
#pragma unroll 4
      for (int tl = 0; tl < n_valid; ++tl) {
        const int tok = warp * 16 + tl;
        const uint8_t* vp = sV + v_chunk * Cfg::kChunkBytes + tok * 128 +
                            ((v_u16 ^ (tok & 7)) << 4) + v_in;
        float2 v[Cfg::kCols / 2];
        if constexpr (Cfg::kCols == 4) {
          const uint2 vw = *reinterpret_cast<const uint2*>(vp);
          v[0] = unpack2<BF16>(vw.x);
          v[1] = unpack2<BF16>(vw.y);
        } else {
          v[0] = unpack2<BF16>(*reinterpret_cast<const uint32_t*>(vp));
        }
        const float* pr = p_w + tl * RMAX;
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
          const float pv = pr[r];
#pragma unroll
          for (int c2 = 0; c2 < Cfg::kCols / 2; ++c2) {
            const float2 a = fma2(make_float2(pv, pv), v[c2],
                                  make_float2(acc[r][2 * c2], acc[r][2 * c2 + 1]));
            acc[r][2 * c2] = a.x;
            acc[r][2 * c2 + 1] = a.y;
          }
        }
      }
      __syncwarp();  // p_w is rewritten by the next tile
      mbar_arrive(empty + s);
    }
    if (named_sync_or(1, kDecConsumers, !ok)) break;

    // ---------------------------------------------------------- end of item
    // Merge the four warps' (m, l, O) by the LSE rule in two rounds through a
    // two-warp buffer (lane l of every warp owns the same columns), then write.
    float* red_m = red;
    float* red_l = red + 4 * RMAX;
    float l_w[RMAX];  // the warp's row sums, the same in every lane
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      float v = (part == 0) ? l_part[r] : 0.f;
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      l_w[r] = v;
    }
    auto publish = [&](int buf) {  // this warp's (m, l, O) -> buffer slot `buf`
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        if (lane == 0) {
          red_m[buf * RMAX + r] = m_run[r];
          red_l[buf * RMAX + r] = l_w[r];
        }
#pragma unroll
        for (int c = 0; c < Cfg::kCols; ++c) accs[(buf * RMAX + r) * D + e0 + c] = acc[r][c];
      }
    };
    auto absorb = [&](int buf) {   // merge buffer slot `buf` into this warp's (m, l, O)
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        const float mo = red_m[buf * RMAX + r];
        const float M = fmaxf(m_run[r], mo);
        const float sa_ = (m_run[r] == -INFINITY) ? 0.f : ex2(m_run[r] - M);
        const float sb_ = (mo == -INFINITY) ? 0.f : ex2(mo - M);
        l_w[r] = l_w[r] * sa_ + red_l[buf * RMAX + r] * sb_;
#pragma unroll
        for (int c = 0; c < Cfg::kCols; ++c)
          acc[r][c] = acc[r][c] * sa_ + accs[(buf * RMAX + r) * D + e0 + c] * sb_;
        m_run[r] = M;
      }
    };
    if (warp >= 2) publish(warp - 2);
    named_sync(1, kDecConsumers);
    if (warp < 2) absorb(warp);
    named_sync(1, kDecConsumers);
    if (warp == 1) publish(0);
    named_sync(1, kDecConsumers);
    if (warp == 0) {
      absorb(0);
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        if (r >= p.R) break;
        const bool live = (m_run[r] != -INFINITY) && (l_w[r] > 0.f);
        const float inv = live ? 1.f / l_w[r] : 0.f;
        const float lse = live ? (m_run[r] + __log2f(l_w[r])) * kLn2 : -INFINITY;
        const int g = r / p.Sq, i = r % p.Sq;
        const int h = itm.hk * p.G + g;
        const size_t row = (static_cast<size_t>(itm.b) * p.Sq + i) * p.H + h;
        if (p.num_splits == 1) {
          uint8_t* orow = static_cast<uint8_t*>(p.out) + (row * D + e0) * 2;
          if constexpr (Cfg::kCols == 4) {
            *reinterpret_cast<uint2*>(orow) =
                make_uint2(pack2<BF16>(acc[r][0] * inv, acc[r][1] * inv),
                           pack2<BF16>(acc[r][2] * inv, acc[r][3] * inv));
          } else {
            *reinterpret_cast<uint32_t*>(orow) = pack2<BF16>(acc[r][0] * inv, acc[r][1] * inv);
          }
          if (lane == 0 && p.lse != nullptr)
            p.lse[(static_cast<size_t>(itm.b) * p.H + h) * p.Sq + i] = lse;
        } else {
          const size_t prow = static_cast<size_t>(itm.split) * p.B * p.Sq * p.H + row;
          float* orow = p.ws_o + prow * D + e0;
#pragma unroll
          for (int c = 0; c < Cfg::kCols; ++c) orow[c] = acc[r][c] * inv;
          if (lane == 0) p.ws_lse[prow] = lse;
        }
      }
    }
    // red[] and accs[] are rewritten by the next item
    named_sync(1, kDecConsumers);
  }
}

}  // namespace fa
