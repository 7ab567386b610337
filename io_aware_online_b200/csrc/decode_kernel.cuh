// decode_kernel.cuh -- split-KV attention of a few query rows against a (paged) KV
// cache, sm_100a.  Changelog post: v2.2 split-KV ("flash-decoding": the KV cache
// is cut along the sequence, each block handles one range, an extra kernel
// reduces) and v2.5 paged KV cache (a block_table addresses the pages);
// "FlashAttention common interfaces" section 3.3 for the argument set.
//
// This path is bound by HBM bandwidth (about 2 FMAs per cache byte), so it runs
// on the CUDA cores and spends its effort on the memory stream:
//   CTA = (split s, KV head hk, sequence b); 160 threads:
//     warps 0-3  consumers: scores, online softmax and P*V for all R = G * Sq
//                query rows of the KV head, so each cache byte is read once
//     warp  4    TMA producer: 64-token K and V tiles of one KV head through a
//                3-stage ring (block_table looked up once per tile)
//   Scores: thread (token pair, quarter of the head dim) -> shuffle reduction.
//   P*V:    thread (pair of head-dim columns, token group) -> register
//           accumulators, reduced across groups at the end of the split.
// Keys past cache_seqlens[b] (page tails, possibly garbage) are masked by
// selection and skipped in P*V, so nothing they hold can reach the output.
#pragma once

#include <climits>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

constexpr int kDecTok = 64;       // tokens per tile
constexpr int kDecStages = 3;
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
  static constexpr int kQOff = kDecStages * kStageBytes;
  static constexpr int kQBytes = RMAX * 4 * kQPartStride * 4;
  static constexpr int kPOff = kQOff + kQBytes;
  static constexpr int kPBytes = kDecTok * RMAX * 4;
  static constexpr int kRedOff = kPOff + kPBytes;
  static constexpr int kRedBytes = 4 * RMAX * 4;
  static constexpr int kBarOff = (kRedOff + kRedBytes + 7) & ~7;
  static constexpr int kMiscOff = kBarOff + 2 * kDecStages * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static constexpr int kPairs = D / 2;                   // head-dim column pairs
  static constexpr int kGroups = kDecConsumers / kPairs; // token groups in P*V
  static_assert(kGroups * kPairs == kDecConsumers, "thread split");
  static_assert(kDecStages * kStageBytes >= kDecConsumers * RMAX * 8, "reduction space");
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

template <int D, bool BF16, int RMAX>
__global__ void __launch_bounds__(kDecThreads)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecodeParams p) {
  using Cfg = DecCfg<D, RMAX>;
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.6931471805599453f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* q_s = reinterpret_cast<float*>(smem + Cfg::kQOff);
  float* p_s = reinterpret_cast<float*>(smem + Cfg::kPOff);
  float* red = reinterpret_cast<float*>(smem + Cfg::kRedOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* empty = full + kDecStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff);

  const int tid = threadIdx.x;
  const int warp = tid / 32, lane = tid % 32;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;

  // ---------------------------------------------------------- key range of this CTA
  const int L = (p.cache_seqlens != nullptr) ? p.cache_seqlens[b] : p.seqlen_k_max;
  const int n_units = (L + p.unit - 1) / p.unit;
  const int per = (n_units + p.num_splits - 1) / p.num_splits;
  const int u_begin = split * per;
  const int u_end = min(n_units, u_begin + per);
  const bool has_left = p.wl >= 0;
  const bool has_right = p.causal || p.wr >= 0;
  const int right = p.causal ? 0 : p.wr;
  const int off = L - p.Sq;  // query i sits at key position i + off
  int kb_lo = u_begin * p.unit;
  int kb_hi = min(u_end * p.unit, L);
  if (has_left) kb_lo = max(kb_lo, off - p.wl);                     // row i = 0
  if (has_right) kb_hi = min(kb_hi, p.Sq - 1 + off + right + 1);    // row i = Sq-1
  kb_lo = max(kb_lo, 0);
  const int t_lo = kb_lo / kDecTok;
  const int n_tiles = (kb_hi > kb_lo) ? (kb_hi + kDecTok - 1) / kDecTok - t_lo : 0;

  if (tid == kDecConsumers) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kDecConsumers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // query rows of this KV head -> shared memory (fp32, split into padded quarters)
  for (int idx = tid; idx < RMAX * D; idx += kDecThreads) {
    const int r = idx / D, e = idx % D;
    float qv = 0.f;
    if (r < p.R) {
      const int g = r / p.Sq, i = r % p.Sq;
      const int h = hk * p.G + g;
      const size_t qi = ((static_cast<size_t>(b) * p.Sq + i) * p.H + h) * D + e;
      if constexpr (BF16)
        qv = __bfloat162float(static_cast<const __nv_bfloat16*>(p.q)[qi]);
      else
        qv = __half2float(static_cast<const __half*>(p.q)[qi]);
    }
    q_s[(r * 4 + e / Cfg::kPart) * Cfg::kQPartStride + e % Cfg::kPart] = qv;
  }
  __syncthreads();
  const WaitCtx w{abort_flag, p.status, p.timeout_ns};
  uint8_t* stage0 = smem;

  if (warp == kDecConsumers / 32) {
    // ======================================================== TMA producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      int last[kDecStages];
      for (int s = 0; s < kDecStages; ++s) last[s] = -1;
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % kDecStages;
        const uint32_t ph = (n / kDecStages) & 1;
        if (!wait_bounded(empty + s, ph ^ 1, w)) break;
        const int tok0 = (t_lo + n) * kDecTok;
        int c2, c3;
        if (p.block_table != nullptr) {
          int blk = p.block_table[static_cast<size_t>(b) * p.max_blocks + tok0 / p.page_size];
          if (blk < 0 || blk >= p.num_blocks) {
            atomicOr(p.status, kDevBadBlock);
            blk = 0;  // read a valid page; the status word reports the fault
          }
          c2 = tok0 % p.page_size;
          c3 = blk;
        } else {
          c2 = tok0;
          c3 = b;
        }
        uint8_t* st = stage0 + s * Cfg::kStageBytes;
        mbar_arrive_expect_tx(full + s, Cfg::kStageBytes);
#pragma unroll
        for (int c = 0; c < Cfg::kChunks; ++c) {
          tma_load_4d(st + c * Cfg::kChunkBytes, &tmK, full + s, c * 64, hk, c2, c3);
          tma_load_4d(st + Cfg::kTileBytes + c * Cfg::kChunkBytes, &tmV, full + s, c * 64, hk,
                      c2, c3);
        }
        last[s] = ph;
      }
      if (*abort_flag) {
        for (int s = 0; s < kDecStages; ++s)
          if (last[s] >= 0) dec_wait_drain(full + s, last[s], p.timeout_ns);
      }
    }
    __syncwarp();
    return;
  }

  // ========================================================== consumers
  // scores: token pair tp (tokens tp and tp + 32), quarter `part` of the head dim
  const int tp = tid / 4, part = tid % 4;
  // P*V: head-dim column pair dp, token group grp
  const int dp = tid % Cfg::kPairs, grp = tid / Cfg::kPairs;
  int lo_r[RMAX], hi_r[RMAX];
  float slope2[RMAX], cpos[RMAX];
#pragma unroll
  for (int r = 0; r < RMAX; ++r) {
    const int i = (r < p.R) ? r % p.Sq : 0;
    const int c = i + off;
    lo_r[r] = (r < p.R && has_left) ? c - p.wl : INT_MIN / 2;
    hi_r[r] = (r < p.R && has_right) ? min(c + right, L - 1) : L - 1;
    const int h = hk * p.G + ((r < p.R) ? r / p.Sq : 0);
    slope2[r] = (p.alibi != nullptr) ? p.alibi[h] * kLog2e : 0.f;
    cpos[r] = static_cast<float>(c);
  }
  float m_run[RMAX], l_part[RMAX];
  float2 acc[RMAX];
#pragma unroll
  for (int r = 0; r < RMAX; ++r) {
    m_run[r] = -INFINITY;
    l_part[r] = 0.f;
    acc[r] = make_float2(0.f, 0.f);
  }

  for (int n = 0; n < n_tiles; ++n) {
    const int s = n % kDecStages;
    const uint32_t ph = (n / kDecStages) & 1;
    const bool ok = wait_bounded(full + s, ph, w);
    const uint8_t* sK = stage0 + s * Cfg::kStageBytes;
    const uint8_t* sV = sK + Cfg::kTileBytes;
    const int tok0 = (t_lo + n) * kDecTok;

    // ---- scores for tokens tp and tp + 32
    float sa[RMAX], sb[RMAX];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) sa[r] = sb[r] = 0.f;
    const int ta = tp, tb = tp + 32;
#pragma unroll
    for (int u = 0; u < Cfg::kPart / 8; ++u) {
      const int e0 = part * Cfg::kPart + u * 8;
      const int chunk = e0 / 64, u16 = (e0 % 64) / 8;
      const uint4 ka = *reinterpret_cast<const uint4*>(sK + chunk * Cfg::kChunkBytes + ta * 128 +
                                                       ((u16 ^ (ta & 7)) << 4));
      const uint4 kb = *reinterpret_cast<const uint4*>(sK + chunk * Cfg::kChunkBytes + tb * 128 +
                                                       ((u16 ^ (tb & 7)) << 4));
      float fa[8], fb[8];
      {
        float2 t0 = unpack2<BF16>(ka.x), t1 = unpack2<BF16>(ka.y), t2 = unpack2<BF16>(ka.z),
               t3 = unpack2<BF16>(ka.w);
        fa[0] = t0.x; fa[1] = t0.y; fa[2] = t1.x; fa[3] = t1.y;
        fa[4] = t2.x; fa[5] = t2.y; fa[6] = t3.x; fa[7] = t3.y;
        t0 = unpack2<BF16>(kb.x); t1 = unpack2<BF16>(kb.y); t2 = unpack2<BF16>(kb.z);
        t3 = unpack2<BF16>(kb.w);
        fb[0] = t0.x; fb[1] = t0.y; fb[2] = t1.x; fb[3] = t1.y;
        fb[4] = t2.x; fb[5] = t2.y; fb[6] = t3.x; fb[7] = t3.y;
      }
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        const float4* qp =
            reinterpret_cast<const float4*>(q_s + (r * 4 + part) * Cfg::kQPartStride + u * 8);
        const float4 q0 = qp[0], q1 = qp[1];
        sa[r] = fmaf(q0.x, fa[0], sa[r]); sa[r] = fmaf(q0.y, fa[1], sa[r]);
        sa[r] = fmaf(q0.z, fa[2], sa[r]); sa[r] = fmaf(q0.w, fa[3], sa[r]);
        sa[r] = fmaf(q1.x, fa[4], sa[r]); sa[r] = fmaf(q1.y, fa[5], sa[r]);
        sa[r] = fmaf(q1.z, fa[6], sa[r]); sa[r] = fmaf(q1.w, fa[7], sa[r]);
        sb[r] = fmaf(q0.x, fb[0], sb[r]); sb[r] = fmaf(q0.y, fb[1], sb[r]);
        sb[r] = fmaf(q0.z, fb[2], sb[r]); sb[r] = fmaf(q0.w, fb[3], sb[r]);
        sb[r] = fmaf(q1.x, fb[4], sb[r]); sb[r] = fmaf(q1.y, fb[5], sb[r]);
        sb[r] = fmaf(q1.z, fb[6], sb[r]); sb[r] = fmaf(q1.w, fb[7], sb[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      sa[r] += __shfl_xor_sync(0xffffffffu, sa[r], 1);
      sa[r] += __shfl_xor_sync(0xffffffffu, sa[r], 2);
      sb[r] += __shfl_xor_sync(0xffffffffu, sb[r], 1);
      sb[r] += __shfl_xor_sync(0xffffffffu, sb[r], 2);
    }
    // ---- score transform (base-2 units) and mask
    const int ja = tok0 + ta, jb = tok0 + tb;
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      float xa = sa[r], xb = sb[r];
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
    }
    // ---- tile max per row: lanes 4 apart hold different tokens
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      float mx = fmaxf(sa[r], sb[r]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      if (lane == 0) red[warp * RMAX + r] = mx;
    }
    if (named_sync_or(1, kDecConsumers, !ok)) break;
    float alpha[RMAX];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      const float mt = fmaxf(fmaxf(red[r], red[RMAX + r]), fmaxf(red[2 * RMAX + r], red[3 * RMAX + r]));
      const float m_new = fmaxf(m_run[r], mt);
      alpha[r] = (m_new == -INFINITY) ? 1.f : ex2(m_run[r] - m_new);
      m_run[r] = m_new;
      const float pa = (sa[r] == -INFINITY) ? 0.f : ex2(sa[r] - m_new);
      const float pb = (sb[r] == -INFINITY) ? 0.f : ex2(sb[r] - m_new);
      if (part == 0) {
        p_s[ta * RMAX + r] = pa;
        p_s[tb * RMAX + r] = pb;
        l_part[r] = fmaf(l_part[r], alpha[r], pa + pb);
      }
    }
    named_sync(1, kDecConsumers);
    // ---- P * V for this thread's column pair over its token group
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      acc[r].x *= alpha[r];
      acc[r].y *= alpha[r];
    }
    const int n_valid = min(kDecTok, L - tok0);  // keys at or past L are never touched
    const int chunk = (2 * dp) / 64, u16 = ((2 * dp) % 64) / 8, wi = (dp & 3) * 4;
#pragma unroll 4
    for (int tok = grp; tok < n_valid; tok += Cfg::kGroups) {
      const uint32_t vw = *reinterpret_cast<const uint32_t*>(
          sV + chunk * Cfg::kChunkBytes + tok * 128 + ((u16 ^ (tok & 7)) << 4) + wi);
      const float2 v2 = unpack2<BF16>(vw);
      const float* pr = p_s + tok * RMAX;
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        const float pv = pr[r];
        acc[r].x = fmaf(pv, v2.x, acc[r].x);
        acc[r].y = fmaf(pv, v2.y, acc[r].y);
      }
    }
    mbar_arrive(empty + s);
  }

  // ---------------------------------------------------------- end of split
  // row sums: part-0 lanes hold partial sums over their tokens
  named_sync(1, kDecConsumers);
#pragma unroll
  for (int r = 0; r < RMAX; ++r) {
    float v = (part == 0) ? l_part[r] : 0.f;
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    if (lane == 0) red[warp * RMAX + r] = v;
  }
  // column-pair accumulators of every token group -> stage memory
  float2* accs = reinterpret_cast<float2*>(stage0);
#pragma unroll
  for (int r = 0; r < RMAX; ++r) accs[(grp * RMAX + r) * Cfg::kPairs + dp] = acc[r];
  named_sync(1, kDecConsumers);
  if (*abort_flag) return;
  if (grp == 0) {
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      if (r >= p.R) break;
      float2 o = acc[r];
      for (int g2 = 1; g2 < Cfg::kGroups; ++g2) {
        const float2 t = accs[(g2 * RMAX + r) * Cfg::kPairs + dp];
        o.x += t.x;
        o.y += t.y;
      }
      const float l = red[r] + red[RMAX + r] + red[2 * RMAX + r] + red[3 * RMAX + r];
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      const float lse = (l > 0.f) ? (m_run[r] + __log2f(l)) * kLn2 : -INFINITY;
      const int g = r / p.Sq, i = r % p.Sq;
      const int h = hk * p.G + g;
      const size_t row = (static_cast<size_t>(b) * p.Sq + i) * p.H + h;
      if (p.num_splits == 1) {
        uint32_t* orow = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(p.out) + row * D * 2);
        orow[dp] = pack2<BF16>(o.x * inv, o.y * inv);
        if (dp == 0 && p.lse != nullptr)
          p.lse[(static_cast<size_t>(b) * p.H + h) * p.Sq + i] = lse;
      } else {
        const size_t prow = static_cast<size_t>(split) * p.B * p.Sq * p.H + row;
        reinterpret_cast<float2*>(p.ws_o + prow * D)[dp] = make_float2(o.x * inv, o.y * inv);
        if (dp == 0) p.ws_lse[prow] = lse;
      }
    }
  }
}

}  // namespace fa
