// bwd_kernel.cuh -- attention backward for sm_100a: dQ, dK, dV of
// O = softmax(mask(softcap(scale Q K^T)) + ALiBi) V, recomputing the attention
// matrix tile by tile from Q, K and the forward's LSE instead of storing it (tag
// page "flash attention": the backward recomputes S and P in on-chip memory).
//
// With X = scale Q K^T, S = c tanh(X / c) under a softcap c (changelog v2.6) and
// S = X otherwise, P = exp(S - LSE), dP = dO V^T, D = rowsum(dO * O),
// dS = P * (dP - D) and dX = dS * (1 - tanh(X / c)^2) (dX = dS without a softcap):
//   dV = P^T dO,  dK = scale * dX^T Q,  dQ = scale * dX K.
// Varlen batches (section 3.2) run each packed sequence as its own problem: a
// CTA reads its sequence's offsets from cu_seqlens and masks the rows of the
// neighbouring sequences that its tiles reach.
// Two kernels, all deterministic (no atomics): bwd_dot_kernel, then bwd_tiles_kernel,
// whose grid holds the dK/dV CTAs followed by the dQ CTAs.
//   bwd_dot_kernel   D for every query row (one warp per row).
//   dK/dV CTAs       one CTA per (128-key block, KV head): K_j and V_j stay in
//                    shared memory while the query blocks (of every query head
//                    reading this KV head) stream past; per block
//                      S^T = K_j Q_i^T, dP^T = V_j dO_i^T   (tcgen05, SS)
//                      P^T, dS^T in registers -> 16-bit in tensor memory
//                      dV += P^T dO_i, dK += dS^T Q_i        (tcgen05, TS)
//                    with dV and dK accumulated in tensor memory.
//   dQ CTAs          one CTA per (128-query block, head): Q_i and dO_i stay in
//                    shared memory while the key blocks stream past; per block
//                      S = Q_i K_j^T, dP = dO_i V_j^T, dS -> 16-bit,
//                      dQ += dS K_j                           (tcgen05)
// Roles per CTA (384 threads): warps 0-7 compute in two warpgroups that split
// each block's columns (thread r of a warpgroup owns tensor-memory lane r: a key
// row in dK/dV, a query row in dQ), warp 8 TMA producer (K, V and the Q stream in
// dK/dV; Q, dO and the K/V streams in dQ), warp 9 MMA issuer (one elected thread;
// it also allocates tensor memory), warp 10 the dO and statistics stream of dK/dV,
// warp 11 idle.  Tensor memory of a dK/dV CTA: S^T [0,128), dP^T [128,256), dV and
// dK from 256; each warpgroup writes its P^T and dS^T as 16-bit pairs over its own
// score columns [64 c, 64 c + 32) once those scores are in registers.  The dQ CTA's
// layout is given above it.  Every wait is bounded.
// Included by bwd.cu (dense batches) and bwd_varlen.cu (packed sequences), which
// compile in parallel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>

#include "fa_internal.h"
#include "fwd_kernel.cuh"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr float kBwdLog2e = 1.4426950408889634f;

// Shared memory of the dK/dV kernel: K_j and V_j, a three-stage ring of Q_i, a
// two-stage ring of dO_i and the column statistics of each dO stage.  Q_i is read
// by S^T(i), early in a block, and by dK(i), its last product: with three stages the
// tile two blocks ahead is requested as soon as dK of the block before is done, so
// it has landed before S^T wants it.  At D = 128 this fills the 227 KiB a CTA may
// have, with no room left to align the base: the kernel relies on the dynamic shared
// memory starting on a 1 KiB boundary (it does, at shared address 0x400, measured)
// and checks it.
template <int D>
struct BwdCfg {
  static constexpr int kChunks = D / 64;              // 128-byte swizzle atoms per row
  static constexpr int kTileBytes = 128 * D * 2;      // one 128-row tile
  static constexpr int kChunkBytes = 128 * 128;
  static constexpr int kQStages = 3, kDoStages = 2;
  static constexpr int kFixA = 0;                     // K_j
  static constexpr int kFixB = kTileBytes;            // V_j
  static constexpr int kQ = 2 * kTileBytes;           // Q ring
  static constexpr int kDo = kQ + kQStages * kTileBytes;  // dO ring
  // column statistics [2 slots][LSE * log2 e | D][kStatPitch] fp32: a tensor copy must
  // start at a column that is a multiple of 4 (16 bytes), so a varlen block whose rows
  // start elsewhere loads from the multiple of 4 below it, kStatLen columns wide, and is
  // read from the remainder on; each copy's destination sits on 128 bytes (the pitch)
  static constexpr int kStatLen = 132;
  static constexpr int kStatPitch = 160;  // 640 bytes: a multiple of 128
  static constexpr int kStat = kDo + kDoStages * kTileBytes;
  static constexpr int kBarOff = kStat + kDoStages * 2 * kStatPitch * 4;
  static_assert(kStat % 128 == 0 && (kStatPitch * 4) % 128 == 0, "tensor copy destinations");
  // fix_full, q_full[3], q_empty[3], do_full[2], do_empty[2], s_full, p_full, done,
  // drain, dp_full, ds_full
  static constexpr int kNumBars = 1 + 2 * kQStages + 2 * kDoStages + 6;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  // at least 116 KiB, so that one CTA fills an SM (each takes all 512 tensor-memory
  // columns; a second one would wait in its allocation for the first to finish)
  static constexpr int kSmemAlloc = (kSmemBytes > 116 * 1024) ? kSmemBytes : 116 * 1024;
  static_assert(kSmemAlloc <= 227 * 1024, "dK/dV tiles exceed shared memory");
  static constexpr int kTmemCols = 512;                 // S^T 128 + dP^T 128 + 2 x D
};

// Shared memory of the dQ kernel: Q_i and dO_i, then separate rings of K_j (three
// stages: K_j is read until dQ(j)) and V_j (two stages: V_j is released once dP(j)
// has run), so that the tiles of block j+1 arrive while block j is processed.
template <int D>
struct DqCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kChunkBytes = 128 * 128;
  static constexpr int kKStages = 3, kVStages = 2;
  static constexpr int kFixA = 0;                      // Q_i
  static constexpr int kFixB = kTileBytes;             // dO_i
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + kKStages * kTileBytes;
  static constexpr int kBarOff = kV + kVStages * kTileBytes;
  // fix_full, k_full[3], k_empty[3], v_full[2], v_empty[2], s_full, p_full[2],
  // dp_read, done, drain, dp_full
  static constexpr int kNumBars = 18;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc =
      (kSmemBytes + 1024 > 116 * 1024) ? kSmemBytes + 1024 : 116 * 1024;
  static_assert(kSmemAlloc <= 227 * 1024, "dQ tiles exceed shared memory");
  static constexpr int kTmemCols = 512;                // S 2 x 128 + dP 128 + dQ <= 128
};

// Key j allowed for query i (bottom-right alignment, off = Sk - Sq).
struct MaskGeo {
  int off, Sk, Sq, wl, right;
  bool has_left, has_right;
  // branch-free, so that a masked tile's loop stays one basic block
  __device__ __forceinline__ bool allowed(int i, int j) const {
    const int c = i + off;
    return (i < Sq) & (j < Sk) & (!has_right | (j <= c + right)) & (!has_left | (j >= c - wl));
  }
  // every (query, key) of the 128 x 128 tile at (i0, j0) allowed: no mask needed
  __device__ __forceinline__ bool tile_open(int i0, int j0) const {
    if (i0 + 127 >= Sq || j0 + 127 >= Sk) return false;
    if (has_right && j0 + 127 > i0 + off + right) return false;
    if (has_left && j0 < i0 + 127 + off - wl) return false;
    return true;
  }
};

__device__ __forceinline__ MaskGeo mask_geo(const BwdParams& p, int Sq, int Sk) {
  MaskGeo g;
  g.off = Sk - Sq;
  g.Sk = Sk;
  g.Sq = Sq;
  g.wl = p.wl;
  g.has_left = p.wl >= 0;
  g.has_right = p.causal || p.wr >= 0;
  g.right = p.causal ? 0 : p.wr;
  return g;
}

// One sequence of the batch: its first query / key row in the packed tensors (0
// when dense), its lengths, and the batch coordinate of the tensor maps.  Varlen
// is a compile-time switch, so that dense kernels keep their lengths in the
// parameter bank rather than in registers.
struct BwdSeq {
  int qs, ks, Sq, Sk, bc;
};
template <bool VARLEN>
__device__ __forceinline__ BwdSeq bwd_seq(const BwdParams& p, int b) {
  BwdSeq q{0, 0, p.Sq, p.Sk, b};
  if constexpr (VARLEN) {
    q.qs = p.cu_q[b];
    q.Sq = p.cu_q[b + 1] - q.qs;
    q.ks = p.cu_k[b];
    q.Sk = p.cu_k[b + 1] - q.ks;
    q.bc = 0;
  }
  return q;
}

// A CTA's (block, head, sequence) from its index lin in a grid of nb blocks x nh heads
// x ns sequences, dispatched in groups of kGridGroup (sequence, head) pairs: blocks
// slowest inside a group, so the heaviest block of every pair in the group starts
// first and the grid ends on light blocks, while at most two groups' streamed tiles
// are live at once and stay in L2.
constexpr int kGridGroup = 8;
struct GridPos {
  int blk, head, seq;
};
__device__ __forceinline__ GridPos grid_pos(long long lin, int nb, int nh, int ns) {
  const long long nhs = static_cast<long long>(nh) * ns;
  const long long per = static_cast<long long>(kGridGroup) * nb;
  const long long g = lin / per, r = lin % per;
  const long long gsz = min(static_cast<long long>(kGridGroup), nhs - g * kGridGroup);
  const long long hs = g * kGridGroup + r % gsz;
  return {static_cast<int>(r / gsz), static_cast<int>(hs % nh), static_cast<int>(hs / nh)};
}

// softcap c: x_raw = Q.K; r = 1 / (exp(2 scale x_raw / c) + 1), tanh(scale x_raw / c) =
// 1 - 2 r, and its derivative factor 1 - tanh^2 = 4 r (1 - r) (no cancellation near
// saturation).  Returns the score in base-2 units, c log2(e) (1 - 2 r), and g.
__device__ __forceinline__ float softcap_score(float x_raw, const BwdParams& p, float* g) {
  const float r = rcp(ex2(x_raw * p.tanh_k) + 1.f);
  *g = 4.f * r * (1.f - r);
  return fmaf(-2.f * p.softcap_log2, r, p.softcap_log2);
}

__device__ __forceinline__ bool wait_drain_bwd(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// D[b, h, i] = sum_c dO[b, i, h, c] * O[b, i, h, c], fp32.  16-byte loads: a row is
// D / 8 lanes (16 at d = 128, 8 at d = 64), a warp takes 32 / (D / 8) rows.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_dot_kernel(const BwdParams p) {
  constexpr int kLanes = D / 8;
  constexpr int kRowsPerWarp = 32 / kLanes;
  const int lane = threadIdx.x % 32;
  const int l = lane % kLanes;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * 8 + threadIdx.x / 32) * kRowsPerWarp +
                      lane / kLanes;  // (b, i, h)
  const int bm = (p.cu_q != nullptr) ? 1 : p.B;  // varlen: one packed batch entry
  const bool live = row < static_cast<int64_t>(bm) * p.Sq * p.H;
  float acc = 0.f;
  if (live) {
    const int64_t at = row * D + l * 8;
    const uint4 o = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.out) + at);
    const uint4 g = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.dout) + at);
    const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 a = unpack2<BF16>(ow[e]);
      const float2 c = unpack2<BF16>(gw[e]);
      acc = fmaf(a.x, c.x, fmaf(a.y, c.y, acc));
    }
  }
#pragma unroll
  for (int m = kLanes / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if (live && l == 0) {
    const int h = static_cast<int>(row % p.H);
    const int64_t bi = row / p.H;  // b * Sq + i
    const int i = static_cast<int>(bi % p.Sq);
    const int b = static_cast<int>(bi / p.Sq);
    const int64_t bh = static_cast<int64_t>(b) * p.H + h;
    p.dvec[bh * p.sq_pad + i] = acc;
    p.lse2[bh * p.sq_pad + i] = p.lse[bh * p.Sq + i] * kBwdLog2e;  // base-2 LSE for P
  }
}

// Both tile passes run 384 threads: two compute warpgroups (warpgroup c takes
// columns [64 c, 64 c + 64) of every 128 x 128 block for the block's 128 rows),
// producer warps 8 (and 10 in dK/dV), warp 9 MMA issuer, the rest idle.
constexpr int kWideThreads = 384;
// registers per thread: 168 at launch (one CTA per SM); the compute warpgroups
// take what the producer, the MMA issuer and the idle warps do not need
constexpr uint32_t kBwdLaunchRegs = 168, kBwdComputeRegs = 208, kBwdOtherRegs = 88;
static_assert(256 * kBwdComputeRegs + 128 * kBwdOtherRegs == kWideThreads * kBwdLaunchRegs,
              "register re-split must add up to the launch registers");

// One CTA per (128-key block kb, KV head hk, batch b).

// O (+)= A B, A (16-bit, 128 keys or queries along K) from tensor memory in two runs
// of 32 columns: [a, a + 32) holds K-steps 0..63 and [a + 64, a + 96) K-steps
// 64..127, because each compute warpgroup writes its 16-bit values over its own
// 64 score columns.  B MN-major as in fwd_issue_pv (16 rows = 2 KiB a step).
__device__ __forceinline__ void bwd_issue_split_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0,
                                                  uint32_t idesc, bool acc) {
  const uint32_t b_lo = static_cast<uint32_t>(b0), b_hi = static_cast<uint32_t>(b0 >> 32);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts(d_tmem, a_tmem + (kk / 4) * 64 + (kk % 4) * 8, desc_pack(b_lo + kk * (2048 >> 4), b_hi),
           idesc, (acc || kk > 0) ? 1u : 0u);
}

template <int D, bool BF16, bool ALIBI, bool SOFTCAP, bool VARLEN>
__device__ __forceinline__ void bwd_dkdv_cta(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                             const CUtensorMap& tmV, const CUtensorMap& tmDO,
                                             const CUtensorMap& tmL, const CUtensorMap& tmD,
                                             const BwdParams& p, long long lin) {
  using Cfg = BwdCfg<D>;
  constexpr int QS = Cfg::kQStages, DS = Cfg::kDoStages;
  extern __shared__ uint8_t smem_raw[];
  // the layout has no slack to align the base: it must already sit on 1 KiB
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // uniform: nothing set up yet
    if (threadIdx.x == 0) atomicOr(p.status, kDevSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // grid: key blocks x KV heads x sequences in groups of (sequence, KV head) pairs
  // (grid_pos): the CTAs that stream one head's query tiles run together and find
  // them in L2; key block 0 (seen by every query block under a causal mask) first
  const GridPos gp = grid_pos(lin, (p.rows_k + 127) / 128, p.Hkv, p.B);
  const int k0 = gp.blk * 128;
  const int hk = gp.head;
  const int b = gp.seq;
  const BwdSeq sq = bwd_seq<VARLEN>(p, b);
  if (k0 >= sq.Sk) return;  // uniform: past this sequence's keys (varlen), nothing set up yet
  const MaskGeo mg = mask_geo(p, sq.Sq, sq.Sk);
  // query rows that see some key of [k0, k1)
  const int k1 = min(k0 + 128, sq.Sk);
  const int q_lo = mg.has_right ? max(0, k0 - mg.off - mg.right) : 0;
  const int q_hi = mg.has_left ? min(sq.Sq - 1, k1 - 1 - mg.off + mg.wl) : sq.Sq - 1;
  const int i_lo = q_lo / 128;
  const int nqb = (q_hi >= q_lo) ? q_hi / 128 - i_lo + 1 : 0;
  const int n_iter = p.G * nqb;  // iteration n: head hk * G + n / nqb, query block i_lo + n % nqb

  uint8_t* fixA = smem + Cfg::kFixA;  // K_j
  uint8_t* fixB = smem + Cfg::kFixB;  // V_j
  uint8_t* q_ring = smem + Cfg::kQ;    // slot n % 3: Q of block n
  uint8_t* do_ring = smem + Cfg::kDo;  // slot n % 2: dO of block n
  float* stat = reinterpret_cast<float*>(smem + Cfg::kStat);  // [dO slot][lse2 | D][pitch]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* fix_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* q_empty = q_full + QS;
  uint64_t* do_full = q_empty + QS;  // dO and the column statistics
  uint64_t* do_empty = do_full + DS;
  uint64_t* s_full = do_empty + DS;
  uint64_t* p_full = s_full + 1;
  uint64_t* done = s_full + 2;
  uint64_t* drain = s_full + 3;
  uint64_t* dp_full = s_full + 4;
  uint64_t* ds_full = s_full + 5;
  static_assert(1 + 2 * QS + 2 * DS + 6 == Cfg::kNumBars, "barrier count");
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);

  if (warp == 8 && lane == 0) {
    mbar_init(fix_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    for (int s = 0; s < DS; ++s) {
      mbar_init(do_full + s, 1);
      mbar_init(do_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 8);   // one arrival per compute warp
    mbar_init(ds_full, 8);
    mbar_init(done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_holder, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const WaitCtx w{abort_flag, p.status, p.timeout_ns};

  // register re-split inside the role branches (a merge of the two limits before
  // them would hold all later code to the smaller one)
  if (warp >= 8) {
   regs_dec<kBwdOtherRegs>();
   if (warp == 8) {
    // ======================================================== TMA producer
    if (lane == 0 && n_iter > 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      tma_prefetch_map(&tmDO);
      mbar_arrive_expect_tx(fix_full, 2 * Cfg::kTileBytes);
      for (int c = 0; c < Cfg::kChunks; ++c) {
        tma_load_4d(fixA + c * Cfg::kChunkBytes, &tmK, fix_full, c * 64, sq.ks + k0, hk, sq.bc);
        tma_load_4d(fixB + c * Cfg::kChunkBytes, &tmV, fix_full, c * 64, sq.ks + k0, hk, sq.bc);
      }
      // the Q stream (the dO stream and the statistics are warp 10's)
      int last[QS];
      for (int s = 0; s < QS; ++s) last[s] = -1;
      for (int n = 0; n < n_iter; ++n) {
        const int s = n % QS;
        const uint32_t ph = (n / QS) & 1;
        const int h = hk * p.G + n / nqb;
        const int qb = (i_lo + n % nqb) * 128;
        if (!wait_bounded(q_empty + s, ph ^ 1, w)) break;
        mbar_arrive_expect_tx(q_full + s, Cfg::kTileBytes);
        for (int c = 0; c < Cfg::kChunks; ++c)
          tma_load_4d(q_ring + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, &tmQ, q_full + s,
                      c * 64, sq.qs + qb, h, sq.bc);
        last[s] = ph;
      }
      if (*abort_flag) {  // let this CTA's own copies land before the smem goes away
        wait_drain_bwd(fix_full, 0, p.timeout_ns);
        for (int s = 0; s < QS; ++s)
          if (last[s] >= 0) wait_drain_bwd(q_full + s, last[s], p.timeout_ns);
      }
    }
    __syncwarp();
   } else if (warp == 10) {
    // ======================================================== TMA producer: dO
    if (lane == 0 && n_iter > 0) {
      int last[DS];
      for (int s = 0; s < DS; ++s) last[s] = -1;
      for (int n = 0; n < n_iter; ++n) {
        const int s = n % DS;
        const uint32_t ph = (n / DS) & 1;
        const int h = hk * p.G + n / nqb;
        const int qb = (i_lo + n % nqb) * 128;
        if (!wait_bounded(do_empty + s, ph ^ 1, w)) break;
        // dO_i and the block's column statistics (LSE * log2 e and D; zero past the
        // end of the rows, where the mask keeps P at 0)
        constexpr int kStatBox = VARLEN ? Cfg::kStatLen : 128;  // the tensor maps' box width
        const int x0 = VARLEN ? ((sq.qs + qb) & ~3) : sq.qs + qb;
        mbar_arrive_expect_tx(do_full + s, Cfg::kTileBytes + 2 * kStatBox * 4);
        for (int c = 0; c < Cfg::kChunks; ++c)
          tma_load_4d(do_ring + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, &tmDO, do_full + s,
                      c * 64, sq.qs + qb, h, sq.bc);
        tma_load_2d(stat + (2 * s) * Cfg::kStatPitch, &tmL, do_full + s, x0, sq.bc * p.H + h);
        tma_load_2d(stat + (2 * s + 1) * Cfg::kStatPitch, &tmD, do_full + s, x0, sq.bc * p.H + h);
        last[s] = ph;
      }
      if (*abort_flag) {
        for (int s = 0; s < DS; ++s)
          if (last[s] >= 0) wait_drain_bwd(do_full + s, last[s], p.timeout_ns);
      }
    }
    __syncwarp();
   } else if (warp == 9) {
    // ======================================================== MMA issuer
    if (lane == 0 && n_iter > 0) {
      constexpr uint32_t idesc_s = f16_idesc(BF16, 128, 128, false, false);
      constexpr uint32_t idesc_acc = f16_idesc(BF16, 128, D, false, true);
      const uint64_t dKk = sw128_desc(smem_u32(fixA), 16, 1024);  // K-major operands
      const uint64_t dVk = sw128_desc(smem_u32(fixB), 16, 1024);
      // Software pipeline, in issue order:
      //   S^T(0), dP^T(0); per block n:
      //   [P^T(n) ready] dV(n), S^T(n+1); [dS^T(n) ready] dK(n), dP^T(n+1)
      // so the compute warps' dS^T(n) overlaps dV(n) and S^T(n+1), and their
      // P^T(n+1) overlaps dK(n) and dP^T(n+1).  A product that overwrites a region
      // (S^T(n+1) over P^T(n), dP^T(n+1) over dS^T(n)) is issued after the one
      // reading it, and each commit covers every earlier product of this thread.
      auto st_q = [&](int n) { return smem_u32(q_ring + (n % QS) * Cfg::kTileBytes); };
      auto st_do = [&](int n) { return smem_u32(do_ring + (n % DS) * Cfg::kTileBytes); };
      bool ok = wait_bounded(fix_full, 0, w) && wait_bounded(q_full, 0, w);
      if (ok) {
        tc_fence_after();
        fwd_issue_qk<D>(tbase, dKk, sw128_desc(st_q(0), 16, 1024), idesc_s);         // S^T(0)
        tc_commit(s_full);
        ok = wait_bounded(do_full, 0, w);
      }
      if (ok) {
        tc_fence_after();
        fwd_issue_qk<D>(tbase + 128, dVk, sw128_desc(st_do(0), 16, 1024), idesc_s);  // dP^T(0)
        tc_commit(dp_full);
      }
      for (int n = 0; n < n_iter && ok; ++n) {
        const bool more = n + 1 < n_iter;
        const int n1 = n + 1;
        if (!(ok = wait_bounded(p_full, n & 1, w))) break;
        tc_fence_after();
        // B operands MN-major: rows are queries, the head dim contiguous
        bwd_issue_split_a(tbase + 256, tbase, sw128_desc(st_do(n), Cfg::kChunkBytes, 1024),
                          idesc_acc, n > 0);                                      // dV(n)
        if (more) {
          if (!(ok = wait_bounded(q_full + n1 % QS, (n1 / QS) & 1, w))) break;
          tc_fence_after();
          fwd_issue_qk<D>(tbase, dKk, sw128_desc(st_q(n1), 16, 1024), idesc_s);      // S^T(n+1)
          tc_commit(s_full);
        }
        if (!(ok = wait_bounded(ds_full, n & 1, w))) break;
        tc_fence_after();
        bwd_issue_split_a(tbase + 256 + D, tbase + 128, sw128_desc(st_q(n), Cfg::kChunkBytes, 1024),
                          idesc_acc, n > 0);                                      // dK(n)
        // Q(n) and dO(n) (with the statistics the compute warps read until dS^T(n))
        // are done with
        tc_commit(q_empty + n % QS);
        tc_commit(do_empty + n % DS);
        if (more) {
          if (!(ok = wait_bounded(do_full + n1 % DS, (n1 / DS) & 1, w))) break;
          tc_fence_after();
          fwd_issue_qk<D>(tbase + 128, dVk, sw128_desc(st_do(n1), 16, 1024), idesc_s);  // dP^T(n+1)
          tc_commit(dp_full);
        }
      }
      if (ok) tc_commit(done);
      tc_commit(drain);
      wait_drain_bwd(drain, 0, p.timeout_ns);  // own MMAs complete before teardown
    }
    __syncwarp();
   }
  } else {
    regs_inc<kBwdComputeRegs>();
    // ======================================================== compute
    const int cg = warp / 4;  // query-column half of every block
    const int r = (warp % 4) * 32 + lane;  // key row within the block = TMEM lane
    const int k = k0 + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    bool ok = true;
    for (int n = 0; n < n_iter; ++n) {
      const int s = n % DS;  // the dO slot holding this block's column statistics
      const int h = hk * p.G + n / nqb;
      const int qb = (i_lo + n % nqb) * 128;
      const float slope2 = ALIBI ? p.alibi[h] * kBwdLog2e : 0.f;
      // the block's column statistics have landed, and S^T is ready
      ok = wait_bounded(do_full + s, (n / DS) & 1, w) && wait_bounded(s_full, n & 1, w);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // varlen: the statistics were loaded from the multiple of 4 below the block's
      // first row (rem > 0 breaks the 16-byte alignment of the vector reads below)
      const int rem = VARLEN ? ((sq.qs + qb) & 3) : 0;
      const float* lse2 = stat + (2 * s) * Cfg::kStatPitch + rem + cg * 64;
      const float* dd = stat + (2 * s + 1) * Cfg::kStatPitch + rem + cg * 64;
      auto ld4 = [&](const float* a) {
        if constexpr (VARLEN)
          return make_float4(a[0], a[1], a[2], a[3]);
        else
          return *reinterpret_cast<const float4*>(a);
      };
      // phase 1: P^T of this half (fp32 in registers), 16-bit copy to columns
      // [64 cg, 64 cg + 32), over this warpgroup's own S^T columns
      const bool open = mg.tile_open(qb, k0);  // uniform: the whole tile is unmasked
      float pf[64];
      uint32_t gh[SOFTCAP ? 32 : 1];  // softcap: 1 - tanh^2 per element, f16 pairs
      {
        uint32_t sv[64];
        tmem_ld32(tbase + cg * 64 + lane_off, sv);
        tmem_ld32(tbase + cg * 64 + 32 + lane_off, sv + 32);
        tmem_ld_wait(sv);
        tmem_ld_wait(sv + 32);

        // every exponential is taken and a masked one then dropped by a select: a
        // branch per element would split the loop into blocks of one exponential
        // each and expose the whole latency of every one
        // one pair in four is evaluated on the FMA pipe (exp2_fma2), the rest on MUFU
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        auto probs = [&](auto masked_t) {
          constexpr bool kMasked = decltype(masked_t)::value;
#pragma unroll
          for (int e = 0; e < 64; e += 4) {
            const float4 l4 = ld4(lse2 + e);  // one broadcast load, four columns
            float2 a[2];
            if constexpr (SOFTCAP) {
              float g4[4], x4[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) x4[u] = softcap_score(__uint_as_float(sv[e + u]), p, &g4[u]);
              a[0] = make_float2(x4[0] - l4.x, x4[1] - l4.y);
              a[1] = make_float2(x4[2] - l4.z, x4[3] - l4.w);
              gh[e / 2] = pack2<false>(g4[0], g4[1]);
              gh[e / 2 + 1] = pack2<false>(g4[2], g4[3]);
            } else {
              a[0] = fma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2,
                          make_float2(-l4.x, -l4.y));
              a[1] = fma2(make_float2(__uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3])), sc2,
                          make_float2(-l4.z, -l4.w));
            }
            if constexpr (ALIBI) {
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float bias = -slope2 * fabsf(static_cast<float>(qb + cg * 64 + e + u + mg.off - k));
                if (u % 2 == 0) a[u / 2].x += bias; else a[u / 2].y += bias;
              }
            }
            const float2 e0 = (e % 8 == 0) ? exp2_fma2(a[0]) : make_float2(ex2(a[0].x), ex2(a[0].y));
            const float2 e1 = make_float2(ex2(a[1].x), ex2(a[1].y));
            const float ev[4] = {e0.x, e0.y, e1.x, e1.y};
#pragma unroll
            for (int u = 0; u < 4; ++u)
              pf[e + u] = (!kMasked || mg.allowed(qb + cg * 64 + e + u, k)) ? ev[u] : 0.f;
          }
        };
        if (open)
          probs(std::false_type{});
        else
          probs(std::true_type{});
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pp[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pp[e] = pack2<BF16>(pf[c * 32 + 2 * e], pf[c * 32 + 2 * e + 1]);
        tmem_st16(tbase + cg * 64 + c * 16 + lane_off, pp);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      // phase 2: dS^T = P^T * (dP^T - D), 16-bit over this warpgroup's own dP^T columns
      ok = wait_bounded(dp_full, n & 1, w);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        uint32_t dp[64];
        tmem_ld32(tbase + 128 + cg * 64 + lane_off, dp);
        tmem_ld32(tbase + 128 + cg * 64 + 32 + lane_off, dp + 32);
        tmem_ld_wait(dp);
        tmem_ld_wait(dp + 32);
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          const float4 d4 = ld4(dd + e);
          pf[e] *= __uint_as_float(dp[e]) - d4.x;
          pf[e + 1] *= __uint_as_float(dp[e + 1]) - d4.y;
          pf[e + 2] *= __uint_as_float(dp[e + 2]) - d4.z;
          pf[e + 3] *= __uint_as_float(dp[e + 3]) - d4.w;
          if constexpr (SOFTCAP) {  // dX = dS (1 - tanh^2)
            const float2 g01 = unpack2<false>(gh[e / 2]), g23 = unpack2<false>(gh[e / 2 + 1]);
            pf[e] *= g01.x;
            pf[e + 1] *= g01.y;
            pf[e + 2] *= g23.x;
            pf[e + 3] *= g23.y;
          }
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t ps[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) ps[e] = pack2<BF16>(pf[c * 32 + 2 * e], pf[c * 32 + 2 * e + 1]);
        tmem_st16(tbase + 128 + cg * 64 + c * 16 + lane_off, ps);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
    }
    // ---- epilogue: dV, scale * dK -> 16-bit
    if (ok && n_iter > 0) ok = wait_bounded(done, 0, w);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const bool row_ok = k < sq.Sk;
      const int64_t ro = ((static_cast<int64_t>(sq.bc) * p.Sk + sq.ks + k) * p.Hkv + hk) * D;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
        uint16_t* dst = static_cast<uint16_t*>(which ? p.dk : p.dv) + ro;
        const float mul = which ? p.scale : 1.f;
#pragma unroll 1
        for (int c2 = cg * (D / 64); c2 < (cg + 1) * (D / 64); ++c2) {  // this half's columns
          uint32_t o[32];
          if (n_iter > 0) {
            tmem_ld32(tbase + 256 + which * D + c2 * 32 + lane_off, o);
            tmem_ld_wait(o);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack2<BF16>(__uint_as_float(o[2 * e]) * mul, __uint_as_float(o[2 * e + 1]) * mul);
          if (row_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c2 * 32);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              d4[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, Cfg::kTmemCols);
  }
}

// One CTA per (128-query block, head h, batch b).  Tensor memory: two S buffers
// [0, 128) and [128, 256) used by alternate key blocks, dP [256, 384), dQ from 384.
// In issue order the products run S(0), dP(0); per block j, once every compute warp
// holds S(j) and dP(j) in registers: S(j+1) [into the other buffer], dP(j+1); then,
// once dS(j) is written, dQ(j).  The math of block j overlaps the products of block
// j+1, and no completion barrier runs two phases ahead of its waiters.
template <int D, bool BF16, bool ALIBI, bool SOFTCAP, bool VARLEN>
__device__ __forceinline__ void bwd_dq_cta(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                           const CUtensorMap& tmV, const CUtensorMap& tmDO,
                                           const BwdParams& p, long long lin) {
  using Cfg = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // grid: query blocks x heads x sequences in groups of (sequence, head) pairs
  // (grid_pos): the CTAs that stream one head's key/value tiles run together and
  // find them in L2; the last query block (the most keys under a causal mask) first
  const int nqb = (p.rows_q + 127) / 128;
  const GridPos gp = grid_pos(lin, nqb, p.H, p.B);
  const int q0 = (nqb - 1 - gp.blk) * 128;
  const int h = gp.head;
  const int b = gp.seq;
  const int hk = h / p.G;
  const BwdSeq sq = bwd_seq<VARLEN>(p, b);
  if (q0 >= sq.Sq) return;  // uniform: past this sequence's rows (varlen), nothing set up yet
  const MaskGeo mg = mask_geo(p, sq.Sq, sq.Sk);
  // keys seen by some query of [q0, q_last]
  const int q_last = min(q0 + 127, sq.Sq - 1);
  const int k_begin = mg.has_left ? max(0, q0 + mg.off - mg.wl) : 0;
  const int k_end = mg.has_right ? min(q_last + mg.off + mg.right, sq.Sk - 1) + 1 : sq.Sk;
  const int j_lo = k_begin / 128;
  const int n_blk = (k_end > k_begin) ? (k_end + 127) / 128 - j_lo : 0;

  constexpr int KS = Cfg::kKStages, VS = Cfg::kVStages;
  uint8_t* fixA = smem + Cfg::kFixA;  // Q_i
  uint8_t* fixB = smem + Cfg::kFixB;  // dO_i
  uint8_t* ring_k = smem + Cfg::kK;   // K_j in stage j % KS
  uint8_t* ring_v = smem + Cfg::kV;   // V_j in stage j % VS
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* fix_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 1 + KS;
  uint64_t* v_full = bars + 1 + 2 * KS;
  uint64_t* v_empty = bars + 1 + 2 * KS + VS;
  uint64_t* s_full = bars + 1 + 2 * KS + 2 * VS;
  // alternating pairs, by block parity: an arrival for block j+2 needs the other
  // side to have finished block j, so neither runs two phases ahead of its waiter
  uint64_t* p_full[2] = {s_full + 1, s_full + 2};   // dS of the block written
  uint64_t* dp_read = s_full + 3;  // every compute warp holds its dP columns in registers
  uint64_t* done = s_full + 4;
  uint64_t* drain = s_full + 5;
  uint64_t* dp_full = s_full + 6;
  static_assert(1 + 2 * KS + 2 * VS + 7 == Cfg::kNumBars, "barrier count");
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);

  if (warp == 8 && lane == 0) {
    mbar_init(fix_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    mbar_init(s_full, 1);
    for (int x = 0; x < 2; ++x) mbar_init(p_full[x], 8);  // dS written: one arrival per compute warp
    mbar_init(dp_full, 1);
    mbar_init(dp_read, 8);
    mbar_init(done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_holder, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const WaitCtx w{abort_flag, p.status, p.timeout_ns};

  // register re-split inside the role branches (a merge of the two limits before
  // them would hold all later code to the smaller one)
  if (warp >= 8) {
   regs_dec<kBwdOtherRegs>();
   if (warp == 8) {
    // ======================================================== TMA producer
    if (lane == 0 && n_blk > 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      tma_prefetch_map(&tmDO);
      mbar_arrive_expect_tx(fix_full, 2 * Cfg::kTileBytes);
      for (int c = 0; c < Cfg::kChunks; ++c) {
        tma_load_4d(fixA + c * Cfg::kChunkBytes, &tmQ, fix_full, c * 64, sq.qs + q0, h, sq.bc);
        tma_load_4d(fixB + c * Cfg::kChunkBytes, &tmDO, fix_full, c * 64, sq.qs + q0, h, sq.bc);
      }
      int last_k[KS], last_v[VS];
      for (int s = 0; s < KS; ++s) last_k[s] = -1;
      for (int s = 0; s < VS; ++s) last_v[s] = -1;
      for (int it = 0; it < n_blk; ++it) {
        const int sk = it % KS, sv = it % VS;
        const uint32_t phk = (it / KS) & 1, phv = (it / VS) & 1;
        const int kb = (j_lo + it) * 128;
        if (!wait_bounded(k_empty + sk, phk ^ 1, w)) break;
        mbar_arrive_expect_tx(k_full + sk, Cfg::kTileBytes);
        for (int c = 0; c < Cfg::kChunks; ++c)
          tma_load_4d(ring_k + sk * Cfg::kTileBytes + c * Cfg::kChunkBytes, &tmK, k_full + sk,
                      c * 64, sq.ks + kb, hk, sq.bc);
        last_k[sk] = phk;
        if (!wait_bounded(v_empty + sv, phv ^ 1, w)) break;
        mbar_arrive_expect_tx(v_full + sv, Cfg::kTileBytes);
        for (int c = 0; c < Cfg::kChunks; ++c)
          tma_load_4d(ring_v + sv * Cfg::kTileBytes + c * Cfg::kChunkBytes, &tmV, v_full + sv,
                      c * 64, sq.ks + kb, hk, sq.bc);
        last_v[sv] = phv;
      }
      if (*abort_flag) {
        wait_drain_bwd(fix_full, 0, p.timeout_ns);
        for (int s = 0; s < KS; ++s)
          if (last_k[s] >= 0) wait_drain_bwd(k_full + s, last_k[s], p.timeout_ns);
        for (int s = 0; s < VS; ++s)
          if (last_v[s] >= 0) wait_drain_bwd(v_full + s, last_v[s], p.timeout_ns);
      }
    }
    __syncwarp();
   } else if (warp == 9) {
    // ======================================================== MMA issuer
    if (lane == 0 && n_blk > 0) {
      constexpr uint32_t idesc_s = f16_idesc(BF16, 128, 128, false, false);
      constexpr uint32_t idesc_acc = f16_idesc(BF16, 128, D, false, true);
      const uint64_t dQk = sw128_desc(smem_u32(fixA), 16, 1024);
      const uint64_t dOk = sw128_desc(smem_u32(fixB), 16, 1024);
      auto st_k = [&](int it) { return smem_u32(ring_k + (it % KS) * Cfg::kTileBytes); };
      auto st_v = [&](int it) { return smem_u32(ring_v + (it % VS) * Cfg::kTileBytes); };
      bool ok = wait_bounded(fix_full, 0, w) && wait_bounded(k_full, 0, w) &&
                wait_bounded(v_full, 0, w);
      if (ok) {
        tc_fence_after();
        fwd_issue_qk<D>(tbase, dQk, sw128_desc(st_k(0), 16, 1024), idesc_s);   // S(0)
        tc_commit(s_full);
        fwd_issue_qk<D>(tbase + 256, dOk, sw128_desc(st_v(0), 16, 1024), idesc_s);  // dP(0)
        tc_commit(dp_full);
        tc_commit(v_empty);  // V_0 is read by dP(0) alone
      }
      for (int it = 0; it < n_blk && ok; ++it) {
        const int s = it & 1;
        const bool more = it + 1 < n_blk;
        // every compute warp has passed its waits on S(j) and dP(j) and holds dP(j):
        // S(j+1) and dP(j+1) may complete now without running two phases ahead of
        // those waits, and dP(j+1) may overwrite the dP columns
        if (!(ok = wait_bounded(dp_read, it & 1, w))) break;
        if (more) {
          const int n1 = it + 1;
          if (!(ok = wait_bounded(k_full + n1 % KS, (n1 / KS) & 1, w))) break;
          tc_fence_after();
          // S(j+1) into the other buffer (its dS(j-1) was read by dQ(j-1), issued before)
          fwd_issue_qk<D>(tbase + (s ^ 1) * 128, dQk, sw128_desc(st_k(n1), 16, 1024), idesc_s);
          tc_commit(s_full);
          if (!(ok = wait_bounded(v_full + n1 % VS, (n1 / VS) & 1, w))) break;
          tc_fence_after();
          fwd_issue_qk<D>(tbase + 256, dOk, sw128_desc(st_v(n1), 16, 1024), idesc_s);  // dP(j+1)
          tc_commit(dp_full);
          tc_commit(v_empty + n1 % VS);
        }
        if (!(ok = wait_bounded(p_full[s], (it >> 1) & 1, w))) break;
        tc_fence_after();
        // dQ += dS K_j: B = K_j MN-major (rows are keys, the head dim contiguous)
        bwd_issue_split_a(tbase + 384, tbase + s * 128,
                          sw128_desc(st_k(it), Cfg::kChunkBytes, 1024), idesc_acc, it > 0);
        tc_commit(k_empty + it % KS);
      }
      if (ok) tc_commit(done);
      tc_commit(drain);
      wait_drain_bwd(drain, 0, p.timeout_ns);
    }
    __syncwarp();
   }
  } else {
    regs_inc<kBwdComputeRegs>();
    // ======================================================== compute
    const int cg = warp / 4;  // key-column half of every block
    const int r = (warp % 4) * 32 + lane;  // query row within the block = TMEM lane
    const int q = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const int64_t idx = (static_cast<int64_t>(sq.bc) * p.H + h) * p.sq_pad + sq.qs + q;
    const float lse2 = (q < sq.Sq) ? p.lse2[idx] : INFINITY;
    const float dd = (q < sq.Sq) ? p.dvec[idx] : 0.f;
    const float slope2 = ALIBI ? p.alibi[h] * kBwdLog2e : 0.f;
    bool ok = true;
    for (int it = 0; it < n_blk; ++it) {
      const int kb = (j_lo + it) * 128;
      ok = wait_bounded(s_full, it & 1, w) && wait_bounded(dp_full, it & 1, w);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tbase + (it & 1) * 128;  // this block's S buffer
      const bool open = mg.tile_open(q0, kb);  // uniform: the whole tile is unmasked
      // this half's 64 key columns of S and dP; dS (16-bit) goes to S columns
      // [64 cg, 64 cg + 32), over this warpgroup's own scores
      uint32_t sv[64], dp[64];
      tmem_ld32(tS + cg * 64 + lane_off, sv);
      tmem_ld32(tS + cg * 64 + 32 + lane_off, sv + 32);
      tmem_ld32(tbase + 256 + cg * 64 + lane_off, dp);
      tmem_ld32(tbase + 256 + cg * 64 + 32 + lane_off, dp + 32);
      tmem_ld_wait(sv);
      tmem_ld_wait(sv + 32);
      tmem_ld_wait(dp);
      tmem_ld_wait(dp + 32);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dp_read);  // dP(j+1) may overwrite the dP columns
      // every exponential is taken, a masked one then dropped by a select (no
      // branch per element: the loop stays one block the scheduler can overlap)
      uint32_t ps[32];
      auto grads = [&](auto masked_t) {
        constexpr bool kMasked = decltype(masked_t)::value;
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          float ds[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int k = kb + cg * 64 + e + u;
            float x, gt = 1.f;
            if constexpr (SOFTCAP)
              x = softcap_score(__uint_as_float(sv[e + u]), p, &gt);
            else
              x = __uint_as_float(sv[e + u]) * p.scale_log2;
            if constexpr (ALIBI) x = fmaf(-slope2, fabsf(static_cast<float>(q + mg.off - k)), x);
            float g = ex2(x - lse2) * (__uint_as_float(dp[e + u]) - dd);
            if constexpr (SOFTCAP) g *= gt;  // dX = dS (1 - tanh^2)
            ds[u] = (!kMasked || mg.allowed(q, k)) ? g : 0.f;
          }
          ps[e / 2] = pack2<BF16>(ds[0], ds[1]);
        }
      };
      if (open)
        grads(std::false_type{});
      else
        grads(std::true_type{});
      tmem_st16(tS + cg * 64 + lane_off, ps);
      tmem_st16(tS + cg * 64 + 16 + lane_off, ps + 16);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full[it & 1]);
    }
    // ---- epilogue: scale * dQ -> 16-bit
    if (ok && n_blk > 0) ok = wait_bounded(done, 0, w);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      uint16_t* dst = static_cast<uint16_t*>(p.dq) +
                      ((static_cast<int64_t>(sq.bc) * p.Sq + sq.qs + q) * p.H + h) * D;
#pragma unroll 1
      for (int c2 = cg * (D / 64); c2 < (cg + 1) * (D / 64); ++c2) {  // this half's columns
        uint32_t o[32];
        if (n_blk > 0) {
          tmem_ld32(tbase + 384 + c2 * 32 + lane_off, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack2<BF16>(__uint_as_float(o[2 * e]) * p.scale,
                              __uint_as_float(o[2 * e + 1]) * p.scale);
        if (q < sq.Sq) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c2 * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            d4[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, Cfg::kTmemCols);
  }
}

// Both tile passes in one grid: CTAs [0, n_kv) are dK/dV CTAs, the rest dQ CTAs.
// The two passes are independent (each reads only the inputs and D), so dQ CTAs
// start on the SMs that the last dK/dV CTAs leave idle, without a second launch.
template <int D, bool BF16, bool ALIBI, bool SOFTCAP, bool VARLEN>
__global__ void __launch_bounds__(kWideThreads, 1)
    bwd_tiles_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmD,
                     const BwdParams p) {
  const long long n_kv =
      static_cast<long long>((p.rows_k + 127) / 128) * p.Hkv * static_cast<long long>(p.B);
  const long long lin = blockIdx.x;
  if (lin < n_kv)
    bwd_dkdv_cta<D, BF16, ALIBI, SOFTCAP, VARLEN>(tmQ, tmK, tmV, tmDO, tmL, tmD, p, lin);
  else
    bwd_dq_cta<D, BF16, ALIBI, SOFTCAP, VARLEN>(tmQ, tmK, tmV, tmDO, p, lin - n_kv);
}

template <int D, bool BF16, bool ALIBI, bool SOFTCAP, bool VARLEN>
cudaError_t launch_bwd_inst(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tl, const CUtensorMap& td,
                            const BwdParams& p, cudaStream_t stream) {
  constexpr int kSmem = BwdCfg<D>::kSmemAlloc > DqCfg<D>::kSmemAlloc ? BwdCfg<D>::kSmemAlloc
                                                                      : DqCfg<D>::kSmemAlloc;
  const long long n_kv =
      static_cast<long long>((p.rows_k + 127) / 128) * p.Hkv * static_cast<long long>(p.B);
  const long long n_q =
      static_cast<long long>((p.rows_q + 127) / 128) * p.H * static_cast<long long>(p.B);
  if (n_kv + n_q > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int64_t rows = static_cast<int64_t>(p.cu_q != nullptr ? 1 : p.B) * p.Sq * p.H;
  constexpr int kRowsPerBlock = 8 * (32 / (D / 8));
  bwd_dot_kernel<D, BF16><<<static_cast<unsigned>((rows + kRowsPerBlock - 1) / kRowsPerBlock), 256,
                            0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  auto kt = bwd_tiles_kernel<D, BF16, ALIBI, SOFTCAP, VARLEN>;
  if ((e = cudaFuncSetAttribute(kt, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem)) !=
      cudaSuccess)
    return e;
  kt<<<static_cast<unsigned>(n_kv + n_q), kWideThreads, kSmem, stream>>>(tq, tk, tv, tdo, tl, td,
                                                                        p);
  return cudaGetLastError();
}

// Dispatch over head dim, dtype, ALiBi and softcap for one varlen setting.
template <bool VARLEN>
cudaError_t launch_bwd_all(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& tdo, const CUtensorMap& tl, const CUtensorMap& td,
                           const BwdParams& p, bool bf16, int d, cudaStream_t stream) {
  const bool al = p.alibi != nullptr;
  const bool sc = p.softcap_log2 > 0.f;
#define FA_BWD_CASE(DD, BF, AL, SC) \
  if (d == DD && bf16 == BF && al == AL && sc == SC)                                       \
    return launch_bwd_inst<DD, BF, AL, SC, VARLEN>(tq, tk, tv, tdo, tl, td, p, stream);
#define FA_BWD_CASES(SC)          \
  FA_BWD_CASE(64, false, false, SC)  \
  FA_BWD_CASE(64, false, true, SC)   \
  FA_BWD_CASE(64, true, false, SC)   \
  FA_BWD_CASE(64, true, true, SC)    \
  FA_BWD_CASE(128, false, false, SC) \
  FA_BWD_CASE(128, false, true, SC)  \
  FA_BWD_CASE(128, true, false, SC)  \
  FA_BWD_CASE(128, true, true, SC)
  FA_BWD_CASES(false)
  FA_BWD_CASES(true)
#undef FA_BWD_CASES
#undef FA_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace fa
