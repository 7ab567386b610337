// fwd_kernel.cuh -- exact attention forward for sm_100a (dense and varlen).
//
// What it computes: O = softmax(mask(softcap(scale Q K^T) + ALiBi)) V and the
// per-row natural-log LSE, by streaming K/V blocks through shared memory with
// online-softmax rescaling (tag page "flash attention": tiling plus online
// softmax, the score matrix never written to HBM).  Argument semantics follow
// "FlashAttention common interfaces" sections 3.1/3.2; the causal mask is
// aligned bottom-right (changelog post, v2.1).
//
// CTA = T 128-row query tiles of one (sequence, head), T = 2 (or T = 1 at D = 64,
// two CTAs per SM); 128 (T + 1) threads:
//   warps 0 .. 4T-1  softmax warpgroup per tile (thread r owns query row r = TMEM
//                    lane r of its tile)
//   warp  4T         TMA producer: Q once, then K_j / V_j blocks into a ring of stages
//   warp  4T+1 ..    tcgen05.mma issuer(s), one elected thread each; the first also
//                    allocates tensor memory.  The rest of that warpgroup idles: it
//                    completes the warpgroup for the register re-split (softmax
//                    threads hold a 128-float score row and take 200 registers).
// Tensor memory (fp32 columns x 128 lanes):
//   D = 128 (T = 2, 512 columns): S_t = Q_t K_j^T at [128 t, 128 t + 128), P_t
//     (16-bit, two per column) aliasing the first 64 columns of S_t, O_t += P_t V_j
//     at [256 + 128 t, ...).  One issuer runs PV_0(j), QK_0(j+1), PV_1(j),
//     QK_1(j+1); each commit to S_t's barrier also covers the PV_t(j) issued before
//     it, so when a softmax warpgroup sees S_t(j+1) it knows P_t(j) has been
//     consumed and O_t is up to date; it may then rescale O_t before releasing
//     P_t(j+1).
//   D = 64 (256 T columns): S_t at [128 t, ...), P_t at [128 T + 64 t, ...), O_t at
//     [192 T + 64 t, ...).  Each tile has its own issuer, and QK_t(j+1) is issued as
//     soon as S_t(j) sits in registers.
// The running max is kept lazily: O is rescaled only when a row's max grows by
// more than 8 (base-2 units); the final O / l and LSE use the same stale max, so
// the result is unchanged.  Blocks that lie fully inside every row's allowed key
// range skip the mask; blocks outside the unit's key range are never loaded.
//
// Work schedule.  A "unit" is the T query tiles (T * 128 rows) of one (sequence,
// head).  Dense calls run persistently: the grid holds as many CTAs as fit on the
// device at once and CTA c takes work items c, c + gridDim.x, ...; items are
// ordered (batch, head)-major so that the CTAs running at any moment share a few
// heads' K/V in L2.  Under a causal or window mask an item pairs unit n-1-u with
// unit u of the same head (the heaviest with the lightest), so every item carries
// the same number of key blocks and a static assignment stays balanced.  The
// roles of a CTA walk the same unit sequence; ring slots and barrier phases run on
// across units, and the next unit's Q is loaded as soon as the last product that
// reads the current Q has completed, so one unit's epilogue overlaps the next
// unit's first products.  Varlen and KV-cache calls take one unit per CTA, the
// heaviest units first.
#pragma once

#include <climits>
#include <type_traits>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 128;          // keys per K/V block
constexpr uint32_t kSoftmaxRegs = 200;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;
// 8-bit P is taken against the running max minus 8, and the running max is lazy
// with a threshold of 0.8 (log2 units): P then stays at or below 2^8.8 < 448, the
// largest E4M3 value, and a probability is subnormal in E4M3 only below 2^-14 of
// the row's largest (2^-14.8 when the running max is 0.8 stale), so the error bound
// of an exact running max holds.  (With an exact max, O was rescaled in most
// blocks: for random scores some row of a warp raises its max at almost every
// block.)
constexpr float kP8Offset = 8.0f;
constexpr float kP8Threshold = 0.8f;

// T query tiles per CTA (1 or 2).  With T = 2 one CTA fills an SM (512 TMEM
// columns, 12 warps); with T = 1 two CTAs share an SM (256 columns and 8 warps
// each) and, being independent, drift out of phase, so that one CTA's
// exponentials overlap the other's loads and reductions.
// E = bytes per input element: 2 (fp16 / bf16) or 1 (E4M3, D = 128 only).
template <int D, int T, int E = 2>
struct FwdCfg {
  static_assert(T == 1 || T == 2, "one or two query tiles per CTA");
  static_assert(T == 2 || (D == 64 && E == 2), "one tile per CTA is laid out for 16-bit D = 64 only");
  static_assert(E == 2 || D == 128, "8-bit inputs are laid out for D = 128 only");
  static constexpr int kThreads = (4 * T + 4) * 32;   // softmax warpgroups + one more
  static constexpr int kMinBlocks = 3 - T;             // CTAs per SM
  // registers a thread launches with, and what the non-softmax warpgroup keeps:
  // T*128*kSoftmaxRegs + 128*kOtherRegs = kThreads * kLaunchRegs
  static constexpr int kLaunchRegs = (T == 2) ? 168 : 128;
  static constexpr uint32_t kOtherRegs = (T == 2) ? 104 : 56;
  static_assert(T * 128 * kSoftmaxRegs + 128 * kOtherRegs == kThreads * kLaunchRegs,
                "register re-split must add up to the launch registers");
  static constexpr int kChunks = D * E / 128;         // 128-byte swizzle atoms per row
  static constexpr int kChunkElems = 128 / E;         // elements per atom row
  static constexpr int kStages = (D * E == 256) ? 2 : (T == 2 ? 4 : 2);  // K and V ring depth
  static constexpr int kTileBytes = 128 * D * E;      // Q tile, K block or V block
  static constexpr int kChunkBytes = 128 * 128;       // 128 rows x 128 bytes
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + T * kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kStages * kTileBytes;
  // q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_full[2],
  // o_final[2], drain[2], s_free[2], pv_done[2], q_empty, desync
  static constexpr int kNumBars = 1 + 4 * kStages + 14;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;  // room to align the base to 1 KiB
  static constexpr int kTmemCols = 256 * T;
  // D = 64: P has its own columns (S Tx128, P Tx64, O Tx64), so the next S can be
  // computed while the softmax still works on the current one.
  // D = 128: S 2x128 + O 2x128 fill the 512 columns and P aliases S.
  static constexpr bool kSepP = (D == 64);
  static constexpr int kPCol = kSepP ? 128 * T : 0;
  static constexpr int kPStride = kSepP ? 64 : 128;
  static constexpr int kOCol = kSepP ? 192 * T : 256;
  // warp roles: 4T softmax warps, then the producer, then the MMA issuer(s)
  static constexpr int kProducerWarp = 4 * T;
  static constexpr int kIssuerWarp = 4 * T + 1;  // also allocates tensor memory
};

// Wait that ignores the abort flag (used to drain this CTA's own in-flight work).
__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// One unit of work: query rows [row0, row0 + T*128) of sequence b, head h, and the
// key blocks [j_lo, j_lo + n_blk) they may attend.
struct FwdUnit {
  int state;               // 0: no more units; 1: nothing at this position; 2: a unit
  int b, h;
  int q0, k0, Sq_b, Sk_b;  // varlen row offsets and this sequence's lengths
  int row0, off;           // first query row; key offset of the bottom-right alignment
  int j_lo, n_blk;
};

// The k-th unit of this CTA (state 0 = no more units, 1 = none at this position,
// 2 = a unit).  Persistent schedule (dense): item = blockIdx.x + m * gridDim.x,
// items ordered (batch, head, pair index); with pairing, k = 2m takes unit
// n-1-pi and k = 2m+1 unit pi of pair pi.  Otherwise one unit per CTA from
// blockIdx, heaviest first.
template <int T, bool KV>
__device__ __forceinline__ FwdUnit fwd_unit_at(const FwdParams& p, int k) {
  FwdUnit u{};
  int b, h, unit;
  int q0 = 0, k0 = 0, Sq_b = p.Sq, Sk_b = p.Sk;
  if (p.persistent) {
    const int n_units = (p.Sq + T * kBM - 1) / (T * kBM);
    const int n_pi = p.pair ? (n_units + 1) / 2 : n_units;
    const int per = p.pair ? 2 : 1;
    const int item = blockIdx.x + (k / per) * gridDim.x;
    if (item >= p.B * p.H * n_pi) return u;  // state 0
    const int pi = item % n_pi;
    const int bh = item / n_pi;
    b = bh / p.H;
    h = bh % p.H;
    if (p.pair) {
      unit = (k % 2 == 0) ? n_units - 1 - pi : pi;
      if (k % 2 == 1 && unit == n_units - 1 - pi) {  // middle unit of an odd count
        u.state = 1;
        return u;
      }
    } else {
      unit = pi;
    }
  } else {
    if (k > 0) return u;
    h = p.tile_major ? blockIdx.y : blockIdx.x;
    b = p.tile_major ? blockIdx.z : blockIdx.y;
    const int zi = static_cast<int>(p.tile_major ? blockIdx.x : blockIdx.z);
    if (p.cu_q != nullptr) {
      q0 = p.cu_q[b];
      Sq_b = p.cu_q[b + 1] - q0;
      k0 = p.cu_k[b];
      Sk_b = p.cu_k[b + 1] - k0;
    } else if (KV) {
      Sk_b = ((p.cache_seqlens != nullptr) ? p.cache_seqlens[b] : p.Sk) + p.k_add;
      // a length the cache cannot hold would read past the block table: clamp, report
      const int cap = (p.block_table != nullptr) ? p.max_blocks * p.page_size : p.Sk;
      if (Sk_b < 0 || Sk_b > cap) {
        if (threadIdx.x == 0) atomicOr(p.status, kDevBadLength);
        Sk_b = min(max(Sk_b, 0), cap);
      }
    }
    const int n_units_b = (Sq_b + T * kBM - 1) / (T * kBM);
    if (zi >= n_units_b) return u;
    unit = n_units_b - 1 - zi;  // heaviest rows first
  }
  u.b = b;
  u.h = h;
  u.q0 = q0;
  u.k0 = k0;
  u.Sq_b = Sq_b;
  u.Sk_b = Sk_b;
  u.row0 = unit * T * kBM;
  u.off = Sk_b - Sq_b;
  // the unit's key range: [lo(first row), hi(last row)] intersected with [0, Sk_b)
  const int right = p.causal ? 0 : p.wr;
  const int r_last = min(u.row0 + T * kBM - 1, Sq_b - 1);
  const int k_begin = (p.wl >= 0) ? max(0, u.row0 + u.off - p.wl) : 0;
  const int k_end = ((p.causal || p.wr >= 0) ? min(r_last + u.off + right, Sk_b - 1) : Sk_b - 1) + 1;
  u.j_lo = k_begin / kBN;
  u.n_blk = (k_end > k_begin) ? (k_end + kBN - 1) / kBN - u.j_lo : 0;
  u.state = 2;
  return u;
}

// EMU: of every 8 pairs of probabilities, EMU are evaluated by exp2_fma2 on the
// FMA pipe and the rest by the MUFU unit (balances the two at small head dims).
// S_t = Q_t K^T into tensor memory: K-major A (Q tile) and B (K block); a step of
// 16 along the head dim is 32 bytes inside a 128-byte swizzle atom, the next atom
// lies 16 KiB further.
// With 8-bit inputs (E = 1) a step is 32 elements, still 32 bytes, through
// tcgen05.mma kind::f8f6f4.
// Descriptors are passed as their low words (start address, leading offset) plus
// the high word they share (stride offset, version, swizzle mode); a step adds
// its byte offset / 16 to the start address field, which cannot carry.
template <int D, int E = 2>
__device__ __forceinline__ void fwd_issue_qk(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                             uint32_t hi, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < D * E / 32; ++kk) {
    const uint32_t o = ((kk / 4) * (128 * 128) + (kk % 4) * 32) >> 4;
    if constexpr (E == 2)
      mma_ss(d_tmem, desc_pack(a_lo + o, hi), desc_pack(b_lo + o, hi), idesc, kk > 0 ? 1u : 0u);
    else
      mma_ss_f8(d_tmem, desc_pack(a_lo + o, hi), desc_pack(b_lo + o, hi), idesc, kk > 0 ? 1u : 0u);
  }
}

// The same product from two full descriptors (their high words must agree: every
// 128-byte-swizzled operand here has a 1 KiB stride offset).
template <int D, int E = 2>
__device__ __forceinline__ void fwd_issue_qk(uint32_t d_tmem, uint64_t a0, uint64_t b0,
                                             uint32_t idesc) {
  fwd_issue_qk<D, E>(d_tmem, static_cast<uint32_t>(a0), static_cast<uint32_t>(b0),
                     static_cast<uint32_t>(a0 >> 32), idesc);
}

// O_t (+)= P_t V: A = P from tensor memory (8 columns hold 16 keys), B = V block,
// MN-major (16 keys = 16 rows = 2 KiB; head-dim atoms 16 KiB apart).
// With 8-bit P and V a step is 32 keys: 8 columns of four E4M3 values, 4 KiB of V.
template <int D, int E = 2>
__device__ __forceinline__ void fwd_issue_pv(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                             uint32_t b_hi, uint32_t idesc, bool acc) {
#pragma unroll
  for (int kk = 0; kk < kBN * E / 32; ++kk) {
    if constexpr (E == 2)
      mma_ts(d_tmem, a_tmem + kk * 8, desc_pack(b_lo + kk * (2048 >> 4), b_hi), idesc,
             (acc || kk > 0) ? 1u : 0u);
    else
      mma_ts_f8(d_tmem, a_tmem + kk * 8, desc_pack(b_lo + kk * (4096 >> 4), b_hi), idesc,
                (acc || kk > 0) ? 1u : 0u);
  }
}

template <int D, int E = 2>
__device__ __forceinline__ void fwd_issue_pv(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0,
                                             uint32_t idesc, bool acc) {
  fwd_issue_pv<D, E>(d_tmem, a_tmem, static_cast<uint32_t>(b0), static_cast<uint32_t>(b0 >> 32),
                     idesc, acc);
}

// FP8: E4M3 Q, K, V (both products on kind::f8f6f4, P rounded to E4M3), bf16 output
// (BF16 must then be true).  KV: K/V from a KV cache (FwdParams::kv_mode); a
// compile-time switch, so the dense kernels carry none of its code.
template <int D, int T, bool BF16, bool SOFTCAP, bool ALIBI, int EMU, bool FP8 = false,
          bool KV = false>
__global__ void __launch_bounds__(FwdCfg<D, T, FP8 ? 1 : 2>::kThreads,
                                  FwdCfg<D, T, FP8 ? 1 : 2>::kMinBlocks)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  static_assert(!FP8 || BF16, "8-bit inputs write a bf16 output");
  constexpr int E = FP8 ? 1 : 2;
  using Cfg = FwdCfg<D, T, E>;
  constexpr int ST = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---------------------------------------------------------- shared memory
  uint8_t* sQ = smem + Cfg::kQOff;
  uint8_t* sK = smem + Cfg::kKOff;
  uint8_t* sV = smem + Cfg::kVOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 1 + ST;
  uint64_t* v_full = bars + 1 + 2 * ST;
  uint64_t* v_empty = bars + 1 + 3 * ST;
  uint64_t* s_full = bars + 1 + 4 * ST;
  uint64_t* p_full = bars + 3 + 4 * ST;
  uint64_t* o_final = bars + 5 + 4 * ST;
  uint64_t* drain = bars + 7 + 4 * ST;    // [2]: one per issuer
  uint64_t* s_free = bars + 9 + 4 * ST;   // softmax has S_t in registers (separate-P layout)
  uint64_t* pv_done = bars + 11 + 4 * ST; // PV_t finished: P_t may be rewritten, O_t rescaled
  uint64_t* q_empty = bars + 13 + 4 * ST; // the last product reading this unit's Q is done
  // D = 64: tile 1 starts its first product only once tile 0 is half way through the
  // exponentials of its first block.  The two tiles then run half a block apart, so
  // that one tile's loads, max pass and P stores overlap the other's exponentials
  // instead of both idling the exponential unit at the same time (+2.5-3% measured).
  uint64_t* desync = bars + 14 + 4 * ST;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);
  constexpr int kIssuers = Cfg::kSepP ? T : 1;

  if (warp == Cfg::kProducerWarp && lane == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, kIssuers);  // one commit per issuer
    mbar_init(desync, 4);
    for (int s = 0; s < ST; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, T);  // released once per tile
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, T);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full + t, 1);
      mbar_init(p_full + t, 4);   // one arrival per softmax warp
      mbar_init(o_final + t, 1);
      mbar_init(s_free + t, 4);
      mbar_init(pv_done + t, 1);
    }
    mbar_init(drain + 0, 1);
    mbar_init(drain + 1, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == Cfg::kIssuerWarp) {
    tmem_alloc(tmem_holder, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const WaitCtx w{abort_flag, p.status, p.timeout_ns};
  const bool varlen = p.cu_q != nullptr;
  if (warp >= Cfg::kProducerWarp) {
   regs_dec<Cfg::kOtherRegs>();
   if (warp == Cfg::kProducerWarp) {
    // ======================================================== TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      int kv_it = 0;  // K/V blocks loaded so far: ring slot kv_it % ST
      int q_cnt = 0;  // units whose Q tiles were loaded
      int last_k[ST], last_v[ST];
      for (int s = 0; s < ST; ++s) last_k[s] = last_v[s] = -1;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const FwdUnit u = fwd_unit_at<T, KV>(p, k);
        if (u.state == 0) break;
        if (u.state == 1 || u.n_blk == 0) continue;
        const int b_coord = varlen ? 0 : u.b;
        const int hk = u.h / p.G;
        // the previous unit's Q stays in place until its last QK product has run
        if (q_cnt > 0 && !(ok = wait_bounded(q_empty, (q_cnt - 1) & 1, w))) break;
        const int qrow = (varlen ? u.q0 : 0) + u.row0;
        const int krow = varlen ? u.k0 : 0;
        mbar_arrive_expect_tx(q_full, T * Cfg::kTileBytes);
        for (int t = 0; t < T; ++t)
          for (int c = 0; c < Cfg::kChunks; ++c)
            tma_load_4d(sQ + t * Cfg::kTileBytes + c * Cfg::kChunkBytes, &tmQ, q_full,
                        c * Cfg::kChunkElems, qrow + t * kBM, u.h, b_coord);
        ++q_cnt;
        for (int it = 0; it < u.n_blk; ++it, ++kv_it) {
          const int s = kv_it % ST;
          const uint32_t ph = (kv_it / ST) & 1;
          const int j = u.j_lo + it;
          if constexpr (!KV) {
            if (!(ok = wait_bounded(k_empty + s, ph ^ 1, w))) break;
            mbar_arrive_expect_tx(k_full + s, Cfg::kTileBytes);
            for (int c = 0; c < Cfg::kChunks; ++c)
              tma_load_4d(sK + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, &tmK, k_full + s,
                          c * Cfg::kChunkElems, krow + j * kBN, hk, b_coord);
            last_k[s] = ph;
            if (!(ok = wait_bounded(v_empty + s, ph ^ 1, w))) break;
            mbar_arrive_expect_tx(v_full + s, Cfg::kTileBytes);
            for (int c = 0; c < Cfg::kChunks; ++c)
              tma_load_4d(sV + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, &tmV, v_full + s,
                          c * Cfg::kChunkElems, krow + j * kBN, hk, b_coord);
            last_v[s] = ph;
          } else {
            // KV cache: the block's two 64-key halves, each inside one page (page_size
            // is a multiple of 64); halves at or past the sequence's end are not
            // loaded (their rows are masked, and V's are zeroed before P.V)
            int row[2], blk[2], nh = 0;
            for (int hh = 0; hh < 2; ++hh) {
              const int pos = j * kBN + hh * 64;
              if (pos >= u.Sk_b) break;
              if (p.block_table != nullptr) {
                int bk = p.block_table[static_cast<int64_t>(u.b) * p.max_blocks + pos / p.page_size];
                if (bk < 0 || bk >= p.num_blocks) {
                  atomicOr(p.status, kDevBadBlock);
                  bk = 0;  // read a valid page; the status word reports the fault
                }
                row[hh] = pos % p.page_size;
                blk[hh] = bk;
              } else {
                row[hh] = pos;
                blk[hh] = u.b;
              }
              ++nh;
            }
            constexpr uint32_t kHalfBytes = Cfg::kChunks * 64 * 128;
            if (!(ok = wait_bounded(k_empty + s, ph ^ 1, w))) break;
            mbar_arrive_expect_tx(k_full + s, nh * kHalfBytes);
            for (int hh = 0; hh < nh; ++hh)
              for (int c = 0; c < Cfg::kChunks; ++c)
                tma_load_4d(sK + s * Cfg::kTileBytes + c * Cfg::kChunkBytes + hh * 64 * 128, &tmK,
                            k_full + s, c * Cfg::kChunkElems, row[hh], hk, blk[hh]);
            last_k[s] = ph;
            if (!(ok = wait_bounded(v_empty + s, ph ^ 1, w))) break;
            mbar_arrive_expect_tx(v_full + s, nh * kHalfBytes);
            for (int hh = 0; hh < nh; ++hh)
              for (int c = 0; c < Cfg::kChunks; ++c)
                tma_load_4d(sV + s * Cfg::kTileBytes + c * Cfg::kChunkBytes + hh * 64 * 128, &tmV,
                            v_full + s, c * Cfg::kChunkElems, row[hh], hk, blk[hh]);
            last_v[s] = ph;
          }
        }
      }
      if (*abort_flag) {  // let this CTA's own copies land before the smem goes away
        if (q_cnt > 0) wait_drain(q_full, (q_cnt - 1) & 1, p.timeout_ns);
        for (int s = 0; s < ST; ++s) {
          if (last_k[s] >= 0) wait_drain(k_full + s, last_k[s], p.timeout_ns);
          if (last_v[s] >= 0) wait_drain(v_full + s, last_v[s], p.timeout_ns);
        }
      }
    }
    __syncwarp();
   } else if (warp == Cfg::kIssuerWarp && !Cfg::kSepP) {
    // ======================================================== MMA issuer (D = 128)
    // One thread alternates the tiles, PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1), so
    // one tile's softmax overlaps the other tile's products.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = f16_idesc(BF16 && !FP8, kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = f16_idesc(BF16 && !FP8, kBM, D, false, true);
      // K-major Q and K (leading offset 16 B) and MN-major V (leading offset one
      // 16 KiB atom column) share the high descriptor word (stride offset 1 KiB)
      const uint64_t dQ0 = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t dV0 = sw128_desc(smem_u32(sV), Cfg::kChunkBytes, 1024);
      const uint32_t hi = static_cast<uint32_t>(dQ0 >> 32);
      const uint32_t q_lo = static_cast<uint32_t>(dQ0);
      const uint32_t k_lo = static_cast<uint32_t>(sw128_desc(smem_u32(sK), 16, 1024));
      const uint32_t v_lo = static_cast<uint32_t>(dV0);
      constexpr uint32_t kTileStep = Cfg::kTileBytes >> 4;
#define FA_QK(T, S)                                                                        \
  fwd_issue_qk<D, E>(tbase + (T) * kBM, q_lo + (T) * kTileStep, k_lo + (S) * kTileStep, hi, \
                     idesc_qk)
#define FA_PV(T, S, ACC)                                                                   \
  fwd_issue_pv<D, E>(tbase + Cfg::kOCol + (T) * D, tbase + Cfg::kPCol + (T) * Cfg::kPStride, \
                     v_lo + (S) * kTileStep, hi, idesc_pv, ACC)
      int kv_it = 0;  // ring position of the unit's first block
      int blk = 0;    // blocks completed per tile so far: s_full / p_full phases
      int q_cnt = 0;  // units started: q_full phase
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const FwdUnit u = fwd_unit_at<T, KV>(p, k);
        if (u.state == 0) break;
        if (u.state == 1 || u.n_blk == 0) continue;
        const int n = u.n_blk;
        ok = wait_bounded(q_full, q_cnt & 1, w) &&
             wait_bounded(k_full + kv_it % ST, (kv_it / ST) & 1, w);
        if (!ok) break;
        tc_fence_after();
        FA_QK(0, kv_it % ST);
        tc_commit(s_full + 0);
        FA_QK(1, kv_it % ST);
        tc_commit(s_full + 1);
        tc_commit(k_empty + kv_it % ST);
        tc_commit(k_empty + kv_it % ST);  // k_empty counts one release per tile
        if (n == 1) tc_commit(q_empty);
        for (int it = 0; it < n; ++it) {
          const int g = kv_it + it;
          const int s = g % ST;
          const uint32_t ph = (g / ST) & 1;
          const bool more = it + 1 < n;
          const int s1 = (g + 1) % ST;
          const uint32_t ph1 = ((g + 1) / ST) & 1;
          const uint32_t pp = (blk + it) & 1;
          if (!(ok = wait_bounded(v_full + s, ph, w))) break;
          if (!(ok = wait_bounded(p_full + 0, pp, w))) break;
          tc_fence_after();
          FA_PV(0, s, it > 0);
          tc_commit(v_empty + s);
          if (more) {
            if (!(ok = wait_bounded(k_full + s1, ph1, w))) break;
            tc_fence_after();
            FA_QK(0, s1);
            tc_commit(s_full + 0);
            tc_commit(k_empty + s1);
          } else {
            tc_commit(o_final + 0);
          }
          if (!(ok = wait_bounded(p_full + 1, pp, w))) break;
          tc_fence_after();
          FA_PV(1, s, it > 0);
          tc_commit(v_empty + s);
          if (more) {
            FA_QK(1, s1);
            tc_commit(s_full + 1);
            tc_commit(k_empty + s1);
            if (it + 2 == n) tc_commit(q_empty);  // that was the unit's last QK
          } else {
            tc_commit(o_final + 1);
          }
        }
#undef FA_QK
#undef FA_PV
        kv_it += n;
        blk += n;
        ++q_cnt;
      }
      tc_commit(drain + 0);
      wait_drain(drain + 0, 0, p.timeout_ns);
    }
    __syncwarp();
   } else if (Cfg::kSepP && warp >= Cfg::kIssuerWarp && warp < Cfg::kIssuerWarp + T) {
    // ======================================================== MMA issuers (D = 64)
    const int t = warp - Cfg::kIssuerWarp;  // this issuer's query tile
    if (lane == 0) {
      constexpr uint32_t idesc_qk = f16_idesc(BF16 && !FP8, kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = f16_idesc(BF16 && !FP8, kBM, D, false, true);
      const uint32_t tS = tbase + t * kBM;
      const uint32_t tP = tbase + Cfg::kPCol + t * Cfg::kPStride;
      const uint32_t tO = tbase + Cfg::kOCol + t * D;
      constexpr uint32_t kTileStep = Cfg::kTileBytes >> 4;
      const uint64_t dQ0 = sw128_desc(smem_u32(sQ), 16, 1024);                  // K-major
      const uint32_t hi = static_cast<uint32_t>(dQ0 >> 32);  // shared by Q, K and V
      const uint32_t q_lo = static_cast<uint32_t>(dQ0) + t * kTileStep;
      const uint32_t k_lo = static_cast<uint32_t>(sw128_desc(smem_u32(sK), 16, 1024));
      const uint32_t v_lo = static_cast<uint32_t>(sw128_desc(smem_u32(sV), Cfg::kChunkBytes, 1024));
#define FA_QK(S) fwd_issue_qk<D, E>(tS, q_lo, k_lo + (S) * kTileStep, hi, idesc_qk)
#define FA_PV(S, ACC) fwd_issue_pv<D, E>(tO, tP, v_lo + (S) * kTileStep, hi, idesc_pv, ACC)
      int kv_it = 0, blk = 0, q_cnt = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const FwdUnit u = fwd_unit_at<T, KV>(p, k);
        if (u.state == 0) break;
        if (u.state == 1 || u.n_blk == 0) continue;
        const int n = u.n_blk;
        ok = wait_bounded(q_full, q_cnt & 1, w) &&
             wait_bounded(k_full + kv_it % ST, (kv_it / ST) & 1, w);
        if (ok && t == 1 && q_cnt == 0) ok = wait_bounded(desync, 0, w);
        if (!ok) break;
        tc_fence_after();
        FA_QK(kv_it % ST);
        tc_commit(s_full + t);
        tc_commit(k_empty + kv_it % ST);
        if (n == 1) tc_commit(q_empty);
        for (int it = 0; it < n; ++it) {
          const int g = kv_it + it;
          const int s = g % ST;
          const uint32_t ph = (g / ST) & 1;
          const bool more = it + 1 < n;
          const int s1 = (g + 1) % ST;
          const uint32_t ph1 = ((g + 1) / ST) & 1;
          const uint32_t pp = (blk + it) & 1;
          // QK_t(j+1) as soon as softmax t holds S_t(j) in registers
          if (more) {
            if (!(ok = wait_bounded(k_full + s1, ph1, w))) break;
            if (!(ok = wait_bounded(s_free + t, pp, w))) break;
            tc_fence_after();
            FA_QK(s1);
            tc_commit(s_full + t);
            tc_commit(k_empty + s1);
            if (it + 2 == n) tc_commit(q_empty);  // that was the unit's last QK
          }
          if (!(ok = wait_bounded(v_full + s, ph, w))) break;
          if (!(ok = wait_bounded(p_full + t, pp, w))) break;
          tc_fence_after();
          FA_PV(s, it > 0);
          tc_commit(pv_done + t);
          tc_commit(v_empty + s);
          if (!more) tc_commit(o_final + t);
        }
#undef FA_QK
#undef FA_PV
        kv_it += n;
        blk += n;
        ++q_cnt;
      }
      // every MMA issued above is complete before tensor memory is released
      tc_commit(drain + t);
      wait_drain(drain + t, 0, p.timeout_ns);
    }
    __syncwarp();
   }
  } else {
    regs_inc<kSoftmaxRegs>();
    // ======================================================== softmax warpgroups
    const int t = warp / 4;
    const int r = threadIdx.x % kBM;
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tS = tbase + t * kBM + lane_off;
    const uint32_t tP = tbase + Cfg::kPCol + t * Cfg::kPStride + lane_off;
    const uint32_t tO = tbase + Cfg::kOCol + t * D + lane_off;
    int blk = 0;    // blocks of this tile so far: s_full / pv_done phases
    int u_cnt = 0;  // units with at least one block: o_final phase
    bool ok = true;
    for (int k = 0; ok; ++k) {
    // what the block loop needs of the unit; the epilogue looks the unit up again
    // (fewer values live across the loop next to the 128-float score row)
    int kb0, n_blk, lo_i, hi_i, lo_rb, hi_ra, Sk_b;
    float slope2, ipo;
    {
      const FwdUnit u = fwd_unit_at<T, KV>(p, k);
      if (u.state == 0) break;
      if (u.state == 1) continue;
      const int off = u.off, Sq_b = u.Sq_b;
      Sk_b = u.Sk_b;
      kb0 = u.j_lo * kBN;
      n_blk = u.n_blk;
      const bool has_left = p.wl >= 0;
      const bool has_right = p.causal || p.wr >= 0;
      const int right = p.causal ? 0 : p.wr;
      // allowed keys of row i: [lo(i), hi(i)] intersected with [0, Sk_b)
      auto lo_of = [&](int i) { return has_left ? i + off - p.wl : INT_MIN / 2; };
      auto hi_of = [&](int i) { return has_right ? min(i + off + right, Sk_b - 1) : Sk_b - 1; };
      const int i = u.row0 + t * kBM + r;  // query row within the sequence
      const int ra = u.row0 + t * kBM;
      const int rb = max(ra, min(ra + kBM - 1, Sq_b - 1));
      lo_i = lo_of(i);
      hi_i = hi_of(i);
      lo_rb = lo_of(rb);
      hi_ra = hi_of(ra);
      slope2 = ALIBI ? p.alibi[u.h] * kLog2e : 0.f;
      ipo = static_cast<float>(i + off);
    }
    float m_use = -INFINITY;  // running max, base-2 units
    float l = 0.f;            // running sum of exp2(x - m_use): gives the LSE
    float lr = 0.f;           // the same sum over P rounded to bf16: normalises O (bf16 only)

    for (int it = 0; it < n_blk; ++it) {
      const int kb = kb0 + it * kBN;
      const uint32_t pp = (blk + it) & 1;
      ok = wait_bounded(s_full + t, pp, w);
      if (!__all_sync(0xffffffffu, ok)) {  // keep the warp's .sync.aligned ops uniform
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tS + c * 32, s + c * 32);
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) tmem_ld_wait(s + c * 32);
      if constexpr (Cfg::kSepP) {  // S_t may now be overwritten by the next QK
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free + t);
      }
      const bool masked = (kb < lo_rb) || (kb + kBN - 1 > hi_ra);
      const int lo_c = lo_i - kb, hi_c = hi_i - kb;  // allowed columns: lo_c <= c <= hi_c
      float factor;  // exponent argument = s * factor - m
      if constexpr (!SOFTCAP && !ALIBI) {
        // raw-score domain: mask here, fold the scale into the exponent below
        // (softmax_scale > 0 here: the host maps 0 to a tiny positive scale)
        if (masked) {
          // test only the bounds that cut into this block for some row of the warp
          // (a causal diagonal block has only the right one)
          const bool cut_lo = __any_sync(0xffffffffu, lo_c > 0);
          const bool cut_hi = __any_sync(0xffffffffu, hi_c < kBN - 1);
          constexpr uint32_t kNegInf = 0xFF800000u;
          if (cut_lo && cut_hi) {
#pragma unroll
            for (int c = 0; c < kBN; ++c) s[c] = (c >= lo_c && c <= hi_c) ? s[c] : kNegInf;
          } else if (cut_hi) {
#pragma unroll
            for (int c = 0; c < kBN; ++c) s[c] = (c <= hi_c) ? s[c] : kNegInf;
          } else if (cut_lo) {
#pragma unroll
            for (int c = 0; c < kBN; ++c) s[c] = (c >= lo_c) ? s[c] : kNegInf;
          }
        }
        factor = p.scale_log2;
      } else {
        const float base = ipo - static_cast<float>(kb);  // ALiBi distance of column c: |base - c|
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          float x = __uint_as_float(s[c]);
          if constexpr (SOFTCAP) {
            // softcap * tanh(scale * x / softcap) in base-2 units, with
            // tanh(y) = 1 - 2 / (exp(2y) + 1)
            const float e = ex2(x * p.tanh_k);
            x = fmaf(-2.f * p.softcap_log2, rcp(e + 1.f), p.softcap_log2);
          } else {
            x *= p.scale_log2;
          }
          if constexpr (ALIBI) x = fmaf(-slope2, fabsf(base - static_cast<float>(c)), x);
          if (masked) x = (c >= lo_c && c <= hi_c) ? x : -INFINITY;
          s[c] = __float_as_uint(x);
        }
        factor = 1.f;
      }
      // ---- row max, online-softmax bookkeeping (lazy rescale), exponentials.
      // With P aliasing S (D = 128) the exponentials are taken speculatively
      // against the running max while the block's row max is reduced in the same
      // loop.  If no row's max grew by more than the rescale threshold, the running
      // max stays as it is and the probabilities are exactly those of the max-first
      // order; otherwise the warp takes the exponentials again against the new max
      // (rows whose max did not move recompute the same values).  The raw scores
      // stay in registers until that check.  Warps with a row that has not met an
      // allowed key yet (running max -inf) take the max-first order.
      const bool spec = !Cfg::kSepP && !FP8 && __all_sync(0xffffffffu, m_use != -INFINITY);
      constexpr float kThreshold = FP8 ? kP8Threshold : kRescaleThreshold;
      bool need = false;
      float alpha = 1.f;
      auto update_max = [&](float m_blk) {
        const float m_new = fmaxf(m_use, m_blk);
        if (m_use == -INFINITY) {
          m_use = m_new;  // nothing accumulated yet: O is zero
        } else if (m_new > m_use + kThreshold) {
          need = true;
          alpha = ex2(m_use - m_new);
          m_use = m_new;
        }
      };
      // four independent chains of three-input max
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
      if (!spec) {
#pragma unroll
        for (int c = 0; c < kBN; c += 8) {
          mx0 = max3f(mx0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
          mx1 = max3f(mx1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
          mx2 = max3f(mx2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
          mx3 = max3f(mx3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
        }
        update_max(fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * factor);
      }
      // probabilities -> 16-bit P.  With separate P columns the whole row is held
      // and the wait for PV_t(j-1) (which still reads P_t) comes only before the
      // stores, so the exponentials overlap it; with P aliasing S each 32-column
      // chunk is stored as soon as it is ready.
      // With separate P columns the first half of the row is computed before the
      // wait for PV_t(j-1) (which still reads P_t) and held in registers; the second
      // half is stored chunk by chunk as it is produced.  With P aliasing S every
      // 32-column chunk is stored as soon as it is ready.
      float2 lsum[kBN / 32], lrnd[kBN / 32];
      uint32_t pk[Cfg::kSepP ? 32 : 16];
      auto exps = [&](auto with_max, auto q_from, auto q_to) {
        constexpr bool kMax = decltype(with_max)::value;
        const float neg_m = (m_use == -INFINITY) ? 0.f : (FP8 ? kP8Offset : 0.f) - m_use;
        const float2 f2 = make_float2(factor, factor), nm2 = make_float2(neg_m, neg_m);
        float2 prev = make_float2(0.f, 0.f);
#pragma unroll
        for (int q4 = decltype(q_from)::value; q4 < decltype(q_to)::value; ++q4) {
          lsum[q4] = make_float2(0.f, 0.f);
          lrnd[q4] = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float s0 = __uint_as_float(s[q4 * 32 + 2 * e]);
            const float s1 = __uint_as_float(s[q4 * 32 + 2 * e + 1]);
            if constexpr (kMax) {
              if (e % 4 == 0) mx0 = max3f(mx0, s0, s1);
              if (e % 4 == 1) mx1 = max3f(mx1, s0, s1);
              if (e % 4 == 2) mx2 = max3f(mx2, s0, s1);
              if (e % 4 == 3) mx3 = max3f(mx3, s0, s1);
            }
            const float2 arg = fma2(make_float2(s0, s1), f2, nm2);
            float2 pp;
            if ((e % 8) < EMU)
              pp = exp2_fma2(arg);
            else
              pp = make_float2(ex2(arg.x), ex2(arg.y));
            lsum[q4] = add2(lsum[q4], pp);
            if constexpr (FP8) {  // four E4M3 values per column, consecutive keys
              if (e % 2 == 0)
                prev = pp;
              else
                pk[e / 2] = pack4_e4m3(prev.x, prev.y, pp.x, pp.y);
            } else {
              const int pi = Cfg::kSepP ? (q4 % 2) * 16 + e : e;
              pk[pi] = pack2<BF16>(pp.x, pp.y);
              // bf16 P is rounded by up to 2^-9: O is normalised by the sum of the
              // rounded values the PV product uses, so that O / lr is an exact convex
              // combination of V rows (fp16's 2^-11 rounding needs no such sum)
              if constexpr (BF16) lrnd[q4] = add2(lrnd[q4], unpack2<true>(pk[pi]));
            }
          }
          if constexpr (FP8)
            tmem_st8(tP + q4 * 8, pk);
          else if constexpr (!Cfg::kSepP)
            tmem_st16(tP + q4 * 16, pk);
          else if (q4 >= 2)
            tmem_st16(tP + q4 * 16, pk + (q4 % 2) * 16);
        }
      };
      using Q0 = std::integral_constant<int, 0>;
      using Q2 = std::integral_constant<int, kBN / 64>;
      using Q4 = std::integral_constant<int, kBN / 32>;
      if constexpr (Cfg::kSepP) {
        exps(std::false_type{}, Q0{}, Q2{});
        if (t == 0 && blk + it == 0 && lane == 0) mbar_arrive(desync);
        // P_t(j-1) must have been consumed (and O_t updated) by PV_t(j-1)
        if (it > 0) {
          ok = wait_bounded(pv_done + t, (blk + it - 1) & 1, w);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        tmem_st16(tP, pk);
        tmem_st16(tP + 16, pk + 16);
        exps(std::false_type{}, Q2{}, Q4{});
      } else if (spec) {
        exps(std::true_type{}, Q0{}, Q4{});
        update_max(fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * factor);
        if (__any_sync(0xffffffffu, need)) exps(std::false_type{}, Q0{}, Q4{});
      } else {
        exps(std::false_type{}, Q0{}, Q4{});
      }
      l *= alpha;
      if constexpr (BF16 && !FP8) lr *= alpha;
      {
        const float2 a = add2(add2(lsum[0], lsum[1]), add2(lsum[2], lsum[3]));
        l += a.x + a.y;
        if constexpr (BF16 && !FP8) {
          const float2 b = add2(add2(lrnd[0], lrnd[1]), add2(lrnd[2], lrnd[3]));
          lr += b.x + b.y;
        }
      }
      // O_t rescale (after the score row is dead: lower register peak); it only
      // has to land before P_t is released to the MMA warp
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tO + c * 16, o);
          tmem_ld_wait16(o);
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st16(tO + c * 16, o);
        }
      }
      // KV cache, last block of the sequence: V rows past its end hold whatever
      // the page tail (or an unloaded half) holds; P is 0 there, but 0 * NaN is
      // NaN in P.V, so this warp zeroes its 32 rows of them before releasing P
      // (both tiles' warps write the same zeros)
      if (KV && kb + kBN > Sk_b) {
        const int s = (blk + it) % ST;
        ok = wait_bounded(v_full + s, ((blk + it) / ST) & 1, w);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        if (kb + r >= Sk_b) {
          uint8_t* vrow = sV + s * Cfg::kTileBytes + r * 128;
#pragma unroll
          for (int c = 0; c < Cfg::kChunks; ++c)
#pragma unroll
            for (int v16 = 0; v16 < 8; ++v16)
              reinterpret_cast<uint4*>(vrow + c * Cfg::kChunkBytes)[v16] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + t);
    }

    // ---- epilogue: O / l -> 16-bit, LSE (natural log)
    if (ok && n_blk > 0) ok = wait_bounded(o_final + t, u_cnt & 1, w);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const FwdUnit u = fwd_unit_at<T, KV>(p, k);
      const int i = u.row0 + t * kBM + r;
      const int Sq_b = u.Sq_b, h = u.h;
      const bool row_ok = i < Sq_b;
      // a row with no allowed key keeps m = -inf (its sum may hold clamped
      // polynomial exponentials of -inf, each <= 2^-126): O = 0, LSE = -inf
      const float norm = (BF16 && !FP8) ? lr : l;
      const bool dead = (m_use == -INFINITY) || !(norm > 0.f);
      // 8-bit inputs: O carries V's descale factor (Q's and K's sit in the scale)
      const float inv = dead ? 0.f : (FP8 ? p.v_descale : 1.f) / norm;
      uint8_t* orow = nullptr;
      if (row_ok) {
        const int64_t ro = varlen ? static_cast<int64_t>(u.q0 + i) * p.o_ss
                                  : static_cast<int64_t>(u.b) * p.o_sb +
                                        static_cast<int64_t>(i) * p.o_ss;
        orow = static_cast<uint8_t*>(p.out) + (ro + static_cast<int64_t>(h) * p.o_sh) * 2;
      }
#pragma unroll 1
      for (int c = 0; c < D / 16; ++c) {
        uint32_t o[16];
        if (n_blk > 0) {
          tmem_ld16(tO + c * 16, o);
          tmem_ld_wait16(o);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = 0u;
        }
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          pk[e] = pack2<BF16>(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      if (row_ok && p.lse != nullptr) {
        const float lse =
            dead ? -INFINITY : (m_use - (FP8 ? kP8Offset : 0.f) + __log2f(l)) * kLn2;
        const int64_t li = varlen ? static_cast<int64_t>(h) * p.total_q + u.q0 + i
                                  : (static_cast<int64_t>(u.b) * p.H + h) * p.Sq + i;
        p.lse[li] = lse;
      }
    }
    blk += n_blk;
    if (n_blk > 0) ++u_cnt;
    }  // units
  }

  // ---------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::kIssuerWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, Cfg::kTmemCols);
  }
}

}  // namespace fa
