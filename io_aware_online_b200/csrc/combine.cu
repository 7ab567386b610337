// combine.cu -- LSE-weighted combine of split partial results
// ("FlashAttention common interfaces" section 3.4 flash_attn_combine; changelog
// post v2.2: the split ranges are reduced by an extra kernel).
//
//   LSE = M + ln sum_s exp(lse_s - M),  M = max_s lse_s
//   O   = sum_s exp(lse_s - LSE) * O_s           (splits with lse_s = -inf skipped)
//
// One warp per output row (b, s, h).  The weights of a row are computed once into
// shared memory; lanes then stream the head-dim columns.  Memory-bound: it reads
// splits * (head_dim + 1) floats per row and writes one row.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fa_internal.h"

namespace fa {

constexpr int kCombineWarps = 4;
constexpr int kCombineMaxSplits = 256;

template <int OUT_DT>
__global__ void __launch_bounds__(kCombineWarps * 32) combine_kernel(const CombineParams p) {
  __shared__ float wts[kCombineWarps][kCombineMaxSplits];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kCombineWarps + warp;
  const int64_t rows = static_cast<int64_t>(p.B) * p.S * p.H;
  if (row >= rows) return;
  const int h = static_cast<int>(row % p.H);
  const int s = static_cast<int>((row / p.H) % p.S);
  const int b = static_cast<int>(row / (static_cast<int64_t>(p.H) * p.S));
  const float* lrow = p.lp + b * p.lp_s[0] + s * p.lp_s[1] + h * p.lp_s[2];
  const float* orow = p.op + b * p.op_s[0] + s * p.op_s[1] + h * p.op_s[2];

  float m = -INFINITY;
  for (int sp = lane; sp < p.splits; sp += 32) m = fmaxf(m, lrow[sp * p.lp_s[3]]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float lse = -INFINITY;
  if (m != -INFINITY) {
    float z = 0.f;
    for (int sp = lane; sp < p.splits; sp += 32) {
      const float l = lrow[sp * p.lp_s[3]];
      z += (l == -INFINITY) ? 0.f : expf(l - m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    lse = m + logf(z);
  }
  for (int sp = lane; sp < p.splits; sp += 32) {
    const float l = lrow[sp * p.lp_s[3]];
    wts[warp][sp] = (l == -INFINITY || lse == -INFINITY) ? 0.f : expf(l - lse);
  }
  __syncwarp();

  const int64_t out_row = row * p.D;
  if (p.op_s[3] == 1 && (p.op_s[4] % 4) == 0 && ((reinterpret_cast<uintptr_t>(orow) & 15) == 0)) {
    // head dim contiguous: each lane owns 4 consecutive columns (one 16-byte load
    // per split), and the split loop is unrolled so that loads overlap
    for (int d0 = lane * 4; d0 < p.D; d0 += 128) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      int sp = 0;
      for (; sp + 4 <= p.splits; sp += 4) {
        float4 v[4];
        float wv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          wv[u] = wts[warp][sp + u];
          v[u] = wv[u] != 0.f ? *reinterpret_cast<const float4*>(orow + (sp + u) * p.op_s[4] + d0)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          acc.x = fmaf(wv[u], v[u].x, acc.x);
          acc.y = fmaf(wv[u], v[u].y, acc.y);
          acc.z = fmaf(wv[u], v[u].z, acc.z);
          acc.w = fmaf(wv[u], v[u].w, acc.w);
        }
      }
      for (; sp < p.splits; ++sp) {
        const float wv = wts[warp][sp];
        if (wv == 0.f) continue;
        const float4 v = *reinterpret_cast<const float4*>(orow + sp * p.op_s[4] + d0);
        acc.x = fmaf(wv, v.x, acc.x);
        acc.y = fmaf(wv, v.y, acc.y);
        acc.z = fmaf(wv, v.z, acc.z);
        acc.w = fmaf(wv, v.w, acc.w);
      }
      // head_dim is a multiple of 4 (checked by the host), so all four columns exist
      if constexpr (OUT_DT == 0) {
        __half* o = static_cast<__half*>(p.out) + out_row + d0;
        o[0] = __float2half_rn(acc.x); o[1] = __float2half_rn(acc.y);
        o[2] = __float2half_rn(acc.z); o[3] = __float2half_rn(acc.w);
      } else if constexpr (OUT_DT == 1) {
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + out_row + d0;
        o[0] = __float2bfloat16_rn(acc.x); o[1] = __float2bfloat16_rn(acc.y);
        o[2] = __float2bfloat16_rn(acc.z); o[3] = __float2bfloat16_rn(acc.w);
      } else {
        float* o = static_cast<float*>(p.out) + out_row + d0;
        o[0] = acc.x; o[1] = acc.y; o[2] = acc.z; o[3] = acc.w;
      }
    }
  } else {
    for (int dd = lane; dd < p.D; dd += 32) {
      float acc = 0.f;
      const float* col = orow + dd * p.op_s[3];
      for (int sp = 0; sp < p.splits; ++sp) {
        const float wv = wts[warp][sp];
        if (wv != 0.f) acc = fmaf(wv, col[sp * p.op_s[4]], acc);
      }
      if constexpr (OUT_DT == 0)
        static_cast<__half*>(p.out)[out_row + dd] = __float2half_rn(acc);
      else if constexpr (OUT_DT == 1)
        static_cast<__nv_bfloat16*>(p.out)[out_row + dd] = __float2bfloat16_rn(acc);
      else
        static_cast<float*>(p.out)[out_row + dd] = acc;
    }
  }
  if (lane == 0 && p.lse != nullptr)
    p.lse[(static_cast<int64_t>(b) * p.H + h) * p.S + s] = lse;
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.S * p.H;
  if (rows == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((rows + kCombineWarps - 1) / kCombineWarps));
  switch (p.out_dtype) {
    case 0: combine_kernel<0><<<grid, kCombineWarps * 32, 0, stream>>>(p); break;
    case 1: combine_kernel<1><<<grid, kCombineWarps * 32, 0, stream>>>(p); break;
    default: combine_kernel<2><<<grid, kCombineWarps * 32, 0, stream>>>(p); break;
  }
  return cudaGetLastError();
}

}  // namespace fa
