// fpd_cp_merge.cuh -- the context-parallel merge kernel for sm_100a.
//
// With a sequence's keys spread over R ranks, each rank's decode over its own
// keys gives a partial (O_r, lse_r) per row (token, head): O_r is normalised
// by that rank's softmax sum and lse_r = ln of the sum.  The attention over
// all keys is the split-KV merge of FlashInfer PR #5591 (Summary: partial_O /
// partial_lse and the split merge), with ranks in place of splits:
//   M = max(max_r lse_r, sigma),  w_r = e^(lse_r - M),
//   Z = sum_r w_r + e^(sigma - M),  out = sum_r w_r O_r / Z,  lse = M + ln Z,
// where sigma is the head's sink logit (-inf without sinks); a sink adds to
// the denominator only, so the ranks' partials carry none.
//
// One warp per row; each lane owns D / 32 consecutive elements and reads
// them from every rank with one 8- or 16-byte load, so a row's R partial rows
// are read once, coalesced.  The op reads R * (D + 1) * 4 bytes and writes
// 2 * D (+ 4) bytes per row: HBM-bound, and for decode-sized calls (a few
// hundred rows) a single wave of latency.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "fpd_ptx.cuh"

namespace fpd {

constexpr int kCpMergeWarps = 8;   // rows per CTA

struct CpMergeParams {
  const float* partials;    // R blocks of `block` floats: [rows][D] O, then [rows] lse
  const float* sinks;       // [Hq] or nullptr
  __nv_bfloat16* out;
  float* lse;               // [rows] or nullptr
  int64_t block;            // floats per rank
  int64_t rows;
  int64_t out_tok_stride;   // elements between consecutive tokens of `out`
  int R, Hq;
};

template <int D>
__global__ void __launch_bounds__(kCpMergeWarps * 32) fpd_cp_merge_kernel(const CpMergeParams p) {
  constexpr int PER = D / 32;
  constexpr float kL2e = 1.4426950408889634f;
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kCpMergeWarps + (threadIdx.x >> 5);
  if (row >= p.rows) return;
  const float* lse_r = p.partials + p.rows * D + row;         // rank r: lse_r[r * block]
  const float* o_r = p.partials + row * D + lane * PER;       // rank r: o_r[r * block + i]

  // the largest partial lse (lanes take ranks lane, lane + 32, ...)
  float mx = -INFINITY;
  for (int r = lane; r < p.R; r += 32) mx = fmaxf(mx, lse_r[(int64_t)r * p.block]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const int hq = (int)(row % p.Hq);
  const float sg = p.sinks ? p.sinks[hq] : -INFINITY;
  const float M = fmaxf(mx, sg);

  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float Z = 0.f;
  if (mx != -INFINITY) {
#pragma unroll 4
    for (int r = 0; r < p.R; ++r) {
      const int64_t off = (int64_t)r * p.block;
      const float l = lse_r[off];   // the same address in every lane
      float v[PER];
      if constexpr (PER == 4) {
        const float4 t = *reinterpret_cast<const float4*>(o_r + off);
        v[0] = t.x, v[1] = t.y, v[2] = t.z, v[3] = t.w;
      } else {
        const float2 t = *reinterpret_cast<const float2*>(o_r + off);
        v[0] = t.x, v[1] = t.y;
      }
      if (l == -INFINITY) continue;   // the rank holds no key of this row
      const float w = fast_exp2((l - M) * kL2e);
      Z += w;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, v[i], acc[i]);
    }
  }
  if (p.sinks && sg != -INFINITY) Z += fast_exp2((sg - M) * kL2e);
  const bool any = Z > 0.f;   // false: no rank and no sink covers the row
  const float inv = any ? 1.0f / Z : 0.f;
  const int64_t tok = row / p.Hq;
  __nv_bfloat16* dst = p.out + tok * p.out_tok_stride + (int64_t)hq * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; i += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv,
                                                                       acc[i + 1] * inv);
  if (lane == 0 && p.lse) p.lse[row] = any ? M + logf(Z) : -INFINITY;
}

}  // namespace fpd
