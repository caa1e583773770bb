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
// With the exchange fused into the ranks' combine kernels (they store their
// rows straight into every rank's gather buffer over NVLink and raise a flag
// there), the merge first waits for the R flags.
//
// One warp per row; each lane owns D / 32 consecutive elements and reads
// them from every rank with one 8- or 16-byte load, so a row's R partial rows
// are read once, coalesced, eight ranks per round trip to memory.  The op
// reads R * (D + 1) * 4 bytes and writes 2 * D (+ 4) bytes per row: HBM-bound
// in principle, and for decode-sized calls (a few hundred rows, partials that
// the exchange has just written to L2) one or two round trips of latency.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "fpd_ptx.cuh"

namespace fpd {

constexpr int kCpMergeWarps = 8;          // rows per CTA
constexpr uint32_t kCpErrTimeout = 0x4u;  // a rank's flag did not arrive in time

struct CpMergeParams {
  const float* partials;    // R blocks of `block` floats: [rows][D] O, then [rows] lse
  const float* sinks;       // [Hq] or nullptr
  __nv_bfloat16* out;
  float* lse;               // [rows] or nullptr
  int64_t block;            // floats per rank
  int64_t rows;
  int64_t out_tok_stride;   // elements between consecutive tokens of `out`
  int R, Hq;
  // WAIT: the partials arrive from the ranks' combine kernels; flags[r]
  // reaches `epoch` once rank r's rows are all in place.
  const uint32_t* flags;
  uint32_t epoch;
  uint64_t timeout_ns;
  uint32_t* status;         // kCpErrTimeout is or-ed in when a flag does not arrive
};

// WAIT: first wait for every rank's flag (one thread per CTA, acquire loads at
// system scope, bounded by timeout_ns of the GPU's global timer); a CTA that
// gives up records kCpErrTimeout and writes nothing.
template <int D, bool WAIT>
__global__ void __launch_bounds__(kCpMergeWarps * 32) fpd_cp_merge_kernel(const CpMergeParams p) {
  constexpr int PER = D / 32;
  constexpr int kBatch = 8;   // ranks whose partials are loaded together
  constexpr float kL2e = 1.4426950408889634f;
  if constexpr (WAIT) {
    __shared__ int arrived;
    if (threadIdx.x < 32) {   // warp 0: lane r polls rank r's flags (r, r + 32, ...)
      const int lane0 = threadIdx.x;
      const uint64_t t0 = global_timer_ns();
      bool ok = true;
      for (uint32_t spins = 0;; ++spins) {
        // acquire loads: once a lane sees its flag, the rows behind it are visible
        bool mine = true;
        for (int r = lane0; r < p.R; r += 32) mine &= ld_acquire_sys(p.flags + r) == p.epoch;
        if (__all_sync(0xffffffffu, mine)) break;
        if (spins >= (1u << 30) || global_timer_ns() - t0 > p.timeout_ns) {
          ok = false;
          break;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (lane0 == 0) {
        if (!ok && p.status) atomicOr(p.status, kCpErrTimeout);
        arrived = ok;
      }
    }
    __syncthreads();
    if (!arrived) return;
  }
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kCpMergeWarps + (threadIdx.x >> 5);
  if (row >= p.rows) return;
  const float* lse_r = p.partials + p.rows * D + row;         // rank r: lse_r[r * block]
  const float* o_r = p.partials + row * D + lane * PER;       // rank r: o_r[r * block + i]
  const int hq = (int)(row % p.Hq);
  const float sg = p.sinks ? p.sinks[hq] : -INFINITY;

  // Running maximum m, sum z and weighted sum acc over the ranks; each batch
  // of kBatch ranks costs one round trip to memory (all of them for R <= 8).
  float m = -INFINITY, z = 0.f;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  for (int r0 = 0; r0 < p.R; r0 += kBatch) {
    float lv[kBatch];
    float x[kBatch][PER];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      lv[u] = -INFINITY;
      if (r0 + u < p.R) {
        const int64_t off = (int64_t)(r0 + u) * p.block;
        lv[u] = lse_r[off];   // the same address in every lane
        if constexpr (PER == 4) {
          const float4 t = *reinterpret_cast<const float4*>(o_r + off);
          x[u][0] = t.x, x[u][1] = t.y, x[u][2] = t.z, x[u][3] = t.w;
        } else {
          const float2 t = *reinterpret_cast<const float2*>(o_r + off);
          x[u][0] = t.x, x[u][1] = t.y;
        }
      }
    }
    float mb = m;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) mb = fmaxf(mb, lv[u]);
    if (mb == -INFINITY) continue;   // no rank of this batch holds a key of the row
    const float sc = m == -INFINITY ? 0.f : fast_exp2((m - mb) * kL2e);
    z *= sc;
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] *= sc;
    m = mb;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (lv[u] == -INFINITY) continue;   // a rank without a key of this row (or past R)
      const float w = fast_exp2((lv[u] - m) * kL2e);
      z += w;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, x[u][i], acc[i]);
    }
  }
  const float M = fmaxf(m, sg);
  const float rr = m == -INFINITY ? 0.f : fast_exp2((m - M) * kL2e);
  const float Z = z * rr + (sg == -INFINITY ? 0.f : fast_exp2((sg - M) * kL2e));
  const bool any = Z > 0.f;   // false: no rank and no sink covers the row
  const float inv = any ? rr / Z : 0.f;
  const int64_t tok = row / p.Hq;
  __nv_bfloat16* dst = p.out + tok * p.out_tok_stride + (int64_t)hq * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; i += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv,
                                                                       acc[i + 1] * inv);
  if (lane == 0 && p.lse) p.lse[row] = any ? M + logf(Z) : -INFINITY;
}

}  // namespace fpd
