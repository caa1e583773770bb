// fpd_cache_write.cuh -- the FP8 (E4M3) KV-cache write kernel for sm_100a.
//
// New tokens' bf16 K and V rows are quantised with the per-tensor scales and
// scattered into the paged caches, following the per-tensor quantisation of
// the standalone cache-writer kernel in the NVFP4 KV-cache serving gist (its
// writer kernel and host wrapper): the reciprocal of the scale is taken once
// in fp32, each element is multiplied by it in fp32, and the product is
// rounded to the nearest E4M3 value, ties to even, saturating at +-448.  A
// token's slot is slot_mapping[t] = page * block_tokens + offset; a negative
// slot marks a padded token, which is skipped.
//
// Layout: key/value [num_tokens, Hkv, D] bf16 with a token stride (elements);
// caches [num_blocks, block_tokens, Hkv, D] E4M3, so the Hkv * D elements of
// one token form one contiguous row on both sides; or head-major caches
// [num_blocks, Hkv, block_tokens, D] (the gist writer's HND layout), where each
// 16-element chunk still lands contiguously inside one head's row.  One thread converts 16
// consecutive elements: two 16-byte loads, one 16-byte store, so a warp reads
// 1 KB and writes 512 B of one row contiguously.  The op is HBM-bound:
// 6 bytes per element (4 read, 2 written).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "fpd_ptx.cuh"

namespace fpd {

constexpr uint32_t kErrSlot = 0x8u;   // a slot_mapping entry past the end of the cache
constexpr int kWriteThreads = 256;
constexpr int kWriteElems = 16;       // elements per thread

struct CacheWriteParams {
  const __nv_bfloat16* key;
  const __nv_bfloat16* value;
  const int64_t* slot_mapping;
  uint8_t* k_cache;
  uint8_t* v_cache;
  uint32_t* status;        // optional: FPD_DEVERR_SLOT is or-ed in
  int64_t key_stride, value_stride;   // elements between consecutive tokens
  int64_t n_slots;         // num_blocks * block_tokens
  int num_tokens;
  int row_chunks;          // Hkv * D / 16
  float k_inv, v_inv;      // 1 / k_scale, 1 / v_scale, rounded to fp32 on the host
  int hnd;                 // head-major pages [num_blocks, Hkv, bt, D] (else token-major)
  int bt;                  // tokens per page (head-major pages)
  int head_chunks;         // D / 16
};

// Eight bf16 (a 16-byte vector) times `inv`, as four e4m3x2 pairs packed into
// two words (element 0 in the lowest byte).
__device__ __forceinline__ uint2 quantise8(const uint4 raw, float inv) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
  float f[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 x = __bfloat1622float2(h[j]);
    f[2 * j] = __fmul_rn(x.x, inv);
    f[2 * j + 1] = __fmul_rn(x.y, inv);
  }
  return make_uint2(f32x4_to_e4m3x4(f[0], f[1], f[2], f[3]),
                    f32x4_to_e4m3x4(f[4], f[5], f[6], f[7]));
}

// Work unit u -> (token, K or V, 16-element chunk of the row); grid-stride.
__global__ void __launch_bounds__(kWriteThreads) fpd_cache_write_kernel(const CacheWriteParams p) {
  const int64_t per_token = 2LL * p.row_chunks;
  const int64_t units = (int64_t)p.num_tokens * per_token;
  for (int64_t u = (int64_t)blockIdx.x * kWriteThreads + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * kWriteThreads) {
    const int t = (int)(u / per_token);
    const int r = (int)(u - (int64_t)t * per_token);
    const bool is_v = r >= p.row_chunks;
    const int c = is_v ? r - p.row_chunks : r;
    const int64_t slot = __ldg(p.slot_mapping + t);
    if (slot < 0) continue;   // padded token
    if (slot >= p.n_slots) {
      if (p.status && c == 0 && !is_v) atomicOr(p.status, kErrSlot);
      continue;
    }
    const __nv_bfloat16* src =
        (is_v ? p.value + (int64_t)t * p.value_stride : p.key + (int64_t)t * p.key_stride) +
        c * kWriteElems;
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(src));
    const uint4 b = __ldcs(reinterpret_cast<const uint4*>(src) + 1);
    const float inv = is_v ? p.v_inv : p.k_inv;
    const uint2 lo = quantise8(a, inv), hi = quantise8(b, inv);
    uint8_t* base = is_v ? p.v_cache : p.k_cache;
    uint8_t* dst;
    if (p.hnd) {   // [page][kv head][in-page slot][d]; slots fit in 32 bits here
      const int s32 = (int)slot;
      const int page = s32 / p.bt, off = s32 - page * p.bt;
      const int h = c / p.head_chunks, part = c - h * p.head_chunks;
      const int Hkv = p.row_chunks / p.head_chunks;
      dst = base + ((((int64_t)page * Hkv + h) * p.bt + off) * p.head_chunks + part) * kWriteElems;
    } else {       // [slot][kv head][d]: a token's row is contiguous
      dst = base + (slot * p.row_chunks + c) * kWriteElems;
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(lo.x, lo.y, hi.x, hi.y);
  }
}

}  // namespace fpd
