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

// ------------------------------------------------------------------ NVFP4 --
//
// NVFP4 cache write: the block recipe of the gist's NVFP4 cache writer (writer
// kernel and quantisation helper) with exact fp32 reciprocals: per 16
// consecutive elements of a token's head row
//   sf   = e4m3_rne_sat((amax * (1/6)) * gs)        gs = 1 / scale
//   osc  = sf == 0 ? 0 : 1 / (e4m3(sf) * (1 / gs))
//   code = e2m1_rne_sat(x * osc)                    (element 2i in the low nibble)
// into head-major pages: data [page][kv head][slot][D/2], scales
// [page][kv head][slot][D/16], each region at its own page stride.  One thread
// per 16-element block: two 16-byte loads, one 8-byte and one 1-byte store.

struct CacheWriteFp4Params {
  const __nv_bfloat16* key;
  const __nv_bfloat16* value;
  const int64_t* slot_mapping;
  uint8_t* k_data;
  uint8_t* k_sf;
  uint8_t* v_data;
  uint8_t* v_sf;
  uint32_t* status;
  int64_t key_stride, value_stride;         // elements between tokens
  int64_t data_page_stride, sf_page_stride;  // bytes between pages
  int64_t n_slots;
  int num_tokens, D, bt;
  int blocks;                               // Hkv * D / 16 per token and side
  float k_gs, v_gs;                         // 1 / k_scale, 1 / v_scale (fp32)
  float k_rgs, v_rgs;                       // 1 / gs (fp32)
};

// Two floats -> one byte of two E2M1 codes (lo in the low nibble), round to
// nearest even, saturating at +-6.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
      "cvt.u16.u8 %0, b;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(kWriteThreads) fpd_cache_write_nvfp4_kernel(
    const CacheWriteFp4Params p) {
  constexpr float kInv6 = 1.0f / 6.0f;
  const int64_t per_token = 2LL * p.blocks;
  const int64_t units = (int64_t)p.num_tokens * per_token;
  const int hb = p.D / 16;   // blocks per head row
  for (int64_t u = (int64_t)blockIdx.x * kWriteThreads + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * kWriteThreads) {
    const int t = (int)(u / per_token);
    const int r = (int)(u - (int64_t)t * per_token);
    const bool is_v = r >= p.blocks;
    const int blk = is_v ? r - p.blocks : r;
    const int64_t slot = __ldg(p.slot_mapping + t);
    if (slot < 0) continue;   // padded token
    if (slot >= p.n_slots) {
      if (p.status && blk == 0 && !is_v) atomicOr(p.status, kErrSlot);
      continue;
    }
    const __nv_bfloat16* src =
        (is_v ? p.value + (int64_t)t * p.value_stride : p.key + (int64_t)t * p.key_stride) +
        blk * 16;
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(src));
    const uint4 b = __ldcs(reinterpret_cast<const uint4*>(src) + 1);
    float x[16];
    const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* hb2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 fa = __bfloat1622float2(ha[j]);
      const float2 fb = __bfloat1622float2(hb2[j]);
      x[2 * j] = fa.x, x[2 * j + 1] = fa.y;
      x[8 + 2 * j] = fb.x, x[8 + 2 * j + 1] = fb.y;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const float gs = is_v ? p.v_gs : p.k_gs;
    const float rgs = is_v ? p.v_rgs : p.k_rgs;
    const float sf_f = __fmul_rn(__fmul_rn(amax, kInv6), gs);
    const uint32_t sfc = f32x4_to_e4m3x4(sf_f, 0.f, 0.f, 0.f) & 0xFFu;
    const float sf_v = __half2float(__ushort_as_half(
        (unsigned short)(e4m3x2_to_f16x2((uint16_t)sfc) & 0xFFFFu)));
    const float osc = sf_v == 0.f ? 0.f : __frcp_rn(__fmul_rn(sf_v, rgs));
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w[i / 4] |= f32x2_to_e2m1x2(__fmul_rn(x[2 * i], osc), __fmul_rn(x[2 * i + 1], osc))
                  << (8 * (i % 4));
    const int page = (int)(slot / p.bt), off = (int)(slot - (int64_t)page * p.bt);
    const int h = blk / hb, j = blk - h * hb;
    const int64_t row = (int64_t)h * p.bt + off;
    uint8_t* data = (is_v ? p.v_data : p.k_data) + (int64_t)page * p.data_page_stride +
                    row * (p.D / 2) + j * 8;
    *reinterpret_cast<uint2*>(data) = make_uint2(w[0], w[1]);
    (is_v ? p.v_sf : p.k_sf)[(int64_t)page * p.sf_page_stride + row * hb + j] = (uint8_t)sfc;
  }
}

}  // namespace fpd
