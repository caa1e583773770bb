// fpd_api.cu -- host side of the C ABI declared in include/fp8_paged_decode.h:
// argument validation, the split planner, TMA descriptor encoding and the
// kernel launch.  No call allocates or frees device memory, and only
// fp8_paged_decode_check_status synchronises.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fp8_paged_decode.h"
#include "fpd_cache_write.cuh"
#include "fpd_cp_merge.cuh"
#include "fpd_kernels.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kHeaderBytes = 256;    // status word, work counter, finished-CTA counter
// Split heuristic, per stage shape (measured on the five synthetic workloads):
// about this many work items per resident CTA slot, and no item below this
// many (token, KV head) rows.  Four-head items carry a larger fixed cost (query
// set-up of four heads, partial results of four heads), so they get fewer,
// larger items.
constexpr int kTargetWaves1 = 8, kMinChunkRows1 = 256;    // one KV head per stage
constexpr int kTargetWaves4 = 5, kMinChunkRows4 = 1024;   // four KV heads per stage
// Four-head items over E4M3 pages of at least this many tokens at
// kTargetWaves4 rounds take one round fewer: long items carry little fixed
// cost per token, and fewer splits leave the combine kernel fewer partials to
// merge (measured: large mixed batch 26 -> 33 pages 206.3 -> 202.5 us and
// 213.0 -> 210.1 us on two boxes, long context 8 -> 10 pages 175.6 -> 173.7
// us on one and equal on the other; the Llama-3-8B-shaped call, 256-token
// items, keeps its 16 pages: 19 pages took 64.4 instead of 60.5 us).  NVFP4
// pages keep kTargetWaves4: their kernel is bound by instruction issue, and
// the larger items lengthened its tail (long context 155.3 -> 168.6 us).
constexpr int kLongItemTokens4 = 512;
constexpr int kMinItemTokens = 48;   // shortest split when a call cannot fill the machine
constexpr int kOccCacheSize = 32;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool supported_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8 || g == 16; }

// q_len query tokens per sequence, 1 .. FPD_MAX_Q_LEN.
fpd_status validate_shape(int B, int Hq, int Hkv, int D, int bt, int max_blocks, int q_len = 1) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bt <= 0 || max_blocks <= 0 || q_len < 1)
    return FPD_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FPD_ERR_INVALID_ARG;
  if (!supported_group(Hq / Hkv)) return FPD_ERR_UNSUPPORTED;
  if (q_len > FPD_MAX_Q_LEN) return FPD_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return FPD_ERR_UNSUPPORTED;
  if (bt != 16 && bt != 32 && bt != 64) return FPD_ERR_UNSUPPORTED;
  if ((int64_t)max_blocks * bt > INT32_MAX) return FPD_ERR_UNSUPPORTED;
  return FPD_OK;
}

// MMA n-tiles (8 columns each) for `cols` columns per KV head.
int n_tiles(int cols) { return cols > 8 ? 2 : 1; }

// Query positions per work item with q_len queries per sequence: a work item's
// MMA columns are its positions x the g query heads of a KV head, at most
// FPD_MQ_COLS (8: one n-tile, 16: two).  A sequence's queries are cut into
// ceil(q_len / P) chunks of near-equal size; each chunk is its own work item
// over the same KV range (g = 16 always takes one position per item).
#ifndef FPD_MQ_COLS
#define FPD_MQ_COLS 16
#endif
int q_per_item(int q_len, int g) {
  if (q_len <= 1) return 1;
  int P = FPD_MQ_COLS / g;
  if (P < 1) P = 1;
  if (P >= q_len) return q_len;
  const int chunks = (q_len + P - 1) / P;
  return (q_len + chunks - 1) / chunks;
}

// KV heads per stage and work item: 4 whenever the KV heads split into groups
// of 4 (one TMA box then covers 16 tokens of 4 heads), else 1.
int heads_per_stage(int Hkv) { return Hkv % 4 == 0 ? 4 : 1; }

// Depth of the shared-memory stage ring (build-time tunable).
#ifndef FPD_STAGES_D128_NT1
#define FPD_STAGES_D128_NT1 3
#endif
#ifndef FPD_STAGES_D128_NT2
#define FPD_STAGES_D128_NT2 4
#endif
#ifndef FPD_STAGES_D64
#define FPD_STAGES_D64 6
#endif
#ifndef FPD_STAGES_HB4_D128
#define FPD_STAGES_HB4_D128 4
#endif
#ifndef FPD_STAGES_HB4_D64
#define FPD_STAGES_HB4_D64 5
#endif
#ifndef FPD_STAGES_HB4_D128_NT2
#define FPD_STAGES_HB4_D128_NT2 4
#endif
// NVFP4 stages are 72 D bytes instead of 128 D: the ring keeps about the same
// bytes in flight with 16 / 9 as many stages.
#ifndef FPD_FP4_STAGES_NUM
#define FPD_FP4_STAGES_NUM 16
#endif
#ifndef FPD_FP4_STAGES_DEN
#define FPD_FP4_STAGES_DEN 9
#endif
int ring_stages(int D, int NT, int HB, bool fp4 = false) {
  int s;
  if (HB == 4)
    s = D == 128 ? (NT == 2 ? FPD_STAGES_HB4_D128_NT2 : FPD_STAGES_HB4_D128) : FPD_STAGES_HB4_D64;
  else if (D == 128) s = NT == 2 ? FPD_STAGES_D128_NT2 : FPD_STAGES_D128_NT1;
  else s = FPD_STAGES_D64;
  return fp4 ? s * FPD_FP4_STAGES_NUM / FPD_FP4_STAGES_DEN : s;
}

// Header ring depth: two slots while an item's query rows are small, one
// otherwise, so that the stage ring keeps its shared memory.
#ifndef FPD_HDR2_MAX_QBYTES
#define FPD_HDR2_MAX_QBYTES 4096
#endif
int header_slots(int D, int cols, int HB) {
  return HB * cols * D * 2 <= FPD_HDR2_MAX_QBYTES ? 2 : 1;
}

// Shared memory of the split kernel with `cols` = q_len * g columns per KV head.
int smem_bytes_for(int D, int cols, int HB, int B, bool fp4 = false) {
  const int NT = n_tiles(cols);
  return fpd::smem_layout(D, NT, HB, ring_stages(D, NT, HB, fp4), header_slots(D, cols, HB), cols,
                          B, fp4)
      .total;
}

// Workspace carve-up: [header 256 B][partial O][partial lse]
struct WsLayout {
  size_t part_o, part_lse, total, zero_prefix;
};

// f32_out: every row goes through the combine, so partials exist for one split too.
WsLayout ws_layout(int B, int Hq, int Hkv, int D, int max_splits, bool f32_out = false) {
  (void)Hkv;
  WsLayout w;
  size_t off = kHeaderBytes;
  w.zero_prefix = off;  // bytes that must be zero before the first call
  const bool parts = max_splits > 1 || f32_out;
  w.part_o = off;
  if (parts) off += align_up((size_t)B * Hq * max_splits * D * sizeof(float), 256);
  w.part_lse = off;
  if (parts) off += align_up((size_t)B * Hq * max_splits * sizeof(float), 256);
  w.total = off;
  return w;
}

// ---- per-device facts, queried once
struct OccEntry {
  int D, NT, HB, mq, fp4, smem, occ;
};
struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int max_smem = 0;
  int n_occ = 0;
  OccEntry occ[kOccCacheSize];
};
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

template <int D, int NT, int HB, bool MQ>
const void* split_kernel_ptr(bool fp4) {
  return fp4 ? reinterpret_cast<const void*>(&fpd::fpd_split_kernel_nvfp4<D, NT, HB, MQ>)
             : reinterpret_cast<const void*>(&fpd::fpd_split_kernel<D, NT, HB, MQ>);
}

template <int HB, bool MQ>
const void* split_kernel_hb(int D, int NT, bool fp4) {
  if (D == 128)
    return NT == 2 ? split_kernel_ptr<128, 2, HB, MQ>(fp4) : split_kernel_ptr<128, 1, HB, MQ>(fp4);
  return NT == 2 ? split_kernel_ptr<64, 2, HB, MQ>(fp4) : split_kernel_ptr<64, 1, HB, MQ>(fp4);
}

// mq: the kernel for several query tokens per sequence; fp4: over NVFP4 pages
const void* split_kernel_for(int D, int NT, int HB, bool mq, bool fp4) {
  if (mq)
    return HB == 4 ? split_kernel_hb<4, true>(D, NT, fp4) : split_kernel_hb<1, true>(D, NT, fp4);
  return HB == 4 ? split_kernel_hb<4, false>(D, NT, fp4) : split_kernel_hb<1, false>(D, NT, fp4);
}

bool current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) {
    cudaGetLastError();
    return false;
  }
  return true;
}

// The per-device facts, queried on first use (call with g_mu held).
DeviceInfo* device_info(int dev) {
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    if (cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&di.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    di.ready = true;
  }
  return &di;
}

// SM count of the current device.
bool device_sm_count(int* num_sms) {
  int dev = 0;
  if (!current_device(&dev)) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  const DeviceInfo* di = device_info(dev);
  if (!di) return false;
  *num_sms = di->num_sms;
  return true;
}

// SM count of the current device and the number of split-kernel CTAs that fit
// on one SM with `smem` bytes of dynamic shared memory (0 if none).  Also sets
// the kernel's dynamic shared-memory limit, which its launch needs.
bool device_occupancy(int D, int NT, int HB, bool mq, bool fp4, int smem, int* num_sms,
                      int* ctas_per_sm) {
  int dev = 0;
  if (!current_device(&dev)) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo* dip = device_info(dev);
  if (!dip) return false;
  DeviceInfo& di = *dip;
  *num_sms = di.num_sms;
  for (int i = 0; i < di.n_occ; ++i) {
    const OccEntry& e = di.occ[i];
    if (e.D == D && e.NT == NT && e.HB == HB && e.mq == (int)mq && e.fp4 == (int)fp4 &&
        e.smem == smem) {
      *ctas_per_sm = e.occ;
      return true;
    }
  }
  int occ = 0;
  const void* fn = split_kernel_for(D, NT, HB, mq, fp4);
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const int dyn_max = di.max_smem - (int)fa.sharedSizeBytes;  // static + dynamic <= opt-in max
  if (smem <= dyn_max) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, fpd::kThreads, smem) !=
            cudaSuccess) {
      cudaGetLastError();
      return false;
    }
  }
  if (di.n_occ < kOccCacheSize)
    di.occ[di.n_occ++] = OccEntry{D, NT, HB, (int)mq, (int)fp4, smem, occ};
  *ctas_per_sm = occ;
  return true;
}

// ---- TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    else
      cudaGetLastError();
  });
  return g_encode;
}

// View a byte cache as a tensor for TMA.
// Token-major pages [num_blocks, bt, Hkv, D], 3-D:
//   HB = 1: (d, kv head, token row), box (D, 1, bt): one page of one head.
//   HB = 4: (d, token row, kv head), box (D, 16, 4): 16 tokens of 4 heads,
//           landing head-major in shared memory (4 tiles of 16 rows).
// Head-major pages [num_blocks, Hkv, bt, D] (hnd), 4-D (d, slot, kv head, page):
//   HB = 1: box (D, bt, 1, 1); HB = 4: box (D, 16, 4, 1).  Both land in shared
//   memory exactly as the token-major boxes do.
bool encode_cache_map(CUtensorMap* map, const void* base, int num_blocks, int bt, int Hkv, int D,
                      int HB, bool hnd) {
  auto enc = encoder();
  if (!enc) return false;
  const cuuint64_t rows = (cuuint64_t)num_blocks * bt;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4];
  cuuint32_t rank = 3;
  if (hnd) {
    rank = 4;
    dims[0] = D, dims[1] = bt, dims[2] = Hkv, dims[3] = num_blocks;
    strides[0] = D, strides[1] = (cuuint64_t)bt * D, strides[2] = (cuuint64_t)Hkv * bt * D;
    box[0] = D, box[1] = HB == 1 ? bt : fpd::kBoxTokens, box[2] = HB, box[3] = 1u;
  } else if (HB == 1) {
    dims[0] = D, dims[1] = Hkv, dims[2] = rows;
    strides[0] = D, strides[1] = (cuuint64_t)Hkv * D;
    box[0] = D, box[1] = 1u, box[2] = bt;
  } else {
    dims[0] = D, dims[1] = rows, dims[2] = Hkv;
    strides[0] = (cuuint64_t)Hkv * D, strides[1] = D;
    box[0] = D, box[1] = fpd::kBoxTokens, box[2] = HB;
  }
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  const CUtensorMapSwizzle swz =
      D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  // No L2 promotion: each box row is one 128-byte (or 64-byte) line of one KV
  // head, and widening it fetches the neighbouring head's line, which is
  // often evicted before its own reader arrives (measured: 18% extra DRAM
  // reads on the windowed, GQA-8 workload with 256-byte promotion).
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// TMA views of NVFP4 pages (head-major, no swizzle: the rows are read by
// plain 8- and 16-byte loads).
//   data:   (d pair, slot, kv head, page), strides (D/2, bt*D/2, data stride);
//           box (D/2, 16, 4, 1) with four heads per stage, (D/2, bt, 1, 1) with one.
//   scales: (the D bytes of 16 tokens' block scales, 16-token group, kv head,
//           page), strides (D, bt*D/16, scale stride); box (D, 1, 4, 1) or
//           (D, bt/16, 1, 1).
// Each box lands in shared memory as rows [head][token][bytes], like the
// E4M3 tiles.
bool encode_nvfp4_map(CUtensorMap* map, const void* base, int num_blocks, int bt, int Hkv, int D,
                      int HB, int64_t page_stride, bool scales) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4];
  if (!scales) {
    dims[0] = D / 2, dims[1] = bt, dims[2] = Hkv, dims[3] = num_blocks;
    strides[0] = D / 2, strides[1] = (cuuint64_t)bt * (D / 2);
    box[0] = D / 2, box[1] = HB == 1 ? bt : fpd::kBoxTokens, box[2] = HB, box[3] = 1u;
  } else {
    dims[0] = D, dims[1] = bt / fpd::kBoxTokens, dims[2] = Hkv, dims[3] = num_blocks;
    strides[0] = D, strides[1] = (cuuint64_t)bt * (D / 16);
    box[0] = D, box[1] = HB == 1 ? bt / fpd::kBoxTokens : 1u, box[2] = HB, box[3] = 1u;
  }
  strides[2] = (cuuint64_t)page_stride;
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Combine launch as a programmatic dependent of the split kernel: its CTAs may
// start while the split kernel drains and wait for it on the device.
template <int D, bool MQ, int NB>
cudaError_t launch_combine_nb(const fpd::CombineParams& c, cudaStream_t st) {
  const int rows_per_cta = c.rows_per_cta;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((c.B * c.q_len * c.Hq + rows_per_cta - 1) / rows_per_cta));
  cfg.blockDim = dim3(c.wpr * rows_per_cta * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fpd::fpd_combine_kernel<D, MQ, NB>, c);
}

// The first-round batch: one warp per row loads min(max_splits, 8) partials.
template <int D, bool MQ>
cudaError_t launch_combine(const fpd::CombineParams& c, cudaStream_t st) {
  if (c.wpr > 1) return launch_combine_nb<D, MQ, fpd::kCombineBatch>(c, st);
  switch (c.max_splits) {
    case 1: return launch_combine_nb<D, MQ, 1>(c, st);
    case 2: return launch_combine_nb<D, MQ, 2>(c, st);
    case 3: return launch_combine_nb<D, MQ, 3>(c, st);
    case 4: return launch_combine_nb<D, MQ, 4>(c, st);
    case 5: return launch_combine_nb<D, MQ, 5>(c, st);
    case 6: return launch_combine_nb<D, MQ, 6>(c, st);
    case 7: return launch_combine_nb<D, MQ, 7>(c, st);
    default: return launch_combine_nb<D, MQ, fpd::kCombineBatch>(c, st);
  }
}

// The split kernel is launched as a programmatic dependent of whatever ran
// before it in the stream: its CTAs may become resident while that kernel
// drains, and its first instruction waits for that kernel's completion, so
// the ordering is that of a plain launch without the launch gap.
template <int D, int NT, int HB, bool MQ>
cudaError_t launch_split(const CUtensorMap& km, const CUtensorMap& vm, const fpd::DecodeParams& p,
                         int ctas, int smem, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(fpd::kThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fpd::fpd_split_kernel<D, NT, HB, MQ>, km, vm, p);
}

template <int HB, bool MQ>
cudaError_t launch_split_hb(int D, int NT, const CUtensorMap& km, const CUtensorMap& vm,
                            const fpd::DecodeParams& p, int ctas, int smem, cudaStream_t st) {
  if (D == 128)
    return NT == 2 ? launch_split<128, 2, HB, MQ>(km, vm, p, ctas, smem, st)
                   : launch_split<128, 1, HB, MQ>(km, vm, p, ctas, smem, st);
  return NT == 2 ? launch_split<64, 2, HB, MQ>(km, vm, p, ctas, smem, st)
                 : launch_split<64, 1, HB, MQ>(km, vm, p, ctas, smem, st);
}

// The NVFP4 split kernel, launched like the E4M3 one (programmatic dependent).
template <int D, int NT, int HB, bool MQ>
cudaError_t launch_split_nvfp4(const CUtensorMap (&maps)[4], const fpd::DecodeParams& p, int ctas,
                               int smem, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(fpd::kThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fpd::fpd_split_kernel_nvfp4<D, NT, HB, MQ>, maps[0], maps[1],
                            maps[2], maps[3], p);
}

template <int HB, bool MQ>
cudaError_t launch_split_nvfp4_hb(int D, int NT, const CUtensorMap (&maps)[4],
                                  const fpd::DecodeParams& p, int ctas, int smem, cudaStream_t st) {
  if (D == 128)
    return NT == 2 ? launch_split_nvfp4<128, 2, HB, MQ>(maps, p, ctas, smem, st)
                   : launch_split_nvfp4<128, 1, HB, MQ>(maps, p, ctas, smem, st);
  return NT == 2 ? launch_split_nvfp4<64, 2, HB, MQ>(maps, p, ctas, smem, st)
                 : launch_split_nvfp4<64, 1, HB, MQ>(maps, p, ctas, smem, st);
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

#ifndef FPD_SINGLE_SPLIT_STAGES
#define FPD_SINGLE_SPLIT_STAGES 6
#endif

// The split plan for a given stage shape (HB KV heads per stage).
void plan_shape(int B, int q_len, int Hq, int Hkv, int D, int bt, int max_blocks,
                int window_left, int num_sms, int64_t slots, int chunk_pages_override, int HB,
                fpd_plan* plan, bool fp4 = false) {
  const int g = Hq / Hkv;
  const int qp = q_per_item(q_len, g);
  const int q_chunks = (q_len + qp - 1) / qp;
  const int cols = qp * g;   // MMA columns of a work item
  const int NT = n_tiles(cols);
  // with one KV head per stage a stage is 64 tokens of whole pages, and a
  // split must be whole stages; four-head stages are 16 tokens of one page
  const int pps = HB == 1 ? fpd::kTileTokens / bt : 1;
  int pages_max = max_blocks;
  if (window_left >= 0) {   // the q_len queries' windows together span window_left + q_len keys
    const int64_t w = ((int64_t)window_left + q_len - 1) / bt + 2;
    if (w < pages_max) pages_max = (int)w;
  }
  const int64_t units = (int64_t)(B > 0 ? B : 1) * (Hkv / HB) * q_chunks;
  const auto round_pps = [pps](int64_t c) { return (int)((c + pps - 1) / pps * pps); };
  const auto splits_at = [pages_max](int c) { return (int64_t)((pages_max + c - 1) / c); };
  int chunk, adapt = 0;
  int64_t grid_items = 0;   // items the grid is sized for (0: those of `chunk`)
  if (chunk_pages_override > 0) {
    chunk = round_pps(chunk_pages_override);
  } else {
    const int waves = HB == 1 ? kTargetWaves1 : kTargetWaves4;
    const int min_rows = HB == 1 ? kMinChunkRows1 : kMinChunkRows4;
    const auto chunk_for = [&](int w) {
      int64_t splits = (w * slots + units - 1) / units;
      if (splits < 1) splits = 1;
      return round_pps((int)((pages_max + splits - 1) / splits));
    };
    chunk = chunk_for(waves);
    if (HB == 4 && !fp4 && (int64_t)chunk * bt >= kLongItemTokens4) chunk = chunk_for(waves - 1);
    const int min_chunk = round_pps(((int64_t)min_rows / HB + bt - 1) / bt);
    if (chunk < min_chunk) {
      // Too few pages for `waves` rounds of items of the minimum size.  Such
      // calls run best as about two items per SM in one round (measured on
      // uniform batches): items of equal size fill every SM alike.
      chunk = min_chunk;
      const int64_t target = 2 * (int64_t)num_sms;
      const int one_round = round_pps((pages_max + (target + units - 1) / units - 1) /
                                      ((target + units - 1) / units));
      const int floor_chunk = round_pps((kMinItemTokens + bt - 1) / bt);
      const int64_t items_min = units * splits_at(chunk);
      if (items_min <= target) {
        // under-filled: split finer, down to items of a few stages, unless
        // the call needs no split at all (then no combine runs)
        if (splits_at(chunk) > 1) chunk = std::max(one_round, floor_chunk);
      } else if (2 * items_min <= 5 * slots && one_round > chunk) {
        // between one and 2.5 rounds: larger items in one round, taken by
        // the kernel only if the sequences turn out to be of about equal
        // length (it sees the lengths; the plan does not); the grid is
        // sized for those items
        adapt = one_round;
        grid_items = units * splits_at(adapt);
      }
    }
  }
  // A call too small to fill the machine whose longest item is only a few
  // stages runs one split per sequence: no combine launch, and the serial
  // chain of a few stages is shorter than a second kernel (tiny batches).
  if (chunk_pages_override == 0) {
    const int64_t stage_tokens = fpd::kTileTokens / HB;
    const int64_t longest = ((int64_t)pages_max * bt + stage_tokens - 1) / stage_tokens;
    const int64_t splits_now = (pages_max + chunk - 1) / chunk;
    if (longest <= FPD_SINGLE_SPLIT_STAGES && units * splits_now < slots)
      chunk = (pages_max + pps - 1) / pps * pps;
  }
  const int max_splits = (pages_max + chunk - 1) / chunk;
  const int64_t items_max = grid_items > 0 ? grid_items : units * max_splits;
  plan->chunk_pages = chunk;
  plan->adapt_chunk_pages = adapt;
  plan->max_splits = max_splits;
  plan->heads_per_stage = HB;
  plan->stage_tokens = fpd::kTileTokens / HB;
  plan->stages = ring_stages(D, NT, HB, fp4);
  plan->header_slots = header_slots(D, cols, HB);
  plan->ctas = (int)(items_max < slots ? items_max : slots);
  plan->smem_bytes = smem_bytes_for(D, cols, HB, B, fp4);
  // partial results for each of the B * q_len query tokens
  plan->workspace_bytes = ws_layout(B * q_len, Hq, Hkv, D, max_splits).total;
  plan->q_per_item = qp;
  plan->q_chunks = q_chunks;
}

// Validates and plans.  The stage shape is four KV heads per stage whenever
// Hkv allows it, also when the four-head items of a call leave CTA slots idle
// (short windows, few sequences): one-head items of the same keys were slower
// on every such shape measured, since each item pays its set-up and epilogue.
fpd_status plan_for(int B, int q_len, int Hq, int Hkv, int D, int bt, int max_blocks,
                    int window_left, int num_sms, int ctas_per_sm, int chunk_pages_override,
                    fpd_plan* plan, bool fp4 = false) {
  if (!plan) return FPD_ERR_INVALID_ARG;
  fpd_status st = validate_shape(B, Hq, Hkv, D, bt, max_blocks, q_len);
  if (st != FPD_OK) return st;
  if (num_sms <= 0 || ctas_per_sm <= 0 || chunk_pages_override < 0) return FPD_ERR_INVALID_ARG;
  const int64_t slots = (int64_t)num_sms * ctas_per_sm;
  const int HB = heads_per_stage(Hkv);
  plan_shape(B, q_len, Hq, Hkv, D, bt, max_blocks, window_left, num_sms, slots,
             chunk_pages_override, HB, plan, fp4);
  return FPD_OK;
}

// The plan on the current device (its SM count and the split kernel's
// occupancy for the chosen stage shape).
fpd_status plan_device(int B, int q_len, int Hq, int Hkv, int D, int bt, int max_blocks,
                       int window_left, int chunk_pages_override, fpd_plan* plan,
                       bool fp4 = false) {
  if (!plan) return FPD_ERR_INVALID_ARG;
  fpd_status st = validate_shape(B, Hq, Hkv, D, bt, max_blocks, q_len);
  if (st != FPD_OK) return st;
  const int cols = q_per_item(q_len, Hq / Hkv) * (Hq / Hkv);   // MMA columns of a work item
  const int HB = heads_per_stage(Hkv);
  int sms = 0, occ = 0;
  if (!device_occupancy(D, n_tiles(cols), HB, q_len > 1, fp4, smem_bytes_for(D, cols, HB, B, fp4),
                        &sms, &occ))
    return FPD_ERR_CUDA;
  if (occ <= 0) return FPD_ERR_UNSUPPORTED;  // the batch's shared-memory table does not fit
  return plan_for(B, q_len, Hq, Hkv, D, bt, max_blocks, window_left, sms, occ,
                  chunk_pages_override, plan, fp4);
}

}  // namespace

extern "C" {

const char* fp8_paged_decode_status_string(fpd_status s) {
  switch (s) {
    case FPD_OK: return "FPD_OK";
    case FPD_ERR_INVALID_ARG: return "FPD_ERR_INVALID_ARG";
    case FPD_ERR_UNSUPPORTED: return "FPD_ERR_UNSUPPORTED";
    case FPD_ERR_WORKSPACE_TOO_SMALL: return "FPD_ERR_WORKSPACE_TOO_SMALL";
    case FPD_ERR_CUDA: return "FPD_ERR_CUDA";
  }
  return "FPD_UNKNOWN_STATUS";
}

const char* fp8_paged_decode_version(void) { return "0.2.0 sm_100a"; }

fpd_status fp8_paged_decode_make_plan(int B, int Hq, int Hkv, int D, int bt, int max_blocks,
                                      int window_left, int num_sms, int ctas_per_sm,
                                      int chunk_pages_override, fpd_plan* plan) {
  return plan_for(B, 1, Hq, Hkv, D, bt, max_blocks, window_left, num_sms, ctas_per_sm,
                  chunk_pages_override, plan);
}

fpd_status fp8_paged_decode_make_plan_qlen(int B, int q_len, int Hq, int Hkv, int D, int bt,
                                           int max_blocks, int window_left, int num_sms,
                                           int ctas_per_sm, int chunk_pages_override,
                                           fpd_plan* plan) {
  return plan_for(B, q_len, Hq, Hkv, D, bt, max_blocks, window_left, num_sms, ctas_per_sm,
                  chunk_pages_override, plan);
}

fpd_status fp8_paged_decode_plan(int B, int Hq, int Hkv, int D, int bt, int max_blocks,
                                 int window_left, int chunk_pages_override, fpd_plan* plan) {
  return plan_device(B, 1, Hq, Hkv, D, bt, max_blocks, window_left, chunk_pages_override, plan);
}

fpd_status fp8_paged_decode_plan_qlen(int B, int q_len, int Hq, int Hkv, int D, int bt,
                                      int max_blocks, int window_left, int chunk_pages_override,
                                      fpd_plan* plan) {
  return plan_device(B, q_len, Hq, Hkv, D, bt, max_blocks, window_left, chunk_pages_override,
                     plan);
}

size_t fp8_paged_decode_workspace_bytes_qlen(int B, int q_len, int Hq, int Hkv, int D, int bt,
                                             int max_blocks, int window_left,
                                             int chunk_pages_override) {
  fpd_plan plan;
  if (plan_device(B, q_len, Hq, Hkv, D, bt, max_blocks, window_left, chunk_pages_override,
                  &plan) != FPD_OK)
    return 0;
  return plan.workspace_bytes;
}

size_t fp8_paged_decode_workspace_bytes_ex(int B, int Hq, int Hkv, int D, int bt, int max_blocks,
                                           int window_left, int chunk_pages_override) {
  fpd_plan plan;
  if (fp8_paged_decode_plan(B, Hq, Hkv, D, bt, max_blocks, window_left, chunk_pages_override,
                            &plan) != FPD_OK)
    return 0;
  return plan.workspace_bytes;
}

size_t fp8_paged_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int bt, int max_blocks,
                                        int window_left) {
  return fp8_paged_decode_workspace_bytes_ex(B, Hq, Hkv, D, bt, max_blocks, window_left, 0);
}

}  // extern "C"

// The descriptor of a token-major, bf16, contiguous call.
static fpd_decode_args plain_args(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_table, const int32_t* seq_lens, int B, int q_len,
                           int Hq, int Hkv, int D, int num_blocks, int bt, int max_blocks,
                           float k_scale, float v_scale, float sm_scale, int window_left,
                           const float* sinks, void* out, float* lse, int chunk_pages_override) {
  fpd_decode_args a;
  std::memset(&a, 0, sizeof a);
  a.q = q;
  a.q_dtype = FPD_Q_BF16;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.kv_layout = FPD_KV_NHD;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.B = B;
  a.q_len = q_len;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = D;
  a.num_blocks = num_blocks;
  a.block_tokens = bt;
  a.max_blocks = max_blocks;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.sm_scale = sm_scale;
  a.window_left = window_left;
  a.sinks = sinks;
  a.out = out;
  a.lse = lse;
  a.chunk_pages_override = chunk_pages_override;
  return a;
}

// The plan of a descriptor's call: its page format sets the kernel, and an
// f32 output keeps a partial for every row.
static fpd_status plan_args_impl(const fpd_decode_args& a, fpd_plan* plan) {
  if (a.kv_format != FPD_KV_E4M3 && a.kv_format != FPD_KV_NVFP4) return FPD_ERR_INVALID_ARG;
  if (a.out_dtype != FPD_OUT_BF16 && a.out_dtype != FPD_OUT_F32) return FPD_ERR_INVALID_ARG;
  const fpd_status st =
      plan_device(a.B, a.q_len, a.Hq, a.Hkv, a.D, a.block_tokens, a.max_blocks, a.window_left,
                  a.chunk_pages_override, plan, a.kv_format == FPD_KV_NVFP4);
  if (st == FPD_OK && a.out_dtype == FPD_OUT_F32)
    plan->workspace_bytes = ws_layout(a.B * a.q_len, a.Hq, a.Hkv, a.D, plan->max_splits, true).total;
  return st;
}

// zero_header: clear the workspace header (status word, work counters) on the
// stream right before the launches, once every argument has passed the checks
// (the allocation-free entry point's shared scratch).
static fpd_status attention_impl(const fpd_decode_args& a, void* workspace,
                                 size_t workspace_bytes, void* stream, void* ev0, void* ev1,
                                 void* ev2, bool zero_header = false) {
  const int B = a.B, q_len = a.q_len, Hq = a.Hq, Hkv = a.Hkv, D = a.D, bt = a.block_tokens;
  const int max_blocks = a.max_blocks, num_blocks = a.num_blocks, window_left = a.window_left;
  fpd_status st = validate_shape(B, Hq, Hkv, D, bt, max_blocks, q_len);
  if (st != FPD_OK) return st;
  if (num_blocks <= 0 || (int64_t)num_blocks * bt >= INT32_MAX) return FPD_ERR_UNSUPPORTED;
  if (!a.q || !a.k_cache || !a.v_cache || !a.block_table || !a.seq_lens ||
      (!a.out && a.cp_ranks <= 0))
    return FPD_ERR_INVALID_ARG;
  if (a.q_dtype != FPD_Q_BF16 && a.q_dtype != FPD_Q_F16) return FPD_ERR_INVALID_ARG;
  if (a.kv_layout != FPD_KV_NHD && a.kv_layout != FPD_KV_HND) return FPD_ERR_INVALID_ARG;
  if (a.kv_format != FPD_KV_E4M3 && a.kv_format != FPD_KV_NVFP4) return FPD_ERR_INVALID_ARG;
  if (a.out_dtype != FPD_OUT_BF16 && a.out_dtype != FPD_OUT_F32) return FPD_ERR_INVALID_ARG;
  const bool fp4 = a.kv_format == FPD_KV_NVFP4;
  const bool f32_out = a.out_dtype == FPD_OUT_F32;
  const bool cp_pub = a.cp_ranks > 0;
  if (a.cp_ranks < 0) return FPD_ERR_INVALID_ARG;
  if (cp_pub) {   // the fused context-parallel exchange
    if (!f32_out || q_len != 1 || !a.cp_gather || !a.cp_flags || a.cp_rank < 0 ||
        a.cp_rank >= a.cp_ranks || a.cp_epoch == 0 || !aligned(a.cp_gather, 8) ||
        !aligned(a.cp_flags, 8) || a.cp_block_floats % 4 != 0 ||
        a.cp_block_floats < (int64_t)B * Hq * (D + 1) ||
        (a.out_token_stride != 0 && a.out_token_stride != (int64_t)Hq * D))
      return FPD_ERR_INVALID_ARG;
  }
  // NVFP4 pages: head-major, data and scale regions at their own page strides
  const int64_t fp4_data = (int64_t)Hkv * bt * (D / 2), fp4_sf = (int64_t)Hkv * bt * (D / 16);
  const int64_t data_stride = a.kv_page_stride ? a.kv_page_stride : fp4_data;
  const int64_t sf_stride = a.sf_page_stride ? a.sf_page_stride : fp4_sf;
  if (fp4) {
    if (a.kv_layout != FPD_KV_HND) return FPD_ERR_UNSUPPORTED;
    if (!a.k_scales || !a.v_scales || !aligned(a.k_scales, 16) || !aligned(a.v_scales, 16))
      return FPD_ERR_INVALID_ARG;
    if (data_stride < fp4_data || sf_stride < fp4_sf || data_stride % 16 != 0 ||
        sf_stride % 16 != 0)
      return FPD_ERR_INVALID_ARG;
  }
  const int64_t row = (int64_t)Hq * D;
  const int64_t q_stride = a.q_token_stride ? a.q_token_stride : row;
  const int64_t o_stride = a.out_token_stride ? a.out_token_stride : row;
  // 16-byte rows: the query rows are bulk-copied and the outputs stored 16 bytes at a time
  if (q_stride < row || o_stride < row || q_stride % 8 != 0 || o_stride % 8 != 0)
    return FPD_ERR_INVALID_ARG;
  if (!aligned(a.q, 16) || (a.out && !aligned(a.out, 16)) || !aligned(a.k_cache, 16) ||
      !aligned(a.v_cache, 16) || !aligned(a.block_table, 4) || !aligned(a.seq_lens, 4) ||
      (a.lse && !aligned(a.lse, 4)) || (a.sinks && !aligned(a.sinks, 4)) ||
      (a.k_scale_dev && !aligned(a.k_scale_dev, 4)) ||
      (a.v_scale_dev && !aligned(a.v_scale_dev, 4)) || (workspace && !aligned(workspace, 16)))
    return FPD_ERR_INVALID_ARG;
  if (!std::isfinite(a.sm_scale) || !(a.sm_scale > 0.f) ||
      !std::isfinite(a.sm_scale * fpd::kLog2e))
    return FPD_ERR_INVALID_ARG;
  const float qk = a.sm_scale * a.k_scale;
  if (!a.k_scale_dev && (!std::isfinite(a.k_scale) || !(qk > 0.f) ||
                         !std::isfinite(qk * fpd::kLog2e)))
    return FPD_ERR_INVALID_ARG;
  if (!a.v_scale_dev && !std::isfinite(a.v_scale)) return FPD_ERR_INVALID_ARG;
  if (a.chunk_pages_override < 0) return FPD_ERR_INVALID_ARG;
  if (B == 0) return FPD_OK;

  const int g = Hq / Hkv;
  fpd_plan plan;
  st = plan_args_impl(a, &plan);
  if (st != FPD_OK) return st;
  if (!workspace || workspace_bytes < plan.workspace_bytes) return FPD_ERR_WORKSPACE_TOO_SMALL;

  const bool hnd = a.kv_layout == FPD_KV_HND;
  CUtensorMap km, vm, maps4[4];
  if (fp4) {   // K data, K scales, V data, V scales
    const int HBp = plan.heads_per_stage;
    if (!encode_nvfp4_map(&maps4[0], a.k_cache, num_blocks, bt, Hkv, D, HBp, data_stride, false) ||
        !encode_nvfp4_map(&maps4[1], a.k_scales, num_blocks, bt, Hkv, D, HBp, sf_stride, true) ||
        !encode_nvfp4_map(&maps4[2], a.v_cache, num_blocks, bt, Hkv, D, HBp, data_stride, false) ||
        !encode_nvfp4_map(&maps4[3], a.v_scales, num_blocks, bt, Hkv, D, HBp, sf_stride, true))
      return FPD_ERR_CUDA;
  } else if (!encode_cache_map(&km, a.k_cache, num_blocks, bt, Hkv, D, plan.heads_per_stage,
                               hnd) ||
             !encode_cache_map(&vm, a.v_cache, num_blocks, bt, Hkv, D, plan.heads_per_stage,
                               hnd)) {
    return FPD_ERR_CUDA;
  }

  const WsLayout wl = ws_layout(B * q_len, Hq, Hkv, D, plan.max_splits, f32_out);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  fpd::DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.block_table = a.block_table;
  p.seq_lens = a.seq_lens;
  p.sinks = a.sinks;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.part_o = reinterpret_cast<float*>(ws + wl.part_o);
  p.part_lse = reinterpret_cast<float*>(ws + wl.part_lse);
  p.status = reinterpret_cast<uint32_t*>(ws);
  p.sched = reinterpret_cast<uint32_t*>(ws) + 1;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.g = g;
  p.bt = bt;
  p.max_blocks = max_blocks;
  p.num_blocks = num_blocks;
  p.window_left = window_left;
  p.chunk_pages = plan.chunk_pages;
  p.max_splits = plan.max_splits;
  p.stages = plan.stages;
  p.hdr_slots = plan.header_slots;
  p.q_len = q_len;
  p.q_per_item = plan.q_per_item;
  p.q_chunks = plan.q_chunks;
  p.lg = __builtin_ctz((unsigned)g);
  p.qk_scale_log2 = qk * fpd::kLog2e;
  p.v_scale = a.v_scale;
  p.q_tok_stride = q_stride;
  p.out_tok_stride = o_stride;
  p.k_scale_dev = a.k_scale_dev;
  p.v_scale_dev = a.v_scale_dev;
  p.sm_scale_log2 = a.sm_scale * fpd::kLog2e;
  p.q_f16 = a.q_dtype == FPD_Q_F16;
  p.kv_hnd = hnd;
  p.combine_all = f32_out;
  p.adapt_chunk = plan.adapt_chunk_pages;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (zero_header && cudaMemsetAsync(workspace, 0, wl.zero_prefix, s) != cudaSuccess)
    return FPD_ERR_CUDA;
  if (ev0 && cudaEventRecord(static_cast<cudaEvent_t>(ev0), s) != cudaSuccess) return FPD_ERR_CUDA;
  cudaError_t e;
  const int NT = n_tiles(plan.q_per_item * g);
  const bool mq = q_len > 1;
  const int ctas = plan.ctas, smem = plan.smem_bytes;
  if (fp4 && plan.heads_per_stage == 4)
    e = mq ? launch_split_nvfp4_hb<4, true>(D, NT, maps4, p, ctas, smem, s)
           : launch_split_nvfp4_hb<4, false>(D, NT, maps4, p, ctas, smem, s);
  else if (fp4)
    e = mq ? launch_split_nvfp4_hb<1, true>(D, NT, maps4, p, ctas, smem, s)
           : launch_split_nvfp4_hb<1, false>(D, NT, maps4, p, ctas, smem, s);
  else if (plan.heads_per_stage == 4)
    e = mq ? launch_split_hb<4, true>(D, NT, km, vm, p, ctas, smem, s)
           : launch_split_hb<4, false>(D, NT, km, vm, p, ctas, smem, s);
  else
    e = mq ? launch_split_hb<1, true>(D, NT, km, vm, p, ctas, smem, s)
           : launch_split_hb<1, false>(D, NT, km, vm, p, ctas, smem, s);
  if (e != cudaSuccess) return FPD_ERR_CUDA;
  if (ev1 && cudaEventRecord(static_cast<cudaEvent_t>(ev1), s) != cudaSuccess) return FPD_ERR_CUDA;
  if (plan.max_splits > 1 || f32_out) {
    fpd::CombineParams c;
    c.seq_lens = a.seq_lens;
    c.sinks = a.sinks;
    c.part_o = p.part_o;
    c.part_lse = p.part_lse;
    c.out = p.out;
    c.out_f32 = f32_out && !cp_pub ? static_cast<float*>(a.out) : nullptr;
    c.cp_ranks = cp_pub ? a.cp_ranks : 0;
    c.cp_rank = a.cp_rank;
    c.cp_gather = a.cp_gather;
    c.cp_flags = a.cp_flags;
    c.cp_done = reinterpret_cast<uint32_t*>(ws) + 4;
    c.cp_block = a.cp_block_floats;
    c.cp_rows = (int64_t)B * Hq;
    c.cp_epoch = a.cp_epoch;
    c.lse = a.lse;
    c.B = B;
    c.q_len = q_len;
    c.Hq = Hq;
    c.bt = bt;
    c.max_blocks = max_blocks;
    c.window_left = window_left;
    c.chunk_word = p.sched + 2;
    c.max_splits = plan.max_splits;
    // enough warps per row that none merges more than one batch of partials
    // (up to 32 warps), and 8 warps per CTA at least
    c.wpr = 1;
    while (c.wpr < 32 && c.wpr * fpd::kCombineBatch < plan.max_splits) c.wpr *= 2;
    c.rows_per_cta = c.wpr >= 8 ? 1 : 8 / c.wpr;
    c.v_scale = a.v_scale;
    c.v_scale_dev = a.v_scale_dev;
    c.out_tok_stride = o_stride;
    if (mq)
      e = D == 128 ? launch_combine<128, true>(c, s) : launch_combine<64, true>(c, s);
    else
      e = D == 128 ? launch_combine<128, false>(c, s) : launch_combine<64, false>(c, s);
    if (e != cudaSuccess) return FPD_ERR_CUDA;
  }
  if (ev2 && cudaEventRecord(static_cast<cudaEvent_t>(ev2), s) != cudaSuccess) return FPD_ERR_CUDA;
  return FPD_OK;
}

extern "C" {

fpd_status fp8_paged_decode_attention_ex(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_table, const int32_t* seq_lens,
                                         int B, int Hq, int Hkv, int D, int num_blocks, int bt,
                                         int max_blocks, float k_scale, float v_scale,
                                         float sm_scale, int window_left, const float* sinks,
                                         void* out, float* lse, void* workspace,
                                         size_t workspace_bytes, void* stream,
                                         int chunk_pages_override) {
  return attention_impl(plain_args(q, k_cache, v_cache, block_table, seq_lens, B, 1, Hq, Hkv, D,
                                   num_blocks, bt, max_blocks, k_scale, v_scale, sm_scale,
                                   window_left, sinks, out, lse, chunk_pages_override),
                        workspace, workspace_bytes, stream, nullptr, nullptr, nullptr);
}

fpd_status fp8_paged_decode_attention_qlen(const void* q, const void* k_cache,
                                           const void* v_cache, const int32_t* block_table,
                                           const int32_t* seq_lens, int B, int q_len, int Hq,
                                           int Hkv, int D, int num_blocks, int bt, int max_blocks,
                                           float k_scale, float v_scale, float sm_scale,
                                           int window_left, const float* sinks, void* out,
                                           float* lse, void* workspace, size_t workspace_bytes,
                                           void* stream, int chunk_pages_override) {
  return attention_impl(plain_args(q, k_cache, v_cache, block_table, seq_lens, B, q_len, Hq,
                                   Hkv, D, num_blocks, bt, max_blocks, k_scale, v_scale, sm_scale,
                                   window_left, sinks, out, lse, chunk_pages_override),
                        workspace, workspace_bytes, stream, nullptr, nullptr, nullptr);
}

fpd_status fp8_paged_decode_attention_args(const fpd_decode_args* args, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  if (!args) return FPD_ERR_INVALID_ARG;
  return attention_impl(*args, workspace, workspace_bytes, stream, nullptr, nullptr, nullptr);
}

fpd_status fp8_paged_decode_attention_args_profiled(const fpd_decode_args* args, void* workspace,
                                                    size_t workspace_bytes, void* stream,
                                                    void* event_before_split,
                                                    void* event_after_split,
                                                    void* event_after_combine) {
  if (!args) return FPD_ERR_INVALID_ARG;
  return attention_impl(*args, workspace, workspace_bytes, stream, event_before_split,
                        event_after_split, event_after_combine);
}

fpd_status fp8_paged_decode_plan_args(const fpd_decode_args* args, fpd_plan* plan) {
  if (!args || !plan) return FPD_ERR_INVALID_ARG;
  return plan_args_impl(*args, plan);
}

size_t fp8_paged_decode_workspace_bytes_args(const fpd_decode_args* args) {
  fpd_plan plan;
  if (fp8_paged_decode_plan_args(args, &plan) != FPD_OK) return 0;
  return plan.workspace_bytes;
}

fpd_status fp8_paged_decode_attention_profiled(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
    const int32_t* seq_lens, int B, int q_len, int Hq, int Hkv, int D, int num_blocks, int bt,
    int max_blocks, float k_scale, float v_scale, float sm_scale, int window_left,
    const float* sinks, void* out, float* lse, void* workspace, size_t workspace_bytes,
    void* stream, int chunk_pages_override, void* event_before_split, void* event_after_split,
    void* event_after_combine) {
  return attention_impl(plain_args(q, k_cache, v_cache, block_table, seq_lens, B, q_len, Hq,
                                   Hkv, D, num_blocks, bt, max_blocks, k_scale, v_scale, sm_scale,
                                   window_left, sinks, out, lse, chunk_pages_override),
                        workspace, workspace_bytes, stream, event_before_split,
                        event_after_split, event_after_combine);
}

fpd_status fp8_paged_decode_attention(const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_table, const int32_t* seq_lens, int B,
                                      int Hq, int Hkv, int D, int num_blocks, int bt,
                                      int max_blocks, float k_scale, float v_scale, float sm_scale,
                                      int window_left, const float* sinks, void* out, float* lse,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  return fp8_paged_decode_attention_ex(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, D,
                                       num_blocks, bt, max_blocks, k_scale, v_scale, sm_scale,
                                       window_left, sinks, out, lse, workspace, workspace_bytes,
                                       stream, 0);
}

}  // extern "C"

namespace {

// Scratch for fp8_paged_decode_attention_noalloc: split partials, work
// counters and status word for callers that cannot allocate.  In host code this name is only
// a stand-in; the device address comes from cudaGetSymbolAddress per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FPD_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per
// device, with that device current).  nullptr on failure.
void* noalloc_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return nullptr;
    }
    g_noalloc_addr[dev] = ptr;
  }
  return g_noalloc_addr[dev];
}

}  // namespace

extern "C" {

fpd_status fp8_paged_decode_attention_noalloc(const void* q, const void* k_cache,
                                              const void* v_cache, const int32_t* block_table,
                                              const int32_t* seq_lens, int B, int Hq, int Hkv,
                                              int D, int num_blocks, int bt, int max_blocks,
                                              float k_scale, float v_scale, float sm_scale,
                                              int window_left, const float* sinks, void* out,
                                              float* lse, void* stream) {
  fpd_status st = validate_shape(B, Hq, Hkv, D, bt, max_blocks);
  if (st != FPD_OK) return st;
  if (B == 0) return FPD_OK;
  fpd_plan plan;
  st = fp8_paged_decode_plan(B, Hq, Hkv, D, bt, max_blocks, window_left, 0, &plan);
  if (st != FPD_OK) return st;
  if (plan.workspace_bytes > FPD_NOALLOC_SCRATCH_BYTES) return FPD_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = noalloc_scratch_address();
  if (!scratch) return FPD_ERR_CUDA;
  // The status word and the work counters must start at zero (the partials
  // are fully rewritten): the header is cleared on the stream after every
  // argument check has passed, so a rejected call enqueues nothing.
  return attention_impl(plain_args(q, k_cache, v_cache, block_table, seq_lens, B, 1, Hq, Hkv, D,
                                   num_blocks, bt, max_blocks, k_scale, v_scale, sm_scale,
                                   window_left, sinks, out, lse, 0),
                        scratch, FPD_NOALLOC_SCRATCH_BYTES, stream, nullptr, nullptr, nullptr,
                        true);
}

fpd_status fp8_paged_decode_cache_write_layout(const void* key, const void* value,
                                               const int64_t* slot_mapping, int num_tokens,
                                               int Hkv, int D, int64_t key_stride,
                                               int64_t value_stride, float k_scale,
                                               float v_scale, void* k_cache, void* v_cache,
                                               int num_blocks, int block_tokens, int kv_layout,
                                               uint32_t* status, void* stream) {
  if (num_tokens < 0 || Hkv <= 0 || D <= 0 || D % 16 != 0 || num_blocks <= 0 ||
      block_tokens <= 0)
    return FPD_ERR_INVALID_ARG;
  if (kv_layout != FPD_KV_NHD && kv_layout != FPD_KV_HND) return FPD_ERR_INVALID_ARG;
  if (kv_layout == FPD_KV_HND && (int64_t)num_blocks * block_tokens >= INT32_MAX)
    return FPD_ERR_UNSUPPORTED;
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
    return FPD_ERR_INVALID_ARG;
  if (num_tokens == 0) return FPD_OK;
  if (!key || !value || !slot_mapping || !k_cache || !v_cache) return FPD_ERR_INVALID_ARG;
  const int64_t row = (int64_t)Hkv * D;
  if (key_stride < row || value_stride < row || key_stride % 8 != 0 || value_stride % 8 != 0)
    return FPD_ERR_INVALID_ARG;
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8) || (status && !aligned(status, 4)))
    return FPD_ERR_INVALID_ARG;
  if (row / fpd::kWriteElems > INT32_MAX) return FPD_ERR_UNSUPPORTED;
  fpd::CacheWriteParams p;
  p.key = static_cast<const __nv_bfloat16*>(key);
  p.value = static_cast<const __nv_bfloat16*>(value);
  p.slot_mapping = slot_mapping;
  p.k_cache = static_cast<uint8_t*>(k_cache);
  p.v_cache = static_cast<uint8_t*>(v_cache);
  p.status = status;
  p.key_stride = key_stride;
  p.value_stride = value_stride;
  p.n_slots = (int64_t)num_blocks * block_tokens;
  p.num_tokens = num_tokens;
  p.row_chunks = (int)(row / fpd::kWriteElems);
  p.k_inv = 1.0f / k_scale;   // fp32 reciprocal, as the reference writer takes it
  p.v_inv = 1.0f / v_scale;
  p.hnd = kv_layout == FPD_KV_HND;
  p.bt = block_tokens;
  p.head_chunks = D / fpd::kWriteElems;
  int sms = 0;
  if (!device_sm_count(&sms)) return FPD_ERR_CUDA;
  const int64_t units = (int64_t)num_tokens * 2 * p.row_chunks;
  const int64_t want = (units + fpd::kWriteThreads - 1) / fpd::kWriteThreads;
  const int64_t cap = (int64_t)sms * 8;   // 8 CTAs of 256 threads fill an SM
  const int grid = (int)(want < cap ? want : cap);
  fpd::fpd_cache_write_kernel<<<grid, fpd::kWriteThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      p);
  return cudaGetLastError() == cudaSuccess ? FPD_OK : FPD_ERR_CUDA;
}

static fpd_status cp_merge_impl(const float* partials, int R, int64_t block_floats, int64_t rows,
                                int Hq, int D, const float* sinks, void* out,
                                int64_t out_token_stride, float* lse, const uint32_t* flags,
                                uint32_t epoch, uint64_t timeout_ns, uint32_t* status,
                                void* stream) {
  if (R < 1 || Hq < 1 || rows < 0 || rows % Hq != 0) return FPD_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FPD_ERR_UNSUPPORTED;
  if (block_floats < rows * (D + 1) || block_floats % 4 != 0) return FPD_ERR_INVALID_ARG;
  const int64_t o_stride = out_token_stride ? out_token_stride : (int64_t)Hq * D;
  if (o_stride < (int64_t)Hq * D || o_stride % 8 != 0) return FPD_ERR_INVALID_ARG;
  if (!partials || !out || !aligned(partials, 16) || !aligned(out, 16) ||
      (lse && !aligned(lse, 4)) || (sinks && !aligned(sinks, 4)) ||
      (flags && !aligned(flags, 4)) || (status && !aligned(status, 4)))
    return FPD_ERR_INVALID_ARG;
  if (rows == 0) return FPD_OK;
  const int64_t grid = (rows + fpd::kCpMergeWarps - 1) / fpd::kCpMergeWarps;
  if (grid > INT32_MAX) return FPD_ERR_UNSUPPORTED;
  fpd::CpMergeParams p;
  p.partials = partials;
  p.sinks = sinks;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.block = block_floats;
  p.rows = rows;
  p.out_tok_stride = o_stride;
  p.R = R;
  p.Hq = Hq;
  p.flags = flags;
  p.epoch = epoch;
  p.timeout_ns = timeout_ns;
  p.status = status;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dim3 g((unsigned)grid), b(fpd::kCpMergeWarps * 32);
  if (flags) {
    if (D == 128) fpd::fpd_cp_merge_kernel<128, true><<<g, b, 0, s>>>(p);
    else fpd::fpd_cp_merge_kernel<64, true><<<g, b, 0, s>>>(p);
  } else {
    if (D == 128) fpd::fpd_cp_merge_kernel<128, false><<<g, b, 0, s>>>(p);
    else fpd::fpd_cp_merge_kernel<64, false><<<g, b, 0, s>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? FPD_OK : FPD_ERR_CUDA;
}

fpd_status fp8_paged_decode_cp_merge(const float* partials, int R, int64_t block_floats,
                                     int64_t rows, int Hq, int D, const float* sinks, void* out,
                                     int64_t out_token_stride, float* lse, void* stream) {
  return cp_merge_impl(partials, R, block_floats, rows, Hq, D, sinks, out, out_token_stride, lse,
                       nullptr, 0, 0, nullptr, stream);
}

fpd_status fp8_paged_decode_cp_merge_wait(const float* gather, int R, int64_t block_floats,
                                          int64_t rows, int Hq, int D, const float* sinks,
                                          void* out, int64_t out_token_stride, float* lse,
                                          const uint32_t* flags, uint32_t epoch,
                                          uint64_t timeout_ns, uint32_t* status, void* stream) {
  if (!flags || epoch == 0 || timeout_ns == 0) return FPD_ERR_INVALID_ARG;
  return cp_merge_impl(gather, R, block_floats, rows, Hq, D, sinks, out, out_token_stride, lse,
                       flags, epoch, timeout_ns, status, stream);
}

fpd_status fp8_paged_decode_cache_write_nvfp4(const void* key, const void* value,
                                              const int64_t* slot_mapping, int num_tokens,
                                              int Hkv, int D, int64_t key_stride,
                                              int64_t value_stride, float k_scale, float v_scale,
                                              void* k_data, void* k_sf, void* v_data, void* v_sf,
                                              int64_t data_page_stride, int64_t sf_page_stride,
                                              int num_blocks, int block_tokens, uint32_t* status,
                                              void* stream) {
  if (num_tokens < 0 || Hkv <= 0 || D <= 0 || D % 16 != 0 || num_blocks <= 0 ||
      block_tokens <= 0)
    return FPD_ERR_INVALID_ARG;
  if ((int64_t)num_blocks * block_tokens >= INT32_MAX) return FPD_ERR_UNSUPPORTED;
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
    return FPD_ERR_INVALID_ARG;
  if (num_tokens == 0) return FPD_OK;
  if (!key || !value || !slot_mapping || !k_data || !k_sf || !v_data || !v_sf)
    return FPD_ERR_INVALID_ARG;
  const int64_t row = (int64_t)Hkv * D;
  const int64_t data_b = (int64_t)Hkv * block_tokens * (D / 2);
  const int64_t sf_b = (int64_t)Hkv * block_tokens * (D / 16);
  const int64_t ds = data_page_stride ? data_page_stride : data_b;
  const int64_t ss = sf_page_stride ? sf_page_stride : sf_b;
  if (key_stride < row || value_stride < row || key_stride % 8 != 0 || value_stride % 8 != 0 ||
      ds < data_b || ss < sf_b || ds % 16 != 0 || ss % 16 != 0)
    return FPD_ERR_INVALID_ARG;
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_data, 16) || !aligned(k_sf, 16) ||
      !aligned(v_data, 16) || !aligned(v_sf, 16) || !aligned(slot_mapping, 8) ||
      (status && !aligned(status, 4)))
    return FPD_ERR_INVALID_ARG;
  if (row / 16 > INT32_MAX) return FPD_ERR_UNSUPPORTED;
  fpd::CacheWriteFp4Params p;
  p.key = static_cast<const __nv_bfloat16*>(key);
  p.value = static_cast<const __nv_bfloat16*>(value);
  p.slot_mapping = slot_mapping;
  p.k_data = static_cast<uint8_t*>(k_data);
  p.k_sf = static_cast<uint8_t*>(k_sf);
  p.v_data = static_cast<uint8_t*>(v_data);
  p.v_sf = static_cast<uint8_t*>(v_sf);
  p.status = status;
  p.key_stride = key_stride;
  p.value_stride = value_stride;
  p.data_page_stride = ds;
  p.sf_page_stride = ss;
  p.n_slots = (int64_t)num_blocks * block_tokens;
  p.num_tokens = num_tokens;
  p.D = D;
  p.bt = block_tokens;
  p.blocks = (int)(row / 16);
  p.k_gs = 1.0f / k_scale;   // the per-tensor "global" scale, fp32
  p.v_gs = 1.0f / v_scale;
  p.k_rgs = 1.0f / p.k_gs;
  p.v_rgs = 1.0f / p.v_gs;
  int sms = 0;
  if (!device_sm_count(&sms)) return FPD_ERR_CUDA;
  const int64_t units = (int64_t)num_tokens * 2 * p.blocks;
  const int64_t want = (units + fpd::kWriteThreads - 1) / fpd::kWriteThreads;
  const int64_t cap = (int64_t)sms * 8;
  const int grid = (int)(want < cap ? want : cap);
  fpd::fpd_cache_write_nvfp4_kernel<<<grid, fpd::kWriteThreads, 0,
                                      static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? FPD_OK : FPD_ERR_CUDA;
}

fpd_status fp8_paged_decode_cache_write(const void* key, const void* value,
                                        const int64_t* slot_mapping, int num_tokens, int Hkv,
                                        int D, int64_t key_stride, int64_t value_stride,
                                        float k_scale, float v_scale, void* k_cache,
                                        void* v_cache, int num_blocks, int block_tokens,
                                        uint32_t* status, void* stream) {
  return fp8_paged_decode_cache_write_layout(key, value, slot_mapping, num_tokens, Hkv, D,
                                             key_stride, value_stride, k_scale, v_scale, k_cache,
                                             v_cache, num_blocks, block_tokens, FPD_KV_NHD,
                                             status, stream);
}

fpd_status fp8_paged_decode_check_status(void* workspace, void* stream, int* device_error_bits,
                                         int clear) {
  if (!workspace || !device_error_bits) return FPD_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t bits = 0;
  if (cudaMemcpyAsync(&bits, workspace, sizeof(bits), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return FPD_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FPD_ERR_CUDA;
  *device_error_bits = (int)bits;
  if (clear) {
    if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s) != cudaSuccess) return FPD_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return FPD_ERR_CUDA;
  }
  return FPD_OK;
}

fpd_status fp8_paged_decode_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < kHeaderBytes) return FPD_ERR_INVALID_ARG;
  if (cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return FPD_ERR_CUDA;
  return FPD_OK;
}

}  // extern "C"
