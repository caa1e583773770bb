// fpd_api.cu -- host side of the C ABI declared in include/fp8_paged_decode.h:
// argument validation, the split planner, TMA descriptor encoding and the two
// kernel launches.  No call allocates or frees device memory, and only
// fp8_paged_decode_check_status synchronises.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fp8_paged_decode.h"
#include "fpd_kernels.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kHeaderBytes = 256;    // status word + padding
constexpr int kTargetWaves = 8;         // CTAs launched ~ this many waves of resident slots
constexpr int kMinChunkTokens = 256;    // shortest KV range worth a CTA of its own
constexpr int kRingBytesTarget = 96 * 1024;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool supported_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8 || g == 16; }

fpd_status validate_shape(int B, int Hq, int Hkv, int D, int bt, int max_blocks) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bt <= 0 || max_blocks <= 0)
    return FPD_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FPD_ERR_INVALID_ARG;
  if (!supported_group(Hq / Hkv)) return FPD_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return FPD_ERR_UNSUPPORTED;
  if (bt != 16 && bt != 32 && bt != 64) return FPD_ERR_UNSUPPORTED;
  if ((int64_t)max_blocks * bt > INT32_MAX) return FPD_ERR_UNSUPPORTED;
  return FPD_OK;
}

int ring_stages(int D) {
  const int stage_bytes = 2 * fpd::kTileTokens * D;
  int s = kRingBytesTarget / stage_bytes;
  return s < 2 ? 2 : (s > 8 ? 8 : s);
}

int smem_bytes_for(int D, int g, int stages) {
  const int NT = g > 8 ? 2 : 1;
  int ring = stages * 2 * fpd::kTileTokens * D;
  const int merge = fpd::kConsumerWarps * NT * 8 * D * 4 + fpd::kConsumerWarps * NT * 8 * 2 * 4;
  if (ring < merge) ring = merge;
  return ring + 2 * stages * 8 + 1024;  // barriers + slack for 1024-byte alignment
}

// ---- per-device facts, queried once
struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int occ[2][2] = {{0, 0}, {0, 0}};  // [D==128][NT==2] CTAs per SM
};
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

template <int D, int NT>
const void* split_kernel_ptr() {
  return reinterpret_cast<const void*>(&fpd::fpd_split_kernel<D, NT>);
}

const void* split_kernel_for(int D, int NT) {
  if (D == 128) return NT == 2 ? split_kernel_ptr<128, 2>() : split_kernel_ptr<128, 1>();
  return NT == 2 ? split_kernel_ptr<64, 2>() : split_kernel_ptr<64, 1>();
}

bool device_info(int dev, DeviceInfo* out) {
  if (dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    di.num_sms = sms;
    for (int dsel = 0; dsel < 2; ++dsel) {
      for (int nsel = 0; nsel < 2; ++nsel) {
        const int D = dsel ? 128 : 64, NT = nsel ? 2 : 1;
        const void* fn = split_kernel_for(D, NT);
        const int smem = smem_bytes_for(D, NT == 2 ? 16 : 8, ring_stages(D));
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
          return false;
        int occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, fpd::kThreads, smem) !=
            cudaSuccess)
          return false;
        di.occ[dsel][nsel] = occ > 0 ? occ : 1;
      }
    }
    di.ready = true;
  }
  *out = di;
  return true;
}

bool current_device_info(DeviceInfo* out, int* dev_out = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (dev_out) *dev_out = dev;
  if (!device_info(dev, out)) {
    cudaGetLastError();
    return false;
  }
  return true;
}

int ctas_per_sm_for(const DeviceInfo& di, int D, int g) {
  return di.occ[D == 128 ? 1 : 0][g > 8 ? 1 : 0];
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

// View a [num_blocks, bt, Hkv, D] byte cache as the 3-D tensor
// (d, kv head, token row) with box (D, 1, bt): one box = one page of one head.
bool encode_cache_map(CUtensorMap* map, const void* base, int num_blocks, int bt, int Hkv, int D) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)num_blocks * bt};
  cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)Hkv * D};
  cuuint32_t box[3] = {(cuuint32_t)D, 1u, (cuuint32_t)bt};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapSwizzle swz =
      D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int NT>
cudaError_t launch_split(const CUtensorMap& km, const CUtensorMap& vm, const fpd::DecodeParams& p,
                         int ctas, int smem, cudaStream_t st) {
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < kMaxDevices && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(&fpd::fpd_split_kernel<D, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  fpd::fpd_split_kernel<D, NT><<<ctas, fpd::kThreads, smem, st>>>(km, vm, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_combine(const fpd::CombineParams& c, cudaStream_t st) {
  const int rows = c.B * c.Hq;
  const int blocks = (rows + 7) / 8;
  fpd::fpd_combine_kernel<D><<<blocks, 256, 0, st>>>(c);
  return cudaGetLastError();
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

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

const char* fp8_paged_decode_version(void) { return "0.1.0 sm_100a"; }

fpd_status fp8_paged_decode_make_plan(int B, int Hq, int Hkv, int D, int bt, int max_blocks,
                                      int window_left, int num_sms, int ctas_per_sm,
                                      int chunk_pages_override, fpd_plan* plan) {
  if (!plan) return FPD_ERR_INVALID_ARG;
  fpd_status st = validate_shape(B, Hq, Hkv, D, bt, max_blocks);
  if (st != FPD_OK) return st;
  if (num_sms <= 0 || ctas_per_sm <= 0 || chunk_pages_override < 0) return FPD_ERR_INVALID_ARG;
  const int g = Hq / Hkv;
  const int pps = fpd::kTileTokens / bt;
  int pages_max = max_blocks;
  if (window_left >= 0) {
    const int64_t w = (int64_t)window_left / bt + 2;
    if (w < pages_max) pages_max = (int)w;
  }
  int chunk;
  if (chunk_pages_override > 0) {
    chunk = chunk_pages_override;
  } else {
    const int64_t units = (int64_t)(B > 0 ? B : 1) * Hkv;
    const int64_t slots = (int64_t)num_sms * ctas_per_sm;
    int64_t splits = (kTargetWaves * slots + units - 1) / units;
    if (splits < 1) splits = 1;
    chunk = (int)((pages_max + splits - 1) / splits);
    const int min_chunk = (kMinChunkTokens + bt - 1) / bt;
    if (chunk < min_chunk) chunk = min_chunk;
  }
  chunk = (chunk + pps - 1) / pps * pps;
  const int max_splits = (pages_max + chunk - 1) / chunk;
  const int stages = ring_stages(D);
  plan->chunk_pages = chunk;
  plan->max_splits = max_splits;
  plan->pages_per_stage = pps;
  plan->stages = stages;
  plan->ctas = (int)((int64_t)B * Hkv * max_splits);
  plan->smem_bytes = smem_bytes_for(D, g, stages);
  size_t ws = kHeaderBytes;
  if (max_splits > 1) {
    ws += align_up((size_t)B * Hq * max_splits * D * sizeof(float), 256);
    ws += align_up((size_t)B * Hq * max_splits * sizeof(float), 256);
  }
  plan->workspace_bytes = ws;
  return FPD_OK;
}

fpd_status fp8_paged_decode_plan(int B, int Hq, int Hkv, int D, int bt, int max_blocks,
                                 int window_left, int chunk_pages_override, fpd_plan* plan) {
  if (!plan) return FPD_ERR_INVALID_ARG;
  fpd_status st = validate_shape(B, Hq, Hkv, D, bt, max_blocks);
  if (st != FPD_OK) return st;
  DeviceInfo di;
  if (!current_device_info(&di)) return FPD_ERR_CUDA;
  return fp8_paged_decode_make_plan(B, Hq, Hkv, D, bt, max_blocks, window_left, di.num_sms,
                                    ctas_per_sm_for(di, D, Hq / Hkv), chunk_pages_override, plan);
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

static fpd_status attention_impl(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* block_table, const int32_t* seq_lens, int B,
                                 int Hq, int Hkv, int D, int num_blocks, int bt, int max_blocks,
                                 float k_scale, float v_scale, float sm_scale, int window_left,
                                 const float* sinks, void* out, float* lse, void* workspace,
                                 size_t workspace_bytes, void* stream, int chunk_pages_override,
                                 void* ev0, void* ev1, void* ev2) {
  fpd_status st = validate_shape(B, Hq, Hkv, D, bt, max_blocks);
  if (st != FPD_OK) return st;
  if (num_blocks <= 0 || (int64_t)num_blocks * bt >= INT32_MAX) return FPD_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !out) return FPD_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_table, 4) || !aligned(seq_lens, 4) || (lse && !aligned(lse, 4)) ||
      (sinks && !aligned(sinks, 4)) || (workspace && !aligned(workspace, 16)))
    return FPD_ERR_INVALID_ARG;
  if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || !std::isfinite(sm_scale))
    return FPD_ERR_INVALID_ARG;
  const float qk = sm_scale * k_scale;
  if (!(qk > 0.f) || !std::isfinite(qk * fpd::kLog2e)) return FPD_ERR_INVALID_ARG;
  if (chunk_pages_override < 0) return FPD_ERR_INVALID_ARG;
  if (B == 0) return FPD_OK;

  const int g = Hq / Hkv;
  fpd_plan plan;
  st = fp8_paged_decode_plan(B, Hq, Hkv, D, bt, max_blocks, window_left, chunk_pages_override,
                             &plan);
  if (st != FPD_OK) return st;
  if (!workspace || workspace_bytes < plan.workspace_bytes) return FPD_ERR_WORKSPACE_TOO_SMALL;

  CUtensorMap km, vm;
  if (!encode_cache_map(&km, k_cache, num_blocks, bt, Hkv, D) ||
      !encode_cache_map(&vm, v_cache, num_blocks, bt, Hkv, D))
    return FPD_ERR_CUDA;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part_o = reinterpret_cast<float*>(ws + kHeaderBytes);
  float* part_lse = reinterpret_cast<float*>(
      ws + kHeaderBytes + align_up((size_t)B * Hq * plan.max_splits * D * sizeof(float), 256));

  fpd::DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.sinks = sinks;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.status = reinterpret_cast<uint32_t*>(ws);
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
  p.pages_per_stage = plan.pages_per_stage;
  p.stages = plan.stages;
  p.qk_scale_log2 = qk * fpd::kLog2e;
  p.v_scale = v_scale;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (ev0 && cudaEventRecord(static_cast<cudaEvent_t>(ev0), s) != cudaSuccess) return FPD_ERR_CUDA;
  const int NT = g > 8 ? 2 : 1;
  if (D == 128)
    e = NT == 2 ? launch_split<128, 2>(km, vm, p, plan.ctas, plan.smem_bytes, s)
                : launch_split<128, 1>(km, vm, p, plan.ctas, plan.smem_bytes, s);
  else
    e = NT == 2 ? launch_split<64, 2>(km, vm, p, plan.ctas, plan.smem_bytes, s)
                : launch_split<64, 1>(km, vm, p, plan.ctas, plan.smem_bytes, s);
  if (e != cudaSuccess) return FPD_ERR_CUDA;
  if (ev1 && cudaEventRecord(static_cast<cudaEvent_t>(ev1), s) != cudaSuccess) return FPD_ERR_CUDA;

  if (plan.max_splits > 1) {
    fpd::CombineParams c;
    c.seq_lens = seq_lens;
    c.sinks = sinks;
    c.part_o = part_o;
    c.part_lse = part_lse;
    c.out = static_cast<__nv_bfloat16*>(out);
    c.lse = lse;
    c.B = B;
    c.Hq = Hq;
    c.bt = bt;
    c.max_blocks = max_blocks;
    c.window_left = window_left;
    c.chunk_pages = plan.chunk_pages;
    c.max_splits = plan.max_splits;
    c.v_scale = v_scale;
    e = D == 128 ? launch_combine<128>(c, s) : launch_combine<64>(c, s);
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
  return attention_impl(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, D, num_blocks, bt,
                        max_blocks, k_scale, v_scale, sm_scale, window_left, sinks, out, lse,
                        workspace, workspace_bytes, stream, chunk_pages_override, nullptr,
                        nullptr, nullptr);
}

fpd_status fp8_paged_decode_attention_profiled(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
    const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int num_blocks, int bt,
    int max_blocks, float k_scale, float v_scale, float sm_scale, int window_left,
    const float* sinks, void* out, float* lse, void* workspace, size_t workspace_bytes,
    void* stream, int chunk_pages_override, void* event_before_split, void* event_after_split,
    void* event_after_combine) {
  return attention_impl(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, D, num_blocks, bt,
                        max_blocks, k_scale, v_scale, sm_scale, window_left, sinks, out, lse,
                        workspace, workspace_bytes, stream, chunk_pages_override,
                        event_before_split, event_after_split, event_after_combine);
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

// Scratch for fp8_paged_decode_attention_noalloc: split partials and status
// word for callers that cannot allocate.  In host code this name is only a
// stand-in; the device address comes from cudaGetSymbolAddress per device.
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
  // the status word must start at zero; the partials are fully rewritten
  if (cudaMemsetAsync(scratch, 0, kHeaderBytes, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return FPD_ERR_CUDA;
  return attention_impl(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, D, num_blocks, bt,
                        max_blocks, k_scale, v_scale, sm_scale, window_left, sinks, out, lse,
                        scratch, FPD_NOALLOC_SCRATCH_BYTES, stream, 0, nullptr, nullptr, nullptr);
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
  if (cudaMemsetAsync(workspace, 0, kHeaderBytes, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return FPD_ERR_CUDA;
  return FPD_OK;
}

}  // extern "C"
