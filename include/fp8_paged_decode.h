/*
 * fp8_paged_decode.h -- C ABI of the B200 (sm_100a) paged FP8 decode attention.
 *
 * The operation (named by the grouped-nf4-gemm solutions page
 * "fp8-paged-attention-for-moe-serving", title and summary): one decode query
 * per sequence attends, through a per-sequence block table, to a paged KV cache
 * stored as E4M3 (OCP e4m3fn) codes with per-tensor scales, with a caller-chosen
 * softmax scale, an optional sliding window and optional per-head attention
 * sinks.  For sequence b and query head h (GQA: g = Hq / Hkv, KV head h / g):
 *
 *   start = window_left >= 0 ? max(0, L_b - 1 - window_left) : 0
 *   s_j   = sm_scale * q[b,h,:] . (k_scale * e4m3(K_b[j, h/g, :]))   j in [start, L_b)
 *   sigma = sinks ? sinks[h] : -inf                (no value; denominator only)
 *   out   = sum_j e^(s_j - m) v_scale e4m3(V_b[j, h/g, :]) / (sum_j e^(s_j - m) + e^(sigma - m))
 *   lse   = m + ln(sum_j e^(s_j - m) + e^(sigma - m)),   m = max(max_j s_j, sigma)
 *
 * K_b[j] lives at k_cache[block_table[b][j / block_tokens]][j % block_tokens]:
 * the FlashInfer/SGLang paged-KV convention (fish-scales-ops README, the note on
 * paged prefill/decode APIs following those conventions; the NVFP4 KV-cache gist,
 * vLLM FlashInfer backend section).  Per-tensor scales follow the gist's cache
 * writer (stored code = x / scale).  window_left is FlashInfer's parameter of the
 * same name (gist, FlashInfer backend patch).  The caller-owned workspace with a
 * size query and no allocation on any call path follows FlashInfer PR #5591,
 * Summary ("caller-owned workspace").
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers of the current CUDA device unless
 *    stated otherwise; all are row-major and contiguous.  The caller owns every
 *    buffer.  The library never allocates, frees or synchronises device memory
 *    (fp8_paged_decode_check_status is the one call that synchronises).
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *    default stream) and the call returns without waiting for it.
 *  - Calls with distinct workspaces may run concurrently.
 *  - Host-detectable errors return a status before anything is launched.
 *  - Data errors found on the device (sequence length outside [0, max_blocks *
 *    block_tokens], block-table entry outside [0, num_blocks) inside the attended
 *    range) never cause an out-of-bounds access: the length is clamped, the page
 *    is read as zeros, and a bit is set in the workspace status word
 *    (FPD_DEVERR_*), readable with fp8_paged_decode_check_status.
 *
 * Beyond the single-query E4M3 call: several query tokens per sequence
 * (_qlen), a descriptor form with fp16 queries, head-major pages, token
 * strides, device scales, NVFP4 pages and an f32 output (_args), the FP8 and
 * NVFP4 cache writers, and context-parallel decode (the f32 partial of a rank,
 * the merge of R ranks' partials, and the exchange fused into the decode with
 * a merge that waits for the ranks' flags).
 */
#ifndef FP8_PAGED_DECODE_H
#define FP8_PAGED_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FPD_OK = 0,
    FPD_ERR_INVALID_ARG = 1,          /* null pointer, negative size, bad alignment, non-finite scale */
    FPD_ERR_UNSUPPORTED = 2,          /* shape outside the supported set (see below) */
    FPD_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace_bytes below the size query's answer */
    FPD_ERR_CUDA = 4                  /* a CUDA runtime/driver call failed */
} fpd_status;

/* Device-side status bits (sticky until cleared). */
#define FPD_DEVERR_SEQ_LEN 0x1u       /* a seq_lens entry was < 0 or > max_blocks * block_tokens (clamped) */
#define FPD_DEVERR_BLOCK_TABLE 0x2u   /* a block-table entry in the attended range was outside [0, num_blocks) (read as zeros) */
#define FPD_DEVERR_TIMEOUT 0x4u       /* a pipeline wait, or a context-parallel merge's wait for a
                                         rank's flag, exceeded its time limit (results invalid) */
#define FPD_DEVERR_SLOT 0x8u          /* cache write: a slot_mapping entry was >= num_blocks * block_tokens (token skipped) */

/* Split plan chosen by the host planner; all fields are outputs. */
typedef struct {
    int chunk_pages;        /* KV pages per split (one work item per sequence, KV head group and split) */
    int max_splits;         /* most splits of any one sequence */
    int heads_per_stage;    /* KV heads per pipeline stage and work item: 4 when Hkv % 4 == 0, else 1 */
    int stage_tokens;       /* tokens per KV head and stage (heads_per_stage * stage_tokens == 64) */
    int stages;             /* depth of the shared-memory ring */
    int header_slots;       /* depth of the work-item header ring (1 or 2) */
    int ctas;               /* grid size of the split kernel */
    int smem_bytes;         /* dynamic shared memory per CTA */
    size_t workspace_bytes; /* bytes this plan needs */
    int q_per_item;         /* query positions per work item (1 with one query per sequence) */
    int q_chunks;           /* work items per sequence, KV head group and split: ceil(q_len / q_per_item) */
    int adapt_chunk_pages;  /* 0, or the larger split size the kernel takes instead of chunk_pages
                               when the sequences are of about equal length (the grid is then
                               sized for its items); max_splits and the workspace follow chunk_pages */
} fpd_plan;

/*
 * Supported shapes: D (head_dim) in {64, 128}; g = Hq / Hkv in {1, 2, 4, 8, 16};
 * block_tokens in {16, 32, 64}; num_blocks * block_tokens < 2^31; q, out and the
 * caches 16-byte aligned.  Anything else returns FPD_ERR_UNSUPPORTED (or
 * FPD_ERR_INVALID_ARG for malformed arguments); there is no fallback path.
 */

/*
 * Host-only planner (no CUDA call): the split plan for a shape on a device with
 * `num_sms` SMs of which `ctas_per_sm` CTAs of the split kernel fit per SM.
 * chunk_pages_override > 0 forces the pages per split (rounded up to whole
 * 64-token stages when a stage holds one KV head); 0 lets the heuristic choose.
 * Returns FPD_OK or the validation error for the shape.
 */
fpd_status fp8_paged_decode_make_plan(int B, int Hq, int Hkv, int D, int block_tokens,
                                      int max_blocks, int window_left, int num_sms,
                                      int ctas_per_sm, int chunk_pages_override,
                                      fpd_plan *plan);

/* The host-only planner for q_len query tokens per sequence (see
 * fp8_paged_decode_attention_qlen); q_len = 1 is fp8_paged_decode_make_plan. */
fpd_status fp8_paged_decode_make_plan_qlen(int B, int q_len, int Hq, int Hkv, int D,
                                           int block_tokens, int max_blocks, int window_left,
                                           int num_sms, int ctas_per_sm,
                                           int chunk_pages_override, fpd_plan *plan);

/*
 * The plan fp8_paged_decode_attention_ex uses on the CURRENT device (its SM
 * count and the split kernel's occupancy, queried once per device).  Returns
 * FPD_ERR_CUDA when no device is usable.
 */
fpd_status fp8_paged_decode_plan(int B, int Hq, int Hkv, int D, int block_tokens, int max_blocks,
                                 int window_left, int chunk_pages_override, fpd_plan *plan);

/*
 * Workspace bytes one fp8_paged_decode_attention call with these sizes needs on
 * the CURRENT device (queries its SM count and the kernel occupancy once).
 * Returns 0 for an unsupported or malformed shape, or when no device is present.
 * The workspace holds a 256-byte header and per-split partial results.  Header
 * words: 0 the sticky FPD_DEVERR_* status bits; 1 and 2 the work counter and
 * the finished-CTA count (reset by the kernel itself); 3 the split size
 * (pages) the last call used; 4 the publishing CTA count of the fused
 * context-parallel exchange (reset by the kernel).  Zero the header once
 * before the first call (fp8_paged_decode_workspace_init); between calls it
 * carries only the status bits and word 3.
 */
size_t fp8_paged_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int block_tokens,
                                        int max_blocks, int window_left);

/* Same, for a forced split size (see fp8_paged_decode_make_plan). */
size_t fp8_paged_decode_workspace_bytes_ex(int B, int Hq, int Hkv, int D, int block_tokens,
                                           int max_blocks, int window_left,
                                           int chunk_pages_override);

/*
 * Paged E4M3 decode attention (the formula at the top of this file).
 *   q            bf16  [B, Hq, D]
 *   k_cache      e4m3  [num_blocks, block_tokens, Hkv, D]   (token-major pages)
 *   v_cache      e4m3  [num_blocks, block_tokens, Hkv, D]
 *   block_table  int32 [B, max_blocks]; entry i is the physical page of the
 *                sequence's tokens [i*block_tokens, (i+1)*block_tokens); only
 *                the pages covering the attended range are read
 *   seq_lens     int32 [B]; L_b, the sequence length including the new token
 *   k_scale, v_scale   per-tensor dequantisation scales (value = code * scale)
 *   sm_scale     softmax scale applied to q.k (sm_scale * k_scale must be > 0)
 *   window_left  < 0: attend all L_b keys; >= 0: the newest window_left + 1
 *   sinks        float [Hq] sink logits (same units as sm_scale * q.k), or NULL
 *   out          bf16  [B, Hq, D] (round to nearest even)
 *   lse          float [B, Hq] natural-log sum of exponentials including the
 *                sink, or NULL (not written).  L_b == 0 gives out = 0 and
 *                lse = sinks[h] (or -inf).
 *   workspace    device buffer of at least fp8_paged_decode_workspace_bytes()
 *                (always >= 256) bytes, 16-byte aligned.  Its first word is the
 *                sticky device status: zero it once after allocating (or call
 *                fp8_paged_decode_workspace_init); the rest is scratch
 *   stream       cudaStream_t
 * Two kernels are enqueued: the split kernel and, when some sequence spans
 * several splits, the combine kernel.
 */
fpd_status fp8_paged_decode_attention(const void *q, const void *k_cache, const void *v_cache,
                                      const int32_t *block_table, const int32_t *seq_lens,
                                      int B, int Hq, int Hkv, int D, int num_blocks,
                                      int block_tokens, int max_blocks, float k_scale,
                                      float v_scale, float sm_scale, int window_left,
                                      const float *sinks, void *out, float *lse,
                                      void *workspace, size_t workspace_bytes, void *stream);

/* Same, with a forced split size (0 = heuristic); for tests and tuning. */
fpd_status fp8_paged_decode_attention_ex(const void *q, const void *k_cache, const void *v_cache,
                                         const int32_t *block_table, const int32_t *seq_lens,
                                         int B, int Hq, int Hkv, int D, int num_blocks,
                                         int block_tokens, int max_blocks, float k_scale,
                                         float v_scale, float sm_scale, int window_left,
                                         const float *sinks, void *out, float *lse,
                                         void *workspace, size_t workspace_bytes, void *stream,
                                         int chunk_pages_override);

/*
 * Several query tokens per sequence (speculative / multi-token decode): each
 * sequence's q_len newest tokens are queries.  Query i sits at position
 * p = seq_lens[b] - q_len + i, attends causally to the keys up to p and, with
 * window_left >= 0, only to the window_left keys before p as well; sinks
 * enter every query's denominator.  A query with p < 0 sees no key (out = 0,
 * lse = its sink, or -inf).  q_len = 1 is fp8_paged_decode_attention_ex.
 * (Multi-token decode rows as routed on the FlashInfer PR #5591 page,
 * "Unsupported" section; MTP decode in the NVFP4 KV-cache serving gist.)
 *   q    bf16 [B, q_len, Hq, D];  out bf16 [B, q_len, Hq, D];  lse f32 [B, q_len, Hq]
 *   other arguments as in fp8_paged_decode_attention_ex; seq_lens include the
 *   q_len new tokens, whose K/V must already be in the cache.
 * Supported: 1 <= q_len <= FPD_MAX_Q_LEN (else FPD_ERR_UNSUPPORTED), any
 * supported g.  A work item covers the KV range of one split for up to 16 / g
 * of the sequence's queries (at least one); longer query runs are cut into
 * several items over the same pages, which then mostly come from L2.  Size the
 * workspace with the _qlen query below.
 */
#define FPD_MAX_Q_LEN 64
fpd_status fp8_paged_decode_attention_qlen(const void *q, const void *k_cache, const void *v_cache,
                                           const int32_t *block_table, const int32_t *seq_lens,
                                           int B, int q_len, int Hq, int Hkv, int D,
                                           int num_blocks, int block_tokens, int max_blocks,
                                           float k_scale, float v_scale, float sm_scale,
                                           int window_left, const float *sinks, void *out,
                                           float *lse, void *workspace, size_t workspace_bytes,
                                           void *stream, int chunk_pages_override);

/* The plan and the workspace bytes for q_len query tokens per sequence. */
fpd_status fp8_paged_decode_plan_qlen(int B, int q_len, int Hq, int Hkv, int D, int block_tokens,
                                      int max_blocks, int window_left, int chunk_pages_override,
                                      fpd_plan *plan);
size_t fp8_paged_decode_workspace_bytes_qlen(int B, int q_len, int Hq, int Hkv, int D,
                                             int block_tokens, int max_blocks, int window_left,
                                             int chunk_pages_override);

/*
 * Interface variants: the general decode call, described by a struct.
 * The layouts and forms are the ones the pages' serving stack uses: the
 * FlashInfer backend of the NVFP4 KV-cache serving gist takes the query in the
 * model dtype (bf16 or fp16), pages in token-major (NHD) or head-major (HND)
 * order (its cache writer writes both), and a query/output that may be a slice
 * of a wider buffer (the fused QKV projection); per-tensor scales kept in
 * device memory let one captured CUDA graph be replayed with new scales.
 */
#define FPD_KV_NHD 0   /* pages [num_blocks, block_tokens, Hkv, D] (token-major) */
#define FPD_KV_HND 1   /* pages [num_blocks, Hkv, block_tokens, D] (head-major) */
#define FPD_Q_BF16 0
#define FPD_Q_F16  1
#define FPD_KV_E4M3  0   /* E4M3 codes, one byte per element */
#define FPD_KV_NVFP4 1   /* E2M1 codes with an E4M3 scale per 16 elements */
#define FPD_OUT_BF16 0   /* out is bf16 */
#define FPD_OUT_F32  1   /* out is f32: the (O, lse) partial of a context-parallel rank */

typedef struct {
    /* query token t = b * q_len + i, head h, element d is at
     * q[t * q_token_stride + h * D + d]; q_token_stride = 0 means Hq * D.
     * Nonzero strides must be >= Hq * D and a multiple of 8 (16 bytes). */
    const void *q;
    int q_dtype;                 /* FPD_Q_BF16 or FPD_Q_F16 */
    int64_t q_token_stride;      /* elements */
    const void *k_cache;         /* e4m3 pages in kv_layout order */
    const void *v_cache;
    int kv_layout;               /* FPD_KV_NHD or FPD_KV_HND */
    const int32_t *block_table;  /* [B, max_blocks] */
    const int32_t *seq_lens;     /* [B], including the q_len new tokens */
    int B, q_len, Hq, Hkv, D, num_blocks, block_tokens, max_blocks;
    float k_scale, v_scale;      /* host scales, used when the device ones are NULL */
    const float *k_scale_dev;    /* device float or NULL; read by the kernels */
    const float *v_scale_dev;    /* device float or NULL */
    float sm_scale;
    int window_left;             /* < 0: no window */
    const float *sinks;          /* [Hq] f32 or NULL */
    /* out is bf16; token t, head h, element d at out[t * out_token_stride + h * D + d];
     * 0 means Hq * D; nonzero: >= Hq * D and a multiple of 8. */
    void *out;
    int64_t out_token_stride;    /* elements */
    float *lse;                  /* [B, q_len, Hq] contiguous, or NULL */
    int chunk_pages_override;    /* 0: heuristic */
    /* Page format.  FPD_KV_NVFP4 (head-major pages only): k_cache / v_cache
     * point at the E2M1 data of page 0, [Hkv][bt][D/2] bytes per page (element
     * 2i of a row in the low nibble of byte i), and k_scales / v_scales at its
     * E4M3 block scales, [Hkv][bt][D/16] bytes per page (one per 16 elements);
     * consecutive pages are kv_page_stride (data) and sf_page_stride (scales)
     * bytes apart, 0 meaning packed.  An element's value is
     * e2m1(code) * e4m3(block scale) * k_scale (v_scale).  The writer's page
     * [K data | K scales | V data | V scales] is four such pointers with one
     * stride.  Strides must be multiples of 16. */
    int kv_format;               /* FPD_KV_E4M3 or FPD_KV_NVFP4 */
    const void *k_scales;
    const void *v_scales;
    int64_t kv_page_stride;
    int64_t sf_page_stride;
    /* Output type.  FPD_OUT_F32: out is f32 with the same element strides
     * (nonzero out_token_stride a multiple of 8, out 16-byte aligned); every
     * row is then finished by the combine kernel, so the workspace holds one
     * partial per row even when no sequence is split: size it with
     * fp8_paged_decode_workspace_bytes_args.  A row with no key and no sink
     * gets out = 0 and lse = -inf, which fp8_paged_decode_cp_merge skips. */
    int out_dtype;               /* FPD_OUT_BF16 or FPD_OUT_F32 */
    /* Context-parallel publishing (cp_ranks > 0): the exchange of the ranks'
     * partials fused into this call.  Needs out_dtype = FPD_OUT_F32, q_len = 1
     * and contiguous out rows (out_token_stride 0 or Hq * D); `out` and `lse`
     * are not written.  The combine kernel stores every row's f32 O and lse
     * straight into slot cp_rank of each rank r's gather buffer cp_gather[r]
     * (cp_block_floats floats per slot: [B*Hq][D] O, then [B*Hq] lse; the
     * fp8_paged_decode_cp_merge layout) over peer memory (NVLink), and when
     * the whole grid has stored its rows it sets word cp_rank of each rank's
     * flag array cp_flags[r] to cp_epoch (one system-scope fence, then the
     * flag stores).
     * cp_gather and cp_flags are device arrays of cp_ranks device pointers
     * (peer pointers from CUDA IPC or another mapping).  Workspace word 4
     * counts the finished CTAs and must be zero between calls (it is reset).
     * A slot must not be rewritten while its rank may still merge it: alternate
     * two sets of gather buffers and flags by the parity of the epoch (a rank
     * can run at most one step ahead of another). */
    float *const *cp_gather;
    uint32_t *const *cp_flags;
    int cp_ranks, cp_rank;
    uint32_t cp_epoch;
    int64_t cp_block_floats;
} fpd_decode_args;

/*
 * The decode call for any combination of the variants above.  q_len, masks,
 * sinks and the workspace are as in fp8_paged_decode_attention_qlen (size the
 * workspace with fp8_paged_decode_workspace_bytes_qlen: the variants do not
 * change it).  Device scales are read on the GPU after the work queued before
 * this call on `stream` has completed, so a kernel earlier in the stream may
 * write them; their validity (finite, > 0) is the caller's: a bad device scale
 * gives NaN or infinite outputs, not an error.  Host scales are validated as in
 * the other calls.  Returns FPD_ERR_INVALID_ARG for a bad stride, dtype or
 * layout code, and the errors of fp8_paged_decode_attention otherwise.
 */
fpd_status fp8_paged_decode_attention_args(const fpd_decode_args *args, void *workspace,
                                           size_t workspace_bytes, void *stream);

/* fp8_paged_decode_attention_args that also records the given cudaEvent_t
 * handles (void*, each may be NULL) on `stream` before the split kernel,
 * between the two kernels and after the combine kernel, as
 * fp8_paged_decode_attention_profiled does. */
fpd_status fp8_paged_decode_attention_args_profiled(const fpd_decode_args *args, void *workspace,
                                                    size_t workspace_bytes, void *stream,
                                                    void *event_before_split,
                                                    void *event_after_split,
                                                    void *event_after_combine);

/* The plan and the workspace bytes of a descriptor's call on the current
 * device (the page format changes the kernel's shared memory and so the
 * plan, and an f32 output needs the partials even for one split).
 * workspace_bytes_args returns 0 for an invalid descriptor. */
fpd_status fp8_paged_decode_plan_args(const fpd_decode_args *args, fpd_plan *plan);
size_t fp8_paged_decode_workspace_bytes_args(const fpd_decode_args *args);

/*
 * Same as fp8_paged_decode_attention_qlen, and additionally records the given
 * cudaEvent_t handles (passed as void*, each may be NULL) on `stream`: one
 * before the split kernel, one between the split and combine kernels, one after
 * the combine kernel.  For measuring each kernel's duration with CUDA events on
 * the stream the kernels run on; the kernels and their arguments are unchanged.
 */
fpd_status fp8_paged_decode_attention_profiled(const void *q, const void *k_cache,
                                               const void *v_cache, const int32_t *block_table,
                                               const int32_t *seq_lens, int B, int q_len, int Hq, int Hkv,
                                               int D, int num_blocks, int block_tokens,
                                               int max_blocks, float k_scale, float v_scale,
                                               float sm_scale, int window_left,
                                               const float *sinks, void *out, float *lse,
                                               void *workspace, size_t workspace_bytes,
                                               void *stream, int chunk_pages_override,
                                               void *event_before_split, void *event_after_split,
                                               void *event_after_combine);

/*
 * Size of the library's static device scratch used by
 * fp8_paged_decode_attention_noalloc: 16 MiB per GPU, held from the first use
 * of the library on that GPU until the process exits.
 */
#define FPD_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * fp8_paged_decode_attention_noalloc -- the decode call for callers that cannot
 * allocate device memory at all: code running where cudaMalloc is unavailable or
 * forbidden (inside a custom allocator, a plug-in whose host owns all device
 * memory, or a capture/replay path that must not create new allocations) and
 * that therefore cannot provide the workspace fp8_paged_decode_attention needs.
 * The pages describe no such entry point; it has no counterpart there.
 *
 * Arguments are those of fp8_paged_decode_attention without the workspace: the
 * caller still passes every input and output.  The split partials and the status
 * word live instead in one static device array of FPD_NOALLOC_SCRATCH_BYTES
 * inside this library.  Behaviour:
 *  - Nothing is allocated or freed: no cudaMalloc/cudaFree and no allocating
 *    library routine on any call.
 *  - A shape whose plan needs more scratch than FPD_NOALLOC_SCRATCH_BYTES is
 *    rejected with FPD_ERR_WORKSPACE_TOO_SMALL, and every other argument error
 *    with its status, before anything is enqueued on the stream.
 *  - The first call on each device looks up the array's device address on that
 *    device (cudaGetSymbolAddress); make that first call before any stream
 *    capture on the device.  A failed lookup returns FPD_ERR_CUDA.
 *  - That address is kept for the life of the process.  Do not call this entry
 *    point on a device after cudaDeviceReset, or after its primary context was
 *    otherwise destroyed and created again: the library would write through
 *    the old context's address.
 *  - Every call, on any stream, shares the one array, which keeps the previous
 *    call's contents; each call zeroes the part that must start at zero (the
 *    status word) on its own stream before its kernels.  Calls whose kernels
 *    overlap on the GPU (different streams, no ordering between them) race on
 *    the array and give wrong results; order them on one stream or use the
 *    workspace entry point.
 *  - Device status bits are kept in the shared array and are not reported.
 */
fpd_status fp8_paged_decode_attention_noalloc(const void *q, const void *k_cache,
                                              const void *v_cache, const int32_t *block_table,
                                              const int32_t *seq_lens, int B, int Hq, int Hkv,
                                              int D, int num_blocks, int block_tokens,
                                              int max_blocks, float k_scale, float v_scale,
                                              float sm_scale, int window_left,
                                              const float *sinks, void *out, float *lse,
                                              void *stream);

/*
 * FP8 KV-cache write: quantise the bf16 K and V rows of new tokens with the
 * per-tensor scales and scatter them into the paged E4M3 caches.  The
 * quantisation is the per-tensor form of the standalone cache-writer kernel in
 * the NVFP4 KV-cache serving gist (writer kernel and host wrapper sections):
 *   code = e4m3_rne_satfinite(float(x) * (1.0f / scale))
 * with the reciprocal rounded to fp32 once and the product rounded to fp32;
 * the E4M3 rounding is to nearest, ties to even, and saturates at +-448
 * (infinities too; NaN stays NaN).
 *   key, value    bf16 [num_tokens, Hkv, D]; token stride key_stride /
 *                 value_stride elements (a multiple of 8; rows contiguous);
 *                 16-byte aligned
 *   slot_mapping  int64 [num_tokens]: slot = page * block_tokens + offset;
 *                 negative = padded token, skipped.  Slots must be distinct
 *                 (two tokens on one slot race).
 *   k_cache, v_cache  e4m3 [num_blocks, block_tokens, Hkv, D] (16-byte
 *                 aligned), written in place at the given slots only
 *   status        optional device word (e.g. a decode workspace's status
 *                 word) that receives FPD_DEVERR_SLOT for a slot past the
 *                 end of the cache; that token is skipped.  NULL: no report.
 * Requires D % 16 == 0, k_scale and v_scale finite and > 0.  Runs on `stream`,
 * allocates nothing, never synchronises; num_tokens == 0 is a no-op.
 */
fpd_status fp8_paged_decode_cache_write(const void *key, const void *value,
                                        const int64_t *slot_mapping, int num_tokens, int Hkv,
                                        int D, int64_t key_stride, int64_t value_stride,
                                        float k_scale, float v_scale, void *k_cache,
                                        void *v_cache, int num_blocks, int block_tokens,
                                        uint32_t *status, void *stream);

/*
 * The cache write into pages of either layout (kv_layout FPD_KV_NHD or
 * FPD_KV_HND); fp8_paged_decode_cache_write is kv_layout = FPD_KV_NHD.  Head-
 * major pages need num_blocks * block_tokens < 2^31.
 */
fpd_status fp8_paged_decode_cache_write_layout(const void *key, const void *value,
                                               const int64_t *slot_mapping, int num_tokens,
                                               int Hkv, int D, int64_t key_stride,
                                               int64_t value_stride, float k_scale,
                                               float v_scale, void *k_cache, void *v_cache,
                                               int num_blocks, int block_tokens, int kv_layout,
                                               uint32_t *status, void *stream);

/*
 * NVFP4 KV-cache write: the block quantisation of the NVFP4 KV-cache serving
 * gist's cache writer (its writer kernel and quantisation helper), with the
 * reciprocals taken exactly in fp32 where the gist uses approximate ones.  For
 * each 16 consecutive elements x of a token's K (V) head row, with
 * gs = 1 / k_scale (1 / v_scale):
 *   scale = e4m3_rne_satfinite((max|x| * (1/6)) * gs)
 *   code  = e2m1_rne_satfinite(x * (1 / (scale * (1 / gs))))   (0 if scale == 0)
 * every product and reciprocal rounded to fp32.  Codes go to the data region
 * and scales to the scale region of head-major NVFP4 pages (see
 * fpd_decode_args: data [Hkv][bt][D/2] bytes, element 2i in the low nibble;
 * scales [Hkv][bt][D/16]), at the given page strides (0 = packed).
 *   key, value, slot_mapping, status: as in fp8_paged_decode_cache_write
 *   k_data, k_sf, v_data, v_sf: 16-byte aligned device pointers to page 0
 * Requires D % 16 == 0, num_blocks * block_tokens < 2^31, strides multiples of
 * 16 and at least the packed region sizes, scales finite and > 0.  NaN inputs
 * give unspecified codes.  Runs on `stream`, allocates nothing.
 */
fpd_status fp8_paged_decode_cache_write_nvfp4(const void *key, const void *value,
                                              const int64_t *slot_mapping, int num_tokens,
                                              int Hkv, int D, int64_t key_stride,
                                              int64_t value_stride, float k_scale, float v_scale,
                                              void *k_data, void *k_sf, void *v_data, void *v_sf,
                                              int64_t data_page_stride, int64_t sf_page_stride,
                                              int num_blocks, int block_tokens, uint32_t *status,
                                              void *stream);

/*
 * Context-parallel decode: the merge.  When each of R ranks holds part of
 * every sequence's KV pages, each computes the decode over its own keys with
 * no sinks and an f32 output (fpd_decode_args.out_dtype = FPD_OUT_F32), the
 * ranks exchange those (O_r, lse_r) partials (an all-gather), and this call
 * folds them into the attention over all keys:
 *   out = sum_r e^(lse_r - M) O_r / Z,   lse = M + ln Z,
 *   Z = sum_r e^(lse_r - M) + e^(sigma - M),   M = max(max_r lse_r, sigma),
 * sigma = sinks[h] (absent: -inf).  This is the split-KV merge of partial O
 * and LSE of FlashInfer PR #5591 (Summary: the workspace's partial_O /
 * partial_lse and its split merge), with ranks in place of splits; that page
 * lists decode context parallelism (DCP) as unsupported ("Unsupported"
 * section), so the partition of the keys is the caller's.
 *   partials     f32, R blocks of block_floats floats, one per rank in any
 *                order: a block's first rows * D floats are O_r [rows][D],
 *                the next rows floats lse_r [rows] (natural log, -inf for a
 *                rank with no key of the row), the rest padding.  rows =
 *                B * q_len * Hq, a row being (token, head) with the head
 *                innermost.  An all-gather of each rank's [O | lse | pad]
 *                buffer produces this layout.
 *   block_floats >= rows * (D + 1), a multiple of 4 (16-byte blocks).
 *   sinks        f32 [Hq] or NULL.
 *   out          bf16; row (t, h) at out[t * out_token_stride + h * D];
 *                out_token_stride 0 means Hq * D.
 *   lse          f32 [rows] or NULL.
 * R >= 1, Hq >= 1, D in {64, 128}, rows >= 0 a multiple of Hq; partials and
 * out 16-byte aligned, out_token_stride a multiple of 8 and >= Hq * D.  A row that
 * no rank and no sink covers gets out = 0 and lse = -inf.  The call enqueues
 * one kernel and does not synchronise.  Errors: FPD_ERR_INVALID_ARG (null
 * pointer, bad alignment, stride or count), FPD_ERR_UNSUPPORTED (D),
 * FPD_ERR_CUDA (launch failure).  Nothing is written on error.
 */
fpd_status fp8_paged_decode_cp_merge(const float *partials, int R, int64_t block_floats,
                                     int64_t rows, int Hq, int D, const float *sinks, void *out,
                                     int64_t out_token_stride, float *lse, void *stream);

/*
 * The merge of a fused exchange: `gather` is this rank's gather buffer, whose
 * R slots the ranks' decode calls fill (fpd_decode_args.cp_gather), and
 * flags[r] (this rank's flag array, device memory) reaches `epoch` once rank
 * r's slot is complete.  Each CTA first waits for all R flags (acquire loads at
 * system scope) for at most timeout_ns nanoseconds of the GPU's global timer;
 * a CTA that gives up or-s FPD_DEVERR_TIMEOUT into *status (device word, may
 * be NULL) and writes nothing.  The other arguments and errors are those of
 * fp8_paged_decode_cp_merge; epoch 0, timeout 0 or a NULL flags pointer is
 * FPD_ERR_INVALID_ARG.  Epochs must change from call to call (the flags keep
 * the last one).
 */
fpd_status fp8_paged_decode_cp_merge_wait(const float *gather, int R, int64_t block_floats,
                                          int64_t rows, int Hq, int D, const float *sinks,
                                          void *out, int64_t out_token_stride, float *lse,
                                          const uint32_t *flags, uint32_t epoch,
                                          uint64_t timeout_ns, uint32_t *status, void *stream);

/*
 * Reads the workspace status word (FPD_DEVERR_* bits) after synchronising
 * `stream`; clears it when `clear` is nonzero.  Writes the bits to
 * *device_error_bits.  Needs a workspace of at least 256 bytes.
 */
fpd_status fp8_paged_decode_check_status(void *workspace, void *stream, int *device_error_bits,
                                         int clear);

/* Enqueue a zeroing of the workspace header (status word) on `stream`. */
fpd_status fp8_paged_decode_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* Human-readable name of a status code (static string). */
const char *fp8_paged_decode_status_string(fpd_status status);

/* Library version string, e.g. "0.1.0 sm_100a". */
const char *fp8_paged_decode_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8_PAGED_DECODE_H */
