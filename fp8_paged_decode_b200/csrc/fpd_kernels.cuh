// fpd_kernels.cuh -- the sm_100a kernel of the paged E4M3 decode attention.
//
// One persistent kernel.  Each CTA (one or more per SM) pulls work items from
// a global counter; an item is (sequence b, group of HB KV heads, KV split)
// and covers up to `chunk_pages` pages of that sequence's attended range.
// Warp 4 is the producer: it first builds the call's work list alone (the
// prefix over sequences of their splits, from seq_lens; the consumer warps
// never wait for it), then for every item it publishes a small header plus the
// item's query rows (bulk copy) in a header ring and streams the item's KV
// with TMA tiled loads into a ring of shared-memory stages.  The stage ring
// runs straight across item boundaries, so HBM reads never wait for an item to
// start.  A stage holds 64 token rows of K and of V, in one of two shapes:
//
//   HB = 4 (the KV head count is a multiple of 4): 16 tokens x 4 KV heads, one
//     TMA box per tensor (D bytes x 16 tokens x 4 heads, 128-byte swizzle).
//     Consumer warp w owns KV head 4j + w of the item for all of its tokens,
//     so an item needs no merge between warps: each warp finishes its own
//     query heads straight from registers.
//   HB = 1: 64 tokens of one KV head, one TMA box per page and tensor; the
//     four consumer warps split the rows 16 apiece and merge in shared memory
//     at the end of the item.
//
// Per consumer warp and stage, 16 token rows of one KV head:
//   S^T = K Q^T      mma.sync m16n8k16, tokens on M, the query heads of the KV
//                    head on N (heads on the MMA N side, as in the "SwapsAb"
//                    orientation of FlashInfer PR #5591, Summary);
//   online softmax   base 2 with a lazy running max: the max moves only when a
//                    tile exceeds it by more than 8 in the exp2 domain (the
//                    lazy-rescale rule of the same PR's Summary);
//   O^T += V^T P^T   mma.sync m16n8k16, head dim on M, heads on N;
// with E4M3 -> f16 conversion in registers (exact) and the per-tensor scales
// folded into the logit scale and the output.  An item that covers its whole
// sequence writes bf16 out and lse (sink folded in).  Otherwise it writes an
// fp32 partial (O / l and log2-sum-exp), and the combine kernel, launched as a
// programmatic dependent of this one (its CTAs start during this kernel's
// tail and wait for its completion; the FP8 paged-MLA route on the FlashInfer
// PR #5591 page, section "Unsupported", launches its split-KV merge the same
// way), merges the partials of every sequence that spans several splits and
// folds in the sink.  The last CTA to leave resets the work counter, so the
// workspace needs zeroing only once after allocation.
//
// Fragment layouts (PTX ISA, mma.m16n8k16 with .f16):
//   A: a0 (row g, cols 2t..2t+1), a1 (row g+8, same), a2 (row g, cols 2t+8..),
//      a3 (row g+8, cols 2t+8..);  B: b0 (rows 2t..2t+1, col g), b1 (rows
//      2t+8.., col g);  C: c0,c1 (row g, cols 2t..2t+1), c2,c3 (row g+8, ...)
//   with g = lane / 4, t = lane % 4.
// Because q.k and P.V are sums, the head-dim index behind each fragment slot
// may be any fixed permutation; the kernel picks the one that makes every
// thread's shared-memory reads contiguous 16-byte vectors:
//   QK k-step ks, slot 2t+u  -> d = t*(D/4) + 4*ks + u      (u in 0..1)
//               slot 2t+8+u  -> d = t*(D/4) + 4*ks + 2 + u
//   PV m-tile i, row g+8h    -> d = g*(D/8) + 2*i + h        (h in 0..1)
// so the O^T rows a thread holds for one query head are the D/8 contiguous
// elements starting at g*D/8.
//
// Every wait (mbarrier phase, consumer-group sync) is bounded in time; on
// expiry the kernel sets FPD_DEVERR_TIMEOUT in the status word and the warp
// leaves, so a fault upstream can never hang the GPU.
#pragma once

#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fpd_ptx.cuh"

namespace fpd {

constexpr int kConsumerWarps = 4;
constexpr int kRowsPerWarp = 16;
constexpr int kTileTokens = kConsumerWarps * kRowsPerWarp;  // token rows per stage and tensor
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxHdrSlots = 2;
constexpr int kHdrBytes = 64;                 // ItemHeader, padded
constexpr int kBoxTokens = 16;                // tokens per TMA box with HB = 4
constexpr float kLazyThreshold = 8.0f;        // log2 units
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint64_t kWaitLimitNs = 500000000ull;  // 0.5 s: far above any legitimate wait
constexpr uint64_t kDrainLimitNs = 50000000ull;  // 50 ms per stage when draining

constexpr uint32_t kErrSeqLen = 0x1u;
constexpr uint32_t kErrBlockTable = 0x2u;
constexpr uint32_t kErrTimeout = 0x4u;

struct DecodeParams {
  const __nv_bfloat16* q;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const float* sinks;
  __nv_bfloat16* out;
  float* lse;
  float* part_o;        // [B, Hq, max_splits, D]
  float* part_lse;      // [B, Hq, max_splits]   (log2 domain)
  uint32_t* status;     // workspace word 0: sticky FPD_DEVERR_* bits
  uint32_t* sched;      // workspace words 1, 2: next work item, CTAs finished;
                        // word 3: the split size the call used (for the combine)
  int B, Hq, Hkv, g, bt, max_blocks, num_blocks, window_left;
  int chunk_pages, max_splits, stages, hdr_slots;
  int q_len;            // query tokens per sequence
  int q_per_item;       // query positions per work item (its columns: q_per_item * g <= 16)
  int q_chunks;         // work items per (sequence, split, KV head group): ceil(q_len / q_per_item)
  int lg;               // log2(g): g is a power of two
  float qk_scale_log2;  // sm_scale * k_scale * log2(e)
  float v_scale;
  // interface variants
  int64_t q_tok_stride;       // elements between consecutive query tokens (>= Hq * D)
  int64_t out_tok_stride;     // elements between consecutive output tokens
  const float* k_scale_dev;   // device scales, read after the grid dependency
  const float* v_scale_dev;   //   resolves; nullptr: the host values above
  float sm_scale_log2;        // sm_scale * log2(e), for a device k_scale
  int q_f16;                  // the query is fp16 (else bf16)
  int kv_hnd;                 // pages are [num_blocks, Hkv, bt, D] (else [.., bt, Hkv, D])
  // nonzero: every row, one split or several, leaves its partial in the
  // workspace and the combine writes it (f32 output, context-parallel
  // publishing)
  int combine_all;
  // > 0: the split size to take instead of chunk_pages when the sequences
  // are of about equal length and chunk_pages gives more items than the grid
  int adapt_chunk;
};

// Bytes of one header slot: the header, then the item's query rows (HB KV
// heads x g query heads x D, bf16).
__host__ __device__ constexpr int hdr_slot_bytes(int D, int HB, int g) {
  return kHdrBytes + ((HB * g * D * 2 + 15) / 16) * 16;
}

// Shared-memory carve-up (byte offsets from a 1024-byte aligned base); used by
// the host to size the launch and by the kernel to find its buffers.  Only
// HB = 1 needs the merge buffer.
struct SmemLayout {
  int ring, merge, qfrag, hdr, prefix, bars, total;
};

// Query fragments kept in shared memory instead of registers (D = 128 with two
// n-tiles: their 32 registers per thread would otherwise spill at the 2-CTA
// register cap).
#ifndef FPD_QFRAG_SMEM
#define FPD_QFRAG_SMEM 1
#endif
__host__ __device__ constexpr bool qfrag_in_smem(int D, int NT) {
  return FPD_QFRAG_SMEM && D == 128 && NT == 2;
}
// Bytes of one consumer warp's query fragments: [NT][D/16 k-steps][32 lanes][2 words].
__host__ __device__ constexpr int qfrag_warp_bytes(int D, int NT) { return NT * (D / 16) * 32 * 8; }

__host__ __device__ constexpr int align_to(int x, int a) { return (x + a - 1) / a * a; }

// NVFP4 stage: four regions [K data | K scales | V data | V scales] holding
// kTileTokens rows each; a row is D / 2 bytes of E2M1 pairs and D / 16 block
// scales.  Every TMA destination in shared memory must sit on a 128-byte
// boundary, so the scale region is 512 bytes even where its rows need only
// 256, and with one head per stage each page's scales start a slot of
// fp4_sf_pitch bytes.
__host__ __device__ constexpr int fp4_data_bytes(int D) { return kTileTokens * D / 2; }
__host__ __device__ constexpr int fp4_sf_bytes(int D) {
  return kTileTokens * D / 16 > 512 ? kTileTokens * D / 16 : 512;
}
__host__ __device__ constexpr int fp4_sf_pitch(int bt, int D) {
  return bt * D / 16 > 128 ? bt * D / 16 : 128;
}

// Bytes the TMA boxes of one NVFP4 stage deliver (without the padding).
__host__ __device__ constexpr int fp4_stage_payload(int D) {
  return 2 * kTileTokens * (D / 2 + D / 16);
}

// Bytes of one ring stage: kTileTokens rows of K and of V.  E4M3 rows are D
// bytes; NVFP4 stages are laid out as above.
__host__ __device__ constexpr int stage_bytes(int D, bool fp4) {
  return fp4 ? 2 * (fp4_data_bytes(D) + fp4_sf_bytes(D)) : 2 * kTileTokens * D;
}

__host__ __device__ inline SmemLayout smem_layout(int D, int NT, int HB, int stages, int hdr_slots,
                                                  int g, int B, bool fp4 = false) {
  SmemLayout L{};
  const int H = NT * 8;
  L.ring = 0;
  L.merge = stages * stage_bytes(D, fp4);
  const int merge_bytes =
      HB == 1 ? kConsumerWarps * H * (D + 4) * 4 + kConsumerWarps * H * 2 * 4 : 0;
  L.qfrag = align_to(L.merge + merge_bytes, 16);
  const int qfrag_bytes = qfrag_in_smem(D, NT) ? kConsumerWarps * qfrag_warp_bytes(D, NT) : 0;
  L.hdr = align_to(L.qfrag + qfrag_bytes, 128);
  L.prefix = align_to(L.hdr + hdr_slots * hdr_slot_bytes(D, HB, g), 16);
  L.bars = align_to(L.prefix + 4 * (B + 1), 16);
  L.total = align_to(L.bars + (2 * stages + 2 * kMaxHdrSlots + 1) * 8, 16) +
            1024;  // + slack to align the base to 1024
  return L;
}

struct ItemHeader {
  int kind;      // 1: work item, -1: no more work
  int b, kvh0, split;
  int ns;        // splits of this sequence (0: empty sequence)
  int n_stages;  // pipeline stages this item consumes
  int t0;        // token of the first row of the item's first stage
  int tok_lo, tok_hi;
  int qpos0;     // position of the item's first query token
  int qrow0;     // index of that query among the sequence's q_len queries
  int npos;      // query positions of the item (its columns: npos * g)
  int pad[4];
};
static_assert(sizeof(ItemHeader) == kHdrBytes, "header size");

// x / d for x >= 0 and d >= 1 (both the same across the warp): a shift when d
// is a power of two (page sizes, head groups), else the division.
__device__ __forceinline__ int div_pos(int x, int d) {
  return (d & (d - 1)) == 0 ? x >> (__ffs(d) - 1) : x / d;
}

// Attended page range of a sequence.
struct SeqRange {
  int L, start, first_page, end_page, n_splits;
};

// The union of the key ranges of the sequence's q_len queries: query i at
// position L - q_len + i sees keys up to its own position and, under a window,
// the window_left keys before it.
__device__ __forceinline__ SeqRange seq_range(int L_raw, int q_len, int bt, int max_blocks,
                                              int window_left, int chunk_pages, uint32_t* status) {
  SeqRange r;
  int L = L_raw;
  const int cap = max_blocks * bt;
  if (L < 0 || L > cap) {
    if (status) atomicOr(status, kErrSeqLen);
    L = L < 0 ? 0 : cap;
  }
  r.L = L;
  r.start = (window_left >= 0) ? max(0, L - q_len - window_left) : 0;
  r.first_page = div_pos(r.start, bt);
  r.end_page = div_pos(L + bt - 1, bt);
  const int n_pages = r.end_page - r.first_page;
  r.n_splits = div_pos(n_pages + chunk_pages - 1, chunk_pages);
  return r;
}

// Work groups (one per split; one for an empty sequence) of a sequence at
// split size `chunk` pages.
__device__ __forceinline__ int groups_of(int L_raw, int q_len, const DecodeParams& p, int chunk) {
  const SeqRange r = seq_range(L_raw, q_len, p.bt, p.max_blocks, p.window_left, chunk, nullptr);
  return r.n_splits > 0 ? r.n_splits : 1;
}

// The producer warp builds the call's work list itself (no other warp needs
// it): the prefix over sequences of their work groups, prefix[b] groups before
// sequence b, in shared memory.  Every CTA builds the same one.
struct WorkPrefix {
  int total;       // work groups of the call
  int first_b;     // sequence of the CTA's first work group (-1: none)
  int first_len;   // its length
};

// Lane l of the producer warp owns sequences [l * per, (l + 1) * per) with
// per = ceil(B / 32): it loads their lengths, sums their work groups and
// writes their prefix entries; one warp scan joins the lanes.  Only the loads
// are unrolled: the code runs once per call, often from cold caches.
__device__ __forceinline__ void lane_range(const DecodeParams& p, int lane, int& b0, int& b1) {
  const int per = (p.B + 31) / 32;
  b0 = min(p.B, lane * per);
  b1 = min(p.B, b0 + per);
}

// Stages the sequence lengths in prefix[1..B] (each lane's loads back to back).
__device__ __forceinline__ void stage_lengths(const DecodeParams& p, int* prefix, int lane) {
  int b0, b1;
  lane_range(p, lane, b0, b1);
#pragma unroll 8
  for (int b = b0; b < b1; ++b) prefix[b + 1] = __ldg(p.seq_lens + b);
}

// From the staged lengths at split size `chunk`: all work groups, and the
// most of one sequence.
__device__ __forceinline__ void length_totals(const DecodeParams& p, int q_len, int chunk,
                                              const int* prefix, int lane, int& total,
                                              int& most) {
  int b0, b1;
  lane_range(p, lane, b0, b1);
  int sum = 0, mx = 0;
#pragma unroll 1
  for (int b = b0; b < b1; ++b) {
    const int g = groups_of(prefix[b + 1], q_len, p, chunk);
    sum += g;
    mx = max(mx, g);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  total = sum;
  most = mx;
}

// Replaces the staged lengths by the prefix at split size `chunk` and finds
// the sequence that holds work group `first_group`.
__device__ __forceinline__ WorkPrefix build_prefix(const DecodeParams& p, int q_len, int chunk,
                                                   int* prefix, int lane, int first_group) {
  int b0, b1;
  lane_range(p, lane, b0, b1);
  int sum = 0;
#pragma unroll 1
  for (int b = b0; b < b1; ++b) sum += groups_of(prefix[b + 1], q_len, p, chunk);
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - sum;
  int fb = -1, fl = 0;
#pragma unroll 1
  for (int b = b0; b < b1; ++b) {
    const int Lb = prefix[b + 1];
    const int before = run;
    run += groups_of(Lb, q_len, p, chunk);
    if (before <= first_group && first_group < run) {
      fb = b;
      fl = Lb;
    }
    prefix[b + 1] = run;
  }
  WorkPrefix w{__shfl_sync(0xffffffffu, incl, 31), -1, 0};
  const unsigned own = __ballot_sync(0xffffffffu, fb >= 0);
  if (own) {
    const int src = __ffs(own) - 1;
    w.first_b = __shfl_sync(0xffffffffu, fb, src);
    w.first_len = __shfl_sync(0xffffffffu, fl, src);
  }
  if (lane == 0) prefix[0] = 0;
  __syncwarp();   // the prefix is complete for the whole warp
  return w;
}

// Byte offset inside a 1024-byte-aligned tile written by TMA with 128-byte
// (D = 128) or 64-byte (D = 64) swizzle: 16-byte chunk index XOR line bits.
template <int D>
__device__ __forceinline__ uint32_t swz(uint32_t off) {
  constexpr uint32_t mask = (D == 128) ? 7u : 3u;
  return off ^ (((off >> 7) & mask) << 4);
}

// Bounded barrier among the four consumer warps (one arrival per warp).
__device__ __forceinline__ bool consumer_sync(uint64_t* bar, uint32_t& parity, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  const bool ok = mbar_wait_bounded(bar, parity, kWaitLimitNs);
  parity ^= 1u;
  return __all_sync(0xffffffffu, ok);
}

// Key ranges of a boundary tile's columns.  With several queries per sequence
// column c of the MMA N side is query position qpos0 + c / g (head c % g); it
// sees the item's tokens [tok_lo, tok_hi) up to its own position and, under a
// window, from `window` tokens before it.  Columns c >= ncols are padding and
// keep the item's range.  With one query every column has the item's range.
struct TileMask {
  int tok_lo, tok_hi, qpos0, window, lg, ncols;
};

// MQ: several query tokens per sequence (columns are (position, head) pairs
// with per-column key ranges); otherwise one query and columns are heads.
// FP4: the stage holds NVFP4 rows (E2M1 pairs and E4M3 block scales, no
// swizzle; the warp's 16 rows start at the pointers passed to tile());
// otherwise E4M3 rows in the swizzled TMA layout.
template <int D, int NT, bool MQ, bool FP4 = false>
struct Consumer {
  static constexpr int KS = D / 16;   // k-steps of the QK MMA
  static constexpr int MT = D / 16;   // m-tiles of the PV MMA
  static constexpr int QW = D / 4;    // contiguous q elements per thread

  uint32_t koff[D / 64];    // swizzled byte offsets of this thread's K reads (row n)
  uint32_t voff[2];         // swizzled byte offsets of its V reads (rows 2t, 2t + 1)
  // Q^T B fragments (f16x2), head = lane / 4 of n-tile: in registers, or (QSM)
  // in this warp's shared-memory area qs, [nt][ks][lane][2]
  static constexpr bool QSM = qfrag_in_smem(D, NT);
  uint32_t qf[QSM ? 1 : NT][QSM ? 1 : KS][2];
  uint32_t* qs;
  float cs[NT][2];          // logit scale (log2) of this thread's C columns
  float m[NT][2];           // running max (log2 domain) of this thread's columns
  float thr[NT][2];         // raw-accumulator threshold that triggers a rescale
  float l[NT][2];           // partial row sums (this thread's tokens only)
  float o[MT][NT][4];       // O^T accumulators

  // Shared-memory read offsets inside a stage tile; the same for every stage.
  // Rows r and r + 8 share the swizzle phase (it depends on r mod 8), so the
  // second row of each pair is the first plus 8 * D.
  __device__ __forceinline__ void setup(int row0, int lane) {
    const int n = lane >> 2, t = lane & 3;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) koff[c] = swz<D>((row0 + n) * D + t * (D / 4) + 16 * c);
    voff[0] = swz<D>((row0 + 2 * t) * D + n * (D / 8));
    voff[1] = swz<D>((row0 + 2 * t + 1) * D + n * (D / 8));
  }

  // qbase: the item's query rows in shared memory, bf16 [position][rows_per_pos][D];
  // column c (query position c / g, head c % g) is row
  // (c / g) * rows_per_pos + w_off + c % g.
  // qk_scale: the logit scale in the log2 domain (sm_scale * k_scale * log2 e).
  __device__ __forceinline__ void init(const DecodeParams& p, float qk_scale,
                                       const __nv_bfloat16* qbase, int rows_per_pos, int w_off,
                                       int ncols, int lane) {
    const int n = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = nt * 8 + n;
      float vals[QW];
      float amax = 0.f;
      if (c < (MQ ? ncols : p.g)) {
        const int qrow = MQ ? (c >> p.lg) * rows_per_pos + w_off + (c & (p.g - 1)) : w_off + c;
        const __nv_bfloat16* src = qbase + qrow * D + t * QW;
        if (p.q_f16) {   // fp16 query: the same 16-bit rows, another decoding
#pragma unroll
          for (int i = 0; i < QW; i += 8) {
            const uint4 raw = *reinterpret_cast<const uint4*>(src + i);
            const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 f = __half22float2(h2[j]);
              vals[i + 2 * j] = f.x;
              vals[i + 2 * j + 1] = f.y;
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < QW; i += 8) {
            const uint4 raw = *reinterpret_cast<const uint4*>(src + i);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 f = __bfloat1622float2(h2[j]);
              vals[i + 2 * j] = f.x;
              vals[i + 2 * j + 1] = f.y;
            }
          }
        }
#pragma unroll
        for (int i = 0; i < QW; ++i) amax = fmaxf(amax, fabsf(vals[i]));
      } else {
#pragma unroll
        for (int i = 0; i < QW; ++i) vals[i] = 0.f;
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      // Power-of-two prescale so the largest |q| of the head sits in [2^14, 2^15):
      // keeps bf16 -> f16 exact for any bf16 magnitude (and fp16 exact, down to
      // 2^-24 of the largest element); undone in the logit scale.
      int e = 0;
      if (amax > 0.f && isfinite(amax)) frexpf(amax, &e);
      const int sh = max(-126, min(126, 15 - e));
      const float fac = ldexpf(1.0f, sh);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const uint32_t w0 = pack_f16x2(vals[4 * ks] * fac, vals[4 * ks + 1] * fac);
        const uint32_t w1 = pack_f16x2(vals[4 * ks + 2] * fac, vals[4 * ks + 3] * fac);
        if constexpr (QSM) {
          *reinterpret_cast<uint2*>(qs + ((nt * KS + ks) * 32 + lane) * 2) = make_uint2(w0, w1);
        } else {
          qf[nt][ks][0] = w0;
          qf[nt][ks][1] = w1;
        }
      }
      // this thread's C columns are columns 2t and 2t+1 of the n-tile; the
      // prescale is a power of two, so undoing it is an exact multiply
      const int sh0 = __shfl_sync(0xffffffffu, sh, (2 * t) * 4);
      const int sh1 = __shfl_sync(0xffffffffu, sh, (2 * t + 1) * 4);
      cs[nt][0] = qk_scale * ldexpf(1.0f, -sh0);
      cs[nt][1] = qk_scale * ldexpf(1.0f, -sh1);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        m[nt][j] = -INFINITY;
        thr[nt][j] = -INFINITY;
        l[nt][j] = 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[i][nt][j] = 0.f;
  }

  // One 16-row slice of a stage.  FULL: every row is inside every column's
  // range; otherwise rows are masked per column (mk).
  // NVFP4 K fragments of rows n and n + 8 (this thread's elements
  // [t*D/4, (t+1)*D/4) of each, D/8 bytes of E2M1 pairs) as f16x2 words in the
  // E4M3 path's order: word 2ks = elements 4ks, 4ks+1; word 2ks+1 = 4ks+2, 4ks+3.
  // Each value is the E2M1 code times its block's E4M3 scale, exact in f16.
  __device__ __forceinline__ void fp4_k_frags(const uint8_t* Kd, const uint8_t* Ks, int lane,
                                              uint32_t (&kh)[2][D / 8]) {
    const int n = lane >> 2, t = lane & 3;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = n + 8 * r;
      uint32_t w[D / 32];
      if constexpr (D == 128) {
        const uint4 v = *reinterpret_cast<const uint4*>(Kd + row * (D / 2) + t * 16);
        w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(Kd + row * (D / 2) + t * 8);
        w[0] = v.x, w[1] = v.y;
      }
      // block scales of this thread's elements: D/64 blocks of 16
      uint32_t sc[D / 64];
      if constexpr (D == 128) {
        const uint32_t s2 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(Ks + row * (D / 16) + 2 * t));
        sc[0] = prmt(s2, s2, 0x1010u);
        sc[1] = prmt(s2, s2, 0x3232u);
      } else {
        const uint32_t s2 = e4m3x2_to_f16x2((uint16_t)Ks[row * (D / 16) + t]);
        sc[0] = prmt(s2, s2, 0x1010u);
      }
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        uint32_t h[4];
        e2m1x8_to_f16x2x4(w[i], h);
#pragma unroll
        for (int j = 0; j < 4; ++j) kh[r][4 * i + j] = hmul2(h[j], sc[(4 * i + j) / 8]);
      }
    }
  }

  // NVFP4 V for the PV MMA: token pairs (2t, 2t+1) and (2t+8, 2t+9), this
  // thread's elements [n*D/8, (n+1)*D/8) (D/16 bytes and one block scale per
  // row).  vp[pr][e] = f16x2(element e of the pair's first token, of its
  // second token), scaled, and zeroed for tokens outside [tok_lo, tok_hi)
  // when not FULL.  The two tokens' codes are interleaved nibble by nibble
  // before the conversion, so one cvt gives the MMA's token pair directly.
  // Lanes alternate which token of a pair they load first so that every load
  // spreads over all the banks (rows 0, 2, 4, 6 alone would share half).
  template <bool FULL>
  __device__ __forceinline__ void fp4_v_pairs(const uint8_t* Vd, const uint8_t* Vs, int tok0,
                                              const TileMask& mk, int lane,
                                              uint32_t (&vp)[2][D / 8]) {
    const int n = lane >> 2, t = lane & 3;
    const int swap = D == 128 ? (t & 1) : (t >> 1);
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const int rowA = 2 * t + 8 * pr;
      const int r0 = rowA + swap, r1 = rowA + 1 - swap;
      uint32_t x[D / 64], y[D / 64], wa[D / 64], wb[D / 64];
      if constexpr (D == 128) {
        const uint2 u = *reinterpret_cast<const uint2*>(Vd + r0 * (D / 2) + n * 8);
        const uint2 v = *reinterpret_cast<const uint2*>(Vd + r1 * (D / 2) + n * 8);
        x[0] = u.x, x[1] = u.y, y[0] = v.x, y[1] = v.y;
      } else {
        x[0] = *reinterpret_cast<const uint32_t*>(Vd + r0 * (D / 2) + n * 4);
        y[0] = *reinterpret_cast<const uint32_t*>(Vd + r1 * (D / 2) + n * 4);
      }
#pragma unroll
      for (int w = 0; w < D / 64; ++w) {
        wa[w] = swap ? y[w] : x[w];
        wb[w] = swap ? x[w] : y[w];
      }
      const int blk = D == 128 ? n : n / 2;   // the block of this thread's elements
      const uint16_t sab = (uint16_t)(Vs[rowA * (D / 16) + blk] |
                                      (Vs[(rowA + 1) * (D / 16) + blk] << 8));
      const uint32_t sc = e4m3x2_to_f16x2(sab);   // (scale of token A, of token B)
      uint32_t mask = 0xffffffffu;
      if (!FULL) {
        const int ta = tok0 + rowA;
        mask = ((ta >= mk.tok_lo && ta < mk.tok_hi) ? 0x0000ffffu : 0u) |
               ((ta + 1 >= mk.tok_lo && ta + 1 < mk.tok_hi) ? 0xffff0000u : 0u);
      }
#pragma unroll
      for (int w = 0; w < D / 64; ++w) {
        // byte j of lo: element 8w+2j of A (low nibble) and of B; hi: 8w+2j+1
        const uint32_t lo = (wa[w] & 0x0F0F0F0Fu) | ((wb[w] << 4) & 0xF0F0F0F0u);
        const uint32_t hi = ((wa[w] >> 4) & 0x0F0F0F0Fu) | (wb[w] & 0xF0F0F0F0u);
        uint32_t L[4], H[4];
        e2m1x8_to_f16x2x4(lo, L);
        e2m1x8_to_f16x2x4(hi, H);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          vp[pr][8 * w + 2 * k] = hmul2(L[k], sc) & mask;
          vp[pr][8 * w + 2 * k + 1] = hmul2(H[k], sc) & mask;
        }
      }
    }
  }

  template <bool FULL>
  __device__ __forceinline__ void tile(const uint8_t* Kt, const uint8_t* Vt, int row0, int tok0,
                                       const TileMask& mk, int lane,
                                       const uint8_t* Ks = nullptr, const uint8_t* Vs = nullptr) {
    const int n = lane >> 2, t = lane & 3;
    // ---- K fragments: rows row0 + n and row0 + n + 8, bytes [t*D/4, (t+1)*D/4)
    uint32_t kw[2][FP4 ? 1 : D / 16];
    uint32_t kh[2][FP4 ? D / 8 : 1];
    if constexpr (FP4) {
      fp4_k_frags(Kt, Ks, lane, kh);
    } else {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(Kt + koff[c] + r * 8 * D);
        kw[r][4 * c + 0] = v.x;
        kw[r][4 * c + 1] = v.y;
        kw[r][4 * c + 2] = v.z;
        kw[r][4 * c + 3] = v.w;
      }
    }
    }
    // ---- S^T = K Q^T, two accumulation chains per n-tile
    float s[NT][2][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[nt][c][j] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a0, a1, a2, a3;
      if constexpr (FP4) {
        a0 = kh[0][2 * ks], a2 = kh[0][2 * ks + 1];
        a1 = kh[1][2 * ks], a3 = kh[1][2 * ks + 1];
      } else {
        e4m3x4_to_f16x2x2(kw[0][ks], a0, a2);
        e4m3x4_to_f16x2x2(kw[1][ks], a1, a3);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
      {
        uint32_t b0, b1;
        if constexpr (QSM) {
          const uint2 w = *reinterpret_cast<const uint2*>(qs + ((nt * KS + ks) * 32 + lane) * 2);
          b0 = w.x, b1 = w.y;
        } else {
          b0 = qf[nt][ks][0], b1 = qf[nt][ks][1];
        }
        mma_16816(s[nt][ks & 1], a0, a1, a2, a3, b0, b1);
      }
    }
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[nt][j] = s[nt][0][j] + s[nt][1][j];

    if constexpr (!FULL && MQ) {
      const int tk0 = tok0 + n, tk1 = tok0 + n + 8;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int c = nt * 8 + 2 * t + j;
          int lo = mk.tok_lo, hi = mk.tok_hi;
          if (c < mk.ncols) {
            const int pos = mk.qpos0 + (c >> mk.lg);   // this column's query position
            hi = min(hi, pos + 1);
            if (mk.window >= 0) lo = max(lo, pos - mk.window);
          }
          if (!(tk0 >= lo && tk0 < hi)) acc[nt][j] = -INFINITY;
          if (!(tk1 >= lo && tk1 < hi)) acc[nt][j + 2] = -INFINITY;
        }
      }
    } else if constexpr (!FULL) {
      const int tk0 = tok0 + n, tk1 = tok0 + n + 8;
      const bool v0 = tk0 >= mk.tok_lo && tk0 < mk.tok_hi;
      const bool v1 = tk1 >= mk.tok_lo && tk1 < mk.tok_hi;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (!v0) acc[nt][0] = acc[nt][1] = -INFINITY;
        if (!v1) acc[nt][2] = acc[nt][3] = -INFINITY;
      }
    }

    // ---- lazy running max
    bool need = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        need |= (acc[nt][j] > thr[nt][j]) || (acc[nt][j + 2] > thr[nt][j]);
    if (__any_sync(0xffffffffu, need)) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float tmax = fmaxf(acc[nt][j], acc[nt][j + 2]);
          tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
          tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
          tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
          const float smax = tmax * cs[nt][j];
          if (smax > m[nt][j] + kLazyThreshold) {
            const float alpha = fast_exp2(m[nt][j] - smax);  // 0 on the first tile
            m[nt][j] = smax;
            thr[nt][j] = (smax + kLazyThreshold) / cs[nt][j];
            l[nt][j] *= alpha;
#pragma unroll
            for (int i = 0; i < MT; ++i) {
              o[i][nt][j] *= alpha;
              o[i][nt][j + 2] *= alpha;
            }
          }
        }
      }
    }

    // ---- probabilities (fp32 sums; f16 copies feed the PV MMA)
    uint32_t pb0[NT], pb1[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float p0 = fast_exp2(fmaf(acc[nt][0], cs[nt][0], -m[nt][0]));
      float p1 = fast_exp2(fmaf(acc[nt][1], cs[nt][1], -m[nt][1]));
      float p2 = fast_exp2(fmaf(acc[nt][2], cs[nt][0], -m[nt][0]));
      float p3 = fast_exp2(fmaf(acc[nt][3], cs[nt][1], -m[nt][1]));
      if (!FULL && MQ) {   // a column with no key yet: every logit and its max are -inf
        if (m[nt][0] == -INFINITY) p0 = p2 = 0.f;
        if (m[nt][1] == -INFINITY) p1 = p3 = 0.f;
      }
      l[nt][0] += p0 + p2;
      l[nt][1] += p1 + p3;
      pb0[nt] = movmatrix_trans(pack_f16x2(p0, p1));   // tokens 2t..2t+1, head n
      pb1[nt] = movmatrix_trans(pack_f16x2(p2, p3));   // tokens 2t+8..2t+9, head n
    }

    if constexpr (FP4) {
      // ---- O^T += V^T P^T from NVFP4 rows: m-tile i takes element 2i (M row n)
      // and 2i+1 (M row n + 8) of this thread's chunk for both token pairs
      uint32_t vp[2][D / 8];
      fp4_v_pairs<FULL>(Vt, Vs, tok0, mk, lane, vp);
#pragma unroll
      for (int i = 0; i < MT; ++i) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816(o[i][nt], vp[0][2 * i], vp[0][2 * i + 1], vp[1][2 * i], vp[1][2 * i + 1],
                    pb0[nt], pb1[nt]);
      }
      return;
    } else {
    // ---- V fragments: token rows 2t, 2t+1, 2t+8, 2t+9; head-dim chunk n
    constexpr int VB = D / 8;  // bytes of one row this thread needs
    uint32_t va[VB / 4], vb[VB / 4], vc[VB / 4], vd[VB / 4];
    if constexpr (D == 128) {
      const uint4 A = *reinterpret_cast<const uint4*>(Vt + voff[0]);
      const uint4 B = *reinterpret_cast<const uint4*>(Vt + voff[1]);
      const uint4 C = *reinterpret_cast<const uint4*>(Vt + voff[0] + 8 * D);
      const uint4 E = *reinterpret_cast<const uint4*>(Vt + voff[1] + 8 * D);
      va[0] = A.x; va[1] = A.y; va[2] = A.z; va[3] = A.w;
      vb[0] = B.x; vb[1] = B.y; vb[2] = B.z; vb[3] = B.w;
      vc[0] = C.x; vc[1] = C.y; vc[2] = C.z; vc[3] = C.w;
      vd[0] = E.x; vd[1] = E.y; vd[2] = E.z; vd[3] = E.w;
    } else {
      const uint2 A = *reinterpret_cast<const uint2*>(Vt + voff[0]);
      const uint2 B = *reinterpret_cast<const uint2*>(Vt + voff[1]);
      const uint2 C = *reinterpret_cast<const uint2*>(Vt + voff[0] + 8 * D);
      const uint2 E = *reinterpret_cast<const uint2*>(Vt + voff[1] + 8 * D);
      va[0] = A.x; va[1] = A.y;
      vb[0] = B.x; vb[1] = B.y;
      vc[0] = C.x; vc[1] = C.y;
      vd[0] = E.x; vd[1] = E.y;
    }
    if (!FULL) {
      // Zero value rows outside the item's range: stale bytes may hold NaN
      // codes and 0 * NaN would poison the accumulator.
      const int tok_lo = mk.tok_lo, tok_hi = mk.tok_hi;
      const int tA = tok0 + 2 * t;
      const uint32_t mA = (tA >= tok_lo && tA < tok_hi) ? 0xffffffffu : 0u;
      const uint32_t mB = (tA + 1 >= tok_lo && tA + 1 < tok_hi) ? 0xffffffffu : 0u;
      const uint32_t mC = (tA + 8 >= tok_lo && tA + 8 < tok_hi) ? 0xffffffffu : 0u;
      const uint32_t mD = (tA + 9 >= tok_lo && tA + 9 < tok_hi) ? 0xffffffffu : 0u;
#pragma unroll
      for (int w = 0; w < VB / 4; ++w) {
        va[w] &= mA;
        vb[w] &= mB;
        vc[w] &= mC;
        vd[w] &= mD;
      }
    }
    // ---- O^T += V^T P^T
#pragma unroll
    for (int w = 0; w < VB / 4; ++w) {
      const uint32_t ab_lo = prmt(va[w], vb[w], 0x5140u);  // d byte 0,1: {A,B} pairs
      const uint32_t ab_hi = prmt(va[w], vb[w], 0x7362u);  // d byte 2,3
      const uint32_t cd_lo = prmt(vc[w], vd[w], 0x5140u);
      const uint32_t cd_hi = prmt(vc[w], vd[w], 0x7362u);
      uint32_t a0, a1, a2, a3;
      e4m3x4_to_f16x2x2(ab_lo, a0, a1);
      e4m3x4_to_f16x2x2(cd_lo, a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816(o[2 * w][nt], a0, a1, a2, a3, pb0[nt], pb1[nt]);
      e4m3x4_to_f16x2x2(ab_hi, a0, a1);
      e4m3x4_to_f16x2x2(cd_hi, a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        mma_16816(o[2 * w + 1][nt], a0, a1, a2, a3, pb0[nt], pb1[nt]);
    }
    }
  }
  // HB = 4: this warp alone covered KV head `kvh` of the item, so its query
  // heads are finished straight from registers.  Thread (n, t) holds, for
  // column nt*8 + 2t + j, the D/8 output elements starting at n*D/8.  The
  // item's columns are queries qrow0 .. qrow0 + ncols / g - 1 of the sequence.
  __device__ __forceinline__ void finish_own(const DecodeParams& p, float v_scale, int b, int kvh,
                                             int split, int ns, int qrow0, int ncols, int lane) {
    constexpr int E = D / 8;   // output elements per thread and query head
    const int n = lane >> 2, t = lane & 3;
    float lsum[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float v = l[nt][j];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        lsum[nt][j] = v;
      }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = nt * 8 + 2 * t + j;   // column: query position c / g, head c % g
        if (c >= (MQ ? ncols : p.g)) continue;
        const int hq = kvh * p.g + (MQ ? c & (p.g - 1) : c);
        const size_t tok = MQ ? (size_t)b * p.q_len + qrow0 + (c >> p.lg) : (size_t)b;
        const size_t row = tok * p.Hq + hq;
        __nv_bfloat16* const orow = p.out + tok * p.out_tok_stride + (size_t)hq * D;
        // false: this query saw no key in the item (only possible with MQ)
        const bool keys = !MQ || lsum[nt][j] > 0.f;
        const bool one = ns == 1 && !p.combine_all;   // finished here, not by the combine
        if (ns == 0 || (one && !keys)) {  // no key at all: out = 0, lse = sigma
          if (p.combine_all) continue;    // the combine writes the row
          uint4* dst = reinterpret_cast<uint4*>(orow + n * E);
#pragma unroll
          for (int k = 0; k < E / 8; ++k) dst[k] = make_uint4(0u, 0u, 0u, 0u);
          if (n == 0 && p.lse) p.lse[row] = p.sinks ? p.sinks[hq] : -INFINITY;
          continue;
        }
        const float lse2 = m[nt][j] + __log2f(lsum[nt][j]);   // log2-sum-exp, no sink
        if (one) {
          float scale = v_scale;
          float lse_out = lse2;
          if (p.sinks) {
            const float sg = p.sinks[hq] * kLog2e;
            const float Mx = fmaxf(lse2, sg);
            const float wsplit = fast_exp2(lse2 - Mx);
            const float Z = wsplit + fast_exp2(sg - Mx);
            scale *= __fdividef(wsplit, Z);
            lse_out = Mx + __log2f(Z);
          }
          const float inv = __fdividef(scale, lsum[nt][j]);
          uint32_t w[MT];
#pragma unroll
          for (int i = 0; i < MT; ++i) w[i] = pack_bf16x2(o[i][nt][j] * inv, o[i][nt][j + 2] * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + n * E);
#pragma unroll
          for (int k = 0; k < E / 8; ++k)
            dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          if (n == 0 && p.lse) p.lse[row] = lse_out * kLn2;
        } else {
          const size_t prow = row * p.max_splits + split;
          const float inv = keys ? __fdividef(1.0f, lsum[nt][j]) : 0.f;   // no key: O = 0
          float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D + n * E);
#pragma unroll
          for (int k = 0; k < E / 4; ++k)
            dst[k] = make_float4(o[2 * k][nt][j] * inv, o[2 * k][nt][j + 2] * inv,
                                 o[2 * k + 1][nt][j] * inv, o[2 * k + 1][nt][j + 2] * inv);
          if (n == 0) p.part_lse[prow] = keys ? lse2 : -INFINITY;
        }
      }
    }
  }
};

// ---------------------------------------------------------------- producer --

// FP4: NVFP4 pages, four tensors per stage (kmap / vmap the E2M1 data, ksmap /
// vsmap the block scales); otherwise E4M3 pages (kmap / vmap).
template <int D, int HB, bool MQ, bool FP4>
__device__ __forceinline__ void producer_loop(const CUtensorMap* kmap, const CUtensorMap* vmap,
                                              const CUtensorMap* ksmap, const CUtensorMap* vsmap,
                                              const DecodeParams& p, uint8_t* smem,
                                              const SmemLayout& L, const int* prefix,
                                              int chunk, int total_items, int hslot_bytes,
                                              uint64_t* full_bar, uint64_t* empty_bar,
                                              uint64_t* hdr_full, uint64_t* hdr_empty, int lane,
                                              WorkPrefix first) {
  constexpr int kTileBytes = kTileTokens * D;
  constexpr int kStage = stage_bytes(D, FP4);
  constexpr int kDataBytes = fp4_data_bytes(D);   // NVFP4 regions of a stage
  constexpr int kSfBytes = fp4_sf_bytes(D);
  constexpr int kStageTokens = kTileTokens / HB;   // tokens of one KV head per stage
  const int stages = p.stages;
  const int n_hslots = p.hdr_slots;
  const int QL = MQ ? p.q_len : 1;                 // query tokens per sequence
  const int QC = MQ ? p.q_chunks : 1;              // query chunks per (group, KV head group)
  const int groups = p.Hkv / HB;                   // KV head groups
  const int pps = HB == 1 ? kStageTokens / p.bt : 1;   // pages per stage (HB = 1)
  const uint32_t page_bytes = (uint32_t)(p.bt * D);
  const uint64_t policy = l2_policy_evict_first();
  if (lane == 0) {
    tma_prefetch_desc(kmap);
    tma_prefetch_desc(vmap);
    if constexpr (FP4) {
      tma_prefetch_desc(ksmap);
      tma_prefetch_desc(vsmap);
    }
  }
  int hs = 0;
  int hslot = 0;
  uint32_t hphase = 0;        // use count of the current header slot, mod 2
  int slot = 0, issued = 0;   // ring position and stages issued so far
  uint32_t phase = 0;         // use count of the current slot, mod 2
  // The first item of every CTA is its own index; later ones come from the
  // shared counter (offset by the grid size).
  uint32_t item = blockIdx.x;
  for (;;) {
    const bool done = item >= (uint32_t)total_items;
    if (hs >= n_hslots) {
      const bool ok = mbar_wait_bounded(&hdr_empty[hslot], hphase ^ 1u, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) atomicOr(p.status, kErrTimeout);
        return;
      }
    }
    uint8_t* hbase = smem + L.hdr + hslot * hslot_bytes;
    ItemHeader* hdr = reinterpret_cast<ItemHeader*>(hbase);
    if (done) {
      if (lane == 0) {
        hdr->kind = -1;
        mbar_arrive(&hdr_full[hslot]);
      }
      return;
    }
    // item -> (group, kv head group, query chunk) -> (sequence, split) by
    // binary search.  The query chunks of one KV range are consecutive items,
    // so they run at about the same time and share the pages in L2.
    const int unit = MQ ? div_pos((int)item, QC) : (int)item;
    const int qc = MQ ? (int)item - unit * QC : 0;
    const int group = div_pos(unit, groups);
    const int kvh0 = (unit - group * groups) * HB;
    int b = first.first_b;   // the first item's sequence came with the prefix
    if (hs > 0) {
      int lo = 0, hi = p.B;   // largest b with prefix[b] <= group
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= group) lo = mid; else hi = mid;
      }
      b = lo;
    }
    const int split = group - prefix[b];
    const SeqRange R = seq_range(hs > 0 ? __ldg(p.seq_lens + b) : first.first_len, QL, p.bt,
                                 p.max_blocks, p.window_left, chunk,
                                 lane == 0 ? p.status : nullptr);
    int pb = 0, pe = 0, tok_lo = 0, tok_hi = 0, t0 = 0, n_st = 0;
    if (R.n_splits > 0) {
      pb = R.first_page + split * chunk;
      pe = min(pb + chunk, R.end_page);
      tok_lo = max(R.start, pb * p.bt);
      tok_hi = min(R.L, pe * p.bt);
      if (HB == 1) {   // whole pages, pps per stage
        t0 = pb * p.bt;
        n_st = (pe - pb + pps - 1) / pps;
      } else {         // the 16-token blocks that touch [tok_lo, tok_hi)
        t0 = tok_lo & ~(kBoxTokens - 1);
        n_st = (tok_hi - t0 + kBoxTokens - 1) / kBoxTokens;
      }
    }
    if (lane == 0) {
      hdr->kind = 1;
      hdr->b = b;
      hdr->kvh0 = kvh0;
      hdr->split = split;
      hdr->ns = R.n_splits;
      hdr->n_stages = n_st;
      hdr->t0 = t0;
      hdr->tok_lo = tok_lo;
      hdr->tok_hi = tok_hi;
      const int qrow0 = MQ ? qc * p.q_per_item : 0;
      const int npos = MQ ? min(p.q_per_item, QL - qrow0) : 1;
      hdr->qpos0 = R.L - QL + qrow0;
      hdr->qrow0 = qrow0;
      hdr->npos = npos;
      // the query rows of the item's KV heads, one copy per query position:
      // [position][HB * g][D] in the slot
      const uint32_t qbytes = (uint32_t)(HB * p.g * D * 2);
      mbar_arrive_expect_tx(&hdr_full[hslot], qbytes * (uint32_t)npos);
      for (int i = 0; i < npos; ++i)
        bulk_load(hbase + kHdrBytes + (size_t)i * qbytes,
                  p.q + ((size_t)b * QL + qrow0 + i) * p.q_tok_stride + (size_t)kvh0 * p.g * D,
                  qbytes, &hdr_full[hslot]);
    }
    ++hs;
    if (++hslot == n_hslots) {
      hslot = 0;
      hphase ^= 1u;
    }

    // the next item: fetched once this item's first loads are on their way
    // (its latency is hidden behind the item's stages)
    uint32_t next = 0;
    bool fetched = false;

    // ---- stream the item's KV; block-table entries 32 at a time
    const int32_t* tbl = p.block_table + (size_t)b * p.max_blocks;
    int batch_base = -1, my_entry = 0;
    for (int s = 0; s < n_st; ++s) {
      if (issued >= stages) {   // wait for the consumers to release the previous use
        const bool ok = mbar_wait_bounded(&empty_bar[slot], phase ^ 1u, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) atomicOr(p.status, kErrTimeout);
          return;
        }
      }
      uint8_t* stage = smem + L.ring + slot * kStage;
      if constexpr (FP4 && HB == 1) {
        // NVFP4, one head: per page four boxes (K data, K scales, V data, V
        // scales), lane 4q + r for page q of the stage
        const int pg0 = pb + s * pps;
        const int np = min(pps, pe - pg0);
        const int rel = pg0 - pb;
        if ((rel & ~31) != batch_base) {
          batch_base = rel & ~31;
          const int idx = pb + batch_base + lane;
          my_entry = (idx < pe) ? __ldg(tbl + idx) : 0;
        }
        const int e = __shfl_sync(0xffffffffu, my_entry, (rel + (lane >> 2)) & 31);
        const bool mine = lane < 4 * np;
        const bool ok = (e >= 0 && e < p.num_blocks);
        if (mine && !ok && (lane & 3) == 0) atomicOr(p.status, kErrBlockTable);
        if (lane == 0)
          mbar_arrive_expect_tx(&full_bar[slot],
                                (uint32_t)(np * p.bt * (D / 2 + D / 16) * 2));
        __syncwarp();
        if (mine) {
          // an invalid page is read from past the end of the pool: TMA zero-fills it
          const int page = ok ? e : p.num_blocks;
          const int q = lane >> 2, r = lane & 3;
          if (r == 0 || r == 2)   // data: (d pair, slot, kv head, page)
            tma_load_4d(stage + (r == 0 ? 0 : kDataBytes + kSfBytes) + q * p.bt * (D / 2),
                        r == 0 ? kmap : vmap, 0, 0, kvh0, page, &full_bar[slot], policy);
          else                    // scales: (16-token group scales, group, kv head, page)
            tma_load_4d(stage + (r == 1 ? kDataBytes : 2 * kDataBytes + kSfBytes) +
                            q * fp4_sf_pitch(p.bt, D),
                        r == 1 ? ksmap : vsmap, 0, 0, kvh0, page, &full_bar[slot], policy);
        }
      } else if constexpr (FP4) {
        // NVFP4, 16 tokens of 4 heads: lanes 0..3 load K data, K scales, V
        // data, V scales of the block
        const int tok = t0 + s * kBoxTokens;
        const int rel = div_pos(tok, p.bt) - pb;
        if ((rel & ~31) != batch_base) {
          batch_base = rel & ~31;
          const int idx = pb + batch_base + lane;
          my_entry = (idx < pe) ? __ldg(tbl + idx) : 0;
        }
        const int e = __shfl_sync(0xffffffffu, my_entry, rel & 31);
        const bool ok = (e >= 0 && e < p.num_blocks);
        if (lane == 0) {
          if (!ok) atomicOr(p.status, kErrBlockTable);
          mbar_arrive_expect_tx(&full_bar[slot], (uint32_t)fp4_stage_payload(D));
        }
        __syncwarp();
        if (lane < 4) {
          const int page = ok ? e : p.num_blocks;
          const int in_page = tok - (rel + pb) * p.bt;   // first slot of the block in its page
          if (lane == 0 || lane == 2)
            tma_load_4d(stage + (lane == 0 ? 0 : kDataBytes + kSfBytes), lane == 0 ? kmap : vmap,
                        0, in_page, kvh0, page, &full_bar[slot], policy);
          else
            tma_load_4d(stage + (lane == 1 ? kDataBytes : 2 * kDataBytes + kSfBytes),
                        lane == 1 ? ksmap : vsmap, 0, in_page / kBoxTokens, kvh0, page,
                        &full_bar[slot], policy);
        }
      } else if constexpr (HB == 1) {
        const int pg0 = pb + s * pps;
        const int np = min(pps, pe - pg0);
        const int rel = pg0 - pb;
        if ((rel & ~31) != batch_base) {
          batch_base = rel & ~31;
          const int idx = pb + batch_base + lane;
          my_entry = (idx < pe) ? __ldg(tbl + idx) : 0;
        }
        // One lane per (page, K or V) box; the boxes are issued side by side.
        const int e = __shfl_sync(0xffffffffu, my_entry, (rel + (lane >> 1)) & 31);
        const bool mine = lane < 2 * np;
        const bool ok = (e >= 0 && e < p.num_blocks);
        if (mine && !ok && (lane & 1) == 0) atomicOr(p.status, kErrBlockTable);
        if (lane == 0) mbar_arrive_expect_tx(&full_bar[slot], 2u * page_bytes * (uint32_t)np);
        __syncwarp();
        if (mine) {
          // an invalid page is read from past the end of the pool: TMA zero-fills it
          uint8_t* dst = stage + (lane & 1) * kTileBytes + (lane >> 1) * page_bytes;
          const CUtensorMap* map = (lane & 1) ? vmap : kmap;
          if (p.kv_hnd)   // (d, slot, kv head, page)
            tma_load_4d(dst, map, 0, 0, kvh0, ok ? e : p.num_blocks, &full_bar[slot], policy);
          else            // (d, kv head, token row)
            tma_load_3d(dst, map, 0, kvh0, ok ? e * p.bt : p.num_blocks * p.bt, &full_bar[slot],
                        policy);
        }
      } else {
        // 16 tokens of HB heads: one box per tensor, lane 0 K and lane 1 V
        const int tok = t0 + s * kBoxTokens;
        const int rel = div_pos(tok, p.bt) - pb;
        if ((rel & ~31) != batch_base) {
          batch_base = rel & ~31;
          const int idx = pb + batch_base + lane;
          my_entry = (idx < pe) ? __ldg(tbl + idx) : 0;
        }
        const int e = __shfl_sync(0xffffffffu, my_entry, rel & 31);
        const bool ok = (e >= 0 && e < p.num_blocks);
        if (lane == 0) {
          if (!ok) atomicOr(p.status, kErrBlockTable);
          mbar_arrive_expect_tx(&full_bar[slot], 2u * kTileBytes);
        }
        __syncwarp();
        if (lane < 2) {
          // an invalid page is read from past the end of the pool: TMA zero-fills it
          const int in_page = tok - (rel + pb) * p.bt;   // first slot of the block in its page
          const CUtensorMap* map = lane ? vmap : kmap;
          if (p.kv_hnd)   // (d, slot, kv head, page)
            tma_load_4d(stage + lane * kTileBytes, map, 0, in_page, kvh0, ok ? e : p.num_blocks,
                        &full_bar[slot], policy);
          else            // (d, token row, kv head)
            tma_load_3d(stage + lane * kTileBytes, map, 0,
                        (ok ? e * p.bt : p.num_blocks * p.bt) + in_page, kvh0, &full_bar[slot],
                        policy);
        }
      }
      ++issued;
      if (++slot == stages) {
        slot = 0;
        phase ^= 1u;
      }
      if (!fetched) {
        if (lane == 0) next = gridDim.x + atomicAdd(&p.sched[0], 1u);
        fetched = true;
      }
    }
    if (!fetched && lane == 0) next = gridDim.x + atomicAdd(&p.sched[0], 1u);
    item = __shfl_sync(0xffffffffu, next, 0);
  }
}

// ------------------------------------------------------------------ kernel --

// CTAs per SM the register budget is sized for (register cap 64K / (160 * n)).
#ifndef FPD_MINB_D128_NT1
#define FPD_MINB_D128_NT1 3
#endif
#ifndef FPD_MINB_D128_NT2
#define FPD_MINB_D128_NT2 2
#endif
template <int D, int NT>
struct MinBlocks {
  static constexpr int value =
      (D == 128) ? (NT == 1 ? FPD_MINB_D128_NT1 : FPD_MINB_D128_NT2) : (NT == 1 ? 4 : 3);
};

// The split kernel's body.  FP4: NVFP4 pages (kmap / vmap the E2M1 data,
// ksmap / vsmap the block scales); otherwise E4M3 pages (kmap / vmap).
template <int D, int NT, int HB, bool MQ, bool FP4>
__device__ __forceinline__ void split_body(const CUtensorMap* kmap, const CUtensorMap* vmap,
                                           const CUtensorMap* ksmap, const CUtensorMap* vsmap,
                                           const DecodeParams& p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int kTileBytes = kTileTokens * D;
  constexpr int kStage = stage_bytes(D, FP4);
  constexpr int kDataBytes = fp4_data_bytes(D);   // NVFP4 regions of a stage
  constexpr int kSfBytes = fp4_sf_bytes(D);
  constexpr int kStageTokens = kTileTokens / HB;
  constexpr int H = NT * 8;
  const int stages = p.stages;
  const int n_hslots = p.hdr_slots;
  // a header slot holds q_len * g query rows per KV head
  const int QL = MQ ? p.q_len : 1;   // query tokens per sequence
  const int QP = MQ ? p.q_per_item : 1;   // query positions per item
  const SmemLayout L = smem_layout(D, NT, HB, stages, n_hslots, QP * p.g, p.B, FP4);
  const int hslot_bytes = hdr_slot_bytes(D, HB, QP * p.g);
  int* prefix = reinterpret_cast<int*>(smem + L.prefix);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty_bar = full_bar + stages;
  uint64_t* hdr_full = empty_bar + stages;
  uint64_t* hdr_empty = hdr_full + kMaxHdrSlots;
  uint64_t* cbar = hdr_empty + kMaxHdrSlots;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // The launch may be a programmatic dependent of the previous kernel in the
  // stream (so that this grid's CTAs are resident when it finishes): nothing
  // is read before that kernel has completed and its writes are visible.
  // (The barriers live in this CTA's shared memory: they are set up while that
  // kernel may still run.)
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumerWarps);
    }
    for (int s = 0; s < kMaxHdrSlots; ++s) {
      mbar_init(&hdr_full[s], 1);
      mbar_init(&hdr_empty[s], kConsumerWarps);
    }
    mbar_init(cbar, kConsumerWarps);
    fence_mbarrier_init();
  }
  __syncthreads();   // the barriers are set up for every warp
  pdl_wait_primary();

  if (warp == kConsumerWarps) {
    // ---- the split size and the prefix over sequences of their work groups.
    // The plan may offer a larger split size for calls of a few rounds of
    // items: taken when the sequences are of about equal length (the longest
    // one's groups times B within 4/3 of all groups), since then its items,
    // one round of about two per SM, fill every SM alike; otherwise the
    // plan's size runs over the grid, sized for the larger items.  Every CTA
    // reaches the same choice from the same lengths.
    const int G = (p.Hkv / HB) * (MQ ? p.q_chunks : 1);   // items per work group
    int chunk = p.chunk_pages;
    stage_lengths(p, prefix, lane);
    if (p.adapt_chunk > 0) {
      int groups = 0, most = 0;
      length_totals(p, QL, chunk, prefix, lane, groups, most);
      if ((int64_t)groups * G > (int64_t)gridDim.x &&
          4 * (int64_t)groups >= 3 * (int64_t)p.B * most)
        chunk = p.adapt_chunk;
    }
    const WorkPrefix w = build_prefix(p, QL, chunk, prefix, lane, (int)blockIdx.x / G);
    if (blockIdx.x == 0 && lane == 0) p.sched[2] = (uint32_t)chunk;
    pdl_launch_dependents();   // the combine kernel may be scheduled from now on
    producer_loop<D, HB, MQ, FP4>(kmap, vmap, ksmap, vsmap, p, smem, L, prefix, chunk,
                                  w.total * G, hslot_bytes, full_bar, empty_bar, hdr_full,
                                  hdr_empty, lane, w);
    return;
  }
  pdl_launch_dependents();

  // -------------------------------------------------------------- consumers
  // scales: host values, or device words (readable now: the grid dependency
  // has resolved)
  const float qk_scale = p.k_scale_dev ? p.sm_scale_log2 * *p.k_scale_dev : p.qk_scale_log2;
  const float v_scale = p.v_scale_dev ? *p.v_scale_dev : p.v_scale;
  Consumer<D, NT, MQ, FP4> cw;
  const int n = lane >> 2, t = lane & 3;
  // HB = 4: this warp's KV head occupies its own 16 rows of each stage.
  // HB = 1: this warp takes rows [16 * warp, 16 * warp + 16) of the stage.
  const int row0 = HB == 1 ? warp * kRowsPerWarp : 0;
  const int tile_off = HB == 1 ? 0 : warp * kRowsPerWarp * D;
  const int tok_off = HB == 1 ? row0 : 0;
  const int sf_off = HB == 1 ? (warp * kRowsPerWarp / p.bt) * fp4_sf_pitch(p.bt, D) +
                                   (warp * kRowsPerWarp % p.bt) * (D / 16)
                             : warp * kRowsPerWarp * (D / 16);
  int hslot = 0;
  uint32_t hphase = 0;
  int slot = 0;             // ring position
  uint32_t phase = 0;       // use count of the current slot, mod 2
  uint32_t cpar = 0;
  bool alive = true;
  cw.setup(row0, lane);
  cw.qs = reinterpret_cast<uint32_t*>(smem + L.qfrag + warp * qfrag_warp_bytes(D, NT));
  for (;;) {
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&hdr_full[hslot], hphase, kWaitLimitNs))) {
      alive = false;
      break;
    }
    const uint8_t* hbase = smem + L.hdr + hslot * hslot_bytes;
    const ItemHeader hd = *reinterpret_cast<const ItemHeader*>(hbase);
    if (hd.kind < 0) break;
    const int ncols = MQ ? hd.npos * p.g : p.g;   // the item's columns per KV head
    cw.init(p, qk_scale, reinterpret_cast<const __nv_bfloat16*>(hbase + kHdrBytes), HB * p.g,
            HB == 1 ? 0 : warp * p.g, ncols, lane);
    // Tiles inside every column's range skip the masks: past the newest key
    // the first query sees, and at or after the oldest key the last query
    // sees (window).  With one query per sequence that is [tok_lo, tok_hi).
    const TileMask mk{hd.tok_lo, hd.tok_hi, hd.qpos0, p.window_left, p.lg, ncols};
    const int full_lo = MQ && p.window_left >= 0
                            ? max(hd.tok_lo, hd.qpos0 + hd.npos - 1 - p.window_left)
                            : hd.tok_lo;
    const int full_hi = MQ ? min(hd.tok_hi, hd.qpos0 + 1) : hd.tok_hi;
    __syncwarp();
    if (lane == 0) mbar_arrive(&hdr_empty[hslot]);
    if (++hslot == n_hslots) {
      hslot = 0;
      hphase ^= 1u;
    }

    for (int s = 0; s < hd.n_stages; ++s) {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full_bar[slot], phase, kWaitLimitNs))) {
        alive = false;
        break;
      }
      const uint8_t* st = smem + L.ring + slot * kStage;
      // E4M3: the swizzled K and V tiles; NVFP4: the warp's 16 rows of the
      // four regions (rows 16 * warp onward, for either stage shape)
      const uint8_t* Kt = FP4 ? st + warp * kRowsPerWarp * (D / 2) : st + tile_off;
      const uint8_t* Vt =
          FP4 ? st + kDataBytes + kSfBytes + warp * kRowsPerWarp * (D / 2) : Kt + kTileBytes;
      // (the scale rows of this warp: head `warp` with four heads per stage;
      // with one head, rows 16 * warp of the stage, in page slot
      // 16 * warp / bt at its row 16 * warp % bt)
      const uint8_t* Ks = FP4 ? st + kDataBytes + sf_off : nullptr;
      const uint8_t* Vs = FP4 ? st + 2 * kDataBytes + kSfBytes + sf_off : nullptr;
      const int tok0 = hd.t0 + s * kStageTokens + tok_off;   // token of this warp's first row
      if (tok0 + kRowsPerWarp > hd.tok_lo && tok0 < hd.tok_hi) {
        if (tok0 >= full_lo && tok0 + kRowsPerWarp <= full_hi)
          cw.template tile<true>(Kt, Vt, row0, tok0, mk, lane, Ks, Vs);
        else
          cw.template tile<false>(Kt, Vt, row0, tok0, mk, lane, Ks, Vs);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[slot]);
      if (++slot == stages) {
        slot = 0;
        phase ^= 1u;
      }
    }
    if (!alive) break;

    if constexpr (HB != 1) {
      cw.finish_own(p, v_scale, hd.b, hd.kvh0 + warp, hd.split, hd.ns, hd.qrow0, ncols, lane);
      continue;
    }

    // ---- HB = 1: merge the four warps of this item
    constexpr int OS = D + 4;                                // padded row: no bank conflicts
    float* Osm = reinterpret_cast<float*>(smem + L.merge);   // [warp][H][OS]
    float* MLsm = Osm + kConsumerWarps * H * OS;             // [warp][H][2]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float lsum = cw.l[nt][j];
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
        const int h = nt * 8 + 2 * t + j;
        if (n == 0) {
          MLsm[(warp * H + h) * 2 + 0] = cw.m[nt][j];
          MLsm[(warp * H + h) * 2 + 1] = lsum;
        }
        // O^T column h: rows d = n*(D/8) + 2i + hh  (hh = 0 -> c0/c1, 1 -> c2/c3)
        float* dst = Osm + ((size_t)warp * H + h) * OS + n * (D / 8);
#pragma unroll
        for (int i = 0; i < Consumer<D, NT, MQ, FP4>::MT; ++i) {
          dst[2 * i + 0] = cw.o[i][nt][j];
          dst[2 * i + 1] = cw.o[i][nt][j + 2];
        }
      }
    }
    if (!consumer_sync(cbar, cpar, lane)) {
      alive = false;
      break;
    }
    const bool single = hd.ns <= 1 && !p.combine_all;   // else the combine finishes the rows
    {
      // thread -> (d, first head); heads step by 128 / D.  The loop body is
      // independent per head, so it is unrolled for overlap.
      constexpr int HPI = kConsumerWarps * 32 / D;
      const int d = tid % D;
#pragma unroll 4
      for (int h = tid / D; h < ncols; h += HPI) {
        // column h: query qrow0 + h / g of the sequence, head h % g
        const int hq = hd.kvh0 * p.g + (MQ ? h & (p.g - 1) : h);
        const size_t tok = MQ ? (size_t)hd.b * QL + hd.qrow0 + (h >> p.lg) : (size_t)hd.b;
        const size_t row = tok * p.Hq + hq;
        __nv_bfloat16* const orow = p.out + tok * p.out_tok_stride + (size_t)hq * D;
        if (hd.ns == 0) {  // empty sequence: out = 0, lse = sigma
          if (p.combine_all) continue;   // the combine writes the row
          orow[d] = __float2bfloat16_rn(0.f);
          if (d == 0 && p.lse) p.lse[row] = p.sinks ? p.sinks[hq] : -INFINITY;
          continue;
        }
        float2 ml[kConsumerWarps];
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w)
          ml[w] = *reinterpret_cast<const float2*>(MLsm + (w * H + h) * 2);
        float M = ml[0].x;
#pragma unroll
        for (int w = 1; w < kConsumerWarps; ++w) M = fmaxf(M, ml[w].x);
        float Lsum = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float sc = (ml[w].x == -INFINITY) ? 0.f : fast_exp2(ml[w].x - M);
          Lsum = fmaf(ml[w].y, sc, Lsum);
          acc = fmaf(Osm[((size_t)w * H + h) * OS + d], sc, acc);
        }
        const float lse2 = M + __log2f(Lsum);   // log2-sum-exp of this split (no sink)
        if (MQ && !(Lsum > 0.f)) {   // this query saw no key in the item
          if (single) {
            orow[d] = __float2bfloat16_rn(0.f);
            if (d == 0 && p.lse) p.lse[row] = p.sinks ? p.sinks[hq] : -INFINITY;
          } else {
            const size_t prow = row * p.max_splits + hd.split;
            p.part_o[prow * D + d] = 0.f;
            if (d == 0) p.part_lse[prow] = -INFINITY;
          }
          continue;
        }
        if (single) {
          float scale = v_scale;
          float lse_out = lse2;
          if (p.sinks) {
            const float sg = p.sinks[hq] * kLog2e;
            const float Mx = fmaxf(lse2, sg);
            const float wsplit = fast_exp2(lse2 - Mx);
            const float Z = wsplit + fast_exp2(sg - Mx);
            scale *= __fdividef(wsplit, Z);
            lse_out = Mx + __log2f(Z);
          }
          orow[d] = __float2bfloat16_rn(acc * __fdividef(scale, Lsum));
          if (d == 0 && p.lse) p.lse[row] = lse_out * kLn2;
        } else {
          const size_t prow = row * p.max_splits + hd.split;
          p.part_o[prow * D + d] = __fdividef(acc, Lsum);
          if (d == 0) p.part_lse[prow] = lse2;
        }
      }
    }
    // the merge scratch is reused by the next item
    if (!consumer_sync(cbar, cpar, lane)) {
      alive = false;
      break;
    }
  }
  if (!alive) {
    // Let loads that may already be issued land before the CTA's shared memory
    // is released (bounded), and report.
    for (int r = 0; r < stages; ++r) {
      mbar_wait_bounded(&full_bar[slot], phase, kDrainLimitNs);
      if (++slot == stages) {
        slot = 0;
        phase ^= 1u;
      }
    }
    if (lane == 0) atomicOr(p.status, kErrTimeout);
    return;
  }
  // The last CTA to finish resets the work counter for the next call.
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(&p.sched[1], 1u) == gridDim.x - 1) {
      atomicExch(&p.sched[0], 0u);
      atomicExch(&p.sched[1], 0u);
    }
  }
}

template <int D, int NT, int HB, bool MQ>
__global__ void __launch_bounds__(kThreads, MinBlocks<D, NT>::value)
fpd_split_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                 const DecodeParams p) {
  split_body<D, NT, HB, MQ, false>(&kmap, &vmap, nullptr, nullptr, p);
}

// The split kernel over NVFP4 pages: TMA views of the K and V data (E2M1
// pairs) and of their block scales.
template <int D, int NT, int HB, bool MQ>
__global__ void __launch_bounds__(kThreads, MinBlocks<D, NT>::value)
fpd_split_kernel_nvfp4(const __grid_constant__ CUtensorMap kdata,
                       const __grid_constant__ CUtensorMap ksf,
                       const __grid_constant__ CUtensorMap vdata,
                       const __grid_constant__ CUtensorMap vsf, const DecodeParams p) {
  split_body<D, NT, HB, MQ, true>(&kdata, &vdata, &ksf, &vsf, p);
}

// ----------------------------------------------------------------- combine --

struct CombineParams {
  const int32_t* seq_lens;
  const float* sinks;
  const float* part_o;
  const float* part_lse;
  __nv_bfloat16* out;
  float* out_f32;     // non-null: f32 output, and every row is merged here
  float* lse;
  int B, q_len, Hq, bt, max_blocks, window_left, max_splits;
  const uint32_t* chunk_word;   // the split size the split kernel used (workspace word 3)
  int wpr;            // warps per row: 1, 2, 4, 8, 16 or 32
  int rows_per_cta;   // rows per CTA (wpr * rows_per_cta <= 32)
  float v_scale;
  const float* v_scale_dev;   // device v_scale or nullptr
  int64_t out_tok_stride;     // elements between consecutive output tokens
  // Context-parallel publishing (cp_ranks > 0): every f32 row goes to slot
  // cp_rank of each rank's gather buffer (cp_gather[r] + cp_rank * cp_block:
  // [cp_rows][D] O, then [cp_rows] lse), and once the whole grid has stored
  // its rows, word cp_rank of each rank's flags is set to cp_epoch.
  float* const* cp_gather;    // device array [cp_ranks] of gather buffers
  uint32_t* const* cp_flags;  // device array [cp_ranks] of flag arrays [cp_ranks]
  uint32_t* cp_done;          // CTAs that finished publishing (zero between calls)
  int64_t cp_block, cp_rows;
  int cp_ranks, cp_rank;
  uint32_t cp_epoch;
};

// A row's lse (natural log): to `lse` if given, or to every rank's gather buffer.
template <int D>
__device__ __forceinline__ void store_lse(const CombineParams& p, int row, float v) {
  if (p.cp_ranks > 0) {
    for (int r = 0; r < p.cp_ranks; ++r)
      p.cp_gather[r][p.cp_rank * p.cp_block + p.cp_rows * D + row] = v;
  } else if (p.lse) {
    p.lse[row] = v;
  }
}

// Context-parallel publishing: once every CTA of the grid has stored its rows
// into all ranks' gather buffers, the last one raises this rank's flag at each
// rank.  Each CTA releases its stores at GPU scope into the count; the last
// one, having seen every count, fences at system scope before the flags, so a
// rank that reads a flag with acquire semantics sees all the rows (release is
// cumulative).  One system-scope fence per grid.  Every thread of the CTA
// calls this.
__device__ __forceinline__ void cp_publish_done(const CombineParams& p) {
  if (p.cp_ranks <= 0) return;
  __syncthreads();   // this CTA's rows are stored
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.cp_done, 1u) == gridDim.x - 1) {   // the grid's last CTA
      __threadfence_system();   // one fence orders every row before all the flags
      *p.cp_done = 0u;          // for the next call
      for (int r = 0; r < p.cp_ranks; ++r)
        st_relaxed_sys(p.cp_flags[r] + p.cp_rank, p.cp_epoch);
    }
  }
}

// One lane's PER consecutive output elements, x[i] * inv: bf16, f32, or f32
// into every rank's gather buffer.
template <int PER>
__device__ __forceinline__ void store_out_row(const CombineParams& p, size_t off, const float* x,
                                              float inv) {
  if (p.cp_ranks > 0) {
    for (int r = 0; r < p.cp_ranks; ++r) {
      float* dst = p.cp_gather[r] + p.cp_rank * p.cp_block + off;
#pragma unroll
      for (int i = 0; i < PER; i += 2)
        *reinterpret_cast<float2*>(dst + i) = make_float2(x[i] * inv, x[i + 1] * inv);
    }
  } else if (p.out_f32) {
    float* dst = p.out_f32 + off;
#pragma unroll
    for (int i = 0; i < PER; i += 2)
      *reinterpret_cast<float2*>(dst + i) = make_float2(x[i] * inv, x[i + 1] * inv);
  } else {
    __nv_bfloat16* dst = p.out + off;
#pragma unroll
    for (int i = 0; i < PER; ++i) dst[i] = __float2bfloat16_rn(x[i] * inv);
  }
}

constexpr int kCombineMaxThreads = 1024;
constexpr int kCombineBatch = 8;   // partials a warp loads before it reduces them

// Rows (sequence, query token, query head) whose sequence spans several splits:
//   out = v_scale sum_s 2^(lse_s - M) o_s / (sum_s 2^(lse_s - M) + 2^(sigma - M)),
//   lse = (M + log2 Z) ln 2,  M = max(max_s lse_s, sigma)  (sigma in log2 units).
// Each row gets `wpr` warps; warp j of a row takes splits j, j + wpr, ...  The
// first kCombineBatch of them are loaded together with the sequence length,
// before the split count is known (in bounds: every row owns max_splits
// partials; entries past the count are never used), so the whole merge costs
// one round trip to memory.  Each warp reduces against its own maximum; the
// row's warps are combined in shared memory.  MQ: several queries per
// sequence, where a split may hold no key of a query (its lse is -inf).
// NB: the partials each warp loads in its first round, min(max_splits, 8) for
// one warp per row (256-thread CTAs; a call with few splits then holds fewer
// registers and fits more CTAs per SM), kCombineBatch otherwise.
template <int NB>
struct CombineBounds {
  static constexpr int threads = NB < kCombineBatch ? 256 : kCombineMaxThreads;
  static constexpr int min_blocks = NB <= 4 ? 6 : (NB <= 6 ? 5 : (NB < kCombineBatch ? 4 : 1));
};
template <int D, bool MQ, int NB = kCombineBatch>
__global__ void __launch_bounds__(CombineBounds<NB>::threads, CombineBounds<NB>::min_blocks)
fpd_combine_kernel(const CombineParams p) {
  constexpr int kMaxWarps = kCombineMaxThreads / 32;
  __shared__ float acc_sm[kMaxWarps][D];
  __shared__ float z_sm[kMaxWarps], m_sm[kMaxWarps];
  pdl_launch_dependents();   // the next call's split kernel may be scheduled
  pdl_wait_primary();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpr = p.wpr;
  const int row = blockIdx.x * p.rows_per_cta + warp / wpr;
  const int j = warp % wpr;
  const int QL = MQ ? p.q_len : 1;   // query tokens per sequence
  const bool in_range = row < p.B * QL * p.Hq;
  constexpr int PER = D / 32;
  const int ms = p.max_splits;
  const float* pl = p.part_lse + (size_t)(in_range ? row : 0) * ms;
  const float* po = p.part_o + (size_t)(in_range ? row : 0) * ms * D + lane * PER;

  // ---- one round of loads: the sequence length, v_scale and this warp's first batch
  const int L_raw = in_range ? p.seq_lens[row / (QL * p.Hq)] : 0;
  const int chunk = (int)*p.chunk_word;
  const float v_scale = p.v_scale_dev ? *p.v_scale_dev : p.v_scale;
  float lv[NB];
  float x[NB][PER];
#pragma unroll
  for (int u = 0; u < NB; ++u) {
    const int s = j + wpr * u;
    lv[u] = -INFINITY;
#pragma unroll
    for (int i = 0; i < PER; ++i) x[u][i] = 0.f;
    if (in_range && s < ms) {
      lv[u] = pl[s];
      if constexpr (PER == 4) {
        const float4 t = *reinterpret_cast<const float4*>(po + (size_t)s * D);
        x[u][0] = t.x, x[u][1] = t.y, x[u][2] = t.z, x[u][3] = t.w;
      } else {
        const float2 t = *reinterpret_cast<const float2*>(po + (size_t)s * D);
        x[u][0] = t.x, x[u][1] = t.y;
      }
    }
  }
  const int ns =
      seq_range(L_raw, QL, p.bt, p.max_blocks, p.window_left, chunk, nullptr)
          .n_splits;
  // rows with one split were written by the split kernel, unless the output is f32
  const bool active = in_range && (ns > 1 || p.out_f32 || p.cp_ranks > 0);

  // ---- this warp's splits against its own maximum m
  float m = -INFINITY, z = 0.f;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  if (active) {
#pragma unroll
    for (int u = 0; u < NB; ++u)
      if (j + wpr * u < ns) m = fmaxf(m, lv[u]);
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      // never touch unused (possibly stale) entries; -inf: no key of the query there
      if (j + wpr * u < ns && (!MQ || lv[u] != -INFINITY)) {
        const float w = fast_exp2(lv[u] - m);
        z += w;
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, x[u][i], acc[i]);
      }
    }
    // splits beyond the first batch (more than wpr * NB of them)
    for (int s = j + wpr * NB; s < ns; s += wpr) {
      const float l = pl[s];
      float v[PER];
      if constexpr (PER == 4) {
        const float4 t = *reinterpret_cast<const float4*>(po + (size_t)s * D);
        v[0] = t.x, v[1] = t.y, v[2] = t.z, v[3] = t.w;
      } else {
        const float2 t = *reinterpret_cast<const float2*>(po + (size_t)s * D);
        v[0] = t.x, v[1] = t.y;
      }
      if (MQ && l == -INFINITY) continue;   // the query saw no key in this split
      if (l > m) {   // rescale to the new maximum (m = -inf: r = 0)
        const float r = fast_exp2(m - l);
        z *= r;
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] *= r;
        m = l;
      }
      const float w = fast_exp2(l - m);
      z += w;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, v[i], acc[i]);
    }
  }

  // ---- merge the row's warps (M = max over warps and the sink) and write
  const int hq = row % p.Hq;
  const float sink2 = (active && p.sinks) ? p.sinks[hq] * kLog2e : -INFINITY;
  // this lane's PER output elements of the row
  const size_t ooff = (size_t)(row / p.Hq) * p.out_tok_stride + (size_t)hq * D + lane * PER;
  if (wpr == 1) {
    if (active) {
      const float M = fmaxf(m, sink2);
      const float r = fast_exp2(m - M);
      const float Z = z * r + (p.sinks ? fast_exp2(sink2 - M) : 0.f);
      // false only for an f32 row with no key and no sink: out = 0, lse = -inf
      const bool any = Z > 0.f;
      const float inv = any ? v_scale * r / Z : 0.f;
      store_out_row<PER>(p, ooff, acc, inv);
      if (lane == 0) store_lse<D>(p, row, any ? (M + __log2f(Z)) * kLn2 : -INFINITY);
    }
    cp_publish_done(p);
    return;
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) acc_sm[warp][lane * PER + i] = acc[i];
  if (lane == 0) {
    z_sm[warp] = z;
    m_sm[warp] = m;
  }
  __syncthreads();
  if (active && j == 0) {   // the row's first warp finishes it
    // lane w < wpr holds warp w's maximum, weight and sum
    const float mw = lane < wpr ? m_sm[warp + lane] : -INFINITY;
    float M = fmaxf(sink2, mw);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float rw = mw == -INFINITY ? 0.f : fast_exp2(mw - M);   // 0: warp without a split
    float Z = lane < wpr ? z_sm[warp + lane] * rw : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, o);
    if (p.sinks) Z += fast_exp2(sink2 - M);
    const bool any = Z > 0.f;   // as above
    const float inv = any ? v_scale / Z : 0.f;
    float a[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) a[i] = 0.f;
    for (int w = 0; w < wpr; ++w) {
      const float r = __shfl_sync(0xffffffffu, rw, w);
#pragma unroll
      for (int i = 0; i < PER; ++i) a[i] = fmaf(acc_sm[warp + w][lane * PER + i], r, a[i]);
    }
    store_out_row<PER>(p, ooff, a, inv);
    if (lane == 0) store_lse<D>(p, row, any ? (M + __log2f(Z)) * kLn2 : -INFINITY);
  }
  cp_publish_done(p);
}

}  // namespace fpd
