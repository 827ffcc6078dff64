// kvq_internal.cuh -- internal types of libkvq (not part of the C ABI).
//
// Device memory of one layer (all regions 256-byte aligned):
//   pages : [max_batch][n_kv_heads][max_pages] x page_bytes   (full 32-token pages)
//   window: [max_batch][n_kv_heads][2][32][head_dim] bf16      (keys, values; slot = token % 32)
//   len   : [max_batch] int32                                  (tokens held per sequence)
// Cache-wide scratch:
//   partials: [slots][G][head_dim + 2] fp32 split-K partial (acc, m, l), slot =
//             (b * n_kv_heads + h) * splits_stride + split
//   merge_ctr: [max_batch * n_kv_heads] int32, zero between launches
//   append_ctr: [max_batch] int32, zero between launches
//   plan  : [4 * max_batch] int32 (T0, n, row offset, work items) for multi-token appends
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <utility>
#include <string>
#include <vector>

#include "kvq.h"

namespace kvq {

constexpr int kPageTokens = 32;   // key group size = tokens per page = window capacity
constexpr int kMaxBatch = 1024;
constexpr int kMaxGqa = 8;
constexpr int kHostLens = 256;    // sequences whose lengths a decode launch can carry in its parameters
// Per-layer quantization error report: kErrBins bins of kErrStride doubles (one
// 128-byte line each), every flush adding into one bin, so concurrent flushes
// seldom update the same address; the report is the sum over bins.
constexpr int kErrBins = 64;
constexpr int kErrStride = 16;

__host__ __device__ inline double* err_bin(double* base, unsigned key) {
  return base ? base + (key % kErrBins) * kErrStride : nullptr;
}

__host__ __device__ constexpr int64_t code_block_bytes(int bits, int D) { return 4LL * D * bits; }

// km: key mode (0 = per-channel keys, D scale/zero pairs; 1 = per-token keys, 32).
// fmt: 0 = integer codes with page metadata, 1 = fp8 e4m3 (no page metadata).
__host__ __device__ constexpr int64_t page_bytes_of(int kb, int vb, int D, int km, int fmt) {
  return code_block_bytes(kb, D) + code_block_bytes(vb, D) +
         ((kb == 16 || fmt) ? 0 : (km ? 128LL : 4LL * D) + 128);
}

// Tensor-core kernel split record: [G][D] accumulators, [G] maxima, [G] sums,
// padded to 4 floats so every record starts 16-byte aligned.
__host__ __device__ constexpr int split_record_floats(int G, int D) { return G * D + ((2 * G + 3) & ~3); }

struct LayerState {
  int kb = 0, vb = 0, km = 0, fmt = 0;
  float* fp8_scales = nullptr;   // fp8 layers: [2][n_kv_heads] key then value scales (device)
  double* err_stats = nullptr;   // [kErrBins][kErrStride]: sums (k-k^)^2, k^2, (v-v^)^2, v^2, element count
  int64_t page_bytes = 0;
  uint8_t* pages = nullptr;
  __nv_bfloat16* window = nullptr;
  int32_t* len = nullptr;
  std::vector<int64_t> host_len;
};

// Parameters of the append kernel.
struct AppendParams {
  uint8_t* pages;
  __nv_bfloat16* window;
  int32_t* len;
  int32_t* ctr;          // append_ctr
  const void* K;
  const void* V;
  const int32_t* plan;   // nullptr: one token per sequence, lengths read from `len`
  int64_t page_bytes;
  int max_pages;
  int n_kv_heads;
  int key_mode;          // 0 = per-channel keys, 1 = per-token keys
  int fmt;               // 0 = integer codes, 1 = fp8 e4m3
  const float* fp8_scales;  // fmt 1: [2][n_kv_heads] key then value scales
  double* err_stats;     // quantization error sums of the layer, see LayerState
  int64_t max_tokens;    // one-token mode: a full sequence is left unchanged and flags err
  int32_t* err;          // cache error flag (2 = one-token append past max_tokens)
};

// Parameters of the decode attention kernel.
struct DecodeParams {
  const uint8_t* pages;
  const __nv_bfloat16* window;
  const int32_t* len;
  const __nv_bfloat16* Q;
  float* out;
  float* partials;
  int32_t* ctr;          // merge_ctr
  int64_t page_bytes;
  int max_pages;
  int n_kv_heads;
  int gqa;               // query heads per KV head
  int batch;             // sequences b < batch are attended
  int chunk;             // CUDA-core kernel: pages per split
  int splits_stride;     // CUDA-core kernel: partial slots per (b, h)
  int n_units;           // tensor-core kernel: total units (host view; an upper bound with device lengths)
  int max_ctas;          // tensor-core kernel: CTAs the partial buffer can serve (2 split records each)
  int sm_count;
  int seg_overhead;      // tensor-core kernel: overhead units leading each segment (>= 0)
  int key_mode;          // 0 = per-channel keys, 1 = per-token keys
  int fmt;               // 0 = integer codes, 1 = fp8 e4m3
  const float* fp8_scales;  // fmt 1: [2][n_kv_heads] key then value scales
  float scale_log2;      // log2(e) / sqrt(head_dim)
  int* err;              // set to nonzero if a bounded wait gave up (may be null)
  int warp_split;        // tensor-core kernel, G <= 4: one warp per segment (if the segments fit the
                         // resident warps) instead of CTAs sharing each segment's pages
  int warp_pairs;        // warp split: two warps per segment (alternate pages, merged in shared
                         // memory) when the pairs also fit the resident warps
  // fused decode step (kvq_decode_step): the warp that owns segment (b, h)'s tail
  // unit first appends that segment's new token; the same buffers as above, writable
  int append;
  uint8_t* step_pages;
  __nv_bfloat16* step_window;
  int32_t* step_len;
  int32_t* append_ctr;           // warp split: [batch], zero between launches
  int32_t* grid_ctr;             // shared split with device lengths: one int, zero between launches
  const __nv_bfloat16* k_new;    // [batch][n_kv_heads][head_dim]
  const __nv_bfloat16* v_new;
  double* err_stats;
  int max_tokens;
  // shared split: the lengths (before this call's append) come from hlen instead of
  // a scan of `len` on the device; with `early` the first page copies are issued
  // before the wait for the preceding kernel (pages below those lengths are not
  // written by it)
  int host_units;
  int early;
  int32_t hlen[kHostLens];
};

// Programmatic dependent launch. Every kernel of the library starts with
// pdl_enter(): it waits for its stream predecessor to complete (with that
// grid's memory visible) before its first global memory access, then lets its
// own successor begin launching. On an ordinary stream the kernels are launched
// with programmatic stream serialization, so a successor's launch and CTA
// placement overlap this kernel's tail; stream order is unchanged. While the
// stream is being captured into a CUDA graph they are launched plainly
// (measured on B200: programmatic edges inside the captured decode step made
// replays slower), and the wait is then a no-op.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Device-scope fetch-add with acquire-release ordering: releases every memory
// access this thread has performed or observed (through a preceding barrier)
// and acquires those released by the other participants.
__device__ __forceinline__ int atomic_add_acq_rel(int* addr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
  return old;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &capture);
  if (e != cudaSuccess) return e;
  cfg.attrs = attr;
  cfg.numAttrs = capture == cudaStreamCaptureStatusNone ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launchers (defined per kernel file); return the CUDA launch error.
// The key mode travels in the parameter blocks (AppendParams/DecodeParams::key_mode).
cudaError_t launch_append(int kb, int vb, int D, kvq_dtype dtype, const AppendParams& p, dim3 grid,
                          cudaStream_t s);
cudaError_t launch_decode_simt(int kb, int vb, int D, const DecodeParams& p, dim3 grid, cudaStream_t s);
// Grid chosen inside: one warp per segment when p.warp_split and the segments fit
// one resident wave, else resident CTAs x SMs capped by n_units and max_ctas.
cudaError_t launch_decode_mma(int kb, int vb, int D, const DecodeParams& p, cudaStream_t s);
// Pages per split-K CTA for a layer-step: about 3 CTAs per SM, at least 8 pages
// (2 per warp) per CTA, and no more than `stride` splits per (sequence, head).
int choose_chunk(int sm_count, int64_t total_pages, int64_t max_pages_per_seq, int64_t stride);
// Overhead units per segment for the tensor-core kernel's balanced slices
// (KVQ_SEG_OVERHEAD_UNITS overrides the default).
int seg_overhead_units();
// Completed 32-token groups of one sequence-head per append CTA in multi-token
// appends (KVQ_APPEND_GROUPS_PER_CTA overrides).
int append_groups_per_cta();
// Message returned by kvq_last_error() on this thread.
void set_last_error(const std::string& msg);
// KVQ_DECODE_KERNEL=simt: the CUDA-core decode kernel instead of the tensor-core one.
bool decode_uses_simt();

// Layer-map dispatcher: the kernel instance for a layer's pair (p.append = 1:
// the fused one-token append + decode attention of kvq_decode_step).
cudaError_t launch_decode(int kb, int vb, int D, const DecodeParams& p, dim3 grid, cudaStream_t s);

}  // namespace kvq

struct kvq_cache {
  int device = 0;
  int n_layers = 0, n_q_heads = 0, n_kv_heads = 0, head_dim = 0, max_batch = 0;
  int64_t max_tokens = 0, max_pages = 0;
  int sm_count = 148;
  std::vector<kvq::LayerState> layers;
  float* partials = nullptr;
  int64_t partial_slots = 0;
  int32_t* merge_ctr = nullptr;
  int32_t* append_ctr = nullptr;
  int32_t* err = nullptr;            // device flag raised by a decode wait that gave up
  int32_t* grid_ctr = nullptr;       // fused step with device lengths: elects the CTA publishing lengths
  int32_t* plan_dev = nullptr;
  int32_t* plan_host = nullptr;      // pinned
  cudaEvent_t plan_done = nullptr;
  bool plan_pending = false;
  void* pool = nullptr;
  size_t pool_bytes = 0;
  bool owns_pool = false;
  int split_pages = 0;
  int warp_pages = -1;               // kvq_set_decode_mode: -1 automatic, 0 never, n > 0 up to n pages
  int64_t launches = 0;
  // Streams this cache launched on, each with the layer its latest launch wrote
  // (-1: none, -2: every layer): a decode may stream pages in under the tail of
  // the preceding kernel unless that kernel is one of ours writing the same layer.
  struct StreamWrite {
    void* stream;
    int layer;
  };
  std::vector<StreamWrite> stream_writes;
  bool stream_table_full = false;
  // A CUDA graph was captured: its replays change the device lengths without the
  // host, so launches read the device lengths until kvq_refresh_lengths.
  bool graph_captured = false;
};
