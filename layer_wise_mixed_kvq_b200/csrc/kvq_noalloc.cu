// kvq_noalloc.cu -- decode attention for callers that cannot allocate device
// memory.
//
// Who needs this: programs whose device memory is owned by someone else. A
// serving engine that reserves all of HBM for its own arena at start-up cannot
// let a library call cudaMalloc behind its back: the call would fail, or break
// the engine's memory accounting. A plug-in hosted inside another runtime
// cannot touch that runtime's allocator. Latency-critical loops must avoid
// cudaMalloc/cudaFree, which can synchronise the whole device. kvq_cache_create
// allocates (device memory, or at least pinned host memory and an event), so
// these callers keep the layer's pages, window and lengths in their own buffers
// and call kvq_decode_attn_noalloc. Its split-K scratch lives in a fixed
// static device array instead of an allocation.
//
// The array below is part of the module image: every GPU that loads the
// library holds its 16 MiB until the process exits. All calls share it, so calls
// whose kernels overlap on the GPU (different streams, or different host
// threads without ordering) race on it and give wrong results; serialise them.

#include <algorithm>
#include <cmath>
#include <mutex>
#include <string>

#include "kvq_internal.cuh"

namespace {

constexpr size_t kScratchBytes = 16u << 20;  // 16 MiB per device
constexpr int kMaxDevices = 64;

// Split-K scratch: an error word (in its own 256-byte slot), the merge counters,
// then (acc, m, l) partial records.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];
constexpr size_t kErrSlot = 256;

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

kvq_status fail(kvq_status st, const std::string& msg) {
  kvq::set_last_error(msg);
  return st;
}

// Device address of g_decode_scratch on the current device, looked up once per
// device (the host-side symbol is only a stand-in and must never be passed to
// a kernel).
kvq_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(KVQ_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(KVQ_EINVAL, "device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p)
      return fail(KVQ_ECUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return KVQ_OK;
}

bool ok_bits(int b) { return b == 2 || b == 4 || b == 8; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" kvq_status kvq_decode_attn_noalloc(kvq_pair pair, int head_dim, int n_q_heads, int n_kv_heads,
                                              const void* pages, int64_t max_pages, const void* window,
                                              const int32_t* seq_len, int64_t max_seq_len, const void* Q,
                                              int batch, float* out, void* stream) {
  if (!((pair.k_bits == 16 && pair.v_bits == 16) || (ok_bits(pair.k_bits) && ok_bits(pair.v_bits))) ||
      pair.key_mode > KVQ_KEY_PER_TOKEN || (pair.k_bits == 16 && pair.key_mode != KVQ_KEY_PER_CHANNEL))
    return fail(KVQ_EINVAL, "unsupported pair");
  if (pair.format != KVQ_FMT_INT)
    return fail(KVQ_EINVAL, "fp8 layers need their per-head scales: use kvq_decode_attn on a cache");
  if (head_dim != 64 && head_dim != 128) return fail(KVQ_EINVAL, "head_dim must be 64 or 128");
  if (n_kv_heads <= 0 || n_q_heads <= 0 || n_q_heads % n_kv_heads != 0 || n_q_heads / n_kv_heads > kvq::kMaxGqa)
    return fail(KVQ_EINVAL, "n_q_heads must be a multiple of n_kv_heads with at most 8 per KV head");
  if (batch <= 0 || batch > kvq::kMaxBatch) return fail(KVQ_EINVAL, "batch must be in [1, 1024]");
  if (max_pages < 0 || max_seq_len < 0 || max_seq_len / kvq::kPageTokens > max_pages || max_pages > (1 << 25))
    return fail(KVQ_EINVAL, "need 0 <= max_seq_len/32 <= max_pages <= 2^25");
  if (!pages || !window || !seq_len || !Q || !out) return fail(KVQ_EINVAL, "null pointer");
  if (!aligned16(pages) || !aligned16(window) || !aligned16(Q) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(seq_len) & 3u))
    return fail(KVQ_EINVAL, "pages, window, Q and out must be 16-byte aligned, seq_len 4-byte aligned");

  const int G = n_q_heads / n_kv_heads;
  const int64_t pairs = (int64_t)batch * n_kv_heads;
  const size_t ctr_bytes = kErrSlot + ((size_t)pairs * 4 + 255) / 256 * 256;  // error word + merge counters
  const size_t rec_bytes = (size_t)G * (head_dim + 2) * 4;  // one split-K record (acc, m, l)
  if (ctr_bytes + 2 * rec_bytes > kScratchBytes)
    return fail(KVQ_ECAPACITY, "batch * n_kv_heads merge counters (4 bytes each) leave no room for split records "
                               "in the 16 MiB static scratch; use fewer sequences per call");
  const int64_t records = (int64_t)((kScratchBytes - ctr_bytes) / rec_bytes);
  const int64_t max_p = max_seq_len / kvq::kPageTokens;
  const int64_t n_units = pairs * (max_p + 1 + kvq::seg_overhead_units());
  if (n_units > INT32_MAX) return fail(KVQ_EINVAL, "too many pages in one call");

  void* base = nullptr;
  kvq_status st = scratch_address(&base);
  if (st != KVQ_OK) return st;
  int32_t* err = static_cast<int32_t*>(base);
  int32_t* ctr = reinterpret_cast<int32_t*>(static_cast<unsigned char*>(base) + kErrSlot);
  float* partials = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + ctr_bytes);

  // same split policy as kvq_decode_attn, sized from the caller's length bound
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t stride = records / pairs;  // CUDA-core kernel: records per (sequence, head)
  const int64_t chunk = stride >= 1 ? kvq::choose_chunk(sms, max_p * pairs, max_p, stride) : max_p + 1;
  const int splits = max_p > 0 ? (int)((max_p + chunk - 1) / chunk) : 1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the merge counters must start at zero; the array keeps the last call's contents
  cudaError_t e = cudaMemsetAsync(ctr, 0, (size_t)pairs * 4, s);
  if (e != cudaSuccess) return fail(KVQ_ECUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));

  kvq::DecodeParams p{};
  p.pages = static_cast<const uint8_t*>(pages);
  p.window = static_cast<const __nv_bfloat16*>(window);
  p.len = seq_len;
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.out = out;
  p.partials = partials;
  p.ctr = ctr;
  p.page_bytes = kvq::page_bytes_of(pair.k_bits, pair.v_bits, head_dim, pair.key_mode, KVQ_FMT_INT);
  p.key_mode = pair.key_mode;
  p.max_pages = (int)max_pages;
  p.n_kv_heads = n_kv_heads;
  p.gqa = G;
  p.chunk = (int)chunk;
  p.splits_stride = (int)std::max<int64_t>(stride, 1);
  p.batch = batch;
  p.n_units = (int)n_units;
  p.err = err;
  p.max_ctas = (int)std::min<int64_t>(
      (int64_t)((kScratchBytes - ctr_bytes) / ((size_t)kvq::split_record_floats(G, head_dim) * 4)) / 2, INT32_MAX);
  p.sm_count = sms;
  p.seg_overhead = kvq::seg_overhead_units();
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)head_dim));
  e = kvq::launch_decode(pair.k_bits, pair.v_bits, head_dim, p, dim3(splits, n_kv_heads, batch), s);
  if (e != cudaSuccess) return fail(KVQ_ECUDA, std::string("decode kernel launch: ") + cudaGetErrorString(e));
  return KVQ_OK;
}

extern "C" kvq_status kvq_noalloc_check(void) {
  void* base = nullptr;
  kvq_status st = scratch_address(&base);
  if (st != KVQ_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  int32_t flag = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&flag, base, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && flag) e = cudaMemset(base, 0, 4);
  if (e != cudaSuccess) return fail(KVQ_ECUDA, std::string("kvq_noalloc_check: ") + cudaGetErrorString(e));
  if (flag)
    return fail(KVQ_ECUDA, "kvq_decode_attn_noalloc: a page copy did not complete within its wait limit; "
                           "the output of that call is wrong");
  return KVQ_OK;
}
