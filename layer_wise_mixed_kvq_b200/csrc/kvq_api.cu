// kvq_api.cu -- the C ABI of libkvq: argument checks, device memory layout,
// host mirror of sequence lengths, and the layer-map dispatcher that picks the
// kernel instance of each layer's (key bits, value bits) pair.
//
// The layer map is fixed at creation: KVTuner applies its offline-searched
// per-layer configuration at inference with no online decision (llms-explorer
// facts page; arXiv 2502.04420 abstract), so dispatch is a table lookup.

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "kvq_internal.cuh"

namespace {

thread_local std::string g_last_error;

kvq_status fail(kvq_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

kvq_status cuda_fail(cudaError_t e, const char* what) {
  g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  return KVQ_ECUDA;
}

bool valid_pair(kvq_pair p) {
  auto ok = [](int b) { return b == 2 || b == 4 || b == 8; };
  if (p.format > KVQ_FMT_FP8 || p.key_mode > KVQ_KEY_PER_TOKEN) return false;
  if (p.k_bits == 16 && p.v_bits == 16) return p.key_mode == KVQ_KEY_PER_CHANNEL && p.format == KVQ_FMT_INT;
  if (p.format == KVQ_FMT_FP8) return p.k_bits == 8 && p.v_bits == 8 && p.key_mode == KVQ_KEY_PER_CHANNEL;
  return ok(p.k_bits) && ok(p.v_bits);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Geometry {
  int64_t max_pages = 0;
  std::vector<size_t> page_region, window_region;
  size_t len_region = 0, partial_region = 0, merge_region = 0, append_region = 0, plan_region = 0, err_region = 0,
         grid_region = 0;
  int64_t partial_slots = 0;
  size_t total = 0;
};

// Split-K partial slots: enough for every (sequence, head) to take 2 splits, and
// at least 16 per SM of a 148-SM part.
int64_t partial_slots_for(int max_batch, int n_kv_heads) {
  return std::max<int64_t>((int64_t)max_batch * n_kv_heads * 2, 148LL * 16);
}

bool make_geometry(const kvq_pair* map, int n_layers, int n_q_heads, int n_kv_heads, int head_dim,
                   int max_batch, int64_t max_tokens, Geometry& g, std::string& why) {
  if (!map || n_layers <= 0) { why = "layer_map is null or n_layers <= 0"; return false; }
  for (int l = 0; l < n_layers; ++l)
    if (!valid_pair(map[l])) {
      why = "layer " + std::to_string(l) + " has an unsupported pair (k_bits, v_bits, key_mode, format) = (" +
            std::to_string(map[l].k_bits) + ", " + std::to_string(map[l].v_bits) + ", " +
            std::to_string(map[l].key_mode) + ", " + std::to_string(map[l].format) + ")";
      return false;
    }
  if (head_dim != 64 && head_dim != 128) { why = "head_dim must be 64 or 128"; return false; }
  if (n_kv_heads <= 0 || n_q_heads <= 0 || n_q_heads % n_kv_heads != 0 ||
      n_q_heads / n_kv_heads > kvq::kMaxGqa) {
    why = "n_q_heads must be a positive multiple of n_kv_heads with at most 8 query heads per KV head";
    return false;
  }
  if (max_batch <= 0 || max_batch > kvq::kMaxBatch) { why = "max_batch must be in [1, 1024]"; return false; }
  if (max_tokens <= 0 || max_tokens > (int64_t)1 << 30) { why = "max_tokens must be in [1, 2^30]"; return false; }
  g.max_pages = max_tokens / kvq::kPageTokens;
  size_t total = 0;
  for (int l = 0; l < n_layers; ++l) {
    size_t pb = (size_t)kvq::page_bytes_of(map[l].k_bits, map[l].v_bits, head_dim, map[l].key_mode,
                                           map[l].format);
    size_t pr = round_up((size_t)max_batch * n_kv_heads * std::max<int64_t>(g.max_pages, 1) * pb);
    size_t wr = round_up((size_t)max_batch * n_kv_heads * 2 * kvq::kPageTokens * head_dim * 2);
    g.page_region.push_back(pr);
    g.window_region.push_back(wr);
    total += pr + wr + round_up((size_t)max_batch * 4) + round_up((size_t)n_kv_heads * 2 * 4) +
             round_up((size_t)kvq::kErrBins * kvq::kErrStride * 8);
  }
  g.len_region = round_up((size_t)max_batch * 4);
  g.partial_slots = partial_slots_for(max_batch, n_kv_heads);
  int G = n_q_heads / n_kv_heads;
  g.partial_region = round_up((size_t)g.partial_slots * G * (head_dim + 2) * 4);
  g.merge_region = round_up((size_t)max_batch * n_kv_heads * 4);
  g.append_region = round_up((size_t)max_batch * 4);
  g.plan_region = round_up((size_t)max_batch * 4 * 4);
  g.err_region = round_up(4);
  g.grid_region = round_up(4);
  total += g.partial_region + g.merge_region + g.append_region + g.plan_region + g.err_region + g.grid_region;
  g.total = total;
  return true;
}

kvq_status check_cache(const kvq_cache* c, int layer) {
  if (!c) return fail(KVQ_EINVAL, "cache is null");
  if (layer < 0 || layer >= c->n_layers) return fail(KVQ_EINVAL, "layer index out of range");
  return KVQ_OK;
}

// The layer the latest launch of this cache on `stream` wrote (-1: none; -2:
// every layer, or unknown because the table of streams overflowed).
int stream_written_layer(const kvq_cache* c, void* stream) {
  for (const auto& w : c->stream_writes)
    if (w.stream == stream) return w.layer;
  return c->stream_table_full ? -2 : -1;
}

void note_stream_write(kvq_cache* c, void* stream, int layer) {
  for (auto& w : c->stream_writes)
    if (w.stream == stream) {
      w.layer = layer;
      return;
    }
  if (c->stream_writes.size() >= 64) {
    c->stream_writes.clear();
    c->stream_table_full = true;
  }
  c->stream_writes.push_back({stream, layer});
}

bool capturing(void* stream) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &st) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return st != cudaStreamCaptureStatusNone;
}

}  // namespace

namespace kvq {
void set_last_error(const std::string& msg) { g_last_error = msg; }

// The tensor-core kernel serves every pair; KVQ_DECODE_KERNEL=simt selects the
// CUDA-core kernel instead (a second, independent implementation for checks).
bool decode_uses_simt() {
  static const bool simt = [] {
    const char* e = std::getenv("KVQ_DECODE_KERNEL");
    return e && std::string(e) == "simt";
  }();
  return simt;
}

cudaError_t launch_decode(int kb, int vb, int D, const DecodeParams& p, dim3 grid, cudaStream_t s) {
  return decode_uses_simt() ? launch_decode_simt(kb, vb, D, p, grid, s) : launch_decode_mma(kb, vb, D, p, s);
}

int seg_overhead_units() {
  static const int v = [] {
    const char* e = std::getenv("KVQ_SEG_OVERHEAD_UNITS");
    int x = e ? std::atoi(e) : 32;
    return x < 0 ? 0 : (x > 256 ? 256 : x);
  }();
  return v;
}

int append_groups_per_cta() {
  static const int v = [] {
    const char* e = std::getenv("KVQ_APPEND_GROUPS_PER_CTA");
    const int n = e ? std::atoi(e) : 0;
    return n >= 1 && n <= 1024 ? n : 8;
  }();
  return v;
}

int choose_chunk(int sm_count, int64_t total_pages, int64_t max_p, int64_t stride) {
  const int64_t target_ctas = (int64_t)sm_count * 3;
  int64_t chunk = std::max<int64_t>(8, (total_pages + target_ctas - 1) / target_ctas);
  if (stride < 1) stride = 1;
  chunk = std::max<int64_t>(chunk, (max_p + stride - 1) / stride);
  return (int)chunk;
}
}  // namespace kvq

extern "C" {

const char* kvq_last_error(void) { return g_last_error.c_str(); }

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_EINVAL: return "KVQ_EINVAL";
    case KVQ_ECAPACITY: return "KVQ_ECAPACITY";
    case KVQ_ENOMEM: return "KVQ_ENOMEM";
    case KVQ_ECUDA: return "KVQ_ECUDA";
  }
  return "KVQ_UNKNOWN";
}

int64_t kvq_page_bytes(kvq_pair pair, int head_dim) {
  if (!valid_pair(pair) || (head_dim != 64 && head_dim != 128)) return 0;
  return kvq::page_bytes_of(pair.k_bits, pair.v_bits, head_dim, pair.key_mode, pair.format);
}

double kvq_equiv_bits(const kvq_pair* map, int n_layers) {
  if (!map || n_layers <= 0) return -1.0;
  double sum = 0.0;
  for (int l = 0; l < n_layers; ++l) {
    if (!valid_pair(map[l])) return -1.0;
    sum += 0.5 * ((double)map[l].k_bits + (double)map[l].v_bits);
  }
  return sum / n_layers;
}

size_t kvq_cache_pool_bytes(const kvq_pair* map, int n_layers, int n_q_heads, int n_kv_heads,
                            int head_dim, int max_batch, int64_t max_tokens) {
  Geometry g;
  std::string why;
  if (!make_geometry(map, n_layers, n_q_heads, n_kv_heads, head_dim, max_batch, max_tokens, g, why)) return 0;
  return g.total;
}

kvq_status kvq_cache_create(const kvq_pair* map, int n_layers, int n_q_heads, int n_kv_heads,
                            int head_dim, int max_batch, int64_t max_tokens, void* device_pool,
                            size_t pool_bytes, kvq_cache** out) {
  if (!out) return fail(KVQ_EINVAL, "out is null");
  *out = nullptr;
  Geometry g;
  std::string why;
  if (!make_geometry(map, n_layers, n_q_heads, n_kv_heads, head_dim, max_batch, max_tokens, g, why))
    return fail(KVQ_EINVAL, why);
  if (device_pool && (reinterpret_cast<uintptr_t>(device_pool) % kAlign) != 0)
    return fail(KVQ_EINVAL, "device_pool must be 256-byte aligned");
  if (device_pool && pool_bytes < g.total)
    return fail(KVQ_ENOMEM, "device_pool is smaller than kvq_cache_pool_bytes()");

  kvq_cache* c = new kvq_cache();
  cudaError_t e = cudaGetDevice(&c->device);
  if (e != cudaSuccess) { delete c; return cuda_fail(e, "cudaGetDevice"); }
  cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, c->device);
  c->n_layers = n_layers;
  c->n_q_heads = n_q_heads;
  c->n_kv_heads = n_kv_heads;
  c->head_dim = head_dim;
  c->max_batch = max_batch;
  c->max_tokens = max_tokens;
  c->max_pages = g.max_pages;
  c->partial_slots = g.partial_slots;

  if (device_pool) {
    c->pool = device_pool;
    c->pool_bytes = pool_bytes;
  } else {
    e = cudaMalloc(&c->pool, g.total);
    if (e != cudaSuccess) {
      delete c;
      cudaGetLastError();
      return fail(KVQ_ENOMEM, std::string("cudaMalloc of the cache pool failed: ") + cudaGetErrorString(e));
    }
    c->owns_pool = true;
    c->pool_bytes = g.total;
  }
  uint8_t* p = static_cast<uint8_t*>(c->pool);
  c->layers.resize(n_layers);
  for (int l = 0; l < n_layers; ++l) {
    kvq::LayerState& L = c->layers[l];
    L.kb = map[l].k_bits;
    L.vb = map[l].v_bits;
    L.km = map[l].key_mode;
    L.fmt = map[l].format;
    L.page_bytes = kvq::page_bytes_of(L.kb, L.vb, head_dim, L.km, L.fmt);
    L.pages = p;
    p += g.page_region[l];
    L.window = reinterpret_cast<__nv_bfloat16*>(p);
    p += g.window_region[l];
    L.len = reinterpret_cast<int32_t*>(p);
    p += g.len_region;
    L.fp8_scales = reinterpret_cast<float*>(p);
    p += round_up((size_t)n_kv_heads * 2 * 4);
    L.err_stats = reinterpret_cast<double*>(p);
    p += round_up((size_t)kvq::kErrBins * kvq::kErrStride * 8);
    L.host_len.assign(max_batch, 0);
  }
  c->partials = reinterpret_cast<float*>(p);
  p += g.partial_region;
  c->merge_ctr = reinterpret_cast<int32_t*>(p);
  p += g.merge_region;
  c->append_ctr = reinterpret_cast<int32_t*>(p);
  p += g.append_region;
  c->plan_dev = reinterpret_cast<int32_t*>(p);
  p += g.plan_region;
  c->err = reinterpret_cast<int32_t*>(p);
  p += g.err_region;
  c->grid_ctr = reinterpret_cast<int32_t*>(p);
  p += g.grid_region;

  e = cudaMallocHost(&c->plan_host, (size_t)max_batch * 4 * sizeof(int32_t));
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->plan_done, cudaEventDisableTiming);
  // lengths and counters start at zero; pages and windows need no initialisation
  const std::vector<float> ones((size_t)n_kv_heads * 2, 1.0f);
  for (int l = 0; l < n_layers && e == cudaSuccess; ++l) {
    e = cudaMemset(c->layers[l].len, 0, (size_t)max_batch * 4);
    if (e == cudaSuccess)
      e = cudaMemcpy(c->layers[l].fp8_scales, ones.data(), ones.size() * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(c->layers[l].err_stats, 0, (size_t)kvq::kErrBins * kvq::kErrStride * 8);
  }
  if (e == cudaSuccess) e = cudaMemset(c->merge_ctr, 0, (size_t)max_batch * n_kv_heads * 4);
  if (e == cudaSuccess) e = cudaMemset(c->append_ctr, 0, (size_t)max_batch * 4);
  if (e == cudaSuccess) e = cudaMemset(c->err, 0, 4);
  if (e == cudaSuccess) e = cudaMemset(c->grid_ctr, 0, 4);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    kvq_status st = cuda_fail(e, "cache initialisation");
    kvq_cache_destroy(c);
    return st;
  }
  *out = c;
  return KVQ_OK;
}

void kvq_cache_destroy(kvq_cache* c) {
  if (!c) return;
  cudaDeviceSynchronize();
  if (c->plan_done) cudaEventDestroy(c->plan_done);
  if (c->plan_host) cudaFreeHost(c->plan_host);
  if (c->owns_pool && c->pool) cudaFree(c->pool);
  delete c;
}

kvq_status kvq_cache_reset(kvq_cache* c, void* stream) {
  if (!c) return fail(KVQ_EINVAL, "cache is null");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (auto& L : c->layers) {
    cudaError_t e = cudaMemsetAsync(L.len, 0, (size_t)c->max_batch * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(L.err_stats, 0, (size_t)kvq::kErrBins * kvq::kErrStride * 8, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    std::fill(L.host_len.begin(), L.host_len.end(), 0);
  }
  note_stream_write(c, stream, -2);
  return KVQ_OK;
}

kvq_status kvq_layer_error(const kvq_cache* c, int layer, kvq_error_stats* out) {
  kvq_status st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (!out) return fail(KVQ_EINVAL, "out is null");
  std::vector<double> bins((size_t)kvq::kErrBins * kvq::kErrStride);
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess)
    e = cudaMemcpy(bins.data(), c->layers[layer].err_stats, bins.size() * 8, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(error report)");
  double h[5] = {0.0, 0.0, 0.0, 0.0, 0.0};
  for (int b = 0; b < kvq::kErrBins; ++b)
    for (int i = 0; i < 5; ++i) h[i] += bins[(size_t)b * kvq::kErrStride + i];
  out->k_sq_err = h[0];
  out->k_sq = h[1];
  out->v_sq_err = h[2];
  out->v_sq = h[3];
  out->elements = (int64_t)h[4];
  return KVQ_OK;
}

kvq_status kvq_set_fp8_scales(kvq_cache* c, int layer, const float* k_scale, const float* v_scale) {
  kvq_status st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  kvq::LayerState& L = c->layers[layer];
  if (L.fmt != KVQ_FMT_FP8) return fail(KVQ_EINVAL, "layer is not an fp8 layer");
  if (!k_scale || !v_scale) return fail(KVQ_EINVAL, "scale arrays are null");
  for (int64_t T : L.host_len)
    if (T != 0) return fail(KVQ_EINVAL, "fp8 scales must be set while the layer is empty");
  std::vector<float> s((size_t)c->n_kv_heads * 2);
  for (int h = 0; h < c->n_kv_heads; ++h) {
    if (!(std::isfinite(k_scale[h]) && k_scale[h] > 0.f && std::isfinite(v_scale[h]) && v_scale[h] > 0.f))
      return fail(KVQ_EINVAL, "fp8 scales must be finite and > 0");
    s[h] = k_scale[h];
    s[c->n_kv_heads + h] = v_scale[h];
  }
  cudaError_t e = cudaMemcpy(L.fp8_scales, s.data(), s.size() * 4, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(fp8 scales)");
  return KVQ_OK;
}

kvq_status kvq_set_split_pages(kvq_cache* c, int pages_per_split) {
  if (!c) return fail(KVQ_EINVAL, "cache is null");
  if (pages_per_split < 0) return fail(KVQ_EINVAL, "pages_per_split must be >= 0");
  c->split_pages = pages_per_split;
  return KVQ_OK;
}

kvq_status kvq_set_decode_mode(kvq_cache* c, int max_pages_per_warp) {
  if (!c) return fail(KVQ_EINVAL, "cache is null");
  if (max_pages_per_warp < -1) return fail(KVQ_EINVAL, "max_pages_per_warp must be >= -1");
  c->warp_pages = max_pages_per_warp;
  return KVQ_OK;
}

kvq_status kvq_append(kvq_cache* c, int layer, const void* K, const void* V, kvq_dtype dtype,
                      const int32_t* n_new, int batch, void* stream) {
  kvq_status st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (dtype != KVQ_BF16 && dtype != KVQ_F32) return fail(KVQ_EINVAL, "dtype must be KVQ_BF16 or KVQ_F32");
  if (!n_new) return fail(KVQ_EINVAL, "n_new is null");
  if (batch <= 0) return fail(KVQ_EINVAL, "batch must be positive");
  if (batch > c->max_batch) return fail(KVQ_ECAPACITY, "batch exceeds max_batch");
  kvq::LayerState& L = c->layers[layer];
  int64_t total = 0;
  bool all_one = true;
  int max_items = 1;
  for (int b = 0; b < batch; ++b) {
    if (n_new[b] < 0) return fail(KVQ_EINVAL, "n_new entries must be >= 0");
    if (L.host_len[b] + n_new[b] > c->max_tokens)
      return fail(KVQ_ECAPACITY, "append would exceed max_tokens for sequence " + std::to_string(b));
    total += n_new[b];
    all_one = all_one && (n_new[b] == 1);
    int64_t T0 = L.host_len[b], T1 = T0 + n_new[b];
    max_items = (int)std::max<int64_t>(max_items, T1 / kvq::kPageTokens - T0 / kvq::kPageTokens);
  }
  if (total == 0) return KVQ_OK;
  if (!K || !V) return fail(KVQ_EINVAL, "K or V is null");
  if (!aligned16(K) || !aligned16(V)) return fail(KVQ_EINVAL, "K and V must be 16-byte aligned");
  if (total > INT32_MAX) return fail(KVQ_EINVAL, "too many tokens in one call");

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  kvq::AppendParams p{};
  p.pages = L.pages;
  p.window = L.window;
  p.len = L.len;
  p.ctr = c->append_ctr;
  p.K = K;
  p.V = V;
  p.page_bytes = L.page_bytes;
  p.max_pages = (int)c->max_pages;
  p.n_kv_heads = c->n_kv_heads;
  p.key_mode = L.km;
  p.fmt = L.fmt;
  p.fp8_scales = L.fp8_scales;
  p.err_stats = L.err_stats;
  p.max_tokens = c->max_tokens;
  p.err = c->err;
  p.plan = nullptr;
  if (!all_one) {
    // multi-token append: per-sequence plan (start, count, row offset, items)
    if (c->plan_pending) {
      cudaError_t e = cudaEventSynchronize(c->plan_done);
      if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    }
    int64_t off = 0;
    for (int b = 0; b < batch; ++b) {
      int64_t T0 = L.host_len[b], T1 = T0 + n_new[b];
      c->plan_host[4 * b + 0] = (int32_t)T0;
      c->plan_host[4 * b + 1] = n_new[b];
      c->plan_host[4 * b + 2] = (int32_t)off;
      c->plan_host[4 * b + 3] = (int32_t)std::max<int64_t>(1, T1 / kvq::kPageTokens - T0 / kvq::kPageTokens);
      off += n_new[b];
    }
    cudaError_t e = cudaMemcpyAsync(c->plan_dev, c->plan_host, (size_t)batch * 16, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(plan)");
    e = cudaEventRecord(c->plan_done, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    c->plan_pending = true;
    p.plan = c->plan_dev;
  }
  // multi-token appends: each CTA quantizes up to append_groups_per_cta() of a
  // sequence-head's completed groups, staging the next while it quantizes one
  const int gpc = kvq::append_groups_per_cta();
  dim3 grid(all_one ? 1 : (max_items + gpc - 1) / gpc, c->n_kv_heads, batch);
  cudaError_t e = kvq::launch_append(L.kb, L.vb, c->head_dim, dtype, p, grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
  c->launches += 1;
  note_stream_write(c, stream, layer);
  if (capturing(stream)) c->graph_captured = true;
  for (int b = 0; b < batch; ++b) L.host_len[b] += n_new[b];
  return KVQ_OK;
}

// One warp (or warp pair) per (sequence, KV head) segment, or CTAs sharing each
// segment's pages. Automatic: the split a cost model predicts faster, fitted to
// both kernels' times on B200 (K4V2..K8V8 pages, batch 8 to 128, 5 to 128 pages
// per sequence): the warp split takes about 5 + 1.0 us per page a warp reads of
// the longest sequence (half its pages with warp pairs), the shared split about
// 11.5 + 0.01 us per segment + 0.15 us per page per SM.
static bool choose_warp_split(const kvq_cache* c, int gqa, int batch, int64_t max_p, int64_t total_pages) {
  if (gqa > 4 || c->warp_pages == 0) return false;
  if (c->warp_pages > 0) return max_p <= c->warp_pages;
  const double segs = (double)batch * c->n_kv_heads;
  // warp pairs (two warps per segment, from 4 pages on, while 2 warps per segment fit
  // about 12 resident warps per SM) halve a warp's pages
  const bool pairs = max_p >= 4 && 2.0 * segs <= 12.0 * c->sm_count;
  const double t_warp = 5.0 + 1.0 * (double)max_p / (pairs ? 2.0 : 1.0);
  const double t_shared = 11.5 + 0.01 * segs + 0.15 * (double)total_pages / c->sm_count;
  return t_warp < t_shared;
}

// Parameters of one decode launch of `layer` over sequences b < batch at the
// host's lengths `lens` (before a fused step's append). Fails with a message
// when the units exceed 32-bit indexing.
static kvq_status decode_params(kvq_cache* c, int layer, const void* Q, int batch, float* out, void* stream,
                                bool append, const std::vector<int64_t>& lens, kvq::DecodeParams& p) {
  const kvq::LayerState& L = c->layers[layer];
  int64_t total_pages = 0, max_p = 0, n_units = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t P = lens[b] / kvq::kPageTokens;
    total_pages += P;
    max_p = std::max(max_p, P);
    n_units += P + 1 + kvq::seg_overhead_units();
  }
  total_pages *= c->n_kv_heads;
  n_units *= c->n_kv_heads;
  if (n_units > INT32_MAX) return fail(KVQ_EINVAL, "too many pages in one call");
  int64_t stride = c->partial_slots / ((int64_t)batch * c->n_kv_heads);
  if (stride < 1) return fail(KVQ_EINVAL, "batch too large for the split-K buffer");
  int chunk = c->split_pages > 0 ? c->split_pages : kvq::choose_chunk(c->sm_count, total_pages, max_p, stride);
  // never more splits than the partial buffer holds
  chunk = (int)std::max<int64_t>(chunk, (max_p + stride - 1) / stride);

  p = kvq::DecodeParams{};
  p.pages = L.pages;
  p.window = L.window;
  p.len = L.len;
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.out = out;
  p.partials = c->partials;
  p.ctr = c->merge_ctr;
  p.page_bytes = L.page_bytes;
  p.max_pages = (int)c->max_pages;
  p.n_kv_heads = c->n_kv_heads;
  p.gqa = c->n_q_heads / c->n_kv_heads;
  p.chunk = chunk;
  p.splits_stride = (int)stride;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)c->head_dim));
  p.err = c->err;
  p.batch = batch;
  p.n_units = (int)n_units;
  {
    // partial region holds partial_slots * G * (D + 2) floats; split records are padded
    const int64_t floats = c->partial_slots * (int64_t)p.gqa * (c->head_dim + 2);
    p.max_ctas = (int)std::min<int64_t>(floats / kvq::split_record_floats(p.gqa, c->head_dim) / 2, INT32_MAX);
  }
  p.sm_count = c->sm_count;
  p.seg_overhead = kvq::seg_overhead_units();
  p.key_mode = L.km;
  p.fmt = L.fmt;
  p.fp8_scales = L.fp8_scales;
  p.warp_split = choose_warp_split(c, p.gqa, batch, max_p + (append ? 1 : 0), total_pages) ? 1 : 0;
  p.warp_pairs = max_p >= 4 ? 1 : 0;  // halving a warp's pages pays from a few pages on
  // The lengths travel in the parameters unless a captured graph may replay this
  // launch (frozen parameters) or replays have moved the device lengths past the
  // host's view. Then the page copies may start under the preceding kernel's
  // tail, unless that kernel is one of ours that wrote this layer.
  const bool capture = capturing(stream);
  if (capture) c->graph_captured = true;
  p.host_units = (!capture && !c->graph_captured && batch <= kvq::kHostLens) ? 1 : 0;
  if (p.host_units) {
    for (int b = 0; b < batch; ++b) p.hlen[b] = (int32_t)lens[b];
    const int w = stream_written_layer(c, stream);
    p.early = (w != layer && w != -2) ? 1 : 0;
  }
  if (append) {
    p.append = 1;
    p.step_pages = L.pages;
    p.step_window = L.window;
    p.step_len = L.len;
    p.append_ctr = c->append_ctr;
    p.grid_ctr = c->grid_ctr;
    p.err_stats = L.err_stats;
    p.max_tokens = (int)std::min<int64_t>(c->max_tokens, INT32_MAX);
  }
  return KVQ_OK;
}

kvq_status kvq_decode_attn(kvq_cache* c, int layer, const void* Q, int batch, float* out, void* stream) {
  kvq_status st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (batch <= 0 || batch > c->max_batch) return fail(KVQ_EINVAL, "batch must be in [1, max_batch]");
  if (!Q || !out) return fail(KVQ_EINVAL, "Q or out is null");
  if (!aligned16(Q) || !aligned16(out)) return fail(KVQ_EINVAL, "Q and out must be 16-byte aligned");
  const kvq::LayerState& L = c->layers[layer];
  kvq::DecodeParams p{};
  st = decode_params(c, layer, Q, batch, out, stream, false, L.host_len, p);
  if (st != KVQ_OK) return st;
  int splits = 1;
  for (int b = 0; b < batch; ++b)
    splits = std::max<int>(splits, (int)((L.host_len[b] / kvq::kPageTokens + p.chunk - 1) / p.chunk));
  dim3 grid(splits, c->n_kv_heads, batch);
  cudaError_t e = kvq::launch_decode(L.kb, L.vb, c->head_dim, p, grid, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  c->launches += 1;
  note_stream_write(c, stream, -1);
  return KVQ_OK;
}

kvq_status kvq_decode_step(kvq_cache* c, int layer, const void* K, const void* V, const void* Q, int batch,
                           float* out, void* stream) {
  kvq_status st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  if (batch <= 0 || batch > c->max_batch) return fail(KVQ_EINVAL, "batch must be in [1, max_batch]");
  if (!K || !V || !Q || !out) return fail(KVQ_EINVAL, "K, V, Q or out is null");
  if (!aligned16(K) || !aligned16(V) || !aligned16(Q) || !aligned16(out))
    return fail(KVQ_EINVAL, "K, V, Q and out must be 16-byte aligned");
  kvq::LayerState& L = c->layers[layer];
  for (int b = 0; b < batch; ++b)
    if (L.host_len[b] + 1 > c->max_tokens)
      return fail(KVQ_ECAPACITY, "append would exceed max_tokens for sequence " + std::to_string(b));
  if (kvq::decode_uses_simt()) {
    // the CUDA-core decode kernel has no fused form: append, then attend
    std::vector<int32_t> ones((size_t)batch, 1);
    st = kvq_append(c, layer, K, V, KVQ_BF16, ones.data(), batch, stream);
    return st != KVQ_OK ? st : kvq_decode_attn(c, layer, Q, batch, out, stream);
  }
  kvq::DecodeParams p{};
  st = decode_params(c, layer, Q, batch, out, stream, true, L.host_len, p);
  if (st != KVQ_OK) return st;
  p.k_new = static_cast<const __nv_bfloat16*>(K);
  p.v_new = static_cast<const __nv_bfloat16*>(V);
  cudaError_t e = kvq::launch_decode_mma(L.kb, L.vb, c->head_dim, p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode step kernel launch");
  for (int b = 0; b < batch; ++b) L.host_len[b] += 1;
  c->launches += 1;
  note_stream_write(c, stream, layer);
  return KVQ_OK;
}

int64_t kvq_seq_len(const kvq_cache* c, int layer, int seq) {
  if (!c || layer < 0 || layer >= c->n_layers || seq < 0 || seq >= c->max_batch) return -1;
  return c->layers[layer].host_len[seq];
}

int64_t kvq_bytes(const kvq_cache* c, int layer, int batch, int include_metadata) {
  if (!c || layer < 0 || layer >= c->n_layers || batch <= 0 || batch > c->max_batch) return -1;
  const kvq::LayerState& L = c->layers[layer];
  const int D = c->head_dim;
  int64_t total = 0;
  for (int b = 0; b < batch; ++b) {
    int64_t T = L.host_len[b], P = T / kvq::kPageTokens, W = T % kvq::kPageTokens;
    int64_t codes = kvq::code_block_bytes(L.kb, D) + kvq::code_block_bytes(L.vb, D);
    total += P * (include_metadata ? L.page_bytes : codes);
    if (include_metadata) total += W * D * 2 * 2;
  }
  return total * c->n_kv_heads;
}

int64_t kvq_export_bytes(const kvq_cache* c, int layer, int batch) {
  if (!c || layer < 0 || layer >= c->n_layers || batch <= 0 || batch > c->max_batch) return -1;
  const kvq::LayerState& L = c->layers[layer];
  int64_t total = 0;
  for (int b = 0; b < batch; ++b) {
    int64_t T = L.host_len[b];
    total += (T / kvq::kPageTokens) * L.page_bytes + (T % kvq::kPageTokens) * c->head_dim * 2 * 2;
  }
  return total * c->n_kv_heads;
}

kvq_status kvq_export_layer(const kvq_cache* c, int layer, int batch, void* host_dst, size_t bytes) {
  kvq_status st = check_cache(c, layer);
  if (st != KVQ_OK) return st;
  int64_t need = kvq_export_bytes(c, layer, batch);
  if (need < 0) return fail(KVQ_EINVAL, "bad batch");
  if (!host_dst || bytes < (size_t)need) return fail(KVQ_EINVAL, "host_dst is null or too small");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  const kvq::LayerState& L = c->layers[layer];
  const int D = c->head_dim, H = c->n_kv_heads;
  uint8_t* dst = static_cast<uint8_t*>(host_dst);
  for (int b = 0; b < batch; ++b)
    for (int h = 0; h < H; ++h) {
      int64_t T = L.host_len[b], P = T / kvq::kPageTokens, W = T % kvq::kPageTokens;
      const uint8_t* pg = L.pages + ((int64_t)(b * H + h) * c->max_pages) * L.page_bytes;
      if (P) {
        e = cudaMemcpy(dst, pg, (size_t)(P * L.page_bytes), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(pages)");
        dst += P * L.page_bytes;
      }
      const __nv_bfloat16* win = L.window + ((int64_t)(b * H + h) * 2) * kvq::kPageTokens * D;
      if (W) {
        e = cudaMemcpy(dst, win, (size_t)(W * D * 2), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(window K)");
        dst += W * D * 2;
        e = cudaMemcpy(dst, win + kvq::kPageTokens * D, (size_t)(W * D * 2), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(window V)");
        dst += W * D * 2;
      }
    }
  return KVQ_OK;
}

kvq_status kvq_sync(kvq_cache* c) {
  if (!c) return fail(KVQ_EINVAL, "cache is null");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetLastError");
  int32_t flag = 0;
  e = cudaMemcpy(&flag, c->err, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(err)");
  if (flag) {
    cudaMemset(c->err, 0, 4);
    if (flag == 2)
      return fail(KVQ_ECAPACITY, "a one-token append (replayed graph) found a sequence at max_tokens; "
                                 "that sequence was left unchanged");
    return fail(KVQ_ECUDA, "decode attention: a page copy did not complete within its wait limit");
  }
  return KVQ_OK;
}

kvq_status kvq_refresh_lengths(kvq_cache* c) {
  if (!c) return fail(KVQ_EINVAL, "cache is null");
  cudaError_t e = cudaDeviceSynchronize();
  std::vector<int32_t> tmp((size_t)c->max_batch);
  for (auto& L : c->layers) {
    if (e == cudaSuccess) e = cudaMemcpy(tmp.data(), L.len, tmp.size() * 4, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) break;
    for (int b = 0; b < c->max_batch; ++b) L.host_len[b] = tmp[b];
  }
  if (e != cudaSuccess) return cuda_fail(e, "kvq_refresh_lengths");
  c->graph_captured = false;
  return KVQ_OK;
}

int64_t kvq_launch_count(const kvq_cache* c) { return c ? c->launches : -1; }

}  // extern "C"
