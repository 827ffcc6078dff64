// kvq_append.cu -- append new tokens to a layer's cache: bf16 window, and on
// every 32nd token a quantize + bit-pack flush into the next page.
//
// KVTuner OpenReview rebuttal, "Computational cost": only the newly generated
// keys and values are quantized online, with the layer's calibrated precision
// pair. Keys are quantized per channel and values per token, both asymmetric
// (llms-explorer facts page; rebuttal "key per-channel-asym and value
// per-token-asym"); a layer in per-token key mode quantizes its keys per token
// like its values (rebuttal section 4, "Per-channel vs. per-token
// quantization"). The group size (32 tokens) and the fp16 scale/zero format
// are this library's choices.
//
// Grid (items, n_kv_heads, batch), 128 threads. Work item i of (b, h) quantizes
// group floor(T0/32) + i when that group completes during this call; item 0
// also rewrites the window afterwards (it is the only item reading old window
// tokens). With no completed group, item 0 only writes the window. A flush
// stages the group's 32 key and value rows in shared memory as bf16 (16-byte
// vector loads), takes the quantizer parameters (a thread per key channel, a
// warp per token), then quantizes every element as it is packed into the
// fragment-ordered page.
//
// Quantizer (bit-exact contract with the CPU oracle; every fp32 step is a
// single IEEE operation, the __f*_rn intrinsics are never contracted):
//   mn, mx = min, max (signed zeros canonicalised to +0)
//   z = fp16_round_down(mn) clamped to >= -65504
//   s = fp16_round_up((mx - z) / qmax) clamped to <= 65504
//   code = s == 0 ? 0 : clamp(rint((x - z) * (1/s)), 0, qmax)
// FP8 layers (e4m3 elements, per-KV-head scale s_h; llms-explorer facts page on
// vLLM FP8 KV caches): code = e4m3(x / s_h), one IEEE division, then round to
// nearest even with saturation at 448.
// Every flush also adds its quantization error to the layer's report: sums of
// (x - x_hat)^2 and x^2 for keys and values, in fp64 (x_hat = code * s + z, or
// e4m3 value * s_h, is exact in fp64).

#include <cuda_fp8.h>

#include "kvq_internal.cuh"
#include "kvq_quant.cuh"

namespace kvq {
namespace {

constexpr int kThreads = 128;

// Write one code block (32 tokens x D) as lane-interleaved 16-byte vectors.
template <int BITS, int D, typename Get>
__device__ __forceinline__ void store_block(uint8_t* blk, bool is_value, Get vals) {
  constexpr int kVectors = (int)(code_block_bytes(BITS, D) / 16);
  for (int v = threadIdx.x; v < kVectors; v += kThreads) {
    int lane = v & 31, vi = v >> 5;
    uint4 q;
    q.x = lane_word<BITS>(lane, 4 * vi + 0, is_value, vals);
    q.y = lane_word<BITS>(lane, 4 * vi + 1, is_value, vals);
    q.z = lane_word<BITS>(lane, 4 * vi + 2, is_value, vals);
    q.w = lane_word<BITS>(lane, 4 * vi + 3, is_value, vals);
    reinterpret_cast<uint4*>(blk)[v] = q;
  }
}

template <bool F32IN>
__device__ __forceinline__ __nv_bfloat16 load_in(const void* base, int64_t idx) {
  if constexpr (F32IN) return __float2bfloat16_rn(reinterpret_cast<const float*>(base)[idx]);
  else return reinterpret_cast<const __nv_bfloat16*>(base)[idx];
}

// Eight consecutive input values as bf16 (a 16-byte vector; fp32 inputs are
// rounded to nearest even). idx is a multiple of 8.
template <bool F32IN>
__device__ __forceinline__ uint4 load8(const void* base, int64_t idx) {
  if constexpr (F32IN) {
    const float4 x = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
    const float4 y = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx + 4);
    auto pack = [](float lo, float hi) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
      return *reinterpret_cast<const uint32_t*>(&b);
    };
    return make_uint4(pack(x.x, x.y), pack(x.z, x.w), pack(y.x, y.y), pack(y.z, y.w));
  } else {
    return *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx);
  }
}

// Integer code blocks, tile by tile. A block's 16-byte vector vi of lane
// (g, t) holds 16/BITS consecutive 16x16 tiles f (tile row dt = f/2, token
// half tt = f%2); element (p, j) of a tile sits at row g + 8(p&1), column
// 2t + j + 8(p>>1), rows being tokens for keys and channels for values. The
// element's code goes to nibble p + 4j of word f (4-bit), to bits
// 2(4u + p + 8j) of word f/2 with u = f%2 (2-bit), or to byte 2(p&1) + j of
// word 2f + p/2 (8-bit): the same layout as lane_word, produced tile by tile so
// that a tile's values and quantizer parameters are loaded once.
//   code(r, p, j, x, i): code of the element with value x and parameter index i.
template <int BITS>
__device__ __forceinline__ void place_tile(uint32_t (&words)[4], int i, const uint32_t (&c)[4][2]) {
  if constexpr (BITS == 4) {
    uint32_t w = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int j = 0; j < 2; ++j) w |= c[p][j] << (4 * (p + 4 * j));
    words[i] = w;
  } else if constexpr (BITS == 2) {
    const int u = i & 1;
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int j = 0; j < 2; ++j) words[i >> 1] |= c[p][j] << (2 * (4 * u + p + 8 * j));
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h)
      words[2 * i + h] = c[2 * h][0] | (c[2 * h][1] << 8) | (c[2 * h + 1][0] << 16) | (c[2 * h + 1][1] << 24);
  }
}

// Vector vi of lane `lane` of the key block (r = 0) or value block (r = 1).
// xs: [32][RS] bf16 rows of the group (tokens); pz, pr: quantizer zero points and
// reciprocals by channel (per-channel keys) or by token (values, per-token keys).
template <int BITS, int RS, typename Code>
__device__ __forceinline__ uint4 pack_vector(int r, bool by_token, int lane, int vi,
                                             const __nv_bfloat16 (*xs)[RS], Code code) {
  constexpr int TPV = 16 / BITS;  // tiles per 16-byte vector
  const int g = lane >> 2, t = lane & 3;
  uint32_t words[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < TPV; ++i) {
    const int f = vi * TPV + i, dt = f >> 1, tt = f & 1;
    uint32_t c[4][2];
    if (r == 0) {
      // keys: rows are tokens 16tt + g (+8), columns channels 16dt + 2t (+1) (+8)
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int tok = 16 * tt + g + 8 * (p & 1), dim = 16 * dt + 2 * t + 8 * (p >> 1);
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[tok][dim]));
        c[p][0] = code(p, 0, x.x, by_token ? tok : dim);
        c[p][1] = code(p, 1, x.y, by_token ? tok : dim + 1);
      }
    } else {
      // values: rows are channels 16dt + g (+8), columns tokens 16tt + 2t (+1) (+8)
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int dim = 16 * dt + g + 8 * (p & 1), tok = 16 * tt + 2 * t + 8 * (p >> 1);
        c[p][0] = code(p, 0, __bfloat162float(xs[tok][dim]), tok);
        c[p][1] = code(p, 1, __bfloat162float(xs[tok + 1][dim]), tok + 1);
      }
    }
    place_tile<BITS>(words, i, c);
  }
  return make_uint4(words[0], words[1], words[2], words[3]);
}

// One integer code block (R = 0 keys, 1 values) of BITS-bit codes, with this
// thread's share of the error report terms.
template <int R, int BITS, int D, int RS>
__device__ __forceinline__ void emit_block(uint8_t* blk, bool per_token_keys, const __nv_bfloat16 (*xs)[RS],
                                           const float* pz, const float* pr, const float* ps, double (&err)[4]) {
  constexpr int qmax = (1 << BITS) - 1;
  const bool by_token = R == 1 || per_token_keys;
  auto code = [&](int, int, float x, int i) -> uint32_t {
    QParams q;
    q.z = pz[i];
    q.r = pr[i];
    q.zero_scale = (q.r == 0.0f);
    const uint32_t c = quant_code(x, q, qmax);
    const double dx = (double)x - ((double)c * (double)ps[i] + (double)q.z);
    err[2 * R] += dx * dx;
    err[2 * R + 1] += (double)x * (double)x;
    return c;
  };
  constexpr int kVectors = (int)(code_block_bytes(BITS, D) / 16);
  for (int v = threadIdx.x; v < kVectors; v += kThreads)
    reinterpret_cast<uint4*>(blk)[v] = pack_vector<BITS, RS>(R, by_token, v & 31, v >> 5, xs, code);
}

template <int KB, int VB, int D, bool F32IN>
__global__ void __launch_bounds__(kThreads) append_kernel(AppendParams a) {
  pdl_enter();
  constexpr bool kBf16Layer = (KB == 16);
  constexpr int RS = D + 8;          // bf16 row stride of the staged rows (16-byte rows, staggered banks)
  constexpr int NP = D > 32 ? D : 32;
  const int b = blockIdx.z, h = blockIdx.y, item = blockIdx.x;
  const int H = a.n_kv_heads;
  __shared__ __align__(16) __nv_bfloat16 xs[2][kPageTokens][RS];  // keys, values of the group
  __shared__ float pz[2][NP], pr[2][NP], ps[2][NP];  // quantizer zero, reciprocal, scale: keys, values
  __shared__ double red[kThreads / 32][4];
  __shared__ int s_T0;
  __nv_bfloat16 k_new, v_new;  // one-token mode: this thread's channel of the new row

  int T0, n, items;
  int64_t off;
  if (a.plan) {
    T0 = a.plan[4 * b];
    n = a.plan[4 * b + 1];
    off = a.plan[4 * b + 2];
    items = a.plan[4 * b + 3];
    if (item >= items) return;
    if (item == 0 && h == 0 && threadIdx.x == 0) a.len[b] = T0 + n;
  } else {
    // One token per sequence; every CTA of sequence b reads the old length,
    // and the last one to have read it publishes the new length (the
    // acquire-release increment orders each CTA's read before the last CTA's
    // write). The host checks capacity before launching, but a replayed CUDA
    // graph does not run host code: a full sequence is left unchanged here and
    // the cache's error flag is raised. The new token's row is loaded first:
    // its address does not depend on the length.
    if (threadIdx.x < D) {
      k_new = load_in<F32IN>(a.K, ((int64_t)b * H + h) * D + threadIdx.x);
      v_new = load_in<F32IN>(a.V, ((int64_t)b * H + h) * D + threadIdx.x);
    }
    if (threadIdx.x == 0) {
      const int t0 = a.len[b];
      s_T0 = t0;
      if (atomic_add_acq_rel(&a.ctr[b], 1) == H - 1) {
        a.ctr[b] = 0;
        if (t0 < a.max_tokens) a.len[b] = t0 + 1;
      }
    }
    __syncthreads();
    T0 = s_T0;
    if (T0 >= a.max_tokens) {
      if (threadIdx.x == 0 && a.err) atomicExch(a.err, 2);
      return;
    }
    n = 1;
    off = b;
    items = 1;
  }
  if (n == 0) return;
  const int T1 = T0 + n;
  const int g0 = T0 / kPageTokens;
  const int ng = T1 / kPageTokens - g0;

  __nv_bfloat16* win = a.window + ((int64_t)(b * H + h) * 2) * kPageTokens * D;

  if (ng > 0) {
    const int g = g0 + item;
    uint8_t* page = a.pages + ((int64_t)(b * H + h) * a.max_pages + g) * a.page_bytes;
    // the group's 32 key and value rows, old window slots first, as 16-byte vectors
    constexpr int VPR = D / 8;
    for (int v = threadIdx.x; v < 2 * kPageTokens * VPR; v += kThreads) {
      const int r = v / (kPageTokens * VPR), rem = v % (kPageTokens * VPR);
      const int tk = rem / VPR, c8 = (rem % VPR) * 8;
      const int tau = g * kPageTokens + tk;
      uint4 x;
      if (tau < T0) {
        x = *reinterpret_cast<const uint4*>(win + (r * kPageTokens + (tau % kPageTokens)) * D + c8);
      } else {
        const int64_t row = off + (tau - T0);
        x = load8<F32IN>(r ? a.V : a.K, (row * H + h) * D + c8);
      }
      *reinterpret_cast<uint4*>(&xs[r][tk][c8]) = x;
    }
    __syncthreads();
    if constexpr (kBf16Layer) {
      store_block<16, D>(page, false, [&](int tok, int dim) { return (uint32_t)__bfloat16_as_ushort(xs[0][tok][dim]); });
      store_block<16, D>(page + code_block_bytes(16, D), true,
                         [&](int tok, int dim) { return (uint32_t)__bfloat16_as_ushort(xs[1][tok][dim]); });
    } else {
      double err[4] = {0.0, 0.0, 0.0, 0.0};  // this thread's share of the error report
      auto add_err = [&](int r, float x, double xh) {
        const double dx = (double)x - xh;
        err[2 * r] += dx * dx;
        err[2 * r + 1] += (double)x * (double)x;
      };
      if (a.fmt != 0) {
        if constexpr (KB == 8 && VB == 8) {
          const float sc[2] = {a.fp8_scales[h], a.fp8_scales[H + h]};
          auto code = [&](int r, int tok, int dim) -> uint32_t {
            const float x = __bfloat162float(xs[r][tok][dim]);
            const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(__fdiv_rn(x, sc[r]), __NV_SATFINITE, __NV_E4M3);
            add_err(r, x, (double)__half2float(__half(__nv_cvt_fp8_to_halfraw(c, __NV_E4M3))) * sc[r]);
            return (uint32_t)c;
          };
          store_block<8, D>(page, false, [&](int tok, int dim) { return code(0, tok, dim); });
          store_block<8, D>(page + code_block_bytes(8, D), true, [&](int tok, int dim) { return code(1, tok, dim); });
        }
      } else {
        const bool per_token_keys = a.key_mode != 0;
        const int nk = per_token_keys ? kPageTokens : D;  // key scale/zero pairs
        uint8_t* vblk = page + code_block_bytes(KB, D);
        __half* kscale = reinterpret_cast<__half*>(vblk + code_block_bytes(VB, D));
        __half* kzero = kscale + nk;
        __half* vscale = kzero + nk;
        __half* vzero = vscale + kPageTokens;
        auto keep = [&](int r, int i, const QParams& q) {
          pz[r][i] = q.z;
          pr[r][i] = q.r;  // 0 for a constant set
          ps[r][i] = __half2float(q.s_h);
        };
        // one warp per token over the head dimension: row r of xs (0 keys, 1 values)
        auto quantize_tokens = [&](int r, int qmax, __half* sdst, __half* zdst) {
          const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
          for (int t = warp; t < kPageTokens; t += kThreads / 32) {
            float mn = __bfloat162float(xs[r][t][lane]), mx = mn;
#pragma unroll
            for (int k = 1; k < D / 32; ++k) {
              const float x = __bfloat162float(xs[r][t][lane + 32 * k]);
              mn = fminf(mn, x);
              mx = fmaxf(mx, x);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            if (lane == 0) {
              const QParams q = make_qparams(mn, mx, qmax);
              sdst[t] = q.s_h;
              zdst[t] = q.z_h;
              keep(r, t, q);
            }
          }
        };
        if (per_token_keys) quantize_tokens(0, (1 << KB) - 1, kscale, kzero);
        // keys (per-channel mode): one thread per channel, over the group's 32 tokens
        for (int d = threadIdx.x; d < (per_token_keys ? 0 : D); d += kThreads) {
          float mn = __bfloat162float(xs[0][0][d]), mx = mn;
#pragma unroll 8
          for (int t = 1; t < kPageTokens; ++t) {
            const float x = __bfloat162float(xs[0][t][d]);
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
          }
          const QParams q = make_qparams(mn, mx, (1 << KB) - 1);
          const int slot = kmeta_slot<D>(d);
          kscale[slot] = q.s_h;
          kzero[slot] = q.z_h;
          keep(0, d, q);
        }
        quantize_tokens(1, (1 << VB) - 1, vscale, vzero);
        __syncthreads();
        // codes, each element quantized as it is packed, and its error report terms
        emit_block<0, KB, D, RS>(page, per_token_keys, xs[0], pz[0], pr[0], ps[0], err);
        emit_block<1, VB, D, RS>(vblk, true, xs[1], pz[1], pr[1], ps[1], err);
      }
      // this flush's error sums: warp shuffles, then one fp64 atomic per sum into
      // one of the layer's bins
      const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        double v = err[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp][i] = v;
      }
      __syncthreads();
      double* bin = err_bin(a.err_stats, blockIdx.x + 131u * blockIdx.y + 8191u * blockIdx.z);
      if (bin && threadIdx.x < 4) {
        double v = 0.0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) v += red[w][threadIdx.x];
        atomicAdd(&bin[threadIdx.x], v);
      }
      if (bin && threadIdx.x == 4) atomicAdd(&bin[4], (double)(kPageTokens * D));
    }
  }

  if (item == 0) {
    __syncthreads();  // the group above may have read old window slots
    const int wstart = (T1 / kPageTokens) * kPageTokens;
    const int from = wstart > T0 ? wstart : T0;
    const int cnt = T1 - from;
    if (!a.plan) {
      if (cnt == 1 && threadIdx.x < D) {  // the new token (cnt = 0: it completed a page)
        const int slot = T0 % kPageTokens;
        win[(0 * kPageTokens + slot) * D + threadIdx.x] = k_new;
        win[(1 * kPageTokens + slot) * D + threadIdx.x] = v_new;
      }
    } else {
      constexpr int VPR = D / 8;
      for (int v = threadIdx.x; v < cnt * VPR; v += kThreads) {
        const int i = v / VPR, c8 = (v % VPR) * 8;
        const int tau = from + i;
        const int64_t row = off + (tau - T0);
        const int slot = tau % kPageTokens;
        *reinterpret_cast<uint4*>(win + (0 * kPageTokens + slot) * D + c8) = load8<F32IN>(a.K, (row * H + h) * D + c8);
        *reinterpret_cast<uint4*>(win + (1 * kPageTokens + slot) * D + c8) = load8<F32IN>(a.V, (row * H + h) * D + c8);
      }
    }
  }
}

template <int KB, int VB, int D>
cudaError_t launch3(kvq_dtype dt, const AppendParams& p, dim3 grid, cudaStream_t s) {
  if (dt == KVQ_F32) return launch_pdl(append_kernel<KB, VB, D, true>, grid, dim3(kThreads), 0, s, p);
  return launch_pdl(append_kernel<KB, VB, D, false>, grid, dim3(kThreads), 0, s, p);
}

template <int D>
cudaError_t launch_d(int kb, int vb, kvq_dtype dt, const AppendParams& p, dim3 grid, cudaStream_t s) {
#define KVQ_PAIR(K_, V_) \
  if (kb == K_ && vb == V_) return launch3<K_, V_, D>(dt, p, grid, s);
  KVQ_PAIR(2, 2) KVQ_PAIR(2, 4) KVQ_PAIR(2, 8)
  KVQ_PAIR(4, 2) KVQ_PAIR(4, 4) KVQ_PAIR(4, 8)
  KVQ_PAIR(8, 2) KVQ_PAIR(8, 4) KVQ_PAIR(8, 8)
  KVQ_PAIR(16, 16)
#undef KVQ_PAIR
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_append(int kb, int vb, int D, kvq_dtype dtype, const AppendParams& p, dim3 grid,
                          cudaStream_t s) {
  if (D == 64) return launch_d<64>(kb, vb, dtype, p, grid, s);
  if (D == 128) return launch_d<128>(kb, vb, dtype, p, grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
