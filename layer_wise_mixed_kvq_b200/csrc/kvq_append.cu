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
// tokens). With no completed group, item 0 only writes the window.
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

template <int KB, int VB, int D, bool F32IN>
__global__ void __launch_bounds__(kThreads) append_kernel(AppendParams a) {
  pdl_enter();
  constexpr bool kBf16Layer = (KB == 16);
  const int b = blockIdx.z, h = blockIdx.y, item = blockIdx.x;
  const int H = a.n_kv_heads;
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
    if constexpr (kBf16Layer) {
      __shared__ uint16_t sv[2][kPageTokens][D];
      for (int idx = threadIdx.x; idx < kPageTokens * D; idx += kThreads) {
        int t = idx / D, d = idx % D;
        int tau = g * kPageTokens + t;
        __nv_bfloat16 kx, vx;
        if (tau < T0) {
          kx = win[(0 * kPageTokens + (tau % kPageTokens)) * D + d];
          vx = win[(1 * kPageTokens + (tau % kPageTokens)) * D + d];
        } else {
          int64_t row = off + (tau - T0);
          kx = load_in<F32IN>(a.K, (row * H + h) * D + d);
          vx = load_in<F32IN>(a.V, (row * H + h) * D + d);
        }
        sv[0][t][d] = __bfloat16_as_ushort(kx);
        sv[1][t][d] = __bfloat16_as_ushort(vx);
      }
      __syncthreads();
      store_block<16, D>(page, false, [&](int tok, int dim) { return (uint32_t)sv[0][tok][dim]; });
      store_block<16, D>(page + code_block_bytes(16, D), true,
                         [&](int tok, int dim) { return (uint32_t)sv[1][tok][dim]; });
    } else {
      __shared__ float xs[2][kPageTokens][D + 1];
      __shared__ uint8_t cs[2][kPageTokens][D];
      for (int idx = threadIdx.x; idx < kPageTokens * D; idx += kThreads) {
        int t = idx / D, d = idx % D;
        int tau = g * kPageTokens + t;
        __nv_bfloat16 kx, vx;
        if (tau < T0) {
          kx = win[(0 * kPageTokens + (tau % kPageTokens)) * D + d];
          vx = win[(1 * kPageTokens + (tau % kPageTokens)) * D + d];
        } else {
          int64_t row = off + (tau - T0);
          kx = load_in<F32IN>(a.K, (row * H + h) * D + d);
          vx = load_in<F32IN>(a.V, (row * H + h) * D + d);
        }
        xs[0][t][d] = __bfloat162float(kx);
        xs[1][t][d] = __bfloat162float(vx);
      }
      __syncthreads();
      double err[4] = {0.0, 0.0, 0.0, 0.0};  // this thread's share of the error report
      auto add_err = [&](int r, float x, double xh) {
        const double dx = (double)x - xh;
        err[2 * r] += dx * dx;
        err[2 * r + 1] += (double)x * (double)x;
      };
      if (a.fmt != 0) {
        if constexpr (KB == 8 && VB == 8) {
          const float ksc = a.fp8_scales[h], vsc = a.fp8_scales[H + h];
          for (int idx = threadIdx.x; idx < kPageTokens * D; idx += kThreads) {
            const int t = idx / D, d = idx % D;
            const __nv_fp8_storage_t ck = __nv_cvt_float_to_fp8(__fdiv_rn(xs[0][t][d], ksc), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8_storage_t cv = __nv_cvt_float_to_fp8(__fdiv_rn(xs[1][t][d], vsc), __NV_SATFINITE, __NV_E4M3);
            cs[0][t][d] = (uint8_t)ck;
            cs[1][t][d] = (uint8_t)cv;
            add_err(0, xs[0][t][d], (double)__half2float(__half(__nv_cvt_fp8_to_halfraw(ck, __NV_E4M3))) * ksc);
            add_err(1, xs[1][t][d], (double)__half2float(__half(__nv_cvt_fp8_to_halfraw(cv, __NV_E4M3))) * vsc);
          }
          __syncthreads();
          store_block<8, D>(page, false, [&](int tok, int dim) { return (uint32_t)cs[0][tok][dim]; });
          store_block<8, D>(page + code_block_bytes(8, D), true, [&](int tok, int dim) { return (uint32_t)cs[1][tok][dim]; });
        }
      } else {
        const bool per_token_keys = a.key_mode != 0;
        const int nk = per_token_keys ? kPageTokens : D;  // key scale/zero pairs
        uint8_t* vblk = page + code_block_bytes(KB, D);
        __half* kscale = reinterpret_cast<__half*>(vblk + code_block_bytes(VB, D));
        __half* kzero = kscale + nk;
        __half* vscale = kzero + nk;
        __half* vzero = vscale + kPageTokens;
        // one warp per token over the head dimension: row r of xs (0 keys, 1 values)
        auto quantize_tokens = [&](int r, int qmax, __half* sdst, __half* zdst) {
          const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
          for (int t = warp; t < kPageTokens; t += kThreads / 32) {
            float mn = xs[r][t][lane], mx = mn;
  #pragma unroll
            for (int k = 1; k < D / 32; ++k) {
              float x = xs[r][t][lane + 32 * k];
              mn = fminf(mn, x);
              mx = fmaxf(mx, x);
            }
  #pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            QParams q = make_qparams(mn, mx, qmax);
            const double s = (double)__half2float(q.s_h), z = (double)q.z;
  #pragma unroll
            for (int k = 0; k < D / 32; ++k) {
              const float x = xs[r][t][lane + 32 * k];
              const uint32_t c = quant_code(x, q, qmax);
              cs[r][t][lane + 32 * k] = (uint8_t)c;
              add_err(r, x, (double)c * s + z);
            }
            if (lane == 0) {
              sdst[t] = q.s_h;
              zdst[t] = q.z_h;
            }
          }
        };
        if (per_token_keys) quantize_tokens(0, (1 << KB) - 1, kscale, kzero);
        // keys (per-channel mode): one thread per channel, over the group's 32 tokens
        for (int d = threadIdx.x; d < (per_token_keys ? 0 : D); d += kThreads) {
          constexpr int qmax = (1 << KB) - 1;
          float mn = xs[0][0][d], mx = mn;
  #pragma unroll 8
          for (int t = 1; t < kPageTokens; ++t) {
            float x = xs[0][t][d];
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
          }
          QParams q = make_qparams(mn, mx, qmax);
          const double s = (double)__half2float(q.s_h), z = (double)q.z;
  #pragma unroll 8
          for (int t = 0; t < kPageTokens; ++t) {
            const uint32_t c = quant_code(xs[0][t][d], q, qmax);
            cs[0][t][d] = (uint8_t)c;
            add_err(0, xs[0][t][d], (double)c * s + z);
          }
          int slot = kmeta_slot<D>(d);
          kscale[slot] = q.s_h;
          kzero[slot] = q.z_h;
        }
        // values: one warp per token, over the head dimension
        quantize_tokens(1, (1 << VB) - 1, vscale, vzero);
        __syncthreads();
        store_block<KB, D>(page, false, [&](int tok, int dim) { return (uint32_t)cs[0][tok][dim]; });
        store_block<VB, D>(vblk, true, [&](int tok, int dim) { return (uint32_t)cs[1][tok][dim]; });
      }
      // this flush's error sums: warp shuffles, then one fp64 atomic per sum
      __shared__ double red[kThreads / 32][4];
      const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        double v = err[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp][i] = v;
      }
      __syncthreads();
      if (a.err_stats && threadIdx.x < 4) {
        double v = 0.0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) v += red[w][threadIdx.x];
        atomicAdd(&a.err_stats[threadIdx.x], v);
      }
      if (a.err_stats && threadIdx.x == 4) atomicAdd(&a.err_stats[4], (double)(kPageTokens * D));
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
      for (int idx = threadIdx.x; idx < cnt * D; idx += kThreads) {
        int i = idx / D, d = idx % D;
        int tau = from + i;
        int64_t row = off + (tau - T0);
        int slot = tau % kPageTokens;
        win[(0 * kPageTokens + slot) * D + d] = load_in<F32IN>(a.K, (row * H + h) * D + d);
        win[(1 * kPageTokens + slot) * D + d] = load_in<F32IN>(a.V, (row * H + h) * D + d);
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
