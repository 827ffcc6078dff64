// kvq_decode_simt.cu -- split-K decode attention over one layer's mixed-precision
// cache on CUDA cores (fp32). Reference design for the tensor-core kernel.
//
// KVTuner OpenReview rebuttal, "Baseline Implementation": decode runs
// FlashAttention-style kernels directly over the int8 / mixed-precision K and V
// cache; "New GQA efficiency results": grouped-query attention, q head hq
// reads KV head hq / G. Dequantization is x = code * s + z with the page's fp16
// scale/zero (keys per channel, values per token).
//
// Grid (splits, n_kv_heads, batch), 128 threads. CTA (s, h, b) covers pages
// [s*chunk, min((s+1)*chunk, P)) of sequence b, KV head h (P = len/32), plus the
// bf16 window when it is the last split. Each CTA keeps an online-softmax state
// (running max m, sum l, accumulator) for its G query heads; with more than one
// split it writes (acc, m, l) to the partial buffer and the last CTA of (b, h)
// to finish merges: out = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s.
// Scores are kept in the log2 domain (scale includes log2(e)).

#include <cuda_fp8.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ void tile_elem(int f, int lane, int e, bool is_value, int& tok, int& dim) {
  int dt = f >> 1, tt = f & 1;
  int g = lane >> 2, t = lane & 3;
  int p = e >> 1, j = e & 1;
  int row = g + 8 * (p & 1);
  int col = 2 * t + j + 8 * (p >> 1);
  if (is_value) { dim = 16 * dt + row; tok = 16 * tt + col; }
  else          { tok = 16 * tt + row; dim = 16 * dt + col; }
}

__device__ __forceinline__ uint32_t lane_word_at(const uint8_t* blk, int lane, int w) {
  return *reinterpret_cast<const uint32_t*>(blk + (((w >> 2) * 32 + lane) * 16 + (w & 3) * 4));
}

// Element e of tile f of lane `lane` in a block of BITS-bit elements.
template <int BITS>
__device__ __forceinline__ uint32_t elem_code(const uint8_t* blk, int f, int lane, int e) {
  if constexpr (BITS == 8) {
    uint32_t w = lane_word_at(blk, lane, 2 * f + (e >> 2));
    return (w >> (8 * (e & 3))) & 0xFFu;
  } else if constexpr (BITS == 4) {
    uint32_t w = lane_word_at(blk, lane, f);
    return (w >> (4 * ((e >> 1) + 4 * (e & 1)))) & 0xFu;
  } else if constexpr (BITS == 2) {
    uint32_t w = lane_word_at(blk, lane, f >> 1);
    return (w >> (2 * (4 * (f & 1) + (e >> 1) + 8 * (e & 1)))) & 0x3u;
  } else {
    uint32_t w = lane_word_at(blk, lane, 4 * f + (e >> 1));
    return (w >> (16 * (e & 1))) & 0xFFFFu;
  }
}

template <int D>
__device__ __forceinline__ int kmeta_channel(int i) {
  int t = i / (D / 4), dt = (i % (D / 4)) / 4, j = i % 4;
  return 16 * dt + 2 * t + (j & 1) + 8 * (j >> 1);
}

template <int KB, int VB, int D>
struct Smem {
  float q[kMaxGqa][D];
  float kd[kPageTokens][D + 1];
  float vd[kPageTokens][D + 1];
  float sc[kMaxGqa][kPageTokens];
  float ks[D], kz[D], vs[kPageTokens], vz[kPageTokens];
  float m[kMaxGqa], l[kMaxGqa], alpha[kMaxGqa];
  int last;
};

__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3)));
}

// Dequantize one full page into kd/vd (fp32). per_token_keys: the page holds 32
// key scales/zeros in token order instead of D in channel-slot order. fp8: the
// elements are e4m3 values times the KV head's scales ksc/vsc.
template <int KB, int VB, int D>
__device__ void load_page(Smem<KB, VB, D>& sm, const uint8_t* page, bool per_token_keys, bool fp8, float ksc,
                          float vsc) {
  constexpr int F = 2 * (D / 16);
  const uint8_t* kblk = page;
  const uint8_t* vblk = page + code_block_bytes(KB, D);
  if constexpr (KB == 16) {
    for (int idx = threadIdx.x; idx < F * 32; idx += kThreads) {
      int f = idx >> 5, lane = idx & 31;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int tok, dim;
        tile_elem(f, lane, e, false, tok, dim);
        sm.kd[tok][dim] = __bfloat162float(__ushort_as_bfloat16((unsigned short)elem_code<16>(kblk, f, lane, e)));
        tile_elem(f, lane, e, true, tok, dim);
        sm.vd[tok][dim] = __bfloat162float(__ushort_as_bfloat16((unsigned short)elem_code<16>(vblk, f, lane, e)));
      }
    }
  } else if (KB == 8 && VB == 8 && fp8) {
    for (int idx = threadIdx.x; idx < F * 32; idx += kThreads) {
      int f = idx >> 5, lane = idx & 31;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int tok, dim;
        tile_elem(f, lane, e, false, tok, dim);
        sm.kd[tok][dim] = e4m3_to_float(elem_code<KB>(kblk, f, lane, e)) * ksc;
        tile_elem(f, lane, e, true, tok, dim);
        sm.vd[tok][dim] = e4m3_to_float(elem_code<VB>(vblk, f, lane, e)) * vsc;
      }
    }
  } else {
    const int nk = per_token_keys ? kPageTokens : D;
    const __half* kscale = reinterpret_cast<const __half*>(vblk + code_block_bytes(VB, D));
    const __half* kzero = kscale + nk;
    const __half* vscale = kzero + nk;
    const __half* vzero = vscale + kPageTokens;
    for (int i = threadIdx.x; i < nk; i += kThreads) {
      int d = per_token_keys ? i : kmeta_channel<D>(i);  // ks/kz indexed by token or by channel
      sm.ks[d] = __half2float(kscale[i]);
      sm.kz[d] = __half2float(kzero[i]);
    }
    for (int t = threadIdx.x; t < kPageTokens; t += kThreads) {
      sm.vs[t] = __half2float(vscale[t]);
      sm.vz[t] = __half2float(vzero[t]);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < F * 32; idx += kThreads) {
      int f = idx >> 5, lane = idx & 31;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int tok, dim;
        tile_elem(f, lane, e, false, tok, dim);
        const int ki = per_token_keys ? tok : dim;
        sm.kd[tok][dim] = fmaf((float)elem_code<KB>(kblk, f, lane, e), sm.ks[ki], sm.kz[ki]);
        tile_elem(f, lane, e, true, tok, dim);
        sm.vd[tok][dim] = fmaf((float)elem_code<VB>(vblk, f, lane, e), sm.vs[tok], sm.vz[tok]);
      }
    }
  }
  __syncthreads();
}

// Fold `ntok` tokens held in kd/vd into the online-softmax state.
template <int KB, int VB, int D, int NACC>
__device__ void attend_tokens(Smem<KB, VB, D>& sm, int G, int ntok, float scale_log2, float (&acc)[NACC]) {
  for (int idx = threadIdx.x; idx < G * kPageTokens; idx += kThreads) {
    int g = idx / kPageTokens, t = idx % kPageTokens;
    float s = -INFINITY;
    if (t < ntok) {
      float a = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) a = fmaf(sm.q[g][d], sm.kd[t][d], a);
      s = a * scale_log2;
    }
    sm.sc[g][t] = s;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    int g = threadIdx.x;
    float mx = sm.m[g];
    for (int t = 0; t < ntok; ++t) mx = fmaxf(mx, sm.sc[g][t]);
    float alpha = (sm.m[g] == -INFINITY) ? 0.f : exp2f(sm.m[g] - mx);
    float sum = 0.f;
    for (int t = 0; t < kPageTokens; ++t) {
      float p = (t < ntok) ? exp2f(sm.sc[g][t] - mx) : 0.f;
      sm.sc[g][t] = p;
      sum += p;
    }
    sm.l[g] = sm.l[g] * alpha + sum;
    sm.m[g] = mx;
    sm.alpha[g] = alpha;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < NACC; ++k) {
    int idx = threadIdx.x + k * kThreads;
    if (idx < G * D) {
      int g = idx / D, d = idx % D;
      float a = acc[k] * sm.alpha[g];
      for (int t = 0; t < ntok; ++t) a = fmaf(sm.sc[g][t], sm.vd[t][d], a);
      acc[k] = a;
    }
  }
  __syncthreads();
}

template <int KB, int VB, int D>
__global__ void __launch_bounds__(kThreads) decode_simt_kernel(DecodeParams p) {
  pdl_enter();
  constexpr int NACC = kMaxGqa * D / kThreads;
  __shared__ Smem<KB, VB, D> sm;
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int H = p.n_kv_heads, G = p.gqa;
  const int T = p.len[b];
  const int P = T / kPageTokens, W = T % kPageTokens;
  const int nsplit = P > 0 ? (P + p.chunk - 1) / p.chunk : 1;
  if (s >= nsplit) return;
  const int p0 = s * p.chunk;
  const int p1 = min(P, p0 + p.chunk);

  for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
    int g = idx / D, d = idx % D;
    sm.q[g][d] = __bfloat162float(p.Q[((int64_t)b * H * G + h * G + g) * D + d]);
  }
  if (threadIdx.x < kMaxGqa) {
    sm.m[threadIdx.x] = -INFINITY;
    sm.l[threadIdx.x] = 0.f;
  }
  float acc[NACC];
#pragma unroll
  for (int k = 0; k < NACC; ++k) acc[k] = 0.f;
  __syncthreads();

  const uint8_t* base = p.pages + ((int64_t)(b * H + h) * p.max_pages) * p.page_bytes;
  for (int pg = p0; pg < p1; ++pg) {
    load_page<KB, VB, D>(sm, base + (int64_t)pg * p.page_bytes, p.key_mode != 0, p.fmt != 0,
                         p.fmt ? p.fp8_scales[h] : 1.f, p.fmt ? p.fp8_scales[p.n_kv_heads + h] : 1.f);
    attend_tokens<KB, VB, D, NACC>(sm, G, kPageTokens, p.scale_log2, acc);
  }
  if (s == nsplit - 1 && W > 0) {
    const __nv_bfloat16* win = p.window + ((int64_t)(b * H + h) * 2) * kPageTokens * D;
    for (int idx = threadIdx.x; idx < W * D; idx += kThreads) {
      int t = idx / D, d = idx % D;
      sm.kd[t][d] = __bfloat162float(win[t * D + d]);
      sm.vd[t][d] = __bfloat162float(win[(kPageTokens + t) * D + d]);
    }
    __syncthreads();
    attend_tokens<KB, VB, D, NACC>(sm, G, W, p.scale_log2, acc);
  }

  float* outp = p.out + ((int64_t)b * H * G + h * G) * D;
  if (nsplit == 1) {
#pragma unroll
    for (int k = 0; k < NACC; ++k) {
      int idx = threadIdx.x + k * kThreads;
      if (idx < G * D) {
        int g = idx / D;
        float l = sm.l[g];
        outp[idx] = l > 0.f ? acc[k] / l : 0.f;
      }
    }
    return;
  }

  // split-K: publish this CTA's partial state, the last CTA merges
  const int64_t slot0 = (int64_t)(b * H + h) * p.splits_stride;
  float* part = p.partials + (slot0 + s) * G * (D + 2);
#pragma unroll
  for (int k = 0; k < NACC; ++k) {
    int idx = threadIdx.x + k * kThreads;
    if (idx < G * D) {
      int g = idx / D, d = idx % D;
      part[g * (D + 2) + d] = acc[k];
    }
  }
  if (threadIdx.x < G) {
    part[threadIdx.x * (D + 2) + D] = sm.m[threadIdx.x];
    part[threadIdx.x * (D + 2) + D + 1] = sm.l[threadIdx.x];
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int prev = atomicAdd(&p.ctr[b * H + h], 1);
    sm.last = (prev == nsplit - 1);
    if (sm.last) p.ctr[b * H + h] = 0;
  }
  __syncthreads();
  if (!sm.last) return;
  __threadfence();
  const float* parts = p.partials + slot0 * G * (D + 2);
  for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
    int g = idx / D, d = idx % D;
    float M = -INFINITY;
    for (int j = 0; j < nsplit; ++j) M = fmaxf(M, __ldcg(parts + ((int64_t)j * G + g) * (D + 2) + D));
    float L = 0.f, O = 0.f;
    for (int j = 0; j < nsplit; ++j) {
      const float* r = parts + ((int64_t)j * G + g) * (D + 2);
      float mj = __ldcg(r + D);
      float w = (mj == -INFINITY) ? 0.f : exp2f(mj - M);
      L = fmaf(w, __ldcg(r + D + 1), L);
      O = fmaf(w, __ldcg(r + d), O);
    }
    outp[idx] = L > 0.f ? O / L : 0.f;
  }
}

template <int D>
cudaError_t launch_d(int kb, int vb, const DecodeParams& p, dim3 grid, cudaStream_t s) {
#define KVQ_PAIR(K_, V_) \
  if (kb == K_ && vb == V_) return launch_pdl(decode_simt_kernel<K_, V_, D>, grid, dim3(kThreads), 0, s, p);
  KVQ_PAIR(2, 2) KVQ_PAIR(2, 4) KVQ_PAIR(2, 8)
  KVQ_PAIR(4, 2) KVQ_PAIR(4, 4) KVQ_PAIR(4, 8)
  KVQ_PAIR(8, 2) KVQ_PAIR(8, 4) KVQ_PAIR(8, 8)
  KVQ_PAIR(16, 16)
#undef KVQ_PAIR
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_simt(int kb, int vb, int D, const DecodeParams& p, dim3 grid, cudaStream_t s) {
  if (D == 64) return launch_d<64>(kb, vb, p, grid, s);
  if (D == 128) return launch_d<128>(kb, vb, p, grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
