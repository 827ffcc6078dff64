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

// Asynchronous 16-byte global -> shared copies (L2 only), committed and
// waited for in groups.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
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

// Fragment loads from the staged rows: matrix m of an x4 load takes its eight
// row addresses from lanes 8m..8m+7, and lane (g, t) = (lane/4, lane%4)
// receives row g, columns 2t and 2t+1 of each matrix (rows and columns
// swapped with .trans).
__device__ __forceinline__ void ldsm_x4(uint32_t (&a)[4], const void* p) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]) : "r"(s));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&a)[4], const void* p) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]) : "r"(s));
}

// Tile (dt, tt) of a code block for this lane: register p holds elements
// (p, 0) and (p, 1) (low, high half), element (p, j) sitting at row g + 8(p&1),
// column 2t + j + 8(p>>1) of the 16x16 tile. Rows are tokens 16tt.. for keys
// (is_value false) and channels 16dt.. for values; xs rows are tokens.
template <int RS>
__device__ __forceinline__ void load_tile(uint32_t (&a)[4], const __nv_bfloat16 (*xs)[RS], bool is_value,
                                          int dt, int tt, int lane) {
  const int m = lane >> 3, r = lane & 7;
  if (is_value) ldsm_x4_trans(a, &xs[16 * tt + 8 * (m >> 1) + r][16 * dt + 8 * (m & 1)]);
  else ldsm_x4(a, &xs[16 * tt + r + 8 * (m & 1)][16 * dt + 8 * (m >> 1)]);
}

// Two elements' codes, as the bits of the fp32 numbers 1.5 * 2^23 + code: for y
// in [0, qmax] the single rounding of the addition is rint(y), round-half-even.
// y = (x - z) * (1/s), x - z formed as x + (-z) (the same IEEE result); with
// CLAMP, y is clamped to [0, qmax] first, which gives clamp(rint(y), 0, qmax) for
// every y (fmaxf also maps a NaN to 0); a zero reciprocal (constant set) gives
// 0. Two elements per packed fp32 operation, each with an explicit rounding mode.
constexpr uint32_t kRintBias = 0x4B400000u;  // bits of 1.5 * 2^23
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, D;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "add.rn.f32x2 D, A, B;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, D;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "mul.rn.f32x2 D, A, B;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, C, D;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "mov.b64 C, {%6, %7};\n\tfma.rn.f32x2 D, A, B, C;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
// m: the two sums 1.5 * 2^23 + code (as floats); u: x - z (rounded, as used for y)
struct CodePair {
  float2 m, u;
};
// Without CLAMP (a group none of whose sets had z or s clamped to fp16's
// range) y already lies in [0, qmax + 2^-14] for every element of its set (z <=
// min, s >= (max - z) / qmax rounded up), so rint(y) is in [0, qmax] without the
// clamp. There the bias is added by two scalar additions: a packed addition
// that directly consumes the packed product measured as a single rounding of
// both on B200 (codes off by one in ~0.04% of elements), while __fadd_rn stays
// its own operation.
template <bool CLAMP>
__device__ __forceinline__ CodePair code_pair(float2 x, float2 nz, float2 r, float qmax) {
  CodePair cp;
  cp.u = add2_rn(x, nz);
  float2 y = mul2_rn(cp.u, r);
  if constexpr (CLAMP) {
    y.x = fminf(fmaxf(y.x, 0.0f), qmax);
    y.y = fminf(fmaxf(y.y, 0.0f), qmax);
    cp.m = add2_rn(y, make_float2(12582912.0f, 12582912.0f));
  } else {
    cp.m = make_float2(__fadd_rn(y.x, 12582912.0f), __fadd_rn(y.y, 12582912.0f));
  }
  return cp;
}

// Error report terms of one element: (x - x_hat)^2 and x^2 in fp64, with
// x_hat = code * s + z exact in fp64 (code < 2^8, s and z fp16 values).
// The code becomes a double through the bits of 2^52 + (code bits).
__device__ __forceinline__ void add_error(double (&e)[2], float x, uint32_t bits, double2 zs) {
  const double c = __hiloint2double(0x43300000, (int)bits) - (4503599627370496.0 + (double)kRintBias);
  const double xd = (double)x;
  const double dx = xd - fma(c, zs.y, zs.x);
  e[0] = fma(dx, dx, e[0]);
  e[1] = fma(xd, xd, e[1]);
}

// Error report terms in fp32 for a pair of elements, for groups whose largest
// magnitude lies in [2^-14, 2^40) (fp16's normal range and above, so z and s
// resolve the data): dx = (x - z) - code * s with x - z the rounded u of the
// code computation and one rounding of the fused multiply-add, dx^2 and x^2
// accumulated in fp32 over one 16-byte vector (at most 32 elements per thread)
// and then added to the fp64 sums. x^2 is exact in fp32 for a bf16 x there; the
// rounding of u (|u| <= (qmax + 1) s) moves a dx by at most 2^-24 |u|, so a
// layer's sum of dx^2 stays within about 2^-23 (qmax + 1) * 3 (below 1e-4 for
// 8-bit codes, far less in practice) of the exact one. Outside that range the
// fp64 terms above are used.
__device__ __forceinline__ void add_error2(float2 (&acc)[2], float2 x, const CodePair& cp, float2 ns) {
  const float2 c = add2_rn(cp.m, make_float2(-12582912.0f, -12582912.0f));  // the codes, exactly
  const float2 dx = fma2_rn(c, ns, cp.u);
  acc[0] = fma2_rn(dx, dx, acc[0]);
  acc[1] = fma2_rn(x, x, acc[1]);
}

// Quantizer parameters of one index (a channel or a token): z and 1/s in fp32
// for the code; -s in fp32 and z, s in fp64 for the error report.
struct QTab {
  const float* nz;     // -z
  const float* r;      // 1/s, 0 for a constant set
  const float* ns;     // -s
  const double2* zs;   // z, s
};

// Integer code block of BITS-bit codes. Lane l's 16-byte vector vi holds tiles
// f = vi * 16/BITS .. (tile row dt = f/2, token half tt = f%2). Element (p, j)
// of tile f goes to nibble p + 4j of word f (4-bit), to bits 2(4u + p + 8j) of
// word f/2 with u = f%2 (2-bit), or to byte 2(p&1) + j of word 2f + p/2 (8-bit).
// MODE 0: keys, one parameter set per channel; 1: keys, one per token;
// 2: values, one per token. e: this thread's error terms of the block, formed
// in fp32 (F32ERR) or fp64. CLAMP: see code_pair.
template <int BITS, int D, int RS, int MODE, bool F32ERR, bool CLAMP>
__device__ __forceinline__ void emit_codes(uint8_t* blk, const __nv_bfloat16 (*xs)[RS], QTab q, double (&e)[2]) {
  constexpr int TPV = 16 / BITS;  // tiles per 16-byte vector
  constexpr int kVectors = (int)(code_block_bytes(BITS, D) / 16);
  constexpr float qmax = (float)((1 << BITS) - 1);
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  // parameters of the element pair (p, 0), (p, 1) of a tile: index h = p>>1
  // (MODE 0, 2: indices i0 + 8h, +1) or h = p&1 (MODE 1: one token for both)
  struct Pair {
    float2 nz, r, ns;
    double2 zs0, zs1;
  };
  auto load_pair = [&](int i, bool one) {
    Pair pr;
    if (one) {
      pr.nz = make_float2(q.nz[i], q.nz[i]);
      pr.r = make_float2(q.r[i], q.r[i]);
      if constexpr (F32ERR) pr.ns = make_float2(q.ns[i], q.ns[i]);
      else pr.zs0 = pr.zs1 = q.zs[i];
    } else {
      pr.nz = *reinterpret_cast<const float2*>(q.nz + i);
      pr.r = *reinterpret_cast<const float2*>(q.r + i);
      if constexpr (F32ERR) {
        pr.ns = *reinterpret_cast<const float2*>(q.ns + i);
      } else {
        pr.zs0 = q.zs[i];
        pr.zs1 = q.zs[i + 1];
      }
    }
    return pr;
  };
  for (int v = threadIdx.x; v < kVectors; v += kThreads) {
    const int vi = v >> 5;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // F32ERR: dx^2, x^2 of this vector
    // one element pair: quantize, add the error terms, add the codes into their fields
    auto put = [&](int i, int p, uint32_t a, const Pair& pr) {
      const float2 x = make_float2(__uint_as_float(a << 16), __uint_as_float(a & 0xFFFF0000u));
      const CodePair cp = code_pair<CLAMP>(x, pr.nz, pr.r, qmax);
      const uint2 bits = make_uint2(__float_as_uint(cp.m.x), __float_as_uint(cp.m.y));
      if constexpr (F32ERR) {
        add_error2(acc, x, cp, pr.ns);
      } else {
        add_error(e, x.x, bits.x, pr.zs0);
        add_error(e, x.y, bits.y, pr.zs1);
      }
      // (bits - bias) << shift is the code in place; words only gain disjoint fields
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t c = (j ? bits.y : bits.x) - kRintBias;
        if constexpr (BITS == 4) w[i] += c << (4 * (p + 4 * j));
        else if constexpr (BITS == 2) w[i >> 1] += c << (2 * (4 * (i & 1) + p + 8 * j));
        else w[2 * i + (p >> 1)] += c << (8 * (2 * (p & 1) + j));
      }
    };
    if constexpr (MODE == 0) {
      // parameters by channel 16dt + 2t + j + 8(p>>1): shared by both token halves
#pragma unroll
      for (int d2 = 0; d2 < TPV / 2; ++d2) {
        const int dt = vi * (TPV / 2) + d2;
        const Pair pr[2] = {load_pair(16 * dt + 2 * t, false), load_pair(16 * dt + 2 * t + 8, false)};
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          uint32_t a[4];
          load_tile<RS>(a, xs, false, dt, tt, lane);
#pragma unroll
          for (int p = 0; p < 4; ++p) put(2 * d2 + tt, p, a[p], pr[p >> 1]);
        }
      }
    } else {
      // parameters by token 16tt + g + 8(p&1) (keys, MODE 1) or 16tt + 2t + j + 8(p>>1)
      // (values): shared by every tile row of a token half
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const Pair pr[2] = {MODE == 1 ? load_pair(16 * tt + g, true) : load_pair(16 * tt + 2 * t, false),
                            MODE == 1 ? load_pair(16 * tt + g + 8, true) : load_pair(16 * tt + 2 * t + 8, false)};
#pragma unroll
        for (int d2 = 0; d2 < TPV / 2; ++d2) {
          const int dt = vi * (TPV / 2) + d2;
          uint32_t a[4];
          load_tile<RS>(a, xs, MODE == 2, dt, tt, lane);
#pragma unroll
          for (int p = 0; p < 4; ++p) put(2 * d2 + tt, p, a[p], pr[MODE == 1 ? (p & 1) : (p >> 1)]);
        }
      }
    }
    reinterpret_cast<uint4*>(blk)[v] = make_uint4(w[0], w[1], w[2], w[3]);
    if constexpr (F32ERR) {
      e[0] += (double)acc[0].x + (double)acc[0].y;
      e[1] += (double)acc[1].x + (double)acc[1].y;
    }
  }
}

// bf16 block (a bf16 layer): the tile registers are the block's words.
template <int D, int RS>
__device__ __forceinline__ void emit_bf16(uint8_t* blk, const __nv_bfloat16 (*xs)[RS], bool is_value) {
  constexpr int kVectors = (int)(code_block_bytes(16, D) / 16);
  const int lane = threadIdx.x & 31;
  for (int v = threadIdx.x; v < kVectors; v += kThreads) {
    const int f = v >> 5;
    uint32_t a[4];
    load_tile<RS>(a, xs, is_value, f >> 1, f & 1, lane);
    reinterpret_cast<uint4*>(blk)[v] = make_uint4(a[0], a[1], a[2], a[3]);
  }
}

template <int KB, int VB, int D, bool F32IN>
__global__ void __launch_bounds__(kThreads, 4) append_kernel(AppendParams a) {
  pdl_enter();
  constexpr bool kBf16Layer = (KB == 16);
  constexpr int RS = D + 8;          // bf16 row stride of the staged rows (16-byte rows, staggered banks)
  constexpr int NP = D > 32 ? D : 32;
  const int b = blockIdx.z, h = blockIdx.y, item = blockIdx.x;
  const int H = a.n_kv_heads;
  __shared__ __align__(16) __nv_bfloat16 xsb[2][2][kPageTokens][RS];  // two groups' key and value rows
  __shared__ __align__(16) float qnz[2][NP];    // quantizer -z by index: keys, values
  __shared__ __align__(16) float qr[2][NP];     // 1/s (0 for a constant set)
  __shared__ __align__(16) float qns[2][NP];    // -s
  __shared__ unsigned s_amax;                   // largest |min| or |max| of the group's sets (float bits)
  __shared__ int s_clamp;                       // a set of the group had z or s clamped to fp16's range
  __shared__ __align__(16) double2 qzs[2][NP];  // z, s in fp64 (error report)
  constexpr int KP = D / 2, KS = kThreads / KP;  // key channel pairs, token splits of the key pass
  __shared__ __nv_bfloat162 kpart[KS][2][KP];   // per-split min, max of each key channel pair
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
    // this CTA's groups are item, item + gridDim.x, ...; the next group's rows
    // are staged (asynchronous 16-byte copies for bf16 inputs) while one group
    // is quantized
    constexpr int VPR = D / 8;
    auto stage = [&](int it, int buf) {
      const int g = g0 + it;
      for (int v = threadIdx.x; v < 2 * kPageTokens * VPR; v += kThreads) {
        const int r = v / (kPageTokens * VPR), rem = v % (kPageTokens * VPR);
        const int tk = rem / VPR, c8 = (rem % VPR) * 8;
        const int tau = g * kPageTokens + tk;  // old window slots first
        const bool from_win = tau < T0;
        const int64_t idx = ((off + (tau - T0)) * H + h) * D + c8;
        const __nv_bfloat16* wsrc = win + (r * kPageTokens + (tau % kPageTokens)) * D + c8;
        if constexpr (F32IN) {
          *reinterpret_cast<uint4*>(&xsb[buf][r][tk][c8]) =
              from_win ? *reinterpret_cast<const uint4*>(wsrc) : load8<true>(r ? a.V : a.K, idx);
        } else {
          cp_async16(&xsb[buf][r][tk][c8],
                     from_win ? wsrc : reinterpret_cast<const __nv_bfloat16*>(r ? a.V : a.K) + idx);
        }
      }
      cp_async_commit();
    };
    double err[4] = {0.0, 0.0, 0.0, 0.0};  // this thread's share of the error report
    int groups = 0;
    stage(item, 0);
    for (int it = item, buf = 0; it < ng; it += gridDim.x, buf ^= 1, ++groups) {
      if (it + (int)gridDim.x < ng) {
        stage(it + (int)gridDim.x, buf ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      const int g = g0 + it;
      uint8_t* page = a.pages + ((int64_t)(b * H + h) * a.max_pages + g) * a.page_bytes;
      auto& xs = xsb[buf];
      if (threadIdx.x == 0) {
        s_amax = 0u;
        s_clamp = 0;
      }
      __syncthreads();
      if constexpr (kBf16Layer) {
        emit_bf16<D, RS>(page, xs[0], false);
        emit_bf16<D, RS>(page + code_block_bytes(16, D), xs[1], true);
      } else {
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
          auto keep = [&](int r, int i, const QParams& q, float mn, float mx) {
            atomicMax(&s_amax, __float_as_uint(fmaxf(fabsf(mn), fabsf(mx))));  // bits order = value order
            if (q.z > mn || __half2float(q.s_h) >= 65504.0f) atomicOr(&s_clamp, 1);
            qnz[r][i] = -q.z;
            qns[r][i] = -__half2float(q.s_h);
            qr[r][i] = q.r;  // 0 for a constant set
            qzs[r][i] = make_double2((double)q.z, (double)__half2float(q.s_h));
          };
          // per-token sets (values; keys in per-token mode): four threads per token,
          // thread u taking the bf16 pairs u, u + 4, ... of the row
          auto token_params = [&](int r, int qmax, __half* sdst, __half* zdst) {
            const int tok = threadIdx.x >> 2, u = threadIdx.x & 3;
            const __nv_bfloat162* row = reinterpret_cast<const __nv_bfloat162*>(&xs[r][tok][0]);
            __nv_bfloat162 mn = row[u], mx = mn;
#pragma unroll
            for (int k = 1; k < D / 8; ++k) {
              mn = __hmin2(mn, row[u + 4 * k]);
              mx = __hmax2(mx, row[u + 4 * k]);
            }
            float fmn = fminf(__low2float(mn), __high2float(mn)), fmx = fmaxf(__low2float(mx), __high2float(mx));
#pragma unroll
            for (int o = 1; o < 4; o <<= 1) {
              fmn = fminf(fmn, __shfl_xor_sync(0xffffffffu, fmn, o));
              fmx = fmaxf(fmx, __shfl_xor_sync(0xffffffffu, fmx, o));
            }
            if (u == 0) {
              const QParams q = make_qparams(fmn, fmx, qmax);
              sdst[tok] = q.s_h;
              zdst[tok] = q.z_h;
              keep(r, tok, q, fmn, fmx);
            }
          };
          token_params(1, (1 << VB) - 1, vscale, vzero);
          if (per_token_keys) {
            token_params(0, (1 << KB) - 1, kscale, kzero);
          } else {
            // keys per channel: thread (split, pair) scans 32/KS tokens of one channel
            // pair; the splits are then combined, one thread per channel
            const int pi = threadIdx.x % KP, sp = threadIdx.x / KP;
            const __nv_bfloat162* col = reinterpret_cast<const __nv_bfloat162*>(&xs[0][sp * (kPageTokens / KS)][0]) + pi;
            __nv_bfloat162 mn = col[0], mx = mn;
#pragma unroll
            for (int k = 1; k < kPageTokens / KS; ++k) {
              mn = __hmin2(mn, col[k * (RS / 2)]);
              mx = __hmax2(mx, col[k * (RS / 2)]);
            }
            kpart[sp][0][pi] = mn;
            kpart[sp][1][pi] = mx;
            __syncthreads();
            for (int d = threadIdx.x; d < D; d += kThreads) {
              float fmn = 0.0f, fmx = 0.0f;
#pragma unroll
              for (int k = 0; k < KS; ++k) {
                const __nv_bfloat162 m0 = kpart[k][0][d >> 1], m1 = kpart[k][1][d >> 1];
                const float x0 = (d & 1) ? __high2float(m0) : __low2float(m0);
                const float x1 = (d & 1) ? __high2float(m1) : __low2float(m1);
                fmn = k ? fminf(fmn, x0) : x0;
                fmx = k ? fmaxf(fmx, x1) : x1;
              }
              const QParams q = make_qparams(fmn, fmx, (1 << KB) - 1);
              const int slot = kmeta_slot<D>(d);
              kscale[slot] = q.s_h;
              kzero[slot] = q.z_h;
              keep(0, d, q, fmn, fmx);
            }
          }
          __syncthreads();
          // codes, each element quantized as it is packed, and its error report terms
          double ek[2] = {0.0, 0.0}, ev[2] = {0.0, 0.0};
          const QTab tk{qnz[0], qr[0], qns[0], qzs[0]}, tv{qnz[1], qr[1], qns[1], qzs[1]};
          const float amax = __uint_as_float(s_amax);
          if (amax >= 0x1p-14f && amax < 0x1p40f && !s_clamp) {
            if (per_token_keys) emit_codes<KB, D, RS, 1, true, false>(page, xs[0], tk, ek);
            else emit_codes<KB, D, RS, 0, true, false>(page, xs[0], tk, ek);
            emit_codes<VB, D, RS, 2, true, false>(vblk, xs[1], tv, ev);
          } else if (amax >= 0x1p-14f && amax < 0x1p40f) {
            if (per_token_keys) emit_codes<KB, D, RS, 1, true, true>(page, xs[0], tk, ek);
            else emit_codes<KB, D, RS, 0, true, true>(page, xs[0], tk, ek);
            emit_codes<VB, D, RS, 2, true, true>(vblk, xs[1], tv, ev);
          } else {
            if (per_token_keys) emit_codes<KB, D, RS, 1, false, true>(page, xs[0], tk, ek);
            else emit_codes<KB, D, RS, 0, false, true>(page, xs[0], tk, ek);
            emit_codes<VB, D, RS, 2, false, true>(vblk, xs[1], tv, ev);
          }
          err[0] += ek[0];
          err[1] += ek[1];
          err[2] += ev[0];
          err[3] += ev[1];
        }
      }
      __syncthreads();  // the staged rows and the parameter tables are reused
    }
    if constexpr (!kBf16Layer) {
      // this CTA's error sums: warp shuffles, then one fp64 atomic per sum into
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
      if (bin && threadIdx.x == 4) atomicAdd(&bin[4], (double)groups * (kPageTokens * D));
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
