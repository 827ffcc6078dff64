// kvq_quant.cuh -- the quantizer and the fragment-order packing shared by the
// append kernel (CTA-wide flush) and the fused decode step (warp-level flush).
//
// Quantizer (bit-exact contract with the CPU oracle; every fp32 step is a
// single IEEE operation, the __f*_rn intrinsics are never contracted):
//   mn, mx = min, max (signed zeros canonicalised to +0)
//   z = fp16_round_down(mn) clamped to >= -65504
//   s = fp16_round_up((mx - z) / qmax) clamped to <= 65504
//   code = s == 0 ? 0 : clamp(rint((x - z) * (1/s)), 0, qmax)
#pragma once

#include "kvq_internal.cuh"

namespace kvq {
namespace {

struct QParams {
  float z, r;
  __half s_h, z_h;
  bool zero_scale;
};

__device__ __forceinline__ QParams make_qparams(float mn, float mx, int qmax) {
  QParams q;
  mn = __fadd_rn(mn, 0.0f);
  mx = __fadd_rn(mx, 0.0f);
  float z = __half2float(__float2half_rd(mn));
  z = fmaxf(z, -65504.0f);
  float d = __fsub_rn(mx, z);
  float ratio = __fdiv_rn(d, (float)qmax);
  float s = __half2float(__float2half_ru(ratio));
  s = fminf(s, 65504.0f);
  q.z = z;
  q.s_h = __float2half_rn(s);   // exact: s is an fp16 value
  q.z_h = __float2half_rn(z);
  q.zero_scale = (s == 0.0f);
  q.r = q.zero_scale ? 0.0f : __fdiv_rn(1.0f, s);
  return q;
}

__device__ __forceinline__ uint32_t quant_code(float x, const QParams& q, int qmax) {
  if (q.zero_scale) return 0u;
  float y = __fmul_rn(__fsub_rn(x, q.z), q.r);
  int c = __float2int_rn(y);
  c = c < 0 ? 0 : (c > qmax ? qmax : c);
  return (uint32_t)c;
}

// Element e of tile f for lane l: (token, channel) it stores.
__device__ __forceinline__ void tile_elem(int f, int lane, int e, bool is_value, int& tok, int& dim) {
  int dt = f >> 1, tt = f & 1;
  int g = lane >> 2, t = lane & 3;
  int p = e >> 1, j = e & 1;
  int row = g + 8 * (p & 1);
  int col = 2 * t + j + 8 * (p >> 1);
  if (is_value) { dim = 16 * dt + row; tok = 16 * tt + col; }
  else          { tok = 16 * tt + row; dim = 16 * dt + col; }
}

// Lane word w of lane `lane` for a block of `BITS`-bit elements read from
// vals(tok, dim).
template <int BITS, typename Get>
__device__ __forceinline__ uint32_t lane_word(int lane, int w, bool is_value, Get vals) {
  uint32_t word = 0;
  int tok, dim;
  if constexpr (BITS == 8) {
    int f = w >> 1, half = w & 1;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      tile_elem(f, lane, 4 * half + k, is_value, tok, dim);
      word |= (vals(tok, dim) & 0xFFu) << (8 * k);
    }
  } else if constexpr (BITS == 4) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      tile_elem(w, lane, e, is_value, tok, dim);
      word |= (vals(tok, dim) & 0xFu) << (4 * ((e >> 1) + 4 * (e & 1)));
    }
  } else if constexpr (BITS == 2) {
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        tile_elem(2 * w + u, lane, e, is_value, tok, dim);
        word |= (vals(tok, dim) & 0x3u) << (2 * (4 * u + (e >> 1) + 8 * (e & 1)));
      }
  } else {  // 16-bit (bf16 bit patterns)
    int f = w >> 2, pair = w & 3;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      tile_elem(f, lane, 2 * pair + k, is_value, tok, dim);
      word |= (vals(tok, dim) & 0xFFFFu) << (16 * k);
    }
  }
  return word;
}

// Key scale/zero slot of channel d (inverse of the documented permutation).
template <int D>
__device__ __forceinline__ int kmeta_slot(int d) {
  int dt = d >> 4, r = d & 15;
  int j = (r & 1) + 2 * (r >> 3);
  int t = (r & 7) >> 1;
  return t * (D / 4) + dt * 4 + j;
}

}  // namespace
}  // namespace kvq
