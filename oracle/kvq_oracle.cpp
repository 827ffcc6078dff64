// kvq_oracle.cpp -- plain CPU oracle for layer-wise mixed-precision KV decode.
//
// TEST INFRASTRUCTURE ONLY. This file is the slow, obviously-correct restatement
// of what the CUDA path computes. Only the tests, the smoke check and the
// benchmark's CPU-baseline leg may load it; the product library never does, and
// the two share no source, header, table or helper.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -shared -fPIC -pthread.
// -ffp-contract=off keeps every fp32 multiply and add a separate IEEE
// operation, which is what makes the packed codes reproducible bit for bit.
//
// What each part follows (sources are the KVTuner pages):
//  * equivalent bitwidth -- llms-explorer "Mixed-precision KV-cache quantization
//    per-layer" facts (3.25-bit Llama-3.1-8B, 4.0-bit Qwen2.5-7B) and the
//    arXiv 2502.04420 abstract: average over layers of (k_bits + v_bits)/2.
//  * byte accounting -- machinoai Q&A, section 2 worked example (BF16 layer 100
//    MiB, FP8 layer half of it, scales and metadata ignored).
//  * key quantizer -- per-channel asymmetric over a token group (facts page;
//    OpenReview rebuttal on KIVI's per-channel per-group keys); group = 32.
//    Second key mode: per-token asymmetric, one (scale, zero) per key token over
//    the head dimension, exactly like values (OpenReview rebuttal, section 4
//    "Per-channel vs. per-token quantization"; facts page: the two modes give
//    different Pareto-optimal pairs). The mode is a per-layer setting.
//  * value quantizer -- per-token asymmetric (OpenReview rebuttal, "value
//    per-token-asym").
//  * only new tokens are quantized, with the layer's fixed pair (OpenReview
//    rebuttal, "Computational cost"); the not-yet-quantized tail (< 32 tokens)
//    stays bf16.
//  * attention -- plain softmax(q.k / sqrt(D)) v decode attention with GQA
//    (OpenReview rebuttal, "New GQA efficiency results"), evaluated in fp64.
//
// Readings where the pages are silent (each also listed in the design notes):
//  * asymmetric = min/max with a float zero point z = group minimum rounded
//    toward -inf to fp16, scale s = (max - z)/qmax rounded toward +inf to fp16,
//    code = clamp(rint((x - z) * (1/s)), 0, qmax), rint = round-half-even.
//    z is clamped to >= -65504 and s to <= 65504 (fp16 finite range).
//  * s == 0 (constant group whose value is fp16-representable): codes are 0.
//  * signed zeros: the min and max of a set are taken as +0 when they are zero.
//  * fp32 inputs are rounded to bf16 (round-to-nearest-even) at entry.
//  * q head h reads KV head h / (Hq/Hkv); softmax scale 1/sqrt(D); no mask.
//  * empty sequence: output 0.
//  * per-token key mode keeps the same 32-token pages and bf16 residual window:
//    a key token is quantized when its page fills, like a value token.
//  * per-layer quantization error report (OpenReview rebuttal, Table 3 and the
//    layer-wise error figures the pages cite: quantization error is tracked
//    per layer): sums over every element a page flush quantizes of
//    (x - x_hat)^2 and x^2, keys and values separately, in fp64, plus the
//    element counts; bf16 layers add nothing.
//  * FP8 layer format (llms-explorer facts page: vLLM-style FP8 KV cache with
//    per-attention-head scales and BF16 skip layers; machinoai Q&A section 2
//    worked example of BF16 and FP8 layers): each key/value element of KV head
//    h is stored as e4m3(x / s_h) with a per-layer, per-head fp32 scale s_h
//    (k and v scales separate, calibrated offline, an input here, default 1).
//    e4m3 = 1 sign, 4 exponent (bias 7), 3 mantissa bits, no infinities,
//    largest finite 448; rounding to nearest, ties to even, and magnitudes
//    above 448 saturate to 448. Dequantized value: e4m3 value * s_h. Same
//    32-token pages (no per-page metadata) and bf16 residual window.
//
// The packed page layout implemented here is the library's documented storage
// format (written out independently below from its definition).

#include <cstdint>
#include <cstring>
#include <cmath>
#include <cstdlib>
#include <vector>
#include <algorithm>
#include <atomic>
#include <thread>
#include <utility>

namespace {

// ---------------------------------------------------------------- formats --

float bits_to_f32(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }
uint32_t f32_to_bits(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }

// fp32 -> bf16, round to nearest, ties to even (finite inputs; NaN kept quiet).
uint16_t f32_to_bf16_rne(float x) {
  if (std::isnan(x)) return 0x7FC0;
  // The bf16 neighbours of x are x with the low 16 bits cleared (toward zero)
  // and the next one away from zero. Pick by comparing the dropped half.
  uint32_t u = f32_to_bits(x);
  uint32_t hi = u >> 16;
  uint32_t lo = u & 0xFFFFu;
  if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1;  // carries into exponent correctly
  return (uint16_t)hi;
}

float bf16_to_f32(uint16_t h) { return bits_to_f32(((uint32_t)h) << 16); }

// Exact value of an fp16 bit pattern as a double.
double f16_value(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0) v = std::ldexp((double)m, -24);                 // subnormal / zero
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = std::ldexp((double)(1024 + m), e - 25);           // (1 + m/1024) * 2^(e-15)
  return sign ? -v : v;
}

// Encode a double that is exactly representable in fp16 (or +-inf) as bits.
uint16_t f16_encode_exact(double v, bool negative_zero) {
  uint16_t sign = (v < 0 || (v == 0 && negative_zero)) ? 0x8000 : 0;
  double a = std::fabs(v);
  if (std::isinf(a)) return sign | 0x7C00;
  if (a == 0) return sign;
  if (a < std::ldexp(1.0, -14)) {                              // subnormal: a = m * 2^-24
    double m = std::ldexp(a, 24);
    return sign | (uint16_t)m;
  }
  int k;                                                       // a = f * 2^k, f in [0.5, 1)
  std::frexp(a, &k);
  int e = k - 1;                                               // a in [2^e, 2^(e+1))
  double mant = std::ldexp(a, 10 - e) - 1024.0;                // 0..1023, exact
  return sign | (uint16_t)((e + 15) << 10) | (uint16_t)mant;
}

// fp32 -> fp16 with a directed rounding: the largest fp16 <= x (down) or the
// smallest fp16 >= x (up). Written from the definition: scale x by the fp16
// spacing of its binade, take floor/ceil, scale back (all exact in double).
uint16_t f32_to_f16_directed(float xf, bool up) {
  double x = (double)xf;
  if (std::isnan(x)) return 0x7E00;
  if (x == 0) return std::signbit(xf) ? 0x8000 : 0;
  const double fmax = 65504.0;
  if (std::isinf(x)) return x > 0 ? 0x7C00 : 0xFC00;
  int k;
  std::frexp(std::fabs(x), &k);
  int e = std::max(k - 1, -14);                                // exponent of x's binade (subnormals share -14)
  double ulp = std::ldexp(1.0, e - 10);
  double q = x / ulp;                                          // exact: division by a power of two
  double r = up ? std::ceil(q) : std::floor(q);
  double v = r * ulp;                                          // may step into the next binade: still exact
  if (v > fmax) return up ? 0x7C00 : f16_encode_exact(fmax, false);
  if (v < -fmax) return up ? f16_encode_exact(-fmax, false) : 0xFC00;
  return f16_encode_exact(v, v == 0 && x < 0);
}

// ------------------------------------------------------------------ e4m3 --

// Value of an e4m3 bit pattern (NaN for S.1111.111).
double e4m3_value(uint8_t c) {
  int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return NAN;
  double v = (e == 0) ? std::ldexp((double)m, -9) : std::ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -v : v;
}

// fp32 -> e4m3: round to nearest, ties to even, saturating at 448 (inf too).
// Written from the definition: the spacing of the e4m3 grid around |x| is
// 2^-9 below 2^-6 (subnormals) and 2^(floor(log2|x|) - 3) above; all exact
// in double.
uint8_t e4m3_encode(float xf) {
  double x = xf;
  uint8_t sign = std::signbit(xf) ? 0x80 : 0x00;
  double a = std::fabs(x);
  if (!(a < 448.0)) return sign | 0x7E;  // 448 (this also saturates inf)
  double spacing;
  if (a < std::ldexp(1.0, -6)) {
    spacing = std::ldexp(1.0, -9);
  } else {
    int ex;
    std::frexp(a, &ex);  // a = f * 2^ex, f in [0.5, 1)
    spacing = std::ldexp(1.0, ex - 1 - 3);
  }
  double q = a / spacing;               // exact (power-of-two spacing)
  double r = std::floor(q);
  double frac = q - r;
  if (frac > 0.5 || (frac == 0.5 && std::fmod(r, 2.0) != 0.0)) r += 1.0;
  double v = r * spacing;               // rounded magnitude, <= 448
  if (v > 448.0) v = 448.0;
  if (v == 0.0) return sign;
  // encode v: subnormal if below 2^-6
  if (v < std::ldexp(1.0, -6)) return sign | (uint8_t)(v / std::ldexp(1.0, -9));
  int ex;
  double f = std::frexp(v, &ex);        // v = f * 2^ex, f in [0.5, 1)
  int e = ex - 1 + 7;                   // biased exponent of 1.m form
  int m = (int)((f * 2.0 - 1.0) * 8.0);  // exact: v has 3 fraction bits
  return sign | (uint8_t)(e << 3) | (uint8_t)m;
}

// ------------------------------------------------------------- quantizer --

// Quantize n values (already bf16-exact fp32) to `bits`-bit unsigned codes with
// one fp16 scale and one fp16 zero. Every fp32 operation is a single IEEE op.
void quantize_set(const float* x, int n, int bits, uint8_t* codes,
                  uint16_t* scale_bits, uint16_t* zero_bits) {
  const int qmax = (1 << bits) - 1;
  float mn = x[0], mx = x[0];
  for (int i = 1; i < n; ++i) { mn = std::min(mn, x[i]); mx = std::max(mx, x[i]); }
  // A set whose minimum (or maximum) is zero may hold both -0 and +0; which one
  // the min/max returns depends on order. Adding +0 makes either one +0.
  mn = mn + 0.0f;
  mx = mx + 0.0f;
  uint16_t zb = f32_to_f16_directed(mn, /*up=*/false);
  float z = (float)f16_value(zb);
  if (z < -65504.0f) { z = -65504.0f; zb = f16_encode_exact(-65504.0, false); }
  float d = mx - z;
  float ratio = d / (float)qmax;
  uint16_t sb = f32_to_f16_directed(ratio, /*up=*/true);
  float s = (float)f16_value(sb);
  if (s > 65504.0f) { s = 65504.0f; sb = f16_encode_exact(65504.0, false); }
  *scale_bits = sb;
  *zero_bits = zb;
  if (s == 0.0f) {
    for (int i = 0; i < n; ++i) codes[i] = 0;
    return;
  }
  float r = 1.0f / s;
  for (int i = 0; i < n; ++i) {
    float t = x[i] - z;
    float y = t * r;
    float c = std::nearbyint(y);                               // default mode: ties to even
    if (c < 0.0f) c = 0.0f;
    if (c > (float)qmax) c = (float)qmax;
    codes[i] = (uint8_t)c;
  }
}

// ---------------------------------------------------------------- layout --
//
// One page = 32 consecutive tokens of one (sequence, KV head):
//   [K code block][V code block][K scales (D fp16)][K zeros (D fp16)]
//   [V scales (32 fp16)][V zeros (32 fp16)]          (quantized pair)
//   per-token key mode: [K scales (32 fp16)][K zeros (32 fp16)] in token order
//   take the place of the D key scales and zeros
//   [K block (bf16)][V block (bf16)]                 (bf16 layer)
// A code block is split into 16x16 tiles f = 2*dt + tt (dt: 16-dim tile,
// tt: 16-token tile). In tile f, lane l = 4g + t owns 8 elements e = 2p + j:
//   row = g + 8*(p & 1), col = 2t + j + 8*(p >> 1)
// K tiles have row = token, col = dim; V tiles have row = dim, col = token.
// Each lane's elements form a stream of 32-bit words:
//   8-bit: tile f -> words 2f, 2f+1; element e in byte e of the pair
//   4-bit: tile f -> word f; element e in nibble (e >> 1) + 4*(e & 1)
//   2-bit: tiles 2w, 2w+1 -> word w; element e of tile 2w+u in 2-bit slot
//          4u + (e >> 1) + 8*(e & 1)
//   bf16 : tile f -> words 4f..4f+3; element e in half-word e
// Lane word w of lane l lives at byte ((w/4)*32 + l)*16 + (w%4)*4 of the block.
// K scale/zero index i (0..D-1) holds channel 16*dt + 2t + (j&1) + 8*(j>>1)
// with t = i / (D/4), dt = (i % (D/4)) / 4, j = i % 4.

struct Elem { int row, col; };

Elem tile_elem(int g, int t, int e) {
  int p = e >> 1, j = e & 1;
  return Elem{g + 8 * (p & 1), 2 * t + j + 8 * (p >> 1)};
}

// Bit offset (within the lane's word stream) of element e of tile f.
int64_t stream_bit(int bits, int f, int e) {
  if (bits == 8) return (int64_t)f * 64 + e * 8;
  if (bits == 4) return (int64_t)f * 32 + 4 * ((e >> 1) + 4 * (e & 1));
  if (bits == 2) return (int64_t)(f >> 1) * 32 + 2 * (4 * (f & 1) + (e >> 1) + 8 * (e & 1));
  return (int64_t)f * 128 + e * 16;                            // bf16
}

int64_t word_byte(int lane, int64_t w) { return ((w / 4) * 32 + lane) * 16 + (w % 4) * 4; }

int64_t code_block_bytes(int bits, int D) { return (int64_t)32 * D * bits / 8; }

// key_mode: 0 = per-channel keys (D scale/zero pairs), 1 = per-token keys (32).
// fmt: 0 = integer codes with fp16 scale/zero, 1 = fp8 e4m3 (8/8 bits, no page metadata).
int64_t page_bytes(int kb, int vb, int D, int key_mode, int fmt) {
  int64_t b = code_block_bytes(kb, D) + code_block_bytes(vb, D);
  if (kb != 16 && !fmt) b += (key_mode ? 128 : (int64_t)4 * D) + 128;
  return b;
}

int kmeta_channel(int i, int D) {
  int t = i / (D / 4), dt = (i % (D / 4)) / 4, j = i % 4;
  return 16 * dt + 2 * t + (j & 1) + 8 * (j >> 1);
}

// Write value v (bits wide) of element (row, col) belonging to lane/tile/elem.
void put_bits(uint8_t* blk, int lane, int64_t bit, int bits, uint32_t v) {
  int64_t w = bit / 32;
  int sh = (int)(bit % 32);
  uint8_t* p = blk + word_byte(lane, w);
  uint32_t word;
  std::memcpy(&word, p, 4);
  uint32_t mask = (bits == 32) ? 0xFFFFFFFFu : ((1u << bits) - 1u);
  word = (word & ~(mask << sh)) | ((v & mask) << sh);
  std::memcpy(p, &word, 4);
}

uint32_t get_bits(const uint8_t* blk, int lane, int64_t bit, int bits) {
  int64_t w = bit / 32;
  int sh = (int)(bit % 32);
  uint32_t word;
  std::memcpy(&word, blk + word_byte(lane, w), 4);
  uint32_t mask = (1u << bits) - 1u;
  return (word >> sh) & mask;
}

// vals[token][dim] (codes, or bf16 bit patterns for the bf16 layer).
void pack_block(uint8_t* blk, const uint16_t* vals, int D, int bits, bool is_value) {
  int F = 2 * (D / 16);
  for (int f = 0; f < F; ++f) {
    int dt = f >> 1, tt = f & 1;
    for (int lane = 0; lane < 32; ++lane) {
      int g = lane >> 2, t = lane & 3;
      for (int e = 0; e < 8; ++e) {
        Elem el = tile_elem(g, t, e);
        int tok = is_value ? 16 * tt + el.col : 16 * tt + el.row;
        int dim = is_value ? 16 * dt + el.row : 16 * dt + el.col;
        put_bits(blk, lane, stream_bit(bits, f, e), bits, vals[tok * D + dim]);
      }
    }
  }
}

void unpack_block(const uint8_t* blk, uint16_t* vals, int D, int bits, bool is_value) {
  int F = 2 * (D / 16);
  for (int f = 0; f < F; ++f) {
    int dt = f >> 1, tt = f & 1;
    for (int lane = 0; lane < 32; ++lane) {
      int g = lane >> 2, t = lane & 3;
      for (int e = 0; e < 8; ++e) {
        Elem el = tile_elem(g, t, e);
        int tok = is_value ? 16 * tt + el.col : 16 * tt + el.row;
        int dim = is_value ? 16 * dt + el.row : 16 * dt + el.col;
        vals[tok * D + dim] = (uint16_t)get_bits(blk, lane, stream_bit(bits, f, e), bits);
      }
    }
  }
}

// Build one page from 32 tokens of bf16 keys/values ([32][D] bit patterns).
// fp8 pages: ksc/vsc are the KV head's fp32 key and value scales.
void build_page(uint8_t* page, const uint16_t* kbf, const uint16_t* vbf, int D, int kb, int vb, int key_mode,
                int fmt, float ksc, float vsc) {
  std::memset(page, 0, (size_t)page_bytes(kb, vb, D, key_mode, fmt));
  uint8_t* kblk = page;
  uint8_t* vblk = page + code_block_bytes(kb, D);
  if (kb == 16) {
    pack_block(kblk, kbf, D, 16, false);
    pack_block(vblk, vbf, D, 16, true);
    return;
  }
  if (fmt) {
    std::vector<uint16_t> kc(32 * D), vc(32 * D);
    for (int i = 0; i < 32 * D; ++i) {
      kc[i] = e4m3_encode(bf16_to_f32(kbf[i]) / ksc);  // one IEEE fp32 division
      vc[i] = e4m3_encode(bf16_to_f32(vbf[i]) / vsc);
    }
    pack_block(kblk, kc.data(), D, 8, false);
    pack_block(vblk, vc.data(), D, 8, true);
    return;
  }
  const int nk = key_mode ? 32 : D;  // key scale/zero pairs in the page
  uint8_t* kscale = vblk + code_block_bytes(vb, D);
  uint8_t* kzero = kscale + 2 * nk;
  uint8_t* vscale = kzero + 2 * nk;
  uint8_t* vzero = vscale + 64;
  std::vector<uint16_t> kc(32 * D), vc(32 * D);
  std::vector<float> col(32), row(D);
  std::vector<uint8_t> codes(std::max(32, D));
  std::vector<uint16_t> ks(D), kz(D);
  if (key_mode) {
    // keys: one set per token over the head dimension
    for (int t = 0; t < 32; ++t) {
      for (int d = 0; d < D; ++d) row[d] = bf16_to_f32(kbf[t * D + d]);
      uint16_t sb, zb;
      quantize_set(row.data(), D, kb, codes.data(), &sb, &zb);
      for (int d = 0; d < D; ++d) kc[t * D + d] = codes[d];
      std::memcpy(kscale + 2 * t, &sb, 2);
      std::memcpy(kzero + 2 * t, &zb, 2);
    }
  } else {
    // keys: one set per channel over the page's 32 tokens
    for (int d = 0; d < D; ++d) {
      for (int t = 0; t < 32; ++t) col[t] = bf16_to_f32(kbf[t * D + d]);
      quantize_set(col.data(), 32, kb, codes.data(), &ks[d], &kz[d]);
      for (int t = 0; t < 32; ++t) kc[t * D + d] = codes[t];
    }
  }
  // values: one set per token over the head dimension
  for (int t = 0; t < 32; ++t) {
    for (int d = 0; d < D; ++d) row[d] = bf16_to_f32(vbf[t * D + d]);
    uint16_t sb, zb;
    quantize_set(row.data(), D, vb, codes.data(), &sb, &zb);
    for (int d = 0; d < D; ++d) vc[t * D + d] = codes[d];
    std::memcpy(vscale + 2 * t, &sb, 2);
    std::memcpy(vzero + 2 * t, &zb, 2);
  }
  pack_block(kblk, kc.data(), D, kb, false);
  pack_block(vblk, vc.data(), D, vb, true);
  if (!key_mode) {
    for (int i = 0; i < D; ++i) {
      int d = kmeta_channel(i, D);
      std::memcpy(kscale + 2 * i, &ks[d], 2);
      std::memcpy(kzero + 2 * i, &kz[d], 2);
    }
  }
}

// Dequantize one page into [32][D] doubles (x = code * s + z, exact in fp64).
void dequant_page(const uint8_t* page, int D, int kb, int vb, int key_mode, int fmt, float ksc, float vsc,
                  double* Kh, double* Vh) {
  std::vector<uint16_t> kc(32 * D), vc(32 * D);
  const uint8_t* kblk = page;
  const uint8_t* vblk = page + code_block_bytes(kb, D);
  unpack_block(kblk, kc.data(), D, kb, false);
  unpack_block(vblk, vc.data(), D, vb, true);
  if (kb == 16) {
    for (int i = 0; i < 32 * D; ++i) { Kh[i] = bf16_to_f32(kc[i]); Vh[i] = bf16_to_f32(vc[i]); }
    return;
  }
  if (fmt) {
    for (int i = 0; i < 32 * D; ++i) {
      Kh[i] = e4m3_value((uint8_t)kc[i]) * (double)ksc;
      Vh[i] = e4m3_value((uint8_t)vc[i]) * (double)vsc;
    }
    return;
  }
  const int nk = key_mode ? 32 : D;
  const uint8_t* kscale = vblk + code_block_bytes(vb, D);
  const uint8_t* kzero = kscale + 2 * nk;
  const uint8_t* vscale = kzero + 2 * nk;
  const uint8_t* vzero = vscale + 64;
  if (key_mode) {
    for (int t = 0; t < 32; ++t) {
      uint16_t sb, zb;
      std::memcpy(&sb, kscale + 2 * t, 2);
      std::memcpy(&zb, kzero + 2 * t, 2);
      double ks = f16_value(sb), kz = f16_value(zb);
      for (int d = 0; d < D; ++d) Kh[t * D + d] = (double)kc[t * D + d] * ks + kz;
    }
  } else {
    std::vector<double> s(D), z(D);
    for (int i = 0; i < D; ++i) {
      uint16_t sb, zb;
      std::memcpy(&sb, kscale + 2 * i, 2);
      std::memcpy(&zb, kzero + 2 * i, 2);
      int d = kmeta_channel(i, D);
      s[d] = f16_value(sb);
      z[d] = f16_value(zb);
    }
    for (int t = 0; t < 32; ++t)
      for (int d = 0; d < D; ++d) Kh[t * D + d] = (double)kc[t * D + d] * s[d] + z[d];
  }
  for (int t = 0; t < 32; ++t) {
    uint16_t sb, zb;
    std::memcpy(&sb, vscale + 2 * t, 2);
    std::memcpy(&zb, vzero + 2 * t, 2);
    double vs = f16_value(sb), vz = f16_value(zb);
    for (int d = 0; d < D; ++d) Vh[t * D + d] = (double)vc[t * D + d] * vs + vz;
  }
}

// ----------------------------------------------------------------- cache --

struct Seq {
  std::vector<std::vector<uint8_t>> pages;   // per KV head: concatenated pages
  std::vector<std::vector<uint16_t>> wk, wv;  // per KV head: window tokens [W][D] bf16
  int64_t len = 0;
};

struct Layer {
  int kb, vb, key_mode, fmt, batch, hkv, D;
  std::vector<Seq> seqs;
  std::vector<float> kscale, vscale;  // fp8 format: per KV head
  double err[4] = {0, 0, 0, 0};       // sum (k - k_hat)^2, sum k^2, sum (v - v_hat)^2, sum v^2
  int64_t elements = 0;               // quantized elements of K (= of V)
};

}  // namespace

extern "C" {

// ---- scalar helpers exposed for the pins --------------------------------
uint16_t oracle_f32_to_bf16(float x) { return f32_to_bf16_rne(x); }
uint16_t oracle_f32_to_f16_rd(float x) { return f32_to_f16_directed(x, false); }
uint16_t oracle_f32_to_f16_ru(float x) { return f32_to_f16_directed(x, true); }
double oracle_f16_value(uint16_t h) { return f16_value(h); }

// Equivalent bitwidth of a layer map: mean over layers of (k + v)/2, a bf16
// layer counting as 16 + 16. Scales and zero points are not counted.
double oracle_equiv_bits(const uint8_t* kbits, const uint8_t* vbits, int n_layers) {
  double sum = 0;
  for (int l = 0; l < n_layers; ++l) sum += ((double)kbits[l] + (double)vbits[l]) / 2.0;
  return sum / n_layers;
}

// Bytes of one layer's K and V for `tokens` tokens per KV head: codes only
// (with_meta = 0, the idealised count of the worked example), or codes plus
// fp16 scale/zero (2 bytes each: D/32 key pairs -- one key pair in per-token key
// mode -- and one value pair per token).
int64_t oracle_layer_bytes(int kbits, int vbits, int key_mode, int fmt, int64_t tokens, int n_kv_heads,
                           int head_dim, int with_meta) {
  int64_t bits = tokens * n_kv_heads * (int64_t)head_dim * (kbits + vbits);
  int64_t bytes = bits / 8;
  if (with_meta && kbits != 16 && !fmt)
    bytes += tokens * n_kv_heads * ((key_mode ? 4 : (int64_t)head_dim * 4 / 32) + 4);
  return bytes;
}

void oracle_quantize(const float* x, int n, int bits, uint8_t* codes, uint16_t* scale_bits,
                     uint16_t* zero_bits) {
  quantize_set(x, n, bits, codes, scale_bits, zero_bits);
}

int64_t oracle_page_bytes(int kb, int vb, int D, int key_mode, int fmt) { return page_bytes(kb, vb, D, key_mode, fmt); }

uint8_t oracle_e4m3_encode(float x) { return e4m3_encode(x); }
double oracle_e4m3_value(uint8_t c) { return e4m3_value(c); }

// Pack/unpack one code block (vals [32][D]); is_value selects the V tiling.
void oracle_pack_block(uint8_t* blk, const uint16_t* vals, int D, int bits, int is_value) {
  std::memset(blk, 0, (size_t)code_block_bytes(bits, D));
  pack_block(blk, vals, D, bits, is_value != 0);
}
void oracle_unpack_block(const uint8_t* blk, uint16_t* vals, int D, int bits, int is_value) {
  unpack_block(blk, vals, D, bits, is_value != 0);
}

void oracle_build_page(uint8_t* page, const uint16_t* kbf, const uint16_t* vbf, int D, int kb, int vb,
                       int key_mode, int fmt, float ksc, float vsc) {
  build_page(page, kbf, vbf, D, kb, vb, key_mode, fmt, ksc, vsc);
}
void oracle_dequant_page(const uint8_t* page, int D, int kb, int vb, int key_mode, int fmt, float ksc, float vsc,
                         double* Kh, double* Vh) {
  dequant_page(page, D, kb, vb, key_mode, fmt, ksc, vsc, Kh, Vh);
}

// ---- one-layer cache simulator -------------------------------------------
void* oracle_layer_new(int kb, int vb, int key_mode, int fmt, int batch, int n_kv_heads, int head_dim) {
  Layer* L = new Layer{kb, vb, kb == 16 ? 0 : key_mode, kb == 16 ? 0 : fmt, batch, n_kv_heads, head_dim, {}, {}, {}};
  L->kscale.assign(n_kv_heads, 1.0f);
  L->vscale.assign(n_kv_heads, 1.0f);
  L->seqs.resize(batch);
  for (auto& s : L->seqs) {
    s.pages.resize(n_kv_heads);
    s.wk.resize(n_kv_heads);
    s.wv.resize(n_kv_heads);
  }
  return L;
}

void oracle_layer_free(void* p) { delete static_cast<Layer*>(p); }

// fp8 format: per-KV-head key and value scales (before the first append).
void oracle_layer_set_fp8_scales(void* p, const float* kscale, const float* vscale) {
  Layer* L = static_cast<Layer*>(p);
  for (int h = 0; h < L->hkv; ++h) {
    L->kscale[h] = kscale[h];
    L->vscale[h] = vscale[h];
  }
}

int64_t oracle_layer_len(void* p, int b) { return static_cast<Layer*>(p)->seqs[b].len; }

// Quantization error report: out = {sum (k - k_hat)^2, sum k^2, sum (v - v_hat)^2,
// sum v^2}; returns the number of quantized key (= value) elements.
int64_t oracle_layer_error(void* p, double* out) {
  Layer* L = static_cast<Layer*>(p);
  for (int i = 0; i < 4; ++i) out[i] = L->err[i];
  return L->elements;
}

// Append n_new[b] tokens to every sequence b < batch. K and V are packed
// [sum(n_new)][n_kv_heads][D] fp32 (rounded to bf16 on entry). Tokens enter the
// window one at a time; the window is quantized as one page the moment it
// holds 32 tokens.
void oracle_layer_append(void* p, const float* K, const float* V, const int32_t* n_new, int batch) {
  Layer* L = static_cast<Layer*>(p);
  const int D = L->D, H = L->hkv;
  const int64_t pb = page_bytes(L->kb, L->vb, D, L->key_mode, L->fmt);
  int64_t row = 0;
  for (int b = 0; b < batch; ++b) {
    Seq& s = L->seqs[b];
    for (int i = 0; i < n_new[b]; ++i, ++row) {
      for (int h = 0; h < H; ++h) {
        const float* kr = K + (row * H + h) * D;
        const float* vr = V + (row * H + h) * D;
        for (int d = 0; d < D; ++d) {
          s.wk[h].push_back(f32_to_bf16_rne(kr[d]));
          s.wv[h].push_back(f32_to_bf16_rne(vr[d]));
        }
        if ((int64_t)s.wk[h].size() == 32LL * D) {
          size_t off = s.pages[h].size();
          s.pages[h].resize(off + pb);
          build_page(s.pages[h].data() + off, s.wk[h].data(), s.wv[h].data(), D, L->kb, L->vb, L->key_mode, L->fmt,
                     L->kscale[h], L->vscale[h]);
          if (L->kb != 16) {
            // quantization error of this flush against its bf16 inputs
            std::vector<double> Kh(32 * D), Vh(32 * D);
            dequant_page(s.pages[h].data() + off, D, L->kb, L->vb, L->key_mode, L->fmt, L->kscale[h], L->vscale[h],
                         Kh.data(), Vh.data());
            for (int i = 0; i < 32 * D; ++i) {
              double k = bf16_to_f32(s.wk[h][i]), v = bf16_to_f32(s.wv[h][i]);
              L->err[0] += (k - Kh[i]) * (k - Kh[i]);
              L->err[1] += k * k;
              L->err[2] += (v - Vh[i]) * (v - Vh[i]);
              L->err[3] += v * v;
            }
            L->elements += 32LL * D;
          }
          s.wk[h].clear();
          s.wv[h].clear();
        }
      }
      s.len += 1;
    }
  }
}

// Export: for b < batch, for each KV head: full pages, then window keys
// [W][D] bf16, then window values [W][D] bf16 (W = len mod 32).
int64_t oracle_layer_export_bytes(void* p, int batch) {
  Layer* L = static_cast<Layer*>(p);
  int64_t n = 0;
  for (int b = 0; b < batch; ++b)
    for (int h = 0; h < L->hkv; ++h)
      n += (int64_t)L->seqs[b].pages[h].size() + 2 * 2 * (int64_t)L->seqs[b].wk[h].size();
  return n;
}

void oracle_layer_export(void* p, int batch, uint8_t* dst) {
  Layer* L = static_cast<Layer*>(p);
  for (int b = 0; b < batch; ++b)
    for (int h = 0; h < L->hkv; ++h) {
      const Seq& s = L->seqs[b];
      std::memcpy(dst, s.pages[h].data(), s.pages[h].size());
      dst += s.pages[h].size();
      std::memcpy(dst, s.wk[h].data(), 2 * s.wk[h].size());
      dst += 2 * s.wk[h].size();
      std::memcpy(dst, s.wv[h].data(), 2 * s.wv[h].size());
      dst += 2 * s.wv[h].size();
    }
}

// Dequantized keys/values of sequence b, KV head h: [len][D] doubles.
void oracle_layer_dequant(void* p, int b, int h, double* Kh, double* Vh) {
  Layer* L = static_cast<Layer*>(p);
  const int D = L->D;
  const Seq& s = L->seqs[b];
  const int64_t pb = page_bytes(L->kb, L->vb, D, L->key_mode, L->fmt);
  int64_t npages = (int64_t)s.pages[h].size() / pb;
  for (int64_t pg = 0; pg < npages; ++pg)
    dequant_page(s.pages[h].data() + pg * pb, D, L->kb, L->vb, L->key_mode, L->fmt, L->kscale[h], L->vscale[h],
                 Kh + pg * 32 * D, Vh + pg * 32 * D);
  int64_t base = npages * 32 * D;
  for (size_t i = 0; i < s.wk[h].size(); ++i) {
    Kh[base + i] = bf16_to_f32(s.wk[h][i]);
    Vh[base + i] = bf16_to_f32(s.wv[h][i]);
  }
}

}  // extern "C"

namespace {

// Decode attention of the G query heads of KV head h of sequence b (fp64).
void attend_one(void* p, const float* Q, int n_q_heads, int b, int h, double* out) {
  Layer* L = static_cast<Layer*>(p);
  const int D = L->D, H = L->hkv, G = n_q_heads / H;
  const double inv_sqrt_d = 1.0 / std::sqrt((double)D);
  const int64_t T = L->seqs[b].len;
  std::vector<double> Kh(T * D), Vh(T * D), sc(T);
  if (T > 0) oracle_layer_dequant(p, b, h, Kh.data(), Vh.data());
  for (int gq = 0; gq < G; ++gq) {
    int hq = h * G + gq;
    double* o = out + ((int64_t)b * n_q_heads + hq) * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (T == 0) continue;
    std::vector<double> q(D);
    for (int d = 0; d < D; ++d)
      q[d] = bf16_to_f32(f32_to_bf16_rne(Q[((int64_t)b * n_q_heads + hq) * D + d]));
    double m = -INFINITY;
    for (int64_t t = 0; t < T; ++t) {
      double acc = 0;
      for (int d = 0; d < D; ++d) acc += q[d] * Kh[t * D + d];
      sc[t] = acc * inv_sqrt_d;
      m = std::max(m, sc[t]);
    }
    double l = 0;
    for (int64_t t = 0; t < T; ++t) { sc[t] = std::exp(sc[t] - m); l += sc[t]; }
    for (int64_t t = 0; t < T; ++t) {
      double w = sc[t] / l;
      for (int d = 0; d < D; ++d) o[d] += w * Vh[t * D + d];
    }
  }
}

}  // namespace

extern "C" {

// Decode attention for every (b < batch, q head): Q [batch][Hq][D] fp32 holding
// bf16 values (rounded on entry), out [batch][Hq][D] fp64. Only the sequences
// listed in `seq_mask` (nonzero) are computed when seq_mask is not null.
void oracle_layer_attend(void* p, const float* Q, int n_q_heads, int batch, const uint8_t* seq_mask,
                         double* out) {
  Layer* L = static_cast<Layer*>(p);
  for (int b = 0; b < batch; ++b) {
    if (seq_mask && !seq_mask[b]) continue;
    for (int h = 0; h < L->hkv; ++h) attend_one(p, Q, n_q_heads, b, h, out);
  }
}

// The same attention with the (sequence, KV head) units shared out over
// n_threads host threads (each unit writes its own output rows, so the result
// is identical to oracle_layer_attend's). Used to time the oracle on every core.
void oracle_layer_attend_threads(void* p, const float* Q, int n_q_heads, int batch, const uint8_t* seq_mask,
                                 double* out, int n_threads) {
  Layer* L = static_cast<Layer*>(p);
  std::vector<std::pair<int, int>> units;
  for (int b = 0; b < batch; ++b)
    if (!seq_mask || seq_mask[b])
      for (int h = 0; h < L->hkv; ++h) units.emplace_back(b, h);
  std::atomic<size_t> next{0};
  auto worker = [&]() {
    for (size_t i = next++; i < units.size(); i = next++)
      attend_one(p, Q, n_q_heads, units[i].first, units[i].second, out);
  };
  const int n = std::max(1, std::min<int>(n_threads, (int)units.size()));
  std::vector<std::thread> pool;
  for (int t = 1; t < n; ++t) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
}

}  // extern "C"
