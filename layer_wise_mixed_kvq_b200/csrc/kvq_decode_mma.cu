// kvq_decode_mma.cu -- split-K decode attention over one layer's mixed-precision
// cache on the tensor cores (warp-level mma.sync m16n8k16, fp32 accumulate).
//
// KVTuner OpenReview rebuttal, "Baseline Implementation": decode runs
// FlashAttention-style kernels directly over the int8 / mixed-precision K and V
// cache; "New GQA efficiency results": grouped-query attention. Keys are
// dequantized per channel (x = code * s_c + z_c over each 32-token page) and
// values per token (x = code * s_t + z_t); "Computational cost": only the new
// token is quantized online, which the fused decode step does in this kernel.
//
// Work splits, 4 warps per CTA, each warp streaming pages through a private
// ring of shared-memory stages filled by bulk copies (cp.async.bulk, one copy
// per page, mbarrier completion) with its own online-softmax state:
//  * shared split (decode_mma_kernel): a persistent grid cuts all (sequence,
//    KV head) segments' units into balanced contiguous slices, one per CTA; the
//    CTA's warps take a segment part's units in turn, merge in shared memory,
//    and either write the output or leave a split record that the last CTA of
//    the segment merges. A segment's units are: overhead units (no work), its
//    tail unit (the bf16 window; in the fused step, the new token's append and
//    then the window or the page that token completed), then its pages.
//  * warp split (decode_warp_kernel, short sequences, G <= 4): each warp
//    attends whole segments alone and writes their outputs.
//
// Per page (32 tokens), token rows (G <= 4): MMA rows are tokens (QK) and value
// channels (PV); the 8 columns are (head c/2, part c%2), part 0 the high and
// part 1 the low f16 half of the operand (hi + lo carries the operand exactly).
//   QK : A = key codes, B = q'_c = q_c * s_c. q is a bf16 value scaled by a power
//        of two into (-1, 1), so it is exact in f16, and s_c is the page's f16
//        scale: hi = RN(q s) (HMUL2) and lo = q s - hi (HFMA2) are exact, i.e. the
//        product is formed without rounding. The z term sum_c q_c z_c is one MMA
//        per 16 channels (B = q on part-0 columns).
//   softmax: online max / sum in the log2 domain, raised lazily (p <= 2^8).
//   PV : A = value codes, B = p' = p * s_t * 2^E as (hi, lo) f16 pairs, moved from
//        the score layout to the B layout by 8x8 transposes (movmatrix); E is a
//        per-segment power of two that keeps p' in f16's normal range whatever
//        the value scales are; sum_t p_t z_t is added per head at the end.
// Head rows (G > 4) put (head, part) on the MMA rows and tokens on the columns.
// Codes enter the tensor core as f16 *subnormals*: masking a packed word with
// 0x000F000F (4-bit), 0x00030003 (2-bit) or byte-permuting with zero (8-bit)
// yields the f16 pair (c_a * 2^-24, c_b * 2^-24) exactly, so unpacking costs one
// logic op per two codes. Codes sitting higher in a word come out multiplied
// by a power of two; those factors are folded, exactly, into q, p', the score
// scale and the output scale (see the sigma/tau constants below).
// bf16 layers and the bf16 window use bf16 MMAs on the raw values.

#include <algorithm>
#include <type_traits>

#include <cuda_fp8.h>

#include "kvq_internal.cuh"
#include "kvq_quant.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kWaitLimit = 1u << 24;   // try_wait polls before a copy is declared lost
constexpr float kTwo24 = 16777216.0f;         // codes are c * 2^-24 inside the MMA
constexpr float kTau = 8.0f;                  // lazy rescale: p may grow to 2^kTau before a rescale
constexpr int kNoExp = -1000;                 // value exponent not chosen yet (no nonzero value scale seen)

// ------------------------------------------------------------ PTX helpers --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: false if the phase did not complete within kWaitLimit polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t it = 0; it < kWaitLimit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// L2 policy for data read exactly once (the streamed pages): evict first, so
// the stream does not push out the small reused data (query rows, windows,
// split records).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void bulk_load_once(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                               uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// Bulk prefetch into L2 (16-byte aligned address, size a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// f16x2 arithmetic, each half rounded to nearest (IEEE binary16).
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t hneg2(uint32_t a) { return a ^ 0x80008000u; }

// 8x8 transpose of 16-bit elements across the warp: lane l holds row l/4,
// columns 2(l%4), 2(l%4)+1 before and after.
__device__ __forceinline__ uint32_t movtrans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ uint32_t b2_bits(__nv_bfloat162 h) { return *reinterpret_cast<uint32_t*>(&h); }

// x = hi + lo with hi = f16(x) and lo = f16(x - hi); (x0, x1) -> low, high halves.
__device__ __forceinline__ void split_f16(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  __half2 h = __floats2half2_rn(x0, x1);
  float2 f = __half22float2(h);
  hi = h2_bits(h);
  lo = h2_bits(__floats2half2_rn(x0 - f.x, x1 - f.y));
}

__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  float2 f = __bfloat1622float2(h);
  hi = b2_bits(h);
  lo = b2_bits(__floats2bfloat162_rn(x0 - f.x, x1 - f.y));
}

// (hi, lo) of one value as one register: low half f16(x), high half f16(x - hi).
__device__ __forceinline__ uint32_t pack_hl_f16(float x) {
  const float h = __half2float(__float2half_rn(x));
  return h2_bits(__floats2half2_rn(h, x - h));
}

__device__ __forceinline__ uint32_t pack_hl_bf16(float x) {
  const float h = __bfloat162float(__float2bfloat16_rn(x));
  return b2_bits(__floats2bfloat162_rn(h, x - h));
}

// hi (part 0) or lo (part 1) halves of (x0, x1) as one register.
__device__ __forceinline__ uint32_t part_f16(float x0, float x1, float partf) {
  __half2 h = __floats2half2_rn(x0, x1);
  float2 f = __half22float2(h);
  return h2_bits(__floats2half2_rn(fmaf(-partf, f.x, x0), fmaf(-partf, f.y, x1)));
}

// 2^k as a float, -126 <= k <= 127.
__device__ __forceinline__ float exp2i(int k) { return __int_as_float((127 + k) << 23); }

// 2^x on the MUFU unit (flushes results below 2^-126 to zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------ configuration --
// PT: per-token key mode (32 key scales/zeros per page instead of D).
// F8: fp8 e4m3 elements (8/8 bits, no page metadata, per-KV-head scales).
template <int KB, int VB, int D, bool PT = false, bool F8 = false>
struct Cfg {
  static constexpr bool kBf16 = (KB == 16);
  static constexpr int KS = D / 16;                       // 16-channel tiles
  static constexpr int PB = (int)page_bytes_of(KB, VB, D, PT ? 1 : 0, F8 ? 1 : 0);
  // token rows: 3 CTAs per SM for small pages (3-4 stages per warp), 2 for larger ones; head rows
  // (64 accumulators per lane) always 2, so they get the registers they need without spilling
  static constexpr int MINB = 2;
  static constexpr int MINB_TOK = PB <= 5000 ? 3 : 2;
  // bytes of stages per warp: with 3 CTAs per SM, 3 x 4 warps x 14 KB; with 2, 2 x 4 x 20 KB, leaving
  // room for the rest of a CTA's shared memory inside its share of the SM
  static constexpr int RING_BUDGET = MINB_TOK == 3 ? 14336 : 20480;
  static constexpr int R = (RING_BUDGET / PB) < 2 ? 2 : ((RING_BUDGET / PB) > 4 ? 4 : (RING_BUDGET / PB));
  static constexpr int STAGE = (PB + 127) / 128 * 128;
  // Power-of-two factors of the subnormal unpack (see file comment).
  //   key n-tile parity 1 (tokens 8..15 of each 16) is sigmaK times parity 0;
  //   key channels 2t+8, 2t+9 of each tile carry tauK relative to 2t, 2t+1;
  //   value output channels with bit 3 set carry sigmaV; value tokens with bit 3
  //   set carry tauV.
  static constexpr float sigmaK = KB == 4 ? 16.f : (KB == 2 ? 4.f : 1.f);
  static constexpr float tauK = KB == 2 ? 16.f : 1.f;
  static constexpr float sigmaV = VB == 4 ? 16.f : (VB == 2 ? 4.f : 1.f);
  static constexpr float tauV = VB == 2 ? 16.f : 1.f;
  // shared memory layout
  static constexpr int RING = kWarps * R * STAGE;
  static constexpr int MBAR_OFF = RING;
  // ring + 2 query-row barriers, then each warp's stage part tags [kWarps][4] and the page counter
  static constexpr int MBAR_BYTES = ((kWarps * R + 2) * 8 + kWarps * 16 + 16 + 127) / 128 * 128;
  // per-warp scratch: value scales and zeros, per-token key scales and zeros
  // (4 x 32 floats), or a flush's quantizer parameters (2 D + 64 floats)
  static constexpr int WSCR_FLOATS = 2 * D + 64 > 128 ? 2 * D + 64 : 128;
  static constexpr int WSCR_OFF = MBAR_OFF + MBAR_BYTES;
  static constexpr int WSCR_STRIDE = (WSCR_FLOATS * 4 + 127) / 128 * 128;
  static constexpr int QZ_OFF = WSCR_OFF + kWarps * WSCR_STRIDE;
  static constexpr int QZ_BYTES = KS * 32 * 16;            // head rows: query operand table
  // 2 x [G][D] bf16 query rows (G <= 4 with token rows, <= 8 with head rows)
  static constexpr int qbuf_bytes(bool tok) { return 2 * (tok ? 4 : kMaxGqa) * D * 2; }
  static constexpr int qbuf_off(bool tok) { return tok ? QZ_OFF : QZ_OFF + QZ_BYTES; }
  static constexpr int merge_off(bool tok) { return qbuf_off(tok) + qbuf_bytes(tok); }
  // then: merge area [kWarps + 1][G][D] + m, l [kWarps + 1][8] floats (one slot per warp and
  // one for the window), unit starts [batch + 1] and lengths [batch] ints
  static int smem_bytes(bool tok, int G, int batch) {
    return merge_off(tok) + ((kWarps + 1) * G * D + 2 * (kWarps + 1) * kMaxGqa) * 4 + (2 * batch + 1) * 4;
  }
  static_assert(PB % 16 == 0, "bulk copies need 16-byte multiples");
};

// Running state of one warp. Head rows: lane (g, t) owns head g, o[n-tile] with
// rows g (hi) and g + 8 (lo). Token rows: lane (g, t) owns head t's scores and
// o[channel tile] (c0/c1: channel g, parts; c2/c3: channel g + 8).
template <int NT>
struct State {
  float o[NT][4];
  float m;             // reference max (log2 domain)
  float l;             // partial sum over this lane's tokens
  float vz;            // partial sum_t p_t z_t over this lane's tokens
  int E;               // integer pages: o is kept in units of 2^-E (p' = p * s * 2^E), kNoExp before
};
template <int D> using WarpState = State<D / 8>;
template <int D> using TokState = State<D / 16>;

template <int NT>
__device__ __forceinline__ void state_init(State<NT>& st) {
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) st.o[j][k] = 0.f;
  st.m = -INFINITY;
  st.l = 0.f;
  st.vz = 0.f;
  st.E = kNoExp;
}

// Value-operand exponent for one integer page whose value scales (lane = token)
// are vs: p' = p * s_t * 2^E stays below 2^15 (p <= 2^kTau) and, for the page's
// largest scale, above 2^6, so the (hi, lo) f16 pair keeps p' to ~22 bits even
// when every scale is far below f16's normal range. E changes (and o is rescaled
// exactly by the power of two) only when the page needs a smaller E or could
// use one larger by more than 8. Warp-uniform. Returns 2^E.
template <int NT>
__device__ __forceinline__ float value_exponent(State<NT>& st, float vs) {
  const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(vs));  // vs >= 0: bit order = value order
  if (mb != 0u) {
    const int e = (int)(mb >> 23) - 127;   // largest scale in [2^e, 2^(e+1)); fp16 scales: -24 <= e <= 15
    const int want = 6 - e;                // 2^8 * 2^(e+1) * 2^want = 2^15
    if (st.E == kNoExp) {
      st.E = want;
    } else if (want < st.E || want > st.E + 8) {
      const float f = exp2i(want - st.E);
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k) st.o[j][k] *= f;
      st.E = want;
    }
  }
  return exp2i(st.E == kNoExp ? 0 : st.E);
}

// ------------------------------------------------------ B fragments of codes --
// Words of one 16-channel tile row dt of a code block for this lane: tiles
// (dt, tt = 0) and (dt, tt = 1). N = 1 (2-bit), 2 (4-bit), 4 (8-bit), 8 (bf16).
template <int BITS>
struct TileWords {
  static constexpr int N = BITS == 2 ? 1 : (BITS == 4 ? 2 : (BITS == 8 ? 4 : 8));
};

template <int BITS>
__device__ __forceinline__ void load_tile_words(const uint8_t* blk, int lane, int dt,
                                                uint32_t (&w)[TileWords<BITS>::N]) {
  constexpr int N = TileWords<BITS>::N;
  const int base = dt * N;  // first lane word
  if constexpr (N >= 4) {
#pragma unroll
    for (int v = 0; v < N / 4; ++v) {
      uint4 q = *reinterpret_cast<const uint4*>(blk + ((base / 4 + v) * 32 + lane) * 16);
      w[4 * v + 0] = q.x;
      w[4 * v + 1] = q.y;
      w[4 * v + 2] = q.z;
      w[4 * v + 3] = q.w;
    }
  } else if constexpr (N == 2) {
    uint2 q = *reinterpret_cast<const uint2*>(blk + ((base >> 2) * 32 + lane) * 16 + (base & 3) * 4);
    w[0] = q.x;
    w[1] = q.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(blk + ((base >> 2) * 32 + lane) * 16 + (base & 3) * 4);
  }
}

// The same words through a 16-byte vector per lane shared by consecutive tile
// rows: 4-bit blocks hold 2 tile rows per vector, 2-bit blocks 4. Called with
// dt = 0, 1, ... in order (unrolled), it loads a vector only at a vector's first
// tile row, so a warp reads whole 512-byte rows (no bank conflicts) with half or
// a quarter of the loads.
template <int BITS>
__device__ __forceinline__ void tile_words(const uint8_t* blk, int lane, int dt, uint4& vec,
                                           uint32_t (&w)[TileWords<BITS>::N]) {
  constexpr int N = TileWords<BITS>::N;
  if constexpr (N >= 4) {
    load_tile_words<BITS>(blk, lane, dt, w);
  } else {
    const int word0 = dt * N;
    if (word0 % 4 == 0) vec = *reinterpret_cast<const uint4*>(blk + ((word0 / 4) * 32 + lane) * 16);
    const uint32_t c[4] = {vec.x, vec.y, vec.z, vec.w};
#pragma unroll
    for (int i = 0; i < N; ++i) w[i] = c[word0 % 4 + i];
  }
}

// B fragments of tile (dt, tt): b[0..1] for the even n-tile (key tokens
// 16tt..16tt+7, or value channels 16dt..16dt+7), b[2..3] for the odd one.
template <int BITS>
__device__ __forceinline__ void tile_frags(const uint32_t (&w)[TileWords<BITS>::N], int tt, uint32_t (&b)[4]) {
  if constexpr (BITS == 4) {
    uint32_t x = w[tt], y = x >> 8;
    b[0] = x & 0x000F000Fu;
    b[1] = y & 0x000F000Fu;
    b[2] = x & 0x00F000F0u;
    b[3] = y & 0x00F000F0u;
  } else if constexpr (BITS == 2) {
    uint32_t x = tt ? (w[0] >> 8) : w[0];
    b[0] = x & 0x00030003u;
    b[1] = x & 0x00300030u;
    b[2] = x & 0x000C000Cu;
    b[3] = x & 0x00C000C0u;
  } else if constexpr (BITS == 8) {
    uint32_t x = w[2 * tt], y = w[2 * tt + 1];
    b[0] = __byte_perm(x, 0u, 0x4140);
    b[1] = __byte_perm(y, 0u, 0x4140);
    b[2] = __byte_perm(x, 0u, 0x4342);
    b[3] = __byte_perm(y, 0u, 0x4342);
  } else {  // bf16 values: the stored words are the fragments
    b[0] = w[4 * tt + 0];
    b[1] = w[4 * tt + 2];
    b[2] = w[4 * tt + 1];
    b[3] = w[4 * tt + 3];
  }
}

// A fragment of tile (dt, tt) from this lane's words (rows: tokens for keys,
// channels for values; columns: channels for keys, tokens for values).
template <int BITS>
__device__ __forceinline__ void tile_afrag(const uint32_t (&w)[TileWords<BITS>::N], int tt, uint32_t (&a)[4]) {
  if constexpr (BITS == 4) {
    uint32_t x = w[tt], y = x >> 8;
    a[0] = x & 0x000F000Fu;   // rows g,   cols 2t..     x1
    a[1] = x & 0x00F000F0u;   // rows g+8, cols 2t..     x16
    a[2] = y & 0x000F000Fu;   // rows g,   cols 2t+8..   x1
    a[3] = y & 0x00F000F0u;   // rows g+8, cols 2t+8..   x16
  } else if constexpr (BITS == 2) {
    uint32_t x = tt ? (w[0] >> 8) : w[0];
    a[0] = x & 0x00030003u;   // x1
    a[1] = x & 0x000C000Cu;   // x4
    a[2] = x & 0x00300030u;   // x16
    a[3] = x & 0x00C000C0u;   // x64
  } else if constexpr (BITS == 8) {
    uint32_t x = w[2 * tt], y = w[2 * tt + 1];
    a[0] = __byte_perm(x, 0u, 0x4140);
    a[1] = __byte_perm(x, 0u, 0x4342);
    a[2] = __byte_perm(y, 0u, 0x4140);
    a[3] = __byte_perm(y, 0u, 0x4342);
  } else {
    a[0] = w[4 * tt + 0];
    a[1] = w[4 * tt + 1];
    a[2] = w[4 * tt + 2];
    a[3] = w[4 * tt + 3];
  }
}

// Two e4m3 bytes of x (bytes 0, 1 for kSelLo; 2, 3 for kSelHi) -> f16x2 whose
// values are the e4m3 values times 2^-8, exactly. prmt puts each byte in the
// low half of a 16-bit lane with its sign replicated into the high byte; a
// shift by 7 moves the seven magnitude bits (4 exponent, 3 mantissa) to f16
// bits 7..13 and a sign copy to bit 15; the mask keeps those. The f16 exponent
// bias (15) exceeds e4m3's (7) by 8, which gives the 2^-8 for normal and
// subnormal codes alike (a subnormal e4m3 m*2^-9 becomes the f16 subnormal
// m*2^7*2^-24).
constexpr uint32_t kSelLo = 0x9180u, kSelHi = 0xB3A2u;
constexpr float kF8Unit = 256.0f;  // true value = f16 value * 2^8

__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t x, uint32_t sel) {
  uint32_t t;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(t) : "r"(x), "r"(sel));
  return (t << 7) & 0xBF80BF80u;
}

// fp8 counterparts of the 8-bit A and B fragments: the same bytes, as f16
// values (times 2^-8) instead of integer codes.
__device__ __forceinline__ void tile_afrag_f8(const uint32_t (&w)[TileWords<8>::N], int tt, uint32_t (&a)[4]) {
  const uint32_t x = w[2 * tt], y = w[2 * tt + 1];
  a[0] = e4m3x2_f16x2(x, kSelLo);
  a[1] = e4m3x2_f16x2(x, kSelHi);
  a[2] = e4m3x2_f16x2(y, kSelLo);
  a[3] = e4m3x2_f16x2(y, kSelHi);
}

__device__ __forceinline__ void tile_frags_f8(const uint32_t (&w)[TileWords<8>::N], int tt, uint32_t (&b)[4]) {
  const uint32_t x = w[2 * tt], y = w[2 * tt + 1];
  b[0] = e4m3x2_f16x2(x, kSelLo);
  b[1] = e4m3x2_f16x2(y, kSelLo);
  b[2] = e4m3x2_f16x2(x, kSelHi);
  b[3] = e4m3x2_f16x2(y, kSelHi);
}

// ---------------------------------------------------------- online softmax --
// Head rows: scores sc[8] (log2 domain; tokens 8j + 2t + {0,1} for n-tile
// j = i/2; masked tokens are -inf). The reference max is raised only when a
// score exceeds it by more than kTau, so p <= 2^kTau. Returns p in sc.
template <int D>
__device__ __forceinline__ void softmax_update(WarpState<D>& st, float (&sc)[8]) {
  float mx = fmaxf(fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3])), fmaxf(fmaxf(sc[4], sc[5]), fmaxf(sc[6], sc[7])));
  // the row maximum is needed only when some score passes the reference by more
  // than kTau: one vote decides (a row's lanes share st.m, so the result is the
  // same as reducing every time)
  if (!__any_sync(0xffffffffu, mx > st.m + kTau)) mx = st.m;
  else {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  }
  if (mx > st.m + kTau) {
    const float alpha = ex2(st.m - mx);  // 0 when st.m = -inf
#pragma unroll
    for (int j = 0; j < D / 8; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) st.o[j][k] *= alpha;
    st.l *= alpha;
    st.vz *= alpha;
    st.m = mx;
  }
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float pv = ex2(sc[i] - st.m);  // ex2(-inf) = 0
    sc[i] = pv;
    sum += pv;
  }
  st.l += sum;
}

// Token rows: scores sc[4] of head t for tokens g + 8i.
template <int D>
__device__ __forceinline__ void tok_softmax_update(TokState<D>& st, float (&sc)[4]) {
  float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
  // the head's maximum over the page is needed only when some score passes the
  // reference by more than kTau: one vote decides (a head's lanes share st.m)
  if (!__any_sync(0xffffffffu, mx > st.m + kTau)) mx = st.m;
  else {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
  }
  if (mx > st.m + kTau) {
    const float alpha = ex2(st.m - mx);
#pragma unroll
    for (int j = 0; j < D / 16; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) st.o[j][k] *= alpha;
    st.l *= alpha;
    st.vz *= alpha;
    st.m = mx;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    sc[i] = ex2(sc[i] - st.m);
    st.l += sc[i];
  }
}

// ----------------------------------------------------------- query operands --
// Power of two k with max |q| * 2^-k < 1 over the warp's query values (bits:
// this lane's largest |q| as float bits); q * 2^-k then fits f16 exactly and
// q * 2^-k * s (s <= 65504) cannot overflow it.
__device__ __forceinline__ int query_shift(float amax) {
  const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
  if (mb == 0u) return 0;
  const int k = (int)(mb >> 23) - 126;
  return k < -100 ? -100 : (k > 100 ? 100 : k);
}

// Token rows: query operands of one segment for lane (g, t), column g = (head
// g/2, part g%2).
template <int D>
struct TokOps {
  // integer per-channel keys: q * 2^-k as f16 pairs of head g/2, channels
  // 16dt + 2t (+1) and 16dt + 2t + 8 (+9), the second pair / tauK;
  // integer per-token keys: the QK B fragments (that q on part-0 columns, 0 on
  // part 1); fp8: the QK B fragments (q * key scale * log2(e)/sqrt(D), parts)
  uint32_t q2[D / 8];
  uint32_t qz[D / 8];   // integer per-channel keys: z-term B fragments (q * 2^-k on part-0 columns)
  uint32_t npart;       // f16x2 0 (part 0) or -1 (part 1)
  float fs0, fs1;       // QK accumulator -> score (log2 units) for n-tiles of parity 0 / 1
  float lsc;            // log2(e)/sqrt(D) * 2^k
  float qsum;           // per-token keys: sum_c q_c * 2^-k of the head this lane scores
};

template <int KB, int D, bool PT, bool F8>
__device__ __forceinline__ void prep_tok_ops(TokOps<D>& ops, const __nv_bfloat16* qrow, bool qvalid, int lane,
                                             float L, float ksc) {
  using C = Cfg<KB, 4, D>;
  constexpr int KS = D / 16;
  const int g = lane >> 2, t = lane & 3;
  const bool part0 = (g & 1) == 0;
  float2 lo[KS], hi[KS];
  float amax = 0.f;
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    uint32_t a = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t);
    uint32_t b = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t + 8);
    if (!qvalid) a = b = 0u;
    lo[dt] = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&a));
    hi[dt] = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&b));
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(lo[dt].x), fabsf(lo[dt].y)), fmaxf(fabsf(hi[dt].x), fabsf(hi[dt].y))));
  }
  if constexpr (F8) {
    const float f = L * ksc, partf = part0 ? 0.f : 1.f;
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      ops.q2[2 * dt] = part_f16(lo[dt].x * f, lo[dt].y * f, partf);
      ops.q2[2 * dt + 1] = part_f16(hi[dt].x * f, hi[dt].y * f, partf);
    }
    ops.fs0 = ops.fs1 = kF8Unit;
    return;
  } else {
    const int k = query_shift(amax);
    const float down = exp2i(-k), lp = L * exp2i(k);
    const float fold = down / C::tauK;
    float qs = 0.f;
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      const uint32_t ql = h2_bits(__floats2half2_rn(lo[dt].x * down, lo[dt].y * down));
      const uint32_t qh = h2_bits(__floats2half2_rn(hi[dt].x * down, hi[dt].y * down));
      const uint32_t qf = C::tauK != 1.f ? h2_bits(__floats2half2_rn(hi[dt].x * fold, hi[dt].y * fold)) : qh;
      qs += (lo[dt].x + lo[dt].y) + (hi[dt].x + hi[dt].y);
      if constexpr (PT) {
        ops.q2[2 * dt] = part0 ? ql : 0u;
        ops.q2[2 * dt + 1] = part0 ? qf : 0u;
      } else {
        ops.q2[2 * dt] = ql;
        ops.q2[2 * dt + 1] = qf;
        ops.qz[2 * dt] = part0 ? ql : 0u;
        ops.qz[2 * dt + 1] = part0 ? qh : 0u;
      }
    }
    ops.npart = part0 ? 0u : 0xBC00BC00u;
    ops.lsc = lp;
    ops.fs0 = kTwo24 * lp;
    ops.fs1 = kTwo24 / C::sigmaK * lp;
    if constexpr (PT) {
      // head g/2's sum over its D channels (the quad holds them), then head t's
      qs += __shfl_xor_sync(0xffffffffu, qs, 1);
      qs += __shfl_xor_sync(0xffffffffu, qs, 2);
      ops.qsum = __shfl_sync(0xffffffffu, qs, 8 * t) * down;
    }
  }
}

// Raw bf16 pairs of q for the bf16 pages and the window (token rows: q on
// part-0 columns, 0 on part 1; head rows: row g).
template <int D>
__device__ __forceinline__ void load_qb(const __nv_bfloat16* qrow, bool keep, int t, uint32_t (&qb)[D / 8]) {
#pragma unroll
  for (int dt = 0; dt < D / 16; ++dt) {
    qb[2 * dt] = keep ? *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t) : 0u;
    qb[2 * dt + 1] = keep ? *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t + 8) : 0u;
  }
}

// ------------------------------------------------------- token-row pages --
// p' of this lane (head t, tokens g + 8i) -> the PV B fragments. r[i] packs
// (hi, lo) of token g + 8i: block i of the [token][(head, part)] matrix in the
// C-fragment layout; an 8x8 transpose turns blocks 2ks, 2ks+1 into the B
// fragment of k-step ks (tokens 16ks + 2t, +1 and 16ks + 8 + 2t, +1; column g).
template <bool BF16>
__device__ __forceinline__ void tok_pv_frags(const float (&pv)[4], uint32_t (&b)[2][2]) {
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) r[i] = BF16 ? pack_hl_bf16(pv[i]) : pack_hl_f16(pv[i]);
  b[0][0] = movtrans(r[0]);
  b[0][1] = movtrans(r[1]);
  b[1][0] = movtrans(r[2]);
  b[1][1] = movtrans(r[3]);
}

// PV of one integer / fp8 / bf16 value block with the B fragments above.
template <int VB, int D, bool F8>
__device__ __forceinline__ void tok_pv(const uint8_t* vblk, TokState<D>& st, const uint32_t (&b)[2][2], int lane) {
  uint4 vec;
#pragma unroll
  for (int dt = 0; dt < D / 16; ++dt) {
    uint32_t w[TileWords<VB>::N];
    tile_words<VB>(vblk, lane, dt, vec, w);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t a[4];
      if constexpr (F8) tile_afrag_f8(w, ks, a);
      else tile_afrag<VB>(w, ks, a);
      if constexpr (VB == 16) mma_bf16(st.o[dt], a[0], a[1], a[2], a[3], b[ks][0], b[ks][1]);
      else mma_f16(st.o[dt], a[0], a[1], a[2], a[3], b[ks][0], b[ks][1]);
    }
  }
}

// Value scales (x 2^E, tauV folded) and zeros of an integer page into the warp's tables.
template <int VB, int NT>
__device__ __forceinline__ void value_tables(const __half* vscale, const __half* vzero, State<NT>& st, float* svf,
                                             float* zvf, int lane) {
  constexpr float tauV = VB == 2 ? 16.f : 1.f;
  const float vs = __half2float(vscale[lane]);
  const float f = value_exponent(st, vs);
  svf[lane] = vs * ((tauV != 1.f && (lane & 8)) ? f * (1.f / tauV) : f);
  zvf[lane] = __half2float(vzero[lane]);
}

// p' = p * s_t * 2^E and the value zero term, then PV.
template <int VB, int D>
__device__ __forceinline__ void tok_int_pv(const uint8_t* vblk, TokState<D>& st, float (&sc)[4], const float* svf,
                                           const float* zvf, int lane) {
  const int g = lane >> 2;
  float pv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    pv[i] = sc[i] * svf[g + 8 * i];
    st.vz = fmaf(sc[i], zvf[g + 8 * i], st.vz);
  }
  uint32_t b[2][2];
  tok_pv_frags<false>(pv, b);
  tok_pv<VB, D, false>(vblk, st, b, lane);
}

// Integer page, per-channel keys.
template <int KB, int VB, int D>
__device__ __forceinline__ void attend_qpage_tok(const uint8_t* page, TokState<D>& st, const TokOps<D>& ops,
                                                 float* wscr, int lane) {
  using C = Cfg<KB, VB, D>;
  const int t = lane & 3;
  const uint8_t* vblk = page + code_block_bytes(KB, D);
  const __half* kscale = reinterpret_cast<const __half*>(vblk + code_block_bytes(VB, D));
  const __half* kzero = kscale + D;
  const __half* vscale = kzero + D;
  const __half* vzero = vscale + kPageTokens;
  float* svf = wscr;
  float* zvf = wscr + kPageTokens;
  value_tables<VB>(vscale, vzero, st, svf, zvf, lane);
  __syncwarp();

  // QK: two token m-tiles, B = exact (hi, lo) of q * s_c; z term: A = z rows, B = q
  float s2[2][4], cz[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int k = 0; k < 4; ++k) s2[mt][k] = 0.f;
  const uint2* srow = reinterpret_cast<const uint2*>(kscale + t * (D / 4));   // channels 2t, 2t+1, 2t+8, 2t+9 per tile
  const uint2* zrow = reinterpret_cast<const uint2*>(kzero + t * (D / 4));
  uint4 vec;
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<KB>::N];
    tile_words<KB>(page, lane, dt, vec, w);
    const uint2 s = srow[dt];
    const uint32_t h0 = hmul2(ops.q2[2 * dt], s.x), h1 = hmul2(ops.q2[2 * dt + 1], s.y);
    const uint32_t b0 = hfma2(ops.q2[2 * dt], s.x, hmul2(h0, ops.npart));
    const uint32_t b1 = hfma2(ops.q2[2 * dt + 1], s.y, hmul2(h1, ops.npart));
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      uint32_t a[4];
      tile_afrag<KB>(w, mt, a);
      mma_f16(s2[mt], a[0], a[1], a[2], a[3], b0, b1);
    }
    const uint2 z = zrow[dt];
    mma_f16(cz, z.x, z.x, z.y, z.y, ops.qz[2 * dt], ops.qz[2 * dt + 1]);
  }
  const float czv = (cz[0] + cz[1]) * ops.lsc;  // head t: sum_c q_c z_c
  float sc[4];
  sc[0] = fmaf(s2[0][0] + s2[0][1], ops.fs0, czv);
  sc[1] = fmaf(s2[0][2] + s2[0][3], ops.fs1, czv);
  sc[2] = fmaf(s2[1][0] + s2[1][1], ops.fs0, czv);
  sc[3] = fmaf(s2[1][2] + s2[1][3], ops.fs1, czv);
  tok_softmax_update<D>(st, sc);
  tok_int_pv<VB, D>(vblk, st, sc, svf, zvf, lane);
}

// Integer page, per-token keys: B = the segment's q (fixed); score of token
// g + 8i for head t = (s_tok * acc + z_tok * sum_c q_c) * log2(e)/sqrt(D) * 2^k.
template <int KB, int VB, int D>
__device__ __forceinline__ void attend_qpage_tok_pt(const uint8_t* page, TokState<D>& st, const TokOps<D>& ops,
                                                    float* wscr, int lane) {
  using C = Cfg<KB, VB, D, true>;
  const int g = lane >> 2;
  const uint8_t* vblk = page + code_block_bytes(KB, D);
  const __half* kscale = reinterpret_cast<const __half*>(vblk + code_block_bytes(VB, D));
  const __half* kzero = kscale + kPageTokens;
  const __half* vscale = kzero + kPageTokens;
  const __half* vzero = vscale + kPageTokens;
  float* svf = wscr;
  float* zvf = wscr + kPageTokens;
  float* kst = wscr + 2 * kPageTokens;
  float* kzt = wscr + 3 * kPageTokens;
  kst[lane] = __half2float(kscale[lane]) * ((lane & 8) ? ops.fs1 : ops.fs0);
  kzt[lane] = __half2float(kzero[lane]) * ops.lsc;
  value_tables<VB>(vscale, vzero, st, svf, zvf, lane);
  __syncwarp();

  float s2[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int k = 0; k < 4; ++k) s2[mt][k] = 0.f;
  uint4 vec;
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<KB>::N];
    tile_words<KB>(page, lane, dt, vec, w);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      uint32_t a[4];
      tile_afrag<KB>(w, mt, a);
      mma_f16(s2[mt], a[0], a[1], a[2], a[3], ops.q2[2 * dt], ops.q2[2 * dt + 1]);
    }
  }
  float sc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int tok = g + 8 * i;
    const float acc = s2[i >> 1][2 * (i & 1)] + s2[i >> 1][2 * (i & 1) + 1];
    sc[i] = fmaf(acc, kst[tok], kzt[tok] * ops.qsum);
  }
  tok_softmax_update<D>(st, sc);
  tok_int_pv<VB, D>(vblk, st, sc, svf, zvf, lane);
}

// fp8 page: A = e4m3 keys/values as f16, B = the segment's q' parts (key scale
// folded in) or p parts.
template <int D>
__device__ __forceinline__ void attend_f8page_tok(const uint8_t* page, TokState<D>& st, const TokOps<D>& ops,
                                                  int lane) {
  constexpr int KS = D / 16;
  float s2[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int k = 0; k < 4; ++k) s2[mt][k] = 0.f;
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    uint32_t w[TileWords<8>::N];
    load_tile_words<8>(page, lane, dt, w);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      uint32_t a[4];
      tile_afrag_f8(w, mt, a);
      mma_f16(s2[mt], a[0], a[1], a[2], a[3], ops.q2[2 * dt], ops.q2[2 * dt + 1]);
    }
  }
  float sc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) sc[i] = (s2[i >> 1][2 * (i & 1)] + s2[i >> 1][2 * (i & 1) + 1]) * kF8Unit;
  tok_softmax_update<D>(st, sc);
  uint32_t b[2][2];
  tok_pv_frags<false>(sc, b);
  tok_pv<8, D, true>(page + code_block_bytes(8, D), st, b, lane);
}

template <int D>
__device__ __forceinline__ void attend_bpage_tok(const uint8_t* page, TokState<D>& st, const uint32_t (&qbp)[D / 8],
                                                 float scale_log2, int lane) {
  constexpr int KS = D / 16;
  float s2[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int k = 0; k < 4; ++k) s2[mt][k] = 0.f;
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    uint32_t w[TileWords<16>::N];
    load_tile_words<16>(page, lane, dt, w);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      uint32_t a[4];
      tile_afrag<16>(w, mt, a);
      mma_bf16(s2[mt], a[0], a[1], a[2], a[3], qbp[2 * dt], qbp[2 * dt + 1]);
    }
  }
  float sc[4] = {(s2[0][0] + s2[0][1]) * scale_log2, (s2[0][2] + s2[0][3]) * scale_log2,
                 (s2[1][0] + s2[1][1]) * scale_log2, (s2[1][2] + s2[1][3]) * scale_log2};
  tok_softmax_update<D>(st, sc);
  uint32_t b[2][2];
  tok_pv_frags<true>(sc, b);
  tok_pv<16, D, false>(page + code_block_bytes(16, D), st, b, lane);
}

// bf16 window (natural [32][D] rows in global memory), W < 32 valid tokens.
template <int D>
__device__ __forceinline__ void attend_window_tok(const __nv_bfloat16* win, int W, TokState<D>& st,
                                                  const uint32_t (&qbp)[D / 8], float scale_log2, int lane) {
  constexpr int KS = D / 16;
  const int g = lane >> 2, t = lane & 3;
  const uint16_t* kw = reinterpret_cast<const uint16_t*>(win);
  const uint16_t* vw = kw + kPageTokens * D;
  auto kpair = [&](int tok, int dim) -> uint32_t {
    return tok < W ? *reinterpret_cast<const uint32_t*>(kw + tok * D + dim) : 0u;
  };
  auto vpair = [&](int tok, int dim) -> uint32_t {
    const uint32_t lo = tok < W ? vw[tok * D + dim] : 0u;
    const uint32_t hi = tok + 1 < W ? vw[(tok + 1) * D + dim] : 0u;
    return lo | (hi << 16);
  };
  float s2[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int k = 0; k < 4; ++k) s2[mt][k] = 0.f;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    if (16 * mt >= W) continue;  // warp-uniform
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      const int r0 = 16 * mt + g, c0 = 16 * dt + 2 * t;
      mma_bf16(s2[mt], kpair(r0, c0), kpair(r0 + 8, c0), kpair(r0, c0 + 8), kpair(r0 + 8, c0 + 8), qbp[2 * dt],
               qbp[2 * dt + 1]);
    }
  }
  float sc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float v = (i & 1) ? (s2[i >> 1][2] + s2[i >> 1][3]) : (s2[i >> 1][0] + s2[i >> 1][1]);
    sc[i] = (g + 8 * i) < W ? v * scale_log2 : -INFINITY;
  }
  tok_softmax_update<D>(st, sc);
  uint32_t b[2][2];
  tok_pv_frags<true>(sc, b);
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    if (16 * ks >= W) continue;  // warp-uniform
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      const int tk = 16 * ks + 2 * t, ch = 16 * dt + g;
      mma_bf16(st.o[dt], vpair(tk, ch), vpair(tk, ch + 8), vpair(tk + 8, ch), vpair(tk + 8, ch + 8), b[ks][0],
               b[ks][1]);
    }
  }
}

// -------------------------------------------------------- head-row pages --
// Query operand table of a segment in shared memory, built by one warp: entry
// (dt, lane) for head g, channels 16dt + 2t (+1) and + 8 (+9):
//   integer per-channel keys: {q01, q89 / tauK, q01, q89} (q * 2^-k as f16 pairs;
//     the first two are the QK A operand, the last two the z-term A operand);
//   integer per-token keys: {q01, q89 / tauK, -, -};
//   fp8: {hi01, lo01, hi89, lo89} of q * key scale * log2(e)/sqrt(D).
struct HeadOps {
  float fs0, fs1, lsc, qsum;
};

template <int KB, int D, bool PT, bool F8>
__device__ __forceinline__ void prep_head_ops(HeadOps& ops, uint32_t* qtab, bool write_tab, const __nv_bfloat16* qrow,
                                              bool qvalid, int lane, float L, float ksc) {
  using C = Cfg<KB, 4, D>;
  constexpr int KS = D / 16;
  const int t = lane & 3;
  float2 lo[KS], hi[KS];
  float amax = 0.f;
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    uint32_t a = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t);
    uint32_t b = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t + 8);
    if (!qvalid) a = b = 0u;
    lo[dt] = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&a));
    hi[dt] = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&b));
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(lo[dt].x), fabsf(lo[dt].y)), fmaxf(fabsf(hi[dt].x), fabsf(hi[dt].y))));
  }
  if constexpr (F8) {
    const float f = L * ksc;
    if (write_tab) {
#pragma unroll
      for (int dt = 0; dt < KS; ++dt) {
        uint4 q4;
        split_f16(lo[dt].x * f, lo[dt].y * f, q4.x, q4.y);
        split_f16(hi[dt].x * f, hi[dt].y * f, q4.z, q4.w);
        *reinterpret_cast<uint4*>(qtab + (dt * 32 + lane) * 4) = q4;
      }
    }
    ops.fs0 = ops.fs1 = kF8Unit;
  } else {
    const int k = query_shift(amax);
    const float down = exp2i(-k), lp = L * exp2i(k);
    const float fold = down / C::tauK;
    float qs = 0.f;
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      qs += (lo[dt].x + lo[dt].y) + (hi[dt].x + hi[dt].y);
      if (write_tab) {
        uint4 q4;
        q4.x = h2_bits(__floats2half2_rn(lo[dt].x * down, lo[dt].y * down));
        q4.w = h2_bits(__floats2half2_rn(hi[dt].x * down, hi[dt].y * down));
        q4.y = C::tauK != 1.f ? h2_bits(__floats2half2_rn(hi[dt].x * fold, hi[dt].y * fold)) : q4.w;
        q4.z = q4.x;
        *reinterpret_cast<uint4*>(qtab + (dt * 32 + lane) * 4) = q4;
      }
    }
    ops.lsc = lp;
    ops.fs0 = kTwo24 * lp;
    ops.fs1 = kTwo24 / C::sigmaK * lp;
    qs += __shfl_xor_sync(0xffffffffu, qs, 1);
    qs += __shfl_xor_sync(0xffffffffu, qs, 2);
    ops.qsum = qs * down;  // head g
  }
}

// PV of head rows: A = p' (hi/lo) per 16-token k-step, B = value codes.
template <int VB, int D, bool F8>
__device__ __forceinline__ void head_pv(const uint8_t* vblk, WarpState<D>& st, const uint32_t (&pa)[2][4], int lane) {
  uint4 vec;
#pragma unroll
  for (int dt = 0; dt < D / 16; ++dt) {
    uint32_t w[TileWords<VB>::N];
    tile_words<VB>(vblk, lane, dt, vec, w);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t b[4];
      if constexpr (F8) tile_frags_f8(w, ks, b);
      else tile_frags<VB>(w, ks, b);
      if constexpr (VB == 16) {
        mma_bf16(st.o[2 * dt], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[0], b[1]);
        mma_bf16(st.o[2 * dt + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[2], b[3]);
      } else {
        mma_f16(st.o[2 * dt], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[0], b[1]);
        mma_f16(st.o[2 * dt + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[2], b[3]);
      }
    }
  }
}

// p' = p * s_t * 2^E (hi/lo) and the value zero term, then PV.
template <int VB, int D>
__device__ __forceinline__ void head_int_pv(const uint8_t* vblk, WarpState<D>& st, const float (&sc)[8],
                                            const float* svf, const float* zvf, int lane) {
  const int t = lane & 3;
  uint32_t pa[2][4];
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    const int t0 = 16 * ks + 2 * t, t1 = t0 + 8;
    const float2 s0 = *reinterpret_cast<const float2*>(svf + t0);
    const float2 s1 = *reinterpret_cast<const float2*>(svf + t1);
    const float2 z0 = *reinterpret_cast<const float2*>(zvf + t0);
    const float2 z1 = *reinterpret_cast<const float2*>(zvf + t1);
    const float p0 = sc[4 * ks + 0], p1 = sc[4 * ks + 1], p2 = sc[4 * ks + 2], p3 = sc[4 * ks + 3];
    split_f16(p0 * s0.x, p1 * s0.y, pa[ks][0], pa[ks][1]);
    split_f16(p2 * s1.x, p3 * s1.y, pa[ks][2], pa[ks][3]);
    st.vz = fmaf(p0, z0.x, fmaf(p1, z0.y, fmaf(p2, z1.x, fmaf(p3, z1.y, st.vz))));
  }
  head_pv<VB, D, false>(vblk, st, pa, lane);
}

// Integer page, per-channel keys: A = exact (hi, lo) of q * s_c, B = key codes.
template <int KB, int VB, int D>
__device__ __forceinline__ void attend_qpage(const uint8_t* page, WarpState<D>& st, const uint32_t* qtab,
                                             const HeadOps& ops, float* wscr, int lane) {
  using C = Cfg<KB, VB, D>;
  const int t = lane & 3;
  const uint8_t* vblk = page + code_block_bytes(KB, D);
  const __half* kscale = reinterpret_cast<const __half*>(vblk + code_block_bytes(VB, D));
  const __half* kzero = kscale + D;
  const __half* vscale = kzero + D;
  const __half* vzero = vscale + kPageTokens;
  float* svf = wscr;
  float* zvf = wscr + kPageTokens;
  value_tables<VB>(vscale, vzero, st, svf, zvf, lane);
  __syncwarp();

  float s4[4][4], cz[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) s4[j][k] = 0.f;
  const uint2* srow = reinterpret_cast<const uint2*>(kscale + t * (D / 4));
  const uint2* zrow = reinterpret_cast<const uint2*>(kzero + t * (D / 4));
  uint4 vec;
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<KB>::N];
    tile_words<KB>(page, lane, dt, vec, w);
    const uint4 q = *reinterpret_cast<const uint4*>(qtab + (dt * 32 + lane) * 4);
    const uint2 s = srow[dt];
    const uint32_t h01 = hmul2(q.x, s.x), h89 = hmul2(q.y, s.y);
    const uint32_t l01 = hfma2(q.x, s.x, hneg2(h01)), l89 = hfma2(q.y, s.y, hneg2(h89));
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      uint32_t b[4];
      tile_frags<KB>(w, tt, b);
      mma_f16(s4[2 * tt], h01, l01, h89, l89, b[0], b[1]);
      mma_f16(s4[2 * tt + 1], h01, l01, h89, l89, b[2], b[3]);
    }
    const uint2 z = zrow[dt];
    mma_f16(cz, q.z, 0u, q.w, 0u, z.x, z.y);
  }
  const float czv = (cz[0] + cz[2]) * ops.lsc;  // every column holds the same sum
  float sc[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float f = (j & 1) ? ops.fs1 : ops.fs0;
    sc[2 * j] = fmaf(s4[j][0] + s4[j][2], f, czv);
    sc[2 * j + 1] = fmaf(s4[j][1] + s4[j][3], f, czv);
  }
  softmax_update<D>(st, sc);
  head_int_pv<VB, D>(vblk, st, sc, svf, zvf, lane);
}

// Integer page, per-token keys: score of head g, token t = (s_t * sum_c q_c
// code_tc + z_t * sum_c q_c) * log2(e)/sqrt(D) * 2^k.
template <int KB, int VB, int D>
__device__ __forceinline__ void attend_qpage_pt(const uint8_t* page, WarpState<D>& st, const uint32_t* qtab,
                                                const HeadOps& ops, float* wscr, int lane) {
  using C = Cfg<KB, VB, D, true>;
  const int t = lane & 3;
  const uint8_t* vblk = page + code_block_bytes(KB, D);
  const __half* kscale = reinterpret_cast<const __half*>(vblk + code_block_bytes(VB, D));
  const __half* kzero = kscale + kPageTokens;
  const __half* vscale = kzero + kPageTokens;
  const __half* vzero = vscale + kPageTokens;
  float* svf = wscr;
  float* zvf = wscr + kPageTokens;
  float* kst = wscr + 2 * kPageTokens;
  float* kzt = wscr + 3 * kPageTokens;
  kst[lane] = __half2float(kscale[lane]) * ((lane & 8) ? ops.fs1 : ops.fs0);
  kzt[lane] = __half2float(kzero[lane]) * ops.lsc;
  value_tables<VB>(vscale, vzero, st, svf, zvf, lane);
  __syncwarp();

  float s4[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) s4[j][k] = 0.f;
  uint4 vec;
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<KB>::N];
    tile_words<KB>(page, lane, dt, vec, w);
    const uint2 q = *reinterpret_cast<const uint2*>(qtab + (dt * 32 + lane) * 4);
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      uint32_t b[4];
      tile_frags<KB>(w, tt, b);
      mma_f16(s4[2 * tt], q.x, 0u, q.y, 0u, b[0], b[1]);
      mma_f16(s4[2 * tt + 1], q.x, 0u, q.y, 0u, b[2], b[3]);
    }
  }
  float sc[8];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const int tok = 8 * j + 2 * t + jj;
      sc[2 * j + jj] = fmaf(s4[j][jj] + s4[j][jj + 2], kst[tok], kzt[tok] * ops.qsum);
    }
  softmax_update<D>(st, sc);
  head_int_pv<VB, D>(vblk, st, sc, svf, zvf, lane);
}

// fp8 page: A = the segment's q' hi/lo fragments with the KV head's key scale
// folded in, B = e4m3 keys as f16 (times 2^-8, undone on the scores); p hi/lo
// against e4m3 values (the value scale and 2^8 are applied once, at the end).
template <int D>
__device__ __forceinline__ void attend_f8page(const uint8_t* page, WarpState<D>& st, const uint32_t* qtab, int lane) {
  constexpr int KS = D / 16;
  float s4[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) s4[j][k] = 0.f;
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    uint32_t w[TileWords<8>::N];
    load_tile_words<8>(page, lane, dt, w);
    const uint4 a = *reinterpret_cast<const uint4*>(qtab + (dt * 32 + lane) * 4);
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      uint32_t b[4];
      tile_frags_f8(w, tt, b);
      mma_f16(s4[2 * tt], a.x, a.y, a.z, a.w, b[0], b[1]);
      mma_f16(s4[2 * tt + 1], a.x, a.y, a.z, a.w, b[2], b[3]);
    }
  }
  float sc[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    sc[2 * j] = (s4[j][0] + s4[j][2]) * kF8Unit;
    sc[2 * j + 1] = (s4[j][1] + s4[j][3]) * kF8Unit;
  }
  softmax_update<D>(st, sc);
  uint32_t pa[2][4];
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    split_f16(sc[4 * ks + 0], sc[4 * ks + 1], pa[ks][0], pa[ks][1]);
    split_f16(sc[4 * ks + 2], sc[4 * ks + 3], pa[ks][2], pa[ks][3]);
  }
  head_pv<8, D, true>(page + code_block_bytes(8, D), st, pa, lane);
}

// One full bf16 page: raw bf16 values, q unscaled (exact in bf16), p hi/lo.
template <int D>
__device__ __forceinline__ void attend_bpage(const uint8_t* page, WarpState<D>& st, const uint32_t (&qb)[D / 8],
                                             float scale_log2, int lane) {
  constexpr int KS = D / 16;
  float s4[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) s4[j][k] = 0.f;
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    uint32_t w[TileWords<16>::N];
    load_tile_words<16>(page, lane, dt, w);
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      uint32_t b[4];
      tile_frags<16>(w, tt, b);
      mma_bf16(s4[2 * tt], qb[2 * dt], 0u, qb[2 * dt + 1], 0u, b[0], b[1]);
      mma_bf16(s4[2 * tt + 1], qb[2 * dt], 0u, qb[2 * dt + 1], 0u, b[2], b[3]);
    }
  }
  float sc[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    sc[2 * j] = s4[j][0] * scale_log2;
    sc[2 * j + 1] = s4[j][1] * scale_log2;
  }
  softmax_update<D>(st, sc);
  uint32_t pa[2][4];
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    split_bf16(sc[4 * ks + 0], sc[4 * ks + 1], pa[ks][0], pa[ks][1]);
    split_bf16(sc[4 * ks + 2], sc[4 * ks + 3], pa[ks][2], pa[ks][3]);
  }
  head_pv<16, D, false>(page + code_block_bytes(16, D), st, pa, lane);
}

// The bf16 window (natural [32][D] rows in global memory), W < 32 valid tokens.
template <int D>
__device__ __forceinline__ void attend_window(const __nv_bfloat16* win, int W, WarpState<D>& st,
                                              const uint32_t (&qb)[D / 8], float scale_log2, int lane) {
  constexpr int KS = D / 16;
  const int g = lane >> 2, t = lane & 3;
  const uint16_t* kw = reinterpret_cast<const uint16_t*>(win);
  const uint16_t* vwp = kw + kPageTokens * D;
  float s4[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) s4[j][k] = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int tok = 8 * j + g;
    if (8 * j >= W) continue;  // warp-uniform
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      uint32_t b0 = 0, b1 = 0;
      if (tok < W) {
        b0 = *reinterpret_cast<const uint32_t*>(kw + tok * D + 16 * dt + 2 * t);
        b1 = *reinterpret_cast<const uint32_t*>(kw + tok * D + 16 * dt + 2 * t + 8);
      }
      mma_bf16(s4[j], qb[2 * dt], 0u, qb[2 * dt + 1], 0u, b0, b1);
    }
  }
  float sc[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int tok = 8 * j + 2 * t;
    sc[2 * j] = tok < W ? s4[j][0] * scale_log2 : -INFINITY;
    sc[2 * j + 1] = tok + 1 < W ? s4[j][1] * scale_log2 : -INFINITY;
  }
  softmax_update<D>(st, sc);
  uint32_t pa[2][4];
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    split_bf16(sc[4 * ks + 0], sc[4 * ks + 1], pa[ks][0], pa[ks][1]);
    split_bf16(sc[4 * ks + 2], sc[4 * ks + 3], pa[ks][2], pa[ks][3]);
  }
  auto vpair = [&](int tok, int dim) -> uint32_t {
    const uint32_t lo = tok < W ? vwp[tok * D + dim] : 0u;
    const uint32_t hi = tok + 1 < W ? vwp[(tok + 1) * D + dim] : 0u;
    return lo | (hi << 16);
  };
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    if (16 * ks >= W) continue;  // warp-uniform
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const uint32_t b0 = vpair(16 * ks + 2 * t, 8 * n + g);
      const uint32_t b1 = vpair(16 * ks + 2 * t + 8, 8 * n + g);
      mma_bf16(st.o[n], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b0, b1);
    }
  }
}

// ---------------------------------------------------- output scaling --
// Integer / fp8 accumulators to true units: acc * 2^24 * 2^-E (/ sigmaV on value
// channels with bit 3 set); fp8: acc * the KV head's value scale * 2^8.
template <int VB, bool TOK, bool F8, int NT>
__device__ __forceinline__ void to_true_units(State<NT>& st, float f8_vscale) {
  if constexpr (F8) {
    const float f = f8_vscale * kF8Unit;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) st.o[j][k] *= f;
  } else if constexpr (VB != 16) {
    constexpr float sigmaV = VB == 4 ? 16.f : (VB == 2 ? 4.f : 1.f);
    const float f = kTwo24 * exp2i(st.E == kNoExp ? 0 : -st.E);
    const float fh = f * (1.f / sigmaV);
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if constexpr (TOK) {
        st.o[j][0] *= f;
        st.o[j][1] *= f;
        st.o[j][2] *= fh;
        st.o[j][3] *= fh;
      } else {
        const float x = (j & 1) ? fh : f;
#pragma unroll
        for (int k = 0; k < 4; ++k) st.o[j][k] *= x;
      }
    }
  }
}

// ------------------------------------------------------------ fused append --
// Warp-level flush of one completed 32-token group (the window's 31 tokens and
// the new token) into `page`, bit-identical to the append kernel's CTA-wide
// flush: the same quantizer and packing (kvq_quant.cuh), only the work split
// differs. It needs no staging buffer: a first pass takes each set's min and
// max and keeps the quantizer parameters in `prm` (this warp's scratch, 2D + 64
// floats); the second pass quantizes each element as it is packed.
template <int BITS, int D, typename Get>
__device__ __forceinline__ void pack_block_warp(uint8_t* blk, bool is_value, int lane, Get vals) {
  constexpr int kPerLane = (int)(code_block_bytes(BITS, D) / 16) / 32;  // 16-byte vectors per lane
#pragma unroll 1
  for (int vi = 0; vi < kPerLane; ++vi) {
    uint4 q;
    q.x = lane_word<BITS>(lane, 4 * vi + 0, is_value, vals);
    q.y = lane_word<BITS>(lane, 4 * vi + 1, is_value, vals);
    q.z = lane_word<BITS>(lane, 4 * vi + 2, is_value, vals);
    q.w = lane_word<BITS>(lane, 4 * vi + 3, is_value, vals);
    reinterpret_cast<uint4*>(blk)[vi * 32 + lane] = q;
  }
}

template <int KB, int VB, int D, bool PT, bool F8>
__device__ __noinline__ void warp_flush(uint8_t* page, const __nv_bfloat16* win, const __nv_bfloat16* kn,
                                        const __nv_bfloat16* vn, float* prm, float ksc, float vsc,
                                        double* err_stats, int lane) {
  // row of token tok (0..31) of keys (r = 0) or values (r = 1)
  auto row = [&](int r, int tok) -> const __nv_bfloat16* {
    return tok < kPageTokens - 1 ? win + (r * kPageTokens + tok) * D : (r ? vn : kn);
  };
  if constexpr (KB == 16) {
    pack_block_warp<16, D>(page, false, lane,
                           [&](int tok, int dim) { return (uint32_t)__bfloat16_as_ushort(row(0, tok)[dim]); });
    pack_block_warp<16, D>(page + code_block_bytes(16, D), true, lane,
                           [&](int tok, int dim) { return (uint32_t)__bfloat16_as_ushort(row(1, tok)[dim]); });
    return;
  } else {
    double err[4] = {0.0, 0.0, 0.0, 0.0};
    auto add_err = [&](int r, float x, double xh) {
      const double dx = (double)x - xh;
      err[2 * r] += dx * dx;
      err[2 * r + 1] += (double)x * (double)x;
    };
    if constexpr (F8) {
      // every element is e4m3(x / s_h) of its KV head's scale
      auto code = [&](int r, int tok, int dim) -> uint32_t {
        const float x = __bfloat162float(row(r, tok)[dim]);
        const float sc = r ? vsc : ksc;
        const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(__fdiv_rn(x, sc), __NV_SATFINITE, __NV_E4M3);
        add_err(r, x, (double)__half2float(__half(__nv_cvt_fp8_to_halfraw(c, __NV_E4M3))) * sc);
        return (uint32_t)c;
      };
      pack_block_warp<8, D>(page, false, lane, [&](int tok, int dim) { return code(0, tok, dim); });
      pack_block_warp<8, D>(page + code_block_bytes(8, D), true, lane,
                            [&](int tok, int dim) { return code(1, tok, dim); });
    } else {
      constexpr int nk = PT ? kPageTokens : D;  // key scale/zero pairs
      uint8_t* vblk = page + code_block_bytes(KB, D);
      __half* kscale = reinterpret_cast<__half*>(vblk + code_block_bytes(VB, D));
      __half* kzero = kscale + nk;
      __half* vscale = kzero + nk;
      __half* vzero = vscale + kPageTokens;
      // quantizer parameters (zero point z and reciprocal r = 1/s, r = 0 for a
      // constant set) of the keys (by channel, or by token) and of the values
      float* kz = prm;
      float* kr = prm + nk;
      float* vz = prm + 2 * nk;
      float* vr = vz + kPageTokens;
      // per token over head_dim (values; keys in per-token mode): lane = token
      auto per_token = [&](int r, int qmax, __half* sdst, __half* zdst, float* zp, float* rp) {
        const __nv_bfloat16* src = row(r, lane);
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll 1
        for (int c8 = 0; c8 < D; c8 += 8) {
          const uint4 raw = *reinterpret_cast<const uint4*>(src + c8);
          const __nv_bfloat16* xv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float x = __bfloat162float(xv[j]);
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
          }
        }
        const QParams q = make_qparams(mn, mx, qmax);
        sdst[lane] = q.s_h;
        zdst[lane] = q.z_h;
        zp[lane] = q.z;
        rp[lane] = q.r;  // 0 for a constant set
      };
      if constexpr (PT) {
        per_token(0, (1 << KB) - 1, kscale, kzero, kz, kr);
      } else {
        // keys per channel over the 32 tokens: lane owns channels lane * NC .. + NC - 1
        constexpr int NC = D / 32;
        const int c0 = lane * NC;
        float mn[NC], mx[NC];
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          mn[j] = INFINITY;
          mx[j] = -INFINITY;
        }
#pragma unroll 1
        for (int tok = 0; tok < kPageTokens; ++tok) {
          const __nv_bfloat16* src = row(0, tok) + c0;
#pragma unroll
          for (int j = 0; j < NC; ++j) {
            const float x = __bfloat162float(src[j]);
            mn[j] = fminf(mn[j], x);
            mx[j] = fmaxf(mx[j], x);
          }
        }
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          const QParams q = make_qparams(mn[j], mx[j], (1 << KB) - 1);
          const int slot = kmeta_slot<D>(c0 + j);
          kscale[slot] = q.s_h;
          kzero[slot] = q.z_h;
          kz[c0 + j] = q.z;
          kr[c0 + j] = q.r;
        }
      }
      per_token(1, (1 << VB) - 1, vscale, vzero, vz, vr);
      __syncwarp();  // parameters and page metadata visible to the warp
      // element (tok, dim) of keys (r = 0) or values (r = 1): its code, counted once in the report
      auto code = [&](int r, int tok, int dim) -> uint32_t {
        const float x = __bfloat162float(row(r, tok)[dim]);
        const int i = (r == 0 && !PT) ? dim : tok;
        QParams q;
        q.z = r ? vz[i] : kz[i];
        q.r = r ? vr[i] : kr[i];
        q.zero_scale = (q.r == 0.0f);
        const int qmax = (1 << (r ? VB : KB)) - 1;
        const uint32_t c = quant_code(x, q, qmax);
        const __half sh = r ? vscale[i] : kscale[(PT ? i : kmeta_slot<D>(i))];
        add_err(r, x, (double)c * (double)__half2float(sh) + (double)q.z);
        return c;
      };
      pack_block_warp<KB, D>(page, false, lane, [&](int tok, int dim) { return code(0, tok, dim); });
      pack_block_warp<VB, D>(vblk, true, lane, [&](int tok, int dim) { return code(1, tok, dim); });
    }
    // this flush's error sums: warp shuffles, then one fp64 atomic per sum
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      double v = err[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      err[i] = v;
    }
    if (err_stats && lane == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) atomicAdd(&err_stats[i], err[i]);
      atomicAdd(&err_stats[4], (double)(kPageTokens * D));
    }
  }
}

// Append segment s's new token: into window slot t0 mod 32, or, when it
// completes a group, quantized with the window's 31 tokens into page t0 / 32.
// Returns true when a page was written.
template <int KB, int VB, int D, bool PT, bool F8>
__device__ __forceinline__ bool append_token(const DecodeParams& p, int s, int h, int t0, float* prm, int lane) {
  __nv_bfloat16* wwin = p.step_window + ((int64_t)s * 2) * kPageTokens * D;
  const __nv_bfloat16* kn = p.k_new + (int64_t)s * D;
  const __nv_bfloat16* vn = p.v_new + (int64_t)s * D;
  bool flushed = false;
  if ((t0 + 1) % kPageTokens != 0) {
    const int slot = t0 % kPageTokens;
    for (int d = 2 * lane; d < D; d += 64) {
      *reinterpret_cast<uint32_t*>(wwin + slot * D + d) = *reinterpret_cast<const uint32_t*>(kn + d);
      *reinterpret_cast<uint32_t*>(wwin + (kPageTokens + slot) * D + d) = *reinterpret_cast<const uint32_t*>(vn + d);
    }
  } else {
    flushed = true;
    warp_flush<KB, VB, D, PT, F8>(p.step_pages + ((int64_t)s * p.max_pages + t0 / kPageTokens) * p.page_bytes, wwin,
                                  kn, vn, prm, F8 ? p.fp8_scales[h] : 1.f, F8 ? p.fp8_scales[p.n_kv_heads + h] : 1.f,
                                  err_bin(p.err_stats, (unsigned)s), lane);
  }
  __syncwarp();  // the window row or the page is complete for every lane
  return flushed;
}

// ------------------------------------------------------------------ kernel --
// Units: per (sequence b, KV head h) segment, V "overhead" units (no work:
// they stand for the fixed cost of starting and merging a segment part, so a
// CTA that spans several segments gets fewer pages), then one tail unit (the
// bf16 window, and in the fused step the new token's append), then the pages.
// Segment (b, h) occupies units [ustart[b] + h * n_b, ... + n_b). The N units
// are cut into gridDim.x balanced contiguous slices, one per CTA. A slice that
// ends inside a segment's overhead units takes no part in that segment: the
// segment's parts are held by the CTAs from the one owning unit start + V on.

// Segment containing unit u.
struct Seg {
  int b, h, start, n;
};

__device__ __forceinline__ Seg seg_of(const int* ustart, int B, int H, int u) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ustart[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  Seg s;
  s.b = lo;
  s.n = (ustart[lo + 1] - ustart[lo]) / H;
  s.h = (u - ustart[lo]) / s.n;
  s.start = ustart[lo] + s.h * s.n;
  return s;
}

// Balanced slices: with N = q * grid + r, CTA c owns
// [c * q + min(c, r), (c + 1) * q + min(c + 1, r)) -- the first r slices hold one
// extra unit. All in 32-bit integers (N < 2^31).
struct Slicer {
  int q, r;
  __device__ __forceinline__ int lo(int c) const { return c * q + min(c, r); }
  __device__ __forceinline__ bool empty(int c) const { return q == 0 && c >= r; }
  // CTA whose slice contains unit u
  __device__ __forceinline__ int cta_of(int u) const {
    const int big = r * (q + 1);
    return u < big ? u / (q + 1) : r + (u - big) / q;
  }
};

// The pages of a CTA's slice, numbered in unit order (ordinals), are handed to
// the CTA's warps by a shared-memory counter, so a warp that runs ahead (or one
// that spent its time on the tail unit) takes more or fewer of them and the
// warps finish a part together. Each warp's producer (lane 0) walks the slice's
// segment parts forward to the part holding the ordinal it drew.
struct PageWalk {
  int a, e;             // segment part [a, e) of the slice
  int k0, n;            // its first page index in the segment and its page count
  int ord0;             // ordinal of its first page
  const uint8_t* base;  // pages of its (b, h)
};

// Advance w to the part holding ordinal o; false when the slice has no page o.
__device__ __forceinline__ bool walk_to(PageWalk& w, int o, const DecodeParams& p, const int* ustart, const int* slen,
                                        int B, int u1) {
  while (o >= w.ord0 + w.n) {
    if (w.e >= u1) return false;
    const int a = w.e;
    const Seg sg = seg_of(ustart, B, p.n_kv_heads, a);
    const int first = sg.start + p.seg_overhead + 1;  // first page unit (after the overhead and tail units)
    const int e = min(sg.start + sg.n, u1);
    const int lo = max(a, first);
    w.ord0 += w.n;
    w.a = a;
    w.e = e;
    w.k0 = lo - first;
    w.n = max(0, e - lo);
    w.base = p.pages + ((int64_t)(sg.b * p.n_kv_heads + sg.h) * p.max_pages) * p.page_bytes;
  }
  return true;
}

template <int KB, int VB, int D, bool TOK, bool PT, bool F8, bool AP>
__global__ void __launch_bounds__(kThreads, TOK ? Cfg<KB, VB, D, PT, F8>::MINB_TOK : Cfg<KB, VB, D, PT, F8>::MINB)
    decode_mma_kernel(const __grid_constant__ DecodeParams p) {
  using C = Cfg<KB, VB, D, PT, F8>;
  using St = typename std::conditional<TOK, TokState<D>, WarpState<D>>::type;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_last;
  const int H = p.n_kv_heads, G = p.gqa, B = p.batch;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  // this lane's query head: row g (head rows) or column head g/2 (token rows)
  const int qh = TOK ? (g >> 1) : g;

  uint8_t* ring = smem + warp * C::R * C::STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::MBAR_OFF) + warp * C::R;
  float* wscr = reinterpret_cast<float*>(smem + C::WSCR_OFF + warp * C::WSCR_STRIDE);
  uint32_t* qtab = reinterpret_cast<uint32_t*>(smem + C::QZ_OFF);
  float* mo = reinterpret_cast<float*>(smem + C::merge_off(TOK));   // [kWarps + 1][G][D]
  float* mm = mo + (kWarps + 1) * G * D;                             // [kWarps + 1][8]
  float* ml = mm + (kWarps + 1) * kMaxGqa;                           // [kWarps + 1][8]
  int* ustart = reinterpret_cast<int*>(ml + (kWarps + 1) * kMaxGqa); // [B + 1]
  int* slen = ustart + B + 1;                                        // [B]: lengths before this call's append
  __nv_bfloat16* qbuf = reinterpret_cast<__nv_bfloat16*>(smem + C::qbuf_off(TOK));  // [2][G][D]
  constexpr int QROWS = TOK ? 4 : kMaxGqa;  // rows per query buffer
  uint64_t* qbars = reinterpret_cast<uint64_t*>(smem + C::MBAR_OFF) + kWarps * C::R;
  int* stage_part = reinterpret_cast<int*>(qbars + 2) + warp * 4;  // [4]: first unit of the part a stage holds
  int* s_taken = reinterpret_cast<int*>(qbars + 2) + kWarps * 4;   // pages of the slice handed out

  // ---- units per sequence: exclusive scan (warp 0), n_b = H * (V + 1 + P_b)
  auto scan_units = [&](bool host) {
    if (warp == 0) {
      int carry = 0;
      for (int b0 = 0; b0 < B; b0 += 32) {
        const int bb = b0 + lane;
        int n = 0;
        if (bb < B) {
          const int T = host ? p.hlen[bb] : p.len[bb];
          slen[bb] = T;
          n = (T / kPageTokens + 1 + p.seg_overhead) * H;
        }
        int x = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (bb < B) ustart[bb] = carry + x - n;
        carry += __shfl_sync(0xffffffffu, x, 31);
      }
      if (lane == 0) ustart[B] = carry;
    }
  };
  if (lane == 0) {
    for (int r = 0; r < C::R; ++r) mbar_init(&bars[r], 1);
    if (warp == 0) {
      mbar_init(&qbars[0], 1);
      mbar_init(&qbars[1], 1);
      *s_taken = 0;
    }
    mbar_init_fence();
  }
  // with the lengths in the parameters the slices are known before the wait for
  // the preceding kernel; otherwise the device lengths are read after it
  if (p.host_units) scan_units(true);
  else pdl_enter();
  if (!p.host_units) scan_units(false);
  __syncthreads();
  if constexpr (AP) {
    // device lengths: the last CTA to have read them publishes the new ones
    // (acquire-release: every CTA's reads are ordered before that write); a full
    // sequence is left unchanged and the cache's error flag raised
    if (!p.host_units && threadIdx.x == 0) {
      if (atomic_add_acq_rel(p.grid_ctr, 1) == (int)gridDim.x - 1) {
        *p.grid_ctr = 0;
        for (int b = 0; b < B; ++b)
          if (slen[b] < p.max_tokens) p.step_len[b] = slen[b] + 1;
      }
    }
  }
  const int N = ustart[B];
  const Slicer sl{N / (int)gridDim.x, N % (int)gridDim.x};
  const int u0 = sl.lo(blockIdx.x), u1 = sl.lo(blockIdx.x + 1);
  bool work = u0 < u1;
  if (work) {
    // nothing to do when the whole slice lies in one segment's overhead units
    const Seg s0 = seg_of(ustart, B, H, u0);
    work = u1 > s0.start + p.seg_overhead;
  }

  // ---- producer: the first R pages of this warp (pages below the lengths the
  // slices were cut from are never written by the preceding kernel when `early`
  // is set, so they may stream in under its tail)
  PageWalk pw;
  pw.a = pw.e = u0;
  pw.k0 = pw.n = pw.ord0 = 0;
  pw.base = nullptr;
  int issued = 0;
  bool pdone = false;  // lane 0: the slice has no more pages for this warp
  const uint64_t pol = l2_evict_first_policy();
  auto grab = [&](int stage) {
    const int o = atomicAdd(s_taken, 1);
    if (!walk_to(pw, o, p, ustart, slen, B, u1)) {
      pdone = true;
      return;
    }
    stage_part[stage] = pw.a;
    mbar_expect_tx(&bars[stage], C::PB);
    bulk_load_once(ring + stage * C::STAGE, pw.base + (int64_t)(pw.k0 + (o - pw.ord0)) * p.page_bytes, C::PB,
                   &bars[stage], pol);
    ++issued;
  };
  auto issue_first = [&]() {
    if (lane == 0 && work)
      for (int r = 0; r < C::R && !pdone; ++r) grab(r);
  };
  if (p.host_units && p.early) issue_first();
  if (p.host_units) pdl_enter();
  if (!(p.host_units && p.early)) issue_first();
  if (!work) return;  // no copy was issued
  issued = __shfl_sync(0xffffffffu, issued, 0);
  __syncwarp();  // the stage tags are visible to the warp

  // ---- query rows: the first part's straight from global memory (a bulk copy
  // would queue behind the page copies), the later parts' by bulk copy into a
  // shared double buffer one part ahead
  const uint32_t qbytes = (uint32_t)(G * D * 2);
  auto issue_q = [&](int unit, int buf) {
    const Seg qs = seg_of(ustart, B, H, unit);
    fence_proxy_async();  // the buffer's previous rows were read through the generic proxy
    mbar_expect_tx(&qbars[buf], qbytes);
    bulk_load(qbuf + buf * QROWS * D, p.Q + (int64_t)(qs.b * H + qs.h) * G * D, qbytes, &qbars[buf]);
  };

  bool ok = true;
  int consumed = 0;
  int cstage = 0;       // consumed % R
  uint32_t cphase = 0;  // (consumed / R) & 1
  int segi = 0;
  for (int a = u0; a < u1; ++segi) {
    const Seg sg = seg_of(ustart, B, H, a);
    const int e = min(sg.start + sg.n, u1);
    if (e <= sg.start + p.seg_overhead) break;  // overhead units only (the slice's last part)
    const int seg = sg.b * H + sg.h;
    const int T = slen[sg.b];
    const int P = T / kPageTokens;
    const int tu = sg.start + p.seg_overhead;  // the tail unit
    const __nv_bfloat16* win = p.window + ((int64_t)seg * 2) * kPageTokens * D;
    if (threadIdx.x == 0 && a <= tu && T % kPageTokens > 0) {
      // this part holds the tail: bring the window's key and value rows into L2
      prefetch_l2(win, (uint32_t)((T % kPageTokens) * D * 2));
      prefetch_l2(win + kPageTokens * D, (uint32_t)((T % kPageTokens) * D * 2));
    }
    // ---- the tail unit (its warp: part index mod 4): the fused step's append
    // happens here, before the query operands are live; its
    // window, or the page it completed, is attended after the warp's pages
    const bool has_tail = a <= tu;  // (e > tu: a part never ends inside the overhead units)
    const bool appends = AP && (p.host_units || T < p.max_tokens);  // device lengths: a full sequence is left as is
    const int win_tokens = appends ? (T + 1) % kPageTokens : T % kPageTokens;
    const bool has_win = has_tail && win_tokens > 0;
    const bool tail_warp = has_tail && segi % kWarps == warp;
    bool tail_page = false;  // the page the new token completed (attended first by the tail warp)
    if constexpr (AP) {
      if (tail_warp) {
        if (!appends) {
          if (lane == 0 && p.err) atomicExch(p.err, 2);
        } else {
          tail_page = append_token<KB, VB, D, PT, F8>(p, seg, sg.h, T, wscr, lane);
          if (p.host_units && sg.h == 0 && lane == 0) p.step_len[sg.b] = T + 1;
        }
      }
    }
    const bool qvalid = qh < G;
    const __nv_bfloat16* qrow;
    if (segi == 0) {
      qrow = p.Q + ((int64_t)seg * G + (qvalid ? qh : 0)) * D;
    } else {
      const bool got = mbar_wait(&qbars[segi & 1], (uint32_t)(((segi - 1) >> 1) & 1));
      if (!__all_sync(0xffffffffu, got)) ok = false;
      qrow = qbuf + (segi & 1) * QROWS * D + (qvalid ? qh : 0) * D;
    }
    // prefetch the next part's query rows (unless that part is overhead units only)
    if (threadIdx.x == 0 && e < u1 && u1 > e + p.seg_overhead) issue_q(e, (segi + 1) & 1);

    // ---- query operands
    const float ksc = F8 ? p.fp8_scales[sg.h] : 1.f;
    TokOps<D> tops;
    HeadOps hops;
    if constexpr (!C::kBf16) {
      if constexpr (TOK) {
        prep_tok_ops<KB, D, PT, F8>(tops, qrow, qvalid, lane, p.scale_log2, ksc);
      } else {
        prep_head_ops<KB, D, PT, F8>(hops, qtab, warp == 0, qrow, qvalid, lane, p.scale_log2, ksc);
        __syncthreads();
      }
    }
    uint32_t qb[D / 8];   // bf16 q for bf16 pages and the window (loaded when needed)
    auto load_qbp = [&]() { load_qb<D>(qrow, qvalid && (!TOK || (g & 1) == 0), t, qb); };
    if constexpr (C::kBf16) load_qbp();

    // a state (true units: the bf16 MMAs) into merge slot `slot`
    auto store_state = [&](St& x, int slot) {
      if constexpr (TOK) {
        float l = x.l, vz = x.vz;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          l += __shfl_xor_sync(0xffffffffu, l, o);
          vz += __shfl_xor_sync(0xffffffffu, vz, o);
        }
        if (t < G) {
          float* dst = mo + (slot * G + t) * D;
#pragma unroll
          for (int j = 0; j < D / 16; ++j) {
            dst[16 * j + g] = x.o[j][0] + x.o[j][1] + vz;
            dst[16 * j + 8 + g] = x.o[j][2] + x.o[j][3] + vz;
          }
          if (g == 0) {
            mm[slot * kMaxGqa + t] = x.m;
            ml[slot * kMaxGqa + t] = l;
          }
        }
      } else {
        float l = x.l + __shfl_xor_sync(0xffffffffu, x.l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        float vz = x.vz + __shfl_xor_sync(0xffffffffu, x.vz, 1);
        vz += __shfl_xor_sync(0xffffffffu, vz, 2);
        if (g < G) {
          float* dst = mo + (slot * G + g) * D;
#pragma unroll
          for (int j = 0; j < D / 8; ++j) {
            dst[8 * j + 2 * t] = x.o[j][0] + x.o[j][2] + vz;
            dst[8 * j + 2 * t + 1] = x.o[j][1] + x.o[j][3] + vz;
          }
          if (t == 0) {
            mm[slot * kMaxGqa + g] = x.m;
            ml[slot * kMaxGqa + g] = l;
          }
        }
      }
    };
    // the bf16 window, by the tail warp before its pages (its L2 reads overlap the
    // other warps' page stream), into the window's merge slot
    if (tail_warp && win_tokens > 0) {
      St wst;
      state_init(wst);
      if constexpr (!C::kBf16) load_qbp();
      if constexpr (TOK) attend_window_tok<D>(win, win_tokens, wst, qb, p.scale_log2, lane);
      else attend_window<D>(win, win_tokens, wst, qb, p.scale_log2, lane);
      store_state(wst, kWarps);
    }

    St st;
    state_init(st);
    auto attend_page = [&](const uint8_t* page) {
      if constexpr (TOK) {
        if constexpr (C::kBf16) attend_bpage_tok<D>(page, st, qb, p.scale_log2, lane);
        else if constexpr (F8) attend_f8page_tok<D>(page, st, tops, lane);
        else if constexpr (PT) attend_qpage_tok_pt<KB, VB, D>(page, st, tops, wscr, lane);
        else attend_qpage_tok<KB, VB, D>(page, st, tops, wscr, lane);
      } else {
        if constexpr (C::kBf16) attend_bpage<D>(page, st, qb, p.scale_log2, lane);
        else if constexpr (F8) attend_f8page<D>(page, st, qtab, lane);
        else if constexpr (PT) attend_qpage_pt<KB, VB, D>(page, st, qtab, hops, wscr, lane);
        else attend_qpage<KB, VB, D>(page, st, qtab, hops, wscr, lane);
      }
    };

    // the page the new token completed (generic loads: it never went through the async proxy)
    if (tail_page) attend_page(p.pages + ((int64_t)seg * p.max_pages + P) * p.page_bytes);

    // ---- this warp's pages of the segment part [a, e): the ring in order, while
    // its stages hold pages of this part
    for (;;) {
      if (!ok || consumed == issued) break;  // a lost copy, or no more pages for this warp
      const int stage = cstage;
      if (stage_part[stage] != a) break;     // the next page belongs to a later part
      const bool arrived = mbar_wait(&bars[stage], cphase);
      if (!__all_sync(0xffffffffu, arrived)) {  // warp-uniform verdict
        ok = false;
        break;
      }
      attend_page(ring + stage * C::STAGE);
      ++consumed;
      if (++cstage == C::R) {
        cstage = 0;
        cphase ^= 1u;
      }
      __syncwarp();
      if (lane == 0 && !pdone) {
        fence_proxy_async();
        grab(stage);
      }
      issued = __shfl_sync(0xffffffffu, issued, 0);
      __syncwarp();  // the stage tag is visible to the warp
    }
    to_true_units<VB, TOK, F8>(st, F8 ? p.fp8_scales[H + sg.h] : 1.f);
    store_state(st, warp);
    __syncthreads();
    const bool whole = has_tail && (e == sg.start + sg.n);
    float* outp = p.out + (int64_t)seg * G * D;
    float* part = p.partials + ((int64_t)blockIdx.x * 2 + (a == u0 ? 0 : 1)) * split_record_floats(G, D);
    const int nslots = kWarps + (has_win ? 1 : 0);
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
      const int gg = idx / D, d = idx % D;
      float M = -INFINITY;
      for (int w = 0; w < nslots; ++w) M = fmaxf(M, mm[w * kMaxGqa + gg]);
      float L = 0.f, O = 0.f;
      for (int w = 0; w < nslots; ++w) {
        const float mw = mm[w * kMaxGqa + gg];
        const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        L = fmaf(f, ml[w * kMaxGqa + gg], L);
        O = fmaf(f, mo[(w * G + gg) * D + d], O);
      }
      if (whole) {
        outp[idx] = L > 0.f ? O / L : 0.f;
      } else {
        // record: [G][D] accumulators, then [G] maxima, then [G] sums
        part[idx] = O;
        if (d == 0) {
          part[G * D + gg] = M;
          part[G * D + G + gg] = L;
        }
      }
    }
    if (!whole) {
      // The last CTA of a split segment merges the slices' partials in slice
      // order (empty slices, possible when CTAs outnumber units, hold nothing).
      const int c_lo = sl.cta_of(tu), c_hi = sl.cta_of(sg.start + sg.n - 1);
      __syncthreads();  // this CTA's partial record is complete
      if (threadIdx.x == 0) {
        int parts = 0;
        for (int c = c_lo; c <= c_hi; ++c) parts += !sl.empty(c);
        const int prev = atomic_add_acq_rel(&p.ctr[seg], 1);
        s_last = (prev == parts - 1);
        if (s_last) p.ctr[seg] = 0;
      }
      __syncthreads();
      if (s_last) {
        // The slices' records, four channels per thread, 4, 8 or 16 records per
        // round with all their loads in flight at once (maximum, sum and
        // accumulators), each weighted by 2^(m_c - M); rounds are joined by online
        // rescaling. An empty slice (or a padding entry of a round) has weight 0 and
        // is read from this CTA's own record in its place.
        const int nrec = c_hi - c_lo + 1;
        const int64_t rec_floats = split_record_floats(G, D);
        for (int i4 = threadIdx.x; i4 < G * D / 4; i4 += kThreads) {
          const int gg = (4 * i4) / D, d = (4 * i4) % D;
          float M = -INFINITY, L = 0.f;
          float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
          // one round of R records starting at record k0
          auto merge_round = [&](auto rounds, int k0) {
            constexpr int R = decltype(rounds)::value;
            float mc[R], lc[R];
            float4 oc[R];
#pragma unroll
            for (int j = 0; j < R; ++j) {
              const int c = c_lo + k0 + j;
              const bool valid = k0 + j < nrec && !sl.empty(c);
              const float* r =
                  valid ? p.partials + ((int64_t)c * 2 + ((sl.lo(c) >= sg.start) ? 0 : 1)) * rec_floats : part;
              const float m = __ldcg(r + G * D + gg);
              mc[j] = valid ? m : -INFINITY;
              lc[j] = __ldcg(r + G * D + G + gg);
              oc[j] = __ldcg(reinterpret_cast<const float4*>(r + gg * D + d));
            }
            float Mn = M;
#pragma unroll
            for (int j = 0; j < R; ++j) Mn = fmaxf(Mn, mc[j]);
            if (Mn == -INFINITY) return;
            const float fa = (M == -INFINITY) ? 0.f : exp2f(M - Mn);
            L *= fa;
            O.x *= fa;
            O.y *= fa;
            O.z *= fa;
            O.w *= fa;
#pragma unroll
            for (int j = 0; j < R; ++j) {
              const float w = (mc[j] == -INFINITY) ? 0.f : exp2f(mc[j] - Mn);
              L = fmaf(w, lc[j], L);
              O.x = fmaf(w, oc[j].x, O.x);
              O.y = fmaf(w, oc[j].y, O.y);
              O.z = fmaf(w, oc[j].z, O.z);
              O.w = fmaf(w, oc[j].w, O.w);
            }
            M = Mn;
          };
          if (nrec <= 4) {
            merge_round(std::integral_constant<int, 4>{}, 0);
          } else if (nrec <= 8) {
            merge_round(std::integral_constant<int, 8>{}, 0);
          } else {
            for (int k0 = 0; k0 < nrec; k0 += 16) merge_round(std::integral_constant<int, 16>{}, k0);
          }
          const float inv = L > 0.f ? 1.f / L : 0.f;
          *reinterpret_cast<float4*>(outp + gg * D + d) = make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
        }
      }
    }
    __syncthreads();  // merge area, query table and s_last are reused by the next segment
    a = e;
  }

  if (!ok) {
    // a copy never completed: report it, then let the copies in flight land
    // (each wait bounded again) before this CTA's shared memory goes away
    if (lane == 0 && p.err) atomicExch(p.err, 1);
    for (int i = consumed; i < issued; ++i) mbar_wait(&bars[i % C::R], (uint32_t)((i / C::R) & 1));
  }
}

// ---------------------------------------------------------- warp-segment kernel --
// Short sequences (token rows, G <= 4): warp w of CTA c attends segments
// s = c * kWarps + w, then s + gridDim.x * kWarps, ... on its own -- query rows
// by bulk copy into the warp's slot, pages through the warp's ring, then the
// window -- and writes the segment's output directly. No CTA barrier, split
// record or merge: at a few pages per segment those fixed costs, not the page
// bytes, are what a shared split spends its time on.
template <int KB, int VB, int D, bool PT, bool F8>
struct WarpCfg {
  using C = Cfg<KB, VB, D, PT, F8>;
  static constexpr int MBAR_OFF = C::RING;
  static constexpr int MBAR_BYTES = ((kWarps * (C::R + 1)) * 8 + 127) / 128 * 128;  // ring + one query barrier
  static constexpr int WSCR_OFF = MBAR_OFF + MBAR_BYTES;
  static constexpr int QBUF_OFF = WSCR_OFF + kWarps * C::WSCR_STRIDE;
  static constexpr int QSLOT = 4 * D * 2;                                            // [4][D] bf16 per warp
  static constexpr int SMEM = QBUF_OFF + kWarps * QSLOT;
  // warp pairs: per pair three barriers (length handed over, state dumped, dump read),
  // the handed-over length, and the second warp's state [32 lanes][D/4 + 3] floats
  static constexpr int DUMP_FLOATS = D / 4 + 3;
  static constexpr int PBAR_OFF = SMEM;
  static constexpr int T0_OFF = PBAR_OFF + (kWarps / 2) * 3 * 8;
  static constexpr int DUMP_OFF = (T0_OFF + (kWarps / 2) * 4 + 15) / 16 * 16;
  static constexpr int SMEM_PAIR = DUMP_OFF + (kWarps / 2) * 32 * DUMP_FLOATS * 4;
};

// AP (kvq_decode_step): before attending segment (b, h) the warp appends its new
// token -- into the window, or, when it completes a group, quantized into the
// next page, which the warp then attends from global memory -- and the last of
// sequence b's H warps to have read the old length publishes the new one (the
// acquire-release increment orders every read before that write).
//
// PAIR: warps 2i and 2i + 1 share a segment -- the first takes its even pages,
// the tail and the window, the second its odd pages -- and the first merges the
// second's state from shared memory before the window and the output. The pair
// syncs on three mbarriers, every wait bounded like the ring's.
template <int KB, int VB, int D, bool PT, bool F8, bool AP = false, bool PAIR = false>
__global__ void __launch_bounds__(kThreads, Cfg<KB, VB, D, PT, F8>::MINB_TOK)
    decode_warp_kernel(const __grid_constant__ DecodeParams p) {
  pdl_enter();
  using C = Cfg<KB, VB, D, PT, F8>;
  using WC = WarpCfg<KB, VB, D, PT, F8>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int H = p.n_kv_heads, G = p.gqa;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int qh = g >> 1;  // column head of this lane
  uint8_t* ring = smem + warp * C::R * C::STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + WC::MBAR_OFF) + warp * (C::R + 1);
  uint64_t* qbar = bars + C::R;
  float* wscr = reinterpret_cast<float*>(smem + WC::WSCR_OFF + warp * C::WSCR_STRIDE);
  __nv_bfloat16* qslot = reinterpret_cast<__nv_bfloat16*>(smem + WC::QBUF_OFF + warp * WC::QSLOT);
  constexpr int SPW = PAIR ? 2 : 1;  // warps per segment
  const int half = PAIR ? (warp & 1) : 0;
  uint64_t* pbar = reinterpret_cast<uint64_t*>(smem + WC::PBAR_OFF) + (warp >> 1) * 3;
  int* t0slot = reinterpret_cast<int*>(smem + WC::T0_OFF) + (warp >> 1);
  float* dump = reinterpret_cast<float*>(smem + WC::DUMP_OFF) + (warp >> 1) * 32 * WC::DUMP_FLOATS +
                lane * WC::DUMP_FLOATS;
  if (lane == 0) {
    for (int r = 0; r <= C::R; ++r) mbar_init(&bars[r], 1);
    if (PAIR && half == 0)
      for (int r = 0; r < 3; ++r) mbar_init(&pbar[r], 1);
    mbar_init_fence();
  }
  if constexpr (PAIR) __syncthreads();  // the pair barriers exist before either warp uses them
  else __syncwarp();

  const int S = p.batch * H;
  const int stride = (int)gridDim.x * kWarps / SPW;
  const uint32_t qbytes = (uint32_t)(G * D * 2);
  const uint64_t pol = l2_evict_first_policy();
  bool ok = true;
  int issued = 0, consumed = 0, nq = 0;
  for (int s = (blockIdx.x * kWarps + warp) / SPW; s < S && ok; s += stride, ++nq) {
    const int b = s / H, h = s % H;
    int T, P;              // tokens attended; pages of the segment (before the new token)
    bool flushed = false;  // AP: page P, just written, is attended too
    if constexpr (AP) {
      int t0 = 0;
      if (PAIR && half == 1) {
        // the first warp of the pair read the length and appended the token
        const bool got = mbar_wait(&pbar[0], (uint32_t)(nq & 1));
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        t0 = *t0slot;
      } else if (lane == 0) {
        t0 = p.step_len[b];
        if (atomic_add_acq_rel(&p.append_ctr[b], 1) == H - 1) {
          p.append_ctr[b] = 0;
          if (t0 < p.max_tokens) p.step_len[b] = t0 + 1;
        }
      }
      t0 = __shfl_sync(0xffffffffu, t0, 0);
      if (PAIR && half == 0 && lane == 0) {
        *t0slot = t0;
        mbar_arrive(&pbar[0]);
      }
      P = t0 / kPageTokens;
      if (t0 < p.max_tokens) {
        T = t0 + 1;
        if (half == 0) flushed = append_token<KB, VB, D, PT, F8>(p, s, h, t0, wscr, lane);
      } else {
        T = t0;  // a full sequence is left unchanged and the cache's error flag raised
        if (half == 0 && lane == 0 && p.err) atomicExch(p.err, 2);
      }
    } else {
      T = p.len[b];
      P = T / kPageTokens;
    }
    const int W = T % kPageTokens;
    // this warp's pages: half, half + SPW, ... (all of them without pairs)
    const int Pn = P > half ? (P - half + SPW - 1) / SPW : 0;
    const uint8_t* base = p.pages + ((int64_t)s * p.max_pages + half) * p.page_bytes;
    const int64_t pstride = (int64_t)SPW * p.page_bytes;
    const __nv_bfloat16* win = p.window + ((int64_t)s * 2) * kPageTokens * D;
    int next = 0;  // next of this warp's pages to copy
    if (lane == 0) {
      fence_proxy_async();  // the slot's previous rows were read through the generic proxy
      mbar_expect_tx(qbar, qbytes);
      bulk_load(qslot, p.Q + (int64_t)s * G * D, qbytes, qbar);
      for (; next < Pn && next < C::R; ++next) {
        const int stage = (issued + next) % C::R;
        mbar_expect_tx(&bars[stage], C::PB);
        bulk_load_once(ring + stage * C::STAGE, base + (int64_t)next * pstride, C::PB, &bars[stage], pol);
      }
      if (W > 0 && half == 0) {
        prefetch_l2(win, (uint32_t)(W * D * 2));
        prefetch_l2(win + kPageTokens * D, (uint32_t)(W * D * 2));
      }
    }
    next = __shfl_sync(0xffffffffu, next, 0);
    issued += next;
    {
      const bool got = mbar_wait(qbar, (uint32_t)(nq & 1));
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
    }
    const bool qvalid = qh < G;
    const __nv_bfloat16* qrow = qslot + (qvalid ? qh : 0) * D;
    TokOps<D> tops;
    if constexpr (!C::kBf16) prep_tok_ops<KB, D, PT, F8>(tops, qrow, qvalid, lane, p.scale_log2, F8 ? p.fp8_scales[h] : 1.f);
    uint32_t qb[D / 8];
    auto load_qbp = [&]() { load_qb<D>(qrow, qvalid && (g & 1) == 0, t, qb); };
    if constexpr (C::kBf16) load_qbp();

    TokState<D> st;
    state_init(st);
    auto attend_page = [&](const uint8_t* page) {
      if constexpr (C::kBf16) attend_bpage_tok<D>(page, st, qb, p.scale_log2, lane);
      else if constexpr (F8) attend_f8page_tok<D>(page, st, tops, lane);
      else if constexpr (PT) attend_qpage_tok_pt<KB, VB, D>(page, st, tops, wscr, lane);
      else attend_qpage_tok<KB, VB, D>(page, st, tops, wscr, lane);
    };
    for (int k = 0; k < Pn; ++k) {
      const int stage = consumed % C::R;
      const bool arrived = mbar_wait(&bars[stage], (uint32_t)((consumed / C::R) & 1));
      if (!__all_sync(0xffffffffu, arrived)) {
        ok = false;
        break;
      }
      attend_page(ring + stage * C::STAGE);
      ++consumed;
      __syncwarp();
      if (next < Pn) {
        if (lane == 0) {
          fence_proxy_async();
          mbar_expect_tx(&bars[stage], C::PB);
          bulk_load_once(ring + stage * C::STAGE, base + (int64_t)next * pstride, C::PB, &bars[stage], pol);
        }
        ++next;
        ++issued;
      }
    }
    if (!ok) break;
    // the page this warp has just written (generic loads: it never went through the async proxy)
    if (flushed) attend_page(p.pages + ((int64_t)s * p.max_pages + P) * p.page_bytes);
    to_true_units<VB, true, F8>(st, F8 ? p.fp8_scales[H + h] : 1.f);
    if constexpr (PAIR) {
      constexpr int NT = D / 16;
      if (half == 1) {
        // hand this warp's state over once the first warp has read the previous one
        bool got = nq == 0 || mbar_wait(&pbar[2], (uint32_t)((nq - 1) & 1));
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int k = 0; k < 4; ++k) dump[4 * j + k] = st.o[j][k];
        dump[4 * NT] = st.m;
        dump[4 * NT + 1] = st.l;
        dump[4 * NT + 2] = st.vz;
        __syncwarp();
        if (lane == 0) mbar_arrive(&pbar[1]);
        __syncwarp();  // every lane has read the query slot before the next segment's copy lands
        continue;
      }
      // merge the second warp's state (same lane layout; heads share st.m per lane)
      const bool got = mbar_wait(&pbar[1], (uint32_t)(nq & 1));
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      const float m1 = dump[4 * NT];
      const float M = fmaxf(st.m, m1);
      const float f0 = (st.m == -INFINITY) ? 0.f : ex2(st.m - M);
      const float f1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M);
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k) st.o[j][k] = st.o[j][k] * f0 + dump[4 * j + k] * f1;
      st.l = st.l * f0 + dump[4 * NT + 1] * f1;
      st.vz = st.vz * f0 + dump[4 * NT + 2] * f1;
      st.m = M;
      __syncwarp();
      if (lane == 0) mbar_arrive(&pbar[2]);
    }
    if (W > 0) {
      if constexpr (!C::kBf16) load_qbp();
      attend_window_tok<D>(win, W, st, qb, p.scale_log2, lane);
    }

    // head t's sum over the warp's tokens, then the output rows of this segment
    float l = st.l, vz = st.vz;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, o);
      vz += __shfl_xor_sync(0xffffffffu, vz, o);
    }
    if (t < G) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float* dst = p.out + ((int64_t)s * G + t) * D;
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        dst[16 * j + g] = (st.o[j][0] + st.o[j][1] + vz) * inv;
        dst[16 * j + 8 + g] = (st.o[j][2] + st.o[j][3] + vz) * inv;
      }
    }
    __syncwarp();  // every lane has read the query slot before the next segment's copy lands
  }

  if (!ok) {
    // a copy never completed: report it, then let the copies in flight land
    // (each wait bounded again) before this CTA's shared memory goes away
    if (lane == 0 && p.err) atomicExch(p.err, 1);
    for (int i = consumed; i < issued; ++i) mbar_wait(&bars[i % C::R], (uint32_t)((i / C::R) & 1));
    mbar_wait(qbar, (uint32_t)(nq & 1));
  }
}

// ---------------------------------------------------------------- launchers --
// One warp per segment when every segment fits one resident wave of warps;
// cudaErrorNotSupported (nothing launched) otherwise.
template <int KB, int VB, int D, bool PT, bool F8, bool AP>
cudaError_t launch_warp(const DecodeParams& p, cudaStream_t s) {
  using WC = WarpCfg<KB, VB, D, PT, F8>;
  static bool configured = false;
  static int occ = 0, occ_pair = 0;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(decode_warp_kernel<KB, VB, D, PT, F8, AP, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, WC::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_warp_kernel<KB, VB, D, PT, F8, AP, false>,
                                                      kThreads, WC::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_warp_kernel<KB, VB, D, PT, F8, AP, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, WC::SMEM_PAIR);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_pair, decode_warp_kernel<KB, VB, D, PT, F8, AP, true>,
                                                      kThreads, WC::SMEM_PAIR);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int64_t segs = (int64_t)p.batch * p.n_kv_heads;
  if (p.warp_pairs) {
    // two warps per segment when the pairs fit one resident wave too
    const int64_t ctas = (2 * segs + kWarps - 1) / kWarps;
    if (ctas >= 1 && ctas <= (int64_t)occ_pair * p.sm_count)
      return launch_pdl(decode_warp_kernel<KB, VB, D, PT, F8, AP, true>, dim3((unsigned)ctas), dim3(kThreads),
                        (size_t)WC::SMEM_PAIR, s, p);
  }
  const int64_t ctas = (segs + kWarps - 1) / kWarps;
  if (ctas < 1 || ctas > (int64_t)occ * p.sm_count) return cudaErrorNotSupported;
  return launch_pdl(decode_warp_kernel<KB, VB, D, PT, F8, AP, false>, dim3((unsigned)ctas), dim3(kThreads),
                    (size_t)WC::SMEM, s, p);
}

// The shared split: resident CTAs per SM x SMs, capped by the units and the
// split-record slots.
template <int KB, int VB, int D, bool TOK, bool PT, bool F8, bool AP>
cudaError_t launch_shared(const DecodeParams& p, cudaStream_t s) {
  using C = Cfg<KB, VB, D, PT, F8>;
  static int configured_smem = 0;
  static int occ_smem = -1, occ_blocks = 0;
  const int smem = C::smem_bytes(TOK, p.gqa, p.batch);
  if (smem > configured_smem) {
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<KB, VB, D, TOK, PT, F8, AP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured_smem = smem;
  }
  if (smem != occ_smem) {
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &occ_blocks, decode_mma_kernel<KB, VB, D, TOK, PT, F8, AP>, kThreads, smem);
    if (e != cudaSuccess) return e;
    occ_smem = smem;
  }
  int64_t grid = (int64_t)(occ_blocks > 0 ? occ_blocks : 1) * p.sm_count;
  grid = std::min<int64_t>(grid, p.n_units);
  grid = std::min<int64_t>(grid, p.max_ctas);
  if (grid < 1) grid = 1;
  return launch_pdl(decode_mma_kernel<KB, VB, D, TOK, PT, F8, AP>, dim3((unsigned)grid), dim3(kThreads),
                    (size_t)smem, s, p);
}

template <int KB, int VB, int D, bool TOK, bool PT, bool F8>
cudaError_t launch4(const DecodeParams& p, cudaStream_t s) {
  if constexpr (TOK) {
    if (p.warp_split) {
      const cudaError_t e =
          p.append ? launch_warp<KB, VB, D, PT, F8, true>(p, s) : launch_warp<KB, VB, D, PT, F8, false>(p, s);
      if (e != cudaErrorNotSupported) return e;
    }
  }
  return p.append ? launch_shared<KB, VB, D, TOK, PT, F8, true>(p, s)
                  : launch_shared<KB, VB, D, TOK, PT, F8, false>(p, s);
}

template <int KB, int VB, int D>
cudaError_t launch3(const DecodeParams& p, cudaStream_t s) {
  // token rows when the query group fits the 8 (head, part) columns
  if constexpr (KB == 8 && VB == 8) {
    if (p.fmt != 0)
      return p.gqa <= 4 ? launch4<KB, VB, D, true, false, true>(p, s) : launch4<KB, VB, D, false, false, true>(p, s);
  }
  if constexpr (KB != 16) {
    if (p.key_mode != 0)
      return p.gqa <= 4 ? launch4<KB, VB, D, true, true, false>(p, s) : launch4<KB, VB, D, false, true, false>(p, s);
  }
  return p.gqa <= 4 ? launch4<KB, VB, D, true, false, false>(p, s) : launch4<KB, VB, D, false, false, false>(p, s);
}

template <int D>
cudaError_t launch_d(int kb, int vb, const DecodeParams& p, cudaStream_t s) {
#define KVQ_PAIR(K_, V_) \
  if (kb == K_ && vb == V_) return launch3<K_, V_, D>(p, s);
  KVQ_PAIR(2, 2) KVQ_PAIR(2, 4) KVQ_PAIR(2, 8)
  KVQ_PAIR(4, 2) KVQ_PAIR(4, 4) KVQ_PAIR(4, 8)
  KVQ_PAIR(8, 2) KVQ_PAIR(8, 4) KVQ_PAIR(8, 8)
  KVQ_PAIR(16, 16)
#undef KVQ_PAIR
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_mma(int kb, int vb, int D, const DecodeParams& p, cudaStream_t s) {
  if (D == 64) return launch_d<64>(kb, vb, p, s);
  if (D == 128) return launch_d<128>(kb, vb, p, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
