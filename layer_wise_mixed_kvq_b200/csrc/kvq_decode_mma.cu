// kvq_decode_mma.cu -- split-K decode attention over one layer's mixed-precision
// cache on the tensor cores (warp-level mma.sync m16n8k16, fp32 accumulate).
//
// KVTuner OpenReview rebuttal, "Baseline Implementation": decode runs
// FlashAttention-style kernels directly over the int8 / mixed-precision K and V
// cache; "New GQA efficiency results": grouped-query attention. Keys are
// dequantized per channel (x = code * s_c + z_c over each 32-token page) and
// values per token (x = code * s_t + z_t).
//
// Work splits, 4 warps per CTA, each warp streaming pages through a private
// ring of shared-memory stages filled by bulk copies (cp.async.bulk, one copy
// per page, mbarrier completion) with its own online-softmax state:
//  * shared split (decode_mma_kernel): a persistent grid cuts all (sequence,
//    KV head) segments' pages into balanced contiguous slices, one per CTA; the
//    CTA's warps take a segment part's pages in turn, merge in shared memory,
//    and either write the output or leave a split record that the last CTA of
//    the segment merges;
//  * warp split (decode_warp_kernel, short sequences, G <= 4): each warp
//    attends whole segments alone and writes their outputs; its fused form
//    first appends the segment's new token (window slot, or a warp-level
//    flush of the completed group into the next page).
//
// Per page (32 tokens), with MMA rows = query heads: row g holds the high f16
// part of head g's operand and row g + 8 the low part (hi + lo carries ~22
// bits), so any G <= 8 fits one 16-row tile and S = C[g] + C[g + 8].
//   z-term : C_z = q_hi/lo x z (z broadcast over the 8 columns): sum_c q_c z_c.
//   QK     : A = q' = q * s_c (hi/lo), B = key codes, accumulators seeded with C_z.
//   softmax: online max / sum in the log2 domain (q carries log2(e)/sqrt(D)).
//   PV     : A = p' = p * s_t (hi/lo, straight from the QK accumulators),
//            B = value codes; sum_t p_t z_t is added per head at the end.
// Codes enter the tensor core as f16 *subnormals*: masking a packed word with
// 0x000F000F (4-bit), 0x00030003 (2-bit) or byte-permuting with zero (8-bit)
// yields the f16 pair (c_a * 2^-24, c_b * 2^-24) exactly, so unpacking costs one
// logic op per two codes. Codes sitting higher in a word come out multiplied
// by a power of two; those factors are folded, exactly, into q', p', the score
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
constexpr float kScaleCapLazy = 255.0f;       // largest value scale for which p' = p * s <= 65504 at p <= 2^kTau

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
  // room for the rest of a CTA's shared memory (about 20-30 KB) inside half an SM
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
  // per-warp key-scale table: row t holds this lane's D/4 scales, rows padded by
  // 4 floats so the four rows fall on different banks
  static constexpr int KSROW = D / 4 + 4;
  // shared memory layout
  static constexpr int RING = kWarps * R * STAGE;
  static constexpr int MBAR_OFF = RING;
  static constexpr int MBAR_BYTES = ((kWarps * R + 2) * 8 + 127) / 128 * 128;  // + 2 query-row barriers
  static constexpr int WSCR_FLOATS = 4 * KSROW + 64 + 160;  // key scales, value scales/zeros, p' transpose tile
  static constexpr int WSCR_OFF = MBAR_OFF + MBAR_BYTES;
  static constexpr int WSCR_STRIDE = (WSCR_FLOATS * 4 + 127) / 128 * 128;
  static constexpr int QZ_OFF = WSCR_OFF + kWarps * WSCR_STRIDE;
  static constexpr int QZ_BYTES = KS * 32 * 16;            // head rows: z-term q fragments
  static constexpr int QBUF_BYTES = 2 * kMaxGqa * D * 2;   // 2 x [8][D] bf16 query rows (= QZ_BYTES)
  // token rows have no z-term fragments in shared memory: their query rows take that place
  static constexpr int qbuf_off(bool tok) { return tok ? QZ_OFF : QZ_OFF + QZ_BYTES; }
  static constexpr int merge_off(bool tok) { return qbuf_off(tok) + QBUF_BYTES; }
  // then: merge area [kWarps][G][D] + m, l [kWarps][8] floats, unit starts [batch + 1] ints
  static int smem_bytes(bool tok, int G, int batch) {
    return merge_off(tok) + (kWarps * G * D + 2 * kWarps * kMaxGqa) * 4 + (batch + 1) * 4;
  }
  static_assert(PB % 16 == 0, "bulk copies need 16-byte multiples");
};

// Per-warp running state for the G heads (lane (g, t) owns head g).
template <int D>
struct WarpState {
  float o[D / 8][4];   // PV accumulators: [n-tile][c0..c3], rows g (hi) and g+8 (lo)
  float m;             // reference max (log2 domain), identical across the quad
  float l;             // partial sum over this lane's tokens
  float vz;            // partial sum_t p_t z_t over this lane's tokens
};

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

// Online-softmax update with this page's scores sc[8] (log2 domain; tokens
// 8j + 2t + {0,1} for n-tile j = i/2; masked tokens are -inf). The reference
// max is raised only when a score exceeds it by more than tau, so p <= 2^tau.
// Returns p in sc.
template <int D>
__device__ __forceinline__ void softmax_update(WarpState<D>& st, float (&sc)[8], float tau) {
  float mx = fmaxf(fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3])), fmaxf(fmaxf(sc[4], sc[5]), fmaxf(sc[6], sc[7])));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  if (mx > st.m + tau) {
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

// ------------------------------------------------------------ page kernels --
// One full quantized page in shared memory -> state.
template <int KB, int VB, int D>
__device__ __forceinline__ void attend_qpage(const uint8_t* page, WarpState<D>& st, const float (&qf)[D / 4],
                                             const uint32_t* qz, float* wscr, int lane) {
  using C = Cfg<KB, VB, D>;
  const int t = lane & 3;
  const uint8_t* vblk = page + code_block_bytes(KB, D);
  const __half* kscale = reinterpret_cast<const __half*>(vblk + code_block_bytes(VB, D));
  const __half* kzero = kscale + D;
  const __half* vscale = kzero + D;
  const __half* vzero = vscale + kPageTokens;
  float* ksf = wscr;                   // [4][KSROW] key scales by lane row t, tauK folded
  float* svf = wscr + 4 * C::KSROW;    // [32] value scales, tauV folded
  float* zvf = svf + kPageTokens;      // [32] value zeros

  // --- scale tables in fp32, converted cooperatively by the warp
  {
    constexpr int NE = D / 32;         // entries per lane, all in one row
    const int i0 = lane * NE;
    float* dst = ksf + (i0 / (D / 4)) * C::KSROW + (i0 % (D / 4));
    if constexpr (NE == 4) {
      const uint2 raw = *reinterpret_cast<const uint2*>(kscale + i0);
      float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
      float2 c = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
      if (C::tauK != 1.f) { c.x *= 1.f / C::tauK; c.y *= 1.f / C::tauK; }  // entries j = 2, 3
      *reinterpret_cast<float4*>(dst) = make_float4(a.x, a.y, c.x, c.y);
    } else {
      const uint32_t raw = *reinterpret_cast<const uint32_t*>(kscale + i0);
      float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw));
      if (C::tauK != 1.f && (i0 & 2)) { a.x *= 1.f / C::tauK; a.y *= 1.f / C::tauK; }
      *reinterpret_cast<float2*>(dst) = a;
    }
  }
  const float vs = __half2float(vscale[lane]);
  svf[lane] = (C::tauV != 1.f && (lane & 8)) ? vs * (1.f / C::tauV) : vs;
  zvf[lane] = __half2float(vzero[lane]);
  // lazy rescaling keeps p <= 2^kTau; p' = p * s must stay inside f16
  const float tau = __any_sync(0xffffffffu, vs > kScaleCapLazy) ? 0.f : kTau;
  __syncwarp();

  // --- QK (A = q' hi/lo, B = key codes) and the z-term (A = q hi/lo, B = z)
  float s4[4][4], cz[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) s4[j][k] = 0.f;
  const float* ksl = ksf + t * C::KSROW;
  const uint32_t* zrow = reinterpret_cast<const uint32_t*>(kzero + t * (D / 4));
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<KB>::N];
    load_tile_words<KB>(page, lane, dt, w);
    const float4 sc4 = *reinterpret_cast<const float4*>(ksl + dt * 4);
    uint32_t ah0, al0, ah1, al1;
    split_f16(qf[dt * 4 + 0] * sc4.x, qf[dt * 4 + 1] * sc4.y, ah0, al0);
    split_f16(qf[dt * 4 + 2] * sc4.z, qf[dt * 4 + 3] * sc4.w, ah1, al1);
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      uint32_t b[4];
      tile_frags<KB>(w, tt, b);
      mma_f16(s4[2 * tt], ah0, al0, ah1, al1, b[0], b[1]);
      mma_f16(s4[2 * tt + 1], ah0, al0, ah1, al1, b[2], b[3]);
    }
    const uint4 a = *reinterpret_cast<const uint4*>(qz + (dt * 32 + lane) * 4);
    const uint2 z = *reinterpret_cast<const uint2*>(zrow + dt * 2);
    mma_f16(cz, a.x, a.y, a.z, a.w, z.x, z.y);
  }
  const float czv = cz[0] + cz[2];  // every column holds the same sum
  float sc[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float f = (j & 1) ? kTwo24 / C::sigmaK : kTwo24;
    sc[2 * j] = fmaf(s4[j][0] + s4[j][2], f, czv);
    sc[2 * j + 1] = fmaf(s4[j][1] + s4[j][3], f, czv);
  }
  softmax_update<D>(st, sc, tau);

  // --- PV: A = p' (hi/lo) per 16-token k-step, B = value codes
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
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<VB>::N];
    load_tile_words<VB>(vblk, lane, dt, w);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t b[4];
      tile_frags<VB>(w, ks, b);
      mma_f16(st.o[2 * dt], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[0], b[1]);
      mma_f16(st.o[2 * dt + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[2], b[3]);
    }
  }
}

// Per-token keys, head rows: score of head g, token t = s_t * sum_c q'_c code_tc
// + z_t * sum_c q'_c. The A operand is the segment's q' hi/lo fragments in
// shared memory (2-bit tauK already folded in); no key-scale table, no z-term MMA.
template <int KB, int VB, int D>
__device__ __forceinline__ void attend_qpage_pt(const uint8_t* page, WarpState<D>& st, const uint32_t* qz,
                                                float qsum, float* wscr, int lane) {
  using C = Cfg<KB, VB, D, true>;
  const int t = lane & 3;
  const uint8_t* vblk = page + code_block_bytes(KB, D);
  const __half* kscale = reinterpret_cast<const __half*>(vblk + code_block_bytes(VB, D));
  const __half* kzero = kscale + kPageTokens;
  const __half* vscale = kzero + kPageTokens;
  const __half* vzero = vscale + kPageTokens;
  float* kst = wscr;                   // [32] key scales x 2^24 (/ sigmaK on tokens with bit 3 set)
  float* kzt = wscr + kPageTokens;     // [32] key zeros
  float* svf = wscr + 4 * C::KSROW;    // [32] value scales, tauV folded
  float* zvf = svf + kPageTokens;      // [32] value zeros
  kst[lane] = __half2float(kscale[lane]) * ((lane & 8) ? kTwo24 / C::sigmaK : kTwo24);
  kzt[lane] = __half2float(kzero[lane]);
  const float vs = __half2float(vscale[lane]);
  svf[lane] = (C::tauV != 1.f && (lane & 8)) ? vs * (1.f / C::tauV) : vs;
  zvf[lane] = __half2float(vzero[lane]);
  const float tau = __any_sync(0xffffffffu, vs > kScaleCapLazy) ? 0.f : kTau;
  __syncwarp();

  float s4[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) s4[j][k] = 0.f;
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<KB>::N];
    load_tile_words<KB>(page, lane, dt, w);
    const uint4 a = *reinterpret_cast<const uint4*>(qz + (dt * 32 + lane) * 4);
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      uint32_t b[4];
      tile_frags<KB>(w, tt, b);
      mma_f16(s4[2 * tt], a.x, a.y, a.z, a.w, b[0], b[1]);
      mma_f16(s4[2 * tt + 1], a.x, a.y, a.z, a.w, b[2], b[3]);
    }
  }
  float sc[8];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const int tok = 8 * j + 2 * t + jj;
      sc[2 * j + jj] = fmaf(s4[j][jj] + s4[j][jj + 2], kst[tok], kzt[tok] * qsum);
    }
  softmax_update<D>(st, sc, tau);

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
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<VB>::N];
    load_tile_words<VB>(vblk, lane, dt, w);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t b[4];
      tile_frags<VB>(w, ks, b);
      mma_f16(st.o[2 * dt], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[0], b[1]);
      mma_f16(st.o[2 * dt + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[2], b[3]);
    }
  }
}

// fp8 page, head rows: A = the segment's q' hi/lo fragments with the KV head's
// key scale folded in, B = e4m3 keys as f16 (times 2^-8, undone on the scores);
// p hi/lo against e4m3 values (the value scale and 2^8 are applied once, to
// the accumulators).
template <int D>
__device__ __forceinline__ void attend_f8page(const uint8_t* page, WarpState<D>& st, const uint32_t* qz, int lane) {
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
    const uint4 a = *reinterpret_cast<const uint4*>(qz + (dt * 32 + lane) * 4);
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
  softmax_update<D>(st, sc, kTau);
  uint32_t pa[2][4];
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    split_f16(sc[4 * ks + 0], sc[4 * ks + 1], pa[ks][0], pa[ks][1]);
    split_f16(sc[4 * ks + 2], sc[4 * ks + 3], pa[ks][2], pa[ks][3]);
  }
  const uint8_t* vblk = page + code_block_bytes(8, D);
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    uint32_t w[TileWords<8>::N];
    load_tile_words<8>(vblk, lane, dt, w);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t b[4];
      tile_frags_f8(w, ks, b);
      mma_f16(st.o[2 * dt], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[0], b[1]);
      mma_f16(st.o[2 * dt + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[2], b[3]);
    }
  }
}

// One full bf16 page: raw bf16 values, q unscaled (exact in bf16), p hi/lo.
template <int D>
__device__ __forceinline__ void attend_bpage(const uint8_t* page, WarpState<D>& st,
                                             const uint32_t (&qb)[D / 8], float scale_log2, int lane) {
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
  softmax_update<D>(st, sc, kTau);
  uint32_t pa[2][4];
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    split_bf16(sc[4 * ks + 0], sc[4 * ks + 1], pa[ks][0], pa[ks][1]);
    split_bf16(sc[4 * ks + 2], sc[4 * ks + 3], pa[ks][2], pa[ks][3]);
  }
  const uint8_t* vblk = page + code_block_bytes(16, D);
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    uint32_t w[TileWords<16>::N];
    load_tile_words<16>(vblk, lane, dt, w);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t b[4];
      tile_frags<16>(w, ks, b);
      mma_bf16(st.o[2 * dt], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[0], b[1]);
      mma_bf16(st.o[2 * dt + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b[2], b[3]);
    }
  }
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
  softmax_update<D>(st, sc, kTau);
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

// Raw bf16 pairs of q for lane (g, t): channels 16dt + 2t (+1) and 16dt + 2t + 8 (+9).
template <int D>
__device__ __forceinline__ void load_qb(const __nv_bfloat16* qrow, bool valid, int t, uint32_t (&qb)[D / 8]) {
#pragma unroll
  for (int dt = 0; dt < D / 16; ++dt) {
    qb[2 * dt] = valid ? *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t) : 0u;
    qb[2 * dt + 1] = valid ? *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t + 8) : 0u;
  }
}

// ============================================================================
// Token-row formulation (G <= 4): MMA rows are tokens (QK) and channels (PV);
// the 8 columns are (head c/2, part c%2) with part 0 = high f16 half and part 1
// = low half of q' (QK) or p' (PV). Lane (g, t) keeps head t's scores for
// tokens g, g+8, g+16, g+24 and head t's output for channels g, g+8 of every
// 16-channel tile. 16 QK + 16 PV + 8 z-term MMAs per page.
template <int D>
struct TokState {
  float o[D / 16][4];  // [channel tile]: c0/c1 = head t parts at channel g, c2/c3 at channel g+8
  float m, l, vz;      // head t: reference max, partial sum over this lane's tokens, sum p*z
};

template <int D>
__device__ __forceinline__ void tok_rescale_update(TokState<D>& st, float (&sc)[4], float tau) {
  float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
  if (mx > st.m + tau) {
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

// hi (part 0) or lo (part 1) f16 halves of (x0, x1) as one register.
__device__ __forceinline__ uint32_t part_f16(float x0, float x1, float partf) {
  __half2 h = __floats2half2_rn(x0, x1);
  float2 f = __half22float2(h);
  return h2_bits(__floats2half2_rn(fmaf(-partf, f.x, x0), fmaf(-partf, f.y, x1)));
}

__device__ __forceinline__ uint32_t part_bf16(float x0, float x1, float partf) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  float2 f = __bfloat1622float2(h);
  return b2_bits(__floats2bfloat162_rn(fmaf(-partf, f.x, x0), fmaf(-partf, f.y, x1)));
}

// Transpose p' (this lane: head t, tokens g + 8i) into the PV B fragments
// (this lane: column g = (head g/2, part g%2), tokens 2t, 2t+1, 2t+8, 2t+9 of
// each 16-token k-step). `ptr` is a per-warp [4][40] float tile.
template <bool BF16>
__device__ __forceinline__ void tok_pfrags(float* ptr, const float (&pv)[4], int lane, float partf,
                                           uint32_t (&b)[2][2]) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) ptr[t * 40 + g + 8 * i] = pv[i];
  __syncwarp();
  const float* row = ptr + (g >> 1) * 40 + 2 * t;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    const float2 lo = *reinterpret_cast<const float2*>(row + 16 * ks);
    const float2 hi = *reinterpret_cast<const float2*>(row + 16 * ks + 8);
    if constexpr (BF16) {
      b[ks][0] = part_bf16(lo.x, lo.y, partf);
      b[ks][1] = part_bf16(hi.x, hi.y, partf);
    } else {
      b[ks][0] = part_f16(lo.x, lo.y, partf);
      b[ks][1] = part_f16(hi.x, hi.y, partf);
    }
  }
  __syncwarp();
}

template <int KB, int VB, int D>
__device__ __forceinline__ void attend_qpage_tok(const uint8_t* page, TokState<D>& st, const float (&qf)[D / 4],
                                                 const uint32_t (&qzb)[D / 8], float* wscr, float partf,
                                                 int lane) {
  using C = Cfg<KB, VB, D>;
  const int g = lane >> 2, t = lane & 3;
  const uint8_t* vblk = page + code_block_bytes(KB, D);
  const __half* kscale = reinterpret_cast<const __half*>(vblk + code_block_bytes(VB, D));
  const __half* kzero = kscale + D;
  const __half* vscale = kzero + D;
  const __half* vzero = vscale + kPageTokens;
  float* ksf = wscr;
  float* svf = wscr + 4 * C::KSROW;
  float* zvf = svf + kPageTokens;
  float* ptr = zvf + kPageTokens;  // [4][40]
  {
    constexpr int NE = D / 32;
    const int i0 = lane * NE;
    float* dst = ksf + (i0 / (D / 4)) * C::KSROW + (i0 % (D / 4));
    if constexpr (NE == 4) {
      const uint2 raw = *reinterpret_cast<const uint2*>(kscale + i0);
      float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
      float2 c = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
      if (C::tauK != 1.f) { c.x *= 1.f / C::tauK; c.y *= 1.f / C::tauK; }
      *reinterpret_cast<float4*>(dst) = make_float4(a.x, a.y, c.x, c.y);
    } else {
      const uint32_t raw = *reinterpret_cast<const uint32_t*>(kscale + i0);
      float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw));
      if (C::tauK != 1.f && (i0 & 2)) { a.x *= 1.f / C::tauK; a.y *= 1.f / C::tauK; }
      *reinterpret_cast<float2*>(dst) = a;
    }
  }
  const float vs = __half2float(vscale[lane]);
  svf[lane] = (C::tauV != 1.f && (lane & 8)) ? vs * (1.f / C::tauV) : vs;
  zvf[lane] = __half2float(vzero[lane]);
  const float tau = __any_sync(0xffffffffu, vs > kScaleCapLazy) ? 0.f : kTau;
  __syncwarp();

  // --- QK: two token m-tiles, B = q' parts; z-term: A = z rows, B = q parts
  float s2[2][4], cz[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int k = 0; k < 4; ++k) s2[mt][k] = 0.f;
  const float* ksl = ksf + t * C::KSROW;
  const uint32_t* zrow = reinterpret_cast<const uint32_t*>(kzero + t * (D / 4));
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<KB>::N];
    load_tile_words<KB>(page, lane, dt, w);
    const float4 sc4 = *reinterpret_cast<const float4*>(ksl + dt * 4);
    const uint32_t b0 = part_f16(qf[dt * 4 + 0] * sc4.x, qf[dt * 4 + 1] * sc4.y, partf);
    const uint32_t b1 = part_f16(qf[dt * 4 + 2] * sc4.z, qf[dt * 4 + 3] * sc4.w, partf);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      uint32_t a[4];
      tile_afrag<KB>(w, mt, a);
      mma_f16(s2[mt], a[0], a[1], a[2], a[3], b0, b1);
    }
    const uint2 z = *reinterpret_cast<const uint2*>(zrow + dt * 2);
    mma_f16(cz, z.x, z.x, z.y, z.y, qzb[2 * dt], qzb[2 * dt + 1]);
  }
  const float czv = cz[0] + cz[1];  // head t: both parts of sum_c q_c z_c
  float sc[4];
  sc[0] = fmaf(s2[0][0] + s2[0][1], kTwo24, czv);
  sc[1] = fmaf(s2[0][2] + s2[0][3], kTwo24 / C::sigmaK, czv);
  sc[2] = fmaf(s2[1][0] + s2[1][1], kTwo24, czv);
  sc[3] = fmaf(s2[1][2] + s2[1][3], kTwo24 / C::sigmaK, czv);
  tok_rescale_update<D>(st, sc, tau);

  // --- p' = p * s_t for tokens g + 8i; value zero term; transpose to B fragments
  float pv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    pv[i] = sc[i] * svf[g + 8 * i];
    st.vz = fmaf(sc[i], zvf[g + 8 * i], st.vz);
  }
  uint32_t pb[2][2];
  tok_pfrags<false>(ptr, pv, lane, partf, pb);

  // --- PV: A = value codes (rows = channels), B = p' parts
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<VB>::N];
    load_tile_words<VB>(vblk, lane, dt, w);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t a[4];
      tile_afrag<VB>(w, ks, a);
      mma_f16(st.o[dt], a[0], a[1], a[2], a[3], pb[ks][0], pb[ks][1]);
    }
  }
}

// Per-token keys, token rows: B = the segment's q' parts (tauK folded, fixed per
// segment); score of token g + 8i for head t = s * acc + z * sum_c q'_c.
template <int KB, int VB, int D>
__device__ __forceinline__ void attend_qpage_tok_pt(const uint8_t* page, TokState<D>& st,
                                                    const uint32_t (&qkb)[D / 8], float qsum, float* wscr,
                                                    float partf, int lane) {
  using C = Cfg<KB, VB, D, true>;
  const int g = lane >> 2;
  const uint8_t* vblk = page + code_block_bytes(KB, D);
  const __half* kscale = reinterpret_cast<const __half*>(vblk + code_block_bytes(VB, D));
  const __half* kzero = kscale + kPageTokens;
  const __half* vscale = kzero + kPageTokens;
  const __half* vzero = vscale + kPageTokens;
  float* kst = wscr;
  float* kzt = wscr + kPageTokens;
  float* svf = wscr + 4 * C::KSROW;
  float* zvf = svf + kPageTokens;
  float* ptr = zvf + kPageTokens;  // [4][40]
  kst[lane] = __half2float(kscale[lane]) * ((lane & 8) ? kTwo24 / C::sigmaK : kTwo24);
  kzt[lane] = __half2float(kzero[lane]);
  const float vs = __half2float(vscale[lane]);
  svf[lane] = (C::tauV != 1.f && (lane & 8)) ? vs * (1.f / C::tauV) : vs;
  zvf[lane] = __half2float(vzero[lane]);
  const float tau = __any_sync(0xffffffffu, vs > kScaleCapLazy) ? 0.f : kTau;
  __syncwarp();

  float s2[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int k = 0; k < 4; ++k) s2[mt][k] = 0.f;
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<KB>::N];
    load_tile_words<KB>(page, lane, dt, w);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      uint32_t a[4];
      tile_afrag<KB>(w, mt, a);
      mma_f16(s2[mt], a[0], a[1], a[2], a[3], qkb[2 * dt], qkb[2 * dt + 1]);
    }
  }
  float sc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int tok = g + 8 * i;
    const float acc = s2[i >> 1][2 * (i & 1)] + s2[i >> 1][2 * (i & 1) + 1];
    sc[i] = fmaf(acc, kst[tok], kzt[tok] * qsum);
  }
  tok_rescale_update<D>(st, sc, tau);

  float pv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    pv[i] = sc[i] * svf[g + 8 * i];
    st.vz = fmaf(sc[i], zvf[g + 8 * i], st.vz);
  }
  uint32_t pb[2][2];
  tok_pfrags<false>(ptr, pv, lane, partf, pb);
#pragma unroll
  for (int dt = 0; dt < C::KS; ++dt) {
    uint32_t w[TileWords<VB>::N];
    load_tile_words<VB>(vblk, lane, dt, w);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t a[4];
      tile_afrag<VB>(w, ks, a);
      mma_f16(st.o[dt], a[0], a[1], a[2], a[3], pb[ks][0], pb[ks][1]);
    }
  }
}

// fp8 page, token rows: A = e4m3 keys/values as f16, B = the segment's q' parts
// (key scale folded in) or p parts.
template <int D>
__device__ __forceinline__ void attend_f8page_tok(const uint8_t* page, TokState<D>& st, const uint32_t (&qkb)[D / 8],
                                                  float* wscr, float partf, int lane) {
  constexpr int KS = D / 16;
  float* ptr = wscr + 4 * (D / 4 + 4) + 2 * kPageTokens;
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
      mma_f16(s2[mt], a[0], a[1], a[2], a[3], qkb[2 * dt], qkb[2 * dt + 1]);
    }
  }
  float sc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) sc[i] = (s2[i >> 1][2 * (i & 1)] + s2[i >> 1][2 * (i & 1) + 1]) * kF8Unit;
  tok_rescale_update<D>(st, sc, kTau);
  uint32_t pb[2][2];
  tok_pfrags<false>(ptr, sc, lane, partf, pb);
  const uint8_t* vblk = page + code_block_bytes(8, D);
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    uint32_t w[TileWords<8>::N];
    load_tile_words<8>(vblk, lane, dt, w);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t a[4];
      tile_afrag_f8(w, ks, a);
      mma_f16(st.o[dt], a[0], a[1], a[2], a[3], pb[ks][0], pb[ks][1]);
    }
  }
}

template <int D>
__device__ __forceinline__ void attend_bpage_tok(const uint8_t* page, TokState<D>& st, const uint32_t (&qbp)[D / 8],
                                                 float* wscr, float partf, float scale_log2, int lane) {
  constexpr int KS = D / 16;
  float* ptr = wscr + 4 * (D / 4 + 4) + 2 * kPageTokens;
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
  tok_rescale_update<D>(st, sc, kTau);
  uint32_t pb[2][2];
  tok_pfrags<true>(ptr, sc, lane, partf, pb);
  const uint8_t* vblk = page + code_block_bytes(16, D);
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    uint32_t w[TileWords<16>::N];
    load_tile_words<16>(vblk, lane, dt, w);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t a[4];
      tile_afrag<16>(w, ks, a);
      mma_bf16(st.o[dt], a[0], a[1], a[2], a[3], pb[ks][0], pb[ks][1]);
    }
  }
}

// bf16 window (natural [32][D] rows in global memory), W < 32 valid tokens.
template <int D>
__device__ __forceinline__ void attend_window_tok(const __nv_bfloat16* win, int W, TokState<D>& st,
                                                  const uint32_t (&qbp)[D / 8], float* wscr, float partf,
                                                  float scale_log2, int lane) {
  constexpr int KS = D / 16;
  const int g = lane >> 2, t = lane & 3;
  float* ptr = wscr + 4 * (D / 4 + 4) + 2 * kPageTokens;
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
  tok_rescale_update<D>(st, sc, kTau);
  uint32_t pb[2][2];
  tok_pfrags<true>(ptr, sc, lane, partf, pb);
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    if (16 * ks >= W) continue;  // warp-uniform
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      const int tk = 16 * ks + 2 * t, ch = 16 * dt + g;
      mma_bf16(st.o[dt], vpair(tk, ch), vpair(tk, ch + 8), vpair(tk + 8, ch), vpair(tk + 8, ch + 8), pb[ks][0],
               pb[ks][1]);
    }
  }
}

// ------------------------------------------------------------------ kernel --
// Units: per (sequence b, KV head h) segment, V "overhead" units (no work:
// they stand for the fixed cost of starting and merging a segment part, so a
// CTA that spans several segments gets fewer pages), then the pages in order,
// then one window unit when T mod 32 > 0 (or one empty unit when T = 0).
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

// Walks the page units of one warp in the order the warp consumes them:
// within each segment part [a, e) of the CTA slice, units a + warp + 4j.
struct PageCursor {
  int u, e;          // candidate unit, end of the current segment part
  int first, P;      // current segment's first page unit and page count
  const uint8_t* base;  // pages of the current (b, h)
};

template <int D>
__device__ __forceinline__ bool cursor_next(PageCursor& c, const DecodeParams& p, const int* ustart, int B, int u1,
                                            int warp) {
  for (;;) {
    if (c.u < c.e) {
      const int k = c.u - c.first;
      if (k >= 0 && k < c.P) return true;
      c.u += kWarps;  // overhead units lead a segment, the window / empty unit ends it
      continue;
    }
    if (c.e >= u1) return false;
    const int a = c.e;
    const Seg sg = seg_of(ustart, B, p.n_kv_heads, a);
    c.first = sg.start + p.seg_overhead;
    c.e = min(sg.start + sg.n, u1);
    c.P = p.len[sg.b] / kPageTokens;
    c.base = p.pages + ((int64_t)(sg.b * p.n_kv_heads + sg.h) * p.max_pages) * p.page_bytes;
    c.u = a + warp;
  }
}

template <int KB, int VB, int D, bool TOK, bool PT, bool F8>
__global__ void __launch_bounds__(kThreads, TOK ? Cfg<KB, VB, D, PT, F8>::MINB_TOK : Cfg<KB, VB, D, PT, F8>::MINB)
    decode_mma_kernel(DecodeParams p) {
  pdl_enter();
  using C = Cfg<KB, VB, D, PT, F8>;
  using State = typename std::conditional<TOK, TokState<D>, WarpState<D>>::type;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_last;
  const int H = p.n_kv_heads, G = p.gqa, B = p.batch;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  // this lane's query head: row g (head rows) or column head g/2 (token rows)
  const int qh = TOK ? (g >> 1) : g;
  const float partf = (float)(g & 1);

  uint8_t* ring = smem + warp * C::R * C::STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::MBAR_OFF) + warp * C::R;
  float* wscr = reinterpret_cast<float*>(smem + C::WSCR_OFF + warp * C::WSCR_STRIDE);
  uint32_t* qz = reinterpret_cast<uint32_t*>(smem + C::QZ_OFF);
  float* mo = reinterpret_cast<float*>(smem + C::merge_off(TOK));   // [kWarps][G][D]
  float* mm = mo + kWarps * G * D;                                   // [kWarps][8]
  float* ml = mm + kWarps * kMaxGqa;                                 // [kWarps][8]
  int* ustart = reinterpret_cast<int*>(ml + kWarps * kMaxGqa);       // [B + 1]
  __nv_bfloat16* qbuf = reinterpret_cast<__nv_bfloat16*>(smem + C::qbuf_off(TOK));  // [2][8][D]
  uint64_t* qbars = reinterpret_cast<uint64_t*>(smem + C::MBAR_OFF) + kWarps * C::R;

  // ---- units per sequence: exclusive scan (warp 0), n_b = H * max(1, P + (W > 0))
  if (warp == 0) {
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int bb = b0 + lane;
      int n = 0;
      if (bb < B) {
        const int T = p.len[bb];
        n = T / kPageTokens + (T % kPageTokens > 0 ? 1 : 0);
        n = ((n > 0 ? n : 1) + p.seg_overhead) * H;
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
  if (lane == 0) {
    for (int r = 0; r < C::R; ++r) mbar_init(&bars[r], 1);
    if (warp == 0) {
      mbar_init(&qbars[0], 1);
      mbar_init(&qbars[1], 1);
    }
    mbar_init_fence();
  }
  __syncthreads();
  const int N = ustart[B];
  const Slicer sl{N / (int)gridDim.x, N % (int)gridDim.x};
  const int u0 = sl.lo(blockIdx.x), u1 = sl.lo(blockIdx.x + 1);
  if (u0 >= u1) return;
  {
    // nothing to do when the whole slice lies in one segment's overhead units
    const Seg s0 = seg_of(ustart, B, H, u0);
    if (u1 <= s0.start + p.seg_overhead) return;
  }

  // ---- query rows arrive by bulk copy (the first one ahead of the page stream)
  const uint32_t qbytes = (uint32_t)(G * D * 2);
  auto issue_q = [&](int unit, int buf) {
    const Seg qs = seg_of(ustart, B, H, unit);
    mbar_expect_tx(&qbars[buf], qbytes);
    bulk_load(qbuf + buf * kMaxGqa * D, p.Q + (int64_t)(qs.b * H + qs.h) * G * D, qbytes, &qbars[buf]);
  };
  if (threadIdx.x == 0) issue_q(u0, 0);

  // ---- producer: the first R page units of this warp
  PageCursor cur;
  cur.u = u0;  // >= e: the first call looks up the segment of u0
  cur.e = u0;
  cur.first = 0;
  cur.P = 0;
  cur.base = nullptr;
  int issued = 0;
  const uint64_t pol = l2_evict_first_policy();
  if (lane == 0) {
    for (int r = 0; r < C::R; ++r) {
      if (!cursor_next<D>(cur, p, ustart, B, u1, warp)) break;
      mbar_expect_tx(&bars[r], C::PB);
      bulk_load_once(ring + r * C::STAGE, cur.base + (int64_t)(cur.u - cur.first) * p.page_bytes, C::PB, &bars[r],
                     pol);
      cur.u += kWarps;
      ++issued;
    }
  }

  bool ok = true;
  int consumed = 0;
  int segi = 0;
  for (int a = u0; a < u1; ++segi) {
    const Seg sg = seg_of(ustart, B, H, a);
    const int e = min(sg.start + sg.n, u1);
    if (e <= sg.start + p.seg_overhead) break;  // overhead units only (the slice's last part)
    const int T = p.len[sg.b];
    const int P = T / kPageTokens, W = T % kPageTokens;
    if (threadIdx.x == 0 && W > 0 && e == sg.start + sg.n) {
      // this part ends with the bf16 window: bring its W key and W value rows into L2
      const __nv_bfloat16* w0 = p.window + ((int64_t)(sg.b * H + sg.h) * 2) * kPageTokens * D;
      prefetch_l2(w0, (uint32_t)(W * D * 2));
      prefetch_l2(w0 + kPageTokens * D, (uint32_t)(W * D * 2));
    }
    const bool qvalid = qh < G;
    {
      const bool got = mbar_wait(&qbars[segi & 1], (uint32_t)((segi >> 1) & 1));
      if (!__all_sync(0xffffffffu, got)) ok = false;
      // prefetch the next segment's query row (unless that part is overhead units only)
      if (threadIdx.x == 0 && e < u1 && u1 > e + p.seg_overhead) issue_q(e, (segi + 1) & 1);
    }
    const __nv_bfloat16* qrow = qbuf + (segi & 1) * kMaxGqa * D + (qvalid ? qh : 0) * D;

    // ---- query operands
    float qf[D / 4];
    uint32_t qb[D / 8];   // bf16 pairs (head rows) or bf16 parts (token rows)
    uint32_t qzb[D / 8];  // token rows: z-term B fragments (q parts); QK B fragments with per-token keys
    float qsum = 0.f;     // per-token keys: sum_c q'_c of the head this lane scores
    auto load_qbp = [&]() {
#pragma unroll
      for (int dt = 0; dt < C::KS; ++dt) {
        uint32_t lo = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t);
        uint32_t hi = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t + 8);
        const bool keep = qvalid && (!TOK || (g & 1) == 0);  // q is exact in bf16: low part is zero
        qb[2 * dt] = keep ? lo : 0u;
        qb[2 * dt + 1] = keep ? hi : 0u;
      }
    };
    if constexpr (C::kBf16) {
      load_qbp();
    } else {
#pragma unroll
      for (int dt = 0; dt < C::KS; ++dt) {
        uint32_t lo = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t);
        uint32_t hi = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t + 8);
        if (!qvalid) lo = hi = 0u;
        const float2 l2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&lo));
        const float2 h2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&hi));
        qf[dt * 4 + 0] = l2.x * p.scale_log2;
        qf[dt * 4 + 1] = l2.y * p.scale_log2;
        qf[dt * 4 + 2] = h2.x * p.scale_log2;
        qf[dt * 4 + 3] = h2.y * p.scale_log2;
      }
      // q parts: the z-term B/A operands (per-channel keys) or the QK operands
      // themselves (per-token keys: the 2-bit tauK channel factor is folded
      // here; fp8: the KV head's key scale is)
      const float qlo = F8 ? p.fp8_scales[sg.h] : 1.f;
      const float qhi = PT ? 1.f / C::tauK : qlo;  // channels 2t+8, 2t+9 of each tile
      if constexpr (TOK) {
#pragma unroll
        for (int dt = 0; dt < C::KS; ++dt) {
          qzb[2 * dt] = part_f16(qf[dt * 4 + 0] * qlo, qf[dt * 4 + 1] * qlo, partf);
          qzb[2 * dt + 1] = part_f16(qf[dt * 4 + 2] * qhi, qf[dt * 4 + 3] * qhi, partf);
        }
      } else {
        if (warp == 0) {
#pragma unroll
          for (int dt = 0; dt < C::KS; ++dt) {
            uint4 q4;
            split_f16(qf[dt * 4 + 0] * qlo, qf[dt * 4 + 1] * qlo, q4.x, q4.y);
            split_f16(qf[dt * 4 + 2] * qhi, qf[dt * 4 + 3] * qhi, q4.z, q4.w);
            *reinterpret_cast<uint4*>(qz + (dt * 32 + lane) * 4) = q4;
          }
        }
        __syncthreads();
      }
      if constexpr (PT) {
        // sum_c q'_c of this lane's query head (its D/4 channels, then the quad)
        float qs = 0.f;
#pragma unroll
        for (int i = 0; i < D / 4; ++i) qs += qf[i];
        qs += __shfl_xor_sync(0xffffffffu, qs, 1);
        qs += __shfl_xor_sync(0xffffffffu, qs, 2);
        // token rows score head t (held by lanes with g = 2t); head rows score head g
        qsum = TOK ? __shfl_sync(0xffffffffu, qs, 8 * t) : qs;
      }
    }

    State st;
#pragma unroll
    for (int j = 0; j < (TOK ? D / 16 : D / 8); ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) st.o[j][k] = 0.f;
    st.m = -INFINITY;
    st.l = 0.f;
    st.vz = 0.f;
    bool converted = C::kBf16;
    // quantized accumulators to true units: acc * 2^24 (/ sigmaV on channels with
    // bit 3 set); fp8: acc * the KV head's value scale
    auto to_true_units = [&]() {
      if constexpr (F8) {
        const float vsc = p.fp8_scales[H + sg.h] * kF8Unit;
#pragma unroll
        for (int j = 0; j < (TOK ? D / 16 : D / 8); ++j)
#pragma unroll
          for (int k = 0; k < 4; ++k) st.o[j][k] *= vsc;
      } else if constexpr (TOK) {
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          st.o[j][0] *= kTwo24;
          st.o[j][1] *= kTwo24;
          st.o[j][2] *= kTwo24 / C::sigmaV;
          st.o[j][3] *= kTwo24 / C::sigmaV;
        }
      } else {
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          const float f = (j & 1) ? kTwo24 / C::sigmaV : kTwo24;
#pragma unroll
          for (int k = 0; k < 4; ++k) st.o[j][k] *= f;
        }
      }
      converted = true;
    };

    // ---- this warp's units of the segment part [a, e)
    for (int u = a + warp; u < e; u += kWarps) {
      const int k = u - sg.start - p.seg_overhead;
      if (k < 0) continue;  // overhead unit: no work
      if (k < P) {
        if (ok) {
          const int stage = consumed % C::R;
          const bool arrived = mbar_wait(&bars[stage], (uint32_t)((consumed / C::R) & 1));
          if (!__all_sync(0xffffffffu, arrived)) {  // warp-uniform verdict
            ok = false;
          } else {
            const uint8_t* page = ring + stage * C::STAGE;
            if constexpr (TOK) {
              if constexpr (C::kBf16) attend_bpage_tok<D>(page, st, qb, wscr, partf, p.scale_log2, lane);
              else if constexpr (F8) attend_f8page_tok<D>(page, st, qzb, wscr, partf, lane);
              else if constexpr (PT) attend_qpage_tok_pt<KB, VB, D>(page, st, qzb, qsum, wscr, partf, lane);
              else attend_qpage_tok<KB, VB, D>(page, st, qf, qzb, wscr, partf, lane);
            } else {
              if constexpr (C::kBf16) attend_bpage<D>(page, st, qb, p.scale_log2, lane);
              else if constexpr (F8) attend_f8page<D>(page, st, qz, lane);
              else if constexpr (PT) attend_qpage_pt<KB, VB, D>(page, st, qz, qsum, wscr, lane);
              else attend_qpage<KB, VB, D>(page, st, qf, qz, wscr, lane);
            }
            ++consumed;
            __syncwarp();
            if (lane == 0 && cursor_next<D>(cur, p, ustart, B, u1, warp)) {
              fence_proxy_async();
              mbar_expect_tx(&bars[stage], C::PB);
              bulk_load_once(ring + stage * C::STAGE, cur.base + (int64_t)(cur.u - cur.first) * p.page_bytes,
                             C::PB, &bars[stage], pol);
              cur.u += kWarps;
              ++issued;
            }
          }
        }
      } else if (W > 0) {
        if constexpr (!C::kBf16) {
          to_true_units();
          load_qbp();
        }
        const __nv_bfloat16* win = p.window + ((int64_t)(sg.b * H + sg.h) * 2) * kPageTokens * D;
        if constexpr (TOK) attend_window_tok<D>(win, W, st, qb, wscr, partf, p.scale_log2, lane);
        else attend_window<D>(win, W, st, qb, p.scale_log2, lane);
      }
    }
    if (!converted) to_true_units();

    // ---- warps -> shared memory, CTA merge
    if constexpr (TOK) {
      float l = st.l, vz = st.vz;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, o);
        vz += __shfl_xor_sync(0xffffffffu, vz, o);
      }
      if (t < G) {
        float* dst = mo + (warp * G + t) * D;
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          dst[16 * j + g] = st.o[j][0] + st.o[j][1] + vz;
          dst[16 * j + 8 + g] = st.o[j][2] + st.o[j][3] + vz;
        }
        if (g == 0) {
          mm[warp * kMaxGqa + t] = st.m;
          ml[warp * kMaxGqa + t] = l;
        }
      }
    } else {
      float l = st.l + __shfl_xor_sync(0xffffffffu, st.l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      float vz = st.vz + __shfl_xor_sync(0xffffffffu, st.vz, 1);
      vz += __shfl_xor_sync(0xffffffffu, vz, 2);
      if (g < G) {
        float* dst = mo + (warp * G + g) * D;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          dst[8 * j + 2 * t] = st.o[j][0] + st.o[j][2] + vz;
          dst[8 * j + 2 * t + 1] = st.o[j][1] + st.o[j][3] + vz;
        }
        if (t == 0) {
          mm[warp * kMaxGqa + g] = st.m;
          ml[warp * kMaxGqa + g] = l;
        }
      }
    }
    __syncthreads();
    const int seg = sg.b * H + sg.h;
    const bool whole = (a <= sg.start + p.seg_overhead) && (e == sg.start + sg.n);
    float* outp = p.out + (int64_t)seg * G * D;
    float* part = p.partials + ((int64_t)blockIdx.x * 2 + (a == u0 ? 0 : 1)) * split_record_floats(G, D);
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
      const int gg = idx / D, d = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mm[w * kMaxGqa + gg]);
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
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
      const int c_lo = sl.cta_of(sg.start + p.seg_overhead), c_hi = sl.cta_of(sg.start + sg.n - 1);
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
        // one pass over the records, online rescaling, four channels per thread
        for (int i4 = threadIdx.x; i4 < G * D / 4; i4 += kThreads) {
          const int gg = (4 * i4) / D, d = (4 * i4) % D;
          float M = -INFINITY, L = 0.f;
          float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
          for (int c = c_lo; c <= c_hi; ++c) {
            if (sl.empty(c)) continue;
            const int slot = (sl.lo(c) >= sg.start) ? 0 : 1;
            const float* r = p.partials + ((int64_t)c * 2 + slot) * split_record_floats(G, D);
            const float mc = __ldcg(r + G * D + gg), lc = __ldcg(r + G * D + G + gg);
            const float4 oc = __ldcg(reinterpret_cast<const float4*>(r + gg * D + d));
            const float Mn = fmaxf(M, mc);
            const float fa = (M == -INFINITY) ? 0.f : exp2f(M - Mn);
            const float fb = (mc == -INFINITY) ? 0.f : exp2f(mc - Mn);
            L = L * fa + lc * fb;
            O.x = O.x * fa + oc.x * fb;
            O.y = O.y * fa + oc.y * fb;
            O.z = O.z * fa + oc.z * fb;
            O.w = O.w * fa + oc.w * fb;
            M = Mn;
          }
          const float inv = L > 0.f ? 1.f / L : 0.f;
          *reinterpret_cast<float4*>(outp + gg * D + d) = make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
        }
      }
    }
    __syncthreads();  // merge area, qz and s_last are reused by the next segment
    a = e;
  }

  if (!ok) {
    // a copy never completed: report it, then let the copies in flight land
    // (each wait bounded again) before this CTA's shared memory goes away
    if (lane == 0 && p.err) atomicExch(p.err, 1);
    for (int i = consumed; i < issued; ++i) mbar_wait(&bars[i % C::R], (uint32_t)((i / C::R) & 1));
  }
}

// ------------------------------------------------------------ fused append --
// Warp-level flush of one completed 32-token group (the window's 31 tokens and
// the new token) into `page`, bit-identical to the append kernel's CTA-wide
// flush: the same quantizer and packing (kvq_quant.cuh), only the work split
// differs. `scr` is this warp's ring (free at a segment's start) and holds the
// codes as bytes, [2][32][D] (bf16 layers: the rows themselves), before they
// are packed in fragment order.
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
                                        const __nv_bfloat16* vn, uint8_t* scr, float ksc, float vsc,
                                        double* err_stats, int lane) {
  // row of token tok (0..31) of keys (r = 0) or values (r = 1)
  auto row = [&](int r, int tok) -> const __nv_bfloat16* {
    return tok < kPageTokens - 1 ? win + (r * kPageTokens + tok) * D : (r ? vn : kn);
  };
  if constexpr (KB == 16) {
    // bf16 layer: stage the 32 rows of keys and values, then pack their bit patterns
    uint16_t* sb = reinterpret_cast<uint16_t*>(scr);  // [2][32][D]
#pragma unroll 1
    for (int i = lane; i < 2 * kPageTokens * D / 8; i += 32) {
      const int r = i / (kPageTokens * D / 8), rem = i % (kPageTokens * D / 8);
      const int tok = rem / (D / 8), c8 = (rem % (D / 8)) * 8;
      *reinterpret_cast<uint4*>(sb + (r * kPageTokens + tok) * D + c8) =
          *reinterpret_cast<const uint4*>(row(r, tok) + c8);
    }
    __syncwarp();
    pack_block_warp<16, D>(page, false, lane, [&](int tok, int dim) { return (uint32_t)sb[tok * D + dim]; });
    pack_block_warp<16, D>(page + code_block_bytes(16, D), true, lane,
                           [&](int tok, int dim) { return (uint32_t)sb[(kPageTokens + tok) * D + dim]; });
    return;
  } else {
    uint8_t* cs = scr;  // [2][32][D] codes
    double err[4] = {0.0, 0.0, 0.0, 0.0};
    auto add_err = [&](int r, float x, double xh) {
      const double dx = (double)x - xh;
      err[2 * r] += dx * dx;
      err[2 * r + 1] += (double)x * (double)x;
    };
    if constexpr (F8) {
      // lane = token: every element is e4m3(x / s_h) of its KV head's scale
#pragma unroll 1
      for (int r = 0; r < 2; ++r) {
        const float sc = r ? vsc : ksc;
        const __nv_bfloat16* src = row(r, lane);
#pragma unroll 1
        for (int c8 = 0; c8 < D; c8 += 8) {
          const uint4 raw = *reinterpret_cast<const uint4*>(src + c8);
          const __nv_bfloat16* xv = reinterpret_cast<const __nv_bfloat16*>(&raw);
          uint32_t packed[2] = {0u, 0u};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float x = __bfloat162float(xv[j]);
            const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(__fdiv_rn(x, sc), __NV_SATFINITE, __NV_E4M3);
            packed[j >> 2] |= (uint32_t)c << (8 * (j & 3));
            add_err(r, x, (double)__half2float(__half(__nv_cvt_fp8_to_halfraw(c, __NV_E4M3))) * sc);
          }
          *reinterpret_cast<uint2*>(cs + (r * kPageTokens + lane) * D + c8) = make_uint2(packed[0], packed[1]);
        }
      }
      __syncwarp();
      pack_block_warp<8, D>(page, false, lane, [&](int tok, int dim) { return (uint32_t)cs[tok * D + dim]; });
      pack_block_warp<8, D>(page + code_block_bytes(8, D), true, lane,
                            [&](int tok, int dim) { return (uint32_t)cs[(kPageTokens + tok) * D + dim]; });
    } else {
      constexpr int nk = PT ? kPageTokens : D;  // key scale/zero pairs
      uint8_t* vblk = page + code_block_bytes(KB, D);
      __half* kscale = reinterpret_cast<__half*>(vblk + code_block_bytes(VB, D));
      __half* kzero = kscale + nk;
      __half* vscale = kzero + nk;
      __half* vzero = vscale + kPageTokens;
      // per token over head_dim (values; keys in per-token mode): lane = token
      auto per_token = [&](int r, int qmax, __half* sdst, __half* zdst) {
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
        const double s = (double)__half2float(q.s_h), z = (double)q.z;
#pragma unroll 1
        for (int c8 = 0; c8 < D; c8 += 8) {
          const uint4 raw = *reinterpret_cast<const uint4*>(src + c8);
          const __nv_bfloat16* xv = reinterpret_cast<const __nv_bfloat16*>(&raw);
          uint32_t packed[2] = {0u, 0u};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float x = __bfloat162float(xv[j]);
            const uint32_t c = quant_code(x, q, qmax);
            packed[j >> 2] |= c << (8 * (j & 3));
            add_err(r, x, (double)c * s + z);
          }
          *reinterpret_cast<uint2*>(cs + (r * kPageTokens + lane) * D + c8) = make_uint2(packed[0], packed[1]);
        }
        sdst[lane] = q.s_h;
        zdst[lane] = q.z_h;
      };
      if constexpr (PT) {
        per_token(0, (1 << KB) - 1, kscale, kzero);
      } else {
        // keys per channel over the 32 tokens: lane owns channels lane * NC .. + NC - 1
        constexpr int NC = D / 32;
        constexpr int qmax = (1 << KB) - 1;
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
        QParams q[NC];
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          q[j] = make_qparams(mn[j], mx[j], qmax);
          const int slot = kmeta_slot<D>(c0 + j);
          kscale[slot] = q[j].s_h;
          kzero[slot] = q[j].z_h;
        }
#pragma unroll 1
        for (int tok = 0; tok < kPageTokens; ++tok) {
          const __nv_bfloat16* src = row(0, tok) + c0;
#pragma unroll
          for (int j = 0; j < NC; ++j) {
            const float x = __bfloat162float(src[j]);
            const uint32_t c = quant_code(x, q[j], qmax);
            cs[tok * D + c0 + j] = (uint8_t)c;
            add_err(0, x, (double)c * (double)__half2float(q[j].s_h) + (double)q[j].z);
          }
        }
      }
      per_token(1, (1 << VB) - 1, vscale, vzero);
      __syncwarp();
      pack_block_warp<KB, D>(page, false, lane, [&](int tok, int dim) { return (uint32_t)cs[tok * D + dim]; });
      pack_block_warp<VB, D>(vblk, true, lane,
                             [&](int tok, int dim) { return (uint32_t)cs[(kPageTokens + tok) * D + dim]; });
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
};

// AP (kvq_decode_step): before attending segment (b, h) the warp appends its new
// token -- into the window, or, when it completes a group, quantized into the
// next page, which the warp then attends from global memory -- and the last of
// sequence b's H warps to have read the old length publishes the new one (the
// acquire-release increment orders every read before that write).
template <int KB, int VB, int D, bool PT, bool F8, bool AP = false>
__global__ void __launch_bounds__(kThreads, Cfg<KB, VB, D, PT, F8>::MINB_TOK)
    decode_warp_kernel(DecodeParams p) {
  pdl_enter();
  using C = Cfg<KB, VB, D, PT, F8>;
  using WC = WarpCfg<KB, VB, D, PT, F8>;
  static_assert(C::R * C::STAGE >= 2 * kPageTokens * D * (C::kBf16 ? 2 : 1), "flush scratch fits the warp's ring");
  extern __shared__ __align__(128) uint8_t smem[];
  const int H = p.n_kv_heads, G = p.gqa;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int qh = g >> 1;  // column head of this lane
  const float partf = (float)(g & 1);
  uint8_t* ring = smem + warp * C::R * C::STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + WC::MBAR_OFF) + warp * (C::R + 1);
  uint64_t* qbar = bars + C::R;
  float* wscr = reinterpret_cast<float*>(smem + WC::WSCR_OFF + warp * C::WSCR_STRIDE);
  __nv_bfloat16* qslot = reinterpret_cast<__nv_bfloat16*>(smem + WC::QBUF_OFF + warp * WC::QSLOT);
  if (lane == 0) {
    for (int r = 0; r <= C::R; ++r) mbar_init(&bars[r], 1);
    mbar_init_fence();
  }
  __syncwarp();

  const int S = p.batch * H;
  const int stride = (int)gridDim.x * kWarps;
  const uint32_t qbytes = (uint32_t)(G * D * 2);
  const uint64_t pol = l2_evict_first_policy();
  bool ok = true;
  int issued = 0, consumed = 0, nq = 0;
  for (int s = blockIdx.x * kWarps + warp; s < S && ok; s += stride, ++nq) {
    const int b = s / H, h = s % H;
    int T, P;              // tokens attended; pages read through the ring
    bool flushed = false;  // AP: page P, just written, is attended too
    if constexpr (AP) {
      int t0 = 0;
      if (lane == 0) {
        t0 = p.step_len[b];
        if (atomic_add_acq_rel(&p.append_ctr[b], 1) == H - 1) {
          p.append_ctr[b] = 0;
          if (t0 < p.max_tokens) p.step_len[b] = t0 + 1;
        }
      }
      t0 = __shfl_sync(0xffffffffu, t0, 0);
      P = t0 / kPageTokens;
      if (t0 < p.max_tokens) {
        T = t0 + 1;
        __nv_bfloat16* wwin = p.step_window + ((int64_t)s * 2) * kPageTokens * D;
        const __nv_bfloat16* kn = p.k_new + (int64_t)s * D;
        const __nv_bfloat16* vn = p.v_new + (int64_t)s * D;
        if (T % kPageTokens != 0) {
          // the new token into window slot t0 mod 32
          const int slot = t0 % kPageTokens;
          for (int d = 2 * lane; d < D; d += 64) {
            *reinterpret_cast<uint32_t*>(wwin + slot * D + d) = *reinterpret_cast<const uint32_t*>(kn + d);
            *reinterpret_cast<uint32_t*>(wwin + (kPageTokens + slot) * D + d) =
                *reinterpret_cast<const uint32_t*>(vn + d);
          }
        } else {
          flushed = true;
          warp_flush<KB, VB, D, PT, F8>(p.step_pages + ((int64_t)s * p.max_pages + P) * p.page_bytes, wwin, kn, vn,
                                        ring, F8 ? p.fp8_scales[h] : 1.f, F8 ? p.fp8_scales[H + h] : 1.f,
                                        p.err_stats, lane);
        }
        __syncwarp();  // the window row or page and the ring scratch are complete for every lane
      } else {
        T = t0;  // a full sequence is left unchanged and the cache's error flag raised
        if (lane == 0 && p.err) atomicExch(p.err, 2);
      }
    } else {
      T = p.len[b];
      P = T / kPageTokens;
    }
    const int W = T % kPageTokens;
    const uint8_t* base = p.pages + ((int64_t)s * p.max_pages) * p.page_bytes;
    const __nv_bfloat16* win = p.window + ((int64_t)s * 2) * kPageTokens * D;
    int next = 0;  // next page of this segment to copy
    if (lane == 0) {
      fence_proxy_async();  // the slot's previous rows were read through the generic proxy
      mbar_expect_tx(qbar, qbytes);
      bulk_load(qslot, p.Q + (int64_t)s * G * D, qbytes, qbar);
      for (; next < P && next < C::R; ++next) {
        const int stage = (issued + next) % C::R;
        mbar_expect_tx(&bars[stage], C::PB);
        bulk_load_once(ring + stage * C::STAGE, base + (int64_t)next * p.page_bytes, C::PB, &bars[stage], pol);
      }
      if (W > 0) {
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
    float qf[D / 4];
    uint32_t qb[D / 8];
    uint32_t qzb[D / 8];
    float qsum = 0.f;
    auto load_qbp = [&]() {
#pragma unroll
      for (int dt = 0; dt < C::KS; ++dt) {
        const uint32_t lo = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t);
        const uint32_t hi = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t + 8);
        const bool keep = qvalid && (g & 1) == 0;  // q is exact in bf16: its low part is zero
        qb[2 * dt] = keep ? lo : 0u;
        qb[2 * dt + 1] = keep ? hi : 0u;
      }
    };
    if constexpr (C::kBf16) {
      load_qbp();
    } else {
#pragma unroll
      for (int dt = 0; dt < C::KS; ++dt) {
        uint32_t lo = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t);
        uint32_t hi = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t + 8);
        if (!qvalid) lo = hi = 0u;
        const float2 l2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&lo));
        const float2 h2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&hi));
        qf[dt * 4 + 0] = l2.x * p.scale_log2;
        qf[dt * 4 + 1] = l2.y * p.scale_log2;
        qf[dt * 4 + 2] = h2.x * p.scale_log2;
        qf[dt * 4 + 3] = h2.y * p.scale_log2;
      }
      const float qlo = F8 ? p.fp8_scales[h] : 1.f;
      const float qhi = PT ? 1.f / C::tauK : qlo;
#pragma unroll
      for (int dt = 0; dt < C::KS; ++dt) {
        qzb[2 * dt] = part_f16(qf[dt * 4 + 0] * qlo, qf[dt * 4 + 1] * qlo, partf);
        qzb[2 * dt + 1] = part_f16(qf[dt * 4 + 2] * qhi, qf[dt * 4 + 3] * qhi, partf);
      }
      if constexpr (PT) {
        float qs = 0.f;
#pragma unroll
        for (int i = 0; i < D / 4; ++i) qs += qf[i];
        qs += __shfl_xor_sync(0xffffffffu, qs, 1);
        qs += __shfl_xor_sync(0xffffffffu, qs, 2);
        qsum = __shfl_sync(0xffffffffu, qs, 8 * t);
      }
    }

    TokState<D> st;
#pragma unroll
    for (int j = 0; j < D / 16; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) st.o[j][k] = 0.f;
    st.m = -INFINITY;
    st.l = 0.f;
    st.vz = 0.f;
    bool converted = C::kBf16;
    auto to_true_units = [&]() {
      if constexpr (F8) {
        const float vsc = p.fp8_scales[H + h] * kF8Unit;
#pragma unroll
        for (int j = 0; j < D / 16; ++j)
#pragma unroll
          for (int k = 0; k < 4; ++k) st.o[j][k] *= vsc;
      } else if constexpr (!C::kBf16) {
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          st.o[j][0] *= kTwo24;
          st.o[j][1] *= kTwo24;
          st.o[j][2] *= kTwo24 / C::sigmaV;
          st.o[j][3] *= kTwo24 / C::sigmaV;
        }
      }
      converted = true;
    };

    for (int k = 0; k < P; ++k) {
      const int stage = consumed % C::R;
      const bool arrived = mbar_wait(&bars[stage], (uint32_t)((consumed / C::R) & 1));
      if (!__all_sync(0xffffffffu, arrived)) {
        ok = false;
        break;
      }
      const uint8_t* page = ring + stage * C::STAGE;
      if constexpr (C::kBf16) attend_bpage_tok<D>(page, st, qb, wscr, partf, p.scale_log2, lane);
      else if constexpr (F8) attend_f8page_tok<D>(page, st, qzb, wscr, partf, lane);
      else if constexpr (PT) attend_qpage_tok_pt<KB, VB, D>(page, st, qzb, qsum, wscr, partf, lane);
      else attend_qpage_tok<KB, VB, D>(page, st, qf, qzb, wscr, partf, lane);
      ++consumed;
      __syncwarp();
      if (next < P) {
        if (lane == 0) {
          fence_proxy_async();
          mbar_expect_tx(&bars[stage], C::PB);
          bulk_load_once(ring + stage * C::STAGE, base + (int64_t)next * p.page_bytes, C::PB, &bars[stage], pol);
        }
        ++next;
        ++issued;
      }
    }
    if (!ok) break;
    if (flushed) {
      // the page this warp has just written (generic loads: it never went through the async proxy)
      const uint8_t* page = base + (int64_t)P * p.page_bytes;
      if constexpr (C::kBf16) attend_bpage_tok<D>(page, st, qb, wscr, partf, p.scale_log2, lane);
      else if constexpr (F8) attend_f8page_tok<D>(page, st, qzb, wscr, partf, lane);
      else if constexpr (PT) attend_qpage_tok_pt<KB, VB, D>(page, st, qzb, qsum, wscr, partf, lane);
      else attend_qpage_tok<KB, VB, D>(page, st, qf, qzb, wscr, partf, lane);
    }
    if (W > 0) {
      if constexpr (!C::kBf16) {
        to_true_units();
        load_qbp();
      }
      attend_window_tok<D>(win, W, st, qb, wscr, partf, p.scale_log2, lane);
    }
    if (!converted) to_true_units();

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

template <int KB, int VB, int D, bool TOK, bool PT, bool F8>
cudaError_t launch4(const DecodeParams& p, cudaStream_t s) {
  using C = Cfg<KB, VB, D, PT, F8>;
  if constexpr (TOK) {
    // short sequences: one warp per segment when every segment fits in one resident wave
    if (p.warp_split) {
      using WC = WarpCfg<KB, VB, D, PT, F8>;
      static bool configured = false;
      static int occ_w = 0;
      if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(decode_warp_kernel<KB, VB, D, PT, F8>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, WC::SMEM);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_w, decode_warp_kernel<KB, VB, D, PT, F8>, kThreads,
                                                          WC::SMEM);
        if (e != cudaSuccess) return e;
        configured = true;
      }
      const int64_t segs = (int64_t)p.batch * p.n_kv_heads;
      const int64_t ctas = (segs + kWarps - 1) / kWarps;
      if (ctas >= 1 && ctas <= (int64_t)occ_w * p.sm_count)
        return launch_pdl(decode_warp_kernel<KB, VB, D, PT, F8>, dim3((unsigned)ctas), dim3(kThreads),
                          (size_t)WC::SMEM, s, p);
    }
  }
  static int configured_smem = 0;
  static int occ_smem = -1, occ_blocks = 0;
  const int smem = C::smem_bytes(TOK, p.gqa, p.batch);
  if (smem > configured_smem) {
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<KB, VB, D, TOK, PT, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess) return e;
    configured_smem = smem;
  }
  if (smem != occ_smem) {
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_blocks, decode_mma_kernel<KB, VB, D, TOK, PT, F8>,
                                                                  kThreads, smem);
    if (e != cudaSuccess) return e;
    occ_smem = smem;
  }
  int64_t grid = (int64_t)(occ_blocks > 0 ? occ_blocks : 1) * p.sm_count;
  grid = std::min<int64_t>(grid, p.n_units);
  grid = std::min<int64_t>(grid, p.max_ctas);
  if (grid < 1) grid = 1;
  return launch_pdl(decode_mma_kernel<KB, VB, D, TOK, PT, F8>, dim3((unsigned)grid), dim3(kThreads), (size_t)smem, s,
                    p);
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

// fused append + decode (one warp per segment); not launched when the segments
// do not fit one resident wave of warps
template <int KB, int VB, int D, bool PT, bool F8>
cudaError_t launch_step4(const DecodeParams& p, cudaStream_t s) {
  using WC = WarpCfg<KB, VB, D, PT, F8>;
  static bool configured = false;
  static int occ = 0;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(decode_warp_kernel<KB, VB, D, PT, F8, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, WC::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_warp_kernel<KB, VB, D, PT, F8, true>, kThreads,
                                                      WC::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int64_t ctas = ((int64_t)p.batch * p.n_kv_heads + kWarps - 1) / kWarps;
  if (ctas < 1 || ctas > (int64_t)occ * p.sm_count) return cudaErrorNotSupported;
  return launch_pdl(decode_warp_kernel<KB, VB, D, PT, F8, true>, dim3((unsigned)ctas), dim3(kThreads),
                    (size_t)WC::SMEM, s, p);
}

template <int KB, int VB, int D>
cudaError_t launch_step3(const DecodeParams& p, cudaStream_t s) {
  if (p.gqa > 4) return cudaErrorNotSupported;
  if constexpr (KB == 8 && VB == 8) {
    if (p.fmt != 0) return launch_step4<KB, VB, D, false, true>(p, s);
  }
  if constexpr (KB != 16) {
    if (p.key_mode != 0) return launch_step4<KB, VB, D, true, false>(p, s);
  }
  return launch_step4<KB, VB, D, false, false>(p, s);
}

template <int D>
cudaError_t launch_step_d(int kb, int vb, const DecodeParams& p, cudaStream_t s) {
#define KVQ_PAIR(K_, V_) \
  if (kb == K_ && vb == V_) return launch_step3<K_, V_, D>(p, s);
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

cudaError_t launch_decode_step(int kb, int vb, int D, const DecodeParams& p, cudaStream_t s) {
  if (D == 64) return launch_step_d<64>(kb, vb, p, s);
  if (D == 128) return launch_step_d<128>(kb, vb, p, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
