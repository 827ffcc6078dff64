// kvq_decode_mma.cu -- split-K decode attention over one layer's mixed-precision
// cache on the tensor cores (warp-level mma.sync m16n8k16, fp32 accumulate).
//
// KVTuner OpenReview rebuttal, "Baseline Implementation": decode runs
// FlashAttention-style kernels directly over the int8 / mixed-precision K and V
// cache; "New GQA efficiency results": grouped-query attention. Keys are
// dequantized per channel (x = code * s_c + z_c over each 32-token page) and
// values per token (x = code * s_t + z_t).
//
// Work split: grid (splits, n_kv_heads, batch), 4 warps per CTA. Each warp
// streams its own pages (p0 + warp, p0 + warp + 4, ...) through a private ring
// of shared-memory stages filled by bulk copies (cp.async.bulk, one copy per
// page, mbarrier completion) and keeps its own online-softmax state. The CTA
// merges its warps, then either writes the output (one split) or a partial
// (acc, m, l) that the last CTA of the (sequence, head) merges.
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

#include "kvq_internal.cuh"

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
template <int KB, int VB, int D>
struct Cfg {
  static constexpr bool kBf16 = (KB == 16);
  static constexpr int KS = D / 16;                       // 16-channel tiles
  static constexpr int PB = (int)page_bytes_of(KB, VB, D);
  // small pages: 3 CTAs per SM with 3-4 stages per warp; larger ones: 2 CTAs per SM
  static constexpr int MINB = PB <= 5000 ? 3 : 2;
  static constexpr int RING_BUDGET = MINB == 3 ? 14336 : 24576;   // bytes of stages per warp
  static constexpr int R = (RING_BUDGET / PB) < 2 ? 2 : ((RING_BUDGET / PB) > 4 ? 4 : (RING_BUDGET / PB));
  static constexpr int STAGE = (PB + 127) / 128 * 128;
  static constexpr int KW = D * KB / 32;                  // 32-bit words of K codes per lane
  static constexpr int VW = D * VB / 32;
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
  static constexpr int MBAR_BYTES = (kWarps * R * 8 + 127) / 128 * 128;
  static constexpr int WSCR_FLOATS = 4 * KSROW + 64;      // key scales, value scales, value zeros
  static constexpr int WSCR_OFF = MBAR_OFF + MBAR_BYTES;
  static constexpr int WSCR_STRIDE = (WSCR_FLOATS * 4 + 127) / 128 * 128;
  static constexpr int QZ_OFF = WSCR_OFF + kWarps * WSCR_STRIDE;
  static constexpr int QZ_BYTES = KS * 32 * 16;
  static constexpr int SMEM = QZ_OFF + QZ_BYTES;
  static_assert(kWarps * kMaxGqa * D * 4 + 2 * kWarps * kMaxGqa * 4 <= RING, "merge area must fit in the ring");
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

// ------------------------------------------------------------------ kernel --
template <int KB, int VB, int D>
__global__ void __launch_bounds__(kThreads, Cfg<KB, VB, D>::MINB) decode_mma_kernel(DecodeParams p) {
  using C = Cfg<KB, VB, D>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_last;
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int H = p.n_kv_heads, G = p.gqa;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int T = p.len[b];
  const int P = T / kPageTokens, W = T % kPageTokens;
  const int nsplit = P > 0 ? (P + p.chunk - 1) / p.chunk : 1;
  if (s >= nsplit) return;
  const int p0 = s * p.chunk;
  const int p1 = min(P, p0 + p.chunk);

  uint8_t* ring = smem + warp * C::R * C::STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::MBAR_OFF) + warp * C::R;
  float* wscr = reinterpret_cast<float*>(smem + C::WSCR_OFF + warp * C::WSCR_STRIDE);
  uint32_t* qz = reinterpret_cast<uint32_t*>(smem + C::QZ_OFF);

  // ---- pipeline start: this warp's pages are p0 + warp + kWarps * i
  const int first = p0 + warp;
  const int n_my = p1 > first ? (p1 - first + kWarps - 1) / kWarps : 0;
  const uint8_t* seq_pages = p.pages + ((int64_t)(b * H + h) * p.max_pages) * p.page_bytes;
  if (lane == 0) {
    for (int r = 0; r < C::R; ++r) mbar_init(&bars[r], 1);
    mbar_init_fence();
  }
  __syncwarp();
  if (lane == 0) {
    for (int i = 0; i < n_my && i < C::R; ++i) {
      mbar_expect_tx(&bars[i], C::PB);
      bulk_load(ring + i * C::STAGE, seq_pages + (int64_t)(first + i * kWarps) * p.page_bytes, C::PB, &bars[i]);
    }
  }

  // ---- query operands (row g = head g; heads >= G are zero)
  const __nv_bfloat16* qrow = p.Q + ((int64_t)b * H * G + (int64_t)h * G + (g < G ? g : 0)) * D;
  float qf[D / 4];  // q * log2(e)/sqrt(D) at this lane's channels (quantized pages)
  if constexpr (!C::kBf16) {
#pragma unroll
    for (int dt = 0; dt < C::KS; ++dt) {
      uint32_t lo = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t);
      uint32_t hi = *reinterpret_cast<const uint32_t*>(qrow + 16 * dt + 2 * t + 8);
      if (g >= G) lo = hi = 0u;
      const float2 l2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&lo));
      const float2 h2 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&hi));
      qf[dt * 4 + 0] = l2.x * p.scale_log2;
      qf[dt * 4 + 1] = l2.y * p.scale_log2;
      qf[dt * 4 + 2] = h2.x * p.scale_log2;
      qf[dt * 4 + 3] = h2.y * p.scale_log2;
    }
    if (warp == 0) {
#pragma unroll
      for (int dt = 0; dt < C::KS; ++dt) {
        uint4 a;
        split_f16(qf[dt * 4 + 0], qf[dt * 4 + 1], a.x, a.y);
        split_f16(qf[dt * 4 + 2], qf[dt * 4 + 3], a.z, a.w);
        *reinterpret_cast<uint4*>(qz + (dt * 32 + lane) * 4) = a;
      }
    }
    __syncthreads();
  }

  WarpState<D> st;
#pragma unroll
  for (int j = 0; j < D / 8; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) st.o[j][k] = 0.f;
  st.m = -INFINITY;
  st.l = 0.f;
  st.vz = 0.f;

  // ---- page loop
  {
    uint32_t qb[D / 8];
    if constexpr (C::kBf16) load_qb<D>(qrow, g < G, t, qb);
    bool ok = true;
    int consumed = 0;
    for (int i = 0; i < n_my; ++i) {
      const int stage = i % C::R;
      const bool arrived = mbar_wait(&bars[stage], (uint32_t)((i / C::R) & 1));
      if (!__all_sync(0xffffffffu, arrived)) {  // warp-uniform verdict
        ok = false;
        break;
      }
      consumed = i + 1;
      const uint8_t* page = ring + stage * C::STAGE;
      if constexpr (C::kBf16) attend_bpage<D>(page, st, qb, p.scale_log2, lane);
      else attend_qpage<KB, VB, D>(page, st, qf, qz, wscr, lane);
      __syncwarp();
      if (lane == 0 && i + C::R < n_my) {
        fence_proxy_async();
        mbar_expect_tx(&bars[stage], C::PB);
        bulk_load(ring + stage * C::STAGE, seq_pages + (int64_t)(first + (i + C::R) * kWarps) * p.page_bytes, C::PB,
                  &bars[stage]);
      }
    }
    if (!ok) {
      // a copy never completed: report it, then let the copies in flight land
      // (each wait bounded again) before this CTA's shared memory goes away
      if (lane == 0 && p.err) atomicExch(p.err, 1);
      const int issued = min(n_my, consumed + C::R);
      for (int i = consumed; i < issued; ++i) mbar_wait(&bars[i % C::R], (uint32_t)((i / C::R) & 1));
    }
  }

  // ---- quantized accumulators to true units: O = acc * 2^24 / sigmaV
  if constexpr (!C::kBf16) {
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const float f = (j & 1) ? kTwo24 / C::sigmaV : kTwo24;
#pragma unroll
      for (int k = 0; k < 4; ++k) st.o[j][k] *= f;
    }
  }
  if (s == nsplit - 1 && W > 0 && warp == kWarps - 1) {
    uint32_t qb[D / 8];
    load_qb<D>(qrow, g < G, t, qb);
    const __nv_bfloat16* win = p.window + ((int64_t)(b * H + h) * 2) * kPageTokens * D;
    attend_window<D>(win, W, st, qb, p.scale_log2, lane);
  }

  // ---- warp results to shared memory (reusing the ring; all copies have landed)
  float l = st.l + __shfl_xor_sync(0xffffffffu, st.l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  float vz = st.vz + __shfl_xor_sync(0xffffffffu, st.vz, 1);
  vz += __shfl_xor_sync(0xffffffffu, vz, 2);
  __syncthreads();
  float* mo = reinterpret_cast<float*>(smem);                  // [kWarps][G][D]
  float* mm = mo + kWarps * kMaxGqa * D;                       // [kWarps][G]
  float* ml = mm + kWarps * kMaxGqa;
  if (g < G) {
    float* dst = mo + (warp * kMaxGqa + g) * D;
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
  __syncthreads();

  // ---- CTA merge over warps, then output or split-K partial
  float* outp = p.out + ((int64_t)b * H * G + (int64_t)h * G) * D;
  const int64_t slot0 = (int64_t)(b * H + h) * p.splits_stride;
  float* part = p.partials + (slot0 + s) * G * (D + 2);
  for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
    const int gg = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mm[w * kMaxGqa + gg]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = mm[w * kMaxGqa + gg];
      const float a = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
      L = fmaf(a, ml[w * kMaxGqa + gg], L);
      O = fmaf(a, mo[(w * kMaxGqa + gg) * D + d], O);
    }
    if (nsplit == 1) {
      outp[idx] = L > 0.f ? O / L : 0.f;
    } else {
      part[gg * (D + 2) + d] = O;
      if (d == 0) {
        part[gg * (D + 2) + D] = M;
        part[gg * (D + 2) + D + 1] = L;
      }
    }
  }
  if (nsplit == 1) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(&p.ctr[b * H + h], 1);
    s_last = (prev == nsplit - 1);
    if (s_last) p.ctr[b * H + h] = 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* parts = p.partials + slot0 * G * (D + 2);
  for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
    const int gg = idx / D, d = idx % D;
    float M = -INFINITY;
    for (int j = 0; j < nsplit; ++j) M = fmaxf(M, __ldcg(parts + ((int64_t)j * G + gg) * (D + 2) + D));
    float L = 0.f, O = 0.f;
    for (int j = 0; j < nsplit; ++j) {
      const float* r = parts + ((int64_t)j * G + gg) * (D + 2);
      const float mj = __ldcg(r + D);
      const float a = (mj == -INFINITY) ? 0.f : exp2f(mj - M);
      L = fmaf(a, __ldcg(r + D + 1), L);
      O = fmaf(a, __ldcg(r + d), O);
    }
    outp[idx] = L > 0.f ? O / L : 0.f;
  }
}

template <int KB, int VB, int D>
cudaError_t launch3(const DecodeParams& p, dim3 grid, cudaStream_t s) {
  using C = Cfg<KB, VB, D>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<KB, VB, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  decode_mma_kernel<KB, VB, D><<<grid, kThreads, C::SMEM, s>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(int kb, int vb, const DecodeParams& p, dim3 grid, cudaStream_t s) {
#define KVQ_PAIR(K_, V_) \
  if (kb == K_ && vb == V_) return launch3<K_, V_, D>(p, grid, s);
  KVQ_PAIR(2, 2) KVQ_PAIR(2, 4) KVQ_PAIR(2, 8)
  KVQ_PAIR(4, 2) KVQ_PAIR(4, 4) KVQ_PAIR(4, 8)
  KVQ_PAIR(8, 2) KVQ_PAIR(8, 4) KVQ_PAIR(8, 8)
  KVQ_PAIR(16, 16)
#undef KVQ_PAIR
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_mma(int kb, int vb, int D, const DecodeParams& p, dim3 grid, cudaStream_t s) {
  if (D == 64) return launch_d<64>(kb, vb, p, grid, s);
  if (D == 128) return launch_d<128>(kb, vb, p, grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
