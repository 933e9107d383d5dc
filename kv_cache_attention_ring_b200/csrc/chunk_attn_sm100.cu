// chunk_attn_sm100.cu -- warp-specialised chunk attention for head_dim 128 on sm_100a.
//
// What it computes ("Runway Characters: Serving a 57B Video Diffusion Transformer for
// Real-Time Conversation", abstract: every call reads the whole FP8 cache, only the
// newest tokens are new; "KREA Real-Time 14B / video-conductor", section "Plastic
// Windows": an additive cache-attention bias on history; "Stream LTX", section
// "Training": block-causal masks):
//   s_ij = softmax_scale * <bf16(RoPE(q_i)), e4m3(kc_j) * ks_j> + [j history] * bias,
//   out_i = sum_j softmax_j(s_i) * e4m3(vc_j) * vs_j.
//
// Design (one CTA = 256 query rows of one head = two 128-row tiles g = 0, 1; keys in
// tiles of 64 slots):
//  * Q.K^T runs on the FP8 tensor core directly on the cached e4m3 K codes (no
//    conversion of K).  The rotated bf16 query row is split exactly into
//    q = r * (hi + lo), hi, lo e4m3, r a power of two (8 significant bits = 4 + 4), so
//    S' = hi.K + lo.K is one f32 accumulation of 2*D/32 kind::f8f6f4 MMAs and
//    s = r * ks * scale * S' (+ bias).  r is per query row, so a row's result never
//    depends on other rows (later blocks cannot change earlier ones, bit for bit).
//  * P.V runs in f16 (11 significant bits): a CTA first finds G, the smallest power of
//    two at or above every V scale of its keys; two converter warps turn V codes into
//    f16(e4m3(vc) * vs / G) in shared memory (|V'| <= 448, one f16 rounding, 2^-11
//    relative); P = f16(p) (p <= 1) is written to tensor memory over the S columns it
//    came from and read from there as the A operand; the epilogue multiplies O by G.
//  * Mode B (KV_QK_FP8): the rotated bf16 row is instead quantised to e4m3 by the write's
//    row rule, and the row scale takes the place of r; S' is one set of D/32 MMAs.
//  * Tensor memory (512 columns): tile g owns two S/P buffers of 64 columns,
//    [128g, 128g+64) and [128g+64, 128g+128), and O_g = [256+128g, 384+128g).  Per key
//    tile j and query tile g the MMA issuer runs P.V_g(j) as soon as P_g(j) is in tensor
//    memory, then S_g(j+2) into the buffer P_g(j) occupied (tensor-core operations of one
//    thread run in issue order), so the softmax finds S_g(j+1) ready after S_g(j).
//  * Warps: 0 TMA producer, 1 MMA issuer, 2-3 V converters + per-key info, 4-7 softmax
//    of tile 0, 8-11 softmax of tile 1 (thread = query row = TMEM lane).
//  * Softmax in log2 units with paired fp32 instructions (f32x2) on the 64-column S row
//    held in registers.  The reference maximum m moves lazily (only when the tile
//    maximum exceeds it by more than 8, a factor 256); O is then rescaled in tensor
//    memory after the previous P.V has completed.  out = O / l is exact regardless of m.
//    A history-only tile with m already set takes one pass (scale, 2^(t - m), P, tile
//    maximum on the way); the first tile, tiles with current or invalid keys, and tiles
//    whose maximum exceeds m by more than 8 take two (maximum first, then 2^(t - m)).
//  * Split over keys (gridDim.z > 1): each CTA takes a contiguous share of the valid
//    tiles and writes fp32 partials (O G, m, l); split_combine_kernel merges them.
//  * Keys are visited in physical slot order; the ring wrap costs nothing (attention
//    does not depend on key order once bias and mask are per key).
// Every mbarrier wait is bounded (about a second); on a timeout the CTA abandons the
// work, writes NaN to its rows and exits.
#include <cuda.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "../../include/kvring.h"

namespace kvring {

namespace {

constexpr int D = 128;
constexpr int BM = 256;                 // query rows per CTA
constexpr int BN = 64;                  // key slots per tile
constexpr int NK = 4;                   // K code stages
constexpr int NV = 4;                   // V code stages
constexpr int NB = 2;                   // V f16 buffers
constexpr int NI = 4;                   // per-key info stages
constexpr int kThreads = 12 * 32;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpConv = 2, kWarpSoft = 4;
constexpr int kConvThreads = 64;        // one converter thread per key slot of a tile
constexpr uint32_t kVPanel = BN * 128u;  // bytes of one 64-column f16 panel of V (64 rows)
constexpr float kRescaleLog2 = 8.f;
constexpr int kInvalidTok = 0x7FFFFFFF;

struct Info {             // per key slot of one tile
  float kscl[BN];         // ks * softmax_scale * log2(e); 0 for invalid slots
  float kb[BN];           // additive log2 logit: bias (history), 0 (current), -inf (invalid)
  int ktok[BN];           // -1 history, token index (current), kInvalidTok (invalid)
  int flag[2];            // per converter warp: tile holds current or invalid keys
  int pad[2];
};

struct Layout {
  static constexpr uint32_t qhi = 0;                            // e4m3 [256][128], sw128
  static constexpr uint32_t qlo = qhi + BM * D;
  static constexpr uint32_t kbuf = qlo + BM * D;                // NK x e4m3 [64][128], sw128
  static constexpr uint32_t vcode = kbuf + NK * BN * D;         // NV x e4m3 [64][128], sw128
  static constexpr uint32_t vh = vcode + NV * BN * D;           // NB x f16 2 panels, sw128
  static constexpr uint32_t info = vh + NB * 2 * kVPanel;      // NI x Info
  static constexpr uint32_t bars = info + NI * sizeof(Info);    // mbarriers
  static constexpr int kNumBars = 2 * NK + 2 * NV + 2 * NB + 2 * NI + 4 + 4 + 1;
  static constexpr uint32_t misc = bars + 8 * kNumBars;         // tmem addr, abort flag, G
  static constexpr uint32_t bytes = misc + 16 + 1024;           // + alignment slack
};
static_assert(Layout::bytes <= 232448, "shared memory budget");
static_assert(Layout::kbuf % 1024 == 0 && Layout::vcode % 1024 == 0 && Layout::vh % 1024 == 0,
              "swizzled operands need 1024-byte alignment");

struct Bars {
  uint64_t* b;
  __device__ uint64_t* kfull(int s) { return b + s; }
  __device__ uint64_t* kempty(int s) { return b + NK + s; }
  __device__ uint64_t* vfull(int s) { return b + 2 * NK + s; }
  __device__ uint64_t* vempty(int s) { return b + 2 * NK + NV + s; }
  __device__ uint64_t* vhfull(int s) { return b + 2 * NK + 2 * NV + s; }
  __device__ uint64_t* vhempty(int s) { return b + 2 * NK + 2 * NV + NB + s; }
  __device__ uint64_t* ifull(int s) { return b + 2 * NK + 2 * NV + 2 * NB + s; }
  __device__ uint64_t* iempty(int s) { return b + 2 * NK + 2 * NV + 2 * NB + NI + s; }
  // buffer `buf` of tile g holds S (sfull) / holds P (pfull); all MMAs are done (ofinal).
  // P-ready is per buffer because the softmax may finish tile j+1 before the MMA issuer
  // has consumed tile j's signal.  The P.V of key tile j (both query tiles) has completed
  // when V buffer j % NB is released (vhempty).
  __device__ uint64_t* sfull(int g, int buf) { return b + 2 * (NK + NV + NB + NI) + 2 * g + buf; }
  __device__ uint64_t* pfull(int g, int buf) { return b + 2 * (NK + NV + NB + NI) + 4 + 2 * g + buf; }
  __device__ uint64_t* ofinal() { return b + 2 * (NK + NV + NB + NI) + 8; }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// e4m3 code of v (RNE, saturating), as a byte.
__device__ __forceinline__ uint32_t e4m3_byte(float v) { return e4m3x2(v, 0.f) & 0xFFu; }

// Exact value of an e4m3 code.
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  return f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)code)).x;
}

// Does tile t (slots [t*BN, t*BN+BN)) hold a valid slot?  Valid slots are the nv slots
// ending at `newest` (mod C).
__device__ __forceinline__ bool tile_valid(int t, int C, int newest, int nv) {
  if (nv <= 0) return false;
  if (nv >= C) return true;
  const int a = t * BN, b = min(C, a + BN);
  int first = newest - nv + 1;
  if (first >= 0) return a <= newest && b > first;
  first += C;  // wrapped: [first, C) and [0, newest]
  return (b > first) || (a <= newest);
}

// Next tile index >= t holding a valid slot (n_tiles if none).
__device__ __forceinline__ int next_tile(int t, int n_tiles, int C, int newest, int nv) {
  while (t < n_tiles && !tile_valid(t, C, newest, nv)) ++t;
  return t;
}

// bf16-rounded rotation of 8 consecutive elements (chunk c) of query row gi.
__device__ __forceinline__ void q_rot8(const AttnArgs& a, int gi, int h, int c, float (&y)[8]) {
  const uint4 raw = __ldg(reinterpret_cast<const uint4*>(a.q + ((size_t)gi * a.H + h) * D) + c);
  const float4* tb = reinterpret_cast<const float4*>(a.rope_q0 + (size_t)gi * D);
  const float4 cs0 = __ldg(tb + 2 * c), cs1 = __ldg(tb + 2 * c + 1);
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  const float cc[4] = {cs0.x, cs0.z, cs1.x, cs1.z};
  const float ss[4] = {cs0.y, cs0.w, cs1.y, cs1.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float x0 = bf16_bits_to_float(w[j] & 0xFFFFu);
    const float x1 = bf16_bits_to_float(w[j] >> 16);
    const float y0 = sub_rn(mul_rn(x0, cc[j]), mul_rn(x1, ss[j]));
    const float y1 = add_rn(mul_rn(x0, ss[j]), mul_rn(x1, cc[j]));
    const uint32_t b = pack_bf16x2(y0, y1);               // bf16 RNE of the rotated pair
    y[2 * j] = bf16_bits_to_float(b & 0xFFFFu);
    y[2 * j + 1] = bf16_bits_to_float(b >> 16);
  }
}

// Exponent k of the smallest power of two r = 2^k with max|bf16(RoPE(q_gi))| / r <= 448
// (448 = 1.75 * 2^8).  Rows beyond n_q or all-zero rows return INT_MIN.
__device__ __forceinline__ int q_exponent(const AttnArgs& a, int gi, int h) {
  if (gi >= a.n_q) return INT_MIN;
  float amax = 0.f;
#pragma unroll 4
  for (int c = 0; c < D / 8; ++c) {
    float y[8];
    q_rot8(a, gi, h, c, y);
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(y[e]));
  }
  if (!(amax > 0.f) || !isfinite(amax)) return INT_MIN;
  int e;
  const float m = frexpf(amax, &e);          // amax = m * 2^e, m in [0.5, 1)
  return (e - 1) - 8 + (m > 0.875f ? 1 : 0);
}

// Split bf16(RoPE(q_gi)) / 2^k exactly into e4m3 hi + lo (4 + 4 significant bits; exact
// for elements within 2^10 of the row's largest) and write both into the swizzled
// K-major operand rows.  Rows beyond n_q get zero codes.
__device__ __forceinline__ void q_split(const AttnArgs& a, int gi, int h, int k, uint8_t* qhi,
                                        uint8_t* qlo, int row) {
  const bool live = gi < a.n_q;
  const float inv_r = ldexpf(1.f, -k);
#pragma unroll 2
  for (int c = 0; c < D / 16; ++c) {
    float y[16];
    if (live) {
      float y0[8], y1[8];
      q_rot8(a, gi, h, 2 * c, y0);
      q_rot8(a, gi, h, 2 * c + 1, y1);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        y[e] = y0[e];
        y[8 + e] = y1[e];
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) y[e] = 0.f;
    }
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t hb = 0, lb = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x = y[4 * j + e] * inv_r;                // exact (power of two)
        const uint32_t hc = e4m3_byte(x);
        const uint32_t lc = e4m3_byte(x - e4m3_value(hc));   // exact difference
        hb |= hc << (8 * e);
        lb |= lc << (8 * e);
      }
      hw[j] = hb;
      lw[j] = lb;
    }
    const uint32_t off = (uint32_t)row * 128u + ((uint32_t)(c ^ (row & 7)) << 4);
    *reinterpret_cast<uint4*>(qhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(qlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

// Mode B: quantise bf16(RoPE(q_gi)) to e4m3 by the write's row rule (scale = amax/448,
// codes = e4m3(y * (448/amax)); zero rows -> scale 0; a non-finite element -> NaN scale)
// into the swizzled K-major operand row; returns the row's scale.  Rows beyond n_q get
// zero codes and scale 0.
__device__ __forceinline__ float q_quant_b(const AttnArgs& a, int gi, int h, uint8_t* qc, int row) {
  if (gi >= a.n_q) {
#pragma unroll
    for (int c = 0; c < D / 16; ++c)
      *reinterpret_cast<uint4*>(qc + row * 128 + ((c ^ (row & 7)) << 4)) = make_uint4(0, 0, 0, 0);
    return 0.f;
  }
  float amax = 0.f;
#pragma unroll 4
  for (int c = 0; c < D / 8; ++c) {
    float y[8];
    q_rot8(a, gi, h, c, y);
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = max_nan(amax, fabsf(y[e]));
  }
  float inv = 0.f, scale = 0.f;
  bool zero = false;
  if (!(amax <= 3.402823466e38f)) {
    scale = __uint_as_float(0x7FC00000u);
  } else {
    inv = amax > 0.f ? div_rn(448.f, amax) : 0.f;
    zero = !(amax > 0.f) || !isfinite(inv);
    scale = zero ? 0.f : div_rn(amax, 448.f);
  }
  const bool bad = isnan(scale);
#pragma unroll 2
  for (int c = 0; c < D / 16; ++c) {
    float y0[8], y1[8];
    q_rot8(a, gi, h, 2 * c, y0);
    q_rot8(a, gi, h, 2 * c + 1, y1);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float* y = j < 2 ? y0 + 4 * j : y1 + 4 * (j - 2);
      const uint32_t lo = e4m3x2(mul_rn(y[0], inv), mul_rn(y[1], inv));
      const uint32_t hi = e4m3x2(mul_rn(y[2], inv), mul_rn(y[3], inv));
      w[j] = bad ? 0x7F7F7F7Fu : zero ? 0u : (lo | (hi << 16));
    }
    *reinterpret_cast<uint4*>(qc + row * 128 + ((c ^ (row & 7)) << 4)) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  return scale;
}

__global__ void __launch_bounds__(kThreads, 1)
    chunk_attn_sm100_kernel(const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars bars{reinterpret_cast<uint64_t*>(sm + Layout::bars)};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Layout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Layout::misc + 4);
  uint32_t* vmax_bits = reinterpret_cast<uint32_t*>(sm + Layout::misc + 8);
  Info* info = reinterpret_cast<Info*>(sm + Layout::info);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int q0 = blockIdx.x * BM;
  const int C = a.C;
  const int n_tiles = (C + BN - 1) / BN;
  const int newest = (int)a.newest_slot, n_valid = (int)a.n_valid;

  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int s = 0; s < NK; ++s) { mbar_init(bars.kfull(s), 1); mbar_init(bars.kempty(s), 1); }
    for (int s = 0; s < NV; ++s) { mbar_init(bars.vfull(s), 1); mbar_init(bars.vempty(s), kConvThreads); }
    for (int s = 0; s < NB; ++s) { mbar_init(bars.vhfull(s), kConvThreads); mbar_init(bars.vhempty(s), 1); }
    for (int s = 0; s < NI; ++s) { mbar_init(bars.ifull(s), kConvThreads); mbar_init(bars.iempty(s), 256); }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bars.sfull(g, 0), 1);
      mbar_init(bars.sfull(g, 1), 1);
      mbar_init(bars.pfull(g, 0), 128);
      mbar_init(bars.pfull(g, 1), 128);
    }
    mbar_init(bars.ofinal(), 1);
    *abort_flag = 0;
    *vmax_bits = 0u;
    fence_mbar_init();
  }
  if (tid == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
  }

  // Q prologue by the softmax warps: thread = query row = TMEM lane; per-row scale r = 2^k
  const int g = (warp - kWarpSoft) >> 2;                 // softmax tile (warps 4..11)
  const int row_in_tile = 32 * (warp & 3) + lane;        // TMEM lane of this thread
  const int gi = q0 + 128 * g + row_in_tile;
  float rowmul = 1.f;
  if (warp >= kWarpSoft) {
    if (a.mode_b) {
      rowmul = q_quant_b(a, gi, h, sm + Layout::qhi, 128 * g + row_in_tile);
    } else {
      int k = q_exponent(a, gi, h);
      k = (k == INT_MIN) ? 0 : max(-126, min(127, k));
      q_split(a, gi, h, k, sm + Layout::qhi, sm + Layout::qlo, 128 * g + row_in_tile);
      rowmul = ldexpf(1.f, k);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // this CTA's slice of the valid tiles (all of them unless split over keys)
  int n_mine, t_first, t_last;
  {
    int T = 0;
    for (int t = next_tile(0, n_tiles, C, newest, n_valid); t < n_tiles;
         t = next_tile(t + 1, n_tiles, C, newest, n_valid))
      ++T;
    const int per = (T + (int)gridDim.z - 1) / (int)gridDim.z;
    const int j0 = min(T, (int)blockIdx.z * per);
    n_mine = min(T, j0 + per) - j0;
    t_first = next_tile(0, n_tiles, C, newest, n_valid);
    for (int k = 0; k < j0; ++k) t_first = next_tile(t_first + 1, n_tiles, C, newest, n_valid);
    t_last = t_first;
    for (int k = 1; k < n_mine; ++k) t_last = next_tile(t_last + 1, n_tiles, C, newest, n_valid);
  }

  // G = 2^e >= every V scale of this CTA's valid keys (converters + softmax warps; the
  // TMA and MMA warps start meanwhile).  Non-negative floats order like their bits.
  float vnorm = 1.f, vnorm_inv = 1.f;
  if (warp >= kWarpConv) {
    constexpr int kN = kThreads - 32 * kWarpConv;
    float mx = 0.f;
    if (n_mine > 0) {
      const int lo = t_first * BN, hi = min(C, (t_last + 1) * BN);
      const float* vsrow = a.v_scale + (size_t)h * C;
#pragma unroll 6
      for (int s = lo + tid - 32 * kWarpConv; s < hi; s += kN) {
        int age = newest - s;
        if (age < 0) age += C;
        if (age < n_valid) mx = fmaxf(mx, __ldg(vsrow + s));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) atomicMax(vmax_bits, __float_as_uint(mx));
    named_bar(3, kN);
    // mx < 2^(b - 126) for biased exponent b; b clamped so that G and 1/G are normal
    const int b = max(1, min(252, (int)((*vmax_bits >> 23) & 0xFFu)));
    vnorm = __uint_as_float((uint32_t)(b + 1) << 23);
    vnorm_inv = __uint_as_float((uint32_t)(253 - b) << 23);
  }

  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;       // fast path: already complete
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, a.timeouts)) return true;
    *abort_flag = 1;
    return false;
  };

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int t = t_first;
      for (int j = 0; j < n_mine; ++j, t = next_tile(t + 1, n_tiles, C, newest, n_valid)) {
        const int sk = j % NK, rk = j / NK;
        if (rk > 0 && !wait(bars.kempty(sk), (rk - 1) & 1)) break;
        mbar_arrive_expect_tx(bars.kfull(sk), BN * D);
        tma_load_3d(sm + Layout::kbuf + sk * BN * D, &tmk, bars.kfull(sk), 0, t * BN, h);
        const int sv = j % NV, rv = j / NV;
        if (rv > 0 && !wait(bars.vempty(sv), (rv - 1) & 1)) break;
        mbar_arrive_expect_tx(bars.vfull(sv), BN * D);
        tma_load_3d(sm + Layout::vcode + sv * BN * D, &tmv, bars.vfull(sv), 0, t * BN, h);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_e4m3_f32(128, BN);
      constexpr uint32_t idO = idesc_f16_f32(128, D, 0, 1);
      const uint32_t sQhi = smem_u32(sm + Layout::qhi), sQlo = smem_u32(sm + Layout::qlo);
      const uint32_t sK = smem_u32(sm + Layout::kbuf), sV = smem_u32(sm + Layout::vh);
      const bool mode_b = a.mode_b != 0;
      // S_g = Q_g K^T into buffer buf of tile g (hi and lo halves of Q accumulate)
      // descriptors are built once; a step of s bytes adds s >> 4 to the start field
      const uint64_t dQhi = smem_desc_sw128(sQhi, 16, 1024), dQlo = smem_desc_sw128(sQlo, 16, 1024);
      const uint64_t dK = smem_desc_sw128(sK, 16, 1024), dV = smem_desc_sw128(sV, kVPanel, 1024);
      // query halves: hi and lo (exact split), or the one e4m3 operand (mode B)
      const int n_halves = mode_b ? 1 : 2;
      auto issue_s = [&](int gg, int buf, int sk) {
        const uint32_t d = tmem + 128 * gg + 64 * buf;
        const uint64_t kd = dK + ((sk * BN * D) >> 4);
        for (int hf = 0; hf < n_halves; ++hf) {
          const uint64_t qd = (hf == 0 ? dQhi : dQlo) + ((gg * 128 * D) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            tc_mma_f8_ss(d, qd + 2 * kk, kd + 2 * kk, idS, (hf | kk) != 0);
        }
      };
      // O_g (+)= P_g V with P_g read from tensor memory (buffer buf)
      auto issue_pv = [&](int gg, int buf, int vbi, uint32_t acc) {
        const uint32_t d = tmem + 256 + 128 * gg;
        const uint32_t p = tmem + 128 * gg + 64 * buf;
        const uint64_t vd = dV + ((vbi * 2 * kVPanel) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          tc_mma_f16_ts(d, p + 8 * kk, vd + 128 * kk, idO, acc | (kk > 0));
      };
      // S_g(jj) into buffer jj & 1; tile 1 of the CTA starts two S groups after tile 0, so
      // the two softmax groups drift apart and take turns on the exp unit.
      auto s_group = [&](int gg, int jj) -> bool {
        const int sk = jj % NK;
        if (gg == 0) {
          if (!wait(bars.kfull(sk), (jj / NK) & 1)) return false;
          tc_fence_after();
        }
        issue_s(gg, jj & 1, sk);
        tc_commit(bars.sfull(gg, jj & 1));
        if (gg == 1) tc_commit(bars.kempty(sk));       // both tiles have read K(jj)
        return true;
      };
      int j = 0;
      bool ok = true;
      for (int gg = 0; gg < 2 && ok; ++gg)
        for (int jj = 0; jj < 2 && jj < n_mine && ok; ++jj) ok = s_group(gg, jj);
      // per key tile j and query tile g: P.V(j) as soon as P_g(j) is ready, then S_g(j + 2)
      // into the buffer P_g(j) occupied (tensor-core operations run in issue order)
      for (; ok && j < n_mine; ++j) {
        if (!(ok = wait(bars.vhfull(j % NB), (j / NB) & 1))) break;
        for (int gg = 0; gg < 2; ++gg) {
          if (!(ok = wait(bars.pfull(gg, j & 1), (j >> 1) & 1))) break;
          tc_fence_after();
          issue_pv(gg, j & 1, j % NB, j > 0);
          if (gg == 1) tc_commit(bars.vhempty(j % NB));
          if (j + 2 < n_mine && !(ok = s_group(gg, j + 2))) break;
        }
      }
      if (j > 0) tc_commit(bars.ofinal());
      else mbar_arrive(bars.ofinal());
    }
  } else if (warp < kWarpSoft) {
    // ------------------------------------------------------------ converters + key info
    // 64 threads; thread ct owns key slot ct of every tile: its info, its V row (f16,
    // scale / G folded in).  The scales of the next tile are loaded while this one converts.
    const int ct = tid - 32 * kWarpConv;          // 0..63
    auto load_scales = [&](int tt, float& ks, float& vs) {
      const int slot = tt * BN + ct;
      const bool in_ring = tt < n_tiles && slot < C;
      ks = in_ring ? __ldg(a.k_scale + (size_t)h * C + slot) : 0.f;
      vs = in_ring ? __ldg(a.v_scale + (size_t)h * C + slot) : 0.f;
    };
    float pks, pvs;
    int t = t_first;
    load_scales(n_mine > 0 ? t : n_tiles, pks, pvs);
    for (int j = 0; j < n_mine; ++j) {
      const int t_next = j + 1 < n_mine ? next_tile(t + 1, n_tiles, C, newest, n_valid) : n_tiles;
      const int si = j % NI;
      bool ok = j < NI || wait(bars.iempty(si), ((j / NI) - 1) & 1);
      if (!named_bar_and(1, kConvThreads, ok)) break;   // uniform decision across converters
      Info& in = info[si];
      const int slot = t * BN + ct;
      float ksv = 0.f, kbv = -INFINITY, vsv = 0.f;
      int tok = kInvalidTok;
      if (slot < C) {
        int age = newest - slot;
        if (age < 0) age += C;
        if (age < n_valid) {
          ksv = pks * a.score_scale_log2;
          vsv = pvs * vnorm_inv;
          if (age < a.n_current) {
            kbv = 0.f;
            tok = a.n_current - 1 - age;
          } else {
            kbv = a.bias_log2;
            tok = -1;
          }
        }
      }
      in.kscl[ct] = ksv;
      in.kb[ct] = kbv;
      in.ktok[ct] = tok;
      const unsigned special = __ballot_sync(0xffffffffu, tok != -1);
      if (lane == 0) in.flag[ct >> 5] = special != 0;
      load_scales(t_next, pks, pvs);                   // prefetch for the next tile
      mbar_arrive(bars.ifull(si));
      const int sv = j % NV, b = j % NB;
      ok = wait(bars.vfull(sv), (j / NV) & 1);
      ok = ok && (j < NB || wait(bars.vhempty(b), ((j / NB) - 1) & 1));
      if (!named_bar_and(2, kConvThreads, ok)) break;
      // V row ct: 8 chunks of 16 codes (128-byte swizzled) -> f16(code * vs / G)
      const uint8_t* vc = sm + Layout::vcode + sv * BN * D + ct * 128;
      uint8_t* vb = sm + Layout::vh + b * 2 * kVPanel;
      const bool dead = tok == kInvalidTok;
      const uint64_t vs2 = f2_pack(vsv, vsv);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 cv = *reinterpret_cast<const uint4*>(vc + ((c ^ (ct & 7)) << 4));
        if (dead) cv = make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w[4] = {cv.x, cv.y, cv.z, cv.w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float a0, a1, b0, b1;
          const float2 lo = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[i] & 0xFFFFu)));
          const float2 hi = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[i] >> 16)));
          f2_unpack(f2_mul(f2_pack(lo.x, lo.y), vs2), a0, a1);
          f2_unpack(f2_mul(f2_pack(hi.x, hi.y), vs2), b0, b1);
          o[2 * i] = pack_f16x2(a0, a1);
          o[2 * i + 1] = pack_f16x2(b0, b1);
        }
        *reinterpret_cast<uint4*>(vb + sw128_offset(ct, 16 * c, kVPanel)) =
            make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(vb + sw128_offset(ct, 16 * c + 8, kVPanel)) =
            make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_smem();
      mbar_arrive(bars.vhfull(b));
      mbar_arrive(bars.vempty(sv));
      t = t_next;
    }
  } else {
    // ------------------------------------------------------------ softmax of tile g
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t t_o = tmem + lane_base + 256 + 128 * g;     // O_g
    int lim;                                                   // visible current keys: tok < lim
    {
      const int64_t qb = gi < a.q_first ? 0 : 1 + (int64_t)(gi - a.q_first) / a.q_block;
      const int64_t l = (int64_t)a.k_first + qb * (int64_t)a.k_block;
      lim = (int)(l < (int64_t)a.n_current ? l : (int64_t)a.n_current);
    }
    const uint64_t r2 = f2_pack(rowmul, rowmul);
    float m_run = -INFINITY, l_run = 0.f;
    int j = 0;
    for (int t = t_first; j < n_mine; t = next_tile(t + 1, n_tiles, C, newest, n_valid), ++j) {
      const int si = j % NI, buf = j & 1;
      const uint32_t t_s = tmem + lane_base + 128 * g + 64 * buf;   // S_g(j) / P_g(j)
      bool ok = wait(bars.sfull(g, buf), (j >> 1) & 1) && wait(bars.ifull(si), (j / NI) & 1);
      if (!__all_sync(0xffffffffu, ok)) break;     // TMEM access below is warp-collective
      tc_fence_after();
      const Info& in = info[si];
      const bool special = (in.flag[0] | in.flag[1]) != 0;
      uint32_t sr[64];
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t (*)[32]>(sr);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t (*)[32]>(sr + 32);
        tmem_ld32(t_s, lo);
        tmem_ld32(t_s + 32, hi);
      }
      tmem_wait_ld();
      const float4* k4s = reinterpret_cast<const float4*>(in.kscl);
      const float m_old = m_run;
      bool move = false, single = false;
      uint64_t sum01 = f2_pack(0.f, 0.f), sum23 = sum01;
      if (!special && __all_sync(0xffffffffu, m_run != -INFINITY)) {
        // single pass against the current reference maximum: p = 2^(S kscl r + bias - m),
        // the tile maximum tracked on the way; kept unless a row's tile maximum exceeds m
        // by more than 2^8 (then the two passes below recompute the tile from S)
        const float off = a.bias_log2 - m_run;
        const uint64_t off2 = f2_pack(off, off);
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int q8 = 0; q8 < 8; ++q8) {
            const int q = 8 * c + q8;
            const float4 ks = k4s[q];
            const uint64_t u01 = f2_mul(f2_pack(__uint_as_float(sr[4 * q]), __uint_as_float(sr[4 * q + 1])),
                                        f2_pack(ks.x, ks.y));
            const uint64_t u23 = f2_mul(f2_pack(__uint_as_float(sr[4 * q + 2]), __uint_as_float(sr[4 * q + 3])),
                                        f2_pack(ks.z, ks.w));
            float u0, u1, u2, u3, t0, t1, t2, t3;
            f2_unpack(u01, u0, u1);
            f2_unpack(u23, u2, u3);
            m0 = max3f(m0, u0, u1);
            m1 = max3f(m1, u2, u3);
            f2_unpack(f2_fma(u01, r2, off2), t0, t1);
            f2_unpack(f2_fma(u23, r2, off2), t2, t3);
            const float p0 = ex2(t0), p1 = ex2(t1), p2 = ex2(t2), p3 = ex2(t3);
            sum01 = f2_add(sum01, f2_pack(p0, p1));
            sum23 = f2_add(sum23, f2_pack(p2, p3));
            pk[2 * q8] = pack_f16x2(p0, p1);
            pk[2 * q8 + 1] = pack_f16x2(p2, p3);
          }
          // P over S columns already read into registers; a recomputation overwrites it
          tmem_st16(t_s + 16 * c, pk);
        }
        const float mloc = fmaf(fmaxf(m0, m1), rowmul, a.bias_log2);
        single = !__any_sync(0xffffffffu, mloc > m_run + kRescaleLog2);
      }
      if (!single) {
        // pass 1, in place: t = S * kscl (* r + bias later) for fast tiles, masked t for the
        // others; row maximum of the tile
        const float4* k4 = reinterpret_cast<const float4*>(in.kscl);
        float m0 = -INFINITY, m1 = -INFINITY;
        if (!special) {
          // key scales in two batches of 8 shared-memory loads, so their latency overlaps
          float4 kq[8];
  #pragma unroll
          for (int q = 0; q < 16; ++q) {
            if ((q & 7) == 0) {
  #pragma unroll
              for (int i = 0; i < 8; ++i) kq[i] = k4[q + i];
            }
            const float4 ks = kq[q & 7];
            float u0, u1, u2, u3;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(sr[4 * q]), __uint_as_float(sr[4 * q + 1])),
                             f2_pack(ks.x, ks.y)), u0, u1);
            f2_unpack(f2_mul(f2_pack(__uint_as_float(sr[4 * q + 2]), __uint_as_float(sr[4 * q + 3])),
                             f2_pack(ks.z, ks.w)), u2, u3);
            sr[4 * q] = __float_as_uint(u0);
            sr[4 * q + 1] = __float_as_uint(u1);
            sr[4 * q + 2] = __float_as_uint(u2);
            sr[4 * q + 3] = __float_as_uint(u3);
            m0 = max3f(m0, u0, u1);
            m1 = max3f(m1, u2, u3);
          }
        } else {
          const float4* b4 = reinterpret_cast<const float4*>(in.kb);
          const int4* t4 = reinterpret_cast<const int4*>(in.ktok);
  #pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float4 ks = k4[q], kb = b4[q];
            const int4 tk = t4[q];
            float u0, u1, u2, u3;
            f2_unpack(f2_fma(f2_mul(f2_pack(__uint_as_float(sr[4 * q]), __uint_as_float(sr[4 * q + 1])),
                                    f2_pack(ks.x, ks.y)), r2, f2_pack(kb.x, kb.y)), u0, u1);
            f2_unpack(f2_fma(f2_mul(f2_pack(__uint_as_float(sr[4 * q + 2]), __uint_as_float(sr[4 * q + 3])),
                                    f2_pack(ks.z, ks.w)), r2, f2_pack(kb.z, kb.w)), u2, u3);
            u0 = tk.x < lim ? u0 : -INFINITY;
            u1 = tk.y < lim ? u1 : -INFINITY;
            u2 = tk.z < lim ? u2 : -INFINITY;
            u3 = tk.w < lim ? u3 : -INFINITY;
            sr[4 * q] = __float_as_uint(u0);
            sr[4 * q + 1] = __float_as_uint(u1);
            sr[4 * q + 2] = __float_as_uint(u2);
            sr[4 * q + 3] = __float_as_uint(u3);
            m0 = max3f(m0, u0, u1);
            m1 = max3f(m1, u2, u3);
          }
        }
        const float mloc = special ? fmaxf(m0, m1) : fmaf(fmaxf(m0, m1), rowmul, a.bias_log2);
        // lazy reference maximum: move m only when the tile maximum exceeds it by more than
        // 2^8 (rows of a tile may differ; everything below is per row)
        move = mloc > m_old + kRescaleLog2 || (m_old == -INFINITY && mloc > -INFINITY);
        if (move) m_run = mloc;
        const float mref = (m_run == -INFINITY) ? 0.f : m_run;
        // pass 2: p = 2^(t - m); P = f16(p) over the S columns of tensor memory
        const float off = special ? -mref : a.bias_log2 - mref;
        const uint64_t mul2 = special ? f2_pack(1.f, 1.f) : r2;
        const uint64_t off2 = f2_pack(off, off);
        sum01 = f2_pack(0.f, 0.f);
        sum23 = sum01;
  #pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
  #pragma unroll
          for (int q8 = 0; q8 < 8; ++q8) {
            const int q = 8 * c + q8;
            float t0, t1, t2, t3;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[4 * q]), __uint_as_float(sr[4 * q + 1])), mul2,
                             off2), t0, t1);
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[4 * q + 2]), __uint_as_float(sr[4 * q + 3])), mul2,
                             off2), t2, t3);
            const float p0 = ex2(t0), p1 = ex2(t1), p2 = ex2(t2), p3 = ex2(t3);   // 2^-inf = 0
            sum01 = f2_add(sum01, f2_pack(p0, p1));
            sum23 = f2_add(sum23, f2_pack(p2, p3));
            pk[2 * q8] = pack_f16x2(p0, p1);
            pk[2 * q8 + 1] = pack_f16x2(p2, p3);
          }
          tmem_st16(t_s + 16 * c, pk);
        }
      }
      float s0, s1, s2, s3;
      f2_unpack(sum01, s0, s1);
      f2_unpack(sum23, s2, s3);
      const bool scale_o = move && m_old != -INFINITY;
      const float alpha = scale_o ? ex2(m_old - m_run) : 1.f;
      l_run = l_run * alpha + ((s0 + s1) + (s2 + s3));
      // rescale O_g once the previous P.V of this tile has landed (rare; warp-collective)
      if (__any_sync(0xffffffffu, scale_o)) {
        // P.V(j - 1) of both tiles has completed once V buffer (j - 1) is released
        ok = wait(bars.vhempty((j - 1) % NB), ((j - 1) / NB) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_o + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(t_o + 32 * c, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars.pfull(g, buf));
      mbar_arrive(bars.iempty(si));
    }
    // ------------------------------------------------------------ epilogue
    const bool ok = __all_sync(0xffffffffu, wait(bars.ofinal(), 0));
    tc_fence_after();
    const bool row_ok = gi < a.n_q;
    const bool any = j > 0;
    if (a.part_o) {
      // split over keys: unnormalised O (relative to m_run, times G) and (m_run, l_run)
      const size_t prow = ((size_t)blockIdx.z * a.n_q + (row_ok ? gi : 0)) * a.H + h;
      float* po = a.part_o + prow * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (any) {
          tmem_ld32(t_o + 32 * c, o);
          tmem_wait_ld();
        }
        if (row_ok) {
          float4* d4 = reinterpret_cast<float4*>(po + 32 * c);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            float4 v;
            v.x = (any && l_run > 0.f) ? __uint_as_float(o[4 * k]) * vnorm : 0.f;
            v.y = (any && l_run > 0.f) ? __uint_as_float(o[4 * k + 1]) * vnorm : 0.f;
            v.z = (any && l_run > 0.f) ? __uint_as_float(o[4 * k + 2]) * vnorm : 0.f;
            v.w = (any && l_run > 0.f) ? __uint_as_float(o[4 * k + 3]) * vnorm : 0.f;
            if (!ok) v.x = v.y = v.z = v.w = __uint_as_float(0x7FC00000u);
            d4[k] = v;
          }
        }
      }
      if (row_ok) {
        float2* pml = reinterpret_cast<float2*>(a.part_ml) +
                      ((size_t)blockIdx.z * a.H + h) * a.n_q + gi;
        *pml = ok ? make_float2(m_run, l_run)
                  : make_float2(__uint_as_float(0x7FC00000u), __uint_as_float(0x7FC00000u));
      }
    } else {
    uint16_t* dst = a.out + ((size_t)(row_ok ? gi : 0) * a.H + h) * D;
    const float inv_l = (l_run > 0.f) ? (1.f / l_run) * vnorm : 0.f;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (any) {
        tmem_ld32(t_o + 32 * c, o);
        tmem_wait_ld();
      }
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float x0 = l_run > 0.f ? __uint_as_float(o[2 * k]) * inv_l : 0.f;
        float x1 = l_run > 0.f ? __uint_as_float(o[2 * k + 1]) * inv_l : 0.f;
        if (!ok) x0 = x1 = __uint_as_float(0x7FC00000u);
        pk[k] = pack_bf16x2(x0, x1);
      }
      if (row_ok) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          d4[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
      }
    }
    if (row_ok && a.lse) {
      float v = (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      if (!ok) v = __uint_as_float(0x7FC00000u);
      a.lse[(size_t)h * a.n_q + gi] = v;
    }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the split partials of one (query row, head) per warp: M = max m_s over splits
// with l_s > 0, w_s = 2^(m_s - M), out = sum w_s O_s / sum w_s l_s, lse = (M + log2 L) ln 2.
__global__ void __launch_bounds__(256) split_combine_kernel(const AttnArgs a, int n_splits) {
  const int wid = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (wid >= a.n_q * a.H) return;                 // whole warp leaves together
  const int gi = wid / a.H, h = wid % a.H;
  const float2* pml = reinterpret_cast<const float2*>(a.part_ml);
  float M = -INFINITY;
  bool bad = false;                               // a split that gave up: NaN out
  for (int z = 0; z < n_splits; ++z) {
    const float2 ml = pml[((size_t)z * a.H + h) * a.n_q + gi];
    bad |= isnan(ml.y);
    if (ml.y > 0.f) M = fmaxf(M, ml.x);
  }
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int z = 0; z < n_splits; ++z) {
    const float2 ml = pml[((size_t)z * a.H + h) * a.n_q + gi];
    if (!(ml.y > 0.f)) continue;
    const float w = ex2(ml.x - M);
    L += w * ml.y;
    const float4 o = reinterpret_cast<const float4*>(
        a.part_o + (((size_t)z * a.n_q + gi) * a.H + h) * D)[lane];
    acc.x += w * o.x;
    acc.y += w * o.y;
    acc.z += w * o.z;
    acc.w += w * o.w;
  }
  float inv = L > 0.f ? 1.f / L : 0.f;
  if (bad) inv = __uint_as_float(0x7FC00000u);
  uint2 pk;
  pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(a.out + ((size_t)gi * a.H + h) * D)[lane] = pk;
  if (lane == 0 && a.lse)
    a.lse[(size_t)h * a.n_q + gi] = bad ? __uint_as_float(0x7FC00000u)
                                    : L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f
                                              : -INFINITY;
}

}  // namespace

int launch_split_combine(const AttnArgs& a, int D_, int n_splits, cudaStream_t s) {
  if (D_ != D) return KV_EUNSUPPORTED;
  const int warps = a.n_q * a.H;
  split_combine_kernel<<<(warps + 7) / 8, 256, 0, s>>>(a, n_splits);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

int launch_attention_sm100_d128(const AttnArgs& a, const void* tmap_k_sw128,
                                const void* tmap_v_sw128, cudaStream_t s, int n_splits) {
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(chunk_attn_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Layout::bytes) != cudaSuccess)
      return KV_ECUDA;
    configured = true;
  }
  CUtensorMap mk, mv;
  memcpy(&mk, tmap_k_sw128, sizeof(mk));
  memcpy(&mv, tmap_v_sw128, sizeof(mv));
  dim3 grid((a.n_q + BM - 1) / BM, a.H, n_splits);
  chunk_attn_sm100_kernel<<<grid, kThreads, Layout::bytes, s>>>(mk, mv, a);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

}  // namespace kvring
