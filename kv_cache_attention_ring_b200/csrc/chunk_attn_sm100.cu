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
// Design (one CTA = 256 query rows of one head = two 128-row tiles g = 0, 1):
//  * Q.K^T runs on the FP8 tensor core directly on the cached e4m3 K codes (no
//    conversion of K).  The rotated bf16 query row is split exactly into
//    q = r * (hi + lo), hi, lo e4m3, r a power of two (8 significant bits = 4 + 4), so
//    S' = hi.K + lo.K is one f32 accumulation of 2*D/32 kind::f8f6f4 MMAs and
//    s = r * ks * scale * S' (+ bias).
//  * P.V runs in bf16: V codes are converted (exactly) to bf16 in shared memory by four
//    converter warps; P = p * vs (bf16) is written to tensor memory over the S columns
//    it came from and read from there as the A operand.
//  * Tensor memory (512 columns): S0/P0 [0,128), S1/P1 [128,256), O0 [256,384),
//    O1 [384,512).  MMA issue order per key tile j:
//      S0(j) PV1(j-1) S1(j) PV0(j)
//    so softmax of tile g overlaps the tensor core working on the other tile.
//  * Warps: 0 TMA producer, 1 MMA issuer, 2-5 V converters + per-key info, 6-9 softmax
//    of tile 0, 10-13 softmax of tile 1 (thread = query row = TMEM lane).
//  * Online softmax in log2 units with lazy rescale of O (only when the row maximum
//    grows by more than 8, i.e. a factor 256); the final O / l is exact regardless.
//  * Keys are visited in physical slot order in 128-slot tiles; the ring wrap costs
//    nothing (attention does not depend on key order once bias and mask are per key).
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
constexpr int BN = 128;                 // key slots per tile
constexpr int NK = 3;                   // K code stages
constexpr int NV = 2;                   // V code stages
constexpr int NB = 2;                   // V bf16 buffers
constexpr int NI = 4;                   // per-key info stages
constexpr int kThreads = 14 * 32;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpConv = 2, kWarpSoft = 6;
constexpr uint32_t kPanel = 128u * 128u;   // one 128-row x 128-byte swizzled panel
constexpr float kRescaleLog2 = 8.f;
constexpr int kInvalidTok = 0x7FFFFFFF;

struct Info {             // per key slot of one tile
  float kscl[BN];         // ks * softmax_scale * log2(e); 0 for invalid slots
  float kb[BN];           // additive log2 logit: bias (history), 0 (current), -inf (invalid)
  int ktok[BN];           // -1 history, token index (current), kInvalidTok (invalid)
  float vscl[BN];         // vs; 0 for invalid slots
  int flag[4];            // per converter warp: tile holds current or invalid keys
};

struct Layout {
  static constexpr uint32_t qhi = 0;                            // e4m3 [256][128], sw128
  static constexpr uint32_t qlo = qhi + BM * D;
  static constexpr uint32_t kbuf = qlo + BM * D;                // NK x e4m3 [128][128], sw128
  static constexpr uint32_t vcode = kbuf + NK * BN * D;         // NV x e4m3 [128][128]
  static constexpr uint32_t vbf = vcode + NV * BN * D;          // NB x bf16 2 panels, sw128
  static constexpr uint32_t info = vbf + NB * 2 * kPanel;       // NI x Info
  static constexpr uint32_t bars = info + NI * sizeof(Info);    // mbarriers
  static constexpr int kNumBars = 2 * NK + 2 * NV + 2 * NB + 2 * NI + 2 + 2 + 1;
  static constexpr uint32_t misc = bars + 8 * kNumBars;         // tmem addr, abort flag
  static constexpr uint32_t bytes = misc + 16 + 1024;           // + alignment slack
};
static_assert(Layout::bytes <= 232448, "shared memory budget");

struct Bars {
  uint64_t* b;
  __device__ uint64_t* kfull(int s) { return b + s; }
  __device__ uint64_t* kempty(int s) { return b + NK + s; }
  __device__ uint64_t* vfull(int s) { return b + 2 * NK + s; }
  __device__ uint64_t* vempty(int s) { return b + 2 * NK + NV + s; }
  __device__ uint64_t* vbfull(int s) { return b + 2 * NK + 2 * NV + s; }
  __device__ uint64_t* vbempty(int s) { return b + 2 * NK + 2 * NV + NB + s; }
  __device__ uint64_t* ifull(int s) { return b + 2 * NK + 2 * NV + 2 * NB + s; }
  __device__ uint64_t* iempty(int s) { return b + 2 * NK + 2 * NV + 2 * NB + NI + s; }
  __device__ uint64_t* sfull(int g) { return b + 2 * NK + 2 * NV + 2 * NB + 2 * NI + g; }
  __device__ uint64_t* pfull(int g) { return b + 2 * NK + 2 * NV + 2 * NB + 2 * NI + 2 + g; }
  __device__ uint64_t* ofinal() { return b + 2 * NK + 2 * NV + 2 * NB + 2 * NI + 4; }
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

__device__ __forceinline__ bool tile_valid(int64_t t, int64_t C, int64_t newest, int64_t nv) {
  if (nv <= 0) return false;
  if (nv >= C) return true;
  const int64_t a = t * BN, b = min(C, a + BN);
  int64_t first = newest - nv + 1;
  if (first >= 0) return a <= newest && b > first;
  first += C;
  return (b > first) || (a <= newest);
}

// Next physical tile index >= t holding a valid slot (n_tiles if none).
__device__ __forceinline__ int64_t next_tile(int64_t t, int64_t n_tiles, int64_t C,
                                             int64_t newest, int64_t nv) {
  while (t < n_tiles && !tile_valid(t, C, newest, nv)) ++t;
  return t;
}

// Rotate query row gi at position q_pos0 + gi, round to bf16, split exactly into
// r * (hi + lo) with e4m3 hi/lo and a power-of-two r; write hi/lo into the swizzled
// K-major operand rows.  Returns r (0 rows beyond n_q give r = 1 and zero codes).
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

// Rotate query row gi at position q_pos0 + gi, round to bf16, split exactly into
// r * (hi + lo) with e4m3 hi/lo and a power-of-two r; write hi/lo into the swizzled
// K-major operand rows.  Returns r.  Rows beyond n_q get zero codes and r = 1.
__device__ __forceinline__ float q_prologue(const AttnArgs& a, int gi, int h, uint8_t* qhi,
                                            uint8_t* qlo, int row) {
  const bool live = gi < a.n_q;
  float amax = 0.f;
  if (live) {
#pragma unroll 4
    for (int c = 0; c < D / 8; ++c) {
      float y[8];
      q_rot8(a, gi, h, c, y);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(y[e]));
    }
  }
  // smallest power of two r with amax / r <= 448 (448 = 1.75 * 2^8), clamped to normals
  int k = 0;
  if (amax > 0.f && isfinite(amax)) {
    int e;
    const float m = frexpf(amax, &e);        // amax = m * 2^e, m in [0.5, 1)
    k = (e - 1) - 8 + (m > 0.875f ? 1 : 0);
    k = max(-126, min(127, k));
  }
  const float r = ldexpf(1.f, k), inv_r = ldexpf(1.f, -k);
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
  return r;
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
  Info* info = reinterpret_cast<Info*>(sm + Layout::info);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int q0 = blockIdx.x * BM;
  const int64_t C = a.C;
  const int64_t n_tiles = (C + BN - 1) / BN;

  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int s = 0; s < NK; ++s) { mbar_init(bars.kfull(s), 1); mbar_init(bars.kempty(s), 1); }
    for (int s = 0; s < NV; ++s) { mbar_init(bars.vfull(s), 1); mbar_init(bars.vempty(s), 128); }
    for (int s = 0; s < NB; ++s) { mbar_init(bars.vbfull(s), 128); mbar_init(bars.vbempty(s), 1); }
    for (int s = 0; s < NI; ++s) { mbar_init(bars.ifull(s), 128); mbar_init(bars.iempty(s), 256); }
    for (int g = 0; g < 2; ++g) { mbar_init(bars.sfull(g), 1); mbar_init(bars.pfull(g), 128); }
    mbar_init(bars.ofinal(), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
  }

  // Q prologue by the softmax warps: thread = query row = TMEM lane
  const int g = (warp - kWarpSoft) >> 2;                 // softmax tile (valid for warps 6..13)
  const int row_in_tile = 32 * (warp & 3) + lane;        // TMEM lane of this thread
  const int gi = q0 + 128 * g + row_in_tile;
  float rowmul = 1.f;
  if (warp >= kWarpSoft)
    rowmul = q_prologue(a, gi, h, sm + Layout::qhi, sm + Layout::qlo, 128 * g + row_in_tile);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, a.timeouts)) return true;
    *abort_flag = 1;
    return false;
  };

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int64_t t = next_tile(0, n_tiles, C, a.newest_slot, a.n_valid);
      for (int j = 0; t < n_tiles; ++j, t = next_tile(t + 1, n_tiles, C, a.newest_slot, a.n_valid)) {
        const int sk = j % NK, rk = j / NK;
        if (rk > 0 && !wait(bars.kempty(sk), (rk - 1) & 1)) break;
        mbar_arrive_expect_tx(bars.kfull(sk), BN * D);
        tma_load_3d(sm + Layout::kbuf + sk * BN * D, &tmk, bars.kfull(sk), 0, (int)(t * BN), h);
        const int sv = j % NV, rv = j / NV;
        if (rv > 0 && !wait(bars.vempty(sv), (rv - 1) & 1)) break;
        mbar_arrive_expect_tx(bars.vfull(sv), BN * D);
        tma_load_3d(sm + Layout::vcode + sv * BN * D, &tmv, bars.vfull(sv), 0, (int)(t * BN), h);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_e4m3_f32(128, BN);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t sQhi = smem_u32(sm + Layout::qhi), sQlo = smem_u32(sm + Layout::qlo);
      const uint32_t sK = smem_u32(sm + Layout::kbuf), sV = smem_u32(sm + Layout::vbf);
      auto issue_s = [&](int gg, int sk) {
        const uint32_t d = tmem + 128 * gg;
        const uint32_t kb = sK + sk * BN * D;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          tc_mma_f8_ss(d, smem_desc_sw128(sQhi + gg * 128 * D + kk * 32, 16, 1024),
                       smem_desc_sw128(kb + kk * 32, 16, 1024), idS, kk > 0);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          tc_mma_f8_ss(d, smem_desc_sw128(sQlo + gg * 128 * D + kk * 32, 16, 1024),
                       smem_desc_sw128(kb + kk * 32, 16, 1024), idS, 1);
      };
      auto issue_pv = [&](int gg, int b, uint32_t acc) {
        const uint32_t d = tmem + 256 + 128 * gg;
        const uint32_t p = tmem + 128 * gg;
        const uint32_t vb = sV + b * 2 * kPanel;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          tc_mma_f16_ts(d, p + 8 * kk, smem_desc_sw128(vb + kk * 2048, kPanel, 1024), idO,
                        acc | (kk > 0));
      };
      int j = 0;
      bool ok = true;
      for (int64_t t = next_tile(0, n_tiles, C, a.newest_slot, a.n_valid); t < n_tiles;
           t = next_tile(t + 1, n_tiles, C, a.newest_slot, a.n_valid), ++j) {
        const int sk = j % NK;
        if (!(ok = wait(bars.kfull(sk), (j / NK) & 1))) break;
        tc_fence_after();
        issue_s(0, sk);
        tc_commit(bars.sfull(0));
        if (j > 0) {
          if (!(ok = wait(bars.pfull(1), (j - 1) & 1))) break;
          tc_fence_after();
          issue_pv(1, (j - 1) % NB, (j - 1) > 0);
          tc_commit(bars.vbempty((j - 1) % NB));
        }
        issue_s(1, sk);
        tc_commit(bars.sfull(1));
        tc_commit(bars.kempty(sk));
        if (!(ok = wait(bars.vbfull(j % NB), (j / NB) & 1))) break;
        if (!(ok = wait(bars.pfull(0), j & 1))) break;
        tc_fence_after();
        issue_pv(0, j % NB, j > 0);
      }
      if (ok && j > 0 && wait(bars.pfull(1), (j - 1) & 1)) {
        tc_fence_after();
        issue_pv(1, (j - 1) % NB, (j - 1) > 0);
        tc_commit(bars.vbempty((j - 1) % NB));
      }
      if (j > 0) tc_commit(bars.ofinal());
      else mbar_arrive(bars.ofinal());
    }
  } else if (warp < kWarpSoft) {
    // ------------------------------------------------------------ converters + key info
    const int ct = tid - 32 * kWarpConv;          // 0..127
    int j = 0;
    for (int64_t t = next_tile(0, n_tiles, C, a.newest_slot, a.n_valid); t < n_tiles;
         t = next_tile(t + 1, n_tiles, C, a.newest_slot, a.n_valid), ++j) {
      const int si = j % NI;
      bool ok = j < NI || wait(bars.iempty(si), ((j / NI) - 1) & 1);
      if (!named_bar_and(1, 128, ok)) break;       // uniform decision across converters
      Info& in = info[si];
      {
        const int64_t slot = t * BN + ct;
        float ksv = 0.f, kbv = -INFINITY, vsv = 0.f;
        int tok = kInvalidTok;
        if (slot < C) {
          int64_t age = a.newest_slot - slot;
          if (age < 0) age += C;
          if (age < a.n_valid) {
            ksv = a.k_scale[(size_t)h * C + slot] * a.score_scale_log2;
            vsv = a.v_scale[(size_t)h * C + slot];
            if (age < a.n_current) {
              kbv = 0.f;
              tok = (int)(a.n_current - 1 - age);
            } else {
              kbv = a.bias_log2;
              tok = -1;
            }
          }
        }
        in.kscl[ct] = ksv;
        in.kb[ct] = kbv;
        in.ktok[ct] = tok;
        in.vscl[ct] = vsv;
        const unsigned special = __ballot_sync(0xffffffffu, tok != -1);
        if (lane == 0) in.flag[ct >> 5] = special != 0;
      }
      named_bar(1, 128);                               // info of this tile complete
      mbar_arrive(bars.ifull(si));
      const int sv = j % NV, b = j % NB;
      ok = wait(bars.vfull(sv), (j / NV) & 1);
      ok = ok && (j < NB || wait(bars.vbempty(b), ((j / NB) - 1) & 1));
      if (!named_bar_and(2, 128, ok)) break;
      const uint8_t* vc = sm + Layout::vcode + sv * BN * D;
      uint8_t* vb = sm + Layout::vbf + b * 2 * kPanel;
#pragma unroll 4
      for (int idx = ct; idx < BN * D / 16; idx += 128) {
        const int row = idx >> 3, c = idx & 7;
        uint4 cv = *reinterpret_cast<const uint4*>(vc + row * D + 16 * c);
        if (in.ktok[row] == kInvalidTok) cv = make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w[4] = {cv.x, cv.y, cv.z, cv.w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 lo = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[i] & 0xFFFFu)));
          const float2 hi = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[i] >> 16)));
          o[2 * i] = pack_bf16x2(lo.x, lo.y);
          o[2 * i + 1] = pack_bf16x2(hi.x, hi.y);
        }
        *reinterpret_cast<uint4*>(vb + sw128_offset(row, 16 * c, kPanel)) =
            make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(vb + sw128_offset(row, 16 * c + 8, kPanel)) =
            make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_smem();
      mbar_arrive(bars.vbfull(b));
      mbar_arrive(bars.vempty(sv));
    }
  } else {
    // ------------------------------------------------------------ softmax of tile g
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t t_s = tmem + lane_base + 128 * g;           // S_g / P_g
    const uint32_t t_o = tmem + lane_base + 256 + 128 * g;     // O_g
    int lim;                                                   // visible current keys: tok < lim
    {
      const int64_t qb = gi < a.q_first ? 0 : 1 + (int64_t)(gi - a.q_first) / a.q_block;
      const int64_t l = (int64_t)a.k_first + qb * (int64_t)a.k_block;
      lim = (int)(l < (int64_t)a.n_current ? l : (int64_t)a.n_current);
    }
    float m_run = -INFINITY, l_run = 0.f;
    int j = 0;
    for (int64_t t = next_tile(0, n_tiles, C, a.newest_slot, a.n_valid); t < n_tiles;
         t = next_tile(t + 1, n_tiles, C, a.newest_slot, a.n_valid), ++j) {
      const int si = j % NI;
      bool ok = wait(bars.sfull(g), j & 1) && wait(bars.ifull(si), (j / NI) & 1);
      if (!__all_sync(0xffffffffu, ok)) break;     // TMEM access below is warp-collective
      tc_fence_after();
      const Info& in = info[si];
      const bool special = (in.flag[0] | in.flag[1] | in.flag[2] | in.flag[3]) != 0;
      // pass 1: row maximum of this tile (log2 units)
      float mloc = -INFINITY;
      if (!special) {
        float umax = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t raw[32];
          tmem_ld32(t_s + 32 * c, raw);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) umax = fmaxf(umax, __uint_as_float(raw[k]) * in.kscl[32 * c + k]);
        }
        mloc = fmaf(umax, rowmul, a.bias_log2);
      } else {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t raw[32];
          tmem_ld32(t_s + 32 * c, raw);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int key = 32 * c + k;
            const float tv = fmaf(__uint_as_float(raw[k]) * in.kscl[key], rowmul, in.kb[key]);
            mloc = fmaxf(mloc, in.ktok[key] < lim ? tv : -INFINITY);
          }
        }
      }
      // lazy rescale of O (warp-collective TMEM access; alpha = 1 for rows that keep m)
      const bool move = mloc > m_run + kRescaleLog2 || (m_run == -INFINITY && mloc > -INFINITY);
      const bool scale_o = move && m_run != -INFINITY;
      const float alpha = scale_o ? ex2(m_run - mloc) : 1.f;
      if (__any_sync(0xffffffffu, scale_o)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_o + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(t_o + 32 * c, o);
        }
      }
      if (move) {
        l_run *= alpha;
        m_run = mloc;
      }
      // pass 2: p = 2^(t - m), P = p * vs (bf16) over the S columns already consumed
      const float mref = (m_run == -INFINITY) ? 0.f : m_run;
      float lsum = 0.f;
      if (!special) {
        const float off = a.bias_log2 - mref;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t raw[32], pk[16];
          tmem_ld32(t_s + 32 * c, raw);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int key = 32 * c + 2 * k;
            const float p0 = ex2(fmaf(__uint_as_float(raw[2 * k]) * in.kscl[key], rowmul, off));
            const float p1 = ex2(fmaf(__uint_as_float(raw[2 * k + 1]) * in.kscl[key + 1], rowmul, off));
            lsum += p0 + p1;
            pk[k] = pack_bf16x2(p0 * in.vscl[key], p1 * in.vscl[key + 1]);
          }
          tmem_st16(t_s + 16 * c, pk);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t raw[32], pk[16];
          tmem_ld32(t_s + 32 * c, raw);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            float pp[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int key = 32 * c + 2 * k + e;
              const float tv = fmaf(__uint_as_float(raw[2 * k + e]) * in.kscl[key], rowmul, in.kb[key]);
              pp[e] = in.ktok[key] < lim ? ex2(tv - mref) : 0.f;
            }
            lsum += pp[0] + pp[1];
            pk[k] = pack_bf16x2(pp[0] * in.vscl[32 * c + 2 * k], pp[1] * in.vscl[32 * c + 2 * k + 1]);
          }
          tmem_st16(t_s + 16 * c, pk);
        }
      }
      l_run += lsum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars.pfull(g));
      mbar_arrive(bars.iempty(si));
    }
    // ------------------------------------------------------------ epilogue
    const bool ok = __all_sync(0xffffffffu, wait(bars.ofinal(), 0));
    tc_fence_after();
    const bool row_ok = gi < a.n_q;
    const bool any = j > 0;
    uint16_t* dst = a.out + ((size_t)(row_ok ? gi : 0) * a.H + h) * D;
    const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
#pragma unroll
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
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

int launch_attention_sm100_d128(const AttnArgs& a, const void* tmap_k_sw128, const void* tmap_v,
                                cudaStream_t s) {
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(chunk_attn_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Layout::bytes) != cudaSuccess)
      return KV_ECUDA;
    configured = true;
  }
  CUtensorMap mk, mv;
  memcpy(&mk, tmap_k_sw128, sizeof(mk));
  memcpy(&mv, tmap_v, sizeof(mv));
  dim3 grid((a.n_q + BM - 1) / BM, a.H);
  chunk_attn_sm100_kernel<<<grid, kThreads, Layout::bytes, s>>>(mk, mv, a);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

}  // namespace kvring
