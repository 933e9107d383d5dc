// chunk_attn.cu -- chunk attention over the FP8 ring ("Runway Characters: Serving a 57B
// Video Diffusion Transformer for Real-Time Conversation", abstract: every attention call
// reads the whole cache while only the newest tokens are new; "KREA Real-Time 14B /
// video-conductor", section "Plastic Windows": an additive cache-attention bias on
// history; "Stream LTX", section "Training": block-causal masks).
//
// One CTA = 128 query rows of one head, 4 warps; thread t owns query row t, which is
// also TMEM lane t.  Keys are visited in physical slot order in tiles of 128 slots
// (softmax attention does not depend on key order once bias and mask are per key), so
// the ring wrap costs nothing: a tile is a TMA box at (slot, head) and slots >= C read
// as zero.  Per tile:
//   TMA:      K and V e4m3 codes [128 slots][D] -> shared memory
//   convert:  codes -> bf16 (exact) into 128-byte-swizzled K-major panels
//   tcgen05:  S = Q K^T  (M=128, N=128, K=D; bf16 in, fp32 in TMEM)
//   softmax:  s = S * ks * scale*log2e + bias; mask; online max with lazy rescale of O
//             (only when the max grows by more than 8 in log2 units); P' = p * vs -> bf16
//   tcgen05:  O += P' V  (M=128, N=D, K=128; V read MN-major)
// Epilogue: out = O / l (bf16), lse = (m + log2 l) * ln 2.
#include <cuda.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "../../include/kvring.h"

namespace kvring {

namespace {

constexpr int BM = 128;          // query rows per CTA
constexpr int BN = 128;          // key slots per tile
constexpr int kThreads = 128;
constexpr uint32_t kPanel = 128u * 128u;   // bytes of one 64-column bf16 panel, 128 rows
constexpr float kRescaleLog2 = 8.0f;       // lazy-rescale threshold (factor 256)

template <int D>
struct Smem {
  static constexpr uint32_t q = 0;                        // bf16 Q   [D/64 panels]
  static constexpr uint32_t k = q + (D / 64) * kPanel;    // bf16 K tile
  static constexpr uint32_t v = k + (D / 64) * kPanel;    // bf16 V tile
  static constexpr uint32_t p = v + (D / 64) * kPanel;    // bf16 P   [2 panels]
  static constexpr uint32_t kc = p + 2 * kPanel;          // e4m3 K codes [BN][D]
  static constexpr uint32_t vc = kc + BN * D;             // e4m3 V codes
  static constexpr uint32_t kscl = vc + BN * D;           // float[BN]
  static constexpr uint32_t kbias = kscl + 4 * BN;        // float[BN]
  static constexpr uint32_t ktok = kbias + 4 * BN;        // int[BN]
  static constexpr uint32_t vscl = ktok + 4 * BN;         // float[BN]
  static constexpr uint32_t bars = vscl + 4 * BN;         // 2 x uint64
  static constexpr uint32_t tmem = bars + 16;             // uint32
  static constexpr uint32_t flag = tmem + 4;
  static constexpr uint32_t bytes = flag + 4 + 1024;      // + slack for 1024 alignment
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Convert 16 e4m3 codes (one uint4) to 16 bf16 values packed in two uint4.
__device__ __forceinline__ void codes16_to_bf16(uint4 c, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 a = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[i] & 0xFFFFu)));
    const float2 b = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[i] >> 16)));
    o[2 * i] = pack_bf16x2(a.x, a.y);
    o[2 * i + 1] = pack_bf16x2(b.x, b.y);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// Does physical tile [t*BN, t*BN+BN) hold a valid slot?  Valid slots are the n_valid
// slots ending at newest (mod C).
__device__ __forceinline__ bool tile_has_valid(int64_t t, int64_t C, int64_t newest,
                                               int64_t n_valid) {
  if (n_valid <= 0) return false;
  if (n_valid >= C) return true;
  const int64_t a = t * BN, b = min(C, a + BN);
  int64_t first = newest - n_valid + 1;
  if (first >= 0) return a <= newest && b > first;
  first += C;  // wrapped: [first, C) and [0, newest]
  return (b > first) || (a <= newest);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_attn_kernel(const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const AttnArgs a) {
  using S = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic on the shared array (an integer round trip
  // would hide from the compiler that sm addresses shared memory)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* kscl = reinterpret_cast<float*>(sm + S::kscl);
  float* kbias = reinterpret_cast<float*>(sm + S::kbias);
  int* ktok = reinterpret_cast<int*>(sm + S::ktok);
  float* vscl = reinterpret_cast<float*>(sm + S::vscl);
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(sm + S::bars);
  uint64_t* mma_bar = tma_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S::tmem);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int h = blockIdx.y;
  const int q0 = blockIdx.x * BM;
  const int64_t C = a.C;

  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(tma_bar, 1);
    mbar_init(mma_bar, 1);
    fence_mbar_init();
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
  }

  // ---- Q prologue: rotate row q0+tid at q_pos0+q0+tid, round to bf16, swizzle into smem
  {
    const int gi = q0 + tid;
    uint8_t* sq = sm + S::q;
    if (gi < a.n_q) {
      const uint4* src = reinterpret_cast<const uint4*>(a.q + ((size_t)gi * a.H + h) * D);
      const float4* tb = reinterpret_cast<const float4*>(a.rope_q0 + (size_t)gi * D);
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
        const uint4 raw = __ldg(src + c);
        const float4 cs0 = __ldg(tb + 2 * c), cs1 = __ldg(tb + 2 * c + 1);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        const float cc[4] = {cs0.x, cs0.z, cs1.x, cs1.z};
        const float ss[4] = {cs0.y, cs0.w, cs1.y, cs1.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float x0 = bf16_bits_to_float(w[j] & 0xFFFFu);
          const float x1 = bf16_bits_to_float(w[j] >> 16);
          const float y0 = sub_rn(mul_rn(x0, cc[j]), mul_rn(x1, ss[j]));
          const float y1 = add_rn(mul_rn(x0, ss[j]), mul_rn(x1, cc[j]));
          o[j] = pack_bf16x2(y0, y1);
        }
        *reinterpret_cast<uint4*>(sq + sw128_offset(tid, 8 * c, kPanel)) =
            make_uint4(o[0], o[1], o[2], o[3]);
      }
    } else {
      for (int c = 0; c < D / 8; ++c)
        *reinterpret_cast<uint4*>(sq + sw128_offset(tid, 8 * c, kPanel)) = make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t t_s = tmem + lane_base;          // S: columns [0, 128)
  const uint32_t t_o = tmem + lane_base + 128;    // O: columns [128, 128 + D)

  // O = 0
  {
    uint32_t z[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) tmem_st32(t_o + 32 * c, z);
    tmem_wait_st();
  }

  // query row constants
  const int gi = q0 + tid;
  int lim;   // current-chunk keys with token index < lim are visible to this row
  {
    const int64_t qb = gi < a.q_first ? 0 : 1 + (int64_t)(gi - a.q_first) / a.q_block;
    const int64_t l = (int64_t)a.k_first + qb * (int64_t)a.k_block;
    lim = (int)(l < (int64_t)a.n_current ? l : (int64_t)a.n_current);
  }
  float m_run = -INFINITY, l_run = 0.f;

  const uint32_t sQ = smem_u32(sm + S::q), sK = smem_u32(sm + S::k), sV = smem_u32(sm + S::v),
                 sP = smem_u32(sm + S::p);
  constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);
  constexpr uint32_t idO = idesc_bf16_f32(BM, D, 0, 1);

  uint32_t tma_phase = 0, mma_phase = 0;
  bool ok = true;
  const int64_t n_tiles = (C + BN - 1) / BN;
  for (int64_t t = 0; t < n_tiles && ok; ++t) {
    if (!tile_has_valid(t, C, a.newest_slot, a.n_valid)) continue;
    if (tid == 0) {
      mbar_arrive_expect_tx(tma_bar, 2u * BN * D);
      tma_load_3d(sm + S::kc, &tmk, tma_bar, 0, (int)(t * BN), h);
      tma_load_3d(sm + S::vc, &tmv, tma_bar, 0, (int)(t * BN), h);
    }
    // per-key classification of slot t*BN + tid
    {
      const int64_t slot = t * BN + tid;
      float ksv = 0.f, bsv = -INFINITY, vsv = 0.f;
      int tok = 0x7FFFFFFF;
      if (slot < C) {
        int64_t age = a.newest_slot - slot;
        if (age < 0) age += C;
        if (age < a.n_valid) {
          ksv = a.k_scale[(size_t)h * C + slot] * a.score_scale_log2;
          vsv = a.v_scale[(size_t)h * C + slot];
          if (age < a.n_current) {
            bsv = 0.f;
            tok = (int)(a.n_current - 1 - age);
          } else {
            bsv = a.bias_log2;
            tok = -1;
          }
        }
      }
      kscl[tid] = ksv;
      kbias[tid] = bsv;
      ktok[tid] = tok;
      vscl[tid] = vsv;
    }
    ok = mbar_wait(tma_bar, tma_phase, a.timeouts);
    tma_phase ^= 1u;
    ok = __syncthreads_and(ok);
    if (!ok) break;

    // codes -> bf16 panels (invalid slots become zero rows)
    {
      constexpr int CPR = D / 16;   // 16-code chunks per row
      const uint8_t* kc = sm + S::kc;
      const uint8_t* vc = sm + S::vc;
      uint8_t* sk = sm + S::k;
      uint8_t* sv = sm + S::v;
#pragma unroll 2
      for (int idx = tid; idx < BN * CPR; idx += kThreads) {
        const int row = idx / CPR, c = idx % CPR;
        uint4 ck = *reinterpret_cast<const uint4*>(kc + row * D + 16 * c);
        uint4 cv = *reinterpret_cast<const uint4*>(vc + row * D + 16 * c);
        if (ktok[row] == 0x7FFFFFFF) {
          ck = make_uint4(0, 0, 0, 0);
          cv = ck;
        }
        uint4 lo, hi;
        codes16_to_bf16(ck, lo, hi);
        *reinterpret_cast<uint4*>(sk + sw128_offset(row, 16 * c, kPanel)) = lo;
        *reinterpret_cast<uint4*>(sk + sw128_offset(row, 16 * c + 8, kPanel)) = hi;
        codes16_to_bf16(cv, lo, hi);
        *reinterpret_cast<uint4*>(sv + sw128_offset(row, 16 * c, kPanel)) = lo;
        *reinterpret_cast<uint4*>(sv + sw128_offset(row, 16 * c + 8, kPanel)) = hi;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // S = Q K^T
    if (tid < 32) {                                   // warp 0; one elected lane issues
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
        el_mma_f16_ss(tmem, smem_desc_sw128(sQ + off, 16, 1024),
                      smem_desc_sw128(sK + off, 16, 1024), idS, kk > 0);
      }
      el_commit(mma_bar);
    }
    ok = mbar_wait(mma_bar, mma_phase, a.timeouts);
    mma_phase ^= 1u;
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();

    // ---- softmax of row tid over this tile
    {
      uint32_t raw[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(t_s + 32 * c, raw[c]);
      tmem_wait_ld();
      float mloc = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int key = 32 * c + j;
          float s = fmaf(__uint_as_float(raw[c][j]), kscl[key], kbias[key]);
          s = (ktok[key] >= lim) ? -INFINITY : s;
          raw[c][j] = __float_as_uint(s);
          mloc = fmaxf(mloc, s);
        }
      }
      // lazy rescale: move the reference max only when it grows by more than 2^8.
      // tcgen05.ld/st are warp-collective, so the warp rescales together when any of its
      // rows needs it (alpha = 1 for the others).
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
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(t_o + 32 * c, o);
        }
        tmem_wait_st();
      }
      if (move) {
        l_run *= alpha;
        m_run = mloc;
      }
      const float mref = (m_run == -INFINITY) ? 0.f : m_run;
      float lsum = 0.f;
      uint8_t* sp = sm + S::p;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {    // 8 keys -> one 16-byte chunk of P
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int k0 = 8 * g + 2 * j;
            const float p0 = ex2(__uint_as_float(raw[c][k0]) - mref);
            const float p1 = ex2(__uint_as_float(raw[c][k0 + 1]) - mref);
            lsum += p0 + p1;
            w[j] = pack_bf16x2(p0 * vscl[32 * c + k0], p1 * vscl[32 * c + k0 + 1]);
          }
          *reinterpret_cast<uint4*>(sp + sw128_offset(tid, 32 * c + 8 * g, kPanel)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      l_run += lsum;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // O += P' V
    if (tid < 32) {                                   // warp 0; one elected lane issues
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        const uint32_t pa = sP + (kk >> 2) * kPanel + (kk & 3) * 32;   // K-major P
        const uint32_t vb = sV + kk * 2048;                            // 16 keys = 2 atoms
        el_mma_f16_ss(tmem + 128, smem_desc_sw128(pa, 16, 1024),
                      smem_desc_sw128(vb, kPanel, 1024), idO, 1);
      }
      el_commit(mma_bar);
    }
    ok = mbar_wait(mma_bar, mma_phase, a.timeouts);
    mma_phase ^= 1u;
    ok = __syncthreads_and(ok);
    tc_fence_after();
  }

  // ---- epilogue (TMEM loads by every lane: they are warp-collective)
  {
    const bool row_ok = gi < a.n_q;
    uint16_t* dst = a.out + ((size_t)(row_ok ? gi : 0) * a.H + h) * D;
    const float inv_l = (ok && l_run > 0.f) ? 1.f / l_run : 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(t_o + 32 * c, o);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float x0 = __uint_as_float(o[2 * j]) * inv_l, x1 = __uint_as_float(o[2 * j + 1]) * inv_l;
        if (!ok) x0 = x1 = __uint_as_float(0x7FC00000u);
        pk[j] = pack_bf16x2(x0, x1);
      }
      if (row_ok) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          d4[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
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
    tmem_dealloc(tmem, 256);
  }
}

template <int D>
int launch_d(const AttnArgs& a, const void* tk, const void* tv, cudaStream_t s) {
  using S = Smem<D>;
  static unsigned char configured[kMaxDevices] = {};
  if (!smem_attr_set(reinterpret_cast<const void*>(chunk_attn_kernel<D>), (int)S::bytes,
                     configured))
    return KV_ECUDA;
  CUtensorMap mk, mv;
  memcpy(&mk, tk, sizeof(mk));
  memcpy(&mv, tv, sizeof(mv));
  dim3 grid((a.n_q + BM - 1) / BM, a.H);
  chunk_attn_kernel<D><<<grid, kThreads, S::bytes, s>>>(mk, mv, a);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

}  // namespace

int launch_attention(const AttnArgs& a, int D, const void* tmap_k, const void* tmap_v,
                     const void* tmap_k_sw128, const void* tmap_v_sw128, cudaStream_t s) {
  if (D == 128) return launch_attention_sm100_d128(a, tmap_k_sw128, tmap_v_sw128, s);
  return launch_d<64>(a, tmap_k, tmap_v, s);
}

}  // namespace kvring
