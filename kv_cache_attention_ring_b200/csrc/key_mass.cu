// key_mass.cu -- attention mass received by history keys, and the content memory's top-M
// selection ("Stream LTX", Inference: the long-context cache is an anchor, a content
// memory and a FIFO of recent blocks; each layer scores its own keys on attention quality
// and temporal diversity and evicts down to a top-M budget).
//
// key_mass_kernel: mass_h[h][c] = sum over query rows i of exp(s_ihc - lse_ih), the
// probability head h of row i gives candidate key c in the attention call whose
// log-sum-exp `lse` the caller passes.  One launch may score several candidate sets of
// that call (their CTAs side by side in the grid).  One CTA takes 4 groups of 128
// candidate keys of one set and head (512 threads) and computes S^T = K Q^T on the tensor core (M = 128 keys per
// group, N = 128 queries per tile, the query split exactly into e4m3 hi + lo as in the
// attention kernel, once per tile for all 512 keys), so every thread owns one key as its
// tensor-memory lane and sums its own row: no cross-thread reduction.
//
// memory_select_kernel: one CTA ranks the candidates (quality = sum over heads of the
// masses; the k-th best key of a frame scores quality * gamma^k; ties toward the lower
// position, then the lower candidate index) and keeps the best M, written as a list of
// source (ring, slot) in ascending candidate order.  memory_gather_kernel copies them
// (K and V codes, scales, positions) into the new memory ring's slots 0 .. kept - 1.
#include <cuda.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "../../include/kvring.h"

namespace kvring {

namespace {

constexpr int D = 128;
constexpr int KM = 128;          // candidate keys per group (tensor-memory lanes)
constexpr int KG = 4;            // groups per CTA: 512 candidates share each query tile's split
constexpr int QN = 128;          // query rows per tile (MMA N)
constexpr int kThreads = 32 * 4 * KG;   // warp w: lane quadrant w % 4 of group w / 4

struct MassLayout {
  static constexpr uint32_t k = 0;                    // KG x e4m3 [128 keys][128], sw128
  static constexpr uint32_t qhi = k + KG * KM * D;    // e4m3 [128 queries][128], sw128
  static constexpr uint32_t qlo = qhi + QN * D;
  static constexpr uint32_t rq = qlo + QN * D;        // per query: r (the split's power of two)
  static constexpr uint32_t lq = rq + QN * 4;         // per query: lse * log2(e), or +inf
  static constexpr uint32_t bar = lq + QN * 4;        // one mbarrier
  static constexpr uint32_t misc = bar + 8;           // tmem address, abort flag
  static constexpr uint32_t bytes = misc + 8 + 1024;  // + alignment slack
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One lane of a query row's group of 8 lanes (16 elements each): row i of head h rotated
// with the main ring's table, rounded to bf16 and split exactly into e4m3 hi + lo with the
// row's power of two r = 2^k (zeros for i >= n_q).  All 8 lanes of the group call it
// together: the row maximum is shuffled among them.
__device__ __forceinline__ void q_split_lane(const KeyMassArgs& a, int i, int h, int lc,
                                             uint32_t (&hw)[4], uint32_t (&lw)[4], int& k) {
  float y[16];
  if (i < a.n_q) {
    const uint4* qp = reinterpret_cast<const uint4*>(a.q + ((size_t)i * a.H + h) * D + 16 * lc);
    const uint4 q0v = __ldg(qp), q1v = __ldg(qp + 1);
    const float4* tb = reinterpret_cast<const float4*>(a.rope_q0 + (size_t)i * D + 16 * lc);
    const uint32_t w[8] = {q0v.x, q0v.y, q0v.z, q0v.w, q1v.x, q1v.y, q1v.z, q1v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 cs = __ldg(tb + j);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t pr = w[2 * j + u];
        const float c = u ? cs.z : cs.x, s = u ? cs.w : cs.y;
        const float x0 = bf16_bits_to_float(pr & 0xFFFFu), x1 = bf16_bits_to_float(pr >> 16);
        const uint32_t b = pack_bf16x2(sub_rn(mul_rn(x0, c), mul_rn(x1, s)),
                                       add_rn(mul_rn(x0, s), mul_rn(x1, c)));
        y[4 * j + 2 * u] = bf16_bits_to_float(b & 0xFFFFu);
        y[4 * j + 2 * u + 1] = bf16_bits_to_float(b >> 16);
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) y[e] = 0.f;
  }
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) amax = max_nan(amax, fabsf(y[e]));
#pragma unroll
  for (int off = 4; off > 0; off >>= 1) amax = max_nan(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  k = 0;
  if (amax > 0.f && amax <= 3.402823466e38f) {
    int e;
    const float m = frexpf(amax, &e);
    k = max(-126, min(127, (e - 1) - 8 + (m > 0.875f ? 1 : 0)));
  }
  const float inv_r = ldexpf(1.f, -k);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float x[4], lv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = y[4 * j + e] * inv_r;
    const uint32_t h01 = e4m3x2(x[0], x[1]), h23 = e4m3x2(x[2], x[3]);
    const float2 d01 = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)h01));
    const float2 d23 = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)h23));
    lv[0] = x[0] - d01.x;
    lv[1] = x[1] - d01.y;
    lv[2] = x[2] - d23.x;
    lv[3] = x[3] - d23.y;
    hw[j] = h01 | (h23 << 16);
    lw[j] = e4m3x2(lv[0], lv[1]) | (e4m3x2(lv[2], lv[3]) << 16);
  }
}

__global__ void __launch_bounds__(kThreads, 1) key_mass_kernel(const KeyMassArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic on the shared array (an integer round trip
  // would hide from the compiler that sm addresses shared memory)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + MassLayout::bar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + MassLayout::misc);
  float* rq = reinterpret_cast<float*>(sm + MassLayout::rq);
  float* lq = reinterpret_cast<float*>(sm + MassLayout::lq);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp >> 2, quad = warp & 3;
  const int krow = 32 * quad + lane;                   // TMEM lane = row in group grp
  const int h = blockIdx.y;
  int set = 0;                                         // candidate set of this CTA
  while (set + 1 < a.n_sets && (int)blockIdx.x >= a.blk_first[set + 1]) ++set;
  const int n_cand = a.n_cand[set], C = a.C[set];
  const int c = ((int)blockIdx.x - a.blk_first[set]) * (KG * KM) + grp * KM + krow;
  const bool live_c = c < n_cand;                      // this thread's candidate

  if (warp == 0) {
    tmem_alloc(tmem_slot, KG * 128);
    tmem_relinquish();
  }
  if (tid == 32) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  // candidate key row: 8 16-byte chunks into the swizzled K-major operand (zero past the
  // candidates); its scale times softmax_scale * log2(e)
  float kscl = 0.f;
  {
    uint4 w[8];
    if (live_c) {
      int slot = a.slot_first[set] + c;
      slot = slot >= C ? slot - C : slot;
      const uint4* src = reinterpret_cast<const uint4*>(a.kc[set] + ((size_t)h * C + slot) * D);
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = __ldg(src + i);
      kscl = __ldg(a.ks[set] + (size_t)h * C + slot) * a.score_scale_log2;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    uint8_t* krow_sm = sm + MassLayout::k + grp * KM * D + krow * 128;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *reinterpret_cast<uint4*>(krow_sm + ((i ^ (krow & 7)) << 4)) = w[i];
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
  constexpr uint32_t idS = idesc_e4m3_f32(KM, QN);
  const uint64_t dK = smem_desc_sw128(smem_u32(sm + MassLayout::k), 16, 1024);
  const uint64_t dQhi = smem_desc_sw128(smem_u32(sm + MassLayout::qhi), 16, 1024);
  const uint64_t dQlo = smem_desc_sw128(smem_u32(sm + MassLayout::qlo), 16, 1024);

  float acc = 0.f;
  bool ok = true;
  const int lc = tid & 7;                              // prologue: 8 lanes per query row
  int phase = 0;
  for (int q0 = 0; q0 < a.n_q && ok; q0 += QN, phase ^= 1) {
    // query tile: rotate, round to bf16, split exactly into e4m3 hi + lo (per-row power
    // of two r), 16 rows per pass of the 128 threads
    for (int rr = tid >> 3; rr < QN; rr += kThreads / 8) {
      const int i = q0 + rr;
      uint32_t hw[4], lw[4];
      int k;
      q_split_lane(a, i, h, lc, hw, lw, k);
      const uint32_t off = (uint32_t)rr * 128u + ((uint32_t)(lc ^ (rr & 7)) << 4);
      *reinterpret_cast<uint4*>(sm + MassLayout::qhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(sm + MassLayout::qlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      if (lc == 0) {
        // rows past n_q, rows that attended nothing (lse not finite): no contribution
        const float l = i < a.n_q ? __ldg(a.lse + (size_t)h * a.n_q + i) : INFINITY;
        const bool use = isfinite(l);
        rq[rr] = use ? ldexpf(1.f, k) : 0.f;
        lq[rr] = use ? l * 1.4426950408889634f : INFINITY;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid < 32) {                                   // warp 0; one elected lane issues
#pragma unroll
      for (int gg = 0; gg < KG; ++gg) {
        const uint64_t kd = dK + ((gg * KM * D) >> 4);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const uint64_t qd = hf == 0 ? dQhi : dQlo;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            el_mma_f8_ss(tmem + 128 * gg, kd + 2 * kk, qd + 2 * kk, idS, (hf | kk) != 0);
        }
      }
      el_commit(bar);
    }
    ok = mbar_wait(bar, phase, a.timeouts);
    tc_fence_after();
    if (__all_sync(0xffffffffu, ok)) {
#pragma unroll 1
      for (int cb = 0; cb < QN; cb += 32) {
        uint32_t sr[32];
        tmem_ld32(tmem + lane_base + 128 * grp + cb, sr);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          // s' = S kscl r + bias - lse (log2 units); 2^-inf = 0 for unused rows
          const float t = fmaf(__uint_as_float(sr[u]) * kscl, rq[cb + u], a.bias_log2) - lq[cb + u];
          acc += ex2f(t);
        }
      }
    }
    tc_fence_before();
    ok = __syncthreads_and(ok);
    tc_fence_after();
  }
  if (!ok) {
    mbar_wait(bar, phase ^ 1, a.timeouts);             // bounded: let an issued MMA land
    acc = __uint_as_float(0x7FC00000u);
  }
  if (live_c) a.mass[set][(size_t)h * n_cand + c] = acc;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, KG * 128);
  }
}

// ------------------------------------------------------------------ pipelined key mass
// With a caller workspace the query split runs once per call instead of once per CTA:
// key_mass_qsplit_kernel writes, per head and tile of 64 query rows, the image the MMA
// reads (hi and lo codes, K-major with the 128-byte swizzle, then r and lse * log2(e) per
// row); key_mass_pipe_kernel streams those images into shared memory with bulk copies,
// NQS tiles ahead, and double-buffers S in tensor memory, so that the MMAs of tile t + 1
// run while the threads sum tile t.  One warp per key group issues that group's eight
// MMAs (a single issuer for all 32 held every other warp at the tile barrier).  Each
// candidate's sum runs over the queries in the same order as in key_mass_kernel.
constexpr int QT = 64;                       // query rows per pipelined tile (MMA N)
constexpr int NQS = 3;                       // tile images in flight
struct QTile {                               // one (head, tile) image, workspace and smem
  static constexpr uint32_t hi = 0;                   // e4m3 [64 queries][128], sw128
  static constexpr uint32_t lo = QT * D;
  static constexpr uint32_t rq = 2 * QT * D;          // per query: r, or 0
  static constexpr uint32_t lq = rq + QT * 4;         // per query: lse * log2(e), or +inf
  static constexpr uint32_t bytes = lq + QT * 4;      // 16,896 (a multiple of 16)
};
struct PipeLayout {
  static constexpr uint32_t k = 0;                    // KG x e4m3 [128 keys][128], sw128
  static constexpr uint32_t qstride = (QTile::bytes + 1023u) & ~1023u;
  static constexpr uint32_t q = k + KG * KM * D;      // NQS tile images, 1024-aligned
  static constexpr uint32_t bar = q + NQS * qstride;  // qfull[NQS], sfull[2]
  static constexpr uint32_t misc = bar + 8 * (NQS + 2);   // tmem address, abort flag
  static constexpr uint32_t bytes = misc + 8 + 1024;      // + alignment slack
};

__global__ void __launch_bounds__(512) key_mass_qsplit_kernel(const KeyMassArgs a) {
  const int t = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int rr = tid >> 3, lc = tid & 7, i = t * QT + rr;
  uint8_t* img = a.qws + ((size_t)h * a.n_qt + t) * QTile::bytes;
  uint32_t hw[4], lw[4];
  int k;
  q_split_lane(a, i, h, lc, hw, lw, k);
  const uint32_t off = (uint32_t)rr * 128u + ((uint32_t)(lc ^ (rr & 7)) << 4);
  *reinterpret_cast<uint4*>(img + QTile::hi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  *reinterpret_cast<uint4*>(img + QTile::lo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  if (lc == 0) {
    // rows past n_q, rows that attended nothing (lse not finite): no contribution
    const float l = i < a.n_q ? __ldg(a.lse + (size_t)h * a.n_q + i) : INFINITY;
    const bool use = isfinite(l);
    reinterpret_cast<float*>(img + QTile::rq)[rr] = use ? ldexpf(1.f, k) : 0.f;
    reinterpret_cast<float*>(img + QTile::lq)[rr] = use ? l * 1.4426950408889634f : INFINITY;
  }
}

__global__ void __launch_bounds__(kThreads, 1) key_mass_pipe_kernel(const KeyMassArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic on the shared array (an integer round trip
  // would hide from the compiler that sm addresses shared memory)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* qfull = reinterpret_cast<uint64_t*>(sm + PipeLayout::bar);
  uint64_t* sfull = qfull + NQS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + PipeLayout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + PipeLayout::misc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp >> 2, quad = warp & 3;
  const int krow = 32 * quad + lane;                   // TMEM lane = row in group grp
  const int h = blockIdx.y;
  int set = 0;                                         // candidate set of this CTA
  while (set + 1 < a.n_sets && (int)blockIdx.x >= a.blk_first[set + 1]) ++set;
  const int n_cand = a.n_cand[set], C = a.C[set];
  const int c = ((int)blockIdx.x - a.blk_first[set]) * (KG * KM) + grp * KM + krow;
  const bool live_c = c < n_cand;                      // this thread's candidate
  const int n_t = a.n_qt;

  if (warp == 0) {
    tmem_alloc(tmem_slot, 2 * KG * QT);                // S double-buffered: 512 columns
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int st = 0; st < NQS; ++st) mbar_init(&qfull[st], 1);
    mbar_init(&sfull[0], KG);                          // one commit per group's issuer
    mbar_init(&sfull[1], KG);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // candidate key row, as in key_mass_kernel
  float kscl = 0.f;
  {
    uint4 w[8];
    if (live_c) {
      int slot = a.slot_first[set] + c;
      slot = slot >= C ? slot - C : slot;
      const uint4* src = reinterpret_cast<const uint4*>(a.kc[set] + ((size_t)h * C + slot) * D);
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = __ldg(src + i);
      kscl = __ldg(a.ks[set] + (size_t)h * C + slot) * a.score_scale_log2;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    uint8_t* krow_sm = sm + PipeLayout::k + grp * KM * D + krow * 128;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *reinterpret_cast<uint4*>(krow_sm + ((i ^ (krow & 7)) << 4)) = w[i];
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
  const uint8_t* img0 = a.qws + (size_t)h * n_t * QTile::bytes;
  int n_loads = 0;                                     // thread 0: tile images requested
  auto load = [&](int t) {
    uint8_t* dst = sm + PipeLayout::q + (t % NQS) * PipeLayout::qstride;
    mbar_arrive_expect_tx(&qfull[t % NQS], QTile::bytes);
    bulk_load(dst, img0 + (size_t)t * QTile::bytes, QTile::bytes, &qfull[t % NQS]);
    n_loads = t + 1;
  };
  if (tid == 0)
    for (int t = 0; t < NQS && t < n_t; ++t) load(t);

  constexpr uint32_t idS = idesc_e4m3_f32(KM, QT);
  const uint64_t dK = smem_desc_sw128(smem_u32(sm + PipeLayout::k), 16, 1024);
  // warp 5 g of group g (one per SM sub-partition), converged: S_g(t) = K_g Q(t)^T into
  // buffer t & 1 once tile t's image has landed
  const bool issuer = warp == 5 * grp;
  int n_mma = 0;                                       // issuers: tiles whose MMAs went out
  auto issue = [&](int t) -> bool {
    if (!mbar_wait_warp(&qfull[t % NQS], (t / NQS) & 1, abort_flag, a.timeouts)) return false;
    tc_fence_after();
    const uint32_t qs = smem_u32(sm + PipeLayout::q + (t % NQS) * PipeLayout::qstride);
    const uint64_t dQhi = smem_desc_sw128(qs + QTile::hi, 16, 1024);
    const uint64_t dQlo = smem_desc_sw128(qs + QTile::lo, 16, 1024);
    const uint64_t kd = dK + ((grp * KM * D) >> 4);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint64_t qd = hf == 0 ? dQhi : dQlo;
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk)
        el_mma_f8_ss(tmem + KG * QT * (t & 1) + QT * grp, kd + 2 * kk, qd + 2 * kk, idS,
                     (hf | kk) != 0);
    }
    el_commit(&sfull[t & 1]);
    n_mma = t + 1;
    return true;
  };

  float acc = 0.f;
  bool ok = true;
  if (issuer && n_t > 0) ok = issue(0);
  for (int t = 0; t < n_t; ++t) {
    // S(t + 1) goes into the buffer every thread finished reading before the last barrier
    if (issuer && ok && t + 1 < n_t) ok = issue(t + 1);
    // S(t), and tile t's image itself (its r and lse are read below; complete already)
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      if (mbar_try_wait(bar, parity)) return true;
      if (*abort_flag) return false;
      if (mbar_wait(bar, parity, a.timeouts)) return true;
      *abort_flag = 1;
      return false;
    };
    bool got = wait(&sfull[t & 1], (t >> 1) & 1) && wait(&qfull[t % NQS], (t / NQS) & 1);
    tc_fence_after();
    if (__all_sync(0xffffffffu, got)) {
      const uint8_t* img = sm + PipeLayout::q + (t % NQS) * PipeLayout::qstride;
      const float4* rq4 = reinterpret_cast<const float4*>(img + QTile::rq);
      const float4* lq4 = reinterpret_cast<const float4*>(img + QTile::lq);
#pragma unroll 1
      for (int cb = 0; cb < QT; cb += 32) {
        uint32_t sr[32];
        tmem_ld32(tmem + lane_base + KG * QT * (t & 1) + QT * grp + cb, sr);
        tmem_wait_ld();
#pragma unroll
        for (int u4 = 0; u4 < 8; ++u4) {
          const float4 r = rq4[cb / 4 + u4], l = lq4[cb / 4 + u4];
          const float rr[4] = {r.x, r.y, r.z, r.w}, ll[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // s' = S kscl r + bias - lse (log2 units); 2^-inf = 0 for unused rows
            const float x = fmaf(__uint_as_float(sr[4 * u4 + e]) * kscl, rr[e], a.bias_log2) - ll[e];
            acc += ex2f(x);
          }
        }
      }
    }
    tc_fence_before();
    ok = __syncthreads_and(ok && got);
    if (!ok) break;
    // tile t's image is free (its MMAs completed before sfull(t) did): refill it
    if (tid == 0 && t + NQS < n_t) load(t + NQS);
  }
  if (!ok) {
    // abandoned: wait (bounded) for the copies and MMAs this CTA issued, the last of
    // each barrier standing for every earlier one on it (an S phase that another issuer
    // never committed to ends the wait by its time limit)
    if (tid == 0)
      for (int u = max(0, n_loads - NQS); u < n_loads; ++u)
        mbar_wait(&qfull[u % NQS], (u / NQS) & 1, a.timeouts);
    if (issuer && lane == 0)
      for (int u = max(0, n_mma - 2); u < n_mma; ++u)
        mbar_wait(&sfull[u & 1], (u >> 1) & 1, a.timeouts);
    acc = __uint_as_float(0x7FC00000u);
  }
  if (live_c) a.mass[set][(size_t)h * n_cand + c] = acc;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * KG * QT);
  }
}

// ------------------------------------------------------------------ selection
constexpr int kSelThreads = 1024;

// Candidates of a selection: quality (then score), index, position, frame; 16 bytes, kept in
// shared memory.  Positions are the rings' int32 slot positions, so frames fit in 32 bits.
struct __align__(16) Cand {
  float q;
  int idx;
  int pos;
  int frame;
};

// (frame asc, quality desc, position asc, index asc)
__device__ __forceinline__ bool before_in_frame(const Cand& x, const Cand& y) {
  if (x.frame != y.frame) return x.frame < y.frame;
  if (x.q != y.q) return x.q > y.q;
  if (x.pos != y.pos) return x.pos < y.pos;
  return x.idx < y.idx;
}

// Bitonic sort of n_pow2 <= EPT * kSelThreads entries of v (padding entries sort last), all
// threads.  Thread t holds entries EPT t .. EPT t + EPT - 1 in registers: pairs closer than
// EPT entries are exchanged in registers, pairs up to 16 EPT apart through warp shuffles,
// and only the wider strides go through shared memory (one barrier each).
__device__ __forceinline__ Cand shfl_cand(const Cand& c, int lane_mask) {
  Cand o;
  o.q = __shfl_xor_sync(0xffffffffu, c.q, lane_mask);
  o.idx = __shfl_xor_sync(0xffffffffu, c.idx, lane_mask);
  o.pos = __shfl_xor_sync(0xffffffffu, c.pos, lane_mask);
  o.frame = __shfl_xor_sync(0xffffffffu, c.frame, lane_mask);
  return o;
}
template <int EPT>
__device__ void bitonic(Cand* v, int n_pow2) {
  const int tid = threadIdx.x;
  const bool live = EPT * tid < n_pow2;                // threads past the entries idle
  Cand x[EPT];
#pragma unroll
  for (int k = 0; k < EPT; ++k) x[k] = live ? v[EPT * tid + k] : v[0];
  for (int size = 2; size <= n_pow2; size <<= 1) {
    int stride = size >> 1;
    if (stride >= 32 * EPT) {                          // wide strides: shared memory
      if (live) {
#pragma unroll
        for (int k = 0; k < EPT; ++k) v[EPT * tid + k] = x[k];
      }
      __syncthreads();
      for (; stride >= 32 * EPT; stride >>= 1) {
        for (int t = tid; t < (n_pow2 >> 1); t += blockDim.x) {
          const int i = ((t & ~(stride - 1)) << 1) | (t & (stride - 1));
          const int j = i + stride;
          const Cand a = v[i], b = v[j];
          const bool up = (i & size) == 0;
          if (up ? before_in_frame(b, a) : before_in_frame(a, b)) {
            v[i] = b;
            v[j] = a;
          }
        }
        __syncthreads();
      }
      if (live) {
#pragma unroll
        for (int k = 0; k < EPT; ++k) x[k] = v[EPT * tid + k];
      }
      __syncthreads();
    }
    for (; stride >= EPT; stride >>= 1) {              // within the warp: shuffles
#pragma unroll
      for (int k = 0; k < EPT; ++k) {
        const int e = EPT * tid + k;
        const Cand o = shfl_cand(x[k], stride / EPT);
        const bool lower = (e & stride) == 0, up = (e & size) == 0;
        const bool mine_first = before_in_frame(x[k], o);
        // the lower entry keeps the first of the pair (descending runs: the last)
        const bool keep_mine = (lower == up) ? mine_first : !mine_first;
        if (live && !keep_mine) x[k] = o;
      }
    }
    // within the thread: the strides below EPT
    auto cx = [&](Cand& a, Cand& b, int e) {
      const bool up = (e & size) == 0;
      if (up ? before_in_frame(b, a) : before_in_frame(a, b)) {
        const Cand t = a;
        a = b;
        b = t;
      }
    };
#pragma unroll
    for (int s = EPT / 2; s >= 1; s >>= 1) {
      if (s < size) {
#pragma unroll
        for (int k = 0; k < EPT; ++k)
          if ((k & s) == 0) cx(x[k], x[k + s], EPT * tid + k);
      }
    }
  }
  if (live) {
#pragma unroll
    for (int k = 0; k < EPT; ++k) v[EPT * tid + k] = x[k];
  }
  __syncthreads();
}

// Block-wide inclusive max-scan of one int per thread (kSelThreads threads).
__device__ int block_max_scan(int x, int* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x = max(x, y);
  }
  if (lane == 31) red[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int w = red[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w = max(w, y);
    }
    red[lane] = w;
  }
  __syncthreads();
  const int r = wid > 0 ? max(x, red[wid - 1]) : x;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kSelThreads) memory_select_kernel(const SelectArgs a) {
  extern __shared__ uint8_t smem_raw[];
  Cand* v = reinterpret_cast<Cand*>(smem_raw);
  __shared__ int red[32];
  __shared__ uint32_t kbits[KV_MEMORY_MAX_CANDIDATES / 32];
  __shared__ int wpre[KV_MEMORY_MAX_CANDIDATES / 32];
  __shared__ int hist[256];
  __shared__ int sel[3];
  const int tid = threadIdx.x;
  const int n = a.n_mem + a.n_fifo;
  int n_pow2 = 4;                                    // at least one thread's four entries
  while (n_pow2 < n) n_pow2 <<= 1;
  for (int i = tid; i < n_pow2; i += blockDim.x) {
    Cand c;
    if (i < n) {
      const bool mem = i < a.n_mem;
      const float* m = mem ? a.mass_mem : a.mass_fifo;
      const int ci = mem ? i : i - a.n_mem;
      const int nc = mem ? a.n_mem : a.n_fifo;
      // quality: the heads' masses added in head order; loads issued eight at a time
      float q = 0.f;
      for (int h0 = 0; h0 < a.H; h0 += 8) {
        float t[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) t[u] = h0 + u < a.H ? __ldg(m + (size_t)(h0 + u) * nc + ci) : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (h0 + u < a.H) q += t[u];
      }
      int slot = (mem ? a.mem_slot_first : a.fifo_slot_first) + ci;
      const int C = mem ? a.mem_C : a.fifo_C;
      slot = slot >= C ? slot - C : slot;
      const long long pos = (mem ? a.mem_pos : a.fifo_pos)[slot];
      c.q = q;
      c.idx = i;
      c.pos = (int)pos;
      c.frame = (int)(pos >= 0 ? pos / a.frame_len : -((-pos + a.frame_len - 1) / a.frame_len));
    } else {
      c.q = -INFINITY;                               // padding sorts last in both orders
      c.idx = 0x7FFFFFFF;
      c.pos = 0x7FFFFFFF;
      c.frame = 0x7FFFFFFF;
    }
    v[i] = c;
  }
  __syncthreads();
  if (n_pow2 > 4 * kSelThreads)                      // up to 8,192 entries: eight per thread
    bitonic<8>(v, n_pow2);
  else
    bitonic<4>(v, n_pow2);
  // rank within the frame: the k-th entry of a frame run scores quality * gamma^k, gamma^k
  // formed by repeated multiplication.  Each thread takes a contiguous chunk; the run in
  // effect at its first entry comes from a max-scan of the chunks' last run starts.
  {
    const int per = (n + kSelThreads - 1) / kSelThreads;
    const int lo = min(tid * per, n), hi = min(lo + per, n);
    int last_start = -1;
    for (int i = lo; i < hi; ++i)
      if (i == 0 || v[i].frame != v[i - 1].frame) last_start = i;
    const int incl = block_max_scan(last_start, red);
    const int before = __shfl_up_sync(0xffffffffu, incl, 1);
    // run start in effect before lo: the previous thread's inclusive value (for the first
    // lane of a warp, the scanned total of the warps before it)
    const int carry = (tid & 31) ? before : (tid > 0 ? red[(tid >> 5) - 1] : -1);
    float scale = 1.f;
    if (lo < hi) {
      const int start = (lo == 0 || v[lo].frame != v[lo - 1].frame) ? lo : max(carry, 0);
      for (int k = start; k < lo; ++k) scale *= a.gamma;
    }
    float qs[8];
    for (int i = lo; i < hi; ++i) {
      if (i > lo) scale = (v[i].frame == v[i - 1].frame) ? scale * a.gamma : 1.f;
      qs[i - lo] = v[i].q * scale;
    }
    __syncthreads();                                 // every frame read before q changes
    for (int i = lo; i < hi; ++i) v[i].q = qs[i - lo];
  }
  __syncthreads();
  // the best min(n, M) by (score desc, position asc, index asc): a radix select over that
  // composite key (unique, since indices are), most significant byte first, marks them in
  // a bitmap of candidate indices without sorting by score
  const int m = n < a.M ? n : a.M;
  const int n_words = (n + 31) >> 5;
  for (int w = tid; w < n_words; w += blockDim.x) kbits[w] = 0u;
  {
    constexpr int kPer = KV_MEMORY_MAX_CANDIDATES / kSelThreads;   // entries i = tid + k * 1024
    uint32_t key[kPer][3];
    int state[kPer];                                 // 0 undecided, 1 kept, 2 dropped
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int i = tid + k * kSelThreads;
      state[k] = i < n ? 0 : 2;
      if (i < n) {
        uint32_t b = __float_as_uint(v[i].q);
        if (b == 0x80000000u) b = 0u;                // -0 ranks as +0
        const uint32_t asc = (b & 0x80000000u) ? ~b : (b | 0x80000000u);   // float order
        key[k][0] = ~asc;                            // higher score first
        key[k][1] = (uint32_t)v[i].pos ^ 0x80000000u;   // lower position first
        key[k][2] = (uint32_t)v[i].idx;              // lower index first (< 2^13)
      } else {
        key[k][0] = key[k][1] = key[k][2] = 0u;
      }
    }
    int r = m;                                       // still to keep among the undecided
    for (int pass = 0; pass < 10; ++pass) {
      const int word = pass < 4 ? 0 : (pass < 8 ? 1 : 2);
      const int shift = pass < 8 ? 24 - 8 * (pass & 3) : 8 - 8 * (pass - 8);
      for (int d = tid; d < 256; d += kSelThreads) hist[d] = 0;
      __syncthreads();
      // the word by constant indices (a runtime index would put key[] in local memory)
      auto digit = [&](int k) -> int {
        const uint32_t w = word == 0 ? key[k][0] : (word == 1 ? key[k][1] : key[k][2]);
        return (int)((w >> shift) & 0xFFu);
      };
#pragma unroll
      for (int k = 0; k < kPer; ++k)
        if (state[k] == 0) atomicAdd(&hist[digit(k)], 1);
      __syncthreads();
      if (tid < 32) {                                // the digit where the r-th key falls
        int c8[8], run = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          c8[e] = hist[8 * tid + e];
          run += c8[e];
        }
        int incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += y;
        }
        int below = incl - run;                      // keys in the digits under 8 tid
        if (below < r && r <= incl) {                // exactly one lane
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (below < r && r <= below + c8[e]) {
              sel[0] = 8 * tid + e;
              sel[1] = below;
              sel[2] = c8[e];
            }
            below += c8[e];
          }
        }
      }
      __syncthreads();
      const int dsel = sel[0], below = sel[1], cnt = sel[2];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        if (state[k] != 0) continue;
        const int d = digit(k);
        state[k] = d < dsel ? 1 : (d > dsel ? 2 : 0);
      }
      r -= below;
      __syncthreads();                               // sel and hist are reused
      if (cnt == r) break;                           // every key left in that digit is kept
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int i = tid + k * kSelThreads;
      if (i < n && state[k] != 2) {                  // kept, or left undecided in a full digit
        state[k] = 1;
        atomicOr(&kbits[v[i].idx >> 5], 1u << (v[i].idx & 31));
      }
    }
  }
  __syncthreads();
  if (tid < 32) {                                    // exclusive prefix of the words' counts
    const int per_w = (n_words + 31) >> 5;
    int run = 0;
    for (int k = 0; k < per_w; ++k) {
      const int w = tid * per_w + k;
      run += w < n_words ? __popc(kbits[w]) : 0;
    }
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (tid >= o) incl += y;
    }
    int base = incl - run;
    for (int k = 0; k < per_w; ++k) {
      const int w = tid * per_w + k;
      if (w < n_words) {
        wpre[w] = base;
        base += __popc(kbits[w]);
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x) {
    const int idx = v[i].idx;
    if (!(kbits[idx >> 5] & (1u << (idx & 31)))) continue;
    const int r = wpre[idx >> 5] + __popc(kbits[idx >> 5] & ((1u << (idx & 31)) - 1u));
    a.kept[r] = idx;
  }
}

// Copy kept candidate r (source: memory ring slot or FIFO slot) into memory_out slot r.
__global__ void __launch_bounds__(256) memory_gather_kernel(const SelectArgs a) {
  const int r = blockIdx.x;                          // kept entry = destination slot
  const int idx = a.kept[r];
  const bool mem = idx < a.n_mem;
  int slot = mem ? a.mem_slot_first + idx : a.fifo_slot_first + (idx - a.n_mem);
  const int C = mem ? a.mem_C : a.fifo_C;
  slot = slot >= C ? slot - C : slot;
  const uint8_t* kc = mem ? a.mem_kc : a.fifo_kc;
  const uint8_t* vc = mem ? a.mem_vc : a.fifo_vc;
  const float* ks = mem ? a.mem_ks : a.fifo_ks;
  const float* vs = mem ? a.mem_vs : a.fifo_vs;
  // 8 lanes per (head, K or V) row of 128 bytes
  for (int t = threadIdx.x; t < a.H * 2 * 8; t += blockDim.x) {
    const int hh = t / 16, which = (t / 8) & 1, part = t & 7;
    const uint8_t* src = (which ? vc : kc) + ((size_t)hh * C + slot) * D;
    uint8_t* dst = (which ? a.out_vc : a.out_kc) + ((size_t)hh * a.out_C + r) * D;
    reinterpret_cast<uint4*>(dst)[part] = reinterpret_cast<const uint4*>(src)[part];
  }
  for (int hh = threadIdx.x; hh < a.H; hh += blockDim.x) {
    a.out_ks[(size_t)hh * a.out_C + r] = ks[(size_t)hh * C + slot];
    a.out_vs[(size_t)hh * a.out_C + r] = vs[(size_t)hh * C + slot];
  }
  if (threadIdx.x == 0) a.out_pos[r] = (mem ? a.mem_pos : a.fifo_pos)[slot];
}

}  // namespace

size_t key_mass_workspace_bytes(int n_q, int n_heads) {
  if (n_q < 0 || n_heads < 1) return 0;
  return (size_t)n_heads * (size_t)((n_q + QT - 1) / QT) * QTile::bytes;
}

int launch_key_mass(const KeyMassArgs& a, cudaStream_t s) {
  // every set's CTAs in one grid: blk_first is the running sum of their block counts
  KeyMassArgs b = a;
  b.blk_first[0] = 0;
  for (int t = 0; t < b.n_sets; ++t)
    b.blk_first[t + 1] = b.blk_first[t] + (b.n_cand[t] + KG * KM - 1) / (KG * KM);
  if (b.blk_first[b.n_sets] == 0 || b.n_q == 0) return KV_OK;
  const dim3 grid((unsigned)b.blk_first[b.n_sets], (unsigned)b.H);
  if (b.qws) {
    static unsigned char configured[kMaxDevices] = {};
    if (!smem_attr_set(reinterpret_cast<const void*>(key_mass_pipe_kernel),
                       (int)PipeLayout::bytes, configured))
      return KV_ECUDA;
    b.n_qt = (b.n_q + QT - 1) / QT;
    key_mass_qsplit_kernel<<<dim3((unsigned)b.n_qt, (unsigned)b.H), 512, 0, s>>>(b);
    if (cudaPeekAtLastError() != cudaSuccess) return KV_ECUDA;
    key_mass_pipe_kernel<<<grid, kThreads, PipeLayout::bytes, s>>>(b);
  } else {
    static unsigned char configured[kMaxDevices] = {};
    if (!smem_attr_set(reinterpret_cast<const void*>(key_mass_kernel), (int)MassLayout::bytes,
                       configured))
      return KV_ECUDA;
    key_mass_kernel<<<grid, kThreads, MassLayout::bytes, s>>>(b);
  }
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

size_t select_smem_bytes(int n) {
  size_t p = 4;
  while ((int)p < n) p <<= 1;
  return p * sizeof(Cand);
}

int launch_memory_select(const SelectArgs& a, cudaStream_t s) {
  const int n = a.n_mem + a.n_fifo;
  const size_t bytes = select_smem_bytes(n);
  static unsigned char configured[kMaxDevices] = {};
  if (!smem_attr_set(reinterpret_cast<const void*>(memory_select_kernel),
                     (int)select_smem_bytes(KV_MEMORY_MAX_CANDIDATES), configured))
    return KV_ECUDA;
  memory_select_kernel<<<1, kSelThreads, bytes, s>>>(a);
  if (cudaPeekAtLastError() != cudaSuccess) return KV_ECUDA;
  const int m = n < a.M ? n : a.M;
  if (m > 0) memory_gather_kernel<<<m, 256, 0, s>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

}  // namespace kvring
