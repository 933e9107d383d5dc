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
//  * P.V runs in f16 on the raw V codes: a CTA first finds G, the smallest power of two
//    at or above every V scale of its keys; each key's V scale is carried by P instead of
//    V, P' = f16(p * vs / G) (p <= 2^8, one f16 rounding, 2^-11 relative), and two
//    converter warps only widen the V codes to f16 (exact) in shared memory.  P' goes to
//    tensor memory over the S columns it came from and is read from there as the A
//    operand; the epilogue multiplies O by G.
//  * Mode B (KV_QK_FP8): the rotated bf16 row is instead quantised to e4m3 by the write's
//    row rule, and the row scale takes the place of r; S' is one set of D/32 MMAs.
//  * Prologue: all 12 warps rotate and split the 256 query rows together (8 lanes per
//    row, coalesced 16-byte loads) and find G; the producer thread has already started
//    the first K/V tile loads.
//  * Tensor memory (512 columns): tile g owns two S/P buffers of 64 columns,
//    [128g, 128g+64) and [128g+64, 128g+128), and O_g = [256+128g, 384+128g).  The MMA
//    warp runs its loop converged and one elected lane issues each instruction; it
//    serves the two query tiles in lockstep: for key tile j it waits for P_0(j)
//    (and V(j) widened), runs P.V_0(j) and S_0(j+2) into the buffer P_0(j) occupied,
//    then does the same for tile 1 (tensor-core operations of one thread run in issue
//    order).  Query tile 1 releases the K stage and the V buffer.
//  * Warps: 0 producer (lane 0 issues the TMA loads of K and V codes; all lanes build the
//    per-key info of each tile: scale, P factor, bias, mask token), 1 MMA issuer,
//    2-3 V converters, 4-7 softmax of tile 0, 8-11 softmax of tile 1 (thread = query
//    row = TMEM lane).
//  * Softmax in log2 units with paired fp32 instructions (f32x2) on the 64-column S row
//    held in registers; P goes back to tensor memory in 8-column pieces.  The reference maximum m moves lazily (only when the tile
//    maximum exceeds it by more than 8, a factor 256); O is then rescaled in tensor
//    memory after the previous P.V has completed.  out = O / l is exact regardless of m.
//    A history-only tile with m already set takes one pass (scale, 2^(t - m), P, tile
//    maximum on the way); the first tile, tiles with current or invalid keys, and tiles
//    whose maximum exceeds m by more than 8 take two (maximum first, then 2^(t - m)).
//  * Epilogue: O / l in bf16 goes through the K/V code stages of shared memory (free once
//    every MMA has completed), so whole 256-byte output rows leave in coalesced stores.
//  * Split over keys (gridDim.z > 1): each CTA takes a contiguous share of the valid
//    tiles and writes fp32 partials (O G, m, l); split_combine_kernel merges them.
//  * Several rings (kMulti): after the main ring's tiles a CTA visits the tiles of up to
//    KV_MAX_RINGS - 1 history-only rings (a persistent anchor, a content memory) in the
//    same pipeline, with each ring's tensor maps, scales and valid range; one softmax
//    covers them all.
//  * Keys are visited in physical slot order; the ring wrap costs nothing (attention
//    does not depend on key order once bias and mask are per key).  A CTA skips the
//    newest current-chunk keys that the block-causal mask hides from all of its rows.
// Every mbarrier wait is bounded (about a second); on a timeout the CTA abandons the
// work, writes NaN to its rows, waits (bounded again) for the copies and MMAs it has
// issued, frees its tensor memory and exits.
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
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpConv = 2, kWarpSoft = 4;
constexpr int kConvThreads = 64;        // one converter thread per key slot of a tile
constexpr uint32_t kVPanel = BN * 128u;  // bytes of one 64-column f16 panel of V (64 rows)
constexpr float kRescaleLog2 = 8.f;
constexpr int kInvalidTok = 0x7FFFFFFF;
constexpr int kRowLanes = 8;            // prologue: lanes per query row (16 elements each)
constexpr int kRowsPerPass = kThreads / kRowLanes;   // 48

struct Info {             // per key slot of one tile
  float kscl[BN];         // ks * softmax_scale * log2(e); 0 for invalid slots
  float w[BN];            // vs / G, the factor P carries for this key's V row; 0 invalid
  float kb[BN];           // additive log2 logit: bias (history), 0 (current), -inf (invalid)
  int ktok[BN];           // -1 history, token index (current), kInvalidTok (invalid)
  int special;            // the tile holds current-chunk or invalid slots
  int pad[3];
};

struct Layout {
  static constexpr uint32_t qhi = 0;                            // e4m3 [256][128], sw128
  static constexpr uint32_t qlo = qhi + BM * D;
  static constexpr uint32_t kbuf = qlo + BM * D;                // NK x e4m3 [64][128], sw128
  static constexpr uint32_t vcode = kbuf + NK * BN * D;         // NV x e4m3 [64][128], sw128
  static constexpr uint32_t vh = vcode + NV * BN * D;           // NB x f16 2 panels, sw128
  static constexpr uint32_t info = vh + NB * 2 * kVPanel;      // NI x Info
  static constexpr uint32_t rows = info + NI * sizeof(Info);    // int gi[256], float rowmul[256]
  static constexpr uint32_t bars = rows + 2 * BM * 4;           // mbarriers
  static constexpr int kNumBars = 2 * NK + 2 * NV + 2 * NB + 2 * NI + 4 + 4 + 1 + NV;
  static constexpr uint32_t misc = bars + 8 * kNumBars;         // tmem addr, abort flag, G
  static constexpr uint32_t bytes = misc + 16 + 1024;           // + alignment slack
};
static_assert(Layout::bytes <= 232448, "shared memory budget");
static_assert(Layout::kbuf % 1024 == 0 && Layout::vcode % 1024 == 0 && Layout::vh % 1024 == 0,
              "swizzled operands need 1024-byte alignment");
static_assert(Layout::bars % 8 == 0 && sizeof(Info) % 16 == 0, "alignment");

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
  // The P.V of key tile j (both query tiles) has completed when V buffer j % NB is
  // released (vhempty).
  __device__ uint64_t* sfull(int g, int buf) { return b + 2 * (NK + NV + NB + NI) + 2 * g + buf; }
  __device__ uint64_t* pfull(int g, int buf) { return b + 2 * (NK + NV + NB + NI) + 4 + 2 * g + buf; }
  __device__ uint64_t* ofinal() { return b + 2 * (NK + NV + NB + NI) + 8; }
  // e4m3-P mode: V code stage s checked (rows of invalid slots zeroed) for the MMAs
  __device__ uint64_t* vready(int s) { return b + 2 * (NK + NV + NB + NI) + 9 + s; }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The valid slots are the nv slots ending at `newest` (mod C), visited tile by tile in
// physical order.  count = number of tiles holding a valid slot; tile(k) = the k-th one.
struct TileSeq {
  int count;
  int split;   // tiles below `split` are taken as they are; from `split` on, add `skip`
  int skip;
  __device__ TileSeq(int C, int newest, int nv) {
    const int n_tiles = (C + BN - 1) / BN;
    split = n_tiles;
    skip = 0;
    if (nv <= 0) {
      count = 0;
    } else if (nv >= C) {
      count = n_tiles;
    } else {
      int first = newest - nv + 1;
      if (first >= 0) {                       // one segment [first, newest]
        const int ta = first / BN, tb = newest / BN;
        count = tb - ta + 1;
        split = 0;
        skip = ta;
      } else {                                // wrapped: [first + C, C) and [0, newest]
        first += C;
        const int tb = newest / BN, ta = first / BN;
        if (ta <= tb) {
          count = n_tiles;                    // the two segments share a tile: all tiles
        } else {
          count = (tb + 1) + (n_tiles - ta);
          split = tb + 1;
          skip = ta - (tb + 1);
        }
      }
    }
  }
  __device__ __forceinline__ int tile(int k) const { return k < split ? k : k + skip; }
};

// Age of slot `slot` (< C): 0 for the newest valid slot; valid iff age < n_valid.
__device__ __forceinline__ int slot_age(int slot, int newest, int C) {
  int age = newest - slot;
  return age < 0 ? age + C : age;
}

// Tensor maps (K and V codes, 128-byte swizzle) of the history-only rings that follow the
// main ring in one launch.
struct ExtraMaps {
  CUtensorMap k[KV_MAX_RINGS - 1];
  CUtensorMap v[KV_MAX_RINGS - 1];
};

// One key tile of the launch: ring r (0 = main ring), tile t of that ring, and the ring's
// scales, capacity and valid range.
struct KeyTile {
  int r, t, C, newest, n_valid;
  const float* ks;
  const float* vs;
};

// Tile k of the CTA's sequence: the main ring's visited tiles first, then each extra
// ring's valid tiles in order (kMulti: the launch reads extra rings).
template <bool kMulti>
__device__ __forceinline__ KeyTile key_tile(const AttnArgs& a, const TileSeq& seq0, int k) {
  KeyTile kt;
  if (!kMulti || k < seq0.count) {
    kt.r = 0;
    kt.t = seq0.tile(k);
    kt.C = a.C;
    kt.newest = (int)a.newest_slot;
    kt.n_valid = (int)a.n_valid;
    kt.ks = a.k_scale;
    kt.vs = a.v_scale;
    return kt;
  }
  k -= seq0.count;
  int x = 0;
  for (; x < a.n_extra - 1; ++x) {
    const int cnt = TileSeq(a.x_C[x], a.x_newest[x], a.x_n_valid[x]).count;
    if (k < cnt) break;
    k -= cnt;
  }
  kt.r = 1 + x;
  kt.t = TileSeq(a.x_C[x], a.x_newest[x], a.x_n_valid[x]).tile(k);
  kt.C = a.x_C[x];
  kt.newest = a.x_newest[x];
  kt.n_valid = a.x_n_valid[x];
  kt.ks = a.x_k_scale[x];
  kt.vs = a.x_v_scale[x];
  return kt;
}

// ------------------------------------------------------------------ query prologue
// 8 lanes per row, 16 consecutive elements per lane (one 16-byte chunk of the e4m3 row).
__device__ __forceinline__ void q_load16(const AttnArgs& a, int gi, int h, int lc, uint4 (&qr)[2],
                                         float4 (&cs)[4]) {
  const uint4* qp = reinterpret_cast<const uint4*>(a.q + ((size_t)gi * a.H + h) * D + 16 * lc);
  qr[0] = __ldg(qp);
  qr[1] = __ldg(qp + 1);
  const float4* tb = reinterpret_cast<const float4*>(a.rope_q0 + (size_t)gi * D + 16 * lc);
#pragma unroll
  for (int i = 0; i < 4; ++i) cs[i] = __ldg(tb + i);
}

// Rotated, bf16-rounded 16 elements of this lane's chunk (the write's binary32 sequence).
__device__ __forceinline__ void q_rot16(const uint4 (&qr)[2], const float4 (&cs)[4], float (&y)[16]) {
  const uint32_t w[8] = {qr[0].x, qr[0].y, qr[0].z, qr[0].w, qr[1].x, qr[1].y, qr[1].z, qr[1].w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float c = (j & 1) ? cs[j >> 1].z : cs[j >> 1].x;
    const float s = (j & 1) ? cs[j >> 1].w : cs[j >> 1].y;
    const float x0 = bf16_bits_to_float(w[j] & 0xFFFFu);
    const float x1 = bf16_bits_to_float(w[j] >> 16);
    const float y0 = sub_rn(mul_rn(x0, c), mul_rn(x1, s));
    const float y1 = add_rn(mul_rn(x0, s), mul_rn(x1, c));
    const uint32_t b = pack_bf16x2(y0, y1);                 // bf16 RNE of the rotated pair
    y[2 * j] = bf16_bits_to_float(b & 0xFFFFu);
    y[2 * j + 1] = bf16_bits_to_float(b >> 16);
  }
}

// Max |y| over the row's 8 lanes (NaN-propagating).
__device__ __forceinline__ float row_amax8(const float (&y)[16]) {
  float m = max3_nan(fabsf(y[0]), fabsf(y[1]), fabsf(y[2]));
#pragma unroll
  for (int i = 3; i < 15; i += 2) m = max3_nan(m, fabsf(y[i]), fabsf(y[i + 1]));
  m = max_nan(m, fabsf(y[15]));
#pragma unroll
  for (int off = kRowLanes / 2; off > 0; off >>= 1)
    m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, off));
  return m;
}

// Mode A: exponent k of the smallest power of two r = 2^k with amax / r <= 448, clamped
// to the normal range (k = 0 for zero or non-finite rows); then y / r = hi + lo exactly
// (hi, lo e4m3: 4 + 4 significant bits cover bf16's 8, for elements within 2^10 of the
// row's largest).  Returns r.
__device__ __forceinline__ float q_split16(const float (&y)[16], float amax, uint4& hi16, uint4& lo16) {
  int k = 0;
  if (amax > 0.f && amax <= 3.402823466e38f) {
    int e;
    const float m = frexpf(amax, &e);          // amax = m * 2^e, m in [0.5, 1)
    k = max(-126, min(127, (e - 1) - 8 + (m > 0.875f ? 1 : 0)));
  }
  const float inv_r = ldexpf(1.f, -k);
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float x[4], hv[4], lv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = y[4 * j + e] * inv_r;             // exact (power of two)
    const uint32_t h01 = e4m3x2(x[0], x[1]), h23 = e4m3x2(x[2], x[3]);
    const float2 d01 = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)h01));
    const float2 d23 = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)h23));
    hv[0] = d01.x;
    hv[1] = d01.y;
    hv[2] = d23.x;
    hv[3] = d23.y;
#pragma unroll
    for (int e = 0; e < 4; ++e) lv[e] = x[e] - hv[e];                    // exact difference
    const uint32_t l01 = e4m3x2(lv[0], lv[1]), l23 = e4m3x2(lv[2], lv[3]);
    hw[j] = h01 | (h23 << 16);
    lw[j] = l01 | (l23 << 16);
  }
  hi16 = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  lo16 = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  return ldexpf(1.f, k);
}

// Mode B: the write's row rule (scale = amax/448, codes = e4m3(y * (448/amax)); zero rows
// -> scale 0, zero codes; a non-finite element -> NaN scale, codes 0x7F).  Returns the
// row's scale.
__device__ __forceinline__ float q_quant16(const float (&y)[16], float amax, uint4& c16) {
  if (!(amax <= 3.402823466e38f)) {
    c16 = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    return __uint_as_float(0x7FC00000u);
  }
  const float inv = amax > 0.f ? div_rn(448.f, amax) : 0.f;
  if (!(amax > 0.f) || !isfinite(inv)) {
    c16 = make_uint4(0u, 0u, 0u, 0u);
    return 0.f;
  }
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t lo = e4m3x2(mul_rn(y[4 * j], inv), mul_rn(y[4 * j + 1], inv));
    const uint32_t hi = e4m3x2(mul_rn(y[4 * j + 2], inv), mul_rn(y[4 * j + 3], inv));
    w[j] = lo | (hi << 16);
  }
  c16 = make_uint4(w[0], w[1], w[2], w[3]);
  return div_rn(amax, 448.f);
}

// kPv8 (KV_PV_FP8): P is quantised to e4m3 as P'' = e4m3(p * vs / G * 2^8) with an exact
// running maximum (p <= 1), and P''.V runs as kind::f8f6f4 MMAs that read the V codes
// straight from their TMA stage (an MN-major e4m3 operand): no converter work, half the
// tensor time of the f16 product, and e4m3's 2^-4 relative rounding on every P element.
template <bool kPv8, bool kModeB, bool kMulti>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_attn_sm100_kernel(const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv,
                            const __grid_constant__ ExtraMaps xm, const AttnArgs a) {
  constexpr float kThr = kPv8 ? 0.f : kRescaleLog2;   // lazy-maximum threshold (log2)
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic on the shared array (an integer round trip
  // would hide from the compiler that sm addresses shared memory)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Bars bars{reinterpret_cast<uint64_t*>(sm + Layout::bars)};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Layout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Layout::misc + 4);
  uint32_t* vmax_bits = reinterpret_cast<uint32_t*>(sm + Layout::misc + 8);
  volatile int* n_issued = reinterpret_cast<volatile int*>(sm + Layout::misc + 12);  // K+V loads
  Info* info = reinterpret_cast<Info*>(sm + Layout::info);
  int* row_gi = reinterpret_cast<int*>(sm + Layout::rows);
  float* row_mul = reinterpret_cast<float*>(sm + Layout::rows + BM * 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int q0 = blockIdx.x * BM;
  // a CTA with at most 128 rows (few queries, a short last block) leaves query tile 1
  // out: none of its MMAs, its softmax warps idle until the epilogue
  const bool one_tile = a.n_rows - q0 <= BM / 2;
  const int C = a.C;
  const int newest = (int)a.newest_slot, n_valid = (int)a.n_valid;

  // Keys this CTA visits: the valid slots, less the newest current-chunk keys that the
  // block-causal mask hides from every one of its rows (the mask limit grows with the row
  // index, so its last row decides; a row list can hold any index, so all are kept then).
  int newest_v = newest, n_visit = n_valid;
  if (!a.rows && a.n_current > 0) {
    const int last = min(q0 + BM, min(a.n_rows, a.n_q)) - 1;
    if (last >= 0) {
      const int64_t qb = last < a.q_first ? 0 : 1 + (int64_t)(last - a.q_first) / a.q_block;
      const int64_t l = (int64_t)a.k_first + qb * (int64_t)a.k_block;
      const int hidden = a.n_current - (int)(l < (int64_t)a.n_current ? l : (int64_t)a.n_current);
      n_visit = n_valid - hidden;
      newest_v = newest - hidden;
      if (newest_v < 0) newest_v += C;
    }
  }
  // this CTA's slice of the visited tiles (all of them unless split over keys): the main
  // ring's, then those of every extra (history-only) ring
  const TileSeq seq(C, newest_v, n_visit);
  int n_total = seq.count;
  if (kMulti)
    for (int x = 0; x < a.n_extra; ++x)
      n_total += TileSeq(a.x_C[x], a.x_newest[x], a.x_n_valid[x]).count;
  int j0, n_mine;
  {
    const int per = (n_total + (int)gridDim.z - 1) / (int)gridDim.z;
    j0 = min(n_total, (int)blockIdx.z * per);
    n_mine = min(n_total, j0 + per) - j0;
  }
  auto tmap_k = [&](int r) -> const CUtensorMap* { return !kMulti || r == 0 ? &tmk : &xm.k[r - 1]; };
  auto tmap_v = [&](int r) -> const CUtensorMap* { return !kMulti || r == 0 ? &tmv : &xm.v[r - 1]; };

  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int s = 0; s < NK; ++s) { mbar_init(bars.kfull(s), 1); mbar_init(bars.kempty(s), 1); }
    for (int s = 0; s < NV; ++s) {
      mbar_init(bars.vfull(s), 1);
      mbar_init(bars.vempty(s), kPv8 ? 1 : kConvThreads);  // released by the MMAs (kPv8)
    }
    for (int s = 0; s < NB; ++s) { mbar_init(bars.vhfull(s), kConvThreads); mbar_init(bars.vhempty(s), 1); }
    for (int s = 0; s < NI; ++s) {
      mbar_init(bars.ifull(s), 32);
      mbar_init(bars.iempty(s), one_tile ? 128 : 256);   // the softmax threads that run
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bars.sfull(g, 0), 1);
      mbar_init(bars.sfull(g, 1), 1);
      mbar_init(bars.pfull(g, 0), 128);
      mbar_init(bars.pfull(g, 1), 128);
    }
    mbar_init(bars.ofinal(), 1);
    for (int s = 0; s < NV; ++s) mbar_init(bars.vready(s), kConvThreads);
    *abort_flag = 0;
    *vmax_bits = 0u;
    *n_issued = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // the first tiles' code loads go out now (their stages start empty) and overlap the
  // prologue below
  const int n_pre = min(n_mine, min(NK, NV));
  if (tid == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
    for (int j = 0; j < n_pre; ++j) {
      const KeyTile kt = key_tile<kMulti>(a, seq, j0 + j);
      mbar_arrive_expect_tx(bars.kfull(j), BN * D);
      tma_load_3d(sm + Layout::kbuf + j * BN * D, tmap_k(kt.r), bars.kfull(j), 0, kt.t * BN, h);
      mbar_arrive_expect_tx(bars.vfull(j), BN * D);
      tma_load_3d(sm + Layout::vcode + j * BN * D, tmap_v(kt.r), bars.vfull(j), 0, kt.t * BN, h);
    }
    *n_issued = n_pre;
  }

  // ------------------------------------------------------------ prologue (all warps)
  // G = 2^e >= every V scale of this CTA's valid keys.  Non-negative floats order like
  // their bits.  Up to 16 loads per thread are in flight at once.
  {
    float mx = 0.f;
    const int n_slots = n_mine * BN;
    for (int base = 0; base < n_slots; base += 16 * kThreads) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int i = base + u * kThreads + tid;
        v[u] = 0.f;
        if (i < n_slots) {
          const KeyTile kt = key_tile<kMulti>(a, seq, j0 + i / BN);
          const int slot = kt.t * BN + (i % BN);
          if (slot < kt.C && slot_age(slot, kt.newest, kt.C) < kt.n_valid)
            v[u] = __ldg(kt.vs + (size_t)h * kt.C + slot);
        }
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) mx = fmaxf(mx, v[u]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) atomicMax(vmax_bits, __float_as_uint(mx));
  }
  // query rows: row r of the CTA is entry q0 + r of the row list (or that index itself);
  // gi = -1 past the list's end or for an index outside [0, n_q) (nothing is computed or
  // written for such a row).  Two rows per lane group in flight.
  {
    const int lc = tid % kRowLanes;
    constexpr bool mode_b = kModeB;
    for (int base = 0; base < BM; base += 2 * kRowsPerPass) {
      int gi[2], r[2];
      uint4 qr[2][2];
      float4 cs[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        r[u] = base + u * kRowsPerPass + tid / kRowLanes;
        const int li = q0 + r[u];
        gi[u] = -1;
        if (r[u] < BM && li < a.n_rows) gi[u] = a.rows ? __ldg(a.rows + li) : li;
        if (gi[u] >= a.n_q) gi[u] = -1;
        if (gi[u] >= 0) {
          q_load16(a, gi[u], h, lc, qr[u], cs[u]);
        } else {
          qr[u][0] = qr[u][1] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int i = 0; i < 4; ++i) cs[u][i] = make_float4(1.f, 0.f, 1.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float y[16];
        q_rot16(qr[u], cs[u], y);                 // zero row for gi = -1
        const float amax = row_amax8(y);          // all lanes take part in the shuffles
        if (r[u] >= BM) continue;
        const uint32_t off = (uint32_t)r[u] * 128u + ((uint32_t)(lc ^ (r[u] & 7)) << 4);
        float rm;
        if (mode_b) {
          uint4 c16;
          rm = q_quant16(y, amax, c16);
          *reinterpret_cast<uint4*>(sm + Layout::qhi + off) = c16;
        } else {
          uint4 hi16, lo16;
          rm = q_split16(y, amax, hi16, lo16);
          *reinterpret_cast<uint4*>(sm + Layout::qhi + off) = hi16;
          *reinterpret_cast<uint4*>(sm + Layout::qlo + off) = lo16;
        }
        if (lc == 0) {
          row_gi[r[u]] = gi[u];
          row_mul[r[u]] = gi[u] >= 0 ? rm : 0.f;
        }
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // mx < 2^(b - 126) for biased exponent b; b clamped so that G and 1/G are normal
  const int gexp = max(1, min(252, (int)((*vmax_bits >> 23) & 0xFFu)));
  // G (times 2^-8 for kPv8, whose P carries 2^8)
  const float vnorm = __uint_as_float((uint32_t)(gexp + 1 - (kPv8 ? 8 : 0)) << 23);
  const float vnorm_inv = __uint_as_float((uint32_t)(253 - gexp) << 23);  // 1 / G

  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;       // fast path: already complete
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, a.timeouts)) return true;
    *abort_flag = 1;
    return false;
  };

  if (warp == kWarpProd) {
    // ------------------------------------------------------------ producer
    // lane 0: TMA loads of the K and V codes of tile j (the first n_pre went out before
    // the prologue); all lanes: the per-key info of tile j, two keys per lane, with the
    // next tile's scales loaded while this one is written.
    auto load_scales = [&](int j, float (&ks)[2], float (&vs)[2]) {
      const KeyTile kt = key_tile<kMulti>(a, seq, j < n_mine ? j0 + j : 0);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int slot = kt.t * BN + lane + 32 * e;
        const bool in_ring = j < n_mine && slot < kt.C;
        ks[e] = in_ring ? __ldg(kt.ks + (size_t)h * kt.C + slot) : 0.f;
        vs[e] = in_ring ? __ldg(kt.vs + (size_t)h * kt.C + slot) : 0.f;
      }
    };
    float pks[2], pvs[2];
    load_scales(0, pks, pvs);
    for (int j = 0; j < n_mine; ++j) {
      const KeyTile kt = key_tile<kMulti>(a, seq, j0 + j);
      const int t = kt.t;
      bool ok = true;
      if (lane == 0 && j >= n_pre) {
        const int sk = j % NK, sv = j % NV;
        ok = j < NK || wait(bars.kempty(sk), ((j / NK) - 1) & 1);
        if (ok) {
          mbar_arrive_expect_tx(bars.kfull(sk), BN * D);
          tma_load_3d(sm + Layout::kbuf + sk * BN * D, tmap_k(kt.r), bars.kfull(sk), 0, t * BN, h);
          ok = j < NV || wait(bars.vempty(sv), ((j / NV) - 1) & 1);
        }
        if (ok) {
          mbar_arrive_expect_tx(bars.vfull(sv), BN * D);
          tma_load_3d(sm + Layout::vcode + sv * BN * D, tmap_v(kt.r), bars.vfull(sv), 0, t * BN, h);
          *n_issued = j + 1;          // tile j's K and V loads are both out
        } else if (*n_issued == j) {
          // K(j) went out but V(j) did not: count K(j) alone (the drain waits on it)
          *n_issued = -(j + 1);
        }
      }
      const int si = j % NI;
      ok = ok && (j < NI || wait(bars.iempty(si), ((j / NI) - 1) & 1));
      if (!__all_sync(0xffffffffu, ok)) break;
      Info& in = info[si];
      bool special = false;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kk = lane + 32 * e, slot = t * BN + kk;
        float ksv = 0.f, kbv = -INFINITY, wv = 0.f;
        int tok = kInvalidTok;
        if (slot < kt.C) {
          const int age = slot_age(slot, kt.newest, kt.C);
          if (age < kt.n_valid) {
            ksv = pks[e] * a.score_scale_log2;
            wv = pvs[e] * vnorm_inv * (kPv8 ? 256.f : 1.f);   // exact: powers of two
            if (kt.r == 0 && age < a.n_current) {           // current chunk: main ring only
              kbv = 0.f;
              tok = a.n_current - 1 - age;
            } else {
              kbv = a.bias_log2;
              tok = -1;
            }
          }
        }
        special |= tok != -1;
        in.kscl[kk] = ksv;
        in.w[kk] = wv;
        in.kb[kk] = kbv;
        in.ktok[kk] = tok;
      }
      special = __any_sync(0xffffffffu, special);
      if (lane == 0) in.special = special ? 1 : 0;
      load_scales(j + 1, pks, pvs);                   // prefetch for the next tile
      mbar_arrive(bars.ifull(si));
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and waits; one elected lane issues each tensor-core
    // instruction (el_*), so every operand is warp-uniform.
    {
      constexpr uint32_t idS = idesc_e4m3_f32(128, BN);
      constexpr uint32_t idO = idesc_f16_f32(128, D, 0, 1);
      constexpr uint32_t idO8 = idesc_e4m3_f32(128, D, 1);     // e4m3 P (TMEM) x V codes (MN)
      const uint32_t sQhi = smem_u32(sm + Layout::qhi), sQlo = smem_u32(sm + Layout::qlo);
      const uint32_t sK = smem_u32(sm + Layout::kbuf), sV = smem_u32(sm + Layout::vh);
      // descriptors are built once; a step of s bytes adds s >> 4 to the start field
      const uint64_t dQhi = smem_desc_sw128(sQhi, 16, 1024), dQlo = smem_desc_sw128(sQlo, 16, 1024);
      const uint64_t dK = smem_desc_sw128(sK, 16, 1024), dV = smem_desc_sw128(sV, kVPanel, 1024);
      // V codes as the B operand: 64 key rows of 128 one-byte d values, 128-byte swizzled
      // (one swizzle atom across d, 8-row groups 1024 bytes apart along the keys)
      const uint64_t dVc = smem_desc_sw128(smem_u32(sm + Layout::vcode), kVPanel, 1024);
      constexpr int kHalves = kModeB ? 1 : 2;      // hi and lo, or the one e4m3 operand
      // S_g(j) = Q_g K(j)^T into buffer j & 1 of tile g
      auto issue_s = [&](int gg, int jj) {
        const uint32_t d = tmem + 128 * gg + 64 * (jj & 1);
        const uint64_t kd = dK + (((jj % NK) * BN * D) >> 4);
#pragma unroll
        for (int hf = 0; hf < kHalves; ++hf) {
          const uint64_t qd = (hf == 0 ? dQhi : dQlo) + ((gg * 128 * D) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            el_mma_f8_ss(d, qd + 2 * kk, kd + 2 * kk, idS, (hf | kk) != 0);
        }
        el_commit(bars.sfull(gg, jj & 1));
      };
      // O_g (+)= P_g(j) V(j) with P_g read from tensor memory (buffer j & 1)
      auto issue_pv = [&](int gg, int jj) {
        const uint32_t d = tmem + 256 + 128 * gg;
        const uint32_t p = tmem + 128 * gg + 64 * (jj & 1);
        if (kPv8) {
          const uint64_t vd = dVc + (((jj % NV) * BN * D) >> 4);
#pragma unroll
          for (int kk = 0; kk < BN / 32; ++kk)         // 32 keys = 8 columns = 32 code rows
            el_mma_f8_ts(d, p + 8 * kk, vd + 256 * kk, idO8, (jj > 0) | (kk > 0));
        } else {
          const uint64_t vd = dV + (((jj % NB) * 2 * kVPanel) >> 4);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            el_mma_f16_ts(d, p + 8 * kk, vd + 128 * kk, idO, (jj > 0) | (kk > 0));
        }
      };
      auto wait_w = [&](uint64_t* bar, uint32_t parity) -> bool {
        return mbar_wait_warp(bar, parity, abort_flag, a.timeouts);
      };
      bool ok = true;
      // S of the first two tiles for both query tiles
      for (int jj = 0; jj < 2 && jj < n_mine && ok; ++jj) {
        if (!(ok = wait_w(bars.kfull(jj % NK), (jj / NK) & 1))) break;
        tc_fence_after();
        issue_s(0, jj);
        if (!one_tile) issue_s(1, jj);
        el_commit(bars.kempty(jj % NK));           // every query tile has read K(jj)
      }
      // lockstep: per key tile j, query tile 0 then query tile 1, blocking waits
      const int last_g = one_tile ? 0 : 1;
      for (int j = 0; ok && j < n_mine; ++j) {
        const bool more = j + 2 < n_mine;
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          if (gg > last_g) break;
          ok = wait_w(bars.pfull(gg, j & 1), (j >> 1) & 1) &&
               (kPv8 ? wait_w(bars.vready(j % NV), (j / NV) & 1)
                     : wait_w(bars.vhfull(j % NB), (j / NB) & 1)) &&
               (!more || wait_w(bars.kfull((j + 2) % NK), ((j + 2) / NK) & 1));
          if (!ok) break;
          tc_fence_after();
          issue_pv(gg, j);
          if (gg == last_g) el_commit(kPv8 ? bars.vempty(j % NV) : bars.vhempty(j % NB));
          if (more) {
            issue_s(gg, j + 2);
            if (gg == last_g) el_commit(bars.kempty((j + 2) % NK));
          }
        }
      }
      if (n_mine > 0) el_commit(bars.ofinal());    // tracks every MMA issued above
      else if (lane == 0) mbar_arrive(bars.ofinal());
    }
  } else if (warp < kWarpSoft) {
    // ------------------------------------------------------------ V converters
    // 64 threads; thread ct owns key slot ct of every tile: its V row widened to f16
    // (exact) into the swizzled MN-major operand; rows of invalid slots become zero.
    // e4m3-P mode: the MMAs read the V codes in place; thread ct only zeroes row ct of the
    // stage when its slot is invalid (stale memory must not reach the MMA: 0 * NaN = NaN).
    const int ct = tid - 32 * kWarpConv;          // 0..63
    for (int j = 0; j < n_mine; ++j) {
      const KeyTile kt = key_tile<kMulti>(a, seq, j0 + j);
      const int slot = kt.t * BN + ct;
      const bool dead = !(slot < kt.C && slot_age(slot, kt.newest, kt.C) < kt.n_valid);
      const int sv = j % NV, b = j % NB;
      bool ok = wait(bars.vfull(sv), (j / NV) & 1);
      if (!kPv8) ok = ok && (j < NB || wait(bars.vhempty(b), ((j / NB) - 1) & 1));
      if (!named_bar_and(2, kConvThreads, ok)) break;
      if (kPv8) {
        if (dead) {
          uint4* row = reinterpret_cast<uint4*>(sm + Layout::vcode + sv * BN * D + ct * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) row[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        mbar_arrive(bars.vready(sv));
        continue;
      }
      const uint8_t* vc = sm + Layout::vcode + sv * BN * D + ct * 128;
      uint8_t* vb = sm + Layout::vh + b * 2 * kVPanel;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 cv = *reinterpret_cast<const uint4*>(vc + ((c ^ (ct & 7)) << 4));
        if (dead) cv = make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w[4] = {cv.x, cv.y, cv.z, cv.w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          o[2 * i] = e4m3x2_to_f16x2((uint16_t)(w[i] & 0xFFFFu));
          o[2 * i + 1] = e4m3x2_to_f16x2((uint16_t)(w[i] >> 16));
        }
        *reinterpret_cast<uint4*>(vb + sw128_offset(ct, 16 * c, kVPanel)) =
            make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(vb + sw128_offset(ct, 16 * c + 8, kVPanel)) =
            make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_smem();
      mbar_arrive(bars.vhfull(b));
      mbar_arrive(bars.vempty(sv));
    }
  } else {
    // ------------------------------------------------------------ softmax of tile g
    const int g = (warp - kWarpSoft) >> 2;                 // softmax tile (warps 4..11)
    const int row = 128 * g + 32 * (warp & 3) + lane;      // CTA row = TMEM lane of tile g
    const int gi = row_gi[row];
    const float rowmul = row_mul[row];
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
    const int n_soft = (g == 1 && one_tile) ? 0 : n_mine;    // tile 1 left out: no rows
    for (; j < n_soft; ++j) {
      const int si = j % NI, buf = j & 1;
      const uint32_t t_s = tmem + lane_base + 128 * g + 64 * buf;   // S_g(j) / P_g(j)
      bool ok = wait(bars.sfull(g, buf), (j >> 1) & 1) && wait(bars.ifull(si), (j / NI) & 1);
      if (!__all_sync(0xffffffffu, ok)) break;     // TMEM access below is warp-collective
      tc_fence_after();
      const Info& in = info[si];
      const bool special = in.special != 0;
      uint32_t sr[64];
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t (*)[32]>(sr);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t (*)[32]>(sr + 32);
        tmem_ld32(t_s, lo);
        tmem_ld32(t_s + 32, hi);
      }
      tmem_wait_ld();
      const float4* k4 = reinterpret_cast<const float4*>(in.kscl);
      const float4* w4 = reinterpret_cast<const float4*>(in.w);
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
        uint32_t p8[16];                               // kPv8: e4m3 P, four keys per word
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[8];
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const int q = 4 * c + q8;
            const float4 ks = k4[q], ww = w4[q];
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
            const uint64_t p01 = f2_pack(ex2(t0), ex2(t1)), p23 = f2_pack(ex2(t2), ex2(t3));
            sum01 = f2_add(sum01, p01);
            sum23 = f2_add(sum23, p23);
            float a0, a1, a2, a3;
            f2_unpack(f2_mul(p01, f2_pack(ww.x, ww.y)), a0, a1);
            f2_unpack(f2_mul(p23, f2_pack(ww.z, ww.w)), a2, a3);
            if (kPv8) {
              p8[q] = e4m3x2(a0, a1) | (e4m3x2(a2, a3) << 16);
            } else {
              pk[2 * q8] = pack_f16x2(a0, a1);
              pk[2 * q8 + 1] = pack_f16x2(a2, a3);
            }
          }
          // P over S columns already read into registers; a recomputation overwrites it
          if (!kPv8) tmem_st8(t_s + 8 * c, pk);
        }
        if (kPv8) tmem_st16(t_s, p8);
        const float mloc = fmaf(fmaxf(m0, m1), rowmul, a.bias_log2);
        single = !__any_sync(0xffffffffu, mloc > m_run + kThr);
      }
      if (!single) {
        // pass 1, in place: t = S * kscl (* r + bias later) for fast tiles, masked t for the
        // others; row maximum of the tile
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
        move = mloc > m_old + kThr || (m_old == -INFINITY && mloc > -INFINITY);
        if (move) m_run = mloc;
        const float mref = (m_run == -INFINITY) ? 0.f : m_run;
        // pass 2: p = 2^(t - m); P' = f16(p * w) over the S columns of tensor memory
        const float off = special ? -mref : a.bias_log2 - mref;
        const uint64_t mul2 = special ? f2_pack(1.f, 1.f) : r2;
        const uint64_t off2 = f2_pack(off, off);
        sum01 = f2_pack(0.f, 0.f);
        sum23 = sum01;
        uint32_t p8[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[8];
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const int q = 4 * c + q8;
            const float4 ww = w4[q];
            float t0, t1, t2, t3;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[4 * q]), __uint_as_float(sr[4 * q + 1])), mul2,
                             off2), t0, t1);
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[4 * q + 2]), __uint_as_float(sr[4 * q + 3])), mul2,
                             off2), t2, t3);
            // 2^-inf = 0
            const uint64_t p01 = f2_pack(ex2(t0), ex2(t1)), p23 = f2_pack(ex2(t2), ex2(t3));
            sum01 = f2_add(sum01, p01);
            sum23 = f2_add(sum23, p23);
            float a0, a1, a2, a3;
            f2_unpack(f2_mul(p01, f2_pack(ww.x, ww.y)), a0, a1);
            f2_unpack(f2_mul(p23, f2_pack(ww.z, ww.w)), a2, a3);
            if (kPv8) {
              p8[q] = e4m3x2(a0, a1) | (e4m3x2(a2, a3) << 16);
            } else {
              pk[2 * q8] = pack_f16x2(a0, a1);
              pk[2 * q8 + 1] = pack_f16x2(a2, a3);
            }
          }
          if (!kPv8) tmem_st8(t_s + 8 * c, pk);
        }
        if (kPv8) tmem_st16(t_s, p8);
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
        ok = kPv8 ? wait(bars.vempty((j - 1) % NV), ((j - 1) / NV) & 1)
                  : wait(bars.vhempty((j - 1) % NB), ((j - 1) / NB) & 1);
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
    const bool row_ok = gi >= 0;
    const bool any = j > 0;
    if (a.part_o) {
      // split over keys: unnormalised O (relative to m_run, times G) and (m_run, l_run)
      // partials are indexed by the row's list entry li (its own index without a list)
      const int li = row_ok ? q0 + row : 0;
      const size_t prow = ((size_t)blockIdx.z * a.n_rows + li) * a.H + h;
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
                      ((size_t)blockIdx.z * a.H + h) * a.n_rows + li;
        *pml = ok ? make_float2(m_run, l_run)
                  : make_float2(__uint_as_float(0x7FC00000u), __uint_as_float(0x7FC00000u));
      }
    } else {
      const float inv_l = (l_run > 0.f) ? (1.f / l_run) * vnorm : 0.f;
      // Rows go through shared memory (the K and V code stages are free once every MMA has
      // completed) so that whole 256-byte rows are stored with coalesced 16-byte stores.
      // After an abandoned wait in any softmax warp, every row is stored directly instead.
      if (named_bar_and(1, 256, ok)) {
        uint8_t* st = sm + Layout::kbuf;                      // [256 rows][256 B], swizzled
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t o[64];
          if (any) {
            uint32_t (&lo)[32] = *reinterpret_cast<uint32_t (*)[32]>(o);
            uint32_t (&hi)[32] = *reinterpret_cast<uint32_t (*)[32]>(o + 32);
            tmem_ld32(t_o + 64 * c, lo);
            tmem_ld32(t_o + 64 * c + 32, hi);
            tmem_wait_ld();
          }
          uint32_t pk[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float x0 = l_run > 0.f ? __uint_as_float(o[2 * k]) * inv_l : 0.f;
            const float x1 = l_run > 0.f ? __uint_as_float(o[2 * k + 1]) * inv_l : 0.f;
            pk[k] = pack_bf16x2(x0, x1);
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int cc = 8 * c + k;                           // 16-byte chunk of the row
            *reinterpret_cast<uint4*>(st + row * 256 + ((cc ^ (row & 15)) << 4)) =
                make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
          }
        }
        named_bar(1, 256);
        const int sw = warp - kWarpSoft;                        // rows [32 sw, 32 sw + 32)
#pragma unroll 4
        for (int it = 0; it < 16; ++it) {
          const int r = 32 * sw + 2 * it + (lane >> 4), cc = lane & 15;
          const int gr = row_gi[r];
          if (gr >= 0)
            *reinterpret_cast<uint4*>(a.out + ((size_t)gr * a.H + h) * D + 8 * cc) =
                *reinterpret_cast<const uint4*>(st + r * 256 + ((cc ^ (r & 15)) << 4));
        }
      } else {
        uint16_t* dst = a.out + ((size_t)(row_ok ? gi : 0) * a.H + h) * D;
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t o[64];
          if (any) {
            uint32_t (&lo)[32] = *reinterpret_cast<uint32_t (*)[32]>(o);
            uint32_t (&hi)[32] = *reinterpret_cast<uint32_t (*)[32]>(o + 32);
            tmem_ld32(t_o + 64 * c, lo);
            tmem_ld32(t_o + 64 * c + 32, hi);
            tmem_wait_ld();
          }
          uint32_t pk[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            float x0 = l_run > 0.f ? __uint_as_float(o[2 * k]) * inv_l : 0.f;
            float x1 = l_run > 0.f ? __uint_as_float(o[2 * k + 1]) * inv_l : 0.f;
            if (!ok) x0 = x1 = __uint_as_float(0x7FC00000u);
            pk[k] = pack_bf16x2(x0, x1);
          }
          if (row_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + 64 * c);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              d4[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
          }
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
    if (lane == 0 && *abort_flag) {
      // abandoned work: wait (bounded, ignoring the abort flag) for the code loads and the
      // MMAs this CTA issued before its shared and tensor memory are released.  Loads of
      // tiles [0, nk) (K) and [0, nv) (V) went out; the last NK resp. NV of them cover
      // every load still in flight.  ofinal is committed after the last MMA on every path.
      const int ni = *n_issued;
      const int nk = ni >= 0 ? ni : -ni, nv = ni >= 0 ? ni : -ni - 1;
      for (int j = max(0, nk - NK); j < nk; ++j)
        mbar_wait(bars.kfull(j % NK), (j / NK) & 1, a.timeouts);
      for (int j = max(0, nv - NV); j < nv; ++j)
        mbar_wait(bars.vfull(j % NV), (j / NV) & 1, a.timeouts);
      mbar_wait(bars.ofinal(), 0, a.timeouts);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the split partials of one (query row, head) per warp: M = max m_s over splits
// with l_s > 0, w_s = 2^(m_s - M), out = sum w_s O_s / sum w_s l_s, lse = (M + log2 L) ln 2.
__global__ void __launch_bounds__(256) split_combine_kernel(const AttnArgs a, int n_splits) {
  const int wid = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (wid >= a.n_rows * a.H) return;              // whole warp leaves together
  // partials of list entry li; the output row is rows[li] (li itself without a list)
  const int li = wid / a.H, h = wid % a.H;
  const int gi = a.rows ? __ldg(a.rows + li) : li;
  if (gi < 0 || gi >= a.n_q) return;
  const float2* pml = reinterpret_cast<const float2*>(a.part_ml);
  float M = -INFINITY;
  bool bad = false;                               // a split that gave up: NaN out
  for (int z = 0; z < n_splits; ++z) {
    const float2 ml = pml[((size_t)z * a.H + h) * a.n_rows + li];
    bad |= isnan(ml.y);
    if (ml.y > 0.f) M = fmaxf(M, ml.x);
  }
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int z = 0; z < n_splits; ++z) {
    const float2 ml = pml[((size_t)z * a.H + h) * a.n_rows + li];
    if (!(ml.y > 0.f)) continue;
    const float w = ex2(ml.x - M);
    L += w * ml.y;
    const float4 o = reinterpret_cast<const float4*>(
        a.part_o + (((size_t)z * a.n_rows + li) * a.H + h) * D)[lane];
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
  const int warps = a.n_rows * a.H;
  split_combine_kernel<<<(warps + 7) / 8, 256, 0, s>>>(a, n_splits);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

int launch_attention_sm100_d128(const AttnArgs& a, const void* tmap_k_sw128,
                                const void* tmap_v_sw128, cudaStream_t s, int n_splits,
                                const void* const* x_tmap_k, const void* const* x_tmap_v) {
  // one instance per (e4m3 P, mode B, extra rings) triple
  using Kernel = void (*)(const CUtensorMap, const CUtensorMap, const ExtraMaps, const AttnArgs);
  static const Kernel kernels[8] = {
      chunk_attn_sm100_kernel<false, false, false>, chunk_attn_sm100_kernel<false, true, false>,
      chunk_attn_sm100_kernel<true, false, false>,  chunk_attn_sm100_kernel<true, true, false>,
      chunk_attn_sm100_kernel<false, false, true>,  chunk_attn_sm100_kernel<false, true, true>,
      chunk_attn_sm100_kernel<true, false, true>,   chunk_attn_sm100_kernel<true, true, true>};
  static unsigned char configured[8][kMaxDevices] = {};
  const int which = (a.n_extra > 0 ? 4 : 0) + (a.pv_fp8 ? 2 : 0) + (a.mode_b ? 1 : 0);
  const Kernel fn = kernels[which];
  if (!smem_attr_set(reinterpret_cast<const void*>(fn), (int)Layout::bytes, configured[which]))
    return KV_ECUDA;
  if (a.n_extra < 0 || a.n_extra > KV_MAX_RINGS - 1 || (a.n_extra > 0 && (!x_tmap_k || !x_tmap_v)))
    return KV_EINVAL;
  CUtensorMap mk, mv;
  memcpy(&mk, tmap_k_sw128, sizeof(mk));
  memcpy(&mv, tmap_v_sw128, sizeof(mv));
  ExtraMaps xm;
  memset(&xm, 0, sizeof(xm));
  for (int x = 0; x < a.n_extra; ++x) {
    memcpy(&xm.k[x], x_tmap_k[x], sizeof(CUtensorMap));
    memcpy(&xm.v[x], x_tmap_v[x], sizeof(CUtensorMap));
  }
  dim3 grid((a.n_rows + BM - 1) / BM, a.H, n_splits);
  fn<<<grid, kThreads, Layout::bytes, s>>>(mk, mv, xm, a);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

}  // namespace kvring
