// kv_rotate.cu -- delta rotation of the cached keys when positions reset ("Runway
// Characters: Serving a 57B Video Diffusion Transformer for Real-Time Conversation",
// abstract: a delta rotation when positions reset, instead of re-encoding the cache).
//
// For every valid slot and head: x = e4m3(code) * scale (binary32), rotate the pairs by
// the angles of delta, requantise by the write rule.  Rows are (head, slot) with the slot
// running fastest, so consecutive rows are consecutive lines of one head's cache.
// G = D/32 lanes per row, 32 codes (two 16-byte loads and stores) per lane.  The angles
// are the same for every row: each lane keeps its 16 pairs' (c, c) and (s, s) in
// registers, so a pair's four products are two paired multiplies (each product still one
// binary32 rounding) and its two sums are single operations.
// Algorithmic traffic per row: D codes + 1 scale read, the same written.
#include "common.cuh"
#include "internal.h"
#include "../../include/kvring.h"

namespace kvring {

namespace {

constexpr int kThreads = 256;
constexpr int kRows = 4;        // rows per lane group: all their loads are in flight at once

// Row maximum over 32 values and G lanes, then the write's row rule for this lane's 32
// values (two 16-byte code words).
template <int G>
__device__ __forceinline__ void quant_row32(const float (&y)[32], uint4& c0, uint4& c1,
                                            float* scale_out) {
  float amax = max3_nan(fabsf(y[0]), fabsf(y[1]), fabsf(y[2]));
#pragma unroll
  for (int i = 3; i < 31; i += 2) amax = max3_nan(amax, fabsf(y[i]), fabsf(y[i + 1]));
  amax = max_nan(amax, fabsf(y[31]));
#pragma unroll
  for (int off = G / 2; off > 0; off >>= 1)
    amax = max_nan(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (!(amax <= 3.402823466e38f)) {
    *scale_out = __uint_as_float(0x7FC00000u);
    c0 = c1 = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    return;
  }
  const float inv = (amax > 0.f) ? div_rn(448.f, amax) : 0.f;
  if (!(amax > 0.f) || !isfinite(inv)) {
    *scale_out = 0.f;
    c0 = c1 = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  *scale_out = div_rn(amax, 448.f);
  const uint64_t inv2 = f2_pack(inv, inv);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float a0, a1, b0, b1;
    f2_unpack(f2_mul(f2_pack(y[4 * i], y[4 * i + 1]), inv2), a0, a1);
    f2_unpack(f2_mul(f2_pack(y[4 * i + 2], y[4 * i + 3]), inv2), b0, b1);
    w[i] = e4m3x2(a0, a1) | (e4m3x2(b0, b1) << 16);
  }
  c0 = make_uint4(w[0], w[1], w[2], w[3]);
  c1 = make_uint4(w[4], w[5], w[6], w[7]);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2) kv_rotate_kernel(const RotateArgs a) {
  constexpr int G = D / 32;
  constexpr int kPass = kThreads / G;
  const int lane_in_row = threadIdx.x % G;
  const int e0 = lane_in_row * 32;
  // (c, c) and (s, s) of this lane's 16 pairs
  uint64_t cc[16], ss[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float c = a.cs[e0 + 2 * i], s = a.cs[e0 + 2 * i + 1];
    cc[i] = f2_pack(c, c);
    ss[i] = f2_pack(s, s);
  }
  const int h = blockIdx.y;
  const int count = (int)a.count;
  const int i0 = blockIdx.x * (kRows * kPass) + threadIdx.x / G;
  uint8_t* const kc_h = a.kc + (size_t)h * a.C * D + e0;
  float* const ks_h = a.ks + (size_t)h * a.C;
  auto slot_of = [&](int k) {
    const int i = min(i0 + k * kPass, count - 1);     // all lanes stay for the shuffles
    int sl = (int)a.first_slot + i;
    return sl >= a.C ? sl - a.C : sl;
  };
  uint4 raw[kRows][2];
  float sc[kRows];
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const int sl = slot_of(k);
    const uint4* p = reinterpret_cast<const uint4*>(kc_h + (size_t)sl * D);
    raw[k][0] = p[0];
    raw[k][1] = p[1];
    sc[k] = ks_h[sl];
  }
  // every lane has read its rows before any store below (rows of a block are disjoint from
  // other blocks' rows; within the block each row is read and written by one lane group)
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const uint32_t w[8] = {raw[k][0].x, raw[k][0].y, raw[k][0].z, raw[k][0].w,
                           raw[k][1].x, raw[k][1].y, raw[k][1].z, raw[k][1].w};
    const uint64_t sc2 = f2_pack(sc[k], sc[k]);
    float y[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 lo = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[j] & 0xFFFFu)));
      const float2 hi = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[j] >> 16)));
      const uint64_t x01 = f2_mul(f2_pack(lo.x, lo.y), sc2);   // pair 2j
      const uint64_t x23 = f2_mul(f2_pack(hi.x, hi.y), sc2);   // pair 2j + 1
      float p0, p1, q0, q1;
      f2_unpack(f2_mul(x01, cc[2 * j]), p0, p1);               // x0 c, x1 c
      f2_unpack(f2_mul(x01, ss[2 * j]), q0, q1);               // x0 s, x1 s
      y[4 * j] = sub_rn(p0, q1);
      y[4 * j + 1] = add_rn(q0, p1);
      f2_unpack(f2_mul(x23, cc[2 * j + 1]), p0, p1);
      f2_unpack(f2_mul(x23, ss[2 * j + 1]), q0, q1);
      y[4 * j + 2] = sub_rn(p0, q1);
      y[4 * j + 3] = add_rn(q0, p1);
    }
    float scale;
    uint4 c0, c1;
    quant_row32<G>(y, c0, c1, &scale);
    if (i0 + k * kPass < count) {
      const int sl = slot_of(k);
      uint4* p = reinterpret_cast<uint4*>(kc_h + (size_t)sl * D);
      p[0] = c0;
      p[1] = c1;
      if (lane_in_row == 0) {
        ks_h[sl] = scale;
        if (h == 0) a.slot_pos[sl] += a.delta;
      }
    }
  }
}

template <int D>
int launch_rotate_d(const RotateArgs& a, cudaStream_t s) {
  constexpr int G = D / 32;
  if (a.count == 0 || a.H == 0) return KV_OK;
  const int64_t per_block = (int64_t)kRows * (kThreads / G);
  const dim3 grid((unsigned)((a.count + per_block - 1) / per_block), (unsigned)a.H);
  kv_rotate_kernel<D><<<grid, kThreads, 0, s>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

}  // namespace

int launch_rotate(const RotateArgs& a, int D, cudaStream_t s) {
  return D == 128 ? launch_rotate_d<128>(a, s) : launch_rotate_d<64>(a, s);
}

}  // namespace kvring
