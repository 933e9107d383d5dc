// kv_rotate.cu -- delta rotation of the cached keys when positions reset ("Runway
// Characters: Serving a 57B Video Diffusion Transformer for Real-Time Conversation",
// abstract: a delta rotation when positions reset, instead of re-encoding the cache).
//
// For every valid slot and head: x = e4m3(code) * scale (binary32), rotate the pairs by
// the angles of delta, requantise by the write rule.  Rows are (head, slot) with the slot
// running fastest, so consecutive rows are consecutive 128-byte lines of one head's
// cache.  G = D/16 lanes per row, 16 codes (one 16-byte load and store) per lane.
// Algorithmic traffic per row: D codes + 1 scale read, the same written.
#include "common.cuh"
#include "internal.h"
#include "../../include/kvring.h"

namespace kvring {

namespace {

constexpr int kThreads = 256;

template <int D>
__global__ void __launch_bounds__(kThreads) kv_rotate_kernel(const RotateArgs a) {
  constexpr int G = D / 16;
  __shared__ float4 s_cs[D / 4];
  if (threadIdx.x < D / 4)
    s_cs[threadIdx.x] = make_float4(a.cs[4 * threadIdx.x], a.cs[4 * threadIdx.x + 1],
                                    a.cs[4 * threadIdx.x + 2], a.cs[4 * threadIdx.x + 3]);
  __syncthreads();

  const int lane_in_row = threadIdx.x % G;
  const int64_t row = (int64_t)blockIdx.x * (kThreads / G) + threadIdx.x / G;
  const int64_t rows = a.count * a.H;
  const bool active = row < rows;
  const int64_t r = active ? row : rows - 1;
  const int h = (int)(r / a.count);
  const int64_t i = r % a.count;
  int64_t slot = a.first_slot + i;
  if (slot >= a.C) slot -= a.C;
  const int e0 = lane_in_row * 16;
  const size_t at = ((size_t)h * a.C + slot);

  const uint4 raw = *reinterpret_cast<const uint4*>(a.kc + at * D + e0);
  const float sc = a.ks[at];
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  float x[16], y[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 lo = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[j] & 0xFFFFu)));
    const float2 hi = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[j] >> 16)));
    x[4 * j] = mul_rn(lo.x, sc);
    x[4 * j + 1] = mul_rn(lo.y, sc);
    x[4 * j + 2] = mul_rn(hi.x, sc);
    x[4 * j + 3] = mul_rn(hi.y, sc);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 cs = s_cs[e0 / 4 + j];
    float x0 = x[4 * j], x1 = x[4 * j + 1];
    y[4 * j] = sub_rn(mul_rn(x0, cs.x), mul_rn(x1, cs.y));
    y[4 * j + 1] = add_rn(mul_rn(x0, cs.y), mul_rn(x1, cs.x));
    x0 = x[4 * j + 2];
    x1 = x[4 * j + 3];
    y[4 * j + 2] = sub_rn(mul_rn(x0, cs.z), mul_rn(x1, cs.w));
    y[4 * j + 3] = add_rn(mul_rn(x0, cs.w), mul_rn(x1, cs.z));
  }

  // requantise (same row rule as the write)
  float amax = 0.f;
  uint32_t bad = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    amax = fmaxf(amax, fabsf(y[k]));
    bad |= (uint32_t)!isfinite(y[k]);
  }
#pragma unroll
  for (int off = G / 2; off > 0; off >>= 1) {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    bad |= __shfl_xor_sync(0xffffffffu, bad, off);
  }
  uint4 q;
  float scale;
  const float inv = (amax > 0.f) ? div_rn(448.f, amax) : 0.f;
  if (bad) {
    scale = __uint_as_float(0x7FC00000u);
    q = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
  } else if (!(amax > 0.f) || !isfinite(inv)) {
    scale = 0.f;
    q = make_uint4(0u, 0u, 0u, 0u);
  } else {
    scale = div_rn(amax, 448.f);
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = e4m3x2(mul_rn(y[4 * j], inv), mul_rn(y[4 * j + 1], inv));
      const uint32_t hi = e4m3x2(mul_rn(y[4 * j + 2], inv), mul_rn(y[4 * j + 3], inv));
      o[j] = lo | (hi << 16);
    }
    q = make_uint4(o[0], o[1], o[2], o[3]);
  }
  // every lane of the row has read its codes before any lane overwrites the row's scale
  __syncwarp();
  if (active) {
    *reinterpret_cast<uint4*>(a.kc + at * D + e0) = q;
    if (lane_in_row == 0) {
      a.ks[at] = scale;
      if (h == 0) a.slot_pos[slot] += a.delta;
    }
  }
}

template <int D>
int launch_rotate_d(const RotateArgs& a, cudaStream_t s) {
  constexpr int G = D / 16;
  const int64_t rows = a.count * a.H;
  if (rows == 0) return KV_OK;
  const int64_t blocks = (rows + (kThreads / G) - 1) / (kThreads / G);
  kv_rotate_kernel<D><<<(unsigned)blocks, kThreads, 0, s>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

}  // namespace

int launch_rotate(const RotateArgs& a, int D, cudaStream_t s) {
  return D == 128 ? launch_rotate_d<128>(a, s) : launch_rotate_d<64>(a, s);
}

}  // namespace kvring
