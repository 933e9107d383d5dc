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
constexpr int kRows = 4;        // rows per lane group: all their loads are in flight at once

// Rotate and requantise one row's 16 codes (this lane's share); returns the new codes and,
// through *scale_out, the row's new scale (the same in every lane of the group).
template <int G>
__device__ __forceinline__ uint4 rotate16(uint4 raw, float sc, const float4* cs4,
                                          float* scale_out) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  const uint64_t sc2 = f2_pack(sc, sc);
  float y[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 lo = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[j] & 0xFFFFu)));
    const float2 hi = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w[j] >> 16)));
    const float4 cs = cs4[j];
    float x0, x1, x2, x3;
    f2_unpack(f2_mul(f2_pack(lo.x, lo.y), sc2), x0, x1);
    f2_unpack(f2_mul(f2_pack(hi.x, hi.y), sc2), x2, x3);
    y[4 * j] = sub_rn(mul_rn(x0, cs.x), mul_rn(x1, cs.y));
    y[4 * j + 1] = add_rn(mul_rn(x0, cs.y), mul_rn(x1, cs.x));
    x0 = x2;
    x1 = x3;
    y[4 * j + 2] = sub_rn(mul_rn(x0, cs.z), mul_rn(x1, cs.w));
    y[4 * j + 3] = add_rn(mul_rn(x0, cs.w), mul_rn(x1, cs.z));
  }
  return quant_row16<G>(y, scale_out);      // the write's row rule
}

// Grid (slot blocks, heads).  A block covers kRows passes of kThreads / G consecutive
// valid slots of head blockIdx.y; lane group g of pass k owns valid slot
// blockIdx.x * (kRows * kThreads / G) + k * (kThreads / G) + g (counted from the oldest).
// Every lane first issues the loads of all its rows, then rotates and stores them.
template <int D>
__global__ void __launch_bounds__(kThreads, 4) kv_rotate_kernel(const RotateArgs a) {
  constexpr int G = D / 16;
  constexpr int kPass = kThreads / G;
  __shared__ float4 s_cs[D / 4];
  if (threadIdx.x < D / 4)
    s_cs[threadIdx.x] = make_float4(a.cs[4 * threadIdx.x], a.cs[4 * threadIdx.x + 1],
                                    a.cs[4 * threadIdx.x + 2], a.cs[4 * threadIdx.x + 3]);

  const int lane_in_row = threadIdx.x % G;
  const int e0 = lane_in_row * 16;
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
  uint4 raw[kRows];
  float sc[kRows];
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const int sl = slot_of(k);
    raw[k] = *reinterpret_cast<const uint4*>(kc_h + (size_t)sl * D);
    sc[k] = ks_h[sl];
  }
  __syncthreads();   // s_cs ready; every lane has read its rows before any store below
  const float4* cs4 = s_cs + e0 / 4;
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    float scale;
    const uint4 q = rotate16<G>(raw[k], sc[k], cs4, &scale);
    if (i0 + k * kPass < count) {
      const int sl = slot_of(k);
      *reinterpret_cast<uint4*>(kc_h + (size_t)sl * D) = q;
      if (lane_in_row == 0) {
        ks_h[sl] = scale;
        if (h == 0) a.slot_pos[sl] += a.delta;
      }
    }
  }
}

template <int D>
int launch_rotate_d(const RotateArgs& a, cudaStream_t s) {
  constexpr int G = D / 16;
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
