// kv_write.cu -- ring write: RoPE on K, per-(token, head) e4m3 quantisation of K and V,
// store into the ring slots ("Runway Characters: Serving a 57B Video Diffusion Transformer
// for Real-Time Conversation", abstract: RoPE and FP8 quantisation applied once per write,
// into a ring cache).
//
// HBM-bound streaming kernel.  A row is one (token, head) pair; G = D/16 threads share a
// row and each owns 16 consecutive elements (8 rotation pairs): 16-byte vector loads of
// the inputs and of the (cos, sin) table, one 16-byte store of 16 codes.  The row's amax
// and non-finite flag are reduced with shuffles inside the G-lane group.  Algorithmic
// traffic per row: 2*D*sizeof(in) read + 2*D codes + 2 scales (+ slot position) written.
#include "common.cuh"
#include "internal.h"
#include "../../include/kvring.h"

namespace kvring {

namespace {

constexpr int kThreads = 256;

template <typename T>
struct In;

template <>
struct In<uint16_t> {  // bf16: 16 elements = two 16-byte loads
  static __device__ __forceinline__ void load16(const void* base, size_t elem, float (&x)[16]) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + elem);
    uint4 a = __ldg(p), b = __ldg(p + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[2 * i] = bf16_bits_to_float(w[i] & 0xFFFFu);
      x[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
    }
  }
};

template <>
struct In<float> {  // fp32: 16 elements = four 16-byte loads
  static __device__ __forceinline__ void load16(const void* base, size_t elem, float (&x)[16]) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 f = __ldg(p + i);
      x[4 * i] = f.x;
      x[4 * i + 1] = f.y;
      x[4 * i + 2] = f.z;
      x[4 * i + 3] = f.w;
    }
  }
};

// Quantise the 16 values this thread owns of a row shared by G lanes; lane 0 of the
// group returns the scale through *scale_out.  Row rule: scale = amax/448, codes =
// e4m3(y * (448/amax)); zero or tiny rows -> 0; non-finite rows -> NaN scale, 0x7F codes.
template <int G>
__device__ __forceinline__ uint4 quant16(const float (&y)[16], float* scale_out) {
  float amax = 0.f;
  uint32_t bad = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    amax = fmaxf(amax, fabsf(y[i]));
    bad |= (uint32_t)!isfinite(y[i]);
  }
#pragma unroll
  for (int off = G / 2; off > 0; off >>= 1) {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    bad |= __shfl_xor_sync(0xffffffffu, bad, off);
  }
  if (bad) {
    *scale_out = __uint_as_float(0x7FC00000u);
    return make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
  }
  const float inv = (amax > 0.f) ? div_rn(448.f, amax) : 0.f;
  if (!(amax > 0.f) || !isfinite(inv)) {
    *scale_out = 0.f;
    return make_uint4(0u, 0u, 0u, 0u);
  }
  *scale_out = div_rn(amax, 448.f);
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t lo = e4m3x2(mul_rn(y[4 * i], inv), mul_rn(y[4 * i + 1], inv));
    const uint32_t hi = e4m3x2(mul_rn(y[4 * i + 2], inv), mul_rn(y[4 * i + 3], inv));
    w[i] = lo | (hi << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int D, typename T>
__global__ void __launch_bounds__(kThreads) kv_write_kernel(const WriteArgs a) {
  constexpr int G = D / 16;                      // lanes per row
  const int lane_in_row = threadIdx.x % G;
  const int64_t row = (int64_t)blockIdx.x * (kThreads / G) + threadIdx.x / G;
  const int64_t rows = (int64_t)a.n * a.H;
  const bool active = row < rows;                // all lanes stay for the shuffles
  const int64_t r = active ? row : rows - 1;
  const int t = (int)(r / a.H), h = (int)(r % a.H);
  int64_t slot = a.w + t;
  if (slot >= a.C) slot -= a.C;
  const int e0 = lane_in_row * 16;
  const size_t in_elem = (size_t)r * D + e0;
  const size_t out_row = ((size_t)h * a.C + slot);

  // K: rotate pairs (2i, 2i+1) by the tabled angle of position pos0 + t.
  float x[16], y[16];
  In<T>::load16(a.k, in_elem, x);
  const float4* tb = reinterpret_cast<const float4*>(a.rope_row0 + (size_t)t * D + e0);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 cs = __ldg(tb + j);   // (c, s) of pairs 2j, 2j+1 of this lane's block
    const float c0 = cs.x, s0 = cs.y, c1 = cs.z, s1 = cs.w;
    float x0 = x[4 * j], x1 = x[4 * j + 1];
    y[4 * j] = sub_rn(mul_rn(x0, c0), mul_rn(x1, s0));
    y[4 * j + 1] = add_rn(mul_rn(x0, s0), mul_rn(x1, c0));
    x0 = x[4 * j + 2];
    x1 = x[4 * j + 3];
    y[4 * j + 2] = sub_rn(mul_rn(x0, c1), mul_rn(x1, s1));
    y[4 * j + 3] = add_rn(mul_rn(x0, s1), mul_rn(x1, c1));
  }
  float kscale;
  const uint4 kq = quant16<G>(y, &kscale);

  // V: quantise as is.
  In<T>::load16(a.v, in_elem, x);
  float vscale;
  const uint4 vq = quant16<G>(x, &vscale);

  if (active) {
    *reinterpret_cast<uint4*>(a.kc + out_row * D + e0) = kq;
    *reinterpret_cast<uint4*>(a.vc + out_row * D + e0) = vq;
    if (lane_in_row == 0) {
      a.ks[out_row] = kscale;
      a.vs[out_row] = vscale;
      if (h == 0) a.slot_pos[slot] = (int32_t)(a.pos0 + t);
    }
  }
}

template <int D>
int launch_write_d(const WriteArgs& a, int in_dtype, cudaStream_t s) {
  constexpr int G = D / 16;
  const int64_t rows = (int64_t)a.n * a.H;
  const int64_t blocks = (rows + (kThreads / G) - 1) / (kThreads / G);
  if (in_dtype == KV_DTYPE_BF16)
    kv_write_kernel<D, uint16_t><<<(unsigned)blocks, kThreads, 0, s>>>(a);
  else
    kv_write_kernel<D, float><<<(unsigned)blocks, kThreads, 0, s>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

}  // namespace

int launch_write(const WriteArgs& a, int D, int in_dtype, cudaStream_t s) {
  return D == 128 ? launch_write_d<128>(a, in_dtype, s) : launch_write_d<64>(a, in_dtype, s);
}

}  // namespace kvring
