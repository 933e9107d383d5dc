// kv_write.cu -- ring write: RoPE on K, per-(token, head) e4m3 quantisation of K and V,
// store into the ring slots ("Runway Characters: Serving a 57B Video Diffusion Transformer
// for Real-Time Conversation", abstract: RoPE and FP8 quantisation applied once per write,
// into a ring cache).
//
// HBM-bound streaming kernel.  A row is one (token, head) pair; G = D/16 threads share a
// row and each owns 16 consecutive elements (8 rotation pairs): 16-byte vector loads of
// the inputs and of the (cos, sin) table, one 16-byte store of 16 codes each for K and V.
// The row's maximum magnitude (NaN-propagating) is reduced with shuffles inside the
// G-lane group.  Algorithmic traffic per row: 2*D*sizeof(in) read + 2*D codes + 2 scales
// (+ slot position) written.
#include "common.cuh"
#include "internal.h"
#include "../../include/kvring.h"

namespace kvring {

namespace {

constexpr int kThreads = 64;         // small blocks: the grid's last partial wave is short
constexpr int kRows = 1;        // rows per lane group (more in flight cost occupancy here)

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

// Grid (token blocks, heads): consecutive rows of a block are consecutive tokens of one
// head, so its code lines and scales are stored contiguously.  A block covers kRows
// passes of kThreads / G tokens; every lane first issues the loads of all its rows (K, V
// and the rotation table), then computes and stores them.
template <int D, typename T>
__global__ void __launch_bounds__(kThreads) kv_write_kernel(const WriteArgs a) {
  constexpr int G = D / 16;                      // lanes per row
  constexpr int kPass = kThreads / G;
  const int lane_in_row = threadIdx.x % G;
  const int e0 = lane_in_row * 16;
  const int h = blockIdx.y;
  const int t0 = blockIdx.x * (kRows * kPass) + threadIdx.x / G;
  float xk[kRows][16], xv[kRows][16];
  float4 cs[kRows][4];
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const int t = min(t0 + k * kPass, a.n - 1);     // all lanes stay for the shuffles
    const size_t in_elem = ((size_t)t * a.H + h) * D + e0;
    In<T>::load16(a.k, in_elem, xk[k]);
    In<T>::load16(a.v, in_elem, xv[k]);
    const float4* tb = reinterpret_cast<const float4*>(a.rope_row0 + (size_t)t * D + e0);
#pragma unroll
    for (int j = 0; j < 4; ++j) cs[k][j] = __ldg(tb + j);   // (c, s) of 2 pairs each
  }
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    // K: rotate pairs (2i, 2i+1) by the tabled angle of position pos0 + t.
    float y[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float c0 = cs[k][j].x, s0 = cs[k][j].y, c1 = cs[k][j].z, s1 = cs[k][j].w;
      float x0 = xk[k][4 * j], x1 = xk[k][4 * j + 1];
      y[4 * j] = sub_rn(mul_rn(x0, c0), mul_rn(x1, s0));
      y[4 * j + 1] = add_rn(mul_rn(x0, s0), mul_rn(x1, c0));
      x0 = xk[k][4 * j + 2];
      x1 = xk[k][4 * j + 3];
      y[4 * j + 2] = sub_rn(mul_rn(x0, c1), mul_rn(x1, s1));
      y[4 * j + 3] = add_rn(mul_rn(x0, s1), mul_rn(x1, c1));
    }
    float kscale, vscale;
    const uint4 kq = quant_row16<G>(y, &kscale);
    const uint4 vq = quant_row16<G>(xv[k], &vscale);     // V: quantised as is
    const int t = t0 + k * kPass;
    if (t < a.n) {
      int64_t slot = a.w + t;
      if (slot >= a.C) slot -= a.C;
      const size_t out_row = (size_t)h * a.C + slot;
      *reinterpret_cast<uint4*>(a.kc + out_row * D + e0) = kq;
      *reinterpret_cast<uint4*>(a.vc + out_row * D + e0) = vq;
      if (lane_in_row == 0) {
        a.ks[out_row] = kscale;
        a.vs[out_row] = vscale;
        if (h == 0) a.slot_pos[slot] = (int32_t)(a.pos0 + t);
      }
    }
  }
}

template <int D>
int launch_write_d(const WriteArgs& a, int in_dtype, cudaStream_t s) {
  constexpr int G = D / 16;
  const int per_block = kRows * (kThreads / G);
  const dim3 grid((unsigned)((a.n + per_block - 1) / per_block), (unsigned)a.H);
  if (in_dtype == KV_DTYPE_BF16)
    kv_write_kernel<D, uint16_t><<<grid, kThreads, 0, s>>>(a);
  else
    kv_write_kernel<D, float><<<grid, kThreads, 0, s>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? KV_OK : KV_ECUDA;
}

}  // namespace

int launch_write(const WriteArgs& a, int D, int in_dtype, cudaStream_t s) {
  return D == 128 ? launch_write_d<128>(a, in_dtype, s) : launch_write_d<64>(a, in_dtype, s);
}

}  // namespace kvring
