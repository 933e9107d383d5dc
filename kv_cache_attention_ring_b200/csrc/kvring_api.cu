// kvring_api.cu -- the C ABI declared in include/kvring.h: argument and state validation,
// ring-head arithmetic, the host-built RoPE table, TMA descriptor encoding, launches.
//
// Ring semantics follow "Runway Characters: Serving a 57B Video Diffusion Transformer for
// Real-Time Conversation" (abstract: a ring cache written once per token, a delta rotation
// when positions reset).  Every check happens here, before anything is enqueued; the
// kernels assume validated arguments.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "../../include/kvring.h"
#include "internal.h"

namespace kvring {
__device__ unsigned int g_wait_timeouts = 0;

// Partials of chunk_attention_split_noalloc: part of the module image, so every device
// that loads the library has its own copy and no call allocates.
__device__ __align__(256) unsigned char g_noalloc_scratch[KV_NOALLOC_SCRATCH_BYTES];

std::mutex g_symbol_mu;
void* g_timeouts_ptr[kMaxDevices] = {};
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of `symbol` on the current device, looked up once per device (with that
// device current) and cached in table[device].
template <typename T>
void* symbol_address(const T& symbol, void* (&table)[kMaxDevices]) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_symbol_mu);
  if (!table[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess) return nullptr;
    table[dev] = p;
  }
  return table[dev];
}

unsigned int* timeout_counter() {
  return static_cast<unsigned int*>(symbol_address(g_wait_timeouts, g_timeouts_ptr));
}

// Device address of the current device's no-alloc scratch.
void* noalloc_scratch() { return symbol_address(g_noalloc_scratch, g_noalloc_ptr); }

// Raise a kernel's dynamic shared-memory limit once per device (the attribute is per
// device context, so a process that drives several GPUs sets it on each).
std::mutex g_smem_mu;
bool smem_attr_set(const void* func, int bytes, unsigned char (&done)[kMaxDevices]) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_smem_mu);
  if (!done[dev]) {
    if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
      return false;
    done[dev] = 1;
  }
  return true;
}
}

using namespace kvring;

namespace {

constexpr uint64_t kMagic = 0x6B7672696E673031ull;  // "kvring01"
constexpr int kOpaqueTmapK = 0;                     // K codes, no swizzle
constexpr int kOpaqueTmapV = 16;                    // V codes, no swizzle
constexpr int kOpaqueTmapKsw = 32;                  // K codes, 128-byte swizzle (D = 128)
constexpr int kOpaqueTmapVsw = 48;                  // V codes, 128-byte swizzle (D = 128)
constexpr int kOpaqueMagic = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t mod_c(int64_t a, int64_t c) {
  int64_t r = a % c;
  return r < 0 ? r + c : r;
}

// (cos, sin) of p * theta_i, theta_i = base^(-2i/D), binary64 angle, rounded to binary32.
void rope_angles(int64_t p, int D, double base, float* out /* [D/2][2] */) {
  for (int i = 0; i < D / 2; ++i) {
    const double theta_i = pow(base, -(2.0 * (double)i) / (double)D);
    const double angle = (double)p * theta_i;
    out[2 * i] = (float)cos(angle);
    out[2 * i + 1] = (float)sin(angle);
  }
}

bool rope_is_3d(const kv_ring_t* kv) {
  return (kv->rope_pairs_t | kv->rope_pairs_h | kv->rope_pairs_w) != 0;
}

// 3-D form: token position p -> (frame, row, column) of a raster-ordered grid_h x grid_w
// frame; pair k of the time/height/width run of n pairs turns by that coordinate times
// base^(-2k/(2n)), binary64, rounded to binary32.
void rope_angles_3d(int64_t p, int D, double base, const int (&pairs)[3], int64_t grid_h,
                    int64_t grid_w, float* out /* [D/2][2] */) {
  const int64_t hw = grid_h * grid_w;
  int64_t f = p / hw;
  if (p < 0 && f * hw != p) f -= 1;                          // floor division
  const int64_t rest = p - f * hw;
  const int64_t coord[3] = {f, rest / grid_w, rest % grid_w};
  int i = 0;
  for (int run = 0; run < 3; ++run) {
    for (int k = 0; k < pairs[run] && i < D / 2; ++k, ++i) {
      const double theta = pow(base, -(2.0 * (double)k) / (double)(2 * pairs[run]));
      const double angle = (double)coord[run] * theta;
      out[2 * i] = (float)cos(angle);
      out[2 * i + 1] = (float)sin(angle);
    }
  }
}

// Angles of position p under the ring's rule.
void ring_angles(const kv_ring_t* kv, int64_t p, float* out) {
  if (!rope_is_3d(kv)) {
    rope_angles(p, kv->head_dim, kv->rope_base, out);
    return;
  }
  const int pairs[3] = {kv->rope_pairs_t, kv->rope_pairs_h, kv->rope_pairs_w};
  rope_angles_3d(p, kv->head_dim, kv->rope_base, pairs, kv->rope_grid_h, kv->rope_grid_w, out);
}

bool rope3d_valid(int D, int pt, int ph, int pw, int gh, int gw) {
  return pt >= 0 && ph >= 0 && pw >= 0 && (int64_t)pt + ph + pw == D / 2 && gh >= 1 &&
         gw >= 1 && (int64_t)gh * gw <= ((int64_t)1 << 24);
}

int check_ring(const kv_ring_t* kv) {
  if (!kv) return KV_EINVAL;
  if (!kv->initialized || kv->opaque[kOpaqueMagic] != kMagic) return KV_ESTATE;
  const int64_t C = kv->capacity;
  if (kv->write_slot < 0 || kv->write_slot >= C || kv->live < 0 || kv->live > C ||
      kv->pending < 0 || kv->pending > C)
    return KV_ESTATE;
  return KV_OK;
}

int64_t valid_slots(const kv_ring_t* kv) {
  const int64_t v = kv->live + kv->pending;
  return v > kv->capacity ? kv->capacity : v;
}

bool in_table(const kv_ring_t* kv, int64_t p_first, int64_t p_last) {
  return p_first >= kv->rope_pos_min && p_last <= kv->rope_pos_max && p_first <= p_last;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D map over codes [H][C][D] bytes; box = D bytes x box_rows slots x 1 head.  Slots
// >= C read as zero.  swizzle128: rows land in shared memory with the 128-byte swizzle
// the tensor core expects for a K-major operand (requires D = 128).
int encode_codes_map(void* base, int H, int C, int D, uint64_t* dst, bool swizzle128,
                     unsigned box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return KV_ECUDA;
  alignas(64) CUtensorMap m;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)C, (cuuint64_t)H};
  const cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)C * (cuuint64_t)D};
  const cuuint32_t box[3] = {(cuuint32_t)D, box_rows, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return KV_ECUDA;
  static_assert(sizeof(CUtensorMap) == 128, "CUtensorMap is 128 bytes");
  memcpy(dst, &m, sizeof(m));
  return KV_OK;
}

}  // namespace

extern "C" {

const char* kv_status_string(int status) {
  switch (status) {
    case KV_OK: return "ok";
    case KV_EINVAL: return "invalid argument (null pointer, shape, dtype, flag or alignment)";
    case KV_ERANGE: return "count or position out of range of the ring or the RoPE table";
    case KV_EUNSUPPORTED: return "unsupported configuration (head_dim or device)";
    case KV_ECUDA: return "CUDA runtime or driver call failed";
    case KV_ESTATE: return "ring not initialised or its state is inconsistent";
    default: return "unknown status";
  }
}

int kv_rope_table_build(float* host_out, int64_t pos_min, int64_t pos_max, int head_dim,
                        double base) {
  if (!host_out || head_dim <= 0 || (head_dim & 1) || pos_max < pos_min || !(base > 0.0))
    return KV_EINVAL;
  for (int64_t p = pos_min; p <= pos_max; ++p)
    rope_angles(p, head_dim, base, host_out + (size_t)(p - pos_min) * head_dim);
  return KV_OK;
}

int kv_rope3d_table_build(float* host_out, int64_t pos_min, int64_t pos_max, int head_dim,
                          double base, int pairs_t, int pairs_h, int pairs_w, int grid_h,
                          int grid_w) {
  if (!host_out || head_dim <= 0 || (head_dim & 1) || pos_max < pos_min || !(base > 0.0))
    return KV_EINVAL;
  if (!rope3d_valid(head_dim, pairs_t, pairs_h, pairs_w, grid_h, grid_w)) return KV_EINVAL;
  const int pairs[3] = {pairs_t, pairs_h, pairs_w};
  for (int64_t p = pos_min; p <= pos_max; ++p)
    rope_angles_3d(p, head_dim, base, pairs, grid_h, grid_w,
                   host_out + (size_t)(p - pos_min) * head_dim);
  return KV_OK;
}

int kv_ring_init(kv_ring_t* kv) {
  if (!kv) return KV_EINVAL;
  kv->initialized = 0;
  if (kv->capacity < 1 || kv->n_heads < 1) return KV_EINVAL;
  if (kv->head_dim != 64 && kv->head_dim != 128) return KV_EUNSUPPORTED;
  if (!kv->k_codes || !kv->v_codes || !kv->k_scale || !kv->v_scale || !kv->slot_pos ||
      !kv->rope_table)
    return KV_EINVAL;
  if (!aligned16(kv->k_codes) || !aligned16(kv->v_codes) || !aligned16(kv->rope_table))
    return KV_EINVAL;
  if (kv->rope_pos_max < kv->rope_pos_min || !(kv->rope_base > 0.0)) return KV_EINVAL;
  if (rope_is_3d(kv) && !rope3d_valid(kv->head_dim, kv->rope_pairs_t, kv->rope_pairs_h,
                                      kv->rope_pairs_w, kv->rope_grid_h, kv->rope_grid_w))
    return KV_EINVAL;
  if ((int64_t)kv->capacity * kv->n_heads > (int64_t)1 << 31) return KV_ERANGE;
  if (kv->n_heads > 65535) return KV_ERANGE;          // heads index grid dimension y
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KV_ECUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return KV_ECUDA;
  if (major != 10 || minor != 0) return KV_EUNSUPPORTED;
  int rc = encode_codes_map(kv->k_codes, kv->n_heads, kv->capacity, kv->head_dim,
                            kv->opaque + kOpaqueTmapK, false, 128u);
  if (rc) return rc;
  rc = encode_codes_map(kv->v_codes, kv->n_heads, kv->capacity, kv->head_dim,
                        kv->opaque + kOpaqueTmapV, false, 128u);
  if (rc) return rc;
  if (kv->head_dim == 128) {   // swizzled 64-slot boxes for the head_dim-128 kernel
    rc = encode_codes_map(kv->k_codes, kv->n_heads, kv->capacity, kv->head_dim,
                          kv->opaque + kOpaqueTmapKsw, true, 64u);
    if (rc) return rc;
    rc = encode_codes_map(kv->v_codes, kv->n_heads, kv->capacity, kv->head_dim,
                          kv->opaque + kOpaqueTmapVsw, true, 64u);
    if (rc) return rc;
  }
  kv->opaque[kOpaqueMagic] = kMagic;
  kv->write_slot = 0;
  kv->live = 0;
  kv->pending = 0;
  kv->initialized = 1;
  return KV_OK;
}

int kv_ring_commit(kv_ring_t* kv) {
  int rc = check_ring(kv);
  if (rc) return rc;
  const int64_t C = kv->capacity;
  kv->write_slot = mod_c(kv->write_slot + kv->pending, C);
  kv->live = kv->live + kv->pending > C ? C : kv->live + kv->pending;
  kv->next_pos += kv->pending;
  kv->pending = 0;
  return KV_OK;
}

int kv_ring_write(kv_ring_t* kv, const void* k, const void* v, int in_dtype, int n_tokens,
                  uint32_t flags, void* stream) {
  int rc = check_ring(kv);
  if (rc) return rc;
  if (!k || !v || !aligned16(k) || !aligned16(v)) return KV_EINVAL;
  if (in_dtype != KV_DTYPE_BF16 && in_dtype != KV_DTYPE_FP32) return KV_EINVAL;
  if (flags & ~KV_COMMIT) return KV_EINVAL;
  if (n_tokens < 1 || n_tokens > kv->capacity) return KV_ERANGE;
  if (n_tokens < kv->pending) return KV_ESTATE;  // a rewrite must cover the pending chunk
  const int64_t p0 = kv->next_pos, p1 = kv->next_pos + n_tokens - 1;
  if (!in_table(kv, p0, p1) || p0 < INT32_MIN || p1 > INT32_MAX) return KV_ERANGE;
  WriteArgs a;
  a.k = k;
  a.v = v;
  a.kc = kv->k_codes;
  a.vc = kv->v_codes;
  a.ks = kv->k_scale;
  a.vs = kv->v_scale;
  a.slot_pos = kv->slot_pos;
  a.rope_row0 = kv->rope_table + (size_t)(p0 - kv->rope_pos_min) * kv->head_dim;
  a.n = n_tokens;
  a.H = kv->n_heads;
  a.C = kv->capacity;
  a.w = kv->write_slot;
  a.pos0 = p0;
  rc = launch_write(a, kv->head_dim, in_dtype, static_cast<cudaStream_t>(stream));
  if (rc) return rc;
  kv->pending = n_tokens;
  if (flags & KV_COMMIT) return kv_ring_commit(kv);
  return KV_OK;
}

int kv_ring_delta_rotate(kv_ring_t* kv, int64_t delta, void* stream) {
  int rc = check_ring(kv);
  if (rc) return rc;
  const int64_t nv = valid_slots(kv);
  const int64_t committed = nv - kv->pending;              // history still in the ring
  const int64_t lo = kv->next_pos - committed + delta;     // oldest valid position after
  const int64_t hi = kv->next_pos + (kv->pending > 0 ? kv->pending - 1 : 0) + delta;
  if (rope_is_3d(kv) && delta % ((int64_t)kv->rope_grid_h * kv->rope_grid_w) != 0)
    return KV_EINVAL;                                      // resets move whole frames
  if (delta < INT32_MIN || delta > INT32_MAX || lo < INT32_MIN || hi > INT32_MAX)
    return KV_ERANGE;
  if (nv > 0) {
    RotateArgs a;
    a.kc = kv->k_codes;
    a.ks = kv->k_scale;
    a.slot_pos = kv->slot_pos;
    a.H = kv->n_heads;
    a.C = kv->capacity;
    a.first_slot = mod_c(kv->write_slot + kv->pending - nv, kv->capacity);
    a.count = nv;
    a.delta = (int32_t)delta;
    ring_angles(kv, delta, a.cs);
    rc = launch_rotate(a, kv->head_dim, static_cast<cudaStream_t>(stream));
    if (rc) return rc;
  }
  kv->next_pos += delta;
  return KV_OK;
}

}  // extern "C"

namespace {

// Shared validation and argument set-up of the chunk-attention entry points.
int attention_args(const kv_ring_t* kv, const void* q, int n_q, int64_t q_pos0, int n_current,
                   const kv_block_mask_t* mask, const kv_cache_bias_t* bias,
                   float softmax_scale, void* out, float* lse, uint32_t flags, AttnArgs* a) {
  int rc = check_ring(kv);
  if (rc) return rc;
  if (flags & ~(KV_QK_FP8 | KV_PV_FP8)) return KV_EINVAL;
  if (n_q < 0 || n_current < 0) return KV_EINVAL;
  if ((flags & (KV_QK_FP8 | KV_PV_FP8)) && kv->head_dim != 128) return KV_EUNSUPPORTED;
  if (n_q == 0) return KV_OK;
  if (!q || !out || !aligned16(q) || !aligned16(out)) return KV_EINVAL;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return KV_EINVAL;
  const float b = bias ? bias->history_bias : 0.f;
  if (isnan(b) || b == INFINITY) return KV_EINVAL;
  kv_block_mask_t m = {1 << 30, 1 << 30, 1 << 30, 1 << 30};
  if (mask) {
    if (mask->q_first_len < 1 || mask->q_block_len < 1 || mask->k_first_len < 1 ||
        mask->k_block_len < 1)
      return KV_EINVAL;
    m = *mask;
  }
  const int64_t nv = valid_slots(kv);
  if (n_current > nv) return KV_ERANGE;
  if (!in_table(kv, q_pos0, q_pos0 + n_q - 1)) return KV_ERANGE;
  if ((int64_t)n_q * kv->n_heads > ((int64_t)1 << 31)) return KV_ERANGE;
  a->q = static_cast<const uint16_t*>(q);
  a->out = static_cast<uint16_t*>(out);
  a->lse = lse;
  a->k_scale = kv->k_scale;
  a->v_scale = kv->v_scale;
  a->rope_q0 = kv->rope_table + (size_t)(q_pos0 - kv->rope_pos_min) * kv->head_dim;
  a->n_q = n_q;
  a->H = kv->n_heads;
  a->C = kv->capacity;
  a->n_current = n_current;
  a->newest_slot = mod_c(kv->write_slot + kv->pending - 1, kv->capacity);
  a->n_valid = nv;
  a->q_first = m.q_first_len;
  a->q_block = m.q_block_len;
  a->k_first = m.k_first_len;
  a->k_block = m.k_block_len;
  const float log2e = 1.4426950408889634f;
  a->score_scale_log2 = softmax_scale * log2e;
  a->bias_log2 = b * log2e;
  a->timeouts = nullptr;
  a->part_o = nullptr;
  a->part_ml = nullptr;
  a->n_extra = 0;
  a->mode_b = (flags & KV_QK_FP8) ? 1 : 0;
  a->pv_fp8 = (flags & KV_PV_FP8) ? 1 : 0;
  a->rows = nullptr;
  a->n_rows = n_q;
  return KV_OK;
}

// The device-side wait-timeout counter (the one CUDA query of the set-up; host validation
// comes first so that argument errors are reported without a device).
int attach_timeouts(AttnArgs* a) {
  a->timeouts = timeout_counter();
  return a->timeouts ? KV_OK : KV_ECUDA;
}

}  // namespace

extern "C" {

int chunk_attention(const kv_ring_t* kv, const void* q, int n_q, int64_t q_pos0,
                    int n_current, const kv_block_mask_t* mask, const kv_cache_bias_t* bias,
                    float softmax_scale, void* out, float* lse, uint32_t flags, void* stream) {
  AttnArgs a;
  int rc = attention_args(kv, q, n_q, q_pos0, n_current, mask, bias, softmax_scale, out, lse,
                          flags, &a);
  if (rc || n_q == 0) return rc;
  if ((rc = attach_timeouts(&a))) return rc;
  return launch_attention(a, kv->head_dim, kv->opaque + kOpaqueTmapK,
                          kv->opaque + kOpaqueTmapV, kv->opaque + kOpaqueTmapKsw,
                          kv->opaque + kOpaqueTmapVsw, static_cast<cudaStream_t>(stream));
}

int chunk_attention_rows(const kv_ring_t* kv, const void* q, int n_q, int64_t q_pos0,
                         int n_current, const int32_t* rows, int n_rows,
                         const kv_block_mask_t* mask, const kv_cache_bias_t* bias,
                         float softmax_scale, void* out, float* lse, int n_splits,
                         void* workspace, size_t workspace_bytes, uint32_t flags,
                         void* stream) {
  AttnArgs a;
  int rc = attention_args(kv, q, n_q, q_pos0, n_current, mask, bias, softmax_scale, out, lse,
                          flags, &a);
  if (rc) return rc;
  if (n_rows < 0 || n_splits < 1 || n_splits > 64) return KV_EINVAL;
  if (n_q == 0 || n_rows == 0) return KV_OK;
  if (kv->head_dim != 128) return KV_EUNSUPPORTED;
  if (!rows || (reinterpret_cast<uintptr_t>(rows) & 3u)) return KV_EINVAL;
  if ((int64_t)n_rows * kv->n_heads > ((int64_t)1 << 31)) return KV_ERANGE;
  if (n_splits > 1) {
    const size_t need = chunk_attention_workspace_size(n_rows, kv->n_heads, kv->head_dim, n_splits);
    if (!workspace || !aligned16(workspace)) return KV_EINVAL;
    if (workspace_bytes < need) return KV_ERANGE;
  }
  if ((rc = attach_timeouts(&a))) return rc;
  a.rows = rows;
  a.n_rows = n_rows;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_splits == 1)
    return launch_attention_sm100_d128(a, kv->opaque + kOpaqueTmapKsw,
                                       kv->opaque + kOpaqueTmapVsw, s, 1);
  a.part_o = static_cast<float*>(workspace);
  a.part_ml = a.part_o + (size_t)n_splits * n_rows * kv->n_heads * kv->head_dim;
  rc = launch_attention_sm100_d128(a, kv->opaque + kOpaqueTmapKsw, kv->opaque + kOpaqueTmapVsw,
                                   s, n_splits);
  if (rc) return rc;
  return launch_split_combine(a, kv->head_dim, n_splits, s);
}

size_t chunk_attention_workspace_size(int n_q, int n_heads, int head_dim, int n_splits) {
  if (n_q < 0 || n_heads < 1 || head_dim < 1 || n_splits < 1) return 0;
  return (size_t)n_splits * (size_t)n_q * (size_t)n_heads * ((size_t)head_dim * 4 + 8);
}

int chunk_attention_suggest_splits(int n_q, int n_heads, int64_t n_keys, int n_sms) {
  if (n_q < 1 || n_heads < 1 || n_keys < 1 || n_sms < 1) return 1;
  const int64_t units = ((int64_t)n_q + 255) / 256 * n_heads;
  const int64_t n_tiles = (n_keys + 63) / 64;
  const double tiles = (double)n_tiles;
  const int z_max = (int)(n_tiles / 4 < 16 ? (n_tiles / 4 < 1 ? 1 : n_tiles / 4) : 16);
  int best = 1;
  double best_cost = 0.0;
  for (int z = 1; z <= z_max; ++z) {
    const int64_t waves = (units * z + n_sms - 1) / n_sms;
    const double cost = (double)waves * (tiles / z + 10.0);
    if (z == 1 || cost < best_cost) {
      best = z;
      best_cost = cost;
    }
  }
  // partials and their merge cost HBM traffic the waves leave out: split only for a clear gain
  const double unsplit = (double)((units + n_sms - 1) / n_sms) * (tiles + 10.0);
  return best_cost <= 0.9 * unsplit ? best : 1;
}

int chunk_attention_split(const kv_ring_t* kv, const void* q, int n_q, int64_t q_pos0,
                          int n_current, const kv_block_mask_t* mask,
                          const kv_cache_bias_t* bias, float softmax_scale, void* out,
                          float* lse, int n_splits, void* workspace, size_t workspace_bytes,
                          uint32_t flags, void* stream) {
  AttnArgs a;
  int rc = attention_args(kv, q, n_q, q_pos0, n_current, mask, bias, softmax_scale, out, lse,
                          flags, &a);
  if (rc || n_q == 0) return rc;
  if (kv->head_dim != 128) return KV_EUNSUPPORTED;
  if (n_splits < 1 || n_splits > 64) return KV_EINVAL;
  const size_t need = chunk_attention_workspace_size(n_q, kv->n_heads, kv->head_dim, n_splits);
  if (!workspace || !aligned16(workspace)) return KV_EINVAL;
  if (workspace_bytes < need) return KV_ERANGE;
  if ((rc = attach_timeouts(&a))) return rc;
  a.part_o = static_cast<float*>(workspace);
  a.part_ml = a.part_o + (size_t)n_splits * n_q * kv->n_heads * kv->head_dim;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = launch_attention_sm100_d128(a, kv->opaque + kOpaqueTmapKsw, kv->opaque + kOpaqueTmapVsw,
                                   s, n_splits);
  if (rc) return rc;
  return launch_split_combine(a, kv->head_dim, n_splits, s);
}

int chunk_attention_split_noalloc(const kv_ring_t* kv, const void* q, int n_q, int64_t q_pos0,
                                  int n_current, const kv_block_mask_t* mask,
                                  const kv_cache_bias_t* bias, float softmax_scale, void* out,
                                  float* lse, int n_splits, uint32_t flags, void* stream) {
  AttnArgs a;
  int rc = attention_args(kv, q, n_q, q_pos0, n_current, mask, bias, softmax_scale, out, lse,
                          flags, &a);
  if (rc || n_q == 0) return rc;
  if (kv->head_dim != 128) return KV_EUNSUPPORTED;
  if (n_splits < 1 || n_splits > 64) return KV_EINVAL;
  const size_t need = chunk_attention_workspace_size(n_q, kv->n_heads, kv->head_dim, n_splits);
  if (need > KV_NOALLOC_SCRATCH_BYTES) return KV_ERANGE;
  if ((rc = attach_timeouts(&a))) return rc;
  void* scratch = noalloc_scratch();
  if (!scratch) return KV_ECUDA;
  a.part_o = static_cast<float*>(scratch);
  a.part_ml = a.part_o + (size_t)n_splits * n_q * kv->n_heads * kv->head_dim;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = launch_attention_sm100_d128(a, kv->opaque + kOpaqueTmapKsw, kv->opaque + kOpaqueTmapVsw,
                                   s, n_splits);
  if (rc) return rc;
  return launch_split_combine(a, kv->head_dim, n_splits, s);
}

int chunk_attention_multi(const kv_ring_t* const* rings, int n_rings, const void* q, int n_q,
                          int64_t q_pos0, int n_current, const kv_block_mask_t* mask,
                          const kv_cache_bias_t* bias, float softmax_scale, void* out,
                          float* lse, int n_splits, void* workspace, size_t workspace_bytes,
                          uint32_t flags, void* stream) {
  if (!rings || n_rings < 1 || n_rings > KV_MAX_RINGS) return KV_EINVAL;
  AttnArgs a[KV_MAX_RINGS];
  for (int r = 0; r < n_rings; ++r) {
    if (!rings[r]) return KV_EINVAL;
    // every ring after the first holds history only
    int rc = attention_args(rings[r], q, n_q, q_pos0, r == 0 ? n_current : 0, mask, bias,
                            softmax_scale, out, lse, flags, &a[r]);
    if (rc) return rc;
    if (rings[r]->n_heads != rings[0]->n_heads || rings[r]->head_dim != rings[0]->head_dim ||
        rings[r]->rope_base != rings[0]->rope_base)
      return KV_EINVAL;
  }
  if (n_q == 0) return KV_OK;
  if (rings[0]->head_dim != 128) return KV_EUNSUPPORTED;
  if (n_splits < 1 || n_splits > 64 || n_rings * n_splits > 64) return KV_EINVAL;
  const int H = rings[0]->n_heads, D = rings[0]->head_dim, S = n_rings * n_splits;
  const size_t need = chunk_attention_workspace_size(n_q, H, D, S);
  if (!workspace || !aligned16(workspace)) return KV_EINVAL;
  if (workspace_bytes < need) return KV_ERANGE;
  if (int rc = attach_timeouts(&a[0])) return rc;
  // One launch reads every ring: each CTA visits the main ring's tiles, then the extra
  // rings' (all history).  The CTAs' fp32 partials go to the workspace only when the
  // keys are split; otherwise the kernel writes out and lse itself.
  AttnArgs m = a[0];
  const void* xk[KV_MAX_RINGS - 1];
  const void* xv[KV_MAX_RINGS - 1];
  m.n_extra = n_rings - 1;
  for (int r = 1; r < n_rings; ++r) {
    m.x_k_scale[r - 1] = a[r].k_scale;
    m.x_v_scale[r - 1] = a[r].v_scale;
    m.x_C[r - 1] = a[r].C;
    m.x_newest[r - 1] = (int)a[r].newest_slot;
    m.x_n_valid[r - 1] = (int)a[r].n_valid;
    xk[r - 1] = rings[r]->opaque + kOpaqueTmapKsw;
    xv[r - 1] = rings[r]->opaque + kOpaqueTmapVsw;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_splits > 1) {
    m.part_o = static_cast<float*>(workspace);
    m.part_ml = m.part_o + (size_t)n_splits * n_q * H * D;
  }
  int rc = launch_attention_sm100_d128(m, rings[0]->opaque + kOpaqueTmapKsw,
                                       rings[0]->opaque + kOpaqueTmapVsw, s, n_splits, xk, xv);
  if (rc || n_splits == 1) return rc;
  return launch_split_combine(m, D, n_splits, s);
}

int chunk_key_mass_multi(const kv_ring_t* main_ring, int n_sets,
                         const kv_ring_t* const* cand_rings, const void* q, int n_q,
                         int64_t q_pos0, const float* lse, const kv_cache_bias_t* bias,
                         float softmax_scale, const int64_t* slot_first, const int* n_cand,
                         float* const* mass, void* workspace, size_t workspace_bytes,
                         void* stream) {
  int rc = check_ring(main_ring);
  if (rc) return rc;
  if (n_sets < 1 || n_sets > KV_KEY_MASS_MAX_SETS || !cand_rings || !slot_first || !n_cand ||
      !mass)
    return KV_EINVAL;
  for (int t = 0; t < n_sets; ++t) {
    const kv_ring_t* cr = cand_rings[t];
    if (!cr) return KV_EINVAL;
    if ((rc = check_ring(cr))) return rc;
    if (main_ring->n_heads != cr->n_heads || main_ring->head_dim != cr->head_dim ||
        main_ring->rope_base != cr->rope_base)
      return KV_EINVAL;
  }
  if (main_ring->head_dim != 128) return KV_EUNSUPPORTED;
  if (n_q < 0) return KV_EINVAL;
  bool any = false;
  for (int t = 0; t < n_sets; ++t) {
    if (n_cand[t] < 0 || n_cand[t] > cand_rings[t]->capacity) return KV_EINVAL;
    if (slot_first[t] < 0 || slot_first[t] >= cand_rings[t]->capacity) return KV_EINVAL;
    any = any || n_cand[t] > 0;
  }
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return KV_EINVAL;
  const float b = bias ? bias->history_bias : 0.f;
  if (isnan(b) || b == INFINITY) return KV_EINVAL;
  if (n_q == 0 || !any) return KV_OK;
  if (!q || !lse || !aligned16(q) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return KV_EINVAL;
  for (int t = 0; t < n_sets; ++t)
    if (n_cand[t] > 0 && (!mass[t] || (reinterpret_cast<uintptr_t>(mass[t]) & 3u)))
      return KV_EINVAL;
  if (workspace && !aligned16(workspace)) return KV_EINVAL;
  if (workspace && workspace_bytes < key_mass_workspace_bytes(n_q, main_ring->n_heads))
    return KV_ERANGE;
  if (!in_table(main_ring, q_pos0, q_pos0 + n_q - 1)) return KV_ERANGE;
  KeyMassArgs a;
  memset(&a, 0, sizeof(a));
  a.q = static_cast<const uint16_t*>(q);
  a.rope_q0 = main_ring->rope_table + (size_t)(q_pos0 - main_ring->rope_pos_min) * 128;
  a.lse = lse;
  a.n_q = n_q;
  a.H = main_ring->n_heads;
  for (int t = 0; t < n_sets; ++t) {
    if (n_cand[t] == 0) continue;                     // nothing to score in this set
    const int u = a.n_sets++;
    a.kc[u] = cand_rings[t]->k_codes;
    a.ks[u] = cand_rings[t]->k_scale;
    a.mass[u] = mass[t];
    a.C[u] = cand_rings[t]->capacity;
    a.n_cand[u] = n_cand[t];
    a.slot_first[u] = (int)slot_first[t];
  }
  a.score_scale_log2 = softmax_scale * 1.4426950408889634f;
  a.bias_log2 = b * 1.4426950408889634f;
  a.qws = static_cast<uint8_t*>(workspace);
  a.timeouts = timeout_counter();
  if (!a.timeouts) return KV_ECUDA;
  return launch_key_mass(a, static_cast<cudaStream_t>(stream));
}

size_t chunk_key_mass_workspace_size(int n_q, int n_heads) {
  return key_mass_workspace_bytes(n_q, n_heads);
}

int chunk_key_mass(const kv_ring_t* main_ring, const kv_ring_t* cand_ring, const void* q,
                   int n_q, int64_t q_pos0, const float* lse, const kv_cache_bias_t* bias,
                   float softmax_scale, int64_t slot_first, int n_cand, float* mass,
                   void* stream) {
  if (!cand_ring) return KV_EINVAL;
  return chunk_key_mass_multi(main_ring, 1, &cand_ring, q, n_q, q_pos0, lse, bias,
                              softmax_scale, &slot_first, &n_cand, &mass, nullptr, 0, stream);
}

int kv_memory_select(const kv_ring_t* memory, const float* mass_memory, const kv_ring_t* fifo,
                     const float* mass_fifo, int64_t fifo_slot_first, int n_fifo, int budget,
                     int64_t frame_len, float gamma, kv_ring_t* memory_out, int32_t* kept,
                     void* stream) {
  int rc = check_ring(fifo);
  if (rc) return rc;
  if ((rc = check_ring(memory_out))) return rc;
  if (memory && (rc = check_ring(memory))) return rc;
  if (memory_out == memory || memory_out == fifo) return KV_EINVAL;
  if (memory_out->k_codes == fifo->k_codes || (memory && memory_out->k_codes == memory->k_codes))
    return KV_EINVAL;
  const kv_ring_t* others[2] = {memory, memory_out};
  for (const kv_ring_t* r : others) {
    if (r && (r->n_heads != fifo->n_heads || r->head_dim != fifo->head_dim)) return KV_EINVAL;
  }
  if (budget < 1 || frame_len < 1 || !(gamma > 0.f) || gamma > 1.f) return KV_EINVAL;
  if (n_fifo < 0 || n_fifo > fifo->capacity) return KV_ERANGE;
  if (fifo_slot_first < 0 || fifo_slot_first >= fifo->capacity) return KV_EINVAL;
  if (budget > memory_out->capacity) return KV_ERANGE;
  const int64_t n_mem = memory ? valid_slots(memory) : 0;
  if (n_mem + n_fifo > KV_MEMORY_MAX_CANDIDATES) return KV_ERANGE;
  if (!kept || (n_mem > 0 && !mass_memory) || (n_fifo > 0 && !mass_fifo)) return KV_EINVAL;
  const int64_t m = n_mem + n_fifo < budget ? n_mem + n_fifo : budget;
  SelectArgs a;
  a.mass_mem = mass_memory;
  a.mass_fifo = mass_fifo;
  a.mem_kc = memory ? memory->k_codes : nullptr;
  a.mem_vc = memory ? memory->v_codes : nullptr;
  a.mem_ks = memory ? memory->k_scale : nullptr;
  a.mem_vs = memory ? memory->v_scale : nullptr;
  a.mem_pos = memory ? memory->slot_pos : nullptr;
  a.mem_C = memory ? memory->capacity : 1;
  a.n_mem = (int)n_mem;
  a.mem_slot_first =
      memory ? (int)mod_c(memory->write_slot + memory->pending - n_mem, memory->capacity) : 0;
  a.fifo_kc = fifo->k_codes;
  a.fifo_vc = fifo->v_codes;
  a.fifo_ks = fifo->k_scale;
  a.fifo_vs = fifo->v_scale;
  a.fifo_pos = fifo->slot_pos;
  a.fifo_C = fifo->capacity;
  a.n_fifo = n_fifo;
  a.fifo_slot_first = (int)fifo_slot_first;
  a.H = fifo->n_heads;
  a.M = budget;
  a.frame_len = frame_len;
  a.gamma = gamma;
  a.kept = kept;
  a.out_kc = memory_out->k_codes;
  a.out_vc = memory_out->v_codes;
  a.out_ks = memory_out->k_scale;
  a.out_vs = memory_out->v_scale;
  a.out_pos = memory_out->slot_pos;
  a.out_C = memory_out->capacity;
  if (m > 0) {
    rc = launch_memory_select(a, static_cast<cudaStream_t>(stream));
    if (rc) return rc;
  }
  memory_out->write_slot = mod_c(m, memory_out->capacity);
  memory_out->live = m;
  memory_out->pending = 0;
  return KV_OK;
}

int kv_wait_timeout_count(uint32_t* host_count) {
  if (!host_count) return KV_EINVAL;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, kvring::g_wait_timeouts, sizeof(v)) != cudaSuccess)
    return KV_ECUDA;
  *host_count = v;
  return KV_OK;
}

}  // extern "C"
