// internal.h -- launch interfaces between the C ABI (kvring_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvring.h"

namespace kvring {

struct WriteArgs {
  const void* k;            // [n][H][D] input dtype
  const void* v;
  uint8_t* kc;              // [H][C][D]
  uint8_t* vc;
  float* ks;                // [H][C]
  float* vs;
  int32_t* slot_pos;        // [C]
  const float* rope_row0;   // table row of position `pos0`: [n][D/2][2] floats follow
  int n, H, C;
  int64_t w;                // first slot
  int64_t pos0;             // position of token 0
};

struct RotateArgs {
  uint8_t* kc;
  float* ks;
  int32_t* slot_pos;
  int H, C;
  int64_t first_slot;       // oldest valid slot
  int64_t count;            // valid slots (contiguous mod C from first_slot)
  int32_t delta;
  float cs[128];            // (cos, sin) of delta * theta_i, i < D/2, interleaved
};

struct AttnArgs {
  const uint16_t* q;        // bf16 [n_q][H][D]
  uint16_t* out;            // bf16 [n_q][H][D]
  float* lse;               // [H][n_q] or null
  const float* k_scale;     // [H][C]
  const float* v_scale;
  const float* rope_q0;     // table row of position q_pos0
  int n_q, H, C;
  int n_current;
  int64_t newest_slot;      // slot of the newest valid token
  int64_t n_valid;          // valid slots
  int q_first, q_block, k_first, k_block;
  float score_scale_log2;   // softmax_scale * log2(e)
  float bias_log2;          // history_bias * log2(e)
  unsigned int* timeouts;   // device counter of waits that gave up
  int mode_b;               // query quantised to e4m3 per row (one MMA set for Q.K^T)
  int pv_fp8;               // P quantised to e4m3, P.V on the raw V codes (fast, less exact)
  // rows computed: the query indices rows[0 .. n_rows) (device int32), or 0 .. n_rows - 1
  // when rows is null (then n_rows = n_q); indices outside [0, n_q) are skipped
  const int32_t* rows;
  int n_rows;
  // split over keys (gridDim.z splits): when part_o is set, each split writes its
  // unnormalised O [split][n_q][H][D] and (m, l) [split][H][n_q] (log2 units) there
  float* part_o;
  float* part_ml;
  // history-only rings read after the main ring in the same launch (chunk_attention_multi):
  // their scales [H][C], capacity, newest valid slot and number of valid slots
  int n_extra;
  const float* x_k_scale[KV_MAX_RINGS - 1];
  const float* x_v_scale[KV_MAX_RINGS - 1];
  int x_C[KV_MAX_RINGS - 1];
  int x_newest[KV_MAX_RINGS - 1];
  int x_n_valid[KV_MAX_RINGS - 1];
};

// Attention mass received by n_cand consecutive slots (from slot_first, mod C) of one
// ring: mass [H][n_cand] (see key_mass.cu).
struct KeyMassArgs {
  const uint16_t* q;        // bf16 [n_q][H][D]
  const float* rope_q0;     // main ring's table row of q_pos0
  const float* lse;         // [H][n_q] natural log, from the attention call
  int n_q, H;
  int n_sets;               // candidate sets, 1 .. KV_KEY_MASS_MAX_SETS
  // set t: candidate ring codes [H][C][D] and scales [H][C], masses [H][n_cand]; its CTAs
  // are blockIdx.x in [blk_first[t], blk_first[t + 1])
  const uint8_t* kc[KV_KEY_MASS_MAX_SETS];
  const float* ks[KV_KEY_MASS_MAX_SETS];
  float* mass[KV_KEY_MASS_MAX_SETS];
  int C[KV_KEY_MASS_MAX_SETS], n_cand[KV_KEY_MASS_MAX_SETS];
  int slot_first[KV_KEY_MASS_MAX_SETS];
  int blk_first[KV_KEY_MASS_MAX_SETS + 1];
  float score_scale_log2;   // softmax_scale * log2(e)
  float bias_log2;          // history_bias * log2(e)
  unsigned int* timeouts;
  uint8_t* qws;             // split query images (workspace), or null: split in every CTA
  int n_qt;                 // their 64-row tiles per head
};

// Bytes of the split query images of n_q rows x n_heads (the pipelined key mass).
size_t key_mass_workspace_bytes(int n_q, int n_heads);

// Top-M selection over a memory ring's slots and a FIFO block, and the gather of the kept
// entries into a fresh ring (see key_mass.cu).
struct SelectArgs {
  const float* mass_mem;    // [H][n_mem]
  const float* mass_fifo;   // [H][n_fifo]
  const uint8_t *mem_kc, *mem_vc, *fifo_kc, *fifo_vc;
  const float *mem_ks, *mem_vs, *fifo_ks, *fifo_vs;
  const int32_t *mem_pos, *fifo_pos;
  int n_mem, mem_slot_first, mem_C;
  int n_fifo, fifo_slot_first, fifo_C;
  int H, M;
  long long frame_len;
  float gamma;
  int32_t* kept;            // [min(n_mem + n_fifo, M)] candidate indices, ascending
  uint8_t *out_kc, *out_vc;
  float *out_ks, *out_vs;
  int32_t* out_pos;
  int out_C;
};

int launch_key_mass(const KeyMassArgs& a, cudaStream_t s);
int launch_memory_select(const SelectArgs& a, cudaStream_t s);
// Shared memory of the selection for n candidates (n rounded up to a power of two).
size_t select_smem_bytes(int n);

// Largest device ordinal the per-device tables cover.
constexpr int kMaxDevices = 64;

// Device address of the library's wait-timeout counter on the current device (looked up
// once per device, then cached).
unsigned int* timeout_counter();

// Set `func`'s dynamic shared-memory limit to `bytes` on the current device unless
// done[device] says it is set already; false if the CUDA call fails.
bool smem_attr_set(const void* func, int bytes, unsigned char (&done)[kMaxDevices]);

int launch_write(const WriteArgs& a, int D, int in_dtype, cudaStream_t s);
int launch_rotate(const RotateArgs& a, int D, cudaStream_t s);
// tmaps: 128-byte CUtensorMap images of the K and V codes without swizzle and with the
// 128-byte swizzle (the latter for D = 128 only).
int launch_attention(const AttnArgs& a, int D, const void* tmap_k, const void* tmap_v,
                     const void* tmap_k_sw128, const void* tmap_v_sw128, cudaStream_t s);
int launch_attention_sm100_d128(const AttnArgs& a, const void* tmap_k_sw128,
                                const void* tmap_v_sw128, cudaStream_t s, int n_splits = 1,
                                const void* const* x_tmap_k = nullptr,
                                const void* const* x_tmap_v = nullptr);
// Merge split partials into out (bf16) and lse.
int launch_split_combine(const AttnArgs& a, int D, int n_splits, cudaStream_t s);

}  // namespace kvring
