/*
 * kvring.h -- C ABI of the ring KV-cache attention library (libkvring.so, sm_100a).
 *
 * One hot path of chunk-wise autoregressive video diffusion, on one GPU:
 *   write side: a ring KV cache; RoPE and FP8 (e4m3, one fp32 scale per token and head)
 *               are applied once, when a token is written; a delta rotation re-rotates
 *               the cached keys when positions reset.
 *   read side:  a chunk of new queries attends over the whole cache under a block-causal
 *               mask, with an additive bias on history slots.
 * Sources: "Runway Characters: Serving a 57B Video Diffusion Transformer for Real-Time
 * Conversation" (abstract: ring cache, RoPE + FP8 once per write, delta rotation on
 * position reset, 240 calls per chunk over a 5,788-slot cache with 757 new tokens);
 * "KREA Real-Time 14B / video-conductor" (section "Plastic Windows": lowering the cache
 * attention bias); "Why Live Video Generation Still Struggles With Timing" (bidirectional
 * inside the current chunk, backward-only across chunks, sliding window of history);
 * "Stream LTX" (section "Training": blocks and causal masks on every attention path).
 *
 * Conventions shared by every entry point
 *  - Ownership: the caller allocates and owns every device buffer and the CUDA stream.
 *    The library allocates no device memory at run time and never synchronises the
 *    stream.  Kernels are enqueued on `stream` (a cudaStream_t; NULL is the legacy default
 *    stream) and read/write only the buffers named in the call, plus the library's own
 *    module-level device state: a wait-timeout counter (kv_wait_timeout_count) and the
 *    scratch of chunk_attention_split_noalloc, one of each per device, present from module
 *    load.  The host keeps, per device, the addresses of those two symbols (looked up on
 *    first use, then cached) and whether each kernel's shared-memory limit has been
 *    raised; these tables are guarded by mutexes.
 *  - Errors: every function returns KV_OK (0) or a negative KV_E* code.  Argument, shape,
 *    state and range errors are detected on the host before anything is enqueued, and
 *    leave the ring state unchanged.  A launch failure returns KV_ECUDA (the CUDA error
 *    is also left for cudaGetLastError).  Faults during execution surface as CUDA errors
 *    at the caller's next synchronisation.  Nothing aborts, throws or traps.
 *  - Concurrency: one kv_ring_t per stream/session.  Calls on the same ring must be
 *    ordered on one stream; the host-side state fields are updated when a call is
 *    enqueued, not when it completes.
 *
 * Numerics (bit-exact contract for codes, scales and slot positions)
 *  - RoPE: 1-D positions, interleaved pairs (x[2i], x[2i+1]); angle p * theta_i with
 *    theta_i = base^(-2i/D) evaluated in binary64 as pow(base, -(2i)/D); the table holds
 *    c = (float)cos(angle), s = (float)sin(angle).  Rotation, in binary32 with separate
 *    round-to-nearest-even operations (no fused multiply-add, no flush to zero):
 *        y0 = (x0*c) - (x1*s),   y1 = (x0*s) + (x1*c).
 *  - Quantisation of a D-element row y: amax = max|y_i|; scale = amax/448,
 *    inv = 448/amax (binary32 divisions); code_i = e4m3(y_i * inv), OCP e4m3fn,
 *    round-to-nearest-even, saturating to +-448.  amax == 0, or 448/amax not finite:
 *    scale 0, codes 0.  A row with a non-finite element: scale NaN (bits 0x7FC00000),
 *    all codes 0x7F.
 *  - Attention: q~ = bf16_rne(RoPE(q, q_pos0 + i)); k~ = e4m3(kc) * ks; v~ = e4m3(vc) * vs;
 *    s_ij = softmax_scale * <q~_i, k~_j> + (slot j is history ? history_bias : 0);
 *    masked pairs are excluded; out_i = sum_j softmax_j(s_i) v~_j; lse_i = log sum exp.
 *    Accumulation is fp32 on tensor cores; accuracy vs an fp64 evaluation of the same
 *    definition is a tolerance, not bit-exact.
 */
#ifndef KVRING_H
#define KVRING_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KV_API __attribute__((visibility("default")))
#else
#define KV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status codes */
#define KV_OK 0
#define KV_EINVAL (-1)        /* null pointer, bad shape, bad dtype, bad flag, misaligned */
#define KV_ERANGE (-2)        /* a count or position outside what the ring/table holds */
#define KV_EUNSUPPORTED (-3)  /* head_dim not 64/128, device is not sm_100, ... */
#define KV_ECUDA (-4)         /* a CUDA runtime/driver call failed */
#define KV_ESTATE (-5)        /* ring not initialised, or state fields inconsistent */

/* ------------------------------------------------------------------ input dtypes */
#define KV_DTYPE_BF16 1
#define KV_DTYPE_FP32 2

/* ------------------------------------------------------------------ flags */
#define KV_COMMIT 1u          /* kv_ring_write: commit the chunk after writing it */
#define KV_QK_FP8 1u          /* chunk_attention*: "mode B" -- the rotated bf16 query row is
                                 also quantised to e4m3 by the write's row rule (one fp32
                                 scale per row) and Q.K^T runs as one e4m3 MMA set instead
                                 of the exact hi + lo pair; head_dim 128 only */
#define KV_PV_FP8 2u          /* chunk_attention*: the fast, less exact P.V -- P (times the
                                 key's V scale) is rounded to e4m3 (2^-4 relative) and P.V
                                 runs as e4m3 MMAs on the raw V codes.  Its error against
                                 the definition is measured and reported, not bounded by
                                 the acceptance tolerance ("KREA Real-Time 14B /
                                 video-conductor", "What didn't": FP8 by default cost
                                 quality); head_dim 128 only */

/* Per-stream ring-head state.  Plain data: the caller fills the shape, the device
 * pointers, the RoPE table fields and next_pos, then calls kv_ring_init.  Copying the
 * struct together with the device buffers it points to is a complete snapshot.
 *
 * Device layouts (all row-major, caller-allocated, 16-byte aligned):
 *   k_codes, v_codes  uint8  [n_heads][capacity][head_dim]   e4m3fn codes
 *   k_scale, v_scale  float  [n_heads][capacity]             one scale per token, head
 *   slot_pos          int32  [capacity]                      RoPE position of each slot
 *   rope_table        float  [rope_pos_max-rope_pos_min+1][head_dim/2][2]  (cos, sin)
 * Ring semantics ("Runway Characters", abstract: a ring cache; "Why Live Video
 * Generation Still Struggles With Timing": a sliding window of recent history):
 *   the pending chunk occupies slots [write_slot, write_slot+pending) mod capacity;
 *   committed history occupies the `live` slots before write_slot (FIFO overwrite);
 *   valid slots = min(live + pending, capacity), the newest ending at
 *   write_slot + pending - 1 (mod capacity). */
typedef struct kv_ring {
  int32_t capacity;          /* C: number of slots, >= 1 */
  int32_t n_heads;           /* H, 1..65535 */
  int32_t head_dim;          /* D: 64 or 128 */
  int32_t initialized;       /* set by kv_ring_init; do not write */
  int64_t write_slot;        /* physical slot of the first pending/next token, [0, C) */
  int64_t live;              /* committed valid slots, [0, C] */
  int64_t pending;           /* tokens written at write_slot but not committed */
  int64_t next_pos;          /* RoPE position of the first pending/next token */
  uint8_t* k_codes;
  uint8_t* v_codes;
  float* k_scale;
  float* v_scale;
  int32_t* slot_pos;
  const float* rope_table;   /* device copy of kv_rope_table_build's output */
  int64_t rope_pos_min;      /* first position held by rope_table */
  int64_t rope_pos_max;      /* last position held by rope_table */
  double rope_base;          /* base used to build the table (for the delta rotation) */
  /* 3-D RoPE (all three pair counts 0 = 1-D RoPE): pairs of the time, height and width
   * runs of the head dimension (their sum is head_dim/2) and the frame grid
   * (rope_grid_h x rope_grid_w tokens per frame, raster order).  The table must then be
   * built by kv_rope3d_table_build with the same values. */
  int32_t rope_pairs_t, rope_pairs_h, rope_pairs_w;
  int32_t rope_grid_h, rope_grid_w;
  int32_t rope_reserved;     /* 0 */
  uint64_t opaque[96];       /* library-owned: encoded TMA descriptors of the caches */
} kv_ring_t;

/* Block-causal mask of the current chunk ("Stream LTX", section "Training": a block is
 * the unit inside which attention is bidirectional; across blocks it only looks back;
 * "Why Live Video Generation Still Struggles With Timing": bidirectional within the
 * chunk, backward across chunks).  Block id of chunk token t:
 *   t < first_len ? 0 : 1 + (t - first_len) / block_len     (queries: q_*, keys: k_*)
 * A current-chunk key is visible iff its block id <= the query's.  History keys are
 * always visible.  block_len = first_len = 1 gives token-causal masking; a length larger
 * than the chunk gives one bidirectional block.  NULL means one block. */
typedef struct kv_block_mask {
  int32_t q_first_len, q_block_len, k_first_len, k_block_len; /* all >= 1 */
} kv_block_mask_t;

/* Additive logit on history slots ("KREA Real-Time 14B / video-conductor", section
 * "Plastic Windows": lowering the cache attention bias opens a plastic window during
 * prompt transitions; read here as a natural-log offset added after softmax_scale).
 * NULL means 0.  -INFINITY removes history entirely. */
typedef struct kv_cache_bias {
  float history_bias;
} kv_cache_bias_t;

/* Fill host_out[(p - pos_min) * D + 2*i + {0,1}] = (cos, sin)(p * theta_i), rounded to
 * binary32, for pos_min <= p <= pos_max and i < D/2, by the RoPE rule above.  Host only
 * ("Runway Characters", abstract: RoPE applied once per write).  host_out holds
 * (pos_max - pos_min + 1) * D floats.  Errors: KV_EINVAL (null, D not even, pos_max <
 * pos_min, base <= 0). */
KV_API int kv_rope_table_build(float* host_out, int64_t pos_min, int64_t pos_max, int head_dim,
                        double base);

/* 3-D RoPE table: the same layout and binary32 rounding as kv_rope_table_build, for the
 * video form of RoPE ("Why Live Video Generation Still Struggles With Timing",
 * Transcript: positions of long streams are calibrated and reset along time; the run
 * split and frame grid are the usual video-DiT layout).  Token position p is frame
 * f = floor(p / (grid_h * grid_w)), row y = floor(p / grid_w) mod grid_h and column
 * x = p mod grid_w; pairs [0, pairs_t) turn by f * theta, the next pairs_h by y * theta,
 * the last pairs_w by x * theta, where the k-th pair of a run of n pairs has
 * theta = base^(-2k / (2n)) (pow in binary64, angle in binary64, cos/sin rounded to
 * binary32).  With pairs (D/2, 0, 0) and a 1 x 1 grid the table is kv_rope_table_build's.
 * The kernels read the table by position, so the write, the query rotation and the
 * attention are unchanged.  Errors: KV_EINVAL (null, pairs negative or not summing to
 * D/2, grid < 1, pos_max < pos_min, base <= 0). */
KV_API int kv_rope3d_table_build(float* host_out, int64_t pos_min, int64_t pos_max, int head_dim,
                                 double base, int pairs_t, int pairs_h, int pairs_w,
                                 int grid_h, int grid_w);

/* Validate a filled kv_ring_t, check the current device is sm_100, encode the TMA
 * descriptors of the caches into kv->opaque, and reset write_slot, live and pending to 0
 * (next_pos is kept).  Must be called again after any device pointer changes.
 * 3-D RoPE fields: all pair counts 0 (1-D), or non-negative counts summing to head_dim/2
 * with rope_grid_h, rope_grid_w >= 1 and rope_grid_h * rope_grid_w <= 2^24.
 * Errors: KV_EINVAL, KV_EUNSUPPORTED, KV_ECUDA. */
KV_API int kv_ring_init(kv_ring_t* kv);

/* Write n_tokens new tokens as the pending chunk ("Runway Characters", abstract: RoPE and
 * FP8 quantisation applied once per write).  k, v: device [n_tokens][H][D] in in_dtype
 * (KV_DTYPE_BF16 or KV_DTYPE_FP32), 16-byte aligned.  Token t goes to slot
 * (write_slot + t) mod C at position next_pos + t: K is rotated then quantised, V is
 * quantised; scales and slot_pos are written.  A previous pending chunk is replaced
 * (denoising passes rewrite the same chunk); the rewrite must be at least as long as the
 * pending chunk it replaces (else KV_ESTATE).  With KV_COMMIT the chunk is then
 * committed as by kv_ring_commit.  Errors: KV_EINVAL, KV_ERANGE (n_tokens < 1 or > C,
 * a position outside the table), KV_ESTATE, KV_ECUDA. */
KV_API int kv_ring_write(kv_ring_t* kv, const void* k, const void* v, int in_dtype, int n_tokens,
                  uint32_t flags, void* stream);

/* Commit the pending chunk: write_slot += pending (mod C), live = min(C, live + pending),
 * next_pos += pending, pending = 0.  Host only.  Errors: KV_EINVAL, KV_ESTATE. */
KV_API int kv_ring_commit(kv_ring_t* kv);

/* Position reset ("Runway Characters", abstract: a delta rotation when positions reset):
 * every valid cached key row is dequantised (code * scale, binary32), rotated by the
 * angles of `delta` (computed on the host by the ring's RoPE rule with kv->rope_base) and
 * requantised by the rule above; slot_pos of valid slots and next_pos shift by delta.
 * V is untouched.  Under 3-D RoPE a reset moves time only: delta must be a whole number
 * of frames (a multiple of rope_grid_h * rope_grid_w), whose angles are zero on the
 * height and width runs (those pairs pass through the rotation unchanged and are
 * requantised with the row).  Errors: KV_EINVAL (also a 3-D delta that is not a whole
 * number of frames), KV_ERANGE (shifted positions leave int32), KV_ESTATE, KV_ECUDA. */
KV_API int kv_ring_delta_rotate(kv_ring_t* kv, int64_t delta, void* stream);

/* Chunk attention ("Runway Characters", abstract: each call reads the whole cache, only
 * the newest tokens are new).  q: device bf16 [n_q][H][D]; query i is rotated at
 * q_pos0 + i.  Keys are the valid slots; the newest n_current of them are the current
 * chunk (masked by `mask`, no bias), the rest are history (bias added, always visible).
 * out: device bf16 [n_q][H][D]; lse: device fp32 [H][n_q] natural-log sum of exp, or
 * NULL.  A row with no visible key gets out = 0 and lse = -inf.  softmax_scale > 0.
 * flags: 0 (the query stays bf16: exact, "mode A"), KV_QK_FP8 (mode B; its result
 * matches the definition evaluated on the quantised-then-dequantised query) and/or
 * KV_PV_FP8 (e4m3 P.V, see above).  Errors: KV_EINVAL (also an unknown flag), KV_ERANGE
 * (n_current > valid slots, a query position outside the table), KV_EUNSUPPORTED
 * (KV_QK_FP8 or KV_PV_FP8 at head_dim 64), KV_ESTATE, KV_ECUDA. */
KV_API int chunk_attention(const kv_ring_t* kv, const void* q, int n_q, int64_t q_pos0,
                    int n_current, const kv_block_mask_t* mask, const kv_cache_bias_t* bias,
                    float softmax_scale, void* out, float* lse, uint32_t flags, void* stream);

/* Chunk attention for a gathered subset of the chunk's query rows ("Why Live Video
 * Generation Still Struggles With Timing", Transcript, the LiveEdit passage: a mask cache
 * finds the edited regions and self-attention is recomputed only there).  q, n_q, q_pos0,
 * n_current, mask, bias, softmax_scale, out, lse and flags mean what they mean for
 * chunk_attention, for the whole chunk of n_q queries.  rows: device int32 [n_rows],
 * 4-byte aligned, the chunk indices of the queries to compute, in any order, duplicates
 * allowed.  For each listed index i in [0, n_q), out[i] and lse[:, i] receive exactly
 * the values chunk_attention writes there (query rotated at q_pos0 + i, block id of i);
 * every other row of out and lse is left as it was (the static regions keep their
 * previous outputs).  A listed index outside [0, n_q) is skipped: nothing is computed or
 * written for it (the indices live on the device, so the host cannot reject them).
 * n_rows = 0 enqueues nothing.  head_dim 128 only.
 * n_splits (1..64) splits the keys as chunk_attention_split does, so that few listed rows
 * still fill the SMs: each split writes fp32 partials per list entry into workspace
 * (device, 16-byte aligned, caller-owned, at least
 * chunk_attention_workspace_size(n_rows, n_heads, head_dim, n_splits) bytes), and one
 * merge writes the listed rows.  With n_splits = 1 the workspace is not used (may be
 * NULL).  Errors: those of chunk_attention, KV_EINVAL (rows null or misaligned,
 * n_rows < 0, n_splits outside 1..64, workspace null or misaligned for n_splits > 1),
 * KV_ERANGE (n_rows * n_heads > 2^31, workspace too small), KV_EUNSUPPORTED
 * (head_dim 64). */
KV_API int chunk_attention_rows(const kv_ring_t* kv, const void* q, int n_q, int64_t q_pos0,
                                int n_current, const int32_t* rows, int n_rows,
                                const kv_block_mask_t* mask, const kv_cache_bias_t* bias,
                                float softmax_scale, void* out, float* lse, int n_splits,
                                void* workspace, size_t workspace_bytes, uint32_t flags,
                                void* stream);

/* Bytes of workspace chunk_attention_split needs: n_splits * n_q * n_heads * (4*head_dim + 8).
 * 0 for invalid arguments. */
KV_API size_t chunk_attention_workspace_size(int n_q, int n_heads, int head_dim, int n_splits);

/* Key splits (1..16) for chunk_attention_split on a GPU of n_sms SMs (148 on B200) that
 * fill it in whole waves: head_dim-128 attention runs one CTA per 256 query rows and
 * head per SM, so n_q queries x n_heads over n_keys valid slots make
 * ceil(n_q / 256) * n_heads CTAs of ceil(n_keys / 64) key tiles each.  The choice
 * minimises waves * (tiles / splits + 10), the 10 standing for a CTA's fixed cost (query
 * prologue, epilogue, partials) in key tiles; ties go to fewer splits, and no split gets
 * fewer than 4 key tiles.  Unless that cost is at most 0.9 of the unsplit one, the answer
 * is 1: the fp32 partials and their merge cost HBM traffic the count leaves out.  Host
 * arithmetic only; 1 for arguments out of range. */
KV_API int chunk_attention_suggest_splits(int n_q, int n_heads, int64_t n_keys, int n_sms);

/* chunk_attention with the keys split over n_splits (1..64) groups of consecutive valid
 * tiles, for few queries over a long ring (e.g. the 25 audio latents of a 1 s block in
 * "Stream LTX", section "Training", attending a 20-block video ring): every split keeps
 * its own online softmax and writes an unnormalised fp32 partial (O, max, sum) into
 * `workspace`; a second kernel merges the partials (max over splits, weights 2^(m_s - M))
 * into out and lse.  Same result and contract as chunk_attention up to fp32 rounding.
 * workspace: device, 16-byte aligned, caller-owned, at least
 * chunk_attention_workspace_size(n_q, H, D, n_splits) bytes, contents need not be
 * initialised; calls that share a workspace must be ordered on one stream.  head_dim 128
 * only.  Errors: those of chunk_attention, KV_EINVAL (n_splits, workspace null or
 * misaligned), KV_ERANGE (workspace too small), KV_EUNSUPPORTED (head_dim 64). */
KV_API int chunk_attention_split(const kv_ring_t* kv, const void* q, int n_q, int64_t q_pos0,
                                 int n_current, const kv_block_mask_t* mask,
                                 const kv_cache_bias_t* bias, float softmax_scale, void* out,
                                 float* lse, int n_splits, void* workspace,
                                 size_t workspace_bytes, uint32_t flags, void* stream);

/* Most rings one chunk_attention_multi call reads. */
#define KV_MAX_RINGS 8

/* Chunk attention over the stream's ring plus history-only rings, such as the first chunk
 * kept as a persistent anchor beside the sliding window ("Why Live Video Generation Still
 * Struggles With Timing", Transcript).  rings[0] is the stream's ring: its newest n_current
 * valid slots are the current chunk, exactly as in chunk_attention.  Every valid slot of
 * rings[1 .. n_rings) is history: always visible, cache_bias added.  The result is softmax
 * attention over the union of all rings' valid slots, with chunk_attention's contract for
 * out, lse, mask, softmax_scale and flags.
 * One launch reads every ring (each CTA visits the main ring's key tiles, then the extra
 * rings', under one online softmax).  The keys of all rings together are split over
 * n_splits groups as in chunk_attention_split; with n_splits > 1 the partials go to the
 * workspace and one merge writes out and lse, with n_splits = 1 the kernel writes them
 * itself.  The workspace must hold at least chunk_attention_workspace_size(n_q, H, 128,
 * n_rings * n_splits) bytes (device, 16-byte aligned, caller-owned, uninitialised is
 * fine); the launch uses its first n_splits slices.
 * rings: host array of n_rings (1..KV_MAX_RINGS) initialised rings with equal n_heads,
 * head_dim (128) and rope_base.  Each ring's RoPE table must cover q_pos0 .. q_pos0 + n_q - 1
 * (checked); the queries are rotated once, from rings[0]'s table, and every ring's keys
 * were rotated with the same angles (kv_rope_table_build with that base).
 * n_rings * n_splits <= 64.
 * Errors, all before anything is enqueued: KV_EINVAL (rings null or n_rings out of range,
 * a null entry, n_splits out of range, rings that differ in heads, head_dim or base, the
 * errors of chunk_attention_split), KV_EUNSUPPORTED (head_dim 64), KV_ERANGE (workspace too
 * small, n_current above rings[0]'s valid slots, a query position outside a table),
 * KV_ESTATE (a ring not initialised), KV_ECUDA. */
KV_API int chunk_attention_multi(const kv_ring_t* const* rings, int n_rings, const void* q,
                                 int n_q, int64_t q_pos0, int n_current,
                                 const kv_block_mask_t* mask, const kv_cache_bias_t* bias,
                                 float softmax_scale, void* out, float* lse, int n_splits,
                                 void* workspace, size_t workspace_bytes, uint32_t flags,
                                 void* stream);

/* Size of the library's own scratch for chunk_attention_split_noalloc: 16 MiB per
 * device.  8 splits of 25 queries x 32 heads x 128 take 3.3 MB; 4 splits of 1,024
 * queries x 8 heads x 128 (17.0 MB) do not fit. */
#define KV_NOALLOC_SCRATCH_BYTES (16u << 20)

/* chunk_attention_split without a caller workspace, for callers that cannot allocate
 * device memory at call time: a real-time loop whose memory was reserved up front (the
 * rings and the model own the whole HBM), code whose allocator must not be entered
 * while a step runs (cudaMalloc and cudaFree can synchronise the device and so stall
 * every other stream), or a plain C caller with no allocator at all.  The pages have no
 * counterpart; this is a convenience of this library.
 * The partials go to a static device buffer of KV_NOALLOC_SCRATCH_BYTES in the library
 * (one per device, 256-byte aligned).  The first call on a device looks up that
 * buffer's address (with that device current) and keeps it; make that first call
 * before any stream capture.  The call allocates nothing: no cudaMalloc, cudaFree or
 * allocating library routine.  Nothing in the scratch has to start at zero (every
 * partial is written before the merge reads it).  There is one scratch per device, so
 * calls that overlap in time on one device (other streams, other threads) race on it
 * and give wrong results: order them on one stream.
 * Arguments and result as chunk_attention_split.  Errors: those of
 * chunk_attention_split, and KV_ERANGE when chunk_attention_workspace_size(n_q, H, D,
 * n_splits) exceeds KV_NOALLOC_SCRATCH_BYTES (checked on the host before any CUDA
 * call); KV_ECUDA when the address lookup fails. */
KV_API int chunk_attention_split_noalloc(const kv_ring_t* kv, const void* q, int n_q,
                                         int64_t q_pos0, int n_current,
                                         const kv_block_mask_t* mask,
                                         const kv_cache_bias_t* bias, float softmax_scale,
                                         void* out, float* lse, int n_splits, uint32_t flags,
                                         void* stream);

/* ------------------------------------------------------------------ content memory
 * "Stream LTX", Inference: the long-context cache is an anchor, a content memory and a
 * FIFO of recent blocks; each layer scores its own keys on attention quality and temporal
 * diversity and evicts down to a top-M budget.  Here the FIFO is the stream's ring, the
 * anchor and the content memory are history-only rings read by chunk_attention_multi, and
 * the two calls below score and select.  The pages give no formula; the reading:
 *   quality of a key = the softmax probability it receives in the newest chunk's
 *     attention call, summed over heads and query rows (chunk_key_mass);
 *   diversity: the k-th best key of a frame (frame = floor(slot position / frame_len))
 *     scores quality * gamma^k; the budget keeps the best M (kv_memory_select). */

/* Attention mass of n_cand slots of cand_ring, the slots (slot_first + c) mod capacity,
 * c < n_cand: mass[h * n_cand + c] = sum over query rows i of exp(s_ihc - lse[h * n_q + i])
 * with s the call's score (softmax_scale * <q~_i, k~_c> + history bias), q~ rotated from
 * main_ring's RoPE table at q_pos0 + i.  q, n_q, q_pos0, bias and softmax_scale must be
 * those of the attention call whose lse [H][n_q] (device, natural log) is passed; the
 * slots must be history keys of that call (always visible, bias added).  Rows whose lse
 * is not finite add nothing.  mass: device fp32 [H][n_cand].  head_dim 128; both rings
 * initialised with equal n_heads, head_dim and rope_base.  Errors: KV_EINVAL (null or
 * misaligned pointers, rings that differ, n_cand < 0 or > capacity, slot_first outside
 * [0, capacity), softmax_scale), KV_ERANGE (a query position outside main_ring's table),
 * KV_EUNSUPPORTED (head_dim 64), KV_ESTATE, KV_ECUDA. */
KV_API int chunk_key_mass(const kv_ring_t* main_ring, const kv_ring_t* cand_ring, const void* q,
                          int n_q, int64_t q_pos0, const float* lse,
                          const kv_cache_bias_t* bias, float softmax_scale,
                          int64_t slot_first, int n_cand, float* mass, void* stream);

/* Most candidate sets of one chunk_key_mass_multi call. */
#define KV_KEY_MASS_MAX_SETS 4

/* chunk_key_mass for n_sets candidate sets of the same attention call in one launch, so
 * that the CTAs of all sets fill the GPU together (an eviction scores the memory ring's
 * slots and the FIFO block the next write overwrites).  Set t: the n_cand[t] slots
 * (slot_first[t] + c) mod capacity of cand_rings[t], masses to mass[t] (device fp32
 * [H][n_cand[t]]).  cand_rings, slot_first, n_cand and mass are host arrays of n_sets
 * entries, 1 <= n_sets <= KV_KEY_MASS_MAX_SETS; sets with n_cand 0 are skipped.
 * workspace: null, or device memory of at least chunk_key_mass_workspace_size(n_q, H)
 * bytes, 16-byte aligned, owned by the caller and free for the call's duration.  With
 * it the query rows are rotated and split once per call (a second kernel before the
 * scoring one) and the scoring CTAs stream them in; without it every CTA splits the
 * rows itself (slower, nothing to allocate).  Each candidate's sum adds its queries in
 * the same order either way.  Other arguments and errors as chunk_key_mass, checked for
 * every set before anything is launched; KV_EINVAL also for n_sets out of range, a null
 * array or a misaligned workspace, KV_ERANGE for a workspace that is too small. */
KV_API int chunk_key_mass_multi(const kv_ring_t* main_ring, int n_sets,
                                const kv_ring_t* const* cand_rings, const void* q, int n_q,
                                int64_t q_pos0, const float* lse,
                                const kv_cache_bias_t* bias, float softmax_scale,
                                const int64_t* slot_first, const int* n_cand,
                                float* const* mass, void* workspace, size_t workspace_bytes,
                                void* stream);

/* Bytes of workspace chunk_key_mass_multi takes for n_q query rows of n_heads heads:
 * n_heads * ceil(n_q / 64) * 16,896.  0 for n_q < 0 or n_heads < 1. */
KV_API size_t chunk_key_mass_workspace_size(int n_q, int n_heads);

/* Largest candidate count (memory slots + FIFO block) of one kv_memory_select call. */
#define KV_MEMORY_MAX_CANDIDATES 8192

/* Content-memory eviction: the candidates are the valid slots of `memory` (oldest first;
 * memory may be NULL for none) and the n_fifo slots (fifo_slot_first + c) mod capacity of
 * `fifo` (the block that the FIFO's next write overwrites), with their masses from
 * chunk_key_mass (device [H][n_mem] and [H][n_fifo]).  quality = sum over heads of the
 * masses (binary32, heads in order); frame = floor(slot_pos / frame_len); the k-th best
 * key of a frame (quality descending, ties toward the lower position, then the lower
 * candidate index) scores quality * gamma^k (binary32); the best min(n, budget) are kept.
 * kept: device int32 workspace of at least min(n_mem + n_fifo, budget) entries; it
 * receives the kept candidate indices (memory slots first, then the FIFO block), in
 * ascending order.  Their K and V codes, scales and positions are copied into slots
 * 0 .. kept - 1 of memory_out (a different ring with the same n_heads and head_dim and
 * capacity >= budget), whose state becomes write_slot = kept mod capacity, live = kept,
 * pending = 0 (next_pos unchanged).  Errors: KV_EINVAL (null or aligned pointers,
 * budget < 1, frame_len < 1, gamma outside (0, 1], memory_out aliasing memory or fifo,
 * rings that differ), KV_ERANGE (more than KV_MEMORY_MAX_CANDIDATES candidates,
 * memory_out too small, n_fifo outside [0, capacity]), KV_ESTATE, KV_ECUDA. */
KV_API int kv_memory_select(const kv_ring_t* memory, const float* mass_memory,
                            const kv_ring_t* fifo, const float* mass_fifo,
                            int64_t fifo_slot_first, int n_fifo, int budget, int64_t frame_len,
                            float gamma, kv_ring_t* memory_out, int32_t* kept, void* stream);

/* Static description of a status code.  Never NULL. */
KV_API const char* kv_status_string(int status);

/* Number of device-side waits (on TMA or tensor-core completion) that gave up after
 * about one second since the library was loaded on the current device.  A kernel whose
 * wait gave up abandons its work, writes NaN to the rows it owned and exits; a non-zero
 * count means those outputs are invalid.  Synchronous (reads a device word).  Errors:
 * KV_EINVAL (null), KV_ECUDA. */
KV_API int kv_wait_timeout_count(uint32_t* host_count);

#ifdef __cplusplus
}
#endif

#endif /* KVRING_H */
