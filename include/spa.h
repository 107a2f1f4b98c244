/*
 * spa.h -- C ABI of libspa: paged / selected-token sparse attention over a
 * block-table KV cache, for NVIDIA B200 (sm_100a).
 *
 * The operation is the staged pipeline described on the onnxruntime pages
 * "[WebGPU] Add PagedAttention metadata and GPT-OSS support" (PR #32277),
 * "[WebGPU] Add SparsePagedAttention" (PR #32533), "[WebGPU] Add
 * DynamicSparseAttention" (PR #32529) and PR #33472 (INT8 KV cache):
 *   1. metadata prepare    -> spa_prepare_metadata
 *   2. KV append scatter   -> spa_append_kv
 *   3.-5. gather, scaled QK + joint softmax with a learned sink,
 *         split-KV partials + log-sum-exp combine -> spa_attention
 *
 * Conventions for every entry point:
 *   - Every pointer is a DEVICE pointer unless marked [host].  All buffers are
 *     owned by the caller; the library allocates no device memory, never
 *     synchronises the stream and never reads device memory from the host, so
 *     every call may be captured into a CUDA graph.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *   - The return value reports HOST-side problems only (SPA_OK or a negative
 *     SPA_ERR_* code; spa_error_string() gives a message).  When an error is
 *     returned nothing was enqueued.
 *   - Problems visible only on the device (malformed lengths, bad block ids,
 *     bad selected indices, host bounds exceeded) are OR-ed into the int32
 *     word `*status` (SPA_ST_* bits).  The caller clears it; kernels never
 *     clear it.  Whatever the inputs, every memory access stays inside the
 *     buffers whose sizes the arguments describe.  When a bit other than
 *     SPA_ST_BAD_IDX is set, the outputs of the affected requests are
 *     unspecified.
 *   - Integer layouts are int32, row-major, densely packed.
 */
#ifndef SPA_H_
#define SPA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so that the header needs no CUDA headers. */
typedef struct CUstream_st* spa_stream_t;

/* Element encodings. */
typedef enum {
  SPA_F32 = 0,  /* IEEE binary32                                   */
  SPA_F16 = 1,  /* IEEE binary16                                   */
  SPA_BF16 = 2, /* bfloat16                                        */
  SPA_I8 = 3    /* signed int8 with per-channel fp32 scales (cache) */
} spa_dtype_t;

/* Host-side return codes. */
#define SPA_OK 0
#define SPA_ERR_INVALID_ARG (-1) /* null required pointer, bad size, H_q % H_kv != 0, bad dtype combination */
#define SPA_ERR_UNSUPPORTED (-2) /* non-causal, main selection combined with window/aux, unsupported D */
#define SPA_ERR_WORKSPACE (-3)   /* workspace missing, too small or misaligned */
#define SPA_ERR_CUDA (-4)        /* a kernel launch failed; see spa_error_string(SPA_ERR_CUDA) */
#define SPA_ERR_SCRATCH_LIMIT (-5) /* spa_attention_noalloc: the call needs more than SPA_NOALLOC_SCRATCH_BYTES */

/* Device status bits (OR-ed into *status). */
#define SPA_ST_BAD_CU 0x1     /* cu_seqlens_q not non-decreasing from 0 to T, or a negative past length */
#define SPA_ST_CAPACITY 0x2   /* a position lies beyond the block table (pos >= MB * block_size) */
#define SPA_ST_BAD_BLOCK 0x4  /* a block-table entry needed by a position is outside [0, num_blocks) */
#define SPA_ST_BOUNDS 0x8     /* a device length exceeds the host bound max_seqlen_q / max_seqlen_k */
#define SPA_ST_BAD_IDX 0x10   /* a selected index is < -1 or beyond its range; it was skipped */
#define SPA_ST_TIMEOUT 0x20   /* a bounded on-chip wait expired; the affected outputs are unspecified */

/*
 * spa_select_topk -- the selection producer ahead of step 3: for every row r
 * (a request, or a query token) and kv head h, the top_k keys of the per-key
 * scores, written as the -1 padded selected-index row that spa_attention's
 * selected mode reads (selected_idx with sel_target = 0).
 * Source: onnxruntime PR #33472, Key Changes (PackedSparseAttentionIndexer:
 * QSA scoring and hierarchical / compact TopK selection) and its experiments
 * note (the compact TopK keeps stable keys, causal tails, capacity stride /
 * padding and overflow handling).  The pages do not define the score, so it
 * is an input.
 *
 *   scores [R, H, n_keys]  fp32 score of key j of row r under kv head h.
 *   bound [R]              last eligible key of row r (the causal tail):
 *                          seqlen_k of spa_prepare_metadata for per-request
 *                          rows, token_pos for per-token rows; keys beyond it,
 *                          or beyond n_keys - 1, are never selected; a
 *                          negative bound gives an empty row.
 *   top_k, sel_width       [host] keys kept per row, 0 <= top_k <= sel_width;
 *                          sel_width is the row capacity of the output.
 *   selected_idx [R, H, sel_width] (output) the kept keys in increasing order,
 *                          then -1 up to sel_width.
 * A key is eligible when its score is neither NaN nor -inf (-inf masks a
 * key); -0 and +0 are equal.  The kept keys are the min(top_k, eligible)
 * largest scores; among equal scores the lower key index is kept first, so
 * the result is unique and bit-exact.  Errors: SPA_ERR_INVALID_ARG for
 * negative sizes, H <= 0, sel_width <= 0, top_k > sel_width or a NULL
 * required pointer.  R = 0 is valid.  One kernel launch.
 */
int spa_select_topk(const float* scores, int32_t R, int32_t H, int32_t n_keys, const int32_t* bound,
                    int32_t top_k, int32_t sel_width, int32_t* selected_idx, spa_stream_t stream);

/*
 * spa_prepare_metadata -- step 1, exact per-request and per-token metadata on
 * the device, replacing a device-to-host readback per layer.
 * Source: "[WebGPU] Add PagedAttention metadata and GPT-OSS support",
 * Description / Changes (host replay-wide bounds; exact seqlen_k and
 * seqlens_q derived on device) and review item T1 (seqlen_k = -1 for an
 * empty request); "[WebGPU] Add SparsePagedAttention", File summaries
 * (token_meta: sanitised per-token metadata).
 *
 * Inputs:
 *   cu_seqlens_q [B+1]  cumulative query lengths; request b owns packed tokens
 *                       [cu[b], cu[b+1]).  Malformed values are clamped to a
 *                       non-decreasing sequence in [0, T] starting at 0 and
 *                       flagged SPA_ST_BAD_CU.
 *   past_seqlens [B]    tokens already resident in the cache (negative -> 0, flagged).
 *   block_table [B, MB] physical block id of each logical block (-1 = unmapped).
 *   B, T                [host] number of requests / packed query tokens.
 *   max_seqlen_q, max_seqlen_k [host] replay-wide bounds; a request with
 *                       q_len > max_seqlen_q or past + q_len > max_seqlen_k
 *                       sets SPA_ST_BOUNDS.
 *   MB, block_size, num_blocks [host] block-table width, tokens per block,
 *                       number of physical blocks in the cache.
 * Outputs:
 *   seqlens_q [B]       q_len[b] = cu'[b+1] - cu'[b]
 *   seqlen_k  [B]       past[b] + q_len[b] - 1 (so -1 for a request with no tokens)
 *   token_batch [T]     request owning token t (-1 if none)
 *   token_pos   [T]     absolute position past[b] + t - cu'[b] (-1 if no owner)
 *   slot_mapping [T]    block_table[b, pos / bs] * bs + pos % bs, or -1 when the
 *                       position is beyond the table (SPA_ST_CAPACITY) or its
 *                       block id is invalid (SPA_ST_BAD_BLOCK)
 *   status              OR-ed status bits.
 * B = 0 or T = 0 is valid (outputs of length 0 are not touched).
 */
int spa_prepare_metadata(const int32_t* cu_seqlens_q, const int32_t* past_seqlens,
                         const int32_t* block_table, int32_t B, int32_t T, int32_t max_seqlen_q,
                         int32_t max_seqlen_k, int32_t MB, int32_t block_size, int32_t num_blocks,
                         int32_t* seqlens_q, int32_t* seqlen_k, int32_t* token_batch,
                         int32_t* token_pos, int32_t* slot_mapping, int32_t* status,
                         spa_stream_t stream);

/*
 * spa_append_kv -- step 2, scatter the current tokens' K/V rows into the paged
 * cache through slot_mapping.
 * Source: "[WebGPU] Add SparsePagedAttention", File summaries (scatter current
 * K/V into the cache using slot_mapping); PR #33472, Key Changes (INT8 KV
 * cache append with key_scale / value_scale).
 *
 *   k_new, v_new [T, H_kv, D]  activation dtype `act` (SPA_F32/F16/BF16).
 *   k_cache, v_cache [num_blocks, block_size, H_kv, D]  dtype `cache`, which is
 *                     either `act` (exact copy) or SPA_I8.
 *   k_scale, v_scale [H_kv, D] fp32, required iff cache == SPA_I8:
 *                     q8 = clamp(rint(float(x) / scale[h, d]), -128, 127),
 *                     IEEE fp32 division, round half to even.
 *   slot_mapping [T]  destination slot of token t; -1 skips the token; a slot
 *                     outside [0, num_blocks * block_size) is skipped and sets
 *                     SPA_ST_BAD_BLOCK.
 * T = 0 is valid.  D must be a multiple of 8 (and of 16 for SPA_I8).
 */
int spa_append_kv(const void* k_new, const void* v_new, int32_t act, void* k_cache, void* v_cache,
                  int32_t cache, const float* k_scale, const float* v_scale,
                  const int32_t* slot_mapping, int32_t T, int32_t H_kv, int32_t D,
                  int32_t block_size, int32_t num_blocks, int32_t* status, spa_stream_t stream);

/*
 * spa_prepare_append_kv -- steps 1 and 2 in one launch: the metadata of
 * spa_prepare_metadata and the scatter of spa_append_kv, with outputs (the
 * five metadata arrays, both caches and the status bits) identical bit for
 * bit to calling those two entry points in sequence with the same arguments.
 * Source: "[WebGPU] Add SparsePagedAttention", File summaries (token_meta and
 * scatter_kv stages) -- fused here so that one warp derives a token's slot and
 * writes its K/V rows.  Argument meaning, layouts and error behaviour are those
 * of the two entry points; H_kv and D describe k_new / v_new and the caches.
 */
int spa_prepare_append_kv(const int32_t* cu_seqlens_q, const int32_t* past_seqlens,
                          const int32_t* block_table, int32_t B, int32_t T, int32_t max_seqlen_q,
                          int32_t max_seqlen_k, int32_t MB, int32_t block_size, int32_t num_blocks,
                          int32_t* seqlens_q, int32_t* seqlen_k, int32_t* token_batch,
                          int32_t* token_pos, int32_t* slot_mapping, const void* k_new,
                          const void* v_new, int32_t act, void* k_cache, void* v_cache, int32_t cache,
                          const float* k_scale, const float* v_scale, int32_t H_kv, int32_t D,
                          int32_t* status, spa_stream_t stream);

/*
 * Arguments of spa_attention (steps 3-5).  `struct_size` must be set to
 * sizeof(spa_attention_args_t) so that the struct can grow compatibly.
 * Sources: "[WebGPU] Add DynamicSparseAttention", Description / Attention
 * (selected main-cache and local-plus-auxiliary modes, joint FP32 stable
 * softmax with optional sink, guarded int32 indices) and QKV and cache (GQA
 * head mapping); "[WebGPU] Add PagedAttention metadata and GPT-OSS support",
 * Description (local window, learned head sink) and review item Q3 (window
 * start); "[WebGPU] Add SparsePagedAttention", File summaries (main and
 * auxiliary partial FP32 softmax state, finalize merge with the sink).
 */
typedef struct spa_attention_args {
  size_t struct_size;
  /* queries and output, [T, H_q, D] in `act` (SPA_F32 / SPA_F16 / SPA_BF16) */
  const void* q;
  void* out;
  int32_t act;
  int32_t T, B, H_q, H_kv, D; /* [host]; H_q must be a positive multiple of H_kv; D in {64, 128} */
  /* paged cache [num_blocks, block_size, H_kv, D] in `cache` (== act, or SPA_I8 with scales) */
  const void* k_cache;
  const void* v_cache;
  int32_t cache;
  const float* k_scale; /* [H_kv, D], SPA_I8 only */
  const float* v_scale; /* [H_kv, D], SPA_I8 only */
  const int32_t* block_table; /* [B, MB] */
  int32_t MB, block_size, num_blocks; /* [host] */
  /* metadata from spa_prepare_metadata */
  const int32_t* cu_seqlens_q; /* [B+1] */
  const int32_t* seqlens_q;    /* [B]   */
  const int32_t* seqlen_k;     /* [B]   total - 1 */
  const int32_t* token_batch;  /* [T]   */
  const int32_t* token_pos;    /* [T]   */
  int32_t max_seqlen_q, max_seqlen_k; /* [host] replay-wide bounds used for launch sizing */
  int32_t is_causal; /* must be 1 */
  int32_t window;    /* > 0: key j visible to position p iff p - window < j <= p; <= 0: off */
  /* selected indices, -1 padded: [T, H_kv, sel_width] (sel_per_request = 0) or
     [B, H_kv, sel_width] (sel_per_request = 1); NULL = no selection */
  const int32_t* selected_idx;
  int32_t sel_width;
  int32_t sel_per_request;
  int32_t sel_target; /* 0: indices address the main cache (no window allowed);
                         1: indices address the auxiliary store; the main cache
                            then contributes its causal window (or all causal
                            keys when window <= 0) */
  /* auxiliary store [B, aux_cap, H_kv, D], same dtype and scales as the main cache */
  const void* aux_k;
  const void* aux_v;
  int32_t aux_cap;
  const int32_t* aux_seqlens; /* [B] valid entries per request */
  const float* sinks; /* [H_q] learned sink logits, not multiplied by scale; NULL = no sink */
  float scale;        /* 0 selects 1/sqrt(D) */
  float* lse;         /* [T, H_q] optional: log of the softmax denominator incl. the sink */
  int32_t num_splits; /* 0 = automatic; otherwise the number of key splits per unit */
  int32_t* status;    /* OR-ed status bits */
  /* One shard of a sequence split across devices ("[WebGPU] Add
     SparsePagedAttention", File summaries: partial FP32 softmax states merged
     by a finalize stage that applies the sink).
     kv_range [B, 2]: main-cache positions lo <= j < hi of request b that this
       call attends (NULL = all).  Keys outside the range are dropped before
       any block-table lookup, so a shard's block table may leave the other
       shards' blocks unmapped (-1) without setting a status bit.  Auxiliary
       entries are not affected.
     partial = 1: the call leaves the shard's partial state for
       spa_merge_partials instead of the output: `out` is FP32 [T, H_q, D],
       the softmax over the shard's attended keys WITHOUT the sink (0 when it
       has none); `lse` is required and holds its log-sum-exp (-inf when
       none); `sinks` is ignored (the merge applies it once). */
  const int32_t* kv_range;
  int32_t partial;
  /* Test hook of the failure detection, 0 in normal use: 1 makes the
     tcgen05 prefill kernel drop one barrier arrival per CTA (on a barrier
     that guards no copy and no MMA) and poll for it only briefly, so that the
     bounded wait expires: every CTA drains its copies and MMAs, frees its
     tensor memory and returns, and SPA_ST_TIMEOUT is set.  Other kernels
     ignore it. */
  int32_t test_expire_wait;
} spa_attention_args_t;

/* Bytes of workspace spa_attention needs for these arguments (0 if none:
   decode with one split per unit, prefill without a local window of at most
   256 keys).  Returns 0 as well for invalid arguments; spa_attention then
   reports the error. */
size_t spa_attention_workspace_size(const spa_attention_args_t* a);

/*
 * spa_attention -- steps 3-5.  For token t (request b, position p) and q
 * head h (kv head h / (H_q / H_kv)):
 *   s_j = scale * <q[t,h], k_j> over the attended set S(t, h_kv),
 *   m = max(max_j s_j, sink_h), l = sum_j exp(s_j - m) + exp(sink_h - m),
 *   out[t,h] = sum_j exp(s_j - m) v_j / l  (0 when S is empty and there is no sink),
 *   lse[t,h] = m + log(l).
 * The attended set is, for the main cache, the causal window (or all causal
 * keys) or the valid selected indices <= p; plus, with sel_target = 1, the
 * valid auxiliary entries of the request.  Keys are processed in splits whose
 * FP32 partial states are merged by log-sum-exp; the result does not depend
 * on num_splits beyond rounding.
 * workspace: device buffer of at least spa_attention_workspace_size() bytes,
 * 256-byte aligned; it may be NULL when the size is 0.  It holds the splits'
 * FP32 partial states (no initialisation needed), for plans that merge by
 * ticket per-unit split tickets, and for prefill with a local window of at
 * most 256 keys (one CTA per SM looping over work items) the work counter
 * the CTAs claim items from: tickets and counter must be zero before the
 * first use and every call leaves them at zero again (also when a bounded
 * wait expired), so zero-fill a new workspace.  Calls that share a workspace
 * must be ordered on one stream.  The whole operation
 * is one kernel launch: on the tensor-core decode kernels the (at most 8)
 * splits of a unit form one thread-block cluster, write their partial states
 * to the workspace, pass a cluster barrier and merge a share of the rows
 * each; otherwise the last CTA to finish a unit's splits merges them.
 */
int spa_attention(const spa_attention_args_t* a, void* workspace, size_t workspace_bytes,
                  spa_stream_t stream);

/*
 * spa_merge_partials -- the merge of a sequence split across R devices: the
 * partial states that R spa_attention calls with partial = 1 left (each over
 * its kv_range of the same requests), gathered into one buffer, combined by
 * log-sum-exp with the sink counted once.
 * Source: "[WebGPU] Add SparsePagedAttention", File summaries (main and
 * auxiliary partial FP32 softmax states; finalize merge with the sink).
 *   part_out [R, T, H_q, D] fp32 (16-byte aligned), part_lse [R, T, H_q] fp32:
 *                   shard r's out and lse.
 *   sinks [H_q]     learned sink logits, or NULL (no sink).
 *   act             dtype of `out` (SPA_F32 / SPA_F16 / SPA_BF16).
 *   out [T, H_q, D], lse [T, H_q] (optional): for each row
 *     M = max(sink, max_r lse_r), L = e^(sink - M) + sum_r e^(lse_r - M),
 *     out = sum_r e^(lse_r - M) out_r / L, lse = M + ln L;
 *     out = 0, lse = -inf when every shard is empty and there is no sink.
 * Errors: SPA_ERR_INVALID_ARG for R <= 0, D not 64 / 128, a bad dtype or a
 * NULL / misaligned required pointer.  T = 0 is valid.  One kernel launch.
 */
int spa_merge_partials(const float* part_out, const float* part_lse, int32_t R, int32_t T, int32_t H_q,
                       int32_t D, const float* sinks, int32_t act, void* out, float* lse, spa_stream_t stream);

/*
 * spa_prepare_append_attention -- steps 1 to 5 as one call: the outputs of
 * spa_prepare_append_kv followed by spa_attention with the same arguments,
 * bit for bit (the metadata arrays, both caches, out, lse and status).
 * Source: "[WebGPU] Add SparsePagedAttention", File summaries (prepare the
 * token metadata, scatter the current K/V into the cache, then attend) --
 * here one kernel launch when the plan picks the warp-MMA decode kernel on a
 * 16-bit cache of the activation dtype, or the tcgen05 decode kernel on a
 * 16-bit or INT8 cache (each CTA derives its unit's metadata from
 * cu_seqlens_q and past_seqlens in shared memory, writes its share of the
 * metadata and of the appended rows, and reads this step's own new rows from
 * k_new / v_new -- INT8 rows quantised exactly as the append quantises
 * them); otherwise the two launches of the staged sequence.
 *   a               the attention arguments; a->seqlens_q, a->seqlen_k,
 *                   a->token_batch and a->token_pos are OUTPUTS here (the
 *                   step-1 arrays, written with spa_prepare_metadata's
 *                   meaning); a->cu_seqlens_q, block_table, MB, block_size,
 *                   num_blocks, max_seqlen_q, max_seqlen_k, k_cache, v_cache,
 *                   cache, k_scale, v_scale, H_kv, D and status play their
 *                   spa_prepare_append_kv roles as well.
 *   past_seqlens [B], k_new, v_new [T, H_kv, D] (dtype a->act, 16-byte
 *                   aligned), slot_mapping [T] (output): as in
 *                   spa_prepare_append_kv.
 *   workspace       as in spa_attention (spa_attention_workspace_size(a)).
 * Errors: those of both entry points; nothing is launched on an error.
 * Memory the caches alias between this step's new slots and older positions
 * (a malformed block table) is read as the staged sequence would only when
 * the two launches are used.
 */
int spa_prepare_append_attention(const spa_attention_args_t* a, const int32_t* past_seqlens,
                                 const void* k_new, const void* v_new, int32_t* slot_mapping, void* workspace,
                                 size_t workspace_bytes, spa_stream_t stream);

/* Kernel launches spa_prepare_append_attention makes for these arguments (1 or
   2), or a negative error code.  Host only. */
int spa_prepare_append_attention_launches(const spa_attention_args_t* a);

/*
 * spa_prepare_qkv_append -- steps 1 and 2 with the QKV prologue between them,
 * in one launch: the metadata of spa_prepare_metadata, then per (token, head)
 * row of q and k an optional RMSNorm and an optional rotary embedding, then q
 * written for the attention and k / v appended as spa_append_kv does.
 * Source: "[WebGPU] Add DynamicSparseAttention", Description -- QKV and cache
 * (packed and unpacked QKV), Position processing (QK RMSNorm; partial and
 * interleaved RoPE; rotary offsets and explicit position IDs); "[WebGPU] Add
 * SparsePagedAttention", Description (packed-QKV split and RoPE ahead of the
 * block-table scatter).  Per row x of a q or k head:
 *   x <- x / sqrt(mean(x^2) + norm_eps) * w             (w = q_ / k_norm_weight)
 *   x <- RoPE on channels [0, rotary_dim): pairs (i, i + rotary_dim/2), or
 *        (2i, 2i+1) when rotary_interleaved: (a, b) -> (a c - b s, b c + a s)
 *        with c, s = cos_cache, sin_cache[position, i]
 *   position = position_ids[t] if given, else token_pos[t] + rotary_offset;
 *   outside [0, max_pos) the row is not rotated and SPA_ST_BOUNDS is set.
 * Results are rounded to `act` (nearest even); k and v are then appended
 * (INT8: q8 = clamp(rint(x / scale), -128, 127) of the rounded x).
 */
typedef struct {
  size_t struct_size;            /* sizeof(spa_qkv_args_t) */
  /* step 1, as spa_prepare_metadata (the five arrays are outputs) */
  const int32_t* cu_seqlens_q;   /* [B + 1] */
  const int32_t* past_seqlens;   /* [B] */
  const int32_t* block_table;    /* [B, MB] */
  int32_t B, T, max_seqlen_q, max_seqlen_k, MB, block_size, num_blocks;
  int32_t* seqlens_q;
  int32_t* seqlen_k;
  int32_t* token_batch;
  int32_t* token_pos;
  int32_t* slot_mapping;
  /* the rows */
  int32_t act;                   /* SPA_F32 / SPA_F16 / SPA_BF16 */
  int32_t H_q, H_kv, D;          /* D = 64 or 128 */
  const void* qkv;               /* packed [T, H_q + 2 H_kv, D]: q, then k, then v heads; or NULL */
  const void* q;                 /* [T, H_q, D]  \                                  */
  const void* k;                 /* [T, H_kv, D]  } when qkv is NULL                 */
  const void* v;                 /* [T, H_kv, D] /                                   */
  /* prologue */
  const float* q_norm_weight;    /* [D] or NULL (no q norm) */
  const float* k_norm_weight;    /* [D] or NULL (no k norm) */
  float norm_eps;
  const float* cos_cache;        /* [max_pos, rotary_dim / 2] or NULL (no rotation) */
  const float* sin_cache;        /* [max_pos, rotary_dim / 2] */
  int32_t max_pos, rotary_dim, rotary_interleaved;   /* rotary_dim even, <= D */
  const int32_t* position_ids;   /* [T] or NULL */
  int32_t rotary_offset;
  /* outputs */
  void* q_out;                   /* [T, H_q, D] act */
  void* k_cache;                 /* [num_blocks, block_size, H_kv, D] */
  void* v_cache;
  int32_t cache;                 /* act or SPA_I8 */
  const float* k_scale;          /* [H_kv, D] iff SPA_I8 */
  const float* v_scale;
  int32_t* status;
} spa_qkv_args_t;

/* Errors: SPA_ERR_INVALID_ARG for a NULL required pointer, a bad dtype pair,
   D not 64 / 128, an odd or oversized rotary_dim, a row pointer not 16-byte
   aligned, or inconsistent sizes; SPA_ERR_UNSUPPORTED for B > 16384.  B = 0 or
   T = 0 is valid. */
int spa_prepare_qkv_append(const spa_qkv_args_t* a, spa_stream_t stream);

/*
 * spa_attention_noalloc -- spa_attention for callers that cannot allocate
 * device memory.  The pages have no counterpart: this entry point exists for
 * callers of this library that cannot provide a workspace -- code running
 * inside a CUDA graph capture (where cudaMalloc is not allowed), plugins whose
 * host runtime owns all device memory, tools that must keep the process's
 * device footprint fixed.  It computes exactly what spa_attention computes
 * (same kernels, same arguments) but takes its scratch from an array built
 * into the library: SPA_NOALLOC_SCRATCH_BYTES on every GPU that loads the
 * library, held until the process exits.  It calls no cudaMalloc / cudaFree
 * and no allocating routine.
 *   - A call whose plan needs more scratch than SPA_NOALLOC_SCRATCH_BYTES
 *     (spa_attention_workspace_size() of the same arguments) returns
 *     SPA_ERR_SCRATCH_LIMIT and enqueues nothing.  Plans whose
 *     spa_attention_workspace_size() is 0 need no scratch at all.
 *   - The first call on each device resolves the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     Every later call made outside a capture resolves it again; a call made
 *     during a capture reuses the address of the last uncaptured call on the
 *     device, so after a context reset (cudaDeviceReset) make one call
 *     outside a capture before capturing again.  If the address cannot be
 *     resolved the call returns SPA_ERR_CUDA.
 *   - Every call on a device shares the array and sees what the previous call
 *     left in it; the values that must start at zero are cleared on `stream`
 *     before the kernel runs (one memset).  Calls that may overlap on the GPU
 *     (different streams, different host threads) race on the array and must
 *     be ordered by the caller.
 */
#define SPA_NOALLOC_SCRATCH_BYTES (8u << 20)
int spa_attention_noalloc(const spa_attention_args_t* a, spa_stream_t stream);

/*
 * spa_attention_plan -- host-only introspection of what spa_attention would
 * launch for these arguments: the number of key splits per unit, the number
 * of kernel launches, and the kernel family (0 = CUDA-core decode,
 * 1 = warp-MMA decode, 2 = tcgen05 prefill, 3 = tcgen05 multi-row decode).  Any output pointer may be
 * NULL.  Returns the same code spa_attention would return for the arguments
 * before launching anything.
 */
int spa_attention_plan(const spa_attention_args_t* a, int32_t* num_splits, int32_t* num_launches,
                       int32_t* kernel_kind);

/* Static message for a return code; for SPA_ERR_CUDA the message of the
   last failed launch in this thread. */
const char* spa_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* SPA_H_ */
