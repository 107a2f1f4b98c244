// C ABI of libspa: argument validation, launch planning and dispatch.
//
// Host code only.  Nothing here allocates device memory, synchronises a
// stream or reads device memory; every decision is taken from host-side
// sizes and the replay-wide bounds max_seqlen_q / max_seqlen_k ("[WebGPU] Add
// PagedAttention metadata and GPT-OSS support", Description: host bounds size
// scratch and choose dispatch, exact lengths stay on the device).
#include <cmath>
#include <cstdio>
#include <cstring>

#include "spa_attn.cuh"
#include "spa_plan.h"

namespace spa {
int launch_prepare_metadata(const int32_t*, const int32_t*, const int32_t*, int, int, int, int, int,
                            int, int, int32_t*, int32_t*, int32_t*, int32_t*, int32_t*, int32_t*,
                            cudaStream_t);
int launch_append_kv(const void*, const void*, int, void*, void*, int, const float*, const float*,
                     const int32_t*, int, int, int, int, int, int32_t*, cudaStream_t);
int launch_prepare_append(const int32_t*, const int32_t*, const int32_t*, int, int, int, int, int, int, int,
                          int32_t*, int32_t*, int32_t*, int32_t*, int32_t*, const void*, const void*, int,
                          void*, void*, int, const float*, const float*, int, int, int32_t*, cudaStream_t);
int launch_attention_scalar_impl(const AttnParams&, int, int, int, cudaStream_t);
size_t scalar_smem_bytes(int D, int max_rows, int nq);
int launch_attention_mma(const AttnParams& p, int act, int cache, int max_rows, cudaStream_t stream);
int mma_supported(int act, int cache, int D, int max_rows);
int mma_key_tile(int D, int max_rows);
int tc_supported(int act, int cache, int D, int max_rows);
int tc_key_tile();
int launch_attention_tc(const AttnParams& p, int act, int cache, cudaStream_t stream);
int launch_step_mma(const AttnParams& p, int act, int max_rows, cudaStream_t stream);
int launch_step_tc(const AttnParams& p, int act, int cache, cudaStream_t stream);
int tc_step_fits(int D, int cache, int B);
int launch_prepare_qkv_append(const QkvParams& P, int act, int cache, cudaStream_t stream);
int mma_step_fits(int D, int max_rows, int B);
int launch_prefill(const AttnParams& p, int act, cudaStream_t stream);
int prefill_supported(const spa_attention_args_t* a);
size_t prefill_ticket_bytes(const spa_attention_args_t* a);

static thread_local char g_cuda_msg[256] = "no CUDA error recorded";

static int check_launch() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(g_cuda_msg, sizeof(g_cuda_msg), "CUDA launch failed: %s (%s)", cudaGetErrorName(e),
             cudaGetErrorString(e));
    return SPA_ERR_CUDA;
  }
  return SPA_OK;
}

static bool act_ok(int d) { return d == SPA_F32 || d == SPA_F16 || d == SPA_BF16; }
static int elt_bytes(int d) { return d == SPA_F32 ? 4 : (d == SPA_I8 ? 1 : 2); }

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int validate_attention(const spa_attention_args_t* a) {
  if (a == nullptr || a->struct_size < sizeof(spa_attention_args_t)) return SPA_ERR_INVALID_ARG;
  if (a->is_causal != 1) return SPA_ERR_UNSUPPORTED;
  if (!act_ok(a->act)) return SPA_ERR_INVALID_ARG;
  if (!(a->cache == a->act || a->cache == SPA_I8)) return SPA_ERR_INVALID_ARG;
  if (a->T < 0 || a->B < 0 || a->H_q <= 0 || a->H_kv <= 0 || a->H_q % a->H_kv != 0)
    return SPA_ERR_INVALID_ARG;
  if (a->H_q / a->H_kv > 128) return SPA_ERR_UNSUPPORTED;
  if (a->D != 64 && a->D != 128) return SPA_ERR_UNSUPPORTED;
  if (a->block_size <= 0 || a->MB <= 0 || a->num_blocks <= 0) return SPA_ERR_INVALID_ARG;
  if ((long long)a->num_blocks * a->block_size * a->H_kv * a->D > (1LL << 40)) return SPA_ERR_INVALID_ARG;
  if ((long long)a->num_blocks * a->block_size >= (1LL << 31)) return SPA_ERR_INVALID_ARG;
  if (a->max_seqlen_q < 0 || a->max_seqlen_k < 0) return SPA_ERR_INVALID_ARG;
  if (a->num_splits < 0) return SPA_ERR_INVALID_ARG;
  if (a->T == 0 || a->B == 0) return SPA_OK;  // nothing to compute; pointers may be null
  if (!a->q || !a->out || !a->k_cache || !a->v_cache || !a->block_table || !a->cu_seqlens_q ||
      !a->seqlens_q || !a->seqlen_k || !a->token_batch || !a->token_pos)
    return SPA_ERR_INVALID_ARG;
  if (a->cache == SPA_I8 && (!a->k_scale || !a->v_scale)) return SPA_ERR_INVALID_ARG;
  if (a->selected_idx) {
    if (a->sel_width <= 0 || a->sel_width > (1 << 24)) return SPA_ERR_INVALID_ARG;
    if (a->sel_target != 0 && a->sel_target != 1) return SPA_ERR_INVALID_ARG;
    if (a->sel_target == 0 && a->window > 0) return SPA_ERR_UNSUPPORTED;
    if (a->sel_target == 1 && (!a->aux_k || !a->aux_v || !a->aux_seqlens || a->aux_cap <= 0))
      return SPA_ERR_INVALID_ARG;
  }
  if (!std::isfinite(a->scale) || a->scale < 0.f) return SPA_ERR_INVALID_ARG;
  if (a->partial != 0 && a->partial != 1) return SPA_ERR_INVALID_ARG;
  if (a->partial && !a->lse) return SPA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a->q) | reinterpret_cast<uintptr_t>(a->out) |
       reinterpret_cast<uintptr_t>(a->k_cache) | reinterpret_cast<uintptr_t>(a->v_cache)) & 15)
    return SPA_ERR_INVALID_ARG;
  if (a->aux_k && ((reinterpret_cast<uintptr_t>(a->aux_k) | reinterpret_cast<uintptr_t>(a->aux_v)) & 15))
    return SPA_ERR_INVALID_ARG;
  return SPA_OK;
}

// Launch plan: which kernel, how units are grouped, how candidates are split.
int make_plan(const spa_attention_args_t* a, Plan* pl) {
  memset(pl, 0, sizeof(*pl));
  const int G = a->H_q / a->H_kv;
  const bool sel_main = a->selected_idx && a->sel_target == 0;
  const bool sel_aux = a->selected_idx && a->sel_target == 1;
  const int maxq = a->max_seqlen_q > 0 ? a->max_seqlen_q : 1;
  if (prefill_supported(a)) {
    pl->kind = kPlanPrefill;
    pl->num_splits = 1;
    pl->ws_count_bytes = prefill_ticket_bytes(a);   // the persistent schedule's work counter
    return SPA_OK;
  }
  // group all tokens of a request when their rows fit one CTA and the
  // candidate list is per request
  const bool per_request_list = !a->selected_idx || a->sel_per_request;
  pl->group_by_request = per_request_list && (long long)maxq * G <= 128;
  pl->max_q = pl->group_by_request ? maxq : 1;
  pl->max_rows = pl->max_q * G;
  if (tc_supported(a->act, a->cache, a->D, pl->max_rows)) pl->kind = kPlanTc;
  else if (mma_supported(a->act, a->cache, a->D, pl->max_rows)) pl->kind = kPlanMma;
  else pl->kind = kPlanScalar;
  const int KT = pl->kind == kPlanTc ? tc_key_tile()
                                     : (pl->kind == kPlanMma ? mma_key_tile(a->D, pl->max_rows) : scalar_key_tile());
  long long n_main;
  if (sel_main) n_main = a->sel_width;
  else if (a->window > 0) n_main = std::min<long long>((long long)a->window + pl->max_q - 1, a->max_seqlen_k);
  else n_main = a->max_seqlen_k;
  long long n_cand = n_main + (sel_aux ? a->sel_width : 0);
  if (n_cand < 1) n_cand = 1;
  const long long tiles = (n_cand + KT - 1) / KT;
  const long long units = pl->group_by_request ? (long long)a->B * a->H_kv : (long long)a->T * a->H_kv;
  if (units > 0x7fffffffLL) return SPA_ERR_INVALID_ARG;
  long long splits;
  if (a->num_splits > 0) {
    splits = a->num_splits;
  } else {
    // units that already fill the GPU run unsplit (no partials, no merge);
    // otherwise split as far as one wave allows (two CTAs per SM, one for
    // the tcgen05 kernel, which holds most of the shared memory)
    const long long slots = pl->kind == kPlanTc ? 148 : 2LL * 148;
    splits = units >= 148 ? 1 : slots / units;
    if (splits > tiles) splits = tiles;
    if (splits > 64) splits = 64;
    if (splits < 1) splits = 1;
  }
  if (splits > 65535) return SPA_ERR_INVALID_ARG;
  long long per_tiles = (tiles + splits - 1) / splits;
  if (a->num_splits == 0) splits = (tiles + per_tiles - 1) / per_tiles;
  pl->num_splits = (int)splits;
  pl->split_len = (int)std::min<long long>(per_tiles * KT, 0x7fffffffLL);
  pl->units = (int)units;
  // split partial states go through the workspace; the splits of a unit
  // merge after a cluster barrier when they fit one cluster (tensor-core
  // decode kernels), otherwise the CTA that finishes last merges (tickets)
  pl->cluster_merge = (pl->kind == kPlanTc || pl->kind == kPlanMma) && pl->num_splits > 1 &&
                      pl->num_splits <= 8;
  if (pl->num_splits > 1) {
    const size_t rows = (size_t)a->T * a->H_q;
    pl->ws_acc_bytes = align256(rows * a->D * sizeof(float) * pl->num_splits);
    pl->ws_ml_bytes = align256(rows * 2 * sizeof(float) * pl->num_splits);
    if (!pl->cluster_merge) pl->ws_count_bytes = align256((size_t)units * sizeof(int));
  }
  if (pl->kind == kPlanScalar &&
      scalar_smem_bytes(a->D, pl->max_rows, pl->max_q) > 200 * 1024)
    return SPA_ERR_UNSUPPORTED;
  return SPA_OK;
}

void fill_params(const spa_attention_args_t* a, const Plan& pl, void* ws, AttnParams* p) {
  memset(p, 0, sizeof(*p));
  p->q = a->q;
  p->out = a->out;
  p->lse = a->lse;
  p->k_cache = a->k_cache;
  p->v_cache = a->v_cache;
  p->k_scale = a->k_scale;
  p->v_scale = a->v_scale;
  p->block_table = a->block_table;
  p->MB = a->MB;
  p->bs = a->block_size;
  p->NB = a->num_blocks;
  p->cu = a->cu_seqlens_q;
  p->seqlens_q = a->seqlens_q;
  p->seqlen_k = a->seqlen_k;
  p->token_batch = a->token_batch;
  p->token_pos = a->token_pos;
  p->T = a->T;
  p->B = a->B;
  p->H_q = a->H_q;
  p->H_kv = a->H_kv;
  p->D = a->D;
  p->G = a->H_q / a->H_kv;
  p->window = a->window;
  p->sel = a->selected_idx;
  p->sel_width = a->selected_idx ? a->sel_width : 0;
  p->sel_per_request = a->sel_per_request;
  p->sel_target = a->sel_target;
  p->aux_k = a->aux_k;
  p->aux_v = a->aux_v;
  p->aux_cap = a->aux_cap;
  p->aux_len = a->aux_seqlens;
  p->sinks = a->partial ? nullptr : a->sinks;   // a shard's partial leaves the sink to the merge
  p->kv_range = a->kv_range;
  p->out_f32 = a->partial;
  p->test_expire_wait = a->test_expire_wait != 0;
  const float scale = a->scale == 0.f ? (float)(1.0 / std::sqrt((double)a->D)) : a->scale;
  p->scale_log2 = scale * kLog2e;
  p->group_by_request = pl.group_by_request;
  p->max_q = pl.kind == kPlanPrefill ? a->max_seqlen_q : pl.max_q;
  p->max_k = a->max_seqlen_k;
  p->num_splits = pl.num_splits;
  p->split_len = pl.split_len;
  p->status = a->status;
  p->cluster_merge = pl.cluster_merge;
  if (pl.kind == kPlanPrefill && pl.ws_count_bytes > 0) p->ws_count = static_cast<int*>(ws);
  if (pl.num_splits > 1) {
    p->ws_acc = static_cast<float*>(ws);
    p->ws_ml = reinterpret_cast<float*>(static_cast<char*>(ws) + pl.ws_acc_bytes);
    if (!pl.cluster_merge)
      p->ws_count = reinterpret_cast<int*>(static_cast<char*>(ws) + pl.ws_acc_bytes + pl.ws_ml_bytes);
  }
}

int run_attention(const spa_attention_args_t* a, const Plan& pl, void* ws, cudaStream_t stream) {
  AttnParams p;
  fill_params(a, pl, ws, &p);
  int rc;
  if (pl.kind == kPlanPrefill) {
    rc = launch_prefill(p, a->act, stream);
    if (rc != SPA_OK) return rc;
    return check_launch();
  }
  if (pl.kind == kPlanTc) rc = launch_attention_tc(p, a->act, a->cache, stream);
  else if (pl.kind == kPlanMma) rc = launch_attention_mma(p, a->act, a->cache, pl.max_rows, stream);
  else rc = launch_attention_scalar_impl(p, a->act, a->cache, pl.max_rows, stream);
  if (rc != SPA_OK) return rc;
  return check_launch();
}

int launches_of(const Plan&) { return 1; }

// The fused step runs as one launch when the plan picks the warp-MMA kernel
// on a cache of the activation dtype and the metadata fits shared memory.
static bool step_fusable(const spa_attention_args_t* a, const Plan& pl) {
  if (a->B > 4096) return false;
  if (pl.kind == kPlanTc) return tc_step_fits(a->D, a->cache, a->B) != 0;
  return pl.kind == kPlanMma && a->cache == a->act && mma_step_fits(a->D, pl.max_rows, a->B);
}

const char* cuda_message() { return g_cuda_msg; }
int check_launch_public() { return check_launch(); }

}  // namespace spa

using namespace spa;

extern "C" {

int spa_prepare_metadata(const int32_t* cu_seqlens_q, const int32_t* past_seqlens,
                         const int32_t* block_table, int32_t B, int32_t T, int32_t max_seqlen_q,
                         int32_t max_seqlen_k, int32_t MB, int32_t block_size, int32_t num_blocks,
                         int32_t* seqlens_q, int32_t* seqlen_k, int32_t* token_batch,
                         int32_t* token_pos, int32_t* slot_mapping, int32_t* status,
                         spa_stream_t stream) {
  if (B < 0 || T < 0 || MB < 0 || block_size <= 0 || num_blocks < 0) return SPA_ERR_INVALID_ARG;
  if (B > 16384) return SPA_ERR_UNSUPPORTED;
  if ((long long)num_blocks * block_size >= (1LL << 31)) return SPA_ERR_INVALID_ARG;
  if (!cu_seqlens_q) return SPA_ERR_INVALID_ARG;
  if (B > 0 && (!past_seqlens || !seqlens_q || !seqlen_k || (MB > 0 && !block_table)))
    return SPA_ERR_INVALID_ARG;
  if (T > 0 && (!token_batch || !token_pos || !slot_mapping)) return SPA_ERR_INVALID_ARG;
  launch_prepare_metadata(cu_seqlens_q, past_seqlens, block_table, B, T, max_seqlen_q, max_seqlen_k,
                          MB, block_size, num_blocks, seqlens_q, seqlen_k, token_batch, token_pos,
                          slot_mapping, status, (cudaStream_t)stream);
  return check_launch();
}

int spa_append_kv(const void* k_new, const void* v_new, int32_t act, void* k_cache, void* v_cache,
                  int32_t cache, const float* k_scale, const float* v_scale,
                  const int32_t* slot_mapping, int32_t T, int32_t H_kv, int32_t D,
                  int32_t block_size, int32_t num_blocks, int32_t* status, spa_stream_t stream) {
  if (!act_ok(act) || !(cache == act || cache == SPA_I8)) return SPA_ERR_INVALID_ARG;
  if (T < 0 || H_kv <= 0 || D <= 0 || block_size <= 0 || num_blocks < 0) return SPA_ERR_INVALID_ARG;
  if ((D * elt_bytes(act)) % 16 != 0) return SPA_ERR_INVALID_ARG;
  if (cache == SPA_I8 && (D % 16 != 0 || !k_scale || !v_scale)) return SPA_ERR_INVALID_ARG;
  if ((long long)num_blocks * block_size >= (1LL << 31)) return SPA_ERR_INVALID_ARG;
  if (T == 0) return SPA_OK;
  if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return SPA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new) |
       reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15)
    return SPA_ERR_INVALID_ARG;
  launch_append_kv(k_new, v_new, act, k_cache, v_cache, cache, k_scale, v_scale, slot_mapping, T,
                   H_kv, D, block_size, num_blocks, status, (cudaStream_t)stream);
  return check_launch();
}

int spa_prepare_append_kv(const int32_t* cu_seqlens_q, const int32_t* past_seqlens,
                          const int32_t* block_table, int32_t B, int32_t T, int32_t max_seqlen_q,
                          int32_t max_seqlen_k, int32_t MB, int32_t block_size, int32_t num_blocks,
                          int32_t* seqlens_q, int32_t* seqlen_k, int32_t* token_batch,
                          int32_t* token_pos, int32_t* slot_mapping, const void* k_new,
                          const void* v_new, int32_t act, void* k_cache, void* v_cache, int32_t cache,
                          const float* k_scale, const float* v_scale, int32_t H_kv, int32_t D,
                          int32_t* status, spa_stream_t stream) {
  // the union of both entry points' checks
  if (B < 0 || T < 0 || MB < 0 || block_size <= 0 || num_blocks < 0) return SPA_ERR_INVALID_ARG;
  if (B > 16384) return SPA_ERR_UNSUPPORTED;
  if ((long long)num_blocks * block_size >= (1LL << 31)) return SPA_ERR_INVALID_ARG;
  if (!cu_seqlens_q) return SPA_ERR_INVALID_ARG;
  if (B > 0 && (!past_seqlens || !seqlens_q || !seqlen_k || (MB > 0 && !block_table)))
    return SPA_ERR_INVALID_ARG;
  if (T > 0 && (!token_batch || !token_pos || !slot_mapping)) return SPA_ERR_INVALID_ARG;
  if (!act_ok(act) || !(cache == act || cache == SPA_I8)) return SPA_ERR_INVALID_ARG;
  if (H_kv <= 0 || D <= 0 || (D * elt_bytes(act)) % 16 != 0) return SPA_ERR_INVALID_ARG;
  if (cache == SPA_I8 && (D % 16 != 0 || !k_scale || !v_scale)) return SPA_ERR_INVALID_ARG;
  if (T > 0) {
    if (!k_new || !v_new || !k_cache || !v_cache) return SPA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new) |
         reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15)
      return SPA_ERR_INVALID_ARG;
  }
  launch_prepare_append(cu_seqlens_q, past_seqlens, block_table, B, T, max_seqlen_q, max_seqlen_k, MB,
                        block_size, num_blocks, seqlens_q, seqlen_k, token_batch, token_pos, slot_mapping,
                        k_new, v_new, act, k_cache, v_cache, cache, k_scale, v_scale, H_kv, D, status,
                        (cudaStream_t)stream);
  return check_launch();
}

size_t spa_attention_workspace_size(const spa_attention_args_t* a) {
  if (validate_attention(a) != SPA_OK) return 0;
  if (a->T == 0 || a->B == 0) return 0;
  Plan pl;
  if (make_plan(a, &pl) != SPA_OK) return 0;
  return pl.ws_acc_bytes + pl.ws_ml_bytes + pl.ws_count_bytes;
}

int spa_attention(const spa_attention_args_t* a, void* workspace, size_t workspace_bytes,
                  spa_stream_t stream) {
  int rc = validate_attention(a);
  if (rc != SPA_OK) return rc;
  if (a->T == 0 || a->B == 0) return SPA_OK;
  Plan pl;
  if ((rc = make_plan(a, &pl)) != SPA_OK) return rc;
  const size_t need = pl.ws_acc_bytes + pl.ws_ml_bytes + pl.ws_count_bytes;
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return SPA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return SPA_ERR_WORKSPACE;
  }
  return run_attention(a, pl, workspace, (cudaStream_t)stream);
}

// Validation of the step-1/2 arguments the fused step adds to `a`.
static int validate_step(const spa_attention_args_t* a, const int32_t* past_seqlens, const void* k_new,
                         const void* v_new, const int32_t* slot_mapping) {
  if (a->B > 16384) return SPA_ERR_UNSUPPORTED;
  if ((long long)a->num_blocks * a->block_size >= (1LL << 31)) return SPA_ERR_INVALID_ARG;
  if (a->B > 0 && (!past_seqlens || !a->seqlens_q || !a->seqlen_k)) return SPA_ERR_INVALID_ARG;
  if (a->T > 0 && (!a->token_batch || !a->token_pos || !slot_mapping || !k_new || !v_new))
    return SPA_ERR_INVALID_ARG;
  if ((a->D * elt_bytes(a->act)) % 16 != 0) return SPA_ERR_INVALID_ARG;
  if (a->cache == SPA_I8 && a->D % 16 != 0) return SPA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & 15) return SPA_ERR_INVALID_ARG;
  return SPA_OK;
}

int spa_prepare_append_attention(const spa_attention_args_t* a, const int32_t* past_seqlens,
                                 const void* k_new, const void* v_new, int32_t* slot_mapping, void* workspace,
                                 size_t workspace_bytes, spa_stream_t stream) {
  int rc = validate_attention(a);
  if (rc != SPA_OK) return rc;
  if ((rc = validate_step(a, past_seqlens, k_new, v_new, slot_mapping)) != SPA_OK) return rc;
  int32_t* seqlens_q = const_cast<int32_t*>(a->seqlens_q);
  int32_t* seqlen_k = const_cast<int32_t*>(a->seqlen_k);
  int32_t* token_batch = const_cast<int32_t*>(a->token_batch);
  int32_t* token_pos = const_cast<int32_t*>(a->token_pos);
  const cudaStream_t st = (cudaStream_t)stream;
  auto staged_prepare = [&]() {
    launch_prepare_append(a->cu_seqlens_q, past_seqlens, a->block_table, a->B, a->T, a->max_seqlen_q,
                          a->max_seqlen_k, a->MB, a->block_size, a->num_blocks, seqlens_q, seqlen_k, token_batch,
                          token_pos, slot_mapping, k_new, v_new, a->act, const_cast<void*>(a->k_cache),
                          const_cast<void*>(a->v_cache), a->cache, a->k_scale, a->v_scale, a->H_kv, a->D,
                          a->status, st);
    return check_launch();
  };
  if (a->T == 0 || a->B == 0) return staged_prepare();
  Plan pl;
  if ((rc = make_plan(a, &pl)) != SPA_OK) return rc;
  const size_t need = pl.ws_acc_bytes + pl.ws_ml_bytes + pl.ws_count_bytes;
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return SPA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return SPA_ERR_WORKSPACE;
  }
  if (!step_fusable(a, pl)) {
    if ((rc = staged_prepare()) != SPA_OK) return rc;
    return run_attention(a, pl, workspace, st);
  }
  AttnParams p;
  fill_params(a, pl, workspace, &p);
  p.past = past_seqlens;
  p.k_new = k_new;
  p.v_new = v_new;
  p.seqlens_q_out = seqlens_q;
  p.seqlen_k_out = seqlen_k;
  p.token_batch_out = token_batch;
  p.token_pos_out = token_pos;
  p.slot_out = slot_mapping;
  p.max_seqlen_q = a->max_seqlen_q;
  p.max_seqlen_k = a->max_seqlen_k;
  rc = pl.kind == kPlanTc ? launch_step_tc(p, a->act, a->cache, st) : launch_step_mma(p, a->act, pl.max_rows, st);
  if (rc != SPA_OK) return rc;
  return check_launch();
}

int spa_prepare_append_attention_launches(const spa_attention_args_t* a) {
  int rc = validate_attention(a);
  if (rc != SPA_OK) return rc;
  if (a->T == 0 || a->B == 0) return 1;
  Plan pl;
  if ((rc = make_plan(a, &pl)) != SPA_OK) return rc;
  return step_fusable(a, pl) ? 1 : 1 + launches_of(pl);
}

int spa_prepare_qkv_append(const spa_qkv_args_t* a, spa_stream_t stream) {
  if (!a || a->struct_size < sizeof(spa_qkv_args_t)) return SPA_ERR_INVALID_ARG;
  if (a->B < 0 || a->T < 0 || a->MB < 0 || a->block_size <= 0 || a->num_blocks < 0) return SPA_ERR_INVALID_ARG;
  if (a->B > 16384) return SPA_ERR_UNSUPPORTED;
  if ((long long)a->num_blocks * a->block_size >= (1LL << 31)) return SPA_ERR_INVALID_ARG;
  if (!act_ok(a->act) || !(a->cache == a->act || a->cache == SPA_I8)) return SPA_ERR_INVALID_ARG;
  if (a->H_q <= 0 || a->H_kv <= 0 || a->H_q % a->H_kv != 0) return SPA_ERR_INVALID_ARG;
  if (a->D != 64 && a->D != 128) return SPA_ERR_INVALID_ARG;
  if (a->cache == SPA_I8 && (!a->k_scale || !a->v_scale)) return SPA_ERR_INVALID_ARG;
  if (!a->cu_seqlens_q) return SPA_ERR_INVALID_ARG;
  if (a->B > 0 && (!a->past_seqlens || !a->seqlens_q || !a->seqlen_k || (a->MB > 0 && !a->block_table)))
    return SPA_ERR_INVALID_ARG;
  if (a->cos_cache) {
    if (!a->sin_cache || a->rotary_dim <= 0 || (a->rotary_dim & 1) || a->rotary_dim > a->D || a->max_pos <= 0)
      return SPA_ERR_INVALID_ARG;
  }
  if (a->T > 0) {
    if (!a->token_batch || !a->token_pos || !a->slot_mapping || !a->q_out || !a->k_cache || !a->v_cache)
      return SPA_ERR_INVALID_ARG;
    if (!a->qkv && (!a->q || !a->k || !a->v)) return SPA_ERR_INVALID_ARG;
    const uintptr_t al = reinterpret_cast<uintptr_t>(a->qkv) | reinterpret_cast<uintptr_t>(a->q) |
                         reinterpret_cast<uintptr_t>(a->k) | reinterpret_cast<uintptr_t>(a->v) |
                         reinterpret_cast<uintptr_t>(a->q_out) | reinterpret_cast<uintptr_t>(a->k_cache) |
                         reinterpret_cast<uintptr_t>(a->v_cache);
    if (al & 15) return SPA_ERR_INVALID_ARG;
  }
  QkvParams P;
  memset(&P, 0, sizeof(P));
  P.cu = a->cu_seqlens_q;
  P.past = a->past_seqlens;
  P.block_table = a->block_table;
  P.B = a->B;
  P.T = a->T;
  P.max_q = a->max_seqlen_q;
  P.max_k = a->max_seqlen_k;
  P.MB = a->MB;
  P.bs = a->block_size;
  P.NB = a->num_blocks;
  P.seqlens_q = a->seqlens_q;
  P.seqlen_k = a->seqlen_k;
  P.token_batch = a->token_batch;
  P.token_pos = a->token_pos;
  P.slot_mapping = a->slot_mapping;
  P.H_q = a->H_q;
  P.H_kv = a->H_kv;
  P.D = a->D;
  P.qkv = a->qkv;
  P.q = a->q;
  P.k = a->k;
  P.v = a->v;
  P.q_norm = a->q_norm_weight;
  P.k_norm = a->k_norm_weight;
  P.eps = a->norm_eps;
  P.cos_cache = a->cos_cache;
  P.sin_cache = a->sin_cache;
  P.max_pos = a->max_pos;
  P.rotary_dim = a->cos_cache ? a->rotary_dim : 0;
  P.interleaved = a->rotary_interleaved != 0;
  P.position_ids = a->position_ids;
  P.rotary_offset = a->rotary_offset;
  P.q_out = a->q_out;
  P.k_cache = a->k_cache;
  P.v_cache = a->v_cache;
  P.k_scale = a->k_scale;
  P.v_scale = a->v_scale;
  P.status = a->status;
  if (a->B == 0 && a->T == 0) return SPA_OK;
  int rc = launch_prepare_qkv_append(P, a->act, a->cache, (cudaStream_t)stream);
  if (rc != SPA_OK) return rc;
  return check_launch();
}

int spa_attention_plan(const spa_attention_args_t* a, int32_t* num_splits, int32_t* num_launches,
                       int32_t* kernel_kind) {
  int rc = validate_attention(a);
  if (rc != SPA_OK) return rc;
  Plan pl;
  memset(&pl, 0, sizeof(pl));
  if (a->T > 0 && a->B > 0 && (rc = make_plan(a, &pl)) != SPA_OK) return rc;
  const bool empty = a->T == 0 || a->B == 0;
  if (num_splits) *num_splits = empty ? 0 : pl.num_splits;
  if (num_launches) *num_launches = empty ? 0 : launches_of(pl);
  if (kernel_kind) *kernel_kind = empty ? -1 : pl.kind;
  return SPA_OK;
}

const char* spa_error_string(int code) {
  switch (code) {
    case SPA_OK: return "ok";
    case SPA_ERR_INVALID_ARG: return "invalid argument";
    case SPA_ERR_UNSUPPORTED: return "unsupported combination of arguments";
    case SPA_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case SPA_ERR_CUDA: return g_cuda_msg;
    case SPA_ERR_SCRATCH_LIMIT:
      return "the call needs more scratch than the library's static array (SPA_NOALLOC_SCRATCH_BYTES); "
             "use spa_attention with a caller workspace";
    default: return "unknown error code";
  }
}

}  // extern "C"
