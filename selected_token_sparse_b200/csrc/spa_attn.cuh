// Device-side parameter block and unit decoding shared by the attention kernels.
#pragma once

#include <climits>

#include "spa_common.cuh"

namespace spa {

constexpr int kPosInvalid = INT_MAX;  // key slot holds nothing
constexpr int kPosAux = INT_MIN;      // auxiliary entry: visible to every row of the request

struct AttnParams {
  const void* q;
  void* out;
  float* lse;
  const void* k_cache;
  const void* v_cache;
  const float* k_scale;
  const float* v_scale;
  const int32_t* block_table;
  int MB, bs, NB;
  const int32_t* cu;
  const int32_t* seqlens_q;
  const int32_t* seqlen_k;
  const int32_t* token_batch;
  const int32_t* token_pos;
  int T, B, H_q, H_kv, D, G;
  int window;
  const int32_t* sel;
  int sel_width, sel_per_request, sel_target;
  const void* aux_k;
  const void* aux_v;
  int aux_cap;
  const int32_t* aux_len;
  const float* sinks;
  float scale_log2;      // softmax scale * log2(e)
  int group_by_request;  // 1: unit = (request, kv head), rows = q_len * G; 0: unit = (token, kv head)
  int max_q;             // tokens per unit bound (host max_seqlen_q, or 1)
  int max_k;             // host bound max_seqlen_k
  int num_splits;
  int split_len;         // candidates per split (multiple of the kernel's key tile)
  float* ws_acc;         // [num_splits, T, H_q, D]
  float* ws_ml;          // [num_splits, T, H_q, 2]
  int32_t* status;
};

// What one CTA works on: a set of query rows sharing one candidate-key list.
struct Unit {
  int b, h_kv, t0, nq;    // request, kv head, first packed token, tokens
  int L;                  // total keys of the request (seqlen_k + 1)
  int p_first, p_last;    // positions of the first / last token
  int lo, n_main, n_aux;  // main candidates [lo, lo + n_main) (or selection slots), aux slots
  int aux_n;              // valid auxiliary entries of the request
  const int32_t* selrow;  // selection row or nullptr
  bool sel_main, sel_aux;
};

__device__ __forceinline__ bool decode_unit(const AttnParams& p, int u, Unit& U) {
  U.h_kv = u % p.H_kv;
  const int g = u / p.H_kv;
  if (p.group_by_request) {
    U.b = g;
    U.t0 = clampi(p.cu[g], 0, p.T);
    U.nq = clampi(p.seqlens_q[g], 0, p.T - U.t0);
    U.nq = min(U.nq, p.max_q);
  } else {
    U.t0 = g;
    U.b = p.token_batch[g];
    U.nq = 1;
  }
  if (U.b < 0 || U.b >= p.B || U.nq <= 0) return false;
  U.L = max(p.seqlen_k[U.b] + 1, 0);
  U.p_first = p.token_pos[U.t0];
  U.p_last = p.token_pos[U.t0 + U.nq - 1];
  U.sel_main = p.sel != nullptr && p.sel_target == 0;
  U.sel_aux = p.sel != nullptr && p.sel_target == 1;
  U.selrow = p.sel ? p.sel + ((long long)(p.sel_per_request ? U.b : U.t0) * p.H_kv + U.h_kv) * p.sel_width
                   : nullptr;
  U.lo = 0;
  if (U.sel_main) {
    U.n_main = p.sel_width;
  } else {
    U.lo = p.window > 0 ? max(0, U.p_first - p.window + 1) : 0;
    const int hi = min(U.p_last + 1, U.L);
    U.n_main = max(hi - U.lo, 0);
  }
  U.n_aux = U.sel_aux ? p.sel_width : 0;
  U.aux_n = U.sel_aux ? min(p.aux_len[U.b], p.aux_cap) : 0;
  return true;
}

// Resolve candidate c of a unit to a cache element offset (or -1) and a key position.
// `from_aux` tells which store the offset addresses.  Status bits go to `bits`.
__device__ __forceinline__ long long resolve_candidate(const AttnParams& p, const Unit& U, int c,
                                                       int& kpos, bool& from_aux, int& bits) {
  kpos = kPosInvalid;
  from_aux = false;
  if (c < U.n_main) {
    int j;
    if (U.sel_main) {
      const int idx = U.selrow[c];
      if (idx == -1) return -1;
      if (idx < -1 || idx >= U.L) {
        bits |= kStBadIdx;
        return -1;
      }
      j = idx;
    } else {
      j = U.lo + c;
    }
    const int lb = j / p.bs;
    if (lb >= p.MB) {
      bits |= kStCapacity;
      return -1;
    }
    const int blk = p.block_table[(long long)U.b * p.MB + lb];
    if (blk < 0 || blk >= p.NB) {
      bits |= kStBadBlock;
      return -1;
    }
    kpos = j;
    return ((long long)blk * p.bs + (j % p.bs)) * p.H_kv * p.D + (long long)U.h_kv * p.D;
  }
  const int idx = U.selrow[c - U.n_main];
  if (idx == -1) return -1;
  if (idx < -1 || idx >= U.aux_n) {
    bits |= kStBadIdx;
    return -1;
  }
  kpos = kPosAux;
  from_aux = true;
  return (((long long)U.b * p.aux_cap + idx) * p.H_kv + U.h_kv) * p.D;
}

__device__ __forceinline__ bool key_visible(int kpos, int prow, int window) {
  if (kpos == kPosAux) return true;
  if (kpos == kPosInvalid) return false;
  return kpos <= prow && (window <= 0 || kpos > prow - window);
}

// Final normalisation of one row with the sink (log2 units).
__device__ __forceinline__ void finalize_row(float m, float l, float sink2, float& a, float& inv_l,
                                             float& lse) {
  const float mf = fmaxf(m, sink2);
  if (mf == -INFINITY) {
    a = 0.f;
    inv_l = 0.f;
    lse = -INFINITY;
    return;
  }
  a = (m == -INFINITY) ? 0.f : exp2f(m - mf);
  const float lf = l * a + ((sink2 == -INFINITY) ? 0.f : exp2f(sink2 - mf));
  inv_l = 1.0f / lf;
  lse = (mf + log2f(lf)) * kLn2;
}

int launch_attention_scalar(const AttnParams& p, int max_rows, cudaStream_t stream);
int launch_combine(const AttnParams& p, cudaStream_t stream);
int scalar_key_tile();

}  // namespace spa
