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
  int* ws_count;         // [units] split tickets; zero between calls
  int32_t* status;
};

// Programmatic dependent launch: let the next kernel in the stream be
// scheduled early, and wait for the previous one before touching memory.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// What one CTA works on: a set of query rows sharing one candidate-key list.
struct Unit {
  int b, h_kv, t0, nq;    // request, kv head, first packed token, tokens
  int L;                  // total keys of the request (seqlen_k + 1)
  int p_first, p_last;    // positions of the first / last token (token i is at p_first + i)
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
  if (p.group_by_request) {
    // the request's tokens sit at past, past + 1, ... with past = L - q_len
    U.p_first = max(U.L - p.seqlens_q[U.b], 0);
  } else {
    U.p_first = p.token_pos[U.t0];
  }
  U.p_last = U.p_first + U.nq - 1;
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

// Log-sum-exp merge of the split partial states of one output row with the
// sink, by one warp (lanes over D); writes out[row] and lse[row].
template <typename ActT, int D>
__device__ __forceinline__ void merge_row(const AttnParams& p, long long row, int h, int lane) {
  constexpr int PER = D / 32;
  const float sink2 = p.sinks ? p.sinks[h] * kLog2e : -INFINITY;
  const long long stride = (long long)p.T * p.H_q;
  float M = sink2;
  for (int s = 0; s < p.num_splits; ++s) M = fmaxf(M, __ldcg(p.ws_ml + (s * stride + row) * 2));
  float o[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) o[i] = 0.f;
  float lse = -INFINITY;
  if (M != -INFINITY) {
    float Lsum = (sink2 == -INFINITY) ? 0.f : exp2f(sink2 - M);
    for (int s = 0; s < p.num_splits; ++s) {
      const float ms = __ldcg(p.ws_ml + (s * stride + row) * 2);
      if (ms == -INFINITY) continue;
      const float w = exp2f(ms - M);
      Lsum += w * __ldcg(p.ws_ml + (s * stride + row) * 2 + 1);
      const float* a = p.ws_acc + (s * stride + row) * D;
#pragma unroll
      for (int i = 0; i < PER; ++i) o[i] = fmaf(w, __ldcg(a + lane + 32 * i), o[i]);
    }
    const float inv = 1.0f / Lsum;
#pragma unroll
    for (int i = 0; i < PER; ++i) o[i] *= inv;
    lse = (M + log2f(Lsum)) * kLn2;
  }
  ActT* out = static_cast<ActT*>(p.out) + row * D;
#pragma unroll
  for (int i = 0; i < PER; ++i) out[lane + 32 * i] = from_f32<ActT>(o[i]);
  if (lane == 0 && p.lse) p.lse[row] = lse;
}

// Called by every thread of a split CTA once its partial states are written.
// The CTA that takes the last ticket of its unit merges all splits of the
// unit's rows (no CTA ever waits for another) and puts the ticket back to 0.
template <typename ActT, int D>
__device__ __forceinline__ void finish_split(const AttnParams& p, int unit, int t0, int nq, int h_kv,
                                             int* smem_flag) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(p.ws_count + unit, 1);
    const int last = prev == p.num_splits - 1;
    if (last) p.ws_count[unit] = 0;
    *smem_flag = last;
  }
  __syncthreads();
  if (!*smem_flag) return;
  __threadfence();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int R = nq * p.G;
  for (int r = warp; r < R; r += nw) {
    const int t = t0 + r / p.G, h = h_kv * p.G + r % p.G;
    merge_row<ActT, D>(p, (long long)t * p.H_q + h, h, lane);
  }
}

int scalar_key_tile();

}  // namespace spa
