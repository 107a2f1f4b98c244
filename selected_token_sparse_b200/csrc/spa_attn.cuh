// Device-side parameter block and unit decoding shared by the attention kernels.
#pragma once

#include <climits>
#include <type_traits>

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
  // fused step (metadata + append + attention in one launch): inputs of step
  // 1-2, and the metadata arrays as outputs
  const int32_t* past;
  const void* k_new;
  const void* v_new;
  int32_t* seqlens_q_out;
  int32_t* seqlen_k_out;
  int32_t* token_batch_out;
  int32_t* token_pos_out;
  int32_t* slot_out;
  int max_seqlen_q;      // host bounds for the step-1 status bits
  int max_seqlen_k;
  int cluster_merge;     // 1: the splits of a unit are one cluster, merged after a cluster barrier
  // one shard of a sequence split across devices: main-cache keys lo <= j < hi
  // of request b ([B, 2], or nullptr for all); out_f32: `out` is fp32 (the
  // shard's partial output; the host passes no sink then)
  const int32_t* kv_range;
  int out_f32;
  // test hook (0 in normal use): the tcgen05 prefill kernel drops one arrival
  // on a barrier that guards no copy or MMA, so that the bounded wait for it
  // expires and the CTA takes its abort path (SPA_ST_TIMEOUT)
  int test_expire_wait;
};

// Parameters of the fused metadata + QKV prologue + append kernel.
struct QkvParams {
  const int32_t* cu;
  const int32_t* past;
  const int32_t* block_table;
  int B, T, max_q, max_k, MB, bs, NB;
  int32_t* seqlens_q;
  int32_t* seqlen_k;
  int32_t* token_batch;
  int32_t* token_pos;
  int32_t* slot_mapping;
  int H_q, H_kv, D;
  const void* qkv;   // packed, or nullptr
  const void* q;
  const void* k;
  const void* v;
  const float* q_norm;
  const float* k_norm;
  float eps;
  const float* cos_cache;
  const float* sin_cache;
  int max_pos, rotary_dim, interleaved;
  const int32_t* position_ids;
  int rotary_offset;
  void* q_out;
  void* k_cache;
  void* v_cache;
  const float* k_scale;
  const float* v_scale;
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
  // fused step only: positions [new_lo, new_hi) are this step's tokens of the
  // request, whose K/V rows are read from k_new / v_new (token new_t0 + j - new_lo)
  int new_lo, new_hi, new_t0;
  int rlo, rhi;           // main-cache key range of this shard (0, INT_MAX: all)
};

// First packed token of request b under the sanitised cumulative lengths
// (the non-decreasing sequence clamped to [0, T] that token ownership follows):
// when request b has tokens and the raw lengths agree with its sanitised
// length, cu[b] is that start; otherwise (malformed lengths only) it is the
// sum of the sanitised lengths of the requests before b.
__device__ __forceinline__ int sanitised_start(const AttnParams& p, int b) {
  const int c0 = p.cu[b], c1 = p.cu[b + 1], q = p.seqlens_q[b];
  if (q > 0 && (long long)c1 - c0 == q) return c0;
  int s = 0;
  for (int i = 0; i < b; ++i) s += max(p.seqlens_q[i], 0);
  return s;
}

// Step-1 metadata as the attention kernels read it: the arrays written by the
// metadata entry points.
struct StagedMeta {
  const AttnParams& p;
  __device__ __forceinline__ int cu(int g) const { return sanitised_start(p, g); }
  __device__ __forceinline__ int seqlens_q(int b) const { return p.seqlens_q[b]; }
  __device__ __forceinline__ int seqlen_k(int b) const { return p.seqlen_k[b]; }
  __device__ __forceinline__ void token(int t, int& b, int& pos) const {
    b = p.token_batch[t];
    pos = p.token_pos[t];
  }
};

template <typename Meta>
__device__ __forceinline__ bool decode_unit_with(const AttnParams& p, const Meta& m, int u, Unit& U) {
  U.h_kv = u % p.H_kv;
  const int g = u / p.H_kv;
  int tpos = -1;
  U.new_lo = U.new_hi = U.new_t0 = 0;
  if (p.group_by_request) {
    U.b = g;
    U.t0 = clampi(m.cu(g), 0, p.T);
    U.nq = clampi(m.seqlens_q(g), 0, p.T - U.t0);
    U.nq = min(U.nq, p.max_q);
  } else {
    U.t0 = g;
    m.token(g, U.b, tpos);
    U.nq = 1;
  }
  if (U.b < 0 || U.b >= p.B || U.nq <= 0) return false;
  U.L = max(m.seqlen_k(U.b) + 1, 0);
  if (p.group_by_request) {
    // the request's tokens sit at past, past + 1, ... with past = L - q_len
    U.p_first = max(U.L - m.seqlens_q(U.b), 0);
  } else {
    U.p_first = tpos;
  }
  U.p_last = U.p_first + U.nq - 1;
  U.rlo = 0;
  U.rhi = INT_MAX;
  if (p.kv_range) {
    U.rlo = max(p.kv_range[2 * U.b], 0);
    U.rhi = p.kv_range[2 * U.b + 1];
  }
  U.sel_main = p.sel != nullptr && p.sel_target == 0;
  U.sel_aux = p.sel != nullptr && p.sel_target == 1;
  U.selrow = p.sel ? p.sel + ((long long)(p.sel_per_request ? U.b : U.t0) * p.H_kv + U.h_kv) * p.sel_width
                   : nullptr;
  U.lo = 0;
  if (U.sel_main) {
    U.n_main = p.sel_width;
  } else {
    U.lo = max(p.window > 0 ? max(0, U.p_first - p.window + 1) : 0, U.rlo);
    const int hi = min(min(U.p_last + 1, U.L), U.rhi);
    U.n_main = max(hi - U.lo, 0);
  }
  U.n_aux = U.sel_aux ? p.sel_width : 0;
  U.aux_n = U.sel_aux ? min(p.aux_len[U.b], p.aux_cap) : 0;
  return true;
}

__device__ __forceinline__ bool decode_unit(const AttnParams& p, int u, Unit& U) {
  return decode_unit_with(p, StagedMeta{p}, u, U);
}

// Resolve candidate c of a unit to a cache element offset (or -1) and a key
// position, in three stages so that callers resolving several candidates per
// thread can keep every stage's loads in flight together:
//   cand_stage1 -> the raw selection entry (selected modes) or the position;
//   cand_stage2 -> the block id of a main-cache key (or -1);
//   cand_finish -> guards (status bits), key position and element offset.
// `from_aux` tells which store the offset addresses.
__device__ __forceinline__ int cand_stage1(const AttnParams& p, const Unit& U, int c) {
  if (c < U.n_main) return U.sel_main ? U.selrow[c] : U.lo + c;
  return U.selrow[c - U.n_main];
}

__device__ __forceinline__ int cand_stage2(const AttnParams& p, const Unit& U, int c, int raw) {
  if (c >= U.n_main) return -1;
  if (U.sel_main && (raw < 0 || raw >= U.L || raw < U.rlo || raw >= U.rhi)) return -1;
  const int lb = raw / p.bs;
  if (lb >= p.MB) return -1;
  return p.block_table[(long long)U.b * p.MB + lb];
}

__device__ __forceinline__ long long cand_finish(const AttnParams& p, const Unit& U, int c, int raw, int blk,
                                                 int& kpos, bool& from_aux, int& bits) {
  kpos = kPosInvalid;
  from_aux = false;
  if (c < U.n_main) {
    if (U.sel_main) {
      if (raw == -1) return -1;
      if (raw < -1 || raw >= U.L) {
        bits |= kStBadIdx;
        return -1;
      }
      if (raw < U.rlo || raw >= U.rhi) return -1;   // another shard's key
    }
    const int j = raw;
    if (j / p.bs >= p.MB) {
      bits |= kStCapacity;
      return -1;
    }
    if (blk < 0 || blk >= p.NB) {
      bits |= kStBadBlock;
      return -1;
    }
    kpos = j;
    return ((long long)blk * p.bs + (j % p.bs)) * p.H_kv * p.D + (long long)U.h_kv * p.D;
  }
  if (raw == -1) return -1;
  if (raw < -1 || raw >= U.aux_n) {
    bits |= kStBadIdx;
    return -1;
  }
  kpos = kPosAux;
  from_aux = true;
  return (((long long)U.b * p.aux_cap + raw) * p.H_kv + U.h_kv) * p.D;
}

__device__ __forceinline__ long long resolve_candidate(const AttnParams& p, const Unit& U, int c,
                                                       int& kpos, bool& from_aux, int& bits) {
  const int raw = cand_stage1(p, U, c);
  return cand_finish(p, U, c, raw, cand_stage2(p, U, c, raw), kpos, from_aux, bits);
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

// Log-sum-exp merge of the split partial states of a unit's rows with the
// sink ("[WebGPU] Add SparsePagedAttention", finalize: every split's running
// max m_s and sum l_s are rescaled to the global max M; the sink joins the
// denominator).  The whole CTA works on it with independent loads so the L2
// latency of the workspace reads overlaps:
//   pass 1, one thread per row: M = max(sink, m_s), L = sum_s 2^(m_s - M) l_s
//           (+ 2^(sink - M)), lse = (M + log2 L) ln 2, kept in shared memory;
//   pass 2, one thread per 4 output columns: o = sum_s 2^(m_s - M) acc_s / L.
// Rows go in chunks of kMergeRows (the shared arrays' size).
constexpr int kMergeRows = 128;

template <typename ActT>
__device__ __forceinline__ void store4(ActT* dst, float a, float b, float c, float d) {
  if constexpr (std::is_same<ActT, float>::value) {
    *reinterpret_cast<float4*>(dst) = make_float4(a, b, c, d);
  } else {
    ActT v[4] = {from_f32<ActT>(a), from_f32<ActT>(b), from_f32<ActT>(c), from_f32<ActT>(d)};
    *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(v);
  }
}

// Four output columns at element offset `off` of `out`: in the activation
// dtype, or fp32 for a shard's partial output.
template <typename ActT>
__device__ __forceinline__ void store_out4(const AttnParams& p, long long off, float a, float b, float c, float d) {
  if (p.out_f32) *reinterpret_cast<float4*>(static_cast<float*>(p.out) + off) = make_float4(a, b, c, d);
  else store4<ActT>(static_cast<ActT*>(p.out) + off, a, b, c, d);
}

template <typename ActT, int D>
__device__ __forceinline__ void merge_rows(const AttnParams& p, int t0, int nq, int h_kv) {
  __shared__ float sM[kMergeRows], sInv[kMergeRows];
  constexpr int C4 = D / 4;
  const long long stride = (long long)p.T * p.H_q;
  const int R = nq * p.G, S = p.num_splits;
  for (int r0 = 0; r0 < R; r0 += kMergeRows) {
    const int nr = min(kMergeRows, R - r0);
    for (int i = threadIdx.x; i < nr; i += blockDim.x) {
      const int r = r0 + i;
      const int h = h_kv * p.G + r % p.G;
      const long long row = (long long)(t0 + r / p.G) * p.H_q + h;
      const float sink2 = p.sinks ? p.sinks[h] * kLog2e : -INFINITY;
      float M = sink2;
#pragma unroll 4
      for (int s = 0; s < S; ++s) M = fmaxf(M, __ldcg(p.ws_ml + (s * stride + row) * 2));
      float inv = 0.f, lse = -INFINITY;
      if (M != -INFINITY) {
        float Lsum = (sink2 == -INFINITY) ? 0.f : exp2f(sink2 - M);
#pragma unroll 4
        for (int s = 0; s < S; ++s) {
          const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.ws_ml + (s * stride + row) * 2));
          if (ml.x != -INFINITY) Lsum += exp2f(ml.x - M) * ml.y;
        }
        inv = 1.0f / Lsum;
        lse = (M + log2f(Lsum)) * kLn2;
      }
      sM[i] = M;
      sInv[i] = inv;
      if (p.lse) p.lse[row] = lse;
    }
    __syncthreads();
    // four output items per thread in flight; out-of-range items re-read the
    // chunk's last item and store nothing
    const int n_items = nr * C4;
    for (int base = threadIdx.x; base < n_items; base += 4 * blockDim.x) {
      int ii[4];
      long long rw[4];
      float Mi[4];
      float4 o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        ii[j] = min(base + j * (int)blockDim.x, n_items - 1);
        const int r = r0 + ii[j] / C4;
        rw[j] = (long long)(t0 + r / p.G) * p.H_q + h_kv * p.G + r % p.G;
        Mi[j] = sM[ii[j] / C4];
        o[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll 2
      for (int s = 0; s < S; ++s) {
        float ms[4];
        float4 a[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          ms[j] = __ldcg(p.ws_ml + (s * stride + rw[j]) * 2);
          a[j] = __ldcg(reinterpret_cast<const float4*>(p.ws_acc + (s * stride + rw[j]) * D + (ii[j] % C4) * 4));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (ms[j] == -INFINITY || Mi[j] == -INFINITY) continue;
          const float w = exp2f(ms[j] - Mi[j]);
          o[j].x = fmaf(w, a[j].x, o[j].x);
          o[j].y = fmaf(w, a[j].y, o[j].y);
          o[j].z = fmaf(w, a[j].z, o[j].z);
          o[j].w = fmaf(w, a[j].w, o[j].w);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (base + j * (int)blockDim.x >= n_items) continue;
        const float inv = sInv[ii[j] / C4];
        store_out4<ActT>(p, rw[j] * D + (ii[j] % C4) * 4, o[j].x * inv, o[j].y * inv, o[j].z * inv, o[j].w * inv);
      }
    }
    __syncthreads();
  }
}

// Split merge inside a thread-block cluster.  The num_splits CTAs of a unit
// form one cluster (rank = split).  Each has written its partial state of the
// unit's rows to the workspace, as the ticket merge's splits do (ws_acc
// [split][T * H_q][D], ws_ml [split][T * H_q][2], log2 units), and passed a
// cluster barrier (release / acquire) after that; then CTA k merges rows k,
// k + S, k + 2S, ... with the sink as merge_rows does, in one pass: each
// thread takes 4 output columns of a row, reads every split's (m, l) and
// partial columns from L2 at once, and forms the weights itself.  No CTA
// reads another's shared memory, so none waits for the others to leave.
// (Pulling the partial states from the peers' shared memory instead costs a
// second cluster barrier and moves them over the SM-to-SM network, which
// measured slower than L2 for these sizes.)
constexpr int kClusterMaxSplits = 8;

// SMAX bounds the split count; IPT items of a thread have their loads in
// flight together.
template <typename ActT, int D, int SMAX, int IPT>
__device__ __forceinline__ void cluster_merge_rows(const AttnParams& p, int t0, int nq, int h_kv) {
  constexpr int C4 = D / 4;
  const int S = p.num_splits, k = (int)cluster_rank();
  const int R = nq * p.G;
  const long long stride = (long long)p.T * p.H_q;
  const int mine = R > k ? (R - k + S - 1) / S : 0;   // rows k, k + S, ...
  const int n_items = mine * C4;
  for (int base = threadIdx.x; base < n_items; base += IPT * blockDim.x) {
    float2 ml[IPT][SMAX];
    float4 a[IPT][SMAX];
    float sink2[IPT];
    long long rw[IPT];
#pragma unroll
    for (int t = 0; t < IPT; ++t) {
      const int it = base + t * blockDim.x;
      const int r = k + (it / C4) * S, c = (it % C4) * 4;
      const int h = h_kv * p.G + r % p.G;
      rw[t] = (long long)(t0 + r / p.G) * p.H_q + h;
      sink2[t] = (p.sinks && it < n_items) ? __ldg(p.sinks + h) * kLog2e : -INFINITY;
#pragma unroll
      for (int s = 0; s < SMAX; ++s) {
        ml[t][s] = make_float2(-INFINITY, 0.f);
        a[t][s] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s < S && it < n_items) {
          ml[t][s] = __ldcg(reinterpret_cast<const float2*>(p.ws_ml + (s * stride + rw[t]) * 2));
          a[t][s] = __ldcg(reinterpret_cast<const float4*>(p.ws_acc + (s * stride + rw[t]) * D + c));
        }
      }
    }
#pragma unroll
    for (int t = 0; t < IPT; ++t) {
      const int it = base + t * blockDim.x;
      if (it >= n_items) continue;
      const int c = (it % C4) * 4;
      float M = sink2[t];
#pragma unroll
      for (int s = 0; s < SMAX; ++s) M = fmaxf(M, ml[t][s].x);
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      float inv = 0.f, lse = -INFINITY;
      if (M != -INFINITY) {
        float Lsum = (sink2[t] == -INFINITY) ? 0.f : exp2f(sink2[t] - M);
#pragma unroll
        for (int s = 0; s < SMAX; ++s) {
          const float w = (ml[t][s].x == -INFINITY) ? 0.f : exp2f(ml[t][s].x - M);
          Lsum += w * ml[t][s].y;
          o.x = fmaf(w, a[t][s].x, o.x);
          o.y = fmaf(w, a[t][s].y, o.y);
          o.z = fmaf(w, a[t][s].z, o.z);
          o.w = fmaf(w, a[t][s].w, o.w);
        }
        inv = 1.0f / Lsum;
        lse = (M + log2f(Lsum)) * kLn2;
      }
      store_out4<ActT>(p, rw[t] * D + c, o.x * inv, o.y * inv, o.z * inv, o.w * inv);
      if (c == 0 && p.lse) p.lse[rw[t]] = lse;
    }
  }
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
  merge_rows<ActT, D>(p, t0, nq, h_kv);
}

int scalar_key_tile();

}  // namespace spa
