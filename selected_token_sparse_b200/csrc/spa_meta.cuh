// Step 1 helpers shared by the metadata kernels and the fused step kernel:
// the sanitised cumulative lengths, the per-request outputs and the per-token
// (request, position, slot) metadata ("[WebGPU] Add PagedAttention metadata
// and GPT-OSS support", Description and Changes; "[WebGPU] Add
// SparsePagedAttention", review notes on the per-token scan and on malformed
// cumulative lengths).  Every caller runs this same code, so their outputs
// agree bit for bit.
#pragma once

#include "spa_attn.cuh"

namespace spa {

// Sanitised cumulative lengths into cs[0..B] (all threads of the block).
// With `past`, the past lengths are copied into past_s[0..B) as well; their
// first loads are issued ahead of the cumulative lengths' so that both are in
// flight together, and the copy is visible once this returns.
template <int NT>
__device__ __forceinline__ void build_cs(const int32_t* __restrict__ cu, int B, int T, int32_t* cs,
                                         const int32_t* __restrict__ past = nullptr, int32_t* past_s = nullptr) {
  __shared__ int32_t warp_max[NT / 32];
  __shared__ int32_t chunk_carry[NT];
  const int tid = threadIdx.x;
  const int pv0 = (past != nullptr && tid < B) ? ld_early(past + tid) : 0;
  const int n = B + 1;
  // contiguous chunk per thread: local prefix max, then a scan over chunk maxima
  const int per = (n + NT - 1) / NT;
  const int c0 = tid * per;
  const int c1 = min(c0 + per, n);
  int run = 0;  // cs[0] = 0 takes part in the maximum
  for (int i = c0; i < c1; ++i) {
    int v = (i == 0) ? 0 : cu[i];
    run = max(run, v);
    cs[i] = run;
  }
  const int lane = tid & 31, warp = tid >> 5;
  int x = (c0 < c1) ? run : 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x = max(x, y);
  }
  if (lane == 31) warp_max[warp] = x;
  if (past != nullptr) {
    if (tid < B) past_s[tid] = pv0;
    for (int b = tid + NT; b < B; b += NT) past_s[b] = past[b];
  }
  __syncthreads();
  int prev_warps = 0;
  for (int w = 0; w < warp; ++w) prev_warps = max(prev_warps, warp_max[w]);
  chunk_carry[tid] = max(x, prev_warps);
  __syncthreads();
  const int carry = (tid == 0) ? 0 : chunk_carry[tid - 1];
  for (int i = c0; i < c1; ++i) cs[i] = min(max(cs[i], carry), T);
  __syncthreads();
}

// build_cs without a block barrier, for B + 1 <= 64: every warp computes the
// clamped cumulative lengths (a shuffle prefix maximum) and copies the past
// lengths itself, and writes them to shared memory (all warps write the same
// values; each reads back only after its own writes).  The caller loaded
// cu[lane], cu[lane + 32] (entries <= B, entry 0 unused) and past[lane],
// past[lane + 32] (entries < B).  Loads still in flight when it runs are not
// waited for, as a block barrier would.
__device__ __forceinline__ void build_cs_warp(int B, int T, int32_t* cs, int32_t* past_s, int cu0, int cu1,
                                              int p0, int p1) {
  const int lane = threadIdx.x & 31;
  const int i0 = lane, i1 = lane + 32;
  int x0 = (i0 == 0 || i0 > B) ? 0 : cu0;
  int x1 = i1 > B ? 0 : cu1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y0 = __shfl_up_sync(0xffffffffu, x0, o);
    const int y1 = __shfl_up_sync(0xffffffffu, x1, o);
    if (lane >= o) {
      x0 = max(x0, y0);
      x1 = max(x1, y1);
    }
  }
  x1 = max(x1, __shfl_sync(0xffffffffu, x0, 31));
  if (i0 <= B) cs[i0] = min(x0, T);
  if (i1 <= B) cs[i1] = min(x1, T);
  if (i0 < B) past_s[i0] = p0;
  if (i1 < B) past_s[i1] = p1;
  __syncwarp();
}

// seqlen_k of a request: past + q_len - 1 (past < 0 counts as 0), as int32.
__device__ __forceinline__ int32_t request_seqlen_k(int past, int q_len) {
  return (int32_t)((long long)max(past, 0) + q_len - 1);
}

// Per-request outputs and the request-level status bits (block 0 only).
// Threads ti = 0 .. nthr - 1 of the block share the work.
__device__ __forceinline__ int per_request(const int32_t* __restrict__ cu, const int32_t* __restrict__ past,
                                           const int32_t* cs, int B, int T, int max_q, int max_k,
                                           int32_t* __restrict__ seqlens_q, int32_t* __restrict__ seqlen_k,
                                           int ti, int nthr) {
  int bits = 0;
  for (int b = ti; b <= B; b += nthr) {
    if (cu[b] != cs[b]) bits |= kStBadCu;
    if (b == B && cs[B] != T) bits |= kStBadCu;
  }
  for (int b = ti; b < B; b += nthr) {
    int pb = past[b];
    if (pb < 0) {
      bits |= kStBadCu;
      pb = 0;
    }
    const int q_len = cs[b + 1] - cs[b];
    const long long total = (long long)pb + q_len;
    seqlens_q[b] = q_len;
    seqlen_k[b] = request_seqlen_k(pb, q_len);
    if (q_len > max_q || total > (long long)max_k) bits |= kStBounds;
  }
  return bits;
}
__device__ __forceinline__ int per_request(const int32_t* __restrict__ cu, const int32_t* __restrict__ past,
                                           const int32_t* cs, int B, int T, int max_q, int max_k,
                                           int32_t* __restrict__ seqlens_q, int32_t* __restrict__ seqlen_k) {
  return per_request(cu, past, cs, B, T, max_q, max_k, seqlens_q, seqlen_k, threadIdx.x, blockDim.x);
}

struct TokenMeta {
  int b, pos, slot;
};

// Owner request (-1 if none) and absolute position (-1 if none) of token t.
__device__ __forceinline__ void token_owner(int t, const int32_t* cs, int B, const int32_t* past, int& b,
                                            int& pos) {
  int lo = 0, hi = B + 1;  // owner = upper_bound(cs[0..B], t) - 1
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (cs[mid] <= t) lo = mid + 1; else hi = mid;
  }
  b = lo - 1;
  pos = -1;
  if (t >= cs[B] || b < 0 || b >= B) {
    b = -1;
    return;
  }
  pos = max(past[b], 0) + (t - cs[b]);
}

// Token metadata in two halves so that the block-table load can be in flight
// while other work runs: the load half finds the owner and position and reads
// the block id, the finish half validates it (status bits) and forms the slot.
struct TokenLoad {
  int b, pos, lb, blk;
};

__device__ __forceinline__ TokenLoad token_meta_load(int t, const int32_t* cs, int B, const int32_t* past,
                                                     const int32_t* __restrict__ block_table, int MB, int bs) {
  TokenLoad l;
  token_owner(t, cs, B, past, l.b, l.pos);
  l.lb = -1;
  l.blk = -1;
  if (l.b >= 0) {
    l.lb = l.pos / bs;
    if (l.lb < MB) l.blk = ld_early(block_table + (long long)l.b * MB + l.lb);
  }
  return l;
}

__device__ __forceinline__ TokenMeta token_meta_finish(const TokenLoad& l, int MB, int bs, int num_blocks,
                                                       int& bits) {
  TokenMeta m = {-1, -1, -1};
  if (l.b < 0) return m;
  m.b = l.b;
  m.pos = l.pos;
  if (l.lb >= MB) bits |= kStCapacity;
  else if (l.blk < 0 || l.blk >= num_blocks) bits |= kStBadBlock;
  else m.slot = l.blk * bs + l.pos % bs;
  return m;
}

// Owner request, absolute position and cache slot of token t.
__device__ __forceinline__ TokenMeta token_meta(int t, const int32_t* cs, int B,
                                                const int32_t* __restrict__ past,
                                                const int32_t* __restrict__ block_table, int MB, int bs,
                                                int num_blocks, int& bits) {
  return token_meta_finish(token_meta_load(t, cs, B, past, block_table, MB, bs), MB, bs, num_blocks, bits);
}

// Step-1 metadata computed in shared memory by the fused step kernel from
// the raw cumulative lengths, their sanitised form cs and the past lengths,
// with the same helpers as the metadata kernels.
struct FusedMeta {
  const int32_t* cu_raw;
  const int32_t* cs;
  const int32_t* past;
  int B;
  __device__ __forceinline__ int cu(int g) const { return cs[g]; }   // request g's first token
  __device__ __forceinline__ int seqlens_q(int b) const { return cs[b + 1] - cs[b]; }
  __device__ __forceinline__ int seqlen_k(int b) const { return request_seqlen_k(past[b], cs[b + 1] - cs[b]); }
  __device__ __forceinline__ void token(int t, int& b, int& pos) const { token_owner(t, cs, B, past, b, pos); }
};

// Candidate offsets of a fused step that address k_new / v_new rather than
// the cache carry this bit.
constexpr long long kNewRow = 1LL << 62;

// Steps 1 and 2 inside the attention CTAs of a fused step.
//
// Request-level part (CTA 0 of split 0): the per-request outputs and, with
// request-grouped units, the metadata of tokens no request owns.
__device__ __forceinline__ void fused_request_outputs(const AttnParams& p, const int32_t* cs, const int32_t* past,
                                                      int& bits, int ti, int nthr) {
  bits |= per_request(p.cu, past, cs, p.B, p.T, p.max_seqlen_q, p.max_seqlen_k, p.seqlens_q_out,
                      p.seqlen_k_out, ti, nthr);
  if (p.group_by_request) {
    for (int t = cs[p.B] + ti; t < p.T; t += nthr) {
      p.token_batch_out[t] = -1;
      p.token_pos_out[t] = -1;
      p.slot_out[t] = -1;
    }
  }
}
__device__ __forceinline__ void fused_request_outputs(const AttnParams& p, const int32_t* cs, const int32_t* past,
                                                      int& bits) {
  fused_request_outputs(p, cs, past, bits, threadIdx.x, blockDim.x);
}

// Token-level part for token t and kv head h_kv (split 0): the token's
// metadata, written by kv head 0.
__device__ __forceinline__ void fused_token_outputs(const AttnParams& p, int t, int h_kv, const TokenMeta& m,
                                                    int tb, int& bits) {
  if (h_kv == 0 && threadIdx.x == 0) {
    bits |= tb;
    p.token_batch_out[t] = m.b;
    p.token_pos_out[t] = m.pos;
    p.slot_out[t] = m.slot;
  }
}

// The token's K/V rows of one kv head go to the cache as 16-byte vectors (an
// exact copy for 16-bit caches): vector v < nv of the K row, v - nv of the V row.
template <typename T16>
__device__ __forceinline__ void fused_store_row_vector(const AttnParams& p, int slot, int h_kv, int v, int nv,
                                                       const uint4& data) {
  const bool isv = v >= nv;
  uint4* dp = reinterpret_cast<uint4*>(static_cast<T16*>(const_cast<void*>(isv ? p.v_cache : p.k_cache)) +
                                       ((long long)slot * p.H_kv + h_kv) * p.D);
  dp[isv ? v - nv : v] = data;
}

template <typename T16>
__device__ __forceinline__ uint4 fused_load_row_vector(const AttnParams& p, int t, int h_kv, int v, int nv) {
  const bool isv = v >= nv;
  const uint4* sp = reinterpret_cast<const uint4*>(static_cast<const T16*>(isv ? p.v_new : p.k_new) +
                                                   ((long long)t * p.H_kv + h_kv) * p.D);
  return ld_early(sp + (isv ? v - nv : v));
}

// Tokens [t_lo, t_hi) of a unit, metadata and rows loaded where they are used.
template <typename T16>
__device__ __forceinline__ void fused_append_tokens(const AttnParams& p, const int32_t* cs, const int32_t* past,
                                                    int t_lo, int t_hi, int h_kv, int& bits) {
  const int nv = p.D * (int)sizeof(T16) / 16;
  for (int t = t_lo; t < t_hi; ++t) {
    int tb = 0;
    const TokenMeta m = token_meta(t, cs, p.B, past, p.block_table, p.MB, p.bs, p.NB, tb);
    fused_token_outputs(p, t, h_kv, m, tb, bits);
    if (m.slot < 0) continue;
    for (int v = threadIdx.x; v < 2 * nv; v += blockDim.x)
      fused_store_row_vector<T16>(p, m.slot, h_kv, v, nv, fused_load_row_vector<T16>(p, t, h_kv, v, nv));
  }
}

// Tokens [t_lo, t_hi) of a unit for kv head h_kv, by threads ti = 0 .. nthr - 1:
// each (token, item) pair finds the token's slot (the thread with item 0 of a
// token writes its metadata, from kv head 0) and stores one item of the rows
// -- a 16-byte vector copied (16-bit caches) or a 16-channel group quantised
// with the shared group quantiser (INT8 caches; `ksc` / `vsc` are this kv
// head's scales), so the cache holds what the append kernels write.
template <typename ActT, typename CacheT>
__device__ __forceinline__ void fused_append_rows(const AttnParams& p, const int32_t* cs, const int32_t* past,
                                                 int t_lo, int t_hi, int h_kv, const float* ksc, const float* vsc,
                                                 int ti, int nthr, int& bits) {
  constexpr bool kI8 = sizeof(CacheT) == 1;
  const int per_row = kI8 ? p.D / 16 : p.D * (int)sizeof(CacheT) / 16;
  const int per_tok = 2 * per_row;
  const int n = max(t_hi - t_lo, 0) * per_tok;
  for (int idx = ti; idx < n; idx += nthr) {
    const int t = t_lo + idx / per_tok, it = idx % per_tok;
    int tb = 0;
    const TokenMeta m = token_meta(t, cs, p.B, past, p.block_table, p.MB, p.bs, p.NB, tb);
    if (it == 0 && h_kv == 0) {
      bits |= tb;
      p.token_batch_out[t] = m.b;
      p.token_pos_out[t] = m.pos;
      p.slot_out[t] = m.slot;
    }
    if (m.slot < 0) continue;
    if constexpr (kI8) {
      const bool isv = it >= per_row;
      const int g = isv ? it - per_row : it;
      Group16<ActT> x;
      x.load(static_cast<const ActT*>(isv ? p.v_new : p.k_new) + ((long long)t * p.H_kv + h_kv) * p.D + g * 16);
      int8_t* dst = static_cast<int8_t*>(const_cast<void*>(isv ? p.v_cache : p.k_cache)) +
                    ((long long)m.slot * p.H_kv + h_kv) * p.D + g * 16;
      *reinterpret_cast<uint4*>(dst) = quant_group16<ActT>(x.v, (isv ? vsc : ksc) + g * 16);
    } else {
      fused_store_row_vector<CacheT>(p, m.slot, h_kv, it, per_row, fused_load_row_vector<CacheT>(p, t, h_kv, it, per_row));
    }
  }
}

}  // namespace spa
