// Step 1 -- metadata prepare (and its fusion with step 2, the KV append).
//
// Derives the exact per-request lengths and the per-token (request, position,
// slot) metadata on the device, so that no device-to-host copy is needed per
// layer ("[WebGPU] Add PagedAttention metadata and GPT-OSS support",
// Description and Changes; worked cases in review item T1).  The per-token
// request index is a binary search over the sanitised cumulative lengths,
// not a linear scan ("[WebGPU] Add SparsePagedAttention", review note on the
// O(batch_size) scan per token and on malformed cumulative lengths).
//
// Every block rebuilds the sanitised cumulative lengths
//   cs[0] = 0,  cs[b] = min(max(cu[1..b], 0), T)
// (a clamped prefix maximum) in shared memory with a block-wide scan; block 0
// also writes the per-request outputs and status bits.
//
// prepare_append_kernel fuses the scatter of the current tokens' K/V rows
// into the same launch (one warp per token: the lanes find the token's slot,
// then copy its rows as 16-byte vectors, quantising for an INT8 cache); its
// outputs are bit-identical to spa_prepare_metadata followed by spa_append_kv.
#include "spa_attn.cuh"
#include "spa_meta.cuh"

namespace spa {

constexpr int kMetaThreads = 256;

__global__ void __launch_bounds__(kMetaThreads)
prepare_metadata_kernel(const int32_t* __restrict__ cu, const int32_t* __restrict__ past,
                        const int32_t* __restrict__ block_table, int B, int T, int max_q,
                        int max_k, int MB, int bs, int num_blocks, int32_t* __restrict__ seqlens_q,
                        int32_t* __restrict__ seqlen_k, int32_t* __restrict__ token_batch,
                        int32_t* __restrict__ token_pos, int32_t* __restrict__ slot_mapping,
                        int32_t* __restrict__ status) {
  extern __shared__ int32_t cs[];  // [B + 1]
  pdl_wait();
  pdl_trigger();
  build_cs<kMetaThreads>(cu, B, T, cs);
  if (blockIdx.x == 0) flag(status, per_request(cu, past, cs, B, T, max_q, max_k, seqlens_q, seqlen_k));
  int bits = 0;
  for (int t = blockIdx.x * kMetaThreads + threadIdx.x; t < T; t += gridDim.x * kMetaThreads) {
    const TokenMeta m = token_meta(t, cs, B, past, block_table, MB, bs, num_blocks, bits);
    token_batch[t] = m.b;
    token_pos[t] = m.pos;
    slot_mapping[t] = m.slot;
  }
  flag(status, bits);
}

// Copy (or quantise) token t's K and V rows for all kv heads into `slot`, by one warp.
template <typename ActT, typename CacheT>
__device__ __forceinline__ void append_token_rows(const ActT* __restrict__ k_new,
                                                  const ActT* __restrict__ v_new,
                                                  CacheT* __restrict__ k_cache, CacheT* __restrict__ v_cache,
                                                  const float* __restrict__ k_scale,
                                                  const float* __restrict__ v_scale, int t, int slot,
                                                  int H_kv, int D, int lane, int first = 0) {
  const long long src_row = (long long)t * H_kv * D;
  const long long dst_row = (long long)slot * H_kv * D;
  if constexpr (sizeof(CacheT) != 1) {
    // exact copy, 16-byte vectors
    constexpr int EPV = 16 / sizeof(ActT);
    const int nvec = H_kv * D / EPV;
    const uint4* ks = reinterpret_cast<const uint4*>(k_new + src_row);
    const uint4* vs = reinterpret_cast<const uint4*>(v_new + src_row);
    uint4* kd = reinterpret_cast<uint4*>(k_cache + dst_row);
    uint4* vd = reinterpret_cast<uint4*>(v_cache + dst_row);
    for (int i = lane; i < nvec; i += 32) {
      kd[i] = ks[i];
      vd[i] = vs[i];
    }
  } else {
    // q8 = clamp(rint(x / scale), -128, 127) per channel, 16 channels per lane
    // step; items below `first` were done by the caller
    const int ngrp = H_kv * D / 16;
    for (int i = first + lane; i < 2 * ngrp; i += 32) {
      const bool isv = i >= ngrp;
      const int e0 = (isv ? i - ngrp : i) * 16;   // element offset within the token's H_kv*D row
      Group16<ActT> g;
      g.load((isv ? v_new : k_new) + src_row + e0);
      int8_t* dst = reinterpret_cast<int8_t*>(isv ? v_cache : k_cache) + dst_row + e0;
      *reinterpret_cast<uint4*>(dst) = quant_group16<ActT>(g.v, (isv ? v_scale : k_scale) + e0);
    }
  }
}

// 16-byte vectors (16-bit caches) or 16-channel groups (INT8 caches) of a
// token's K and V rows each lane loads before the metadata is known, so the
// copy does not wait for them; INT8 groups are quantised while the token's
// block-table entry is in flight
constexpr int kAppendPre = 2;

template <typename ActT, typename CacheT>
__global__ void __launch_bounds__(kMetaThreads)
prepare_append_kernel(const int32_t* __restrict__ cu, const int32_t* __restrict__ past,
                      const int32_t* __restrict__ block_table, int B, int T, int max_q, int max_k, int MB,
                      int bs, int num_blocks, int32_t* __restrict__ seqlens_q,
                      int32_t* __restrict__ seqlen_k, int32_t* __restrict__ token_batch,
                      int32_t* __restrict__ token_pos, int32_t* __restrict__ slot_mapping,
                      const ActT* __restrict__ k_new, const ActT* __restrict__ v_new,
                      CacheT* __restrict__ k_cache, CacheT* __restrict__ v_cache,
                      const float* __restrict__ k_scale, const float* __restrict__ v_scale, int H_kv,
                      int D, int32_t* __restrict__ status) {
  extern __shared__ int32_t cs[];  // [B + 1] cumulative lengths, then [B] past lengths
  int32_t* past_s = cs + B + 1;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int wpb = kMetaThreads / 32;
  const int t_first = blockIdx.x * wpb + (threadIdx.x >> 5);
  constexpr bool kCopy = sizeof(CacheT) != 1;
  constexpr int EPV = 16 / sizeof(ActT);
  const int nvec = H_kv * D / EPV;
  uint4 kpre[kAppendPre], vpre[kAppendPre];
  if constexpr (kCopy) {
    if (t_first < T) {
      const uint4* ks = reinterpret_cast<const uint4*>(k_new + (long long)t_first * H_kv * D);
      const uint4* vs = reinterpret_cast<const uint4*>(v_new + (long long)t_first * H_kv * D);
#pragma unroll
      for (int i = 0; i < kAppendPre; ++i) {
        const int v = lane + 32 * i;
        if (v < nvec) {
          kpre[i] = ks[v];
          vpre[i] = vs[v];
        }
      }
    }
  }
  const int ngrp = H_kv * D / 16;   // INT8: 16-channel groups of a K (or V) row
  Group16<ActT> gpre[kAppendPre];
  uint4 qpre[kAppendPre];
  if constexpr (!kCopy) {
    if (t_first < T) {
#pragma unroll
      for (int i = 0; i < kAppendPre; ++i) {
        const int it = lane + 32 * i;
        if (it < 2 * ngrp) {
          const bool isv = it >= ngrp;
          gpre[i].load((isv ? v_new : k_new) + (long long)t_first * H_kv * D + (isv ? it - ngrp : it) * 16);
        }
      }
    }
  }
  build_cs<kMetaThreads>(cu, B, T, cs, past, past_s);   // ends with a block barrier: past_s is visible too
  if (blockIdx.x == 0) flag(status, per_request(cu, past_s, cs, B, T, max_q, max_k, seqlens_q, seqlen_k));
  int bits = 0;
  for (int t = t_first; t < T; t += gridDim.x * wpb) {
    int tb = 0;  // every lane computes the same metadata; lane 0 reports and writes it
    const TokenLoad tl = token_meta_load(t, cs, B, past_s, block_table, MB, bs);
    if constexpr (!kCopy) {
      if (t == t_first) {
#pragma unroll
        for (int i = 0; i < kAppendPre; ++i) {
          const int it = lane + 32 * i;
          if (it < 2 * ngrp) {
            const bool isv = it >= ngrp;
            qpre[i] = quant_group16<ActT>(gpre[i].v, (isv ? v_scale : k_scale) + (isv ? it - ngrp : it) * 16);
          }
        }
      }
    }
    const TokenMeta m = token_meta_finish(tl, MB, bs, num_blocks, tb);
    if (lane == 0) {
      bits |= tb;
      token_batch[t] = m.b;
      token_pos[t] = m.pos;
      slot_mapping[t] = m.slot;
    }
    if (m.slot < 0) continue;
    if constexpr (kCopy) {
      if (t == t_first) {
        uint4* kd = reinterpret_cast<uint4*>(k_cache + (long long)m.slot * H_kv * D);
        uint4* vd = reinterpret_cast<uint4*>(v_cache + (long long)m.slot * H_kv * D);
#pragma unroll
        for (int i = 0; i < kAppendPre; ++i) {
          const int v = lane + 32 * i;
          if (v < nvec) {
            kd[v] = kpre[i];
            vd[v] = vpre[i];
          }
        }
        const uint4* ks = reinterpret_cast<const uint4*>(k_new + (long long)t * H_kv * D);
        const uint4* vs = reinterpret_cast<const uint4*>(v_new + (long long)t * H_kv * D);
        for (int v = lane + 32 * kAppendPre; v < nvec; v += 32) {
          kd[v] = ks[v];
          vd[v] = vs[v];
        }
        continue;
      }
    }
    if constexpr (!kCopy) {
      if (t == t_first) {
#pragma unroll
        for (int i = 0; i < kAppendPre; ++i) {
          const int it = lane + 32 * i;
          if (it < 2 * ngrp) {
            const bool isv = it >= ngrp;
            int8_t* dst = reinterpret_cast<int8_t*>(isv ? v_cache : k_cache) + (long long)m.slot * H_kv * D +
                          (isv ? it - ngrp : it) * 16;
            *reinterpret_cast<uint4*>(dst) = qpre[i];
          }
        }
        append_token_rows<ActT, CacheT>(k_new, v_new, k_cache, v_cache, k_scale, v_scale, t, m.slot, H_kv, D,
                                        lane, 32 * kAppendPre);
        continue;
      }
    }
    append_token_rows<ActT, CacheT>(k_new, v_new, k_cache, v_cache, k_scale, v_scale, t, m.slot, H_kv, D, lane);
  }
  flag(status, bits);
}

static size_t cs_smem(int B) { return sizeof(int32_t) * (size_t)(B + 1); }
static size_t cs_past_smem(int B) { return sizeof(int32_t) * (size_t)(2 * B + 1); }

template <typename K>
static void allow_smem(K kern, size_t smem) {
  if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

int launch_prepare_metadata(const int32_t* cu, const int32_t* past, const int32_t* block_table,
                            int B, int T, int max_q, int max_k, int MB, int bs, int num_blocks,
                            int32_t* seqlens_q, int32_t* seqlen_k, int32_t* token_batch,
                            int32_t* token_pos, int32_t* slot_mapping, int32_t* status,
                            cudaStream_t stream) {
  int grid = (T + kMetaThreads - 1) / kMetaThreads;
  if (grid < 1) grid = 1;
  if (grid > 148 * 8) grid = 148 * 8;
  const size_t smem = cs_smem(B);
  allow_smem(prepare_metadata_kernel, smem);
  return launch_pdl(prepare_metadata_kernel, dim3(grid), dim3(kMetaThreads), smem, stream, cu, past,
                    block_table, B, T, max_q, max_k, MB, bs, num_blocks, seqlens_q, seqlen_k, token_batch,
                    token_pos, slot_mapping, status);
}

template <typename ActT, typename CacheT>
static int launch_pa(const int32_t* cu, const int32_t* past, const int32_t* block_table, int B, int T,
                     int max_q, int max_k, int MB, int bs, int num_blocks, int32_t* seqlens_q,
                     int32_t* seqlen_k, int32_t* token_batch, int32_t* token_pos, int32_t* slot_mapping,
                     const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                     const float* k_scale, const float* v_scale, int H_kv, int D, int32_t* status,
                     cudaStream_t stream) {
  const int wpb = kMetaThreads / 32;
  int grid = (T + wpb - 1) / wpb;
  if (grid < 1) grid = 1;
  if (grid > 148 * 8) grid = 148 * 8;
  const size_t smem = cs_past_smem(B);
  auto kern = prepare_append_kernel<ActT, CacheT>;
  allow_smem(kern, smem);
  return launch_pdl(kern, dim3(grid), dim3(kMetaThreads), smem, stream, cu, past, block_table, B, T, max_q,
                    max_k, MB, bs, num_blocks, seqlens_q, seqlen_k, token_batch, token_pos, slot_mapping,
                    static_cast<const ActT*>(k_new), static_cast<const ActT*>(v_new),
                    static_cast<CacheT*>(k_cache), static_cast<CacheT*>(v_cache), k_scale, v_scale, H_kv, D,
                    status);
}

int launch_prepare_append(const int32_t* cu, const int32_t* past, const int32_t* block_table, int B, int T,
                          int max_q, int max_k, int MB, int bs, int num_blocks, int32_t* seqlens_q,
                          int32_t* seqlen_k, int32_t* token_batch, int32_t* token_pos,
                          int32_t* slot_mapping, const void* k_new, const void* v_new, int act,
                          void* k_cache, void* v_cache, int cache, const float* k_scale,
                          const float* v_scale, int H_kv, int D, int32_t* status, cudaStream_t stream) {
#define SPA_PA(A, C)                                                                                     \
  return launch_pa<A, C>(cu, past, block_table, B, T, max_q, max_k, MB, bs, num_blocks, seqlens_q,       \
                         seqlen_k, token_batch, token_pos, slot_mapping, k_new, v_new, k_cache, v_cache, \
                         k_scale, v_scale, H_kv, D, status, stream)
  if (cache == SPA_I8) {
    if (act == SPA_F32) SPA_PA(float, int8_t);
    if (act == SPA_F16) SPA_PA(__half, int8_t);
    SPA_PA(__nv_bfloat16, int8_t);
  }
  if (act == SPA_F32) SPA_PA(float, float);
  if (act == SPA_F16) SPA_PA(__half, __half);
  SPA_PA(__nv_bfloat16, __nv_bfloat16);
#undef SPA_PA
}

}  // namespace spa
