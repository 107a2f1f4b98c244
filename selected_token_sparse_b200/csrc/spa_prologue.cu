// Steps 1 and 2 with the QKV prologue in between, in one launch: metadata,
// then for every (token, head) row of q, k and v the prologue, then q is
// written for the attention and k / v are appended to the paged cache.
//
// Prologue ("[WebGPU] Add DynamicSparseAttention", Description: QKV and cache
// -- packed and unpacked QKV; Position processing -- QK RMSNorm, partial and
// interleaved RoPE, rotary offsets and explicit position IDs; "[WebGPU] Add
// SparsePagedAttention", Description -- packed-QKV split and RoPE ahead of the
// block-table scatter):
//   x  = the row of head h of q or k (packed [T, H_q + 2 H_kv, D]: q heads,
//        then k heads, then v heads; or separate q / k / v tensors);
//   x <- x / sqrt(mean(x^2) + eps) * w                 (when w is given)
//   x <- RoPE(x, position)  on the first rotary_dim channels, pairs
//        (i, i + rotary_dim/2) or (2i, 2i+1): (a, b) -> (a c - b s, b c + a s),
//        c / s = cos_cache / sin_cache[position, i]   (when the caches are given)
//   position = position_ids[t], or the token's position + rotary_offset; a
//        position outside [0, max_pos) leaves the row unrotated (BOUNDS).
// q leaves rounded to the activation dtype; k and v are rounded to it and
// then appended exactly as spa_append_kv does (copy, or INT8 per-channel
// quantisation of the rounded value).  v has no prologue.
//
// One warp per (token, head) row: lane l holds channels [l E, l E + E),
// E = D / 32; the sum of squares is a warp reduction; a rotation reads its
// pair partner through a per-warp row in shared memory.
#include "spa_attn.cuh"
#include "spa_meta.cuh"

namespace spa {

constexpr int kProThreads = 256;


template <typename T>
__device__ __forceinline__ T from_f32_rn(float x) {
  return from_f32<T>(x);
}

template <typename ActT, typename CacheT, int E>
__global__ void __launch_bounds__(kProThreads, 1)
prepare_qkv_append_kernel(const QkvParams P) {
  extern __shared__ int32_t pro_smem[];   // cs [B + 1], past [B], then per-warp rows [8][D]
  int32_t* cs = pro_smem;
  int32_t* past_s = cs + P.B + 1;
  float* rows = reinterpret_cast<float*>(past_s + P.B + ((2 * P.B + 1) & 1));   // 8-byte aligned
  constexpr int D = E * 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* xrow = rows + warp * D;
  pdl_wait();
  pdl_trigger();
  const int NH = P.H_q + 2 * P.H_kv;
  const long long rows_total = (long long)P.T * NH;
  // source row (token t, head hh) of the packed or separate q / k / v
  auto row_src = [&](int t, int hh) -> const ActT* {
    if (P.qkv) return static_cast<const ActT*>(P.qkv) + ((long long)t * NH + hh) * D;
    const int kind = hh < P.H_q ? 0 : (hh < P.H_q + P.H_kv ? 1 : 2);
    const int h = kind == 0 ? hh : (kind == 1 ? hh - P.H_q : hh - P.H_q - P.H_kv);
    const void* base = kind == 0 ? P.q : (kind == 1 ? P.k : P.v);
    return static_cast<const ActT*>(base) + ((long long)t * (kind == 0 ? P.H_q : P.H_kv) + h) * D;
  };
  // Issued first: the lengths every warp scans by itself (B + 1 <= 64:
  // build_cs_warp, no block barrier that would wait for the loads in flight)
  const bool warp_scan = P.B + 1 <= 64;
  int pc0 = 0, pc1 = 0, pp0 = 0, pp1 = 0;
  if (warp_scan) {
    pc0 = (lane >= 1 && lane <= P.B) ? ld_early(P.cu + lane) : 0;
    pc1 = lane + 32 <= P.B ? ld_early(P.cu + lane + 32) : 0;
    pp0 = lane < P.B ? ld_early(P.past + lane) : 0;
    pp1 = lane + 32 < P.B ? ld_early(P.past + lane + 32) : 0;
  }
  // the warp's first row, its norm weights and (with explicit position ids)
  // its rotary rows are loaded before the metadata is known
  const long long r0 = (long long)blockIdx.x * (kProThreads / 32) + warp;
  const bool rope = P.cos_cache != nullptr && P.rotary_dim > 0;
  const int rd = P.rotary_dim, half = rd / 2;
  ActT x0[E];
  float w0[E], c0[E], s0[E];
  int pos0 = -1;
  if (r0 < rows_total) {
    const int t0 = (int)(r0 / NH), hh0 = (int)(r0 % NH);
    const ActT* src = row_src(t0, hh0);
#pragma unroll
    for (int e = 0; e < E; ++e) x0[e] = src[lane * E + e];
    const int kind0 = hh0 < P.H_q ? 0 : (hh0 < P.H_q + P.H_kv ? 1 : 2);
    const float* w = kind0 == 0 ? P.q_norm : (kind0 == 1 ? P.k_norm : nullptr);
#pragma unroll
    for (int e = 0; e < E; ++e) w0[e] = w != nullptr ? ld_early(w + lane * E + e) : 0.f;
    if (rope && kind0 != 2 && P.position_ids != nullptr) {
      pos0 = ld_early(P.position_ids + t0);
      if (pos0 >= 0 && pos0 < P.max_pos) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int d = lane * E + e;
          const int i = d >= rd ? 0 : (P.interleaved ? d >> 1 : (d < half ? d : d - half));
          c0[e] = ld_early(P.cos_cache + (long long)pos0 * half + i);
          s0[e] = ld_early(P.sin_cache + (long long)pos0 * half + i);
        }
      }
    }
  }
  if (warp_scan) build_cs_warp(P.B, P.T, cs, past_s, pc0, pc1, pp0, pp1);
  else build_cs<kProThreads>(P.cu, P.B, P.T, cs, P.past, past_s);   // ends with a block barrier
  int bits = 0;
  if (blockIdx.x == 0)
    bits |= per_request(P.cu, past_s, cs, P.B, P.T, P.max_q, P.max_k, P.seqlens_q, P.seqlen_k);
  for (long long r = r0; r < rows_total; r += (long long)gridDim.x * (kProThreads / 32)) {
    const int t = (int)(r / NH), hh = (int)(r % NH);
    const TokenLoad l = token_meta_load(t, cs, P.B, past_s, P.block_table, P.MB, P.bs);
    float x[E];   // the row, read before this iteration's metadata stores
    if (r == r0) {
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = to_f32(x0[e]);
    } else {
      const ActT* src = row_src(t, hh);
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = to_f32(src[lane * E + e]);
    }
    const int kind = hh < P.H_q ? 0 : (hh < P.H_q + P.H_kv ? 1 : 2);   // q, k, v
    const int h = kind == 0 ? hh : (kind == 1 ? hh - P.H_q : hh - P.H_q - P.H_kv);
    // the rotary position and its cos / sin entries, loaded while the
    // block-table entry is in flight (l.pos is -1 for a token no request owns)
    const bool pre = r == r0 && P.position_ids != nullptr;   // loaded up front
    const int pos = !rope || kind == 2 ? -1
                    : (pre ? pos0 : (P.position_ids ? P.position_ids[t] : l.pos + P.rotary_offset));
    const bool rot = rope && kind != 2 && pos >= 0 && pos < P.max_pos;
    const float* w = kind == 0 ? P.q_norm : (kind == 1 ? P.k_norm : nullptr);
    float wv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) wv[e] = r == r0 ? w0[e] : (w != nullptr ? ld_early(w + lane * E + e) : 0.f);
    float cv[E], sv[E];
    if (rot) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int d = lane * E + e;
        const int i = d >= rd ? 0 : (P.interleaved ? d >> 1 : (d < half ? d : d - half));
        cv[e] = pre ? c0[e] : ld_early(P.cos_cache + (long long)pos * half + i);
        sv[e] = pre ? s0[e] : ld_early(P.sin_cache + (long long)pos * half + i);
      }
    }
    int tb = 0;
    const TokenMeta m = token_meta_finish(l, P.MB, P.bs, P.NB, tb);
    if (hh == 0 && lane == 0) {
      bits |= tb;
      P.token_batch[t] = m.b;
      P.token_pos[t] = m.pos;
      P.slot_mapping[t] = m.slot;
    }
    if (kind != 0 && m.slot < 0) continue;   // nothing to append
    if (kind != 2) {
      if (w != nullptr) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = 1.0f / sqrtf(ss / (float)D + P.eps);
#pragma unroll
        for (int e = 0; e < E; ++e) x[e] = x[e] * inv * wv[e];
      }
      if (rope) {
        if (rot) {
#pragma unroll
          for (int e = 0; e < E; ++e) xrow[lane * E + e] = x[e];
          __syncwarp();
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const int d = lane * E + e;
            if (d >= rd) continue;
            int partner;
            bool first;
            if (P.interleaved) {
              first = (d & 1) == 0;
              partner = d ^ 1;
            } else {
              first = d < half;
              partner = first ? d + half : d - half;
            }
            const float y = xrow[partner];
            x[e] = first ? (x[e] * cv[e] - y * sv[e]) : (x[e] * cv[e] + y * sv[e]);
          }
          __syncwarp();
        } else {
          bits |= kStBounds;
        }
      }
    }
    if (kind == 0) {
      ActT* dst = static_cast<ActT*>(P.q_out) + ((long long)t * P.H_q + h) * D;
#pragma unroll
      for (int e = 0; e < E; ++e) dst[lane * E + e] = from_f32_rn<ActT>(x[e]);
      continue;
    }
    // append: the value rounded to the activation dtype, copied or quantised
    const long long drow = ((long long)m.slot * P.H_kv + h) * D;
    if constexpr (sizeof(CacheT) != 1) {
      CacheT* dst = static_cast<CacheT*>(kind == 1 ? P.k_cache : P.v_cache) + drow;
#pragma unroll
      for (int e = 0; e < E; ++e) dst[lane * E + e] = from_f32_rn<CacheT>(x[e]);
    } else {
      const float* sc = (kind == 1 ? P.k_scale : P.v_scale) + (long long)h * D;
      int8_t* dst = static_cast<int8_t*>(kind == 1 ? P.k_cache : P.v_cache) + drow;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float xr = to_f32(from_f32_rn<ActT>(x[e]));
        float q8 = rintf(__fdiv_rn(xr, sc[lane * E + e]));
        q8 = fminf(fmaxf(q8, -128.0f), 127.0f);
        dst[lane * E + e] = static_cast<int8_t>(static_cast<int>(q8));
      }
    }
  }
  flag(P.status, bits);
}

size_t prologue_smem_bytes(int B, int D) {
  return sizeof(int32_t) * (size_t)(2 * B + 2) + sizeof(float) * (size_t)(kProThreads / 32) * D;
}

template <typename ActT, typename CacheT>
static int launch_pro_t(const QkvParams& P, cudaStream_t stream) {
  const int NH = P.H_q + 2 * P.H_kv;
  const long long rows = (long long)P.T * NH;
  long long grid = (rows + (kProThreads / 32) - 1) / (kProThreads / 32);
  if (grid < 1) grid = 1;
  if (grid > 148 * 16) grid = 148 * 16;
  const size_t smem = prologue_smem_bytes(P.B, P.D);
  if (P.D == 64) {
    auto kern = prepare_qkv_append_kernel<ActT, CacheT, 2>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch_pdl(kern, dim3((unsigned)grid), dim3(kProThreads), smem, stream, P);
  }
  auto kern = prepare_qkv_append_kernel<ActT, CacheT, 4>;
  if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kProThreads), smem, stream, P);
}

int launch_prepare_qkv_append(const QkvParams& P, int act, int cache, cudaStream_t stream) {
  if (cache == SPA_I8) {
    if (act == SPA_F32) return launch_pro_t<float, int8_t>(P, stream);
    if (act == SPA_F16) return launch_pro_t<__half, int8_t>(P, stream);
    return launch_pro_t<__nv_bfloat16, int8_t>(P, stream);
  }
  if (act == SPA_F32) return launch_pro_t<float, float>(P, stream);
  if (act == SPA_F16) return launch_pro_t<__half, __half>(P, stream);
  return launch_pro_t<__nv_bfloat16, __nv_bfloat16>(P, stream);
}

}  // namespace spa
