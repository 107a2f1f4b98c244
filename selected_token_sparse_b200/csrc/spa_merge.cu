// Merge of the partial states of a sequence split across devices.
//
// "[WebGPU] Add SparsePagedAttention", File summaries: the attention leaves
// partial FP32 softmax states that a finalize stage merges, applying the
// sink.  When one request's keys are spread over R devices, each device's
// spa_attention call (partial = 1, its kv_range) leaves o_r -- the softmax
// over its keys, without the sink -- and lse_r; after an all-gather this
// kernel forms, per (token, q head),
//   M = max(sink, max_r lse_r),  L = e^(sink - M) + sum_r e^(lse_r - M),
//   out = sum_r e^(lse_r - M) o_r / L,  lse = M + ln L
// (out = 0, lse = -inf when M = -inf), in log2 units on the device.
//
// One warp per (token, q head) row; a lane owns D / 32 adjacent columns and
// reads every shard's columns with vector loads, the shards' loads in flight
// together.  The work is a pass over R x rows x D fp32 values: HBM bound.
#include "spa_attn.cuh"

namespace spa {

int check_launch_public();

constexpr int kMergeThreads = 256;

template <typename ActT, int D>
__global__ void __launch_bounds__(kMergeThreads)
merge_partials_kernel(const float* __restrict__ part_out, const float* __restrict__ part_lse, int R, long long rows,
                      int H_q, const float* __restrict__ sinks, void* out, float* lse_out) {
  pdl_wait();
  pdl_trigger();
  constexpr int CPL = D / 32;   // columns per lane: 4 (D = 128) or 2 (D = 64)
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int h = (int)(row % H_q);
  const float sink2 = sinks ? sinks[h] * kLog2e : -INFINITY;
  float M = sink2;
  for (int r = 0; r < R; ++r) M = fmaxf(M, part_lse[r * rows + row] * kLog2e);
  float o[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) o[i] = 0.f;
  float L = 0.f, lse = -INFINITY;
  if (M != -INFINITY) {
    L = (sink2 == -INFINITY) ? 0.f : exp2f(sink2 - M);
    int r = 0;
    for (; r + 4 <= R; r += 4) {
      float w[4], v[4][CPL];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float l2 = part_lse[(r + u) * rows + row] * kLog2e;
        w[u] = (l2 == -INFINITY) ? 0.f : exp2f(l2 - M);
        const float* src = part_out + ((r + u) * rows + row) * D + lane * CPL;
        if constexpr (CPL == 4) {
          const float4 x = *reinterpret_cast<const float4*>(src);
          v[u][0] = x.x; v[u][1] = x.y; v[u][2] = x.z; v[u][3] = x.w;
        } else {
          const float2 x = *reinterpret_cast<const float2*>(src);
          v[u][0] = x.x; v[u][1] = x.y;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        L += w[u];
#pragma unroll
        for (int i = 0; i < CPL; ++i) o[i] = fmaf(w[u], v[u][i], o[i]);
      }
    }
    for (; r < R; ++r) {
      const float l2 = part_lse[r * rows + row] * kLog2e;
      const float w = (l2 == -INFINITY) ? 0.f : exp2f(l2 - M);
      const float* src = part_out + (r * rows + row) * D + lane * CPL;
      L += w;
#pragma unroll
      for (int i = 0; i < CPL; ++i) o[i] = fmaf(w, src[i], o[i]);
    }
    const float inv = 1.0f / L;
#pragma unroll
    for (int i = 0; i < CPL; ++i) o[i] *= inv;
    lse = (M + log2f(L)) * kLn2;
  }
  ActT* dst = static_cast<ActT*>(out) + row * D + lane * CPL;
#pragma unroll
  for (int i = 0; i < CPL; ++i) dst[i] = from_f32<ActT>(o[i]);
  if (lse_out && lane == 0) lse_out[row] = lse;
}

template <typename ActT>
static int launch_merge(const float* po, const float* pl, int R, long long rows, int H_q, int D, const float* sinks,
                        void* out, float* lse, cudaStream_t stream) {
  const dim3 grid((unsigned)((rows + kMergeThreads / 32 - 1) / (kMergeThreads / 32)));
  if (D == 128)
    return launch_pdl(merge_partials_kernel<ActT, 128>, grid, dim3(kMergeThreads), 0, stream, po, pl, R, rows, H_q,
                      sinks, out, lse);
  return launch_pdl(merge_partials_kernel<ActT, 64>, grid, dim3(kMergeThreads), 0, stream, po, pl, R, rows, H_q,
                    sinks, out, lse);
}

}  // namespace spa

using namespace spa;

extern "C" int spa_merge_partials(const float* part_out, const float* part_lse, int32_t R, int32_t T, int32_t H_q,
                                  int32_t D, const float* sinks, int32_t act, void* out, float* lse,
                                  spa_stream_t stream) {
  if (R <= 0 || T < 0 || H_q <= 0 || (D != 64 && D != 128)) return SPA_ERR_INVALID_ARG;
  if (act != SPA_F32 && act != SPA_F16 && act != SPA_BF16) return SPA_ERR_INVALID_ARG;
  if ((long long)T * H_q * D * R > (1LL << 40)) return SPA_ERR_INVALID_ARG;
  if (T == 0) return SPA_OK;
  if (!part_out || !part_lse || !out) return SPA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(part_out) & 15) return SPA_ERR_INVALID_ARG;
  const long long rows = (long long)T * H_q;
  const cudaStream_t st = (cudaStream_t)stream;
  int rc;
  if (act == SPA_F32) rc = launch_merge<float>(part_out, part_lse, R, rows, H_q, D, sinks, out, lse, st);
  else if (act == SPA_F16) rc = launch_merge<__half>(part_out, part_lse, R, rows, H_q, D, sinks, out, lse, st);
  else rc = launch_merge<__nv_bfloat16>(part_out, part_lse, R, rows, H_q, D, sinks, out, lse, st);
  if (rc != SPA_OK) return rc;
  return check_launch_public();
}
