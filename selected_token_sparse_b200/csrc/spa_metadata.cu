// Step 1 -- metadata prepare.
//
// Derives the exact per-request lengths and the per-token (request, position,
// slot) metadata on the device, so that no device-to-host copy is needed per
// layer ("[WebGPU] Add PagedAttention metadata and GPT-OSS support",
// Description and Changes; worked cases in review item T1).  The per-token
// request index is a binary search over the sanitised cumulative lengths,
// not a linear scan ("[WebGPU] Add SparsePagedAttention", review note on the
// O(batch_size) scan per token and on malformed cumulative lengths).
//
// One launch.  Every block rebuilds the sanitised cumulative lengths
//   cs[0] = 0,  cs[b] = min(max(cu[1..b], 0), T)
// (a clamped prefix maximum) in shared memory with a block-wide scan; block 0
// also writes the per-request outputs and status bits; every thread then
// handles tokens in a grid-stride loop.
#include "spa_common.cuh"

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
  __shared__ int32_t warp_max[kMetaThreads / 32];
  __shared__ int32_t chunk_carry[kMetaThreads];
  const int tid = threadIdx.x;
  const int n = B + 1;
  // contiguous chunk per thread: local prefix max, then a scan over chunk maxima
  const int per = (n + kMetaThreads - 1) / kMetaThreads;
  const int c0 = tid * per;
  const int c1 = min(c0 + per, n);
  int run = 0;  // cs[0] = 0 takes part in the maximum
  for (int i = c0; i < c1; ++i) {
    int v = (i == 0) ? 0 : cu[i];
    run = max(run, v);
    cs[i] = run;
  }
  // inclusive scan (max) of chunk maxima across the block
  int lane = tid & 31, warp = tid >> 5;
  int x = (c0 < c1) ? run : 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x = max(x, y);
  }
  if (lane == 31) warp_max[warp] = x;
  __syncthreads();
  int prev_warps = 0;
  for (int w = 0; w < warp; ++w) prev_warps = max(prev_warps, warp_max[w]);
  int incl = max(x, prev_warps);
  chunk_carry[tid] = incl;
  __syncthreads();
  int carry = (tid == 0) ? 0 : chunk_carry[tid - 1];
  for (int i = c0; i < c1; ++i) cs[i] = min(max(cs[i], carry), T);
  __syncthreads();

  if (blockIdx.x == 0) {
    int bits = 0;
    for (int b = tid; b <= B; b += kMetaThreads) {
      int raw = (b == 0) ? cu[0] : cu[b];
      if (raw != cs[b]) bits |= kStBadCu;
      if (b == B && cs[B] != T) bits |= kStBadCu;
    }
    for (int b = tid; b < B; b += kMetaThreads) {
      int p = past[b];
      if (p < 0) {
        bits |= kStBadCu;
        p = 0;
      }
      int q_len = cs[b + 1] - cs[b];
      long long total = (long long)p + q_len;
      seqlens_q[b] = q_len;
      seqlen_k[b] = (int32_t)(total - 1);
      if (q_len > max_q || total > (long long)max_k) bits |= kStBounds;
    }
    flag(status, bits);
  }

  int bits = 0;
  for (int t = blockIdx.x * kMetaThreads + tid; t < T; t += gridDim.x * kMetaThreads) {
    // owner = upper_bound(cs[0..B], t) - 1, valid iff t < cs[B]
    int lo = 0, hi = n;  // search in [lo, hi)
    while (lo < hi) {
      int mid = (lo + hi) >> 1;
      if (cs[mid] <= t) lo = mid + 1; else hi = mid;
    }
    int b = lo - 1;
    if (t >= cs[B] || b < 0 || b >= B) {
      token_batch[t] = -1;
      token_pos[t] = -1;
      slot_mapping[t] = -1;
      continue;
    }
    int p0 = max(past[b], 0);
    int pos = p0 + (t - cs[b]);
    token_batch[t] = b;
    token_pos[t] = pos;
    int lb = pos / bs;
    int slot = -1;
    if (lb >= MB) {
      bits |= kStCapacity;
    } else {
      int blk = block_table[(long long)b * MB + lb];
      if (blk < 0 || blk >= num_blocks) bits |= kStBadBlock;
      else slot = blk * bs + pos % bs;
    }
    slot_mapping[t] = slot;
  }
  flag(status, bits);
}

int launch_prepare_metadata(const int32_t* cu, const int32_t* past, const int32_t* block_table,
                            int B, int T, int max_q, int max_k, int MB, int bs, int num_blocks,
                            int32_t* seqlens_q, int32_t* seqlen_k, int32_t* token_batch,
                            int32_t* token_pos, int32_t* slot_mapping, int32_t* status,
                            cudaStream_t stream) {
  int grid = (T + kMetaThreads - 1) / kMetaThreads;
  if (grid < 1) grid = 1;
  if (grid > 148 * 8) grid = 148 * 8;
  size_t smem = sizeof(int32_t) * (size_t)(B + 1);
  if (smem > 48 * 1024) {
    cudaFuncSetAttribute(prepare_metadata_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
  }
  prepare_metadata_kernel<<<grid, kMetaThreads, smem, stream>>>(
      cu, past, block_table, B, T, max_q, max_k, MB, bs, num_blocks, seqlens_q, seqlen_k,
      token_batch, token_pos, slot_mapping, status);
  return 0;
}

}  // namespace spa
