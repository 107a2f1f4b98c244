// Step 2 -- KV append scatter.
//
// Writes the current tokens' K/V rows into the paged cache at slot_mapping[t]
// ("[WebGPU] Add SparsePagedAttention", File summaries: scatter current K/V
// into the cache using slot_mapping).  With an INT8 cache each element is
// quantised with its channel's scale (onnxruntime PR #33472, Key Changes:
// INT8 KV cache append with key_scale / value_scale):
//   q8 = clamp(rint(x / scale[h, d]), -128, 127), IEEE fp32 division, ties to even.
//
// Pure bandwidth: one thread moves one 16-byte chunk of the destination row,
// so loads and stores are 16-byte vectors and a warp covers whole rows.
#include "spa_attn.cuh"

namespace spa {

constexpr int kAppendThreads = 256;

// Float caches: exact copy of 16-byte chunks.
__global__ void __launch_bounds__(kAppendThreads)
append_copy_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                   uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                   const int32_t* __restrict__ slot_mapping, int T, int H_kv, int chunks_per_row,
                   long long num_slots, int32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  const long long per_tensor = (long long)T * H_kv * chunks_per_row;
  int bits = 0;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < 2 * per_tensor;
       i += (long long)gridDim.x * blockDim.x) {
    const bool is_v = i >= per_tensor;
    const long long j = is_v ? i - per_tensor : i;
    const int c = (int)(j % chunks_per_row);
    const long long row = j / chunks_per_row;  // t * H_kv + h
    const int t = (int)(row / H_kv);
    const int h = (int)(row % H_kv);
    const int slot = slot_mapping[t];
    if (slot < 0) continue;
    if ((long long)slot >= num_slots) {
      bits |= kStBadBlock;
      continue;
    }
    const long long dst = ((long long)slot * H_kv + h) * chunks_per_row + c;
    if (is_v) v_cache[dst] = v_new[j];
    else k_cache[dst] = k_new[j];
  }
  flag(status, bits);
}

template <typename ActT>
__device__ __forceinline__ float load_act(const ActT* p) { return to_f32(*p); }

// INT8 cache: each thread produces 16 consecutive int8 of one row.
template <typename ActT>
__global__ void __launch_bounds__(kAppendThreads)
append_int8_kernel(const ActT* __restrict__ k_new, const ActT* __restrict__ v_new,
                   int8_t* __restrict__ k_cache, int8_t* __restrict__ v_cache,
                   const float* __restrict__ k_scale, const float* __restrict__ v_scale,
                   const int32_t* __restrict__ slot_mapping, int T, int H_kv, int D,
                   long long num_slots, int32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  const int chunks_per_row = D / 16;
  const long long per_tensor = (long long)T * H_kv * chunks_per_row;
  int bits = 0;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < 2 * per_tensor;
       i += (long long)gridDim.x * blockDim.x) {
    const bool is_v = i >= per_tensor;
    const long long j = is_v ? i - per_tensor : i;
    const int c = (int)(j % chunks_per_row);
    const long long row = j / chunks_per_row;
    const int t = (int)(row / H_kv);
    const int h = (int)(row % H_kv);
    const int slot = slot_mapping[t];
    if (slot < 0) continue;
    if ((long long)slot >= num_slots) {
      bits |= kStBadBlock;
      continue;
    }
    const ActT* src = (is_v ? v_new : k_new) + row * D + c * 16;
    const float* sc = (is_v ? v_scale : k_scale) + (long long)h * D + c * 16;
    Group16<ActT> g;
    g.load(src);
    int8_t* dst = (is_v ? v_cache : k_cache) + ((long long)slot * H_kv + h) * D + c * 16;
    *reinterpret_cast<uint4*>(dst) = quant_group16<ActT>(g.v, sc);
  }
  flag(status, bits);
}

static int grid_for(long long work) {
  long long g = (work + kAppendThreads - 1) / kAppendThreads;
  if (g < 1) g = 1;
  if (g > 148 * 16) g = 148 * 16;
  return (int)g;
}

int launch_append_kv(const void* k_new, const void* v_new, int act, void* k_cache, void* v_cache,
                     int cache, const float* k_scale, const float* v_scale,
                     const int32_t* slot_mapping, int T, int H_kv, int D, int block_size,
                     int num_blocks, int32_t* status, cudaStream_t stream) {
  const long long num_slots = (long long)num_blocks * block_size;
  if (cache != SPA_I8) {
    const int elt = act == SPA_F32 ? 4 : 2;
    const int chunks = D * elt / 16;
    const long long work = 2LL * T * H_kv * chunks;
    return launch_pdl(append_copy_kernel, dim3(grid_for(work)), dim3(kAppendThreads), 0, stream,
                      (const uint4*)k_new, (const uint4*)v_new, (uint4*)k_cache, (uint4*)v_cache,
                      slot_mapping, T, H_kv, chunks, num_slots, status);
  }
  const long long work = 2LL * T * H_kv * (D / 16);
  const int g = grid_for(work);
  switch (act) {
    case SPA_F32:
      launch_pdl(append_int8_kernel<float>, dim3(g), dim3(kAppendThreads), 0, stream,
          (const float*)k_new, (const float*)v_new, (int8_t*)k_cache, (int8_t*)v_cache, k_scale,
          v_scale, slot_mapping, T, H_kv, D, num_slots, status);
      break;
    case SPA_F16:
      launch_pdl(append_int8_kernel<__half>, dim3(g), dim3(kAppendThreads), 0, stream,
          (const __half*)k_new, (const __half*)v_new, (int8_t*)k_cache, (int8_t*)v_cache, k_scale,
          v_scale, slot_mapping, T, H_kv, D, num_slots, status);
      break;
    default:
      launch_pdl(append_int8_kernel<__nv_bfloat16>, dim3(g), dim3(kAppendThreads), 0, stream,
          (const __nv_bfloat16*)k_new, (const __nv_bfloat16*)v_new, (int8_t*)k_cache,
          (int8_t*)v_cache, k_scale, v_scale, slot_mapping, T, H_kv, D, num_slots, status);
      break;
  }
  return 0;
}

}  // namespace spa
