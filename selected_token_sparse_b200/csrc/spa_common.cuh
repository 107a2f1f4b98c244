// Shared device helpers of libspa (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "spa.h"

namespace spa {

constexpr int kStBadCu = SPA_ST_BAD_CU;
constexpr int kStCapacity = SPA_ST_CAPACITY;
constexpr int kStBadBlock = SPA_ST_BAD_BLOCK;
constexpr int kStBounds = SPA_ST_BOUNDS;
constexpr int kStBadIdx = SPA_ST_BAD_IDX;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ void flag(int32_t* status, int bits) {
  if (status != nullptr && bits != 0) atomicOr(status, bits);
}

// Exact conversions of one encoded element to fp32.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// INT8 K/V quantisation of one group of 16 channels: q8 = clamp(rint(x / scale),
// -128, 127) with an IEEE fp32 division, the 16 bytes packed in channel order.
// `x` holds the group's values as they were loaded (16-byte vectors).
template <typename ActT>
__device__ __forceinline__ uint4 quant_group16(const uint4* x, const float* __restrict__ sc) {
  const ActT* v = reinterpret_cast<const ActT*>(x);
  alignas(16) int8_t q[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    float r = rintf(__fdiv_rn(to_f32(v[e]), sc[e]));
    r = fminf(fmaxf(r, -128.0f), 127.0f);
    q[e] = static_cast<int8_t>(static_cast<int>(r));
  }
  return *reinterpret_cast<const uint4*>(q);
}
// The 16-byte vectors of a group of 16 values (16-byte aligned).
template <typename ActT>
struct Group16 {
  static constexpr int NV = 16 * (int)sizeof(ActT) / 16;
  uint4 v[NV];
  __device__ __forceinline__ void load(const ActT* src) {
#pragma unroll
    for (int i = 0; i < NV; ++i) v[i] = reinterpret_cast<const uint4*>(src)[i];
  }
};
__device__ __forceinline__ float to_f32(int8_t x) { return static_cast<float>(x); }

// Round-to-nearest-even conversion of an fp32 value to the output encoding.
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// cp.async: 16-byte global -> shared copy, zero-filled when src_bytes == 0.
// Residual of a 16-bit pair: given x, y and their rounding to T packed in `hi`
// (x in the low half), the pair (x - T(x), y - T(y)) rounded to T.  A product
// P V with 16-bit P is run as P_hi V + P_lo V where P's own rounding would
// show in the output -- bf16 P (8 bits: a row dominated by one key carries
// that key's 2^-9 rounding), and fp16 P against integer-valued INT8 V (values
// up to 127 before the scale) -- so that P keeps about twice its bits.
template <typename T> __device__ __forceinline__ uint32_t residual_pair(float x, float y, uint32_t hi);
template <> __device__ __forceinline__ uint32_t residual_pair<__nv_bfloat16>(float x, float y, uint32_t hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(x - __uint_as_float(hi << 16), y - __uint_as_float(hi & 0xffff0000u));
  return *reinterpret_cast<uint32_t*>(&v);
}
template <> __device__ __forceinline__ uint32_t residual_pair<__half>(float x, float y, uint32_t hi) {
  const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&hi));
  __half2 v = __floats2half2_rn(x - h.x, y - h.y);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void cp_async_16(void* smem, const void* gmem, bool valid) {
  uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  int src_bytes = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Global loads issued where they are written: volatile asm keeps the
// compiler from sinking a read-only load to its first use, so a value needed
// late can be in flight from early on.
__device__ __forceinline__ int ld_early(const int32_t* p) {
  int v;
  asm volatile("ld.global.b32 %0, [%1];\n" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ float ld_early(const float* p) {
  float v;
  asm volatile("ld.global.f32 %0, [%1];\n" : "=f"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ld_early(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// ---- named barriers (id 0 is __syncthreads): a sync of `n` threads, and the
// OR / AND of a predicate over them
__device__ __forceinline__ void bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool bar_red_or(bool x, int id, int n) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.or.pred po, %2, %3, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)x), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool bar_red_and(bool x, int id, int n) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.and.pred po, %2, %3, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)x), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// ---- thread-block clusters: rank and barrier
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster; its memory writes before it
// (shared and global: release / acquire at cluster scope) are visible to every
// thread of the cluster after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while its predecessor in the stream is still running; it must execute
// griddepcontrol.wait before touching memory that predecessor writes.
template <typename... KArgs, typename... Args>
static int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  return 0;
}

// launch_pdl with the grid's y dimension in clusters of `cluster_y` CTAs.
template <typename... KArgs, typename... Args>
static int launch_pdl_cluster_y(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                cudaStream_t stream, int cluster_y, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = cluster_y;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  return 0;
}

}  // namespace spa
