// Steps 3-5 for long causal query runs (prefill / chunked prefill) on the
// fifth-generation tensor cores (tcgen05, TMEM accumulators, TMA).
//
// The dense QK^T and PV tiles of a causal (optionally windowed) prefill are
// real contractions, so they run as 128x128xD tcgen05.mma tiles:
//
//   CTA  = one q head x one 128-row q tile of one request; launched longest
//          tiles first (q tiles in reverse order) so the ragged tail balances.
//   TMA  = Q tile (3-D map over [T, H_q, D]) once; per 128-key step a K and a V
//          tile gathered from the paged cache with a 4-D map over
//          [num_blocks, block_size, H_kv, D] whose block coordinate comes from
//          the block table (one box per cache block; an unmapped block is
//          loaded from an out-of-range coordinate, i.e. zeros, and masked).
//          128-byte swizzle, no multicast.
//   MMA  = one elected thread: S = Q K^T (SS form, fp32 in TMEM columns
//          [0,128)), then O += P V (TS form: P read from TMEM, V MN-major).
//   softmax = 128 threads, thread i owns row i (TMEM lane i): masks the
//          causal / window / unmapped keys, keeps a running max in log2
//          units that is only raised (and O, l rescaled) when a tile's max
//          exceeds it by more than 8, so P <= 2^8 fits fp16 / bf16 and most
//          tiles skip the O rescale; P overwrites S in TMEM as packed pairs.
//   sink = folded into the final normalisation (denominator only).
//
// The key loop starts at the earliest window tile, rounded down to the tile
// size, and keeps per-row visibility checks ("[WebGPU] Add PagedAttention
// metadata and GPT-OSS support", review item Q3); the sink semantics follow
// the same page's Description and "[WebGPU] Add DynamicSparseAttention"
// (joint FP32 stable softmax with optional sink).
//
// Every mbarrier wait is bounded; on expiry the kernel sets SPA_ST_TIMEOUT,
// drains what it issued (again bounded), frees its TMEM and returns.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "spa_attn.cuh"
#include "spa_sm100.cuh"

namespace spa {

using namespace sm100;

constexpr int kPfBM = 128;   // q rows per CTA (TMEM lanes)
constexpr int kPfBN = 128;   // keys per step
constexpr uint32_t kPfTmemCols = 256;
constexpr uint32_t kPfWaitLimit = 1u << 20;   // polls before a wait is declared lost

template <int D>
struct PfCfg {
  static constexpr int NCH = D / 64;                  // 128-byte chunks along D
  static constexpr int CHUNK = 128 * 128;             // one chunk of a 128-row tile (bytes)
  static constexpr int TILE = NCH * CHUNK;            // Q, K or V tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_BAR = OFF_V + TILE;        // 5 mbarriers
  static constexpr int OFF_TMEM = OFF_BAR + 64;       // TMEM base address holder
  static constexpr int OFF_MASK = OFF_TMEM + 16;      // box validity per tile (2 slots)
  static constexpr int OFF_FLAG = OFF_MASK + 16;      // abort flag
  static constexpr int BYTES = OFF_FLAG + 16;
  // + alignment slack; at least 80 KB so that no more than two CTAs (2 x 256
  // TMEM columns) are ever resident on one SM
  static constexpr int SMEM = (BYTES + 1024 > 80 * 1024) ? BYTES + 1024 : 80 * 1024;
  static constexpr uint32_t TX_TILE = (uint32_t)TILE;
};

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }

template <typename T>
__device__ __forceinline__ uint32_t pack_pair(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pack_pair<__half>(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <>
__device__ __forceinline__ uint32_t pack_pair<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct PfGeom {
  int b, h, h_kv, t_begin, q0, rows, past, L, k_lo, k_hi, ntiles;
};

// Block id of the cache block holding key `key` (or -1), with status bits for
// keys that must exist (key < k_hi).
__device__ __forceinline__ int pf_block(const AttnParams& p, int b, int key, bool needed, int& bits) {
  const int lb = key / p.bs;
  if (lb >= p.MB) {
    if (needed) bits |= kStCapacity;
    return -1;
  }
  const int blk = p.block_table[(long long)b * p.MB + lb];
  if (blk < 0 || blk >= p.NB) {
    if (needed) bits |= kStBadBlock;
    return -1;
  }
  return blk;
}

// Issue the TMA loads of one K or V tile (keys [kb, kb + 128)); returns the
// validity mask of its boxes (bit i: box i maps to a cache block).
__device__ __forceinline__ uint32_t pf_issue_kv(const AttnParams& p, const PfGeom& g,
                                                const CUtensorMap* map, unsigned char* dst,
                                                uint64_t* bar, int kb, int box_rows, int nch,
                                                int& bits, uint32_t tx) {
  mbar_arrive_expect_tx(bar, tx);
  uint32_t mask = 0;
  const int nbox = kPfBN / box_rows;
  for (int i = 0; i < nbox; ++i) {
    const int key0 = kb + i * box_rows;
    const int blk = pf_block(p, g.b, key0, key0 < g.k_hi, bits);
    if (blk >= 0) mask |= 1u << i;
    const int cblk = blk >= 0 ? blk : p.NB;  // out of range: the box reads zeros
    const int row = key0 % p.bs;
    for (int c = 0; c < nch; ++c)
      tma_load_4d(dst + c * (128 * 128) + i * box_rows * 128, map, bar, c * 64, g.h_kv, row, cblk);
  }
  return mask;
}

template <typename T, int D>
__global__ void __launch_bounds__(128, 1)
prefill_tcgen05_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       int n_qt, int box_rows, int max_tiles) {
  using C = PfCfg<D>;
  constexpr uint32_t FMT = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t IDESC_S = idesc_f16(FMT, kPfBM, kPfBN, 0);
  constexpr uint32_t IDESC_O = idesc_f16(FMT, kPfBM, D, 1);
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  pdl_wait();
  pdl_trigger();

  // ---- geometry (uniform across the CTA)
  PfGeom g;
  g.h = blockIdx.x;
  g.b = blockIdx.z;
  const int qt = n_qt - 1 - (int)blockIdx.y;
  g.t_begin = clampi(p.cu[g.b], 0, p.T);
  const int q_len = clampi(p.seqlens_q[g.b], 0, p.T - g.t_begin);
  g.q0 = qt * kPfBM;
  if (g.q0 >= q_len) return;
  g.rows = min(kPfBM, q_len - g.q0);
  g.L = max(p.seqlen_k[g.b] + 1, 0);
  g.past = max(g.L - q_len, 0);
  g.h_kv = g.h / p.G;
  const int p_first = g.past + g.q0;
  const int p_last = p_first + g.rows - 1;
  g.k_lo = p.window > 0 ? max(0, p_first - p.window + 1) : 0;
  g.k_lo = (g.k_lo / kPfBN) * kPfBN;
  g.k_hi = min(p_last + 1, g.L);
  g.ntiles = g.k_hi > g.k_lo ? (g.k_hi - g.k_lo + kPfBN - 1) / kPfBN : 0;
  g.ntiles = min(g.ntiles, max_tiles);

  unsigned char* sQ = smem + C::OFF_Q;
  unsigned char* sK = smem + C::OFF_K;
  unsigned char* sV = smem + C::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_k = bars + 1;
  uint64_t* bar_v = bars + 2;
  uint64_t* bar_s = bars + 3;
  uint64_t* bar_o = bars + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  volatile uint32_t* kmask = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MASK);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);

  int bits = 0;
  if (tid == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(bars + i, 1);
    fence_mbar_init();
    *abort_flag = 0;
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, kPfTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tmem_S = tmem;         // S (fp32, 128 cols); P (packed, 64 cols) overlays it
  const uint32_t tmem_O = tmem + 128;   // O (fp32, D cols)
  const uint32_t lane_off = (uint32_t)(32 * warp) << 16;

  // outstanding async work issued by thread 0 (for the drain on abort)
  int pend_q = 0, pend_k = 0, pend_v = 0, pend_s = 0, pend_o = 0;
  uint32_t ph_k = 0, ph_v = 0, ph_o = 0;

  if (tid == 0 && g.ntiles > 0) {
    mbar_arrive_expect_tx(bar_q, C::TX_TILE);
    for (int c = 0; c < C::NCH; ++c)
      tma_load_3d(sQ + c * C::CHUNK, &tm_q, bar_q, c * 64, g.h, g.t_begin + g.q0);
    pend_q = 1;
    kmask[0] = pf_issue_kv(p, g, &tm_k, sK, bar_k, g.k_lo, box_rows, C::NCH, bits, C::TX_TILE);
    pend_k = 1;
    pf_issue_kv(p, g, &tm_v, sV, bar_v, g.k_lo, box_rows, C::NCH, bits, C::TX_TILE);
    pend_v = 1;
  }
  __syncthreads();

  // softmax state of row `tid`
  const int prow = g.past + g.q0 + tid;
  float m_used = -INFINITY;   // log2 units
  float l_sum = 0.f;
  const float sl2 = p.scale_log2;

  for (int j = 0; j < g.ntiles; ++j) {
    const int kb = g.k_lo + j * kPfBN;
    // ---- producer / MMA thread: V_j, then S_j = Q K_j^T
    if (tid == 0) {
      bool ok = true;
      if (j > 0) {
        ok = mbar_wait(bar_o, ph_o, kPfWaitLimit);   // PV_{j-1} done: V buffer and P free
        if (ok) {
          ph_o ^= 1;
          pend_o = 0;
          pf_issue_kv(p, g, &tm_v, sV, bar_v, kb, box_rows, C::NCH, bits, C::TX_TILE);
          pend_v = 1;
        }
      }
      if (ok && j == 0) {
        ok = mbar_wait(bar_q, 0, kPfWaitLimit);
        if (ok) pend_q = 0;
      }
      if (ok) ok = mbar_wait(bar_k, ph_k, kPfWaitLimit);
      if (ok) {
        ph_k ^= 1;
        pend_k = 0;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk / 4, koff = (kk % 4) * 32;
          const uint64_t ad = smem_desc_sw128(smem_u32(sQ + c * C::CHUNK + koff), 16, 1024);
          const uint64_t bd = smem_desc_sw128(smem_u32(sK + c * C::CHUNK + koff), 16, 1024);
          mma_ss(tmem_S, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar_s);
        pend_s = 1;
      } else {
        *abort_flag = 1;
      }
    }
    // ---- everyone: wait for S_j (the decision to go on is CTA-uniform)
    const bool got_s = mbar_wait(bar_s, j & 1, kPfWaitLimit, abort_flag);
    if (__syncthreads_or(!got_s || *abort_flag)) {
      if (tid == 0) *abort_flag = 1;
      break;
    }
    if (tid == 0) {
      pend_s = 0;
      // K buffer is free: prefetch K_{j+1}
      if (j + 1 < g.ntiles) {
        kmask[(j + 1) & 1] = pf_issue_kv(p, g, &tm_k, sK, bar_k, kb + kPfBN, box_rows, C::NCH, bits,
                                         C::TX_TILE);
        pend_k = 1;
      }
    }
    tc_fence_after();
    {
      const uint32_t vmask = kmask[j & 1];
      uint32_t s[kPfBN];
#pragma unroll
      for (int c = 0; c < kPfBN / 32; ++c) tmem_ld32(tmem_S + lane_off + c * 32, s + c * 32);
      tmem_wait_ld();
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kPfBN; ++c) {
        const int key = kb + c;
        const bool vis = key < g.k_hi && key <= prow && (p.window <= 0 || key > prow - p.window) &&
                         ((vmask >> (c / box_rows)) & 1u);
        const float v = vis ? u2f(s[c]) * sl2 : -INFINITY;
        s[c] = __float_as_uint(v);
        mx = fmaxf(mx, v);
      }
      // lazy rescale: raise the reference max only when it grows by > 8 (x256).
      // The TMEM loads / stores of O are warp-collective, so the whole warp
      // takes the branch when any of its rows needs it (alpha = 1 otherwise).
      const bool need = mx > m_used + 8.0f;
      const float m_new = need ? mx : m_used;
      const float alpha = need ? ((m_used == -INFINITY) ? 0.f : exp2f(m_used - m_new)) : 1.f;
      if (j > 0 && __any_sync(0xffffffffu, need && m_used != -INFINITY)) {
        uint32_t o[32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          tmem_ld32(tmem_O + lane_off + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(u2f(o[e]) * alpha);
          tmem_st32(tmem_O + lane_off + c * 32, o);
        }
      }
      l_sum *= alpha;
      m_used = m_new;
      uint32_t pk[kPfBN / 2];
      float ls = 0.f;
#pragma unroll
      for (int c = 0; c < kPfBN; c += 2) {
        const float a = u2f(s[c]), bb = u2f(s[c + 1]);
        const float pa = (a == -INFINITY) ? 0.f : exp2f(a - m_used);
        const float pb = (bb == -INFINITY) ? 0.f : exp2f(bb - m_used);
        ls += pa + pb;
        pk[c / 2] = pack_pair<T>(pa, pb);
      }
      l_sum += ls;
#pragma unroll
      for (int c = 0; c < kPfBN / 64; ++c) tmem_st32(tmem_S + lane_off + c * 32, pk + c * 32);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    // ---- MMA thread: O += P V_j
    if (tid == 0) {
      tc_fence_after();
      if (mbar_wait(bar_v, ph_v, kPfWaitLimit)) {
        ph_v ^= 1;
        pend_v = 0;
#pragma unroll
        for (int kk = 0; kk < kPfBN / 16; ++kk) {
          const uint64_t bd = smem_desc_sw128(smem_u32(sV + kk * 2048), C::CHUNK, 1024);
          mma_ts(tmem_O, tmem_S + kk * 8, bd, IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar_o);
        pend_o = 1;
      } else {
        *abort_flag = 1;
      }
    }
    __syncthreads();
    if (*abort_flag) break;
  }

  // ---- epilogue: wait for the last PV, normalise with the sink, store
  __syncthreads();
  bool have_o = g.ntiles > 0 && !*abort_flag;
  if (have_o) {
    const bool got = mbar_wait(bar_o, (g.ntiles - 1) & 1, kPfWaitLimit, abort_flag);
    if (__syncthreads_or(!got)) {
      if (tid == 0) *abort_flag = 1;
    } else if (tid == 0) {
      pend_o = 0;
    }
  }
  __syncthreads();
  have_o = have_o && !*abort_flag;
  if (*abort_flag) {
    bits |= SPA_ST_TIMEOUT;
    if (tid == 0) {   // drain whatever is still in flight, bounded
      if (pend_q) mbar_wait(bar_q, 0, kPfWaitLimit);
      if (pend_k) mbar_wait(bar_k, ph_k, kPfWaitLimit);
      if (pend_v) mbar_wait(bar_v, ph_v, kPfWaitLimit);
      if (pend_s || pend_o) mbar_wait(bar_o, ph_o, kPfWaitLimit);
    }
  } else {
    const bool mine = tid < g.rows;
    const int t = g.t_begin + g.q0 + tid;
    const long long orow = (long long)t * p.H_q + g.h;
    const float sink2 = p.sinks ? p.sinks[g.h] * kLog2e : -INFINITY;
    float a, inv_l, lse;
    finalize_row(m_used, l_sum, sink2, a, inv_l, lse);
    const float f = a * inv_l;
    T* out = static_cast<T*>(p.out) + orow * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (have_o) {   // CTA-uniform: every thread takes part in the warp-wide load
        tmem_ld32(tmem_O + lane_off + c * 32, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (mine) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 v;
          v.x = pack_pair<T>(u2f(o[e + 0]) * f, u2f(o[e + 1]) * f);
          v.y = pack_pair<T>(u2f(o[e + 2]) * f, u2f(o[e + 3]) * f);
          v.z = pack_pair<T>(u2f(o[e + 4]) * f, u2f(o[e + 5]) * f);
          v.w = pack_pair<T>(u2f(o[e + 6]) * f, u2f(o[e + 7]) * f);
          *reinterpret_cast<uint4*>(out + c * 32 + e) = v;
        }
      }
    }
    if (mine && p.lse) p.lse[orow] = lse;
  }
  flag(p.status, bits);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kPfTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

int prefill_supported(const spa_attention_args_t* a) {
  if (a->act != SPA_F16 && a->act != SPA_BF16) return 0;
  if (a->cache != a->act) return 0;
  if (a->D != 64 && a->D != 128) return 0;
  if (a->selected_idx) return 0;
  const int G = a->H_q / a->H_kv;
  if (!(a->max_seqlen_q >= 64 || (long long)a->max_seqlen_q * G > 128)) return 0;
  const int bs = a->block_size;
  if (bs < 16 || (bs & (bs - 1)) != 0) return 0;
  if ((reinterpret_cast<uintptr_t>(a->q) | reinterpret_cast<uintptr_t>(a->k_cache) |
       reinterpret_cast<uintptr_t>(a->v_cache)) & 15)
    return 0;
  if (a->B > 65535 || a->H_q > 65535) return 0;
  return encode_fn() != nullptr;
}

static int encode(CUtensorMap* m, CUtensorMapDataType dt, cuuint32_t rank, const void* base,
                  const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode_fn()(m, dt, rank, const_cast<void*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SPA_OK : SPA_ERR_INVALID_ARG;
}

template <typename T, int D>
static int launch_pf(const AttnParams& p, CUtensorMapDataType dt, cudaStream_t stream) {
  using C = PfCfg<D>;
  const int box_rows = p.bs < kPfBN ? p.bs : kPfBN;
  CUtensorMap tq, tk, tv;
  const cuuint64_t qd[3] = {(cuuint64_t)D, (cuuint64_t)p.H_q, (cuuint64_t)p.T};
  const cuuint64_t qs[2] = {(cuuint64_t)D * 2, (cuuint64_t)p.H_q * D * 2};
  const cuuint32_t qb[3] = {64, 1, (cuuint32_t)kPfBM};
  const cuuint64_t kd[4] = {(cuuint64_t)D, (cuuint64_t)p.H_kv, (cuuint64_t)p.bs, (cuuint64_t)p.NB};
  const cuuint64_t ks[3] = {(cuuint64_t)D * 2, (cuuint64_t)p.H_kv * D * 2,
                            (cuuint64_t)p.bs * p.H_kv * D * 2};
  const cuuint32_t kbx[4] = {64, 1, (cuuint32_t)box_rows, 1};
  int rc;
  if ((rc = encode(&tq, dt, 3, p.q, qd, qs, qb)) != SPA_OK) return rc;
  if ((rc = encode(&tk, dt, 4, p.k_cache, kd, ks, kbx)) != SPA_OK) return rc;
  if ((rc = encode(&tv, dt, 4, p.v_cache, kd, ks, kbx)) != SPA_OK) return rc;
  const int n_qt = (p.max_q + kPfBM - 1) / kPfBM;
  const int max_tiles = (p.max_k + kPfBN - 1) / kPfBN + 1;
  auto kern = prefill_tcgen05_kernel<T, D>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  dim3 grid(p.H_q, n_qt, p.B);
  return launch_pdl(kern, grid, dim3(128), C::SMEM, stream, p, tq, tk, tv, n_qt, box_rows, max_tiles);
}

int launch_prefill(const AttnParams& p, int act, cudaStream_t stream) {
  if (p.T == 0 || p.B == 0 || p.max_q == 0) return SPA_OK;
  if (act == SPA_BF16) {
    if (p.D == 64) return launch_pf<__nv_bfloat16, 64>(p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, stream);
    return launch_pf<__nv_bfloat16, 128>(p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, stream);
  }
  if (p.D == 64) return launch_pf<__half, 64>(p, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, stream);
  return launch_pf<__half, 128>(p, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, stream);
}

}  // namespace spa
