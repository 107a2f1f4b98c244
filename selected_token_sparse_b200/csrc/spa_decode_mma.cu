// Steps 3-5 on tensor cores for 16-bit activations (fp16 / bf16 caches, and
// INT8 caches dequantised to fp16 in shared memory).
//
// Decode attention is a skinny contraction: one CTA owns a unit (all G q
// heads of one kv head, for one token or all tokens of one request: R = G*S_q
// rows) and one split of its candidate keys, so every gathered K/V row is read
// from HBM once and used by all R rows.  At G*2 flops per byte the math must
// not run on the FP32 pipe, but R is far below a 128-row tcgen05 tile, so the
// contraction uses warp-level m16n8k16 MMAs (rows padded to 16) while the
// kernel's real work is the gather:
//
//   * candidates (window positions, or selected / auxiliary slots) are resolved
//     through the block table with every guard of the scalar path, by the
//     threads that copy the rows, and
//   * K/V rows are copied as 16-byte cp.async chunks into a 3-stage ring of
//     64-key tiles in XOR-swizzled shared memory (conflict-free ldmatrix),
//     keeping two tiles in flight while one is consumed.
//
// Warps split a key tile (KW slices) and/or the row tiles (RT); each keeps
// its own online-softmax state (log2 units) and merges through shared memory
// at the end.  With one split the learned sink is folded in and the output
// written; otherwise FP32 partial states go to the workspace for the
// log-sum-exp combine, after a cluster barrier (up to 8 splits) or by ticket
// ("[WebGPU] Add SparsePagedAttention", File summaries;
// "[WebGPU] Add DynamicSparseAttention", Attention: joint FP32 stable softmax
// with optional sink; onnxruntime PR #33472: INT8 per-channel K/V scales).
#include <type_traits>

#include "spa_attn.cuh"
#include "spa_meta.cuh"

namespace spa {

#ifdef SPA_PHASE_PROBE
// Phase probe, compiled only into the separate probe library (build.py
// --probe): thread 0 of every CTA stamps %globaltimer at the phase boundaries
// below; the host reads the stamps of the last launch back.
constexpr int kProbeCtas = 8192, kProbeSlots = 16;
static __device__ unsigned long long g_phase_mma[kProbeCtas * kProbeSlots];
__device__ __forceinline__ void phase_stamp(int i) {
  const int c = blockIdx.y * gridDim.x + blockIdx.x;
  if (threadIdx.x != 0 || c >= kProbeCtas) return;
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  g_phase_mma[c * kProbeSlots + i] = t;
}
#define SPA_PHASE(i) phase_stamp(i)
#else
#define SPA_PHASE(i) ((void)0)
#endif

constexpr int kMmaCandChunk = 512;   // candidates resolved at once

// Keys per tile: one 128-key tile (one softmax pass, four 32-key warp slices)
// for single-row-tile units with D = 64, otherwise 64-key tiles in a 3-deep ring.
constexpr int mma_kt(int D, int rt) { return (D == 64 && rt == 1) ? 128 : 64; }
int mma_key_tile(int D, int max_rows) { return mma_kt(D, (max_rows + 15) / 16); }

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename T> struct MmaName;
template <> struct MmaName<__half> { static constexpr bool bf16 = false; };
template <> struct MmaName<__nv_bfloat16> { static constexpr bool bf16 = true; };

template <typename MT>
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, const uint32_t* b) {
  if constexpr (MmaName<MT>::bf16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* p) {
  uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, const void* p) {
  uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}

template <typename MT>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (MmaName<MT>::bf16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

// Byte offset of 16-byte chunk `c` of row `r` in a swizzled tile with `cpr` chunks per row.
__device__ __forceinline__ int swz(int r, int c, int cpr) { return (r * cpr + (c ^ (r & 7))) * 16; }

template <typename ActT, typename CacheT, int D, int RT, int KW>
struct MmaCfg {
  using MT = typename std::conditional<sizeof(CacheT) == 1, __half, ActT>::type;
  static constexpr bool kInt8 = sizeof(CacheT) == 1;
  static constexpr int KT = mma_kt(D, RT);
  static constexpr int STAGES = KT == 128 ? 2 : 3;  // cp.async ring depth
  static constexpr int CAND_TILES = kMmaCandChunk / KT;
  static constexpr int NW = RT * KW;
  static constexpr int NT = NW * 32;
  static constexpr int KS = KT / KW;            // keys per warp slice
  static constexpr int CPR = D * 2 / 16;        // 16-byte chunks per 16-bit row
  static constexpr int RAW_CPR = D * (int)sizeof(CacheT) / 16;
  static constexpr int TILE16 = KT * D * 2;                   // one converted K or V tile
  static constexpr int RAW_TILE = KT * D * (int)sizeof(CacheT);
  static constexpr int ROWS = RT * 16;
  // shared memory layout (bytes)
  static constexpr int OFF_Q = 0;                                      // Q (int8 path: q*ks, high part)
  static constexpr int OFF_QLO = OFF_Q + ROWS * D * 2;                 // int8 path: low part
  static constexpr int OFF_RAW = OFF_QLO + (kInt8 ? ROWS * D * 2 : 0); // stages x (K, V) raw
  static constexpr int OFF_CONV = OFF_RAW + STAGES * 2 * RAW_TILE;  // int8 only: (K, V) fp16
  static constexpr int OFF_KPOS = OFF_CONV + (kInt8 ? 2 * TILE16 : 0);
  static constexpr int OFF_SCALE = OFF_KPOS + STAGES * KT * 4;
  static constexpr int OFF_PROW = OFF_SCALE + (kInt8 ? 2 * D * 4 : 0);
  static constexpr int OFF_CAND = OFF_PROW + 128 * 4;                  // resolved candidates
  static constexpr int END = OFF_CAND + kMmaCandChunk * (8 + 4);
  // the cross-warp merge reuses the K/V ring once every tile is consumed
  static constexpr int OFF_RED = OFF_RAW;
  static constexpr int RED_BYTES = (KW > 1) ? NW * 32 * (D / 2 + 4) * 4 : 0;
  static constexpr int SMEM = END;
  static_assert(OFF_RED + RED_BYTES <= OFF_KPOS, "the merge buffer must not reach the scales / positions");
};

// FUSED: one launch of the whole step (16-bit caches).  Every CTA rebuilds
// the sanitised cumulative lengths and reads the past lengths into shared
// memory (after the kernel's own layout), decodes its unit from them with the
// metadata kernels' helpers, writes its share of the step-1/2 outputs, and
// reads candidates at this step's new positions from k_new / v_new -- the
// bytes the append writes, so the result equals the staged sequence.
template <typename ActT, typename CacheT, int D, int RT, int KW, bool FUSED>
__global__ void __launch_bounds__(RT * KW * 32)
decode_mma_kernel(const AttnParams p) {
  using C = MmaCfg<ActT, CacheT, D, RT, KW>;
  using MT = typename C::MT;
  constexpr int KT = C::KT, NT = C::NT, KS = C::KS, CPR = C::CPR, RAW_CPR = C::RAW_CPR;
  constexpr int kMmaStages = C::STAGES, kMmaCandTiles = C::CAND_TILES;
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wr = warp % RT;   // row tile of this warp
  const int wk = warp / RT;   // key slice of this warp
  __shared__ int last_flag;
  SPA_PHASE(0);
  pdl_wait();
  pdl_trigger();
  SPA_PHASE(1);

  // Issued first: the lengths every warp scans by itself (fused step, B + 1 <= 64:
  // build_cs_warp, no block barrier that would wait for the loads in flight).
  const bool warp_scan = FUSED && p.B + 1 <= 64;
  int pc0 = 0, pc1 = 0, pp0 = 0, pp1 = 0;
  if (warp_scan) {
    pc0 = (lane >= 1 && lane <= p.B) ? ld_early(p.cu + lane) : 0;
    pc1 = lane + 32 <= p.B ? ld_early(p.cu + lane + 32) : 0;
    pp0 = lane < p.B ? ld_early(p.past + lane) : 0;
    pp1 = lane + 32 < p.B ? ld_early(p.past + lane + 32) : 0;
  }

  // Q rows of the unit in 16-byte chunks (row r = token r / G, head r % G).
  // A per-token unit knows its token from the block index, so its loads are
  // in flight while the unit's metadata loads resolve.
  constexpr int QPER = (C::ROWS * CPR + NT - 1) / NT;
  const ActT* q = static_cast<const ActT*>(p.q);
  uint4 qv[QPER];
  auto load_q = [&](int tq, int rows) {
#pragma unroll
    for (int k = 0; k < QPER; ++k) {
      const int e = tid + k * NT, r = e / CPR, c = e % CPR;
      qv[k] = make_uint4(0, 0, 0, 0);
      if (e < C::ROWS * CPR && r < rows)
        qv[k] = *reinterpret_cast<const uint4*>(q + ((long long)(tq + r / p.G) * p.H_q +
                                                     (blockIdx.x % p.H_kv) * p.G + r % p.G) * D + c * 8);
    }
  };
  if (!p.group_by_request) load_q(blockIdx.x / p.H_kv, p.G);
  // fused step, split 0: this thread's vector of the unit's first token's
  // new K/V row is loaded early (a per-token unit knows its token now) and
  // stored into the cache while the split's K/V copies are in flight
  constexpr int NV = D * 2 / 16;
  const bool app_thread = FUSED && blockIdx.y == 0 && tid < 2 * NV;
  uint4 app_data = make_uint4(0, 0, 0, 0);
  if constexpr (FUSED) {
    if (app_thread && !p.group_by_request)
      app_data = fused_load_row_vector<CacheT>(p, blockIdx.x / p.H_kv, blockIdx.x % p.H_kv, tid, NV);
  }

  // Per-request selection rows: the unit's request and kv head follow from the
  // block index, so the first chunk's selection entries can be in flight
  // while the unit's metadata is read (and their block-table entries right
  // after); resolve_chunk(0) then only applies the guards.
  constexpr int RPT = (kMmaCandChunk + NT - 1) / NT;
  const bool pre = p.group_by_request && p.sel != nullptr && p.sel_target == 0 && p.sel_per_request;
  int pre_raw[RPT], pre_blk[RPT];
  if (pre) {
    const int32_t* selrow = p.sel + (long long)blockIdx.x * p.sel_width;   // (request, kv head) = block index
    const int cb = blockIdx.y * p.split_len, ce = min(cb + p.split_len, p.sel_width);
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      const int i = tid + k * NT;
      pre_raw[k] = (i < kMmaCandChunk && cb + i < ce) ? ld_early(selrow + cb + i) : -1;
    }
  }

  Unit U;
  bool has_rows;
  int bits = 0;
  int32_t* cs_s = nullptr;
  int32_t* past_s = nullptr;
  if constexpr (FUSED) {
    cs_s = reinterpret_cast<int32_t*>(smem + C::SMEM);
    past_s = cs_s + p.B + 1;
    if (warp_scan) build_cs_warp(p.B, p.T, cs_s, past_s, pc0, pc1, pp0, pp1);
    else build_cs<NT>(p.cu, p.B, p.T, cs_s, p.past, past_s);   // ends with a block barrier
    has_rows = decode_unit_with(p, FusedMeta{p.cu, cs_s, past_s, p.B}, blockIdx.x, U);
    if (has_rows) {
      U.new_lo = max(past_s[U.b], 0);
      U.new_hi = U.new_lo + (cs_s[U.b + 1] - cs_s[U.b]);
      U.new_t0 = cs_s[U.b];
    }
    if (p.group_by_request && !has_rows) {
      if (blockIdx.y == 0) {
        const int b = blockIdx.x / p.H_kv;
        if (blockIdx.x == 0) fused_request_outputs(p, cs_s, past_s, bits);
        fused_append_tokens<CacheT>(p, cs_s, past_s, cs_s[b], cs_s[b + 1], blockIdx.x % p.H_kv, bits);
      }
      flag(p.status, bits);
      return;
    }
  } else {
    has_rows = decode_unit(p, blockIdx.x, U);
    if (p.group_by_request && !has_rows) return;
  }
  if (pre) {
    const int b = blockIdx.x / p.H_kv;
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      const int raw = pre_raw[k];
      pre_blk[k] = (raw >= 0 && raw / p.bs < p.MB) ? ld_early(p.block_table + (long long)b * p.MB + raw / p.bs) : -1;
    }
  }
  SPA_PHASE(2);
  const int split = blockIdx.y;
  const int G = p.G;
  const int nq = p.group_by_request ? U.nq : 1;
  const int R = nq * G;
  const int t0 = has_rows ? U.t0 : blockIdx.x / p.H_kv;
  const int h_kv = blockIdx.x % p.H_kv;

  unsigned char* q_s = smem + C::OFF_Q;
  int* kpos_s = reinterpret_cast<int*>(smem + C::OFF_KPOS);
  float* ksc_s = reinterpret_cast<float*>(smem + C::OFF_SCALE);
  float* vsc_s = ksc_s + D;
  int* prow_s = reinterpret_cast<int*>(smem + C::OFF_PROW);

  if (p.group_by_request) load_q(t0, R);

  // ---- Q rows -> swizzled smem.  INT8 caches keep K exact (|k8| <= 128 is
  // exact in fp16): the key scale is folded into q in fp32 and q*ks is split
  // into fp16 high and low parts, so S = k8.hi + k8.lo carries ~22 bits.
  if constexpr (C::kInt8) {
    for (int d = tid; d < D; d += NT) {
      ksc_s[d] = p.k_scale[h_kv * D + d];
      vsc_s[d] = p.v_scale[h_kv * D + d];
    }
    __syncthreads();
  }
#pragma unroll
  for (int k = 0; k < QPER; ++k) {
    const int e = tid + k * NT, r = e / CPR, c = e % CPR;
    if (e >= C::ROWS * CPR) continue;
    uint4 v = qv[k];
    if constexpr (C::kInt8) {
      const ActT* x8 = reinterpret_cast<const ActT*>(&qv[k]);
      alignas(16) __half hi[8];
      alignas(16) __half lo[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x = to_f32(x8[i]) * ksc_s[c * 8 + i];
        hi[i] = __float2half_rn(x);
        lo[i] = __float2half_rn(x - __half2float(hi[i]));
      }
      v = *reinterpret_cast<const uint4*>(hi);
      *reinterpret_cast<uint4*>(smem + C::OFF_QLO + swz(r, c, CPR)) = *reinterpret_cast<const uint4*>(lo);
    }
    *reinterpret_cast<uint4*>(q_s + swz(r, c, CPR)) = v;
  }
  for (int i = tid; i < 128; i += NT) prow_s[i] = (i < nq && has_rows) ? U.p_first + i : -1;

  // ---- candidate range of this split
  const int n_total = has_rows ? U.n_main + U.n_aux : 0;
  const int c_begin = split * p.split_len;
  const int c_end = min(c_begin + p.split_len, n_total);
  const int ntiles = c_end > c_begin ? (c_end - c_begin + KT - 1) / KT : 0;
  const CacheT* kc = static_cast<const CacheT*>(p.k_cache);
  const CacheT* vc = static_cast<const CacheT*>(p.v_cache);
  const CacheT* ak = static_cast<const CacheT*>(p.aux_k);
  const CacheT* av = static_cast<const CacheT*>(p.aux_v);
  const CacheT* kn = static_cast<const CacheT*>(p.k_new);
  const CacheT* vn = static_cast<const CacheT*>(p.v_new);

  // Issue the copies of tile `it` into its ring stage.  Thread `tid` copies
  // chunk (tid % RAW_CPR) of rows tid / RAW_CPR, + NT / RAW_CPR, ...
  // Candidates are resolved (selection slot / window position -> block table
  // -> row offset, with every guard) a chunk of tiles at a time by all threads
  // at once, so the index loads of many rows are in flight together and the
  // copy loop below reads ready offsets.
  long long* cand_off = reinterpret_cast<long long*>(smem + C::OFF_CAND);
  int* cand_kpos = reinterpret_cast<int*>(smem + C::OFF_CAND + kMmaCandChunk * 8);
  auto resolve_chunk = [&](int first_tile) {
    // every stage's loads of this thread's candidates are in flight together
    int raw[RPT], blk[RPT];
    if (pre && first_tile == 0) {
      // the prefetched entries; cand_finish rejects what cand_stage2 would have
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        raw[k] = pre_raw[k];
        blk[k] = pre_blk[k];
      }
    } else {
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        const int i = tid + k * NT, cand = c_begin + first_tile * KT + i;
        raw[k] = (i < kMmaCandChunk && cand < c_end) ? cand_stage1(p, U, cand) : -1;
      }
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        const int i = tid + k * NT, cand = c_begin + first_tile * KT + i;
        blk[k] = (i < kMmaCandChunk && cand < c_end) ? cand_stage2(p, U, cand, raw[k]) : -1;
      }
    }
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      const int i = tid + k * NT, cand = c_begin + first_tile * KT + i;
      if (i >= kMmaCandChunk) continue;
      int kp = kPosInvalid;
      bool from_aux = false;
      long long off = -1;
      if (cand < c_end) off = cand_finish(p, U, cand, raw[k], blk[k], kp, from_aux, bits);
      if constexpr (FUSED) {
        // this step's tokens: read the row the append writes from its source
        if (off >= 0 && kp >= U.new_lo && kp < U.new_hi)
          off = (((long long)(U.new_t0 + kp - U.new_lo) * p.H_kv + U.h_kv) * D) | kNewRow;
      }
      cand_off[i] = off;
      cand_kpos[i] = kp;
    }
  };
  auto issue = [&](int it) {
    const int stage = it % kMmaStages;
    unsigned char* kraw = smem + C::OFF_RAW + stage * 2 * C::RAW_TILE;
    unsigned char* vraw = kraw + C::RAW_TILE;
    const int c = tid % RAW_CPR;
    for (int row = tid / RAW_CPR; row < KT; row += NT / RAW_CPR) {
      const int ci = (it % kMmaCandTiles) * KT + row;
      const int kp = cand_kpos[ci];
      long long off = cand_off[ci];
      const bool from_aux = kp == kPosAux;
      const bool ok = off >= 0;
      const CacheT* kb = from_aux ? ak : kc;
      const CacheT* vb = from_aux ? av : vc;
      if constexpr (FUSED) {
        if (ok && (off & kNewRow)) {
          off &= ~kNewRow;
          kb = kn;
          vb = vn;
        }
      }
      const CacheT* ksrc = ok ? kb + off + c * (16 / sizeof(CacheT)) : kc;
      const CacheT* vsrc = ok ? vb + off + c * (16 / sizeof(CacheT)) : vc;
      const int dst = C::kInt8 ? (row * RAW_CPR + c) * 16 : swz(row, c, CPR);
      cp_async_16(kraw + dst, ksrc, ok);
      cp_async_16(vraw + dst, vsrc, ok);
      if (c == 0) kpos_s[stage * KT + row] = kp;
    }
  };

  // per-warp state: rows (lane/4) and (lane/4 + 8) of row tile wr
  float m_r[2] = {-INFINITY, -INFINITY};
  float l_r[2] = {0.f, 0.f};
  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  uint32_t qf[C::kInt8 ? 1 : D / 16][4];

  SPA_PHASE(3);
  if (ntiles > 0) resolve_chunk(0);
  __syncthreads();
  SPA_PHASE(4);
#pragma unroll
  for (int s = 0; s < kMmaStages - 1; ++s) {
    if (s < ntiles) issue(s);
    cp_async_commit();
  }
  // fused step, split 0: the first token of the unit (-1: none) and its
  // block-table entry, in flight until the end
  int app_t = -1;
  TokenLoad app_tl;
  if constexpr (FUSED) {
    if (split == 0) {
      if (!p.group_by_request) {
        app_t = blockIdx.x / p.H_kv;
      } else {
        const int b = blockIdx.x / p.H_kv;
        if (cs_s[b + 1] > cs_s[b]) app_t = cs_s[b];
        if (app_t >= 0 && app_thread) app_data = fused_load_row_vector<CacheT>(p, app_t, h_kv, tid, NV);
      }
      if (app_t >= 0) app_tl = token_meta_load(app_t, cs_s, p.B, past_s, p.block_table, p.MB, p.bs);
      // steps 1-2 of the first token while this split's K/V copies are in
      // flight: no CTA reads the cache rows it writes (keys at this step's
      // positions are read from k_new / v_new)
      if (blockIdx.x == 0) fused_request_outputs(p, cs_s, past_s, bits);
      if (app_t >= 0) {
        int tb = 0;
        const TokenMeta m = token_meta_finish(app_tl, p.MB, p.bs, p.NB, tb);
        fused_token_outputs(p, app_t, h_kv, m, tb, bits);
        if (app_thread && m.slot >= 0) fused_store_row_vector<CacheT>(p, m.slot, h_kv, tid, NV, app_data);
      }
    }
  }
  __syncthreads();
  // Q fragments for this warp's row tile stay in registers (16-bit caches)
  if constexpr (!C::kInt8) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int r = wr * 16 + (lane & 15);
      const int ch = kk * 2 + (lane >> 4);
      ldsm_x4(qf[kk], q_s + swz(r, ch, CPR));
    }
  }
  const int r0 = wr * 16 + (lane >> 2);
  const int r1 = r0 + 8;
  // the epilogue's sink logits, in flight from here
  float sink_raw[2] = {-INFINITY, -INFINITY};
  if (p.sinks && p.num_splits == 1) {
    if (r0 < R) sink_raw[0] = ld_early(p.sinks + h_kv * G + r0 % G);
    if (r1 < R) sink_raw[1] = ld_early(p.sinks + h_kv * G + r1 % G);
  }
  const int prow0 = r0 < R ? prow_s[r0 / G] : -1;
  const int prow1 = r1 < R ? prow_s[r1 / G] : -1;
  const float sl2 = p.scale_log2;

  SPA_PHASE(5);
  for (int it = 0; it < ntiles; ++it) {
    const int nxt = it + kMmaStages - 1;
    if (nxt < ntiles && nxt % kMmaCandTiles == 0) {
      // every thread is past the copies that read the previous chunk
      resolve_chunk(nxt);
      __syncthreads();
    }
    if (nxt < ntiles) issue(nxt);
    cp_async_commit();
    cp_async_wait<kMmaStages - 1>();
    __syncthreads();
    const int stage = it % kMmaStages;
    const unsigned char* ks;
    const unsigned char* vs;
    if constexpr (C::kInt8) {
      // dequantise the raw int8 stage into fp16 tiles (per-channel scales)
      const int8_t* kraw = reinterpret_cast<const int8_t*>(smem + C::OFF_RAW + stage * 2 * C::RAW_TILE);
      const int8_t* vraw = kraw + C::RAW_TILE;
      unsigned char* kconv = smem + C::OFF_CONV;
      unsigned char* vconv = kconv + C::TILE16;
      for (int e = tid; e < KT * RAW_CPR * 2; e += NT) {
        const bool isv = e >= KT * RAW_CPR;
        const int ee = isv ? e - KT * RAW_CPR : e;
        const int row = ee / RAW_CPR, c = ee % RAW_CPR;
        const int8_t* src = (isv ? vraw : kraw) + (row * RAW_CPR + c) * 16;
        const int4 raw = *reinterpret_cast<const int4*>(src);
        const int8_t* b8 = reinterpret_cast<const int8_t*>(&raw);
        alignas(16) __half h[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) h[i] = __int2half_rn(static_cast<int>(b8[i]));   // exact
        unsigned char* dst = isv ? vconv : kconv;
        *reinterpret_cast<uint4*>(dst + swz(row, 2 * c, CPR)) = *reinterpret_cast<const uint4*>(h);
        *reinterpret_cast<uint4*>(dst + swz(row, 2 * c + 1, CPR)) =
            *reinterpret_cast<const uint4*>(h + 8);
      }
      __syncthreads();
      ks = kconv;
      vs = vconv;
    } else {
      ks = smem + C::OFF_RAW + stage * 2 * C::RAW_TILE;
      vs = ks + C::RAW_TILE;
    }
    const int* kpos = kpos_s + stage * KT;

    // S = Q K^T for this warp's 16 rows x KS keys
    float s[KS / 8][4];
#pragma unroll
    for (int j = 0; j < KS / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t qh[4], ql[4];
      if constexpr (C::kInt8) {
        const int r = wr * 16 + (lane & 15);
        const int ch = kk * 2 + (lane >> 4);
        ldsm_x4(qh, q_s + swz(r, ch, CPR));
        ldsm_x4(ql, smem + C::OFF_QLO + swz(r, ch, CPR));
      }
#pragma unroll
      for (int j = 0; j < KS / 8; j += 2) {
        uint32_t b[4];
        const int mi = lane >> 3;
        const int krow = wk * KS + j * 8 + (mi >> 1) * 8 + (lane & 7);
        ldsm_x4(b, ks + swz(krow, kk * 2 + (mi & 1), CPR));
        if constexpr (C::kInt8) {
          mma16816<MT>(s[j], qh, b);
          mma16816<MT>(s[j + 1], qh, b + 2);
          mma16816<MT>(s[j], ql, b);
          mma16816<MT>(s[j + 1], ql, b + 2);
        } else {
          mma16816<MT>(s[j], qf[kk], b);
          mma16816<MT>(s[j + 1], qf[kk], b + 2);
        }
      }
    }
    // mask, scale, online softmax (rows r0, r1)
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < KS / 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = wk * KS + j * 8 + (lane & 3) * 2 + e;
        const int kp = kpos[key];
        s[j][e] = key_visible(kp, prow0, p.window) ? s[j][e] * sl2 : -INFINITY;
        s[j][2 + e] = key_visible(kp, prow1, p.window) ? s[j][2 + e] * sl2 : -INFINITY;
        mx0 = fmaxf(mx0, s[j][e]);
        mx1 = fmaxf(mx1, s[j][2 + e]);
      }
    }
#pragma unroll
    for (int o2 = 1; o2 <= 2; o2 <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
    }
    // The reference max is raised only when a tile's max exceeds it by more
    // than 8 (log2 units): p = 2^(s - m) then stays <= 256 (exact range in
    // fp16 / bf16) and O is rescaled only on those tiles.
    const bool up0 = mx0 > m_r[0] + 8.0f, up1 = mx1 > m_r[1] + 8.0f;
    const float mn0 = up0 ? mx0 : m_r[0], mn1 = up1 ? mx1 : m_r[1];
    const float al0 = (up0 && m_r[0] != -INFINITY) ? ex2f(m_r[0] - mn0) : 1.f;
    const float al1 = (up1 && m_r[1] != -INFINITY) ? ex2f(m_r[1] - mn1) : 1.f;
    // masked scores are -inf and give 0 once the row max is finite
    const float ms0 = (mn0 == -INFINITY) ? 0.f : mn0, ms1 = (mn1 == -INFINITY) ? 0.f : mn1;
    m_r[0] = mn0;
    m_r[1] = mn1;
    float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
    for (int j = 0; j < KS / 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s[j][e] = ex2f(s[j][e] - ms0);
        s[j][2 + e] = ex2f(s[j][2 + e] - ms1);
        ls0 += s[j][e];
        ls1 += s[j][2 + e];
      }
    }
    l_r[0] = l_r[0] * al0 + ls0;
    l_r[1] = l_r[1] * al1 + ls1;
    if (__any_sync(0xffffffffu, up0 || up1)) {
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        o[n][0] *= al0;
        o[n][1] *= al0;
        o[n][2] *= al1;
        o[n][3] *= al1;
      }
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < KS / 16; ++kk) {
      uint32_t a[4];
      a[0] = pack2<MT>(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack2<MT>(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack2<MT>(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack2<MT>(s[2 * kk + 1][2], s[2 * kk + 1][3]);
      // bf16 P, and fp16 P against INT8 V, run as P_hi V + P_lo V (see residual_pair)
      constexpr bool kPLo = MmaName<MT>::bf16 || C::kInt8;
      uint32_t al[4];
      if constexpr (kPLo) {
        al[0] = residual_pair<MT>(s[2 * kk][0], s[2 * kk][1], a[0]);
        al[1] = residual_pair<MT>(s[2 * kk][2], s[2 * kk][3], a[1]);
        al[2] = residual_pair<MT>(s[2 * kk + 1][0], s[2 * kk + 1][1], a[2]);
        al[3] = residual_pair<MT>(s[2 * kk + 1][2], s[2 * kk + 1][3], a[3]);
      }
#pragma unroll
      for (int n = 0; n < D / 8; n += 2) {
        uint32_t b[4];
        const int mi = lane >> 3;
        const int vrow = wk * KS + kk * 16 + (mi & 1) * 8 + (lane & 7);
        ldsm_x4_t(b, vs + swz(vrow, n + (mi >> 1), CPR));
        mma16816<MT>(o[n], a, b);
        mma16816<MT>(o[n + 1], a, b + 2);
        if constexpr (kPLo) {
          mma16816<MT>(o[n], al, b);
          mma16816<MT>(o[n + 1], al, b + 2);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  __syncthreads();
  SPA_PHASE(6);

  // row sums across the quad
#pragma unroll
  for (int o2 = 1; o2 <= 2; o2 <<= 1) {
    l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], o2);
    l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], o2);
  }

  // Merge of the KW key slices of each row tile: every warp publishes its
  // state, then warp (wr, wk) combines and writes the wk-th share of the
  // output columns (8-column blocks [wk * NPW, (wk + 1) * NPW)).
  constexpr int NB8 = D / 8;
  constexpr int NPW = NB8 / KW;
  const int n_lo = wk * NPW;
  float fo[NPW][4];
  float mf[2], lf[2];
  if constexpr (KW > 1) {
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
    constexpr int PER = D / 2 + 4;
    float* mine = red + (warp * 32 + lane) * PER;
#pragma unroll
    for (int n = 0; n < NB8; ++n)
      *reinterpret_cast<float4*>(mine + n * 4) = make_float4(o[n][0], o[n][1], o[n][2], o[n][3]);
    *reinterpret_cast<float4*>(mine + D / 2) = make_float4(m_r[0], m_r[1], l_r[0], l_r[1]);
    __syncthreads();
    float4 ml[KW];
#pragma unroll
    for (int k2 = 0; k2 < KW; ++k2)
      ml[k2] = *reinterpret_cast<const float4*>(red + ((k2 * RT + wr) * 32 + lane) * PER + D / 2);
    mf[0] = mf[1] = -INFINITY;
#pragma unroll
    for (int k2 = 0; k2 < KW; ++k2) {
      mf[0] = fmaxf(mf[0], ml[k2].x);
      mf[1] = fmaxf(mf[1], ml[k2].y);
    }
    float w0[KW], w1[KW];
    lf[0] = lf[1] = 0.f;
#pragma unroll
    for (int k2 = 0; k2 < KW; ++k2) {
      w0[k2] = (mf[0] == -INFINITY) ? 0.f : ex2f(ml[k2].x - mf[0]);
      w1[k2] = (mf[1] == -INFINITY) ? 0.f : ex2f(ml[k2].y - mf[1]);
      lf[0] = fmaf(w0[k2], ml[k2].z, lf[0]);
      lf[1] = fmaf(w1[k2], ml[k2].w, lf[1]);
    }
#pragma unroll
    for (int nn = 0; nn < NPW; ++nn) fo[nn][0] = fo[nn][1] = fo[nn][2] = fo[nn][3] = 0.f;
#pragma unroll
    for (int k2 = 0; k2 < KW; ++k2) {
      const float* other = red + ((k2 * RT + wr) * 32 + lane) * PER;
#pragma unroll
      for (int nn = 0; nn < NPW; ++nn) {
        const float4 x = *reinterpret_cast<const float4*>(other + (n_lo + nn) * 4);
        fo[nn][0] = fmaf(w0[k2], x.x, fo[nn][0]);
        fo[nn][1] = fmaf(w0[k2], x.y, fo[nn][1]);
        fo[nn][2] = fmaf(w1[k2], x.z, fo[nn][2]);
        fo[nn][3] = fmaf(w1[k2], x.w, fo[nn][3]);
      }
    }
  } else {
#pragma unroll
    for (int nn = 0; nn < NPW; ++nn) {
      fo[nn][0] = o[nn][0];
      fo[nn][1] = o[nn][1];
      fo[nn][2] = o[nn][2];
      fo[nn][3] = o[nn][3];
    }
    mf[0] = m_r[0];
    mf[1] = m_r[1];
    lf[0] = l_r[0];
    lf[1] = l_r[1];
  }
  if constexpr (C::kInt8) {   // O = vs * sum_j p_j v8_j (V stayed exact)
#pragma unroll
    for (int nn = 0; nn < NPW; ++nn) {
      const int d = (n_lo + nn) * 8 + (lane & 3) * 2;
      fo[nn][0] *= vsc_s[d];
      fo[nn][1] *= vsc_s[d + 1];
      fo[nn][2] *= vsc_s[d];
      fo[nn][3] *= vsc_s[d + 1];
    }
  }

  // write this warp's columns of rows r0, r1
#pragma unroll
  for (int hrow = 0; hrow < 2; ++hrow) {
    const int r = hrow ? r1 : r0;
    if (r >= R) continue;
    const int t = t0 + r / G, h = h_kv * G + r % G;
    const long long row = (long long)t * p.H_q + h;
    if (p.num_splits == 1) {
      const float sink2 = p.sinks ? sink_raw[hrow] * kLog2e : -INFINITY;
      float a, inv_l, lse;
      finalize_row(mf[hrow], lf[hrow], sink2, a, inv_l, lse);
      const float f = a * inv_l;
      ActT* out = static_cast<ActT*>(p.out) + row * D;
      float* out32 = static_cast<float*>(p.out) + row * D;
#pragma unroll
      for (int nn = 0; nn < NPW; ++nn) {
        const int d = (n_lo + nn) * 8 + (lane & 3) * 2;
        if (p.out_f32)
          *reinterpret_cast<float2*>(out32 + d) = make_float2(fo[nn][hrow * 2 + 0] * f, fo[nn][hrow * 2 + 1] * f);
        else
          *reinterpret_cast<uint32_t*>(out + d) = pack2<ActT>(fo[nn][hrow * 2 + 0] * f, fo[nn][hrow * 2 + 1] * f);
      }
      if (wk == 0 && (lane & 3) == 0 && p.lse) p.lse[row] = lse;
    } else {
      const long long wrow = (long long)split * p.T * p.H_q + row;
      float* acc = p.ws_acc + wrow * D;
#pragma unroll
      for (int nn = 0; nn < NPW; ++nn) {
        const int d = (n_lo + nn) * 8 + (lane & 3) * 2;
        *reinterpret_cast<float2*>(acc + d) = make_float2(fo[nn][hrow * 2], fo[nn][hrow * 2 + 1]);
      }
      if (wk == 0 && (lane & 3) == 0) {
        p.ws_ml[wrow * 2 + 0] = mf[hrow];
        p.ws_ml[wrow * 2 + 1] = lf[hrow];
      }
    }
  }

  SPA_PHASE(7);
  // fused step: a request-grouped unit's further tokens (steps 1-2)
  if constexpr (FUSED) {
    if (split == 0 && app_t >= 0 && p.group_by_request) {
      const int b = blockIdx.x / p.H_kv;
      fused_append_tokens<CacheT>(p, cs_s, past_s, app_t + 1, cs_s[b + 1], h_kv, bits);
    }
  }
  flag(p.status, bits);
  SPA_PHASE(8);
  if (p.num_splits > 1) {
    if (p.cluster_merge) {
      // the unit's splits are one cluster: once every split's partial state
      // is in the workspace, each CTA merges a share of the rows
      cluster_sync();
      SPA_PHASE(10);
      if (p.num_splits <= 4) cluster_merge_rows<ActT, D, 4, 2>(p, t0, nq, h_kv);
      else cluster_merge_rows<ActT, D, kClusterMaxSplits, 1>(p, t0, nq, h_kv);
      SPA_PHASE(11);
    } else {
      finish_split<ActT, D>(p, blockIdx.x, t0, nq, h_kv, &last_flag);
    }
  }
  SPA_PHASE(9);
}

// ---------------------------------------------------------------------------
// dispatch
// ---------------------------------------------------------------------------

size_t mma_fused_extra_smem(int B);

int mma_supported(int act, int cache, int D, int max_rows) {
  if (act != SPA_F16 && act != SPA_BF16) return 0;
  if (!(cache == act || cache == SPA_I8)) return 0;
  if (D != 64 && D != 128) return 0;
  return max_rows >= 1 && max_rows <= 128;
}

template <typename ActT, typename CacheT, int D, int RT, int KW, bool FUSED>
static int launch_rt(const AttnParams& p, cudaStream_t stream) {
  using C = MmaCfg<ActT, CacheT, D, RT, KW>;
  auto kern = decode_mma_kernel<ActT, CacheT, D, RT, KW, FUSED>;
  const size_t smem = C::SMEM + (FUSED ? mma_fused_extra_smem(p.B) : 0);
  if (smem > 227 * 1024) return SPA_ERR_UNSUPPORTED;
  if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int units = p.group_by_request ? p.B * p.H_kv : p.T * p.H_kv;
  dim3 grid(units, p.num_splits);
  if (p.cluster_merge) return launch_pdl_cluster_y(kern, grid, dim3(C::NT), smem, stream, p.num_splits, p);
  return launch_pdl(kern, grid, dim3(C::NT), smem, stream, p);
}

template <typename ActT, typename CacheT, int D, bool FUSED>
static int launch_d(const AttnParams& p, int max_rows, cudaStream_t stream) {
  const int rt = (max_rows + 15) / 16;
  switch (rt) {
    case 1: return launch_rt<ActT, CacheT, D, 1, 4, FUSED>(p, stream);
    case 2: return launch_rt<ActT, CacheT, D, 2, 2, FUSED>(p, stream);
    case 3: return launch_rt<ActT, CacheT, D, 3, 1, FUSED>(p, stream);
    case 4: return launch_rt<ActT, CacheT, D, 4, 1, FUSED>(p, stream);
    case 5:
    case 6: return launch_rt<ActT, CacheT, D, 6, 1, FUSED>(p, stream);
    default: return launch_rt<ActT, CacheT, D, 8, 1, FUSED>(p, stream);
  }
}

template <typename ActT, typename CacheT, bool FUSED>
static int launch_dd(const AttnParams& p, int max_rows, cudaStream_t stream) {
  if (p.D == 64) return launch_d<ActT, CacheT, 64, FUSED>(p, max_rows, stream);
  return launch_d<ActT, CacheT, 128, FUSED>(p, max_rows, stream);
}

int launch_attention_mma(const AttnParams& p, int act, int cache, int max_rows, cudaStream_t stream) {
  if (act == SPA_F16) {
    if (cache == SPA_I8) return launch_dd<__half, int8_t, false>(p, max_rows, stream);
    return launch_dd<__half, __half, false>(p, max_rows, stream);
  }
  if (cache == SPA_I8) return launch_dd<__nv_bfloat16, int8_t, false>(p, max_rows, stream);
  return launch_dd<__nv_bfloat16, __nv_bfloat16, false>(p, max_rows, stream);
}

// Shared memory the fused step adds: cumulative lengths [B + 1] and past lengths [B].
size_t mma_fused_extra_smem(int B) { return sizeof(int32_t) * (size_t)(2 * B + 1); }

// Whether the fused step fits one CTA's shared memory (16-bit caches).
template <int D>
static size_t smem_rt(int rt) {
  switch (rt) {
    case 1: return MmaCfg<__half, __half, D, 1, 4>::SMEM;
    case 2: return MmaCfg<__half, __half, D, 2, 2>::SMEM;
    case 3: return MmaCfg<__half, __half, D, 3, 1>::SMEM;
    case 4: return MmaCfg<__half, __half, D, 4, 1>::SMEM;
    case 5:
    case 6: return MmaCfg<__half, __half, D, 6, 1>::SMEM;
    default: return MmaCfg<__half, __half, D, 8, 1>::SMEM;
  }
}
int mma_step_fits(int D, int max_rows, int B) {
  const int rt = (max_rows + 15) / 16;
  const size_t base = D == 64 ? smem_rt<64>(rt) : smem_rt<128>(rt);
  return base + mma_fused_extra_smem(B) <= 227 * 1024;
}

// The whole step in one launch (16-bit caches whose dtype is the activations').
int launch_step_mma(const AttnParams& p, int act, int max_rows, cudaStream_t stream) {
  if (act == SPA_F16) return launch_dd<__half, __half, true>(p, max_rows, stream);
  return launch_dd<__nv_bfloat16, __nv_bfloat16, true>(p, max_rows, stream);
}

}  // namespace spa

#ifdef SPA_PHASE_PROBE
// Probe library only: copy / clear the phase stamps of decode_mma_kernel.
extern "C" int spa_probe_read_mma(void* host, size_t bytes) {
  if (bytes > sizeof(spa::g_phase_mma)) bytes = sizeof(spa::g_phase_mma);
  return (int)cudaMemcpyFromSymbol(host, spa::g_phase_mma, bytes);
}
extern "C" int spa_probe_clear_mma() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, spa::g_phase_mma) != cudaSuccess) return -1;
  return (int)cudaMemset(p, 0, sizeof(spa::g_phase_mma));
}
#endif
