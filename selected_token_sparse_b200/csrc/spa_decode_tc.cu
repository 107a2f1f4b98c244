// Steps 3-5 for units with many query rows (multi-token decode: G q heads x
// S_q tokens sharing one kv head's candidate list, up to 128 rows) on the
// fifth-generation tensor cores.
//
// With tens of rows per kv head every gathered K/V row feeds a 96- or
// 128-row contraction, so the unit is one M = 128 tcgen05 tile.  The CTA
// runs three roles that overlap:
//
//   * producer warps (4): resolve the candidates (window positions, selected
//     or auxiliary slots) through the block table with every guard, gather
//     64-key tiles, and place them as fp16 / bf16 K and V tiles
//     (128-byte-swizzled; V is the MN-major B operand of PV, the same bytes)
//     in a three-stage ring.  Rows are gathered with cp.async (16-bit rows
//     straight into place; INT8 rows into a raw staging ring, converted to
//     exact fp16 integers).  A tile's "full" barrier is released
//     when it is in place; its "empty" barrier is committed by the MMAs that
//     read it, so the next tiles are prepared while this one is computed;
//   * softmax warps (4, one thread per TMEM lane = one row of the unit:
//     token i, head g -> row i*G + g): the row's q goes into tensor memory
//     (INT8 caches fold the key scale into q, split into fp16 high and low
//     parts, so S = Q_hi K^T + Q_lo K^T carries ~22 bits); per tile, the
//     row's 64 scores from TMEM, masked by key position (causal / window for
//     the main cache, always visible for auxiliary entries), a lazily raised
//     max in log2 units, P into one of two TMEM buffers of its own; at the
//     end O is scaled by the value scale (INT8), normalised with the sink and
//     written (one split) or left in the workspace as a partial state and
//     merged with the unit's other splits (up to 8 splits form a
//     thread-block cluster and merge after a cluster barrier, more merge by
//     ticket);
//   * an MMA warp (one thread): S = Q K^T into one of two TMEM buffers, the
//     next tile's S ahead of this tile's PV so that it is computed while the
//     softmax runs, and O += P V (A from TMEM) once the four softmax warps
//     have placed P.
//
// Sources: "[WebGPU] Add DynamicSparseAttention" (Attention: selected and
// local-plus-auxiliary modes, joint FP32 stable softmax with optional sink),
// "[WebGPU] Add SparsePagedAttention" (partial FP32 state, finalize merge),
// onnxruntime PR #33472 (INT8 per-channel K/V scales; 12 q heads per kv head
// with S <= 8 decode).
#include <type_traits>

#include "spa_attn.cuh"
#include "spa_meta.cuh"
#include "spa_sm100.cuh"

namespace spa {

using namespace sm100;

#ifdef SPA_PHASE_PROBE
// Phase probe, compiled only into the separate probe library (build.py
// --probe): the given thread of every CTA stamps %globaltimer at a phase
// boundary; the host reads the stamps of the last launch back.
constexpr int kTcProbeCtas = 4096, kTcProbeSlots = 16;
static __device__ unsigned long long g_phase_tc[kTcProbeCtas * kTcProbeSlots];
__device__ __forceinline__ void tc_phase_stamp(int i, int t) {
  const int c = blockIdx.y * gridDim.x + blockIdx.x;
  if ((int)threadIdx.x != t || c >= kTcProbeCtas) return;
  unsigned long long v;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(v));
  g_phase_tc[c * kTcProbeSlots + i] = v;
}
#define SPA_PHASE_T(i, t) tc_phase_stamp(i, t)
#else
#define SPA_PHASE_T(i, t) ((void)0)
#endif

constexpr int kTcKT = 64;                       // keys per tile (MMA N)
constexpr int kTcStages = 3;                    // K/V tiles in the ring
constexpr int kTcCons = 128;                    // softmax threads (4 warps, one per row)
constexpr int kTcProd = 128;                    // producer threads (4 warps)
constexpr int kTcMmaTid = kTcCons + kTcProd;    // the MMA-issuing thread (its own warp)
constexpr int kTcThreads = kTcCons + kTcProd + 32;
constexpr int kTcBarProd = 2;                   // named barrier of the producers
constexpr int kTcCandTiles = 8;                 // tiles whose candidates are resolved at once
constexpr int kTcCand = kTcCandTiles * kTcKT;
// tensor memory columns: S[2] | O | P[2] (packed 16-bit pairs) | Q_hi | Q_lo |
// P_lo[2] (P residuals for bf16 P and INT8 caches; see residual_pair)
constexpr uint32_t kTcColS = 0, kTcColO = 128, kTcColP = 256, kTcColQ = 320, kTcColPlo = 448;
constexpr uint32_t kTcTmemCols = 512;
constexpr uint32_t kTcWaitLimit = 1u << 20;
constexpr int kTcStageTok = 64;   // fused INT8 step: tokens of a request whose new rows are staged

int tc_key_tile() { return kTcKT; }

template <typename ActT, typename CacheT, int D>
struct TcCfg {
  static constexpr bool kInt8 = sizeof(CacheT) == 1;
  using MT = typename std::conditional<kInt8, __half, ActT>::type;
  // P as P_hi + P_lo (residual_pair): bf16 P, or fp16 P against INT8 V
  static constexpr bool kPLo = kInt8 || std::is_same<MT, __nv_bfloat16>::value;
  static constexpr int NCH = D / 64;
  static constexpr int KCHUNK = kTcKT * 128;          // one 64-column chunk of a 64-row tile
  static constexpr int KTILE = NCH * KCHUNK;          // 64 rows x D, 16-bit, swizzled
  static constexpr int ROW_BYTES = D * (int)sizeof(CacheT);
  static constexpr int RAW = kTcKT * ROW_BYTES;       // one staged INT8 K or V tile
  static constexpr int RAW_ST = kInt8 ? 2 : 0;        // raw stages (INT8)
  static constexpr int OFF_CONV = 0;                                   // [stage][K, V]
  static constexpr int OFF_RAW = OFF_CONV + kTcStages * 2 * KTILE;     // INT8: [raw stage][K, V]
  static constexpr int END_RING = OFF_RAW + RAW_ST * 2 * RAW;
  static constexpr int OFF_KVIS = END_RING;                          // [stage][64] row intervals
  static constexpr int OFF_TVIS = OFF_KVIS + kTcStages * kTcKT * 8;           // [stage] tile seen by every row
  static constexpr int OFF_CAND = OFF_TVIS + 16;                    // [2 chunks] offsets + positions
  static constexpr int OFF_SCALE = OFF_CAND + 2 * kTcCand * 12;     // INT8: ks, vs
  static constexpr int NBAR = 2 * kTcStages + 7;   // full, empty, s[2], o[2], p[2], q
  static constexpr int OFF_BAR = OFF_SCALE + (kInt8 ? 2 * D * 4 : 0);
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;                  // tmem holder, abort flag
  static constexpr int BYTES = (OFF_MISC + 16 + 15) & ~15;   // what follows (fused step) is 16-byte aligned
  // at least 120 KB, so one CTA holds an SM and its 512 TMEM columns
  static constexpr int SMEM = BYTES + 1024 > 120 * 1024 ? BYTES + 1024 : 120 * 1024;
};

// byte offset of 16-byte unit u (0 .. D/8-1) of row r in a ROWS-row swizzled tile
template <int ROWS>
__device__ __forceinline__ int sw_off(int r, int u) {
  const int c = u >> 3, uu = u & 7;
  return c * (ROWS * 128) + (r >> 3) * 1024 + (r & 7) * 128 + ((uu ^ (r & 7)) << 4);
}

template <typename T>
__device__ __forceinline__ uint32_t pk_pair(float lo, float hi) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Four signed bytes -> two fp16 pairs holding the same integers, exactly:
// with the sign bit flipped a byte is u = x + 128 in [0, 255]; placed under
// the fp16 exponent of 1024 (high byte 0x64) it reads 1024 + u, and
// subtracting 1152 leaves x.
__device__ __forceinline__ void i8x4_to_h2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t x = w ^ 0x80808080u;
  uint32_t a = __byte_perm(x, 0x64646464u, 0x4140);
  uint32_t b = __byte_perm(x, 0x64646464u, 0x4342);
  const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));  // 1152
  __half2 ha = __hsub2(*reinterpret_cast<__half2*>(&a), bias);
  __half2 hb = __hsub2(*reinterpret_cast<__half2*>(&b), bias);
  lo = *reinterpret_cast<uint32_t*>(&ha);
  hi = *reinterpret_cast<uint32_t*>(&hb);
}

template <typename ActT>
__device__ __forceinline__ uint4 pack8(const float* x) {
  uint4 r;
  r.x = pk_pair<ActT>(x[0], x[1]);
  r.y = pk_pair<ActT>(x[2], x[3]);
  r.z = pk_pair<ActT>(x[4], x[5]);
  r.w = pk_pair<ActT>(x[6], x[7]);
  return r;
}

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t* r) {
  static_assert(N == 16 || N == 32, "columns");
  if constexpr (N == 32) tmem_st32(taddr, r);
  else tmem_st16(taddr, r);
}

// FUSED: one launch of the whole step.  Every CTA rebuilds the sanitised
// cumulative lengths and reads the past lengths into shared memory (after the
// kernel's own layout), decodes its unit from them with the metadata
// kernels' helpers, reads candidates at this step's new positions from k_new
// / v_new (INT8: quantised exactly as the append quantises them), and the
// producer warps of split 0 write the unit's share of the step-1/2 outputs
// once their gather is done.
template <typename ActT, typename CacheT, int D, bool FUSED>
__global__ void __launch_bounds__(kTcThreads, 1)
decode_tc_kernel(const AttnParams p) {
  using C = TcCfg<ActT, CacheT, D>;
  using MT = typename C::MT;
  constexpr uint32_t FMT = std::is_same<MT, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t IDESC_S = idesc_f16(FMT, 128, kTcKT, 0);
  constexpr uint32_t IDESC_O = idesc_f16(FMT, 128, D, 1);
  constexpr int KT = kTcKT, NST = kTcStages;
  constexpr int CPR = C::ROW_BYTES / 16;   // 16-byte chunks per gathered row
  constexpr uint32_t QCOLS = D / 2;        // TMEM columns of one Q part (two 16-bit values each)
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool softmax = tid < kTcCons;
  const bool producer = !softmax && tid < kTcCons + kTcProd;
  const int ptid = tid - kTcCons;             // producer thread index
  const int row = tid;                        // softmax: the S / O row (TMEM lane)
  __shared__ int last_flag;
  SPA_PHASE_T(0, 0);
  pdl_wait();
  pdl_trigger();
  SPA_PHASE_T(1, 0);

  // Issued before the metadata is known: the lengths every warp scans by
  // itself (fused step, B + 1 <= 64: build_cs_warp, no block barrier that
  // would wait for loads in flight) and the INT8 scales of the kv head.
  const bool warp_scan = FUSED && p.B + 1 <= 64;
  int pc0 = 0, pc1 = 0, pp0 = 0, pp1 = 0;
  if (warp_scan) {
    pc0 = (lane >= 1 && lane <= p.B) ? ld_early(p.cu + lane) : 0;
    pc1 = lane + 32 <= p.B ? ld_early(p.cu + lane + 32) : 0;
    pp0 = lane < p.B ? ld_early(p.past + lane) : 0;
    pp1 = lane + 32 < p.B ? ld_early(p.past + lane + 32) : 0;
  }
  float ks_r = 0.f, vs_r = 0.f;
  if (C::kInt8 && tid < D) {
    ks_r = ld_early(p.k_scale + (blockIdx.x % p.H_kv) * D + tid);
    vs_r = ld_early(p.v_scale + (blockIdx.x % p.H_kv) * D + tid);
  }

  Unit U;
  bool has_rows;
  int bits = 0;
  int32_t* cs_s = nullptr;
  int32_t* past_s = nullptr;
  int8_t* stage_s = nullptr;   // fused INT8 step: [token][K, V][D] quantised new rows
  if constexpr (FUSED) {
    cs_s = reinterpret_cast<int32_t*>(smem + C::BYTES);
    past_s = cs_s + p.B + 1;
    stage_s = reinterpret_cast<int8_t*>(smem + C::BYTES + ((sizeof(int32_t) * (2 * p.B + 1) + 15) & ~size_t(15)));
    if (warp_scan) build_cs_warp(p.B, p.T, cs_s, past_s, pc0, pc1, pp0, pp1);
    else build_cs<kTcThreads>(p.cu, p.B, p.T, cs_s, p.past, past_s);   // ends with a block barrier
    has_rows = decode_unit_with(p, FusedMeta{p.cu, cs_s, past_s, p.B}, blockIdx.x, U);
    if (has_rows) {
      U.new_lo = max(past_s[U.b], 0);
      U.new_hi = U.new_lo + (cs_s[U.b + 1] - cs_s[U.b]);
      U.new_t0 = cs_s[U.b];
    }
    if (p.group_by_request && !has_rows) {
      // no attention rows: split 0 still writes the request's outputs and appends
      if (blockIdx.y == 0) {
        const int b = blockIdx.x / p.H_kv, hk = blockIdx.x % p.H_kv;
        if (blockIdx.x == 0) fused_request_outputs(p, cs_s, past_s, bits, tid, kTcThreads);
        fused_append_rows<ActT, CacheT>(p, cs_s, past_s, cs_s[b], cs_s[b + 1], hk, p.k_scale + hk * D,
                                        p.v_scale + hk * D, tid, kTcThreads, bits);
      }
      flag(p.status, bits);
      return;
    }
  } else {
    has_rows = decode_unit(p, blockIdx.x, U);
    if (p.group_by_request && !has_rows) return;
  }
  SPA_PHASE_T(2, 0);
  const int split = blockIdx.y;
  const int G = p.G;
  const int nq = p.group_by_request ? U.nq : 1;
  const int R = nq * G;
  const int t0 = has_rows ? U.t0 : blockIdx.x / p.H_kv;
  const int h_kv = blockIdx.x % p.H_kv;
  const int n_total = has_rows ? U.n_main + U.n_aux : 0;
  const int c_begin = split * p.split_len;
  const int c_end = min(c_begin + p.split_len, n_total);
  const int ntiles = c_end > c_begin ? (c_end - c_begin + KT - 1) / KT : 0;
  // query positions of the unit's rows: [p_lo, p_hi]
  const int p_lo = has_rows ? U.p_first : 0, p_hi = has_rows ? U.p_last : -1;
  // fused INT8 step: the request's new rows fit the staging area
  const bool staged_new = FUSED && C::kInt8 && has_rows && U.new_hi - U.new_lo <= kTcStageTok;

  int2* kvis_s = reinterpret_cast<int2*>(smem + C::OFF_KVIS);
  int* tvis_s = reinterpret_cast<int*>(smem + C::OFF_TVIS);
  // candidate chunks are double-buffered: resolving chunk c + 1 leaves the
  // tiles of chunk c still in flight untouched
  long long* cand_off = reinterpret_cast<long long*>(smem + C::OFF_CAND);
  int* cand_kpos = reinterpret_cast<int*>(smem + C::OFF_CAND + 2 * kTcCand * 8);
  float* ksc = reinterpret_cast<float*>(smem + C::OFF_SCALE);
  float* vsc = ksc + D;
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);   // [NST] tile in place
  uint64_t* bar_empty = bar_full + NST;   // [NST] tile's MMAs complete (tcgen05.commit)
  uint64_t* bar_s = bar_empty + NST;      // [2] S of tile j in buffer j % 2 complete
  uint64_t* bar_o = bar_s + 2;            // [2] PV of tile j (P buffer j % 2) complete
  uint64_t* bar_p = bar_o + 2;            // [2] P of tile j placed by the four softmax warps
  uint64_t* bar_q = bar_p + 2;            // Q in tensor memory (four softmax warps)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);

  if (tid == 0) {
    for (int i = 0; i < C::NBAR; ++i) mbar_init(bar_full + i, i >= 2 * NST + 4 ? kTcCons / 32 : 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, kTcTmemCols);
    tmem_relinquish();
  }
  if (C::kInt8 && tid < D) {
    ksc[tid] = ks_r;
    vsc[tid] = vs_r;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // softmax: Q row `row` (token row / G, head row % G), loaded after the
  // set-up barrier (which would otherwise wait for it: the producers' path
  // is the critical one; the softmax warps wait for S(0) long after)
  constexpr int QV = D / 8;
  uint4 qv[QV];
  float sink_raw = -INFINITY;
  if (softmax) {
#pragma unroll
    for (int k = 0; k < QV; ++k) qv[k] = make_uint4(0, 0, 0, 0);
    if (row < R) {
      const uint4* src = reinterpret_cast<const uint4*>(
          static_cast<const ActT*>(p.q) + ((long long)(t0 + row / G) * p.H_q + h_kv * G + row % G) * D);
#pragma unroll
      for (int k = 0; k < QV; ++k) qv[k] = src[k];
    }
    // the epilogue's (or the cluster merge's) sink logit of row `row`
    if (p.sinks && p.num_splits == 1 && row < R) sink_raw = ld_early(p.sinks + h_kv * G + row % G);
  }

  if (producer) {
    // =================== producers: candidates, gather, conversion ===================
    const CacheT* kc = static_cast<const CacheT*>(p.k_cache);
    const CacheT* vc = static_cast<const CacheT*>(p.v_cache);
    const CacheT* ak = static_cast<const CacheT*>(p.aux_k);
    const CacheT* av = static_cast<const CacheT*>(p.aux_v);
    // slot of candidate r of tile j: chunk buffer (j / 8) % 2, tile (j % 8)
    auto cslot = [](int j, int r) { return ((j / kTcCandTiles) & 1) * kTcCand + (j % kTcCandTiles) * KT + r; };
    auto resolve_chunk = [&](int first_tile) {
      // every stage's loads of this thread's candidates are in flight together
      constexpr int RPT = kTcCand / kTcProd;
      const int buf = ((first_tile / kTcCandTiles) & 1) * kTcCand;
      static_assert(kTcCand % kTcProd == 0, "candidates per thread");
      int raw[RPT], blk[RPT];
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        const int cand = c_begin + first_tile * KT + ptid + k * kTcProd;
        raw[k] = cand < c_end ? cand_stage1(p, U, cand) : -1;
      }
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        const int cand = c_begin + first_tile * KT + ptid + k * kTcProd;
        blk[k] = cand < c_end ? cand_stage2(p, U, cand, raw[k]) : -1;
      }
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        const int i = ptid + k * kTcProd, cand = c_begin + first_tile * KT + i;
        int kp = kPosInvalid;
        bool from_aux = false;
        long long off = -1;
        if (cand < c_end) off = cand_finish(p, U, cand, raw[k], blk[k], kp, from_aux, bits);
        if constexpr (FUSED) {
          // this step's tokens: read the row the append writes from its source
          if (off >= 0 && kp >= U.new_lo && kp < U.new_hi)
            off = (((long long)(U.new_t0 + kp - U.new_lo) * p.H_kv + U.h_kv) * D) | kNewRow;
        }
        cand_off[buf + i] = off;
        cand_kpos[buf + i] = kp;
      }
    };
    // cp.async copies of tile j: into the raw ring (INT8) or straight into the
    // swizzled K / V stage (16-bit caches)
    constexpr int NIT = KT * CPR * 2 / kTcProd;   // 16-byte chunks per producer thread and tile
    static_assert(KT * CPR * 2 % kTcProd == 0, "chunks per thread");
    auto issue = [&](int j) {
      bool any_new = false;   // fused INT8 step: rows of this step's tokens, quantised below
#pragma unroll 8
      for (int k = 0; k < NIT; ++k) {
        const int e = ptid + k * kTcProd;
        const bool isv = e >= KT * CPR;
        const int ee = isv ? e - KT * CPR : e;
        const int r = ee / CPR, ch = ee % CPR;
        const int ci = cslot(j, r);
        long long off = cand_off[ci];
        const int kp = cand_kpos[ci];
        const bool okr = off >= 0;
        const CacheT* base = isv ? (kp == kPosAux ? av : vc) : (kp == kPosAux ? ak : kc);
        if constexpr (FUSED) {
          if (okr && (off & kNewRow)) {
            if constexpr (C::kInt8) {
              any_new = true;
              continue;
            } else {
              off &= ~kNewRow;
              base = static_cast<const CacheT*>(isv ? p.v_new : p.k_new);
            }
          }
        }
        const CacheT* src = okr ? base + off + ch * (16 / sizeof(CacheT)) : kc;
        unsigned char* dst;
        if constexpr (C::kInt8) {
          dst = smem + C::OFF_RAW + ((j & 1) * 2 + (isv ? 1 : 0)) * C::RAW + r * C::ROW_BYTES + ch * 16;
        } else {
          dst = smem + C::OFF_CONV + ((j % NST) * 2 + (isv ? 1 : 0)) * C::KTILE + sw_off<KT>(r, ch);
        }
        cp_async_16(dst, src, okr);
      }
      if constexpr (FUSED && C::kInt8) {
        if (any_new) {
          // each such 16-byte chunk is 16 channels of a k_new / v_new row:
          // copied from the staged rows, or quantised here with this kv
          // head's scales when the request has too many new tokens to stage
          for (int k = 0; k < NIT; ++k) {
            const int e = ptid + k * kTcProd;
            const bool isv = e >= KT * CPR;
            const int ee = isv ? e - KT * CPR : e;
            const int r = ee / CPR, ch = ee % CPR;
            const long long off = cand_off[cslot(j, r)];
            if (off < 0 || !(off & kNewRow)) continue;
            uint4 q8;
            if (staged_new) {
              const int tj = cand_kpos[cslot(j, r)] - U.new_lo;
              q8 = *reinterpret_cast<const uint4*>(stage_s + (tj * 2 + (isv ? 1 : 0)) * D + ch * 16);
            } else {
              Group16<ActT> g;
              g.load(static_cast<const ActT*>(isv ? p.v_new : p.k_new) + (off & ~kNewRow) + ch * 16);
              q8 = quant_group16<ActT>(g.v, (isv ? vsc : ksc) + ch * 16);
            }
            *reinterpret_cast<uint4*>(smem + C::OFF_RAW + ((j & 1) * 2 + (isv ? 1 : 0)) * C::RAW +
                                      r * C::ROW_BYTES + ch * 16) = q8;
          }
        }
      }
    };
    // each key's interval [a, b] of query positions that see it (auxiliary
    // entries: all; empty slots: none; main-cache key j: j .. j + window - 1,
    // or j .. with no window); returns whether every key this thread placed
    // is visible to every row of the unit
    auto place_vis = [&](int j) -> bool {
      const int st = j % NST;
      bool all_vis = true;
      for (int r = ptid; r < KT; r += kTcProd) {
        const int kp = cand_kpos[cslot(j, r)];
        int a = kp, b = INT_MAX;
        if (kp == kPosAux) {
          a = INT_MIN;
        } else if (kp == kPosInvalid) {
          a = INT_MAX;
          b = INT_MIN;
        } else if (p.window > 0 && kp <= INT_MAX - p.window) {
          b = kp + p.window - 1;
        }
        kvis_s[st * KT + r] = make_int2(a, b);
        all_vis = all_vis && a <= p_lo && b >= p_hi;
      }
      return all_vis;
    };
    bool ok = true;
    auto wait_empty = [&](int j) {   // the MMAs of tile j - NST (same stage) are complete
      if (j >= NST && ok)
        ok = mbar_wait(bar_empty + j % NST, ((j / NST) - 1) & 1, kTcWaitLimit, abort_flag);
    };
    auto publish = [&](int j, bool all_vis) {   // tile j in place: release its full barrier
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      const bool tv = bar_red_and(all_vis, kTcBarProd, kTcProd);
      if (ptid == 0) {
        tvis_s[j % NST] = tv ? 1 : 0;
        mbar_arrive(bar_full + j % NST);
      }
    };
    // fused INT8 step: the request's new rows (this step's tokens, kv head
    // h_kv) are loaded with the first candidates' loads, quantised once into
    // the staging area, and split 0 appends them to the cache from there
    constexpr int PRE = 1;
    const int per_tok = 2 * (D / 16);
    const int n_new = (FUSED && C::kInt8 && staged_new) ? (U.new_hi - U.new_lo) * per_tok : 0;
    Group16<ActT> pre_g[PRE];
    TokenLoad pre_tl[PRE];
    if constexpr (FUSED && C::kInt8) {
#pragma unroll
      for (int k = 0; k < PRE; ++k) {
        const int idx = ptid + k * kTcProd;
        if (idx < n_new) {
          const int t = U.new_t0 + idx / per_tok, it = idx % per_tok;
          const bool isv = it >= D / 16;
          pre_g[k].load(static_cast<const ActT*>(isv ? p.v_new : p.k_new) + ((long long)t * p.H_kv + h_kv) * D +
                        (isv ? it - D / 16 : it) * 16);
          if (split == 0) pre_tl[k] = token_meta_load(t, cs_s, p.B, past_s, p.block_table, p.MB, p.bs);
        }
      }
    }
    SPA_PHASE_T(3, kTcCons);
    if (ntiles > 0) resolve_chunk(0);
    SPA_PHASE_T(4, kTcCons);
    if constexpr (FUSED && C::kInt8) {
      for (int idx = ptid; idx < n_new; idx += kTcProd) {
        const int k = (idx - ptid) / kTcProd;
        const int tj = idx / per_tok, it = idx % per_tok;
        const int t = U.new_t0 + tj;
        const bool isv = it >= D / 16;
        const int g = isv ? it - D / 16 : it;
        Group16<ActT> x;
        TokenLoad tl;
        if (k < PRE) {
          x = pre_g[k < PRE ? k : 0];
          if (split == 0) tl = pre_tl[k < PRE ? k : 0];
        } else {
          x.load(static_cast<const ActT*>(isv ? p.v_new : p.k_new) + ((long long)t * p.H_kv + h_kv) * D + g * 16);
          if (split == 0) tl = token_meta_load(t, cs_s, p.B, past_s, p.block_table, p.MB, p.bs);
        }
        const uint4 q8 = quant_group16<ActT>(x.v, (isv ? vsc : ksc) + g * 16);
        *reinterpret_cast<uint4*>(stage_s + (tj * 2 + (isv ? 1 : 0)) * D + g * 16) = q8;
        if (split == 0) {
          int tb = 0;
          const TokenMeta m = token_meta_finish(tl, p.MB, p.bs, p.NB, tb);
          if (it == 0 && h_kv == 0) {
            bits |= tb;
            p.token_batch_out[t] = m.b;
            p.token_pos_out[t] = m.pos;
            p.slot_out[t] = m.slot;
          }
          if (m.slot >= 0)
            *reinterpret_cast<uint4*>(static_cast<int8_t*>(const_cast<void*>(isv ? p.v_cache : p.k_cache)) +
                                      ((long long)m.slot * p.H_kv + h_kv) * D + g * 16) = q8;
        }
      }
    }
    SPA_PHASE_T(13, kTcCons);
    bar_sync(kTcBarProd, kTcProd);
    if constexpr (C::kInt8) {
      if (ntiles > 0) issue(0);
      cp_async_commit();
      for (int j = 0; j < ntiles && ok; ++j) {
        if (j + 1 < ntiles) {
          if ((j + 1) % kTcCandTiles == 0) {
            bar_sync(kTcBarProd, kTcProd);   // the copies of the previous chunk are issued
            resolve_chunk(j + 1);
            bar_sync(kTcBarProd, kTcProd);
          }
          issue(j + 1);   // raw stage (j+1) & 1 held tile j - 1, converted already
        }
        cp_async_commit();
        if (j == 0) SPA_PHASE_T(14, kTcCons);
        cp_async_wait<1>();
        bar_sync(kTcBarProd, kTcProd);   // tile j's raw rows landed (every producer's copies)
        if (j == 0) SPA_PHASE_T(15, kTcCons);
        wait_empty(j);
        if (bar_red_or(!ok, kTcBarProd, kTcProd)) {
          ok = false;
          break;
        }
        unsigned char* kcv = smem + C::OFF_CONV + (j % NST) * 2 * C::KTILE;
        unsigned char* vcv = kcv + C::KTILE;
        const unsigned char* rawp = smem + C::OFF_RAW + (j & 1) * 2 * C::RAW;
        // every raw chunk of this thread is read before any is converted
        uint4 rv[NIT];
#pragma unroll
        for (int k = 0; k < NIT; ++k) {
          const int e = ptid + k * kTcProd;
          const bool isv = e >= KT * CPR;
          const int ee = isv ? e - KT * CPR : e;
          rv[k] = *reinterpret_cast<const uint4*>(rawp + (isv ? C::RAW : 0) + (ee / CPR) * C::ROW_BYTES + (ee % CPR) * 16);
        }
#pragma unroll
        for (int k = 0; k < NIT; ++k) {
          const int e = ptid + k * kTcProd;
          const bool isv = e >= KT * CPR;
          const int ee = isv ? e - KT * CPR : e;
          const int r = ee / CPR, ch = ee % CPR;
          uint4 h0, h1;
          i8x4_to_h2x2(rv[k].x, h0.x, h0.y);
          i8x4_to_h2x2(rv[k].y, h0.z, h0.w);
          i8x4_to_h2x2(rv[k].z, h1.x, h1.y);
          i8x4_to_h2x2(rv[k].w, h1.z, h1.w);
          unsigned char* dst = isv ? vcv : kcv;
          *reinterpret_cast<uint4*>(dst + sw_off<KT>(r, 2 * ch)) = h0;
          *reinterpret_cast<uint4*>(dst + sw_off<KT>(r, 2 * ch + 1)) = h1;
        }
        publish(j, place_vis(j));
        if (j == 0) SPA_PHASE_T(5, kTcCons);
      }
    } else {
      // NST tiles in flight; tile j + NST goes into tile j's stage once its MMAs are done
      for (int j = 0; j < NST && j < ntiles; ++j) {
        issue(j);
        cp_async_commit();
      }
      for (int j = 0; j < ntiles && ok; ++j) {
        // groups committed after tile j's: min(j + NST - 1, ntiles - 1) - j
        const int newer = min(j + NST - 1, ntiles - 1) - j;
        if (newer >= 2) cp_async_wait<2>();
        else if (newer == 1) cp_async_wait<1>();
        else cp_async_wait<0>();
        bar_sync(kTcBarProd, kTcProd);   // tile j landed (every producer's copies)
        publish(j, place_vis(j));
        if (j == 0) SPA_PHASE_T(5, kTcCons);
        const int n = j + NST;
        if (n < ntiles) {
          if (n % kTcCandTiles == 0) {
            bar_sync(kTcBarProd, kTcProd);
            resolve_chunk(n);
            bar_sync(kTcBarProd, kTcProd);
          }
          wait_empty(n);
          if (bar_red_or(!ok, kTcBarProd, kTcProd)) {
            ok = false;
            break;
          }
          issue(n);
          cp_async_commit();
        }
      }
    }
    cp_async_wait<0>();   // no copy outlives the CTA's use of the ring
    if (!ok) *abort_flag = 1;
    if constexpr (FUSED) {
      // steps 1-2 of the unit's tokens, off the attention's critical path
      if (split == 0) {
        if (blockIdx.x == 0) fused_request_outputs(p, cs_s, past_s, bits, ptid, kTcProd);
        int t_lo = blockIdx.x / p.H_kv, t_hi = t_lo + 1;
        if (p.group_by_request) {
          t_lo = cs_s[t_lo];
          t_hi = cs_s[blockIdx.x / p.H_kv + 1];
        }
        // staged INT8 rows were appended at the start
        if (!(C::kInt8 && staged_new && p.group_by_request))
          fused_append_rows<ActT, CacheT>(p, cs_s, past_s, t_lo, t_hi, h_kv, ksc, vsc, ptid, kTcProd, bits);
      }
    }
  }

  // S of tile n into buffer n % 2: A = Q from tensor memory, B = the tile's
  // K rows (K-major, 128-byte swizzle)
  auto issue_s = [&](int n) {
    const unsigned char* kt = smem + C::OFF_CONV + (n % NST) * 2 * C::KTILE;
    const uint32_t dS = tmem + kTcColS + (n & 1) * KT;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c = kk / 4, koff = (kk % 4) * 32;
      const uint64_t bd = smem_desc_sw128(smem_u32(kt + c * C::KCHUNK + koff), 16, 1024);
      mma_ts(dS, tmem + kTcColQ + kk * 8, bd, IDESC_S, kk > 0 ? 1u : 0u);
      if constexpr (C::kInt8) mma_ts(dS, tmem + kTcColQ + QCOLS + kk * 8, bd, IDESC_S, 1u);
    }
    tc_commit(bar_s + (n & 1));
  };
  if (tid == kTcMmaTid && ntiles > 0) {
    // =================== MMA thread ===================
    // order: S(0), then per tile j: S(j + 1), PV(j).  S(j + 1) overwrites the
    // scores of tile j - 1, which the softmax warps read before placing P(j - 1),
    // which PV(j - 1) waited for.
    bool ok = mbar_wait(bar_q, 0, kTcWaitLimit, abort_flag) && mbar_wait(bar_full, 0, kTcWaitLimit, abort_flag);
    int s_iss = 0, pv_iss = 0;   // S and PV groups issued (each committed to its buffer's barrier)
    if (ok) {
      tc_fence_after();
      issue_s(0);
      ++s_iss;
    }
    for (int j = 0; j < ntiles && ok; ++j) {
      const int st = j % NST, sb = j & 1;
      if (j + 1 < ntiles) {
        ok = mbar_wait(bar_full + (j + 1) % NST, ((j + 1) / NST) & 1, kTcWaitLimit, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_s(j + 1);
        ++s_iss;
      }
      ok = mbar_wait(bar_p + sb, (j >> 1) & 1, kTcWaitLimit, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const unsigned char* vt = smem + C::OFF_CONV + st * 2 * C::KTILE + C::KTILE;
#pragma unroll
      for (int kk = 0; kk < KT / 16; ++kk) {
        const uint64_t bd = smem_desc_sw128(smem_u32(vt + kk * 2048), C::KCHUNK, 1024);
        mma_ts(tmem + kTcColO, tmem + kTcColP + sb * (KT / 2) + kk * 8, bd, IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
        if constexpr (C::kPLo) mma_ts(tmem + kTcColO, tmem + kTcColPlo + sb * (KT / 2) + kk * 8, bd, IDESC_O, 1u);
      }
      tc_commit(bar_o + sb);
      tc_commit(bar_empty + st);   // the stage is free once S and PV of this tile complete
      ++pv_iss;
    }
    if (!ok) {
      *abort_flag = 1;
      // the MMAs already issued complete before the tensor memory is freed
      // (bounded; the latest commit on a barrier covers every earlier MMA)
      if (s_iss > 0) mbar_wait(bar_s + ((s_iss - 1) & 1), ((s_iss - 1) >> 1) & 1, kTcWaitLimit);
      if (pv_iss > 0) mbar_wait(bar_o + ((pv_iss - 1) & 1), ((pv_iss - 1) >> 1) & 1, kTcWaitLimit);
    }
  }

  float m_used = -INFINITY, l_sum = 0.f;
  const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
  const uint32_t tO = tmem + kTcColO + lane_off;
  if (softmax) {
    // ---- Q row `row` -> tensor memory (the A operand of S); INT8 caches fold
    // the key scale into q and split it into fp16 high and low parts
    {
      // 32 columns (64 values) at a time
#pragma unroll
      for (int c = 0; c < (int)QCOLS; c += 32) {
        uint32_t qh[32];
        if constexpr (!C::kInt8) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 u = qv[c / 4 + k];
            qh[4 * k + 0] = u.x;
            qh[4 * k + 1] = u.y;
            qh[4 * k + 2] = u.z;
            qh[4 * k + 3] = u.w;
          }
          tmem_st32(tmem + lane_off + kTcColQ + c, qh);
        } else {
          uint32_t ql[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const ActT* x8 = reinterpret_cast<const ActT*>(&qv[c / 4 + k]);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const int d = (c / 4 + k) * 8 + e;
              const float x0 = to_f32(x8[e]) * ksc[d];
              const float x1 = to_f32(x8[e + 1]) * ksc[d + 1];
              const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
              const __half l0 = __float2half_rn(x0 - __half2float(h0));
              const __half l1 = __float2half_rn(x1 - __half2float(h1));
              __half2 hh = __halves2half2(h0, h1), ll = __halves2half2(l0, l1);
              qh[4 * k + e / 2] = *reinterpret_cast<uint32_t*>(&hh);
              ql[4 * k + e / 2] = *reinterpret_cast<uint32_t*>(&ll);
            }
          }
          tmem_st32(tmem + lane_off + kTcColQ + c, qh);
          tmem_st32(tmem + lane_off + kTcColQ + QCOLS + c, ql);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_q);
    }
    SPA_PHASE_T(6, 0);
    const float sl2 = p.scale_log2;
    const int prow = (row < R && has_rows) ? U.p_first + row / G : -1;
    bool lost = false;
    for (int j = 0; j < ntiles; ++j) {
      const int st = j % NST, sb = j & 1;
      // S(j) complete; the tile's visibility flags were placed before its full barrier
      const bool got = mbar_wait(bar_s + sb, (j >> 1) & 1, kTcWaitLimit, abort_flag) &&
                       mbar_wait(bar_full + st, (j / NST) & 1, kTcWaitLimit, abort_flag);
      if (__any_sync(0xffffffffu, !got)) {
        lost = true;
        break;
      }
      if (j == 0) SPA_PHASE_T(7, 0);
      tc_fence_after();
      // ---- softmax of row `row` over the tile's 64 keys
      const bool tile_vis = tvis_s[st] != 0;
      uint32_t v[KT];
      tmem_ld32(tmem + kTcColS + lane_off + sb * KT, v);
      tmem_ld32(tmem + kTcColS + lane_off + sb * KT + 32, v + 32);
      tmem_wait_ld();
      float mx0 = -INFINITY, mx1 = -INFINITY;
      if (tile_vis) {
#pragma unroll
        for (int e = 0; e < KT; e += 2) {
          mx0 = fmaxf(mx0, __uint_as_float(v[e]));
          mx1 = fmaxf(mx1, __uint_as_float(v[e + 1]));
        }
      } else {
        const int4* kv4 = reinterpret_cast<const int4*>(kvis_s + st * KT);
#pragma unroll
        for (int e = 0; e < KT; e += 2) {
          const int4 w = kv4[e / 2];
          const float x0 = (prow >= w.x && prow <= w.y) ? __uint_as_float(v[e]) : -INFINITY;
          const float x1 = (prow >= w.z && prow <= w.w) ? __uint_as_float(v[e + 1]) : -INFINITY;
          v[e] = __float_as_uint(x0);
          v[e + 1] = __float_as_uint(x1);
          mx0 = fmaxf(mx0, x0);
          mx1 = fmaxf(mx1, x1);
        }
      }
      const float mx = fmaxf(mx0, mx1) * sl2;
      const bool need = mx > m_used + 8.0f;
      const float m_new = need ? mx : m_used;
      const float alpha = need ? ((m_used == -INFINITY) ? 0.f : ex2a(m_used - m_new)) : 1.f;
      if (j > 0 && __any_sync(0xffffffffu, need && m_used != -INFINITY)) {
        // O is rescaled in place once the previous tile's PV is complete
        if (!mbar_wait(bar_o + ((j - 1) & 1), ((j - 1) >> 1) & 1, kTcWaitLimit, abort_flag)) *abort_flag = 1;
        tc_fence_after();
        uint32_t o[32];
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
      }
      m_used = m_new;
      const float nm = (m_used == -INFINITY) ? 0.f : -m_used;
      float ls0 = 0.f, ls1 = 0.f;
      constexpr bool kLo = C::kPLo;
      uint32_t pk[KT / 2], pl[kLo ? KT / 2 : 1];
#pragma unroll
      for (int e = 0; e < KT; e += 2) {
        const float pa = ex2a(fmaf(__uint_as_float(v[e]), sl2, nm));
        const float pb = ex2a(fmaf(__uint_as_float(v[e + 1]), sl2, nm));
        ls0 += pa;
        ls1 += pb;
        pk[e / 2] = pk_pair<MT>(pa, pb);
        if constexpr (kLo) pl[e / 2] = residual_pair<MT>(pa, pb, pk[e / 2]);
      }
      l_sum = l_sum * alpha + (ls0 + ls1);
      // P buffer sb was last read by the PV of tile j - 2
      if (j >= 2) {
        if (!mbar_wait(bar_o + sb, ((j - 2) >> 1) & 1, kTcWaitLimit, abort_flag)) *abort_flag = 1;
        tc_fence_after();
      }
      // packed P of the 64 keys -> the buffer's 32 columns
      tmem_st32(tmem + kTcColP + lane_off + sb * (KT / 2), pk);
      if constexpr (kLo) tmem_st32(tmem + kTcColPlo + lane_off + sb * (KT / 2), pl);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p + sb);
    }
    // O is complete once the last tile's PV is
    if (!lost && ntiles > 0) {
      if (!mbar_wait(bar_o + ((ntiles - 1) & 1), ((ntiles - 1) >> 1) & 1, kTcWaitLimit, abort_flag))
        *abort_flag = 1;
      tc_fence_after();
    }
    if (lost) *abort_flag = 1;
    SPA_PHASE_T(8, 0);
  }
  // every role is done with the rings (the producers drained their copies)
  __syncthreads();
  const bool lost = *abort_flag != 0;
  if (lost) bits |= SPA_ST_TIMEOUT;

  // ---- epilogue (softmax warps): row `row`; O (x value scale) -> output or
  // partial state
  if (softmax) {
    const bool have_o = ntiles > 0 && !lost;
    const int tt = t0 + row / max(G, 1), h = h_kv * G + row % G;
    const long long orow = (long long)tt * p.H_q + h;
    const bool mine = row < R;
    float f = 1.f, lse = -INFINITY;
    if (p.num_splits == 1) {
      const float sink2 = (p.sinks && mine) ? sink_raw * kLog2e : -INFINITY;
      float a, inv_l;
      finalize_row(m_used, l_sum, sink2, a, inv_l, lse);
      f = a * inv_l;
    }
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (have_o) {
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (!mine) continue;
      const int col = c * 32;
      float ov[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) ov[e] = __uint_as_float(o[e]) * (C::kInt8 ? vsc[col + e] : 1.f);
      if (p.num_splits == 1) {
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] *= f;
        if (p.out_f32) {
          float4* out = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * D + col);
#pragma unroll
          for (int e = 0; e < 32; e += 4) out[e / 4] = make_float4(ov[e], ov[e + 1], ov[e + 2], ov[e + 3]);
        } else {
          uint4* out = reinterpret_cast<uint4*>(static_cast<ActT*>(p.out) + orow * D + col);
#pragma unroll
          for (int e = 0; e < 32; e += 8) out[e / 8] = pack8<ActT>(ov + e);
        }
      } else {
        float* acc = p.ws_acc + ((long long)split * p.T * p.H_q + orow) * D + col;
#pragma unroll
        for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(acc + e) = make_float4(ov[e], ov[e + 1], ov[e + 2], ov[e + 3]);
      }
    }
    if (mine) {
      if (p.num_splits == 1) {
        if (p.lse) p.lse[orow] = lse;
      } else {
        const long long wrow = (long long)split * p.T * p.H_q + orow;
        p.ws_ml[wrow * 2 + 0] = m_used;
        p.ws_ml[wrow * 2 + 1] = l_sum;
      }
    }
  }
  SPA_PHASE_T(9, 0);
  flag(p.status, bits);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
  if (p.num_splits > 1) {
    if (p.cluster_merge) {
      // every split's partial state is in the workspace once the cluster
      // barrier passes; each CTA merges a share of the rows
      cluster_sync();
      SPA_PHASE_T(11, 0);
      if (p.num_splits <= 4) cluster_merge_rows<ActT, D, 4, 3>(p, t0, nq, h_kv);
      else cluster_merge_rows<ActT, D, kClusterMaxSplits, 1>(p, t0, nq, h_kv);
      SPA_PHASE_T(12, 0);
    } else {
      finish_split<ActT, D>(p, blockIdx.x, t0, nq, h_kv, &last_flag);
    }
  }
  SPA_PHASE_T(10, 0);
}

int tc_supported(int act, int cache, int D, int max_rows) {
  if (act != SPA_F16 && act != SPA_BF16) return 0;
  if (!(cache == act || cache == SPA_I8)) return 0;
  if (D != 64 && D != 128) return 0;
  return max_rows > 32 && max_rows <= 128;
}

// Shared memory the fused step adds: cumulative lengths [B + 1] and past
// lengths [B], then (INT8) the staged new rows [kTcStageTok][K, V][D].
static size_t tc_fused_extra_smem(int B, int cache, int D) {
  return ((sizeof(int32_t) * (size_t)(2 * B + 1) + 15) & ~size_t(15)) +
         (cache == SPA_I8 ? (size_t)kTcStageTok * 2 * D : 0);
}

template <typename ActT, typename CacheT, int D, bool FUSED>
static int launch_tc_t(const AttnParams& p, cudaStream_t stream) {
  using C = TcCfg<ActT, CacheT, D>;
  static_assert(C::SMEM <= 227 * 1024, "shared memory");
  static_assert(C::SMEM >= C::BYTES + 1024, "the fused step's arrays follow the aligned layout");
  static_assert(C::BYTES % 16 == 0, "the staged rows are 16-byte vectors");
  auto kern = decode_tc_kernel<ActT, CacheT, D, FUSED>;
  const size_t smem = C::SMEM + (FUSED ? tc_fused_extra_smem(p.B, C::kInt8 ? SPA_I8 : SPA_F16, D) : 0);
  if (smem > 227 * 1024) return SPA_ERR_UNSUPPORTED;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int units = p.group_by_request ? p.B * p.H_kv : p.T * p.H_kv;
  if (p.cluster_merge)
    return launch_pdl_cluster_y(kern, dim3(units, p.num_splits), dim3(kTcThreads), smem, stream, p.num_splits, p);
  return launch_pdl(kern, dim3(units, p.num_splits), dim3(kTcThreads), smem, stream, p);
}

template <bool FUSED>
static int launch_tc_any(const AttnParams& p, int act, int cache, cudaStream_t stream) {
  if (act == SPA_F16) {
    if (cache == SPA_I8) return p.D == 64 ? launch_tc_t<__half, int8_t, 64, FUSED>(p, stream)
                                          : launch_tc_t<__half, int8_t, 128, FUSED>(p, stream);
    return p.D == 64 ? launch_tc_t<__half, __half, 64, FUSED>(p, stream)
                     : launch_tc_t<__half, __half, 128, FUSED>(p, stream);
  }
  if (cache == SPA_I8) return p.D == 64 ? launch_tc_t<__nv_bfloat16, int8_t, 64, FUSED>(p, stream)
                                        : launch_tc_t<__nv_bfloat16, int8_t, 128, FUSED>(p, stream);
  return p.D == 64 ? launch_tc_t<__nv_bfloat16, __nv_bfloat16, 64, FUSED>(p, stream)
                   : launch_tc_t<__nv_bfloat16, __nv_bfloat16, 128, FUSED>(p, stream);
}

int launch_attention_tc(const AttnParams& p, int act, int cache, cudaStream_t stream) {
  return launch_tc_any<false>(p, act, cache, stream);
}

// The whole step in one launch.
int launch_step_tc(const AttnParams& p, int act, int cache, cudaStream_t stream) {
  return launch_tc_any<true>(p, act, cache, stream);
}

// Whether the fused step fits one CTA's shared memory.
int tc_step_fits(int D, int cache, int B) {
  size_t base;
  if (cache == SPA_I8) base = D == 64 ? TcCfg<__half, int8_t, 64>::SMEM : TcCfg<__half, int8_t, 128>::SMEM;
  else base = D == 64 ? TcCfg<__half, __half, 64>::SMEM : TcCfg<__half, __half, 128>::SMEM;
  return base + tc_fused_extra_smem(B, cache, D) <= 227 * 1024;
}

}  // namespace spa

#ifdef SPA_PHASE_PROBE
// Probe library only: copy / clear the phase stamps of decode_tc_kernel.
extern "C" int spa_probe_read_tc(void* host, size_t bytes) {
  if (bytes > sizeof(spa::g_phase_tc)) bytes = sizeof(spa::g_phase_tc);
  return (int)cudaMemcpyFromSymbol(host, spa::g_phase_tc, bytes);
}
extern "C" int spa_probe_clear_tc() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, spa::g_phase_tc) != cudaSuccess) return -1;
  return (int)cudaMemset(p, 0, sizeof(spa::g_phase_tc));
}
#endif
