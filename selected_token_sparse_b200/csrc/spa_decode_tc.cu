// Steps 3-5 for units with many query rows (multi-token decode: G q heads x
// S_q tokens sharing one kv head's candidate list, up to 128 rows) on the
// fifth-generation tensor cores.
//
// With tens of rows per kv head every gathered K/V row feeds a 96- or
// 128-row contraction, so the unit is one M = 128 tcgen05 tile:
//
//   * the unit's rows (token i, head g) -> row i*G + g of a Q tile in shared
//     memory, 128-byte-swizzled K-major; INT8 caches keep K exact (|k8| <= 128
//     is exact in fp16) and fold the key scale into q, split into fp16 high
//     and low tiles, so S = Q_hi K^T + Q_lo K^T carries ~22 bits;
//   * candidates (window positions, selected or auxiliary slots) are resolved
//     up front through the block table with every guard; rows are gathered
//     with cp.async into a double-buffered staging area (the next 128-key
//     tile streams in while this one is computed); INT8 rows are converted to
//     fp16 integers into the swizzled K and V tiles (V is the MN-major B
//     operand of PV, the same bytes), 16-bit rows are copied there as is;
//   * S = Q K^T (tcgen05.mma into TMEM), 128 softmax threads (thread i owns
//     row i) mask by key position (causal / window for the main cache,
//     always visible for auxiliary entries), keep a lazily raised max in log2
//     units, write P over S in TMEM, then O += P V (A from TMEM);
//   * O is scaled by the value scale (INT8), then either normalised with the
//     sink and written (one split) or written as a partial state merged by the
//     CTA that takes the unit's last ticket.
//
// Sources: "[WebGPU] Add DynamicSparseAttention" (Attention: selected and
// local-plus-auxiliary modes, joint FP32 stable softmax with optional sink),
// "[WebGPU] Add SparsePagedAttention" (partial FP32 state, finalize merge),
// onnxruntime PR #33472 (INT8 per-channel K/V scales; 12 q heads per kv head
// with S <= 8 decode).
#include <type_traits>

#include "spa_attn.cuh"
#include "spa_sm100.cuh"

namespace spa {

using namespace sm100;

constexpr int kTcKT = 128;                      // keys per tile (MMA N)
constexpr int kTcThreads = 256;                 // two warps per TMEM lane quadrant
constexpr int kTcCandTiles = 4;                 // tiles whose candidates are resolved at once
constexpr int kTcCand = kTcCandTiles * kTcKT;
constexpr uint32_t kTcTmemCols = 256;           // S [0,128) | O [128, 128 + D)
constexpr uint32_t kTcWaitLimit = 1u << 20;

int tc_key_tile() { return kTcKT; }

template <typename ActT, typename CacheT, int D>
struct TcCfg {
  static constexpr bool kInt8 = sizeof(CacheT) == 1;
  using MT = typename std::conditional<kInt8, __half, ActT>::type;
  static constexpr int NCH = D / 64;
  static constexpr int TILE = NCH * 128 * 128;        // one 128-row 16-bit tile, swizzled
  static constexpr int ROW_BYTES = D * (int)sizeof(CacheT);
  static constexpr int RAW = kTcKT * ROW_BYTES;       // one staged K or V tile (INT8 only)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_QLO = OFF_Q + TILE;
  static constexpr int OFF_KV = OFF_QLO + (kInt8 ? TILE : 0);
  // 16-bit caches: 2 stages x (K, V) swizzled tiles; INT8: one (K, V) pair of
  // converted tiles plus 2 stages x (K, V) raw staging
  static constexpr int KV_BYTES = kInt8 ? 2 * TILE + 2 * 2 * RAW : 2 * 2 * TILE;
  static constexpr int OFF_KVIS = OFF_KV + KV_BYTES;              // [2][128] visible row-position intervals
  static constexpr int OFF_CAND = OFF_KVIS + 2 * kTcKT * 8;      // candidate offsets + positions
  static constexpr int OFF_RED = OFF_CAND + kTcCand * 12;        // [2][128] row max, [2][128] row sum
  static constexpr int OFF_SCALE = OFF_RED + 4 * 128 * 4;        // INT8: ks, vs
  static constexpr int OFF_BAR = OFF_SCALE + (kInt8 ? 2 * D * 4 : 0);
  static constexpr int OFF_MISC = OFF_BAR + 16;                  // tmem holder
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM = BYTES + 1024;
  // cluster split merge: partial o [128][D + 4] and (m, l) [128][2], fp32, over
  // the K/V staging once every tile is consumed
  static constexpr int OFF_PART = OFF_KV;
  static constexpr int PART_ML = OFF_PART + 128 * (D + 4) * 4;
  static_assert(PART_ML + 128 * 2 * 4 <= OFF_KV + KV_BYTES, "partial state must fit the K/V staging");
};

// byte offset of 16-byte unit u (0 .. D/8-1) of row r in a 128-row swizzled tile
__device__ __forceinline__ int sw_off(int r, int u) {
  const int c = u >> 3, uu = u & 7;
  return c * 16384 + (r >> 3) * 1024 + (r & 7) * 128 + ((uu ^ (r & 7)) << 4);
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

template <typename ActT, typename CacheT, int D>
__global__ void __launch_bounds__(kTcThreads, 1)
decode_tc_kernel(const AttnParams p) {
  using C = TcCfg<ActT, CacheT, D>;
  using MT = typename C::MT;
  constexpr uint32_t FMT = std::is_same<MT, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t IDESC_S = idesc_f16(FMT, 128, kTcKT, 0);
  constexpr uint32_t IDESC_O = idesc_f16(FMT, 128, D, 1);
  constexpr int KT = kTcKT, NT = kTcThreads;
  constexpr int HK = KT / 2, HD = D / 2;   // key columns / O columns per warp half
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;   // the S / O row (TMEM lane) this thread works on
  __shared__ int last_flag;
  pdl_wait();
  pdl_trigger();

  Unit U;
  const bool has_rows = decode_unit(p, blockIdx.x, U);
  if (p.group_by_request && !has_rows) return;
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

  unsigned char* sQ = smem + C::OFF_Q;
  unsigned char* sQlo = smem + C::OFF_QLO;
  int2* kvis_s = reinterpret_cast<int2*>(smem + C::OFF_KVIS);
  long long* cand_off = reinterpret_cast<long long*>(smem + C::OFF_CAND);
  int* cand_kpos = reinterpret_cast<int*>(smem + C::OFF_CAND + kTcCand * 8);
  float* red_max = reinterpret_cast<float*>(smem + C::OFF_RED);
  float* red_l = red_max + 2 * 128;
  float* ksc = reinterpret_cast<float*>(smem + C::OFF_SCALE);
  float* vsc = ksc + D;
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_o = bar_s + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);

  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, kTcTmemCols);
    tmem_relinquish();
  }
  if constexpr (C::kInt8) {
    for (int d = tid; d < D; d += NT) {
      ksc[d] = p.k_scale[h_kv * D + d];
      vsc[d] = p.v_scale[h_kv * D + d];
    }
  }
  int bits = 0;
  auto resolve_chunk = [&](int first_tile) {
    // every stage's loads of this thread's candidates are in flight together
    constexpr int RPT = kTcCand / NT;
    static_assert(kTcCand % NT == 0, "candidates per thread");
    int raw[RPT], blk[RPT];
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      const int cand = c_begin + first_tile * KT + tid + k * NT;
      raw[k] = cand < c_end ? cand_stage1(p, U, cand) : -1;
    }
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      const int cand = c_begin + first_tile * KT + tid + k * NT;
      blk[k] = cand < c_end ? cand_stage2(p, U, cand, raw[k]) : -1;
    }
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      const int i = tid + k * NT, cand = c_begin + first_tile * KT + i;
      int kp = kPosInvalid;
      bool from_aux = false;
      long long off = -1;
      if (cand < c_end) off = cand_finish(p, U, cand, raw[k], blk[k], kp, from_aux, bits);
      cand_off[i] = off;
      cand_kpos[i] = kp;
    }
  };
  // Q rows (row r = token r / G, head r % G) in coalesced 16-byte units; the
  // loads are in flight while the candidates resolve
  constexpr int QU = D / 8;
  constexpr int QPER = 128 * QU / NT;
  uint4 qv[QPER];
  {
    const ActT* q = static_cast<const ActT*>(p.q);
#pragma unroll
    for (int k = 0; k < QPER; ++k) {
      const int i = tid + k * NT, r = i / QU, u = i % QU;
      qv[k] = make_uint4(0, 0, 0, 0);
      if (r < R)
        qv[k] = *reinterpret_cast<const uint4*>(q + ((long long)(t0 + r / G) * p.H_q + h_kv * G + r % G) * D + u * 8);
    }
  }
  // the epilogue's sink logit of row `row`, in flight from here
  const float sink_raw = (p.sinks && p.num_splits == 1 && row < R) ? ld_early(p.sinks + h_kv * G + row % G)
                                                                   : -INFINITY;
  if (ntiles > 0) resolve_chunk(0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
  const uint32_t tS = tmem + lane_off;
  const uint32_t tO = tmem + 128 + lane_off + half * HD;

  // ---- gather of tile `it` into stage it % 2 (cp.async, 16-byte chunks).
  // Each key also gets the interval [a, b] of query positions that see it
  // (auxiliary entries: all; empty slots: none; main-cache key j: j .. j +
  // window - 1, or j .. with no window).  Returns whether every key this
  // thread placed is visible to every row of the unit.
  const CacheT* kc = static_cast<const CacheT*>(p.k_cache);
  const CacheT* vc = static_cast<const CacheT*>(p.v_cache);
  const CacheT* ak = static_cast<const CacheT*>(p.aux_k);
  const CacheT* av = static_cast<const CacheT*>(p.aux_v);
  constexpr int CPR = C::ROW_BYTES / 16;   // 16-byte chunks per gathered row
  auto issue = [&](int it) -> bool {
    const int st = it & 1;
    bool all_vis = true;
    for (int e = tid; e < KT * CPR * 2; e += NT) {
      const bool isv = e >= KT * CPR;
      const int ee = isv ? e - KT * CPR : e;
      const int r = ee / CPR, ch = ee % CPR;
      const int ci = (it % kTcCandTiles) * KT + r;
      const long long off = cand_off[ci];
      const int kp = cand_kpos[ci];
      const bool okr = off >= 0;
      const CacheT* base = isv ? (kp == kPosAux ? av : vc) : (kp == kPosAux ? ak : kc);
      const CacheT* src = okr ? base + off + ch * (16 / sizeof(CacheT)) : kc;
      unsigned char* dst;
      if constexpr (C::kInt8) {
        dst = smem + C::OFF_KV + 2 * C::TILE + (st * 2 + (isv ? 1 : 0)) * C::RAW + r * C::ROW_BYTES + ch * 16;
      } else {
        dst = smem + C::OFF_KV + (st * 2 + (isv ? 1 : 0)) * C::TILE + sw_off(r, ch);
      }
      cp_async_16(dst, src, okr);
      if (!isv && ch == 0) {
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
    }
    return all_vis;
  };
  bool vis_cur = true;
  if (ntiles > 0) vis_cur = issue(0);
  cp_async_commit();

  // ---- Q tile in swizzled shared memory (overlaps the first gather); INT8
  // caches fold the key scale into q and split it into fp16 high and low tiles
  {
#pragma unroll
    for (int k = 0; k < QPER; ++k) {
      const int i = tid + k * NT, r = i / QU, u = i % QU;
      if constexpr (!C::kInt8) {
        *reinterpret_cast<uint4*>(sQ + sw_off(r, u)) = qv[k];
      } else {
        const ActT* x8 = reinterpret_cast<const ActT*>(&qv[k]);
        alignas(16) __half h8[8], l8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float x = to_f32(x8[e]) * ksc[u * 8 + e];
          h8[e] = __float2half_rn(x);
          l8[e] = __float2half_rn(x - __half2float(h8[e]));
        }
        *reinterpret_cast<uint4*>(sQ + sw_off(r, u)) = *reinterpret_cast<const uint4*>(h8);
        *reinterpret_cast<uint4*>(sQlo + sw_off(r, u)) = *reinterpret_cast<const uint4*>(l8);
      }
    }
  }

  float m_used = -INFINITY, l_sum = 0.f;
  const float sl2 = p.scale_log2;
  const int prow = (row < R && has_rows) ? U.p_first + row / G : -1;
  bool lost = false;
  for (int it = 0; it < ntiles; ++it) {
    const int st = it & 1;
    const int nxt = it + 1;
    if (nxt < ntiles && nxt % kTcCandTiles == 0) {
      __syncthreads();   // copies of the previous chunk are issued
      resolve_chunk(nxt);
      __syncthreads();
    }
    bool vis_nxt = true;
    if (nxt < ntiles) vis_nxt = issue(nxt);   // stage nxt & 1 was released by PV(it - 1)
    cp_async_commit();
    cp_async_wait<1>();
    const bool tile_vis = __syncthreads_and(vis_cur);
    vis_cur = vis_nxt;
    const unsigned char* kt;
    const unsigned char* vt;
    if constexpr (C::kInt8) {
      // PV(it - 1) finished reading the converted tiles (waited below)
      unsigned char* kcv = smem + C::OFF_KV;
      unsigned char* vcv = kcv + C::TILE;
      const unsigned char* raw = smem + C::OFF_KV + 2 * C::TILE + st * 2 * C::RAW;
#pragma unroll 2
      for (int e = tid; e < KT * CPR * 2; e += NT) {
        const bool isv = e >= KT * CPR;
        const int ee = isv ? e - KT * CPR : e;
        const int r = ee / CPR, ch = ee % CPR;
        const uint4 rv = *reinterpret_cast<const uint4*>(raw + (isv ? C::RAW : 0) + r * C::ROW_BYTES + ch * 16);
        uint4 h0, h1;
        i8x4_to_h2x2(rv.x, h0.x, h0.y);
        i8x4_to_h2x2(rv.y, h0.z, h0.w);
        i8x4_to_h2x2(rv.z, h1.x, h1.y);
        i8x4_to_h2x2(rv.w, h1.z, h1.w);
        unsigned char* dst = isv ? vcv : kcv;
        *reinterpret_cast<uint4*>(dst + sw_off(r, 2 * ch)) = h0;
        *reinterpret_cast<uint4*>(dst + sw_off(r, 2 * ch + 1)) = h1;
      }
      kt = kcv;
      vt = vcv;
    } else {
      kt = smem + C::OFF_KV + st * 2 * C::TILE;
      vt = kt + C::TILE;
    }
    // generic-proxy smem writes (Q, converted tiles, cp.async data) must be
    // visible to the tensor core's async proxy
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int c = kk / 4, koff = (kk % 4) * 32;
        const uint64_t bd = smem_desc_sw128(smem_u32(kt + c * 16384 + koff), 16, 1024);
        mma_ss(tmem, smem_desc_sw128(smem_u32(sQ + c * 16384 + koff), 16, 1024), bd, IDESC_S,
               kk > 0 ? 1u : 0u);
        if constexpr (C::kInt8)
          mma_ss(tmem, smem_desc_sw128(smem_u32(sQlo + c * 16384 + koff), 16, 1024), bd, IDESC_S, 1u);
      }
      tc_commit(bar_s);
    }
    const bool got = mbar_wait(bar_s, it & 1, kTcWaitLimit);
    if (__syncthreads_or(!got)) {
      lost = true;
      break;
    }
    tc_fence_after();
    // ---- softmax of row `row` over this half's 64 keys of the tile; the two
    // halves exchange their maxima through shared memory
    uint32_t v[HK];
    tmem_ld32(tS + half * HK, v);
    tmem_ld32(tS + half * HK + 32, v + 32);
    tmem_wait_ld();
    float mx0 = -INFINITY, mx1 = -INFINITY;
    if (tile_vis) {
#pragma unroll
      for (int e = 0; e < HK; e += 2) {
        mx0 = fmaxf(mx0, __uint_as_float(v[e]));
        mx1 = fmaxf(mx1, __uint_as_float(v[e + 1]));
      }
    } else {
      const int4* kv4 = reinterpret_cast<const int4*>(kvis_s + st * KT + half * HK);
#pragma unroll
      for (int e = 0; e < HK; e += 2) {
        const int4 w = kv4[e / 2];
        const float x0 = (prow >= w.x && prow <= w.y) ? __uint_as_float(v[e]) : -INFINITY;
        const float x1 = (prow >= w.z && prow <= w.w) ? __uint_as_float(v[e + 1]) : -INFINITY;
        v[e] = __float_as_uint(x0);
        v[e + 1] = __float_as_uint(x1);
        mx0 = fmaxf(mx0, x0);
        mx1 = fmaxf(mx1, x1);
      }
    }
    red_max[half * 128 + row] = fmaxf(mx0, mx1);
    __syncthreads();
    const float mx = fmaxf(red_max[row], red_max[128 + row]) * sl2;
    const bool need = mx > m_used + 8.0f;
    const float m_new = need ? mx : m_used;
    const float alpha = need ? ((m_used == -INFINITY) ? 0.f : ex2a(m_used - m_new)) : 1.f;
    if (it > 0 && __any_sync(0xffffffffu, need && m_used != -INFINITY)) {
      uint32_t o[32];
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
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
    uint32_t pk[HK / 2];
#pragma unroll
    for (int e = 0; e < HK; e += 2) {
      const float pa = ex2a(fmaf(__uint_as_float(v[e]), sl2, nm));
      const float pb = ex2a(fmaf(__uint_as_float(v[e + 1]), sl2, nm));
      ls0 += pa;
      ls1 += pb;
      pk[e / 2] = pk_pair<MT>(pa, pb);
    }
    // packed P of keys [half*64, half*64 + 64) -> columns [half*32, half*32 + 32);
    // every S column was read into registers before the barrier above
    tmem_st32(tS + half * (HK / 2), pk);
    l_sum = l_sum * alpha + (ls0 + ls1);
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < KT / 16; ++kk) {
        const uint64_t bd = smem_desc_sw128(smem_u32(vt + kk * 2048), 16384, 1024);
        mma_ts(tmem + 128, tmem + kk * 8, bd, IDESC_O, (it > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(bar_o);
    }
    // the next tile's staging / conversion and S reuse what PV reads
    const bool gone = mbar_wait(bar_o, it & 1, kTcWaitLimit);
    if (__syncthreads_or(!gone)) {
      lost = true;
      break;
    }
    tc_fence_after();
  }
  cp_async_wait<0>();
  red_l[half * 128 + row] = l_sum;
  __syncthreads();
  l_sum = red_l[row] + red_l[128 + row];
  if (lost) bits |= SPA_ST_TIMEOUT;

  // ---- epilogue: row `row`, this half's D/2 columns; O (x value scale) ->
  // output or partial state
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
  for (int c = 0; c < HD / 32; ++c) {
    uint32_t o[32];
    if (have_o) {
      tmem_ld32(tO + c * 32, o);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = 0u;
    }
    if (!mine) continue;
    const int col = half * HD + c * 32;
    float ov[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) ov[e] = __uint_as_float(o[e]) * (C::kInt8 ? vsc[col + e] : 1.f);
    if (p.num_splits == 1) {
#pragma unroll
      for (int e = 0; e < 32; ++e) ov[e] *= f;
      uint4* out = reinterpret_cast<uint4*>(static_cast<ActT*>(p.out) + orow * D + col);
#pragma unroll
      for (int e = 0; e < 32; e += 8) out[e / 8] = pack8<ActT>(ov + e);
    } else if (p.cluster_merge) {
      float* po = reinterpret_cast<float*>(smem + C::OFF_PART) + row * (D + 4) + col;
#pragma unroll
      for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(po + e) = make_float4(ov[e], ov[e + 1], ov[e + 2], ov[e + 3]);
    } else {
      float* acc = p.ws_acc + ((long long)split * p.T * p.H_q + orow) * D + col;
#pragma unroll
      for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(acc + e) = make_float4(ov[e], ov[e + 1], ov[e + 2], ov[e + 3]);
    }
  }
  if (mine && half == 0) {
    if (p.num_splits == 1) {
      if (p.lse) p.lse[orow] = lse;
    } else if (p.cluster_merge) {
      *reinterpret_cast<float2*>(smem + C::PART_ML + row * 8) = make_float2(m_used, l_sum);
    } else {
      const long long wrow = (long long)split * p.T * p.H_q + orow;
      p.ws_ml[wrow * 2 + 0] = m_used;
      p.ws_ml[wrow * 2 + 1] = l_sum;
    }
  }
  flag(p.status, bits);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
  if (p.num_splits > 1) {
    if (p.cluster_merge) {
      cluster_sync();
      cluster_merge_rows<ActT, D>(p, t0, nq, h_kv, reinterpret_cast<const float*>(smem + C::OFF_PART),
                                  reinterpret_cast<const float*>(smem + C::PART_ML));
      cluster_sync();
    } else {
      finish_split<ActT, D>(p, blockIdx.x, t0, nq, h_kv, &last_flag);
    }
  }
}

int tc_supported(int act, int cache, int D, int max_rows) {
  if (act != SPA_F16 && act != SPA_BF16) return 0;
  if (!(cache == act || cache == SPA_I8)) return 0;
  if (D != 64 && D != 128) return 0;
  return max_rows > 32 && max_rows <= 128;
}

template <typename ActT, typename CacheT, int D>
static int launch_tc_t(const AttnParams& p, cudaStream_t stream) {
  using C = TcCfg<ActT, CacheT, D>;
  static_assert(C::SMEM <= 227 * 1024, "shared memory");
  auto kern = decode_tc_kernel<ActT, CacheT, D>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  const int units = p.group_by_request ? p.B * p.H_kv : p.T * p.H_kv;
  if (p.cluster_merge)
    return launch_pdl_cluster_y(kern, dim3(units, p.num_splits), dim3(kTcThreads), C::SMEM, stream, p.num_splits, p);
  return launch_pdl(kern, dim3(units, p.num_splits), dim3(kTcThreads), C::SMEM, stream, p);
}

int launch_attention_tc(const AttnParams& p, int act, int cache, cudaStream_t stream) {
  if (act == SPA_F16) {
    if (cache == SPA_I8) return p.D == 64 ? launch_tc_t<__half, int8_t, 64>(p, stream)
                                          : launch_tc_t<__half, int8_t, 128>(p, stream);
    return p.D == 64 ? launch_tc_t<__half, __half, 64>(p, stream) : launch_tc_t<__half, __half, 128>(p, stream);
  }
  if (cache == SPA_I8) return p.D == 64 ? launch_tc_t<__nv_bfloat16, int8_t, 64>(p, stream)
                                        : launch_tc_t<__nv_bfloat16, int8_t, 128>(p, stream);
  return p.D == 64 ? launch_tc_t<__nv_bfloat16, __nv_bfloat16, 64>(p, stream)
                   : launch_tc_t<__nv_bfloat16, __nv_bfloat16, 128>(p, stream);
}

}  // namespace spa
