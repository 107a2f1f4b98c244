// Steps 3-5 for long causal query runs (prefill / chunked prefill) on the
// fifth-generation tensor cores (tcgen05, TMEM accumulators, TMA).
//
// The dense QK^T and PV tiles of a causal (optionally windowed) prefill are
// real contractions, so they run as 128x128xD tcgen05.mma tiles, and the
// kernel is organised so that the tensor core and the softmax overlap:
//
//   item   = two 128-row q tiles (A, B) of one request that read one kv
//            head: the same rows of two q heads when the group size is even
//            (both tiles see the same key tiles), else two consecutive tiles
//            of one q head; each q tile runs only the key tiles its own rows
//            can see.  Causal items run one CTA each, longest first;
//            window-bounded items run persistently, one CTA per SM claiming
//            items from a work counter in the workspace (pf_geom_load and
//            the kernel's comment give the orders and the claim protocol).
//   TMEM   = S_A | S_B | O_A | O_B (4 x 128 columns); P of a tile overwrites
//            its S as packed 16-bit pairs and feeds the PV MMA from TMEM.
//   warp 9 = K/V producer (one thread): K and V tiles through a ring of 3
//            stages (D = 64) or 2 (D = 128) from the paged cache (4-D tensor
//            map over [num_blocks, block_size, H_kv, D]; the block id is a
//            coordinate taken from the block table, read before the wait for
//            a free stage; an unmapped block is read from an out-of-range
//            coordinate, i.e. zeros, and masked; 128-byte swizzle; no
//            multicast); on the persistent schedule it also claims the items.
//   warp 8 = MMA issuer (one thread) and the Q loads (two Q buffers at
//            D = 64: the next item's Q lands during this item).  Per 128-key
//            step j and q tile t it issues PV_t(j) (O_t += P_t V_j) as soon as
//            the softmax group hands over P_t, then S_t(j + 1), so one
//            group's MMAs run on the tensor core while the other group's
//            softmax runs on the CUDA cores.
//   warps 0-3 / 4-7 = softmax of tile A / B: thread i owns row i (TMEM lane i)
//            and reads its row of S from TMEM once per step; masks only the
//            tiles that cross the causal diagonal, the window edge, the end
//            of the keys or an unmapped block; keeps a running max in log2
//            units that is raised (O rescaled in TMEM) only when a tile's max
//            exceeds it by more than 8, so P <= 2^8; the scale is folded into
//            one FFMA ahead of ex2.approx.  16-bit output leaves through
//            per-warp tiled stores at D = 64.
//   registers: warps 8-11 (warps 10-11 idle) hand registers to the softmax
//            warpgroups (setmaxnreg), which need a row of S in registers.
//   sink   = folded into the final normalisation (denominator only).
//
// The key loop starts at the earliest window tile, rounded down to the tile
// size, and keeps per-row visibility checks ("[WebGPU] Add PagedAttention
// metadata and GPT-OSS support", review item Q3); the sink semantics follow
// the same page's Description and "[WebGPU] Add DynamicSparseAttention"
// (joint FP32 stable softmax with optional sink).
//
// Every mbarrier wait is bounded; on expiry the kernel sets SPA_ST_TIMEOUT,
// the other roles give up at their next wait, the issuing thread drains its
// copies and MMAs (bounded), the CTA frees its TMEM and returns.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "spa_attn.cuh"
#include "spa_sm100.cuh"

namespace spa {

using namespace sm100;

#ifdef SPA_PHASE_PROBE
// Phase probe, compiled only into the separate probe library (build.py
// --probe): a few threads of every CTA stamp %globaltimer at the points
// listed in phase_probe.PF_SLOTS; the host reads the stamps of the last launch.
constexpr int kPfProbeCtas = 2048, kPfProbeSlots = 64;
static __device__ unsigned long long g_phase_pf[kPfProbeCtas * kPfProbeSlots];
__device__ __forceinline__ void pf_stamp(int i) {
  if (blockIdx.x >= kPfProbeCtas || i < 0 || i >= kPfProbeSlots) return;
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  g_phase_pf[blockIdx.x * kPfProbeSlots + i] = t;
}
#define SPA_PF_STAMP(cond, i) \
  do {                          \
    if (cond) pf_stamp(i);      \
  } while (0)
#else
#define SPA_PF_STAMP(cond, i) ((void)0)
#endif

constexpr int kPfBM = 128;   // q rows per tile (TMEM lanes)
constexpr int kPfBN = 128;   // keys per step
constexpr uint32_t kPfTmemCols = 512;
constexpr uint32_t kPfWaitLimit = 1u << 20;   // polls before a wait is declared lost
constexpr int kPfRing = 4;                     // item slots of the dynamic schedule
// 3 warpgroups: softmax A (warps 0-3), softmax B (4-7), and warps 8-11: the
// MMA warp, the K/V TMA warp and two idle warps.  The kernel is compiled for
// kPfLaunchRegs registers a thread (one CTA per SM); the third warpgroup hands
// registers to the softmax warpgroups (setmaxnreg), which hold a whole row of
// S: 4 x 128 x (kPfSoftmaxRegs - 168) = 128 x (168 - kPfIssueRegs) registers.
constexpr int kPfThreads = 12 * 32;
constexpr int kPfLaunchRegs = 168;
constexpr int kPfSoftmaxRegs = 200;
constexpr int kPfIssueRegs = 104;
static_assert(2 * (kPfSoftmaxRegs - kPfLaunchRegs) == kPfLaunchRegs - kPfIssueRegs,
              "the registers released by the issue warpgroup must cover the softmax warpgroups' increase");
static_assert(kPfThreads * kPfLaunchRegs <= 65536, "one CTA per SM");

template <int D>
struct PfCfg {
  static constexpr int NCH = D / 64;                  // 128-byte chunks along D
  static constexpr int CHUNK = 128 * 128;             // one chunk of a 128-row tile (bytes)
  static constexpr int TILE = NCH * CHUNK;            // one Q, K or V tile
  // Q buffers (tiles A and B each): two where they fit next to the K/V ring,
  // so that the next item's Q lands while this item runs
  static constexpr int NQB = D == 64 ? 2 : 1;
  static constexpr int OFF_Q = 0;                     // [NQB][2] tiles
  // K/V ring stages: three where they fit, so that the next item's first two
  // key tiles are in flight while this item's last ones are in use
  static constexpr int NST = D == 64 ? 3 : 2;
  static constexpr int OFF_K = OFF_Q + NQB * 2 * TILE;   // NST stages
  static constexpr int OFF_V = OFF_K + NST * TILE;     // NST stages
  // output staging (tiles A and B) for tiled stores of full 16-bit O tiles,
  // where it fits
  static constexpr int NOST = D == 64 ? 2 : 0;
  static constexpr int OFF_OST = OFF_V + NST * TILE;
  static constexpr int OFF_BAR = OFF_OST + NOST * TILE;   // mbarriers
  static constexpr int NBAR = 1 + 3 * NST + 8 + 2 * kPfRing;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int OFF_FLAG = OFF_TMEM + 8;
  static constexpr int OFF_RING = OFF_FLAG + 8;       // [kPfRing] item indices
  static constexpr int BYTES = OFF_RING + 4 * kPfRing;
  // + alignment slack; above half of the SM's shared memory so that exactly
  // one CTA (holding all 512 TMEM columns) is resident per SM
  static constexpr int SMEM = (BYTES + 1024 > 120 * 1024) ? BYTES + 1024 : 120 * 1024;
  static constexpr uint32_t TX_TILE = (uint32_t)TILE;
  static_assert(SMEM <= 227 * 1024, "one CTA's shared memory");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_OST % 1024 == 0 && OFF_BAR % 8 == 0,
                "128-byte-swizzled tiles start on 1024-byte boundaries");
};

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }

// max(a, b, c) in one instruction (three-input max.f32 of sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

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

// bf16 P runs as P_hi V + P_lo V (residual_pair); fp16 P keeps 11 bits
template <typename T>
constexpr bool kPfLo = std::is_same<T, __nv_bfloat16>::value;

struct PfGeom {
  int b, h_kv, t_begin, q_len, past, L, k_lo, k_hi, ntiles;
  int hq[2];     // per q tile: its q head
  int k_first;   // first key any row of the item attends (k_lo is it rounded down to a tile)
  int rlo;       // first key of this shard's range (0: all)
  int q0[2], rows[2];   // per q tile: first row within the request, rows present (0 = absent)
  // per q tile: the key steps [j_lo, j_hi) holding a key some row of the tile
  // may see (causal / window / shard limits); the item's key tiles are their union
  int j_lo[2], j_hi[2];
};

// Block id of box `lane` of the key tile starting at kb (-1 when the lane has
// no box, the box lies beyond the table or the table holds -1); a volatile
// load, so that it is issued here, a tile ahead of its use.
__device__ __forceinline__ int pf_block_id(const AttnParams& p, int b, int kb, int lane, int nbox,
                                           int box_shift) {
  if (lane >= nbox) return -1;
  const int lb = (kb + (lane << box_shift)) / p.bs;
  return lb < p.MB ? ld_early(p.block_table + (long long)b * p.MB + lb) : -1;
}

// Block ids of the boxes of one key tile (keys [kb, kb + 128)) in boxes of
// box_rows rows (one cache block, or 128 rows of one block): independent
// loads, issued ahead of the wait for a free ring stage; they serve both K
// and V.
struct PfIds {
  int raw[8];
};

__device__ __forceinline__ PfIds pf_kv_ids(const AttnParams& p, const PfGeom& g, int kb, int box_rows) {
  const int nbox = kPfBN / box_rows;   // <= 8 (block_size >= 16)
  PfIds ids;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    ids.raw[i] = -1;
    if (i < nbox) {
      const int lb = (kb + i * box_rows) / p.bs;
      if (lb < p.MB) ids.raw[i] = ld_early(p.block_table + (long long)g.b * p.MB + lb);
    }
  }
  return ids;
}

// TMA loads of that key tile of K and of V, box by box.
__device__ __forceinline__ void pf_issue_kv(const AttnParams& p, const PfGeom& g, const PfIds& ids,
                                            const CUtensorMap* map_k, const CUtensorMap* map_v,
                                            unsigned char* dst_k, unsigned char* dst_v, uint64_t* bar_k,
                                            uint64_t* bar_v, int kb, int box_rows, int nch, int& bits,
                                            uint32_t tx) {
  const int nbox = kPfBN / box_rows;
  const int* raw = ids.raw;
  mbar_arrive_expect_tx(bar_k, tx);
  mbar_arrive_expect_tx(bar_v, tx);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i >= nbox) break;
    const int key0 = kb + i * box_rows;
    const bool needed = key0 < g.k_hi && key0 + box_rows > g.k_first;   // some key of the box is attended
    const int lb = key0 / p.bs;
    int blk = -1;
    if (lb >= p.MB) {
      if (needed) bits |= kStCapacity;
    } else if (raw[i] < 0 || raw[i] >= p.NB) {
      if (needed) bits |= kStBadBlock;
    } else {
      blk = raw[i];
    }
    const int cblk = blk >= 0 ? blk : p.NB;  // out of range: the box reads zeros
    const int row = key0 % p.bs;
    for (int c = 0; c < nch; ++c) {
      tma_load_4d(dst_k + c * (128 * 128) + i * box_rows * 128, map_k, bar_k, c * 64, g.h_kv, row, cblk);
      tma_load_4d(dst_v + c * (128 * 128) + i * box_rows * 128, map_v, bar_v, c * 64, g.h_kv, row, cblk);
    }
  }
}

// Work items.  An item is two 128-row q tiles (A, B) of one request that
// read the same kv head: with an even group size G, the same q rows of two
// q heads of one kv head ("head pair": both tiles see exactly the same key
// tiles, so the two softmax groups run in step); otherwise two consecutive q
// tiles of one q head ("tile pair"); `mode` bit 0 selects head pairs.
// Items enumerate heads fastest, then requests, then the q-row slots from the
// last (longest) down, for one CTA per item scheduled by the hardware (the
// longest start first); or, for the persistent schedule (`mode` bit 1),
// heads fastest, then slots from the first, then requests, which spreads
// each request's items, and the empty slots past its end, evenly over the
// CTAs' fixed strides.
//
// The per-request values an item's geometry is computed from are loaded in
// one batch of independent loads (issued where pf_geom_load is called, so
// that their latency can overlap other work before pf_geom_finish).
struct PfRaw {
  int b, h, slot, c0, c1, q, lk, r0, r1;
};

__device__ __forceinline__ PfRaw pf_geom_load(const AttnParams& p, int item, int n_slots, int mode) {
  PfRaw r;
  const int hn = (mode & 1) ? p.H_q / 2 : p.H_q;   // head slots per request
  if (mode & 2) {
    const int rest = item / hn;
    r.h = item - rest * hn;
    r.b = rest / n_slots;
    r.slot = rest - r.b * n_slots;
  } else {
    const int per_slot = hn * p.B;
    const int pz = item / per_slot, rem = item - pz * per_slot;
    r.b = rem / hn;
    r.h = rem - r.b * hn;
    r.slot = n_slots - 1 - pz;
  }
  r.c0 = ld_early(p.cu + r.b);
  r.c1 = ld_early(p.cu + r.b + 1);
  r.q = ld_early(p.seqlens_q + r.b);
  r.lk = ld_early(p.seqlen_k + r.b);
  r.r0 = p.kv_range ? ld_early(p.kv_range + 2 * r.b) : 0;
  r.r1 = p.kv_range ? ld_early(p.kv_range + 2 * r.b + 1) : INT_MAX;
  return r;
}

// Geometry of a work item.  Returns false for an empty item.
__device__ __forceinline__ bool pf_geom_finish(const AttnParams& p, const PfRaw& r, int max_tiles, int mode,
                                               PfGeom& g) {
  g.b = r.b;
  int start = r.c0;   // the request's first token, as sanitised_start forms it
  if (!(r.q > 0 && (long long)r.c1 - r.c0 == r.q)) {
    start = 0;
    for (int i = 0; i < g.b; ++i) start += max(p.seqlens_q[i], 0);
  }
  g.t_begin = clampi(start, 0, p.T);
  g.q_len = clampi(r.q, 0, p.T - g.t_begin);
  if (mode & 1) {   // head pair: q heads 2h, 2h + 1 (one kv head, G even), the same rows
    g.hq[0] = 2 * r.h;
    g.hq[1] = 2 * r.h + 1;
    g.q0[0] = g.q0[1] = r.slot * kPfBM;
  } else {    // tile pair: q head h, rows of two consecutive tiles
    g.hq[0] = g.hq[1] = r.h;
    g.q0[0] = r.slot * 2 * kPfBM;
    g.q0[1] = g.q0[0] + kPfBM;
  }
  if (g.q0[0] >= g.q_len) return false;
  g.rows[0] = min(kPfBM, g.q_len - g.q0[0]);
  g.rows[1] = max(0, min(kPfBM, g.q_len - g.q0[1]));
  g.L = max(r.lk + 1, 0);
  g.past = max(g.L - g.q_len, 0);
  g.h_kv = g.hq[0] / p.G;
  const int last_row = g.rows[1] > 0 ? g.q0[1] + g.rows[1] - 1 : g.q0[0] + g.rows[0] - 1;
  const int p_first = g.past + g.q0[0];
  const int p_last = g.past + last_row;
  g.rlo = max(r.r0, 0);
  const int rhi = r.r1;
  g.k_first = max(p.window > 0 ? max(0, p_first - p.window + 1) : 0, g.rlo);
  g.k_lo = (g.k_first / kPfBN) * kPfBN;
  g.k_hi = min(min(p_last + 1, g.L), rhi);
  g.ntiles = g.k_hi > g.k_lo ? (g.k_hi - g.k_lo + kPfBN - 1) / kPfBN : 0;
  g.ntiles = min(g.ntiles, max_tiles);
  for (int t = 0; t < 2; ++t) {
    g.j_lo[t] = g.j_hi[t] = 0;
    if (g.rows[t] <= 0) continue;
    const int lo_row = g.past + g.q0[t], hi_row = lo_row + g.rows[t] - 1;
    const int first = max(p.window > 0 ? max(0, lo_row - p.window + 1) : 0, g.rlo);
    const int hi = min(hi_row + 1, g.k_hi);
    if (hi <= first) continue;
    g.j_lo[t] = min((first - g.k_lo) / kPfBN, g.ntiles);
    g.j_hi[t] = max(min((hi - g.k_lo + kPfBN - 1) / kPfBN, g.ntiles), g.j_lo[t]);
  }
  return true;
}

__device__ __forceinline__ bool pf_geom(const AttnParams& p, int item, int n_slots, int max_tiles, int mode,
                                        PfGeom& g) {
  return pf_geom_finish(p, pf_geom_load(p, item, n_slots, mode), max_tiles, mode, g);
}

// Items: one CTA per item (grid = items), or persistent with a static
// stride (items blockIdx.x, blockIdx.x + gridDim.x, ...), or persistent with
// a dynamic schedule (`mode` bit 2, a work counter in the workspace): every
// CTA starts with item blockIdx.x, then its producer thread claims items
// gridDim.x + atomicAdd(counter, 1) as it needs them and publishes them, two
// ahead, through a ring of kPfRing slots in shared memory (bar_if: slot
// written, bar_ie: slot read by the MMA thread and the 8 softmax warps);
// every role reads the same sequence, ended by -1.  The last CTA to finish
// puts the counter back to zero.
// The K/V ring and every barrier's phases run on across items (phases come
// from counters, not step indices); the next item's Q is loaded as soon as
// the current item's last P has been observed (its S MMAs are complete), and
// a tile's first PV of an item waits until the softmax group has read the
// previous item's O out of TMEM (bar_e).
template <typename T, int D, bool DYN>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_tcgen05_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o, int n_slots, int mode, int box_rows,
                       int box_shift, int max_tiles, int n_items) {
  using C = PfCfg<D>;
  constexpr uint32_t FMT = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t IDESC_S = idesc_f16(FMT, kPfBM, kPfBN, 0);
  constexpr uint32_t IDESC_O = idesc_f16(FMT, kPfBM, D, 1);
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_trigger();
  SPA_PF_STAMP(tid == 0, 0);

  unsigned char* const sQ = smem + C::OFF_Q;   // Q tile t of buffer qb at sQ + (2 qb + t) TILE
  unsigned char* sK = smem + C::OFF_K;
  unsigned char* sV = smem + C::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  constexpr int NS = C::NST;
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_kf = bars + 1;               // [NS] K stage full
  uint64_t* bar_vf = bar_kf + NS;            // [NS] V stage full
  uint64_t* bar_ke = bar_vf + NS;            // [NS] K/V stage empty (every MMA reading it is complete)
  uint64_t* bar_s = bar_ke + NS;             // [2] S of tile A / B written
  uint64_t* bar_o = bar_s + 2;               // [2] PV of tile A / B done
  uint64_t* bar_p = bar_o + 2;               // [2] P of tile A / B in TMEM (4 warps arrive)
  uint64_t* bar_e = bar_p + 2;               // [2] O of tile A / B read out by its epilogue (4 warps arrive)
  uint64_t* bar_if = bar_e + 2;              // [kPfRing] item slot written (producer)
  uint64_t* bar_ie = bar_if + kPfRing;       // [kPfRing] item slot read (MMA thread + 8 softmax warps)
  volatile int* ring = reinterpret_cast<volatile int*>(smem + C::OFF_RING);
  constexpr bool dyn = DYN;   // `mode` bit 2 (the instance without it carries none of its code)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(bar_kf + i, 1);
      mbar_init(bar_vf + i, 1);
      mbar_init(bar_ke + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s + i, 1);
      mbar_init(bar_o + i, 1);
      mbar_init(bar_p + i, 4);
      mbar_init(bar_e + i, 4);
    }
    for (int i = 0; i < kPfRing; ++i) {
      mbar_init(bar_if + i, 1);
      mbar_init(bar_ie + i, 9);
    }
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, kPfTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  int bits = 0;
  int kv_issued = 0;   // K/V tiles the producer has issued (its thread only)
  // test hook: the MMA thread's waits for P give up after a few polls, and
  // softmax warp 0 drops its first arrival (see AttnParams::test_expire_wait)
  const uint32_t p_wait_limit = p.test_expire_wait ? 256u : kPfWaitLimit;

  // the next item, from `item` on, with key tiles (others need no tensor work)
  auto next_work = [&](int& item, PfGeom& gg) {
    while (item < n_items && !(pf_geom(p, item, n_slots, max_tiles, mode, gg) && gg.ntiles > 0)) item += gridDim.x;
    return item < n_items;
  };
  // registers: warpgroup 2 (issue: warps 8-11) releases, the softmax
  // warpgroups take them, each at the head of its role's code
  if (warp >= 10) {
    setmaxnreg_dec<kPfIssueRegs>();
  } else if (warp == 9) {
    setmaxnreg_dec<kPfIssueRegs>();
    // =================== K/V producer: the NS-stage ring over the CTA's key tiles ===================
    // Tile c of the stream goes to stage c % NS once the MMAs of tile c - NS
    // are complete (bar_ke), so the loads run ahead of the MMA warp.
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int c = 0;
      bool ok = true;
      int item = blockIdx.x;
      PfGeom g;
      // dynamic schedule: claim items (from `it` on; -1: from the counter)
      // until one has q rows, or -1 when none is left.  Items without key
      // tiles are published too: the softmax warps write their rows.
      const int hn = (mode & 1) ? p.H_q / 2 : p.H_q;
      auto claim = [&](int it) -> int {
        PfGeom gg;
        for (;;) {
          if (it < 0) it = (int)gridDim.x + atomicAdd(p.ws_count, 1);
          if (it >= n_items) return -1;
          const PfRaw r = pf_geom_load(p, it, n_slots, mode);
          if (pf_geom_finish(p, r, max_tiles, mode, gg)) {
            return it;
          } else {
            // past the request's last q rows: so are the request's other heads
            // at this slot and, in request-major order, its later slots
            const int skip = (mode & 2) ? (r.b + 1) * n_slots * hn : (it / hn + 1) * hn;
            atomicMax(p.ws_count, skip - (int)gridDim.x);
          }
          it = -1;
        }
      };
      int k_pub = 0;   // items published
      auto publish = [&](int it) {
        const int sl = k_pub % kPfRing;
        if (k_pub >= kPfRing) ok = ok && mbar_wait(bar_ie + sl, ((k_pub / kPfRing) - 1) & 1, kPfWaitLimit, abort_flag);
        if (!ok) return;
        ring[sl] = it;
        mbar_arrive(bar_if + sl);
        ++k_pub;
      };
      int nxt = -1, nnx = -1;
      if (dyn) {
        item = claim((int)blockIdx.x < n_items ? (int)blockIdx.x : n_items);
        publish(item);
        if (item >= 0) {
          nxt = claim(-1);
          publish(nxt);
        }
      }
      while (ok && (dyn ? (item >= 0 && pf_geom(p, item, n_slots, max_tiles, mode, g)) : next_work(item, g))) {
        if (dyn && g.ntiles == 0 && nxt >= 0) {   // no tiles to issue: keep two items published ahead now
          nnx = claim(-1);
          publish(nnx);
        }
        for (int j = 0; j < g.ntiles && ok; ++j) {
          const int st = c % NS;
          const PfIds ids = pf_kv_ids(p, g, g.k_lo + j * kPfBN, box_rows);
          if (c >= NS) ok = mbar_wait(bar_ke + st, ((c / NS) - 1) & 1, kPfWaitLimit, abort_flag);
          if (!ok) break;
          pf_issue_kv(p, g, ids, &tm_k, &tm_v, sK + st * C::TILE, sV + st * C::TILE, bar_kf + st, bar_vf + st,
                      g.k_lo + j * kPfBN, box_rows, C::NCH, bits, C::TX_TILE);
          SPA_PF_STAMP(c < 4, 40 + c);   // K/V tile c of the CTA's stream issued
          kv_issued = ++c;
          if (dyn && j == 0 && nxt >= 0) {   // keep two items published ahead
            nnx = claim(-1);
            publish(nnx);
          }
        }
        if (dyn) {
          item = nxt;
          nxt = nnx;
          nnx = -1;
        } else {
          item += gridDim.x;
        }
      }
      if (!ok) {   // the copies still in flight land before the CTA leaves (bounded)
        *abort_flag = 1;
        bits |= SPA_ST_TIMEOUT;
        for (int k = c >= NS ? c - NS : 0; k < c; ++k) {
          mbar_wait(bar_kf + k % NS, (k / NS) & 1, kPfWaitLimit);
          mbar_wait(bar_vf + k % NS, (k / NS) & 1, kPfWaitLimit);
        }
      }
    }
  } else if (warp == 8) {
    setmaxnreg_dec<kPfIssueRegs>();
    // =================== MMA issuer and Q loads (one thread) ===================
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      // Q of an item into buffer qb (completes one phase of bar_q; at most
      // one such phase is outstanding at a time)
      auto issue_q = [&](const PfGeom& gg, int qb) {
        const bool two = gg.rows[1] > 0;
        unsigned char* const dq = sQ + 2 * qb * C::TILE;
        mbar_arrive_expect_tx(bar_q, (two ? 2 : 1) * C::TX_TILE);
        for (int c = 0; c < C::NCH; ++c) {
          tma_load_3d(dq + c * C::CHUNK, &tm_q, bar_q, c * 64, gg.hq[0], gg.t_begin + gg.q0[0]);
          if (two)
            tma_load_3d(dq + C::TILE + c * C::CHUNK, &tm_q, bar_q, c * 64, gg.hq[1], gg.t_begin + gg.q0[1]);
        }
      };
      int c_use = 0;                              // key tiles consumed (stream index)
      int q_iss = 0, q_seen = 0;
      int s_iss[2] = {0, 0}, o_iss[2] = {0, 0}, o_seen[2] = {0, 0}, p_seen[2] = {0, 0};
      int e_due[2] = {0, 0}, e_seen[2] = {0, 0}, ke_iss[NS] = {};
      bool ok = true;
      int k_get = 0;   // item slots read (dynamic schedule)
      // the CTA's next item after `it` (first: its first item); false when none is left
      auto take = [&](int& it, PfGeom& gg, bool first) -> bool {
        if (!dyn) {
          if (!first) it += gridDim.x;
          return next_work(it, gg);
        }
        for (;;) {   // items without key tiles need no tensor work
          const int sl = k_get % kPfRing;
          ok = ok && mbar_wait(bar_if + sl, (k_get / kPfRing) & 1, kPfWaitLimit, abort_flag);
          if (!ok) return false;
          it = ring[sl];
          mbar_arrive(bar_ie + sl);
          ++k_get;
          if (it < 0) return false;
          if (pf_geom(p, it, n_slots, max_tiles, mode, gg) && gg.ntiles > 0) return true;
        }
      };
      int ci = blockIdx.x;
      PfGeom g;
      bool have = take(ci, g, true);
      if (have) {
        issue_q(g, 0);
        ++q_iss;
      }
      int cn = ci;     // with two Q buffers: the next item, taken up while this one runs
      PfGeom gn;
      bool have_n = false;
      SPA_PF_STAMP(true, 44);   // first Q issued
      // wait for the outstanding PV of tile t (at most one)
      auto pv_done = [&](int t) {
        while (ok && o_seen[t] < o_iss[t]) {
          ok = mbar_wait(bar_o + t, o_seen[t] & 1, kPfWaitLimit, abort_flag);
          if (ok) ++o_seen[t];
        }
      };
      // S_t = Q_t K^T for the key tile in `stage` (Q from buffer qb)
      auto issue_s = [&](int t, int stage, int qb) {
        tc_fence_after();
        const uint32_t tS = tmem + t * 128;
        unsigned char* const sq = sQ + (2 * qb + t) * C::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk / 4, koff = (kk % 4) * 32;
          const uint64_t ad = smem_desc_sw128(smem_u32(sq + c * C::CHUNK + koff), 16, 1024);
          const uint64_t bd = smem_desc_sw128(smem_u32(sK + stage * C::TILE + c * C::CHUNK + koff), 16, 1024);
          mma_ss(tS, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar_s + t);
        ++s_iss[t];
      };
      // Per step j and q tile t: PV_t(j) as soon as P_t(j) is in TMEM, then
      // S_t(j+1) once PV_t(j) is done -- each softmax group gets its next S
      // without waiting for the other group, so one group's softmax overlaps
      // the other's MMAs.
      while (have && ok) {
        const int ntq = g.rows[1] > 0 ? 2 : 1;
        auto need = [&](int t, int j) { return t ? (j >= g.j_lo[1] && j < g.j_hi[1]) : (j >= g.j_lo[0] && j < g.j_hi[0]); };
        bool pv_any[2] = {false, false};   // a PV of tile t issued in this item
        const int qb = q_seen % C::NQB;    // this item's Q buffer
        {   // step 0: S of every q tile that sees key tile 0 (after the tile's previous PV)
          const int st = c_use % NS;
          const uint32_t ph = (c_use / NS) & 1;
          ok = mbar_wait(bar_kf + st, ph, kPfWaitLimit, abort_flag);
          SPA_PF_STAMP(q_seen < 2, 45 + 2 * q_seen);   // item's first K tile landed
          if (ok) {
            ok = mbar_wait(bar_q, q_seen & 1, kPfWaitLimit, abort_flag);
            SPA_PF_STAMP(q_seen < 2, 46 + 2 * q_seen);   // item's Q landed
            if (ok) ++q_seen;
          }
          for (int t = 0; t < ntq && ok; ++t) {
            if (!need(t, 0)) continue;
            pv_done(t);   // S_t overwrites P_t of the tile's previous step
            if (ok) issue_s(t, st, qb);
          }
        }
        if constexpr (C::NQB == 2) {
          // the other buffer held the previous item's Q, whose S MMAs are all
          // complete (every P of that item was observed): the next item's Q
          // goes there now and lands while this item runs
          if (ok) {
            cn = ci;
            have_n = take(cn, gn, false);
            if (have_n) {
              issue_q(gn, qb ^ 1);
              ++q_iss;
            }
          }
        }
        for (int j = 0; j < g.ntiles && ok; ++j) {
          const int st = c_use % NS;
          const uint32_t ph = (c_use / NS) & 1;
          const bool more = j + 1 < g.ntiles;
          const int st1 = (c_use + 1) % NS;
          const uint32_t ph1 = ((c_use + 1) / NS) & 1;
          bool k_next = false;
          ok = mbar_wait(bar_vf + st, ph, kPfWaitLimit, abort_flag);
          for (int t = 0; t < ntq && ok; ++t) {
            if (need(t, j)) {
              ok = mbar_wait(bar_p + t, p_seen[t] & 1, p_wait_limit, abort_flag);
              if (ok) ++p_seen[t];
              // the first PV of an item overwrites O_t: the previous epilogue must have read it
              while (ok && !pv_any[t] && e_seen[t] < e_due[t]) {
                ok = mbar_wait(bar_e + t, e_seen[t] & 1, kPfWaitLimit, abort_flag);
                if (ok) ++e_seen[t];
              }
              if (!ok) break;
              tc_fence_after();
              const uint32_t tP = tmem + t * 128;
              const uint32_t tO = tmem + 256 + t * 128;
              const uint32_t acc0 = pv_any[t] ? 1u : 0u;
#pragma unroll
              for (int kk = 0; kk < kPfBN / 16; ++kk) {
                const uint64_t bd = smem_desc_sw128(smem_u32(sV + st * C::TILE + kk * 2048), C::CHUNK, 1024);
                if constexpr (kPfLo<T>) {   // P_hi and P_lo of 64-key halves (see the softmax)
                  const uint32_t col = (kk / 4) * 64 + (kk % 4) * 8;
                  mma_ts(tO, tP + col, bd, IDESC_O, kk > 0 ? 1u : acc0);
                  mma_ts(tO, tP + col + 32, bd, IDESC_O, 1u);
                } else {
                  mma_ts(tO, tP + kk * 8, bd, IDESC_O, kk > 0 ? 1u : acc0);
                }
              }
              tc_commit(bar_o + t);
              ++o_iss[t];
              pv_any[t] = true;
            }
            if (t == ntq - 1) {   // every MMA reading this stage is issued: it empties on completion
              tc_commit(bar_ke + st);
              ++ke_iss[st];
            }
            if (more && need(t, j + 1)) {
              if (!k_next) {
                ok = mbar_wait(bar_kf + st1, ph1, kPfWaitLimit, abort_flag);
                k_next = true;
              }
              pv_done(t);   // P_t(j) consumed: S_t(j+1) may overwrite it
              if (ok) issue_s(t, st1, qb);
            }
          }
          if (!ok) break;
          ++c_use;
        }
        if (!ok) break;
        for (int t = 0; t < ntq; ++t)
          if (pv_any[t]) ++e_due[t];
        // every P of this item was observed, so its S MMAs are complete: Q may be replaced
        if constexpr (C::NQB == 2) {
          ci = cn;
          g = gn;
          have = have_n;
        } else {
          have = take(ci, g, false);
          if (have) {
            issue_q(g, 0);
            ++q_iss;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        bits |= SPA_ST_TIMEOUT;
        // drain, bounded: the latest commit of each barrier covers every MMA
        // issued before it; then the Q copies whose arrival was not observed
        for (int t = 0; t < 2; ++t) {
          if (s_iss[t] > 0) mbar_wait(bar_s + t, (s_iss[t] - 1) & 1, kPfWaitLimit);
          if (o_iss[t] > o_seen[t]) mbar_wait(bar_o + t, (o_iss[t] - 1) & 1, kPfWaitLimit);
        }
        for (int q = q_seen; q < q_iss; ++q) mbar_wait(bar_q, q & 1, kPfWaitLimit);
      }
      // the last stage-empty arrivals land before the CTA leaves (bounded)
      for (int st = 0; st < NS; ++st)
        if (ke_iss[st] > 0) mbar_wait(bar_ke + st, (ke_iss[st] - 1) & 1, kPfWaitLimit);
    }
  } else {
    setmaxnreg_inc<kPfSoftmaxRegs>();
    // =================== softmax group t (warps 4t .. 4t+3) ===================
    const int t = warp >> 2;
    const int r = tid & 127;                      // row within the q tile (TMEM lane)
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + t * 128 + lane_off;
    const uint32_t tO = tmem + 256 + t * 128 + lane_off;
    const float sl2 = p.scale_log2;
    int s_seen = 0, o_seen = 0;   // bar_s / bar_o phases this group has consumed
    bool ok = true;
    int n_it = 0;   // items this group has worked on (probe only)
    // probe: softmax thread 0 of group A (base 1) and of group B (base 21), items 0 and 1
    const bool pr = (tid == 0 || tid == 128);
    const int pbase = tid == 0 ? 1 : 21;
    (void)pr;
    (void)pbase;
    // the raw per-request values of the group's next item are loaded ahead
    // (before the current item's epilogue), so that its geometry is ready
    int k_get = 0;   // item slots this warp has read (dynamic schedule)
    // the warp's next item after `prev` (-1: its first), or -1 when none is left
    auto take = [&](int prev) -> int {
      if (!dyn) {
        const int it = prev < 0 ? (int)blockIdx.x : prev + (int)gridDim.x;
        return it < n_items ? it : -1;
      }
      const int sl = k_get % kPfRing;
      const bool got = __all_sync(0xffffffffu, mbar_wait(bar_if + sl, (k_get / kPfRing) & 1, kPfWaitLimit,
                                                         abort_flag));
      if (!got) {
        ok = false;
        return -1;
      }
      const int it = ring[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_ie + sl);
      ++k_get;
      return it;
    };
    int item = take(-1);
    PfRaw raw;
    if (item >= 0) raw = pf_geom_load(p, item, n_slots, mode);
    for (; item >= 0 && ok;) {
      PfGeom g;
      const bool valid = pf_geom_finish(p, raw, max_tiles, mode, g);
      const int item_next = take(item);
      if (!ok) break;
      const int q0_t = t ? g.q0[1] : g.q0[0];
      const int rows_t = t ? g.rows[1] : g.rows[0];
      if (!valid || rows_t <= 0) {
        if (item_next >= 0) raw = pf_geom_load(p, item_next, n_slots, mode);
        item = item_next;
        continue;
      }
      const int prow = g.past + q0_t + r;
      const int p_lo = g.past + q0_t;                         // first row of this tile
      const int p_hi = g.past + q0_t + rows_t - 1;
      float m_used = -INFINITY;   // log2 units
      float l_sum = 0.f;
      const int nbox0 = kPfBN >> box_shift;
      // the key steps this tile sees; the MMA thread issues S and PV for these only
      const int j_lo = t ? g.j_lo[1] : g.j_lo[0], j_hi = t ? g.j_hi[1] : g.j_hi[0];
      int blk_next = j_hi > j_lo ? pf_block_id(p, g.b, g.k_lo + j_lo * kPfBN, lane, nbox0, box_shift) : -1;
      SPA_PF_STAMP(pr && n_it < 2, pbase + n_it * 10);   // item geometry known
      for (int j = j_lo; j < j_hi; ++j) {
        ok = mbar_wait(bar_s + t, s_seen & 1, kPfWaitLimit, abort_flag);
        SPA_PF_STAMP(pr && n_it < 2 && j < 3, pbase + n_it * 10 + 1 + 2 * j);   // S(j) ready
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        ++s_seen;
        tc_fence_after();
        const int kb = g.k_lo + j * kPfBN;
        // which cache blocks of this tile are mapped (bit i: box i; lane i read
        // block i one tile ahead), and does any key of the tile need a mask for
        // any row of this q tile?
        const int nbox = kPfBN >> box_shift;   // <= 8 (block_size >= 16)
        const uint32_t boxmask = __ballot_sync(0xffffffffu, lane < nbox && blk_next >= 0 && blk_next < p.NB);
        if (j + 1 < j_hi) blk_next = pf_block_id(p, g.b, kb + kPfBN, lane, nbox, box_shift);
        const bool all_mapped = boxmask == (1u << nbox) - 1u;
        const bool full = all_mapped && kb + kPfBN - 1 <= p_lo && kb + kPfBN <= g.k_hi &&
                          (p.window <= 0 || kb > p_hi - p.window) && kb >= g.rlo;
        // visibility of key column c (only consulted on tiles that need a mask):
        // the row's causal / window / end-of-keys limits as a column interval
        // [c_lo, c_hi), and the mapped-block bitmask
        const int c_hi = min(min(prow + 1, g.k_hi) - kb, kPfBN);
        const int c_lo = max(p.window > 0 ? max(prow - p.window + 1 - kb, 0) : 0, g.rlo - kb);
        // visibility of the 32 columns of chunk c4 as a bitmask: the row's
        // causal / window / end-of-keys interval and the mapped blocks
        auto chunk_bits = [&](int c4) -> uint32_t {
          const int base = c4 * 32;
          const int lo = clampi(c_lo - base, 0, 32), hi = clampi(c_hi - base, 0, 32);
          uint32_t m = (hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u)) & ~(lo >= 32 ? 0xffffffffu : ((1u << lo) - 1u));
          if (box_shift >= 5) {
            if (!((boxmask >> (base >> box_shift)) & 1u)) m = 0u;
          } else {   // 16-row boxes: two per chunk
            if (!((boxmask >> (base >> 4)) & 1u)) m &= 0xffff0000u;
            if (!((boxmask >> ((base >> 4) + 1)) & 1u)) m &= 0x0000ffffu;
          }
          return m;
        };
        // the whole row of S in registers: four loads, one wait
        uint32_t v[kPfBN];
#pragma unroll
        for (int c4 = 0; c4 < kPfBN / 32; ++c4) tmem_ld32(tS + c4 * 32, v + c4 * 32);
        uint32_t msk[kPfBN / 32];
#pragma unroll
        for (int c4 = 0; c4 < kPfBN / 32; ++c4) msk[c4] = full ? 0xffffffffu : chunk_bits(c4);
        tmem_wait_ld();
        // hidden keys (masked tiles) count as -inf in the max and give p = 0
        if (!full) {
#pragma unroll
          for (int e = 0; e < kPfBN; ++e)
            if (!((msk[e / 32] >> (e % 32)) & 1u)) v[e] = __float_as_uint(-INFINITY);
        }
        // row max in four independent three-input max chains
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int e = 0; e < kPfBN; e += 2) mq[(e / 2) & 3] = fmax3(mq[(e / 2) & 3], u2f(v[e]), u2f(v[e + 1]));
        float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
        SPA_PF_STAMP(tid == 0 && n_it == 0 && j == 1, 51);   // probe: step 1's row max known
        mx *= sl2;   // scores in log2 units (scale > 0)
        // lazy rescale: raise the reference max only when it grows by > 8 (x256).
        // The TMEM loads / stores of O are warp-collective, so the whole warp
        // takes the branch when any of its rows needs it (alpha = 1 otherwise).
        const bool need = mx > m_used + 8.0f;
        const float m_new = need ? mx : m_used;
        const float alpha = need ? ((m_used == -INFINITY) ? 0.f : ex2(m_used - m_new)) : 1.f;
        const bool rescale = j > 0 && __any_sync(0xffffffffu, need && m_used != -INFINITY);
        l_sum *= alpha;
        m_used = m_new;
        const float nm = (m_used == -INFINITY) ? 0.f : -m_used;
        SPA_PF_STAMP(tid == 0 && n_it == 0 && j == 1, 52);   // probe: step 1's rescale decided
        // P = 2^(s*scale - m) (ex2(-inf) = 0 for hidden keys), packed in pairs
        // into the TMEM columns that held the scores: fp16 P of keys hh*64 ..
        // hh*64+63 in columns hh*32 ..; bf16 P_hi and P_lo (residual_pair) in
        // columns hh*64 .. and hh*64+32 ..
        float lq[4] = {0.f, 0.f, 0.f, 0.f};   // four independent sum chains
#pragma unroll
        for (int hh = 0; hh < kPfBN / 64; ++hh) {
          uint32_t pk[32], pl[kPfLo<T> ? 32 : 1];
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const float pa = ex2(fmaf(u2f(v[hh * 64 + e]), sl2, nm));
            const float pb = ex2(fmaf(u2f(v[hh * 64 + e + 1]), sl2, nm));
            lq[(e / 2) & 3] += pa + pb;
            pk[e / 2] = pack_pair<T>(pa, pb);
            if constexpr (kPfLo<T>) pl[e / 2] = residual_pair<T>(pa, pb, pk[e / 2]);
          }
          if constexpr (kPfLo<T>) {
            tmem_st32(tS + hh * 64, pk);
            tmem_st32(tS + hh * 64 + 32, pl);
          } else {
            tmem_st32(tS + hh * 32, pk);
          }
        }
        // O *= alpha before this step's PV accumulates into it (the PV waits
        // for this group's P arrival below)
        if (rescale) {
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(u2f(o[e]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
        }
        l_sum += (lq[0] + lq[1]) + (lq[2] + lq[3]);
        SPA_PF_STAMP(tid == 0 && n_it == 0 && j == 1, 53);   // probe: step 1's P stores issued
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        const bool drop = p.test_expire_wait && warp == 0 && j == 0 && item == (int)blockIdx.x;
        if (lane == 0 && !drop) mbar_arrive(bar_p + t);
        SPA_PF_STAMP(pr && n_it < 2 && j < 3, pbase + n_it * 10 + 2 + 2 * j);   // P(j) handed over
      }
      if (!ok) break;
      if (item_next >= 0) raw = pf_geom_load(p, item_next, n_slots, mode);
      const int hq = g.hq[t];
      const float sink_v = p.sinks ? ld_early(p.sinks + hq) : 0.f;
      // ---- epilogue: wait for the last PV of this tile, normalise with the sink, store
      bool have_o = j_hi > j_lo;
      if (have_o) {
        have_o = mbar_wait(bar_o + t, (o_seen + (j_hi - j_lo) - 1) & 1, kPfWaitLimit, abort_flag);
        o_seen += j_hi - j_lo;
        if (!__all_sync(0xffffffffu, have_o)) {
          ok = false;
          break;
        }
      }
      SPA_PF_STAMP(pr && n_it < 2, pbase + n_it * 10 + 7);   // last PV complete
        tc_fence_after();
        const bool mine = r < rows_t;
        const int tok = g.t_begin + q0_t + r;
        const long long orow = (long long)tok * p.H_q + hq;
        const float sink2 = p.sinks ? sink_v * kLog2e : -INFINITY;
        float a, inv_l, lse;
        finalize_row(m_used, l_sum, sink2, a, inv_l, lse);
        const float f = a * inv_l;
        T* out = static_cast<T*>(p.out) + orow * D;
        // 16-bit output (`mode` bit 3): each warp whose 32 rows are all
        // present writes them to its 128-byte-swizzled 4 KB of the group's
        // staging tile (lane l's 16-byte chunk c at l * 128 + (c ^ (l & 7)) *
        // 16) and its lane 0 stores them with one tiled store, instead of 32
        // rows of scattered stores; no other warp takes part
        const int w4 = warp & 3;
        const bool tma_o = C::NOST > 0 && (mode & 8) && 32 * (w4 + 1) <= rows_t;   // warp-uniform
        unsigned char* const stg = smem + C::OFF_OST + t * C::TILE + w4 * 4096;
        if (tma_o) {
          if (lane == 0) bulk_wait_read0();   // the warp's previous store has read its staging rows
          __syncwarp();
        }
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (have_o) {   // warp-uniform: every lane takes part in the warp-wide load
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
          if (tma_o) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 v;
              v.x = pack_pair<T>(u2f(o[e + 0]) * f, u2f(o[e + 1]) * f);
              v.y = pack_pair<T>(u2f(o[e + 2]) * f, u2f(o[e + 3]) * f);
              v.z = pack_pair<T>(u2f(o[e + 4]) * f, u2f(o[e + 5]) * f);
              v.w = pack_pair<T>(u2f(o[e + 6]) * f, u2f(o[e + 7]) * f);
              const int ch = c * 4 + e / 8;
              *reinterpret_cast<uint4*>(stg + lane * 128 + ((ch ^ (lane & 7)) << 4)) = v;
            }
          } else if (mine && p.out_f32) {
            float* o32 = static_cast<float*>(p.out) + orow * D + c * 32;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(o32 + e) =
                  make_float4(u2f(o[e]) * f, u2f(o[e + 1]) * f, u2f(o[e + 2]) * f, u2f(o[e + 3]) * f);
          } else if (mine) {
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
        if (tma_o) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tm_o, stg, 0, hq, g.t_begin + q0_t + 32 * w4);
            bulk_commit();
          }
        }
        if (mine && p.lse) p.lse[orow] = lse;
      if (j_hi > j_lo) {   // O_t may now be overwritten by the next item
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_e + t);
      }
      SPA_PF_STAMP(pr && n_it < 2, pbase + n_it * 10 + 8);   // epilogue stored
      ++n_it;
      item = item_next;
    }
    if (!ok) *abort_flag = 1;
    if (C::NOST > 0 && lane == 0) bulk_wait0();   // this warp's tiled stores are done
  }
  __syncthreads();
  if (*abort_flag) {
    bits |= SPA_ST_TIMEOUT;
    // another role gave up: the producer's last NS K/V tiles may still be in
    // flight although it finished issuing normally; they land before the CTA
    // leaves (bounded; the latest phase of each stage is unambiguous)
    if (warp == 9 && lane == 0)
      for (int k = kv_issued >= NS ? kv_issued - NS : 0; k < kv_issued; ++k) {
        mbar_wait(bar_kf + k % NS, (k / NS) & 1, kPfWaitLimit);
        mbar_wait(bar_vf + k % NS, (k / NS) & 1, kPfWaitLimit);
      }
  }
  flag(p.status, bits);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kPfTmemCols);
  }
  // dynamic schedule: every role of this CTA is done claiming; the last CTA
  // to get here puts the work counter (and this ticket) back to zero
  if (dyn && tid == 0) {
    __threadfence();
    if (atomicAdd(p.ws_count + 1, 1) == (int)gridDim.x - 1) {
      atomicExch(p.ws_count, 0);
      atomicExch(p.ws_count + 1, 0);
    }
  }
  SPA_PF_STAMP(tid == 0, 50);   // CTA end
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

// Short items (a window of at most two key tiles) run persistently, one CTA
// per SM looping over them (see launch_pf).
static bool pf_persistent(int window) { return window > 0 && window <= 2 * kPfBN; }

// Workspace of a prefill plan: the persistent schedule's work counter and
// its end-of-launch ticket (zero between calls).
size_t prefill_ticket_bytes(const spa_attention_args_t* a) { return pf_persistent(a->window) ? 256 : 0; }

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
  int box_shift = 0;
  while ((1 << box_shift) < box_rows) ++box_shift;
  CUtensorMap tq, tk, tv, to;
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
  // tiled stores of the output, 32 rows of one head per box: 16-bit output
  // (not a shard's fp32 partial) with room for the staging tiles
  const bool tma_out = C::NOST > 0 && !p.out_f32 && (reinterpret_cast<uintptr_t>(p.out) & 15) == 0;
  const cuuint32_t ob[3] = {64, 1, 32};
  to = tq;
  if (tma_out && (rc = encode(&to, dt, 3, p.out, qd, qs, ob)) != SPA_OK) return rc;
  // head pairs when the group size is even, tile pairs otherwise (see pf_geom_load)
  const int hp = (p.G % 2 == 0) ? 1 : 0;
  const int n_slots = hp ? (p.max_q + kPfBM - 1) / kPfBM : (p.max_q + 2 * kPfBM - 1) / (2 * kPfBM);
  const long long items = (long long)(hp ? p.H_q / 2 : p.H_q) * p.B * n_slots;
  if (items > 0x7fffffffLL) return SPA_ERR_UNSUPPORTED;
  const int max_tiles = (p.max_k + kPfBN - 1) / kPfBN + 1;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const bool persistent = pf_persistent(p.window);
  // persistent items are claimed from a counter in the workspace when there is one
  const bool dyn = persistent && p.ws_count != nullptr;
  auto kern = dyn ? prefill_tcgen05_kernel<T, D, true> : prefill_tcgen05_kernel<T, D, false>;
  // the register hand-over (setmaxnreg) balances only at the launch register
  // count it was written for: a build with another count is not launched
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != kPfLaunchRegs) {
    cudaGetLastError();
    return SPA_ERR_UNSUPPORTED;
  }
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  // persistent: one CTA per SM (all of TMEM, over half the shared memory);
  // the item order of each schedule is described at pf_geom_load
  // Short items (a window of at most two key tiles) run persistently, one CTA
  // per SM looping over them, so the per-CTA set-up and pipeline fill are paid
  // once per SM; long causal items keep one CTA each, which the hardware
  // schedules dynamically (a static assignment of the unequal causal items
  // measured slower).
  const int grid = persistent ? (int)std::min<long long>(items, std::max(sms, 1)) : (int)items;
  const int mode = hp | (persistent ? 2 : 0) | (dyn ? 4 : 0) | (tma_out ? 8 : 0);
  return launch_pdl(kern, dim3(grid), dim3(kPfThreads), C::SMEM, stream, p, tq, tk, tv, to, n_slots, mode, box_rows,
                    box_shift, max_tiles, (int)items);
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

#ifdef SPA_PHASE_PROBE
// Probe library only: copy / clear the phase stamps of prefill_tcgen05_kernel.
extern "C" int spa_probe_read_pf(void* host, size_t bytes) {
  if (bytes > sizeof(spa::g_phase_pf)) bytes = sizeof(spa::g_phase_pf);
  return (int)cudaMemcpyFromSymbol(host, spa::g_phase_pf, bytes);
}
extern "C" int spa_probe_clear_pf() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, spa::g_phase_pf) != cudaSuccess) return -1;
  return (int)cudaMemset(p, 0, sizeof(spa::g_phase_pf));
}
#endif
