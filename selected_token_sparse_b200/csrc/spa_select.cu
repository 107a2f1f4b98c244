// Selection producer: the top_k keys of per-key scores, as the -1 padded,
// increasing selected-index rows that the attention's selected mode reads.
//
// Source: onnxruntime PR #33472, Key Changes (PackedSparseAttentionIndexer:
// QSA scoring and hierarchical / compact TopK selection ahead of
// DynamicSparseAttention) and its experiments note (the compact TopK keeps
// stable keys, causal tails, capacity stride / padding and overflow
// handling).  The pages do not define the score; it is an input.
//
// One CTA of 1024 threads per (row, kv head):
//   1. the row's candidate scores (keys 0..bound) are read once, coalesced,
//      and kept in shared memory as order-preserving 32-bit keys (NaN and
//      -inf, which are never selected, become 0; -0 becomes +0);
//   2. when more than top_k keys are eligible, a radix select over three
//      digits of 11, 11 and 10 bits (a 2048-bin shared histogram per digit)
//      finds the exact k-th largest key T and how many keys equal to T are
//      still to be taken -- the first ones by index (stable);
//   3. a compaction over contiguous per-warp segments (ballot / popc counts,
//      one scan over the 32 warps) writes every kept index at its rank among
//      the kept ones, so the row comes out in increasing index order;
//   4. the rest of the row, up to its capacity sel_width, is -1.
// Rows longer than the shared-memory capacity read their scores again from
// global memory (L2) in every pass instead.
#include "spa_attn.cuh"

namespace spa {

int check_launch_public();

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelStageKeys = 48 * 1024;   // keys kept in shared memory (192 KB)

// Order-preserving key of a score: larger score, larger key; 0 = not eligible.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;                       // -0 ties with +0
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;     // NaN
  if (u == 0xff800000u) return 0u;                    // -inf masks the key
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // >= 0x00800000 for eligible keys
}

constexpr int kSelBins = 2048;   // radix digits of 11, 11 and 10 bits

struct SelShared {
  uint32_t hist[kSelBins];
  int warp_gt[kSelWarps];
  int warp_eq[kSelWarps];
  int red[kSelWarps];
  int digit, above, in_bin;
};

__global__ void __launch_bounds__(kSelThreads, 1)
select_topk_kernel(const float* __restrict__ scores, int H, int n_keys, const int32_t* __restrict__ bound,
                   int top_k, int sel_width, int32_t* __restrict__ out, int staged, int vec) {
  extern __shared__ uint32_t sel_keys[];
  __shared__ SelShared sh;
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long row = blockIdx.x;
  const int r = (int)(row / H);
  const float* src = scores + row * (long long)n_keys;
  int32_t* dst = out + row * (long long)sel_width;
  const int last = min(bound[r], n_keys - 1);
  const int n = last + 1 > 0 ? last + 1 : 0;   // candidate keys 0 .. last

  auto key_at = [&](int j) -> uint32_t { return staged ? sel_keys[j] : score_key(__ldg(src + j)); };

  // 1. stage the keys and count the eligible ones.  Rows whose start is
  // 16-byte aligned are read with 16-byte vectors, eight in flight per thread
  // (a 32768-key row in one batch).
  int elig = 0;
  if (vec) {
    const float4* src4 = reinterpret_cast<const float4*>(src);
    const int n4 = (n + 3) >> 2;
    for (int i0 = 0; i0 < n4; i0 += 8 * kSelThreads) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kSelThreads + tid;
        v[u] = i < n4 ? __ldg(src4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kSelThreads + tid;
        if (i >= n4) continue;
        const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t k[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          k[e] = 4 * i + e < n ? score_key(x[e]) : 0u;   // keys beyond the bound are not candidates
          elig += k[e] != 0u;
        }
        if (staged) *reinterpret_cast<uint4*>(sel_keys + 4 * i) = make_uint4(k[0], k[1], k[2], k[3]);
      }
    }
  } else {
    for (int j0 = 0; j0 < n; j0 += 8 * kSelThreads) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * kSelThreads + tid;
        v[u] = j < n ? __ldg(src + j) : __int_as_float(0xff800000);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * kSelThreads + tid;
        const uint32_t k = score_key(v[u]);
        elig += k != 0u;
        if (staged && j < n) sel_keys[j] = k;
      }
    }
  }
  elig = __reduce_add_sync(0xffffffffu, elig);
  if (lane == 0) sh.red[warp] = elig;
  __syncthreads();
  if (warp == 0) {
    const int e = __reduce_add_sync(0xffffffffu, sh.red[lane]);
    if (lane == 0) sh.red[0] = e;
  }
  __syncthreads();
  const int E = sh.red[0];

  // 2. the threshold: keep keys > T, plus the first need_eq keys equal to T
  uint32_t T = 0u;
  int need_eq = 0;
  if (E > top_k && top_k > 0) {
    uint32_t prefix = 0u, pmask = 0u;
    int k_rem = top_k;
    bool exact = true;
    // digits: bits 31..21, 20..10, 9..0 (the first spreads the sign, the
    // exponent and two mantissa bits over 2048 bins)
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const uint32_t dmask = pass == 2 ? 1023u : 2047u;
      const int nbins = (int)dmask + 1;
      for (int i = tid; i < nbins; i += kSelThreads) sh.hist[i] = 0u;
      __syncthreads();
      for (int j0 = 0; j0 < n; j0 += kSelThreads) {
        const int j = j0 + tid;
        const uint32_t k = j < n ? key_at(j) : 0u;
        if (k != 0u && (k & pmask) == prefix) atomicAdd(&sh.hist[(k >> shift) & dmask], 1u);
      }
      __syncthreads();
      {
        // block-wide: thread t holds the bins nbins-1-bpt*t ... (largest
        // digits first); an inclusive scan over the threads finds the bin
        // where the count of larger keys reaches k_rem
        const int bpt = nbins / kSelThreads;   // 2 or 1
        const int b0 = nbins - 1 - tid * bpt;
        const int c0 = (int)sh.hist[b0];
        const int c1 = bpt == 2 ? (int)sh.hist[b0 - 1] : 0;
        int incl = c0 + c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (lane == 31) sh.red[warp] = incl;
        __syncthreads();
        int before = 0;
        for (int w = 0; w < warp; ++w) before += sh.red[w];
        incl += before;
        const int excl = incl - c0 - c1;
        if (excl < k_rem && k_rem <= incl) {
          if (excl + c0 >= k_rem) {
            sh.digit = b0;
            sh.above = excl;
            sh.in_bin = c0;
          } else {
            sh.digit = b0 - 1;
            sh.above = excl + c0;
            sh.in_bin = c1;
          }
        }
      }
      __syncthreads();
      const int d = sh.digit;
      k_rem -= sh.above;
      prefix |= (uint32_t)d << shift;
      pmask |= dmask << shift;
      if (sh.in_bin == k_rem) {   // every key of this bin is kept: no tie to split
        T = prefix - 1u;          // keys with this prefix are >= prefix
        need_eq = 0;
        exact = false;
        break;
      }
      __syncthreads();            // sh.* is rewritten by the next pass
    }
    if (exact) {
      T = prefix;
      need_eq = k_rem;
    }
  }
  const int kept = E < top_k ? E : top_k;

  // 3. compaction in index order over contiguous per-warp segments
  const int seg = ((n + kSelWarps - 1) / kSelWarps + 31) & ~31;
  const int beg = warp * seg, end = min(beg + seg, n);
  int gt_w = 0, eq_w = 0;
  if (kept > 0) {
    for (int j0 = beg; j0 < end; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t k = j < end ? key_at(j) : 0u;
      gt_w += __popc(__ballot_sync(0xffffffffu, k > T));
      eq_w += __popc(__ballot_sync(0xffffffffu, need_eq > 0 && k == T));
    }
  }
  if (lane == 0) {
    sh.warp_gt[warp] = gt_w;
    sh.warp_eq[warp] = eq_w;
  }
  __syncthreads();
  if (kept > 0) {
    int gt_before = 0, eq_before = 0;
    for (int w = 0; w < warp; ++w) {
      gt_before += sh.warp_gt[w];
      eq_before += sh.warp_eq[w];
    }
    int pos = gt_before + min(eq_before, need_eq);
    int eq_seen = eq_before;
    const unsigned lt = (1u << lane) - 1u;
    for (int j0 = beg; j0 < end; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t k = j < end ? key_at(j) : 0u;
      const bool is_eq = need_eq > 0 && k == T;
      const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
      const bool take = k > T || (is_eq && eq_seen + __popc(eqm & lt) < need_eq);
      const unsigned tm = __ballot_sync(0xffffffffu, take);
      if (take) dst[pos + __popc(tm & lt)] = j;
      pos += __popc(tm);
      eq_seen += __popc(eqm);
    }
  }
  // 4. padding up to the row's capacity
  for (int i = kept + tid; i < sel_width; i += kSelThreads) dst[i] = -1;
}

// ---------------------------------------------------------------------------
// Rows that fit shared memory with 16-byte aligned scores.  Every warp owns a
// contiguous segment of the row (a multiple of 128 keys; each lane takes 4
// consecutive keys per step, so a warp step is 128 keys in index order).
// After the histogram of the first digit, only the keys of the threshold bin
// can change the answer: they go (key, index) to a candidate buffer, and the
// two remaining digits are resolved on that buffer alone.  The per-warp
// counts the final write needs are gathered on the way (keys above the bin in
// the candidate pass, the buffer's keys once the threshold is exact), so the
// row is read from shared memory twice after staging (the first digit's
// histogram is counted while staging): the candidate pass and the write pass.  When the threshold bin
// is larger than the buffer (e.g. all scores equal), the remaining digits and
// the counts run over the whole row instead.
constexpr int kFastStageKeys = 40 * 1024;   // keys staged (160 KB)
constexpr int kFastCand = 4096;             // candidate buffer entries (32 KB)

struct FastShared {
  uint32_t hist[kSelBins];
  uint32_t hist1[kSelBins];   // CTA pair: digit 2's histogram (digit 3 reuses hist)
  uint32_t histc[kSelBins];   // CTA pair: both halves' histogram of the current digit
  int e_loc, peer_gt, peer_eq;
  int warp_el[kSelWarps];
  int warp_gt[kSelWarps];
  int warp_eq[kSelWarps];
  int red[kSelWarps];
  int digit, above, in_bin, nbuf;
};

// inclusive and exclusive warp prefix sums of x
__device__ __forceinline__ int warp_excl_scan(int x, int lane, int& total) {
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  total = __shfl_sync(0xffffffffu, incl, 31);
  return incl - x;
}

// Block-wide search of the histogram bin where the count of larger keys
// reaches k_rem (bins ordered from the largest digit); results in fs.
__device__ __forceinline__ void find_digit(FastShared& fs, const uint32_t* hist, int nbins, int k_rem, int tid,
                                           int lane, int warp) {
  const int bpt = nbins / kSelThreads;   // 2 or 1
  const int b0 = nbins - 1 - tid * bpt;
  const int c0 = (int)hist[b0];
  const int c1 = bpt == 2 ? (int)hist[b0 - 1] : 0;
  int incl = c0 + c1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) fs.red[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += fs.red[w];
  incl += before;
  const int excl = incl - c0 - c1;
  if (excl < k_rem && k_rem <= incl) {
    if (excl + c0 >= k_rem) {
      fs.digit = b0;
      fs.above = excl;
      fs.in_bin = c0;
    } else {
      fs.digit = b0 - 1;
      fs.above = excl + c0;
      fs.in_bin = c1;
    }
  }
  __syncthreads();
}

// The same word of shared memory in the other CTA of a pair (cluster of 2).
__device__ __forceinline__ uint32_t pair_addr(const void* p, uint32_t peer) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n"
               : "=r"(r)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))), "r"(peer));
  return r;
}
__device__ __forceinline__ uint32_t pair_ld(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];\n" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void pair_st(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}

// PAIR: a row's candidates are split over a CTA pair (a cluster of two along
// y; rank = blockIdx.y): each stages and scans its half, the pair exchanges
// every digit's histogram (and the eligible count) through distributed
// shared memory after a cluster barrier, so both take the same digits; at
// the end rank 0 hands its kept counts to rank 1, which writes after them.
// Rows with few (row, kv head) pairs use twice the SMs this way.
template <bool PAIR>
__global__ void __launch_bounds__(kSelThreads, 1)
select_topk_fast_kernel(const float* __restrict__ scores, int H, int n_keys, const int32_t* __restrict__ bound,
                        int top_k, int sel_width, int32_t* __restrict__ out) {
  extern __shared__ __align__(16) uint32_t fast_smem[];
  __shared__ FastShared fs;
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long row = blockIdx.x;
  const int rank = PAIR ? (int)blockIdx.y : 0;
  const uint32_t peer = (uint32_t)(rank ^ 1);
  const int r = (int)(row / H);
  int32_t* dst = out + row * (long long)sel_width;
  const int last = min(bound[r], n_keys - 1);
  const int n_row = last + 1 > 0 ? last + 1 : 0;
  // this CTA's candidates: [lo_c, lo_c + n) of the row (lo_c a multiple of 128)
  const int half = PAIR ? ((((n_row + 1) / 2) + 127) & ~127) : n_row;
  const int lo_c = PAIR ? min(rank * half, n_row) : 0;
  const int n = PAIR ? min(half, n_row - lo_c) : n_row;
  const float4* src4 = reinterpret_cast<const float4*>(scores + row * (long long)n_keys + lo_c);
  uint32_t* keys = fast_smem;                                           // [n_keys or half]
  uint32_t* buf_key = fast_smem + ((PAIR ? half : ((n_keys + 3) & ~3)));   // [kFastCand]
  int* buf_idx = reinterpret_cast<int*>(buf_key + kFastCand);           // [kFastCand]
  const int seg = (((n + kSelWarps - 1) / kSelWarps) + 127) & ~127;     // keys per warp
  const int beg = min(warp * seg, n), end = min(beg + seg, n);
  // both halves' histogram of the digit counted in `h` (PAIR), after a
  // cluster barrier that publishes this CTA's own
  auto combine = [&](const uint32_t* h, int nbins) {
    cluster_sync();
    for (int i = tid; i < nbins; i += kSelThreads) fs.histc[i] = h[i] + pair_ld(pair_addr(h + i, peer));
    __syncthreads();
  };

  // 1. staging: this warp's segment as 16-byte vectors, 8 in flight per lane;
  // the histogram of the first digit (bits 31..21) is counted on the way
  for (int i = tid; i < kSelBins; i += kSelThreads) fs.hist[i] = 0u;
  __syncthreads();
  int elig = 0;
  if (beg < end) {   // (a warp past the row's end has an empty segment)
    const int i_beg = beg >> 2, i_end = (end + 3) >> 2;
    for (int i0 = i_beg; i0 < i_end; i0 += 8 * 32) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * 32 + lane;
        v[u] = i < i_end ? __ldg(src4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * 32 + lane;
        if (i >= i_end) continue;
        const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t k[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          k[e] = 4 * i + e < end ? score_key(x[e]) : 0u;
          elig += k[e] != 0u;
          if (k[e] != 0u) atomicAdd(&fs.hist[k[e] >> 21], 1u);
        }
        *reinterpret_cast<uint4*>(keys + 4 * i) = make_uint4(k[0], k[1], k[2], k[3]);
      }
    }
  }
  elig = __reduce_add_sync(0xffffffffu, elig);
  if (lane == 0) {
    fs.warp_el[warp] = elig;
    fs.warp_gt[warp] = 0;
    fs.warp_eq[warp] = 0;
  }
  if (tid == 0) fs.nbuf = 0;
  __syncthreads();
  int E = 0;
  for (int w = 0; w < kSelWarps; ++w) E += fs.warp_el[w];
  const int E_loc = E;
  if constexpr (PAIR) {
    if (tid == 0) fs.e_loc = E;
    combine(fs.hist, kSelBins);   // its barrier also publishes e_loc
    E += (int)pair_ld(pair_addr(&fs.e_loc, peer));
  }

  // one warp step: the 4 keys of this lane at step start j0 (index order)
  auto lane_keys = [&](int j0, uint32_t (&k)[4]) {
    const int j = j0 + 4 * lane;
    const uint4 v = j < end ? *reinterpret_cast<const uint4*>(keys + j) : make_uint4(0u, 0u, 0u, 0u);
    k[0] = v.x; k[1] = v.y; k[2] = v.z; k[3] = v.w;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (j + e >= end) k[e] = 0u;
  };

  // e-major view of a warp step: key j0 + 32 e + lane (index order is e, then lane)
  const uint32_t lt_mask = (1u << lane) - 1u;
  auto key_e = [&](int j0, int e) -> uint32_t {
    const int j = j0 + 32 * e + lane;
    return j < end ? keys[j] : 0u;
  };

  uint32_t T = 0u;
  int need_eq = 0;
  if (E > top_k && top_k > 0) {
    // 2a. the first digit (its histogram was counted while staging)
    find_digit(fs, PAIR ? fs.histc : fs.hist, kSelBins, top_k, tid, lane, warp);
    const uint32_t d1 = (uint32_t)fs.digit;
    int k_rem = top_k - fs.above;
    const int in1 = fs.in_bin;
    uint32_t prefix = d1 << 21, pmask = 2047u << 21;
    bool exact = true;
    if (in1 == k_rem) {   // the whole bin is kept
      T = prefix - 1u;
      exact = false;
    }
    const bool use_buf = exact && in1 <= kFastCand;
    // 2b. candidate pass: per-warp count of keys above the bin; the bin's
    // keys (key, index) into the buffer
    int gt_above = 0;
    for (int j0 = beg; j0 < end; j0 += 128) {
      uint32_t k[4], bb[4];
      int tot = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        k[e] = key_e(j0, e);
        const uint32_t dg = k[e] >> 21;
        gt_above += (k[e] != 0u && dg > d1) ? 1 : 0;
        bb[e] = __ballot_sync(0xffffffffu, use_buf && k[e] != 0u && dg == d1);
        tot += __popc(bb[e]);
      }
      if (tot > 0) {   // warp-uniform
        int base = 0;
        if (lane == 0) base = atomicAdd(&fs.nbuf, tot);
        base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if ((bb[e] >> lane) & 1u) {
            const int at = base + __popc(bb[e] & lt_mask);
            buf_key[at] = k[e];
            buf_idx[at] = j0 + 32 * e + lane;
          }
          base += __popc(bb[e]);
        }
      }
    }
    gt_above = __reduce_add_sync(0xffffffffu, gt_above);
    __syncthreads();
    const int nb = use_buf ? fs.nbuf : 0;
    // 2c. the remaining digits (bits 20..10, 9..0) on the buffer, or on the
    // whole row when the bin did not fit
    for (int pass = 1; pass < 3 && exact; ++pass) {
      const int shift = pass == 1 ? 10 : 0;
      const uint32_t dmask = pass == 2 ? 1023u : 2047u;
      const int nbins = (int)dmask + 1;
      // PAIR: digit 2 counts into hist1 (the peer may still read digit 1's
      // hist until the barrier in combine), digit 3 into hist again
      uint32_t* h = (PAIR && pass == 1) ? fs.hist1 : fs.hist;
      for (int i = tid; i < nbins; i += kSelThreads) h[i] = 0u;
      __syncthreads();
      if (use_buf) {
        for (int i = tid; i < nb; i += kSelThreads) {
          const uint32_t k = buf_key[i];
          if ((k & pmask) == prefix) atomicAdd(&h[(k >> shift) & dmask], 1u);
        }
      } else {
        for (int j0 = beg; j0 < end; j0 += 128) {
          uint32_t k[4];
          lane_keys(j0, k);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (k[e] != 0u && (k[e] & pmask) == prefix) atomicAdd(&h[(k[e] >> shift) & dmask], 1u);
        }
      }
      __syncthreads();
      if constexpr (PAIR) combine(h, nbins);
      find_digit(fs, PAIR ? fs.histc : h, nbins, k_rem, tid, lane, warp);
      k_rem -= fs.above;
      prefix |= (uint32_t)fs.digit << shift;
      pmask |= dmask << shift;
      if (fs.in_bin == k_rem) {
        T = prefix - 1u;
        exact = false;
      }
      __syncthreads();   // fs is rewritten by the next pass
    }
    if (exact) {
      T = prefix;
      need_eq = k_rem;
    }
    // 2d. per-warp counts of kept-above (> T) and equal (== T) keys
    if (use_buf) {
      if (lane == 0) fs.warp_gt[warp] = gt_above;
      __syncthreads();
      for (int i = tid; i < nb; i += kSelThreads) {
        const uint32_t k = buf_key[i];
        const int w = buf_idx[i] / seg;
        if (k > T) atomicAdd(&fs.warp_gt[w], 1);
        else if (need_eq > 0 && k == T) atomicAdd(&fs.warp_eq[w], 1);
      }
    } else {
      int g = 0, q = 0;
      for (int j0 = beg; j0 < end; j0 += 128) {
        uint32_t k[4];
        lane_keys(j0, k);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          g += k[e] > T ? 1 : 0;
          q += (need_eq > 0 && k[e] == T) ? 1 : 0;
        }
      }
      g = __reduce_add_sync(0xffffffffu, g);
      q = __reduce_add_sync(0xffffffffu, q);
      if (lane == 0) {
        fs.warp_gt[warp] = g;
        fs.warp_eq[warp] = q;
      }
    }
    __syncthreads();
  } else {
    // every eligible key is kept (or none, top_k = 0): keys > 0
    if (lane == 0) fs.warp_gt[warp] = top_k > 0 ? fs.warp_el[warp] : 0;
    __syncthreads();
  }
  const int kept = E < top_k ? E : top_k;
  // PAIR: rank 0's kept-above and equal counts, for rank 1's positions
  int base_gt = 0, base_eq = 0;
  if constexpr (PAIR) {
    if (rank == 0 && tid == 0) {
      int g = 0, q = 0;
      for (int w = 0; w < kSelWarps; ++w) {
        g += fs.warp_gt[w];
        q += fs.warp_eq[w];
      }
      pair_st(pair_addr(&fs.peer_gt, peer), (uint32_t)g);
      pair_st(pair_addr(&fs.peer_eq, peer), (uint32_t)q);
    }
    cluster_sync();   // the last access to the peer's shared memory precedes it
    if (rank == 1) {
      base_gt = fs.peer_gt;
      base_eq = fs.peer_eq;
    }
  }
  (void)E_loc;

  // 3. write pass: kept indices in increasing order
  if (kept > 0) {
    int pos = base_gt, eq_seen = base_eq;
    for (int w = 0; w < warp; ++w) {
      pos += fs.warp_gt[w];
      eq_seen += fs.warp_eq[w];
    }
    pos += min(eq_seen, need_eq);
    for (int j0 = beg; j0 < end; j0 += 128) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t k = key_e(j0, e);
        bool take = k > T;
        uint32_t bt = __ballot_sync(0xffffffffu, take);
        if (need_eq > 0) {   // keys equal to T: the first need_eq of them by index
          const bool eq = k == T;
          const uint32_t be = __ballot_sync(0xffffffffu, eq);
          if (be != 0u) {
            take = take || (eq && eq_seen + __popc(be & lt_mask) < need_eq);
            bt = __ballot_sync(0xffffffffu, take);
            eq_seen += __popc(be);
          }
        }
        if (take) dst[pos + __popc(bt & lt_mask)] = lo_c + j0 + 32 * e + lane;
        pos += __popc(bt);
      }
    }
  }
  // 4. padding up to the row's capacity (shared by the pair)
  for (int i = kept + (PAIR ? rank * kSelThreads : 0) + tid; i < sel_width; i += (PAIR ? 2 : 1) * kSelThreads)
    dst[i] = -1;
}

}  // namespace spa

using namespace spa;

extern "C" int spa_select_topk(const float* scores, int32_t R, int32_t H, int32_t n_keys, const int32_t* bound,
                               int32_t top_k, int32_t sel_width, int32_t* selected_idx, spa_stream_t stream) {
  if (R < 0 || H <= 0 || n_keys < 0 || top_k < 0 || sel_width <= 0 || top_k > sel_width)
    return SPA_ERR_INVALID_ARG;
  if ((long long)R * H > 0x7fffffffLL) return SPA_ERR_INVALID_ARG;
  if (R == 0) return SPA_OK;
  if (!selected_idx || !bound || (n_keys > 0 && !scores)) return SPA_ERR_INVALID_ARG;
  const int staged = n_keys <= kSelStageKeys ? 1 : 0;
  // whole-row 16-byte vectors: every row starts 16-byte aligned
  const int vec = (n_keys % 4 == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0) ? 1 : 0;
  if (vec && n_keys > 0 && n_keys <= kFastStageKeys) {
    // few rows: each row over a CTA pair (twice the SMs, one wave at most)
    const bool pair = 2LL * R * H <= 148 && n_keys >= 2 * 128;
    const size_t keys_smem = pair ? (size_t)((((n_keys + 1) / 2) + 127) & ~127) * 4 : (size_t)((n_keys + 3) & ~3) * 4;
    const size_t fsm = keys_smem + (size_t)kFastCand * 8;
    auto kern = pair ? select_topk_fast_kernel<true> : select_topk_fast_kernel<false>;
    // (the static shared memory counts toward the default 48 KB as well: always opt in)
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsm) != cudaSuccess)
      return check_launch_public();
    const int rc = pair ? launch_pdl_cluster_y(kern, dim3((unsigned)(R * H), 2), dim3(kSelThreads), fsm,
                                               (cudaStream_t)stream, 2, scores, H, n_keys, bound, top_k, sel_width,
                                               selected_idx)
                        : launch_pdl(kern, dim3((unsigned)(R * H)), dim3(kSelThreads), fsm, (cudaStream_t)stream,
                                     scores, H, n_keys, bound, top_k, sel_width, selected_idx);
    if (rc != SPA_OK) return rc;
    return check_launch_public();
  }
  const size_t smem = staged ? (size_t)(n_keys > 0 ? ((n_keys + 3) & ~3) : 4) * sizeof(uint32_t) : 0;
  if (staged && smem > 48 * 1024) {
    if (cudaFuncSetAttribute(select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSelStageKeys * (int)sizeof(uint32_t)) != cudaSuccess)
      return check_launch_public();
  }
  const int rc = launch_pdl(select_topk_kernel, dim3((unsigned)(R * H)), dim3(kSelThreads), smem,
                            (cudaStream_t)stream, scores, H, n_keys, bound, top_k, sel_width, selected_idx, staged,
                            vec);
  if (rc != SPA_OK) return rc;
  return check_launch_public();
}
