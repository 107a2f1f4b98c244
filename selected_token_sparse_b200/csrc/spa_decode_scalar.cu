// Steps 3-5 on CUDA cores: gather of the attended keys, scaled QK, online
// max-stable softmax with the learned sink, and split-KV partial states.
//
// This is the fp32 path (its 1e-5 tolerance rules out reduced-precision
// tensor-core inputs) and the general path for units whose rows do not fit
// the tensor-core kernels.  One CTA = one unit (a set of query rows sharing
// one candidate-key list: all G q heads of one kv head, for one token or for
// all tokens of one request) x one split of its candidate list.
//
// Per key tile: 32 threads resolve candidates (selection slot or window
// position -> block table -> cache row, with all guards), the CTA stages the
// K/V rows in shared memory as fp32 (INT8 rows dequantised with their
// per-channel scales), computes the masked scores, updates each row's
// running (max, sum) with one warp per row, and accumulates P.V into
// per-thread registers.  The state is in log2 units (scale * log2 e folded
// in once).  With one split the sink is applied here and the output written
// directly; otherwise FP32 partial states go to the workspace for the
// log-sum-exp combine ("[WebGPU] Add SparsePagedAttention", File summaries:
// main / auxiliary partial FP32 softmax state and finalize merge).
#include "spa_attn.cuh"

namespace spa {

constexpr int kScalarThreads = 256;
constexpr int kScalarKT = 32;
constexpr int kScalarMaxRows = 128;

int scalar_key_tile() { return kScalarKT; }

template <int D>
struct ScalarSmem {
  static size_t bytes(int R, int nq) {
    size_t f = (size_t)R * D + (size_t)kScalarKT * (D + 1) + (size_t)kScalarKT * D +
               (size_t)R * kScalarKT + 3 * (size_t)R;
    size_t i = (size_t)nq + kScalarKT * 2;  // prow, kpos, kaux
    return f * 4 + i * 4 + kScalarKT * 8 + 16;
  }
};

template <typename ActT, typename CacheT, int D>
__global__ void __launch_bounds__(kScalarThreads)
decode_scalar_kernel(const AttnParams p) {
  constexpr int NT = kScalarThreads;
  constexpr int KT = kScalarKT;
  constexpr int NW = NT / 32;
  constexpr int MAXO = kScalarMaxRows * D / NT;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ int last_flag;
  pdl_wait();
  pdl_trigger();

  Unit U;
  const bool has_rows = decode_unit(p, blockIdx.x, U);
  const int split = blockIdx.y;
  int nq = 1;
  if (p.group_by_request) {
    if (!has_rows) return;  // empty request: no rows to write
    nq = U.nq;
  }
  const int G = p.G;
  const int R = nq * G;
  const int t0 = has_rows ? U.t0 : blockIdx.x / p.H_kv;
  const int h_kv = blockIdx.x % p.H_kv;

  // shared-memory carve-up
  float* q_s = reinterpret_cast<float*>(smem_raw);
  float* k_s = q_s + R * D;
  float* v_s = k_s + KT * (D + 1);
  float* p_s = v_s + KT * D;
  float* m_s = p_s + R * KT;
  float* l_s = m_s + R;
  float* al_s = l_s + R;
  int* prow_s = reinterpret_cast<int*>(al_s + R);
  int* kpos_s = prow_s + nq;
  int* kaux_s = kpos_s + KT;
  long long* koff_s = reinterpret_cast<long long*>(
      (reinterpret_cast<uintptr_t>(kaux_s + KT) + 7) & ~uintptr_t(7));

  const ActT* q = static_cast<const ActT*>(p.q);
  for (int e = tid; e < R * D; e += NT) {
    const int r = e / D, d = e % D;
    const int t = t0 + r / G, h = h_kv * G + r % G;
    q_s[e] = to_f32(q[((long long)t * p.H_q + h) * D + d]);
  }
  for (int r = tid; r < R; r += NT) {
    m_s[r] = -INFINITY;
    l_s[r] = 0.f;
  }
  for (int i = tid; i < nq; i += NT) prow_s[i] = has_rows ? U.p_first + i : -1;

  float acc[MAXO];
#pragma unroll
  for (int i = 0; i < MAXO; ++i) acc[i] = 0.f;

  int bits = 0;
  const int n_total = has_rows ? U.n_main + U.n_aux : 0;
  const int c_begin = split * p.split_len;
  const int c_end = min(c_begin + p.split_len, n_total);
  const CacheT* kc = static_cast<const CacheT*>(p.k_cache);
  const CacheT* vc = static_cast<const CacheT*>(p.v_cache);
  const CacheT* ak = static_cast<const CacheT*>(p.aux_k);
  const CacheT* av = static_cast<const CacheT*>(p.aux_v);
  const bool int8 = sizeof(CacheT) == 1;
  __syncthreads();

  for (int ct = c_begin; ct < c_end; ct += KT) {
    if (tid < KT) {
      const int c = ct + tid;
      int kp = kPosInvalid;
      bool aux = false;
      long long off = -1;
      if (c < c_end) off = resolve_candidate(p, U, c, kp, aux, bits);
      kpos_s[tid] = kp;
      kaux_s[tid] = aux;
      koff_s[tid] = off;
    }
    __syncthreads();
    for (int e = tid; e < KT * D; e += NT) {
      const int k = e / D, d = e % D;
      const long long off = koff_s[k];
      float kv = 0.f, vv = 0.f;
      if (off >= 0) {
        const CacheT* kb = kaux_s[k] ? ak : kc;
        const CacheT* vb = kaux_s[k] ? av : vc;
        kv = to_f32(kb[off + d]);
        vv = to_f32(vb[off + d]);
        if (int8) {
          kv *= p.k_scale[h_kv * D + d];
          vv *= p.v_scale[h_kv * D + d];
        }
      }
      k_s[k * (D + 1) + d] = kv;
      v_s[k * D + d] = vv;
    }
    __syncthreads();
    for (int e = tid; e < R * KT; e += NT) {
      const int r = e / KT, k = e % KT;
      float s = -INFINITY;
      if (key_visible(kpos_s[k], prow_s[r / G], p.window)) {
        float dot = 0.f;
        const float* qr = q_s + r * D;
        const float* kr = k_s + k * (D + 1);
#pragma unroll 16
        for (int d = 0; d < D; ++d) dot = fmaf(qr[d], kr[d], dot);
        s = dot * p.scale_log2;
      }
      p_s[e] = s;
    }
    __syncthreads();
    for (int r = warp; r < R; r += NW) {
      const float s = p_s[r * KT + lane];
      float mx = s;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = m_s[r];
      const float m_new = fmaxf(m_old, mx);
      const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_old - m_new);
      const float pv = (s == -INFINITY) ? 0.f : exp2f(s - m_new);
      p_s[r * KT + lane] = pv;
      float sum = pv;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        l_s[r] = l_s[r] * alpha + sum;
        m_s[r] = m_new;
        al_s[r] = alpha;
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < MAXO; ++i) {
      const int o = tid + i * NT;
      if (o < R * D) {
        const int r = o / D, d = o % D;
        float a = acc[i] * al_s[r];
        const float* pr = p_s + r * KT;
#pragma unroll 8
        for (int k = 0; k < KT; ++k) a = fmaf(pr[k], v_s[k * D + d], a);
        acc[i] = a;
      }
    }
    __syncthreads();
  }
  flag(p.status, bits);

  if (p.num_splits == 1) {
    ActT* out = static_cast<ActT*>(p.out);
#pragma unroll
    for (int i = 0; i < MAXO; ++i) {
      const int o = tid + i * NT;
      if (o < R * D) {
        const int r = o / D, d = o % D;
        const int t = t0 + r / G, h = h_kv * G + r % G;
        const float sink2 = p.sinks ? p.sinks[h] * kLog2e : -INFINITY;
        float a, inv_l, lse;
        finalize_row(m_s[r], l_s[r], sink2, a, inv_l, lse);
        const long long oi = ((long long)t * p.H_q + h) * D + d;
        if (p.out_f32) static_cast<float*>(p.out)[oi] = acc[i] * a * inv_l;
        else out[oi] = from_f32<ActT>(acc[i] * a * inv_l);
        if (d == 0 && p.lse) p.lse[(long long)t * p.H_q + h] = lse;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < MAXO; ++i) {
      const int o = tid + i * NT;
      if (o < R * D) {
        const int r = o / D, d = o % D;
        const int t = t0 + r / G, h = h_kv * G + r % G;
        const long long row = ((long long)split * p.T + t) * p.H_q + h;
        p.ws_acc[row * D + d] = acc[i];
        if (d == 0) {
          p.ws_ml[row * 2 + 0] = m_s[r];
          p.ws_ml[row * 2 + 1] = l_s[r];
        }
      }
    }
    finish_split<ActT, D>(p, blockIdx.x, t0, nq, h_kv, &last_flag);
  }
}

template <typename ActT, typename CacheT, int D>
static int launch_scalar_t(const AttnParams& p, int max_rows, cudaStream_t stream) {
  const int nq = p.group_by_request ? p.max_q : 1;
  const size_t smem = ScalarSmem<D>::bytes(max_rows, nq);
  auto kern = decode_scalar_kernel<ActT, CacheT, D>;
  if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int units = p.group_by_request ? p.B * p.H_kv : p.T * p.H_kv;
  dim3 grid(units, p.num_splits);
  return launch_pdl(kern, grid, dim3(kScalarThreads), smem, stream, p);
}

template <typename ActT, typename CacheT>
static int launch_scalar_d(const AttnParams& p, int max_rows, cudaStream_t stream) {
  if (p.D == 64) return launch_scalar_t<ActT, CacheT, 64>(p, max_rows, stream);
  return launch_scalar_t<ActT, CacheT, 128>(p, max_rows, stream);
}

int launch_attention_scalar_impl(const AttnParams& p, int act, int cache, int max_rows,
                                 cudaStream_t stream) {
  switch (act) {
    case SPA_F32:
      if (cache == SPA_I8) return launch_scalar_d<float, int8_t>(p, max_rows, stream);
      return launch_scalar_d<float, float>(p, max_rows, stream);
    case SPA_F16:
      if (cache == SPA_I8) return launch_scalar_d<__half, int8_t>(p, max_rows, stream);
      return launch_scalar_d<__half, __half>(p, max_rows, stream);
    default:
      if (cache == SPA_I8) return launch_scalar_d<__nv_bfloat16, int8_t>(p, max_rows, stream);
      return launch_scalar_d<__nv_bfloat16, __nv_bfloat16>(p, max_rows, stream);
  }
}

size_t scalar_smem_bytes(int D, int max_rows, int nq) {
  return D == 64 ? ScalarSmem<64>::bytes(max_rows, nq) : ScalarSmem<128>::bytes(max_rows, nq);
}

}  // namespace spa
