// attn_portable.cu -- CUDA-core: fork attention for any head dim
// (multiple of 32, <= 256) in fp32 or bf16.  The fp32 workloads run here; the
// bf16 d=128 workloads run the tensor-core kernel in attn_tc.cu.
//
// One warp per (query token, query head).  The warp walks exactly the key
// spans of the token's isolated sequence (kongchang.com article on Flide,
// "ForkAttention" section; attention-mask section: no key of another branch):
//   1. the request's past rows (checkpointed history),
//   2. every token of each strict ancestor, root first (anc CSR row),
//   3. the node's own tokens up to and including the query (causal, diagonal
//      included).
// Keys are taken 32 at a time (one per lane) with an fp32 online softmax in
// the exp2 domain; each lane owns d/32 output dims.
#include "common.cuh"

namespace flide {
namespace {

constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T>
struct PortableArgs {
  const T *q, *k, *v, *pk, *pv;
  T *out;
  flide_tree_index x;
  int Hq, Hkv, d;
  int past_rows;  // rows of the packed past buffers
  float qscale;   // scale * log2(e)
};

template <typename T>
__device__ __forceinline__ void attend_span(const PortableArgs<T> &a, const T *kb,
                                            const T *vb, int row0, int len, int kvh,
                                            const float *qs, float &m, float &l,
                                            float (&acc)[8]) {
  const int lane = threadIdx.x & 31;
  const int nd = a.d >> 5;
  for (int j0 = 0; j0 < len; j0 += 32) {
    const int j = j0 + lane;
    const bool valid = j < len;
    float s = -INFINITY;
    if (valid) {
      const T *kr = kb + ((size_t)(row0 + j) * a.Hkv + kvh) * a.d;
      float dot = 0.f;
      for (int c = 0; c < a.d; ++c) dot = fmaf(qs[c], load_f(kr + c), dot);
      s = dot;
    }
    const float m_new = fmaxf(m, warp_max(s));
    const float corr = (m == -INFINITY) ? 0.f : exp2f(m - m_new);
    const float p = valid ? exp2f(s - m_new) : 0.f;
    l = l * corr + warp_sum(p);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= corr;
    const int cnt = min(32, len - j0);
    for (int jj = 0; jj < cnt; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const T *vr = vb + ((size_t)(row0 + j0 + jj) * a.Hkv + kvh) * a.d;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i < nd) acc[i] = fmaf(pj, load_f(vr + lane + 32 * i), acc[i]);
    }
    m = m_new;
  }
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
attn_portable_kernel(PortableArgs<T> a) {
  extern __shared__ float q_smem[];
  const flide_tree_index &x = a.x;
  if (failed(x.status)) return;
  const int T_act = x.counts[FLIDE_CNT_T];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float *qs = q_smem + warp * a.d;
  const int G = a.Hq / a.Hkv;
  const long rows = (long)T_act * a.Hq;
  for (long row = (long)blockIdx.x * kWarps + warp; row < rows; row += (long)gridDim.x * kWarps) {
    const int t = (int)(row / a.Hq), h = (int)(row % a.Hq);
    const int kvh = h / G;
    const int Nact = x.counts[FLIDE_CNT_N];
    // debug build: the token's node and request index the tree arrays
    const int n = x.token_node[t];
    if (!in_bounds(x.status, x.counts, n, Nact, 301) ||
        !in_bounds(x.status, x.counts, x.node_req[n], x.R, 302))
      continue;
    const int r = x.node_req[n];
    __syncwarp();
    for (int c = lane; c < a.d; c += 32)
      qs[c] = load_f(a.q + ((size_t)t * a.Hq + h) * a.d + c) * a.qscale;
    __syncwarp();
    float m = -INFINITY, l = 0.f;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    // 1. past rows of the request
    const int p0 = x.past_start[r], plen = x.past_start[r + 1] - p0;
    if (plen > 0) {
      if (!a.pk) {
        set_status(x.status, FLIDE_ERR_SHAPE);
        continue;
      }
      if (p0 < 0 || (long)p0 + plen > a.past_rows) {  // past buffers shorter than the tree's past
        set_status(x.status, FLIDE_ERR_CAPACITY);
        continue;
      }
      attend_span(a, a.pk, a.pv, p0, plen, kvh, qs, m, l, acc);
    }
    // 2. strict ancestors, root first
    const int a0 = x.anc_ptr[n], a1 = x.anc_ptr[n + 1] - 1;
    for (int i = a0; i < a1; ++i) {
      const int an = x.anc_node[checked(x.status, x.counts, i, (long long)x.N * (x.max_depth + 1), 303)];
      if (!in_bounds(x.status, x.counts, an, Nact, 304)) continue;
      const int s0 = x.node_start[an], sl = x.node_start[an + 1] - s0;
      if (sl > 0) attend_span(a, a.k, a.v, s0, sl, kvh, qs, m, l, acc);
    }
    // 3. own node up to and including t
    const int own0 = x.node_start[n];
    attend_span(a, a.k, a.v, own0, t - own0 + 1, kvh, qs, m, l, acc);
    const float inv = 1.f / l;
    T *o = a.out + ((size_t)t * a.Hq + h) * a.d;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < (a.d >> 5)) store_f(o + lane + 32 * i, acc[i] * inv);
  }
}

template <typename T>
int launch(const void *q, const void *k, const void *v, const void *pk, const void *pv,
           int past_rows, const flide_tree_index *x, int Hq, int Hkv, int d, float scale,
           void *out, cudaStream_t s) {
  PortableArgs<T> a;
  a.q = (const T *)q; a.k = (const T *)k; a.v = (const T *)v;
  a.pk = (const T *)pk; a.pv = (const T *)pv; a.out = (T *)out;
  a.x = *x; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.past_rows = pk ? past_rows : 0;
  a.qscale = scale * kLog2e;
  long rows = (long)x->T * Hq;
  long blocks = (rows + kWarps - 1) / kWarps;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  attn_portable_kernel<T><<<(int)blocks, kWarps * 32, kWarps * d * sizeof(float), s>>>(a);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}

}  // namespace

int fork_attn_portable(const void *q, const void *k, const void *v, const void *pk,
                       const void *pv, int past_rows, const flide_tree_index *x, int Hq,
                       int Hkv, int d, int dtype, float scale, void *out, cudaStream_t s) {
  if (d <= 0 || d % 32 != 0 || d > 256) return FLIDE_ERR_SHAPE;
  if (dtype == FLIDE_F32) return launch<float>(q, k, v, pk, pv, past_rows, x, Hq, Hkv, d, scale, out, s);
  if (dtype == FLIDE_BF16)
    return launch<__nv_bfloat16>(q, k, v, pk, pv, past_rows, x, Hq, Hkv, d, scale, out, s);
  return FLIDE_ERR_SHAPE;
}

}  // namespace flide
