// gdn_portable.cu -- CUDA-core: the Gated DeltaNet fork scan, token
// by token, level by level through the tree.
//
// Per head the state S (dv x dk, fp32) follows the gated delta rule
//   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
//   o_t = S_t q_t,   alpha_t = exp(g_t),
// computed as S <- alpha S + (beta v - alpha beta (S k)) k^T.  Rows of S are
// independent (the update mixes columns only), so a CTA owns 32 rows of one
// head's state: 128 threads = 32 rows x 4 column groups, each thread keeping
// dk/4 state entries in registers.
//
// Forking (kongchang.com article on Flide, Gated DeltaNet box; techfi24.com,
// "Exact State Forking"): level 0 runs every root from state_in (the prefix
// scan, done once per request), and writes the root's end state to its
// node-state slot -- the checkpoint.  Level L runs every node of depth L from
// its parent's saved end state, so a branch never recomputes its ancestors and
// siblings never see each other.  Nodes with children save their end state for
// the next level.  Levels are separate launches, ordered by the stream.
#include "common.cuh"

namespace flide {
namespace {

constexpr int kThreads = 128;
constexpr int kRows = 32;  // state rows per CTA

template <typename T>
struct GdnArgs {
  const T *q, *k, *v;
  const float *g, *beta, *state_in;
  T *out;
  float *node_state;
  flide_tree_index x;
  int H, dk, dv, n_slots, level;
};

template <typename T, int DK>
__global__ void __launch_bounds__(kThreads)
gdn_level_kernel(GdnArgs<T> a) {
  constexpr int CPT = DK / 4;       // state entries per thread
  constexpr int TC = (4096 / DK) < 64 ? (4096 / DK) : 64;  // tokens staged per round
  __shared__ __align__(16) float sk[TC][DK];
  __shared__ __align__(16) float sq[TC][DK];
  __shared__ float sv[TC][kRows];
  __shared__ float salpha[TC], sbeta[TC];

  const flide_tree_index &x = a.x;
  if (failed(x.status)) return;
  const int lvl = a.level;
  const int l0 = x.level_ptr[lvl], l1 = x.level_ptr[lvl + 1];
  const int nblk = a.dv / kRows;
  const long items = (long)(l1 - l0) * a.H * nblk;
  const int tid = threadIdx.x;
  const int row = tid >> 2, cg = tid & 3;
  const size_t SS = (size_t)a.dv * a.dk;

  for (long it = blockIdx.x; it < items; it += gridDim.x) {
    const int blk = (int)(it % nblk);
    const int h = (int)((it / nblk) % a.H);
    const int n = x.level_node[l0 + (int)(it / ((long)nblk * a.H))];
    // debug build: node, request and parent index the tree arrays (the whole
    // block takes the same branch: one item per block)
    if (!in_bounds(x.status, x.counts, n, x.counts[FLIDE_CNT_N], 321) ||
        !in_bounds(x.status, x.counts, x.node_req[n], x.R, 322))
      return;
    const int r = x.node_req[n];
    const int vrow = blk * kRows + row;

    // starting state: parent's end state, or the request's state_in
    float S[CPT];
    const float *src = nullptr;
    if (lvl == 0) {
      if (a.state_in) src = a.state_in + ((size_t)r * a.H + h) * SS;
    } else {
      const int pg = x.anc_node[x.anc_ptr[n + 1] - 2];  // parent (global id)
      if (!in_bounds(x.status, x.counts, pg, x.counts[FLIDE_CNT_N], 323)) return;
      const int ps = x.state_slot[pg];
      if (ps < 0 || ps >= a.n_slots) { set_status(x.status, FLIDE_ERR_CAPACITY); return; }
      src = a.node_state + ((size_t)ps * a.H + h) * SS;
    }
#pragma unroll
    for (int i = 0; i < CPT / 4; ++i) {
      float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (src) s4 = *(const float4 *)(src + (size_t)vrow * a.dk + 16 * i + 4 * cg);
      S[4 * i] = s4.x; S[4 * i + 1] = s4.y; S[4 * i + 2] = s4.z; S[4 * i + 3] = s4.w;
    }

    const int t0 = x.node_start[n], t1 = x.node_start[n + 1];
    if (!in_bounds(x.status, x.counts, t0, x.counts[FLIDE_CNT_T] + 1, 324) ||
        !in_bounds(x.status, x.counts, t1, x.counts[FLIDE_CNT_T] + 1, 324))
      return;
    for (int tb = t0; tb < t1; tb += TC) {
      const int cnt = min(TC, t1 - tb);
      __syncthreads();
      for (int e = tid; e < cnt * DK; e += kThreads) {
        const int j = e / DK, c = e % DK;
        const size_t off = ((size_t)(tb + j) * a.H + h) * DK + c;
        sk[j][c] = load_f(a.k + off);
        sq[j][c] = load_f(a.q + off);
      }
      for (int e = tid; e < cnt * kRows; e += kThreads) {
        const int j = e / kRows, rr = e % kRows;
        sv[j][rr] = load_f(a.v + ((size_t)(tb + j) * a.H + h) * a.dv + blk * kRows + rr);
      }
      for (int j = tid; j < cnt; j += kThreads) {
        salpha[j] = expf(a.g[(size_t)(tb + j) * a.H + h]);
        sbeta[j] = a.beta[(size_t)(tb + j) * a.H + h];
      }
      __syncthreads();
      for (int j = 0; j < cnt; ++j) {
        float kk[CPT];
#pragma unroll
        for (int i = 0; i < CPT / 4; ++i) {
          float4 k4 = *(const float4 *)&sk[j][16 * i + 4 * cg];
          kk[4 * i] = k4.x; kk[4 * i + 1] = k4.y; kk[4 * i + 2] = k4.z; kk[4 * i + 3] = k4.w;
        }
        float u0 = 0.f, u1 = 0.f;
#pragma unroll
        for (int i = 0; i < CPT; i += 2) {
          u0 = fmaf(S[i], kk[i], u0);
          u1 = fmaf(S[i + 1], kk[i + 1], u1);
        }
        float u = u0 + u1;
        u += __shfl_xor_sync(0xffffffffu, u, 1);
        u += __shfl_xor_sync(0xffffffffu, u, 2);
        const float alpha = salpha[j], beta = sbeta[j];
        const float coef = beta * sv[j][row] - alpha * beta * u;
#pragma unroll
        for (int i = 0; i < CPT; ++i) S[i] = fmaf(coef, kk[i], alpha * S[i]);
        float o0 = 0.f, o1 = 0.f;
#pragma unroll
        for (int i = 0; i < CPT / 4; ++i) {
          float4 q4 = *(const float4 *)&sq[j][16 * i + 4 * cg];
          o0 = fmaf(S[4 * i], q4.x, o0);
          o1 = fmaf(S[4 * i + 1], q4.y, o1);
          o0 = fmaf(S[4 * i + 2], q4.z, o0);
          o1 = fmaf(S[4 * i + 3], q4.w, o1);
        }
        float o = o0 + o1;
        o += __shfl_xor_sync(0xffffffffu, o, 1);
        o += __shfl_xor_sync(0xffffffffu, o, 2);
        if (cg == 0) store_f(a.out + ((size_t)(tb + j) * a.H + h) * a.dv + vrow, o);
      }
    }

    const int slot = x.state_slot[n];
    if (slot >= 0) {
      if (slot >= a.n_slots) {
        set_status(x.status, FLIDE_ERR_CAPACITY);
      } else {
        float *dst = a.node_state + ((size_t)slot * a.H + h) * SS + (size_t)vrow * a.dk;
#pragma unroll
        for (int i = 0; i < CPT / 4; ++i)
          *(float4 *)(dst + 16 * i + 4 * cg) =
              make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
      }
    }
  }
}

template <typename T, int DK>
int launch_levels(GdnArgs<T> a, cudaStream_t s) {
  for (int lvl = 0; lvl <= a.x.max_depth; ++lvl) {
    a.level = lvl;
    gdn_level_kernel<T, DK><<<148 * 4, kThreads, 0, s>>>(a);
    FLIDE_LAUNCH_CHECK();
  }
  return FLIDE_OK;
}

template <typename T>
int launch_dtype(GdnArgs<T> a, cudaStream_t s) {
  switch (a.dk) {
    case 32: return launch_levels<T, 32>(a, s);
    case 64: return launch_levels<T, 64>(a, s);
    case 128: return launch_levels<T, 128>(a, s);
    case 256: return launch_levels<T, 256>(a, s);
    default: return FLIDE_ERR_SHAPE;
  }
}

template <typename T>
GdnArgs<T> make_args(const void *q, const void *k, const void *v, const float *g,
                     const float *beta, const float *state_in, const flide_tree_index *x,
                     int H, int dk, int dv, void *out, float *node_state, int n_slots) {
  GdnArgs<T> a;
  a.q = (const T *)q; a.k = (const T *)k; a.v = (const T *)v;
  a.g = g; a.beta = beta; a.state_in = state_in;
  a.out = (T *)out; a.node_state = node_state; a.x = *x;
  a.H = H; a.dk = dk; a.dv = dv; a.n_slots = n_slots; a.level = 0;
  return a;
}

}  // namespace

int fork_gdn_portable(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, const float *state_in, const flide_tree_index *x,
                      int H, int dk, int dv, int dtype, void *out, float *node_state,
                      int n_slots, cudaStream_t s) {
  if (dv <= 0 || dv % kRows != 0) return FLIDE_ERR_SHAPE;
  if (dtype == FLIDE_F32)
    return launch_dtype(make_args<float>(q, k, v, g, beta, state_in, x, H, dk, dv, out,
                                         node_state, n_slots), s);
  if (dtype == FLIDE_BF16)
    return launch_dtype(make_args<__nv_bfloat16>(q, k, v, g, beta, state_in, x, H, dk, dv,
                                                 out, node_state, n_slots), s);
  return FLIDE_ERR_SHAPE;
}

}  // namespace flide
