// state.cu -- checkpoint save and resume.
//
// A growing agent history resumes from checkpoints saved by earlier passes
// instead of being recomputed (kongchang.com article on Flide, "ForkAttention"
// section; techfi24.com, "Exact State Forking": the state at a decision point
// is copied, not rebuilt).  For attention the checkpoint is the K/V rows of
// the shared prefix (past rows followed by the root's rows); for Gated DeltaNet
// it is the fp32 state after the root's last token.  Both are plain device
// copies with 16-byte vector accesses.
#include "common.cuh"

namespace flide {
namespace {

constexpr int kMaxResumeR = 4096;

__device__ __forceinline__ int upper_bound_i(const int32_t *a, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (a[mid] > key) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Copies `bytes` (multiple of 16) from src to dst with 16-byte accesses,
// spread over the threads of one warp-group-sized loop.
__device__ __forceinline__ void copy_row(char *dst, const char *src, int bytes, int lane,
                                         int nthreads) {
  for (int b = lane * 16; b < bytes; b += nthreads * 16)
    *(int4 *)(dst + b) = *(const int4 *)(src + b);
}

__global__ void save_kv_kernel(flide_tree_index x, const char *k, const char *v,
                               const char *pk, const char *pv, int row_bytes, char *ck,
                               char *cv, int ckpt_rows) {
  if (failed(x.status)) return;
  const int C = x.counts[FLIDE_CNT_CKPT_ROWS];
  if (C > ckpt_rows) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(x.status, FLIDE_ERR_CAPACITY);
    return;
  }
  const int R = x.R;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (int i = warp; i < C; i += nwarps) {
    const int r = upper_bound_i(x.ckpt_start, R + 1, i) - 1;
    if (!in_bounds(x.status, x.counts, r, R, 401)) continue;  // debug build
    const int o = i - x.ckpt_start[r];
    const int plen = x.past_start[r + 1] - x.past_start[r];
    const char *sk, *sv;
    if (o < plen) {
      sk = pk + (size_t)(x.past_start[r] + o) * row_bytes;
      sv = pv + (size_t)(x.past_start[r] + o) * row_bytes;
    } else {
      // the root is the first node of the request
      int root = -1;
      // the request owns at least one node here (it has root rows)
      root = upper_bound_i(x.node_req, x.counts[FLIDE_CNT_N], r - 1);
      if (!in_bounds(x.status, x.counts, root, x.counts[FLIDE_CNT_N], 402) ||
          !in_bounds(x.status, x.counts, (long long)x.node_start[root] + (o - plen), x.counts[FLIDE_CNT_T], 403))
        continue;  // debug build: the root row lies in the stream
      const size_t t = (size_t)x.node_start[root] + (o - plen);
      sk = k + t * row_bytes;
      sv = v + t * row_bytes;
    }
    copy_row(ck + (size_t)i * row_bytes, sk, row_bytes, lane, 32);
    copy_row(cv + (size_t)i * row_bytes, sv, row_bytes, lane, 32);
  }
}

__global__ void save_state_kernel(flide_tree_index x, const float *node_state, int H,
                                  int SS, float *ckpt_S) {
  if (failed(x.status)) return;
  const int R = x.R;
  const int N = x.counts[FLIDE_CNT_N];
  const long per_req = (long)H * SS / 4;  // float4 units
  const long total = (long)R * per_req;
  for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long)gridDim.x * blockDim.x) {
    const int r = (int)(e / per_req);
    const long w = e % per_req;
    // root = first node whose request is r (node_req is non-decreasing)
    const int root = upper_bound_i(x.node_req, N, r - 1);
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (root < N && x.node_req[root] == r) {
      const int slot = x.state_slot[root];
      // debug build: the root's slot lies in the node-state buffer the tree needs
      if (in_bounds(x.status, x.counts, slot, x.counts[FLIDE_CNT_SLOTS], 404))
        val = ((const float4 *)(node_state + (size_t)slot * H * SS))[w];
    }
    ((float4 *)(ckpt_S + (size_t)r * H * SS))[w] = val;
  }
}

__global__ void resume_kernel(int R, const int32_t *src_req, int src_R,
                              const int32_t *src_start, const char *sk, const char *sv,
                              const float *sS, int row_bytes, int H, int SS,
                              int32_t *past_len, char *pk, char *pv, int past_rows,
                              float *state_in, int32_t *status) {
  __shared__ int32_t off[kMaxResumeR + 1];
  __shared__ int scratch[40];
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  int carry = 0;
  for (int b = 0; b < R; b += blockDim.x) {
    const int r = b + threadIdx.x;
    int len = 0;
    if (r < R) {
      const int s = src_req[r];
      if (s >= src_R) s_bad = FLIDE_ERR_INVALID;
      else if (s >= 0) len = src_start[s + 1] - src_start[s];
    }
    int tot;
    const int ex = block_excl_scan(len, scratch, &tot);
    if (r < R) off[r] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) off[R] = carry;
  __syncthreads();
  if (s_bad || carry > past_rows) {
    if (blockIdx.x == 0 && threadIdx.x == 0)
      set_status(status, s_bad ? s_bad : FLIDE_ERR_CAPACITY);
    return;
  }
  if (blockIdx.x == 0)
    for (int r = threadIdx.x; r < R; r += blockDim.x) past_len[r] = off[r + 1] - off[r];
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (int i = warp; i < carry; i += nwarps) {
    const int r = upper_bound_i(off, R + 1, i) - 1;
    const size_t srow = (size_t)src_start[src_req[r]] + (i - off[r]);
    copy_row(pk + (size_t)i * row_bytes, sk + srow * row_bytes, row_bytes, lane, 32);
    copy_row(pv + (size_t)i * row_bytes, sv + srow * row_bytes, row_bytes, lane, 32);
  }
  if (state_in) {
    const long per_req = (long)H * SS / 4;
    for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < (long)R * per_req;
         e += (long)gridDim.x * blockDim.x) {
      const int r = (int)(e / per_req);
      const int s = src_req[r];
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s >= 0) val = ((const float4 *)(sS + (size_t)s * H * SS))[e % per_req];
      ((float4 *)(state_in + (size_t)r * H * SS))[e % per_req] = val;
    }
  }
}

}  // namespace

int state_save(const flide_tree_index *x, const void *k, const void *v, const void *pk,
               const void *pv, int Hkv, int d, int dtype, const float *node_state, int H,
               int dk, int dv, void *ck, void *cv, float *cS, int ckpt_rows, cudaStream_t s) {
  if (!x) return FLIDE_ERR_SHAPE;
  const int es = dtype == FLIDE_BF16 ? 2 : (dtype == FLIDE_F32 ? 4 : 0);
  if (!es) return FLIDE_ERR_SHAPE;
  // every argument is checked before the first launch, so a refused call
  // leaves the checkpoint untouched
  const long row_bytes = (long)Hkv * d * es;
  if (Hkv > 0 && (d <= 0 || row_bytes % 16 != 0 || row_bytes > (1 << 30) || !k || !v || !ck || !cv))
    return FLIDE_ERR_SHAPE;
  if (H > 0 && (!node_state || !cS || dk <= 0 || dv <= 0 || ((long)dk * dv) % 4 != 0))
    return FLIDE_ERR_SHAPE;
  if (Hkv > 0) {
    save_kv_kernel<<<148 * 4, 256, 0, s>>>(*x, (const char *)k, (const char *)v,
                                           (const char *)pk, (const char *)pv, (int)row_bytes,
                                           (char *)ck, (char *)cv, ckpt_rows);
    FLIDE_LAUNCH_CHECK();
  }
  if (H > 0) {
    save_state_kernel<<<148 * 4, 256, 0, s>>>(*x, node_state, H, dk * dv, cS);
    FLIDE_LAUNCH_CHECK();
  }
  return FLIDE_OK;
}

int state_resume(int R, const int32_t *src_req, int src_R, const int32_t *src_start,
                 const void *sk, const void *sv, const float *sS, int Hkv, int d, int dtype,
                 int H, int dk, int dv, int32_t *past_len, void *pk, void *pv,
                 int past_rows, float *state_in, int32_t *status, cudaStream_t s) {
  const int es = dtype == FLIDE_BF16 ? 2 : (dtype == FLIDE_F32 ? 4 : 0);
  if (!es || R < 0 || !src_req || !src_start || !past_len || !status) return FLIDE_ERR_SHAPE;
  if (R > kMaxResumeR) return FLIDE_ERR_CAPACITY;  // the kernel's shared offset table
  const long row_bytes = (long)Hkv * d * es;
  if (row_bytes <= 0 || row_bytes % 16 != 0 || !sk || !sv || !pk || !pv) return FLIDE_ERR_SHAPE;
  if (state_in && (!sS || ((long)dk * dv) % 4 != 0 || H <= 0)) return FLIDE_ERR_SHAPE;
  resume_kernel<<<148 * 2, 256, 0, s>>>(R, src_req, src_R, src_start, (const char *)sk,
                                         (const char *)sv, sS, (int)row_bytes, H, dk * dv,
                                         past_len, (char *)pk, (char *)pv, past_rows, state_in,
                                         status);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}

}  // namespace flide
