// tree_index.cu -- the tree-index builder.
//
// Turns the parent arrays of a batch of decision requests into the indices the
// layer kernels navigate (kongchang.com article on Flide, "ForkAttention"
// section: the logical tree of every request is encoded as GPU-resident
// indices over one flattened token stream, topology expressed as metadata).
//
// Two launches:
//   tree_nodes_kernel  one CTA of 1024 threads: validation, the node-level
//                      prefix sums (node_start, past_start, anc_ptr,
//                      ckpt_start), depth by walking parent pointers, the
//                      ancestor CSR, ctx_len, nodes grouped by level and
//                      node-state slots.  N is small (thousands), so one CTA
//                      does it in a few microseconds without a grid sync.
//   tree_tokens_kernel grid-stride over tokens: token_node by binary search
//                      over node_start, token_pos from ctx_len.
#include "common.cuh"

namespace flide {

namespace {

constexpr int kNodeThreads = 1024;

// Exclusive prefix sum of f(i), i < L, into out[0..L]; out[L] = total.
template <typename F>
__device__ int block_scan_array(int L, F f, int32_t *out, int *scratch) {
  int carry = 0;
  for (int base = 0; base < L; base += blockDim.x) {
    int i = base + threadIdx.x;
    int v = i < L ? f(i) : 0;
    int tot;
    int ex = block_excl_scan(v, scratch, &tot);
    if (i < L) out[i] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) out[L] = carry;
  __syncthreads();
  return carry;
}

__device__ __forceinline__ int upper_bound(const int32_t *a, int n, int key) {
  int lo = 0, hi = n;  // first i in [0, n) with a[i] > key, or n
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (a[mid] > key) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Sum of one 64-bit value per thread across the block (blockDim.x a multiple
// of 32, <= 1024); `scratch` holds >= 32 entries.
__device__ long long block_sum_ll(long long v, long long *scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  long long tot = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += scratch[w];
  __syncthreads();
  return tot;
}

__global__ void __launch_bounds__(kNodeThreads)
tree_nodes_kernel(flide_tree_desc d, flide_tree_index x) {
  // capacities checked are the descriptor's (never above the index's)
  __shared__ int scratch[40];
  __shared__ int s_err, s_N, s_depth;
  const int tid = threadIdx.x;
  const int R = d.R;
  const int32_t *rp = d.req_node_ptr;
  if (tid == 0) {
    s_err = 0;
    s_depth = 0;
    s_N = rp[R];
    if (rp[0] != 0) s_err = FLIDE_ERR_INVALID;
    else if (s_N < 0 || s_N > d.N) s_err = FLIDE_ERR_CAPACITY;
  }
  __syncthreads();
  for (int r = tid; r <= R; r += blockDim.x) {
    x.req_node[r] = rp[r];
    if (r < R && (rp[r + 1] < rp[r] || d.past_len[r] < 0)) atomicCAS(&s_err, 0, FLIDE_ERR_INVALID);
  }
  __syncthreads();
  if (s_err) {
    if (tid == 0) set_status(x.status, s_err);
    return;
  }
  const int N = s_N;

  // node -> request, and the per-node rules
  for (int n = tid; n < N; n += blockDim.x) {
    int r = upper_bound(rp, R + 1, n) - 1;
    x.node_req[n] = r;
    int local = n - rp[r];
    int p = d.parent[n], s = d.seg_len[n];
    bool ok = local == 0 ? (p == -1 && s >= 0) : (p >= 0 && p < local && s >= 1);
    if (!ok) atomicCAS(&s_err, 0, FLIDE_ERR_INVALID);
  }
  __syncthreads();
  if (s_err) {
    if (tid == 0) set_status(x.status, s_err);
    return;
  }

  // Totals in 64 bits first: the prefix sums below are int32 (the kernels'
  // index type), so tokens beyond the capacity, or past rows plus tokens
  // beyond 2^31 - 1 (positions, context lengths and checkpoint rows add
  // them), are refused before any sum can wrap.
  {
    __shared__ long long sum_scratch[32];
    long long ts = 0, ps = 0;
    for (int n = tid; n < N; n += blockDim.x) ts += d.seg_len[n];
    for (int r = tid; r < R; r += blockDim.x) ps += d.past_len[r];
    ts = block_sum_ll(ts, sum_scratch);
    ps = block_sum_ll(ps, sum_scratch);
    if (ts > d.T || ts + ps > 0x7fffffffLL) {
      if (tid == 0) set_status(x.status, FLIDE_ERR_CAPACITY);
      return;
    }
  }
  const int T = block_scan_array(N, [&](int i) { return (int)d.seg_len[i]; }, x.node_start, scratch);
  const int P = block_scan_array(R, [&](int i) { return (int)d.past_len[i]; }, x.past_start, scratch);

  // depth by walking parents (parent < self, so the walk ends)
  for (int n = tid; n < N; n += blockDim.x) {
    int r = x.node_req[n], base = rp[r];
    int cur = n, dep = 0;
    while (d.parent[cur] >= 0) { cur = base + d.parent[cur]; ++dep; }
    x.depth[n] = dep;
    atomicMax(&s_depth, dep);
  }
  __syncthreads();
  if (tid == 0 && s_depth > d.max_depth) s_err = FLIDE_ERR_CAPACITY;
  __syncthreads();
  if (s_err) {
    if (tid == 0) set_status(x.status, s_err);
    return;
  }
  const int D = s_depth;

  const int A = block_scan_array(N, [&](int i) { return (int)x.depth[i] + 1; }, x.anc_ptr, scratch);
  (void)A;
  // ancestor rows (root first) and context lengths
  const long long anc_cap = (long long)x.N * (x.max_depth + 1);
  for (int n = tid; n < N; n += blockDim.x) {
    int r = x.node_req[n], base = rp[r];
    int row = x.anc_ptr[n];
    int cur = n, ctx = d.past_len[r];
    for (int i = x.depth[n]; i >= 0; --i) {
      if (in_bounds(x.status, x.counts, (long long)row + i, anc_cap, 101)) x.anc_node[row + i] = cur;
      ctx += d.seg_len[cur];
      if (i > 0) cur = base + d.parent[cur];
    }
    x.ctx_len[n] = ctx;
  }

  // nodes grouped by level, ascending node id within a level
  int placed = 0;
  for (int lvl = 0; lvl <= D; ++lvl) {
    if (tid == 0) x.level_ptr[lvl] = placed;
    int carry = 0;
    for (int b = 0; b < N; b += blockDim.x) {
      int n = b + tid;
      int f = (n < N && x.depth[n] == lvl) ? 1 : 0;
      int tot;
      int ex = block_excl_scan(f, scratch, &tot);
      if (f && in_bounds(x.status, x.counts, placed + carry + ex, x.N, 102))
        x.level_node[placed + carry + ex] = n;
      carry += tot;
    }
    placed += carry;
  }
  for (int lvl = D + 1 + tid; lvl <= x.max_depth + 1; lvl += blockDim.x) x.level_ptr[lvl] = N;

  // State slots.  A root keeps its slot for the whole call (its end state is
  // the request's checkpoint).  An inner node at depth L >= 1 is read only by
  // the depth-(L+1) launch, so inner nodes of odd depths share one region and
  // those of even depths another, each sized by its largest level: depth L's
  // slots are rewritten at depth L+2, after depth L+1 has read them.  Leaves
  // have no slot.
  for (int n = tid; n < N; n += blockDim.x) x.state_slot[n] = 0;
  __syncthreads();
  for (int n = tid; n < N; n += blockDim.x) {
    int p = d.parent[n];
    if (p >= 0 && in_bounds(x.status, x.counts, rp[x.node_req[n]] + p, N, 103))
      x.state_slot[rp[x.node_req[n]] + p] = 1;  // has children
  }
  __syncthreads();
  // inner nodes per level (L >= 1), for the two regions' sizes
  int size_odd = 0, size_even = 0;
  for (int lvl = 1; lvl <= D; ++lvl) {
    const int a0 = x.level_ptr[lvl], a1 = x.level_ptr[lvl + 1];
    int cnt = 0;
    for (int b = a0; b < a1; b += blockDim.x) {
      const int k = b + tid;
      const int f = (k < a1 && x.state_slot[checked(x.status, x.counts, x.level_node[k], N, 104)] == 1) ? 1 : 0;
      int tot;
      block_excl_scan(f, scratch, &tot);
      cnt += tot;
    }
    if (lvl & 1) size_odd = max(size_odd, cnt); else size_even = max(size_even, cnt);
  }
  // roots first, in level order (depth 0 is one level)
  int roots = 0;
  {
    const int a0 = x.level_ptr[0], a1 = x.level_ptr[1];
    for (int b = a0; b < a1; b += blockDim.x) {
      const int k = b + tid;
      int tot;
      const int ex = block_excl_scan(k < a1 ? 1 : 0, scratch, &tot);
      if (k < a1) x.state_slot[checked(x.status, x.counts, x.level_node[k], N, 105)] = roots + ex;
      roots += tot;
    }
  }
  for (int lvl = 1; lvl <= D; ++lvl) {
    const int a0 = x.level_ptr[lvl], a1 = x.level_ptr[lvl + 1];
    const int base = roots + ((lvl & 1) ? 0 : size_odd);
    int carry = 0;
    for (int b = a0; b < a1; b += blockDim.x) {
      const int k = b + tid;
      const int n = k < a1 ? (int)checked(x.status, x.counts, x.level_node[k], N, 106) : -1;
      const int f = (n >= 0 && x.state_slot[n] == 1) ? 1 : 0;
      int tot;
      const int ex = block_excl_scan(f, scratch, &tot);
      if (n >= 0) x.state_slot[n] = f ? base + carry + ex : -1;
      carry += tot;
    }
  }
  const int slots = roots + size_odd + size_even;

  // checkpoint rows: past + root tokens of every request
  const int C = block_scan_array(R, [&](int r) {
    int root_len = rp[r + 1] > rp[r] ? (int)d.seg_len[rp[r]] : 0;
    return (int)d.past_len[r] + root_len;
  }, x.ckpt_start, scratch);

  int root_tok = 0;
  for (int b = 0; b < R; b += blockDim.x) {
    int r = b + tid;
    int v = (r < R && rp[r + 1] > rp[r]) ? (int)d.seg_len[rp[r]] : 0;
    int tot;
    block_excl_scan(v, scratch, &tot);
    root_tok += tot;
  }
  if (tid == 0) {
    x.counts[FLIDE_CNT_N] = N;
    x.counts[FLIDE_CNT_T] = T;
    x.counts[FLIDE_CNT_PAST] = P;
    x.counts[FLIDE_CNT_DEPTH] = D;
    x.counts[FLIDE_CNT_SLOTS] = slots;
    x.counts[FLIDE_CNT_BRANCH_TOK] = T - root_tok;
    x.counts[FLIDE_CNT_ROOT_TOK] = root_tok;
    x.counts[FLIDE_CNT_CKPT_ROWS] = C;
    if (s_err) set_status(x.status, s_err);
  }
}

__global__ void tree_tokens_kernel(flide_tree_index x) {
  if (failed(x.status)) return;
  const int N = x.counts[FLIDE_CNT_N];
  const int T = x.counts[FLIDE_CNT_T];
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
    int n = upper_bound(x.node_start, N + 1, t) - 1;
    // nodes with zero tokens share a start with their successor; upper_bound
    // already picks the last node starting at or before t, which holds t.
    if (!in_bounds(x.status, x.counts, n, N, 107)) continue;
    x.token_node[t] = n;
    x.token_pos[t] = x.ctx_len[n] - (x.node_start[n + 1] - x.node_start[n]) + (t - x.node_start[n]);
  }
}

}  // namespace

int tree_build(const flide_tree_desc *d, flide_tree_index *x, cudaStream_t s) {
  if (!d || !x || !x->status) return FLIDE_ERR_SHAPE;
  if (d->R < 0 || d->N < 0 || d->T < 0 || d->max_depth < 0) return FLIDE_ERR_SHAPE;
  if (d->R > x->R || d->N > x->N || d->T > x->T || d->max_depth > x->max_depth)
    return FLIDE_ERR_CAPACITY;
  if (!d->req_node_ptr || !d->past_len || (d->N > 0 && (!d->parent || !d->seg_len)))
    return FLIDE_ERR_SHAPE;
  if (cudaMemsetAsync(x->status, 0, sizeof(int32_t), s) != cudaSuccess) return FLIDE_ERR_CUDA;
  if (cudaMemsetAsync(x->counts, 0, sizeof(int32_t) * FLIDE_COUNTS, s) != cudaSuccess)
    return FLIDE_ERR_CUDA;
  flide_tree_index xi = *x;
  tree_nodes_kernel<<<1, kNodeThreads, 0, s>>>(*d, xi);
  FLIDE_LAUNCH_CHECK();
  int blocks = (d->T + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (blocks < 1) blocks = 1;
  tree_tokens_kernel<<<blocks, 256, 0, s>>>(xi);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}

}  // namespace flide
