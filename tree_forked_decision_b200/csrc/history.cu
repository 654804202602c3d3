// history.cu -- multi-step agent history in a block-paged checkpoint pool.
//
// An agent makes decision after decision on a growing history: each step's
// root (the new observation) is appended to what came before and the next
// step resumes from it, so the shared prefix is never recomputed
// (kongchang.com article on Flide, closing section: growing agent histories
// and checkpoint reuse; techfi24.com, "Exact State Forking").  The pool keeps every
// request's history K/V rows in fixed-size blocks (a block table per request,
// blocks from a shared free list) and its latest GDN state in a per-request
// slot:
//   flide_pool_*            host allocator: blocks, block tables, lengths
//   flide_history_append    after a step: the batch's root rows -> the
//                           requests' blocks; the roots' end states -> slots
//   flide_history_gather    before a step: histories -> packed past K/V,
//                           past_len and GDN state_in for the batch
#include <cstring>
#include <new>
#include <vector>

#include "common.cuh"

struct flide_pool {
  int32_t n_blocks, block_rows, max_requests, max_blocks;
  std::vector<int32_t> table;    // [max_requests][max_blocks], -1 = none
  std::vector<int32_t> length;   // rows held per request
  std::vector<int32_t> nblocks;  // blocks held per request
  std::vector<int32_t> free_list;
  std::vector<int64_t> pending;  // per request: rows a batch append adds (0 between calls)
};

namespace flide {
namespace {

constexpr int kMaxGatherR = 4096;

__device__ __forceinline__ int upper_bound_h(const int32_t *a, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] > key) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// one row of `bytes` (a multiple of 16) by the lanes of a warp; up to four
// 16-byte loads per lane are issued before their stores
__device__ __forceinline__ void copy_row16(char *dst, const char *src, int bytes, int lane) {
  for (int o0 = lane * 16; o0 < bytes; o0 += 4 * 32 * 16) {
    uint4 t[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int o = o0 + u * 32 * 16;
      if (o < bytes) t[u] = __ldg(reinterpret_cast<const uint4 *>(src + o));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int o = o0 + u * 32 * 16;
      if (o < bytes) *reinterpret_cast<uint4 *>(dst + o) = t[u];
    }
  }
}

// physical pool row of logical history row `row` of pool slot `s`, or -1
__device__ __forceinline__ long pool_row(const int32_t *table, int max_blocks, int block_rows,
                                         int s, int row) {
  const int b = row / block_rows;
  if (b >= max_blocks) return -1;
  const int blk = table[(size_t)s * max_blocks + b];
  return blk < 0 ? -1 : (long)blk * block_rows + row % block_rows;
}

__global__ void history_append_kernel(flide_tree_index x, const int32_t *req_slot,
                                      const int32_t *start, const int32_t *table, int max_blocks,
                                      int block_rows, const char *k, const char *v, char *pool_k,
                                      char *pool_v, int row_bytes, const float *node_state,
                                      int state_floats, float *pool_S) {
  if (failed(x.status)) return;
  const int R = x.R;
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  // rows: one warp per (request, root row)
  for (int r = 0; r < R; ++r) {
    const int s = req_slot[r];
    const int n0 = x.req_node[r], n1 = x.req_node[r + 1];
    if (s < 0 || n1 <= n0) continue;
    const int t0 = x.node_start[n0], len = x.node_start[n0 + 1] - t0;
    for (int i = warp; i < len; i += nwarps) {
      const long pr = pool_row(table, max_blocks, block_rows, s, start[r] + i);
      if (pr < 0) {
        if (lane == 0) set_status(x.status, FLIDE_ERR_CAPACITY);
        continue;
      }
      // debug build: the root row lies in the stream (pool block ids come from
      // the host allocator; their range is not passed to the device)
      if (!in_bounds(x.status, x.counts, (long long)t0 + i, x.counts[FLIDE_CNT_T], 502)) continue;
      copy_row16(pool_k + pr * row_bytes, k + (size_t)(t0 + i) * row_bytes, row_bytes, lane);
      copy_row16(pool_v + pr * row_bytes, v + (size_t)(t0 + i) * row_bytes, row_bytes, lane);
    }
    // the root's end state becomes the request's state
    if (node_state && pool_S) {
      const int slot = x.state_slot[n0];
      if (slot < 0 || !in_bounds(x.status, x.counts, slot, x.counts[FLIDE_CNT_SLOTS], 501)) continue;
      const float4 *src = reinterpret_cast<const float4 *>(node_state + (size_t)slot * state_floats);
      float4 *dst = reinterpret_cast<float4 *>(pool_S + (size_t)s * state_floats);
      for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < state_floats / 4;
           e += gridDim.x * blockDim.x)
        dst[e] = src[e];
    }
  }
}

__global__ void history_gather_kernel(int R, const int32_t *req_slot, int max_requests,
                                      const int32_t *hist_len, const int32_t *table, int max_blocks,
                                      int block_rows, const char *pool_k, const char *pool_v,
                                      int row_bytes, const float *pool_S, int state_floats,
                                      int32_t *past_len, char *pk, char *pv, int past_rows,
                                      float *state_in, int32_t *status) {
  __shared__ int32_t off[kMaxGatherR + 1];
  __shared__ int scratch[40];
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  int carry = 0;
  for (int b = 0; b < R; b += blockDim.x) {
    const int r = b + threadIdx.x;
    int len = 0;
    if (r < R) {
      const int s = req_slot[r];
      if (s >= max_requests) s_bad = FLIDE_ERR_INVALID;
      else if (s >= 0) len = hist_len[s];
    }
    int tot;
    const int ex = block_excl_scan(len, scratch, &tot);
    if (r < R) off[r] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) off[R] = carry;
  __syncthreads();
  if (s_bad || (pk != nullptr && carry > past_rows)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, s_bad ? s_bad : FLIDE_ERR_CAPACITY);
    return;
  }
  if (blockIdx.x == 0)
    for (int r = threadIdx.x; r < R; r += blockDim.x) past_len[r] = off[r + 1] - off[r];
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int i = warp; pk != nullptr && i < carry; i += nwarps) {
    const int r = upper_bound_h(off, R + 1, i) - 1;
    const long pr = pool_row(table, max_blocks, block_rows, req_slot[r], i - off[r]);
    if (pr < 0) {
      if (lane == 0) set_status(status, FLIDE_ERR_INVALID);
      continue;
    }
    copy_row16(pk + (size_t)i * row_bytes, pool_k + pr * row_bytes, row_bytes, lane);
    copy_row16(pv + (size_t)i * row_bytes, pool_v + pr * row_bytes, row_bytes, lane);
  }
  if (state_in) {
    const long per = state_floats / 4;
    for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < (long)R * per;
         e += (long)gridDim.x * blockDim.x) {
      const int r = (int)(e / per);
      const int s = req_slot[r];
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s >= 0 && pool_S) val = reinterpret_cast<const float4 *>(pool_S + (size_t)s * state_floats)[e % per];
      reinterpret_cast<float4 *>(state_in)[e] = val;
    }
  }
}

}  // namespace
}  // namespace flide

extern "C" {

flide_pool *flide_pool_create(int32_t n_blocks, int32_t block_rows, int32_t max_requests,
                              int32_t max_blocks_per_request) {
  if (n_blocks < 0 || block_rows <= 0 || max_requests <= 0 || max_blocks_per_request <= 0)
    return nullptr;
  flide_pool *p = new (std::nothrow) flide_pool;
  if (!p) return nullptr;
  try {  // no exception may cross the C ABI
    p->n_blocks = n_blocks;
    p->block_rows = block_rows;
    p->max_requests = max_requests;
    p->max_blocks = max_blocks_per_request;
    p->table.assign((size_t)max_requests * max_blocks_per_request, -1);
    p->length.assign(max_requests, 0);
    p->nblocks.assign(max_requests, 0);
    p->pending.assign(max_requests, 0);
    p->free_list.resize(n_blocks);
    for (int32_t b = 0; b < n_blocks; ++b) p->free_list[b] = n_blocks - 1 - b;  // handed out 0, 1, ...
  } catch (...) {
    delete p;
    return nullptr;
  }
  return p;
}

void flide_pool_destroy(flide_pool *p) { delete p; }

int64_t flide_pool_append(flide_pool *p, int32_t slot, int32_t n) {
  if (!p || slot < 0 || slot >= p->max_requests || n < 0) return -FLIDE_ERR_INVALID;
  const int64_t start = p->length[slot];
  const int64_t need = (start + n + p->block_rows - 1) / p->block_rows;
  if (need > p->max_blocks || start + n > INT32_MAX) return -FLIDE_ERR_CAPACITY;
  if (need - p->nblocks[slot] > (int64_t)p->free_list.size()) return -FLIDE_ERR_CAPACITY;
  while (p->nblocks[slot] < need) {
    const int32_t b = p->free_list.back();
    p->free_list.pop_back();
    p->table[(size_t)slot * p->max_blocks + p->nblocks[slot]++] = b;
  }
  p->length[slot] = (int32_t)(start + n);
  return start;
}

int flide_pool_append_batch(flide_pool *p, int32_t n, const int32_t *slots, const int32_t *counts,
                            int32_t *starts) {
  if (!p || n < 0 || (n > 0 && (!slots || !counts || !starts))) return FLIDE_ERR_SHAPE;
  for (int32_t i = 0; i < n; ++i)
    if (slots[i] >= p->max_requests || (slots[i] >= 0 && counts[i] < 0)) return FLIDE_ERR_INVALID;
  // check the whole batch before any reservation: per request the rows it
  // gains (a request may appear more than once), then its block need
  for (int32_t i = 0; i < n; ++i)
    if (slots[i] >= 0) p->pending[slots[i]] += counts[i];
  int status = FLIDE_OK;
  int64_t blocks = 0;
  for (int32_t i = 0; i < n && status == FLIDE_OK; ++i) {
    const int32_t s = slots[i];
    if (s < 0 || p->pending[s] < 0) continue;  // skipped, or counted already (marked negative)
    const int64_t len = (int64_t)p->length[s] + p->pending[s];
    const int64_t need = (len + p->block_rows - 1) / p->block_rows;
    if (need > p->max_blocks || len > INT32_MAX) status = FLIDE_ERR_CAPACITY;
    blocks += need - p->nblocks[s];
    p->pending[s] = -1 - p->pending[s];
  }
  if (status == FLIDE_OK && blocks > (int64_t)p->free_list.size()) status = FLIDE_ERR_CAPACITY;
  for (int32_t i = 0; i < n; ++i)
    if (slots[i] >= 0) p->pending[slots[i]] = 0;
  if (status != FLIDE_OK) return status;
  for (int32_t i = 0; i < n; ++i)  // cannot fail now
    starts[i] = slots[i] < 0 ? -1 : (int32_t)flide_pool_append(p, slots[i], counts[i]);
  return FLIDE_OK;
}

int flide_pool_release(flide_pool *p, int32_t slot) {
  if (!p || slot < 0 || slot >= p->max_requests) return FLIDE_ERR_INVALID;
  for (int32_t i = p->nblocks[slot] - 1; i >= 0; --i) {
    int32_t &e = p->table[(size_t)slot * p->max_blocks + i];
    p->free_list.push_back(e);
    e = -1;
  }
  p->nblocks[slot] = 0;
  p->length[slot] = 0;
  return FLIDE_OK;
}

int32_t flide_pool_length(const flide_pool *p, int32_t slot) {
  if (!p || slot < 0 || slot >= p->max_requests) return -FLIDE_ERR_INVALID;
  return p->length[slot];
}

int32_t flide_pool_free_blocks(const flide_pool *p) { return p ? (int32_t)p->free_list.size() : 0; }

int flide_pool_export(const flide_pool *p, int32_t *table, int32_t *lengths) {
  if (!p || !table || !lengths) return FLIDE_ERR_SHAPE;
  std::memcpy(table, p->table.data(), p->table.size() * sizeof(int32_t));
  std::memcpy(lengths, p->length.data(), p->length.size() * sizeof(int32_t));
  return FLIDE_OK;
}

int flide_history_append(const flide_tree_index *idx, const int32_t *req_slot,
                         const int32_t *start, const int32_t *table, int32_t max_blocks,
                         int32_t block_rows, const void *k, const void *v, void *pool_k,
                         void *pool_v, int32_t Hkv, int32_t d, int32_t dtype,
                         const float *node_state, int32_t H, int32_t dk, int32_t dv,
                         float *pool_S, flide_stream stream) {
  using namespace flide;
  if (!idx || !req_slot || !start || !table || !k || !v || !pool_k || !pool_v) return FLIDE_ERR_SHAPE;
  if (max_blocks <= 0 || block_rows <= 0 || Hkv <= 0 || d <= 0) return FLIDE_ERR_SHAPE;
  const int es = dtype == FLIDE_BF16 ? 2 : dtype == FLIDE_F32 ? 4 : dtype == FLIDE_E4M3 ? 1 : 0;
  if (!es) return FLIDE_ERR_SHAPE;
  const long row_bytes = (long)Hkv * d * es;
  if (row_bytes % 16) return FLIDE_ERR_SHAPE;
  const long sf = (long)H * dk * dv;
  if ((node_state != nullptr) != (pool_S != nullptr) || (node_state && (H <= 0 || sf % 4)))
    return FLIDE_ERR_SHAPE;
  if (idx->R <= 0) return FLIDE_OK;
  history_append_kernel<<<148 * 2, 256, 0, (cudaStream_t)stream>>>(
      *idx, req_slot, start, table, max_blocks, block_rows, (const char *)k, (const char *)v,
      (char *)pool_k, (char *)pool_v, (int)row_bytes, node_state, (int)sf, pool_S);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}

int flide_history_gather(int32_t R, const int32_t *req_slot, int32_t max_requests,
                         const int32_t *hist_len, const int32_t *table, int32_t max_blocks,
                         int32_t block_rows, const void *pool_k, const void *pool_v, int32_t Hkv,
                         int32_t d, int32_t dtype, const float *pool_S, int32_t H, int32_t dk,
                         int32_t dv, int32_t *past_len, void *past_k, void *past_v,
                         int32_t past_rows, float *state_in, int32_t *status, flide_stream stream) {
  using namespace flide;
  if (!req_slot || !hist_len || !table || !pool_k || !pool_v || !past_len || !status)
    return FLIDE_ERR_SHAPE;
  if (R < 0 || R > kMaxGatherR) return FLIDE_ERR_CAPACITY;
  if (max_requests <= 0 || max_blocks <= 0 || block_rows <= 0 || Hkv <= 0 || d <= 0 || past_rows < 0)
    return FLIDE_ERR_SHAPE;
  if (past_rows > 0 && (!past_k || !past_v)) return FLIDE_ERR_SHAPE;
  if ((past_k == nullptr) != (past_v == nullptr)) return FLIDE_ERR_SHAPE;
  const int es = dtype == FLIDE_BF16 ? 2 : dtype == FLIDE_F32 ? 4 : dtype == FLIDE_E4M3 ? 1 : 0;
  if (!es) return FLIDE_ERR_SHAPE;
  const long row_bytes = (long)Hkv * d * es;
  if (row_bytes % 16) return FLIDE_ERR_SHAPE;
  const long sf = (long)H * dk * dv;
  if (state_in && (H <= 0 || sf % 4)) return FLIDE_ERR_SHAPE;
  if (R == 0) return FLIDE_OK;
  history_gather_kernel<<<148 * 2, 256, 0, (cudaStream_t)stream>>>(
      R, req_slot, max_requests, hist_len, table, max_blocks, block_rows, (const char *)pool_k,
      (const char *)pool_v, (int)row_bytes, pool_S, (int)sf, past_len, (char *)past_k,
      (char *)past_v, past_rows, state_in, status);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}

}  // extern "C"
