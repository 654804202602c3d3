// schedule.cu -- memory-bounded, depth-first scheduling of the GDN node states.
//
// The GDN keeps one fp32 state (H x dv x dk) for every node whose children
// continue from it, and memory for cloned states is what limits how many
// options one call can hold (techfi24.com, "Limites et perspectives": past a
// few dozen options the memory grows linearly with them).  Fork = isolation
// lets a request's tree be cut below its root: every level-1 subtree needs
// only the root's end state, so the roots run once (their end states saved)
// and the subtrees run afterwards in groups, each group a batch of its own
// whose zero-token roots resume from the saved states.  A group's batch needs
// roots + (widest odd depth) + (widest even depth) slots, counting inner nodes
// only, as flide_tree_build assigns them.
//
//   flide_plan_state_groups  host planner: whole level-1 subtrees, in stream
//                            order, packed greedily into groups whose batches
//                            need at most max_slots slots
//   flide_copy_rows          device row gather / scatter between the full
//                            stream and a group's compact stream
#include <algorithm>
#include <vector>

#include "common.cuh"

namespace flide {
namespace {

constexpr int kThreads = 256;

// dst row dst_idx[i] (or i) <- src row src_idx[i] (or i), row_bytes bytes;
// one warp per row, 16-byte words when both rows allow it, else 4-byte words
__global__ void copy_rows_kernel(char *dst, const char *src, const int32_t *dst_idx,
                                 const int32_t *src_idx, int n, long row_bytes, int wide) {
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int i = warp; i < n; i += nwarps) {
    const long d = dst_idx ? dst_idx[i] : i, s = src_idx ? src_idx[i] : i;
    if (wide) {
      const uint4 *sp = reinterpret_cast<const uint4 *>(src + s * row_bytes);
      uint4 *dp = reinterpret_cast<uint4 *>(dst + d * row_bytes);
      for (long w = lane; w < row_bytes / 16; w += 32) dp[w] = sp[w];
    } else {
      const uint32_t *sp = reinterpret_cast<const uint32_t *>(src + s * row_bytes);
      uint32_t *dp = reinterpret_cast<uint32_t *>(dst + d * row_bytes);
      for (long w = lane; w < row_bytes / 4; w += 32) dp[w] = sp[w];
    }
  }
}

// slots a batch needs: one per root, plus the widest odd and even depth's
// inner-node count (depth >= 1)
int batch_slots(int roots, const std::vector<int> &inner_at_depth) {
  int odd = 0, even = 0;
  for (size_t d = 1; d < inner_at_depth.size(); ++d) {
    if (d & 1) odd = std::max(odd, inner_at_depth[d]);
    else even = std::max(even, inner_at_depth[d]);
  }
  return roots + odd + even;
}

}  // namespace
}  // namespace flide

using namespace flide;

namespace {

int plan_state_groups(int32_t R, const int32_t *req_node_ptr, const int32_t *parent,
                      int32_t max_slots, int32_t *node_group, int32_t *n_groups) {
  if (R < 0 || !req_node_ptr || !node_group || !n_groups || max_slots < 1) return FLIDE_ERR_SHAPE;
  if (req_node_ptr[0] != 0) return FLIDE_ERR_INVALID;
  for (int r = 0; r < R; ++r)  // monotone, so N below is a node count
    if (req_node_ptr[r + 1] < req_node_ptr[r]) return FLIDE_ERR_INVALID;
  const int N = req_node_ptr[R];
  if (N > 0 && !parent) return FLIDE_ERR_SHAPE;
  // per node: depth, level-1 ancestor (global id), whether it has children
  std::vector<int> depth(N, 0), top(N, -1), has_child(N, 0);
  for (int r = 0; r < R; ++r) {
    const int n0 = req_node_ptr[r], n1 = req_node_ptr[r + 1];
    if (n1 < n0) return FLIDE_ERR_INVALID;
    for (int n = n0; n < n1; ++n) {
      const int p = parent[n];
      if (n == n0) {
        if (p != -1) return FLIDE_ERR_INVALID;
        continue;
      }
      if (p < 0 || n0 + p >= n) return FLIDE_ERR_INVALID;
      const int pg = n0 + p;
      depth[n] = depth[pg] + 1;
      top[n] = depth[n] == 1 ? n : top[pg];
      has_child[pg] = 1;
    }
  }
  // per level-1 subtree: inner nodes at each depth
  std::vector<std::vector<int>> sub(N);
  for (int n = 0; n < N; ++n)
    if (top[n] >= 0 && has_child[n]) {
      std::vector<int> &v = sub[top[n]];
      if ((int)v.size() <= depth[n]) v.resize(depth[n] + 1, 0);
      ++v[depth[n]];
    }
  int g = -1, roots_in_group = 0, last_req = -1;
  std::vector<int> acc;
  for (int r = 0; r < R; ++r) {
    const int n0 = req_node_ptr[r], n1 = req_node_ptr[r + 1];
    if (n1 > n0) node_group[n0] = -1;
    for (int n = n0 + 1; n < n1; ++n) {
      if (depth[n] != 1) {
        node_group[n] = node_group[top[n]];
        continue;
      }
      // try to add subtree n to the open group
      std::vector<int> trial = acc;
      if (trial.size() < sub[n].size()) trial.resize(sub[n].size(), 0);
      for (size_t d = 0; d < sub[n].size(); ++d) trial[d] += sub[n][d];
      const int trial_roots = roots_in_group + (last_req != r ? 1 : 0);
      if (g < 0 || batch_slots(trial_roots, trial) > max_slots) {
        // a new group holding this subtree alone
        std::vector<int> alone = sub[n];
        if (batch_slots(1, alone) > max_slots) return FLIDE_ERR_CAPACITY;
        ++g;
        acc = alone;
        roots_in_group = 1;
      } else {
        acc.swap(trial);
        roots_in_group = trial_roots;
      }
      last_req = r;
      node_group[n] = g;
    }
  }
  *n_groups = g + 1;
  return FLIDE_OK;
}

// Slots flide_tree_build assigns to the whole batch: every non-empty
// request's root, plus the widest odd and even depth's inner nodes.
int tree_state_slots(int32_t R, const int32_t *req_node_ptr, const int32_t *parent,
                     int32_t *slots) {
  if (R < 0 || !req_node_ptr || !slots) return FLIDE_ERR_SHAPE;
  if (req_node_ptr[0] != 0) return FLIDE_ERR_INVALID;
  for (int r = 0; r < R; ++r)
    if (req_node_ptr[r + 1] < req_node_ptr[r]) return FLIDE_ERR_INVALID;
  const int N = req_node_ptr[R];
  if (N > 0 && !parent) return FLIDE_ERR_SHAPE;
  std::vector<int> depth(N, 0), has_child(N, 0), inner_at_depth;
  int roots = 0;
  for (int r = 0; r < R; ++r) {
    const int n0 = req_node_ptr[r], n1 = req_node_ptr[r + 1];
    if (n1 > n0) ++roots;
    for (int n = n0; n < n1; ++n) {
      const int p = parent[n];
      if (n == n0) {
        if (p != -1) return FLIDE_ERR_INVALID;
        continue;
      }
      if (p < 0 || n0 + p >= n) return FLIDE_ERR_INVALID;
      depth[n] = depth[n0 + p] + 1;
      has_child[n0 + p] = 1;
    }
  }
  for (int n = 0; n < N; ++n)
    if (has_child[n] && depth[n] >= 1) {
      if ((int)inner_at_depth.size() <= depth[n]) inner_at_depth.resize(depth[n] + 1, 0);
      ++inner_at_depth[depth[n]];
    }
  *slots = batch_slots(roots, inner_at_depth);
  return FLIDE_OK;
}

}  // namespace

extern "C" {

int flide_tree_state_slots(int32_t R, const int32_t *req_node_ptr, const int32_t *parent,
                           int32_t *slots) {
  try {  // no exception may cross the C ABI: out of host memory reads as capacity
    return tree_state_slots(R, req_node_ptr, parent, slots);
  } catch (...) {
    return FLIDE_ERR_CAPACITY;
  }
}

int flide_plan_state_groups(int32_t R, const int32_t *req_node_ptr, const int32_t *parent,
                            int32_t max_slots, int32_t *node_group, int32_t *n_groups) {
  try {  // no exception may cross the C ABI: out of host memory reads as capacity
    return plan_state_groups(R, req_node_ptr, parent, max_slots, node_group, n_groups);
  } catch (...) {
    return FLIDE_ERR_CAPACITY;
  }
}

int flide_copy_rows(void *dst, const void *src, const int32_t *dst_idx, const int32_t *src_idx,
                    int32_t n, int64_t row_bytes, flide_stream stream) {
  if (n < 0 || row_bytes <= 0 || row_bytes % 4) return FLIDE_ERR_SHAPE;
  if (n == 0) return FLIDE_OK;
  if (!dst || !src) return FLIDE_ERR_SHAPE;
  if ((uintptr_t)dst % 4 || (uintptr_t)src % 4) return FLIDE_ERR_SHAPE;
  const int wide = row_bytes % 16 == 0 && (uintptr_t)dst % 16 == 0 && (uintptr_t)src % 16 == 0;
  const int blocks = std::min(148 * 4, (n + kThreads / 32 - 1) / (kThreads / 32));
  copy_rows_kernel<<<blocks, kThreads, 0, (cudaStream_t)stream>>>(
      (char *)dst, (const char *)src, dst_idx, src_idx, n, (long)row_bytes, wide);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}

}  // extern "C"
