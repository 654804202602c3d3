// api.cu -- the extern "C" boundary of libflide.so (declared in include/flide.h).
//
// Host-side argument checks, the layout of the tree index over one
// caller-owned device buffer, and dispatch to the kernels.  Nothing here
// allocates memory or synchronises the stream.
#include <cstring>

#include "common.cuh"

namespace flide {
int tree_build(const flide_tree_desc *d, flide_tree_index *x, cudaStream_t s);
int fork_attn_portable(const void *q, const void *k, const void *v, const void *pk,
                       const void *pv, int past_rows, const flide_tree_index *x, int Hq,
                       int Hkv, int d, int dtype, float scale, void *out, cudaStream_t s);
bool fork_attn_tc_supported(const flide_tree_index *x, int Hq, int Hkv, int d, int dtype);
int fork_attn_tc(const void *q, const void *k, const void *v, const void *pk, const void *pv,
                 int past_rows, const flide_tree_index *x, int Hq, int Hkv, int dtype,
                 const float *descale, float scale, void *out, cudaStream_t s,
                 const PagedPast *paged);
bool fork_gdn_tc_supported(int dk, int dv, int dtype);
int fork_gdn_tc(const void *q, const void *k, const void *v, const float *g, const float *beta,
                const float *state_in, const flide_tree_index *x, int H, void *out,
                float *node_state, int n_slots, cudaStream_t s, int dtype, const float *descale);
int fork_gdn_portable(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, const float *state_in, const flide_tree_index *x,
                      int H, int dk, int dv, int dtype, void *out, float *node_state,
                      int n_slots, cudaStream_t s);
int state_save(const flide_tree_index *x, const void *k, const void *v, const void *pk,
               const void *pv, int Hkv, int d, int dtype, const float *node_state, int H,
               int dk, int dv, void *ck, void *cv, float *cS, int ckpt_rows, cudaStream_t s);
int state_resume(int R, const int32_t *src_req, int src_R, const int32_t *src_start,
                 const void *sk, const void *sv, const float *sS, int Hkv, int d, int dtype,
                 int H, int dk, int dv, int32_t *past_len, void *pk, void *pv, int past_rows,
                 float *state_in, int32_t *status, cudaStream_t s);

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// int32 entries of the per-call scratch `work`: the attention's per-request
// item table and the GDN's per-level node groups (see their kernels)
int64_t work_entries(int32_t R, int32_t N) {
  return 4 * (int64_t)(R + 1) + 3 * (int64_t)(N + 1) + 1024;
}

struct Layout {
  size_t off[18];
  size_t total;
};

// Sub-array sizes (int32 entries) in the order of flide_tree_index's pointers.
bool layout(int32_t R, int32_t N, int32_t T, int32_t D, Layout *L) {
  if (R < 0 || N < 0 || T < 0 || D < 0) return false;
  const int64_t n[17] = {1,
                         FLIDE_COUNTS,
                         (int64_t)N + 1,
                         N,
                         N,
                         (int64_t)N + 1,
                         (int64_t)N * ((int64_t)D + 1),
                         N,
                         T,
                         T,
                         (int64_t)R + 1,
                         (int64_t)R + 1,
                         (int64_t)D + 2,
                         N,
                         N,
                         (int64_t)R + 1,
                         work_entries(R, N)};
  // the kernels index every sub-array with int32
  for (int i = 0; i < 17; ++i)
    if (n[i] > INT32_MAX) return false;
  size_t o = 0;
  for (int i = 0; i < 17; ++i) {
    L->off[i] = o;
    o = align_up(o + (size_t)(n[i] > 0 ? n[i] : 1) * sizeof(int32_t));
  }
  L->off[17] = o;
  L->total = o;
  return true;
}

}  // namespace
}  // namespace flide

using namespace flide;

extern "C" {

size_t flide_tree_index_bytes(int32_t R, int32_t N, int32_t T, int32_t max_depth) {
  Layout L;
  if (!layout(R, N, T, max_depth, &L)) return 0;
  return L.total;
}

int flide_tree_index_init(flide_tree_index *idx, void *dev_buf, size_t bytes, int32_t R,
                          int32_t N, int32_t T, int32_t max_depth) {
  Layout L;
  if (!idx || !dev_buf || !layout(R, N, T, max_depth, &L)) return FLIDE_ERR_SHAPE;
  if (((uintptr_t)dev_buf) % kAlign != 0) return FLIDE_ERR_SHAPE;
  if (bytes < L.total) return FLIDE_ERR_CAPACITY;
  char *b = (char *)dev_buf;
  int32_t **ptrs[17] = {&idx->status,     &idx->counts,     &idx->node_start, &idx->node_req,
                        &idx->depth,      &idx->anc_ptr,    &idx->anc_node,   &idx->ctx_len,
                        &idx->token_node, &idx->token_pos,  &idx->past_start, &idx->req_node,
                        &idx->level_ptr,  &idx->level_node, &idx->state_slot, &idx->ckpt_start,
                        &idx->work};
  for (int i = 0; i < 17; ++i) *ptrs[i] = (int32_t *)(b + L.off[i]);
  idx->R = R;
  idx->N = N;
  idx->T = T;
  idx->max_depth = max_depth;
  idx->work_len = work_entries(R, N);
  return FLIDE_OK;
}

int flide_tree_build(const flide_tree_desc *desc, flide_tree_index *idx, flide_stream stream) {
  return tree_build(desc, idx, (cudaStream_t)stream);
}

int flide_fork_attn(const void *q, const void *k, const void *v, const void *past_k,
                    const void *past_v, int32_t past_rows, flide_tree_index *idx, int32_t Hq,
                    int32_t Hkv, int32_t d, int32_t dtype, float scale, void *out,
                    int32_t flags, flide_stream stream) {
  if (!idx || !q || !k || !v || !out) return FLIDE_ERR_SHAPE;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || past_rows < 0) return FLIDE_ERR_SHAPE;
  if ((past_k == nullptr) != (past_v == nullptr)) return FLIDE_ERR_SHAPE;
  if (past_k == nullptr) past_rows = 0;
  if (dtype == FLIDE_E4M3) return FLIDE_ERR_SHAPE;  // needs descale factors: flide_fork_attn_fp8
  if (!(flags & FLIDE_FLAG_PORTABLE) && fork_attn_tc_supported(idx, Hq, Hkv, d, dtype))
    return fork_attn_tc(q, k, v, past_k, past_v, past_rows, idx, Hq, Hkv, dtype, nullptr, scale,
                        out, (cudaStream_t)stream, nullptr);
  return fork_attn_portable(q, k, v, past_k, past_v, past_rows, idx, Hq, Hkv, d, dtype, scale,
                            out, (cudaStream_t)stream);
}

int flide_fork_attn_fp8(const void *q, const void *k, const void *v, const void *past_k,
                        const void *past_v, int32_t past_rows, flide_tree_index *idx, int32_t Hq,
                        int32_t Hkv, int32_t d, const float *descale, float scale, void *out,
                        flide_stream stream) {
  if (!idx || !q || !k || !v || !out || !descale) return FLIDE_ERR_SHAPE;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || past_rows < 0) return FLIDE_ERR_SHAPE;
  if ((past_k == nullptr) != (past_v == nullptr)) return FLIDE_ERR_SHAPE;
  if (past_k == nullptr) past_rows = 0;
  if (!fork_attn_tc_supported(idx, Hq, Hkv, d, FLIDE_E4M3)) return FLIDE_ERR_SHAPE;
  return fork_attn_tc(q, k, v, past_k, past_v, past_rows, idx, Hq, Hkv, FLIDE_E4M3, descale,
                      scale, out, (cudaStream_t)stream, nullptr);
}

int flide_fork_attn_paged(const void *q, const void *k, const void *v, const void *pool_k,
                          const void *pool_v, int32_t n_blocks, int32_t block_rows,
                          const int32_t *block_table, int32_t max_blocks, const int32_t *req_slot,
                          int32_t n_slots, flide_tree_index *idx, int32_t Hq, int32_t Hkv,
                          int32_t d, int32_t dtype, const float *descale, float scale, void *out,
                          flide_stream stream) {
  if (!idx || !q || !k || !v || !out || !pool_k || !pool_v || !block_table || !req_slot)
    return FLIDE_ERR_SHAPE;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return FLIDE_ERR_SHAPE;
  if (n_blocks <= 0 || max_blocks <= 0 || n_slots <= 0 || block_rows <= 0 || block_rows % 128)
    return FLIDE_ERR_SHAPE;
  if ((int64_t)n_blocks * block_rows > 0x7fffffffLL) return FLIDE_ERR_CAPACITY;
  if (dtype == FLIDE_E4M3 && !descale) return FLIDE_ERR_SHAPE;
  if (!fork_attn_tc_supported(idx, Hq, Hkv, d, dtype)) return FLIDE_ERR_SHAPE;
  const PagedPast pp{block_table, req_slot, max_blocks, block_rows, n_blocks, n_slots};
  return fork_attn_tc(q, k, v, pool_k, pool_v, n_blocks * block_rows, idx, Hq, Hkv, dtype,
                      dtype == FLIDE_E4M3 ? descale : nullptr, scale, out, (cudaStream_t)stream,
                      &pp);
}

int flide_fork_gdn(const void *q, const void *k, const void *v, const float *g,
                   const float *beta, const float *state_in, flide_tree_index *idx, int32_t H,
                   int32_t dk, int32_t dv, int32_t dtype, void *out, float *node_state,
                   int32_t n_state_slots, int32_t flags, flide_stream stream) {
  if (!idx || !q || !k || !v || !g || !beta || !out || !node_state) return FLIDE_ERR_SHAPE;
  if (H <= 0 || n_state_slots <= 0) return FLIDE_ERR_SHAPE;
  if (dtype == FLIDE_E4M3) return FLIDE_ERR_SHAPE;  // needs descale factors: flide_fork_gdn_fp8
  if (!(flags & FLIDE_FLAG_PORTABLE) && fork_gdn_tc_supported(dk, dv, dtype))
    return fork_gdn_tc(q, k, v, g, beta, state_in, idx, H, out, node_state, n_state_slots,
                       (cudaStream_t)stream, dtype, nullptr);
  return fork_gdn_portable(q, k, v, g, beta, state_in, idx, H, dk, dv, dtype, out, node_state,
                           n_state_slots, (cudaStream_t)stream);
}

int flide_fork_gdn_fp8(const void *q, const void *k, const void *v, const float *descale,
                       const float *g, const float *beta, const float *state_in,
                       flide_tree_index *idx, int32_t H, int32_t dk, int32_t dv, void *out,
                       float *node_state, int32_t n_state_slots, flide_stream stream) {
  if (!idx || !q || !k || !v || !descale || !g || !beta || !out || !node_state)
    return FLIDE_ERR_SHAPE;
  if (H <= 0 || n_state_slots <= 0) return FLIDE_ERR_SHAPE;
  if (!fork_gdn_tc_supported(dk, dv, FLIDE_E4M3)) return FLIDE_ERR_SHAPE;
  return fork_gdn_tc(q, k, v, g, beta, state_in, idx, H, out, node_state, n_state_slots,
                     (cudaStream_t)stream, FLIDE_E4M3, descale);
}

int flide_state_save(const flide_tree_index *idx, const void *k, const void *v,
                     const void *past_k, const void *past_v, int32_t Hkv, int32_t d,
                     int32_t dtype, const float *node_state, int32_t H, int32_t dk, int32_t dv,
                     void *ckpt_k, void *ckpt_v, float *ckpt_S, int32_t ckpt_rows,
                     flide_stream stream) {
  return state_save(idx, k, v, past_k, past_v, Hkv, d, dtype, node_state, H, dk, dv, ckpt_k,
                    ckpt_v, ckpt_S, ckpt_rows, (cudaStream_t)stream);
}

int flide_state_resume(int32_t R, const int32_t *src_req, int32_t src_R,
                       const int32_t *src_ckpt_start, const void *src_k, const void *src_v,
                       const float *src_S, int32_t Hkv, int32_t d, int32_t dtype, int32_t H,
                       int32_t dk, int32_t dv, int32_t *past_len, void *past_k, void *past_v,
                       int32_t past_rows, float *state_in, int32_t *status,
                       flide_stream stream) {
  return state_resume(R, src_req, src_R, src_ckpt_start, src_k, src_v, src_S, Hkv, d, dtype, H,
                      dk, dv, past_len, past_k, past_v, past_rows, state_in, status,
                      (cudaStream_t)stream);
}

int32_t flide_debug_bounds(void) { return kBoundsChecks ? 1 : 0; }

const char *flide_strerror(int32_t code) {
  switch (code) {
    case FLIDE_OK: return "ok";
    case FLIDE_ERR_INVALID: return "malformed tree or argument";
    case FLIDE_ERR_SHAPE: return "unsupported shape, dtype or null argument";
    case FLIDE_ERR_CAPACITY: return "tree or data exceeds the given capacities";
    case FLIDE_ERR_CUDA: return "CUDA call failed";
    case FLIDE_ERR_TIMEOUT: return "bounded device wait expired";
    case FLIDE_ERR_BOUNDS: return "device index out of bounds (bounds-checked build)";
    default: return "unknown status";
  }
}

}  // extern "C"
