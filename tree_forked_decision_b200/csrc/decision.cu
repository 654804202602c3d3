// decision.cu -- decision scoring over a request's options on the 5th-generation
// tensor cores (sm_100a).
//
// Decision models answer with probabilities over a few candidate options
// (openai-hub.com news article on the Flide release, paragraphs on Jev-like
// decision models), compared to a high-precision reference by total variation
// distance (kongchang.com article on Flide, "total variation distance" box).
// Scoring used here: each leaf of a request's tree is an option whose score is
// the log-likelihood of the branch tokens on its path,
//   log p_t = h_t . w_{y_t} - logsumexp_v (h_t . w_v)      (LM head W [V, D]),
// and the decision is the softmax of the leaves' path scores per request.
//
// flide_branch_logprob: one CTA per (tile of up to 128 branch tokens of one
// request, slice of the vocabulary).  Per vocabulary tile of 128 the CTA forms
// S = H_tile W_tile^T (M = N = 128, K = D in steps of 16; H and W chunks of 64
// columns stream through a 3-stage TMA ring, 128-byte swizzle) in one of two
// TMEM buffers, so four epilogue warps (one row per thread) fold tile v into a
// running max / sum of exponentials (exp2 domain) while the tensor core forms
// tile v+1; the target's logit is picked when its tile passes.  Each CTA writes
// (max, sum, target logit) per row; a merge kernel combines the slices.
// flide_option_probs: per request, segment sums of log p over each node's
// tokens, path sums down the ancestor lists, softmax over the leaves.
// Every wait is bounded (2 s); on expiry the CTA records FLIDE_ERR_TIMEOUT.
#include <cstddef>

#include "common.cuh"
#include "sm100.cuh"

namespace flide {
namespace {

using namespace sm100;

constexpr int BM = 128;        // branch-token rows per CTA
constexpr int BV = 128;        // vocabulary entries per tile
constexpr int KC = 64;         // hidden columns per stage (128 bytes of bf16)
constexpr int kStages = 3;
constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr int SM_H = 0;                      // stage s: s * 16384, 128 rows x 128 B
constexpr int SM_W = kStages * 16384;        // stage s: s * 16384
constexpr int SM_BAR = 2 * kStages * 16384;
constexpr int SM_MISC = SM_BAR + 128;
constexpr int SMEM_BYTES = SM_MISC + 64 + 1024;

enum {
  B_FULL = 0,                 // [kStages]
  B_EMPTY = kStages,          // [kStages]
  B_S_FULL = 2 * kStages,     // [2 TMEM buffers]
  B_S_FREE = 2 * kStages + 2, // [2], 4 epilogue warp arrivals
  B_DRAIN = 2 * kStages + 4,
  NUM_BARS = 2 * kStages + 5
};

struct LpParams {
  flide_tree_index x;
  const int32_t *targets;
  float *partial;  // [n_split][T][3]: max (natural log units), sum of exp, target logit
  int D, V, n_split, tbl;  // tbl: offset of the per-request tile table in x.work
};

__device__ __forceinline__ int upper_bound_i(const int32_t *a, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] > key) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Row tiles of branch tokens per request, prefix-summed into work[tbl .. tbl+R].
__global__ void lp_items_kernel(flide_tree_index x, int tbl) {
  __shared__ int scratch[40];
  if (failed(x.status)) {
    if (threadIdx.x == 0) x.work[tbl + x.R] = 0;
    return;
  }
  const int R = x.R;
  int carry = 0;
  for (int b = 0; b < R; b += blockDim.x) {
    const int r = b + threadIdx.x;
    int cnt = 0;
    if (r < R) {
      const int n0 = x.req_node[r], n1 = x.req_node[r + 1];
      if (n1 > n0) cnt = (x.node_start[n1] - x.node_start[n0 + 1] + BM - 1) / BM;
    }
    int tot;
    const int ex = block_excl_scan(cnt, scratch, &tot);
    if (r < R) x.work[tbl + r] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) x.work[tbl + R] = carry;
}

__global__ void __launch_bounds__(kThreads, 1)
branch_logprob_kernel(const __grid_constant__ CUtensorMap tm_h,
                      const __grid_constant__ CUtensorMap tm_w, const LpParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sb = smem_u32(smem);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM_MISC);
  int *abort_flag = reinterpret_cast<int *>(smem + SM_MISC + 4);
  volatile int *vabort = abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const flide_tree_index &x = p.x;
  auto bar = [&](int i) -> uint32_t { return sb + SM_BAR + 8 * i; };

  // work item: tile of branch rows of one request
  const int R = x.R, item = blockIdx.x, split = blockIdx.y;
  const int32_t *tbl = x.work + p.tbl;
  const bool valid = !failed(x.status) && item < tbl[R];
  int row0 = 0, nrows = 0;
  if (valid) {
    const int r = upper_bound_i(tbl, R + 1, item) - 1;
    const int br = x.node_start[x.req_node[r] + 1], end = x.node_start[x.req_node[r + 1]];
    row0 = br + (item - tbl[r]) * BM;
    nrows = min(BM, end - row0);
  }
  const int nvt = p.V / BV;
  const int v0 = (int)((long)split * nvt / p.n_split), v1 = (int)((long)(split + 1) * nvt / p.n_split);
  const int nkc = p.D / KC;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(bar(i), (i == B_S_FREE || i == B_S_FREE + 1) ? 4u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sb + SM_MISC, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (valid && nrows > 0 && v1 > v0) {
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        prefetch_tmap(&tm_h);
        prefetch_tmap(&tm_w);
        int L = 0;
        bool ok = true;
        for (int v = v0; v < v1 && ok; ++v) {
          for (int kc = 0; kc < nkc; ++kc, ++L) {
            const int st = L % kStages;
            if (L >= kStages && !mbar_wait(bar(B_EMPTY + st), (L / kStages - 1) & 1, vabort, kTimeoutNs)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(B_FULL + st), 2 * BM * KC * 2);
            tma_load_2d(sb + SM_H + st * 16384, &tm_h, bar(B_FULL + st), kc * KC, row0);
            tma_load_2d(sb + SM_W + st * 16384, &tm_w, bar(B_FULL + st), kc * KC, v * BV);
          }
        }
        // drain the copies still in flight into this CTA's shared memory
        for (int l = max(0, L - kStages); l < L; ++l)
          mbar_wait(bar(B_FULL + l % kStages), (l / kStages) & 1, vabort, kTimeoutNs, false);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA
      const uint32_t issue = lane == 0 ? 1u : 0u;
      constexpr uint32_t id = idesc_bf16(BM, BV, false);
      const uint64_t dh = sdesc_sw128(sb + SM_H, 16, 1024), dw = sdesc_sw128(sb + SM_W, 16, 1024);
      auto wait = [&](int b, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar(b), parity, vabort, kTimeoutNs));
      };
      bool ok = true;
      int L = 0;
      for (int v = v0; v < v1 && ok; ++v) {
        const int vi = v - v0, b = vi & 1;
        if (vi >= 2 && !(ok = wait(B_S_FREE + b, ((vi >> 1) - 1) & 1))) break;
        for (int kc = 0; kc < nkc; ++kc, ++L) {
          const int st = L % kStages;
          if (!(ok = wait(B_FULL + st, (L / kStages) & 1))) break;
          tc_fence_after();
          const uint64_t o = (uint64_t)(st * (16384 >> 4));
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ok16 = (uint64_t)(k * (32 >> 4));
            mma_bf16_if(issue, tmem + b * 128, dh + o + ok16, dw + o + ok16, id,
                        (kc > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit_if(issue, bar(B_EMPTY + st));
        }
        if (!ok) break;
        mma_commit_if(issue, bar(B_S_FULL + b));
      }
      // all MMAs issued by this warp complete before TMEM is released
      mma_commit_if(issue, bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, vabort, kTimeoutNs, false);
    } else {
      // ------------------------------------------------------------ epilogue
      const int lg = warp & 3, row = lg * 32 + lane;
      const uint32_t tl = tmem + ((uint32_t)(lg * 32) << 16);
      const bool real = row < nrows;
      const int y = real ? p.targets[row0 + row] : -1;
      // debug build: a target outside the vocabulary would score no logit
      if (real) in_bounds(p.x.status, p.x.counts, y, p.V, 601);
      float m2 = -INFINITY, s = 0.f, tgt = -INFINITY;  // running max (log2 units), sum, target logit
      bool ok = true;
      for (int v = v0; v < v1; ++v) {
        const int vi = v - v0, b = vi & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + b), (vi >> 1) & 1, vabort, kTimeoutNs))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int ycol = y - v * BV;  // target's column in this tile, if any
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t r32[32];
          tmem_ld32(tl + b * 128 + 32 * c4, r32);
          float cm = -INFINITY;
#pragma unroll
          for (int i = 0; i < 32; ++i) cm = fmaxf(cm, __uint_as_float(r32[i]));
          const float mn = fmaxf(m2, cm * kLog2e);
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) acc += ex2_approx(fmaf(__uint_as_float(r32[i]), kLog2e, -mn));
          s = s * ex2_approx(m2 - mn) + acc;
          m2 = mn;
          const int yi = ycol - 32 * c4;  // in [0, 32) when the target is in this chunk
#pragma unroll
          for (int i = 0; i < 32; ++i) tgt = (yi == i) ? __uint_as_float(r32[i]) : tgt;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_S_FREE + b));
      }
      if (ok && real) {
        float *out = p.partial + ((size_t)split * x.T + row0 + row) * 3;
        out[0] = m2 * kLn2;
        out[1] = s;
        out[2] = tgt;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) set_status(x.status, FLIDE_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// log p_t for every branch token from the slices' (max, sum, target logit);
// root tokens get NaN.
__global__ void lp_merge_kernel(flide_tree_index x, const float *partial, int n_split, float *logp) {
  if (failed(x.status)) return;
  const int T = x.counts[FLIDE_CNT_T];
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
    const int n = x.token_node[t];
    if (x.depth[n] == 0) {
      logp[t] = __int_as_float(0x7fc00000);
      continue;
    }
    float M = -INFINITY, tg = -INFINITY;
    for (int sp = 0; sp < n_split; ++sp) {
      const float *q = partial + ((size_t)sp * x.T + t) * 3;
      M = fmaxf(M, q[0]);
      tg = fmaxf(tg, q[2]);
    }
    float S = 0.f;
    for (int sp = 0; sp < n_split; ++sp) {
      const float *q = partial + ((size_t)sp * x.T + t) * 3;
      S += q[1] * __expf(q[0] - M);
    }
    logp[t] = tg - M - __logf(S);
  }
}

// Per request: node segment sums of log p, path sums, softmax over leaves.
__global__ void option_probs_kernel(flide_tree_index x, const float *logp, float *path, float *prob) {
  __shared__ float red[32];
  if (failed(x.status)) return;
  const int r = blockIdx.x;
  const int n0 = x.req_node[r], n1 = x.req_node[r + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (n1 <= n0) return;
  // segment sums (warp per node) into prob[] as scratch
  for (int n = n0 + warp; n < n1; n += nw) {
    float acc = 0.f;
    if (x.depth[n] > 0)
      for (int t = x.node_start[n] + lane; t < x.node_start[n + 1]; t += 32) acc += logp[t];
    acc = warp_sum(acc);
    if (lane == 0) prob[n] = acc;
  }
  __syncthreads();
  // path sums over the non-root ancestors (root .. self lists)
  for (int n = n0 + threadIdx.x; n < n1; n += blockDim.x) {
    float acc = 0.f;
    for (int a = x.anc_ptr[n] + 1; a < x.anc_ptr[n + 1]; ++a) acc += prob[x.anc_node[a]];
    path[n] = acc;
  }
  __syncthreads();
  auto is_leaf = [&](int n) { return x.depth[n] > 0 && x.state_slot[n] < 0; };
  float mx = -INFINITY;
  for (int n = n0 + threadIdx.x; n < n1; n += blockDim.x)
    if (is_leaf(n)) mx = fmaxf(mx, path[n]);
  mx = warp_max(mx);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (warp == 0) {
    float v = lane < nw ? red[lane] : -INFINITY;
    v = warp_max(v);
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  mx = red[0];
  __syncthreads();
  float sm = 0.f;
  for (int n = n0 + threadIdx.x; n < n1; n += blockDim.x)
    if (is_leaf(n)) sm += __expf(path[n] - mx);
  sm = warp_sum(sm);
  if (lane == 0) red[warp] = sm;
  __syncthreads();
  if (warp == 0) {
    float v = lane < nw ? red[lane] : 0.f;
    v = warp_sum(v);
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  sm = red[0];
  for (int n = n0 + threadIdx.x; n < n1; n += blockDim.x)
    prob[n] = is_leaf(n) ? __expf(path[n] - mx) / sm : 0.f;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_lp() {
  static std::atomic<EncodeTiledFn> cached{nullptr};  // host threads may race on a first call
  EncodeTiledFn fn = cached.load(std::memory_order_acquire);
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = (EncodeTiledFn)ptr;
      cached.store(fn, std::memory_order_release);
    }
  }
  return fn;
}

// [rows, cols] bf16 row-major as a 2-D tensor (col, row); box 64 x 128, 128-byte swizzle
bool make_map_2d(CUtensorMap *m, const void *base, long rows, int cols) {
  EncodeTiledFn enc = encode_fn_lp();
  if (!enc || rows <= 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {KC, BM};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Vocabulary slices per row tile.  The host cannot see how many of the T
// stream tokens are branch tokens (that lives on the device), so it splits the
// vocabulary up to this many ways whenever the vocabulary has the tiles: a few
// branch-row tiles then still cover the GPU, and surplus CTAs exit at once.
constexpr int kMaxSplit = 16;

}  // namespace
}  // namespace flide

extern "C" size_t flide_branch_logprob_workspace_bytes(int32_t T, int32_t V) {
  if (T <= 0 || V <= 0) return 0;
  const int nvt = V / flide::BV;
  const int split = nvt < flide::kMaxSplit ? (nvt > 0 ? nvt : 1) : flide::kMaxSplit;
  return (size_t)split * (size_t)T * 3 * sizeof(float);
}

extern "C" int flide_branch_logprob(const void *h, const void *w_lm, const int32_t *targets,
                                    const flide_tree_index *idx, int32_t D, int32_t V,
                                    int32_t dtype, float *logp, void *workspace,
                                    size_t workspace_bytes, flide_stream stream) {
  using namespace flide;
  if (!idx || !h || !w_lm || !targets || !logp || !workspace) return FLIDE_ERR_SHAPE;
  if (dtype != FLIDE_BF16 || D <= 0 || D % KC != 0 || V <= 0 || V % BV != 0) return FLIDE_ERR_SHAPE;
  if (idx->R < 0 || idx->T < 0) return FLIDE_ERR_SHAPE;
  if (idx->work_len < 2 * (int64_t)(idx->R + 1)) return FLIDE_ERR_CAPACITY;
  cudaStream_t s = (cudaStream_t)stream;
  if (idx->T == 0 || idx->R == 0) return FLIDE_OK;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLIDE_ERR_CUDA;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // row tiles: at most T/128 + R
  const long tiles_ub = (long)idx->T / BM + idx->R;
  const int nvt = V / BV;
  int split = max(1, min(nvt, kMaxSplit));
  while (split > 1 && (size_t)split * (size_t)idx->T * 3 * sizeof(float) > workspace_bytes) --split;
  if ((size_t)split * (size_t)idx->T * 3 * sizeof(float) > workspace_bytes) return FLIDE_ERR_CAPACITY;

  CUtensorMap mh, mw;
  if (!make_map_2d(&mh, h, idx->T, D) || !make_map_2d(&mw, w_lm, V, D)) return FLIDE_ERR_CUDA;
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(branch_logprob_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return FLIDE_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
  }
  const int tbl = idx->R + 1;  // work[R+1 .. 2R+2): per-request row-tile table
  lp_items_kernel<<<1, 1024, 0, s>>>(*idx, tbl);
  FLIDE_LAUNCH_CHECK();
  LpParams prm;
  prm.x = *idx;
  prm.targets = targets;
  prm.partial = static_cast<float *>(workspace);
  prm.D = D;
  prm.V = V;
  prm.n_split = split;
  prm.tbl = tbl;
  if (tiles_ub > 0x7fffffffL) return FLIDE_ERR_CAPACITY;
  branch_logprob_kernel<<<dim3((unsigned)tiles_ub, (unsigned)split), kThreads, SMEM_BYTES, s>>>(
      mh, mw, prm);
  FLIDE_LAUNCH_CHECK();
  const int blocks = (int)min(((long)idx->T + 255) / 256, 4L * sms);
  lp_merge_kernel<<<blocks, 256, 0, s>>>(*idx, prm.partial, split, logp);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}

extern "C" int flide_option_probs(const flide_tree_index *idx, const float *logp, float *path_logp,
                                  float *prob, flide_stream stream) {
  using namespace flide;
  if (!idx || !logp || !path_logp || !prob) return FLIDE_ERR_SHAPE;
  if (idx->R <= 0) return FLIDE_OK;
  option_probs_kernel<<<idx->R, 256, 0, (cudaStream_t)stream>>>(*idx, logp, path_logp, prob);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}
