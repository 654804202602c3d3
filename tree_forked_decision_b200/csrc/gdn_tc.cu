// gdn_tc.cu -- Gated DeltaNet fork scan on the 5th-generation tensor cores
// (sm_100a): bf16 or e4m3 q/k/v, dk = dv = 128, fp32 state and accumulation.
//
// Per head the state S (dv x dk) follows the gated delta rule
//   S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,  o_t = S_t q_t.
// Forking (kongchang.com article on Flide, Gated DeltaNet box; techfi24.com,
// "Exact State Forking"): every root scans from its request's state_in (the
// prefix, once) and saves its end state; every other node starts from its
// parent's saved end state; nodes with children save their end state too.
// One launch per tree level, ordered by the stream.
//
// Chunked form used here (C = 64 tokens; the same sums grouped differently,
// equal in exact arithmetic).  With G_i the running sum of g inside the chunk,
// gamma_i = exp(G_i) and S0 the state before the chunk,
//   A_ij = b_i (gamma_i/gamma_j) k_i.k_j  (j < i),   T = (I + A)^-1,
//   W = T diag(b gamma) K,   U = T diag(b) V,   Delta = U - W S0^T,
//   O = diag(gamma) Q S0^T + (M o QK^T) Delta,  M_ij = gamma_i/gamma_j (j <= i),
//   S_end = gamma_last S0 + Delta^T diag(gamma_last/gamma) K.
// Only the last three lines need the state; everything above them is a
// function of the chunk's own inputs.  The kernel below (gdn_ws_kernel) runs
// the two parts in different warps, chunk c+1's state-free part while chunk
// c's state products run.
//
// Work items (built per level by gdn_groups_kernel): a root, an inner node or
// a node longer than one chunk is a "scan" item (its chunks in order, state
// carried in TMEM, end state saved when the node has a slot); runs of
// consecutive sibling leaves that fit one chunk are packed into one item with
// a block-diagonal mask, so no leaf sees another.  Items x heads are spread
// over a persistent grid of one CTA per SM that takes them, longest group
// first, from a shared counter.  Every wait is bounded (2 s).
#include <cstddef>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "sm100.cuh"

namespace flide {
namespace {

using namespace sm100;

constexpr int C = 64;    // tokens per chunk
constexpr int D = 128;   // dk = dv
constexpr uint64_t kTimeoutNs = 2000000000ull;

struct GdnTcParams {
  flide_tree_index x;
  const float *descale;  // e4m3 inputs: {q, k, v} descale factors
  const float *g, *beta, *state_in;
  __nv_bfloat16 *out;
  float *node_state;
  int H, n_slots, level, goff;
};

// work[goff] = number of groups; work[goff+1+g] = first level position of
// group g; work[goff+2+N+g] = its node count; work[goff+2+2N+k] = the group
// of rank k, longest first; work[goff+2+3N] = the next item to hand out.
__device__ __forceinline__ int *groups_n(const flide_tree_index &x, int goff) { return x.work + goff; }
__device__ __forceinline__ int *groups_start(const flide_tree_index &x, int goff) {
  return x.work + goff + 1;
}
__device__ __forceinline__ int *groups_count(const flide_tree_index &x, int goff) {
  return x.work + goff + 2 + x.N;
}
__device__ __forceinline__ int *groups_order(const flide_tree_index &x, int goff) {
  return x.work + goff + 2 + 2 * x.N;
}
__device__ __forceinline__ int *groups_next(const flide_tree_index &x, int goff) {
  return x.work + goff + 2 + 3 * x.N;
}
constexpr int kMaxSortedGroups = 2048;  // more groups than this keep level order

// Groups the nodes of one level: a root, a node with a state slot or a node
// longer than a chunk is alone; consecutive leaves (consecutive ids) with the
// same parent are packed greedily while they fit one chunk.
__global__ void gdn_groups_kernel(flide_tree_index x, int level, int goff) {
  __shared__ int scratch[40];
  int *flag = groups_count(x, goff);  // temporary flags, then counts
  int *gstart = groups_start(x, goff);
  if (failed(x.status)) {
    if (threadIdx.x == 0) {
      *groups_n(x, goff) = 0;
      *groups_next(x, goff) = 0;
    }
    return;
  }
  const int L0 = x.level_ptr[level], n = x.level_ptr[level + 1] - L0;
  auto seg = [&](int node) { return x.node_start[node + 1] - x.node_start[node]; };
  auto alone = [&](int node) { return level == 0 || x.state_slot[node] >= 0 || seg(node) > C; };
  auto parent_of = [&](int node) { return x.anc_node[x.anc_ptr[node + 1] - 2]; };
  // 1: run starts
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    const int node = x.level_node[L0 + k];
    // debug build: a level's nodes index the tree arrays
    if (!in_bounds(x.status, x.counts, node, x.counts[FLIDE_CNT_N], 311) ||
        (k > 0 && !in_bounds(x.status, x.counts, x.level_node[L0 + k - 1], x.counts[FLIDE_CNT_N], 311))) {
      flag[k] = 1;
      continue;
    }
    int f = 1;
    if (k > 0) {
      const int prev = x.level_node[L0 + k - 1];
      f = alone(node) || alone(prev) || prev + 1 != node || parent_of(prev) != parent_of(node);
    }
    flag[k] = f;
  }
  __syncthreads();
  // 2: one thread per run packs it greedily by tokens
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    if (!flag[k]) continue;
    int tok = 0;
    for (int e = k; e < n && (e == k || !flag[e]); ++e) {
      const int sl = seg(x.level_node[L0 + e]);
      if (e > k && tok + sl > C) {
        flag[e] = 2;  // starts a new group inside the run
        tok = 0;
      }
      tok += sl;
    }
  }
  __syncthreads();
  // 3: compact the group starts
  int carry = 0;
  for (int b = 0; b < n; b += blockDim.x) {
    const int k = b + threadIdx.x;
    const int f = (k < n && flag[k] != 0) ? 1 : 0;
    int tot;
    const int ex = block_excl_scan(f, scratch, &tot);
    if (f) gstart[carry + ex] = k;
    carry += tot;
  }
  __syncthreads();
  // 4: counts
  for (int g = threadIdx.x; g < carry; g += blockDim.x)
    flag[g] = (g + 1 < carry ? gstart[g + 1] : n) - gstart[g];
  __syncthreads();
  // 5: hand-out order, longest group (in tokens) first, so the persistent
  //    CTAs' greedy pick-up of items stays balanced; ties keep level order
  __shared__ int len[kMaxSortedGroups];
  int *order = groups_order(x, goff);
  if (carry <= kMaxSortedGroups) {
    for (int g = threadIdx.x; g < carry; g += blockDim.x) {
      const int first = x.level_node[L0 + gstart[g]], last = x.level_node[L0 + gstart[g] + flag[g] - 1];
      len[g] = x.node_start[last + 1] - x.node_start[first];
    }
    __syncthreads();
    for (int g = threadIdx.x; g < carry; g += blockDim.x) {
      const int lg = len[g];
      int rank = 0;
      for (int o = 0; o < carry; ++o) rank += (len[o] > lg) || (len[o] == lg && o < g);
      order[rank] = g;
    }
  } else {
    for (int g = threadIdx.x; g < carry; g += blockDim.x) order[g] = g;
  }
  if (threadIdx.x == 0) {
    *groups_n(x, goff) = carry;
    *groups_next(x, goff) = 0;
  }
}

// Self-check (both builds): records the first failed check of a work item
// (site, value) in the index's check slots and FLIDE_ERR_INVALID in the status
// word; the caller skips the item.
__device__ __forceinline__ void check_fail(const flide_tree_index &x, int site, long val) {
  if (atomicCAS(&x.counts[FLIDE_CNT_CHECK_SITE], 0, site) == 0) x.counts[FLIDE_CNT_CHECK_VALUE] = (int)val;
  set_status(x.status, FLIDE_ERR_INVALID);
}

// 8 bf16 values (one 16-byte chunk q of a 128-byte row) into a swizzled row
__device__ __forceinline__ void st_chunk(uint8_t *base, int row, int q, uint4 v) {
  *reinterpret_cast<uint4 *>(base + row * 128 + ((q ^ (row & 7)) << 4)) = v;
}

// 16 x 16 x 16 block products of the triangular solve on the warp's tensor
// path: mma.sync m16n8k8 with tf32 inputs (rounded to nearest) and fp32
// accumulation.  Fragments (g = lane / 4, t = lane % 4): A rows g, g+8 and
// columns t, t+4 of each 8-wide K step; B rows t, t+4 of the step and column
// g of each 8-wide N tile; the accumulator holds rows g, g+8 and columns 2t,
// 2t+1 of each N tile.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint4 pack8(const float *f) {
  uint4 v;
  v.x = pack_bf16x2(f[0], f[1]);
  v.y = pack_bf16x2(f[2], f[3]);
  v.z = pack_bf16x2(f[4], f[5]);
  v.w = pack_bf16x2(f[6], f[7]);
  return v;
}

// 16 e4m3 codes (one 16-byte chunk) to 16 floats, exactly
__device__ __forceinline__ void decode16_e4m3(uint4 raw, float (&f)[16]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const __half2_raw hr =
          __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> (16 * h2)), __NV_E4M3);
      const float2 f2 = __half22float2(__half2(hr));
      f[4 * i + 2 * h2] = f2.x;
      f[4 * i + 2 * h2 + 1] = f2.y;
    }
  }
}

// ---- warp-specialised fork scan ---------------------------------------------
//
// The same chunked form, with the chunk's work split by what it depends on.
// Everything but the state products -- the segmented gate scan, [Q;K][Q;K]^T,
// the decay masks, T = (I + A)^-1, W, U and the bf16 operand tiles -- depends
// only on the chunk's own inputs, so a "prep" warpgroup computes it for chunk
// c+1 while a "chain" warpgroup runs chunk c's state products:
//   X = [U; 0] + [-W; diag(gamma) Q] S0^T       (rows 0-63: Delta, 64-127: gamma Q S0^T)
//   X[64:] += (M o QK^T) Delta                   (the chunk's outputs)
//   S = gamma_last S0 + Delta'^T K               (Delta' = Delta gamma_last / gamma)
// With gamma folded into Q's rows the output needs no second accumulator; the
// extra rounding is one bf16 rounding of gamma_i q_i, like the bf16 copy of S0.
// Roles (512 threads): warps 0-7 prep (two per TMEM lane quadrant), 8
// producer (items, per-token scalars, TMA), 10-11 epilogue (output rows, TMEM
// lanes 64-127), 12-15 chain (TMEM lanes 0-127); warp 9 idles.  A warp reaches
// TMEM lanes 32 (w % 4) .. +31.  The producer runs ahead through a ring of four chunk
// jobs, so the pipeline flows across items: a new item's first chunk starts
// from its parent's state (global) while the previous item drains.  Every
// handshake is an mbarrier whose next phase can only complete after its waiter
// has consumed the current one, and every wait is bounded.  One thread of a
// role polls a barrier while the rest of the role parks on a named barrier.  The chain's tiles
// are single-buffered: the prep writes [-W; gamma Q] for chunk c+1 once chunk
// c's first product has read them, and copies K once c's update has.
namespace ws {

constexpr int kThreads = 512;
// Role of each warp (the critical prep warpgroup first).
constexpr int kPrepWarp0 = 0, kPrepWarps = 8, kProducerWarp = 8, kEpiWarp0 = 10, kChainWarp0 = 12;
constexpr int BAR_PREP = 1, BAR_CHAIN = 2, BAR_EPI = 3;  // named barriers

// shared-memory map, bytes from a 1024-aligned base
constexpr int KQ = 0;          // stage s at +32768 s; dk slab b at +16384 b: Q rows at +0, K rows at +8192
constexpr int V = 65536;       // dv slab b at +8192 b (64 token rows)
constexpr int MQK = 81920;     // stage s at +8192 s: rows 64-127 of a [junk; M o QK^T] A tile
constexpr int CA = 98304;      // [-W; gamma Q] A tile, dk slab b at +16384 b
constexpr int CK = 131072;     // K rows for the state update (MN-major B), dk slab b at +8192 b
constexpr int SD = 147456;     // bf16 S0 (dk slab b at +16384 b); then Delta (+0) and Delta' (+16384)
constexpr int TT = 180224;     // T' (+0), T'' (+8192), zeros (+16384); solve scratch during the solve
constexpr int PM = 204800;     // fp32 [64][68]: T below the diagonal, A^T above it
constexpr int P_LD = 68;       // row stride: 16-byte rows, and 8 consecutive rows on distinct banks
constexpr int JOB = PM + C * P_LD * 4;  // 4 chunk jobs
constexpr int JOB_BYTES = 1600;
constexpr int BARS = JOB + 4 * JOB_BYTES;
enum {
  KQ_FULL = 0, KQ_EMPTY = 2, V_FULL = 4, V_EMPTY = 5, JOB_FULL = 6, JOB_FREE = 10, GRAM = 14,
  WU = 15, READY = 16, CA_FREE = 17, XDONE = 18, SO = 19, XFREE = 21, DRAIN_P = 23,  // SO: 2
  DRAIN_C = 24, CK_FREE = 25, NBARS = 26
};
constexpr int MISC = BARS + 8 * NBARS;  // TMEM address, abort flag
constexpr int SMEM_BYTES = MISC + 16 + 1024;
static_assert(JOB % 16 == 0 && BARS % 8 == 0, "job slots and barriers must be aligned");
static_assert(SMEM_BYTES <= 232448, "shared memory over the 227 KB limit");

// TMEM columns
// S: state; X: [U; 0] -> [Delta; gamma Q S0^T] -> outputs; G: [Q;K][Q;K]^T,
// written for chunk c+1 while chunk c is solved; W: T' K
constexpr uint32_t T_S = 0, T_X = 128, T_G = 256, T_W = 384;

// One chunk of one (item, head), written by the producer: header, beta, the
// segmented log2 decay G2, gamma = 2^G2, the separable decay factors
// f_j = 2^(gref - G2_j), the state-update scales gamma_last / gamma_j and each
// token's segment start; read by the prep, the chain and the epilogue.
struct Job {
  int stop, cbeg, n, h, first, update, save, sep;
  const float *src;  // first chunk: start state [dv][dk], nullptr = zero
  float *dst;        // save: end state [dv][dk]
  float gam_last, gref, pad0, pad1;
  float beta[C], g2[C], gam[C], f[C], dsc[C];
  int lo[C];  // first token of the token's segment (C for tokens past the chunk)
};
static_assert(sizeof(Job) <= JOB_BYTES, "job slot too small");

__device__ __forceinline__ void role_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// every thread of the role gets the AND of the role's predicates
__device__ __forceinline__ bool role_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// fp32 tile entry T(r, c) of the solve area: below the diagonal the solved
// value, 1 on it, 0 above (where A^T is kept)
__device__ __forceinline__ float t_at(const float *Pm, int r, int c) {
  return r > c ? Pm[r * P_LD + c] : (r == c ? 1.f : 0.f);
}
// A(r, c) for r > c, kept transposed above the diagonal
__device__ __forceinline__ float a_at(const float *Pm, int r, int c) { return Pm[c * P_LD + r]; }

// acc (16 x 8) += X (16 x 16) Y (16 x 8) with tf32 inputs (m16n8k8, two K
// steps); X and Y given as element functions
template <typename FX, typename FY>
__device__ __forceinline__ void mma16x8(float (&acc)[4], FX X, FY Y, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int kk = 0; kk < 16; kk += 8) {
    mma_tf32_16x8x8(acc, to_tf32(X(g, kk + t)), to_tf32(X(g + 8, kk + t)), to_tf32(X(g, kk + t + 4)),
                    to_tf32(X(g + 8, kk + t + 4)), to_tf32(Y(kk + t, g)), to_tf32(Y(kk + t + 4, g)));
  }
}

// Per-token scalars of one chunk into its job, one warp, two consecutive
// tokens (t0 = 2 lane, t0 + 1) per lane: the segmented inclusive scan of g
// (segments = the nodes of a packed group; s0/s1 = segment ids, -1 past the
// chunk), G2 = log2 decay, gamma, the separable factors, the state-update
// scales gamma_last / gamma_j and each token's segment start.  Kept out of
// line: inlined into the producer loop its shuffle chain was scheduled badly.
__device__ __noinline__ void gate_scan(Job *jb, int lane, int n, float b0, float b1, float a0,
                                       float a1, int s0, int s1) {
  const int t0 = 2 * lane, t1 = t0 + 1;
  const bool v0 = s0 >= 0, v1 = s1 >= 0;
  const int prev_s1 = __shfl_up_sync(0xffffffffu, s1, 1);
  const bool cont0 = lane > 0 && prev_s1 == s0;  // token t0 continues token t0 - 1
  float v = (s1 == s0) ? a0 + a1 : a1;
  int f = (s1 != s0 || !cont0) ? 1 : 0;
  const int st0 = cont0 ? -1 : t0, st1 = (s1 == s0) ? -1 : t1;  // segment starts
  int m = max(st0, st1);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float pv = __shfl_up_sync(0xffffffffu, v, o);
    const int pf = __shfl_up_sync(0xffffffffu, f, o);
    const int pm = __shfl_up_sync(0xffffffffu, m, o);
    if (lane >= o) {
      if (!f) v += pv;
      f |= pf;
      m = max(m, pm);
    }
  }
  const float carry = __shfl_up_sync(0xffffffffu, v, 1);
  const int mprev = __shfl_up_sync(0xffffffffu, m, 1);
  const int lo0 = max(lane > 0 ? mprev : -1, st0), lo1 = max(lo0, st1);
  const float G0 = a0 + (cont0 ? carry : 0.f);
  const float g0 = G0 * 1.4426950408889634f;
  const float g1 = ((s1 == s0) ? G0 + a1 : a1) * 1.4426950408889634f;
  float mx = fmaxf(v0 ? g0 : -INFINITY, v1 ? g1 : -INFINITY);
  float mn = fminf(v0 ? g0 : INFINITY, v1 ? g1 : INFINITY);
  mx = warp_max(mx);
  mn = -warp_max(-mn);
  const bool sep = !(mx - mn > 100.f);  // also true when no token is valid
  const float gref = (mx >= mn) ? 0.5f * (mx + mn) : 0.f;
  const float glast = __shfl_sync(0xffffffffu, (n - 1) & 1 ? g1 : g0, (n - 1) >> 1);
  jb->beta[t0] = b0;
  jb->beta[t1] = b1;
  jb->g2[t0] = g0;
  jb->g2[t1] = g1;
  jb->gam[t0] = ex2_approx(g0);
  jb->gam[t1] = ex2_approx(g1);
  jb->f[t0] = sep ? ex2_approx(gref - g0) : 0.f;
  jb->f[t1] = sep ? ex2_approx(gref - g1) : 0.f;
  jb->dsc[t0] = v0 ? ex2_approx(glast - g0) : 0.f;
  jb->dsc[t1] = v1 ? ex2_approx(glast - g1) : 0.f;
  jb->lo[t0] = v0 ? lo0 : C;
  jb->lo[t1] = v1 ? lo1 : C;
  if (lane == 0) {
    jb->gam_last = ex2_approx(glast);
    jb->gref = gref;
    jb->sep = sep ? 1 : 0;
  }
}

}  // namespace ws

template <bool F8>
__global__ void __launch_bounds__(ws::kThreads, 1)
gdn_ws_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const GdnTcParams p) {
  using namespace ws;
  extern __shared__ uint8_t smem_raw[];
  // 1024-aligned base by pointer arithmetic on the shared array, so the
  // compiler keeps the shared address space (shared, not generic, accesses)
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const flide_tree_index &x = p.x;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + MISC);
  int *abort_flag = reinterpret_cast<int *>(smem + MISC + 4);
  auto bar = [&](int i) -> uint32_t { return sb + BARS + 8 * i; };
  auto job = [&](int j) -> Job * { return reinterpret_cast<Job *>(smem + JOB + j * JOB_BYTES); };
  const float dsq = F8 ? p.descale[0] : 1.f, dsk = F8 ? p.descale[1] : 1.f,
              dsv = F8 ? p.descale[2] : 1.f;

  if (tid == 0) {
    for (int i = 0; i < NBARS; ++i) mbar_init(bar(i), i >= JOB_FREE && i < JOB_FREE + 4 ? 2 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // the zero rows of the [T''; 0] tile
  for (int i = tid; i < 8192 / 16; i += ws::kThreads)
    reinterpret_cast<uint4 *>(smem + TT + 16384)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(sb + MISC, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int *vabort = abort_flag;
  const int Tact = x.counts[FLIDE_CNT_T];

  if (warp == kProducerWarp) {
    // ---------------- producer: items -> chunk jobs, per-token scalars, TMA
    const int n_groups = failed(x.status) ? 0 : *groups_n(x, p.goff);
    const int L0 = x.level_ptr[p.level];
    const long long items = (long long)n_groups * p.H;
    const int Nact = x.counts[FLIDE_CNT_N];
    uint32_t seq = 0;
    int last_kq[2] = {-1, -1}, last_v = -1;  // last issued load per buffer (drain)
    bool ok = true;
    auto wait_w = [&](uint32_t b, uint32_t parity) -> bool {  // lane 0 polls
      bool r = true;
      if (lane == 0) r = mbar_wait(b, parity, vabort, kTimeoutNs);
      return __shfl_sync(0xffffffffu, (int)r, 0) != 0;
    };
    // claims job slot `seq` (all lanes), false if the wait gave up
    auto claim = [&](Job *&jb) -> bool {
      if (!wait_w(bar(JOB_FREE + (seq & 3)), ((seq >> 2) & 1) ^ 1)) return false;
      jb = job(seq & 3);
      return true;
    };
    // V of the previous chunk (issued one chunk behind its K and Q)
    bool pend_v = false;
    uint32_t pv_seq = 0;
    int pv_cbeg = 0, pv_h = 0;
    auto issue_v = [&]() -> bool {
      if (!pend_v) return true;
      if (!wait_w(bar(V_EMPTY), (pv_seq & 1) ^ 1)) return false;
      if (lane == 0) {
        const uint32_t vb = sb + V, fb = bar(V_FULL);
        if (F8) {
          mbar_arrive_expect_tx(fb, 8192);
          tma_load_3d(vb + 8192, &tm_v, fb, 0, pv_h, pv_cbeg);
        } else {
          mbar_arrive_expect_tx(fb, 16384);
          tma_load_3d(vb, &tm_v, fb, 0, pv_h, pv_cbeg);
          tma_load_3d(vb + 8192, &tm_v, fb, 64, pv_h, pv_cbeg);
        }
      }
      last_v = (int)pv_seq;
      pend_v = false;
      return true;
    };
    for (;;) {
      unsigned long long it = 0;
      if (lane == 0) it = (unsigned long long)atomicAdd(groups_next(x, p.goff), 1);
      it = __shfl_sync(0xffffffffu, it, 0);
      bool stop = (long long)it >= items || *vabort;
      int h = 0, tbeg = 0, tend = 0, n0 = 0, slot = -1, r = 0, cnt = 0;
      const float *src = nullptr;
      if (!stop) {
        const int rk = (int)(it / p.H);
        h = (int)(it % p.H);
        const int grp = groups_order(x, p.goff)[rk];
        int site = 0;
        long val = 0;
        int k0 = 0;
        if (grp < 0 || grp >= n_groups) {
          site = 6; val = grp;
        } else {
          k0 = groups_start(x, p.goff)[grp];
          cnt = groups_count(x, p.goff)[grp];
          if (k0 < 0 || cnt < 1 || L0 + k0 + cnt > Nact) { site = 1; val = k0 * 100000L + cnt; }
        }
        int n1 = 0;
        if (!site) {
          n0 = x.level_node[L0 + k0];
          n1 = x.level_node[L0 + k0 + cnt - 1];
          if (n0 < 0 || n1 < n0 || n1 >= Nact) { site = 2; val = n0 * 100000L + n1; }
        }
        if (!site) {
          tbeg = x.node_start[n0];
          tend = x.node_start[n1 + 1];
          if (tbeg < 0 || tend < tbeg || tend > Tact) { site = 3; val = tend; }
        }
        if (!site) {
          slot = x.state_slot[n0];
          r = x.node_req[n0];
          if (r < 0 || r >= x.R || (slot >= 0 && slot >= p.n_slots)) { site = 4; val = r * 100000L + slot; }
        }
        if (!site) {
          if (p.level == 0) {
            if (p.state_in) src = p.state_in + ((size_t)r * p.H + h) * D * D;
          } else {
            const int pa = x.anc_ptr[n0 + 1] - 2;
            // debug build: the parent entry and the parent node index the tree arrays
            const bool pok = pa >= 0 && x.depth[n0] >= 1 &&
                             in_bounds(x.status, x.counts, pa, (long long)x.N * (x.max_depth + 1), 313) &&
                             in_bounds(x.status, x.counts, x.anc_node[pa], Nact, 314);
            const int ps = pok ? x.state_slot[x.anc_node[pa]] : -1;
            if (ps < 0 || ps >= p.n_slots) { site = 5; val = ps; }
            else src = p.node_state + ((size_t)ps * p.H + h) * D * D;
          }
        }
        if (site) {
          if (lane == 0) check_fail(x, site, val);
          stop = true;
        }
      }
      if (stop) {
        if (!issue_v()) { ok = false; break; }
        Job *jb;
        if (!claim(jb)) { ok = false; break; }
        if (lane == 0) jb->stop = 1;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(JOB_FULL + (seq & 3)));
        break;
      }
      const bool scan = cnt == 1;
      float *dst = (scan && slot >= 0) ? p.node_state + ((size_t)slot * p.H + h) * D * D : nullptr;
      const int nchunks = (tend - tbeg + C - 1) / C;
      if (nchunks == 0) {
        // a node without tokens (a root whose prefix is all past): its end
        // state is its start state
        if (dst) {
          for (int i = lane; i < D * D / 4; i += 32)
            reinterpret_cast<float4 *>(dst)[i] =
                src ? reinterpret_cast<const float4 *>(src)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      for (int c = 0; c < nchunks; ++c, ++seq) {
        Job *jb;
        if (!claim(jb)) { ok = false; break; }
        const int cbeg = tbeg + c * C;
        const int n = min(C, tend - cbeg);
        // the job first: per-token scalars and the gate scan, as soon as the
        // slot is free, so the scan (slow next to the prep's shared-memory
        // traffic) is done long before the prep starts this chunk
        const int t0 = 2 * lane, t1 = t0 + 1;
        const bool v0 = t0 < n && cbeg + t0 < Tact, v1 = t1 < n && cbeg + t1 < Tact;
        const size_t i0 = (size_t)(cbeg + t0) * p.H + h, i1 = i0 + p.H;
        const float b0 = v0 ? p.beta[i0] : 0.f, b1 = v1 ? p.beta[i1] : 0.f;
        const float a0 = v0 ? p.g[i0] : 0.f, a1 = v1 ? p.g[i1] : 0.f;
        const int s0 = v0 ? x.token_node[cbeg + t0] - n0 : -1;
        const int s1 = v1 ? x.token_node[cbeg + t1] - n0 : -1;
        // debug build: a token of the item belongs to one of its nodes
        if (v0) in_bounds(x.status, x.counts, s0, cnt, 315);
        if (v1) in_bounds(x.status, x.counts, s1, cnt, 315);
        if (lane == 0) {
          jb->stop = 0;
          jb->cbeg = cbeg;
          jb->n = n;
          jb->h = h;
          jb->first = c == 0;
          jb->update = scan && (c + 1 < nchunks || slot >= 0);
          jb->save = scan && slot >= 0 && c + 1 == nchunks;
          jb->src = src;
          jb->dst = dst;
        }
        gate_scan(jb, lane, n, b0, b1, a0, a1, s0, s1);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(JOB_FULL + (seq & 3)));
        // then K and Q into stage s
        const int s = seq & 1;
        if (!wait_w(bar(KQ_EMPTY + s), ((seq >> 1) & 1) ^ 1)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t kq = sb + KQ + s * 32768, fb = bar(KQ_FULL + s);
          if (F8) {  // e4m3 codes (one 128-byte row per token) into the second slabs
            mbar_arrive_expect_tx(fb, 16384);
            tma_load_3d(kq + 16384, &tm_q, fb, 0, h, cbeg);
            tma_load_3d(kq + 16384 + 8192, &tm_k, fb, 0, h, cbeg);
          } else {
            mbar_arrive_expect_tx(fb, 32768);
            tma_load_3d(kq, &tm_q, fb, 0, h, cbeg);
            tma_load_3d(kq + 16384, &tm_q, fb, 64, h, cbeg);
            tma_load_3d(kq + 8192, &tm_k, fb, 0, h, cbeg);
            tma_load_3d(kq + 16384 + 8192, &tm_k, fb, 64, h, cbeg);
          }
        }
        last_kq[s] = (int)(seq >> 1);
        // the previous chunk's V: its buffer frees when that chunk's prep
        // has used the previous V, long before this point in steady state
        if (!issue_v()) { ok = false; break; }
        pend_v = true;
        pv_seq = seq;
        pv_cbeg = cbeg;
        pv_h = h;
      }
      if (!ok) break;
    }
    // every issued load lands before the CTA can exit
    if (lane == 0) {
      for (int s = 0; s < 2; ++s)
        if (last_kq[s] >= 0) mbar_wait(bar(KQ_FULL + s), last_kq[s] & 1, vabort, kTimeoutNs, false);
      if (last_v >= 0) mbar_wait(bar(V_FULL), last_v & 1, vabort, kTimeoutNs, false);
    }
    __syncwarp();
  } else if (warp >= kPrepWarp0 && warp < kPrepWarp0 + kPrepWarps) {
    // ---------------- prep: everything of a chunk that does not need the state.
    // Two warps per TMEM lane quadrant (warps w and w + 4); the second of each
    // pair takes the other half of every column range.
    const int pt = tid - kPrepWarp0 * 32;         // 0 .. 255
    const int pw = warp - kPrepWarp0;             // 0 .. 7
    const int hb = pw >> 2;                       // column half
    const int row = (warp & 3) * 32 + lane;       // this thread's TMEM lane
    const uint32_t tlp = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    float *Pm = reinterpret_cast<float *>(smem + PM);
    float *Xs = reinterpret_cast<float *>(smem + TT);  // 4 blocks of 16 x 17 during the solve
    constexpr int XS_LD = 17;
    constexpr int NP = 32 * kPrepWarps;
    bool issued = false;  // MMAs in flight (pt == 0), for the drain
    auto wait_r = [&](uint32_t b, uint32_t parity) -> bool {  // one poller, the rest park
      bool r = true;
      if (pt == 0) r = mbar_wait(b, parity, vabort, kTimeoutNs);
      return role_and(BAR_PREP, NP, r);
    };
    // e4m3 codes (one swizzled 128-byte row per token, staged in the second
    // slab) -> the bf16 tiles: dims 0-63 to the first slab, dims 64-127 over
    // the codes themselves, so every code is read before any is overwritten.
    // Exact: every e4m3 value is a bf16 value.  base = first slab, ss = slab
    // stride, tiles = 8 KB tiles per slab (tile t at +8192 t).
    auto expand_e4m3 = [&](uint8_t *base, int ss, int tiles) {
      uint4 raw[4];
      const int per = tiles * C * 8 / NP;  // 16-byte code chunks per thread (2 or 4)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (u >= per) break;
        const int e = pt + NP * u, tt = e >> 9, r = (e >> 3) & (C - 1), j = e & 7;
        raw[u] = *reinterpret_cast<const uint4 *>(base + ss + tt * 8192 + r * 128 + ((j ^ (r & 7)) << 4));
      }
      role_sync(BAR_PREP, NP);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (u >= per) break;
        const int e = pt + NP * u, tt = e >> 9, r = (e >> 3) & (C - 1), j = e & 7;
        float f[16];
        decode16_e4m3(raw[u], f);
        uint8_t *dst = base + (j >> 2) * ss + tt * 8192;
        st_chunk(dst, r, 2 * (j & 3), pack8(f));
        st_chunk(dst, r, 2 * (j & 3) + 1, pack8(f + 8));
      }
    };
    // A chunk's start: its job, its Q and K (rows past its tokens zeroed:
    // they may hold another node's tokens or uninitialised memory) and its
    // [Q;K][Q;K]^T into G.  1 = the producer's stop job, -1 = a wait gave up.
    auto start_chunk = [&](uint32_t sq) -> int {
      // the job and its [Q;K] tiles (a stop job has none), one barrier
      bool r = true;
      if (pt == 0) {
        r = mbar_wait(bar(JOB_FULL + (sq & 3)), (sq >> 2) & 1, vabort, kTimeoutNs);
        if (r && !job(sq & 3)->stop) r = mbar_wait(bar(KQ_FULL + (sq & 1)), (sq >> 1) & 1, vabort, kTimeoutNs);
      }
      if (!role_and(BAR_PREP, NP, r)) return -1;
      const Job *jn = job(sq & 3);
      if (jn->stop) return 1;
      const int nn = jn->n, ss = sq & 1;
      uint8_t *kqn = smem + KQ + ss * 32768;
      if (F8) {
        expand_e4m3(kqn, 16384, 2);
        if (nn < C) role_sync(BAR_PREP, NP);  // the zeroing below rewrites expanded rows
      }
      if (nn < C) {
        for (int e = pt; e < 4 * C * 8; e += NP) {  // (slab, Q|K, row, 16-byte chunk)
          const int r = (e >> 3) & (C - 1);
          if (r >= nn)
            *reinterpret_cast<uint4 *>(kqn + (e >> 10) * 16384 + ((e >> 9) & 1) * 8192 + r * 128 +
                                       (e & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (F8 || nn < C) {
        fence_proxy_async_smem();
        role_sync(BAR_PREP, NP);
      }
      if (pt == 0) {
        tc_fence_after();
        const uint32_t kqa = sb + KQ + ss * 32768;
        constexpr uint32_t id = idesc_bf16(128, 128, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t d = sdesc_sw128(kqa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          mma_bf16(tmem + T_G, d, d, id, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(GRAM));
        issued = true;
      }
      __syncwarp();
      return 0;
    };
    int next = start_chunk(0);
    for (uint32_t seq = 0; next == 0; ++seq) {
      Job *jb = job(seq & 3);
      const int n = jb->n, s = seq & 1;
      const uint32_t kq = sb + KQ + s * 32768;
      uint8_t *kqp = smem + KQ + s * 32768;
      if (!wait_r(bar(GRAM), seq & 1)) break;
      tc_fence_after();
      // -- 3. decay masks from the Gram columns 64-127 (k_j): rows 0-63 are
      //       q_i . k_j -> (M o QK^T) in bf16; rows 64-127 are k_i . k_j -> A
      //       (fp32, kept transposed above the diagonal of the solve area)
      {
        const bool sep = jb->sep != 0;
        const bool qrow = row < C;
        const int i = row & (C - 1);
        const float G2i = jb->g2[i];
        const int lo = jb->lo[i], hi = qrow ? i : i - 1;  // visible j: lo <= j <= hi
        const float sc = qrow ? dsq * dsk : jb->beta[i] * (dsk * dsk);
        const float ei = sc * (sep ? ex2_approx(G2i - jb->gref) : 1.f);
        uint32_t d[32];
        tmem_ld32(tlp + T_G + 64 + 32 * hb, d);
        uint8_t *mq = smem + MQK + s * 8192;
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // 8 columns at a time
          const int j0 = 32 * hb + 8 * q;
          const float4 fa = reinterpret_cast<const float4 *>(sep ? jb->f : jb->g2)[j0 >> 2];
          const float4 fb = reinterpret_cast<const float4 *>(sep ? jb->f : jb->g2)[(j0 >> 2) + 1];
          const float fj[8] = {fa.x, fa.y, fa.z, fa.w, fb.x, fb.y, fb.z, fb.w};
          float e[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = j0 + u;
            const float ratio = sep ? ei * fj[u] : ei * ex2_approx(G2i - fj[u]);
            e[u] = (j >= lo && j <= hi) ? ratio * __uint_as_float(d[8 * q + u]) : 0.f;
          }
          if (qrow) {
            st_chunk(mq, i, 4 * hb + q, pack8(e));
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              if (j0 + u < i) Pm[(j0 + u) * P_LD + i] = e[u];
          }
        }
      }
      tc_fence_before();
      role_sync(BAR_PREP, NP);
      // the next chunk's job, Q, K and Gram, behind this chunk's solve
      next = start_chunk(seq + 1);
      if (next < 0) break;
      // -- 4. T = (I + A)^-1: the four diagonal 16 x 16 blocks by substitution,
      //       then the off-diagonal blocks by doubling: T_10, T_32 from
      //       T_ii (-A_ij) T_jj, then the lower-left 32 x 32 block the same way
      if (pt < C) {
        // column cc of the diagonal block at r0, right-looking: as soon as
        // t_i is final every later row k takes its term -A(k, i) t_i, so one
        // FMA per step is on the critical path.  Column i of the block's A
        // (row r0 + i of the transposed copy) is contiguous: four 16-byte
        // loads, issued one step ahead.
        const int r0 = 16 * (pt >> 4), cc = pt & 15;
        float tcol[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) tcol[k] = 0.f;
        float4 nx[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) nx[q] = reinterpret_cast<const float4 *>(Pm + r0 * P_LD + r0)[q];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float col[16] = {nx[0].x, nx[0].y, nx[0].z, nx[0].w, nx[1].x, nx[1].y, nx[1].z, nx[1].w,
                                 nx[2].x, nx[2].y, nx[2].z, nx[2].w, nx[3].x, nx[3].y, nx[3].z, nx[3].w};
          if (i + 1 < 16) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              nx[q] = reinterpret_cast<const float4 *>(Pm + (r0 + i + 1) * P_LD + r0)[q];
          }
          const float ti = (i == cc) ? 1.f : (i > cc ? tcol[i] : 0.f);
          tcol[i] = ti;
#pragma unroll
          for (int k = i + 1; k < 16; ++k) tcol[k] = fmaf(-col[k], ti, tcol[k]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i > cc) Pm[(r0 + i) * P_LD + r0 + cc] = tcol[i];
      }
      role_sync(BAR_PREP, NP);
      if (pw < 4) {
        // T_10 (warps 0, 1: column halves) and T_32 (warps 2, 3)
        const int I = (pw >> 1) ? 3 : 1, J = I - 1, half = pw & 1;
        const int rI = 16 * I, cJ = 16 * J, cn = cJ + 8 * half;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        mma16x8(acc, [&](int r, int k) { return a_at(Pm, rI + r, cJ + k); },
                [&](int k, int c) { return t_at(Pm, cJ + k, cn + c); }, lane);
        float *xs = Xs + pw * 16 * XS_LD;
        const int g = lane >> 2, t = lane & 3;
        xs[g * XS_LD + 2 * t] = acc[0];
        xs[g * XS_LD + 2 * t + 1] = acc[1];
        xs[(g + 8) * XS_LD + 2 * t] = acc[2];
        xs[(g + 8) * XS_LD + 2 * t + 1] = acc[3];
        __syncwarp();
        float acc2[4] = {0.f, 0.f, 0.f, 0.f};
        mma16x8(acc2, [&](int r, int k) { return t_at(Pm, rI + r, rI + k); },
                [&](int k, int c) { return xs[k * XS_LD + c]; }, lane);
        Pm[(rI + g) * P_LD + cn + 2 * t] = -acc2[0];
        Pm[(rI + g) * P_LD + cn + 2 * t + 1] = -acc2[1];
        Pm[(rI + g + 8) * P_LD + cn + 2 * t] = -acc2[2];
        Pm[(rI + g + 8) * P_LD + cn + 2 * t + 1] = -acc2[3];
      }
      role_sync(BAR_PREP, NP);
      {
        // lower-left 32 x 32: X_IJ = sum_{K=J..1} A_IK T_KJ, then
        // T_IJ = -sum_{K=2..I} T_IK X_KJ; block (I, J) = (2 + (b >> 1), b & 1)
        // for b = pw >> 1, column tile nt = pw & 1 of it
        const int blk = pw >> 1, nt = pw & 1;
        const int I = 2 + (blk >> 1), J = blk & 1;
        const int g = lane >> 2, t = lane & 3;
        float *xs = Xs + blk * 16 * XS_LD;
        {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int K = 0; K <= 1; ++K)
            if (K >= J)
              mma16x8(acc, [&](int r, int k) { return a_at(Pm, 16 * I + r, 16 * K + k); },
                      [&](int k, int c) { return t_at(Pm, 16 * K + k, 16 * J + 8 * nt + c); }, lane);
          xs[g * XS_LD + 8 * nt + 2 * t] = acc[0];
          xs[g * XS_LD + 8 * nt + 2 * t + 1] = acc[1];
          xs[(g + 8) * XS_LD + 8 * nt + 2 * t] = acc[2];
          xs[(g + 8) * XS_LD + 8 * nt + 2 * t + 1] = acc[3];
        }
        role_sync(BAR_PREP, NP);
        {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int K = 2; K <= 3; ++K) {
            if (K > I) continue;
            const float *xk = Xs + (2 * (K - 2) + J) * 16 * XS_LD;
            mma16x8(acc, [&](int r, int k) { return t_at(Pm, 16 * I + r, 16 * K + k); },
                    [&](int k, int c) { return xk[k * XS_LD + 8 * nt + c]; }, lane);
          }
          const int cn = 16 * J + 8 * nt;
          Pm[(16 * I + g) * P_LD + cn + 2 * t] = -acc[0];
          Pm[(16 * I + g) * P_LD + cn + 2 * t + 1] = -acc[1];
          Pm[(16 * I + g + 8) * P_LD + cn + 2 * t] = -acc[2];
          Pm[(16 * I + g + 8) * P_LD + cn + 2 * t + 1] = -acc[3];
        }
      }
      role_sync(BAR_PREP, NP);
      // -- 5. T' = T diag(b gamma), T'' = T diag(b) as bf16 K-major A tiles
      {
        // row i along the warp (8 consecutive rows fall on distinct banks),
        // 16-column quarter qq per warp pair
        const int i = pt & (C - 1), qq = pt >> 6;
        const float *trow = Pm + i * P_LD + 16 * qq;
        uint8_t *t1 = smem + TT, *t2 = smem + TT + 8192;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float4 lo4 = reinterpret_cast<const float4 *>(trow + 8 * q)[0];
          const float4 hi4 = reinterpret_cast<const float4 *>(trow + 8 * q)[1];
          const float tr[8] = {lo4.x, lo4.y, lo4.z, lo4.w, hi4.x, hi4.y, hi4.z, hi4.w};
          float f1[8], f2[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = 16 * qq + 8 * q + u;
            const float tv = j < i ? tr[u] : (j == i ? 1.f : 0.f), b = jb->beta[j];
            f1[u] = tv * (b * jb->gam[j] * dsk);
            f2[u] = tv * (b * dsv);
          }
          st_chunk(t1, i, 2 * qq + q, pack8(f1));
          st_chunk(t2, i, 2 * qq + q, pack8(f2));
        }
      }
      // -- 6. V (rows past the chunk zeroed), then W = T' K -> W and
      //       U = [T''; 0] V -> X once the epilogue of chunk seq-1 has read X
      // T' and T'' are written; V has arrived and X is free (the epilogue of
      // chunk seq-1 has read it): one barrier for the three.  The e4m3 path
      // expands V's codes first and waits for X after, so the expansion runs
      // while the epilogue may still hold X.
      fence_proxy_async_smem();
      {
        bool r = true;
        if (pt == 0) {
          r = mbar_wait(bar(V_FULL), seq & 1, vabort, kTimeoutNs);
          if (!F8) r = r && mbar_wait(bar(XFREE), (seq & 1) ^ 1, vabort, kTimeoutNs);
        }
        if (!role_and(BAR_PREP, NP, r)) break;
      }
      if (F8) {
        expand_e4m3(smem + V, 8192, 1);
        if (n < C) role_sync(BAR_PREP, NP);  // the zeroing below rewrites expanded rows
      }
      if (n < C) {
        for (int e = pt; e < 2 * C * 8; e += NP) {
          const int r = (e >> 3) & (C - 1);
          if (r >= n)
            *reinterpret_cast<uint4 *>(smem + V + (e >> 9) * 8192 + r * 128 + (e & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (F8) {
        fence_proxy_async_smem();
        if (!wait_r(bar(XFREE), (seq & 1) ^ 1)) break;
      } else if (n < C) {
        fence_proxy_async_smem();
        role_sync(BAR_PREP, NP);
      }
      if (pt == 0) {
        tc_fence_after();
        constexpr uint32_t id = idesc_bf16(128, 128, true);
        const uint32_t xs_t = tmem + T_X;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_bf16(tmem + T_W, sdesc_sw128(sb + TT + kk * 32, 16, 1024),
                   sdesc_sw128(kq + 8192 + kk * 2048, 16384, 1024), id, kk > 0 ? 1u : 0u);
          mma_bf16(xs_t, sdesc_sw128(sb + TT + 8192 + kk * 32, 16, 1024),
                   sdesc_sw128(sb + V + kk * 2048, 8192, 1024), id, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(WU));
      }
      __syncwarp();
      // -- 7. W and U are done (V is free again), and the chain's tiles, once
      //       chunk seq-1's chain has finished with them: [-W; gamma Q] (read
      //       by its first product) and K (by its update); both are long free
      //       when the prep is the slower role.  One barrier.
      {
        bool r = true;
        if (pt == 0) {
          r = mbar_wait(bar(WU), seq & 1, vabort, kTimeoutNs);
          if (r) mbar_arrive(bar(V_EMPTY));
          r = r && mbar_wait(bar(CA_FREE), (seq & 1) ^ 1, vabort, kTimeoutNs) &&
              mbar_wait(bar(CK_FREE), (seq & 1) ^ 1, vabort, kTimeoutNs);
        }
        if (!role_and(BAR_PREP, NP, r)) break;
      }
      tc_fence_after();
      if (row < C) {
        // W row = token (TMEM lanes 0-63), dk half hb
        uint32_t w[64];
        tmem_ld64(tlp + T_W + 64 * hb, w);
        uint8_t *dst = smem + CA + hb * 16384;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float f[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) f[u] = -__uint_as_float(w[8 * q + u]);
          st_chunk(dst, row, q, pack8(f));
        }
      } else {
        const int i = row - C;  // gamma_i q_i into tile rows 64-127 (same swizzle phase), dk half hb
        const float gq = jb->gam[i] * dsq;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int off = i * 128 + ((q ^ (i & 7)) << 4);
          const uint4 raw = *reinterpret_cast<const uint4 *>(kqp + hb * 16384 + off);
          const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
          float f[8];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 v2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[u]));
            f[2 * u] = v2.x * gq;
            f[2 * u + 1] = v2.y * gq;
          }
          *reinterpret_cast<uint4 *>(smem + CA + hb * 16384 + 8192 + off) = pack8(f);
        }
      }
      for (int e = pt; e < 2 * C * 8; e += NP) {  // K rows: same rows, same swizzle
        const int b = e >> 9, rest = (e & 511) * 16;
        *reinterpret_cast<uint4 *>(smem + CK + b * 8192 + rest) =
            *reinterpret_cast<const uint4 *>(kqp + b * 16384 + 8192 + rest);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      role_sync(BAR_PREP, NP);
      if (pt == 0) {
        mbar_arrive(bar(READY));
        mbar_arrive(bar(KQ_EMPTY + s));
      }
    }
    if (pt == 0 && issued && *vabort) {  // MMAs still in flight after a timeout
      mma_commit(bar(DRAIN_P));
      mbar_wait(bar(DRAIN_P), 0, vabort, kTimeoutNs, false);
    }
  } else if (warp >= kChainWarp0) {
    // ---------------- chain: the state products, chunk after chunk
    const int row = tid - kChainWarp0 * 32;  // TMEM lane = state row (dv) / token row
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    bool issued = false;
    auto wait_r = [&](uint32_t b, uint32_t parity) -> bool {  // one poller, the rest park
      bool r = true;
      if (row == 0) r = mbar_wait(b, parity, vabort, kTimeoutNs);
      return role_and(BAR_CHAIN, 128, r);
    };
    for (uint32_t seq = 0;; ++seq) {
      const int j = seq & 3;
      if (!wait_r(bar(JOB_FULL + j), (seq >> 2) & 1)) break;
      Job *jb = job(j);
      if (jb->stop) break;
      const int s = seq & 1;
      const bool first = jb->first, update = jb->update, save = jb->save;
      const float *src = jb->src;
      float *dst = jb->dst;
      if (!wait_r(bar(READY), seq & 1)) break;
      const float gl = jb->gam_last;
      const uint32_t xt = T_X;
      // -- S0 as the bf16 B operand; S <- gamma_last S for the update
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint32_t v[64];
        if (first) {
#pragma unroll
          for (int i = 0; i < 64; i += 4) {
            const float4 f4 = src ? *reinterpret_cast<const float4 *>(src + (size_t)row * D + 64 * b + i)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
            v[i] = __float_as_uint(f4.x);
            v[i + 1] = __float_as_uint(f4.y);
            v[i + 2] = __float_as_uint(f4.z);
            v[i + 3] = __float_as_uint(f4.w);
          }
        } else {
          tmem_ld64(tl + T_S + 64 * b, v);
        }
        uint8_t *s0 = smem + SD + b * 16384;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float f[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) f[u] = __uint_as_float(v[8 * q + u]);
          st_chunk(s0, row, q, pack8(f));
        }
        if (update) {
#pragma unroll
          for (int i = 0; i < 64; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * gl);
          tmem_st64(tl + T_S + 64 * b, v);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      role_sync(BAR_CHAIN, 128);
      if (row == 0) {
        tc_fence_after();
        constexpr uint32_t id = idesc_bf16(128, 128, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t o = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16(tmem + xt, sdesc_sw128(sb + CA + o, 16, 1024), sdesc_sw128(sb + SD + o, 16, 1024),
                   id, 1u);
        }
        mma_commit(bar(XDONE));
        issued = true;
      }
      __syncwarp();
      if (!wait_r(bar(XDONE), seq & 1)) break;
      tc_fence_after();
      if (row == 0) mbar_arrive(bar(CA_FREE));
      // -- Delta (token rows 0-63) as the MN-major B of (M o QK^T) Delta, and
      //    Delta' = Delta gamma_last / gamma_j as the MN-major A of the update
      if (row < C) {
        const float dj = jb->dsc[row] * dsk;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          uint32_t v[64];
          tmem_ld64(tl + xt + 64 * b, v);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float f[8], f2[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              f[u] = __uint_as_float(v[8 * q + u]);
              f2[u] = f[u] * dj;
            }
            st_chunk(smem + SD + b * 8192, row, q, pack8(f));
            if (update) st_chunk(smem + SD + 16384 + b * 8192, row, q, pack8(f2));
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      role_sync(BAR_CHAIN, 128);
      if (row == 0) {
        tc_fence_after();
        const uint32_t mq = sb + MQK + s * 8192 - 8192;  // [junk; M o QK^T]
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          if (update)
            mma_bf16(tmem + T_S, sdesc_sw128(sb + SD + 16384 + kk * 2048, 8192, 1024),
                     sdesc_sw128(sb + CK + kk * 2048, 8192, 1024),
                     idesc_bf16_ex(128, 128, true, true, false), 1u);
          mma_bf16(tmem + xt, sdesc_sw128(mq + kk * 32, 16, 1024),
                   sdesc_sw128(sb + SD + kk * 2048, 8192, 1024), idesc_bf16(128, 128, true), 1u);
        }
        mma_commit(bar(SO + s));
      }
      __syncwarp();
      if (!wait_r(bar(SO + s), (seq >> 1) & 1)) break;
      tc_fence_after();
      if (row == 0) {
        mbar_arrive(bar(CK_FREE));
        mbar_arrive(bar(JOB_FREE + j));
      }
      if (save) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          uint32_t v[64];
          tmem_ld64(tl + T_S + 64 * b, v);
          float *d = dst + (size_t)row * D + 64 * b;
#pragma unroll
          for (int i = 0; i < 64; i += 4)
            *reinterpret_cast<float4 *>(d + i) =
                make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                            __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
        }
      }
    }
    if (row == 0 && issued && *vabort) {
      mma_commit(bar(DRAIN_C));
      mbar_wait(bar(DRAIN_C), 0, vabort, kTimeoutNs, false);
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 2) {
    // ---------------- epilogue: output rows (TMEM lanes 64-127 of X)
    const int i = tid - kEpiWarp0 * 32;  // token of the chunk
    const uint32_t tle = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    auto wait_r = [&](uint32_t b, uint32_t parity) -> bool {  // one poller, the rest park
      bool r = true;
      if (i == 0) r = mbar_wait(b, parity, vabort, kTimeoutNs);
      return role_and(BAR_EPI, 64, r);
    };
    for (uint32_t seq = 0;; ++seq) {
      const int j = seq & 3;
      if (!wait_r(bar(JOB_FULL + j), (seq >> 2) & 1)) break;
      Job *jb = job(j);
      if (jb->stop) break;
      const int s = seq & 1, cbeg = jb->cbeg, n = jb->n, h = jb->h;
      if (!wait_r(bar(SO + s), (seq >> 1) & 1)) break;
      tc_fence_after();
      const bool valid = i < n && cbeg + i < Tact;
      __nv_bfloat16 *o = p.out + ((size_t)(cbeg + i) * p.H + h) * D;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint32_t v[64];
        tmem_ld64(tle + T_X + 64 * b, v);
        if (valid) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = __uint_as_float(v[8 * q + u]);
            *reinterpret_cast<uint4 *>(o + 64 * b + 8 * q) = pack8(f);
          }
        }
      }
      tc_fence_before();
      role_sync(BAR_EPI, 64);
      if (i == 0) {
        mbar_arrive(bar(XFREE));
        mbar_arrive(bar(JOB_FREE + j));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *vabort) set_status(x.status, FLIDE_ERR_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---- host ------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_gdn() {
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

// [rows, heads, 128] bf16 (esz 2) or e4m3 (esz 1) as a 3-D tensor (dim, head,
// row); box of 128 bytes of dims x 1 x 64 rows
bool make_map_gdn(CUtensorMap *m, const void *base, int heads, long rows, int esz) {
  EncodeTiledFn enc = encode_fn_gdn();
  if (!enc || rows <= 0) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)128 * esz, (cuuint64_t)heads * 128 * esz};
  cuuint32_t box[3] = {(cuuint32_t)(128 / esz), 1, (cuuint32_t)C};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void *>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool fork_gdn_tc_supported(int dk, int dv, int dtype) {
  return (dtype == FLIDE_BF16 || dtype == FLIDE_E4M3) && dk == D && dv == D &&
         encode_fn_gdn() != nullptr;
}

int fork_gdn_tc(const void *q, const void *k, const void *v, const float *g, const float *beta,
                const float *state_in, const flide_tree_index *x, int H, void *out,
                float *node_state, int n_slots, cudaStream_t s, int dtype, const float *descale) {
  const bool f8 = dtype == FLIDE_E4M3;
  if (f8 && !descale) return FLIDE_ERR_SHAPE;
  const int esz = f8 ? 1 : 2;
  CUtensorMap mq, mk, mv;
  const long T = x->T > 0 ? x->T : 1;
  if (!make_map_gdn(&mq, q, H, T, esz) || !make_map_gdn(&mk, k, H, T, esz) ||
      !make_map_gdn(&mv, v, H, T, esz))
    return FLIDE_ERR_CUDA;
  static std::atomic<bool> attr_set[2][64];  // zero-initialised: false
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLIDE_ERR_CUDA;
  if (dev < 0 || dev >= 64 || !attr_set[f8][dev].load(std::memory_order_acquire)) {
    const cudaError_t e =
        f8 ? cudaFuncSetAttribute(gdn_ws_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  ws::SMEM_BYTES)
           : cudaFuncSetAttribute(gdn_ws_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  ws::SMEM_BYTES);
    if (e != cudaSuccess) return FLIDE_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[f8][dev].store(true, std::memory_order_release);
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  GdnTcParams prm;
  prm.x = *x;
  prm.descale = descale;
  prm.g = g;
  prm.beta = beta;
  prm.state_in = state_in;
  prm.out = (__nv_bfloat16 *)out;
  prm.node_state = node_state;
  prm.H = H;
  prm.n_slots = n_slots;
  prm.goff = 4 * (x->R + 1);  // after the attention's per-request table
  for (int lvl = 0; lvl <= x->max_depth; ++lvl) {
    prm.level = lvl;
    gdn_groups_kernel<<<1, 1024, 0, s>>>(*x, lvl, prm.goff);
    FLIDE_LAUNCH_CHECK();
    if (f8)
      gdn_ws_kernel<true><<<sms, ws::kThreads, ws::SMEM_BYTES, s>>>(mq, mk, mv, prm);
    else
      gdn_ws_kernel<false><<<sms, ws::kThreads, ws::SMEM_BYTES, s>>>(mq, mk, mv, prm);
    FLIDE_LAUNCH_CHECK();
  }
  return FLIDE_OK;
}

}  // namespace flide
