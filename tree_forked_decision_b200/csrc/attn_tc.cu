// attn_tc.cu -- fork attention on the 5th-generation tensor cores (sm_100a):
// bf16 q/k/v, head dim 128, fp32 accumulation and online softmax.
//
// What it computes (kongchang.com article on Flide, "ForkAttention" and
// attention-mask sections): every query token attends to exactly the keys of
// its isolated sequence -- its request's past rows, all tokens of its
// ancestors, its own node's tokens up to itself -- so each branch equals an
// isolated forward pass while the shared prefix is stored and read once.
//
// Work decomposition.  One CTA per work item = (request, kv head, tile of
// query tokens).  A tile packs the G = Hq/Hkv query heads of one kv head with
// 128/G consecutive tokens into 128 MMA rows (row = token*G + head), so one
// K/V tile in shared memory serves every query head of the group and, for a
// branch tile, the queries of several sibling branches at once.  Tiles never
// straddle the root/branch boundary of a request.  Key tiles come from a short
// list of spans:
//   past  rows of the packed checkpoint buffer      (all visible)
//   root  the request's root segment                (branch tiles: all
//         visible; root tiles: causal, keys up to the tile's last token)
//   tree  per level L >= 1, the stream range covering the level-L ancestors
//         of the tile's rows; key j of node m is visible to a row of node n
//         iff m is n's level-L ancestor and (m != n or j <= the row's token)
// Item order is (request, kv head) major with the costliest tiles first, so
// CTAs that read the same K/V run together and share it through L2.
//
// CTA roles (192 threads):
//   warps 0-3  softmax: thread = one MMA row = one TMEM lane; reads S from
//              TMEM, masks, online softmax in the exp2 domain with lazy
//              rescaling of O (only when the running max grows by > 2^8),
//              writes P (bf16) to shared memory, final normalisation + store.
//   warp 4     producer: TMA loads of Q once and of K/V tiles into a
//              2-stage ring (128-byte swizzle).
//   warp 5     MMA issuer: S = Q K^T into one of two TMEM buffers, then
//              O += P V into a TMEM accumulator (tcgen05.mma kind::f16,
//              M = N = 128, K = 16 per instruction).
// TMEM: S0 cols [0,128), S1 [128,256), O [256,384) of a 512-column allocation.
// Every wait is bounded; on expiry the CTA records FLIDE_ERR_TIMEOUT, drains
// its in-flight copies and MMAs, frees TMEM and exits.
#include <cstddef>

#include "common.cuh"
#include "sm100.cuh"

namespace flide {
int fork_attn_portable(const void *q, const void *k, const void *v, const void *pk,
                       const void *pv, const flide_tree_index *x, int Hq, int Hkv, int d,
                       int dtype, float scale, void *out, cudaStream_t s);
namespace {

using namespace sm100;

constexpr int BM = 128;  // MMA rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int NS = 2;    // K/V stages
constexpr int kMaxLevels = 8;
constexpr int kMaxSpans = 2 + kMaxLevels;
constexpr int kThreads = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// shared-memory map, bytes from a 1024-aligned base
constexpr int SM_Q = 0;                   // 2 slabs x [128 rows x 128 B]
constexpr int SM_KV = 32768;              // stage s: K slab0, K slab1, V slab0, V slab1
constexpr int SM_P = SM_KV + NS * 65536;  // 2 slabs x [128 rows x 128 B]
constexpr int SM_BAR = SM_P + 32768;
constexpr int SM_MISC = SM_BAR + 256;
constexpr int SMEM_BYTES = SM_MISC + 1024 + 1024;

enum {
  B_Q = 0,
  B_KV_FULL = 1,
  B_KV_FREE = B_KV_FULL + NS,
  B_S_FULL = B_KV_FREE + NS,
  B_S_FREE = B_S_FULL + 2,
  B_P_FULL = B_S_FREE + 2,
  B_PV_DONE = B_P_FULL + 1,
  B_DRAIN = B_PV_DONE + 1,
  NUM_BARS = B_DRAIN + 1
};

enum { SRC_STREAM = 0, SRC_PAST = 1 };
enum { KIND_FULL = 0, KIND_CAUSAL = 1, KIND_TREE = 2 };

struct Span {
  int src, start, len, kind, level, tile0;
};

struct Misc {
  uint32_t tmem_base;
  int abort;
  int valid;
  int n_spans, n_tiles;
  int r, hk, t0, ntok;
  Span spans[kMaxSpans];
};

struct TcParams {
  flide_tree_index x;
  __nv_bfloat16 *out;
  int Hq, Hkv, G, mtok, has_past;
  float qk_log2;  // scale * log2(e)
};

__device__ __forceinline__ int upper_bound_dev(const int32_t *a, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (a[mid] > key) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Item counts per request: Hkv * (branch tiles + root tiles), prefix-summed
// into work[0..R].
__global__ void attn_items_kernel(flide_tree_index x, int Hkv, int mtok) {
  __shared__ int scratch[40];
  if (failed(x.status)) return;
  const int R = x.R;
  int carry = 0;
  for (int b = 0; b < R; b += blockDim.x) {
    const int r = b + threadIdx.x;
    int cnt = 0;
    if (r < R) {
      const int n0 = x.req_node[r], n1 = x.req_node[r + 1];
      if (n1 > n0) {
        const int rs = x.node_start[n0], re = x.node_start[n0 + 1], end = x.node_start[n1];
        cnt = Hkv * ((re - rs + mtok - 1) / mtok + (end - re + mtok - 1) / mtok);
      }
    }
    int tot;
    const int ex = block_excl_scan(cnt, scratch, &tot);
    if (r < R) x.work[r] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) x.work[R] = carry;
}

// Decodes this CTA's work item and builds its key spans (run by one warp).
__device__ void decode_item(const TcParams &p, Misc &ms, int lane) {
  const flide_tree_index &x = p.x;
  const int R = x.R;
  const int item = blockIdx.x;
  int valid = !failed(x.status) && item < x.work[R];
  if (!valid) {
    if (lane == 0) ms.valid = 0;
    return;
  }
  const int r = upper_bound_dev(x.work, R + 1, item) - 1;
  const int local = item - x.work[r];
  const int root = x.req_node[r];
  const int root_start = x.node_start[root];
  const int br_start = x.node_start[root + 1];
  const int req_end = x.node_start[x.req_node[r + 1]];
  const int mtok = p.mtok;
  const int nrt = (br_start - root_start + mtok - 1) / mtok;
  const int nbt = (req_end - br_start + mtok - 1) / mtok;
  const int per = nrt + nbt;
  const int hk = local / per, w = local % per;
  const bool branch = w < nbt;
  int t0, ntok;
  if (branch) {
    t0 = br_start + w * mtok;
    ntok = min(mtok, req_end - t0);
  } else {
    const int i = nrt - 1 - (w - nbt);
    t0 = root_start + i * mtok;
    ntok = min(mtok, br_start - t0);
  }
  Span sp[kMaxSpans];
  int ns = 0;
  const int p0 = x.past_start[r], plen = x.past_start[r + 1] - p0;
  if (plen > 0) {
    if (!p.has_past) {
      if (lane == 0) {
        set_status(x.status, FLIDE_ERR_SHAPE);
        ms.valid = 0;
      }
      return;
    }
    sp[ns++] = Span{SRC_PAST, p0, plen, KIND_FULL, 0, 0};
  }
  if (branch) {
    if (br_start > root_start) sp[ns++] = Span{SRC_STREAM, root_start, br_start - root_start, KIND_FULL, 0, 0};
    for (int lvl = 1; lvl <= kMaxLevels; ++lvl) {
      int mn = INT_MAX, mx = -1;
      for (int i = lane; i < ntok; i += 32) {
        const int n = x.token_node[t0 + i];
        if (x.depth[n] >= lvl) {
          const int a = x.anc_node[x.anc_ptr[n] + lvl];
          mn = min(mn, a);
          mx = max(mx, a);
        }
      }
      mn = __reduce_min_sync(0xffffffffu, mn);
      mx = __reduce_max_sync(0xffffffffu, mx);
      if (mx < 0) break;
      const int s0 = x.node_start[mn];
      sp[ns++] = Span{SRC_STREAM, s0, x.node_start[mx + 1] - s0, KIND_TREE, lvl, 0};
    }
  } else {
    sp[ns++] = Span{SRC_STREAM, root_start, t0 + ntok - root_start, KIND_CAUSAL, 0, 0};
  }
  int tiles = 0;
  for (int s = 0; s < ns; ++s) {
    sp[s].tile0 = tiles;
    tiles += (sp[s].len + BN - 1) / BN;
  }
  if (lane == 0) {
    ms.valid = 1;
    ms.n_spans = ns;
    ms.n_tiles = tiles;
    ms.r = r;
    ms.hk = hk;
    ms.t0 = t0;
    ms.ntok = ntok;
    for (int s = 0; s < ns; ++s) ms.spans[s] = sp[s];
  }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_pk,
               const __grid_constant__ CUtensorMap tm_pv, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sb = smem_u32(smem);
  Misc &ms = *reinterpret_cast<Misc *>(smem + SM_MISC);
  volatile int *abort_flag = &ms.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const flide_tree_index &x = p.x;
  auto bar = [&](int i) -> uint32_t { return sb + SM_BAR + 8 * i; };

  if (warp == 4) {
    if (lane == 0) {
      for (int i = 0; i < NUM_BARS; ++i) {
        uint32_t cnt = 1;
        if (i == B_S_FREE || i == B_S_FREE + 1 || i == B_P_FULL) cnt = 4;
        mbar_init(bar(i), cnt);
      }
      ms.abort = 0;
      fence_mbar_init();
    }
    decode_item(p, ms, lane);
  } else if (warp == 5) {
    tmem_alloc(sb + SM_MISC + (uint32_t)offsetof(Misc, tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_base;

  if (ms.valid) {
    const int n_spans = ms.n_spans, n_tiles = ms.n_tiles;
    const int hk = ms.hk, t0 = ms.t0, ntok = ms.ntok;
    if (warp == 4) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        mbar_arrive_expect_tx(bar(B_Q), BM * 128 * 2);
        tma_load_3d(sb + SM_Q, &tm_q, bar(B_Q), 0, hk * p.G, t0);
        tma_load_3d(sb + SM_Q + 16384, &tm_q, bar(B_Q), 64, hk * p.G, t0);
        int j = 0;
        bool ok = true;
        for (int s = 0; s < n_spans && ok; ++s) {
          const Span sp = ms.spans[s];
          const CUtensorMap *mk = sp.src == SRC_PAST ? &tm_pk : &tm_k;
          const CUtensorMap *mv = sp.src == SRC_PAST ? &tm_pv : &tm_v;
          for (int off = 0; off < sp.len; off += BN, ++j) {
            const int st = j % NS;
            if (j >= NS && !mbar_wait(bar(B_KV_FREE + st), ((j / NS) - 1) & 1, abort_flag, kTimeoutNs)) {
              ok = false;
              break;
            }
            const uint32_t dst = sb + SM_KV + st * 65536;
            const int row = sp.start + off;
            mbar_arrive_expect_tx(bar(B_KV_FULL + st), 65536);
            tma_load_3d(dst, mk, bar(B_KV_FULL + st), 0, hk, row);
            tma_load_3d(dst + 16384, mk, bar(B_KV_FULL + st), 64, hk, row);
            tma_load_3d(dst + 32768, mv, bar(B_KV_FULL + st), 0, hk, row);
            tma_load_3d(dst + 49152, mv, bar(B_KV_FULL + st), 64, hk, row);
          }
        }
        if (!ok) {
          // drain the copies still in flight into this CTA's shared memory
          mbar_wait(bar(B_Q), 0, abort_flag, kTimeoutNs, false);
          for (int jj = max(0, j - NS); jj < j; ++jj)
            mbar_wait(bar(B_KV_FULL + jj % NS), (jj / NS) & 1, abort_flag, kTimeoutNs, false);
        }
      }
    } else if (warp == 5) {
      // ------------------------------------------------------------ MMA
      if (lane == 0) {
        constexpr uint32_t id_s = idesc_bf16(BM, BN, false);
        constexpr uint32_t id_pv = idesc_bf16(BM, 128, true);
        bool ok = mbar_wait(bar(B_Q), 0, abort_flag, kTimeoutNs);
        auto do_pv = [&](int i) -> bool {
          if (!mbar_wait(bar(B_P_FULL), i & 1, abort_flag, kTimeoutNs)) return false;
          tc_fence_after();
          const int st = i % NS;
          const uint32_t vb = sb + SM_KV + st * 65536 + 32768;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = sdesc_sw128(sb + SM_P + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(vb + kk * 2048, 16384, 1024);
            mma_bf16(tmem + 256, a, b, id_pv, (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(B_KV_FREE + st));
          mma_commit(bar(B_PV_DONE));
          return true;
        };
        int j = 0;
        for (; ok && j < n_tiles; ++j) {
          const int st = j % NS;
          if (!mbar_wait(bar(B_KV_FULL + st), (j / NS) & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
          if (j >= 2 && !mbar_wait(bar(B_S_FREE + (j & 1)), ((j >> 1) - 1) & 1, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = sb + SM_KV + st * 65536;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = sdesc_sw128(sb + SM_Q + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(kb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            mma_bf16(tmem + (j & 1) * 128, a, b, id_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_S_FULL + (j & 1)));
          if (j >= 1 && !do_pv(j - 1)) { ok = false; break; }
        }
        if (ok) do_pv(n_tiles - 1);
        // all MMAs issued by this thread complete before TMEM is released
        mma_commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0, abort_flag, kTimeoutNs, false);
      }
    } else {
      // ------------------------------------------------------------ softmax
      const int row = warp * 32 + lane;
      const int tokr = row / p.G, g = row % p.G;
      const bool valid_row = tokr < ntok;
      const int t = t0 + tokr;
      const int row_node = valid_row ? x.token_node[t] : -1;
      const int row_depth = valid_row ? x.depth[row_node] : -1;
      const int row_anc = valid_row ? x.anc_ptr[row_node] : 0;
      const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
      float m_used = -INFINITY, l = 0.f;
      uint8_t *P = smem + SM_P;
      bool ok = true;
      int j = 0;
      for (int s = 0; s < n_spans && ok; ++s) {
        const Span sp = ms.spans[s];
        const int a_row = (sp.kind == KIND_TREE && valid_row && row_depth >= sp.level)
                              ? x.anc_node[row_anc + sp.level]
                              : -2;
        for (int off = 0; off < sp.len; off += BN, ++j) {
          const int buf = j & 1;
          // every lane waits; the warp proceeds only if all lanes saw the phase
          if (!__all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + buf), (j >> 1) & 1, abort_flag, kTimeoutNs))) {
            ok = false;
            break;
          }
          tc_fence_after();
          float sv[BN];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t rr[32];
            tmem_ld32(lane_base + buf * 128 + c4 * 32, rr);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[c4 * 32 + i] = __uint_as_float(rr[i]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_S_FREE + buf));
          const int rem = sp.len - off;
          if (sp.kind != KIND_FULL || rem < BN) {
            const int key0 = sp.start + off;
#pragma unroll
            for (int c = 0; c < BN; ++c) {
              bool vis = c < rem;
              const int key = key0 + c;
              if (sp.kind == KIND_CAUSAL) vis = vis && key <= t;
              if (sp.kind == KIND_TREE) {
                const int kn = vis ? x.token_node[key] : -1;
                vis = vis && kn == a_row && (kn != row_node || key <= t);
              }
              if (!vis) sv[c] = -INFINITY;
            }
          }
          float smax = -INFINITY;
#pragma unroll
          for (int c = 0; c < BN; ++c) smax = fmaxf(smax, sv[c]);
          const float mt = smax * p.qk_log2;
          if (j == 0) {
            m_used = mt;
          } else {
            if (!__all_sync(0xffffffffu, mbar_wait(bar(B_PV_DONE), (j - 1) & 1, abort_flag, kTimeoutNs))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const bool need = mt > m_used + kRescaleThreshold;
            if (__any_sync(0xffffffffu, need)) {
              const float f = need ? exp2f(m_used - mt) : 1.f;
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                uint32_t rr[32];
                tmem_ld32(lane_base + 256 + c4 * 32, rr);
#pragma unroll
                for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * f);
                tmem_st32(lane_base + 256 + c4 * 32, rr);
              }
              l *= f;
              if (need) m_used = mt;
            }
          }
          const float m_sub = (m_used == -INFINITY) ? 0.f : m_used;
          float rs = 0.f;
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            sv[c] = exp2f(fmaf(sv[c], p.qk_log2, -m_sub));
            rs += sv[c];
          }
          l += rs;
#pragma unroll
          for (int sl = 0; sl < 2; ++sl) {
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              const int c0 = sl * 64 + ch * 8;
              uint4 pk;
              __nv_bfloat162 b0 = __floats2bfloat162_rn(sv[c0 + 0], sv[c0 + 1]);
              __nv_bfloat162 b1 = __floats2bfloat162_rn(sv[c0 + 2], sv[c0 + 3]);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(sv[c0 + 4], sv[c0 + 5]);
              __nv_bfloat162 b3 = __floats2bfloat162_rn(sv[c0 + 6], sv[c0 + 7]);
              pk.x = *reinterpret_cast<uint32_t *>(&b0);
              pk.y = *reinterpret_cast<uint32_t *>(&b1);
              pk.z = *reinterpret_cast<uint32_t *>(&b2);
              pk.w = *reinterpret_cast<uint32_t *>(&b3);
              *reinterpret_cast<uint4 *>(P + sl * 16384 + row * 128 + ((ch ^ (row & 7)) << 4)) = pk;
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_P_FULL));
        }
      }
      if (ok && __all_sync(0xffffffffu, mbar_wait(bar(B_PV_DONE), (n_tiles - 1) & 1, abort_flag, kTimeoutNs))) {
        tc_fence_after();
        const float inv = 1.f / l;
        __nv_bfloat16 *o = p.out + ((size_t)t * p.Hq + hk * p.G + g) * 128;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t rr[32];
          tmem_ld32(lane_base + 256 + c4 * 32, rr);
          if (valid_row) {
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              uint4 pk;
              __nv_bfloat162 b0 = __floats2bfloat162_rn(__uint_as_float(rr[q8 * 8 + 0]) * inv, __uint_as_float(rr[q8 * 8 + 1]) * inv);
              __nv_bfloat162 b1 = __floats2bfloat162_rn(__uint_as_float(rr[q8 * 8 + 2]) * inv, __uint_as_float(rr[q8 * 8 + 3]) * inv);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(rr[q8 * 8 + 4]) * inv, __uint_as_float(rr[q8 * 8 + 5]) * inv);
              __nv_bfloat162 b3 = __floats2bfloat162_rn(__uint_as_float(rr[q8 * 8 + 6]) * inv, __uint_as_float(rr[q8 * 8 + 7]) * inv);
              pk.x = *reinterpret_cast<uint32_t *>(&b0);
              pk.y = *reinterpret_cast<uint32_t *>(&b1);
              pk.z = *reinterpret_cast<uint32_t *>(&b2);
              pk.w = *reinterpret_cast<uint32_t *>(&b3);
              *reinterpret_cast<uint4 *>(o + c4 * 32 + q8 * 8) = pk;
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (ms.valid && ms.abort && threadIdx.x == 0) set_status(x.status, FLIDE_ERR_TIMEOUT);
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---- host ------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)ptr;
  }
  return fn;
}

// [rows, heads, 128] bf16 viewed as a 3-D tensor (dim, head, row); box of
// 64 dims x box_heads heads x box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int heads, long rows, int box_heads,
              int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || rows <= 0) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {256, (cuuint64_t)heads * 256};
  cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool fork_attn_tc_supported(const flide_tree_index *x, int Hq, int Hkv, int d, int dtype) {
  if (dtype != FLIDE_BF16 || d != 128 || Hkv <= 0 || Hq % Hkv != 0) return false;
  const int G = Hq / Hkv;
  if (G > BM || BM % G != 0) return false;
  if (x->max_depth > kMaxLevels) return false;
  return encode_fn() != nullptr;
}

int fork_attn_tc(const void *q, const void *k, const void *v, const void *pk, const void *pv,
                 int past_rows, const flide_tree_index *x, int Hq, int Hkv, float scale,
                 void *out, cudaStream_t s) {
  const int G = Hq / Hkv;
  const int mtok = BM / G;
  CUtensorMap mq, mk, mv, mpk, mpv;
  const long T = x->T > 0 ? x->T : 1;
  if (!make_map(&mq, q, Hq, T, G, mtok)) return FLIDE_ERR_CUDA;
  if (!make_map(&mk, k, Hkv, T, 1, BN)) return FLIDE_ERR_CUDA;
  if (!make_map(&mv, v, Hkv, T, 1, BN)) return FLIDE_ERR_CUDA;
  const bool has_past = pk != nullptr && past_rows > 0;
  if (!make_map(&mpk, has_past ? pk : k, Hkv, has_past ? past_rows : T, 1, BN)) return FLIDE_ERR_CUDA;
  if (!make_map(&mpv, has_past ? pv : v, Hkv, has_past ? past_rows : T, 1, BN)) return FLIDE_ERR_CUDA;

  // the shared-memory opt-in is per device; remember it for the first 64
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLIDE_ERR_CUDA;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return FLIDE_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  attn_items_kernel<<<1, 1024, 0, s>>>(*x, Hkv, mtok);
  FLIDE_LAUNCH_CHECK();
  TcParams prm;
  prm.x = *x;
  prm.out = (__nv_bfloat16 *)out;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = G;
  prm.mtok = mtok;
  prm.has_past = has_past ? 1 : 0;
  prm.qk_log2 = scale * kLog2e;
  const long grid = (long)Hkv * ((x->T + mtok - 1) / mtok + 2L * x->R);
  if (grid <= 0) return FLIDE_OK;
  if (grid > 0x7fffffffL) return FLIDE_ERR_CAPACITY;
  attn_tc_kernel<<<(unsigned)grid, kThreads, SMEM_BYTES, s>>>(mq, mk, mv, mpk, mpv, prm);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}

}  // namespace flide

// ---- entry point without caller-provided scratch ---------------------------
//
// flide_fork_attn keeps its per-call work table (one int32 per request plus
// one) in the caller's index buffer, idx->work.  flide_fork_attn_noalloc runs
// the same kernels but takes that table from the fixed array below, which
// every GPU that loads libflide.so holds until the process exits (64 KB).

namespace flide {
namespace {

constexpr int kNoAllocMaxRequests = 16384;
static __device__ __align__(256) int32_t g_noalloc_work[kNoAllocMaxRequests + 1];

// Device address of g_noalloc_work on the current device.  In host code the
// array's name only stands in for the symbol, so the address is looked up once
// per device with that device current and cached.
int32_t *noalloc_work_ptr() {
  static int32_t *cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_work) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64) cached[dev] = (int32_t *)p;
  return (int32_t *)p;
}

}  // namespace
}  // namespace flide

extern "C" int flide_fork_attn_noalloc(const void *q, const void *k, const void *v,
                                       const void *past_k, const void *past_v,
                                       int32_t past_rows, const flide_tree_index *idx,
                                       int32_t Hq, int32_t Hkv, int32_t d, int32_t dtype,
                                       float scale, void *out, int32_t flags,
                                       flide_stream stream) {
  using namespace flide;
  if (!idx || !q || !k || !v || !out) return FLIDE_ERR_SHAPE;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || past_rows < 0) return FLIDE_ERR_SHAPE;
  if ((past_k == nullptr) != (past_v == nullptr)) return FLIDE_ERR_SHAPE;
  if (past_k == nullptr) past_rows = 0;
  if (idx->R < 0 || idx->R > kNoAllocMaxRequests) return FLIDE_ERR_CAPACITY;
  if (!(flags & FLIDE_FLAG_PORTABLE) && fork_attn_tc_supported(idx, Hq, Hkv, d, dtype)) {
    int32_t *work = noalloc_work_ptr();
    if (!work) return FLIDE_ERR_CUDA;
    flide_tree_index x = *idx;  // same index, work table moved to the fixed array
    x.work = work;
    x.work_len = kNoAllocMaxRequests + 1;
    return fork_attn_tc(q, k, v, past_k, past_v, past_rows, &x, Hq, Hkv, scale, out,
                        (cudaStream_t)stream);
  }
  // the CUDA-core kernel keeps no per-call table
  return fork_attn_portable(q, k, v, past_k, past_v, idx, Hq, Hkv, d, dtype, scale, out,
                            (cudaStream_t)stream);
}
