// attn_tc.cu -- fork attention on the 5th-generation tensor cores (sm_100a):
// bf16 or e4m3 q/k/v, head dim 128, fp32 accumulation and online softmax.
//
// What it computes (kongchang.com article on Flide, "ForkAttention" and
// attention-mask sections): every query token attends to exactly the keys of
// its isolated sequence -- its request's past rows, all tokens of its
// ancestors, its own node's tokens up to itself -- so each branch equals an
// isolated forward pass while the shared prefix is stored and read once.
//
// Work decomposition.  One CTA per work item = (request, kv head, tile of
// query tokens).  The G = Hq/Hkv query heads of one kv head are packed with
// the tokens into MMA rows (row = token*G + head), so one K/V tile in shared
// memory serves every query head of the group and, for a branch tile, the
// queries of several sibling branches at once.  A tile is 256 rows, split into
// two 128-row halves that share the K/V stream.  Tiles never straddle the
// root/branch boundary of a request.  Key tiles come from a short list of
// spans:
//   past  rows of the packed checkpoint buffer      (all visible)
//   root  the request's root segment                (branch tiles: all
//         visible; root tiles: causal, keys up to the tile's last token)
//   tree  per level L >= 1, the stream range covering the level-L ancestors
//         of the tile's rows; key j of node m is visible to a row of node n
//         iff m is n's level-L ancestor and (m != n or j <= the row's token)
// Item order is (request, kv head) major with the costliest tiles first, so
// CTAs that read the same K/V run together and share it through L2.
//
// CTA roles (320 threads):
//   warps 0-3, 4-7  softmax of half 0 and half 1: thread = one MMA row = one
//              TMEM lane; loads its S row from TMEM, masks, online softmax in
//              the exp2 domain (O rescaled in TMEM only when the running max
//              grows by more than 2^8), writes P as bf16 back into the S
//              columns it has consumed, final normalisation and store.
//   warp 8     producer: TMA loads of Q once and of K and V tiles into two
//              2-stage rings (128-byte swizzle).
//   warp 9     MMA issuer (one thread): per key tile j
//                S0(j) = Q0 K^T, S1(j) = Q1 K^T      (A, B from shared memory)
//                O0 += P0(j) V, O1 += P1(j) V        (A = P from TMEM)
//              issued as ... PV0(j), S0(j+1), PV1(j), S1(j+1) ... so one
//              half's softmax overlaps the other half's matrix work.  S(j+1)
//              overwrites the columns PV(j) reads; the tensor core executes one
//              thread's MMAs in issue order, and the commit after S(j+1)
//              tells the softmax warps that PV(j) has finished too.
// TMEM (512 columns): half h owns [256h, 256h+128) for S / P and
// [256h+128, 256h+256) for O.
// Every wait is bounded; on expiry the CTA records FLIDE_ERR_TIMEOUT, drains
// its in-flight copies and MMAs, frees TMEM and exits.
//
// e4m3 variant (F8 = true): q, k, v and the past rows are e4m3 codes with one
// descale factor per tensor (q, k, v; past rows share k's and v's).  A 128-dim
// row is one 128-byte swizzle row, so Q, K and V tiles are half the bytes;
// S = Q K^T and O += P V run as kind::f8f6f4 MMAs (K = 32 per instruction).
// P is written to TMEM as e4m3, four keys per column, scaled by 2^6: the O
// rescale threshold is 2^2 instead of 2^8, so p <= 4 and 2^6 p <= 256 stays
// below the format's largest value 448, and weights down to 2^-12 keep a
// normal e4m3 code.  One exponential pair in eight is evaluated on the FMA
// pipe (ex2_poly2).  The row sum uses the unrounded p; the descale factors of
// q and k fold into the softmax scale and v's into the final normalisation.
#include <cstddef>

#include "common.cuh"
#include "sm100.cuh"

namespace flide {
int fork_attn_portable(const void *q, const void *k, const void *v, const void *pk,
                       const void *pv, int past_rows, const flide_tree_index *x, int Hq,
                       int Hkv, int d, int dtype, float scale, void *out, cudaStream_t s);
namespace {

using namespace sm100;

constexpr int BM = 128;  // MMA rows per half
constexpr int BN = 128;  // keys per tile
constexpr int kMaxLevels = 8;
constexpr int kMaxSpans = 2 + kMaxLevels;
constexpr int kThreads = 320;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// shared-memory map, bytes from a 1024-aligned base
constexpr int SM_Q = 0;            // half h, slab s: h*32768 + s*16384  [128 rows x 128 B]
constexpr int SM_K = 65536;        // stage st: st*32768 (+ slab*16384)
constexpr int SM_V = 131072;       // stage st: st*32768 (+ slab*16384)
constexpr int SM_BAR = 196608;
constexpr int SM_MISC = SM_BAR + 256;
constexpr int SMEM_BYTES = SM_MISC + 1024 + 1024;

enum {
  B_Q = 0,
  B_K_FULL = 1,    // [2]
  B_K_FREE = 3,    // [2]
  B_V_FULL = 5,    // [2]
  B_V_FREE = 7,    // [2]
  B_S_FULL = 9,    // [2 halves]
  B_P_FULL = 11,   // [2 halves], 4 warp arrivals
  B_O_FULL = 13,
  B_DRAIN = 14,
  NUM_BARS = 15
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
  int slot;  // paged past: the request's history slot
  Span spans[kMaxSpans];
};

struct TcParams {
  flide_tree_index x;
  __nv_bfloat16 *out;
  const float *descale;            // e4m3 inputs: {q, k, v} descale factors
  // paged past (block_table != nullptr): history row i of request r is pool
  // row block_table[req_slot[r] * max_blocks + i / block_rows] * block_rows +
  // i % block_rows; block_rows is a multiple of the key tile
  const int32_t *block_table, *req_slot;
  int max_blocks, block_rows, n_blocks, n_slots;
  int Hq, Hkv, G, mtok, has_past;  // mtok = tokens per 128-row half
  int past_rows;                   // rows of the packed past buffers (unpaged)
  float qk_log2;                   // scale * log2(e)
};

__device__ __forceinline__ int upper_bound_dev(const int32_t *a, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (a[mid] > key) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Item counts per request: Hkv * (branch tiles + root tiles) of `ttok`
// tokens each, prefix-summed into work[0..R].
__global__ void attn_items_kernel(flide_tree_index x, int Hkv, int ttok) {
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
        cnt = Hkv * ((re - rs + ttok - 1) / ttok + (end - re + ttok - 1) / ttok);
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
  const int valid = !failed(x.status) && item < x.work[R];
  if (!valid) {
    if (lane == 0) ms.valid = 0;
    return;
  }
  const int r = upper_bound_dev(x.work, R + 1, item) - 1;
  const int Nact = x.counts[FLIDE_CNT_N], Tact = x.counts[FLIDE_CNT_T];
  // debug build: the request, its root and its node range index the tree arrays
  if (!in_bounds(x.status, x.counts, r, R, 201) ||
      !in_bounds(x.status, x.counts, x.req_node[r], Nact, 202) ||
      !in_bounds(x.status, x.counts, x.req_node[r + 1], Nact + 1, 203)) {
    if (lane == 0) ms.valid = 0;
    return;
  }
  const int local = item - x.work[r];
  const int root = x.req_node[r];
  const int root_start = x.node_start[root];
  const int br_start = x.node_start[root + 1];
  const int req_end = x.node_start[x.req_node[r + 1]];
  const int ttok = 2 * p.mtok;
  const int nrt = (br_start - root_start + ttok - 1) / ttok;
  const int nbt = (req_end - br_start + ttok - 1) / ttok;
  const int per = nrt + nbt;
  const int hk = local / per, w = local % per;
  const bool branch = w < nbt;
  int t0, ntok;
  if (branch) {
    t0 = br_start + w * ttok;
    ntok = min(ttok, req_end - t0);
  } else {
    const int i = nrt - 1 - (w - nbt);
    t0 = root_start + i * ttok;
    ntok = min(ttok, br_start - t0);
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
    // a packed past shorter than the tree's past rows: the tensor map would
    // return zeros past its end, so refuse instead of attending to them
    if (!p.block_table && (p0 < 0 || (long)p0 + plen > p.past_rows)) {
      if (lane == 0) {
        set_status(x.status, FLIDE_ERR_CAPACITY);
        ms.valid = 0;
      }
      return;
    }
    sp[ns++] = Span{SRC_PAST, p0, plen, KIND_FULL, 0, 0};
    if (p.block_table) {
      const int slot = p.req_slot[r];
      if (slot < 0 || slot >= p.n_slots || plen > (long)p.max_blocks * p.block_rows) {
        if (lane == 0) {
          set_status(x.status, FLIDE_ERR_INVALID);
          ms.valid = 0;
        }
        return;
      }
      if (lane == 0) ms.slot = slot;
    }
  }
  if (branch) {
    if (br_start > root_start) sp[ns++] = Span{SRC_STREAM, root_start, br_start - root_start, KIND_FULL, 0, 0};
    for (int lvl = 1; lvl <= kMaxLevels; ++lvl) {
      int mn = INT_MAX, mx = -1;
      for (int i = lane; i < ntok; i += 32) {
        const int n = (int)checked(x.status, x.counts, x.token_node[checked(x.status, x.counts, t0 + i, Tact, 204)],
                                   Nact, 205);
        if (x.depth[n] >= lvl) {
          const int a = x.anc_node[checked(x.status, x.counts, (long long)x.anc_ptr[n] + lvl,
                                           (long long)x.N * (x.max_depth + 1), 206)];
          mn = min(mn, a);
          mx = max(mx, a);
        }
      }
      mn = __reduce_min_sync(0xffffffffu, mn);
      mx = __reduce_max_sync(0xffffffffu, mx);
      if (mx < 0) break;
      if (!in_bounds(x.status, x.counts, mn, Nact, 207) || !in_bounds(x.status, x.counts, mx, Nact, 207)) {
        if (lane == 0) ms.valid = 0;
        return;
      }
      const int s0 = x.node_start[mn];
      sp[ns++] = Span{SRC_STREAM, s0, x.node_start[mx + 1] - s0, KIND_TREE, lvl, 0};
    }
  } else {
    sp[ns++] = Span{SRC_STREAM, root_start, t0 + ntok - root_start, KIND_CAUSAL, 0, 0};
  }
  // debug build: every stream span lies inside the stream, the tile's tokens too
  for (int s = 0; s < ns; ++s)
    if (sp[s].src == SRC_STREAM &&
        (!in_bounds(x.status, x.counts, sp[s].start, Tact + 1, 208) ||
         !in_bounds(x.status, x.counts, (long long)sp[s].start + sp[s].len, Tact + 1, 208))) {
      if (lane == 0) ms.valid = 0;
      return;
    }
  if (!in_bounds(x.status, x.counts, t0, Tact, 209) ||
      !in_bounds(x.status, x.counts, (long long)t0 + ntok, Tact + 1, 209)) {
    if (lane == 0) ms.valid = 0;
    return;
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

// (span, offset) of key tile j; spans are few, a linear walk is cheap
__device__ __forceinline__ void tile_at(const Misc &ms, int j, Span &sp, int &off) {
  int s = 0;
  while (s + 1 < ms.n_spans && ms.spans[s + 1].tile0 <= j) ++s;
  sp = ms.spans[s];
  off = (j - sp.tile0) * BN;
}

template <bool F8>
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
  constexpr int kEsz = F8 ? 1 : 2;    // bytes per element
  constexpr int kSlabs = F8 ? 1 : 2;  // 128-byte swizzle slabs per 128-dim row

  if (warp == 8) {
    if (lane == 0) {
      for (int i = 0; i < NUM_BARS; ++i)
        mbar_init(bar(i), (i == B_P_FULL || i == B_P_FULL + 1) ? 4u : 1u);
      ms.abort = 0;
      fence_mbar_init();
    }
    decode_item(p, ms, lane);
  } else if (warp == 9) {
    tmem_alloc(sb + SM_MISC + (uint32_t)offsetof(Misc, tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_base;

  if (ms.valid) {
    const int n_tiles = ms.n_tiles;
    const int hk = ms.hk, t0 = ms.t0, ntok = ms.ntok;
    if (warp == 8) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        mbar_arrive_expect_tx(bar(B_Q), 2 * BM * 128 * kEsz);
        for (int h = 0; h < 2; ++h)
          for (int s = 0; s < kSlabs; ++s)
            tma_load_3d(sb + SM_Q + h * 32768 + s * 16384, &tm_q, bar(B_Q), 64 * s, hk * p.G,
                        t0 + h * p.mtok);
        int jk = 0, jv = 0;  // tiles issued
        bool ok = true;
        for (int j = 0; j < n_tiles && ok; ++j) {
          Span sp;
          int off;
          tile_at(ms, j, sp, off);
          const CUtensorMap *mk = sp.src == SRC_PAST ? &tm_pk : &tm_k;
          const CUtensorMap *mv = sp.src == SRC_PAST ? &tm_pv : &tm_v;
          int row = sp.start + off;
          if (sp.src == SRC_PAST && p.block_table) {
            // a key tile lies inside one block (block_rows % BN == 0)
            int b = p.block_table[checked(x.status, x.counts,
                                          (long long)ms.slot * p.max_blocks + off / p.block_rows,
                                          (long long)p.n_slots * p.max_blocks, 210)];
            if (b < 0 || b >= p.n_blocks) {
              set_status(x.status, FLIDE_ERR_INVALID);  // no block: read block 0, flag the call
              b = 0;
            }
            row = b * p.block_rows + off % p.block_rows;
          }
          const int st = j & 1;
          if (j >= 2 && !mbar_wait(bar(B_K_FREE + st), ((j >> 1) - 1) & 1, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(B_K_FULL + st), BN * 128 * kEsz);
          tma_load_3d(sb + SM_K + st * 32768, mk, bar(B_K_FULL + st), 0, hk, row);
          if (!F8) tma_load_3d(sb + SM_K + st * 32768 + 16384, mk, bar(B_K_FULL + st), 64, hk, row);
          ++jk;
          if (j >= 2 && !mbar_wait(bar(B_V_FREE + st), ((j >> 1) - 1) & 1, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(B_V_FULL + st), BN * 128 * kEsz);
          tma_load_3d(sb + SM_V + st * 32768, mv, bar(B_V_FULL + st), 0, hk, row);
          if (!F8) tma_load_3d(sb + SM_V + st * 32768 + 16384, mv, bar(B_V_FULL + st), 64, hk, row);
          ++jv;
        }
        if (!ok) {
          // drain the copies still in flight into this CTA's shared memory
          mbar_wait(bar(B_Q), 0, abort_flag, kTimeoutNs, false);
          for (int jj = max(0, jk - 2); jj < jk; ++jj)
            mbar_wait(bar(B_K_FULL + (jj & 1)), (jj >> 1) & 1, abort_flag, kTimeoutNs, false);
          for (int jj = max(0, jv - 2); jj < jv; ++jj)
            mbar_wait(bar(B_V_FULL + (jj & 1)), (jj >> 1) & 1, abort_flag, kTimeoutNs, false);
        }
      }
    } else if (warp == 9) {
      // ------------------------------------------------------------ MMA
      if (lane == 0) {
        constexpr uint32_t id_s = F8 ? idesc_e4m3(BM, BN, false) : idesc_bf16(BM, BN, false);
        constexpr uint32_t id_pv = F8 ? idesc_e4m3(BM, 128, true) : idesc_bf16(BM, 128, true);
        // one instruction covers 32 bytes of K: 16 bf16 or 32 e4m3 elements;
        // in both cases 8 TMEM columns of P and 32 bytes of a K-major row
        auto qk = [&](int h, int st) {
#pragma unroll
          for (int kk = 0; kk < 4 * kSlabs; ++kk) {
            const uint64_t a = sdesc_sw128(sb + SM_Q + h * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(sb + SM_K + st * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            if (F8) mma_f8(tmem + h * 256, a, b, id_s, kk > 0 ? 1u : 0u);
            else mma_bf16(tmem + h * 256, a, b, id_s, kk > 0 ? 1u : 0u);
          }
        };
        auto pv = [&](int h, int st, bool acc) {
#pragma unroll
          for (int kk = 0; kk < 4 * kSlabs; ++kk) {
            // V is MN-major: one 128-byte row per key, K advances by keys
            const uint64_t b = sdesc_sw128(sb + SM_V + st * 32768 + kk * (F8 ? 4096 : 2048), 16384, 1024);
            if (F8)
              mma_f8_ts(tmem + h * 256 + 128, tmem + h * 256 + kk * 8, b, id_pv, (acc || kk > 0) ? 1u : 0u);
            else
              mma_bf16_ts(tmem + h * 256 + 128, tmem + h * 256 + kk * 8, b, id_pv,
                          (acc || kk > 0) ? 1u : 0u);
          }
        };
        bool ok = mbar_wait(bar(B_Q), 0, abort_flag, kTimeoutNs) &&
                  mbar_wait(bar(B_K_FULL), 0, abort_flag, kTimeoutNs);
        if (ok) {
          tc_fence_after();
          qk(0, 0);
          mma_commit(bar(B_S_FULL + 0));
          qk(1, 0);
          mma_commit(bar(B_S_FULL + 1));
          mma_commit(bar(B_K_FREE + 0));
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int sv = j & 1, sk = (j + 1) & 1;
          const bool more = j + 1 < n_tiles;
          if (!mbar_wait(bar(B_V_FULL + sv), (j >> 1) & 1, abort_flag, kTimeoutNs) ||
              !mbar_wait(bar(B_P_FULL + 0), j & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
          tc_fence_after();
          pv(0, sv, j > 0);
          if (more) {
            if (!mbar_wait(bar(B_K_FULL + sk), ((j + 1) >> 1) & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
            tc_fence_after();
            qk(0, sk);
            mma_commit(bar(B_S_FULL + 0));
          }
          if (!mbar_wait(bar(B_P_FULL + 1), j & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
          tc_fence_after();
          pv(1, sv, j > 0);
          mma_commit(bar(B_V_FREE + sv));
          if (more) {
            qk(1, sk);
            mma_commit(bar(B_S_FULL + 1));
            mma_commit(bar(B_K_FREE + sk));
          }
        }
        if (ok) mma_commit(bar(B_O_FULL));
        // all MMAs issued by this thread complete before TMEM is released
        mma_commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0, abort_flag, kTimeoutNs, false);
      }
    } else {
      // ------------------------------------------------------------ softmax
      const int h = warp >> 2;                      // half
      const int row = (warp & 3) * 32 + lane;       // TMEM lane = MMA row in the half
      const int tokr = h * p.mtok + row / p.G, g = row % p.G;
      const bool valid_row = tokr < ntok;
      const int t = t0 + tokr;
      const int row_node = valid_row ? x.token_node[t] : -1;
      const int row_depth = valid_row ? x.depth[row_node] : -1;
      const int row_anc = valid_row ? x.anc_ptr[row_node] : 0;
      const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's lanes
      const uint32_t t_s = tl + h * 256, t_o = tl + h * 256 + 128;
      const float c = F8 ? p.qk_log2 * p.descale[0] * p.descale[1] : p.qk_log2;
      constexpr float kThreshold = F8 ? 2.0f : kRescaleThreshold;
      constexpr float kPShift = F8 ? 6.0f : 0.0f;  // P stored as 2^kPShift p
      float m_used = -INFINITY, l = 0.f;
      int span_tile0 = -1, vis_lo = 0, vis_hi = 0;
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + h), j & 1, abort_flag, kTimeoutNs))) {
          ok = false;
          break;
        }
        tc_fence_after();
        Span sp;
        int off;
        tile_at(ms, j, sp, off);
        uint32_t sr[128];
        tmem_ld128(t_s, sr);
        // The keys this row sees inside one span form one range [vis_lo,
        // vis_hi) of key indices: the whole span (past rows, the root for a
        // branch tile), keys up to the row's own token (causal root), or the
        // token segment of the row's level-L ancestor, cut after the row's
        // own token when that ancestor is the row's own node (tree level).
        // The range is refreshed when the span changes; a tile is masked
        // with two integer bounds, and not at all when it is fully visible
        // to every row of the warp.
        if (sp.tile0 != span_tile0) {
          span_tile0 = sp.tile0;
          vis_lo = sp.start;
          vis_hi = sp.start + sp.len;
          if (valid_row && sp.kind == KIND_CAUSAL) {
            vis_hi = min(vis_hi, t + 1);
          } else if (valid_row && sp.kind == KIND_TREE) {
            if (row_depth >= sp.level) {
              const int a = x.anc_node[row_anc + sp.level];
              vis_lo = x.node_start[a];
              vis_hi = a == row_node ? t + 1 : x.node_start[a + 1];
            } else {
              vis_hi = vis_lo;
            }
          }
          vis_hi = max(vis_hi, vis_lo);
        }
        {
          const int key0 = sp.start + off;
          const int lo = min(max(vis_lo - key0, 0), BN), hi = min(max(vis_hi - key0, 0), BN);
          if (!__all_sync(0xffffffffu, lo == 0 && hi == BN)) {
            const uint32_t w = (uint32_t)(hi - lo);
#pragma unroll
            for (int i = 0; i < BN; ++i)
              if ((uint32_t)(i - lo) >= w) sr[i] = 0xff800000u;  // -inf
          }
        }
        // row max: 8 chains of three-input max
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = __uint_as_float(sr[k]);
#pragma unroll
        for (int i = 8; i < BN; i += 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mx[k] = fmax3f(mx[k], __uint_as_float(sr[i + 2 * k]), __uint_as_float(sr[i + 2 * k + 1]));
        }
        const float smax = fmaxf(fmax3f(mx[0], mx[1], mx[2]),
                                 fmax3f(fmax3f(mx[3], mx[4], mx[5]), mx[6], mx[7]));
        const float mt = smax * c;
        if (j == 0) {
          m_used = mt;
        } else {
          // PV(j-1) of this half is complete (it precedes S(j) in issue order)
          const bool need = mt > m_used + kThreshold;
          if (__any_sync(0xffffffffu, need)) {
            const float f = need ? exp2f(m_used - mt) : 1.f;
#pragma unroll 1
            for (int c4 = 0; c4 < 4; ++c4) {
              uint32_t r32[32];
              tmem_ld32(t_o + 32 * c4, r32);
#pragma unroll
              for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(__uint_as_float(r32[i]) * f);
              tmem_st32(t_o + 32 * c4, r32);
            }
            l *= f;
            if (need) m_used = mt;
          }
        }
        const float m_sub = ((m_used == -INFINITY) ? 0.f : m_used) - kPShift;
        // p = 2^(s*c - m): paired scale-and-shift, SFU exp2, paired row-sum
        // chains; P packed to bf16x2 in place into sr[0..63]
        const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m_sub, -m_sub);
        uint64_t acc[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = 0ull;
        if (F8) {
          // P as e4m3 codes, four keys per word, into sr[0..31]
#pragma unroll
          for (int i = 0; i < BN; i += 4) {
            float x0, x1, x2, x3;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), c2, nm2), x0, x1);
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[i + 2]), __uint_as_float(sr[i + 3])), c2, nm2), x2, x3);
            // one pair in eight on the FMA pipe: the special-function unit's
            // exp2 throughput bounds this loop once the MMAs take e4m3
            float e0, e1;
            if ((i >> 2) % 4 == 0) {
              f2_unpack(ex2_poly2(x0, x1), e0, e1);
            } else {
              e0 = ex2_approx(x0);
              e1 = ex2_approx(x1);
            }
            const float e2 = ex2_approx(x2), e3 = ex2_approx(x3);
            acc[(i >> 1) & 3] = f2_add(acc[(i >> 1) & 3], f2_pack(e0, e1));
            acc[((i >> 1) + 1) & 3] = f2_add(acc[((i >> 1) + 1) & 3], f2_pack(e2, e3));
            sr[i >> 2] = pack_e4m3x4(e0, e1, e2, e3);
          }
        } else {
#pragma unroll
          for (int i = 0; i < BN; i += 2) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), c2, nm2), x0, x1);
            const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
            acc[(i >> 1) & 3] = f2_add(acc[(i >> 1) & 3], f2_pack(e0, e1));
            sr[i >> 1] = pack_bf16x2(e0, e1);
          }
        }
        {
          float a0, a1, b0, b1, c0, c1, d0, d1;
          f2_unpack(acc[0], a0, a1);
          f2_unpack(acc[1], b0, b1);
          f2_unpack(acc[2], c0, c1);
          f2_unpack(acc[3], d0, d1);
          l += ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
        }
        if (F8) tmem_st32(t_s, *reinterpret_cast<uint32_t(*)[32]>(sr));
        else tmem_st64(t_s, *reinterpret_cast<uint32_t(*)[64]>(sr));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_P_FULL + h));
      }
      if (ok && __all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL), 0, abort_flag, kTimeoutNs))) {
        tc_fence_after();
        uint32_t orr[128];
        tmem_ld128(t_o, orr);
        if (valid_row) {
          const float inv = (F8 ? p.descale[2] : 1.f) / l;
          __nv_bfloat16 *o = p.out + ((size_t)t * p.Hq + hk * p.G + g) * 128;
#pragma unroll
          for (int q8 = 0; q8 < 16; ++q8) {
            uint4 v4;
            v4.x = pack_bf16x2(__uint_as_float(orr[q8 * 8 + 0]) * inv, __uint_as_float(orr[q8 * 8 + 1]) * inv);
            v4.y = pack_bf16x2(__uint_as_float(orr[q8 * 8 + 2]) * inv, __uint_as_float(orr[q8 * 8 + 3]) * inv);
            v4.z = pack_bf16x2(__uint_as_float(orr[q8 * 8 + 4]) * inv, __uint_as_float(orr[q8 * 8 + 5]) * inv);
            v4.w = pack_bf16x2(__uint_as_float(orr[q8 * 8 + 6]) * inv, __uint_as_float(orr[q8 * 8 + 7]) * inv);
            *reinterpret_cast<uint4 *>(o + q8 * 8) = v4;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (ms.valid && ms.abort && threadIdx.x == 0) set_status(x.status, FLIDE_ERR_TIMEOUT);
  if (warp == 9) {
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

// [rows, heads, 128] bf16 (esz 2) or e4m3 (esz 1) viewed as a 3-D tensor
// (dim, head, row); box of 128 bytes of dims x box_heads heads x box_rows
// rows, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int heads, long rows, int box_heads,
              int box_rows, int esz) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || rows <= 0) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)128 * esz, (cuuint64_t)heads * 128 * esz};
  cuuint32_t box[3] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void *>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool fork_attn_tc_supported(const flide_tree_index *x, int Hq, int Hkv, int d, int dtype) {
  if ((dtype != FLIDE_BF16 && dtype != FLIDE_E4M3) || d != 128 || Hkv <= 0 || Hq % Hkv != 0) return false;
  const int G = Hq / Hkv;
  if (G > BM || BM % G != 0) return false;
  if (x->max_depth > kMaxLevels) return false;
  return encode_fn() != nullptr;
}

int fork_attn_tc(const void *q, const void *k, const void *v, const void *pk, const void *pv,
                 int past_rows, const flide_tree_index *x, int Hq, int Hkv, int dtype,
                 const float *descale, float scale, void *out, cudaStream_t s,
                 const PagedPast *paged) {
  const int G = Hq / Hkv;
  const int mtok = BM / G;  // tokens per 128-row half; a tile is 2*mtok tokens
  const bool f8 = dtype == FLIDE_E4M3;
  const int esz = f8 ? 1 : 2;
  if (f8 && descale == nullptr) return FLIDE_ERR_SHAPE;
  CUtensorMap mq, mk, mv, mpk, mpv;
  const long T = x->T > 0 ? x->T : 1;
  if (!make_map(&mq, q, Hq, T, G, mtok, esz)) return FLIDE_ERR_CUDA;
  if (!make_map(&mk, k, Hkv, T, 1, BN, esz)) return FLIDE_ERR_CUDA;
  if (!make_map(&mv, v, Hkv, T, 1, BN, esz)) return FLIDE_ERR_CUDA;
  const bool has_past = pk != nullptr && past_rows > 0;
  if (!make_map(&mpk, has_past ? pk : k, Hkv, has_past ? past_rows : T, 1, BN, esz)) return FLIDE_ERR_CUDA;
  if (!make_map(&mpv, has_past ? pv : v, Hkv, has_past ? past_rows : T, 1, BN, esz)) return FLIDE_ERR_CUDA;

  // the shared-memory opt-in is per device and kernel; remember it for the
  // first 64 devices
  static std::atomic<bool> attr_set[2][64];  // zero-initialised: false
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLIDE_ERR_CUDA;
  if (dev < 0 || dev >= 64 || !attr_set[f8][dev].load(std::memory_order_acquire)) {
    const cudaError_t e =
        f8 ? cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)
           : cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return FLIDE_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[f8][dev].store(true, std::memory_order_release);
  }
  attn_items_kernel<<<1, 1024, 0, s>>>(*x, Hkv, 2 * mtok);
  FLIDE_LAUNCH_CHECK();
  TcParams prm;
  prm.x = *x;
  prm.out = (__nv_bfloat16 *)out;
  prm.descale = descale;
  prm.block_table = paged ? paged->block_table : nullptr;
  prm.req_slot = paged ? paged->req_slot : nullptr;
  prm.max_blocks = paged ? paged->max_blocks : 0;
  prm.block_rows = paged ? paged->block_rows : 0;
  prm.n_blocks = paged ? paged->n_blocks : 0;
  prm.n_slots = paged ? paged->n_slots : 0;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = G;
  prm.mtok = mtok;
  prm.has_past = has_past ? 1 : 0;
  prm.past_rows = has_past ? past_rows : 0;
  prm.qk_log2 = scale * kLog2e;
  const long grid = (long)Hkv * ((x->T + 2 * mtok - 1) / (2 * mtok) + 2L * x->R);
  if (grid <= 0) return FLIDE_OK;
  if (grid > 0x7fffffffL) return FLIDE_ERR_CAPACITY;
  if (f8)
    attn_tc_kernel<true><<<(unsigned)grid, kThreads, SMEM_BYTES, s>>>(mq, mk, mv, mpk, mpv, prm);
  else
    attn_tc_kernel<false><<<(unsigned)grid, kThreads, SMEM_BYTES, s>>>(mq, mk, mv, mpk, mpv, prm);
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
  static std::atomic<int32_t *> cached[64];  // zero-initialised: null
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64) {
    int32_t *c = cached[dev].load(std::memory_order_acquire);
    if (c) return c;
  }
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_work) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64) cached[dev].store((int32_t *)p, std::memory_order_release);
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
  if (dtype == FLIDE_E4M3) return FLIDE_ERR_SHAPE;  // needs descale factors: flide_fork_attn_fp8
  if (idx->R < 0 || idx->R > kNoAllocMaxRequests) return FLIDE_ERR_CAPACITY;
  if (!(flags & FLIDE_FLAG_PORTABLE) && fork_attn_tc_supported(idx, Hq, Hkv, d, dtype)) {
    int32_t *work = noalloc_work_ptr();
    if (!work) return FLIDE_ERR_CUDA;
    flide_tree_index x = *idx;  // same index, work table moved to the fixed array
    x.work = work;
    x.work_len = kNoAllocMaxRequests + 1;
    return fork_attn_tc(q, k, v, past_k, past_v, past_rows, &x, Hq, Hkv, dtype, nullptr, scale,
                        out, (cudaStream_t)stream, nullptr);
  }
  // the CUDA-core kernel keeps no per-call table
  return fork_attn_portable(q, k, v, past_k, past_v, past_rows, idx, Hq, Hkv, d, dtype, scale,
                            out, (cudaStream_t)stream);
}
