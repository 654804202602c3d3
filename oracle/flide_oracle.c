/*
 * flide_oracle.c -- plain, slow CPU oracle for the ForkAttention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load this library.  The product path (the CUDA
 * library under tree_forked_decision_b200/csrc) shares no code with it and
 * never calls it.
 *
 * What it computes, and where each definition comes from (pages on Flide,
 * "tree-forked decision inference"):
 *
 *   - One decision request = a shared prefix (the root node) plus option
 *     branches, possibly nested, laid out in one flattened token stream
 *     (kongchang.com article, introduction; "ForkAttention" section).
 *   - Fork equals isolation: every query of a branch must give exactly what an
 *     isolated forward pass over prefix + ancestors + own branch gives
 *     (kongchang.com, "ForkAttention" section).  Branch tokens must not attend
 *     to other branches (kongchang.com, attention-mask section).
 *   - Gated DeltaNet keeps a per-branch recurrent state that evolves in the same
 *     update order as in isolation (kongchang.com, Gated DeltaNet box).  The
 *     recurrence itself is the gated delta rule
 *     S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t
 *     (the pages describe the layer only in words; this is its standard form).
 *   - A resumed request starts from checkpointed history: past K/V rows for
 *     attention and a saved state for GDN (kongchang.com, "ForkAttention"
 *     section, resume from checkpoints; techfi24.com, "Exact State Forking").
 *
 * Everything is done literally: each branch is rebuilt as its own isolated
 * sequence and run with textbook causal softmax attention or the token-by-token
 * recurrence, in double precision.  Inputs are float32 arrays (bf16 values are
 * exactly representable in float32, so a caller upcasts them first).
 *
 * Readings taken where the pages are silent:
 *   attention scale is passed in (1/sqrt(d)); query head h uses kv head h/G with
 *   G = Hq/Hkv; the own segment is causal with the diagonal included; GDN has
 *   no 1/sqrt(dk) on q; gates arrive as g = log(alpha).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_INVALID 1
#define OR_NOMEM 2

/* ------------------------------------------------------------------------ */
/* Tree structure                                                            */
/* ------------------------------------------------------------------------ */

/* Checks the tree rules: per request, local node 0 is the root (parent -1),
 * every other node has 0 <= parent < self and at least one token; the root may
 * hold zero tokens (its whole prefix can come from the checkpointed past). */
static int validate(int R, const int *req_node_ptr, const int *parent,
                    const int *seg_len, const int *past_len) {
  if (req_node_ptr[0] != 0) return OR_INVALID;
  for (int r = 0; r < R; ++r) {
    int n0 = req_node_ptr[r], n1 = req_node_ptr[r + 1];
    if (n1 < n0) return OR_INVALID;
    if (past_len[r] < 0) return OR_INVALID;
    for (int n = n0; n < n1; ++n) {
      int local = n - n0;
      if (local == 0) {
        if (parent[n] != -1) return OR_INVALID;
        if (seg_len[n] < 0) return OR_INVALID;
      } else {
        if (parent[n] < 0 || parent[n] >= local) return OR_INVALID;
        if (seg_len[n] < 1) return OR_INVALID;
      }
    }
  }
  return OR_OK;
}

/* Request of a global node, by linear search over the request ranges. */
static int node_request(int R, const int *req_node_ptr, int n) {
  for (int r = 0; r < R; ++r)
    if (n >= req_node_ptr[r] && n < req_node_ptr[r + 1]) return r;
  return -1;
}

/* Ancestors of node n (global ids), written root first and n last; returns the
 * count (= depth + 1).  Found by walking parent pointers upward. */
static int ancestors(const int *req_node_ptr, const int *parent, int r, int n,
                     int *out, int cap) {
  int tmp_count = 0;
  int cur = n;
  /* first pass: count */
  while (1) {
    ++tmp_count;
    int p = parent[cur];
    if (p < 0) break;
    cur = req_node_ptr[r] + p;
  }
  if (tmp_count > cap) return -1;
  cur = n;
  for (int i = tmp_count - 1; i >= 0; --i) {
    out[i] = cur;
    int p = parent[cur];
    cur = (p < 0) ? -1 : req_node_ptr[r] + p;
  }
  return tmp_count;
}

/*
 * Index arrays of the flattened stream (kongchang.com "ForkAttention": the
 * request tree encoded as indices over one flat token stream):
 *   node_start[N+1]  running sum of seg_len over nodes in stream order
 *   token_node[T]    node holding each stream token
 *   token_pos[T]     position of the token in its branch's isolated sequence:
 *                    past_len + tokens of strict ancestors + offset in node
 *   depth[N]         number of edges from the request root
 *   anc_ptr[N+1]     CSR row pointers, row n = ancestors of n, root first
 *   anc_node[...]    CSR entries (global node ids), row length depth+1
 *   ctx_len[N]       past_len + tokens of ancestors and the node itself
 * Returns OR_OK or OR_INVALID.  anc_node must hold sum(depth+1) entries;
 * anc_cap bounds it.
 */
int oracle_tree_index(int R, const int *req_node_ptr, const int *parent,
                      const int *seg_len, const int *past_len,
                      int *node_start, int *token_node, int *token_pos,
                      int *depth, int *anc_ptr, int *anc_node, int anc_cap,
                      int *ctx_len) {
  int st = validate(R, req_node_ptr, parent, seg_len, past_len);
  if (st != OR_OK) return st;
  int N = req_node_ptr[R];
  node_start[0] = 0;
  for (int n = 0; n < N; ++n) node_start[n + 1] = node_start[n] + seg_len[n];

  int *chain = (int *)malloc(sizeof(int) * (size_t)(N > 0 ? N : 1));
  if (!chain) return OR_NOMEM;
  anc_ptr[0] = 0;
  for (int n = 0; n < N; ++n) {
    int r = node_request(R, req_node_ptr, n);
    int cnt = ancestors(req_node_ptr, parent, r, n, chain, N);
    depth[n] = cnt - 1;
    if (anc_ptr[n] + cnt > anc_cap) { free(chain); return OR_NOMEM; }
    anc_ptr[n + 1] = anc_ptr[n] + cnt;
    int ctx = past_len[r];
    for (int i = 0; i < cnt; ++i) {
      anc_node[anc_ptr[n] + i] = chain[i];
      ctx += seg_len[chain[i]];
    }
    ctx_len[n] = ctx;
    int before = past_len[r];
    for (int i = 0; i + 1 < cnt; ++i) before += seg_len[chain[i]];
    for (int j = 0; j < seg_len[n]; ++j) {
      token_node[node_start[n] + j] = n;
      token_pos[node_start[n] + j] = before + j;
    }
  }
  free(chain);
  return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Isolated key lists                                                        */
/* ------------------------------------------------------------------------ */

/* The key rows an isolated forward pass for stream token t sees, in order:
 * the request's past rows (negative codes -1-i for past row i of the packed
 * past buffer), then every token of the root and of each later ancestor, then
 * the node's own tokens up to and including t.  Returns the count. */
static int isolated_keys(int R, const int *req_node_ptr, const int *parent,
                         const int *seg_len, const int *past_len,
                         const int *node_start, int t, int *keys, int cap,
                         int *chain) {
  int N = req_node_ptr[R];
  int n = -1;
  for (int i = 0; i < N; ++i)
    if (t >= node_start[i] && t < node_start[i + 1]) { n = i; break; }
  if (n < 0) return -1;
  int r = node_request(R, req_node_ptr, n);
  int past_off = 0;
  for (int i = 0; i < r; ++i) past_off += past_len[i];
  int cnt = ancestors(req_node_ptr, parent, r, n, chain, N);
  int m = 0;
  for (int i = 0; i < past_len[r]; ++i) {
    if (m >= cap) return -1;
    keys[m++] = -1 - (past_off + i);
  }
  for (int a = 0; a + 1 < cnt; ++a)
    for (int j = 0; j < seg_len[chain[a]]; ++j) {
      if (m >= cap) return -1;
      keys[m++] = node_start[chain[a]] + j;
    }
  for (int j = node_start[n]; j <= t; ++j) {
    if (m >= cap) return -1;
    keys[m++] = j;
  }
  return m;
}

/* ------------------------------------------------------------------------ */
/* Attention                                                                 */
/* ------------------------------------------------------------------------ */

/*
 * Textbook softmax attention of one query row over its isolated sequence
 * (kongchang.com "ForkAttention": each branch query equals the isolated
 * forward pass; attention-mask section: no cross-branch keys).
 *   s_j = scale * <q_t^h, k_j^{h/G}>,  o = sum_j softmax(s)_j v_j
 * in double precision with the maximum subtracted before exp.
 *
 * Layouts: q [T, Hq, d], k and v [T, Hkv, d], past_k and past_v
 * [sum(past_len), Hkv, d] packed in request order; all float32.
 * Rows to compute: (row_tok[i], row_head[i]) for i < n_rows, output
 * out[i*d .. i*d+d).  Threads: OpenMP over rows when built with -fopenmp.
 */
int oracle_attention_rows(int R, const int *req_node_ptr, const int *parent,
                          const int *seg_len, const int *past_len, int Hq,
                          int Hkv, int d, const float *q, const float *k,
                          const float *v, const float *past_k,
                          const float *past_v, double scale, int n_rows,
                          const int *row_tok, const int *row_head,
                          double *out) {
  int st = validate(R, req_node_ptr, parent, seg_len, past_len);
  if (st != OR_OK) return st;
  if (Hkv <= 0 || Hq % Hkv != 0) return OR_INVALID;
  int G = Hq / Hkv;
  int N = req_node_ptr[R];
  int *node_start = (int *)malloc(sizeof(int) * (size_t)(N + 1));
  if (!node_start) return OR_NOMEM;
  node_start[0] = 0;
  for (int n = 0; n < N; ++n) node_start[n + 1] = node_start[n] + seg_len[n];
  int T = node_start[N];
  int max_past = 0;
  for (int r = 0; r < R; ++r) max_past = past_len[r] > max_past ? past_len[r] : max_past;
  int cap = T + max_past + 1;
  int err = OR_OK;

#pragma omp parallel
  {
    int *keys = (int *)malloc(sizeof(int) * (size_t)cap);
    int *chain = (int *)malloc(sizeof(int) * (size_t)(N + 1));
    double *s = (double *)malloc(sizeof(double) * (size_t)cap);
    double *acc = (double *)malloc(sizeof(double) * (size_t)d);
    if (!keys || !chain || !s || !acc) {
#pragma omp atomic write
      err = OR_NOMEM;
    } else {
#pragma omp for schedule(dynamic, 4)
      for (int i = 0; i < n_rows; ++i) {
        int t = row_tok[i], h = row_head[i];
        int kvh = h / G;
        int m = isolated_keys(R, req_node_ptr, parent, seg_len, past_len,
                              node_start, t, keys, cap, chain);
        if (m <= 0) {
#pragma omp atomic write
          err = OR_INVALID;
          continue;
        }
        const float *qr = q + ((size_t)t * Hq + h) * d;
        double mx = -INFINITY;
        for (int j = 0; j < m; ++j) {
          const float *kr = keys[j] >= 0
              ? k + ((size_t)keys[j] * Hkv + kvh) * d
              : past_k + ((size_t)(-1 - keys[j]) * Hkv + kvh) * d;
          double dot = 0.0;
          for (int c = 0; c < d; ++c) dot += (double)qr[c] * (double)kr[c];
          s[j] = dot * scale;
          if (s[j] > mx) mx = s[j];
        }
        double denom = 0.0;
        for (int c = 0; c < d; ++c) acc[c] = 0.0;
        for (int j = 0; j < m; ++j) {
          double p = exp(s[j] - mx);
          denom += p;
          const float *vr = keys[j] >= 0
              ? v + ((size_t)keys[j] * Hkv + kvh) * d
              : past_v + ((size_t)(-1 - keys[j]) * Hkv + kvh) * d;
          for (int c = 0; c < d; ++c) acc[c] += p * (double)vr[c];
        }
        for (int c = 0; c < d; ++c) out[(size_t)i * d + c] = acc[c] / denom;
      }
    }
    free(keys); free(chain); free(s); free(acc);
  }
  free(node_start);
  return err;
}

/* ------------------------------------------------------------------------ */
/* Gated DeltaNet                                                            */
/* ------------------------------------------------------------------------ */

/* One token of the gated delta rule on the dv x dk state S (row-major, S[i][c]):
 *   u = S k;  S <- alpha (S - beta u k^T) + beta v k^T,  alpha = exp(g).
 * Equal to S <- alpha S (I - beta k k^T) + beta v k^T. */
static void gdn_step(double *S, int dk, int dv, const float *kt,
                     const float *vt, double g, double beta, double *u) {
  double alpha = exp(g);
  for (int i = 0; i < dv; ++i) {
    double acc = 0.0;
    for (int c = 0; c < dk; ++c) acc += S[(size_t)i * dk + c] * (double)kt[c];
    u[i] = acc;
  }
  for (int i = 0; i < dv; ++i) {
    double w = beta * u[i];
    double bv = beta * (double)vt[i];
    for (int c = 0; c < dk; ++c) {
      double kc = (double)kt[c];
      S[(size_t)i * dk + c] = alpha * (S[(size_t)i * dk + c] - w * kc) + bv * kc;
    }
  }
}

/* o = S q */
static void gdn_read(const double *S, int dk, int dv, const float *qt,
                     double *o) {
  for (int i = 0; i < dv; ++i) {
    double acc = 0.0;
    for (int c = 0; c < dk; ++c) acc += S[(size_t)i * dk + c] * (double)qt[c];
    o[i] = acc;
  }
}

/*
 * Gated DeltaNet over the tree, one selected (request, head) pair at a time.
 * Layouts: q, k [T, H, dk]; v [T, H, dv]; g, beta [T, H] (g = log alpha);
 * state_in [R, H, dv, dk] float32 or NULL (zero start); state_in_f64 the same
 * in double (used instead when non-NULL); out [T, H, dv] doubles (only
 * tokens of selected requests/heads are written); node_state_out
 * [N, H, dv, dk] doubles or NULL: the state after each node's last token.
 *
 * memoise = 0: every node is recomputed in isolation from state_in along
 *   root -> ... -> parent -> node (the definition).
 * memoise = 1: nodes in index order; a node starts from its parent's end
 *   state (the root from state_in).  Same operations on the same values in the
 *   same order, so the results equal memoise = 0 bit for bit.
 */
int oracle_gdn(int R, const int *req_node_ptr, const int *parent,
               const int *seg_len, int H, int dk, int dv, const float *q,
               const float *k, const float *v, const float *g,
               const float *beta, const float *state_in,
               const double *state_in_f64, int memoise,
               int n_sel, const int *sel_req, const int *sel_head,
               double *out, double *node_state_out) {
  int N = req_node_ptr[R];
  int *past_zero = (int *)calloc((size_t)(R > 0 ? R : 1), sizeof(int));
  if (!past_zero) return OR_NOMEM;
  int st = validate(R, req_node_ptr, parent, seg_len, past_zero);
  free(past_zero);
  if (st != OR_OK) return st;
  int *node_start = (int *)malloc(sizeof(int) * (size_t)(N + 1));
  if (!node_start) return OR_NOMEM;
  node_start[0] = 0;
  for (int n = 0; n < N; ++n) node_start[n + 1] = node_start[n] + seg_len[n];
  size_t SS = (size_t)dk * dv;
  int err = OR_OK;

#pragma omp parallel
  {
    double *S = (double *)malloc(sizeof(double) * SS);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    double *o = (double *)malloc(sizeof(double) * (size_t)dv);
    int *chain = (int *)malloc(sizeof(int) * (size_t)(N + 1));
    if (!S || !u || !o || !chain) {
#pragma omp atomic write
      err = OR_NOMEM;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int si = 0; si < n_sel; ++si) {
        int r = sel_req[si], h = sel_head[si];
        int n0 = req_node_ptr[r], n1 = req_node_ptr[r + 1];
        double *ends = NULL;
        if (memoise) {
          ends = (double *)malloc(sizeof(double) * SS * (size_t)(n1 - n0 > 0 ? n1 - n0 : 1));
          if (!ends) {
#pragma omp atomic write
            err = OR_NOMEM;
            continue;
          }
        }
        for (int n = n0; n < n1; ++n) {
          /* starting state */
          if (memoise && parent[n] >= 0) {
            memcpy(S, ends + (size_t)parent[n] * SS, sizeof(double) * SS);
          } else if (state_in_f64) {
            memcpy(S, state_in_f64 + ((size_t)r * H + h) * SS, sizeof(double) * SS);
          } else if (state_in) {
            const float *s0 = state_in + ((size_t)r * H + h) * SS;
            for (size_t e = 0; e < SS; ++e) S[e] = (double)s0[e];
          } else {
            for (size_t e = 0; e < SS; ++e) S[e] = 0.0;
          }
          if (!memoise) {
            int cnt = ancestors(req_node_ptr, parent, r, n, chain, N);
            for (int a = 0; a + 1 < cnt; ++a)
              for (int t = node_start[chain[a]]; t < node_start[chain[a] + 1]; ++t)
                gdn_step(S, dk, dv, k + ((size_t)t * H + h) * dk,
                         v + ((size_t)t * H + h) * dv,
                         (double)g[(size_t)t * H + h],
                         (double)beta[(size_t)t * H + h], u);
          }
          for (int t = node_start[n]; t < node_start[n + 1]; ++t) {
            gdn_step(S, dk, dv, k + ((size_t)t * H + h) * dk,
                     v + ((size_t)t * H + h) * dv,
                     (double)g[(size_t)t * H + h],
                     (double)beta[(size_t)t * H + h], u);
            gdn_read(S, dk, dv, q + ((size_t)t * H + h) * dk, o);
            for (int i = 0; i < dv; ++i) out[((size_t)t * H + h) * dv + i] = o[i];
          }
          if (memoise) memcpy(ends + (size_t)(n - n0) * SS, S, sizeof(double) * SS);
          if (node_state_out)
            memcpy(node_state_out + ((size_t)n * H + h) * SS, S, sizeof(double) * SS);
        }
        free(ends);
      }
    }
    free(S); free(u); free(o); free(chain);
  }
  free(node_start);
  return err;
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
