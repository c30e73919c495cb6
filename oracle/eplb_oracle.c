/*
 * eplb_oracle.c -- plain, slow CPU oracle of the EPLB hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * Sources (cited by page title and section):
 *   [EPLB]  page "DualPipe и EPLB: конвейер в обе стороны и балансировщик
 *           экспертов", Part 2 "EPLB — балансировщик нагрузки для
 *           параллелизма экспертов": sections "Алгоритм" (hierarchical and
 *           global policies), "Интерфейс и пример" (worked example) and the
 *           appendix "Приложение: код eplb.py" (functions balanced_packing,
 *           replicate_experts, rebalance_experts_hierarchical,
 *           rebalance_experts).
 *   [LPLB]  page "DeepSeek开源LPLB：基于线性规划的MoE负载均衡器...", usage
 *           example (planner.run maps logical to physical indices).
 *
 * Arithmetic readings (the pages compute in float32 with an unstable sort):
 *   - loads are integers 0 <= w < 2^40; every comparison is exact;
 *   - load / replica-count ratios are compared by cross-multiplication;
 *   - a sum of ratios w/c is held as the integer  sum w * (LAMBDA / c),
 *     LAMBDA = lcm of the counts in that row; scaling by a positive constant
 *     changes no comparison;
 *   - sorts are stable descending: (value desc, index asc);
 *   - the lightest-pack choice takes the lowest pack index among equals
 *     (first minimum, as Python's min does);
 *   - the heaviest-per-replica choice takes the lowest expert index among
 *     equals (first maximum, as torch's max does).
 *
 * Parity pins for every function here live in tests/test_oracle_pins.py.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef __int128 i128;

#define ORACLE_OK 0
#define ORACLE_ERR_SHAPE 2
#define ORACLE_ERR_DIVISIBILITY 3
#define ORACLE_ERR_RANGE 4
#define ORACLE_ERR_SLOTS 5
#define ORACLE_ERR_ALLOC 9

#define LOAD_LIMIT (((int64_t)1) << 40)

/* ------------------------------------------------------------------------ */
/* S1: load counting.  [EPLB] section "От переводчика: термины": the load of */
/* an expert is the number of tokens the router sent it in the observation   */
/* period.  counts[l, e] = #{(t, k) : idx[l, t, k] == e}.  Indices outside   */
/* [0, E) are not counted; their number is added to *bad.                    */
/* ------------------------------------------------------------------------ */
void oracle_count_loads(const int32_t *idx, int64_t L, int64_t T, int32_t K,
                        int32_t E, int64_t *counts, int accumulate,
                        uint64_t *bad) {
  uint64_t nbad = 0;
  if (!accumulate) memset(counts, 0, sizeof(int64_t) * (size_t)(L * E));
  for (int64_t l = 0; l < L; ++l) {
    for (int64_t t = 0; t < T; ++t) {
      for (int32_t k = 0; k < K; ++k) {
        int32_t e = idx[(l * T + t) * K + k];
        if (e < 0 || e >= E) {
          ++nbad;
          continue;
        }
        counts[l * E + e] += 1;
      }
    }
  }
  if (bad) *bad += nbad;
}

/* ------------------------------------------------------------------------ */
/* S2: sliding-window accumulation.  [EPLB] section "Алгоритм" preamble:     */
/* load is commonly predicted by a moving average over history.              */
/* snap[s, l, e] = sum_{u = max(0, s-W+1)}^{s} steps[u, l, e], emitted for   */
/* s_first <= s < S into snaps[s - s_first].  Exact integers: the running    */
/* sum adds row s and removes row s-W.                                        */
/* ------------------------------------------------------------------------ */
void oracle_window(const int64_t *steps, int64_t S, int64_t L, int32_t E,
                   int64_t W, int64_t s_first, int64_t *snaps) {
  int64_t C = L * (int64_t)E;
  int64_t *acc = (int64_t *)calloc((size_t)(C > 0 ? C : 1), sizeof(int64_t));
  for (int64_t s = 0; s < S; ++s) {
    for (int64_t c = 0; c < C; ++c) {
      acc[c] += steps[s * C + c];
      if (s - W >= 0) acc[c] -= steps[(s - W) * C + c];
    }
    if (s >= s_first)
      memcpy(snaps + (s - s_first) * C, acc, sizeof(int64_t) * (size_t)C);
  }
  free(acc);
}

/* ------------------------------------------------------------------------ */
/* balanced_packing ([EPLB] appendix, balanced_packing): put n weighted      */
/* items into m packs of exactly n/m items.  Items are visited heaviest      */
/* first (stable: equal weights by ascending index); each goes to the        */
/* lightest pack that still has room (lowest index among equally light).     */
/* When n/m == 1 the pages short-cut to item i -> pack i, rank 0.            */
/* ------------------------------------------------------------------------ */
typedef struct {
  i128 w;
  int idx;
} item_t;

static int cmp_desc_stable(const void *a, const void *b) {
  const item_t *x = (const item_t *)a, *y = (const item_t *)b;
  if (x->w > y->w) return -1;
  if (x->w < y->w) return 1;
  return (x->idx > y->idx) - (x->idx < y->idx);
}

static int balanced_packing(const i128 *weight, int n, int m, int *pack_index,
                            int *rank_in_pack) {
  if (m <= 0 || n % m != 0) return ORACLE_ERR_DIVISIBILITY;
  int per_pack = n / m;
  if (per_pack == 1) {
    for (int i = 0; i < n; ++i) {
      pack_index[i] = i;
      rank_in_pack[i] = 0;
    }
    return ORACLE_OK;
  }
  item_t *order = (item_t *)malloc(sizeof(item_t) * (size_t)n);
  i128 *pack_weights = (i128 *)calloc((size_t)m, sizeof(i128));
  int *pack_items = (int *)calloc((size_t)m, sizeof(int));
  if (!order || !pack_weights || !pack_items) {
    free(order); free(pack_weights); free(pack_items);
    return ORACLE_ERR_ALLOC;
  }
  for (int i = 0; i < n; ++i) {
    order[i].w = weight[i];
    order[i].idx = i;
  }
  qsort(order, (size_t)n, sizeof(item_t), cmp_desc_stable);
  for (int j = 0; j < n; ++j) {
    int g = order[j].idx;
    int pack = -1;
    for (int p = 0; p < m; ++p) {
      if (pack_items[p] >= per_pack) continue;
      if (pack < 0 || pack_weights[p] < pack_weights[pack]) pack = p;
    }
    pack_index[g] = pack;
    rank_in_pack[g] = pack_items[pack];
    pack_weights[pack] += weight[g];
    pack_items[pack] += 1;
  }
  free(order);
  free(pack_weights);
  free(pack_items);
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* replicate_experts ([EPLB] appendix, replicate_experts): grow num_log      */
/* experts to num_phy replicas.  Physical j < num_log is expert j; each      */
/* further replica goes to the expert with the largest load per replica      */
/* weight/logcnt (first maximum), whose replica rank is its count before     */
/* the increment.                                                             */
/* ------------------------------------------------------------------------ */
static void replicate_experts(const int64_t *weight, int num_log, int num_phy,
                              int *phy2log, int *rank, int *logcnt) {
  for (int i = 0; i < num_log; ++i) {
    phy2log[i] = i;
    rank[i] = 0;
    logcnt[i] = 1;
  }
  for (int i = num_log; i < num_phy; ++i) {
    int best = 0;
    for (int j = 1; j < num_log; ++j) {
      /* weight[j]/logcnt[j] > weight[best]/logcnt[best] */
      if ((i128)weight[j] * logcnt[best] > (i128)weight[best] * logcnt[j])
        best = j;
    }
    phy2log[i] = best;
    rank[i] = logcnt[best];
    logcnt[best] += 1;
  }
}

static i128 gcd128(i128 a, i128 b) {
  while (b != 0) {
    i128 t = a % b;
    a = b;
    b = t;
  }
  return a;
}

/* ------------------------------------------------------------------------ */
/* One row of the hierarchical policy ([EPLB] section "Иерархическая         */
/* балансировка" and its flowchart), in three steps:                          */
/*   1. spread the expert groups over the nodes so that the nodes' loads are  */
/*      balanced (balanced_packing of the G group loads into N nodes, G/N     */
/*      groups each); a node's experts are then its groups in the order the   */
/*      packing seated them, each group's experts in index order;             */
/*   2. copy experts inside every node (replicate_experts of the node's E/N   */
/*      loads to its P/N slots);                                               */
/*   3. lay each node's copies onto the node's GPUs so that the GPUs' loads   */
/*      are balanced (balanced_packing of the copies' loads w / copies into   */
/*      gpus/N GPUs, P/gpus copies each).                                      */
/* Physical slot of a copy: node * (P/N) + GPU-in-node * (P/gpus) + its seat  */
/* on that GPU.  The global policy calls this with one group on one node.     */
/* ------------------------------------------------------------------------ */
static int plan_row(const int64_t *weight, int E, int P, int G, int N, int gpus,
                    int32_t *phy2log, int32_t *phyrank, int32_t *logcnt) {
  if (E % G != 0 || G % N != 0 || gpus % N != 0 || P % gpus != 0)
    return ORACLE_ERR_DIVISIBILITY;
  const int gsize = E / G;              /* experts per group */
  const int per_node = E / N;           /* experts per node */
  const int slots_per_node = P / N;
  const int slots_per_gpu = P / gpus;
  const int gpus_per_node = gpus / N;
  int rc = ORACLE_OK;

  i128 *group_load = (i128 *)calloc((size_t)G, sizeof(i128));
  int *node_of_group = (int *)malloc(sizeof(int) * (size_t)G);
  int *seat_of_group = (int *)malloc(sizeof(int) * (size_t)G);
  int *member = (int *)malloc(sizeof(int) * (size_t)E);       /* [N][per_node] expert ids */
  int64_t *node_w = (int64_t *)malloc(sizeof(int64_t) * (size_t)per_node);
  int *owner = (int *)malloc(sizeof(int) * (size_t)slots_per_node);   /* copy -> member */
  int *copy_rank = (int *)malloc(sizeof(int) * (size_t)slots_per_node);
  int *copies = (int *)malloc(sizeof(int) * (size_t)per_node);
  i128 *copy_w = (i128 *)malloc(sizeof(i128) * (size_t)slots_per_node);
  int *gpu_of_copy = (int *)malloc(sizeof(int) * (size_t)slots_per_node);
  int *seat_of_copy = (int *)malloc(sizeof(int) * (size_t)slots_per_node);
  if (!group_load || !node_of_group || !seat_of_group || !member || !node_w || !owner ||
      !copy_rank || !copies || !copy_w || !gpu_of_copy || !seat_of_copy) {
    rc = ORACLE_ERR_ALLOC;
    goto out;
  }

  /* 1. groups over nodes */
  for (int e = 0; e < E; ++e) group_load[e / gsize] += weight[e];
  rc = balanced_packing(group_load, G, N, node_of_group, seat_of_group);
  if (rc) goto out;
  for (int g = 0; g < G; ++g) {
    int first = node_of_group[g] * per_node + seat_of_group[g] * gsize;
    for (int j = 0; j < gsize; ++j) member[first + j] = g * gsize + j;
  }

  for (int n = 0; n < N; ++n) {
    const int *mine = member + n * per_node;

    /* 2. copies inside node n */
    for (int i = 0; i < per_node; ++i) node_w[i] = weight[mine[i]];
    replicate_experts(node_w, per_node, slots_per_node, owner, copy_rank, copies);
    for (int i = 0; i < per_node; ++i) logcnt[mine[i]] = copies[i];

    /* 3. copies over node n's GPUs.  A copy carries w / copies; the packing
       compares sums of these ratios exactly by scaling all of them by one
       common multiple D of the copy counts (any D gives the same order).
       With one copy per GPU the packing is the identity and reads no loads.
       A row whose D would exceed 2^62 cannot be held exactly: rejected. */
    for (int j = 0; j < slots_per_node; ++j) copy_w[j] = 0;
    if (slots_per_gpu > 1) {
      i128 D = 1;
      for (int i = 0; i < per_node; ++i) {
        D = D / gcd128(D, copies[i]) * copies[i];
        if (D > ((i128)1 << 62)) { rc = ORACLE_ERR_RANGE; goto out; }
      }
      for (int j = 0; j < slots_per_node; ++j)
        copy_w[j] = (i128)node_w[owner[j]] * (D / copies[owner[j]]);
    }
    rc = balanced_packing(copy_w, slots_per_node, gpus_per_node, gpu_of_copy, seat_of_copy);
    if (rc) goto out;
    for (int j = 0; j < slots_per_node; ++j) {
      int slot = n * slots_per_node + gpu_of_copy[j] * slots_per_gpu + seat_of_copy[j];
      phy2log[slot] = mine[owner[j]];
      phyrank[slot] = copy_rank[j];
    }
  }

out:
  free(group_load); free(node_of_group); free(seat_of_group); free(member);
  free(node_w); free(owner); free(copy_rank); free(copies); free(copy_w);
  free(gpu_of_copy); free(seat_of_copy);
  return rc;
}

/* ------------------------------------------------------------------------ */
/* rebalance_experts ([EPLB] appendix rebalance_experts, sections            */
/* "Иерархическая балансировка" / "Глобальная балансировка"): the            */
/* hierarchical policy when num_groups % num_nodes == 0, otherwise the same  */
/* procedure with one group on one node (global policy).  Then log2phy:      */
/* [E, X] filled with -1 and log2phy[phy2log[p], phyrank[p]] = p.  The pages */
/* size X as the largest logcnt; here the caller passes X and any logcnt     */
/* above it is an error.  phyrank, which the pages compute but do not        */
/* return, is returned too.                                                   */
/* ------------------------------------------------------------------------ */
int oracle_rebalance(const int64_t *loads, int64_t R, int32_t E, int32_t P,
                     int32_t G, int32_t N, int32_t gpus, int32_t X,
                     int32_t *phy2log, int32_t *phyrank, int32_t *logcnt,
                     int32_t *log2phy) {
  if (R < 0 || E <= 0 || P <= 0 || G <= 0 || N <= 0 || gpus <= 0 || X <= 0)
    return ORACLE_ERR_SHAPE;
  if (P < E) return ORACLE_ERR_SHAPE;
  if (E % G != 0 || P % gpus != 0) return ORACLE_ERR_DIVISIBILITY;
  int g = G, n = N;
  if (G % N != 0) { g = 1; n = 1; } /* global policy: gpus % N is not needed */
  for (int64_t r = 0; r < R; ++r) {
    const int64_t *w = loads + r * E;
    for (int e = 0; e < E; ++e)
      if (w[e] < 0 || w[e] >= LOAD_LIMIT) return ORACLE_ERR_RANGE;
    int32_t *p2l = phy2log + r * P, *prk = phyrank + r * P, *cnt = logcnt + r * E;
    int rc = plan_row(w, E, P, g, n, gpus, p2l, prk, cnt);
    if (rc) return rc;
    int32_t *l2p = log2phy + r * (int64_t)E * X;
    for (int64_t i = 0; i < (int64_t)E * X; ++i) l2p[i] = -1;
    for (int p = 0; p < P; ++p) {
      if (prk[p] >= X) return ORACLE_ERR_SLOTS;
      l2p[(int64_t)p2l[p] * X + prk[p]] = p;
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* S5: redirect.  [LPLB] usage example: the planner maps each token's        */
/* logical expert index to a physical expert index.  The replica rule is     */
/* this library's fixed choice: token t of a layer (global index t0 + t)     */
/* uses replica (t0 + t) mod logcnt[l, e], the same for all K slots.         */
/* out[l, t, k] = log2phy[l, e, (t0 + t) mod logcnt[l, e]], e = idx[l,t,k]; */
/* an index outside [0, E) gives -1 and is counted in *bad.                  */
/* ------------------------------------------------------------------------ */
void oracle_redirect(const int32_t *idx, int64_t L, int64_t T, int32_t K,
                     int32_t E, const int32_t *log2phy, int32_t X,
                     const int32_t *logcnt, int64_t t0, int32_t *out,
                     uint64_t *bad) {
  uint64_t nbad = 0;
  for (int64_t l = 0; l < L; ++l) {
    for (int64_t t = 0; t < T; ++t) {
      for (int32_t k = 0; k < K; ++k) {
        int64_t pos = (l * T + t) * K + k;
        int32_t e = idx[pos];
        if (e < 0 || e >= E) {
          out[pos] = -1;
          ++nbad;
          continue;
        }
        int64_t c = logcnt[l * E + e];
        int64_t slot = (t0 + t) % c;
        out[pos] = log2phy[(l * E + e) * (int64_t)X + slot];
      }
    }
  }
  if (bad) *bad += nbad;
}

/* ------------------------------------------------------------------------ */
/* Single-row entry points of the two building blocks, for pin tests.        */
/* ------------------------------------------------------------------------ */
int oracle_balanced_packing(const int64_t *weight, int32_t n, int32_t m,
                            int32_t *pack_index, int32_t *rank_in_pack) {
  i128 *w = (i128 *)malloc(sizeof(i128) * (size_t)(n > 0 ? n : 1));
  int *pi = (int *)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
  int *ri = (int *)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
  if (!w || !pi || !ri) { free(w); free(pi); free(ri); return ORACLE_ERR_ALLOC; }
  for (int i = 0; i < n; ++i) w[i] = weight[i];
  int rc = balanced_packing(w, n, m, pi, ri);
  for (int i = 0; rc == ORACLE_OK && i < n; ++i) {
    pack_index[i] = pi[i];
    rank_in_pack[i] = ri[i];
  }
  free(w); free(pi); free(ri);
  return rc;
}

/* Same, items given as exact fractions num[i] / den[i] (den > 0), compared  */
/* through the common denominator lcm(den).                                   */
int oracle_balanced_packing_frac(const int64_t *num, const int32_t *den,
                                 int32_t n, int32_t m, int32_t *pack_index,
                                 int32_t *rank_in_pack) {
  i128 lambda = 1;
  for (int i = 0; i < n; ++i) {
    if (den[i] <= 0) return ORACLE_ERR_RANGE;
    lambda = lambda / gcd128(lambda, den[i]) * den[i];
    if (lambda > ((i128)1 << 62)) return ORACLE_ERR_RANGE;
  }
  i128 *w = (i128 *)malloc(sizeof(i128) * (size_t)(n > 0 ? n : 1));
  int *pi = (int *)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
  int *ri = (int *)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
  if (!w || !pi || !ri) { free(w); free(pi); free(ri); return ORACLE_ERR_ALLOC; }
  for (int i = 0; i < n; ++i) w[i] = (i128)num[i] * (lambda / den[i]);
  int rc = balanced_packing(w, n, m, pi, ri);
  for (int i = 0; rc == ORACLE_OK && i < n; ++i) {
    pack_index[i] = pi[i];
    rank_in_pack[i] = ri[i];
  }
  free(w); free(pi); free(ri);
  return rc;
}

void oracle_replicate_experts(const int64_t *weight, int32_t num_log,
                              int32_t num_phy, int32_t *phy2log, int32_t *rank,
                              int32_t *logcnt) {
  int *p = (int *)malloc(sizeof(int) * (size_t)num_phy);
  int *r = (int *)malloc(sizeof(int) * (size_t)num_phy);
  int *c = (int *)malloc(sizeof(int) * (size_t)num_log);
  replicate_experts(weight, num_log, num_phy, p, r, c);
  for (int i = 0; i < num_phy; ++i) { phy2log[i] = p[i]; rank[i] = r[i]; }
  for (int i = 0; i < num_log; ++i) logcnt[i] = c[i];
  free(p); free(r); free(c);
}

/* ------------------------------------------------------------------------ */
/* Plan quality ([EPLB] box "От переводчика: что сделать руками", exercise  */
/* 2, and the per-GPU load range of "От переводчика: что на рисунке"): the   */
/* load of GPU g is the sum of w[e] / logcnt[e] over its replicas.  fp64,    */
/* summed in slot order p = g*ppg, g*ppg + 1, ...; stats[r] = {min, max,     */
/* mean, mean / max} over the GPUs (balancedness 1 when max is 0).           */
/* ------------------------------------------------------------------------ */
void oracle_plan_stats(const int64_t *loads, const int32_t *phy2log, const int32_t *logcnt,
                       int64_t R, int32_t E, int32_t P, int32_t gpus, double *gpu_load,
                       double *stats) {
  const int ppg = P / gpus;
  for (int64_t r = 0; r < R; ++r) {
    double mn = 0, mx = 0, sum = 0;
    for (int g = 0; g < gpus; ++g) {
      double acc = 0.0;
      for (int k = 0; k < ppg; ++k) {
        int e = phy2log[r * P + g * ppg + k];
        acc += (double)loads[r * E + e] / (double)logcnt[r * E + e];
      }
      gpu_load[r * gpus + g] = acc;
      if (g == 0 || acc < mn) mn = acc;
      if (g == 0 || acc > mx) mx = acc;
      sum += acc;
    }
    double mean = sum / gpus;
    stats[r * 4 + 0] = mn;
    stats[r * 4 + 1] = mx;
    stats[r * 4 + 2] = mean;
    stats[r * 4 + 3] = mx > 0 ? mean / mx : 1.0;
  }
}

/* ------------------------------------------------------------------------ */
/* Physical -> logical load fold: logical[r, e] = sum of phys[r, p] over the */
/* physical slots p with phy2log[r, p] == e (the serving engine records      */
/* load per physical expert and folds it before rebalancing).                */
/* ------------------------------------------------------------------------ */
void oracle_fold_loads(const int64_t *phys, const int32_t *phy2log, int64_t R, int32_t E,
                       int32_t P, int64_t *logical) {
  memset(logical, 0, sizeof(int64_t) * (size_t)(R * E));
  for (int64_t r = 0; r < R; ++r)
    for (int p = 0; p < P; ++p) logical[r * E + phy2log[r * P + p]] += phys[r * P + p];
}

/* Initial map, the plan before any load is measured: the physical experts  */
/* are the routed ones followed by the redundant ones (vLLM eplb_state        */
/* glossary), and with every expert taken as equally loaded replicate_experts */
/* gives each redundant slot to the lowest-index expert with the fewest       */
/* replicas, so the redundant slots cycle through the experts from 0:         */
/* phy2log[p] = p mod E, phyrank[p] = p div E.                                */
void oracle_initial_map(int64_t R, int32_t E, int32_t P, int32_t *phy2log, int32_t *phyrank) {
  for (int64_t r = 0; r < R; ++r)
    for (int p = 0; p < P; ++p) {
      phy2log[r * P + p] = p % E;
      phyrank[r * P + p] = p / E;
    }
}

/* ------------------------------------------------------------------------ */
/* Plan diff: which new physical slots need their expert's weights copied.   */
/* GPU g keeps min(old_g(e), new_g(e)) replicas of expert e in place; going  */
/* through g's new slots in order, a slot whose expert still has a kept      */
/* replica to spare is kept (src = -1), every other slot copies from the     */
/* lowest old physical slot that held its expert.  moves[r] = slots copied.  */
/* ------------------------------------------------------------------------ */
int oracle_plan_diff(const int32_t *old_p2l, const int32_t *new_p2l, int64_t R, int32_t E,
                     int32_t P, int32_t gpus, int32_t *src, int32_t *moves) {
  if (gpus <= 0 || P % gpus != 0) return ORACLE_ERR_DIVISIBILITY;
  const int ppg = P / gpus;
  int *first_old = (int *)malloc(sizeof(int) * (size_t)E);
  int *old_cnt = (int *)malloc(sizeof(int) * (size_t)E);
  if (!first_old || !old_cnt) { free(first_old); free(old_cnt); return ORACLE_ERR_ALLOC; }
  for (int64_t r = 0; r < R; ++r) {
    const int32_t *o = old_p2l + r * P, *n = new_p2l + r * P;
    for (int e = 0; e < E; ++e) first_old[e] = -1;
    for (int p = P - 1; p >= 0; --p) first_old[o[p]] = p;
    int m = 0;
    for (int g = 0; g < gpus; ++g) {
      for (int e = 0; e < E; ++e) old_cnt[e] = 0;
      for (int k = 0; k < ppg; ++k) old_cnt[o[g * ppg + k]] += 1;
      for (int k = 0; k < ppg; ++k) {
        int p = g * ppg + k, e = n[p];
        if (old_cnt[e] > 0) {
          old_cnt[e] -= 1;
          src[r * P + p] = -1;
        } else {
          src[r * P + p] = first_old[e];
          ++m;
        }
      }
    }
    moves[r] = m;
  }
  free(first_old);
  free(old_cnt);
  return ORACLE_OK;
}
