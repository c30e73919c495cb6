/*
 * eplb.h -- C ABI of libeplb.so, the B200 (sm_100a) hot path of the
 * Expert-Parallelism Load Balancer: count expert loads, accumulate them over
 * a sliding window, rebalance every MoE layer into a replica/placement plan,
 * and redirect token indices to physical replicas.
 *
 * Sources cited below:
 *   [EPLB] page "DualPipe и EPLB: конвейер в обе стороны и балансировщик
 *          экспертов", Part 2 "EPLB": section "Алгоритм" (hierarchical and
 *          global policies, moving-average load prediction), box
 *          "От переводчика: термины" (load = routed tokens), section
 *          "Интерфейс и пример" and the appendix eplb.py (rebalance_experts,
 *          balanced_packing, replicate_experts).
 *   [LPLB] page "DeepSeek开源LPLB：基于线性规划的MoE负载均衡器...", usage
 *          example: a planner maps the router's logical indices to physical
 *          indices.
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" are caller-owned global memory on the current
 *     CUDA device; the library allocates nothing and keeps no state besides
 *     a per-device cache of launch limits.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream).
 *     The return value covers host-side argument checks and launch errors.
 *     Data-dependent errors (an index or load out of range, a wait that ran
 *     out) are reported through the optional device word `status`: when it
 *     is non-NULL the first error code of the call is stored there with an
 *     atomic compare-and-swap from EPLB_OK; callers clear it beforehand.
 *   - Layouts are dense row-major (C order), element strides as stated.
 *   - Integer indices are int32; loads and counts are int64.
 */
#ifndef EPLB_H_
#define EPLB_H_

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum eplb_status {
  EPLB_OK = 0,
  EPLB_ERR_NULL = 1,          /* a required pointer is NULL */
  EPLB_ERR_SHAPE = 2,         /* negative or inconsistent sizes, P < E */
  EPLB_ERR_DIVISIBILITY = 3,  /* E % G, gpus % N or P % gpus is not 0 */
  EPLB_ERR_RANGE = 4,         /* a load outside [0, 2^40), an exact ratio too wide,
                                 a logcnt outside [1, X] given to redirect */
  EPLB_ERR_SLOTS = 5,         /* an expert got more replicas than log2phy slots X */
  EPLB_ERR_CUDA = 6,          /* a CUDA runtime call or launch failed */
  EPLB_ERR_TIMEOUT = 7,       /* reserved: an in-kernel wait gave up (no current kernel waits) */
  EPLB_ERR_ALIGN = 8,         /* a pointer lacks the alignment stated below */
  EPLB_ERR_LIMIT = 9,         /* a size beyond the limits stated in this header */
  EPLB_ERR_INTERNAL = 10      /* checking build only: an internal index check failed (the
                                 access it guards was skipped); never from a normal build */
} eplb_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *eplb_status_string(int32_t status);

/* Message of the last CUDA error seen by a call on this host thread. */
const char *eplb_last_cuda_error(void);

/* ABI version of this library: (major << 16) | minor. */
int32_t eplb_abi_version(void);

/* 1 if this library is the checking build (internal index checks compiled
 * in, built with `python -m moe_expert_load_eplb_b200.build --checks` as
 * libeplb_checks.so), else 0.  The checking build has the same ABI and
 * results; it is slower and meant for tests. */
int32_t eplb_checking_build(void);

/*
 * S1 -- load counting.  [EPLB] "От переводчика: термины": the load of an
 * expert is the number of tokens the router sent it.
 *
 *   counts[l, e] (+)= #{ (t, k) : idx[l, t, k] == e }
 *
 * idx      device int32 [L, T, K] (16-byte aligned); values outside [0, E)
 *          are skipped and their number is added to *bad.
 * counts   device int64 [L, E]; overwritten (accumulate == 0) or added to.
 * bad      device uint64 word, nullable; added to, never cleared.
 * Counting has no data-dependent error: the call takes no status word.
 * Limits:  1 <= E <= 1024, K >= 1, 0 <= L < 2^31, T >= 0, T * K < 2^31.
 * Integer atomics make the result independent of scheduling.
 */
eplb_status eplb_count_loads(const int32_t *idx, int64_t L, int64_t T, int32_t K,
                             int32_t E, int64_t *counts, int32_t accumulate,
                             unsigned long long *bad, cudaStream_t stream);

/*
 * S2 -- sliding-window accumulation.  [EPLB] "Алгоритм": expert load is
 * commonly predicted by a moving average over historical statistics; the
 * window sum is that average times W.
 *
 *   snaps[s - s_first, l, e] = sum_{u = max(0, s-W+1)}^{s} steps[u, l, e],
 *   for s_first <= s < S.
 *
 * steps    device int64 [S, L, E].
 * snaps    device int64 [S - s_first, L, E]; must not overlap steps.
 * zero_row -1, or a row of steps to clear after it has been read (with a
 *          ring of per-step counts: the slot the next step counts into, so
 *          that eplb_count_loads can add to it with accumulate = 1 and no
 *          separate clearing launch).
 * W >= 1 (W >= S gives running totals); 0 <= s_first < S; -1 <= zero_row < S.
 * Sums are exact; wrap-around of int64 is the caller's concern.  No
 * data-dependent error exists, so the call takes no status word.
 * With a ring buffer of the last W per-step counts, s_first = S - 1 = W - 1
 * returns the current window sum (row order does not change a full sum).
 */
eplb_status eplb_window_accumulate(int64_t *steps, int64_t S, int64_t L, int32_t E,
                                   int64_t W, int64_t s_first, int64_t *snaps, int64_t zero_row,
                                   cudaStream_t stream);

/*
 * S3/S4 -- rebalance_experts over R independent rows ([EPLB] "Алгоритм",
 * appendix rebalance_experts / rebalance_experts_hierarchical /
 * balanced_packing / replicate_experts).  Policy: hierarchical when
 * G % N == 0, otherwise the same procedure with one group on one node
 * (global).  Per row:
 *   1. group loads -> balanced_packing over N nodes (G/N groups each);
 *   2. replicate_experts inside every node (E/N -> P/N replicas, each extra
 *      replica to the largest load per replica, lowest index on ties);
 *   3. replica loads w/cnt -> balanced_packing over the node's gpus/N GPUs
 *      (P/gpus replicas each; heaviest first, stable; lightest non-full
 *      GPU, lowest index on ties);
 * all comparisons exact (integer cross-products, sums of w/cnt over a
 * common denominator).  Outputs:
 *   phy2log[r, p]  logical expert of physical slot p (slot p lives on GPU
 *                  p / (P/gpus), node p / (P/N));
 *   phyrank[r, p]  replica rank of slot p among its expert's replicas;
 *   logcnt[r, e]   replicas of expert e;
 *   log2phy[r, e, k] = physical slot of replica k of e, -1 for k >= logcnt.
 *
 * loads    device int64 [R, E], each in [0, 2^40) (else the row's outputs
 *          are -1 / 0 and *status = EPLB_ERR_RANGE).
 * phy2log, phyrank  device int32 [R, P]; logcnt device int32 [R, E];
 * log2phy  device int32 [R, E, X].  X = (P - E) / N + 1 (hierarchical) or
 *          P - E + 1 (global) always suffices; with a smaller X, replicas of
 *          rank >= X are left out of log2phy and *status = EPLB_ERR_SLOTS.
 * gpu_load device double [R, gpus], nullable; stats device double [R, 4],
 *          nullable: the plan quality of each row's new plan, computed in the
 *          same launch while the plan is still on chip -- exactly the figures
 *          of eplb_plan_stats(loads, phy2log, logcnt) (same fp64 operations in
 *          the same order, so bit-identical).  Rows rejected with
 *          EPLB_ERR_RANGE get NaN.
 * Limits:  1 <= E <= 1024, E <= P <= 2048, G | E, gpus | P, N | gpus (hierarchical),
 *          X >= 1, R >= 0.
 */
eplb_status eplb_rebalance(const int64_t *loads, int64_t R, int32_t E, int32_t P,
                           int32_t G, int32_t N, int32_t gpus, int32_t X,
                           int32_t *phy2log, int32_t *phyrank, int32_t *logcnt,
                           int32_t *log2phy, double *gpu_load, double *stats,
                           int32_t *status, cudaStream_t stream);

/*
 * S2 + S3/S4 for a serving ring -- rebalance from the window sum of a ring
 * of per-step counts, in one launch:
 *   loads[r, e] = sum_{w < W} ring[w, r, e]     (the window of the last W
 *                 steps, row order irrelevant: eplb_window_accumulate with
 *                 S = W, s_first = W - 1)
 * then exactly eplb_rebalance on those loads (same outputs, plan quality,
 * limits, errors).
 * ring       device int64 [W, R, E]; each window sum must lie in [0, 2^40).
 * zero_slot  -1, or the ring row to clear after it has been read (the slot
 *            the next step's counts go to, e.g. with eplb_count_redirect and
 *            accumulate = 1); the rest of the ring is only read.
 * loads_out  device int64 [R, E], nullable: receives the window sums.
 */
eplb_status eplb_rebalance_window(int64_t *ring, int64_t W, int64_t zero_slot, int64_t R,
                                  int32_t E, int32_t P, int32_t G, int32_t N, int32_t gpus,
                                  int32_t X, int64_t *loads_out, int32_t *phy2log,
                                  int32_t *phyrank, int32_t *logcnt, int32_t *log2phy,
                                  double *gpu_load, double *stats, int32_t *status,
                                  cudaStream_t stream);

/*
 * S5 -- redirect logical expert indices to physical replicas ([LPLB] usage
 * example: logical indices in, physical indices out).  Replica rule (this
 * library's fixed choice; the pages leave it open): token t of the call is
 * global token t0 + t and uses replica (t0 + t) mod logcnt[l, e] for every
 * one of its K slots, so shards of one batch redirect consistently.
 *
 *   out[l, t, k] = log2phy[l, e, (t0 + t) mod logcnt[l, e]],  e = idx[l, t, k]
 *
 * idx, out device int32 [L, T, K], both 16-byte aligned, not overlapping.
 *          An index outside [0, E) gives -1 and is added to *bad; a logcnt
 *          outside [1, X] gives -1 and *status = EPLB_ERR_RANGE.
 * log2phy  device int32 [L, E, X]; logcnt device int32 [L, E].
 * Limits:  1 <= E <= 1024, 1 <= X, E * X <= 32768, T * K < 2^31, L < 2^31,
 *          0 <= t0, t0 + T < 2^31.
 */
eplb_status eplb_redirect(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                          const int32_t *log2phy, int32_t X, const int32_t *logcnt,
                          int64_t t0, int32_t *out, unsigned long long *bad,
                          int32_t *status, cudaStream_t stream);

/*
 * S1 + S5 fused -- count the loads of a batch and redirect it in one pass over
 * its indices (each index read from HBM once: 8 bytes per index instead of
 * 4 + 8).  Same contracts as eplb_count_loads for idx / counts / accumulate /
 * bad and as eplb_redirect for log2phy / X / logcnt / t0 / out / status; an
 * index outside [0, E) is added to *bad once.  This is the serving order the
 * EPLB pages describe ([EPLB] "Алгоритм": the plan comes from a moving
 * average of past loads): the tables are the plan in force, built from
 * earlier steps, while this batch's counts feed the next plan.
 * Limits:  those of both calls.
 */
eplb_status eplb_count_redirect(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                                int64_t *counts, int32_t accumulate, const int32_t *log2phy,
                                int32_t X, const int32_t *logcnt, int64_t t0, int32_t *out,
                                unsigned long long *bad, int32_t *status, cudaStream_t stream);

/*
 * The serving step in one launch (S1 + S5, then S2 + S3/S4 per layer).  The
 * pages plan from a moving average of recent loads ([EPLB] "Алгоритм") and
 * route with the plan in force ([LPLB] usage example); this call does both
 * for one batch:
 *   1. exactly eplb_count_redirect(idx, ..., counts = ring + slot * L * E,
 *      accumulate = 1, log2phy, X, logcnt, t0, out, bad): the batch is
 *      counted into ring slot `slot` and redirected with the plan in force;
 *   2. then, for every layer l, exactly eplb_rebalance_window on row l of the
 *      ring [W, L, E] (the window sum over all W slots, this batch included)
 *      into next_phy2log / next_phyrank / next_logcnt / next_log2phy, writing
 *      loads_out and the plan quality gpu_load [L, gpus] / stats [L, 4] (all
 *      nullable) and clearing ring row zero_slot (-1: none) after the sum
 *      was read.
 * A layer's plan is built by the CTA that finishes the layer's last chunk,
 * while other layers are still being redirected.
 * ring         device int64 [W, L, E]; ring[slot] must hold the counts that
 *              should be added to (normally zero: cleared by the previous
 *              step's zero_slot).
 * next_*       the next plan, same shapes as eplb_rebalance's outputs with X
 *              slots; must not be the plan in force (log2phy / logcnt).
 * layer_done   device uint32 [L], caller-owned, all zero before the call; the
 *              call leaves it all zero again.  One array per stream: two
 *              calls in flight at once must not share it.
 * Limits and errors: those of eplb_count_redirect and of eplb_rebalance with
 *              R = L; 0 <= slot < W; -1 <= zero_slot < W.  T may be 0 (the
 *              plan is then rebuilt from the ring alone).
 */
eplb_status eplb_serve_step(const int32_t *idx, int64_t L, int64_t T, int32_t K, int32_t E,
                            const int32_t *log2phy, int32_t X, const int32_t *logcnt, int64_t t0,
                            int32_t *out, unsigned long long *bad, int64_t *ring, int64_t W,
                            int64_t slot, int64_t zero_slot, int32_t P, int32_t G, int32_t N,
                            int32_t gpus, int64_t *loads_out, int32_t *next_phy2log,
                            int32_t *next_phyrank, int32_t *next_logcnt, int32_t *next_log2phy,
                            double *gpu_load, double *stats, uint32_t *layer_done,
                            int32_t *status, cudaStream_t stream);

/*
 * eplb_serve_step without the caller's layer_done array: the per-layer
 * counters live in a library-owned device array (4096 layers, one per
 * device, zero at load and left zero by every call), so the call allocates
 * nothing and needs no work buffer.  The pages have no counterpart to this
 * entry point; it is a convenience form of eplb_serve_step with identical
 * results.
 * Because all calls on one device share that array, two calls of this entry
 * point must not be in flight at the same time on one device (e.g. on two
 * streams without ordering between them); use eplb_serve_step with one
 * layer_done array per stream for that.
 * Errors: those of eplb_serve_step, and EPLB_ERR_LIMIT when L > 4096 (checked
 * before anything else).
 */
eplb_status eplb_serve_step_noalloc(const int32_t *idx, int64_t L, int64_t T, int32_t K,
                                    int32_t E, const int32_t *log2phy, int32_t X,
                                    const int32_t *logcnt, int64_t t0, int32_t *out,
                                    unsigned long long *bad, int64_t *ring, int64_t W,
                                    int64_t slot, int64_t zero_slot, int32_t P, int32_t G,
                                    int32_t N, int32_t gpus, int64_t *loads_out,
                                    int32_t *next_phy2log, int32_t *next_phyrank,
                                    int32_t *next_logcnt, int32_t *next_log2phy, double *gpu_load,
                                    double *stats, int32_t *status, cudaStream_t stream);

/*
 * Plan quality ([EPLB] box "От переводчика: что на рисунке": per-GPU load of
 * the worked example, 86.5 .. 156, mean 129; exercise 2 of "что сделать
 * руками": compare max / mean between policies).  Per row r:
 *   gpu_load[r, g] = sum over GPU g's slots p (p / (P/gpus) == g, in slot
 *                    order) of loads[r, phy2log[r,p]] / logcnt[r, phy2log[r,p]]
 *   stats[r] = { min_g, max_g, mean_g (summed in GPU order), mean / max }
 *              (balancedness 1 when max is 0).
 * fp64 with round-to-nearest adds and divides in exactly that order.
 * loads int64 [R, E]; phy2log int32 [R, P]; logcnt int32 [R, E]; gpu_load
 * double [R, gpus] and stats double [R, 4], either may be NULL (not both).
 * A slot naming no expert in [0, E) or an expert with logcnt < 1 is skipped
 * and *status = EPLB_ERR_RANGE.  Limits: gpus | P, gpus <= 16384.
 */
eplb_status eplb_plan_stats(const int64_t *loads, const int32_t *phy2log, const int32_t *logcnt,
                            int64_t R, int32_t E, int32_t P, int32_t gpus, double *gpu_load,
                            double *stats, int32_t *status, cudaStream_t stream);

/*
 * Fold loads recorded per physical expert into loads per logical expert:
 *   logical[r, e] = sum of phys[r, p] over slots p with phy2log[r, p] == e.
 * A serving engine counts routed tokens after redirection (physical space,
 * e.g. eplb_count_loads with E = P on redirected indices) and folds them
 * before the next rebalance.  phys int64 [R, P]; phy2log int32 [R, P];
 * logical int64 [R, E] (overwritten).  Slots naming no expert in [0, E) are
 * skipped and *status = EPLB_ERR_RANGE.  Limits: E <= 4096.
 */
eplb_status eplb_fold_loads(const int64_t *phys, const int32_t *phy2log, int64_t R, int32_t E,
                            int32_t P, int64_t *logical, int32_t *status, cudaStream_t stream);

/*
 * The plan before any load is known (vLLM eplb_state glossary, context only:
 * the routed experts in slots 0 .. E-1, then the redundant slots).  With every expert taken as
 * equally loaded, replicate_experts gives each redundant slot to the
 * lowest-index expert with the fewest replicas, so they cycle from expert 0:
 *   phy2log[r, p] = p mod E,  phyrank[r, p] = p div E  (phyrank nullable).
 */
eplb_status eplb_initial_map(int64_t R, int32_t E, int32_t P, int32_t *phy2log, int32_t *phyrank,
                             cudaStream_t stream);

/*
 * Plan diff: which slots of a new plan must fetch their expert's weights.
 * GPU g (slots g*P/gpus ..) keeps min(old_g(e), new_g(e)) replicas of each
 * expert e in place; going through g's new slots in order, slot p keeps its
 * expert when fewer earlier new slots of g hold it than old slots of g did:
 *   src[r, p] = -1 (kept) or the lowest old slot holding phy2log_new[r, p]
 *               (-2 if no old slot holds it);
 *   moves[r]  = number of slots with src != -1 (nullable).
 * old / new phy2log int32 [R, P]; src int32 [R, P].  Entries outside [0, E)
 * give src = -2 and *status = EPLB_ERR_RANGE.  Limits: gpus | P, E <= 8192.
 */
eplb_status eplb_plan_diff(const int32_t *old_phy2log, const int32_t *new_phy2log, int64_t R,
                           int32_t E, int32_t P, int32_t gpus, int32_t *src, int32_t *moves,
                           int32_t *status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EPLB_H_ */
