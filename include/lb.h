/*
 * lb.h -- C ABI of the B200 (sm_100a) library for the per-layer MoE
 * expert-parallel load-balancing decision path.
 *
 * Sources the operations follow (page titles and sections):
 *   [Libra]  "Libra: Effective yet Efficient Load Balancing for Large-Scale
 *            MoE Inference" (project README), Key Ideas.
 *   [FB]     "FreeBalance: Pre-Routing Online MoE Load Balancing via Residual
 *            Workload Prediction", sec. 2.1-2.2, sec. 3.2 eq. 2-5, Algorithm 1.
 *   [Relief] "A Per-Step Load-Balancing Engine for Expert-Parallel MoE
 *            Serving", The Per-Step Optimum Problem; Methodology, The Relief
 *            Algorithm, Algorithm 1; Three Deployments.
 *
 * Model.  G expert-parallel ranks are modelled logically on one GPU.  A
 * problem has T tokens; token t comes from source rank src(t) = t / (T/G)
 * (one contiguous batch per rank), expert e lives at home(e) = e / (E/G).
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers to caller-owned memory; the
 *     library allocates no device memory and keeps no pointer after return.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     stream-ordered and asynchronous; none of them synchronizes the host,
 *     except lb_get_status.
 *   - `nbatch` >= 1 independent problems of identical shape are processed
 *     by one call; every per-problem array is laid out problem-major and
 *     contiguous (problem b starts at b * per-problem size).
 *   - Return codes: LB_OK; LB_EINVAL for a bad argument (nothing launched);
 *     LB_ECUDA if a launch failed; LB_ENOSPACE if a workspace is too small.
 *     Bad DATA found on the device (an expert id out of range, a repeated id
 *     in a token's row, an inconsistent plan or split) never traps: the
 *     kernel skips the offending element and sets a bit in a per-device
 *     status word that lb_get_status reads.
 *   - int32 counts: T * k * nbatch must be < 2^31.
 */
#ifndef LB_H_
#define LB_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    LB_OK = 0,
    LB_EINVAL = 1,    /* bad argument, nothing launched */
    LB_ECUDA = 2,     /* a CUDA call or launch failed */
    LB_EDATA = 3,     /* bad data seen on the device (lb_get_status) */
    LB_ENOSPACE = 4   /* workspace smaller than required */
};

/* Bits of the device status word (lb_get_status). */
enum {
    LB_DEV_BAD_IDS = 1,      /* expert id out of [0,E) or repeated in a row */
    LB_DEV_TIMEOUT = 2,      /* a bounded wait inside a kernel gave up */
    LB_DEV_BAD_PLAN = 4,     /* plan blob inconsistent (e.g. round not rank-disjoint) */
    LB_DEV_BAD_SPLIT = 8     /* split does not cover the remote tokens it should */
};

/* Limits. */
#define LB_MAX_E_GATE 256    /* experts per gate call (one tcgen05 MMA N) */
#define LB_MAX_K_GATE 16     /* top-k of the gate */
#define LB_MAX_G 64          /* logical ranks */
#define LB_MAX_E 1024        /* experts in the integer stages */
#define LB_MAX_K 32          /* experts per token in the integer stages */
#define LB_MAX_N 32          /* replica slots per rank */

/* ------------------------------------------------------------------------
 * Step 1 -- lookahead gate + top-k   [FB sec. 3.2 eq. 2-5, sec. 2.1; Libra,
 * Key Ideas, lookahead predictor]
 *   logit[b,t,e] = sum_h h[b,t,h] * w[b,e,h] + bias[b,e]   (fp32 accumulate)
 *   ids[b,t,0..k-1] = the k largest logits of row t, in descending order,
 *                     equal logits ordered by ascending expert id.  The
 *                     ranking compares fp32 logits with their ceil(log2 E)
 *                     lowest bits dropped: logits closer than a relative
 *                     2^(ceil(log2 E) - 23) order like equal ones.
 * The same call is the "normal" router when given the layer's own input.
 *   h       bf16 [nbatch, T, H] row-major, 16-byte aligned
 *   w       bf16 [nbatch, E, H] (row e = expert e's gate weights), 16-byte aligned
 *   bias    fp32 [nbatch, E] or NULL (no bias)
 *   ids     int32 [nbatch, T, k]                          (output)
 *   logits  fp32 [nbatch, T, E] or NULL                    (optional output)
 * Limits: 1 <= E <= LB_MAX_E_GATE, 1 <= k <= min(E, LB_MAX_K_GATE),
 * H >= 8 and H % 8 == 0, T >= 0.  T need not be a multiple of the tile.
 * ------------------------------------------------------------------------ */
int lb_predict_topk(const void *h, const void *w, const float *bias,
                    int nbatch, int T, int H, int E, int k,
                    int32_t *ids, float *logits, void *stream);

/* ------------------------------------------------------------------------
 * Step 1 over a chain of layers -- both gates that read one hidden state,
 * in one pass   [FB sec. 3.2 eq. 2-5: layer l's routing is predicted from
 * the hidden state that precedes it, with layer l's own gate]
 * Hidden state h_j (j = 0..L) is the input of layer j-1's normal router and
 * of layer j's lookahead, so one read of h_j serves both:
 *   ids_pred[l] = top-k(h[l]   . w[l]^T + bias[l])   l = 0..L-1  (lookahead)
 *   ids_act[l]  = top-k(h[l+1] . w[l]^T + bias[l])   l = 0..L-1  (normal)
 * Layer 0's lookahead reads h_0, the state before layer 0.  Each row's
 * ranking is that of lb_predict_topk (descending, ties to the lower id),
 * and the logits equal lb_predict_topk's up to fp32 summation order.
 *   h            bf16 [L+1, T, H] row-major, 16-byte aligned
 *   w            bf16 [L, E, H], 16-byte aligned (gates of consecutive
 *                layers adjacent in memory)
 *   bias         fp32 [L, E] or NULL
 *   ids_pred     int32 [L, T, k]                          (output)
 *   ids_act      int32 [L, T, k]                          (output)
 *   logits_pred, logits_act   fp32 [L, T, E] or NULL       (optional outputs)
 * Limits: 16 <= E <= 128 with E % 16 == 0 (the two gates form one MMA tile
 * of N = 2E <= 256 columns), 1 <= k <= min(E, LB_MAX_K_GATE), H >= 8 and
 * H % 8 == 0, 1 <= L <= 65534, T >= 0.  Other shapes: LB_EINVAL (call
 * lb_predict_topk twice instead).  Tuning knobs of lb_gate_tuning that apply
 * to the persistent kernel (stages, CTAs per SM, boxes per stage) apply here.
 * ------------------------------------------------------------------------ */
int lb_predict_topk_chain(const void *h, const void *w, const float *bias,
                          int L, int T, int H, int E, int k,
                          int32_t *ids_pred, int32_t *ids_act,
                          float *logits_pred, float *logits_act, void *stream);

/* Tuning knobs of lb_predict_topk and lb_predict_topk_chain (process-wide;
 * 0 = automatic choice): pipeline stages per CTA (2..8, clamped to what the
 * CTA's shared memory holds); split of H across a
 * CTA cluster (1, 2, 4, 8 or 16), or of N (-2, -4, -8: the S CTAs of a
 * cluster share a token tile, each ranking Epad/S experts, their lists
 * merged over distributed shared memory); persistent kernel (1, 2 or 4 = that many
 * CTAs per SM walking the token tiles with a TMEM accumulator, double-
 * buffered where TMEM allows; 3 = CTA pairs: clusters of two CTAs, one per
 * SM, sharing one MMA of M = 256 over 256-token work units, each CTA
 * loading its 128 tokens and half of the MMA's N weight rows, k <= 8;
 * 5, 7 or 6 = lb_predict_topk only: CTA pairs with H split over two, three
 * or four pairs, one cluster of 4, 6 or 8 CTAs per 256-token unit, the partial
 * accumulators summed by a reduce-scatter over distributed shared memory,
 * k <= 8 and every pair given at least one 64-column block of H;
 * -1 = one CTA per tile); 64-column boxes per
 * pipeline stage of the persistent kernel (1, 2 or 4); token tiles per work
 * unit of the persistent kernel (1 or 2: two tiles share every W box, each
 * with its own accumulator, halving W's L2 traffic); at most max_ctas CTAs
 * in the persistent kernel's grid (0 = its CTAs per SM on every SM; fewer
 * leave SMs to kernels that run beside it on other streams).
 * Automatic: lb_predict_topk_chain with E = 128 (N = 256) and k <= 8 runs
 * CTA pairs; lb_predict_topk with k <= 8, E > 48 and H >= 2048 runs CTA
 * pairs with H split over the most pairs whose clusters fit the device
 * at once: four (from 8 units of 256 tokens, or any number for E > 128),
 * else three (from 8 units), else two (from 16 units; up to twice what
 * fits at once for E > 128); otherwise, with at least two token tiles per SM and E <= 128,
 * persistent with two CTAs per SM (one when two double-buffered
 * accumulators of the MMA's N do not fit TMEM twice) and one tile per unit;
 * otherwise one CTA
 * per tile; when the tiles alone do not fill the GPU, H split across the
 * largest cluster that keeps one wave (at most 8, 16 for one or two tiles),
 * or N split in two where that cluster would be two or fewer.  Results do not depend on the knobs beyond fp32 rounding of
 * split-H partial sums.  LB_EINVAL for values out of range. */
int lb_gate_tuning(int stages, int split, int persistent, int kbox, int tiles_per_unit,
                   int max_ctas);

/* Launch options (process-wide; results are identical under every option).
 * programmatic_dependent_launch = 1 (the default): every kernel without a
 * thread-block cluster, and lb_assign's clustered prep, is launched with
 * programmatic stream serialization, so its launch is processed while the
 * previous kernel on the stream runs; each kernel waits for its
 * predecessor's completion (and the visibility of its writes) before it
 * touches global memory.  The one exception: the prep of lb_assign and
 * lb_decide (or lb_decide's fused kernel when it has no plan step) lets the
 * scatter that follows it start once past its own wait, and the scatter
 * reads the counts and the plan, which that kernel does not write, before
 * its wait.  0 = plain stream order.
 * max_block_threads (0 = 1024, or 256, 512, 1024): the largest thread block
 * the integer kernels use (lb_assign's prep and scatter take up to 1024
 * threads; count, plan and split 512).  512 lets a block of every integer
 * kernel share an SM with one CTA of the persistent gate, so that the
 * integer stages of one batch can run on a second stream beside the gate
 * of the next (with lb_gate_tuning's max_ctas leaving one gate CTA on some
 * SMs).  lb_solve's cluster launch is not affected.  LB_EINVAL for other
 * values. */
int lb_launch_options(int programmatic_dependent_launch, int max_block_threads);

/* ------------------------------------------------------------------------
 * Step 2 -- per-rank histograms   [FB sec. 3.2 eq. 5; Algorithm 1,
 * aggregation of expert workloads; Libra, Key Ideas, "its own tokens"]
 *   cnt[b,g,e] = #{(t,j) : src(t) = g, ids[b,t,j] = e}
 *   ids  int32 [nbatch, T, k];   cnt int32 [nbatch, G, E]   (output)
 * Limits: T % G == 0, 1 <= G <= LB_MAX_G, 1 <= E <= LB_MAX_E,
 * 1 <= k <= LB_MAX_K.  Ids out of range or repeated in a row are skipped and
 * flagged (LB_DEV_BAD_IDS).
 * ------------------------------------------------------------------------ */
int lb_count(const int32_t *ids, int nbatch, int T, int k, int E, int G,
             int32_t *cnt, void *stream);

/* ------------------------------------------------------------------------
 * Step 3 -- locality-aware replica plan   [Libra, Key Ideas, locality-aware
 * expert replication planning, phases 1 and 2; Relief, The Relief
 * Algorithm (replica edges, edge-coloured round schedule)]
 * Phase 1: each rank g imports up to L experts it does not host, those its
 *   own tokens request most, order (cnt[g,e] desc, e asc); never one with
 *   cnt[g,e] == 0.
 * Load model: a token whose source holds its expert is served there; the
 *   rest of expert e's tokens (m[e]) are served at home(e).
 * Phase 2: at most sum_g (N - used[g]) times: u = most-loaded rank (lowest
 *   id on ties); among u's home experts with m[e] > 0 that some rank can
 *   still take (does not hold e, has a free slot), the one with the largest
 *   m[e] (lowest id on ties); v = least-loaded such rank (lowest id on ties);
 *   c = cnt[v,e] becomes local to v and d = min(m[e]-c, max(0, lu-lv) >> 1)
 *   more is credited to v (lu = load[u]-c, lv = load[v]+c); stop if no
 *   candidate or c + d == 0.
 * Edges: one transfer (home(e) -> r, e) per replica, ordered by e then r;
 *   schedule: greedy edge colouring in that order (lowest round free at both
 *   ends); rounds are rank-disjoint.
 *   cnt   int32 [nbatch, G, E] (predicted counts)
 *   plan  caller-allocated [nbatch] blobs of lb_plan_bytes(G,E,N) bytes each
 *         (output; layout below)
 * Limits: E % G == 0, G <= LB_MAX_G, E <= LB_MAX_E, 0 <= L <= N <=
 * min(LB_MAX_N, E - E/G), and the counts plus planning tables fit in one
 * SM's shared memory (about G*E*4 + 32*G*N bytes <= 224 KB; every shape of
 * the pages fits: G*E <= 32768 at N <= 16).
 * ------------------------------------------------------------------------ */
size_t lb_plan_bytes(int G, int E, int N);
int lb_plan_replicas(const int32_t *cnt, int nbatch, int G, int E, int N, int L,
                     void *plan, void *stream);

/* Plan blob layout (byte offsets from the start of one problem's blob).
 * All fields int32 except holds (uint8).  Edge arrays hold n_edges valid
 * entries in schedule order (round by round, edge order inside a round).
 *   hdr[16]        n_edges, n_rounds, n_phase1, n_phase2, G, E, N, L, 0...
 *   used[G]        replica slots used per rank
 *   slots[G*N]     expert id per slot, -1 if empty (phase-1 slots first)
 *   slot_phase[G*N] 1 or 2, 0 if empty
 *   plan_load[G]   load model after phase 2
 *   edge_u[G*N]    home rank of the transfer
 *   edge_v[G*N]    replica rank
 *   edge_e[G*N]    expert
 *   edge_round[G*N]
 *   round_ptr[G*N+1] edges of round r are [round_ptr[r], round_ptr[r+1])
 *   rep_ptr[E+1]   edges of expert e, by ascending replica rank, are
 *   rep_edge[G*N]    rep_edge[rep_ptr[e] .. rep_ptr[e+1]) (schedule indices)
 *   holds[G*E]     uint8, 1 if rank g holds expert e (home or replica)   */
typedef struct {
    size_t hdr, used, slots, slot_phase, plan_load, edge_u, edge_v, edge_e,
        edge_round, round_ptr, rep_ptr, rep_edge, holds, total;
} lb_plan_layout;
int lb_plan_layout_of(int G, int E, int N, lb_plan_layout *out);

/* ------------------------------------------------------------------------
 * Step 3, alternative -- budgeted pairwise expert swaps   [FreeBalance sec.
 * 3.3 eq. 6-10; Algorithm 1]
 * Instead of replicating experts, exchange pairs of experts between ranks
 * (every rank keeps its expert count; no replica, no split).
 *   nhat[e] = sum_g cnt[b,g,e];  L[r] = sum_{e: pi[e]=r} nhat[e]
 *   loop: u = most-loaded rank, v = least-loaded rank (lowest id on ties);
 *     stop if L[u] - L[v] <= tau;
 *     candidates: a on u, b on v, neither moved yet; their swap gives
 *       L'[u] = L[u] - nhat[a] + nhat[b], L'[v] = L[v] - nhat[b] + nhat[a]
 *       (eq. 6-7) and benefit Delta = Phi(L) - Phi(L') with
 *       Phi(L) = max_r L[r] + gamma * sum_r (L[r] - mean)^2 (eq. 8),
 *       evaluated in double as (L[u] - max L') + gamma * (integer change of
 *       the squared term), one rounded product and one rounded sum;
 *     cost C = alpha + 2 * expert_bytes / beta (eq. 9, every expert the same
 *       size); a candidate needs Delta > 0 and C within the residual budgets
 *       of u, of v (`budget` each) and of the pair (u, v) (`link_budget`);
 *     take the largest Delta / C (Delta when C = 0), ties to the smaller
 *       (a, b); swap; update loads and residual budgets; no candidate: stop.
 *   cnt            int32 [nbatch, G, E] predicted counts (lb_count)
 *   placement      int32 [nbatch, E] owner rank of each expert, or NULL for
 *                  the even placement e / (E/G)
 *   gamma, tau >= 0; alpha >= 0 (per-swap overhead), beta > 0 (bandwidth),
 *   expert_bytes >= 0, budget and link_budget >= 0 (+inf allowed), in the
 *   units of C
 *   placement_out  int32 [nbatch, E]                       (output)
 *   swaps_out      int32 [nbatch, lb_swaps_capacity(E), 4]: (u, v, a, b)
 *                  in acceptance order                      (output)
 *   n_swaps        int32 [nbatch]                          (output)
 *   loads          int32 [nbatch, G] rank loads under placement_out (output)
 * Limits: G <= LB_MAX_G, E <= LB_MAX_E, E % G == 0.  A placement entry
 * outside [0, G) sets LB_DEV_BAD_PLAN and that problem gets n_swaps = 0
 * (its other outputs unspecified).
 * ------------------------------------------------------------------------ */
int lb_swaps_capacity(int E);   /* rows of swaps_out per problem: E / 2 (at least 1) */
int lb_plan_swaps(const int32_t *cnt, const int32_t *placement, int nbatch, int G, int E,
                  double gamma, double tau, double alpha, double beta, double expert_bytes,
                  double budget, double link_budget, int32_t *placement_out,
                  int32_t *swaps_out, int32_t *n_swaps, int32_t *loads, void *stream);

/* ------------------------------------------------------------------------
 * Step 4 -- Relief split   [Relief, Methodology, Algorithm 1; The Per-Step
 * Optimum Problem]
 * Remote mass of expert e: R_e = tokens of e whose source does not hold e.
 * For a replicated expert with m edges (ascending replica rank j=0..m-1):
 *   tok_j = R_e/m + (j < R_e % m), mass_j = tok_j (all start at home).
 * L[i] = own tokens of experts i holds + R_e of every expert homed on i.
 * Each pass visits the rounds in order and, inside a round, every transfer:
 *   gap = L[u]-L[v]; delta = min(|gap| >> 1, gap > 0 ? mass : tok - mass);
 *   if delta > 0: L[u] -= sgn(gap) delta; L[v] += sgn(gap) delta;
 *                 mass -= sgn(gap) delta.
 * At most `passes` passes; stops after a pass that moved nothing.
 *   cnt        int32 [nbatch, G, E] (actual counts)
 *   plan       [nbatch] plan blobs from lb_plan_replicas
 *   tok, mass  int32 [nbatch, G*N] (schedule order; entries past n_edges = 0;
 *              may be NULL when G*N == 0)
 *   loads      int32 [nbatch, G];  passes_run int32 [nbatch]   (outputs)
 * Limits: as lb_plan_replicas; 0 <= passes <= 4096.
 * ------------------------------------------------------------------------ */
int lb_split(const int32_t *cnt, const void *plan, int nbatch, int G, int E, int N,
             int passes, int32_t *tok, int32_t *mass, int32_t *loads,
             int32_t *passes_run, void *stream);

/* ------------------------------------------------------------------------
 * Step 4, ablation variants   [Relief, Ablation Results, Table III; The
 * Relief Algorithm, key properties (Q11.20)]
 * The same inputs, starting point and outputs as lb_split, with the pass
 * replaced by variant:
 *   0 Relief (as lb_split)      1 no reverse move (home -> replica only)
 *   2 Jacobi: loads snapshotted per pass, moves of |gap| >> 2
 *   3 hash split: remote tokens divided equally over home and replicas
 *     (home first, remainders to the first holders); no passes
 *   4 water-filling: experts in ascending id, each poured over its holders
 *     from the lowest load up (integer levels, leftovers in holder order,
 *     replicas capped at their edge's tokens)
 *   5 proportional: experts in ascending id, remote tokens divided in
 *     proportion to (max base load - base load + 1), largest remainders,
 *     a replica's excess over its edge's tokens kept at home
 *   6 fp32 Relief (exact halving; masses rounded to nearest, ties to even)
 *   7 Q11.20 Relief (units of 2^-f tokens, f = 20 - s, s the smallest shift
 *     keeping the total load below 2^11; masses rounded to nearest, ties up)
 * Passes end after a pass that changes nothing (all but 3).
 * Limits: as lb_split, G <= 64; rounds of at most 32 transfers.  A plan
 * whose header or round table is inconsistent sets LB_DEV_BAD_PLAN.
 * ------------------------------------------------------------------------ */
int lb_split_variant(const int32_t *cnt, const void *plan, int nbatch, int G, int E, int N,
                     int passes, int variant, int32_t *tok, int32_t *mass, int32_t *loads,
                     int32_t *passes_run, void *stream);

/* ------------------------------------------------------------------------
 * Step 5 -- destinations + stable permutation   [Libra, Key Ideas,
 * two-stage locality-aware execution and token sharding; FB sec. 2.2]
 * For assignment f = t*k + j (e = ids[t,j], s = src(t)):
 *   s holds e -> dest = s; e unreplicated -> dest = home(e); otherwise
 *   q = rank of f among e's remote assignments (ascending f); edge j covers
 *   q in [sum_{i<j} tok_i, ... + tok_j): its first mass_j stay at home(e),
 *   the rest go to the edge's replica rank.
 * perm = stable sort of f by key dest*E + e; offs = exclusive prefix sum of
 * the bucket sizes over all G*E keys, offs[G*E] = T*k.
 *   ids        int32 [nbatch, T, k];  cnt int32 [nbatch, G, E] (lb_count of ids)
 *   plan, tok, mass: from lb_plan_replicas and lb_split
 *   dest       int32 [nbatch, T, k]; perm int32 [nbatch, T*k] (problem-local f)
 *   offs       int32 [nbatch, G*E+1]                       (outputs)
 *   workspace  device scratch of >= lb_assign_workspace_bytes(...) bytes,
 *              256-byte aligned, caller-owned; contents need not be cleared.
 * Limits: T % G == 0, G <= LB_MAX_G, E <= LB_MAX_E, k <= LB_MAX_K.
 * ------------------------------------------------------------------------ */
size_t lb_assign_workspace_bytes(int nbatch, int T, int k, int G, int E, int N);
int lb_assign(const int32_t *ids, const int32_t *cnt, const void *plan,
              const int32_t *tok, const int32_t *mass, int nbatch, int T, int k,
              int G, int E, int N, int32_t *dest, int32_t *perm, int32_t *offs,
              void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Steps 3-5 in two launches -- plan (optional), split, assign   [Libra, Key
 * Ideas; Relief, Algorithm 1; FB sec. 2.2]
 * The same bytes as, in order,
 *   lb_plan_replicas(cnt_pred, nbatch, G, E, N, L, plan)   (if cnt_pred)
 *   lb_split(cnt, plan, nbatch, G, E, N, passes, tok, mass, loads, passes_run)
 *   lb_assign(ids, cnt, plan, tok, mass, nbatch, T, k, G, E, N, dest, perm,
 *             offs, workspace, workspace_bytes)
 * For count tables of fewer than 4096 keys (G*E) the plan, the split and
 * the assign's tables of each problem are made by one block in series (one
 * launch) and the scatter is a second launch; for larger tables, where the
 * separate launches measured faster, the four run as separate launches.
 *   cnt_pred   int32 [nbatch, G, E] or NULL.  NULL: plan is an input (a blob
 *              of lb_plan_replicas) and L is ignored; else plan is written.
 *   other arguments, limits and errors: as the three calls (L, N: as
 *   lb_plan_replicas when cnt_pred is given).
 * ------------------------------------------------------------------------ */
int lb_decide(const int32_t *cnt_pred, const int32_t *cnt, const int32_t *ids,
              void *plan, int nbatch, int T, int k, int G, int E, int N, int L,
              int passes, int32_t *tok, int32_t *mass, int32_t *loads,
              int32_t *passes_run, int32_t *dest, int32_t *perm, int32_t *offs,
              void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Steps 2, 4 and 5 fused -- the per-step decision on the actual ids in one
 * launch   [FB sec. 3.2 eq. 5; Relief, Algorithm 1; Libra, Key Ideas]
 * Computes exactly what lb_count, then lb_split, then lb_assign compute
 * (same outputs, same layouts, bit for bit), with one thread-block cluster
 * per problem: its CTAs count slices of the tokens, CTA 0 combines the counts
 * over distributed shared memory and runs the split and the permutation
 * tables, then every CTA scatters its slice.
 *   ids, plan, passes: as lb_count / lb_split
 *   cnt [nbatch,G,E], tok, mass [nbatch,G*N], loads [nbatch,G],
 *   passes_run [nbatch], dest [nbatch,T,k], perm [nbatch,T*k],
 *   offs [nbatch,G*E+1]: outputs
 *   workspace: >= lb_assign_workspace_bytes(...) bytes, 256-byte aligned
 * Limits: those of lb_count, lb_split and lb_assign together.  Shapes whose
 * cluster tables do not fit one SM's shared memory run as the three separate
 * launches, with the same results.
 * ------------------------------------------------------------------------ */
int lb_solve(const int32_t *ids, const void *plan, int nbatch, int T, int k, int G, int E,
             int N, int passes, int32_t *cnt, int32_t *tok, int32_t *mass, int32_t *loads,
             int32_t *passes_run, int32_t *dest, int32_t *perm, int32_t *offs,
             void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * lb_assign without a caller workspace (the pages have no counterpart; this
 * is a convenience of this library).
 * For callers that cannot provide device scratch memory: a runtime whose
 * device memory all belongs to its own arena, or a plain-C caller with no
 * device allocator (cudaMalloc would also synchronize the device mid-step).
 * Same arguments, outputs and limits as lb_assign, minus the workspace; the
 * scratch is a fixed device array of LB_NOALLOC_SCRATCH_BYTES inside the
 * library, which every GPU that loads the library holds until exit.
 *   - Calls whose lb_assign_workspace_bytes(...) exceeds
 *     LB_NOALLOC_SCRATCH_BYTES return LB_ENOSPACE (lb_last_error says why);
 *     use lb_assign for those.
 *   - It allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *     library routine.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current) and, like the first call of any
 *     entry point, raises its kernels' shared-memory limits on that device;
 *     make that first call before any stream capture.
 *   - All calls share the one array: calls that overlap on the GPU (for
 *     example on two streams) race and give wrong results.  The scratch keeps
 *     the last call's contents; every call fully rewrites what it reads, so
 *     nothing needs clearing.
 * ------------------------------------------------------------------------ */
#define LB_NOALLOC_SCRATCH_BYTES (1u << 20)
int lb_assign_noalloc(const int32_t *ids, const int32_t *cnt, const void *plan,
                      const int32_t *tok, const int32_t *mass, int nbatch, int T, int k,
                      int G, int E, int N, int32_t *dest, int32_t *perm, int32_t *offs,
                      void *stream);

/* ------------------------------------------------------------------------
 * Status and diagnostics (not from the pages).
 * lb_get_status: synchronizes the current device, writes the status word of
 * the current device to *flags (LB_DEV_* bits) and clears it when `clear`
 * is non-zero.  Returns LB_OK, LB_EDATA if any data bit is set, or LB_ECUDA.
 * lb_strerror: static text for a return code.
 * ------------------------------------------------------------------------ */
int lb_get_status(int32_t *flags, int clear);
const char *lb_strerror(int code);
/* Text of the CUDA error behind this thread's last LB_ECUDA return. */
const char *lb_last_error(void);
int lb_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LB_H_ */
