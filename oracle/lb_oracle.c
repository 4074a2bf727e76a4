/*
 * Plain, slow CPU oracle for the per-layer MoE expert-parallel load-balancing
 * decision path.  TEST INFRASTRUCTURE ONLY: the product path never links,
 * loads or calls this file.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Each function follows the definition on the pages it cites, in the order
 * the pages give, with no blocking, fusion or reordering:
 *
 *   orc_gate          lookahead gate + top-k
 *                     (FreeBalance deep dive, sec. 2.1 and sec. 3.2 eq. 2-5;
 *                      Libra README, "Key Ideas", lookahead predictor)
 *   orc_count         per-rank token->expert histogram
 *                     (FreeBalance sec. 3.2 eq. 5; Algorithm 1, aggregation step)
 *   orc_plan          locality-aware replica planning, phase 1 and phase 2,
 *                     replica edges and their round schedule
 *                     (Libra README, "Key Ideas", replication planning;
 *                      Relief summary, "The Relief Algorithm", key properties)
 *   orc_split         Relief bidirectional pairwise relaxation
 *                     (Relief summary, Methodology, Algorithm 1)
 *   orc_assign        final destination per token-assignment and the stable
 *                     (rank, expert) grouping permutation
 *                     (Libra README, "Key Ideas", two-stage execution;
 *                      FreeBalance sec. 2.2)
 *   orc_split_optimum exact integer min-max over the same per-edge feasible
 *                     set (Relief summary, "The Per-Step Optimum Problem")
 *   orc_plan_swaps    budgeted pairwise expert-swap planning, the alternative
 *                     to replication (FreeBalance sec. 3.3 eq. 6-10,
 *                     Algorithm 1)
 *   orc_split_variant the split variants of Relief's ablation (Relief,
 *                     Ablation Results, Table III; Key Properties, Q11.20)
 *
 * Readings taken where the pages are silent are stated beside the code that
 * takes them.  Return codes: 0 ok, 1 invalid argument, 3 bad data.
 *
 * Parity status: every function is pinned by tests under tests/ (hand-worked
 * examples, closed forms, invariants, brute force, independent library
 * computations of the same definition).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_EDATA 3

/* Threads the OpenMP parts (the gate) use; reported with CPU timings. */
int orc_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* bf16 -> double, exactly: a bf16 value is the high half of an IEEE float. */
static double orc_bf16(uint16_t x)
{
    uint32_t u = ((uint32_t)x) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Gate + top-k.                                                            */
/*   logit[t,e] = sum_h h[t,h] * W[e,h] + b[e]  (W stored [E,H])            */
/* accumulated in double, then rounded once to float.  Top-k ranks the      */
/* float logits in descending order; equal values go to the lower expert    */
/* id.  No softmax: it is monotone and does not change the chosen ids.      */
/* ------------------------------------------------------------------------ */
int orc_gate(const uint16_t *h, const uint16_t *w, const float *bias,
             int64_t T, int H, int E, int k,
             float *logits /* [T,E] or NULL */, int32_t *ids /* [T,k] */)
{
    if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E || !h || !w || !ids)
        return ORC_EINVAL;
    int bad = 0;
#pragma omp parallel
    {
        float *row = (float *)malloc(sizeof(float) * (size_t)E);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        if (!row || !taken) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                const uint16_t *ht = h + t * (int64_t)H;
                for (int e = 0; e < E; ++e) {
                    const uint16_t *we = w + (int64_t)e * H;
                    double acc = 0.0;
                    for (int c = 0; c < H; ++c)
                        acc += orc_bf16(ht[c]) * orc_bf16(we[c]);
                    if (bias)
                        acc += (double)bias[e];
                    row[e] = (float)acc;
                    if (logits)
                        logits[t * (int64_t)E + e] = row[e];
                }
                memset(taken, 0, (size_t)E);
                for (int j = 0; j < k; ++j) {
                    int best = -1;
                    for (int e = 0; e < E; ++e) {
                        if (taken[e])
                            continue;
                        if (best < 0 || row[e] > row[best])
                            best = e;
                    }
                    taken[best] = 1;
                    ids[t * (int64_t)k + j] = best;
                }
            }
        }
        free(row);
        free(taken);
    }
    return bad ? ORC_EINVAL : ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Count.  Source rank of token t is src(t) = t / (T/G): each rank          */
/* contributes one contiguous batch of T/G tokens.                          */
/*   cnt[g,e] = #{(t,j) : src(t) = g, ids[t,j] = e}                         */
/* A row with an id outside [0,E) or a repeated id is bad data.             */
/* ------------------------------------------------------------------------ */
int orc_count(const int32_t *ids, int64_t T, int k, int E, int G, int32_t *cnt)
{
    if (T < 0 || k <= 0 || E <= 0 || G <= 0 || T % G != 0 || !cnt)
        return ORC_EINVAL;
    memset(cnt, 0, sizeof(int32_t) * (size_t)G * (size_t)E);
    if (T == 0)
        return ORC_OK;
    int64_t Tg = T / G;
    for (int64_t t = 0; t < T; ++t) {
        int g = (int)(t / Tg);
        for (int j = 0; j < k; ++j) {
            int32_t e = ids[t * k + j];
            if (e < 0 || e >= E)
                return ORC_EDATA;
            for (int jj = 0; jj < j; ++jj)
                if (ids[t * k + jj] == e)
                    return ORC_EDATA;
            cnt[(int64_t)g * E + e] += 1;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Plan.                                                                    */
/* home(e) = e / (E/G)  (even placement, FreeBalance sec. 2.2).             */
/*                                                                          */
/* Phase 1 (Libra, phase 1): every rank g, independently, imports up to L   */
/* experts it does not host, those its own tokens request most: order       */
/* (cnt[g,e] desc, e asc); an expert none of g's tokens requests is never   */
/* imported.                                                                */
/*                                                                          */
/* Load model used by phase 2: an assignment whose source rank holds its    */
/* expert is served there (Libra's MoE_local); all other "remote" mass of   */
/* expert e, m[e], is served at home(e).                                    */
/*                                                                          */
/* Phase 2 (Libra, phase 2), at most sum_g (N - used[g]) iterations:        */
/*   u = most-loaded rank (lowest id on ties);                              */
/*   candidates = experts homed on u with m[e] > 0, order (m desc, e asc);  */
/*   the first candidate with an eligible rank (does not hold e, has a free */
/*   slot) is taken, v = least-loaded eligible rank (lowest id on ties);    */
/*   none -> stop.                                                          */
/*   v's own tokens of e become local (c = cnt[v,e]); the replica is then   */
/*   credited with d = min(m' , max(0, lu - lv) >> 1) of the remaining      */
/*   remote mass (the same truncating halving the split uses).  c + d == 0  */
/*   -> stop, else commit.                                                  */
/*                                                                          */
/* Edges: one transfer (u = home(e), v = r, e) per replica, e ascending     */
/* then r ascending.  Schedule: greedy edge colouring in edge order, each   */
/* edge takes the lowest round where neither endpoint is busy; the output   */
/* lists the edges round by round, in edge order inside a round.           */
/* ------------------------------------------------------------------------ */
int orc_plan(const int32_t *cnt, int G, int E, int N, int L,
             uint8_t *holds /* [G,E] */, int32_t *used /* [G] */,
             int32_t *slots /* [G,N] */, int32_t *slot_phase /* [G,N] */,
             int64_t *plan_load /* [G] */,
             int32_t *edge_u, int32_t *edge_v, int32_t *edge_e /* [G*N] */,
             int32_t *edge_round /* [G*N] */, int32_t *round_ptr /* [G*N+1] */,
             int32_t *n_edges_out, int32_t *n_rounds_out)
{
    if (G <= 0 || E <= 0 || E % G != 0 || N < 0 || L < 0 || L > N ||
        N > E - E / G)
        return ORC_EINVAL;
    const int Eg = E / G;
    for (int64_t i = 0; i < (int64_t)G * E; ++i)
        if (cnt[i] < 0)
            return ORC_EDATA;

    memset(holds, 0, (size_t)G * (size_t)E);
    for (int e = 0; e < E; ++e)
        holds[(int64_t)(e / Eg) * E + e] = 1;
    for (int g = 0; g < G; ++g)
        used[g] = 0;
    for (int64_t i = 0; i < (int64_t)G * N; ++i) {
        slots[i] = -1;
        slot_phase[i] = 0;
    }

    /* phase 1 */
    for (int g = 0; g < G; ++g) {
        for (int pick = 0; pick < L; ++pick) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (e / Eg == g || holds[(int64_t)g * E + e])
                    continue;
                int32_t c = cnt[(int64_t)g * E + e];
                if (c <= 0)
                    continue;
                if (best < 0 || c > cnt[(int64_t)g * E + best])
                    best = e;
            }
            if (best < 0)
                break;
            holds[(int64_t)g * E + best] = 1;
            slots[(int64_t)g * N + used[g]] = best;
            slot_phase[(int64_t)g * N + used[g]] = 1;
            used[g] += 1;
        }
    }

    /* load model */
    int64_t *m = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *load = (int64_t *)calloc((size_t)G, sizeof(int64_t));
    unsigned char *tried = (unsigned char *)malloc((size_t)E);
    if (!m || !load || !tried) {
        free(m); free(load); free(tried);
        return ORC_EINVAL;
    }
    for (int e = 0; e < E; ++e)
        for (int s = 0; s < G; ++s)
            if (!holds[(int64_t)s * E + e])
                m[e] += cnt[(int64_t)s * E + e];
    for (int r = 0; r < G; ++r) {
        int64_t x = 0;
        for (int e = 0; e < E; ++e)
            if (holds[(int64_t)r * E + e])
                x += cnt[(int64_t)r * E + e];
        for (int e = r * Eg; e < (r + 1) * Eg; ++e)
            x += m[e];
        load[r] = x;
    }

    /* phase 2 */
    int64_t iters = 0;
    for (int g = 0; g < G; ++g)
        iters += N - used[g];
    for (int64_t it = 0; it < iters; ++it) {
        int u = 0;
        for (int r = 1; r < G; ++r)
            if (load[r] > load[u])
                u = r;
        memset(tried, 0, (size_t)E);
        int ce = -1, cv = -1;
        for (;;) {
            int best = -1;
            for (int e = u * Eg; e < (u + 1) * Eg; ++e) {
                if (tried[e] || m[e] <= 0)
                    continue;
                if (best < 0 || m[e] > m[best])
                    best = e;
            }
            if (best < 0)
                break;
            tried[best] = 1;
            int v = -1;
            for (int r = 0; r < G; ++r) {
                if (holds[(int64_t)r * E + best] || used[r] >= N)
                    continue;
                if (v < 0 || load[r] < load[v])
                    v = r;
            }
            if (v >= 0) {
                ce = best;
                cv = v;
                break;
            }
        }
        if (ce < 0)
            break;
        int64_t c = cnt[(int64_t)cv * E + ce];
        int64_t mr = m[ce] - c;
        int64_t lu = load[u] - c;
        int64_t lv = load[cv] + c;
        int64_t gap = lu - lv;
        int64_t d = gap > 0 ? (gap >> 1) : 0;
        if (d > mr)
            d = mr;
        if (c + d == 0)
            break;
        holds[(int64_t)cv * E + ce] = 1;
        slots[(int64_t)cv * N + used[cv]] = ce;
        slot_phase[(int64_t)cv * N + used[cv]] = 2;
        used[cv] += 1;
        m[ce] = mr - d;
        load[u] = lu - d;
        load[cv] = lv + d;
    }
    for (int r = 0; r < G; ++r)
        plan_load[r] = load[r];
    free(m);
    free(load);
    free(tried);

    /* edges in edge order */
    int64_t maxe = (int64_t)G * N;
    int32_t *ou = (int32_t *)malloc(sizeof(int32_t) * (size_t)(maxe + 1));
    int32_t *ov = (int32_t *)malloc(sizeof(int32_t) * (size_t)(maxe + 1));
    int32_t *oe = (int32_t *)malloc(sizeof(int32_t) * (size_t)(maxe + 1));
    int32_t *orr = (int32_t *)malloc(sizeof(int32_t) * (size_t)(maxe + 1));
    unsigned char *busy = (unsigned char *)calloc((size_t)G * (size_t)(maxe + 1), 1);
    if (!ou || !ov || !oe || !orr || !busy) {
        free(ou); free(ov); free(oe); free(orr); free(busy);
        return ORC_EINVAL;
    }
    int ne = 0;
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < G; ++r)
            if (r != e / Eg && holds[(int64_t)r * E + e]) {
                ou[ne] = e / Eg;
                ov[ne] = r;
                oe[ne] = e;
                ne++;
            }
    /* greedy colouring */
    int nr = 0;
    for (int i = 0; i < ne; ++i) {
        int c = 0;
        while (busy[(int64_t)ou[i] * (maxe + 1) + c] || busy[(int64_t)ov[i] * (maxe + 1) + c])
            c++;
        busy[(int64_t)ou[i] * (maxe + 1) + c] = 1;
        busy[(int64_t)ov[i] * (maxe + 1) + c] = 1;
        orr[i] = c;
        if (c + 1 > nr)
            nr = c + 1;
    }
    /* list round by round, edge order inside a round */
    int pos = 0;
    for (int c = 0; c < nr; ++c) {
        round_ptr[c] = pos;
        for (int i = 0; i < ne; ++i)
            if (orr[i] == c) {
                edge_u[pos] = ou[i];
                edge_v[pos] = ov[i];
                edge_e[pos] = oe[i];
                edge_round[pos] = c;
                pos++;
            }
    }
    round_ptr[nr] = pos;
    *n_edges_out = ne;
    *n_rounds_out = nr;
    free(ou); free(ov); free(oe); free(orr); free(busy);
    return ORC_OK;
}

/* Per-expert view of the edges: the edges of expert e ordered by replica
 * rank ascending (this is edge order), with their positions in the
 * schedule-ordered arrays.  Returns 0 or ORC_EDATA on an invalid edge list. */
static int orc_edges_by_expert(int G, int E, const uint8_t *holds, int n_edges,
                               const int32_t *edge_u, const int32_t *edge_v,
                               const int32_t *edge_e,
                               int32_t *rep_cnt /* [E] */,
                               int32_t *rep_ptr /* [E+1] */,
                               int32_t *rep_edge /* [n_edges] */)
{
    const int Eg = E / G;
    for (int e = 0; e < E; ++e)
        rep_cnt[e] = 0;
    for (int i = 0; i < n_edges; ++i) {
        int e = edge_e[i];
        if (e < 0 || e >= E || edge_u[i] != e / Eg || edge_v[i] < 0 ||
            edge_v[i] >= G || edge_v[i] == edge_u[i] ||
            !holds[(int64_t)edge_v[i] * E + e])
            return ORC_EDATA;
        rep_cnt[e]++;
    }
    rep_ptr[0] = 0;
    for (int e = 0; e < E; ++e)
        rep_ptr[e + 1] = rep_ptr[e] + rep_cnt[e];
    for (int e = 0; e < E; ++e) {
        /* selection of this expert's edges in ascending replica rank */
        int w = rep_ptr[e];
        for (int r = 0; r < G; ++r)
            for (int i = 0; i < n_edges; ++i)
                if (edge_e[i] == e && edge_v[i] == r)
                    rep_edge[w++] = i;
        if (w != rep_ptr[e + 1])
            return ORC_EDATA; /* duplicate edge */
    }
    return ORC_OK;
}

/* Starting split of each replicated expert: its remote mass R_e (tokens from
 * sources that do not hold e) is partitioned over its m replica edges,
 * j = 0..m-1 in ascending replica rank: tok_j = R_e/m + (j < R_e mod m).
 * Every token starts at home: mass_j = tok_j.  Fixed load of rank i: its own
 * tokens of experts it holds, plus the remote mass of its unreplicated home
 * experts. */
static void orc_split_start(const int32_t *cnt, int G, int E, const uint8_t *holds,
                            const int32_t *rep_cnt, const int32_t *rep_ptr,
                            const int32_t *rep_edge, int64_t *R,
                            int64_t *fixed, int32_t *tok)
{
    const int Eg = E / G;
    for (int e = 0; e < E; ++e) {
        int64_t r = 0;
        for (int s = 0; s < G; ++s)
            if (!holds[(int64_t)s * E + e])
                r += cnt[(int64_t)s * E + e];
        R[e] = r;
    }
    for (int i = 0; i < G; ++i) {
        int64_t x = 0;
        for (int e = 0; e < E; ++e)
            if (holds[(int64_t)i * E + e])
                x += cnt[(int64_t)i * E + e];
        for (int e = i * Eg; e < (i + 1) * Eg; ++e)
            if (rep_cnt[e] == 0)
                x += R[e];
        fixed[i] = x;
    }
    for (int e = 0; e < E; ++e) {
        int mcount = rep_cnt[e];
        for (int j = 0; j < mcount; ++j) {
            int i = rep_edge[rep_ptr[e] + j];
            tok[i] = (int32_t)(R[e] / mcount + (j < R[e] % mcount ? 1 : 0));
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Split: Relief, Algorithm 1, integer token counts.                        */
/* L[i] starts at fixed[i] plus every edge's mass at its home u.  A pass    */
/* visits the rounds in order and the transfers of a round (rank-disjoint,  */
/* so their order inside the round does not matter):                        */
/*   gap = L[u] - L[v]; delta = |gap| >> 1;                                 */
/*   limit = gap > 0 ? mass : tok - mass; delta = min(delta, limit);        */
/*   if delta > eps: L[u] -= sgn(gap) delta; L[v] += sgn(gap) delta;        */
/*                   mass -= sgn(gap) delta.                                */
/* eps = 0.  Up to `passes` passes; the loop ends after a pass that moved   */
/* nothing (a fixpoint, so later passes would change nothing).              */
/* passes_run = passes executed, that last no-move pass included.           */
/* ------------------------------------------------------------------------ */
int orc_split(const int32_t *cnt, int G, int E, const uint8_t *holds,
              int n_edges, const int32_t *edge_u, const int32_t *edge_v,
              const int32_t *edge_e, int n_rounds, const int32_t *round_ptr,
              int passes, int32_t *tok, int32_t *mass, int64_t *loads,
              int32_t *passes_run)
{
    if (G <= 0 || E <= 0 || E % G != 0 || n_edges < 0 || n_rounds < 0 || passes < 0)
        return ORC_EINVAL;
    if (round_ptr[0] != 0 || round_ptr[n_rounds] != n_edges)
        return ORC_EDATA;
    /* every round must be rank-disjoint */
    unsigned char *seen = (unsigned char *)calloc((size_t)G, 1);
    int32_t *rep_cnt = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *rep_ptr = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *rep_edge = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_edges + 1));
    int64_t *R = (int64_t *)malloc(sizeof(int64_t) * (size_t)E);
    int64_t *fixed = (int64_t *)malloc(sizeof(int64_t) * (size_t)G);
    int rc = ORC_OK;
    if (!seen || !rep_cnt || !rep_ptr || !rep_edge || !R || !fixed) {
        rc = ORC_EINVAL;
        goto done;
    }
    for (int r = 0; r < n_rounds; ++r) {
        memset(seen, 0, (size_t)G);
        if (round_ptr[r + 1] < round_ptr[r]) { rc = ORC_EDATA; goto done; }
        for (int i = round_ptr[r]; i < round_ptr[r + 1]; ++i) {
            if (edge_u[i] < 0 || edge_u[i] >= G || edge_v[i] < 0 || edge_v[i] >= G ||
                seen[edge_u[i]] || seen[edge_v[i]]) {
                rc = ORC_EDATA;
                goto done;
            }
            seen[edge_u[i]] = 1;
            seen[edge_v[i]] = 1;
        }
    }
    rc = orc_edges_by_expert(G, E, holds, n_edges, edge_u, edge_v, edge_e,
                             rep_cnt, rep_ptr, rep_edge);
    if (rc != ORC_OK)
        goto done;
    orc_split_start(cnt, G, E, holds, rep_cnt, rep_ptr, rep_edge, R, fixed, tok);
    for (int i = 0; i < G; ++i)
        loads[i] = fixed[i];
    for (int i = 0; i < n_edges; ++i) {
        mass[i] = tok[i];
        loads[edge_u[i]] += tok[i];
    }
    *passes_run = 0;
    for (int p = 1; p <= passes; ++p) {
        int moved = 0;
        for (int r = 0; r < n_rounds; ++r) {
            for (int i = round_ptr[r]; i < round_ptr[r + 1]; ++i) {
                int u = edge_u[i], v = edge_v[i];
                int64_t gap = loads[u] - loads[v];
                int64_t delta = (gap < 0 ? -gap : gap) >> 1;
                int64_t limit = gap > 0 ? (int64_t)mass[i] : (int64_t)(tok[i] - mass[i]);
                if (delta > limit)
                    delta = limit;
                if (delta > 0) {
                    int64_t sd = gap > 0 ? delta : -delta;
                    loads[u] -= sd;
                    loads[v] += sd;
                    mass[i] -= (int32_t)sd;
                    moved = 1;
                }
            }
        }
        *passes_run = p;
        if (!moved)
            break;
    }
done:
    free(seen); free(rep_cnt); free(rep_ptr); free(rep_edge); free(R); free(fixed);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Assign.  For assignment f = t*k + j with e = ids[t,j], s = src(t):       */
/*   s holds e                -> dest = s   (served locally)                */
/*   e has no replica         -> dest = home(e)                             */
/*   otherwise: q = rank of f among the remote assignments of e, in         */
/*   ascending f; edge j (ascending replica rank) covers q in               */
/*   [off_j, off_j + tok_j); the first mass_j of that range stay at home(e),*/
/*   the other tok_j - mass_j go to the edge's replica rank.                */
/* perm: stable counting sort of f by key dest*E + e; offs[key] is the      */
/* exclusive prefix sum of the bucket sizes, offs[G*E] = T*k.               */
/* ------------------------------------------------------------------------ */
int orc_assign(const int32_t *ids, int64_t T, int k, int G, int E,
               const uint8_t *holds, int n_edges, const int32_t *edge_u,
               const int32_t *edge_v, const int32_t *edge_e,
               const int32_t *tok, const int32_t *mass,
               int32_t *dest, int32_t *perm, int32_t *offs /* [G*E+1] */)
{
    if (T < 0 || k <= 0 || G <= 0 || E <= 0 || E % G != 0 || T % G != 0 || n_edges < 0)
        return ORC_EINVAL;
    const int Eg = E / G;
    const int64_t nf = T * k;
    const int64_t nkeys = (int64_t)G * E;
    int32_t *rep_cnt = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *rep_ptr = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *rep_edge = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_edges + 1));
    int64_t *qctr = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *fill = (int64_t *)calloc((size_t)(nkeys + 1), sizeof(int64_t));
    int rc = ORC_OK;
    if (!rep_cnt || !rep_ptr || !rep_edge || !qctr || !fill) {
        rc = ORC_EINVAL;
        goto done;
    }
    rc = orc_edges_by_expert(G, E, holds, n_edges, edge_u, edge_v, edge_e,
                             rep_cnt, rep_ptr, rep_edge);
    if (rc != ORC_OK)
        goto done;
    for (int i = 0; i < n_edges; ++i)
        if (tok[i] < 0 || mass[i] < 0 || mass[i] > tok[i]) { rc = ORC_EDATA; goto done; }

    const int64_t Tg = T > 0 ? T / G : 1;
    for (int64_t f = 0; f < nf; ++f) {
        int64_t t = f / k;
        int e = ids[f];
        if (e < 0 || e >= E) { rc = ORC_EDATA; goto done; }
        int s = (int)(t / Tg);
        int home = e / Eg;
        int d;
        if (holds[(int64_t)s * E + e]) {
            d = s;
        } else if (rep_cnt[e] == 0) {
            d = home;
        } else {
            int64_t q = qctr[e]++;
            int64_t off = 0;
            d = -1;
            for (int jj = 0; jj < rep_cnt[e]; ++jj) {
                int i = rep_edge[rep_ptr[e] + jj];
                if (q < off + tok[i]) {
                    d = (q - off < mass[i]) ? home : edge_v[i];
                    break;
                }
                off += tok[i];
            }
            if (d < 0) { rc = ORC_EDATA; goto done; } /* split covers fewer tokens */
        }
        dest[f] = d;
    }
    /* every remote token of a replicated expert must be covered exactly */
    for (int e = 0; e < E; ++e) {
        if (rep_cnt[e] == 0)
            continue;
        int64_t tot = 0;
        for (int jj = 0; jj < rep_cnt[e]; ++jj)
            tot += tok[rep_edge[rep_ptr[e] + jj]];
        if (tot != qctr[e]) { rc = ORC_EDATA; goto done; }
    }
    /* stable counting sort by key = dest*E + e */
    for (int64_t f = 0; f < nf; ++f)
        fill[(int64_t)dest[f] * E + ids[f]] += 1;
    {
        int64_t run = 0;
        for (int64_t key = 0; key < nkeys; ++key) {
            int64_t sz = fill[key];
            offs[key] = (int32_t)run;
            fill[key] = run;
            run += sz;
        }
        offs[nkeys] = (int32_t)run;
    }
    for (int64_t f = 0; f < nf; ++f) {
        int64_t key = (int64_t)dest[f] * E + ids[f];
        perm[fill[key]++] = (int32_t)f;
    }
done:
    free(rep_cnt); free(rep_ptr); free(rep_edge); free(qctr); free(fill);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Exact per-step optimum over the same feasible set as the split: fixed    */
/* loads stay, each replica edge's tok_j tokens may be divided in any       */
/* integer way between its two ranks.  Minimum over those of max_i L_i,     */
/* found by binary search on z with a max-flow feasibility test             */
/* (source -> edge (cap tok_j) -> {u_j, v_j} -> rank i (cap z - fixed_i)    */
/* -> sink).  Flow integrality makes the result the exact integer optimum.  */
/* This is the min-max program of the Relief summary in integer form.       */
/* Returns the optimum (>= 0) or a negative error code.                     */
/* ------------------------------------------------------------------------ */
typedef struct {
    int n, m, cap_m;
    int *head, *nxt, *to;
    int64_t *cap;
    int *level, *it, *queue;
} orc_flow;

static int orc_flow_init(orc_flow *f, int n, int max_edges)
{
    f->n = n;
    f->m = 0;
    f->cap_m = 2 * max_edges;
    f->head = (int *)malloc(sizeof(int) * (size_t)n);
    f->nxt = (int *)malloc(sizeof(int) * (size_t)f->cap_m);
    f->to = (int *)malloc(sizeof(int) * (size_t)f->cap_m);
    f->cap = (int64_t *)malloc(sizeof(int64_t) * (size_t)f->cap_m);
    f->level = (int *)malloc(sizeof(int) * (size_t)n);
    f->it = (int *)malloc(sizeof(int) * (size_t)n);
    f->queue = (int *)malloc(sizeof(int) * (size_t)n);
    if (!f->head || !f->nxt || !f->to || !f->cap || !f->level || !f->it || !f->queue)
        return -1;
    for (int i = 0; i < n; ++i)
        f->head[i] = -1;
    return 0;
}

static void orc_flow_free(orc_flow *f)
{
    free(f->head); free(f->nxt); free(f->to); free(f->cap);
    free(f->level); free(f->it); free(f->queue);
}

static void orc_flow_add(orc_flow *f, int a, int b, int64_t c)
{
    f->to[f->m] = b; f->cap[f->m] = c; f->nxt[f->m] = f->head[a]; f->head[a] = f->m++;
    f->to[f->m] = a; f->cap[f->m] = 0; f->nxt[f->m] = f->head[b]; f->head[b] = f->m++;
}

static int orc_flow_bfs(orc_flow *f, int s, int t)
{
    for (int i = 0; i < f->n; ++i)
        f->level[i] = -1;
    int qh = 0, qt = 0;
    f->queue[qt++] = s;
    f->level[s] = 0;
    while (qh < qt) {
        int a = f->queue[qh++];
        for (int x = f->head[a]; x >= 0; x = f->nxt[x])
            if (f->cap[x] > 0 && f->level[f->to[x]] < 0) {
                f->level[f->to[x]] = f->level[a] + 1;
                f->queue[qt++] = f->to[x];
            }
    }
    return f->level[t] >= 0;
}

static int64_t orc_flow_dfs(orc_flow *f, int a, int t, int64_t pushed)
{
    if (a == t)
        return pushed;
    for (; f->it[a] >= 0; f->it[a] = f->nxt[f->it[a]]) {
        int x = f->it[a];
        int b = f->to[x];
        if (f->cap[x] <= 0 || f->level[b] != f->level[a] + 1)
            continue;
        int64_t got = orc_flow_dfs(f, b, t, pushed < f->cap[x] ? pushed : f->cap[x]);
        if (got > 0) {
            f->cap[x] -= got;
            f->cap[x ^ 1] += got;
            return got;
        }
    }
    return 0;
}

static int64_t orc_maxflow(orc_flow *f, int s, int t)
{
    int64_t total = 0;
    while (orc_flow_bfs(f, s, t)) {
        for (int i = 0; i < f->n; ++i)
            f->it[i] = f->head[i];
        int64_t got;
        while ((got = orc_flow_dfs(f, s, t, INT64_MAX)) > 0)
            total += got;
    }
    return total;
}

int64_t orc_split_optimum(const int32_t *cnt, int G, int E, const uint8_t *holds,
                          int n_edges, const int32_t *edge_u, const int32_t *edge_v,
                          const int32_t *edge_e)
{
    if (G <= 0 || E <= 0 || E % G != 0 || n_edges < 0)
        return -ORC_EINVAL;
    int32_t *rep_cnt = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *rep_ptr = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *rep_edge = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_edges + 1));
    int32_t *tok = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_edges + 1));
    int64_t *R = (int64_t *)malloc(sizeof(int64_t) * (size_t)E);
    int64_t *fixed = (int64_t *)malloc(sizeof(int64_t) * (size_t)G);
    int64_t result = -ORC_EINVAL;
    if (!rep_cnt || !rep_ptr || !rep_edge || !tok || !R || !fixed)
        goto done;
    if (orc_edges_by_expert(G, E, holds, n_edges, edge_u, edge_v, edge_e,
                            rep_cnt, rep_ptr, rep_edge) != ORC_OK) {
        result = -ORC_EDATA;
        goto done;
    }
    orc_split_start(cnt, G, E, holds, rep_cnt, rep_ptr, rep_edge, R, fixed, tok);
    {
        int64_t total = 0, need = 0, lo = 0, hi = 0;
        for (int i = 0; i < G; ++i) {
            total += fixed[i];
            if (fixed[i] > lo)
                lo = fixed[i];
        }
        for (int i = 0; i < n_edges; ++i) {
            total += tok[i];
            need += tok[i];
        }
        hi = total;
        /* smallest z in [lo, hi] that is feasible; hi is always feasible */
        int n = n_edges + G + 2, src = n_edges + G, snk = n_edges + G + 1;
        while (lo < hi) {
            int64_t z = lo + (hi - lo) / 2;
            orc_flow f;
            if (orc_flow_init(&f, n, 3 * n_edges + G + 1) != 0) {
                orc_flow_free(&f);
                result = -ORC_EINVAL;
                goto done;
            }
            for (int i = 0; i < n_edges; ++i) {
                orc_flow_add(&f, src, i, tok[i]);
                orc_flow_add(&f, i, n_edges + edge_u[i], tok[i]);
                orc_flow_add(&f, i, n_edges + edge_v[i], tok[i]);
            }
            for (int r = 0; r < G; ++r)
                orc_flow_add(&f, n_edges + r, snk, z - fixed[r]);
            int64_t got = orc_maxflow(&f, src, snk);
            orc_flow_free(&f);
            if (got == need)
                hi = z;
            else
                lo = z + 1;
        }
        result = lo;
    }
done:
    free(rep_cnt); free(rep_ptr); free(rep_edge); free(tok); free(R); free(fixed);
    return result;
}


/* ------------------------------------------------------------------------
 * Budgeted pairwise expert-swap planning (FreeBalance sec. 3.3, eq. 6-10;
 * Algorithm 1, the loop over beneficial swaps).
 *
 * Expert workloads: nhat[e] = sum_g cnt[g, e] (the predicted counts).
 * Rank loads under the placement pi: L[r] = sum_{e: pi[e] = r} nhat[e].
 * Exchanging expert a on rank u with expert b on rank v changes only
 *   L'[u] = L[u] - nhat[a] + nhat[b],   L'[v] = L[v] - nhat[b] + nhat[a]   (eq. 6-7).
 * Objective Phi(L) = max_r L[r] + gamma * sum_r (L[r] - Lbar)^2 (eq. 8);
 * benefit Delta = Phi(L) - Phi(L').  Lbar does not change under a swap, so
 * the change of the squared term is the integer
 *   (L[u]^2 + L[v]^2) - (L'[u]^2 + L'[v]^2)
 * and Delta = (max L - max L') + gamma * that, evaluated in double as one
 * product then one sum (reading: the pages fix no precision).
 * Cost of a swap C = alpha + (S(a) + S(b)) / beta with S(e) = expert_bytes
 * for every expert (eq. 9); budgets (eq. 10 gives their value): every rank
 * may spend at most `budget`, every rank pair at most `link_budget`.
 * Loop (Algorithm 1 with the frontier of sec. 3.3):
 *   u = most-loaded rank, v = least-loaded rank (lowest id on ties);
 *   stop when L[u] - L[v] <= tau;
 *   candidates: a on u, b on v, neither moved yet in this plan, Delta > 0,
 *   C within the residual budgets of u, v and the pair (u, v);
 *   take the largest Delta / C (Delta alone when C = 0); ties by (u, v,
 *   a, b) ascending (u, v are fixed here, so by a then b);
 *   no candidate: stop; else swap, update loads and budgets, repeat.
 * Outputs: pi_out[E], swaps[4 * n] (u, v, a, b) in acceptance order, the
 * swap count, final loads[G].  pi_in NULL = the even placement e / (E/G).
 * ------------------------------------------------------------------------ */
int orc_plan_swaps(const int32_t *cnt, const int32_t *pi_in, int G, int E, double gamma, double tau,
                   double alpha, double beta, double expert_bytes, double budget, double link_budget,
                   int32_t *pi_out, int32_t *swaps, int32_t *n_swaps, int64_t *loads)
{
    if (G < 1 || E < 1 || E % G != 0 || !cnt || !pi_out || !swaps || !n_swaps || !loads || !(beta > 0.0) ||
        !(gamma >= 0.0) || !(alpha >= 0.0) || !(expert_bytes >= 0.0) || !(tau >= 0.0) || !(budget >= 0.0) ||
        !(link_budget >= 0.0))
        return 1;
    int64_t *nhat = calloc((size_t)E, sizeof(int64_t));
    double *res_rank = calloc((size_t)G, sizeof(double));
    double *res_link = calloc((size_t)G * G, sizeof(double));
    uint8_t *moved = calloc((size_t)E, 1);
    if (!nhat || !res_rank || !res_link || !moved) {
        free(nhat); free(res_rank); free(res_link); free(moved);
        return 1;
    }
    for (int g = 0; g < G; ++g)
        for (int e = 0; e < E; ++e) nhat[e] += cnt[(int64_t)g * E + e];
    for (int e = 0; e < E; ++e) {
        const int r = pi_in ? pi_in[e] : e / (E / G);
        if (r < 0 || r >= G) {
            free(nhat); free(res_rank); free(res_link); free(moved);
            return 3;
        }
        pi_out[e] = r;
    }
    for (int r = 0; r < G; ++r) loads[r] = 0;
    for (int e = 0; e < E; ++e) loads[pi_out[e]] += nhat[e];
    for (int r = 0; r < G; ++r) res_rank[r] = budget;
    for (int i = 0; i < G * G; ++i) res_link[i] = link_budget;
    const double cost = alpha + (expert_bytes + expert_bytes) / beta;

    int n = 0;
    for (;;) {
        int u = 0, v = 0;
        for (int r = 1; r < G; ++r) {
            if (loads[r] > loads[u]) u = r;
            if (loads[r] < loads[v]) v = r;
        }
        if ((double)(loads[u] - loads[v]) <= tau) break;
        /* the largest load over the ranks the swap leaves alone */
        int64_t rest = INT64_MIN;
        for (int r = 0; r < G; ++r)
            if (r != u && r != v && loads[r] > rest) rest = loads[r];
        int best_a = -1, best_b = -1;
        double best_ratio = 0.0;
        const int feasible = res_rank[u] >= cost && res_rank[v] >= cost && res_link[u * G + v] >= cost;
        for (int a = 0; a < E && feasible; ++a) {
            if (pi_out[a] != u || moved[a]) continue;
            for (int b = 0; b < E; ++b) {
                if (pi_out[b] != v || moved[b]) continue;
                const int64_t lu = loads[u] - nhat[a] + nhat[b];
                const int64_t lv = loads[v] - nhat[b] + nhat[a];
                int64_t mx = lu > lv ? lu : lv;
                if (rest > mx) mx = rest;
                const int64_t dsq = (loads[u] * loads[u] + loads[v] * loads[v]) - (lu * lu + lv * lv);
                const double prod = gamma * (double)dsq;
                const double delta = (double)(loads[u] - mx) + prod;
                if (!(delta > 0.0)) continue;
                /* a free swap (cost 0) ranks by its benefit alone */
                const double ratio = cost > 0.0 ? delta / cost : delta;
                /* a ascending, then b ascending: a strict '>' keeps the first */
                if (best_a < 0 || ratio > best_ratio) {
                    best_a = a;
                    best_b = b;
                    best_ratio = ratio;
                }
            }
        }
        if (best_a < 0) break;
        const int a = best_a, b = best_b;
        pi_out[a] = v;
        pi_out[b] = u;
        moved[a] = moved[b] = 1;
        loads[u] = loads[u] - nhat[a] + nhat[b];
        loads[v] = loads[v] - nhat[b] + nhat[a];
        res_rank[u] -= cost;
        res_rank[v] -= cost;
        res_link[u * G + v] -= cost;
        res_link[v * G + u] -= cost;
        swaps[4 * n + 0] = u;
        swaps[4 * n + 1] = v;
        swaps[4 * n + 2] = a;
        swaps[4 * n + 3] = b;
        ++n;
    }
    *n_swaps = n;
    free(nhat); free(res_rank); free(res_link); free(moved);
    return 0;
}


/* ------------------------------------------------------------------------
 * Split variants (Relief, Ablation Results, Table III; The Relief Algorithm,
 * key properties: all-integer Q11.20).  Same edges, schedule and starting
 * point as orc_split (remote mass partitioned equally over a replicated
 * expert's edges, all of it at home).  Readings of the variants, which the
 * pages name without spelling out:
 *   0 RELIEF      the reference (orc_split).
 *   1 NO_REVERSE  Relief without the reverse move: a transfer only moves
 *                 tokens from home to the replica (limit = 0 when the
 *                 replica is the heavier end).
 *   2 JACOBI      snapshot loads, damped: every transfer of a pass reads the
 *                 loads of the pass start and moves |gap| >> 2 (a quarter in
 *                 place of a half), capped as in Relief; all moves of the
 *                 pass are applied together.
 *   3 HASH        the load-oblivious split of a hash router: a replicated
 *                 expert's remote tokens are divided equally over its holders
 *                 (home first, then replicas by rank; remainders to the
 *                 first holders).  No passes.
 *   4 WATER       water-filling relaxation: each pass visits the replicated
 *                 experts in ascending id; an expert's remote tokens are
 *                 taken off its holders and poured back from the lowest load
 *                 up (integer levels; the tokens left over at the last level
 *                 go to the holders at that level in holder order), a
 *                 replica never receiving more than its edge's tokens.
 *   5 PROPORTIONAL each pass, each replicated expert (ascending id) divides
 *                 its remote tokens over its holders in proportion to
 *                 (max base load - base load + 1) (largest remainders, ties
 *                 in holder order); a replica's excess over its edge's tokens
 *                 stays at home.
 *   6 FP32        Relief in single precision: loads and masses in fp32, the
 *                 gap halved exactly (no truncation); at the end every mass
 *                 is rounded to the nearest token (ties to even) and the
 *                 loads recomputed.
 *   7 Q1120       Relief in the engine's Q11.20 fixed point: quantities in
 *                 units of 2^-f tokens, f = 20 - s with s the smallest shift
 *                 that keeps the total load below 2^11 (11 integer bits);
 *                 truncating halves at that resolution; at the end every mass
 *                 is rounded to the nearest token (ties up) and the loads
 *                 recomputed.
 * Passes end early after a pass that changed nothing (variants 0-2, 4-7).
 * ------------------------------------------------------------------------ */
enum { ORC_SV_RELIEF = 0, ORC_SV_NO_REVERSE, ORC_SV_JACOBI, ORC_SV_HASH, ORC_SV_WATER, ORC_SV_PROPORTIONAL,
       ORC_SV_FP32, ORC_SV_Q1120, ORC_SV_COUNT };

/* Integer water-filling of R tokens over n holders with base loads B and
 * capacities cap: the largest level lam with sum min(cap, max(0, lam - B)) <= R,
 * then one more token to each holder still below its cap at that level, in
 * holder order, until R is used up. */
static void orc_water_fill(int n, const int64_t *B, const int64_t *cap, int64_t R, int64_t *a)
{
    int64_t lo = B[0], hi = B[0];
    for (int h = 1; h < n; ++h) {
        if (B[h] < lo) lo = B[h];
        if (B[h] > hi) hi = B[h];
    }
    hi += R + 1;
    /* f(lam) is non-decreasing; find the largest lam in [lo, hi] with f <= R */
    while (lo < hi) {
        int64_t mid = lo + (hi - lo + 1) / 2, f = 0;
        for (int h = 0; h < n; ++h) {
            int64_t x = mid - B[h];
            if (x < 0) x = 0;
            if (x > cap[h]) x = cap[h];
            f += x;
        }
        if (f <= R) lo = mid; else hi = mid - 1;
    }
    int64_t used = 0;
    for (int h = 0; h < n; ++h) {
        int64_t x = lo - B[h];
        if (x < 0) x = 0;
        if (x > cap[h]) x = cap[h];
        a[h] = x;
        used += x;
    }
    for (int h = 0; h < n && used < R; ++h)
        if (B[h] + a[h] <= lo && a[h] < cap[h]) { a[h] += 1; used += 1; }
}

int orc_split_variant(const int32_t *cnt, int G, int E, const uint8_t *holds, int n_edges, const int32_t *edge_u,
                      const int32_t *edge_v, const int32_t *edge_e, int n_rounds, const int32_t *round_ptr,
                      int passes, int variant, int32_t *tok, int32_t *mass, int64_t *loads, int32_t *passes_run)
{
    if (variant < 0 || variant >= ORC_SV_COUNT)
        return ORC_EINVAL;
    if (variant == ORC_SV_RELIEF)
        return orc_split(cnt, G, E, holds, n_edges, edge_u, edge_v, edge_e, n_rounds, round_ptr, passes, tok, mass,
                         loads, passes_run);
    if (G <= 0 || E <= 0 || E % G != 0 || n_edges < 0 || n_rounds < 0 || passes < 0)
        return ORC_EINVAL;
    if (round_ptr[0] != 0 || round_ptr[n_rounds] != n_edges)
        return ORC_EDATA;
    int32_t *rep_cnt = malloc(sizeof(int32_t) * (size_t)E);
    int32_t *rep_ptr = malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *rep_edge = malloc(sizeof(int32_t) * (size_t)(n_edges + 1));
    int64_t *R = malloc(sizeof(int64_t) * (size_t)E);
    int64_t *fixed = malloc(sizeof(int64_t) * (size_t)G);
    int64_t *snap = malloc(sizeof(int64_t) * (size_t)G);
    int64_t *B = malloc(sizeof(int64_t) * (size_t)(G + 1));
    int64_t *cap = malloc(sizeof(int64_t) * (size_t)(G + 1));
    int64_t *a = malloc(sizeof(int64_t) * (size_t)(G + 1));
    int64_t *wt = malloc(sizeof(int64_t) * (size_t)(G + 1));
    int64_t *rm = malloc(sizeof(int64_t) * (size_t)(G + 1));
    float *Lf = malloc(sizeof(float) * (size_t)G);
    float *mf = malloc(sizeof(float) * (size_t)(n_edges + 1));
    int64_t *Lq = malloc(sizeof(int64_t) * (size_t)G);
    int64_t *mq = malloc(sizeof(int64_t) * (size_t)(n_edges + 1));
    int rc = ORC_OK;
    if (!rep_cnt || !rep_ptr || !rep_edge || !R || !fixed || !snap || !B || !cap || !a || !wt || !rm || !Lf ||
        !mf || !Lq || !mq) {
        rc = ORC_EINVAL;
        goto done;
    }
    for (int r = 0; r < n_rounds; ++r) {
        if (round_ptr[r + 1] < round_ptr[r]) { rc = ORC_EDATA; goto done; }
        for (int i = round_ptr[r]; i < round_ptr[r + 1]; ++i)
            for (int i2 = round_ptr[r]; i2 < i; ++i2)
                if (edge_u[i] == edge_u[i2] || edge_u[i] == edge_v[i2] || edge_v[i] == edge_u[i2] ||
                    edge_v[i] == edge_v[i2]) { rc = ORC_EDATA; goto done; }
    }
    rc = orc_edges_by_expert(G, E, holds, n_edges, edge_u, edge_v, edge_e, rep_cnt, rep_ptr, rep_edge);
    if (rc != ORC_OK)
        goto done;
    orc_split_start(cnt, G, E, holds, rep_cnt, rep_ptr, rep_edge, R, fixed, tok);
    for (int i = 0; i < G; ++i)
        loads[i] = fixed[i];
    for (int i = 0; i < n_edges; ++i) {
        mass[i] = tok[i];
        loads[edge_u[i]] += tok[i];
    }
    *passes_run = 0;

    if (variant == ORC_SV_NO_REVERSE || variant == ORC_SV_JACOBI) {
        for (int p = 1; p <= passes; ++p) {
            int moved = 0;
            if (variant == ORC_SV_JACOBI)
                for (int i = 0; i < G; ++i) snap[i] = loads[i];
            for (int r = 0; r < n_rounds; ++r)
                for (int i = round_ptr[r]; i < round_ptr[r + 1]; ++i) {
                    const int u = edge_u[i], v = edge_v[i];
                    const int64_t gap = variant == ORC_SV_JACOBI ? snap[u] - snap[v] : loads[u] - loads[v];
                    int64_t delta = (gap < 0 ? -gap : gap) >> (variant == ORC_SV_JACOBI ? 2 : 1);
                    int64_t limit = gap > 0 ? (int64_t)mass[i]
                                            : (variant == ORC_SV_NO_REVERSE ? 0 : (int64_t)(tok[i] - mass[i]));
                    if (delta > limit) delta = limit;
                    if (delta > 0) {
                        const int64_t sd = gap > 0 ? delta : -delta;
                        loads[u] -= sd;
                        loads[v] += sd;
                        mass[i] -= (int32_t)sd;
                        moved = 1;
                    }
                }
            *passes_run = p;
            if (!moved) break;
        }
    } else if (variant == ORC_SV_HASH) {
        for (int e = 0; e < E; ++e) {
            const int m = rep_cnt[e];
            if (m == 0) continue;
            const int64_t q = R[e] / (m + 1), rem = R[e] % (m + 1);
            const int home = e / (E / G);
            for (int j = 0; j < m; ++j) {
                const int i = rep_edge[rep_ptr[e] + j];
                int64_t share = q + (j + 1 < rem ? 1 : 0);   /* holder j + 1; holder 0 is home */
                if (share > tok[i]) share = tok[i];
                mass[i] = (int32_t)(tok[i] - share);
                loads[home] -= share;
                loads[edge_v[i]] += share;
            }
        }
    } else if (variant == ORC_SV_WATER || variant == ORC_SV_PROPORTIONAL) {
        for (int p = 1; p <= passes; ++p) {
            int changed = 0;
            for (int e = 0; e < E; ++e) {
                const int m = rep_cnt[e];
                if (m == 0) continue;
                const int home = e / (E / G);
                /* holders: 0 = home, j + 1 = replica of edge j; base loads without e's remote tokens */
                int64_t at_home = 0;
                for (int j = 0; j < m; ++j) at_home += mass[rep_edge[rep_ptr[e] + j]];
                B[0] = loads[home] - at_home;
                cap[0] = R[e];
                for (int j = 0; j < m; ++j) {
                    const int i = rep_edge[rep_ptr[e] + j];
                    B[j + 1] = loads[edge_v[i]] - (tok[i] - mass[i]);
                    cap[j + 1] = tok[i];
                }
                const int n = m + 1;
                if (variant == ORC_SV_WATER) {
                    orc_water_fill(n, B, cap, R[e], a);
                } else {
                    int64_t M = B[0], W = 0, used = 0;
                    for (int h = 1; h < n; ++h) if (B[h] > M) M = B[h];
                    for (int h = 0; h < n; ++h) { wt[h] = M - B[h] + 1; W += wt[h]; }
                    for (int h = 0; h < n; ++h) {
                        a[h] = (R[e] * wt[h]) / W;
                        rm[h] = (R[e] * wt[h]) % W;
                        used += a[h];
                    }
                    /* largest remainders, ties in holder order */
                    while (used < R[e]) {
                        int best = 0;
                        for (int h = 1; h < n; ++h) if (rm[h] > rm[best]) best = h;
                        a[best] += 1;
                        rm[best] = -1;
                        used += 1;
                    }
                    for (int h = 1; h < n; ++h)
                        if (a[h] > cap[h]) { a[0] += a[h] - cap[h]; a[h] = cap[h]; }
                }
                loads[home] = B[0] + a[0];
                for (int j = 0; j < m; ++j) {
                    const int i = rep_edge[rep_ptr[e] + j];
                    const int32_t nm = (int32_t)(tok[i] - a[j + 1]);
                    if (nm != mass[i]) changed = 1;
                    mass[i] = nm;
                    loads[edge_v[i]] = B[j + 1] + a[j + 1];
                }
            }
            *passes_run = p;
            if (!changed) break;
        }
    } else if (variant == ORC_SV_FP32) {
        for (int i = 0; i < G; ++i) Lf[i] = (float)fixed[i];
        for (int i = 0; i < n_edges; ++i) {
            mf[i] = (float)tok[i];
            Lf[edge_u[i]] += (float)tok[i];   /* in edge order, one rounded sum at a time */
        }
        for (int p = 1; p <= passes; ++p) {
            int moved = 0;
            for (int r = 0; r < n_rounds; ++r)
                for (int i = round_ptr[r]; i < round_ptr[r + 1]; ++i) {
                    const int u = edge_u[i], v = edge_v[i];
                    const float gap = Lf[u] - Lf[v];
                    float delta = (gap < 0.0f ? -gap : gap) * 0.5f;
                    const float limit = gap > 0.0f ? mf[i] : (float)tok[i] - mf[i];
                    if (delta > limit) delta = limit;
                    if (delta > 0.0f) {
                        const float sd = gap > 0.0f ? delta : -delta;
                        Lf[u] -= sd;
                        Lf[v] += sd;
                        mf[i] -= sd;
                        moved = 1;
                    }
                }
            *passes_run = p;
            if (!moved) break;
        }
        for (int i = 0; i < G; ++i) loads[i] = fixed[i];
        for (int i = 0; i < n_edges; ++i) {
            float x = rintf(mf[i]);   /* nearest, ties to even (default rounding mode) */
            if (x < 0.0f) x = 0.0f;
            if (x > (float)tok[i]) x = (float)tok[i];
            mass[i] = (int32_t)x;
            loads[edge_u[i]] += mass[i];
            loads[edge_v[i]] += tok[i] - mass[i];
        }
    } else { /* ORC_SV_Q1120 */
        int64_t total = 0;
        for (int i = 0; i < G; ++i) total += loads[i];
        int s = 0;
        while ((total >> s) >= 2048) ++s;
        const int f = 20 - s;   /* fractional bits at this scale (total < 2^31 so s <= 20) */
        for (int i = 0; i < G; ++i) Lq[i] = loads[i] << f;
        for (int i = 0; i < n_edges; ++i) mq[i] = (int64_t)tok[i] << f;
        for (int p = 1; p <= passes; ++p) {
            int moved = 0;
            for (int r = 0; r < n_rounds; ++r)
                for (int i = round_ptr[r]; i < round_ptr[r + 1]; ++i) {
                    const int u = edge_u[i], v = edge_v[i];
                    const int64_t gap = Lq[u] - Lq[v];
                    int64_t delta = (gap < 0 ? -gap : gap) >> 1;   /* truncating halve at 2^-f */
                    const int64_t limit = gap > 0 ? mq[i] : ((int64_t)tok[i] << f) - mq[i];
                    if (delta > limit) delta = limit;
                    if (delta > 0) {
                        const int64_t sd = gap > 0 ? delta : -delta;
                        Lq[u] -= sd;
                        Lq[v] += sd;
                        mq[i] -= sd;
                        moved = 1;
                    }
                }
            *passes_run = p;
            if (!moved) break;
        }
        for (int i = 0; i < G; ++i) loads[i] = fixed[i];
        for (int i = 0; i < n_edges; ++i) {
            int64_t x = f > 0 ? (mq[i] + ((int64_t)1 << (f - 1))) >> f : mq[i];
            if (x < 0) x = 0;
            if (x > tok[i]) x = tok[i];
            mass[i] = (int32_t)x;
            loads[edge_u[i]] += mass[i];
            loads[edge_v[i]] += tok[i] - mass[i];
        }
    }
done:
    free(rep_cnt); free(rep_ptr); free(rep_edge); free(R); free(fixed); free(snap); free(B); free(cap); free(a);
    free(wt); free(rm); free(Lf); free(mf); free(Lq); free(mq);
    return rc;
}
