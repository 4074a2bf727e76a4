// Step 4: the per-step split (Relief, Methodology, Algorithm 1; The Per-Step
// Optimum Problem for the edge/weight structure).
//
// One CTA per problem.  Everything the split reads (counts, replica edges,
// round schedule, per-expert edge lists) is first staged into shared memory
// with coalesced loads, so no loop ever waits on L2.  Setup is one thread per
// expert (holder mask, remote mass, equal integer partition of the remote
// mass over the expert's edges) and one warp per rank (starting loads).
//
// The passes run in one warp with the load table in registers: lane j owns
// ranks j and j+32.  A round of the schedule is rank-disjoint, so every rank
// has at most one partner per round; a per-(round, rank) table built once
// names it.  Both owners of a transfer fetch the other's load with one
// shuffle and compute the same delta from the same (L[u], L[v], tok, mass),
// so a round costs a shuffle and a few integer operations, with no shared
// memory round trip on the dependency chain.  Each side keeps its own copy
// of the edge's mass, so no two lanes write the same word.  A pass that moves
// nothing is a fixpoint, so the loop stops there with identical results.
// Schedules too long for the table fall back to one lane per transfer with
// the loads in shared memory and __syncwarp between rounds.
#pragma once
#include "common.cuh"
#include "maskbits.cuh"
#include "plan.cuh"

namespace lb {
namespace split {

constexpr int THREADS = 512;

// Rounds the per-(round, rank) transfer table holds (at most 96 KB of it,
// 16 bytes per slot).
__host__ __device__ inline int table_rounds(int G, int N) {
    const int cap = (96 * 1024) / (16 * G);
    return G * N < cap ? G * N : cap;
}

// Shared-memory carve-up of one problem's split.
struct View {
    uint64_t *hold;     // [E]   holder ranks of each expert (bit g)
    int32_t *cnt;       // [G*E]
    int32_t *R;         // [E]   remote mass
    int32_t *rep_ptr;   // [E+1]
    int32_t *rep_edge;  // [GN]
    int32_t *eu, *ev, *ee;  // [GN] schedule order
    int32_t *er;        // [GN]  each edge's round
    int32_t *rptr;      // [GN+1]
    int32_t *tk, *mu, *mv;  // [GN] tok, mass (home side), mass (replica side)
    int4 *tab;          // [(RC+1)*G] (round, rank) slots: {code, tok, own-side mass, 0}; row nr idle
    int32_t *Ls;        // [64]
};

__host__ __device__ inline size_t smem_bytes(int G, int E, int N) {
    const size_t GN = static_cast<size_t>(G) * N;
    return static_cast<size_t>(E) * 8 + static_cast<size_t>(G) * E * 4 + static_cast<size_t>(E) * 4 +
           (static_cast<size_t>(E) + 1) * 4 + GN * 4 * 8 + (GN + 1) * 4 +
           (static_cast<size_t>(table_rounds(G, N)) + 1) * G * 16 + 64 * 4 + 64;
}

__device__ inline View carve(uint8_t *sm, int G, int E, int N) {
    const int GN = G * N;
    View v;
    v.hold = reinterpret_cast<uint64_t *>(sm);
    v.cnt = reinterpret_cast<int32_t *>(v.hold + E);
    v.R = v.cnt + G * E;
    v.rep_ptr = v.R + E;
    v.rep_edge = v.rep_ptr + E + 1;
    v.eu = v.rep_edge + GN;
    v.ev = v.eu + GN;
    v.ee = v.ev + GN;
    v.er = v.ee + GN;
    v.rptr = v.er + GN;
    v.tk = v.rptr + GN + 1;
    v.mu = v.tk + GN;
    v.mv = v.mu + GN;
    // 16-byte aligned table after the int32 arrays
    uintptr_t t = reinterpret_cast<uintptr_t>(v.mv + GN);
    t = (t + 15) & ~static_cast<uintptr_t>(15);
    v.tab = reinterpret_cast<int4 *>(t);
    v.Ls = reinterpret_cast<int32_t *>(v.tab + (table_rounds(G, N) + 1) * G);   // one idle row past the rounds
    return v;
}

// Slot (round r, rank x) of the table, seen from x: code = partner lane
// (bits 0-4), partner is rank lane+32 (bit 5), x is the transfer's home rank
// (bit 6), edge index (bits 8-23); tok; the mass on x's side (home side: the
// edge's mass; replica side: tok - mass).  An idle slot names x itself as
// partner with tok = mass = 0, so it computes a zero move with no branch.
__device__ __forceinline__ int slot_code(int partner, bool home, int edge) {
    return (partner & 31) | ((partner >> 5) << 5) | (home ? 64 : 0) | (edge << 8);
}

// Relief passes (Algorithm 1), symmetric form.  For a transfer between x and
// its partner y in a round: diff = L[x] - L[y]; the heavier side sends
// min(|diff| >> 1, mass on its side), the lighter side receives the same
// amount, limited by the partner's side (tok - own).  Both sides compute the
// same delta, so this is exactly gap/limit/update of Algorithm 1 seen from u
// and from v.  Lane j owns ranks j and (TWO) j+32; one full warp calls it.
template <bool TWO>
__device__ int relax_passes_regs(int G, int nr, int passes, const View &v) {
    const int lane = threadIdx.x & 31;
    const bool ha = lane < G, hb = TWO && lane + 32 < G;
    // lanes that own no rank read column 0 and compute throw-away moves:
    // nobody shuffles from them and they store nothing
    const int ca = ha ? lane : 0, cb = hb ? lane + 32 : 0;
    int La = ha ? v.Ls[lane] : 0;
    int Lb = hb ? v.Ls[lane + 32] : 0;
    int pr = 0;
    for (int p = 1; p <= passes; ++p) {
        // a move changes the loads at both its ends, so a pass moved something
        // exactly when some load differs from its value at the pass's start
        const int La0 = La, Lb0 = Lb;
        int4 A = v.tab[ca];
        int4 B = TWO ? v.tab[cb] : make_int4(0, 0, 0, 0);
        // four rounds per loop body: one round's table loads and mass stores
        // then sit in the shadow of the next rounds' shuffle chains (decode
        // shape, G = 64: the passes 15 % shorter; unrolling by 2 or 8 gained
        // nothing there; for G <= 32 four rounds measure the same as the
        // compiler's own unrolling, and forcing none was 15-25 % slower)
#pragma unroll 4
        for (int r = 0; r < nr; ++r) {
            const int4 a = A, b = B;
            // next round's slots (row nr is an idle row, so no bound check)
            A = v.tab[(r + 1) * G + ca];
            if (TWO) B = v.tab[(r + 1) * G + cb];
            // every shuffle before any update: a lane may own both ends
            const int pa = a.x & 31;
            int xa = __shfl_sync(kFull, La, pa);
            int xb = 0;
            if (TWO) {
                const int ya = __shfl_sync(kFull, Lb, pa);
                const int pb = b.x & 31;
                const int xl = __shfl_sync(kFull, La, pb);
                const int xh = __shfl_sync(kFull, Lb, pb);
                xa = (a.x & 32) ? ya : xa;
                xb = (b.x & 32) ? xh : xl;
            }
            {
                const int diff = La - xa;
                const int d = min((diff < 0 ? -diff : diff) >> 1, diff > 0 ? a.z : a.y - a.z);
                const int delta = diff > 0 ? -d : d;
                La += delta;
                if (ha) v.tab[r * G + lane].z = a.z + delta;   // unchanged value when delta is 0
            }
            if (TWO) {
                const int diff = Lb - xb;
                const int d = min((diff < 0 ? -diff : diff) >> 1, diff > 0 ? b.z : b.y - b.z);
                const int delta = diff > 0 ? -d : d;
                Lb += delta;
                if (hb) v.tab[r * G + lane + 32].z = b.z + delta;
            }
        }
        pr = p;
        if (!__any_sync(kFull, (ha && La != La0) || (hb && Lb != Lb0))) break;
    }
    if (ha) v.Ls[lane] = La;
    if (hb) v.Ls[lane + 32] = Lb;
    __syncwarp();
    return pr;
}

// Fallback for schedules longer than the table: one lane per transfer of a
// round, loads in shared memory.  Returns passes run; sets *bad on a round of
// more than 32 transfers (impossible for a valid plan with G <= 64).
__device__ int relax_passes_smem(int ne, int nr, int passes, const View &v, int *bad) {
    const int lane = threadIdx.x & 31;
    int pr = 0;
    for (int p = 1; p <= passes; ++p) {
        int moved = 0;
        for (int r = 0; r < nr; ++r) {
            const int a = v.rptr[r], n = v.rptr[r + 1] - a;
            if (n > 32 || n < 0 || a < 0 || a + n > ne) {
                if (lane == 0) *bad = 1;
                continue;
            }
            if (lane < n) {
                const int i = a + lane;
                const int u = v.eu[i], w = v.ev[i];
                const int Lu = v.Ls[u], Lw = v.Ls[w];
                const int gap = Lu - Lw;
                int d = (gap < 0 ? -gap : gap) >> 1;
                d = min(d, gap > 0 ? v.mu[i] : v.tk[i] - v.mu[i]);
                if (d > 0) {
                    const int sd = gap > 0 ? d : -d;
                    v.Ls[u] = Lu - sd;
                    v.Ls[w] = Lw + sd;
                    v.mu[i] -= sd;
                    moved = 1;
                }
            }
            __syncwarp();
        }
        pr = p;
        if (!__any_sync(kFull, moved)) break;
    }
    return pr;
}

// The expert whose slice [rep_ptr[e], rep_ptr[e+1]) of the per-expert edge
// lists holds position j: the largest e < E with rep_ptr[e] <= j (binary
// search; every index stays in [0, E] whatever rep_ptr holds).
__device__ __forceinline__ int list_expert(const int32_t *rep_ptr, int E, int j) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rep_ptr[mid] <= j) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// The whole split of one problem by one CTA.  Inputs: the problem's counts
// (global) and plan blob (global).  Leaves tok in v.tk, mass in v.mu, loads in
// v.Ls, and returns passes run.  All threads of the CTA must call it.
__device__ int split_problem(const int32_t *__restrict__ cnt, const uint8_t *__restrict__ blob, int G, int E,
                             int N, int passes, const View &v, int &ne_out, int *bad) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int GN = G * N, Eg = E / G;
    const plan::Layout LY = plan::layout(G, E, N);
    const int32_t *hdr = reinterpret_cast<const int32_t *>(blob + LY.hdr);
    int ne = hdr[0], nr = hdr[1];
    if (ne < 0 || ne > GN || nr < 0 || nr > GN) {
        *bad = 1;
        ne = 0;
        nr = 0;
    }
    const int RC = table_rounds(G, N);
    const bool use_table = nr <= RC;
    LB_TICK(0);

    // ---- stage inputs (coalesced)
    stage_i32(v.cnt, cnt, G * E);
    {
        const int32_t *p_eu = reinterpret_cast<const int32_t *>(blob + LY.edge_u);
        const int32_t *p_ev = reinterpret_cast<const int32_t *>(blob + LY.edge_v);
        const int32_t *p_ee = reinterpret_cast<const int32_t *>(blob + LY.edge_e);
        const int32_t *p_rep_edge = reinterpret_cast<const int32_t *>(blob + LY.rep_edge);
        const int32_t *p_er = reinterpret_cast<const int32_t *>(blob + LY.edge_round);
        for (int i = tid; i < ne; i += blockDim.x) {
            v.er[i] = p_er[i];
            v.eu[i] = p_eu[i];
            v.ev[i] = p_ev[i];
            v.ee[i] = p_ee[i];
            v.rep_edge[i] = p_rep_edge[i];
            v.tk[i] = 0;
            v.mu[i] = 0;
            v.mv[i] = 0;
        }
        for (int r = tid; r < G; r += blockDim.x) v.Ls[r] = 0;
        const int32_t *p_rptr = reinterpret_cast<const int32_t *>(blob + LY.round_ptr);
        for (int r = tid; r <= nr; r += blockDim.x) v.rptr[r] = p_rptr[r];
        const int32_t *p_rep_ptr = reinterpret_cast<const int32_t *>(blob + LY.rep_ptr);
        for (int e = tid; e <= E; e += blockDim.x) v.rep_ptr[e] = p_rep_ptr[e];
        if (use_table)
            for (int x = tid; x < (nr + 1) * G; x += blockDim.x) {
                const int rank = x % G;
                v.tab[x] = make_int4(slot_code(rank, false, 0), 0, 0, 0);
            }
    }
    __syncthreads();
    LB_TICK(1);

    // ---- holders, remote mass, starting loads, equal partition.  Edge work
    // is spread over the CTA by position in the per-expert edge lists (a hot
    // expert can hold tens of replicas: one thread per expert walking its
    // list left the whole CTA waiting on that one thread).
    // (a) per expert: its home as first holder; an edge range that is not a
    //     valid slice of the list is flagged and treated as empty (R = -1
    //     marks it until (c)).
    for (int e = tid; e < E; e += blockDim.x) {
        const int a = v.rep_ptr[e], z = v.rep_ptr[e + 1];
        const bool ok = !(a < 0 || z > ne || z < a);
        if (!ok) *bad = 1;
        v.hold[e] = 1ull << (e / Eg);
        v.R[e] = ok ? 0 : -1;
    }
    __syncthreads();
    // (b) per list position: validate the edge and add its replica rank to
    //     the expert's holders
    const int npos = max(0, min(v.rep_ptr[E], ne));
    for (int j = tid; j < npos; j += blockDim.x) {
        const int e = list_expert(v.rep_ptr, E, j);
        if (v.R[e] < 0 || j < v.rep_ptr[e] || j >= v.rep_ptr[e + 1]) continue;
        const int i = v.rep_edge[j];
        if (i < 0 || i >= ne || v.ee[i] != e || v.eu[i] != e / Eg || v.ev[i] < 0 || v.ev[i] >= G) {
            *bad = 1;
            continue;
        }
        or_bit64(&v.hold[e], v.ev[i]);
    }
    __syncthreads();
    // (c) per expert: remote mass R (tokens of ranks that hold no copy); the
    //     home serves its own tokens of e and, at the start, all of R.  The
    //     replica holders left in the mask are claimed in (d).
    for (int e = tid; e < E; e += blockDim.x) {
        const int h = e / Eg;
        const uint64_t hm = v.hold[e];
        int R = 0;
        for (int g = 0; g < G; ++g)
            if (!((hm >> g) & 1ull)) R += v.cnt[g * E + e];
        atomicAdd(&v.Ls[h], v.cnt[h * E + e] + R);
        v.R[e] = R;
        v.hold[e] = hm & ~(1ull << h);
    }
    __syncthreads();
    // (d) per list position: the equal integer partition of R over the
    //     expert's edges (the first R mod m edges take one more), and the
    //     starting load of the edge's replica rank: its own tokens of e, added
    //     by whichever edge clears the rank's bit first (once per holder, as
    //     the mask counts it; integer sums, so the order is immaterial)
    for (int j = tid; j < npos; j += blockDim.x) {
        const int e = list_expert(v.rep_ptr, E, j);
        const int a = v.rep_ptr[e], z = v.rep_ptr[e + 1];
        if (j < a || j >= z || a < 0 || z > ne || z < a) continue;
        const int i = v.rep_edge[j];
        if (i < 0 || i >= ne) continue;
        const int m = z - a, R = v.R[e];
        const int t = R / m + (j - a < R % m ? 1 : 0);
        v.tk[i] = t;
        v.mu[i] = t;
        v.mv[i] = t;
        const int w = v.ev[i];
        if (v.ee[i] == e && v.eu[i] == e / Eg && w >= 0 && w < G) {
            if (clear_bit64(&v.hold[e], w)) atomicAdd(&v.Ls[w], v.cnt[w * E + e]);
        }
    }
    LB_TICK(7);
    __syncthreads();
    LB_TICK(2);

    // ---- the round table: one thread per edge, at the (round, rank) slots of
    // both its ends (the plan blob gives each edge's round)
    LB_TICK(5);
    if (use_table) {
        for (int i = tid; i < ne; i += blockDim.x) {
            const int r = v.er[i];
            const int u = v.eu[i], w = v.ev[i];
            if (r < 0 || r >= nr || i < v.rptr[r] || i >= v.rptr[r + 1]) {
                *bad = 1;
                continue;
            }
            if (u < 0 || u >= G || w < 0 || w >= G || u == w) continue;
            const int t = v.tk[i];
            v.tab[r * G + u] = make_int4(slot_code(w, true, i), t, t, 0);
            v.tab[r * G + w] = make_int4(slot_code(u, false, i), t, 0, 0);
        }
    }
    LB_TICK(8);
    __syncthreads();
    LB_TICK(3);

    // ---- passes: one warp
    __shared__ int pr_s;
    if (warp == 0) {
        int pr;
        if (use_table)
            pr = (G > 32) ? relax_passes_regs<true>(G, nr, passes, v) : relax_passes_regs<false>(G, nr, passes, v);
        else
            pr = relax_passes_smem(ne, nr, passes, v, bad);
        if (lane == 0) pr_s = pr;
        LB_TICK(6);
    }
    __syncthreads();
    if (use_table) {
        // the edge's mass is the mass on its home side
        for (int x = tid; x < nr * G; x += blockDim.x) {
            const int4 c = v.tab[x];
            if (c.x & 64) v.mu[(c.x >> 8) & 0xffff] = c.z;
        }
        __syncthreads();
    }
    LB_TICK(4);
    ne_out = ne;
    return pr_s;
}

__global__ void __launch_bounds__(THREADS)
    split_kernel(const int32_t *__restrict__ cnt_all, const uint8_t *__restrict__ plan_all, size_t stride, int G,
                 int E, int N, int passes, int32_t *__restrict__ tok_all, int32_t *__restrict__ mass_all,
                 int32_t *__restrict__ loads_all, int32_t *__restrict__ passes_run_all) {
    extern __shared__ __align__(16) uint8_t sm[];
    pdl_begin();
    __shared__ int bad;
    const int tid = threadIdx.x, b = blockIdx.x, GN = G * N;
    if (tid == 0) bad = 0;
    __syncthreads();
    const View v = carve(sm, G, E, N);
    int ne = 0;
    const int pr = split_problem(cnt_all + static_cast<int64_t>(b) * G * E, plan_all + static_cast<size_t>(b) * stride,
                                 G, E, N, passes, v, ne, &bad);
    int32_t *tok = tok_all + static_cast<int64_t>(b) * GN;
    int32_t *mass = mass_all + static_cast<int64_t>(b) * GN;
    for (int i = tid; i < GN; i += blockDim.x) {
        tok[i] = i < ne ? v.tk[i] : 0;
        mass[i] = i < ne ? v.mu[i] : 0;
    }
    for (int r = tid; r < G; r += blockDim.x) loads_all[static_cast<int64_t>(b) * G + r] = v.Ls[r];
    if (tid == 0) {
        passes_run_all[b] = pr;
        if (bad) flag(LB_DEV_BAD_PLAN);
    }
}

}  // namespace split
}  // namespace lb
