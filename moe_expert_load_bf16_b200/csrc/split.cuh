// Step 4: the per-step split (Relief, Methodology, Algorithm 1; The Per-Step
// Optimum Problem for the edge/weight structure).
//
// One CTA per problem.  Setup is parallel (remote mass per expert, rank
// loads by warp reductions, equal integer partition of each replicated
// expert's remote mass over its edges).  The passes run in one warp: a round
// is rank-disjoint, so with G <= 64 it has at most 32 transfers, one per
// lane; the load table lives in shared memory, every transfer of a round
// reads and writes its two entries with no atomics, and __syncwarp commits
// the round so the next one reads what it wrote (Gauss-Seidel).  A pass that
// moves nothing is a fixpoint, so the loop stops there with identical
// results.
#pragma once
#include "common.cuh"
#include "plan.cuh"

namespace lb {
namespace split {

constexpr int THREADS = 256;

__host__ __device__ inline size_t smem_bytes(int G, int E, int N) {
    const size_t GN = static_cast<size_t>(G) * N;
    return static_cast<size_t>(E) * 8 + static_cast<size_t>(E) * 4 + GN * 4 * 4 + (GN + 1) * 4;
}

__global__ void __launch_bounds__(THREADS)
    split_kernel(const int32_t *__restrict__ cnt_all, const uint8_t *__restrict__ plan_all,
                 size_t stride, int G, int E, int N, int passes, int32_t *__restrict__ tok_all,
                 int32_t *__restrict__ mass_all, int32_t *__restrict__ loads_all,
                 int32_t *__restrict__ passes_run_all) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int GN = G * N;
    uint64_t *hold = reinterpret_cast<uint64_t *>(sm);
    int32_t *R = reinterpret_cast<int32_t *>(hold + E);
    int32_t *eu = R + E;
    int32_t *ev = eu + GN;
    int32_t *tk = ev + GN;
    int32_t *ms = tk + GN;
    int32_t *rptr = ms + GN;
    __shared__ int Ls[LB_MAX_G];
    __shared__ int bad;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
    const int b = blockIdx.x;
    const int32_t *cnt = cnt_all + static_cast<int64_t>(b) * G * E;
    const uint8_t *blob = plan_all + static_cast<size_t>(b) * stride;
    const plan::Layout LY = plan::layout(G, E, N);
    const int32_t *hdr = reinterpret_cast<const int32_t *>(blob + LY.hdr);
    const int32_t *p_eu = reinterpret_cast<const int32_t *>(blob + LY.edge_u);
    const int32_t *p_ev = reinterpret_cast<const int32_t *>(blob + LY.edge_v);
    const int32_t *p_ee = reinterpret_cast<const int32_t *>(blob + LY.edge_e);
    const int32_t *p_rptr = reinterpret_cast<const int32_t *>(blob + LY.round_ptr);
    const int32_t *p_rep_ptr = reinterpret_cast<const int32_t *>(blob + LY.rep_ptr);
    const int32_t *p_rep_edge = reinterpret_cast<const int32_t *>(blob + LY.rep_edge);
    int32_t *tok = tok_all + static_cast<int64_t>(b) * GN;
    int32_t *mass = mass_all + static_cast<int64_t>(b) * GN;
    const int Eg = E / G;

    int ne = hdr[0], nr = hdr[1];
    if (tid == 0) bad = 0;
    if (ne < 0 || ne > GN || nr < 0 || nr > GN) {
        if (tid == 0) flag(LB_DEV_BAD_PLAN);
        ne = 0;
        nr = 0;
    }
    for (int e = tid; e < E; e += blockDim.x) hold[e] = 1ull << (e / Eg);
    for (int i = tid; i < ne; i += blockDim.x) {
        eu[i] = p_eu[i];
        ev[i] = p_ev[i];
    }
    for (int r = tid; r <= nr; r += blockDim.x) rptr[r] = p_rptr[r];
    __syncthreads();
    for (int i = tid; i < ne; i += blockDim.x) {
        const int e = p_ee[i], v = ev[i];
        if (e < 0 || e >= E || v < 0 || v >= G || eu[i] != e / Eg) {
            bad = 1;
            eu[i] = 0;   // neutralise: a self-loop never moves anything
            ev[i] = 0;
            continue;
        }
        atomicOr(reinterpret_cast<unsigned long long *>(&hold[e]), 1ull << v);
    }
    for (int i = tid; i < ne; i += blockDim.x) {
        tk[i] = 0;
        ms[i] = 0;
    }
    __syncthreads();

    // remote mass per expert
    for (int e = tid; e < E; e += blockDim.x) {
        const uint64_t hm = hold[e];
        int s = 0;
        for (int g = 0; g < G; ++g)
            if (!((hm >> g) & 1ull)) s += cnt[g * E + e];
        R[e] = s;
    }
    __syncthreads();
    // starting loads: own tokens of held experts + remote mass of home experts
    for (int r = warp; r < G; r += nwarps) {
        int x = 0;
        for (int e = lane; e < E; e += 32) {
            if ((hold[e] >> r) & 1ull) x += cnt[r * E + e];
            if (e / Eg == r) x += R[e];
        }
        x = __reduce_add_sync(kFull, x);
        if (lane == 0) Ls[r] = x;
    }
    // equal integer partition over each expert's edges (ascending replica rank)
    for (int e = tid; e < E; e += blockDim.x) {
        const int a = p_rep_ptr[e], z = p_rep_ptr[e + 1];
        const int mcount = z - a;
        if (a < 0 || z > ne || mcount < 0) {
            bad = 1;
            continue;
        }
        if (mcount == 0) continue;
        const int q = R[e] / mcount, rem = R[e] % mcount;
        for (int j = 0; j < mcount; ++j) {
            const int i = p_rep_edge[a + j];
            if (i < 0 || i >= ne) {
                bad = 1;
                continue;
            }
            const int t = q + (j < rem ? 1 : 0);
            tk[i] = t;
            ms[i] = t;
        }
    }
    __syncthreads();

    // passes: one warp
    if (warp == 0) {
        int pr = 0;
        for (int p = 1; p <= passes; ++p) {
            int moved = 0;
            for (int r = 0; r < nr; ++r) {
                const int a = rptr[r], n = rptr[r + 1] - a;
                if (n > 32 || n < 0 || a < 0 || a + n > ne) {
                    if (lane == 0) bad = 1;
                    continue;
                }
                if (lane < n) {
                    const int i = a + lane;
                    const int u = eu[i], v = ev[i];
                    const int Lu = Ls[u], Lv = Ls[v];
                    const int gap = Lu - Lv;
                    int d = (gap < 0 ? -gap : gap) >> 1;
                    const int lim = gap > 0 ? ms[i] : tk[i] - ms[i];
                    d = min(d, lim);
                    if (d > 0) {
                        const int sd = gap > 0 ? d : -d;
                        Ls[u] = Lu - sd;
                        Ls[v] = Lv + sd;
                        ms[i] -= sd;
                        moved = 1;
                    }
                }
                __syncwarp();
            }
            pr = p;
            if (!__any_sync(kFull, moved)) break;
        }
        if (lane == 0) passes_run_all[b] = pr;
    }
    __syncthreads();
    for (int i = tid; i < GN; i += blockDim.x) {
        tok[i] = i < ne ? tk[i] : 0;
        mass[i] = i < ne ? ms[i] : 0;
    }
    for (int r = tid; r < G; r += blockDim.x) loads_all[static_cast<int64_t>(b) * G + r] = Ls[r];
    if (tid == 0 && bad) flag(LB_DEV_BAD_PLAN);
}

}  // namespace split
}  // namespace lb
