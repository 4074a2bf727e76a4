// Budgeted pairwise expert-swap planning (FreeBalance sec. 3.3 eq. 6-10,
// Algorithm 1): the alternative to replication planning, in which experts
// change owner in pairs and no replica is created.
//
// One CTA per problem.  All threads sum the predicted per-rank counts into
// expert workloads nhat[e] and build the placement; then warp 0 runs the
// greedy loop with every per-rank quantity in registers (lane r holds ranks r
// and r + 32: loads and residual rank budgets):
//   u = most-loaded rank, v = least-loaded rank (lowest id on ties), one
//     redux.sync each plus a ballot;
//   stop when L[u] - L[v] <= tau;
//   the unmoved experts on u and on v are compacted (ascending id) into two
//     shared-memory lists by ballots;
//   each lane scores candidate pairs (a from u's list, b from v's list):
//     L'[u] = L[u] - nhat[a] + nhat[b], L'[v] = L[v] - nhat[b] + nhat[a]
//     (eq. 6-7), Delta = (L[u] - max(L'[u], L'[v], max of the other ranks))
//     + gamma * ((L[u]^2 + L[v]^2) - (L'[u]^2 + L'[v]^2)) (eq. 8: the mean
//     does not move, so the squared term changes by that integer), in double
//     with one rounded product and one rounded sum; ratio = Delta / C
//     (Delta alone when C = 0);
//   a warp reduction keeps the largest ratio, ties to the smaller (a, b);
//   the swap is taken if Delta > 0 and C fits the residual budgets of u, v
//     and the pair (u, v); loads, budgets and the placement are updated.
// Every rank's loads fit int32 (the counts sum to T*k < 2^31); the squared
// terms are taken in int64.
#pragma once
#include "common.cuh"

namespace lb {
namespace swaps {

constexpr int THREADS = 256;

struct Params {
    const int32_t *cnt;     // [B, G, E] predicted counts
    const int32_t *pi_in;   // [B, E] or null (even placement)
    int G, E;
    double gamma, tau, cost, budget, link_budget;
    int32_t *pi_out;        // [B, E]
    int32_t *swaps;         // [B, max_swaps, 4]
    int32_t *n_swaps;       // [B]
    int32_t *loads;         // [B, G]
    int max_swaps;
};

__host__ __device__ inline size_t smem_bytes(int G, int E) {
    // nhat, pi, two candidate lists (int32 each), moved (bytes, padded), link budgets
    return static_cast<size_t>(E) * 4 * 4 + ((static_cast<size_t>(E) + 15) & ~static_cast<size_t>(15)) +
           static_cast<size_t>(G) * G * 8 + 64;
}

// Best candidate so far: larger ratio wins, equal ratios go to the smaller
// (a, b).  a < 0 = none.
struct Best {
    double ratio;
    int a, b;
};

__device__ __forceinline__ bool better(double r1, int a1, int b1, double r2, int a2, int b2) {
    if (a2 < 0) return a1 >= 0;
    if (a1 < 0) return false;
    if (r1 != r2) return r1 > r2;
    return a1 < a2 || (a1 == a2 && b1 < b2);
}

__global__ void __launch_bounds__(THREADS) swaps_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t sm[];
    pdl_begin();
    const int G = p.G, E = p.E, b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    double *res_link = reinterpret_cast<double *>(sm);
    int32_t *nhat = reinterpret_cast<int32_t *>(res_link + static_cast<size_t>(G) * G);
    int32_t *pi = nhat + E;
    int32_t *list_u = pi + E;
    int32_t *list_v = list_u + E;
    uint8_t *moved = reinterpret_cast<uint8_t *>(list_v + E);
    __shared__ int bad;
    if (tid == 0) bad = 0;
    __syncthreads();

    const int32_t *cnt = p.cnt + static_cast<int64_t>(b) * G * E;
    const int Eg = E / G;
    for (int e = tid; e < E; e += blockDim.x) {
        int s = 0;
        for (int g = 0; g < G; ++g) s += cnt[static_cast<int64_t>(g) * E + e];
        nhat[e] = s;
        int r = p.pi_in != nullptr ? p.pi_in[static_cast<int64_t>(b) * E + e] : e / Eg;
        if (r < 0 || r >= G) {
            bad = 1;
            r = e / Eg;
        }
        pi[e] = r;
        moved[e] = 0;
    }
    for (int i = tid; i < G * G; i += blockDim.x) res_link[i] = p.link_budget;
    __syncthreads();
    if (bad) {
        if (tid == 0) {
            p.n_swaps[b] = 0;
            flag(LB_DEV_BAD_PLAN);
        }
        return;
    }
    if (warp != 0) return;

    // ---- the greedy loop, warp 0; lane r holds ranks r and r + 32
    int L0 = 0, L1 = 0;   // loads of ranks lane, lane + 32
    for (int e = 0; e < E; ++e) {
        const int r = pi[e];
        if (r == lane) L0 += nhat[e];
        if (r == lane + 32) L1 += nhat[e];
    }
    const bool has0 = lane < G, has1 = lane + 32 < G;
    double R0 = p.budget, R1 = p.budget;   // residual rank budgets
    const double cost = p.cost;
    int n = 0;
    int32_t *sw = p.swaps + static_cast<int64_t>(b) * p.max_swaps * 4;
    for (;;) {
        // u = argmax (lowest id), v = argmin (lowest id)
        const int mx0 = has0 ? L0 : INT_MIN, mx1 = has1 ? L1 : INT_MIN;
        const int lmax = __reduce_max_sync(kFull, max(mx0, mx1));
        const unsigned bu0 = __ballot_sync(kFull, has0 && L0 == lmax), bu1 = __ballot_sync(kFull, has1 && L1 == lmax);
        const int u = bu0 ? __ffs(bu0) - 1 : 32 + __ffs(bu1) - 1;
        const int mn0 = has0 ? L0 : INT_MAX, mn1 = has1 ? L1 : INT_MAX;
        const int lmin = __reduce_min_sync(kFull, min(mn0, mn1));
        const unsigned bv0 = __ballot_sync(kFull, has0 && L0 == lmin), bv1 = __ballot_sync(kFull, has1 && L1 == lmin);
        const int v = bv0 ? __ffs(bv0) - 1 : 32 + __ffs(bv1) - 1;
        if (static_cast<double>(lmax - lmin) <= p.tau) break;
        // the largest load over the ranks the swap leaves alone
        const int o0 = (has0 && lane != u && lane != v) ? L0 : INT_MIN;
        const int o1 = (has1 && lane + 32 != u && lane + 32 != v) ? L1 : INT_MIN;
        const int rest = __reduce_max_sync(kFull, max(o0, o1));
        // residual budgets of u, v and the pair
        const double Ru = __shfl_sync(kFull, u < 32 ? R0 : R1, u & 31);
        const double Rv = __shfl_sync(kFull, v < 32 ? R0 : R1, v & 31);
        const double Ruv = res_link[u * G + v];
        if (!(Ru >= cost && Rv >= cost && Ruv >= cost)) break;   // no candidate can be feasible
        // unmoved experts of u and of v, ascending id
        int nu = 0, nv = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const bool ok = e < E && !moved[e];
            const int r = e < E ? pi[e] : -1;
            const unsigned mu = __ballot_sync(kFull, ok && r == u), mv = __ballot_sync(kFull, ok && r == v);
            if (ok && r == u) list_u[nu + __popc(mu & lanemask_lt())] = e;
            if (ok && r == v) list_v[nv + __popc(mv & lanemask_lt())] = e;
            nu += __popc(mu);
            nv += __popc(mv);
        }
        __syncwarp();
        const int Lu = lmax, Lv = lmin;
        const long long sq0 = static_cast<long long>(Lu) * Lu + static_cast<long long>(Lv) * Lv;
        Best best{0.0, -1, -1};
        for (int q = lane; q < nu * nv; q += 32) {
            const int ia = q / nv, ib = q - ia * nv;
            const int a = list_u[ia], bb = list_v[ib];
            const int lu = Lu - nhat[a] + nhat[bb], lv = Lv - nhat[bb] + nhat[a];
            const int mx = max(max(lu, lv), rest);
            const long long dsq = sq0 - (static_cast<long long>(lu) * lu + static_cast<long long>(lv) * lv);
            const double prod = __dmul_rn(p.gamma, static_cast<double>(dsq));
            const double delta = __dadd_rn(static_cast<double>(Lu - mx), prod);
            if (!(delta > 0.0)) continue;
            const double ratio = cost > 0.0 ? __ddiv_rn(delta, cost) : delta;
            if (better(ratio, a, bb, best.ratio, best.a, best.b)) best = Best{ratio, a, bb};
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const double r2 = __shfl_xor_sync(kFull, best.ratio, off);
            const int a2 = __shfl_xor_sync(kFull, best.a, off), b2 = __shfl_xor_sync(kFull, best.b, off);
            if (better(r2, a2, b2, best.ratio, best.a, best.b)) best = Best{r2, a2, b2};
        }
        if (best.a < 0 || n >= p.max_swaps) break;
        const int a = best.a, bb = best.b;
        const int x = nhat[a] - nhat[bb];
        __syncwarp();
        if (lane == 0) {
            pi[a] = v;
            pi[bb] = u;
            moved[a] = moved[bb] = 1;
            res_link[u * G + v] -= cost;
            res_link[v * G + u] -= cost;
            sw[4 * n + 0] = u;
            sw[4 * n + 1] = v;
            sw[4 * n + 2] = a;
            sw[4 * n + 3] = bb;
        }
        if (lane == (u & 31)) {
            if (u < 32) { L0 -= x; R0 -= cost; } else { L1 -= x; R1 -= cost; }
        }
        if (lane == (v & 31)) {
            if (v < 32) { L0 += x; R0 -= cost; } else { L1 += x; R1 -= cost; }
        }
        __syncwarp();
        ++n;
    }
    __syncwarp();
    for (int e = lane; e < E; e += 32) p.pi_out[static_cast<int64_t>(b) * E + e] = pi[e];
    int32_t *lo = p.loads + static_cast<int64_t>(b) * G;
    if (has0) lo[lane] = L0;
    if (has1) lo[lane + 32] = L1;
    if (lane == 0) p.n_swaps[b] = n;
}

}  // namespace swaps
}  // namespace lb
