// Steps 2, 4 and 5 in one launch: per-rank counts, the Relief split and the
// destinations + stable permutation of one problem (FreeBalance sec. 3.2 eq.
// 5; Relief, Algorithm 1; Libra README, Key Ideas), the per-step decision on
// the actual ids.
//
// One thread-block cluster of C CTAs per problem.  The source blocks (one per
// logical rank) are divided among the CTAs: whole blocks when C <= G, or P =
// C/G row-aligned parts of one block when C > G.
//   1. every CTA counts the ids of its slice into shared memory;
//   -- cluster barrier --
//   2. CTA 0 sums the counts over distributed shared memory into cnt, runs
//      the split and the permutation tables (offsets, per-block bases,
//      replica segments) exactly as lb_split and lb_assign do;
//   -- cluster barrier (releases CTA 0's global writes to the cluster) --
//   3. every CTA scatters its slice; a part's per-expert start inside its
//      block is the sum of the earlier parts' counts, read over DSMEM;
//   -- cluster barrier (keeps every CTA's counts alive for the readers) --
// The results are the ones the three separate calls produce, bit for bit.
#pragma once
#include "assign.cuh"
#include "common.cuh"
#include "split.cuh"

namespace lb {
namespace solve {

constexpr int THREADS = 1024;   // the scatter maps one warp to one lane of its cross-warp scan

__host__ __device__ inline bool use_parts(int G, int C) { return C > G; }
__host__ __device__ inline int segs_per_cta(int G, int C) { return C > G ? 1 : G / C; }

__host__ __device__ inline size_t head_bytes(int G, int E, int C) {
    return ((static_cast<size_t>(segs_per_cta(G, C)) + 1) * E * 4 + 15) & ~static_cast<size_t>(15);
}

__host__ __device__ inline size_t smem_bytes(int G, int E, int N, int C) {
    size_t w = split::smem_bytes(G, E, N);
    const size_t p = assign::prep_smem_bytes(G, E, N), sc = assign::scatter_smem_bytes(G, E, N);
    w = w > p ? w : p;
    w = w > sc ? w : sc;
    return head_bytes(G, E, C) + w;
}

__global__ void __launch_bounds__(THREADS, 1)
    solve_kernel(const assign::Args a, int passes, int32_t *__restrict__ loads_out,
                 int32_t *__restrict__ passes_run_out) {
    extern __shared__ __align__(16) uint8_t sm[];
    pdl_begin();
    __shared__ int bad_ids, bad_plan;
    const int G = a.G, E = a.E, N = a.N, k = a.k, T = a.T, GN = G * N;
    const int tid = threadIdx.x;
    const int C = gridDim.x;
    const int crank = static_cast<int>(cluster_ctarank());
    const int b = blockIdx.y;
    const bool parts = use_parts(G, C);
    const int P = parts ? C / G : 1;
    const int nseg = segs_per_cta(G, C);
    const int Tg = T / G;
    int32_t *hist = reinterpret_cast<int32_t *>(sm);   // [nseg][E]
    int32_t *prefix = hist + nseg * E;                  // [E]
    uint8_t *work = sm + head_bytes(G, E, C);

    // slice sidx of this CTA: source block g, rows [r0, r1) of the block
    auto slice = [&](int sidx, int &g, int &r0, int &r1) {
        if (parts) {
            g = crank / P;
            const int q = crank - g * P;
            r0 = static_cast<int>(static_cast<int64_t>(Tg) * q / P);
            r1 = static_cast<int>(static_cast<int64_t>(Tg) * (q + 1) / P);
        } else {
            g = crank * nseg + sidx;
            r0 = 0;
            r1 = Tg;
        }
    };

    // ---- 1. count this CTA's slice
    if (tid == 0) {
        bad_ids = 0;
        bad_plan = 0;
    }
    for (int i = tid; i < nseg * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int32_t *ids = a.ids + static_cast<int64_t>(b) * T * k;
    for (int sidx = 0; sidx < nseg; ++sidx) {
        int g, r0, r1;
        slice(sidx, g, r0, r1);
        const int32_t *rows = ids + (static_cast<int64_t>(g) * Tg) * k;
        for (int r = r0 + tid; r < r1; r += blockDim.x) {
            const int32_t *row = rows + static_cast<int64_t>(r) * k;
            int v[LB_MAX_K];
#pragma unroll
            for (int j = 0; j < LB_MAX_K; ++j) v[j] = j < k ? __ldg(row + j) : -1;
#pragma unroll
            for (int j = 0; j < LB_MAX_K; ++j) {
                if (j >= k) break;
                bool ok = v[j] >= 0 && v[j] < E;
#pragma unroll
                for (int jj = 0; jj < j; ++jj) ok = ok && v[jj] != v[j];
                if (ok)
                    atomicAdd(&hist[sidx * E + v[j]], 1);
                else
                    bad_ids = 1;
            }
        }
    }
    __syncthreads();
    cluster_sync();

    // ---- 2. CTA 0: counts, split, permutation tables
    if (crank == 0) {
        int32_t *cnt = const_cast<int32_t *>(a.cnt) + static_cast<int64_t>(b) * G * E;
        const uint32_t hist_s = smem_u32(hist);
        for (int idx = tid; idx < G * E; idx += blockDim.x) {
            const int g = idx / E, e = idx - g * E;
            int sum = 0;
            if (parts) {
                for (int q = 0; q < P; ++q) sum += ld_cluster_i32(mapa_shared(hist_s + e * 4, g * P + q));
            } else {
                const int owner = g / nseg, sidx = g - owner * nseg;
                sum = ld_cluster_i32(mapa_shared(hist_s + (sidx * E + e) * 4, owner));
            }
            cnt[idx] = sum;
        }
        __syncthreads();
        const split::View v = split::carve(work, G, E, N);
        int ne = 0;
        const int pr = split::split_problem(cnt, a.plan + static_cast<size_t>(b) * a.plan_stride, G, E, N, passes, v,
                                            ne, &bad_plan);
        int32_t *tok = const_cast<int32_t *>(a.tok) + static_cast<int64_t>(b) * GN;
        int32_t *mass = const_cast<int32_t *>(a.mass) + static_cast<int64_t>(b) * GN;
        for (int i = tid; i < GN; i += blockDim.x) {
            tok[i] = i < ne ? v.tk[i] : 0;
            mass[i] = i < ne ? v.mu[i] : 0;
        }
        for (int r = tid; r < G; r += blockDim.x) loads_out[static_cast<int64_t>(b) * G + r] = v.Ls[r];
        if (tid == 0) passes_run_out[b] = pr;
        __syncthreads();
        assign::prep_problem(a, b, work);
    }
    cluster_sync();

    // ---- 3. scatter this CTA's slice
    const int nitems = Tg * k;
    __shared__ int bad_sc;
    if (tid == 0) bad_sc = 0;
    const assign::ScatterView sv = assign::scatter_carve(work, G, E, N);
    assign::scatter_setup(a, b, sv);
    if (!parts && nitems <= assign::WARP_BLOCK_MAX) {
        assign::scatter_blocks_warp_any(a, b, crank * nseg, (crank + 1) * nseg, sv, &bad_sc);
        __syncthreads();
    } else {
        for (int sidx = 0; sidx < nseg; ++sidx) {
            int g, r0, r1;
            slice(sidx, g, r0, r1);
            if (parts) {
                const int q = crank - g * P;
                const uint32_t hist_s = smem_u32(hist);
                for (int e = tid; e < E; e += blockDim.x) {
                    int acc = 0;
                    for (int qq = 0; qq < q; ++qq) acc += ld_cluster_i32(mapa_shared(hist_s + e * 4, g * P + qq));
                    prefix[e] = acc;
                }
                __syncthreads();
            }
            assign::scatter_block_cta_any(a, b, g, r0 * k, min(r1 * k, nitems), parts ? prefix : nullptr, sv,
                                          &bad_sc);
        }
    }
    if (tid == 0 && bad_sc) flag(LB_DEV_BAD_SPLIT);
    cluster_sync();
    if (tid == 0) {
        if (bad_ids) flag(LB_DEV_BAD_IDS);
        if (bad_plan) flag(LB_DEV_BAD_PLAN);
    }
}

}  // namespace solve
}  // namespace lb
