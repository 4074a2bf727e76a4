// The per-problem stages of the decision in one CTA: the replica plan
// (optional), the Relief split and the permutation tables, in series
// (Libra README, Key Ideas; Relief, Algorithm 1; FreeBalance sec. 2.2).
// Each of the three is latency-bound work for one CTA per problem; run as
// separate launches, each pays a kernel boundary and stages its inputs from
// global memory again.  Here the plan blob, the split and the tables are
// produced one after the other by the same block (global writes made
// before a block barrier are visible to the whole block), and the scatter
// follows as its own launch.  Bytes out are those of lb_plan_replicas,
// lb_split and lb_assign's first launch.
#pragma once

#include <algorithm>

#include "assign.cuh"
#include "common.cuh"
#include "plan.cuh"
#include "split.cuh"

namespace lb {
namespace decide {

constexpr int THREADS = 512;

// The fused form is used for count tables of fewer than 4096 keys (G * E).
// Measured on B200, one problem per launch, against separate launches:
// faster for OLMoE (G=8, E=64: 30.8 against 32.8 us for count + split +
// assign), Qwen3-235B (G=8, E=128: 61.9 against 63.8) and a G=64, E=256
// decode step of T=64 (50.8 against 55.3), slower for that decode step at
// T >= 1024, where the split runs many rounds (129 against 125 us at
// T=1024, 190.5 against 174 at T=4096).
inline bool fused_for(int G, int E) { return static_cast<long long>(G) * E < 4096; }

// Dynamic shared memory: the stages run in series over the same bytes.
__host__ __device__ inline size_t smem_bytes(int G, int E, int N, bool with_plan) {
    size_t m = split::smem_bytes(G, E, N);
    const size_t p = assign::prep_smem_bytes(G, E, N);
    if (p > m) m = p;
    if (with_plan && plan::smem_bytes(G, E, N) > m) m = plan::smem_bytes(G, E, N);
    return m;
}

// CTA b: problem b.  PLAN: the plan blob is written from cnt_pred first
// (else a.plan is an input).  Then the split of a.cnt over the blob (tok,
// mass, loads, passes_run) and the tables of the scatter (offs, workspace).
template <bool PLAN>
__global__ void __launch_bounds__(THREADS)
    decide_kernel(const int32_t *__restrict__ cnt_pred_all, int L, const assign::Args a, int passes,
                  int32_t *__restrict__ loads_all, int32_t *__restrict__ passes_run_all) {
    extern __shared__ __align__(16) uint8_t sm[];
    pdl_begin();
    // without the plan step the scatter that follows may start now: what it
    // reads before its own wait (the counts and the plan) is not written here
    if (!PLAN) assign::pdl_signal_dependents();
    __shared__ int bad;
    const int tid = threadIdx.x, b = blockIdx.x;
    const int G = a.G, E = a.E, N = a.N, GN = G * N;
    uint8_t *blob = const_cast<uint8_t *>(a.plan) + static_cast<size_t>(b) * a.plan_stride;
    if (PLAN) plan::plan_problem(cnt_pred_all + static_cast<int64_t>(b) * G * E, G, E, N, L, blob, sm);

    if (tid == 0) bad = 0;
    __syncthreads();
    const split::View v = split::carve(sm, G, E, N);
    int ne = 0;
    const int pr = split::split_problem(a.cnt + static_cast<int64_t>(b) * G * E, blob, G, E, N, passes, v, ne, &bad);
    int32_t *tok = const_cast<int32_t *>(a.tok) + static_cast<int64_t>(b) * GN;
    int32_t *mass = const_cast<int32_t *>(a.mass) + static_cast<int64_t>(b) * GN;
    for (int i = tid; i < GN; i += blockDim.x) {
        tok[i] = i < ne ? v.tk[i] : 0;
        mass[i] = i < ne ? v.mu[i] : 0;
    }
    for (int r = tid; r < G; r += blockDim.x) loads_all[static_cast<int64_t>(b) * G + r] = v.Ls[r];
    if (tid == 0) {
        passes_run_all[b] = pr;
        if (bad) flag(LB_DEV_BAD_PLAN);
    }
    __syncthreads();
    assign::prep_problem(a, b, sm);
}

}  // namespace decide
}  // namespace lb
