// Step 2: per-rank token->expert histograms (FreeBalance sec. 3.2 eq. 5 and
// Algorithm 1's aggregation step, per source rank as in Libra's phase 1).
//
// One CTA per (problem, source rank): it owns output row cnt[b,g,:], so it
// writes it with plain stores (no global atomics, no memset); or a cluster
// of CTAs per rank when the ranks alone underfill the GPU (below).  Rows of k ids
// stream in with 16-byte loads (thread per token row); the histogram lives in
// shared memory.  A row with an id outside [0,E) or a repeated id has that id
// skipped and LB_DEV_BAD_IDS raised.
#pragma once
#include "common.cuh"

namespace lb {
namespace count {

constexpr int THREADS = 512;

template <int K, bool VEC>
__device__ __forceinline__ void load_row(const int32_t *src, int k, int (&e)[K]) {
    if (VEC && K % 4 == 0 && k == K) {
        const int4 *s4 = reinterpret_cast<const int4 *>(src);
#pragma unroll
        for (int q = 0; q < K / 4; ++q) {
            const int4 x = __ldg(s4 + q);
            e[4 * q] = x.x;
            e[4 * q + 1] = x.y;
            e[4 * q + 2] = x.z;
            e[4 * q + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < K; ++j) e[j] = j < k ? __ldg(src + j) : -1;
    }
}

template <int K, bool VEC>
__global__ void __launch_bounds__(THREADS)
    count_kernel(const int32_t *__restrict__ ids, int T, int k, int E, int G,
                 int32_t *__restrict__ cnt) {
    extern __shared__ int hist[];
    pdl_begin();
    __shared__ int bad;
    const int g = blockIdx.x, b = blockIdx.y;
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    const int Tg = T / G;
    const int32_t *base = ids + (static_cast<int64_t>(b) * T + static_cast<int64_t>(g) * Tg) * k;
    for (int r = threadIdx.x; r < Tg; r += blockDim.x) {
        int e[K];
        load_row<K, VEC>(base + static_cast<int64_t>(r) * k, k, e);
#pragma unroll
        for (int j = 0; j < K; ++j) {
            if (j >= k) break;
            bool okj = e[j] >= 0 && e[j] < E;
#pragma unroll
            for (int jj = 0; jj < j; ++jj) okj = okj && (e[jj] != e[j]);
            if (okj)
                atomicAdd(&hist[e[j]], 1);
            else
                bad = 1;
        }
    }
    __syncthreads();
    int32_t *out = cnt + (static_cast<int64_t>(b) * G + g) * E;
    for (int e = threadIdx.x; e < E; e += blockDim.x) out[e] = hist[e];
    if (threadIdx.x == 0 && bad) flag(LB_DEV_BAD_IDS);
}

// The same rows over a cluster of S CTAs per (problem, source rank), for
// when one CTA per rank would leave most SMs idle (one problem: G CTAs).
// CTA c of the cluster counts rows [c R, (c+1) R) of the rank (R = Tg / S,
// rounded up) into its own shared-memory histogram; after a cluster barrier
// it sums experts [c E/S, (c+1) E/S) over the S histograms (distributed
// shared memory reads) and writes them; a second barrier keeps every
// histogram alive until all reads are done.  Same counts, same flags.
template <int K, bool VEC>
__global__ void __launch_bounds__(THREADS)
    count_kernel_cluster(const int32_t *__restrict__ ids, int T, int k, int E, int G, int S,
                         int32_t *__restrict__ cnt) {
    extern __shared__ int hist[];
    __shared__ int bad;
    const int c = static_cast<int>(cluster_ctarank());
    const int g = static_cast<int>(blockIdx.x) / S, b = blockIdx.y;
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    const int Tg = T / G, rps = (Tg + S - 1) / S;
    const int r0 = min(Tg, c * rps), r1 = min(Tg, r0 + rps);
    const int32_t *base = ids + (static_cast<int64_t>(b) * T + static_cast<int64_t>(g) * Tg) * k;
    for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
        int e[K];
        load_row<K, VEC>(base + static_cast<int64_t>(r) * k, k, e);
#pragma unroll
        for (int j = 0; j < K; ++j) {
            if (j >= k) break;
            bool okj = e[j] >= 0 && e[j] < E;
#pragma unroll
            for (int jj = 0; jj < j; ++jj) okj = okj && (e[jj] != e[j]);
            if (okj)
                atomicAdd(&hist[e[j]], 1);
            else
                bad = 1;
        }
    }
    cluster_sync();   // every slice's histogram complete
    const int eps = (E + S - 1) / S;
    int32_t *out = cnt + (static_cast<int64_t>(b) * G + g) * E;
    const uint32_t h0 = smem_u32(hist);
    for (int e = c * eps + threadIdx.x; e < min(E, (c + 1) * eps); e += blockDim.x) {
        int sum = 0;
        for (int q = 0; q < S; ++q) sum += ld_cluster_i32(mapa_shared(h0 + 4u * e, static_cast<uint32_t>(q)));
        out[e] = sum;
    }
    cluster_sync();   // no CTA leaves while another reads its histogram
    if (threadIdx.x == 0 && bad) flag(LB_DEV_BAD_IDS);
}

}  // namespace count
}  // namespace lb
