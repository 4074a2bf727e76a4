// Step 5: destination of every token-assignment and the stable (rank, expert)
// grouping permutation (Libra README, Key Ideas: tokens whose expert sits on
// their own GPU stay local, remote tokens go to GPUs holding a replica;
// FreeBalance sec. 2.2: dispatch groups tokens by device).
//
// Everything global about the permutation follows from the per-rank counts,
// the plan and the split, because source ranks own contiguous token ranges:
//   q0[g,e]   = remote assignments of e in source blocks before g
//   offs      = exclusive scan of the (rank, expert) bucket sizes
//   base[g,e] = where block g's assignments of e start in their bucket
//               (or q0 for a replicated expert's remote assignments, whose
//               destination depends on their rank q among e's remote ones).
// The prep kernel (one CTA per problem) computes these from cnt, plan and
// split without reading the ids.  The scatter kernel (one CTA per (problem,
// source block)) then needs only each assignment's rank among the earlier
// assignments of the same expert in its block: warps take consecutive
// 32-assignment steps with __match_any_sync ranks and per-warp counters in
// shared memory, a per-expert scan across warps keeps block order, and each
// assignment's slot is base + rank (plus the segment arithmetic for a
// replicated expert).  Positions never come from atomics, so the permutation
// is deterministic and stable.
#pragma once
#include "common.cuh"
#include "plan.cuh"

namespace lb {
namespace assign {

constexpr int PREP_THREADS = 1024;
constexpr int SC_THREADS = 1024;
constexpr int SC_WARPS = SC_THREADS / 32;
constexpr int SC_STEPS = 4;   // 32-assignment steps per warp per chunk

// Workspace per problem (int32 words): base[G*E], seg_qoff[GN], seg_cum[GN],
// seg_rep[GN]; rounded to 256 bytes.
__host__ __device__ inline size_t ws_words(int G, int E, int N) {
    const size_t w = static_cast<size_t>(G) * E + 3 * static_cast<size_t>(G) * N;
    return (w + 63) & ~static_cast<size_t>(63);
}

__host__ __device__ inline size_t prep_smem_bytes(int E) {
    return static_cast<size_t>(E) * 8 + static_cast<size_t>(E) * 4 * 2;
}

__host__ __device__ inline size_t scatter_smem_bytes(int E) {
    return static_cast<size_t>(E) * 8 + static_cast<size_t>(E) * 4 * 3 +
           static_cast<size_t>(SC_WARPS) * E * 4 * 2;
}

struct Args {
    const int32_t *ids, *cnt, *tok, *mass;
    const uint8_t *plan;
    size_t plan_stride;
    int T, k, G, E, N;
    int32_t *dest, *perm, *offs, *ws;
    size_t ws_stride;   // words per problem
};

__device__ __forceinline__ int clampi(int x, int lo, int hi) { return min(max(x, lo), hi); }

__global__ void __launch_bounds__(PREP_THREADS) prep_kernel(const Args a) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int G = a.G, E = a.E, N = a.N, GN = G * N, NK = G * E;
    uint64_t *hold = reinterpret_cast<uint64_t *>(sm);
    int32_t *homeadd = reinterpret_cast<int32_t *>(hold + E);
    int32_t *rcnt = homeadd + E;
    __shared__ int wsum[PREP_THREADS / 32];
    __shared__ int bad;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x;
    const int32_t *cnt = a.cnt + static_cast<int64_t>(b) * NK;
    const uint8_t *blob = a.plan + static_cast<size_t>(b) * a.plan_stride;
    const plan::Layout LY = plan::layout(G, E, N);
    const int32_t *hdr = reinterpret_cast<const int32_t *>(blob + LY.hdr);
    const int32_t *p_ev = reinterpret_cast<const int32_t *>(blob + LY.edge_v);
    const int32_t *p_ee = reinterpret_cast<const int32_t *>(blob + LY.edge_e);
    const int32_t *rep_ptr = reinterpret_cast<const int32_t *>(blob + LY.rep_ptr);
    const int32_t *rep_edge = reinterpret_cast<const int32_t *>(blob + LY.rep_edge);
    const int32_t *tok = a.tok + static_cast<int64_t>(b) * GN;
    const int32_t *mass = a.mass + static_cast<int64_t>(b) * GN;
    int32_t *offs = a.offs + static_cast<int64_t>(b) * (NK + 1);
    int32_t *base = a.ws + static_cast<size_t>(b) * a.ws_stride;
    int32_t *seg_qoff = base + NK;
    int32_t *seg_cum = seg_qoff + GN;
    int32_t *seg_rep = seg_cum + GN;
    const int Eg = E / G;
    int ne = hdr[0];
    if (tid == 0) bad = 0;
    if (ne < 0 || ne > GN) ne = 0;

    for (int e = tid; e < E; e += blockDim.x) hold[e] = 1ull << (e / Eg);
    __syncthreads();
    for (int i = tid; i < ne; i += blockDim.x) {
        const int e = p_ee[i], v = p_ev[i];
        if (e >= 0 && e < E && v >= 0 && v < G)
            atomicOr(reinterpret_cast<unsigned long long *>(&hold[e]), 1ull << v);
        else
            bad = 1;
    }
    __syncthreads();

    // q0 (into base, temporarily), remote mass, replica segments
    for (int e = tid; e < E; e += blockDim.x) {
        const uint64_t hm = hold[e];
        int run = 0;
        for (int g = 0; g < G; ++g) {
            base[g * E + e] = run;
            if (!((hm >> g) & 1ull)) run += cnt[g * E + e];
        }
        int r0 = rep_ptr[e], r1 = rep_ptr[e + 1];
        if (r0 < 0 || r1 > ne || r1 < r0) {
            bad = 1;
            r0 = r1 = 0;
        }
        rcnt[e] = r1 - r0;
        int qo = 0, cm = 0;
        for (int j = r0; j < r1; ++j) {
            const int i = rep_edge[j];
            if (i < 0 || i >= ne) {
                bad = 1;
                continue;
            }
            seg_qoff[i] = qo;
            seg_cum[i] = cm;
            qo += tok[i];
            cm += mass[i];
        }
        if (r1 > r0 && qo != run) bad = 1;
        homeadd[e] = (r1 > r0) ? cm : run;
    }
    __syncthreads();

    // bucket sizes over keys r*E+e, block-wide exclusive scan -> offs
    const int per = (NK + blockDim.x - 1) / blockDim.x;
    const int k0 = min(NK, tid * per), k1 = min(NK, k0 + per);
    auto bucket = [&](int key) -> int {
        const int r = key / E, e = key - r * E;
        const int h = e / Eg;
        int s = 0;
        if ((hold[e] >> r) & 1ull) s += cnt[key];
        if (r == h) {
            s += homeadd[e];
        } else if (((hold[e] >> r) & 1ull) && rcnt[e] > 0) {
            for (int j = rep_ptr[e]; j < rep_ptr[e + 1]; ++j) {
                const int i = rep_edge[j];
                if (i >= 0 && i < ne && p_ev[i] == r) s += tok[i] - mass[i];
            }
        }
        return s;
    };
    int local = 0;
    for (int key = k0; key < k1; ++key) local += bucket(key);
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int x = lane < (blockDim.x >> 5) ? wsum[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(kFull, x, off);
            if (lane >= off) x += y;
        }
        if (lane < (blockDim.x >> 5)) wsum[lane] = x;   // inclusive per warp
    }
    __syncthreads();
    int run = (warp > 0 ? wsum[warp - 1] : 0) + incl - local;
    for (int key = k0; key < k1; ++key) {
        offs[key] = run;
        run += bucket(key);
    }
    if (tid == blockDim.x - 1) offs[NK] = wsum[(blockDim.x >> 5) - 1];
    __syncthreads();

    // final base per (block g, expert e)
    for (int key = tid; key < NK; key += blockDim.x) {
        const int g = key / E, e = key - g * E;
        const int h = e / Eg;
        const int q0 = base[key];
        const int r0 = rep_ptr[e], r1 = rcnt[e] > 0 ? rep_ptr[e + 1] : r0;
        int out;
        if ((hold[e] >> g) & 1ull) {
            int before = 0;
            if (g == h) {
                if (r1 == r0) {
                    before = q0;
                } else {
                    for (int j = r0; j < r1; ++j) {
                        const int i = rep_edge[j];
                        if (i >= 0 && i < ne) before += clampi(q0 - seg_qoff[i], 0, mass[i]);
                    }
                }
            } else {
                for (int j = r0; j < r1; ++j) {
                    const int i = rep_edge[j];
                    if (i >= 0 && i < ne && p_ev[i] == g)
                        before = clampi(q0 - seg_qoff[i] - mass[i], 0, tok[i] - mass[i]);
                }
            }
            out = offs[key] + before;
        } else if (r1 == r0) {
            out = offs[h * E + e] + (h < g ? cnt[h * E + e] : 0) + q0;
        } else {
            out = q0;
        }
        base[key] = out;
    }
    for (int i = tid; i < ne; i += blockDim.x) {
        const int e = p_ee[i], v = p_ev[i];
        seg_rep[i] = (e >= 0 && e < E && v >= 0 && v < G) ? offs[v * E + e] : 0;
    }
    if (tid == 0 && bad) flag(LB_DEV_BAD_SPLIT);
}

__global__ void __launch_bounds__(SC_THREADS) scatter_kernel(const Args a) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int G = a.G, E = a.E, N = a.N, GN = G * N, NK = G * E, k = a.k;
    uint64_t *hold = reinterpret_cast<uint64_t *>(sm);
    int32_t *rcnt = reinterpret_cast<int32_t *>(hold + E);
    int32_t *base_s = rcnt + E;
    int32_t *run = base_s + E;
    int32_t *wcnt = run + E;                  // [SC_WARPS][E]
    int32_t *pre = wcnt + SC_WARPS * E;       // [SC_WARPS][E]
    __shared__ int bad;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = blockIdx.x, b = blockIdx.y;
    const int32_t *cnt = a.cnt + static_cast<int64_t>(b) * NK;
    const uint8_t *blob = a.plan + static_cast<size_t>(b) * a.plan_stride;
    const plan::Layout LY = plan::layout(G, E, N);
    const int32_t *hdr = reinterpret_cast<const int32_t *>(blob + LY.hdr);
    const int32_t *p_ev = reinterpret_cast<const int32_t *>(blob + LY.edge_v);
    const int32_t *p_ee = reinterpret_cast<const int32_t *>(blob + LY.edge_e);
    const int32_t *rep_ptr = reinterpret_cast<const int32_t *>(blob + LY.rep_ptr);
    const int32_t *rep_edge = reinterpret_cast<const int32_t *>(blob + LY.rep_edge);
    const int32_t *tok = a.tok + static_cast<int64_t>(b) * GN;
    const int32_t *mass = a.mass + static_cast<int64_t>(b) * GN;
    const int32_t *offs = a.offs + static_cast<int64_t>(b) * (NK + 1);
    const int32_t *ws = a.ws + static_cast<size_t>(b) * a.ws_stride;
    const int32_t *seg_qoff = ws + NK;
    const int32_t *seg_cum = seg_qoff + GN;
    const int32_t *seg_rep = seg_cum + GN;
    const int Eg = E / G;
    const int Tg = a.T / G;
    const int nitems = Tg * k;
    const int64_t f0 = static_cast<int64_t>(g) * nitems;         // problem-local flat index
    const int32_t *ids = a.ids + static_cast<int64_t>(b) * a.T * k;
    int32_t *dest = a.dest + static_cast<int64_t>(b) * a.T * k;
    int32_t *perm = a.perm + static_cast<int64_t>(b) * a.T * k;
    const int nf = a.T * k;
    int ne = hdr[0];
    if (ne < 0 || ne > GN) ne = 0;

    if (tid == 0) bad = 0;
    for (int e = tid; e < E; e += blockDim.x) {
        hold[e] = 1ull << (e / Eg);
        const int r0 = rep_ptr[e], r1 = rep_ptr[e + 1];
        rcnt[e] = (r0 < 0 || r1 > ne || r1 < r0) ? 0 : r1 - r0;
        base_s[e] = ws[g * E + e];
        run[e] = 0;
    }
    __syncthreads();
    for (int i = tid; i < ne; i += blockDim.x) {
        const int e = p_ee[i], v = p_ev[i];
        if (e >= 0 && e < E && v >= 0 && v < G)
            atomicOr(reinterpret_cast<unsigned long long *>(&hold[e]), 1ull << v);
    }
    __syncthreads();

    constexpr int CH = SC_WARPS * 32 * SC_STEPS;
    int32_t *wrow = wcnt + warp * E;
    for (int cs = 0; cs < nitems; cs += CH) {
        for (int e = lane; e < E; e += 32) wrow[e] = 0;
        __syncwarp();
        int es[SC_STEPS], loc[SC_STEPS];
#pragma unroll
        for (int s = 0; s < SC_STEPS; ++s) {
            const int i = cs + warp * 32 * SC_STEPS + s * 32 + lane;
            int e = -1;
            if (i < nitems) {
                e = __ldg(ids + f0 + i);
                if (e < 0 || e >= E) {
                    bad = 1;
                    e = -1;
                }
            }
            const unsigned peers = __match_any_sync(kFull, e);
            const int rnk = __popc(peers & lanemask_lt());
            const int cur = e >= 0 ? wrow[e] : 0;
            __syncwarp();
            if (e >= 0 && lane == 31 - __clz(peers)) wrow[e] = cur + __popc(peers);
            __syncwarp();
            es[s] = e;
            loc[s] = cur + rnk;
        }
        __syncthreads();
        for (int e = tid; e < E; e += blockDim.x) {
            int acc = run[e];
            for (int w = 0; w < SC_WARPS; ++w) {
                const int t = wcnt[w * E + e];
                pre[w * E + e] = acc;
                acc += t;
            }
            run[e] = acc;
        }
        __syncthreads();
#pragma unroll
        for (int s = 0; s < SC_STEPS; ++s) {
            const int e = es[s];
            if (e < 0) continue;
            const int i = cs + warp * 32 * SC_STEPS + s * 32 + lane;
            const int rho = pre[warp * E + e] + loc[s];
            const int h = e / Eg;
            int d, p;
            if ((hold[e] >> g) & 1ull) {
                d = g;
                p = base_s[e] + rho;
            } else if (rcnt[e] == 0) {
                d = h;
                p = base_s[e] + rho;
            } else {
                const int q = base_s[e] + rho;
                d = -1;
                p = -1;
                for (int j = rep_ptr[e]; j < rep_ptr[e] + rcnt[e]; ++j) {
                    const int ei = rep_edge[j];
                    if (ei < 0 || ei >= ne) break;
                    const int qo = seg_qoff[ei];
                    const int t = tok[ei];
                    if (q < qo + t) {
                        const int w = q - qo, mss = mass[ei];
                        if (w < mss) {
                            d = h;
                            p = offs[h * E + e] + (h < g ? cnt[h * E + e] : 0) + seg_cum[ei] + w;
                        } else {
                            const int v = p_ev[ei];
                            if (v < 0 || v >= G) break;
                            d = v;
                            p = seg_rep[ei] + (v < g ? cnt[v * E + e] : 0) + (w - mss);
                        }
                        break;
                    }
                }
            }
            const int64_t f = f0 + i;
            if (d < 0 || p < 0 || p >= nf) {
                bad = 1;
                continue;
            }
            dest[f] = d;
            perm[p] = static_cast<int32_t>(f);
        }
    }
    __syncthreads();
    if (tid == 0 && bad) flag(LB_DEV_BAD_SPLIT);
}

}  // namespace assign
}  // namespace lb
