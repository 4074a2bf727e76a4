// Split variants of Relief's ablation (Relief, Ablation Results, Table III;
// The Relief Algorithm, key properties: all-integer Q11.20): the same replica
// edges, round schedule and starting point as the split kernel, with the
// pass replaced by one of
//   0 RELIEF        the reference pass (Algorithm 1);
//   1 NO_REVERSE    no reverse move: only home -> replica moves;
//   2 JACOBI        loads snapshotted at the pass start, moves of a quarter
//                   of the snapshot gap (damped), applied as they come;
//   3 HASH          the load-oblivious equal split of a hash router over
//                   home and replicas (home first, remainders to the first
//                   holders); no passes;
//   4 WATER         water-filling: replicated experts in ascending id, each
//                   expert's remote tokens poured over its holders from the
//                   lowest load up (integer levels, leftovers in holder
//                   order, a replica capped at its edge's tokens);
//   5 PROPORTIONAL  replicated experts in ascending id, remote tokens divided
//                   in proportion to (max base load - base load + 1), largest
//                   remainders (ties in holder order), a replica's excess over
//                   its edge's tokens kept at home;
//   6 FP32          Relief in fp32 (exact halving), masses rounded to the
//                   nearest token (ties to even) at the end;
//   7 Q1120         Relief in Q11.20: units of 2^-f tokens, f = 20 - s, s the
//                   smallest shift keeping the total load below 2^11;
//                   masses rounded to the nearest token (ties up) at the end.
// A pass that changes nothing ends the loop (0-2, 4-7).
//
// One CTA per problem: all threads stage the plan and compute the remote
// mass, the fixed loads and the equal partition; warp 0 runs the passes.  In
// the Relief-like variants a round's transfers are rank-disjoint, so lane j
// takes transfer j of the round (rounds hold at most G/2 <= 32 transfers);
// the water-filling and proportional variants take one expert at a time
// with one lane per holder (home = holder 0) and warp reductions.
#pragma once
#include "common.cuh"
#include "plan.cuh"

namespace lb {
namespace splitv {

constexpr int THREADS = 256;
enum { RELIEF = 0, NO_REVERSE, JACOBI, HASH, WATER, PROPORTIONAL, FP32, Q1120, COUNT };

struct Params {
    const int32_t *cnt;
    const uint8_t *plan;
    size_t plan_stride;
    int G, E, N, passes, variant;
    int32_t *tok, *mass, *loads, *passes_run;
};

__host__ __device__ inline size_t smem_bytes(int G, int E, int N) {
    const size_t GN = static_cast<size_t>(G) * N;
    // int64: loads, snapshot, Q loads [G]; Q masses [GN]; int32: R [E], rep_ptr [E+1], eu, ev, ee, rep_edge,
    // tok, mass [GN], round_ptr [GN+1]; float: loads [G], masses [GN]; u64 holder masks [E]
    return static_cast<size_t>(G) * 8 * 3 + GN * 8 + static_cast<size_t>(E) * 8 +
           (static_cast<size_t>(E) * 2 + 1 + GN * 7 + 1) * 4 + (static_cast<size_t>(G) + GN) * 4 + 64;
}

__device__ __forceinline__ long long warp_sum_ll(long long x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(kFull, x, off);
    return x;
}
__device__ __forceinline__ long long warp_min_ll(long long x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x = min(x, __shfl_xor_sync(kFull, x, off));
    return x;
}
__device__ __forceinline__ long long warp_max_ll(long long x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x = max(x, __shfl_xor_sync(kFull, x, off));
    return x;
}

__global__ void __launch_bounds__(THREADS) split_variant_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t sm[];
    pdl_begin();
    const int G = p.G, E = p.E, N = p.N, GN = G * N, b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    long long *L = reinterpret_cast<long long *>(sm);
    long long *snap = L + G;
    long long *Lq = snap + G;
    long long *mq = Lq + G;
    uint64_t *hold = reinterpret_cast<uint64_t *>(mq + GN);
    int32_t *R = reinterpret_cast<int32_t *>(hold + E);
    int32_t *rep_ptr = R + E;
    int32_t *eu = rep_ptr + E + 1;
    int32_t *ev = eu + GN;
    int32_t *ee = ev + GN;
    int32_t *rep_edge = ee + GN;
    int32_t *tk = rep_edge + GN;
    int32_t *ms = tk + GN;
    int32_t *rptr = ms + GN;
    float *Lf = reinterpret_cast<float *>(rptr + GN + 1);
    float *mf = Lf + G;
    __shared__ int bad, ne_s, nr_s;

    const uint8_t *blob = p.plan + static_cast<size_t>(b) * p.plan_stride;
    const plan::Layout LY = plan::layout(G, E, N);
    const int32_t *cnt = p.cnt + static_cast<int64_t>(b) * G * E;
    if (tid == 0) {
        const int32_t *hdr = reinterpret_cast<const int32_t *>(blob + LY.hdr);
        int ne = hdr[0], nr = hdr[1];
        bad = (ne < 0 || ne > GN || nr < 0 || nr > GN) ? 1 : 0;
        ne_s = bad ? 0 : ne;
        nr_s = bad ? 0 : nr;
    }
    __syncthreads();
    const int ne = ne_s, nr = nr_s, Eg = E / G;
    {
        const int32_t *p_eu = reinterpret_cast<const int32_t *>(blob + LY.edge_u);
        const int32_t *p_ev = reinterpret_cast<const int32_t *>(blob + LY.edge_v);
        const int32_t *p_ee = reinterpret_cast<const int32_t *>(blob + LY.edge_e);
        const int32_t *p_re = reinterpret_cast<const int32_t *>(blob + LY.rep_edge);
        const int32_t *p_rp = reinterpret_cast<const int32_t *>(blob + LY.rep_ptr);
        const int32_t *p_rr = reinterpret_cast<const int32_t *>(blob + LY.round_ptr);
        for (int i = tid; i < ne; i += blockDim.x) {
            eu[i] = p_eu[i];
            ev[i] = p_ev[i];
            ee[i] = p_ee[i];
            rep_edge[i] = p_re[i];
            if (eu[i] < 0 || eu[i] >= G || ev[i] < 0 || ev[i] >= G || ee[i] < 0 || ee[i] >= E || rep_edge[i] < 0 ||
                rep_edge[i] >= ne)
                bad = 1;
        }
        for (int e = tid; e <= E; e += blockDim.x) rep_ptr[e] = p_rp[e];
        for (int r = tid; r <= nr; r += blockDim.x) rptr[r] = p_rr[r];
    }
    __syncthreads();
    for (int r = tid; r < nr; r += blockDim.x)
        if (rptr[r] < 0 || rptr[r + 1] < rptr[r] || rptr[r + 1] > ne || rptr[r + 1] - rptr[r] > 32) bad = 1;
    for (int e = tid; e < E; e += blockDim.x)
        if (rep_ptr[e] < 0 || rep_ptr[e + 1] < rep_ptr[e] || rep_ptr[e + 1] > ne) bad = 1;
    __syncthreads();
    if (bad) {
        if (tid == 0) {
            flag(LB_DEV_BAD_PLAN);
            p.passes_run[b] = 0;
        }
        return;
    }
    // per expert: holders (home + replica ranks), remote mass, equal partition
    for (int e = tid; e < E; e += blockDim.x) {
        uint64_t hm = 1ull << (e / Eg);
        for (int j = rep_ptr[e]; j < rep_ptr[e + 1]; ++j) hm |= 1ull << ev[rep_edge[j]];
        int r = 0;
        for (int g = 0; g < G; ++g)
            if (!((hm >> g) & 1ull)) r += cnt[static_cast<int64_t>(g) * E + e];
        hold[e] = hm;
        R[e] = r;
        const int m = rep_ptr[e + 1] - rep_ptr[e];
        for (int j = 0; j < m; ++j) {
            const int i = rep_edge[rep_ptr[e] + j];
            tk[i] = r / m + (j < r % m ? 1 : 0);
            ms[i] = tk[i];
        }
    }
    __syncthreads();
    // fixed loads: own tokens of held experts + remote mass of unreplicated home experts;
    // then every edge's mass at its home
    for (int i = tid; i < G; i += blockDim.x) {
        long long x = 0;
        for (int e = 0; e < E; ++e) {
            if ((hold[e] >> i) & 1ull) x += cnt[static_cast<int64_t>(i) * E + e];
            if (e / Eg == i && rep_ptr[e + 1] == rep_ptr[e]) x += R[e];
        }
        snap[i] = x;   // fixed load, kept in snap until the passes
        float xf = static_cast<float>(x);
        long long l = x;
        for (int k = 0; k < ne; ++k)
            if (eu[k] == i) {
                l += tk[k];
                xf = __fadd_rn(xf, static_cast<float>(tk[k]));   // in schedule order, as the reference sums
            }
        L[i] = l;
        Lf[i] = xf;
    }
    __syncthreads();
    if (warp != 0) return;
    // fixed loads move to registers: lane r holds ranks r and r + 32
    const long long F0 = lane < G ? snap[lane] : 0, F1 = lane + 32 < G ? snap[lane + 32] : 0;
    __syncwarp();
    const int variant = p.variant;
    int pr = 0;

    if (variant == RELIEF || variant == NO_REVERSE || variant == JACOBI) {
        for (int pass = 1; pass <= p.passes; ++pass) {
            if (variant == JACOBI) {
                for (int i = lane; i < G; i += 32) snap[i] = L[i];
                __syncwarp();
            }
            bool moved = false;
            for (int r = 0; r < nr; ++r) {
                const int i = rptr[r] + lane;
                if (i < rptr[r + 1]) {
                    const int u = eu[i], v = ev[i];
                    const long long gap = variant == JACOBI ? snap[u] - snap[v] : L[u] - L[v];
                    long long delta = (gap < 0 ? -gap : gap) >> (variant == JACOBI ? 2 : 1);
                    const long long limit = gap > 0 ? ms[i] : (variant == NO_REVERSE ? 0 : tk[i] - ms[i]);
                    if (delta > limit) delta = limit;
                    if (delta > 0) {
                        const long long sd = gap > 0 ? delta : -delta;
                        L[u] -= sd;
                        L[v] += sd;
                        ms[i] -= static_cast<int>(sd);
                        moved = true;
                    }
                }
                __syncwarp();
            }
            pr = pass;
            if (!__any_sync(kFull, moved)) break;
        }
    } else if (variant == FP32) {
        for (int pass = 1; pass <= p.passes; ++pass) {
            bool moved = false;
            for (int i = lane; i < ne; i += 32) mf[i] = pass == 1 ? static_cast<float>(tk[i]) : mf[i];
            __syncwarp();
            for (int r = 0; r < nr; ++r) {
                const int i = rptr[r] + lane;
                if (i < rptr[r + 1]) {
                    const int u = eu[i], v = ev[i];
                    const float gap = __fsub_rn(Lf[u], Lf[v]);
                    float delta = __fmul_rn(gap < 0.0f ? -gap : gap, 0.5f);
                    const float limit = gap > 0.0f ? mf[i] : __fsub_rn(static_cast<float>(tk[i]), mf[i]);
                    if (delta > limit) delta = limit;
                    if (delta > 0.0f) {
                        const float sd = gap > 0.0f ? delta : -delta;
                        Lf[u] = __fsub_rn(Lf[u], sd);
                        Lf[v] = __fadd_rn(Lf[v], sd);
                        mf[i] = __fsub_rn(mf[i], sd);
                        moved = true;
                    }
                }
                __syncwarp();
            }
            pr = pass;
            if (!__any_sync(kFull, moved)) break;
        }
        if (p.passes < 1)
            for (int i = lane; i < ne; i += 32) mf[i] = static_cast<float>(tk[i]);
        __syncwarp();
        for (int i = lane; i < ne; i += 32) {
            float x = rintf(mf[i]);
            x = fminf(fmaxf(x, 0.0f), static_cast<float>(tk[i]));
            ms[i] = static_cast<int>(x);
        }
    } else if (variant == Q1120) {
        long long tot = warp_sum_ll((lane < G ? L[lane] : 0) + (lane + 32 < G ? L[lane + 32] : 0));
        int s = 0;
        while ((tot >> s) >= 2048) ++s;
        const int f = 20 - s;
        for (int i = lane; i < G; i += 32) Lq[i] = L[i] << f;
        for (int i = lane; i < ne; i += 32) mq[i] = static_cast<long long>(tk[i]) << f;
        __syncwarp();
        for (int pass = 1; pass <= p.passes; ++pass) {
            bool moved = false;
            for (int r = 0; r < nr; ++r) {
                const int i = rptr[r] + lane;
                if (i < rptr[r + 1]) {
                    const int u = eu[i], v = ev[i];
                    const long long gap = Lq[u] - Lq[v];
                    long long delta = (gap < 0 ? -gap : gap) >> 1;
                    const long long limit = gap > 0 ? mq[i] : (static_cast<long long>(tk[i]) << f) - mq[i];
                    if (delta > limit) delta = limit;
                    if (delta > 0) {
                        const long long sd = gap > 0 ? delta : -delta;
                        Lq[u] -= sd;
                        Lq[v] += sd;
                        mq[i] -= sd;
                        moved = true;
                    }
                }
                __syncwarp();
            }
            pr = pass;
            if (!__any_sync(kFull, moved)) break;
        }
        for (int i = lane; i < ne; i += 32) {
            long long x = f > 0 ? (mq[i] + (1ll << (f - 1))) >> f : mq[i];
            x = min(max(x, 0ll), static_cast<long long>(tk[i]));
            ms[i] = static_cast<int>(x);
        }
    } else if (variant == HASH) {
        for (int e = lane; e < E; e += 32) {
            const int m = rep_ptr[e + 1] - rep_ptr[e];
            if (m == 0) continue;
            const int q = R[e] / (m + 1), rem = R[e] % (m + 1);
            for (int j = 0; j < m; ++j) {
                const int i = rep_edge[rep_ptr[e] + j];
                const int share = min(q + (j + 1 < rem ? 1 : 0), tk[i]);
                ms[i] = tk[i] - share;
            }
        }
    } else {   // WATER, PROPORTIONAL: one expert at a time, lane h = holder h (h and h + 32)
        for (int pass = 1; pass <= p.passes; ++pass) {
            bool changed = false;
            for (int e = 0; e < E; ++e) {
                const int m = rep_ptr[e + 1] - rep_ptr[e];
                if (m == 0) continue;
                const int home = e / Eg, n = m + 1, Re = R[e];
                long long at_home = 0;
                for (int j = lane; j < m; j += 32) at_home += ms[rep_edge[rep_ptr[e] + j]];
                at_home = warp_sum_ll(at_home);
                // holders h0 = lane, h1 = lane + 32: base load, capacity, edge
                long long B[2], cap[2], a[2];
                int ei[2];
                bool in[2];
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int h = lane + 32 * t;
                    in[t] = h < n;
                    ei[t] = (in[t] && h > 0) ? rep_edge[rep_ptr[e] + h - 1] : -1;
                    if (!in[t]) {
                        B[t] = 0;
                        cap[t] = 0;
                    } else if (h == 0) {
                        B[t] = L[home] - at_home;
                        cap[t] = Re;
                    } else {
                        B[t] = L[ev[ei[t]]] - (tk[ei[t]] - ms[ei[t]]);
                        cap[t] = tk[ei[t]];
                    }
                    a[t] = 0;
                }
                if (variant == WATER) {
                    long long lo = warp_min_ll(min(in[0] ? B[0] : LLONG_MAX, in[1] ? B[1] : LLONG_MAX));
                    long long hi = warp_max_ll(max(in[0] ? B[0] : LLONG_MIN, in[1] ? B[1] : LLONG_MIN)) + Re + 1;
                    while (lo < hi) {
                        const long long mid = lo + (hi - lo + 1) / 2;
                        long long fl = 0;
#pragma unroll
                        for (int t = 0; t < 2; ++t)
                            if (in[t]) fl += min(cap[t], max(0ll, mid - B[t]));
                        fl = warp_sum_ll(fl);
                        if (fl <= Re) lo = mid; else hi = mid - 1;
                    }
                    long long used = 0;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        a[t] = in[t] ? min(cap[t], max(0ll, lo - B[t])) : 0;
                        used += a[t];
                    }
                    used = warp_sum_ll(used);
                    // leftovers: holders at the level with room, in holder order
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const bool el = in[t] && B[t] + a[t] <= lo && a[t] < cap[t];
                        const unsigned bal = __ballot_sync(kFull, el);
                        const int before = __popc(bal & lanemask_lt()) +
                                           (t == 1 ? __popc(__ballot_sync(kFull, in[0] && B[0] + a[0] <= lo &&
                                                                                    a[0] < cap[0])) : 0);
                        if (el && before < Re - used) a[t] += 1;
                    }
                } else {
                    const long long M = warp_max_ll(max(in[0] ? B[0] : LLONG_MIN, in[1] ? B[1] : LLONG_MIN));
                    long long w[2], rm[2];
#pragma unroll
                    for (int t = 0; t < 2; ++t) w[t] = in[t] ? M - B[t] + 1 : 0;
                    const long long W = warp_sum_ll(w[0] + w[1]);
                    long long used = 0;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        a[t] = in[t] ? (static_cast<long long>(Re) * w[t]) / W : 0;
                        rm[t] = in[t] ? (static_cast<long long>(Re) * w[t]) % W : -1;
                        used += a[t];
                    }
                    used = warp_sum_ll(used);
                    // largest remainders, ties in holder order: one holder per round
                    for (long long k = used; k < Re; ++k) {
                        const long long best = warp_max_ll(max(rm[0], rm[1]));
                        const unsigned b0 = __ballot_sync(kFull, rm[0] == best), b1 = __ballot_sync(kFull, rm[1] == best);
                        const int hb = b0 ? __ffs(b0) - 1 : 32 + __ffs(b1) - 1;
                        if (hb == lane) { a[0] += 1; rm[0] = -1; }
                        if (hb == lane + 32) { a[1] += 1; rm[1] = -1; }
                    }
                    // a replica's excess over its edge's tokens stays at home
                    long long excess = 0;
#pragma unroll
                    for (int t = 0; t < 2; ++t)
                        if (in[t] && lane + 32 * t > 0 && a[t] > cap[t]) {
                            excess += a[t] - cap[t];
                            a[t] = cap[t];
                        }
                    excess = warp_sum_ll(excess);
                    if (lane == 0) a[0] += excess;
                }
                __syncwarp();
                bool ch = false;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int h = lane + 32 * t;
                    if (!in[t]) continue;
                    if (h == 0) {
                        L[home] = B[t] + a[t];
                    } else {
                        const int nm = static_cast<int>(tk[ei[t]] - a[t]);
                        ch |= nm != ms[ei[t]];
                        ms[ei[t]] = nm;
                        L[ev[ei[t]]] = B[t] + a[t];
                    }
                }
                changed |= __any_sync(kFull, ch);
                __syncwarp();
            }
            pr = pass;
            if (!changed) break;
        }
    }
    __syncwarp();
    // outputs; loads recomputed from the masses (fixed + home masses + replica shares)
    for (int i = lane; i < ne; i += 32) {
        p.tok[static_cast<int64_t>(b) * GN + i] = tk[i];
        p.mass[static_cast<int64_t>(b) * GN + i] = ms[i];
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int r = lane + 32 * t;
        if (r >= G) continue;
        long long x = t == 0 ? F0 : F1;
        for (int i = 0; i < ne; ++i) {
            if (eu[i] == r) x += ms[i];
            if (ev[i] == r) x += tk[i] - ms[i];
        }
        p.loads[static_cast<int64_t>(b) * G + r] = static_cast<int32_t>(x);
    }
    if (lane == 0) p.passes_run[b] = pr;
}

}  // namespace splitv
}  // namespace lb
