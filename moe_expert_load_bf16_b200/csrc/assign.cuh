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
// split without reading the ids; counts and plan are staged in shared memory
// first.  The scatter kernel (one CTA per (problem, source block)) then needs
// only each assignment's rank among the earlier assignments of the same
// expert in its block: warps take consecutive 32-assignment steps with
// __match_any_sync ranks and per-warp counters in shared memory, a warp
// shuffle scan across warps keeps block order, and each assignment's slot is
// base + rank, or, for a replicated expert's remote assignment, a short walk
// over the expert's replica segments (staged in shared memory).  Positions
// never come from atomics, so the permutation is deterministic and stable.
#pragma once
#include "common.cuh"
#include "plan.cuh"

namespace lb {
namespace assign {

constexpr int PREP_THREADS = 1024;
constexpr int SC_THREADS = 1024;
constexpr int SC_WARPS = SC_THREADS / 32;
constexpr int SC_STEPS = 8;   // 32-assignment steps per warp per chunk
static_assert(SC_WARPS == 32, "the cross-warp scan maps one warp's counts to one lane");

// Workspace per problem (int32 words): base[G*E], seg_qoff[GN], seg_cum[GN],
// seg_rep[GN]; rounded to 256 bytes.
__host__ __device__ inline size_t ws_words(int G, int E, int N) {
    const size_t w = static_cast<size_t>(G) * E + 3 * static_cast<size_t>(G) * N;
    return (w + 63) & ~static_cast<size_t>(63);
}

__host__ __device__ inline size_t prep_smem_bytes(int G, int E, int N) {
    const size_t GN = static_cast<size_t>(G) * N;
    return static_cast<size_t>(E) * 8 + static_cast<size_t>(G) * E * 4 * 2 + static_cast<size_t>(E) * 4 * 3 +
           (static_cast<size_t>(E) + 1) * 4 + GN * 4 * 7 + 64;
}

// Shared memory of the scatter: per-expert tables (holders, replica count,
// CSR start, home count), the per-(CTA or warp) block bases and running
// counts, the per-warp counter tables, and the replica segments.
__host__ __device__ inline size_t scatter_smem_bytes(int G, int E, int N) {
    const size_t GN = static_cast<size_t>(G) * N, EP = static_cast<size_t>(E) + 1;
    return static_cast<size_t>(E) * 8 + static_cast<size_t>(E) * 4 * 3 + (static_cast<size_t>(E) + 1) * 4 +
           static_cast<size_t>(SC_WARPS) * EP * 4 * 3 + GN * 4 * 7 + 64;
}

// Source blocks of at most this many assignments are scattered one block per
// warp (no block-wide barrier); larger ones by the whole CTA.
constexpr int WARP_BLOCK_MAX = 2048;

struct Args {
    const int32_t *ids, *cnt, *tok, *mass;
    const uint8_t *plan;
    size_t plan_stride;
    int T, k, G, E, N;
    int32_t *dest, *perm, *offs, *ws;
    size_t ws_stride;   // words per problem
};

__device__ __forceinline__ int clampi(int x, int lo, int hi) { return min(max(x, lo), hi); }

// Tables of problem b for its scatter: offs, base[g,e], replica segments.
// All threads of the CTA call it; `sm` holds prep_smem_bytes(G,E,N) bytes.
__device__ void prep_problem(const Args &a, int b, uint8_t *sm) {
    const int G = a.G, E = a.E, N = a.N, GN = G * N, NK = G * E;
    uint64_t *hold = reinterpret_cast<uint64_t *>(sm);
    int32_t *cnt_s = reinterpret_cast<int32_t *>(hold + E);
    int32_t *homeadd = cnt_s + NK;
    int32_t *rcnt = homeadd + E;
    int32_t *rtot = rcnt + E;
    int32_t *rep_ptr = rtot + E;     // [E+1]
    int32_t *rep_edge = rep_ptr + E + 1;
    int32_t *ev = rep_edge + GN;
    int32_t *ee = ev + GN;
    int32_t *tk = ee + GN;
    int32_t *ms = tk + GN;
    int32_t *sq = ms + GN;           // segment start in q
    int32_t *sc = sq + GN;           // mass of earlier segments
    int32_t *osz = sc + GN;          // [NK] bucket sizes, then their exclusive scan
    __shared__ int wsum[32];
    __shared__ int bad;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t *cnt = a.cnt + static_cast<int64_t>(b) * NK;
    const uint8_t *blob = a.plan + static_cast<size_t>(b) * a.plan_stride;
    const plan::Layout LY = plan::layout(G, E, N);
    const int32_t *hdr = reinterpret_cast<const int32_t *>(blob + LY.hdr);
    int32_t *offs = a.offs + static_cast<int64_t>(b) * (NK + 1);
    int32_t *base = a.ws + static_cast<size_t>(b) * a.ws_stride;
    int32_t *seg_qoff = base + NK;
    int32_t *seg_cum = seg_qoff + GN;
    int32_t *seg_rep = seg_cum + GN;
    const int Eg = E / G;
    int ne = hdr[0];
    if (tid == 0) bad = 0;
    if (ne < 0 || ne > GN) ne = 0;

    // ---- stage inputs
    LB_TICK(20);
    stage_i32(cnt_s, cnt, NK);
    {
        const int32_t *p_ev = reinterpret_cast<const int32_t *>(blob + LY.edge_v);
        const int32_t *p_ee = reinterpret_cast<const int32_t *>(blob + LY.edge_e);
        const int32_t *p_rep_edge = reinterpret_cast<const int32_t *>(blob + LY.rep_edge);
        const int32_t *p_rep_ptr = reinterpret_cast<const int32_t *>(blob + LY.rep_ptr);
        const int32_t *tok = a.tok + static_cast<int64_t>(b) * GN;
        const int32_t *mass = a.mass + static_cast<int64_t>(b) * GN;
        for (int i = tid; i < ne; i += blockDim.x) {
            ev[i] = p_ev[i];
            ee[i] = p_ee[i];
            rep_edge[i] = p_rep_edge[i];
            tk[i] = tok[i];
            ms[i] = mass[i];
        }
        for (int e = tid; e <= E; e += blockDim.x) rep_ptr[e] = p_rep_ptr[e];
    }
    __syncthreads();

    // ---- per expert: holders, remote mass, replica segments
    for (int e = tid; e < E; e += blockDim.x) {
        const int h = e / Eg;
        int r0 = rep_ptr[e], r1 = rep_ptr[e + 1];
        if (r0 < 0 || r1 > ne || r1 < r0) {
            bad = 1;
            r0 = r1 = 0;
        }
        uint64_t hm = 1ull << h;
        int qo = 0, cm = 0;
        for (int j = r0; j < r1; ++j) {
            const int i = rep_edge[j];
            if (i < 0 || i >= ne || ee[i] != e || ev[i] < 0 || ev[i] >= G) {
                bad = 1;
                continue;
            }
            hm |= 1ull << ev[i];
            sq[i] = qo;
            sc[i] = cm;
            qo += tk[i];
            cm += ms[i];
        }
        int R = 0;
        for (int g = 0; g < G; ++g)
            if (!((hm >> g) & 1ull)) R += cnt_s[g * E + e];
        if (r1 > r0 && qo != R) bad = 1;
        hold[e] = hm;
        rcnt[e] = r1 - r0;
        rtot[e] = R;
        homeadd[e] = (r1 > r0) ? cm : R;
    }
    __syncthreads();
    LB_TICK(21);

    // ---- bucket sizes over keys r*E+e: own tokens of held experts, the home
    // share of each expert, and every edge's replica share (tok - mass)
    for (int r = warp; r < G; r += (blockDim.x >> 5)) {
        for (int e = lane; e < E; e += 32) {
            const uint64_t hm = hold[e];
            int sz = ((hm >> r) & 1ull) ? cnt_s[r * E + e] : 0;
            sz += (e >= r * Eg && e < (r + 1) * Eg) ? homeadd[e] : 0;
            osz[r * E + e] = sz;
        }
    }
    __syncthreads();
    for (int i = tid; i < ne; i += blockDim.x) {
        const int e = ee[i], v = ev[i];
        if (e >= 0 && e < E && v >= 0 && v < G) osz[v * E + e] += tk[i] - ms[i];   // one edge per (v, e)
    }
    __syncthreads();
    // block-wide exclusive scan, in place: warp w scans its contiguous
    // segment of keys 32 at a time (conflict-free, coalesced), then the warp
    // totals are scanned and added back; offs (global) gets a copy
    {
        const int nw = blockDim.x >> 5;
        const int seg = ((NK + nw - 1) / nw + 31) & ~31;
        const int s0 = min(NK, warp * seg), s1 = min(NK, s0 + seg);
        int carry = 0;
        for (int kb = s0; kb < s1; kb += 32) {
            const int key = kb + lane;
            const int x0 = key < s1 ? osz[key] : 0;
            int x = x0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(kFull, x, off);
                if (lane >= off) x += y;
            }
            if (key < s1) osz[key] = carry + x - x0;
            carry += __shfl_sync(kFull, x, 31);
        }
        if (lane == 0) wsum[warp] = carry;
        __syncthreads();
        if (warp == 0) {
            const int c = lane < nw ? wsum[lane] : 0;
            int x = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(kFull, x, off);
                if (lane >= off) x += y;
            }
            if (lane < nw) wsum[lane] = x - c;   // exclusive per warp
            if (lane == nw - 1) offs[NK] = x;
        }
        __syncthreads();
        const int add = wsum[warp];
        for (int key = s0 + lane; key < s1; key += 32) {
            const int o = osz[key] + add;
            osz[key] = o;
            offs[key] = o;
        }
    }
    __syncthreads();
    LB_TICK(22);

    // ---- base per (block g, expert e): thread per expert, g ascending with
    // the running remote prefix q0 and a cursor into the expert's replica
    // edges (ordered by ascending replica rank)
    for (int e = tid; e < E; e += blockDim.x) {
        const int h = e / Eg;
        const uint64_t hm = hold[e];
        const int r0 = rep_ptr[e], m = rcnt[e];
        int j = r0;
        int q0 = 0;
        for (int g = 0; g < G; ++g) {
            int out;
            if ((hm >> g) & 1ull) {
                int before = 0;
                if (g == h) {
                    if (m == 0) {
                        before = q0;
                    } else {
                        for (int jj = r0; jj < r0 + m; ++jj) {
                            const int i = rep_edge[jj];
                            if (i >= 0 && i < ne) before += clampi(q0 - sq[i], 0, ms[i]);
                        }
                    }
                } else {
                    while (j < r0 + m && !(rep_edge[j] >= 0 && rep_edge[j] < ne && ev[rep_edge[j]] >= g)) ++j;
                    if (j < r0 + m) {
                        const int i = rep_edge[j];
                        if (ev[i] == g) before = clampi(q0 - sq[i] - ms[i], 0, tk[i] - ms[i]);
                    }
                }
                out = osz[g * E + e] + before;
            } else if (m == 0) {
                out = osz[h * E + e] + (h < g ? cnt_s[h * E + e] : 0) + q0;
            } else {
                out = q0;
            }
            base[g * E + e] = out;
            if (!((hm >> g) & 1ull)) q0 += cnt_s[g * E + e];
        }
    }
    for (int i = tid; i < ne; i += blockDim.x) {
        const int e = ee[i], v = ev[i];
        seg_qoff[i] = sq[i];
        seg_cum[i] = sc[i];
        seg_rep[i] = (e >= 0 && e < E && v >= 0 && v < G) ? osz[v * E + e] : 0;
    }
    __syncthreads();
    LB_TICK(23);
    if (tid == 0 && bad) flag(LB_DEV_BAD_SPLIT);
    __syncthreads();
}

__global__ void __launch_bounds__(PREP_THREADS) prep_kernel(const Args a) {
    extern __shared__ __align__(16) uint8_t sm[];
    prep_problem(a, blockIdx.x, sm);
}

// ---- scatter ---------------------------------------------------------------
// Peers of this lane's expert id among the warp's lanes (bit-by-bit ballots:
// a fixed log2(E) collectives, where __match_any_sync serialises over the
// distinct values in the warp).  Lanes with e < 0 are excluded.
__device__ __forceinline__ unsigned warp_peers(int e, int nbits) {
    unsigned m = __ballot_sync(kFull, e >= 0);
    for (int bit = 0; bit < nbits; ++bit) {
        const bool on = (e >> bit) & 1;
        const unsigned bb = __ballot_sync(kFull, on);
        m &= on ? bb : ~bb;
    }
    return m;
}

struct ScatterView {
    uint64_t *hold;     // [E]
    int32_t *rcnt;      // [E] replica edges of e
    int32_t *rep0;      // [E+1] first CSR position of e
    int32_t *homecnt;   // [E] cnt[home(e), e]
    int32_t *homeoff;   // [E] offs[home(e)*E + e]
    int32_t *base;      // [SC_WARPS][EP] block bases (row 0 only in CTA mode)
    int32_t *wcnt;      // [SC_WARPS][EP]
    int32_t *pre;       // [SC_WARPS][EP] (CTA mode) / unused
    int32_t *s_qoff, *s_tok, *s_mass, *s_cum, *s_rep, *s_v, *s_vcnt;   // [GN] per CSR position
};

__device__ inline ScatterView scatter_carve(uint8_t *sm, int G, int E, int N) {
    const int GN = G * N, EP = E + 1;
    ScatterView v;
    v.hold = reinterpret_cast<uint64_t *>(sm);
    v.rcnt = reinterpret_cast<int32_t *>(v.hold + E);
    v.rep0 = v.rcnt + E;
    v.homecnt = v.rep0 + E + 1;
    v.homeoff = v.homecnt + E;
    v.base = v.homeoff + E;
    v.wcnt = v.base + SC_WARPS * EP;
    v.pre = v.wcnt + SC_WARPS * EP;
    v.s_qoff = v.pre + SC_WARPS * EP;
    v.s_tok = v.s_qoff + GN;
    v.s_mass = v.s_tok + GN;
    v.s_cum = v.s_mass + GN;
    v.s_rep = v.s_cum + GN;
    v.s_v = v.s_rep + GN;
    v.s_vcnt = v.s_v + GN;
    return v;
}

// Per-problem tables every block shares (built once per CTA): holder masks,
// replica segments in per-expert CSR order (start in q, tok, mass, mass of
// earlier segments, bucket start on the replica rank, replica rank, the
// replica rank's own count of e), and per expert its home bucket start and
// home count.  The per-block terms are added per assignment.
__device__ void scatter_setup(const Args &a, int b, const ScatterView &v) {
    const int G = a.G, E = a.E, N = a.N, GN = G * N, NK = G * E;
    const int tid = threadIdx.x;
    const int32_t *cnt = a.cnt + static_cast<int64_t>(b) * NK;
    const uint8_t *blob = a.plan + static_cast<size_t>(b) * a.plan_stride;
    const plan::Layout LY = plan::layout(G, E, N);
    const int32_t *hdr = reinterpret_cast<const int32_t *>(blob + LY.hdr);
    const int32_t *p_ev = reinterpret_cast<const int32_t *>(blob + LY.edge_v);
    const int32_t *p_rep_ptr = reinterpret_cast<const int32_t *>(blob + LY.rep_ptr);
    const int32_t *p_rep_edge = reinterpret_cast<const int32_t *>(blob + LY.rep_edge);
    const int32_t *tok = a.tok + static_cast<int64_t>(b) * GN;
    const int32_t *mass = a.mass + static_cast<int64_t>(b) * GN;
    const int32_t *offs = a.offs + static_cast<int64_t>(b) * (NK + 1);
    const int32_t *ws = a.ws + static_cast<size_t>(b) * a.ws_stride;
    const int32_t *seg_qoff = ws + NK;
    const int32_t *seg_cum = seg_qoff + GN;
    const int32_t *seg_rep = seg_cum + GN;
    const int Eg = E / G;
    int ne = hdr[0];
    if (ne < 0 || ne > GN) ne = 0;
    for (int e = tid; e <= E; e += blockDim.x) v.rep0[e] = p_rep_ptr[e];
    // per CSR position j (parallel): segment data
    for (int j = tid; j < ne; j += blockDim.x) {
        const int i = p_rep_edge[j];
        const bool ok = i >= 0 && i < ne;
        const int w = ok ? p_ev[i] : -1;
        if (!ok || w < 0 || w >= G) {
            v.s_tok[j] = 0;   // an empty segment: never matched
            v.s_qoff[j] = 0x7fffffff;
            v.s_v[j] = 0;
            continue;
        }
        v.s_qoff[j] = seg_qoff[i];
        v.s_tok[j] = tok[i];
        v.s_mass[j] = mass[i];
        v.s_cum[j] = seg_cum[i];
        v.s_rep[j] = seg_rep[i];
        v.s_v[j] = w;
    }
    __syncthreads();
    for (int j = tid; j < ne; j += blockDim.x) {
        // the expert of CSR position j: last e with rep0[e] <= j
        int lo = 0, hi = E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (v.rep0[mid] <= j) lo = mid; else hi = mid - 1;
        }
        v.s_vcnt[j] = cnt[v.s_v[j] * E + lo];
    }
    for (int e = tid; e < E; e += blockDim.x) {
        const int h = e / Eg;
        int r0 = v.rep0[e], r1 = v.rep0[e + 1];
        if (r0 < 0 || r1 > ne || r1 < r0) r0 = r1 = 0;
        uint64_t hm = 1ull << h;
        for (int j = r0; j < r1; ++j)
            if (v.s_tok[j] > 0 || v.s_qoff[j] != 0x7fffffff) hm |= 1ull << v.s_v[j];
        v.hold[e] = hm;
        v.rcnt[e] = r1 - r0;
        v.homecnt[e] = cnt[h * E + e];
        v.homeoff[e] = offs[h * E + e];
    }
    __syncthreads();
}

// Destination rank and permutation slot of an assignment of expert e from
// source block g whose rank among the block's earlier assignments of e is
// rho; bse = base[g, e].  Returns false if the tables do not place it.
__device__ __forceinline__ bool place(const ScatterView &v, int Eg, int g, int e, int bse, int rho, int &d, int &p) {
    const uint64_t hm = v.hold[e];
    if ((hm >> g) & 1ull) {
        d = g;
        p = bse + rho;
        return true;
    }
    const int h = e / Eg;
    const int m = v.rcnt[e];
    if (m == 0) {
        d = h;
        p = bse + rho;
        return true;
    }
    const int q = bse + rho;
    // last segment starting at or before q (starts ascend along the CSR)
    int lo = v.rep0[e], hi = lo + m - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (v.s_qoff[mid] <= q) lo = mid; else hi = mid - 1;
    }
    const int qo = v.s_qoff[lo], t = v.s_tok[lo];
    if (!(q >= qo && q < qo + t)) return false;
    const int w = q - qo, mss = v.s_mass[lo];
    if (w < mss) {
        d = h;
        p = v.homeoff[e] + (h < g ? v.homecnt[e] : 0) + v.s_cum[lo] + w;
    } else {
        const int r = v.s_v[lo];
        d = r;
        p = v.s_rep[lo] + (r < g ? v.s_vcnt[lo] : 0) + (w - mss);
    }
    return true;
}

// Whole blocks, one per warp (blocks g0, g0 + SC_WARPS, ... below g1): the
// warp walks the block's assignments 32 at a time in order, ranking each
// among the earlier ones of its expert with bit-ballot peers and a per-warp
// running count in shared memory.  No block-wide barrier.
__device__ void scatter_blocks_warp(const Args &a, int b, int g0, int g1, const ScatterView &v, int *bad) {
    const int G = a.G, E = a.E, k = a.k, EP = E + 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int Eg = E / G, Tg = a.T / G, nitems = Tg * k, nf = a.T * k;
    const int nbits = E > 1 ? 32 - __clz(E - 1) : 1;
    const int32_t *ids = a.ids + static_cast<int64_t>(b) * a.T * k;
    int32_t *dest = a.dest + static_cast<int64_t>(b) * a.T * k;
    int32_t *perm = a.perm + static_cast<int64_t>(b) * a.T * k;
    const int32_t *wsb = a.ws + static_cast<size_t>(b) * a.ws_stride;
    int32_t *cntw = v.wcnt + warp * EP;
    int32_t *basew = v.base + warp * EP;
    for (int g = g0 + warp; g < g1; g += SC_WARPS) {
        for (int e = lane; e < E; e += 32) {
            cntw[e] = 0;
            basew[e] = wsb[g * E + e];
        }
        __syncwarp();
        const int64_t f0 = static_cast<int64_t>(g) * nitems;
        for (int i0 = 0; i0 < nitems; i0 += 32) {
            const int i = i0 + lane;
            int e = -1;
            if (i < nitems) {
                e = __ldg(ids + f0 + i);
                if (e < 0 || e >= E) {
                    *bad = 1;
                    e = -1;
                }
            }
            const unsigned peers = warp_peers(e, nbits);
            const int rnk = __popc(peers & lanemask_lt());
            const int cur = e >= 0 ? cntw[e] : 0;
            __syncwarp();
            if (e >= 0 && lane == 31 - __clz(peers)) cntw[e] = cur + __popc(peers);
            if (e >= 0) {
                int d, pp;
                if (place(v, Eg, g, e, basew[e], cur + rnk, d, pp) && pp >= 0 && pp < nf) {
                    dest[f0 + i] = d;
                    perm[pp] = static_cast<int32_t>(f0 + i);
                } else {
                    *bad = 1;
                }
            }
            __syncwarp();
        }
    }
}

// Assignments [i0, i1) of one block by the whole CTA (large blocks): warps
// take consecutive 32-assignment steps, then a shuffle scan across warps
// turns per-warp counts into block-order ranks.  `prefix` (shared memory,
// E entries) holds each expert's assignments in the block before i0, or is
// null when i0 == 0.
__device__ void scatter_block_cta(const Args &a, int b, int g, int i0, int i1, const int32_t *prefix,
                                  const ScatterView &v, int *bad) {
    const int G = a.G, E = a.E, k = a.k, EP = E + 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Eg = E / G, Tg = a.T / G, nitems = Tg * k, nf = a.T * k;
    const int nbits = E > 1 ? 32 - __clz(E - 1) : 1;
    const int64_t f0 = static_cast<int64_t>(g) * nitems;
    const int32_t *ids = a.ids + static_cast<int64_t>(b) * a.T * k;
    int32_t *dest = a.dest + static_cast<int64_t>(b) * a.T * k;
    int32_t *perm = a.perm + static_cast<int64_t>(b) * a.T * k;
    const int32_t *wsb = a.ws + static_cast<size_t>(b) * a.ws_stride;
    int32_t *run = v.base + EP;   // row 1 of the base table: running counts
    for (int e = tid; e < E; e += blockDim.x) {
        v.base[e] = wsb[g * E + e];
        run[e] = prefix != nullptr ? prefix[e] : 0;
    }
    __syncthreads();
    constexpr int CH = SC_WARPS * 32 * SC_STEPS;
    int32_t *wrow = v.wcnt + warp * EP;
    const int iend = min(i1, nitems);
    for (int cs = i0; cs < iend; cs += CH) {
        for (int e = lane; e < E; e += 32) wrow[e] = 0;
        __syncwarp();
        int es[SC_STEPS], loc[SC_STEPS];
#pragma unroll
        for (int s = 0; s < SC_STEPS; ++s) {
            const int i = cs + warp * 32 * SC_STEPS + s * 32 + lane;
            es[s] = i < iend ? __ldg(ids + f0 + i) : -1;
        }
#pragma unroll
        for (int s = 0; s < SC_STEPS; ++s) {
            int e = es[s];
            if (e >= E || e < -1 || (e == -1 && cs + warp * 32 * SC_STEPS + s * 32 + lane < iend)) {
                *bad = 1;
                e = -1;
            }
            const unsigned peers = warp_peers(e, nbits);
            const int rnk = __popc(peers & lanemask_lt());
            const int cur = e >= 0 ? wrow[e] : 0;
            __syncwarp();
            if (e >= 0 && lane == 31 - __clz(peers)) wrow[e] = cur + __popc(peers);
            __syncwarp();
            es[s] = e;
            loc[s] = cur + rnk;
        }
        __syncthreads();
        for (int e = warp; e < E; e += SC_WARPS) {
            const int c = v.wcnt[lane * EP + e];
            int x = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(kFull, x, off);
                if (lane >= off) x += y;
            }
            const int r = run[e];
            v.pre[lane * EP + e] = r + x - c;
            __syncwarp();
            if (lane == 31) run[e] = r + x;
        }
        __syncthreads();
#pragma unroll
        for (int s = 0; s < SC_STEPS; ++s) {
            const int e = es[s];
            if (e < 0) continue;
            const int i = cs + warp * 32 * SC_STEPS + s * 32 + lane;
            int d, pp;
            if (place(v, Eg, g, e, v.base[e], v.pre[warp * EP + e] + loc[s], d, pp) && pp >= 0 && pp < nf) {
                dest[f0 + i] = d;
                perm[pp] = static_cast<int32_t>(f0 + i);
            } else {
                *bad = 1;
            }
        }
        __syncthreads();   // pre/run are rewritten by the next chunk
    }
    __syncthreads();
}

// Scatter kernel: CTA (x, problem y).  Small blocks: CTA x takes blocks
// [x*SC_WARPS, (x+1)*SC_WARPS), one per warp.  Large blocks: CTA x takes
// block x.
__global__ void __launch_bounds__(SC_THREADS) scatter_kernel(const Args a) {
    extern __shared__ __align__(16) uint8_t sm[];
    __shared__ int bad;
    if (threadIdx.x == 0) bad = 0;
    const ScatterView v = scatter_carve(sm, a.G, a.E, a.N);
    LB_TICK(10);
    scatter_setup(a, blockIdx.y, v);
    LB_TICK(11);
    const int nitems = (a.T / a.G) * a.k;
    if (nitems <= WARP_BLOCK_MAX) {
        const int g0 = blockIdx.x * SC_WARPS;
        scatter_blocks_warp(a, blockIdx.y, g0, min(a.G, g0 + SC_WARPS), v, &bad);
        __syncthreads();
    } else {
        scatter_block_cta(a, blockIdx.y, blockIdx.x, 0, nitems, nullptr, v, &bad);
    }
    LB_TICK(12);
    if (threadIdx.x == 0 && bad) flag(LB_DEV_BAD_SPLIT);
}

}  // namespace assign
}  // namespace lb
