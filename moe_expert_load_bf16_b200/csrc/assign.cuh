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
// The prep kernel (one CTA per problem, or a cluster of 8 CTAs per problem
// when one problem's key table is large) computes these from cnt, plan and
// split without reading the ids; counts and plan are staged in shared memory
// first.  The scatter kernel (one CTA per (problem, source block) or slice
// of one, or one warp per block when many problems' small blocks fill the
// GPU) then needs only each assignment's rank among the earlier assignments
// of the same expert in its block: in the CTA forms with top-k up to 8, one
// token per lane and per-warp lane masks of each expert (the rank is the
// count of earlier lanes holding it); otherwise warps take consecutive
// 32-assignment steps and find each lane's peers (same expert) with one
// ballot per bit of the expert id.
// Per-warp counters in shared memory and a per-expert scan down the warps'
// counters keep block order, and each assignment's slot is base + rank, or,
// for a replicated expert's remote assignment, found by searching the
// expert's replica segments (staged in shared memory).  Positions never come
// from atomics, so the permutation is deterministic and stable.
#pragma once
#include "common.cuh"
#include "maskbits.cuh"
#include "plan.cuh"

namespace lb {
namespace assign {

constexpr int PREP_THREADS = 1024;
constexpr int SC_THREADS = 1024;   // scatter CTA for one problem's latency (the throughput launch uses 512)
constexpr int SC_WARPS = SC_THREADS / 32;
constexpr int SC_STEPS = 8;   // 32-assignment steps per warp per chunk
constexpr int TOK_QUEUE = 256;   // token path: queued slots per warp (32 lanes x 8 ids)

// Workspace per problem (int32 words): base[G*E], seg_qoff[GN], seg_cum[GN],
// seg_rep[GN]; rounded to 256 bytes.
__host__ __device__ inline size_t ws_words(int G, int E, int N) {
    const size_t w = static_cast<size_t>(G) * E + 3 * static_cast<size_t>(G) * N;
    return (w + 63) & ~static_cast<size_t>(63);
}

__host__ __device__ inline size_t prep_smem_bytes(int G, int E, int N) {
    const size_t GN = static_cast<size_t>(G) * N;
    return static_cast<size_t>(E) * 8 + static_cast<size_t>(G) * E * 4 * 2 + static_cast<size_t>(E) * 4 * 3 +
           (static_cast<size_t>(E) + 1) * 4 + GN * 4 * 7 + static_cast<size_t>(E) * 4 * 11 + 64;
}

// Shared memory of the scatter: per-expert tables (holders, replica count,
// CSR start, home count), the per-(CTA or warp) block bases and running
// counts, the per-warp counter tables, and the replica segments.
__host__ __device__ inline size_t scatter_smem_bytes(int G, int E, int N, int nw = SC_WARPS) {
    const size_t GN = static_cast<size_t>(G) * N, EP = static_cast<size_t>(E) + 1;
    return static_cast<size_t>(E) * 8 + static_cast<size_t>(E) * 4 * 6 + (static_cast<size_t>(E) + 1) * 4 +
           static_cast<size_t>(nw) * EP * 4 * 3 + static_cast<size_t>(nw) * TOK_QUEUE * 8 + GN * 4 * 7 + 64;
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
    int slices = 1;     // scatter CTAs per large source block (token-aligned slices)
    int cta_blocks = 0; // 1: small blocks (<= WARP_BLOCK_MAX assignments) one per CTA as well
};

__device__ __forceinline__ int clampi(int x, int lo, int hi) { return min(max(x, lo), hi); }

// Exclusive scan of one 64-bit value per thread over the CTA (every thread
// calls it; wtot is 32 words of shared memory); `total` gets the CTA's sum.
__device__ __forceinline__ uint64_t cta_exclusive_scan_u64(uint64_t x, uint64_t *wtot, uint64_t &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint64_t s = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint64_t y = __shfl_up_sync(kFull, s, off);
        if (lane >= off) s += y;
    }
    if (lane == 31) wtot[warp] = s;
    __syncthreads();
    if (warp == 0) {
        uint64_t w = lane < nw ? wtot[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint64_t y = __shfl_up_sync(kFull, w, off);
            if (lane >= off) w += y;
        }
        if (lane < nw) wtot[lane] = w;   // inclusive per warp
    }
    __syncthreads();
    const uint64_t before = warp > 0 ? wtot[warp - 1] : 0;
    total = wtot[nw - 1];
    __syncthreads();   // wtot is reused by the next call
    return before + s - x;
}

// Tables of problem b for its scatter: offs, base[g,e], replica segments.
// All threads of the CTA call it; `sm` holds prep_smem_bytes(G,E,N) bytes.
__device__ void prep_problem(const Args &a, int b, uint8_t *sm, int C = 1, int c = 0) {
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
    int32_t *csum = osz + NK;        // [E][8] remote counts per chunk of 8 blocks
    int32_t *qh = csum + E * 8;      // [E] remote assignments before the home block
    int32_t *bh = qh + E;            // [E] the home block's share of the edges' segments
    int32_t *hc = bh + E;            // [E] cnt[home(e), e] (the counts' table then holds q0)
    __shared__ int wsum[32];
    __shared__ uint64_t wscan[32];
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
    // a cluster of C CTAs shares one problem (C divides G): CTA c owns the
    // (rank, expert) keys of ranks [rlo, rhi); the per-expert work is done by
    // every CTA, the per-key work by the owner, the scan's carries and the
    // few home-rank offsets a CTA needs from another cross over distributed
    // shared memory
    const int rlo = c * (G / C), rhi = rlo + G / C;
    const int K0 = rlo * E, K1 = rhi * E;
    __shared__ int cta_total;
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
    // per-expert scratch of the segment scan below (the arrays' own contents
    // are written later): the scan's value at e's first CSR position and
    // past its last, for tok (high word) and mass (low word)
    int32_t *hT = rcnt, *hM = rtot, *eT = homeadd, *eM = qh;
    for (int e = tid; e < E; e += blockDim.x) {
        hold[e] = 0ull;
        hT[e] = hM[e] = eT[e] = eM[e] = 0;
    }
    __syncthreads();
    LB_TICK(60);

    // ---- per CSR position j (in parallel: a hot expert's tens of edges
    // would otherwise be one thread's serial walk): its edge and expert
    // (checked against the expert's CSR range), the holder bit, and an
    // exclusive scan of (tok, mass) over the positions.  A segment's start
    // in q (and its mass before) is the scan at its position less the scan
    // at its expert's first position.
    {
        uint64_t carry = 0;
        for (int j0 = 0; j0 < ne; j0 += blockDim.x) {   // ne is the same in every thread
            const int j = j0 + tid;
            int i = -1, e = -1;
            uint64_t val = 0;
            if (j < ne) {
                i = rep_edge[j];
                if (i >= 0 && i < ne) {
                    e = ee[i];
                    const int v = ev[i];
                    if (e < 0 || e >= E || v < 0 || v >= G || j < rep_ptr[e] || j >= rep_ptr[e + 1]) {
                        e = -1;
                    } else {
                        or_bit64(&hold[e], v);
                        val = (static_cast<uint64_t>(static_cast<uint32_t>(tk[i])) << 32) |
                              static_cast<uint32_t>(ms[i]);
                    }
                }
                if (e < 0) bad = 1;
            }
            uint64_t tot;
            const uint64_t x = carry + cta_exclusive_scan_u64(val, wscan, tot);
            carry += tot;
            if (e >= 0) {
                sq[i] = static_cast<int>(x >> 32);   // made relative to the expert's first position below
                sc[i] = static_cast<int>(static_cast<uint32_t>(x));
                if (j == rep_ptr[e]) {
                    hT[e] = static_cast<int>(x >> 32);
                    hM[e] = static_cast<int>(static_cast<uint32_t>(x));
                }
                if (j == rep_ptr[e + 1] - 1) {
                    eT[e] = static_cast<int>((x + val) >> 32);
                    eM[e] = static_cast<int>(static_cast<uint32_t>(x + val));
                }
            }
        }
    }
    __syncthreads();
    LB_TICK(61);

    // ---- remote counts of e per chunk of 8 blocks (blocks that hold no copy
    // of e); per edge, its segment's start relative to its expert's first
    const int nch = (G + 7) >> 3;
    for (int x = tid; x < E * nch; x += blockDim.x) {
        const int e = x % E, ch = x / E;
        const uint64_t hm = hold[e] | (1ull << (e / Eg));
        int sum = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int g = ch * 8 + u;
            if (g < G && !((hm >> g) & 1ull)) sum += cnt_s[g * E + e];
        }
        csum[e * 8 + ch] = sum;
    }
    for (int i = tid; i < ne; i += blockDim.x) {
        const int e = ee[i];
        if (e >= 0 && e < E) {
            sq[i] -= hT[e];
            sc[i] -= hM[e];
        }
    }
    __syncthreads();
    LB_TICK(62);

    // ---- per expert: holders, remote total, remote assignments before the
    // home block (q0 there), the home count
    for (int e = tid; e < E; e += blockDim.x) {
        const int h = e / Eg;
        int r0 = rep_ptr[e], r1 = rep_ptr[e + 1];
        if (r0 < 0 || r1 > ne || r1 < r0) {
            bad = 1;
            r0 = r1 = 0;
        }
        const uint64_t hm = hold[e] | (1ull << h);
        // (the scan's scratch shares these arrays: read before they are written)
        const int qo = r1 > r0 ? eT[e] - hT[e] : 0, cm = r1 > r0 ? eM[e] - hM[e] : 0;
        int R = 0, qhome = 0;
        for (int c2 = 0; c2 < nch; ++c2) {
            const int cs = csum[e * 8 + c2];
            R += cs;
            qhome += c2 < (h >> 3) ? cs : 0;
        }
        for (int g = h & ~7; g < h; ++g)
            if (!((hm >> g) & 1ull)) qhome += cnt_s[g * E + e];
        if (r1 > r0 && qo != R) bad = 1;
        hold[e] = hm;
        rcnt[e] = r1 - r0;
        rtot[e] = R;
        homeadd[e] = (r1 > r0) ? cm : R;
        qh[e] = qhome;
        bh[e] = 0;
        hc[e] = cnt_s[h * E + e];
    }
    __syncthreads();
    LB_TICK(21);

    // ---- bucket sizes over keys r*E+e: own tokens of held experts, the home
    // share of each expert, and every edge's replica share (tok - mass)
    for (int r = rlo + warp; r < rhi; r += (blockDim.x >> 5)) {
        for (int e = lane; e < E; e += 32) {
            const uint64_t hm = hold[e];
            int sz = ((hm >> r) & 1ull) ? cnt_s[r * E + e] : 0;
            sz += (e >= r * Eg && e < (r + 1) * Eg) ? homeadd[e] : 0;
            osz[r * E + e] = sz;
        }
    }
    __syncthreads();
    LB_TICK(24);
    for (int i = tid; i < ne; i += blockDim.x) {
        const int e = ee[i], v = ev[i];
        if (e >= 0 && e < E && v >= rlo && v < rhi) osz[v * E + e] += tk[i] - ms[i];   // one edge per (v, e)
    }
    __syncthreads();
    LB_TICK(25);
    // block-wide exclusive scan, in place: warp w scans its contiguous
    // segment of keys 32 at a time (conflict-free, coalesced), then the warp
    // totals are scanned and added back; offs (global) gets a copy
    {
        const int nw = blockDim.x >> 5;
        const int seg = ((K1 - K0 + nw - 1) / nw + 31) & ~31;
        const int s0 = min(K1, K0 + warp * seg), s1 = min(K1, s0 + seg);
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
            const int wc = lane < nw ? wsum[lane] : 0;
            int x = wc;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(kFull, x, off);
                if (lane >= off) x += y;
            }
            if (lane < nw) wsum[lane] = x - wc;   // exclusive per warp
            if (lane == nw - 1) cta_total = x;
        }
        __syncthreads();
        LB_TICK(26);
        // the keys of lower-ranked CTAs come first
        int pre = 0;
        if (C > 1) {
            cluster_sync();
            // (every warp reads the lower CTAs' totals at once, one per lane)
            const int t = lane < c ? ld_cluster_i32(mapa_shared(smem_u32(&cta_total), static_cast<uint32_t>(lane))) : 0;
            pre = __reduce_add_sync(kFull, t);
        }
        LB_TICK(27);
        if (c == C - 1 && tid == 0) offs[NK] = pre + cta_total;
        const int add = wsum[warp] + pre;
        for (int key = s0 + lane; key < s1; key += 32) {
            const int o = osz[key] + add;
            osz[key] = o;
            offs[key] = o;
        }
    }
    __syncthreads();
    LB_TICK(22);

    // ---- base per (block g, expert e).  q0(g, e) = remote assignments of e
    // in the blocks before g (blocks that hold no copy of e).  In parallel
    // steps: (1) q0 of the own rows' blocks from the chunk sums above,
    // written over the counts' table in shared memory (each count is read
    // before its slot is overwritten; the home counts were kept in hc, q0 at
    // the home block in qh); (2) per edge, the home block's share of its
    // segment and the replica holder's base; (3) every other (g, e).
    {
        const int ch0 = rlo >> 3, ch1 = (rhi + 7) >> 3;
        for (int x = tid; x < E * (ch1 - ch0); x += blockDim.x) {
            const int e = x % E, ch = ch0 + x / E;
            const uint64_t hm = hold[e];
            int q0 = 0;
            for (int c2 = 0; c2 < ch; ++c2) q0 += csum[e * 8 + c2];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int g = ch * 8 + u;
                if (g >= G) break;
                const int cg = cnt_s[g * E + e];
                if (g >= rlo && g < rhi) cnt_s[g * E + e] = q0;
                if (!((hm >> g) & 1ull)) q0 += cg;
            }
        }
    }
    LB_TICK(28);
    __syncthreads();
    LB_TICK(29);
    for (int i = tid; i < ne; i += blockDim.x) {
        // (in a plan every edge of e sits once in e's list; a list that does
        // not match its edges was flagged above)
        const int e = ee[i], v = ev[i];
        if (e < 0 || e >= E || v < 0 || v >= G || rcnt[e] == 0) continue;
        atomicAdd(&bh[e], clampi(qh[e] - sq[i], 0, ms[i]));
        if (v != e / Eg && v >= rlo && v < rhi && ((hold[e] >> v) & 1ull)) {
            const int q0 = cnt_s[v * E + e];
            base[v * E + e] = osz[v * E + e] + clampi(q0 - sq[i] - ms[i], 0, tk[i] - ms[i]);
        }
    }
    __syncthreads();
    LB_TICK(55);
    if (C > 1) cluster_sync();   // every CTA's offsets final before the home-rank reads below
    LB_TICK(56);
    for (int x = K0 + tid; x < K1; x += blockDim.x) {
        const int g = x / E, e = x - g * E;
        const int h = e / Eg;
        const uint64_t hm = hold[e];
        const bool held = (hm >> g) & 1ull;
        if (held && g != h) continue;   // replica holders: set in (3)
        const int m = rcnt[e], q0 = cnt_s[x];
        int out;
        if (held) {
            out = osz[x] + (m == 0 ? q0 : bh[e]);
        } else if (m == 0) {
            // the home rank's offset, from its owner (all scans are done:
            // the cluster barrier above)
            const int oh = (h >= rlo && h < rhi)
                               ? osz[h * E + e]
                               : ld_cluster_i32(mapa_shared(smem_u32(&osz[h * E + e]),
                                                            static_cast<uint32_t>(h / (G / C))));
            out = oh + (h < g ? hc[e] : 0) + q0;
        } else {
            out = q0;
        }
        base[x] = out;
    }
    LB_TICK(57);
    for (int i = tid; i < ne; i += blockDim.x) {
        const int e = ee[i], v = ev[i];
        const bool ok = e >= 0 && e < E && v >= 0 && v < G;
        if (c == 0) {
            seg_qoff[i] = sq[i];
            seg_cum[i] = sc[i];
            if (!ok) seg_rep[i] = 0;
        }
        if (ok && v >= rlo && v < rhi) seg_rep[i] = osz[v * E + e];   // by the rank's owner
    }
    __syncthreads();
    LB_TICK(23);
    if (tid == 0 && bad) flag(LB_DEV_BAD_SPLIT);
    __syncthreads();
    if (C > 1) cluster_sync();   // no CTA leaves while another reads its offsets
}

// Both prep kernels (and the fused decide kernel without its plan step) let
// the scatter launch as soon as every CTA has passed its own wait (the
// scatter then builds its tables from the counts and the plan, and waits for
// its predecessor to complete before reading the split and the prep's
// outputs).
__device__ __forceinline__ void pdl_signal_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__global__ void __launch_bounds__(PREP_THREADS) prep_kernel(const Args a) {
    extern __shared__ __align__(16) uint8_t sm[];
    pdl_begin();
    pdl_signal_dependents();
    prep_problem(a, blockIdx.x, sm);
}

// One problem per cluster of gridDim.x CTAs (each owning G / gridDim.x ranks
// of the key table), for a single problem's latency when G x E is large.
__global__ void __launch_bounds__(PREP_THREADS) prep_kernel_cluster(const Args a) {
    extern __shared__ __align__(16) uint8_t sm[];
    pdl_begin();
    pdl_signal_dependents();
    prep_problem(a, blockIdx.y, sm, static_cast<int>(gridDim.x), static_cast<int>(cluster_ctarank()));
}

// ---- scatter ---------------------------------------------------------------
// Peers of this lane's expert id among the warp's lanes (bit-by-bit ballots:
// a fixed NB collectives, where __match_any_sync serialises over the distinct
// values in the warp).  Lanes with e < 0 are excluded.  NB >= the bits of the
// largest id; extra bits are zero for every valid id and change nothing.
template <int NB>
__device__ __forceinline__ unsigned warp_peers(int e) {
    unsigned m = __ballot_sync(kFull, e >= 0);
#pragma unroll
    for (int bit = 0; bit < NB; ++bit) {
        const unsigned on = (e >> bit) & 1u;
        const unsigned bb = __ballot_sync(kFull, on);
        m &= bb ^ (on - 1u);   // bb where the bit is set, ~bb where it is clear
    }
    return m;
}

struct ScatterView {
    uint64_t *hold;     // [E]
    int32_t *rcnt;      // [E] replica edges of e
    int32_t *rep0;      // [E+1] first CSR position of e
    int32_t *homecnt;   // [E] cnt[home(e), e]
    int32_t *homeoff;   // [E] offs[home(e)*E + e]
    int32_t *home;      // [E] home(e)
    int32_t *cls;       // [E] CTA mode: class of e for the CTA's source block (see scatter_block_cta)
    int32_t *sfirst;    // [E] CTA mode: replica segment of the block's first remote rank of e
    int32_t *base;      // [warps][EP] block bases (row 0 only in CTA mode)
    int32_t *wcnt;      // [warps][EP] per-warp counts (CTA mode: scanned in place into prefixes)
    uint32_t *lmask;    // [warps][EP] token path: lanes whose token holds e (kept zero between steps)
    int2 *queue;        // [warps][TOK_QUEUE] token path: slots of replicated experts' remote assignments
    int32_t *s_qoff, *s_tok, *s_mass, *s_cum, *s_rep, *s_v, *s_vcnt;   // [GN] per CSR position
};

__device__ inline ScatterView scatter_carve(uint8_t *sm, int G, int E, int N, int nw = SC_WARPS) {
    const int GN = G * N, EP = E + 1;
    ScatterView v;
    v.hold = reinterpret_cast<uint64_t *>(sm);
    v.queue = reinterpret_cast<int2 *>(v.hold + E);   // 8-byte aligned after the 8-byte masks
    v.rcnt = reinterpret_cast<int32_t *>(v.queue + nw * TOK_QUEUE);
    v.rep0 = v.rcnt + E;
    v.homecnt = v.rep0 + E + 1;
    v.homeoff = v.homecnt + E;
    v.home = v.homeoff + E;
    v.cls = v.home + E;
    v.sfirst = v.cls + E;
    v.base = v.sfirst + E;
    v.wcnt = v.base + nw * EP;
    v.lmask = reinterpret_cast<uint32_t *>(v.wcnt + nw * EP);
    v.s_qoff = reinterpret_cast<int32_t *>(v.lmask + nw * EP);
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
//
// In two parts.  scatter_setup_inputs reads only the counts and the plan
// (inputs that were final before the scatter's predecessor started); the
// scatter kernel runs it before waiting on that predecessor (the prep, or
// the fused decide kernel without its plan step), which signals its
// dependents as soon as it is past its own wait, so this part overlaps it.
// scatter_setup_tables then reads the split (tok, mass) and the prep's
// outputs (segment starts, replica bucket starts, offsets).  A kernel that
// precedes the scatter and writes the counts or the plan must not signal
// early.
__device__ void scatter_setup_inputs(const Args &a, int b, const ScatterView &v) {
    const int G = a.G, E = a.E, N = a.N, GN = G * N, NK = G * E;
    const int tid = threadIdx.x;
    const int32_t *cnt = a.cnt + static_cast<int64_t>(b) * NK;
    const uint8_t *blob = a.plan + static_cast<size_t>(b) * a.plan_stride;
    const plan::Layout LY = plan::layout(G, E, N);
    const int32_t *hdr = reinterpret_cast<const int32_t *>(blob + LY.hdr);
    const int32_t *p_ev = reinterpret_cast<const int32_t *>(blob + LY.edge_v);
    const int32_t *p_rep_ptr = reinterpret_cast<const int32_t *>(blob + LY.rep_ptr);
    const int32_t *p_rep_edge = reinterpret_cast<const int32_t *>(blob + LY.rep_edge);
    const int Eg = E / G;
    // (loads through L2 only: the data is a completed kernel's output, read
    // before this kernel's wait)
    int ne = __ldcg(hdr);
    if (ne < 0 || ne > GN) ne = 0;
    for (int e = tid; e <= E; e += blockDim.x) v.rep0[e] = __ldcg(p_rep_ptr + e);
    for (int e = tid; e < E; e += blockDim.x) v.hold[e] = 1ull << (e / Eg);   // home; replica holders ORed below
    // per CSR position j (parallel): segment data; s_qoff marks a position
    // invalid (and holds 0 otherwise until the tables' part), s_cum holds
    // the edge index until then
    for (int j = tid; j < ne; j += blockDim.x) {
        const int i = __ldcg(p_rep_edge + j);
        const bool ok = i >= 0 && i < ne;
        const int w = ok ? __ldcg(p_ev + i) : -1;
        if (!ok || w < 0 || w >= G) {
            v.s_tok[j] = 0;   // an empty segment: never matched
            v.s_qoff[j] = 0x7fffffff;
            v.s_v[j] = 0;
            continue;
        }
        v.s_qoff[j] = 0;
        v.s_cum[j] = i;
        v.s_v[j] = w;
    }
    __syncthreads();
    LB_TICK(63);
    for (int j = tid; j < ne; j += blockDim.x) {
        // the expert of CSR position j: last e with rep0[e] <= j
        int lo = 0, hi = E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (v.rep0[mid] <= j) lo = mid; else hi = mid - 1;
        }
        v.s_vcnt[j] = __ldcg(cnt + v.s_v[j] * E + lo);
        if (v.s_qoff[j] != 0x7fffffff) or_bit64(&v.hold[lo], v.s_v[j]);
    }
    LB_TICK(9);
    for (int e = tid; e < E; e += blockDim.x) {
        const int h = e / Eg;
        int r0 = v.rep0[e], r1 = v.rep0[e + 1];
        if (r0 < 0 || r1 > ne || r1 < r0) r0 = r1 = 0;
        v.rcnt[e] = r1 - r0;
        v.homecnt[e] = __ldcg(cnt + h * E + e);
        v.home[e] = h;
    }
    __syncthreads();
}

__device__ void scatter_setup_tables(const Args &a, int b, const ScatterView &v) {
    const int G = a.G, E = a.E, N = a.N, GN = G * N, NK = G * E;
    const int tid = threadIdx.x;
    const uint8_t *blob = a.plan + static_cast<size_t>(b) * a.plan_stride;
    const int32_t *hdr = reinterpret_cast<const int32_t *>(blob + plan::layout(G, E, N).hdr);
    const int32_t *offs = a.offs + static_cast<int64_t>(b) * (NK + 1);
    const int32_t *ws = a.ws + static_cast<size_t>(b) * a.ws_stride;
    const int32_t *seg_qoff = ws + NK;
    const int32_t *seg_cum = seg_qoff + GN;
    const int32_t *seg_rep = seg_cum + GN;
    const int32_t *tok = a.tok + static_cast<int64_t>(b) * GN;
    const int32_t *mass = a.mass + static_cast<int64_t>(b) * GN;
    const int Eg = E / G;
    int ne = hdr[0];
    if (ne < 0 || ne > GN) ne = 0;
    for (int j = tid; j < ne; j += blockDim.x) {
        if (v.s_qoff[j] == 0x7fffffff) continue;
        const int i = v.s_cum[j];
        v.s_tok[j] = tok[i];
        v.s_mass[j] = mass[i];
        v.s_qoff[j] = seg_qoff[i];
        v.s_cum[j] = seg_cum[i];
        v.s_rep[j] = seg_rep[i];
    }
    for (int e = tid; e < E; e += blockDim.x) v.homeoff[e] = offs[(e / Eg) * E + e];
    __syncthreads();
}

__device__ void scatter_setup(const Args &a, int b, const ScatterView &v) {
    scatter_setup_inputs(a, b, v);
    scatter_setup_tables(a, b, v);
}

// Destination rank and permutation slot of an assignment of expert e from
// source block g whose rank among the block's earlier assignments of e is
// rho; bse = base[g, e].  Returns false if the tables do not place it.
// A replicated expert's remote assignment with rank q among e's remote ones:
// the replica segment covering q decides between home(e) and the replica.
__device__ __forceinline__ bool place_remote(const ScatterView &v, int g, int e, int q, int &d, int &p) {
    const int h = v.home[e];
    const int m = v.rcnt[e];
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

__device__ __forceinline__ bool place(const ScatterView &v, int g, int e, int bse, int rho, int &d, int &p) {
    const uint64_t hm = v.hold[e];
    if ((hm >> g) & 1ull) {
        d = g;
        p = bse + rho;
        return true;
    }
    if (v.rcnt[e] == 0) {
        d = v.home[e];
        p = bse + rho;
        return true;
    }
    return place_remote(v, g, e, bse + rho, d, p);
}

// Whole blocks, one per warp (blocks g0, g0 + SC_WARPS, ... below g1): the
// warp walks the block's assignments 32 at a time in order, ranking each
// among the earlier ones of its expert with bit-ballot peers and a per-warp
// running count in shared memory.  No block-wide barrier.
template <int NB>
__device__ void scatter_blocks_warp(const Args &a, int b, int g0, int g1, const ScatterView &v, int *bad) {
    const int G = a.G, E = a.E, k = a.k, EP = E + 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int Tg = a.T / G, nitems = Tg * k, nf = a.T * k;
    const int32_t *ids = a.ids + static_cast<int64_t>(b) * a.T * k;
    int32_t *dest = a.dest + static_cast<int64_t>(b) * a.T * k;
    int32_t *perm = a.perm + static_cast<int64_t>(b) * a.T * k;
    const int32_t *wsb = a.ws + static_cast<size_t>(b) * a.ws_stride;
    const int nw = blockDim.x >> 5;
    int32_t *cntw = v.wcnt + warp * EP;
    int32_t *basew = v.base + warp * EP;
    for (int g = g0 + warp; g < g1; g += nw) {
        for (int e = lane; e < E; e += 32) {
            cntw[e] = 0;
            basew[e] = wsb[g * E + e];
        }
        __syncwarp();
        const int64_t f0 = static_cast<int64_t>(g) * nitems;
        // ids of the next PF steps in flight (a ring of registers), so no step
        // waits on its own global load
        constexpr int PF = 4;
        int ring[PF];
#pragma unroll
        for (int q = 0; q < PF; ++q) ring[q] = (q * 32 + lane < nitems) ? __ldg(ids + f0 + q * 32 + lane) : -1;
        for (int i0 = 0; i0 < nitems; i0 += 32) {
            const int i = i0 + lane;
            int e = ring[0];
#pragma unroll
            for (int q = 0; q + 1 < PF; ++q) ring[q] = ring[q + 1];
            ring[PF - 1] = (i + PF * 32 < nitems) ? __ldg(ids + f0 + i + PF * 32) : -1;
            if (i < nitems && (e < 0 || e >= E)) {
                *bad = 1;
                e = -1;
            }
            if (i >= nitems) e = -1;
            const unsigned peers = warp_peers<NB>(e);
            const int rnk = __popc(peers & lanemask_lt());
            const int cur = e >= 0 ? cntw[e] : 0;
            __syncwarp();
            if (e >= 0 && lane == 31 - __clz(peers)) cntw[e] = cur + __popc(peers);
            if (e >= 0) {
                int d, pp;
                if (place(v, g, e, basew[e], cur + rnk, d, pp) && pp >= 0 && pp < nf) {
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
// take consecutive 32-assignment steps, then a scan down the per-warp counts
// (one thread per expert) turns them into block-order ranks.  `prefix` (shared memory,
// E entries) holds each expert's assignments in the block before i0, or is
// null when i0 == 0.
template <int NB>
__device__ void scatter_block_cta(const Args &a, int b, int g, int i0, int i1, const int32_t *prefix,
                                  const ScatterView &v, int *bad) {
    const int G = a.G, E = a.E, k = a.k, EP = E + 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Tg = a.T / G, nitems = Tg * k, nf = a.T * k;
    const int fbase = g * nitems;   // problem-local index of the block's first assignment
    const int64_t pb = static_cast<int64_t>(b) * a.T * k;
    const int32_t *ids = a.ids + pb + fbase;   // this block's assignments
    int32_t *dest = a.dest + pb + fbase;
    int32_t *perm = a.perm + pb;               // the problem's permutation
    const int32_t *wsb = a.ws + static_cast<size_t>(b) * a.ws_stride;
    int32_t *run = v.base + EP;   // row 1 of the base table: running counts
    // Class of each expert for this source block: (g << 2) | 0 when g holds
    // it (served locally), (home << 2) | 1 when it has no replica (served at
    // home), 2 when it is replicated elsewhere (the split decides).  In the
    // first two classes an assignment's slot is base + rank.  For the third,
    // sfirst[e] is the replica segment holding the block's first remote rank
    // of e here; later ranks only move forward from it.
    for (int e = tid; e < E; e += blockDim.x) {
        const int bse = wsb[g * E + e];
        const int r0 = prefix != nullptr ? prefix[e] : 0;
        v.base[e] = bse;
        run[e] = r0;
        const bool local = (v.hold[e] >> g) & 1ull;
        const int m = v.rcnt[e];
        v.cls[e] = local ? (g << 2) : (m == 0 ? (v.home[e] << 2) | 1 : 2);
        int sf = 0;
        if (!local && m > 0) {
            const int q = bse + r0;
            int lo = v.rep0[e], hi = lo + m - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (v.s_qoff[mid] <= q) lo = mid; else hi = mid - 1;
            }
            sf = lo;
        }
        v.sfirst[e] = sf;
    }
    __syncthreads();
    const int nw = blockDim.x >> 5;
    const int CH = nw * 32 * SC_STEPS;
    int32_t *wrow = v.wcnt + warp * EP;
    const int32_t *prow = v.wcnt + warp * EP;   // after the scan: the warp's prefixes
    const int iend = min(i1, nitems);
    const unsigned lt = lanemask_lt();
    int badl = 0;
    for (int cs = i0; cs < iend; cs += CH) {
        for (int e = lane; e < E; e += 32) wrow[e] = 0;
        __syncwarp();
        const int ib = cs + warp * 32 * SC_STEPS + lane;   // this lane's index at step 0
        int es[SC_STEPS], loc[SC_STEPS];
#pragma unroll
        for (int s = 0; s < SC_STEPS; ++s) es[s] = ib + s * 32 < iend ? __ldg(ids + ib + s * 32) : -1;
#pragma unroll
        for (int s = 0; s < SC_STEPS; ++s) {
            int e = es[s];
            if (ib + s * 32 < iend && static_cast<unsigned>(e) >= static_cast<unsigned>(E)) {
                badl = 1;
                e = -1;
            }
            const unsigned peers = warp_peers<NB>(e);
            const int cur = e >= 0 ? wrow[e] : 0;
            __syncwarp();
            if (e >= 0 && (peers >> lane) == 1u) wrow[e] = cur + __popc(peers);   // highest peer lane
            __syncwarp();
            es[s] = e;
            loc[s] = cur + __popc(peers & lt);
        }
        __syncthreads();
        // per expert, an exclusive scan down the warps' counts (one thread per
        // expert walking the nw rows; the rows are per-warp, the columns
        // consecutive, so the walkers' loads hit distinct banks)
        for (int e = tid; e < E; e += blockDim.x) {
            int acc = run[e];
            for (int w = 0; w < nw; ++w) {
                const int c = v.wcnt[w * EP + e];
                v.wcnt[w * EP + e] = acc;   // in place: each row becomes its warp's prefix
                acc += c;
            }
            run[e] = acc;
        }
        __syncthreads();
#pragma unroll
        for (int s = 0; s < SC_STEPS; ++s) {
            const int e = es[s];
            if (e < 0) continue;
            const int i = ib + s * 32;
            const int c = v.cls[e];
            const int q = v.base[e] + prow[e] + loc[s];
            int d = c >> 2, pp = q;
            bool ok = true;
            if ((c & 3) == 2) {
                // the segment covering q: forward from the block's first one
                const int last = v.rep0[e] + v.rcnt[e] - 1;
                int j = v.sfirst[e];
                while (j < last && v.s_qoff[j + 1] <= q) ++j;
                const int qo = v.s_qoff[j], t = v.s_tok[j];
                ok = q >= qo && q < qo + t;
                const int w = q - qo, mss = v.s_mass[j];
                if (w < mss) {
                    const int h = v.home[e];
                    d = h;
                    pp = v.homeoff[e] + (h < g ? v.homecnt[e] : 0) + v.s_cum[j] + w;
                } else {
                    const int r = v.s_v[j];
                    d = r;
                    pp = v.s_rep[j] + (r < g ? v.s_vcnt[j] : 0) + (w - mss);
                }
            }
            if (ok && static_cast<unsigned>(pp) < static_cast<unsigned>(nf)) {
                dest[i] = d;
                perm[pp] = fbase + i;
            } else {
                badl = 1;
            }
        }
        __syncthreads();   // pre/run are rewritten by the next chunk
    }
    if (badl) *bad = 1;
    __syncthreads();
}

// Token path of the CTA-mode scatter (k <= KT <= 8; [i0, i1) whole tokens).
// One token per lane: its k ids are distinct, so the rank of (t, j) among
// the block's earlier assignments of e = ids[t, j] is the number of earlier
// tokens holding e.  Every lane ORs its bit into a per-warp mask word of each
// of its experts; a slot's rank inside the warp's 32 tokens is then
// popc(mask & lanes below), and the lowest lane holding e records the warp's
// count of e for the scan down the warps.  A few operations per slot in
// place of a ballot per id bit per 32 assignments; dest rows are written as
// 16-byte vectors.  An id out of range gets dest = -1 and no permutation
// slot, and is flagged.
template <int KT>
__device__ void scatter_block_tok(const Args &a, int b, int g, int i0, int i1, const int32_t *prefix,
                                  const ScatterView &v, int *bad) {
    const int G = a.G, E = a.E, k = a.k, EP = E + 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Tg = a.T / G, nitems = Tg * k, nf = a.T * k;
    const int fbase = g * nitems;
    const int64_t pb = static_cast<int64_t>(b) * a.T * k;
    const int32_t *ids = a.ids + pb + fbase;
    int32_t *dest = a.dest + pb + fbase;
    int32_t *perm = a.perm + pb;
    const int32_t *wsb = a.ws + static_cast<size_t>(b) * a.ws_stride;
    int32_t *run = v.base + EP;
    const int nw = blockDim.x >> 5;
    for (int e = tid; e < E; e += blockDim.x) {
        const int bse = wsb[g * E + e];
        const int r0 = prefix != nullptr ? prefix[e] : 0;
        v.base[e] = bse;
        run[e] = r0;
        const bool local = (v.hold[e] >> g) & 1ull;
        const int m = v.rcnt[e];
        v.cls[e] = local ? (g << 2) : (m == 0 ? (v.home[e] << 2) | 1 : 2);
        int sf = 0;
        if (!local && m > 0) {
            const int q = bse + r0;
            int lo = v.rep0[e], hi = lo + m - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (v.s_qoff[mid] <= q) lo = mid; else hi = mid - 1;
            }
            sf = lo;
        }
        v.sfirst[e] = sf;
    }
    LB_TICK(58);
    for (int x = tid; x < nw * EP; x += blockDim.x) v.lmask[x] = 0u;
    __syncthreads();
    LB_TICK(59);
    int32_t *wrow = v.wcnt + warp * EP;
    const int32_t *prow = v.wcnt + warp * EP;   // after the scan: the warp's prefixes
    uint32_t *lm = v.lmask + warp * EP;
    const unsigned lt = lanemask_lt();
    const bool vec = KT == k && (KT % 4) == 0 && ((reinterpret_cast<uintptr_t>(ids) | reinterpret_cast<uintptr_t>(dest)) &
                                                  15) == 0;
    const int tb0 = i0 / k, tb1 = min(i1, nitems) / k;
    int badl = 0;
    // The next chunk's ids are loaded one chunk ahead (registers), so no
    // chunk waits on a global load.
    int nx[KT];
    auto load_ids = [&](int tt) {
        const bool ok = tt < tb1;
        if (ok && vec) {
#pragma unroll
            for (int j = 0; j < KT; j += 4) {
                const int4 x = __ldg(reinterpret_cast<const int4 *>(ids + tt * KT + j));
                nx[j] = x.x;
                nx[j + 1] = x.y;
                nx[j + 2] = x.z;
                nx[j + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < KT; ++j) nx[j] = (ok && j < k) ? __ldg(ids + tt * k + j) : -1;
        }
    };
    load_ids(tb0 + warp * 32 + lane);
    for (int cs = tb0; cs < tb1; cs += nw * 32) {
        const bool first = cs == tb0;
        if (first) LB_TICK(13);
        for (int e = lane; e < E; e += 32) wrow[e] = 0;
        const int t = cs + warp * 32 + lane;   // this lane's token (block-local)
        const bool tv = t < tb1;
        int ev[KT];
#pragma unroll
        for (int j = 0; j < KT; ++j) ev[j] = nx[j];
        load_ids(t + nw * 32);
        // ids out of range take no slot (a row repeating an id is lb_count's
        // to flag: its slots are then unspecified, every write stays in range)
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            if (tv && j < k && static_cast<unsigned>(ev[j]) >= static_cast<unsigned>(E)) {
                badl = 1;
                ev[j] = -1;
            }
        }
        __syncwarp();   // wrow zeroed before the leaders below write it
#pragma unroll
        for (int j = 0; j < KT; ++j)
            if (ev[j] >= 0) atomicOr(&lm[ev[j]], 1u << lane);
        __syncwarp();
        int loc[KT];    // rank inside the warp's tokens | (warp count of e if this lane leads e) << 8
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            loc[j] = 0;
            if (ev[j] >= 0) {
                const unsigned msk = lm[ev[j]];
                const unsigned below = msk & lt;
                loc[j] = __popc(below) | (below == 0u ? __popc(msk) << 8 : 0);
            }
        }
        __syncwarp();   // every lane has read the masks before they are cleared
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            if (ev[j] >= 0 && (loc[j] >> 8) != 0) {
                wrow[ev[j]] = loc[j] >> 8;
                lm[ev[j]] = 0u;
            }
        }
        if (first) LB_TICK(14);
        __syncthreads();
        for (int e = tid; e < E; e += blockDim.x) {
            int acc = run[e];
            const int bse = v.base[e];
            for (int w = 0; w < nw; ++w) {
                const int c = v.wcnt[w * EP + e];
                v.wcnt[w * EP + e] = bse + acc;   // in place: each row becomes its warp's first slot of e
                acc += c;
            }
            run[e] = acc;
        }
        __syncthreads();
        // Slots served where they are (held locally, or unreplicated: home)
        // are placed now; a replicated expert's remote slots (a minority,
        // but present in nearly every 32-lane slot column) go to the warp's
        // queue and are resolved 32 at a time with every lane busy.
        if (first) LB_TICK(15);
        int2 *qw = v.queue + warp * TOK_QUEUE;
        int qn = 0;   // queued items (warp-uniform)
        int dv[KT];
#pragma unroll
        for (int j = 0; j < KT; ++j) {
            dv[j] = -1;
            const int e = ev[j];
            const int c = e >= 0 ? v.cls[e] : 0;
            const bool rem = e >= 0 && (c & 3) == 2;
            const unsigned rmask = __ballot_sync(kFull, rem);
            if (rem) {
                const int slot = qn + __popc(rmask & lt);
                qw[slot] = make_int2(t * k + j, e | ((loc[j] & 0xff) << 16));
                loc[j] = slot | (1 << 30);   // this slot's answer comes back through the queue
            } else if (e >= 0) {
                const int pp = prow[e] + (loc[j] & 0xff);
                if (static_cast<unsigned>(pp) < static_cast<unsigned>(nf)) {
                    perm[pp] = fbase + t * k + j;
                    dv[j] = c >> 2;
                } else {
                    badl = 1;
                }
            }
            qn += __popc(rmask);
        }
        if (first) LB_TICK(16);
        __syncwarp();
        for (int i0q = 0; i0q < qn; i0q += 32) {
            const int iq = i0q + lane;
            if (iq < qn) {
                const int2 it = qw[iq];
                const int fl = it.x, e = it.y & 0xffff;
                const int q = prow[e] + (it.y >> 16);
                // the segment covering q: forward from the block's first one
                const int last = v.rep0[e] + v.rcnt[e] - 1;
                int jj = v.sfirst[e];
                while (jj < last && v.s_qoff[jj + 1] <= q) ++jj;
                const int qo = v.s_qoff[jj], tk = v.s_tok[jj];
                const int w = q - qo, mss = v.s_mass[jj];
                int d, pp;
                if (w < mss) {
                    const int h = v.home[e];
                    d = h;
                    pp = v.homeoff[e] + (h < g ? v.homecnt[e] : 0) + v.s_cum[jj] + w;
                } else {
                    const int r = v.s_v[jj];
                    d = r;
                    pp = v.s_rep[jj] + (r < g ? v.s_vcnt[jj] : 0) + (w - mss);
                }
                if (q >= qo && q < qo + tk && static_cast<unsigned>(pp) < static_cast<unsigned>(nf)) {
                    perm[pp] = fbase + fl;
                } else {
                    badl = 1;
                    d = -1;
                }
                qw[iq].x = d;
            }
        }
        if (first) LB_TICK(17);
        __syncwarp();
#pragma unroll
        for (int j = 0; j < KT; ++j)
            if (loc[j] & (1 << 30)) dv[j] = qw[loc[j] & 0xffff].x;
        if (tv) {
            if (vec) {
#pragma unroll
                for (int j = 0; j < KT; j += 4)
                    *reinterpret_cast<int4 *>(dest + t * KT + j) = make_int4(dv[j], dv[j + 1], dv[j + 2], dv[j + 3]);
            } else {
#pragma unroll
                for (int j = 0; j < KT; ++j)
                    if (j < k) dest[t * k + j] = dv[j];
            }
        }
        if (first) LB_TICK(18);
        __syncthreads();   // pre/run are rewritten by the next chunk
        if (first) LB_TICK(19);
    }
    if (badl) *bad = 1;
    __syncthreads();
}

// Bits of the largest expert id, rounded up to an instantiated width.
__device__ __forceinline__ int id_bits(int E) {
    const int nb = E > 1 ? 32 - __clz(E - 1) : 1;
    return nb <= 4 ? 4 : nb <= 6 ? 6 : nb <= 8 ? 8 : 10;
}

__device__ inline void scatter_blocks_warp_any(const Args &a, int b, int g0, int g1, const ScatterView &v,
                                               int *bad) {
    switch (id_bits(a.E)) {
        case 4: scatter_blocks_warp<4>(a, b, g0, g1, v, bad); break;
        case 6: scatter_blocks_warp<6>(a, b, g0, g1, v, bad); break;
        case 8: scatter_blocks_warp<8>(a, b, g0, g1, v, bad); break;
        default: scatter_blocks_warp<10>(a, b, g0, g1, v, bad); break;
    }
}

__device__ inline void scatter_block_cta_any(const Args &a, int b, int g, int i0, int i1, const int32_t *prefix,
                                             const ScatterView &v, int *bad) {
    const int nitems = (a.T / a.G) * a.k;
    if (a.k <= 8 && i0 % a.k == 0 && (i1 % a.k == 0 || i1 >= nitems)) {
        if (a.k <= 2) scatter_block_tok<2>(a, b, g, i0, i1, prefix, v, bad);
        else if (a.k <= 4) scatter_block_tok<4>(a, b, g, i0, i1, prefix, v, bad);
        else scatter_block_tok<8>(a, b, g, i0, i1, prefix, v, bad);
        return;
    }
    switch (id_bits(a.E)) {
        case 4: scatter_block_cta<4>(a, b, g, i0, i1, prefix, v, bad); break;
        case 6: scatter_block_cta<6>(a, b, g, i0, i1, prefix, v, bad); break;
        case 8: scatter_block_cta<8>(a, b, g, i0, i1, prefix, v, bad); break;
        default: scatter_block_cta<10>(a, b, g, i0, i1, prefix, v, bad); break;
    }
}

// Scatter kernel: CTA (x, problem y) of W = blockDim.x / 32 warps (32 for
// one problem's latency; 16 when many problems fill the GPU, so that two CTAs
// share an SM and one's barriers overlap the other's work).  Small blocks:
// CTA x takes blocks [x*W, (x+1)*W), one per warp, unless a.cta_blocks asks
// for one block per CTA (few problems: the blocks then spread over more SMs).
// Large blocks: CTA x takes block x (or a slice of it).
__global__ void __launch_bounds__(SC_THREADS) scatter_kernel(const Args a) {
    extern __shared__ __align__(16) uint8_t sm[];
    __shared__ int bad;
    if (threadIdx.x == 0) bad = 0;
    const int nw = blockDim.x >> 5;
    const ScatterView v = scatter_carve(sm, a.G, a.E, a.N, nw);
    LB_TICK(10);
    // Launched after the prep or the fused decide kernel: the counts and the
    // plan were final before either started, so the tables built from them
    // are built before waiting on it.
    scatter_setup_inputs(a, blockIdx.y, v);
    pdl_begin();
    scatter_setup_tables(a, blockIdx.y, v);
    LB_TICK(11);
    const int nitems = (a.T / a.G) * a.k;
    if (nitems <= WARP_BLOCK_MAX && !a.cta_blocks) {
        const int g0 = blockIdx.x * nw;
        scatter_blocks_warp_any(a, blockIdx.y, g0, min(a.G, g0 + nw), v, &bad);
        __syncthreads();
    } else {
        // CTA x scatters slice x mod S of source block x / S (S = a.slices
        // token-aligned slices, so that one problem's few blocks spread over
        // more SMs).  A slice's ranks continue the block's earlier slices:
        // the CTA first counts each expert's valid ids there (the scatter's
        // own ranking counts the same ones).
        const int S = a.slices;
        const int g = static_cast<int>(blockIdx.x) / S, sl = static_cast<int>(blockIdx.x) - g * S;
        const int Tg = a.T / a.G, tps = (Tg + S - 1) / S;
        const int t0 = min(Tg, sl * tps);
        const int i0 = t0 * a.k, i1 = sl == S - 1 ? nitems : min(Tg, t0 + tps) * a.k;
        const int32_t *prefix = nullptr;
        if (S > 1) {
            int32_t *pref = v.base + 2 * (a.E + 1);   // (rows 0 and 1 serve the block; nw >= 8 here)
            for (int e = threadIdx.x; e < a.E; e += blockDim.x) pref[e] = 0;
            __syncthreads();
            const int32_t *ids = a.ids + static_cast<int64_t>(blockIdx.y) * a.T * a.k + static_cast<int64_t>(g) * nitems;
            const unsigned E = static_cast<unsigned>(a.E);
            int n4 = 0;
            if ((reinterpret_cast<uintptr_t>(ids) & 15) == 0) {
                n4 = i0 >> 2;
                const int4 *ids4 = reinterpret_cast<const int4 *>(ids);
#pragma unroll 4
                for (int x = threadIdx.x; x < n4; x += blockDim.x) {
                    const int4 q = __ldg(ids4 + x);
                    if (static_cast<unsigned>(q.x) < E) atomicAdd(&pref[q.x], 1);
                    if (static_cast<unsigned>(q.y) < E) atomicAdd(&pref[q.y], 1);
                    if (static_cast<unsigned>(q.z) < E) atomicAdd(&pref[q.z], 1);
                    if (static_cast<unsigned>(q.w) < E) atomicAdd(&pref[q.w], 1);
                }
            }
            for (int x = 4 * n4 + threadIdx.x; x < i0; x += blockDim.x) {
                const int e = __ldg(ids + x);
                if (static_cast<unsigned>(e) < E) atomicAdd(&pref[e], 1);
            }
            __syncthreads();
            prefix = pref;
        }
        scatter_block_cta_any(a, blockIdx.y, g, i0, i1, prefix, v, &bad);
    }
    LB_TICK(12);
    if (threadIdx.x == 0 && bad) flag(LB_DEV_BAD_SPLIT);
}

}  // namespace assign
}  // namespace lb
