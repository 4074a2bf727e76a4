// Step 3: locality-aware replica planning (Libra README, Key Ideas,
// locality-aware expert replication planning, phases 1 and 2) and the
// replica edges with their round schedule (Relief, The Relief Algorithm:
// edge colouring of the replica graph, computed once per placement).
//
// One CTA per problem; the predicted counts are staged in shared memory.
//   phase 1: one warp per rank; each pick is a warp arg-max (redux.sync max
//            on the count, then redux.sync min on the id among the maxima).
//   load model: thread per expert (remote mass), warp per rank (loads).
//   phase 2: a single warp runs the sequential greedy loop; rank loads and
//            slot counts live in registers (lane r holds ranks r and r+32),
//            holder sets are 64-bit masks per expert, and every arg-max /
//            arg-min is one redux.sync plus a ballot.
//   edges:   per-expert replica counts, warp scan, parallel edge emission
//            (expert ascending, rank ascending).
//   rounds:  greedy colouring in edge order by one thread, each rank's busy
//            rounds as 64-bit words in shared memory; the stable order by round
//            from per-round counts, a warp scan and each edge's rank among
//            the earlier edges of its round.
#pragma once
#include "common.cuh"

namespace lb {
namespace plan {

constexpr int THREADS = 512;

struct Layout {
    size_t hdr, used, slots, slot_phase, plan_load, edge_u, edge_v, edge_e, edge_round, round_ptr,
        rep_ptr, rep_edge, holds, total;
};

__host__ __device__ inline Layout layout(int G, int E, int N) {
    Layout L;
    const size_t GN = static_cast<size_t>(G) * N;
    size_t o = 0;
    L.hdr = o;        o += 16 * 4;
    L.used = o;       o += static_cast<size_t>(G) * 4;
    L.slots = o;      o += GN * 4;
    L.slot_phase = o; o += GN * 4;
    L.plan_load = o;  o += static_cast<size_t>(G) * 4;
    L.edge_u = o;     o += GN * 4;
    L.edge_v = o;     o += GN * 4;
    L.edge_e = o;     o += GN * 4;
    L.edge_round = o; o += GN * 4;
    L.round_ptr = o;  o += (GN + 1) * 4;
    L.rep_ptr = o;    o += (static_cast<size_t>(E) + 1) * 4;
    L.rep_edge = o;   o += GN * 4;
    L.holds = o;      o += static_cast<size_t>(G) * E;
    L.total = (o + 255) & ~static_cast<size_t>(255);
    return L;
}

// Dynamic shared memory of plan_kernel.
__host__ __device__ inline size_t smem_bytes(int G, int E, int N) {
    const size_t GN = static_cast<size_t>(G) * N;
    const size_t W = (GN + 63) / 64 + 1;
    return static_cast<size_t>(E) * 8            // hold masks
           + static_cast<size_t>(G) * W * 8      // busy round masks
           + static_cast<size_t>(G) * E * 4      // counts
           + static_cast<size_t>(E) * 4          // remote mass m
           + (static_cast<size_t>(E) + 1) * 4    // edge offset per expert
           + GN * 4 * 2                          // slots, slot phase
           + GN * 4 * 5                          // eu, ev, ee, er, pos
           + (GN + 1) * 4 * 2;                   // round ptr, round fill
}

// The whole plan of one problem by one CTA: counts cnt [G, E] (global) in,
// the blob (global) out; `sm` holds smem_bytes(G, E, N) bytes.  All threads
// of the CTA call it; it ends with a block barrier.
__device__ void plan_problem(const int32_t *__restrict__ cnt, int G, int E, int N, int L, uint8_t *__restrict__ blob,
                             uint8_t *sm) {
    const int GN = G * N;
    const int W = (GN + 63) / 64 + 1;
    uint64_t *hold = reinterpret_cast<uint64_t *>(sm);
    uint64_t *busy = hold + E;
    int32_t *cnt_s = reinterpret_cast<int32_t *>(busy + static_cast<size_t>(G) * W);
    int32_t *m = cnt_s + static_cast<size_t>(G) * E;
    int32_t *eoff = m + E;
    int32_t *slots = eoff + E + 1;
    int32_t *phase = slots + GN;
    int32_t *eu = phase + GN;
    int32_t *ev = eu + GN;
    int32_t *ee = ev + GN;
    int32_t *er = ee + GN;
    int32_t *pos = er + GN;
    int32_t *rptr = pos + GN;
    int32_t *rfill = rptr + GN + 1;
    __shared__ int used_s[LB_MAX_G], load_s[LB_MAX_G];
    __shared__ int n_edges_s, n_rounds_s, n_p2_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
    const Layout LY = layout(G, E, N);
    const int Eg = E / G;

    LB_TICK(30);
    stage_i32(cnt_s, cnt, G * E);
    for (int e = tid; e < E; e += blockDim.x) hold[e] = 1ull << (e / Eg);
    for (int i = tid; i < G * W; i += blockDim.x) busy[i] = 0ull;
    for (int i = tid; i < GN; i += blockDim.x) {
        slots[i] = -1;
        phase[i] = 0;
    }
    if (tid < LB_MAX_G) used_s[tid] = 0;
    __syncthreads();

    LB_TICK(31);
    // ---------------- phase 1: each rank imports its L most-requested foreign experts
    for (int g = warp; g < G; g += nwarps) {
        for (int pick = 0; pick < L; ++pick) {
            int bc = 0, be = 0x7fffffff;
            for (int e = lane; e < E; e += 32) {
                if ((e < g * Eg || e >= (g + 1) * Eg) && !((hold[e] >> g) & 1ull)) {
                    const int c = cnt_s[g * E + e];
                    if (c > bc) {
                        bc = c;
                        be = e;
                    }
                }
            }
            const int mc = __reduce_max_sync(kFull, bc);
            if (mc <= 0) break;
            const int me = __reduce_min_sync(kFull, bc == mc ? be : 0x7fffffff);
            if (lane == 0) {
                atomicOr(reinterpret_cast<unsigned long long *>(&hold[me]), 1ull << g);
                slots[g * N + used_s[g]] = me;
                phase[g * N + used_s[g]] = 1;
                used_s[g] += 1;
            }
            __syncwarp();
        }
    }
    __syncthreads();

    LB_TICK(32);
    // ---------------- load model: per expert, its remote mass m[e] (tokens of
    // sources that do not hold it) stays at home; every holder serves its own
    // tokens.  Rank loads are integer sums, so their order is immaterial.
    if (tid < LB_MAX_G) load_s[tid] = 0;
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        const uint64_t hm = hold[e];
        int s = 0;
        for (int g = 0; g < G; ++g)
            if (!((hm >> g) & 1ull)) s += cnt_s[g * E + e];
        m[e] = s;
        for (uint64_t mk = hm; mk; mk &= mk - 1) {
            const int g = __ffsll(static_cast<long long>(mk)) - 1;
            atomicAdd(&load_s[g], cnt_s[g * E + e]);
        }
        atomicAdd(&load_s[e / Eg], s);
    }
    __syncthreads();

    LB_TICK(33);
    // ---------------- phase 2: sequential greedy, one warp
    __shared__ int total_s;
    if (warp == 0) {
        int x = 0;
        for (int r = lane; r < G; r += 32) x += load_s[r];
        x = __reduce_add_sync(kFull, x);
        if (lane == 0) total_s = x;
    }
    __syncthreads();
    if (warp == 0 && total_s < (1 << 21)) {
        // Every load and remote mass is below 2^21, so each arg-reduction is
        // one redux over a packed 32-bit key: (load, 63 - rank) + 1 for the
        // most-loaded rank (lowest rank on ties), (mass, 1023 - position) for
        // the candidate expert (lowest id on ties), (load, rank) for the
        // least-loaded eligible rank.  Same choices as the general loop below.
        const bool ha = lane < G, hb = lane + 32 < G;
        int la = ha ? load_s[lane] : 0, lb = hb ? load_s[lane + 32] : 0;
        int ua = ha ? used_s[lane] : N, ub = hb ? used_s[lane + 32] : N;
        const int iters = __reduce_add_sync(kFull, (ha ? N - ua : 0) + (hb ? N - ub : 0));
        uint64_t freem = static_cast<uint64_t>(__ballot_sync(kFull, ha && ua < N)) |
                         (static_cast<uint64_t>(__ballot_sync(kFull, hb && ub < N)) << 32);
        int np2 = 0;
        for (int it = 0; it < iters; ++it) {
            const unsigned ka = ha ? ((static_cast<unsigned>(la) << 6) | static_cast<unsigned>(63 - lane)) + 1u : 0u;
            const unsigned kb = hb ? ((static_cast<unsigned>(lb) << 6) | static_cast<unsigned>(31 - lane)) + 1u : 0u;
            const unsigned ku = __reduce_max_sync(kFull, max(ka, kb));
            const int u = 63 - static_cast<int>((ku - 1u) & 63u);
            const int mx = static_cast<int>((ku - 1u) >> 6);
            unsigned kc = 0u;
            for (int q = lane; q < Eg; q += 32) {
                const int e = u * Eg + q;
                const int me = m[e];
                if (me > 0 && (~hold[e] & freem) != 0ull)
                    kc = max(kc, (static_cast<unsigned>(me) << 10) | static_cast<unsigned>(1023 - q));
            }
            kc = __reduce_max_sync(kFull, kc);
            if (kc == 0u) break;
            const int ce = u * Eg + (1023 - static_cast<int>(kc & 1023u));
            const uint64_t hce = hold[ce];
            const int mce = static_cast<int>(kc >> 10);
            const uint64_t V = ~hce & freem;
            const bool ea = (V >> lane) & 1ull, eb = (V >> (lane + 32)) & 1ull;
            const unsigned kva = ea ? (static_cast<unsigned>(la) << 6) | static_cast<unsigned>(lane) : 0xffffffffu;
            const unsigned kvb = eb ? (static_cast<unsigned>(lb) << 6) | static_cast<unsigned>(lane + 32) : 0xffffffffu;
            const unsigned kv = __reduce_min_sync(kFull, min(kva, kvb));
            const int v = static_cast<int>(kv & 63u);
            const int mn = static_cast<int>(kv >> 6);
            const int c = cnt_s[v * E + ce];
            const int mr = mce - c;
            const int lu = mx - c, lv = mn + c;
            const int gap = lu - lv;
            const int d = min(gap > 0 ? (gap >> 1) : 0, mr);
            if (c + d == 0) break;
            const int used_v = __shfl_sync(kFull, v < 32 ? ua : ub, v & 31);
            if (lane == 0) {
                hold[ce] = hce | (1ull << v);
                slots[v * N + used_v] = ce;
                phase[v * N + used_v] = 2;
                m[ce] = mr - d;
            }
            if (used_v + 1 >= N) freem &= ~(1ull << v);
            const bool own_u = lane == (u & 31), own_v = lane == (v & 31);
            la = (own_u && u < 32) ? lu - d : la;
            lb = (own_u && u >= 32) ? lu - d : lb;
            la = (own_v && v < 32) ? lv + d : la;
            lb = (own_v && v >= 32) ? lv + d : lb;
            ua += (own_v && v < 32) ? 1 : 0;
            ub += (own_v && v >= 32) ? 1 : 0;
            ++np2;
            __syncwarp();
        }
        if (ha) { load_s[lane] = la; used_s[lane] = ua; }
        if (hb) { load_s[lane + 32] = lb; used_s[lane + 32] = ub; }
        if (lane == 0) n_p2_s = np2;
    } else if (warp == 0) {
        const bool ha = lane < G, hb = lane + 32 < G;
        int la = ha ? load_s[lane] : INT_MIN, lb = hb ? load_s[lane + 32] : INT_MIN;
        int ua = ha ? used_s[lane] : N, ub = hb ? used_s[lane + 32] : N;
        const int iters = __reduce_add_sync(kFull, (ha ? N - ua : 0) + (hb ? N - ub : 0));
        int np2 = 0;
        for (int it = 0; it < iters; ++it) {
            const int mx = __reduce_max_sync(kFull, max(la, lb));
            const unsigned bxa = __ballot_sync(kFull, ha && la == mx);
            const unsigned bxb = __ballot_sync(kFull, hb && lb == mx);
            const int u = bxa ? __ffs(bxa) - 1 : 32 + __ffs(bxb) - 1;
            const uint64_t freem = static_cast<uint64_t>(__ballot_sync(kFull, ha && ua < N)) |
                                   (static_cast<uint64_t>(__ballot_sync(kFull, hb && ub < N)) << 32);
            int bm = 0, be = 0x7fffffff;
            for (int q = lane; q < Eg; q += 32) {
                const int e = u * Eg + q;
                const int me = m[e];
                const bool ok = me > bm && (~hold[e] & freem) != 0ull;
                bm = ok ? me : bm;
                be = ok ? e : be;
            }
            const int mm = __reduce_max_sync(kFull, bm);
            if (mm <= 0) break;
            const int ce = __reduce_min_sync(kFull, bm == mm ? be : 0x7fffffff);
            const uint64_t hce = hold[ce];
            const int mce = m[ce];
            const uint64_t V = ~hce & freem;
            const bool ea = (V >> lane) & 1ull, eb = (V >> (lane + 32)) & 1ull;
            const int mn = __reduce_min_sync(kFull, min(ea ? la : INT_MAX, eb ? lb : INT_MAX));
            const unsigned bva = __ballot_sync(kFull, ea && la == mn);
            const unsigned bvb = __ballot_sync(kFull, eb && lb == mn);
            const int v = bva ? __ffs(bva) - 1 : 32 + __ffs(bvb) - 1;
            const int c = cnt_s[v * E + ce];
            const int mr = mce - c;
            const int lu = mx - c, lv = mn + c;
            const int gap = lu - lv;
            const int d = min(gap > 0 ? (gap >> 1) : 0, mr);
            if (c + d == 0) break;
            const int used_v = __shfl_sync(kFull, v < 32 ? ua : ub, v & 31);
            if (lane == 0) {
                hold[ce] = hce | (1ull << v);
                slots[v * N + used_v] = ce;
                phase[v * N + used_v] = 2;
                m[ce] = mr - d;
            }
            const bool own_u = lane == (u & 31), own_v = lane == (v & 31);
            la = (own_u && u < 32) ? lu - d : la;
            lb = (own_u && u >= 32) ? lu - d : lb;
            la = (own_v && v < 32) ? lv + d : la;
            lb = (own_v && v >= 32) ? lv + d : lb;
            ua += (own_v && v < 32) ? 1 : 0;
            ub += (own_v && v >= 32) ? 1 : 0;
            ++np2;
            __syncwarp();
        }
        if (ha) { load_s[lane] = la; used_s[lane] = ua; }
        if (hb) { load_s[lane + 32] = lb; used_s[lane + 32] = ub; }
        if (lane == 0) n_p2_s = np2;
    }
    __syncthreads();

    LB_TICK(34);
    // ---------------- edges: expert ascending, replica rank ascending
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < E; base += 32) {
            const int e = base + lane;
            int x = e < E ? __popcll(hold[e]) - 1 : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(kFull, x, off);
                if (lane >= off) x += y;
            }
            if (e < E) eoff[e + 1] = carry + x;
            carry += __shfl_sync(kFull, x, 31);
        }
        if (lane == 0) {
            eoff[0] = 0;
            n_edges_s = carry;
        }
    }
    __syncthreads();
    const int ne = n_edges_s;
    for (int e = tid; e < E; e += blockDim.x) {
        const int h = e / Eg;
        uint64_t mask = hold[e] & ~(1ull << h);
        int idx = eoff[e];
        while (mask) {
            const int r = __ffsll(static_cast<long long>(mask)) - 1;
            mask &= mask - 1;
            eu[idx] = h;
            ev[idx] = r;
            ee[idx] = e;
            ++idx;
        }
    }
    __syncthreads();

    LB_TICK(35);
    // ---------------- greedy colouring, edge order: one thread, each rank's
    // busy rounds as W 64-bit words in shared memory.  An edge costs one
    // round of independent loads (both ranks' first two words), a find-first
    // and two stores.  Measured at the decode shape (128 edges, 67 rounds):
    // 17.5 us, against 22.1 us for a warp holding 128-bit masks in registers
    // (eight shuffles per edge), 19.4 us for 32-bit words scanned in a loop,
    // and 24.8 us with the next edge's words loaded ahead and forwarded in
    // registers (a longer chain of 64-bit selects).
    if (tid == 0) {
        int nr = 0;
        for (int i = 0; i < ne; ++i) {
            uint64_t *bu = busy + eu[i] * W, *bv = busy + ev[i] * W;
            const uint64_t u0 = bu[0], v0 = bv[0];
            const uint64_t u1 = W > 1 ? bu[1] : ~0ull, v1 = W > 1 ? bv[1] : ~0ull;
            int c;
            uint64_t ou, ov;   // the words that take the round's bit
            if (~(u0 | v0)) {
                c = __ffsll(static_cast<long long>(~(u0 | v0))) - 1;
                ou = u0;
                ov = v0;
            } else if (~(u1 | v1)) {
                c = 64 + __ffsll(static_cast<long long>(~(u1 | v1))) - 1;
                ou = u1;
                ov = v1;
            } else {
                // past 128 rounds (W words cover more rounds than a plan has edges)
                c = 0;
                for (int w = 2; w < W; ++w) {
                    const uint64_t x = bu[w] | bv[w];
                    if (~x) {
                        c = w * 64 + __ffsll(static_cast<long long>(~x)) - 1;
                        break;
                    }
                }
                ou = bu[c >> 6];
                ov = bv[c >> 6];
            }
            const uint64_t bit = 1ull << (c & 63);
            bu[c >> 6] = ou | bit;
            bv[c >> 6] = ov | bit;   // (an edge joins two ranks)
            er[i] = c;
            nr = max(nr, c + 1);
        }
        n_rounds_s = nr;
    }
    __syncthreads();
    LB_TICK(38);
    {
        // stable order by round: position = start of the round + earlier
        // edges (in edge order) of the same round
        const int nrr = n_rounds_s;
        for (int r = tid; r <= nrr; r += blockDim.x) rfill[r] = 0;
        __syncthreads();
        for (int i = tid; i < ne; i += blockDim.x) atomicAdd(&rfill[er[i]], 1);
        __syncthreads();
        if (warp == 0) {
            int carry = 0;
            for (int base = 0; base < nrr; base += 32) {
                const int r = base + lane;
                int x = r < nrr ? rfill[r] : 0;
                const int own = x;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(kFull, x, off);
                    if (lane >= off) x += y;
                }
                if (r < nrr) rptr[r] = carry + x - own;
                carry += __shfl_sync(kFull, x, 31);
            }
            if (lane == 0) rptr[nrr] = carry;
        }
        __syncthreads();
        for (int i = tid; i < ne; i += blockDim.x) {
            const int r = er[i];
            int before = 0;
            for (int j = 0; j < i; ++j) before += er[j] == r;
            pos[i] = rptr[r] + before;
        }
    }
    __syncthreads();
    const int nr = n_rounds_s;

    LB_TICK(36);
    // ---------------- write the blob
    int32_t *hdr = reinterpret_cast<int32_t *>(blob + LY.hdr);
    if (tid == 0) {
        int np1 = 0;
        for (int i = 0; i < GN; ++i) np1 += phase[i] == 1;
        hdr[0] = ne;
        hdr[1] = nr;
        hdr[2] = np1;
        hdr[3] = n_p2_s;
        hdr[4] = G;
        hdr[5] = E;
        hdr[6] = N;
        hdr[7] = L;
        for (int i = 8; i < 16; ++i) hdr[i] = 0;
    }
    int32_t *o_used = reinterpret_cast<int32_t *>(blob + LY.used);
    int32_t *o_load = reinterpret_cast<int32_t *>(blob + LY.plan_load);
    for (int g = tid; g < G; g += blockDim.x) {
        o_used[g] = used_s[g];
        o_load[g] = load_s[g];
    }
    int32_t *o_slots = reinterpret_cast<int32_t *>(blob + LY.slots);
    int32_t *o_phase = reinterpret_cast<int32_t *>(blob + LY.slot_phase);
    int32_t *o_eu = reinterpret_cast<int32_t *>(blob + LY.edge_u);
    int32_t *o_ev = reinterpret_cast<int32_t *>(blob + LY.edge_v);
    int32_t *o_ee = reinterpret_cast<int32_t *>(blob + LY.edge_e);
    int32_t *o_er = reinterpret_cast<int32_t *>(blob + LY.edge_round);
    int32_t *o_rep_edge = reinterpret_cast<int32_t *>(blob + LY.rep_edge);
    for (int i = tid; i < GN; i += blockDim.x) {
        o_slots[i] = slots[i];
        o_phase[i] = phase[i];
        if (i >= ne) {
            o_eu[i] = -1;
            o_ev[i] = -1;
            o_ee[i] = -1;
            o_er[i] = -1;
            o_rep_edge[i] = -1;
        }
    }
    for (int i = tid; i < ne; i += blockDim.x) {
        const int p = pos[i];
        o_eu[p] = eu[i];
        o_ev[p] = ev[i];
        o_ee[p] = ee[i];
        o_er[p] = er[i];
        o_rep_edge[i] = p;
    }
    int32_t *o_rptr = reinterpret_cast<int32_t *>(blob + LY.round_ptr);
    for (int r = tid; r <= GN; r += blockDim.x) o_rptr[r] = r <= nr ? rptr[r] : ne;
    int32_t *o_rep_ptr = reinterpret_cast<int32_t *>(blob + LY.rep_ptr);
    for (int e = tid; e <= E; e += blockDim.x) o_rep_ptr[e] = eoff[e];
    uint8_t *o_holds = blob + LY.holds;
    for (int g = warp; g < G; g += nwarps)
        for (int e = lane; e < E; e += 32) o_holds[g * E + e] = static_cast<uint8_t>((hold[e] >> g) & 1ull);
    // padding to the blob's 256-byte size: written too, so a blob is fully
    // determined by its inputs
    for (size_t i = LY.holds + static_cast<size_t>(G) * E + tid; i < LY.total; i += blockDim.x) blob[i] = 0;
    __syncthreads();
    LB_TICK(37);
}

__global__ void __launch_bounds__(THREADS)
    plan_kernel(const int32_t *__restrict__ cnt_all, int G, int E, int N, int L,
                uint8_t *__restrict__ plan_all, size_t stride) {
    extern __shared__ __align__(16) uint8_t sm[];
    pdl_begin();
    const int b = blockIdx.x;
    plan_problem(cnt_all + static_cast<int64_t>(b) * G * E, G, E, N, L, plan_all + static_cast<size_t>(b) * stride,
                 sm);
}

}  // namespace plan
}  // namespace lb
