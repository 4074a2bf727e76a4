// Step 1: lookahead gate GEMM + top-k, fused (FreeBalance sec. 3.2 eq. 2-5;
// Libra README, Key Ideas, lookahead predictor).
//
// One CTA owns a 128-token tile of one problem.  TMA streams h[128 x 64] and
// W[Epad x 64] bf16 tiles (128-byte swizzle) through a ring of shared-memory
// stages; one thread issues tcgen05.mma (M=128, N=Epad, K=16) into a TMEM
// accumulator of Epad fp32 columns; after the last k-block, TMEM holds the
// 128 x E logit tile and the epilogue does the top-k without another pass
// over memory.
//
// Split of H across a cluster (SPLITK): when there are too few token tiles to
// fill the GPU, `split` CTAs of one cluster each take 1/split of H; each CTA
// stages its partial tile in its own shared memory, and after a cluster
// barrier CTA r reduces rows [r*128/split, (r+1)*128/split) over all
// partials (in fixed CTA order, so results are deterministic), adds the bias
// and ranks them, with `split` threads per row merged by warp shuffles.
//
// Top-k: each thread keeps a sorted list of its KMAX best (value desc, id
// asc) fed in ascending expert order with a strict '>' so equal logits keep
// the lower id first; lists of several threads merge by repeated
// (max value, min id) shuffles.
#pragma once
#include "common.cuh"

namespace lb {
namespace gate {

constexpr int BM = 128;        // tokens per tile (UMMA M)
constexpr int BK = 64;         // bf16 per k-block: one 128-byte swizzle row
constexpr int UK = 16;         // UMMA K for bf16
constexpr int THREADS = 128;   // 4 warps; warp 0 lane 0 = TMA, warp 1 lane 0 = MMA
constexpr int MAX_STAGES = 8;

// One thread's tensor copies are served one after another (measured on
// B200: one issuing thread feeds an SM at about 38 GB/s from L2 however many
// copies it has in flight; each further issuing thread adds about as much,
// up to the SM's share of L2 bandwidth).  The producer of the pair split-H
// gate is therefore a whole warp, box j of stage slot s issued by lane
// (s * nbox + j) mod 32.  (The persistent and per-tile gates keep one
// issuing lane: their MMAs, not their loads, set the pace, and the same
// change measured slower there, 1278 against 1084 us on the 16-layer
// Qwen3-235B-shaped chain.)
__device__ __forceinline__ bool issues_box(int s, int nbox, int j, int lane) {
    return ((s * nbox + j) & 31) == lane;
}

// Producer wait of a whole warp on a stage's empty barrier: lane 0 waits and
// the warp learns the outcome (0 go on, 1 timed out, 2 aborted elsewhere).
__device__ __forceinline__ int warp_wait_empty(uint64_t *bar, uint32_t parity, const int *abort_flag, int lane) {
    int st = 0;
    if (lane == 0) st = !mbar_wait(bar, parity) ? 1 : (*reinterpret_cast<const volatile int *>(abort_flag) ? 2 : 0);
    return __shfl_sync(0xffffffffu, st, 0);
}

struct Params {
    const float *bias;   // [B,E] or null
    int32_t *ids;        // [B,T,k]
    float *logits;       // [B,T,E] or null
    int T, H, E, Epad, k, nkb, split, stages;
    int kbox;            // persistent kernel: 64-column boxes per pipeline stage
    uint32_t tmem_cols;
    // Chain mode (persistent kernel only): problem b = 0..L is hidden state
    // h_b, and its B tile is rows [(b-1)E, (b+1)E) of the [L*E, H] stack of
    // gates, i.e. W_{b-1} then W_b (rows outside the stack read as zeros).
    // Columns [0,E) rank into ids/logits of layer b-1 (its normal router),
    // columns [E,2E) into ids2/logits2 of layer b (its lookahead).
    int chain, L;
    int32_t *ids2;       // [L,T,k]
    float *logits2;      // [L,T,E] or null
    int nbuf;            // persistent kernel: TMEM accumulator buffers (2 = double-buffered, 1)
};

// Ranking keys.  A logit x and its expert id c (c <= mask, mask = 2^ib - 1)
// pack into one 32-bit key whose unsigned order is the ranking order: the
// bits of x mapped to an order-preserving unsigned integer (negative values
// complemented, the sign bit set on the others), with its ib low bits
// replaced by mask - c.  Larger keys rank first.  Logits that agree in all
// but their ib lowest bits (a relative difference below 2^(ib-23), far under
// the resolution of bf16 inputs) rank by ascending id, exactly like equal
// logits.  One key per candidate turns the sorted insertion into a chain of
// min/max operations with no branches, whatever the lanes of a warp hold.
__device__ __forceinline__ uint32_t id_mask(int E) {
    return E > 1 ? 0xffffffffu >> __clz(E - 1) : 0u;
}
__device__ __forceinline__ uint32_t rank_key(float x, int c, uint32_t mask) {
    const uint32_t u = __float_as_uint(x);
    const uint32_t o = u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
    return (o & ~mask) | (mask - static_cast<uint32_t>(c));
}
__device__ __forceinline__ int key_id(uint32_t key, uint32_t mask) {
    return static_cast<int>(mask - (key & mask));
}

template <int KMAX>
struct TopK {
    uint32_t key[KMAX];   // descending
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) key[j] = 0u;   // below every real key
    }
    __device__ __forceinline__ void push(uint32_t x) {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            const uint32_t hi = max(key[j], x);
            x = min(key[j], x);
            key[j] = hi;
        }
    }
    // Merge the lists of `width` adjacent lanes (width a power of two <= 32);
    // every lane of the group ends up with the merged list in `out`.  Keys
    // of different lanes differ (their ids do), so exactly one lane pops.
    __device__ __forceinline__ void merge(int width, uint32_t (&out)[KMAX]) {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            uint32_t h = key[0];
            for (int off = width >> 1; off > 0; off >>= 1) h = max(h, __shfl_xor_sync(kFull, h, off));
            out[j] = h;
            const bool pop = (key[0] == h);
#pragma unroll
            for (int q = 0; q < KMAX - 1; ++q) key[q] = pop ? key[q + 1] : key[q];
            if (pop) key[KMAX - 1] = 0u;
        }
    }
};

// Split of N across a cluster (SPLITN): the S CTAs of a cluster share one
// token tile; CTA r loads the tile's h rows and rows [r Nc, (r+1) Nc) of W
// (Nc = Epad / S; the B map's box is Nc rows), accumulates the tile's logits
// for those experts over all of H, ranks them per row, and leaves its sorted
// key list of each row in shared memory.  After a cluster barrier, CTA r
// merges rows [r BM/S, (r+1) BM/S) over the S lists (distributed shared
// memory reads) and writes their ids.  Keys carry the global expert id, so
// the merge is a plain top-k of the S lists: the same ranking as one CTA.
template <int KMAX, bool SPLITK, bool SPLITN = false>
__global__ void __launch_bounds__(THREADS, 1)
    gate_topk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const Params p) {
    static_assert(!(SPLITK && SPLITN), "one split at a time");
    extern __shared__ uint8_t smem_raw[];
    pdl_begin();
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    __shared__ __align__(8) uint64_t full_bar[MAX_STAGES];
    __shared__ __align__(8) uint64_t empty_bar[MAX_STAGES];
    __shared__ __align__(8) uint64_t acc_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int aborted;
    __shared__ float bias_s[LB_MAX_E_GATE];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y;
    const int S = (SPLITK || SPLITN) ? p.split : 1;
    const int crank = (SPLITK || SPLITN) ? static_cast<int>(cluster_ctarank()) : 0;
    const int mtile = blockIdx.x / S;
    const int m0 = mtile * BM;
    const int kb_per = SPLITN ? p.nkb : (p.nkb + S - 1) / S;
    const int kb0 = SPLITN ? 0 : crank * kb_per;
    const int nk = max(0, min(p.nkb, kb0 + kb_per) - kb0);
    const int Nc = SPLITN ? p.Epad / S : p.Epad;   // the MMA's N: this CTA's experts
    const int c_off = SPLITN ? crank * Nc : 0;     // its first expert
    const uint32_t a_bytes = BM * 128u;
    const uint32_t stage_bytes = a_bytes + static_cast<uint32_t>(Nc) * 128u;
    const int stages = p.stages;

    for (int c = tid; c < p.Epad; c += THREADS)
        bias_s[c] = (p.bias != nullptr && c < p.E) ? p.bias[static_cast<int64_t>(b) * p.E + c] : 0.f;
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&acc_bar, 1);
        aborted = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            int issued = 0;
            for (int i = 0; i < nk; ++i) {
                const int s = i % stages;
                const uint32_t ph = (i / stages) & 1;
                if (!mbar_wait(&empty_bar[s], ph ^ 1)) {
                    atomicExch(&aborted, 1);
                    flag(LB_DEV_TIMEOUT);
                    break;
                }
                if (*reinterpret_cast<volatile int *>(&aborted)) break;
                uint8_t *sa = smem + static_cast<size_t>(s) * stage_bytes;
                mbar_arrive_expect_tx(&full_bar[s], stage_bytes);
                tma_load_3d(&tmA, sa, &full_bar[s], (kb0 + i) * BK, m0, b);
                tma_load_3d(&tmB, sa + a_bytes, &full_bar[s], (kb0 + i) * BK, c_off, b);
                ++issued;
            }
            // Never leave with copies in flight into this CTA's shared memory:
            // wait (bounded) for the latest phase of every stage used.
            for (int s = 0; s < stages && s < issued; ++s) {
                const int last = s + ((issued - 1 - s) / stages) * stages;
                if (!mbar_wait(&full_bar[s], (last / stages) & 1)) flag(LB_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            const uint32_t idesc = umma_idesc_bf16(BM, Nc);
            for (int i = 0; i < nk; ++i) {
                const int s = i % stages;
                const uint32_t ph = (i / stages) & 1;
                if (!mbar_wait(&full_bar[s], ph)) {
                    atomicExch(&aborted, 1);
                    flag(LB_DEV_TIMEOUT);
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
                const uint32_t sb = sa + a_bytes;
#pragma unroll
                for (int kk = 0; kk < BK / UK; ++kk) {
                    umma_bf16(tmem, sw128_kmajor_desc(sa + kk * UK * 2), sw128_kmajor_desc(sb + kk * UK * 2),
                              idesc, (i > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&empty_bar[s]);   // stage free once these MMAs have read it
            }
            umma_commit(&acc_bar);            // accumulator complete
        }
    }
    __syncwarp();

    // ---------------- epilogue: all four warps, thread tid <-> TMEM lane tid
    bool ok = mbar_wait(&acc_bar, 0);
    if (!ok) flag(LB_DEV_TIMEOUT);
    tc_fence_after();
    ok = ok && (nk > 0) && !*reinterpret_cast<volatile int *>(&aborted);
    ok = __all_sync(kFull, ok);   // tcgen05.ld below is warp-collective
    const int64_t rowbase = static_cast<int64_t>(b) * p.T;
    const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);

    if constexpr (SPLITN) {
        // rank this CTA's experts per row; hand the list over in shared
        // memory (the pipeline buffers are free: acc_bar completed)
        const int row = m0 + tid;
        const bool valid = ok && row < p.T;
        const uint32_t kmask = id_mask(p.E);
        TopK<KMAX> tk;
        tk.init();
        float *lrow = (p.logits != nullptr && valid) ? p.logits + (rowbase + row) * p.E : nullptr;
        if (ok) {
            for (int c0 = 0; c0 < Nc; c0 += 16) {
                uint32_t r[16];
                tmem_ld16(tl + c0, r);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int c = c_off + c0 + q;
                    const float x = __uint_as_float(r[q]) + bias_s[c];
                    tk.push(c < p.E ? rank_key(x, c, kmask) : 0u);
                    if (lrow && c < p.E) lrow[c] = x;
                }
            }
        }
        uint32_t *lists = reinterpret_cast<uint32_t *>(smem);   // [BM][KMAX]
#pragma unroll
        for (int j = 0; j < KMAX; ++j) lists[tid * KMAX + j] = tk.key[j];
        cluster_sync();   // every CTA of the cluster passes both barriers, always
        const int R = BM / S;
        if (tid < R) {
            const int trow = crank * R + tid;
            const int grow_ = m0 + trow;
            TopK<KMAX> mg;
            mg.init();
            const uint32_t laddr = smem_u32(lists + trow * KMAX);
            for (int s2 = 0; s2 < S; ++s2) {
                const uint32_t ra = mapa_shared(laddr, s2);
#pragma unroll
                for (int j = 0; j < KMAX; ++j) mg.push(static_cast<uint32_t>(ld_cluster_i32(ra + 4 * j)));
            }
            if (grow_ < p.T) {
                int32_t *out = p.ids + (rowbase + grow_) * p.k;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (j < p.k) out[j] = key_id(mg.key[j], kmask);
            }
        }
        cluster_sync();   // keep this CTA's lists alive until all readers are done
    } else if constexpr (!SPLITK) {
        const int row = m0 + tid;
        const bool valid = ok && row < p.T;
        const uint32_t kmask = id_mask(p.E);
        TopK<KMAX> tk;
        tk.init();
        float *lrow = (p.logits != nullptr && valid) ? p.logits + (rowbase + row) * p.E : nullptr;
        if (ok) {
            for (int c0 = 0; c0 < p.Epad; c0 += 16) {
                uint32_t r[16];
                tmem_ld16(tl + c0, r);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int c = c0 + q;
                    const float x = __uint_as_float(r[q]) + bias_s[c];
                    tk.push(c < p.E ? rank_key(x, c, kmask) : 0u);
                    if (lrow && c < p.E) lrow[c] = x;
                }
            }
        }
        if (valid) {
            int32_t *out = p.ids + (rowbase + row) * p.k;
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if (j < p.k) out[j] = key_id(tk.key[j], kmask);
        }
    } else {
        // Stage the partial tile in this CTA's shared memory (pipeline buffers
        // are free: every TMA write landed and every MMA read finished before
        // acc_bar completed).
        const int PS = p.Epad + 4;   // padded row stride in floats
        float *part = reinterpret_cast<float *>(smem);
        if (ok) {
            for (int c0 = 0; c0 < p.Epad; c0 += 16) {
                uint32_t r[16];
                tmem_ld16(tl + c0, r);
                tmem_wait_ld();
                float4 *dst = reinterpret_cast<float4 *>(part + tid * PS + c0);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                         __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
            }
        } else {
            for (int c = 0; c < p.Epad; ++c) part[tid * PS + c] = 0.f;
        }
        cluster_sync();   // every CTA of the cluster passes both barriers, always
        const int R = BM / S;          // rows this CTA finishes
        const int rl = tid / S, pp = tid % S;
        const int trow = crank * R + rl;
        const int row = m0 + trow;
        const int C = p.Epad / S;      // columns per thread (multiple of 4)
        const uint32_t kmask = id_mask(p.E);
        TopK<KMAX> tk;
        tk.init();
        const bool valid = row < p.T;
        float *lrow = (p.logits != nullptr && valid) ? p.logits + (rowbase + row) * p.E : nullptr;
        const uint32_t pbase = smem_u32(part + trow * PS);
        for (int c = pp * C; c < pp * C + C; c += 4) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s = 0; s < S; ++s) {
                const float4 x = ld_cluster_f4(mapa_shared(pbase + c * 4, s));
                acc.x += x.x;
                acc.y += x.y;
                acc.z += x.z;
                acc.w += x.w;
            }
            const float xs[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int cc = c + q;
                if (cc < p.E) {
                    const float x = xs[q] + bias_s[cc];
                    tk.push(rank_key(x, cc, kmask));
                    if (lrow) lrow[cc] = x;
                }
            }
        }
        uint32_t best[KMAX];
        tk.merge(S, best);
        if (valid && pp == 0) {
            int32_t *out = p.ids + (rowbase + row) * p.k;
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if (j < p.k) out[j] = key_id(best[j], kmask);
        }
        cluster_sync();   // keep this CTA's partials alive until all readers are done
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}


// ---------------------------------------------------------------------------
// Persistent variant, for when the token tiles fill the GPU.  One or two CTAs
// per SM walk the work units blockIdx.x, blockIdx.x + gridDim.x, ... of all
// problems; a unit is MP consecutive 128-token tiles that share every W box
// (one MMA per tile and k-block into its own accumulator), so W crosses
// from L2 once per MP tiles.  Warp 0 (one lane) keeps the TMA ring full across tile
// boundaries, warp 1 (one lane) issues the MMAs, and 8 or 16 warps run the
// epilogue.  The TMEM
// accumulator is double-buffered (2 x Epad columns), so the top-k of tile i
// overlaps the loads and MMAs of tile i+1.  h is streamed once (L2
// evict-first); W is re-read by every tile of its problem (L2 evict-last).
//
// In chain mode (see Params) the kernel evaluates both gates that read one
// hidden state: h_b feeds the normal router of layer b-1 (gate W_{b-1}) and
// the lookahead of layer b (gate W_b, FreeBalance sec. 3.2, predicted
// routing from the previous layer's hidden state).  The two gates are
// adjacent rows of the stacked [L*E, H] weights, so one N = 2E MMA tile per
// k-block covers both, and each hidden state crosses HBM once instead of
// twice.
// Epilogue warp sets: ES = 2 (eight epilogue warps, two per TMEM lane
// quadrant) or ES = 4 (sixteen; used at one CTA per SM, where the registers
// allow it and the wide tiles need the top-k throughput).
template <int ES>
struct Shape {
    static constexpr int THREADS = 64 + 128 * ES;   // warp 0 TMA, warp 1 MMA, 4 * ES epilogue warps
    static constexpr int EPI = 128 * ES;            // epilogue threads
};

// The ES epilogue warps of TMEM lane quadrant q meet at named barrier 1 + q
// (ids and thread counts as immediates, so the kernel reserves barriers 0..4).
template <int ID, int CNT>
__device__ __forceinline__ bool quad_all_id(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pa, pb;\n\t"
        "setp.ne.u32 pa, %1, 0;\n\t"
        "bar.red.and.pred pb, %2, %3, pa;\n\t"
        "selp.u32 %0, 1, 0, pb;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "n"(ID), "n"(CNT)
        : "memory");
    return r != 0;
}
template <int ID, int CNT>
__device__ __forceinline__ void quad_sync_id() {
    asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(CNT) : "memory");
}
template <int CNT>
__device__ __forceinline__ bool quad_all(int q, bool v) {
    switch (q) {
        case 0: return quad_all_id<1, CNT>(v);
        case 1: return quad_all_id<2, CNT>(v);
        case 2: return quad_all_id<3, CNT>(v);
        default: return quad_all_id<4, CNT>(v);
    }
}
template <int CNT>
__device__ __forceinline__ void quad_sync(int q) {
    switch (q) {
        case 0: quad_sync_id<1, CNT>(); break;
        case 1: quad_sync_id<2, CNT>(); break;
        case 2: quad_sync_id<3, CNT>(); break;
        default: quad_sync_id<4, CNT>(); break;
    }
}

// Merge a sorted key list with another sorted list read back from shared
// memory (ok[j * 32] for this lane): pairwise best against the reversed
// other list, then a half-cleaner cascade (bitonic); the result is the best
// KMAX of both, sorted.
template <int KMAX>
__device__ __forceinline__ void merge_sorted(uint32_t (&key)[KMAX], const uint32_t *ok) {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) key[j] = max(key[j], ok[(KMAX - 1 - j) * 32]);
#pragma unroll
    for (int st = KMAX / 2; st > 0; st >>= 1) {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if ((j & st) == 0) {
                const uint32_t hi = max(key[j], key[j + st]), lo = min(key[j], key[j + st]);
                key[j] = hi;
                key[j + st] = lo;
            }
        }
    }
}

// PAIR: the CTAs of each cluster of two share one MMA of M = 256 (see the
// CTA-pair helpers in common.cuh).  A work unit is then two consecutive
// 128-token tiles, one per CTA; each CTA loads its own h rows and half of
// the unit's B rows (chain mode: CTA 0 the gate W_{b-1}, CTA 1 the gate W_b),
// so every W byte crosses into one SM per unit instead of two.  Rank 0's
// producer expects the bytes of both CTAs' loads on its own full barrier
// (rank 1's loads complete there), rank 0's MMA warp issues every MMA and
// commits to the stage-free and accumulator-full barriers of both CTAs, and
// the epilogue warps of both CTAs release an accumulator buffer on rank 0's
// empty barrier.  Each CTA ranks its own 128 rows of each M-tile.  With
// MP = 2 a unit is two such pair tiles (512 tokens) sharing every W box,
// each into its own accumulator (sixteen epilogue warps, ES = 4).
template <int KMAX, int ES, int MP, bool PAIR = false>
__global__ void __launch_bounds__(Shape<ES>::THREADS, ES == 2 ? 2 : 1)
    gate_topk_persistent(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const Params p, int mtiles, int ntiles) {
    static_assert(!PAIR || ES == 4, "CTA pairs: sixteen epilogue warps");
    extern __shared__ uint8_t smem_raw[];
    pdl_begin();
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    __shared__ __align__(8) uint64_t full_bar[MAX_STAGES];
    __shared__ __align__(8) uint64_t empty_bar[MAX_STAGES];
    __shared__ __align__(8) uint64_t acc_full[2];
    __shared__ __align__(8) uint64_t acc_empty[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int aborted;
    // each epilogue warp's copy of its columns' bias; lists handed over for
    // merging: per quadrant, the lists of every part but the first of each
    // gate (chain: 2 gates x (ES/2 - 1) parts; normal: 1 gate x (ES - 1))
    constexpr int MLISTS = ES - MP > 1 ? ES - MP : 1;
    // (a warp ranks a whole gate only with 8 epilogue warps and two tiles per
    // unit; every other layout splits a gate of at most 256 columns in two)
    constexpr int BW = (ES == 2 && MP == 2) ? LB_MAX_E_GATE : LB_MAX_E_GATE / 2;
    __shared__ __align__(16) float bias_w[4 * ES][BW];
    __shared__ uint32_t merge_k[4][MLISTS][KMAX][32];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t a_box = BM * 128u, b_box = static_cast<uint32_t>(PAIR ? p.Epad / 2 : p.Epad) * 128u;
    const int kbox = p.kbox;
    // work units: PAIR walks units of two tiles per cluster, else one per CTA
    const int crank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
    const int ufirst = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int ustep = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    const uint32_t a_bytes = a_box * kbox * MP;         // A boxes first (M-tile by M-tile), then B boxes
    const uint32_t stage_bytes = (a_box * MP + b_box) * kbox;
    const int stages = p.stages;
    const int nks = (p.nkb + kbox - 1) / kbox;          // stages per work unit (boxes past H read zeros)
    const int nbuf = p.nbuf;
    const uint32_t bufcols = p.tmem_cols / nbuf;        // TMEM columns of one accumulator buffer (MP tiles)

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            // PAIR: one arrival per epilogue warp of both CTAs (on rank 0's)
            mbar_init(&acc_empty[i], PAIR ? 2 * (Shape<ES>::EPI / 32) : Shape<ES>::EPI);
        }
        mbar_init(&drain_bar, 1);
        aborted = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(&tmem_slot, p.tmem_cols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&tmem_slot, p.tmem_cols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    // PAIR: both CTAs' barriers are initialized and their TMEM allocated
    // before either signals the other
    if constexpr (PAIR) cluster_sync();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    volatile int *abort_flag = &aborted;
    // rank 0's copies of the barriers every CTA of the pair signals
    const uint32_t full0 = PAIR ? mapa_shared(smem_u32(&full_bar[0]), 0) : smem_u32(&full_bar[0]);
    const uint32_t accempty0 = PAIR ? mapa_shared(smem_u32(&acc_empty[0]), 0) : smem_u32(&acc_empty[0]);

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            const uint64_t pol_a = l2_policy_evict_first(), pol_b = l2_policy_evict_last();
            int it = 0;
            bool ok = true;
            for (int tile = ufirst; tile < ntiles && ok; tile += ustep) {
                const int b = tile / mtiles;
                // PAIR: M-tile mt of the unit is rows [mt 2BM, (mt+1) 2BM) of it,
                // this CTA's half of them starting at m0 + mt 2BM
                const int m0 = PAIR ? (tile - b * mtiles) * 2 * BM * MP + crank * BM : (tile - b * mtiles) * BM * MP;
                for (int ks = 0; ks < nks; ++ks, ++it) {
                    const int s = it % stages;
                    const uint32_t ph = (it / stages) & 1;
                    if (!mbar_wait(&empty_bar[s], ph ^ 1) || *abort_flag) {
                        atomicExch(&aborted, 1);
                        flag(LB_DEV_TIMEOUT);
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + static_cast<size_t>(s) * stage_bytes;
                    if constexpr (PAIR) {
                        // rank 0 expects both CTAs' bytes; each CTA loads its
                        // own h rows and its half of the B rows
                        if (crank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * stage_bytes);
                        const uint32_t fb = full0 + static_cast<uint32_t>(s) * 8u;
#pragma unroll
                        for (int mt = 0; mt < MP; ++mt)
                            for (int j = 0; j < kbox; ++j)
                                tma_load_3d_pair(&tmA, sa + (mt * kbox + j) * a_box, fb, (ks * kbox + j) * BK,
                                                 m0 + mt * 2 * BM, b, pol_a);
                        const int half = p.Epad / 2;
                        const int by = (p.chain ? (b - 1) * p.E : 0) + crank * half, bz = p.chain ? 0 : b;
                        for (int j = 0; j < kbox; ++j)
                            tma_load_3d_pair(&tmB, sa + a_bytes + j * b_box, fb, (ks * kbox + j) * BK, by, bz, pol_b);
                    } else {
                        mbar_arrive_expect_tx(&full_bar[s], stage_bytes);
#pragma unroll
                        for (int mt = 0; mt < MP; ++mt)
                            for (int j = 0; j < kbox; ++j)
                                tma_load_3d_hint(&tmA, sa + (mt * kbox + j) * a_box, &full_bar[s],
                                                 (ks * kbox + j) * BK, m0 + mt * BM, b, pol_a);
                        const int by = p.chain ? (b - 1) * p.E : 0, bz = p.chain ? 0 : b;
                        for (int j = 0; j < kbox; ++j)
                            tma_load_3d_hint(&tmB, sa + a_bytes + j * b_box, &full_bar[s], (ks * kbox + j) * BK, by,
                                             bz, pol_b);
                    }
                }
            }
            // no copies left in flight into this CTA's shared memory (PAIR:
            // rank 0's full barriers count both CTAs' copies; rank 1 is held
            // at the closing cluster barrier until rank 0 has seen them land)
            if (!PAIR || crank == 0) {
                for (int s = 0; s < stages && s < it; ++s) {
                    const int last = s + ((it - 1 - s) / stages) * stages;
                    if (!mbar_wait(&full_bar[s], (last / stages) & 1)) flag(LB_DEV_TIMEOUT);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && (!PAIR || crank == 0)) {
            // ---------------- MMA issuer (PAIR: rank 0 only)
            const uint32_t idesc = umma_idesc_bf16(PAIR ? 2 * BM : BM, p.Epad);
            int it = 0, tl = 0;
            bool ok = true;
            for (int tile = ufirst; tile < ntiles && ok; tile += ustep, ++tl) {
                const int buf = tl % nbuf;
                const uint32_t use = static_cast<uint32_t>(tl / nbuf);
                if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1) || *abort_flag) {
                    atomicExch(&aborted, 1);
                    flag(LB_DEV_TIMEOUT);
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + buf * bufcols;   // M-tile mt accumulates at d + mt * Epad
                for (int ks = 0; ks < nks; ++ks, ++it) {
                    const int s = it % stages;
                    const uint32_t ph = (it / stages) & 1;
                    if (!mbar_wait(&full_bar[s], ph)) {
                        atomicExch(&aborted, 1);
                        flag(LB_DEV_TIMEOUT);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
                    for (int j = 0; j < kbox; ++j) {
                        const uint32_t sb = st + a_bytes + j * b_box;
#pragma unroll
                        for (int mt = 0; mt < MP; ++mt) {
                            const uint32_t sa = st + (mt * kbox + j) * a_box;
#pragma unroll
                            for (int kk = 0; kk < BK / UK; ++kk) {
                                const uint32_t acc = (ks > 0 || j > 0 || kk > 0) ? 1u : 0u;
                                if constexpr (PAIR)
                                    umma_bf16_pair(d + mt * static_cast<uint32_t>(p.Epad),
                                                   sw128_kmajor_desc(sa + kk * UK * 2),
                                                   sw128_kmajor_desc(sb + kk * UK * 2), idesc, acc);
                                else
                                    umma_bf16(d + mt * static_cast<uint32_t>(p.Epad), sw128_kmajor_desc(sa + kk * UK * 2),
                                              sw128_kmajor_desc(sb + kk * UK * 2), idesc, acc);
                            }
                        }
                    }
                    if constexpr (PAIR) umma_commit_pair(&empty_bar[s], 3);
                    else umma_commit(&empty_bar[s]);
                }
                if constexpr (PAIR) umma_commit_pair(&acc_full[buf], 3);
                else umma_commit(&acc_full[buf]);
            }
            // every MMA this CTA issued has finished before TMEM is freed
            if constexpr (PAIR) umma_commit_pair(&drain_bar, 1);
            else umma_commit(&drain_bar);
            if (!mbar_wait(&drain_bar, 0)) flag(LB_DEV_TIMEOUT);
        }
    } else {
        // ---------------- epilogue: warps 2 .. 2 + 4 ES - 1.  TMEM lane
        // quadrant q = warp % 4 (rows q*32..q*32+31); set s = (warp - 2) / 4
        // picks a gate and a part of its columns: chain mode has 2 gates of
        // ES/2 parts, normal mode 1 gate of ES parts.  Each warp ranks its
        // part; the first part's warp of each gate merges the other parts'
        // lists (handed over in shared memory) and writes the ids.  The ES
        // warps of a quadrant take the same decisions (quadrant barriers),
        // so they always meet at the same barriers.
        constexpr int QCNT = 32 * ES;
        constexpr int RS = ES / MP;                    // sets per M-tile of the work unit
        const int q = warp & 3;
        const int set = (warp - 2) >> 2;
        const int mt = set % MP;                       // the M-tile this warp ranks
        const int rr = set / MP;
        const int GP = p.chain ? RS / 2 : RS;          // parts per gate
        const int NG = p.chain ? 2 : 1;                // gates
        const int gate_id = rr / GP, part = rr - gate_id * GP;
        const int width = p.chain ? p.E : p.Epad;
        const int pw = ((width + GP - 1) / GP + 15) / 16 * 16;
        const int gbase = p.chain ? gate_id * p.E : 0;  // first column of this warp's gate
        const int cbeg = gbase + part * pw;
        const int cend = min(gbase + width, cbeg + pw);
        const int rloc = q * 32 + lane;
        float *wb = bias_w[warp - 2];
        uint32_t *mk = &merge_k[q][0][0][0];
        const uint32_t kmask = id_mask(p.E);
        const int mbase = (mt * NG + gate_id) * (GP - 1);  // this (M-tile, gate)'s hand-over lists
        const int mslot = mbase + part - 1;                 // this warp's list (part > 0)
        int tl = 0;
        for (int tile = ufirst; tile < ntiles; tile += ustep, ++tl) {
            const int buf = tl % nbuf;
            const uint32_t use = static_cast<uint32_t>(tl / nbuf);
            const int b = tile / mtiles;
            const int m0 = PAIR ? (tile - b * mtiles) * 2 * BM * MP + mt * 2 * BM + crank * BM
                                : (tile - b * mtiles) * BM * MP + mt * BM;
            // The layer this warp's columns belong to (uniform over the tile).
            const int layer = p.chain ? b - 1 + gate_id : b;
            const bool live = layer >= 0 && (!p.chain || layer < p.L);   // the gate has a layer here
            const bool active = live && cbeg < cend;
            // This tile's bias for the warp's columns into its own shared-
            // memory slice, before the wait for the accumulator: under the
            // full load of the h stream a global load takes microseconds,
            // and here its latency hides behind the tile's MMAs.  (The warp
            // finished reading the previous tile's copy in program order.)
            for (int c = cbeg + lane; c < cend; c += 32) {
                const int cc = c - gbase;
                wb[c - cbeg] = (p.bias != nullptr && active && cc < p.E) ? p.bias[static_cast<int64_t>(layer) * p.E + cc]
                                                                        : 0.f;
            }
            __syncwarp();
            bool ok = mbar_wait(&acc_full[buf], use & 1) && !*abort_flag;
            ok = quad_all<QCNT>(q, ok);
            if (!ok) {
                if (lane == 0) {
                    atomicExch(&aborted, 1);
                    flag(LB_DEV_TIMEOUT);
                }
                break;
            }
            tc_fence_after();
            const int row = m0 + rloc;
            const bool valid = row < p.T;
            const uint32_t tl_addr =
                tmem + buf * bufcols + mt * static_cast<uint32_t>(p.Epad) + (static_cast<uint32_t>(q * 32) << 16);
            int32_t *ids_out = (p.chain && gate_id == 1) ? p.ids2 : p.ids;
            float *lg_out = (p.chain && gate_id == 1) ? p.logits2 : p.logits;
            const int64_t grow = static_cast<int64_t>(layer) * p.T + row;
            float *lrow = (lg_out != nullptr && valid && active) ? lg_out + grow * p.E : nullptr;
            TopK<KMAX> tk;
            tk.init();
            if (active) {
                // 32 columns per TMEM load and wait (16 for a part's last
                // odd block); the bias as 16-byte shared-memory reads
                for (int c0 = cbeg; c0 < cend; c0 += 32) {
                    uint32_t r[32];
                    const bool full = c0 + 32 <= cend;   // warp-uniform
                    if (full)
                        tmem_ld32(tl_addr + c0, r);
                    else
                        tmem_ld16(tl_addr + c0, *reinterpret_cast<uint32_t(*)[16]>(r));
                    tmem_wait_ld();
                    const float4 *b4 = reinterpret_cast<const float4 *>(wb + (c0 - cbeg));
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4) {
                        if (j4 < 4 || full) {
                            const float4 bb = b4[j4];
                            const float bj[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int c = c0 + 4 * j4 + u - gbase;   // expert id within the gate
                                const float x = __uint_as_float(r[4 * j4 + u]) + bj[u];
                                tk.push(c < p.E ? rank_key(x, c, kmask) : 0u);
                                if (lrow && c < p.E) lrow[c] = x;
                            }
                        }
                    }
                }
            }
            // this warp's TMEM reads are done: the buffer may be overwritten
            tc_fence_before();
            if constexpr (PAIR) {
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(accempty0 + static_cast<uint32_t>(buf) * 8u);
            } else {
                mbar_arrive(&acc_empty[buf]);
            }
            if (GP > 1) {
                if (part > 0) {
#pragma unroll
                    for (int j = 0; j < KMAX; ++j) {
                        mk[(mslot * KMAX + j) * 32 + lane] = tk.key[j];
                    }
                }
                quad_sync<QCNT>(q);
                if (part == 0) {
                    for (int o = 1; o < GP; ++o) {
                        const int sl = mbase + o - 1;
                        merge_sorted<KMAX>(tk.key, mk + sl * KMAX * 32 + lane);
                    }
                }
                quad_sync<QCNT>(q);   // the lists may be refilled only after the merges read them
            }
            if (part == 0 && live && valid) {
                int32_t *out = ids_out + grow * p.k;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (j < p.k) out[j] = key_id(tk.key[j], kmask);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // PAIR: neither CTA leaves (or frees TMEM) while the other may still
    // signal its barriers, read its TMEM or be written by its copies
    if constexpr (PAIR) cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem, p.tmem_cols);
        else tmem_dealloc(tmem, p.tmem_cols);
    }
}

// ---------------------------------------------------------------------------
// Top KMAX of two descending key lists, into a (descending): the elementwise
// maximum of a and b reversed holds the KMAX largest keys of both as a
// bitonic sequence, which a half-cleaner network then sorts.
template <int KMAX>
__device__ __forceinline__ void merge_top(uint32_t (&a)[KMAX], const uint32_t (&b)[KMAX]) {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) a[j] = max(a[j], b[KMAX - 1 - j]);
#pragma unroll
    for (int st = KMAX / 2; st >= 1; st >>= 1)
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if ((j & st) == 0) {
                const uint32_t hi = max(a[j], a[j + st]), lo = min(a[j], a[j + st]);
                a[j] = hi;
                a[j + st] = lo;
            }
}

// Four keys into a descending top-KMAX list: sort them (the optimal network
// of five comparators), then merge as above with the four standing in for a
// list padded with the smallest key.  About half the operations of four
// separate insertions for KMAX = 8.
__device__ __forceinline__ void cmp_swap_desc(uint32_t &x, uint32_t &y) {
    const uint32_t hi = max(x, y), lo = min(x, y);
    x = hi;
    y = lo;
}
template <int KMAX>
__device__ __forceinline__ void push4(uint32_t (&a)[KMAX], uint32_t k0, uint32_t k1, uint32_t k2, uint32_t k3) {
    cmp_swap_desc(k0, k1);
    cmp_swap_desc(k2, k3);
    cmp_swap_desc(k0, k2);
    cmp_swap_desc(k1, k3);
    cmp_swap_desc(k1, k2);
    const uint32_t bk[4] = {k0, k1, k2, k3};
    constexpr int m = KMAX < 4 ? KMAX : 4;
#pragma unroll
    for (int j = KMAX - m; j < KMAX; ++j) a[j] = max(a[j], bk[KMAX - 1 - j]);
#pragma unroll
    for (int st = KMAX / 2; st >= 1; st >>= 1)
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if ((j & st) == 0) cmp_swap_desc(a[j], a[j + st]);
}

// First of the rows [row0(q), row0(q+1)) of its 128 that the CTA of pair q
// ranks: q BM / KS rounded up to a multiple of 8 (slices of 64 for two pairs,
// 48, 40, 40 for three, 32 for four).
template <int KS>
__device__ __forceinline__ int pair_slice_row0(int q) {
    return ((q * BM) / KS + 7) & ~7;
}

// CTA pairs with H split over KS pairs (per-tile, one 256-token unit per
// cluster of 2 KS CTAs; the per-layer gate of wide shapes whose token tiles
// underfill the GPU, such as the decode shape).  Ranks 2p and 2p+1 form pair
// p; within a pair, as in the persistent kernel, the even rank issues one
// tcgen05.mma of M = 256 for both, each CTA loading its own 128 tokens and
// half of the N = Epad weight rows.  Pair p accumulates k-blocks
// [p kper, (p+1) kper), kper = ceil(nkb / KS).
//
// The partial accumulators are summed by a reduce-scatter over distributed
// shared memory.  Each CTA copies its partial (128 rows x Epad fp32) from
// TMEM into its own shared memory (rows of SR = Epad rounded up to 32
// floats, float4 group g of row r stored at g ^ (r mod 8), which keeps both
// the row-per-lane writes and the row-major reads free of bank conflicts).
// After a cluster barrier (every MMA of the cluster done, so every CTA's
// pipeline buffers are free), it sends the rows that pair p' ranks (a
// slice of about 128 / KS rows, see pair_slice_row0) to the CTA of pair p'
// holding the same tokens, as bulk shared-to-shared copies of four rows,
// each issued by its own lane and completing on the receiver's mbarrier.
// Each CTA then ranks its own rows: its partial plus the received ones in
// pair order (deterministic) plus the bias, 8 or 16 threads per row over
// interleaved float4 groups, their lists merged by shuffles.
template <int KMAX, int KS>
__global__ void __launch_bounds__(Shape<4>::THREADS, 1)
    gate_topk_pairk(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Params p) {
    constexpr int RMAX = ((BM + KS - 1) / KS + 7) & ~7;        // largest row slice
    constexpr int TPR = Shape<4>::EPI / RMAX >= 16 ? 16 : 8;   // ranking threads per row
    static_assert(KS >= 2 && KS <= 4, "two to four pairs");
    static_assert(Shape<4>::EPI / TPR >= RMAX, "a ranking slot for every row of a slice");
    static_assert(TPR <= 32 && 32 % TPR == 0, "a row's ranking threads share a warp");
    extern __shared__ uint8_t smem_raw[];
    pdl_begin();
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    __shared__ __align__(8) uint64_t full_bar[MAX_STAGES];
    __shared__ __align__(8) uint64_t empty_bar[MAX_STAGES];
    __shared__ __align__(8) uint64_t acc_full;
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ __align__(8) uint64_t recv_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int aborted;
    __shared__ __align__(16) float bias_s[LB_MAX_E_GATE];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int crank = static_cast<int>(cluster_ctarank());
    const int pair = crank >> 1, half = crank & 1, lead = crank & ~1;
    const int b = blockIdx.y;
    const int unit = static_cast<int>(blockIdx.x) / (2 * KS);
    const int m0 = unit * 2 * BM + half * BM;   // this CTA's 128 rows
    const int kper = (p.nkb + KS - 1) / KS;
    const int kb0 = pair * kper;
    const int kend = min(p.nkb, kb0 + kper);
    const int kbox = p.kbox;
    const int nks = (max(0, kend - kb0) + kbox - 1) / kbox;   // stages of kbox boxes
    const uint32_t a_box = BM * 128u, b_box = static_cast<uint32_t>(p.Epad / 2) * 128u;
    const uint32_t a_bytes = a_box * kbox;
    const uint32_t stage_bytes = (a_box + b_box) * kbox;
    const int stages = p.stages;
    const int SR = (p.Epad + 31) & ~31;                         // staged row stride (floats)
    const int R = pair_slice_row0<KS>(pair + 1) - pair_slice_row0<KS>(pair);   // rows this CTA ranks
    if (tid == 0) {
        LB_TICK_ANY(40);
        LB_CTA_TIME(0);
    }

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&drain_bar, 1);
        mbar_init(&recv_bar, 1);
        aborted = 0;
        fence_mbar_init();
        // the other pairs' slices of this CTA's rows land on recv_bar
        mbar_arrive_expect_tx(&recv_bar, static_cast<uint32_t>((KS - 1) * R * SR) * 4u);
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_slot, p.tmem_cols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // every CTA's barriers and TMEM exist before any signal
    tc_fence_after();
    if (tid == 0) LB_TICK_ANY(41);
    const uint32_t tmem = tmem_slot;
    volatile int *abort_flag = &aborted;
    const uint32_t full0 = mapa_shared(smem_u32(&full_bar[0]), static_cast<uint32_t>(lead));
    const uint16_t pair_mask = static_cast<uint16_t>(3u << lead);

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs of the pair; the whole
        // warp, one lane per box)
        const uint64_t pol_a = l2_policy_evict_first(), pol_b = l2_policy_evict_last();
        const int nbox = 2 * kbox;
        int it = 0;
        for (int ks = 0; ks < nks; ++ks, ++it) {
            const int s = it % stages;
            const uint32_t ph = (it / stages) & 1;
            if (warp_wait_empty(&empty_bar[s], ph ^ 1, &aborted, lane) != 0) {
                if (lane == 0) {
                    atomicExch(&aborted, 1);
                    flag(LB_DEV_TIMEOUT);
                }
                break;
            }
            uint8_t *sa = smem + static_cast<size_t>(s) * stage_bytes;
            if (half == 0 && lane == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * stage_bytes);
            __syncwarp();
            const uint32_t fb = full0 + static_cast<uint32_t>(s) * 8u;
            for (int j = 0; j < kbox; ++j) {
                // boxes past this pair's share of H read real data (the next
                // pair's, or zeros past H) but are never multiplied: the MMA
                // stops at kend
                const int kx = (kb0 + ks * kbox + j) * BK;
                if (issues_box(s, nbox, j, lane)) tma_load_3d_pair(&tmA, sa + j * a_box, fb, kx, m0, b, pol_a);
                if (issues_box(s, nbox, kbox + j, lane))
                    tma_load_3d_pair(&tmB, sa + a_bytes + j * b_box, fb, kx, half * (p.Epad / 2), b, pol_b);
            }
        }
        if (half == 0 && lane == 0) {
            for (int s = 0; s < stages && s < it; ++s) {
                const int last = s + ((it - 1 - s) / stages) * stages;
                if (!mbar_wait(&full_bar[s], (last / stages) & 1)) flag(LB_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && half == 0) {
            // ---------------- MMA issuer (the pair's even rank)
            const uint32_t idesc = umma_idesc_bf16(2 * BM, p.Epad);
            int it = 0;
            bool first = true;
            for (int ks = 0; ks < nks; ++ks, ++it) {
                const int s = it % stages;
                const uint32_t ph = (it / stages) & 1;
                if (!mbar_wait(&full_bar[s], ph) || *abort_flag) {
                    atomicExch(&aborted, 1);
                    flag(LB_DEV_TIMEOUT);
                    break;
                }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
                for (int j = 0; j < kbox; ++j) {
                    if (kb0 + ks * kbox + j >= kend) break;   // this pair's share of H only
                    const uint32_t sa = st + j * a_box, sb = st + a_bytes + j * b_box;
#pragma unroll
                    for (int kk = 0; kk < BK / UK; ++kk) {
                        umma_bf16_pair(tmem, sw128_kmajor_desc(sa + kk * UK * 2), sw128_kmajor_desc(sb + kk * UK * 2),
                                       idesc, first ? 0u : 1u);
                        first = false;
                    }
                }
                umma_commit_pair(&empty_bar[s], pair_mask);
            }
            LB_TICK_ANY(44);
            umma_commit_pair(&acc_full, pair_mask);
            umma_commit_pair(&drain_bar, static_cast<uint16_t>(1u << lead));
            if (!mbar_wait(&drain_bar, 0)) flag(LB_DEV_TIMEOUT);
        }
    }
    __syncwarp();

    // ---------------- epilogue warps 2..17
    const bool epi = warp >= 2;
    const int ew = warp - 2;
    float *stage_f = reinterpret_cast<float *>(smem);   // [128][SR], reusing the pipeline buffers
    float *recv_f = stage_f + BM * SR;                   // [KS-1][RMAX][SR]
    bool ok = true;
    if (epi) {
        // the bias, staged by the epilogue warps while the main loop runs (its
        // load is off the path to the first tiles); the cluster barrier after
        // the partials are staged orders it before the ranking reads it
        for (int c = tid - 64; c < p.Epad; c += Shape<4>::EPI)
            bias_s[c] = (p.bias != nullptr && c < p.E) ? p.bias[static_cast<int64_t>(b) * p.E + c] : 0.f;
        ok = mbar_wait(&acc_full, 0) && !*abort_flag;
        if (!ok && lane == 0) flag(LB_DEV_TIMEOUT);
        ok = __all_sync(kFull, ok);
        tc_fence_after();
        if (tid == 64) LB_TICK_ANY(47);
        // TMEM lane quadrant q = warp % 4, a quarter of the columns per warp
        const int q = warp & 3, part = ew >> 2;
        const int pw = ((p.Epad + 3) / 4 + 15) / 16 * 16;
        const int cbeg = part * pw, cend = min(p.Epad, cbeg + pw);
        const int r = q * 32 + lane;
        float *srow = stage_f + r * SR;
        const uint32_t tl_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
        for (int c0 = cbeg; c0 < cend; c0 += 32) {
            // two loads of 16 columns per wait (cend - c0 is a multiple of 16)
            uint32_t v[2][16];
            const bool two = c0 + 16 < cend;
            tmem_ld16(tl_addr + c0, v[0]);
            if (two) tmem_ld16(tl_addr + c0 + 16, v[1]);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (u >= 4 && !two) break;
                const int g = (c0 >> 2) + u;
                const uint32_t *w = v[u >> 2] + 4 * (u & 3);
                *reinterpret_cast<float4 *>(srow + ((g ^ (r & 7)) << 2)) =
                    make_float4(__uint_as_float(w[0]), __uint_as_float(w[1]), __uint_as_float(w[2]),
                                __uint_as_float(w[3]));
            }
        }
        if (tid == 64) LB_TICK_ANY(54);
        fence_proxy_async_smem();   // the staged rows, before the bulk copies read them
    }
    cluster_sync();   // every partial staged; every CTA's buffers free for the slices
    if (epi && ew == 0) {
        // chunks of 4 rows, one lane each (one thread's bulk copies are served
        // one after another)
        if (lane == 0) LB_TICK_ANY(48);
        const int slot = pair;   // this pair's slot at every receiver of a higher pair (pair - 1 below)
        for (int o = 0; o < KS - 1; ++o) {
            const int pp = o < pair ? o : o + 1;   // receiving pair
            const uint32_t dst_rank = static_cast<uint32_t>(2 * pp + half);
            const int r0 = pair_slice_row0<KS>(pp), nch = (pair_slice_row0<KS>(pp + 1) - r0) / 4;
            const int dslot = pair < pp ? slot : slot - 1;
            for (int ch = lane; ch < nch; ch += 32)
                bulk_copy_to_cta(mapa_shared(smem_u32(recv_f + (dslot * RMAX + ch * 4) * SR), dst_rank),
                                 smem_u32(stage_f + (r0 + ch * 4) * SR), static_cast<uint32_t>(4 * SR) * 4u,
                                 mapa_shared(smem_u32(&recv_bar), dst_rank));
        }
    }
    if (epi) {
        const bool got = mbar_wait(&recv_bar, 0);
        if (!got && lane == 0) flag(LB_DEV_TIMEOUT);
        if (tid == 64) LB_TICK_ANY(52);
        const int lr = ew * (32 / TPR) + lane / TPR;   // row within this CTA's slice
        const int pt = lane % TPR;
        const bool active = lr < R;                    // (a slot per row; spare slots rank nothing)
        const int r = pair_slice_row0<KS>(pair) + lr;  // row within the CTA's 128
        const int row = m0 + r;
        const bool valid = ok && got && active && row < p.T;
        const uint32_t kmask = id_mask(p.E);
        const int64_t grow = static_cast<int64_t>(b) * p.T + row;
        float *lrow = (p.logits != nullptr && valid) ? p.logits + grow * p.E : nullptr;
        TopK<KMAX> tk;
        tk.init();
        const float *own = stage_f + r * SR;
        for (int g = pt; active && g < (p.Epad >> 2); g += TPR) {
            const int sg = (g ^ (r & 7)) << 2;
            float4 x = *reinterpret_cast<const float4 *>(own + sg);
#pragma unroll
            for (int o = 0; o < KS - 1; ++o) {
                const float4 y = *reinterpret_cast<const float4 *>(recv_f + (o * RMAX + lr) * SR + sg);
                x.x += y.x;
                x.y += y.y;
                x.z += y.z;
                x.w += y.w;
            }
            const float4 bv = *reinterpret_cast<const float4 *>(bias_s + 4 * g);
            const float xs[4] = {x.x + bv.x, x.y + bv.y, x.z + bv.z, x.w + bv.w};
            uint32_t key[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = 4 * g + u;
                key[u] = c < p.E ? rank_key(xs[u], c, kmask) : 0u;
                if (lrow && c < p.E) lrow[c] = xs[u];
            }
            push4<KMAX>(tk.key, key[0], key[1], key[2], key[3]);
        }
        if (tid == 64) LB_TICK_ANY(53);
#pragma unroll
        for (int d = 1; d < TPR; d <<= 1) {
            uint32_t o[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) o[j] = __shfl_xor_sync(kFull, tk.key[j], d);
            merge_top<KMAX>(tk.key, o);
        }
        if (tid == 64) LB_TICK_ANY(49);
        if (pt == 0 && valid) {
            int32_t *out = p.ids + grow * p.k;
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if (j < p.k) out[j] = key_id(tk.key[j], kmask);
        }
    }
    if (tid == 64) LB_TICK_ANY(50);
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // no CTA leaves while a slice copy may still read its shared memory
    if (tid == 0) {
        LB_TICK_ANY(51);
        LB_CTA_TIME(1);
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, p.tmem_cols);
    }
}

}  // namespace gate
}  // namespace lb
