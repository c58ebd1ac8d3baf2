// topk_core.cuh -- the per-query block selection of the walk-through
// (news.rkmt.cn/news/25027, section 五 step 3): 4 local blocks + the 12
// highest-scoring remote blocks (score desc, then lower id), optionally limited
// to the candidates of a page-aware bitmap.  topk_select runs one query on a
// CTA (few long rows: decode); topk_warp_select runs one query on a warp (many
// rows: a prefill chunk), with the same steps at warp scope.
//
// Every candidate's ranking key is the 64-bit composite
// (order-preserving fp32 key << 32 | ~id): distinct, larger for a higher score
// and, among equal scores, for the lower id.
//   1. The candidates' scores are read once from L2 as order-preserving keys
//      (masked-out candidates get key 0): into registers for rows of up to
//      8 T candidates, else into shared memory.
//   2. Threshold: the 12th largest of 16 group maxima (groups of T/16
//      threads).  Those 12 maxima are 12 distinct candidates at or above it, so
//      every member of the top 12 is at or above it too.
//   3. Survivors (keys >= threshold; typically a few dozen) are appended to a
//      shared list and ranked by counting; ranks 0..11 are the answer.
//   4. One warp writes the 12 ids in ascending order plus the 4 local blocks.
// If the survivors overflow their list (heavily tied scores) the CTA falls
// back to an exact two-level extraction (12 rounds of a warp-wide max per warp,
// then 12 rounds over the warps' survivors).
#pragma once

#include "common.cuh"

namespace uocr {

constexpr int kSurvivorCap = 2048;          // survivor list capacity (16 KiB)
constexpr int kTopkGroups = 16;             // threshold from 16 group maxima (>= kRemote)

// Larger key <=> larger float; -0 and +0 map to the same key (they compare equal): adding +0
// turns -0 into +0 (round to nearest), then negative floats have all bits flipped and
// non-negative ones the sign bit set.
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);
    return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}

__device__ __forceinline__ uint64_t composite(uint32_t key, int j) {
    return ((uint64_t)key << 32) | (uint32_t)(~(uint32_t)j);
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

// Keys of one query's candidates: staged in shared memory, or read from the scores row.
// A candidate that the optional candidate mask excludes gets key 0, below every real key
// (order_key never returns 0 for a non-NaN score).
struct KeySource {
    const uint32_t *smem;
    const float *row;
    const uint32_t *mask;   // this sequence's candidate bitmap, or NULL
    __device__ __forceinline__ uint32_t raw(int j) const {
        // both loads are issued before either is used
        const float f = __ldcg(row + j);
        const bool ok = !mask || ((__ldg(mask + (j >> 5)) >> (j & 31)) & 1u);
        return ok ? order_key(f) : 0u;
    }
    __device__ __forceinline__ uint32_t operator()(int j) const { return smem ? smem[j] : raw(j); }
};

// Largest composite strictly below `cap` among candidates j = first, first + stride, ... < n
// (0 when there is none; a real composite is never 0 because ~j != 0 for j < 2^31 - 1).
__device__ __forceinline__ uint64_t best_below(const KeySource &key, int first, int stride, int n,
                                               uint64_t cap) {
    uint64_t best = 0;
    for (int j = first; j < n; j += stride) {
        const uint64_t c = composite(key(j), j);
        if (c < cap && c > best) best = c;
    }
    return best;
}

// Exact fallback: the top kRemote composites of candidates [0, nc) into out_c[0..11].
// Called by every thread of a CTA of T threads.
template <int T>
__device__ void topk_two_level(const KeySource &key, int nc, uint64_t *s_cand, uint64_t *out_c) {
    constexpr int kW = T / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint64_t cap = ~0ull;
    uint64_t mine = best_below(key, tid, T, nc, cap);
#pragma unroll 1
    for (int k = 0; k < kRemote; ++k) {
        const uint64_t w = warp_max_u64(mine);
        if (lane == 0) s_cand[warp * kRemote + k] = w;   // 0 when the warp ran out of candidates
        if (mine == w && w != 0) {
            cap = mine;
            mine = best_below(key, tid, T, nc, cap);
        }
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int kPer = kW * kRemote / 32;   // survivors per lane
        static_assert(kW * kRemote % 32 == 0, "warps x 12 survivors must fill whole lanes");
        uint64_t c[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) c[e] = s_cand[lane * kPer + e];
#pragma unroll 1
        for (int k = 0; k < kRemote; ++k) {
            uint64_t best = 0;
            int at = -1;
#pragma unroll
            for (int e = 0; e < kPer; ++e)
                if (c[e] > best) {
                    best = c[e];
                    at = e;
                }
            const uint64_t w = warp_max_u64(best);
            if (best == w && at >= 0) {
#pragma unroll
                for (int e = 0; e < kPer; ++e)
                    if (e == at) c[e] = 0;
            }
            if (lane == 0) out_c[k] = w;
        }
    }
    __syncthreads();
}


constexpr int kTopkRegKeys = 8;            // rows of at most 8 T candidates keep their keys in registers

template <int T>
struct TopkShared {
    uint64_t surv[kSurvivorCap];
    uint64_t cand[(T / 32) * kRemote];
    uint64_t top[kRemote];
    uint32_t gmax[kTopkGroups];
    uint32_t thr;
    int n;
    int allowed;
};

// Selection of one query with nb causal blocks from its score row; every thread of a CTA of
// T threads calls it (the CTA-wide barriers inside must be reached by all of them).
// s_keys: shared staging for at least nb - 4 keys, or NULL to read the row from L2 each pass.
// out: the query's 16 selection slots.
template <int T>
__device__ void topk_select(const float *row, int nb, const uint32_t *mask, uint32_t *s_keys,
                            TopkShared<T> &sm, int32_t *out) {
    constexpr int kW = T / 32;
    constexpr int kGroup = T / kTopkGroups;     // threads per group: 16 or 32
    static_assert(kGroup == 16 || kGroup == 32, "16 groups of a half-warp or a warp");
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int nc = nb - kLocal > 0 ? nb - kLocal : 0;
    if (nc <= kRemote && !mask) {
        // every causal block fits in the 16 slots
        if (tid < kSel) out[tid] = tid < nb ? tid : -1;
        return;
    }
    KeySource key{nullptr, row, mask};
    if (tid == 0) {
        sm.n = 0;
        sm.allowed = 0;
    }
    __syncthreads();

    // ---- 1. stage keys, 2. per-thread then per-group maximum
    // Rows of at most kTopkRegKeys * T candidates: a thread holds one chunk of kTopkRegKeys
    // consecutive candidates in registers (two 16-byte loads on an aligned row, else scalar
    // loads, all issued before any is used; one byte of a word of the candidate mask).  Chunk k
    // goes to thread (k % 16) * kGroup + k / 16, so that consecutive chunks fall in different
    // groups and every group holds candidates whenever the row has 16 chunks: a short row packed
    // into the first groups would leave the other group maxima at 0, the threshold at 0 and
    // every candidate a survivor.  Longer rows are staged in shared memory (or re-read from L2
    // when they do not fit there).
    static_assert(kTopkRegKeys == 8, "a thread's candidates are two float4 and one byte of a mask word");
    const bool in_regs = nc <= kTopkRegKeys * T;
    // first candidate of this thread's chunk on the register path
    const int jr = kTopkRegKeys * ((tid % kGroup) * kTopkGroups + tid / kGroup);
    uint32_t kr[kTopkRegKeys];
    uint32_t tmax = 0;
    int allowed = 0;
    if (in_regs) {
        float f[kTopkRegKeys];
        if ((reinterpret_cast<uintptr_t>(row) & 15) == 0 && jr + kTopkRegKeys <= nc) {
            const float4 a = __ldcg(reinterpret_cast<const float4 *>(row + jr));
            const float4 b = __ldcg(reinterpret_cast<const float4 *>(row + jr) + 1);
            f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
            f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
        } else {
#pragma unroll
            for (int u = 0; u < kTopkRegKeys; ++u) f[u] = jr + u < nc ? __ldcg(row + jr + u) : 0.f;
        }
        const uint32_t mbits = mask ? (jr < nc ? __ldg(mask + (jr >> 5)) >> (jr & 31) : 0u) : 0xffu;
#pragma unroll
        for (int u = 0; u < kTopkRegKeys; ++u) {
            kr[u] = (jr + u < nc && ((mbits >> u) & 1u)) ? order_key(f[u]) : 0u;
            tmax = kr[u] > tmax ? kr[u] : tmax;
            allowed += kr[u] != 0u;
        }
    } else {
        // batches of kTopkRegKeys loads per thread, all issued before any is used
        for (int jb = 0; jb < nc; jb += kTopkRegKeys * T) {
            uint32_t kk[kTopkRegKeys];
#pragma unroll
            for (int u = 0; u < kTopkRegKeys; ++u) {
                const int j = jb + u * T + tid;
                kk[u] = j < nc ? key.raw(j) : 0u;
            }
#pragma unroll
            for (int u = 0; u < kTopkRegKeys; ++u) {
                const int j = jb + u * T + tid;
                if (j < nc && s_keys) s_keys[j] = kk[u];
                tmax = kk[u] > tmax ? kk[u] : tmax;
                allowed += kk[u] != 0u;
            }
        }
        if (s_keys) key.smem = s_keys;
    }
    uint32_t gm = tmax;
    if (kGroup == 32) {
        gm = __reduce_max_sync(0xffffffffu, gm);
    } else {
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
            const uint32_t other = __shfl_xor_sync(0xffffffffu, gm, o);
            gm = other > gm ? other : gm;
        }
    }
    if (tid % kGroup == 0) sm.gmax[tid / kGroup] = gm;
    if (mask) {
        const int wa = __reduce_add_sync(0xffffffffu, allowed);
        if (lane == 0) atomicAdd(&sm.allowed, wa);
    }
    __syncthreads();

    if (mask && sm.allowed <= kRemote) {
        // no more allowed candidates than remote slots: take them all, in id order
        if (warp == 0) {
            int pos = 0;
            for (int base = 0; base < nc; base += 32) {
                const int j = base + lane;
                const bool take = j < nc && key(j) != 0u;
                const unsigned m = __ballot_sync(0xffffffffu, take);
                if (take) out[pos + __popc(m & ((1u << lane) - 1u))] = j;
                pos += __popc(m);
            }
            const int n_loc = nb < kLocal ? nb : kLocal;
            if (lane < n_loc) out[pos + lane] = nb - n_loc + lane;
            if (lane >= pos + n_loc && lane < kSel) out[lane] = -1;
        }
        return;
    }

    // ---- threshold = the kRemote-th largest group maximum (with multiplicity)
    if (warp == 0) {
        const uint32_t v = lane < kTopkGroups ? sm.gmax[lane] : 0u;
        int gt = 0, ge = 0;
#pragma unroll
        for (int w = 0; w < kTopkGroups; ++w) {
            const uint32_t o = sm.gmax[w];
            gt += o > v;
            ge += o >= v;
        }
        const bool is_thr = lane < kTopkGroups && gt <= kRemote - 1 && kRemote - 1 < ge;
        const unsigned who = __ballot_sync(0xffffffffu, is_thr);
        if (lane == __ffs(who) - 1) sm.thr = v;
    }
    __syncthreads();
    const uint32_t thr = sm.thr;

    // ---- 3. survivors: every candidate at or above the threshold
    auto append = [&](uint32_t k, int j, bool keep) {
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        if (m) {
            const int leader = __ffs(m) - 1;
            int base = 0;
            if (lane == leader) base = atomicAdd(&sm.n, __popc(m));
            base = __shfl_sync(0xffffffffu, base, leader);
            const int slot = base + __popc(m & ((1u << lane) - 1u));
            if (keep && slot < kSurvivorCap) sm.surv[slot] = composite(k, j);
        }
    };
    if (in_regs) {
        // this thread's survivors (the staged path's test), placed by one warp prefix sum and
        // one shared atomic per warp
        unsigned keep = 0;
#pragma unroll
        for (int u = 0; u < kTopkRegKeys; ++u)
            if (jr + u < nc && kr[u] >= thr) keep |= 1u << u;
        const int cnt = __popc(keep);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int wtot = __shfl_sync(0xffffffffu, incl, 31);
        int base = 0;
        if (wtot > 0) {
            if (lane == 31) base = atomicAdd(&sm.n, wtot);
            base = __shfl_sync(0xffffffffu, base, 31) + incl - cnt;
#pragma unroll
            for (int u = 0; u < kTopkRegKeys; ++u)
                if ((keep >> u) & 1u) {
                    if (base < kSurvivorCap) sm.surv[base] = composite(kr[u], jr + u);
                    ++base;
                }
        }
    } else {
    for (int j0 = 0; j0 < nc; j0 += T) {
        const int j = j0 + tid;
        const uint32_t k = j < nc ? key(j) : 0u;
        const bool keep = j < nc && k >= thr;
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        if (m) {
            const int leader = __ffs(m) - 1;
            int base = 0;
            if (lane == leader) base = atomicAdd(&sm.n, __popc(m));
            base = __shfl_sync(0xffffffffu, base, leader);
            const int slot = base + __popc(m & ((1u << lane) - 1u));
            if (keep && slot < kSurvivorCap) sm.surv[slot] = composite(k, j);
        }
    }
    }
    __syncthreads();
    const int n = sm.n;
    if (n <= 32) {
        // one survivor per lane of warp 0, ranked by counting over shuffles
        if (warp == 0) {
            const uint64_t c = lane < n ? sm.surv[lane] : 0ull;
            int rank = 0;
            for (int b = 0; b < n; ++b) rank += __shfl_sync(0xffffffffu, c, b) > c;
            if (lane < n && rank < kRemote) sm.top[rank] = c;
        }
        __syncthreads();
    } else if (n <= kSurvivorCap) {
        for (int a = tid; a < n; a += T) {
            const uint64_t c = sm.surv[a];
            int rank = 0;
            for (int b = 0; b < n; ++b) rank += sm.surv[b] > c;
            if (rank < kRemote) sm.top[rank] = c;
        }
        __syncthreads();
    } else {
        topk_two_level<T>(key, nc, sm.cand, sm.top);
    }

    // ---- 4. the 12 remote ids ascending, then the 4 local blocks
    if (warp == 0) {
        const int id = lane < kRemote ? (int)~(uint32_t)(sm.top[lane] & 0xffffffffu) : 0x7fffffff;
        int rank = 0;
#pragma unroll
        for (int k = 0; k < kRemote; ++k) {
            const int other = __shfl_sync(0xffffffffu, id, k);
            rank += other < id;
        }
        if (lane < kRemote) out[rank] = id;
        if (lane < kLocal) out[kRemote + lane] = nb - kLocal + lane;
    }
    (void)kW;
}

// ------------------------------------------------------------ one warp per query
constexpr int kWarpSurvivorCap = 256;       // per-warp survivor list (2 KiB)

struct TopkWarpShared {
    uint64_t surv[kWarpSurvivorCap];
    uint64_t top[kRemote];
};

// The 12 remote ids of `top` ascending into out[0..11], the local blocks into out[12..15].
__device__ __forceinline__ void topk_warp_emit(const uint64_t *top, int nb, int lane, int32_t *out) {
    const int id = lane < kRemote ? (int)~(uint32_t)(top[lane] & 0xffffffffu) : 0x7fffffff;
    int rank = 0;
#pragma unroll
    for (int k = 0; k < kRemote; ++k) rank += __shfl_sync(0xffffffffu, id, k) < id;
    if (lane < kRemote) out[rank] = id;
    if (lane < kLocal) out[kRemote + lane] = nb - kLocal + lane;
}

// Keys of the 4 candidates j .. j + 3 (j % 4 == 0, all < nc) from one aligned 16-byte load;
// the 4 share one word of the candidate mask.
__device__ __forceinline__ void keys4(const float *row, const uint32_t *mask, int j, uint32_t (&k)[4]) {
    const float4 v = __ldcg(reinterpret_cast<const float4 *>(row + j));
    const uint32_t mw = mask ? __ldg(mask + (j >> 5)) >> (j & 31) : 0xfu;
    k[0] = (mw & 1u) ? order_key(v.x) : 0u;
    k[1] = (mw & 2u) ? order_key(v.y) : 0u;
    k[2] = (mw & 4u) ? order_key(v.z) : 0u;
    k[3] = (mw & 8u) ? order_key(v.w) : 0u;
}

constexpr int kRegQuads = 16;   // rows of up to 32 x 4 x 16 = 2048 candidates keep their keys in registers

// Selection of one query with nb causal blocks by one warp.  Lane l holds the candidates
// 4l .. 4l + 3, 4l + 128 .., read as aligned float4.  A row of at most 2048 candidates whose
// start is 16-byte aligned is read once into registers (16 loads in flight per lane); other
// rows are read twice from L2 (maxima, then survivors), in float4 where aligned.  Threshold
// = the 12th largest of the 32 lane maxima; the survivors at or above it are ranked by
// counting; more than kWarpSurvivorCap survivors (heavily tied scores) take the exact
// fallback of 12 rounds of a warp-wide maximum.
__device__ void topk_warp_select(const float *row, int nb, const uint32_t *mask, TopkWarpShared &sm,
                                 int32_t *out) {
    const int lane = threadIdx.x & 31;
    const unsigned below = (1u << lane) - 1u;
    const int nc = nb - kLocal > 0 ? nb - kLocal : 0;
    if (nc <= kRemote && !mask) {
        if (lane < kSel) out[lane] = lane < nb ? lane : -1;
        return;
    }
    const KeySource key{nullptr, row, mask};
    const bool aligned = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
    const bool in_regs = aligned && nc <= 128 * kRegQuads;
    const int n_vec = aligned ? (nc & ~3) : 0;

    uint32_t kr[kRegQuads][4];
    uint32_t tmax = 0;
    int allowed = 0;
    if (in_regs) {
        // every load is issued before any is used: the whole quads first, then the mask words
        // (one branch: the mask pointer is the same for the warp), then the one partial quad
        float4 v[kRegQuads];
#pragma unroll
        for (int q = 0; q < kRegQuads; ++q) {
            const int j = 128 * q + 4 * lane;
            v[q] = j + 3 < nc ? __ldcg(reinterpret_cast<const float4 *>(row + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        uint32_t mw[kRegQuads];
        if (mask) {
#pragma unroll
            for (int q = 0; q < kRegQuads; ++q) {
                const int j = 128 * q + 4 * lane;
                mw[q] = j < nc ? __ldg(mask + (j >> 5)) >> (j & 31) : 0u;
            }
        } else {
#pragma unroll
            for (int q = 0; q < kRegQuads; ++q) mw[q] = 0xfu;
        }
#pragma unroll
        for (int q = 0; q < kRegQuads; ++q) {
            const int j = 128 * q + 4 * lane;
            const float f[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
            if (!mask && 128 * q + 127 < nc) {
                // every lane's quad is whole and unmasked (the same for the warp): keys only
#pragma unroll
                for (int e = 0; e < 4; ++e) kr[q][e] = order_key(f[e]);
                continue;
            }
            if (j < nc && j + 3 >= nc) {   // the quad that holds the row's end: scalar reads
                v[q].x = __ldcg(row + j);
                v[q].y = j + 1 < nc ? __ldcg(row + j + 1) : 0.f;
                v[q].z = j + 2 < nc ? __ldcg(row + j + 2) : 0.f;
            }
            const float g[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) kr[q][e] = (j + e < nc && ((mw[q] >> e) & 1u)) ? order_key(g[e]) : 0u;
        }
#pragma unroll
        for (int q = 0; q < kRegQuads; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) tmax = kr[q][e] > tmax ? kr[q][e] : tmax;
        if (mask) {   // (the count of allowed candidates matters only with a mask)
#pragma unroll
            for (int q = 0; q < kRegQuads; ++q)
#pragma unroll
                for (int e = 0; e < 4; ++e) allowed += kr[q][e] != 0u;
        }
    } else {
#pragma unroll 4
        for (int j = 4 * lane; j < n_vec; j += 128) {
            uint32_t k[4];
            keys4(row, mask, j, k);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                tmax = k[e] > tmax ? k[e] : tmax;
                allowed += k[e] != 0u;
            }
        }
        for (int j = n_vec + lane; j < nc; j += 32) {
            const uint32_t k = key(j);
            tmax = k > tmax ? k : tmax;
            allowed += k != 0u;
        }
    }
    if (mask && __reduce_add_sync(0xffffffffu, allowed) <= kRemote) {
        // no more allowed candidates than remote slots: take them all, in id order
        int pos = 0;
        for (int base = 0; base < nc; base += 32) {
            const int j = base + lane;
            const bool take = j < nc && key(j) != 0u;
            const unsigned m = __ballot_sync(0xffffffffu, take);
            if (take) out[pos + __popc(m & below)] = j;
            pos += __popc(m);
        }
        const int n_loc = nb < kLocal ? nb : kLocal;
        if (lane < n_loc) out[pos + lane] = nb - n_loc + lane;
        if (lane >= pos + n_loc && lane < kSel) out[lane] = -1;
        return;
    }

    // the 12th largest lane maximum, with multiplicity
    int gt = 0, ge = 0;
#pragma unroll
    for (int w = 0; w < 32; ++w) {
        const uint32_t o = __shfl_sync(0xffffffffu, tmax, w);
        gt += o > tmax;
        ge += o >= tmax;
    }
    const unsigned who = __ballot_sync(0xffffffffu, gt <= kRemote - 1 && kRemote - 1 < ge);
    const uint32_t thr = __shfl_sync(0xffffffffu, tmax, __ffs(who) - 1);

    int n = 0;   // warp-uniform survivor count
    auto append = [&](bool keep, uint32_t k, int j) {
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        const int slot = n + __popc(m & below);
        if (keep && slot < kWarpSurvivorCap) sm.surv[slot] = composite(k, j);
        n += __popc(m);
    };
    if (in_regs) {
        // each lane counts its survivors, takes its place in the list from a prefix sum over the
        // lanes and writes them there: no warp-wide step per candidate (the list's order does not
        // matter, the ranking below orders it)
        int mine = 0;
#pragma unroll
        for (int q = 0; q < kRegQuads; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) mine += (128 * q + 4 * lane + e < nc && kr[q][e] >= thr) ? 1 : 0;
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int slot = incl - mine;
        n = __shfl_sync(0xffffffffu, incl, 31);
#pragma unroll
        for (int q = 0; q < kRegQuads; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = 128 * q + 4 * lane + e;
                if (j < nc && kr[q][e] >= thr) {
                    if (slot < kWarpSurvivorCap) sm.surv[slot] = composite(kr[q][e], j);
                    ++slot;
                }
            }
    } else {
        // every lane runs the same number of iterations (the ballots need the whole warp)
#pragma unroll 4
        for (int j0 = 0; j0 < n_vec; j0 += 128) {
            const int j = j0 + 4 * lane;
            uint32_t k[4] = {0u, 0u, 0u, 0u};
            if (j < n_vec) keys4(row, mask, j, k);
#pragma unroll
            for (int e = 0; e < 4; ++e) append(j < n_vec && k[e] >= thr, k[e], j + e);
        }
        for (int j0 = n_vec; j0 < nc; j0 += 32) {
            const int j = j0 + lane;
            const uint32_t k = j < nc ? key(j) : 0u;
            append(j < nc && k >= thr, k, j);
        }
    }
    __syncwarp();
    if (n <= kWarpSurvivorCap) {
        for (int a = lane; a < n; a += 32) {
            const uint64_t c = sm.surv[a];
            int rank = 0;
            for (int b = 0; b < n; ++b) rank += sm.surv[b] > c;
            if (rank < kRemote) sm.top[rank] = c;
        }
    } else {
        uint64_t cap = ~0ull;
        uint64_t mine = best_below(key, lane, 32, nc, cap);
#pragma unroll 1
        for (int k = 0; k < kRemote; ++k) {
            const uint64_t w = warp_max_u64(mine);
            if (lane == 0) sm.top[k] = w;
            if (mine == w && w != 0) {
                cap = mine;
                mine = best_below(key, lane, 32, nc, cap);
            }
        }
    }
    __syncwarp();
    topk_warp_emit(sm.top, nb, lane, out);
}

}  // namespace uocr
