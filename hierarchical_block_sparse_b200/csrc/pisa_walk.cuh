// pisa_walk.cuh -- one warp walks the key pyramid for one query (close reading
// §04 4.2-4.4, Eq.(5)-(7), (11); §5.3 forced/causal rules).
//
// Lane c of the warp owns candidate c (at most g*K = 2K <= 32 candidates per
// level, Eq.(6)). Dot products are batched 32 at a time: every lane holds
// D/32 elements of each of the G query rows, and slot s = row * G + head of a
// reduce-scatter collects one (row, head) dot per lane. Scores are kept in
// log2 units (q is pre-scaled by log2(e)/sqrt(d)), which leaves every ranking
// unchanged.
#pragma once

#include "pisa_device.cuh"

namespace pisa {

template <typename T, int D, int G>
struct Walk {
    static constexpr int VD = D / 32;  // elements of a row per lane
    static constexpr int RB = 32 / G;  // rows finished per reduce-scatter

    // q rows of the group, pre-scaled: q[h][e] for e in [lane*VD, lane*VD+VD)
    float q[G][VD];

    __device__ __forceinline__ void load_q(const T* const* qrow, float scale, int lane) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            Ld<T, VD>::run(qrow[h] + lane * VD, q[h]);
#pragma unroll
            for (int e = 0; e < VD; ++e) q[h][e] *= scale;
        }
    }

    template <typename R>
    __device__ __forceinline__ void dots_into(float (&v)[32], int r, const R* row, bool ok,
                                              int lane) const {
        float x[VD];
        if (ok) {
            Ld<R, VD>::run(row + lane * VD, x);
        } else {
#pragma unroll
            for (int e = 0; e < VD; ++e) x[e] = 0.f;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < VD; ++e) s = fmaf(q[h][e], x[e], s);
            v[r * G + h] = s;
        }
    }

    // Eq.(7) at level l >= 2 for the candidates flagged in `need` (one per
    // lane): LSE over the (up to 2) existing child summaries at level l-1,
    // summed over the G heads (Eq.11). `child_lvl` points at level l-1 of this
    // head's pyramid; children with first token >= n_keys do not exist.
    __device__ __forceinline__ float score_internal(int cand, unsigned need, const float* child_lvl,
                                                    int64_t span_child, int64_t n_keys,
                                                    int lane, int variant = 0) const {
        float my = -INFINITY;
        constexpr int CPB = RB / 2;  // candidates finished per batch
        for (int bi = 0; bi < 32 / CPB; ++bi) {
            if (((need >> (bi * CPB)) & ((CPB == 32 ? 0xffffffffu : ((1u << CPB) - 1u)))) == 0u) continue;
            float v[32];
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const int rho = bi * RB + r;
                const int c = rho >> 1;
                const int child = 2 * __shfl_sync(kFull, cand, c) + (rho & 1);
                const bool ok = ((need >> c) & 1u) && (int64_t)child * span_child < n_keys;
                dots_into(v, r, child_lvl + (int64_t)child * D, ok, lane);
            }
            float z = reduce_scatter32(v, lane);
            {
                const int rho = bi * RB + lane / G;
                const int c = rho >> 1;
                const int child = 2 * __shfl_sync(kFull, cand, c) + (rho & 1);
                const bool ok = ((need >> c) & 1u) && (int64_t)child * span_child < n_keys;
                if (!ok) z = -INFINITY;
            }
            // score over the two children of the same head: partner lane is lane ^ G
            const float z2 = __shfl_xor_sync(kFull, z, G);
            float s = pair_score(z, z2, variant);
#pragma unroll
            for (int o = 1; o < G; o <<= 1) s += __shfl_xor_sync(kFull, s, o);
            // candidate c of this batch sits in lanes [(c - bi*CPB) * 2G, +2G)
            const int src = ((lane - bi * CPB) * 2 * G) & 31;
            const float got = __shfl_sync(kFull, s, src);
            if (lane >= bi * CPB && lane < (bi + 1) * CPB) my = got;
        }
        return my;
    }

    // Eq.(7) at the leaves: exact LSE over each flagged candidate's raw keys
    // [leaf*C, min(leaf*C + C, n_keys)), summed over the G heads.
    __device__ __forceinline__ float score_leaves(int cand, unsigned need, const T* Kh, int C,
                                                  int64_t n_keys, int lane, int variant = 0) const {
        float my = -INFINITY;
        while (need) {
            const int c = __ffs(need) - 1;
            need &= need - 1;
            const int leaf = __shfl_sync(kFull, cand, c);
            const int64_t lo = (int64_t)leaf * C, hi = min((int64_t)leaf * C + C, n_keys);
            const float s = variant == 0 ? leaf_lse(Kh, lo, hi, lane) : leaf_moments_score(Kh, lo, hi, lane, variant);
            if (lane == c) my = s;
        }
        return my;
    }

    // PISA-1 / PISA-2 score over the raw keys [lo, hi), summed over the G heads
    __device__ __forceinline__ float leaf_moments_score(const T* Kh, int64_t lo, int64_t hi, int lane,
                                                        int variant) const {
        Moments mo;  // head lane % G
        for (int64_t r0 = lo; r0 < hi; r0 += RB) {
            float v[32];
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const int64_t row = r0 + r;
                dots_into(v, r, Kh + row * D, row < hi, lane);
            }
            const float z = reduce_scatter32(v, lane);
            if (r0 + lane / G < hi) mo.add(z);
        }
#pragma unroll
        for (int o = G; o < 32; o <<= 1) {
            const float nb = __shfl_xor_sync(kFull, mo.n, o), mb = __shfl_xor_sync(kFull, mo.mean, o),
                        m2b = __shfl_xor_sync(kFull, mo.m2, o);
            mo.merge(nb, mb, m2b);
        }
        float r = mo.score(variant);
#pragma unroll
        for (int o = 1; o < G; o <<= 1) r += __shfl_xor_sync(kFull, r, o);
        return r;
    }

    // sum over heads of log2-sum-exp2 of the scaled dots with rows [lo, hi)
    __device__ __forceinline__ float leaf_lse(const T* Kh, int64_t lo, int64_t hi, int lane) const {
        float m = -INFINITY, s = 0.f;  // running state of head (lane % G)
        for (int64_t r0 = lo; r0 < hi; r0 += RB) {
            float v[32];
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const int64_t row = r0 + r;
                dots_into(v, r, Kh + row * D, row < hi, lane);
            }
            const float z = reduce_scatter32(v, lane);
            if (r0 + lane / G < hi) {
                const float mn = fmaxf(m, z);
                s = s * exp2f(m - mn) + exp2f(z - mn);
                m = mn;
            }
        }
#pragma unroll
        for (int o = G; o < 32; o <<= 1) {
            const float m2 = __shfl_xor_sync(kFull, m, o);
            const float s2 = __shfl_xor_sync(kFull, s, o);
            const float mn = fmaxf(m, m2);
            s = (mn == -INFINITY) ? 0.f : s * exp2f(m - mn) + s2 * exp2f(m2 - mn);
            m = mn;
        }
        float r = m + log2f(s);
#pragma unroll
        for (int o = 1; o < G; o <<= 1) r += __shfl_xor_sync(kFull, r, o);
        return r;
    }
};

// Per-level candidate bookkeeping (close reading §04 4.2 and §5.3).
struct LevelState {
    bool valid;      // lane holds an existing, causally eligible candidate
    bool forced;     // candidate is on a forced path (kept, never ranked)
    unsigned vmask;  // lanes with valid candidates
    int n;           // number of valid candidates
};

__device__ __forceinline__ LevelState level_state(int cand, int l, int C, int64_t n_keys, int64_t t,
                                                  int causal, const Forced& F) {
    LevelState s;
    const int64_t first = (int64_t)cand * ((int64_t)C << (l - 1));
    s.valid = cand >= 0 && first < n_keys && (!causal || first <= t);
    s.forced = s.valid && F.has(cand, l);
    s.vmask = __ballot_sync(kFull, s.valid);
    s.n = __popc(s.vmask);
    return s;
}

// Keep the candidates of this level: all of them when there are at most K,
// else forced first then best score (ties: lower index). Afterwards lanes
// 0..kept-1 hold the kept node ids (ordered by rank); returns kept.
__device__ __forceinline__ int keep_topk(int& id, float score, const LevelState& s, int K, int lane) {
    float key;
    if (s.n <= K) key = s.valid ? 0.f : -INFINITY;
    else key = !s.valid ? -INFINITY : (s.forced ? INFINITY : score);
    int ix = s.valid ? id : 0x7fffffff;
    warp_sort_desc(key, ix, lane);
    id = ix;
    return s.n < K ? s.n : K;
}

// Keep-set of a scored level without a sort: every lane counts the lanes that
// rank before it (higher key, then lower node index) with 31 independent
// shuffles, so the keep decision has no long dependent chain. Keys: +inf
// forced, the score otherwise. The walk keeps its valid candidates in
// ascending node order across the lanes (the root starts in lane 0, and both
// the gather by rank and this keep preserve lane order, so the children
// 2p, 2p + 1 of ascending parents ascend too): "lower index" is "lower lane",
// and only the key crosses lanes. Invalid lanes send NaN, which ranks before
// no one. Lanes 0..kept-1 of the result hold the kept ids in lane order;
// returns kept (and, if asked, the mask of kept candidate lanes).
__device__ __forceinline__ int keep_topk_lane(int& id, float key, bool valid, int K, int lane,
                                              unsigned* kmask_out = nullptr) {
    const float kv = valid ? key : __int_as_float(0x7fc00000);
    int before = 0;
#pragma unroll
    for (int o = 1; o < 32; ++o) {
        const float ok = __shfl_xor_sync(kFull, kv, o);
        const int hb = o >= 16 ? 4 : o >= 8 ? 3 : o >= 4 ? 2 : o >= 2 ? 1 : 0;
        const bool lower = (lane >> hb) & 1;  // lane ^ o < lane
        before += (ok > key || (ok == key && lower)) ? 1 : 0;
    }
    const unsigned kmask = __ballot_sync(kFull, valid && before < K);
    if (kmask_out) *kmask_out = kmask;  // bit c: candidate lane c is kept
    const int kept = __popc(kmask);
    int src = 0;
#pragma unroll
    for (int step = 16; step >= 1; step >>= 1) {
        const int probe = src + step;
        if (probe <= 31 && __popc(kmask & ((1u << probe) - 1u)) <= lane) src = probe;
    }
    id = __shfl_sync(kFull, id, src);
    return kept;
}

// Lanes 0..n-1 of the result hold the valid candidates in lane order
// (a gather by rank: the lane holding the r-th set bit of vmask).
__device__ __forceinline__ int compact_by_rank(int cand, unsigned vmask, int rank) {
    int src = 0;
#pragma unroll
    for (int step = 16; step >= 1; step >>= 1) {
        const int probe = src + step;
        if (__popc(vmask & ((1u << probe) - 1u)) <= rank && probe <= 31) src = probe;
    }
    return __shfl_sync(kFull, cand, src);
}

}  // namespace pisa
