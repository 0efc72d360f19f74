// pisa_attn.cuh -- warp-level online-softmax accumulator for attention over
// selected blocks (close reading §02, Eq.(2)).
//
// Keys are visited 32/G rows at a time: a reduce-scatter gives lane
// l = row*G + head the scaled logit of that (row, head); a running max per
// head rescales the fp32 output accumulator each lane keeps for its D/32
// output columns of every head. Logits never leave registers.
#pragma once

#include "pisa_walk.cuh"

namespace pisa {

template <typename T, int D, int G>
struct AttnAcc {
    static constexpr int VD = D / 32;
    static constexpr int RB = 32 / G;
    float o[G][VD];
    float m;     // running max (log2 units) of head lane % G
    float lsum;  // this lane's share of the softmax denominator of head lane % G

    __device__ __forceinline__ void init() {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < VD; ++e) o[h][e] = 0.f;
        m = -INFINITY;
        lsum = 0.f;
    }

    // rows [lo, hi) of one block; all of them visible to the query
    __device__ __forceinline__ void block(const Walk<T, D, G>& w, const T* Kh, const T* Vh, int64_t lo,
                                          int64_t hi, int lane) {
        for (int64_t r0 = lo; r0 < hi; r0 += RB) {
            float v[32];
#pragma unroll
            for (int r = 0; r < RB; ++r) w.dots_into(v, r, Kh + (r0 + r) * D, r0 + r < hi, lane);
            float z = reduce_scatter32(v, lane);
            if (r0 + lane / G >= hi) z = -INFINITY;
            float cm = z;
#pragma unroll
            for (int off = G; off < 32; off <<= 1) cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, off));
            const float mn = fmaxf(m, cm);  // finite: row r0 is visible
            const float alpha = exp2f(m - mn);
            const float pz = exp2f(z - mn);
            lsum = lsum * alpha + pz;
            m = mn;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float ah = __shfl_sync(kFull, alpha, h);
#pragma unroll
                for (int e = 0; e < VD; ++e) o[h][e] *= ah;
            }
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                if (r0 + r < hi) {
                    float x[VD];
                    Ld<T, VD>::run(Vh + (r0 + r) * D + lane * VD, x);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float ph = __shfl_sync(kFull, pz, r * G + h);
#pragma unroll
                        for (int e = 0; e < VD; ++e) o[h][e] = fmaf(ph, x[e], o[h][e]);
                    }
                }
            }
        }
    }

    // normalise; returns per-head denominators in lanes 0..G-1 (lane h -> head h)
    __device__ __forceinline__ void finish(int lane) {
        float l = lsum;
#pragma unroll
        for (int off = G; off < 32; off <<= 1) l += __shfl_xor_sync(kFull, l, off);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float lh = __shfl_sync(kFull, l, h);
            const float inv = lh > 0.f ? 1.f / lh : 0.f;
#pragma unroll
            for (int e = 0; e < VD; ++e) o[h][e] *= inv;
        }
    }
};

}  // namespace pisa
