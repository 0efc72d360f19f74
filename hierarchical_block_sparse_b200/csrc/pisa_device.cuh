// pisa_device.cuh -- device-side building blocks shared by the PISA kernels:
// pyramid geometry, vector loads that widen bf16/fp32 to fp32, the warp
// reduce-scatter used for batched dot products, and warp bitonic sorts.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pisa {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kMaxLevels = 32;
constexpr float kLog2e = 1.4426950408889634f;

// Pyramid geometry (close reading §04 4.1, Eq.(3)): M_1 = ceil(N/C),
// M_{l+1} = ceil(M_l / 2); levels are stored leaves first, one after another.
struct Geom {
    int L;                        // number of levels (0 for an empty sequence)
    int64_t M[kMaxLevels + 1];    // nodes per level, index 1..L
    int64_t off[kMaxLevels + 1];  // first row of each level inside one head's pyramid
    int64_t rows;                 // rows per (b, kv-head) pyramid
};

// Host and device: returns L, or -1 when more than kMaxLevels levels are needed.
__host__ __device__ inline int make_geom(int64_t N, int C, Geom* g) {
    g->L = 0;
    g->rows = 0;
    if (N <= 0 || C <= 0) return 0;
    int L = 1;
    g->M[1] = (N + C - 1) / C;
    g->off[1] = 0;
    while (g->M[L] > 1) {
        if (L + 1 > kMaxLevels) return -1;
        g->M[L + 1] = (g->M[L] + 1) / 2;
        g->off[L + 1] = g->off[L] + g->M[L];
        ++L;
    }
    g->L = L;
    g->rows = g->off[L] + g->M[L];
    return L;
}

// ---- widening loads: VD consecutive elements -> fp32 ------------------------

template <typename T, int VD>
struct Ld;

template <>
struct Ld<float, 4> {
    static __device__ __forceinline__ void run(const float* p, float* o) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
};
template <>
struct Ld<float, 2> {
    static __device__ __forceinline__ void run(const float* p, float* o) {
        const float2 v = __ldg(reinterpret_cast<const float2*>(p));
        o[0] = v.x; o[1] = v.y;
    }
};
template <>
struct Ld<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void run(const __nv_bfloat16* p, float* o) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xffff0000u);
        o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xffff0000u);
    }
};
template <>
struct Ld<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void run(const __nv_bfloat16* p, float* o) {
        const unsigned v = __ldg(reinterpret_cast<const unsigned*>(p));
        o[0] = __uint_as_float(v << 16); o[1] = __uint_as_float(v & 0xffff0000u);
    }
};

// 16-byte load widened to 16/sizeof(T) floats (used by the pooling kernels).
template <typename T>
struct Ld16;
template <>
struct Ld16<float> {
    static constexpr int E = 4;
    static __device__ __forceinline__ void run(const float* p, float* o) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
};
template <>
struct Ld16<__nv_bfloat16> {
    static constexpr int E = 8;
    static __device__ __forceinline__ void run(const __nv_bfloat16* p, float* o) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

// store VD fp32 values as T
template <typename T, int VD>
__device__ __forceinline__ void store_vec(T* p, const float* v);
template <>
__device__ __forceinline__ void store_vec<float, 4>(float* p, const float* v) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void store_vec<float, 2>(float* p, const float* v) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
}
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 4>(__nv_bfloat16* p, const float* v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 u;
    u.x = *reinterpret_cast<unsigned*>(&a);
    u.y = *reinterpret_cast<unsigned*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 2>(__nv_bfloat16* p, const float* v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    *reinterpret_cast<__nv_bfloat162*>(p) = a;
}

// ---- warp reduce-scatter ------------------------------------------------------
// Every lane holds 32 partial sums v[0..31] (slot s of lane l = lane l's share
// of dot product s). After 31 exchanges lane l holds the full sum of slot l.
// Used with slot = row * G + head so one pass finishes 32/G rows for G heads.
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const bool hi = (lane & w) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float send = hi ? v[i] : v[i + w];
            const float keep = hi ? v[i + w] : v[i];
            v[i] = keep + __shfl_xor_sync(kFull, send, w);
        }
    }
    return v[0];
}

// ---- node scores from the children's logits (close reading §04 4.3) ------------
// Logits are in log2 units on the GPU (z2 = z * log2(e)). Eq.(7): LSE; PISA-1:
// the mean; PISA-2: mean + var / 2 in nats, which is mean2 + var2 * ln(2) / 2
// in log2 units (a positive multiple: every ranking is preserved).
constexpr float kHalfLn2 = 0.34657359027997264f;

// score of a node from the logits of its (up to) two children; a missing
// child is -inf. Symmetric in (a, b).
__device__ __forceinline__ float pair_score(float a, float b, int variant) {
    if (a == -INFINITY) return b;
    if (b == -INFINITY) return a;
    if (variant == 0) {
        const float m = fmaxf(a, b);
        return m + log2f(exp2f(a - m) + exp2f(b - m));
    }
    const float mean = 0.5f * (a + b);
    if (variant == 1) return mean;
    const float h = 0.5f * (a - b);
    return mean + kHalfLn2 * h * h;
}

// PTX approximate base-2 exponential and logarithm (flush-to-zero): about
// 2^-22 relative error, far below the selection's 1e-4 tie band and the bf16
// rounding of attention probabilities.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log2(2^a + 2^b) = max + log2(1 + 2^(min - max)); b may be -inf (a child
// that does not exist), a is finite
__device__ __forceinline__ float lse2_pair(float a, float b) {
    const float m = fmaxf(a, b);
    return m + lg2_approx(1.f + ex2_approx(fminf(a, b) - m));
}

// count, mean and sum of squared deviations of a set of logits (mergeable)
struct Moments {
    float n = 0.f, mean = 0.f, m2 = 0.f;
    __device__ __forceinline__ void add(float x) {
        n += 1.f;
        const float d = x - mean;
        mean += d / n;
        m2 += d * (x - mean);
    }
    __device__ __forceinline__ void merge(float nb, float meanb, float m2b) {
        if (nb == 0.f) return;
        if (n == 0.f) {
            n = nb;
            mean = meanb;
            m2 = m2b;
            return;
        }
        const float nn = n + nb, d = meanb - mean;
        mean += d * (nb / nn);
        m2 += m2b + d * d * (n * nb / nn);
        n = nn;
    }
    // PISA-1 / PISA-2 score (variant 1 / 2)
    __device__ __forceinline__ float score(int variant) const {
        if (n == 0.f) return -INFINITY;
        return variant == 1 ? mean : mean + kHalfLn2 * (m2 / n);
    }
};

// ---- warp bitonic sorts -----------------------------------------------------------

// (ka, ia) ranks before (kb, ib): larger key first, then lower index.
__device__ __forceinline__ bool ranks_before(float ka, int ia, float kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// Sort the warp's 32 (key, idx) pairs so that lane 0 holds the best-ranked.
__device__ __forceinline__ void warp_sort_desc(float& key, int& idx, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const float ok = __shfl_xor_sync(kFull, key, j);
            const int oi = __shfl_xor_sync(kFull, idx, j);
            const bool lower = (lane & j) == 0;
            const bool desc = (lane & k) == 0 || k == 32;
            const bool self_first = ranks_before(key, idx, ok, oi);
            const bool keep = (lower == desc) ? self_first : !self_first;
            if (!keep) { key = ok; idx = oi; }
        }
    }
}

// Sort 32 ints ascending across the warp (lane 0 smallest).
__device__ __forceinline__ void warp_sort_asc(int& v, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const int o = __shfl_xor_sync(kFull, v, j);
            const bool lower = (lane & j) == 0;
            const bool asc = (lane & k) == 0 || k == 32;
            const bool self_first = v < o;
            const bool keep = (lower == asc) ? self_first : !self_first;
            if (!keep) v = o;
        }
    }
}

// Forced leaves of query t (close reading §5.3): first, previous, current.
struct Forced {
    int f0, f1, f2;  // -1 when absent
    __device__ __forceinline__ Forced(int64_t t, int C, int causal, int mask) {
        const int c = (int)(t / C);
        f0 = (mask & 1) ? 0 : -1;
        f1 = ((mask & 2) && c >= 1) ? c - 1 : -1;
        f2 = ((mask & 4) || causal) ? c : -1;
    }
    // node at level l (1 = leaves) is an ancestor of (or is) a forced leaf
    __device__ __forceinline__ bool has(int node, int l) const {
        const int s = l - 1;
        return (f0 >= 0 && (f0 >> s) == node) || (f1 >= 0 && (f1 >> s) == node) ||
               (f2 >= 0 && (f2 >> s) == node);
    }
};

}  // namespace pisa
