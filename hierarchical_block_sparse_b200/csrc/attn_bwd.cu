// attn_bwd.cu -- backward of the attention over fixed selected leaf blocks
// (close reading §02 Eq.(2); §5.3: with the selection fixed, the gradient
// flows only through the selected attention entries).
//
// One warp per (b, kv-head, t) serves the G query heads that share the
// selection, as the forward does. Pass 1 recomputes each head's softmax
// statistics over the selected keys (log-sum-exp L and output o, with the
// forward's online accumulator) and D = dO . o. Pass 2 visits the same keys
// again, 32/G rows at a time through the reduce-scatter of the forward:
//   p = 2^(z - L)  (z: the log2-unit logit),  dp = dO . v,  ds = p (dp - D),
//   dq += ds k,  dK_j += sum_h ds q_h / sqrt(d),  dV_j += sum_h p dO_h,
// with dK and dV rows added to fp32 buffers by vector reductions (several
// queries select the same key) and dq stored once per (head, t).
#include "pisa_internal.h"
#include "pisa_attn.cuh"

namespace pisa {

template <int VD>
__device__ __forceinline__ void red_add_vec(float* p, const float* v) {
    if constexpr (VD == 4) {
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]),
                     "f"(v[3])
                     : "memory");
    } else {
        asm volatile("red.global.add.v2.f32 [%0], {%1, %2};\n" ::"l"(p), "f"(v[0]), "f"(v[1]) : "memory");
    }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(256) attn_bwd_kernel(const T* __restrict__ Q, const T* __restrict__ Kmat,
                                                       const T* __restrict__ Vmat, const int32_t* __restrict__ idx,
                                                       const T* __restrict__ dO, float* __restrict__ dQ,
                                                       float* __restrict__ dK, float* __restrict__ dV, AttnParams p) {
    constexpr int VD = D / 32;
    constexpr int RB = 32 / G;
    const int lane = threadIdx.x & 31;
    const int64_t unit = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t units = (int64_t)p.B * p.Hkv * p.N;
    if (unit >= units) return;
    const int64_t bh = unit / p.N;
    const int64_t t = unit - bh * p.N;
    const int64_t b = bh / p.Hkv;
    const int kvh = (int)(bh - b * p.Hkv);
    const float inv_sqrt_d = p.qscale / kLog2e;

    Walk<T, D, G> w;  // q rows scaled by log2(e) / sqrt(d)
    const T* qrow[G];
    float dov[G][VD];  // dO rows, this lane's columns
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const int64_t row = ((b * p.Hq + (int64_t)kvh * G + h) * p.N) + t;
        qrow[h] = Q + row * D;
        Ld<T, VD>::run(dO + row * D + lane * VD, dov[h]);
    }
    w.load_q(qrow, p.qscale, lane);
    const T* Kh = Kmat + bh * p.N * D;
    const T* Vh = Vmat + bh * p.N * D;
    float* dKh = dK + bh * p.N * D;
    float* dVh = dV + bh * p.N * D;
    const int my_blk = lane < p.K ? idx[unit * p.K + lane] : -1;
    auto block_range = [&](int k, int64_t& lo, int64_t& hi) {
        const int blk = __shfl_sync(kFull, my_blk, k);
        lo = (int64_t)blk * p.C;
        hi = min(lo + p.C, (int64_t)p.N);
        if (p.causal) hi = min(hi, t + 1);
        return blk >= 0 && lo < hi;
    };

    // pass 1: L (log2 units, head lane % G), o and D = dO . o per head
    AttnAcc<T, D, G> acc;
    acc.init();
    for (int k = 0; k < p.K; ++k) {
        int64_t lo, hi;
        if (block_range(k, lo, hi)) acc.block(w, Kh, Vh, lo, hi, lane);
    }
    float l = acc.lsum;
#pragma unroll
    for (int o = G; o < 32; o <<= 1) l += __shfl_xor_sync(kFull, l, o);
    const float Lme = acc.m + log2f(l);  // this lane's head: lane % G
    acc.finish(lane);
    float Dh[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < VD; ++e) s = fmaf(dov[h][e], acc.o[h][e], s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
        Dh[h] = s;
    }
    float Dme = Dh[0];
#pragma unroll
    for (int h = 1; h < G; ++h)
        if (lane % G == h) Dme = Dh[h];

    // pass 2
    float dq[G][VD];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < VD; ++e) dq[h][e] = 0.f;
    for (int k = 0; k < p.K; ++k) {
        int64_t lo, hi;
        if (!block_range(k, lo, hi)) continue;
        for (int64_t r0 = lo; r0 < hi; r0 += RB) {
            float vz[32], vp[32];
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const int64_t row = r0 + r;
                const bool ok = row < hi;
                w.dots_into(vz, r, Kh + row * D, ok, lane);
                float x[VD];
                if (ok) {
                    Ld<T, VD>::run(Vh + row * D + lane * VD, x);
                } else {
#pragma unroll
                    for (int e = 0; e < VD; ++e) x[e] = 0.f;
                }
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float s = 0.f;
#pragma unroll
                    for (int e = 0; e < VD; ++e) s = fmaf(dov[h][e], x[e], s);
                    vp[r * G + h] = s;
                }
            }
            const float z = reduce_scatter32(vz, lane);   // slot lane = r * G + h
            const float dp = reduce_scatter32(vp, lane);
            const bool live = r0 + lane / G < hi;
            const float pr = live ? exp2f(z - Lme) : 0.f;
            const float ds = pr * (dp - Dme);
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const int64_t row = r0 + r;
                float dsr[G], pr_r[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    dsr[h] = __shfl_sync(kFull, ds, r * G + h);
                    pr_r[h] = __shfl_sync(kFull, pr, r * G + h);
                }
                if (row < hi) {
                    float kx[VD], dk[VD], dv[VD];
                    Ld<T, VD>::run(Kh + row * D + lane * VD, kx);
#pragma unroll
                    for (int e = 0; e < VD; ++e) {
                        dk[e] = 0.f;
                        dv[e] = 0.f;
                    }
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int e = 0; e < VD; ++e) {
                            dq[h][e] = fmaf(dsr[h], kx[e], dq[h][e]);
                            dk[e] = fmaf(dsr[h], w.q[h][e], dk[e]);  // q scaled by log2(e)/sqrt(d)
                            dv[e] = fmaf(pr_r[h], dov[h][e], dv[e]);
                        }
#pragma unroll
                    for (int e = 0; e < VD; ++e) dk[e] *= 1.f / kLog2e;
                    red_add_vec<VD>(dKh + row * D + lane * VD, dk);
                    red_add_vec<VD>(dVh + row * D + lane * VD, dv);
                }
            }
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int e = 0; e < VD; ++e) dq[h][e] *= inv_sqrt_d;
        store_vec<float, VD>(dQ + (((b * p.Hq + (int64_t)kvh * G + h) * p.N) + t) * D + lane * VD, dq[h]);
    }
}

template <typename T, int D, int G>
static cudaError_t launch_bwd_t(const void* Q, const void* K, const void* V, const int32_t* idx, const void* dO,
                                float* dQ, float* dK, float* dV, const AttnParams& p, cudaStream_t st) {
    const int64_t units = (int64_t)p.B * p.Hkv * p.N;
    attn_bwd_kernel<T, D, G><<<(unsigned)((units + 7) / 8), 256, 0, st>>>(
        (const T*)Q, (const T*)K, (const T*)V, idx, (const T*)dO, dQ, dK, dV, p);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_bwd_d(const void* Q, const void* K, const void* V, const int32_t* idx, const void* dO,
                                float* dQ, float* dK, float* dV, const AttnParams& p, cudaStream_t st) {
    switch (p.Hq / p.Hkv) {
        case 1: return launch_bwd_t<T, D, 1>(Q, K, V, idx, dO, dQ, dK, dV, p, st);
        case 2: return launch_bwd_t<T, D, 2>(Q, K, V, idx, dO, dQ, dK, dV, p, st);
        case 4: return launch_bwd_t<T, D, 4>(Q, K, V, idx, dO, dQ, dK, dV, p, st);
        case 8: return launch_bwd_t<T, D, 8>(Q, K, V, idx, dO, dQ, dK, dV, p, st);
        case 16: return launch_bwd_t<T, D, 16>(Q, K, V, idx, dO, dQ, dK, dV, p, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bwd(int dtype, int d, const void* Q, const void* K, const void* V, const int32_t* idx,
                            const void* dO, float* dQ, float* dK, float* dV, const AttnParams& p, cudaStream_t st) {
    if (dtype == 1) {
        if (d == 128) return launch_bwd_d<__nv_bfloat16, 128>(Q, K, V, idx, dO, dQ, dK, dV, p, st);
        if (d == 64) return launch_bwd_d<__nv_bfloat16, 64>(Q, K, V, idx, dO, dQ, dK, dV, p, st);
    } else {
        if (d == 128) return launch_bwd_d<float, 128>(Q, K, V, idx, dO, dQ, dK, dV, p, st);
        if (d == 64) return launch_bwd_d<float, 64>(Q, K, V, idx, dO, dQ, dK, dV, p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pisa
