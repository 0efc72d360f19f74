// decode.cu -- decode path (close reading §5.1 last paragraph; §5.3 "decode
// cache").
//
// append_kernel: one warp per (b, kv-head) writes the new key/value row at
// pos[b], recomputes that leaf's mean from its cached rows and the new key,
// then each ancestor as the mean of its existing children: O(C + L) rows.
//
// decode_kernel: the single-stage fused step, one CTA (8 warps) per
// (b, kv-head). Warp 0 carries the walk's bookkeeping; at every scored level
// all warps compute the child dot products together (one round of gathers
// per level), all warps then split the leaf scoring (exact LSE over raw keys)
// and, after warp 0's final Top-K, the attention over the kept blocks;
// partial softmax states are merged through shared memory.
#include "pisa_internal.h"
#include "pisa_attn.cuh"

namespace pisa {

template <typename T, int D>
__global__ void __launch_bounds__(128) append_kernel(T* __restrict__ Kc, T* __restrict__ Vc,
                                                     float* __restrict__ pyr, const T* __restrict__ k_new,
                                                     const T* __restrict__ v_new, const int32_t* __restrict__ pos,
                                                     DecodeParams p) {
    constexpr int VD = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t unit = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (unit >= (int64_t)p.B * p.Hkv) return;
    const int64_t b = unit / p.Hkv;
    const int64_t n = pos[b];
    if (n < 0 || n >= p.N) return;
    T* Kh = Kc + unit * p.N * D;
    T* Vh = Vc + unit * p.N * D;
    float* P = pyr + unit * p.geom.rows * D;

    // new rows: copy the caller's elements verbatim
    float kn[VD], vn[VD];
    Ld<T, VD>::run(k_new + unit * D + lane * VD, kn);
    Ld<T, VD>::run(v_new + unit * D + lane * VD, vn);
    store_vec<T, VD>(Kh + n * D + lane * VD, kn);
    store_vec<T, VD>(Vh + n * D + lane * VD, vn);

    // leaf mean over [leaf*C, n] (rows before n from the cache)
    const int64_t leaf = n / p.C, lo = leaf * p.C;
    float acc[VD];
#pragma unroll
    for (int e = 0; e < VD; ++e) acc[e] = kn[e];
    int64_t r = lo;
    for (; r + 3 < n; r += 4) {
        float x0[VD], x1[VD], x2[VD], x3[VD];
        Ld<T, VD>::run(Kh + r * D + lane * VD, x0);
        Ld<T, VD>::run(Kh + (r + 1) * D + lane * VD, x1);
        Ld<T, VD>::run(Kh + (r + 2) * D + lane * VD, x2);
        Ld<T, VD>::run(Kh + (r + 3) * D + lane * VD, x3);
#pragma unroll
        for (int e = 0; e < VD; ++e) acc[e] += (x0[e] + x1[e]) + (x2[e] + x3[e]);
    }
    for (; r < n; ++r) {
        float x[VD];
        Ld<T, VD>::run(Kh + r * D + lane * VD, x);
#pragma unroll
        for (int e = 0; e < VD; ++e) acc[e] += x[e];
    }
    const float inv = 1.f / (float)(n - lo + 1);
#pragma unroll
    for (int e = 0; e < VD; ++e) acc[e] *= inv;
    store_vec<float, VD>(P + (p.geom.off[1] + leaf) * D + lane * VD, acc);

    // ancestors: mean of the existing children at length n + 1
    const int64_t len = n + 1;
    int64_t node = leaf;
    for (int l = 1; l < p.geom.L; ++l) {
        const int64_t sib = node ^ 1;
        if (sib * ((int64_t)p.C << (l - 1)) < len) {
            float s[VD];
            Ld<float, VD>::run(P + (p.geom.off[l] + sib) * D + lane * VD, s);
#pragma unroll
            for (int e = 0; e < VD; ++e) acc[e] = (acc[e] + s[e]) * 0.5f;
        }
        node >>= 1;
        store_vec<float, VD>(P + (p.geom.off[l + 1] + node) * D + lane * VD, acc);
    }
}

// CTAs per SM the decode kernel is sized for: with G <= 2 four CTAs of 8
// warps fit (64 registers a thread), so a step of up to 4 * 148 (b, kv-head)
// units runs in one wave.
template <int G>
constexpr int decode_min_blocks() { return G <= 2 ? 4 : (G <= 4 ? 2 : 1); }

template <typename T, int D, int G>
__global__ void __launch_bounds__(256, decode_min_blocks<G>()) decode_kernel(
    const T* __restrict__ q_new, const T* __restrict__ Kc, const T* __restrict__ Vc, const float* __restrict__ pyr,
    const int32_t* __restrict__ pos, int32_t* __restrict__ idx, T* __restrict__ out, DecodeParams p) {
    constexpr int VD = D / 32;
    constexpr int NW = 8;
    constexpr int RB = 32 / G;                  // rows per reduce-scatter batch
    constexpr int ROWS_W = 64 / NW;             // child rows per warp at a scored level
    constexpr int NRB = RB < ROWS_W ? RB : ROWS_W;
    extern __shared__ __align__(16) float dsm[];  // [NW][G][D] partial outputs
    __shared__ int s_cand[32];
    __shared__ float s_dot[64][G];
    __shared__ float s_score[32];
    __shared__ int s_sel[32];
    __shared__ unsigned s_need;
    __shared__ int s_level;
    __shared__ float s_m[NW][G], s_l[NW][G];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t unit = blockIdx.x;  // b * Hkv + kvh
    const int64_t b = unit / p.Hkv;
    const int kvh = (int)(unit - b * p.Hkv);
    const int64_t t = pos[b];
    if (t < 0 || t >= p.N) {
        if (threadIdx.x < p.K) idx[unit * p.K + threadIdx.x] = -1;
        for (int i = threadIdx.x; i < G * D; i += blockDim.x)
            out[((b * p.Hq + (int64_t)kvh * G) * D) + i] = (T)0.f;
        return;
    }
    const int64_t n_keys = t + 1;
    const T* Kh = Kc + unit * p.N * D;
    const T* Vh = Vc + unit * p.N * D;
    const float* P = pyr + unit * p.geom.rows * D;
    const Forced F(t, p.C, 1, p.forced_mask);

    Walk<T, D, G> w;
    {
        const T* qrow[G];
#pragma unroll
        for (int h = 0; h < G; ++h) qrow[h] = q_new + (b * p.Hq + (int64_t)kvh * G + h) * D;
        w.load_q(qrow, p.qscale, lane);
    }

    // Internal levels. Warp 0 carries the walk (lane c = candidate c, valid
    // candidates in ascending node order) and passes alone through the levels
    // that need no dot products; at a scored level all warps compute the
    // <= 64 child dots (8 rows each, loads in flight together) into s_dot.
    int cand = lane == 0 ? 0 : -1;  // warp 0's walk state
    int l = p.geom.L;
    for (;;) {
        if (warp == 0) {
            unsigned need = 0;
            for (; l >= 2; --l) {
                const LevelState s = level_state(cand, l, p.C, n_keys, t, 1, F);
                if (s.n <= p.K) {
                    const int parent = compact_by_rank(cand, s.vmask, lane >> 1);
                    cand = lane < 2 * s.n ? 2 * parent + (lane & 1) : -1;
                    continue;
                }
                const unsigned fmask = __ballot_sync(kFull, s.forced);
                if (__popc(fmask) >= p.K) {  // the forced nodes fill the budget
                    int id = cand;
                    const int kept = keep_topk_lane(id, s.forced ? INFINITY : -INFINITY, s.valid, p.K, lane);
                    const int parent = __shfl_sync(kFull, id, lane >> 1);
                    cand = lane < 2 * kept ? 2 * parent + (lane & 1) : -1;
                    continue;
                }
                need = s.vmask & ~fmask;
                break;
            }
            s_cand[lane] = cand;
            if (lane == 0) {
                s_level = l;
                s_need = need;
            }
        }
        __syncthreads();
        const int lv = s_level;
        if (lv < 2) break;
        {
            const unsigned need = s_need;
            const int64_t span_child = (int64_t)p.C << (lv - 2);
            const float* child_lvl = P + p.geom.off[lv - 1] * D;
#pragma unroll
            for (int r0 = warp * ROWS_W; r0 < warp * ROWS_W + ROWS_W; r0 += NRB) {
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.f;
#pragma unroll
                for (int r = 0; r < NRB; ++r) {
                    const int rho = r0 + r, c = rho >> 1;
                    const int64_t child = 2 * (int64_t)s_cand[c] + (rho & 1);
                    const bool ok = ((need >> c) & 1u) && child * span_child < n_keys;
                    w.dots_into(v, r, child_lvl + (ok ? child : 0) * D, ok, lane);
                }
                const float z = reduce_scatter32(v, lane);  // lane = r * G + h
                if (lane < NRB * G) s_dot[r0 + lane / G][lane % G] = z;
            }
        }
        __syncthreads();
        if (warp == 0) {  // scores (Eq.7, summed over the group: Eq.11) and the keep
            const LevelState s = level_state(cand, l, p.C, n_keys, t, 1, F);
            const bool mine = (s_need >> lane) & 1u;
            float score = -INFINITY;
            if (mine) {
                const bool has1 = (2 * (int64_t)cand + 1) * ((int64_t)p.C << (l - 2)) < n_keys;
                score = 0.f;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float z0 = s_dot[2 * lane][h], z1 = has1 ? s_dot[2 * lane + 1][h] : -INFINITY;
                    const float m = fmaxf(z0, z1);
                    score += m + log2f(exp2f(z0 - m) + exp2f(z1 - m));
                }
            }
            int id = cand;
            const int kept = keep_topk_lane(id, s.forced ? INFINITY : score, s.valid, p.K, lane);
            const int parent = __shfl_sync(kFull, id, lane >> 1);
            cand = lane < 2 * kept ? 2 * parent + (lane & 1) : -1;
            --l;
        }
    }

    // leaves: warp 0 flags the candidates to score; exact LSE over raw keys
    if (warp == 0) {
        const LevelState s = level_state(cand, 1, p.C, n_keys, t, 1, F);
        const unsigned fmask = __ballot_sync(kFull, s.forced);
        s_score[lane] = -INFINITY;
        if (lane == 0) s_need = (s.n > p.K && __popc(fmask) < p.K) ? (s.vmask & ~fmask) : 0u;
    }
    __syncthreads();
    {
        const unsigned need = s_need;
        for (int c = warp; c < 32; c += NW) {
            if (!((need >> c) & 1u)) continue;
            const int leaf = s_cand[c];
            const float sc = w.leaf_lse(Kh, (int64_t)leaf * p.C, min((int64_t)leaf * p.C + p.C, n_keys), lane);
            if (lane == 0) s_score[c] = sc;
        }
    }
    __syncthreads();

    if (warp == 0) {  // final Top-K: kept leaves come out in ascending order
        const LevelState s = level_state(cand, 1, p.C, n_keys, t, 1, F);
        int id = cand, kept;
        if (s.n <= p.K) {
            id = compact_by_rank(cand, s.vmask, lane);
            kept = s.n;
        } else {
            kept = keep_topk_lane(id, s.forced ? INFINITY : s_score[lane], s.valid, p.K, lane);
        }
        const int out_id = lane < kept ? id : -1;
        if (lane < p.K) idx[unit * p.K + lane] = out_id;
        s_sel[lane] = lane < p.K ? out_id : -1;
    }
    __syncthreads();

    // attention over the kept blocks, blocks spread over the warps
    AttnAcc<T, D, G> acc;
    acc.init();
    for (int k = warp; k < p.K; k += NW) {
        const int blk = s_sel[k];
        if (blk < 0) continue;
        const int64_t lo = (int64_t)blk * p.C;
        const int64_t hi = min(lo + p.C, n_keys);
        if (lo < hi) acc.block(w, Kh, Vh, lo, hi, lane);
    }
    float lsum = acc.lsum;
#pragma unroll
    for (int o = G; o < 32; o <<= 1) lsum += __shfl_xor_sync(kFull, lsum, o);
    if (lane < G) {
        s_m[warp][lane] = acc.m;
        s_l[warp][lane] = lsum;
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < VD; ++e) dsm[(warp * G + h) * D + lane * VD + e] = acc.o[h][e];
    __syncthreads();

    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int h = i / D;
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, s_m[ww][h]);
        float den = 0.f, num = 0.f;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) {
            const float sc = s_m[ww][h] == -INFINITY ? 0.f : exp2f(s_m[ww][h] - M);
            den += s_l[ww][h] * sc;
            num += dsm[(ww * G + h) * D + (i - h * D)] * sc;
        }
        const float val = den > 0.f ? num / den : 0.f;
        out[((b * p.Hq + (int64_t)kvh * G) * D) + i] = (T)val;
    }
}

template <typename T, int D>
static cudaError_t launch_append_t(void* Kc, void* Vc, float* pyr, const void* k_new, const void* v_new,
                                   const int32_t* pos, const DecodeParams& p, cudaStream_t st) {
    const int64_t units = (int64_t)p.B * p.Hkv;
    append_kernel<T, D><<<(unsigned)((units + 3) / 4), 128, 0, st>>>((T*)Kc, (T*)Vc, pyr, (const T*)k_new,
                                                                      (const T*)v_new, pos, p);
    return cudaGetLastError();
}

cudaError_t launch_append(int dtype, int d, void* Kc, void* Vc, float* pyr, const void* k_new, const void* v_new,
                          const int32_t* pos, const DecodeParams& p, cudaStream_t st) {
    if (dtype == 1) {
        if (d == 128) return launch_append_t<__nv_bfloat16, 128>(Kc, Vc, pyr, k_new, v_new, pos, p, st);
        if (d == 64) return launch_append_t<__nv_bfloat16, 64>(Kc, Vc, pyr, k_new, v_new, pos, p, st);
    } else {
        if (d == 128) return launch_append_t<float, 128>(Kc, Vc, pyr, k_new, v_new, pos, p, st);
        if (d == 64) return launch_append_t<float, 64>(Kc, Vc, pyr, k_new, v_new, pos, p, st);
    }
    return cudaErrorInvalidValue;
}

template <typename T, int D, int G>
static cudaError_t launch_decode_t(const void* q, const void* Kc, const void* Vc, const float* pyr,
                                   const int32_t* pos, int32_t* idx, void* o, const DecodeParams& p,
                                   cudaStream_t st) {
    const size_t smem = sizeof(float) * 8 * G * D;
    auto kern = decode_kernel<T, D, G>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<(unsigned)((int64_t)p.B * p.Hkv), 256, smem, st>>>((const T*)q, (const T*)Kc, (const T*)Vc, pyr, pos,
                                                               idx, (T*)o, p);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_decode_d(const void* q, const void* Kc, const void* Vc, const float* pyr,
                                   const int32_t* pos, int32_t* idx, void* o, const DecodeParams& p,
                                   cudaStream_t st) {
    switch (p.Hq / p.Hkv) {
        case 1: return launch_decode_t<T, D, 1>(q, Kc, Vc, pyr, pos, idx, o, p, st);
        case 2: return launch_decode_t<T, D, 2>(q, Kc, Vc, pyr, pos, idx, o, p, st);
        case 4: return launch_decode_t<T, D, 4>(q, Kc, Vc, pyr, pos, idx, o, p, st);
        case 8: return launch_decode_t<T, D, 8>(q, Kc, Vc, pyr, pos, idx, o, p, st);
        case 16: return launch_decode_t<T, D, 16>(q, Kc, Vc, pyr, pos, idx, o, p, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(int dtype, int d, const void* q_new, const void* Kc, const void* Vc, const float* pyr,
                          const int32_t* pos, int32_t* idx, void* o, const DecodeParams& p, cudaStream_t st) {
    if (dtype == 1) {
        if (d == 128) return launch_decode_d<__nv_bfloat16, 128>(q_new, Kc, Vc, pyr, pos, idx, o, p, st);
        if (d == 64) return launch_decode_d<__nv_bfloat16, 64>(q_new, Kc, Vc, pyr, pos, idx, o, p, st);
    } else {
        if (d == 128) return launch_decode_d<float, 128>(q_new, Kc, Vc, pyr, pos, idx, o, p, st);
        if (d == 64) return launch_decode_d<float, 64>(q_new, Kc, Vc, pyr, pos, idx, o, p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pisa
