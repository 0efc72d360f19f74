// bsa_tc.cu -- flat block selection (close reading §02, Eq.(1)) as a
// tensor-core contraction: the quadratic comparison the pyramid walk is
// measured against, built the way a dense selection is built on B200.
//
// A CTA takes 128 MMA rows (128/G consecutive positions of one (b, kv-head)
// times the G heads of the group) and streams every leaf summary the tile can
// see (causal: up to its last position) in chunks of 128 leaves:
// S = Q_tile x leaves^T on tcgen05 into TMEM, the fp32 summaries as bf16 high
// and low parts (two exact products per element, accumulated in fp32). Each
// row's Eq.(1) score of a leaf is q . k_bar / sqrt(d) summed over the group's
// heads (lanes of one position are adjacent, so the sum is a butterfly of
// shuffles). The forced leaves (first, previous, current) count against K and
// are kept; the other eligible leaves compete for the rest by score, ties to
// the lower leaf. Every row keeps a sorted top list in registers and inserts
// only what beats its current K-th key; warps 0-3 take the first 64 columns of
// each chunk and warps 4-7 the last 64, and one warp per position merges the
// two lists at the end. Output rows are sorted ascending, -1 padded, as from
// the per-query kernel (bsa.cu).
#include <cmath>

#include "pisa_internal.h"
#include "pisa_walk.cuh"
#include "tc.cuh"

namespace pisa {
namespace {

constexpr int kBtThreads = 256;
constexpr int kBtCols = 128;  // leaves per chunk
constexpr int kD = 128;
constexpr int kTop = 16;      // K <= 16
constexpr int kNone = 0x7fffffff;

struct BtSmem {
    uint8_t q[32768];              // A: 128 rows x 128 bf16, K-major
    uint8_t b[2][2][32768];        // B[buffer][hi, lo]: 128 leaf rows x 128 bf16
    float key[2][128][kTop];       // per warpgroup and position: its best keys, descending
    int32_t id[2][128][kTop];
    uint64_t mbar[2];
    uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t idesc_n(int n) {  // kind::f16, bf16 x bf16 -> fp32, both K-major, M = 128
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

template <int G>
__global__ void __launch_bounds__(kBtThreads, 1) bsa_tc_kernel(const __nv_bfloat16* __restrict__ Q,
                                                               const __nv_bfloat16* __restrict__ pyr_hi,
                                                               const __nv_bfloat16* __restrict__ pyr_lo,
                                                               int32_t* __restrict__ idx, int tiles_per_head,
                                                               int* __restrict__ err, SelectParams p) {
    constexpr int P = 128 / G;
    extern __shared__ __align__(1024) uint8_t dsm[];
    BtSmem& S = *reinterpret_cast<BtSmem*>(dsm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t nbh = (int64_t)p.B * p.Hkv;
    const int64_t bh = blockIdx.x % nbh;
    const int tile = tiles_per_head - 1 - (int)(blockIdx.x / nbh);  // latest positions (most leaves) first
    const int64_t b = bh / p.Hkv;
    const int kvh = (int)(bh - b * p.Hkv);
    const int t0 = tile * P;
    const int64_t M1 = p.geom.M[1];

    if (warp == 0) tc::tmem_alloc(&S.tmem_base, 256);
    if (tid == 0) {
        tc::mbar_init(&S.mbar[0], 1);
        tc::mbar_init(&S.mbar[1], 1);
        tc::fence_mbar_init();
    }
    const uint32_t q_smem = tc::smem_u32(S.q);
    for (int i = tid; i < 128 * 16; i += kBtThreads) {
        const int r = (i >> 7) * 8 + (i & 7), c = (i >> 3) & 15;  // 8 rows x 16-byte chunk: 128 contiguous bytes
        const int t = t0 + r / G;
        const __nv_bfloat16* src = Q + (((b * p.Hq + (int64_t)kvh * G + (r % G)) * p.N) + (t < p.N ? t : 0)) * kD + c * 8;
        if (t < p.N) tc::cp_async16(q_smem + tc::kmajor128_off(r, c), src);
        else tc::cp_async_zero16(q_smem + tc::kmajor128_off(r, c), src);
    }
    tc::cp_async_commit();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    const int t_last = min(t0 + P, p.N) - 1;
    const int64_t n_tile = p.causal ? min(M1, (int64_t)t_last / p.C + 1) : M1;  // leaves any row can see
    const int nch = (int)((n_tile + kBtCols - 1) / kBtCols);
    const __nv_bfloat16* Hh = pyr_hi + bh * p.geom.rows * kD;  // level 1 (the leaves) starts at row 0
    const __nv_bfloat16* Hl = pyr_lo + bh * p.geom.rows * kD;
    auto gather = [&](int k, int buf) {
        const int n = (int)min((int64_t)kBtCols, n_tile - (int64_t)k * kBtCols);
        const uint32_t dh = tc::smem_u32(S.b[buf][0]), dl = tc::smem_u32(S.b[buf][1]);
        for (int i = tid; i < ((n + 7) & ~7) * 32; i += kBtThreads) {
            // 8 rows of one core-matrix group per 16-byte chunk: each 8 lanes fill 128 contiguous bytes
            const int row = (i >> 8) * 8 + (i & 7), part = (i >> 3) & 31, c = part & 15;
            if (row >= n) continue;
            const int64_t leaf = (int64_t)k * kBtCols + row;
            const __nv_bfloat16* src = (part < 16 ? Hh : Hl) + leaf * kD + c * 8;
            tc::cp_async16((part < 16 ? dh : dl) + tc::kmajor128_off(row, c), src);
        }
        tc::cp_async_commit();
    };

    // this thread's row: position, head, eligibility and its share of the budget
    const int r = tid & 127, wg = tid >> 7;
    const int pos = r / G, h = r % G;
    const int t = t0 + pos;
    const bool live = t < p.N && h == 0;
    const Forced F(t < p.N ? t : 0, p.C, p.causal, p.forced_mask);
    const int64_t c_max = p.causal ? min(M1 - 1, (int64_t)(t < p.N ? t : 0) / p.C) : M1 - 1;
    int nf = 0;
    {
        const int f[3] = {F.f0, F.f1, F.f2};
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            bool dup = false;
#pragma unroll
            for (int j = 0; j < i; ++j) dup = dup || f[j] == f[i];
            if (f[i] >= 0 && f[i] <= c_max && !dup) ++nf;
        }
    }
    const int Kp = p.K - nf;  // places for the ranked leaves
    // this row's best keys so far, descending (ties: the lower leaf first), in
    // shared memory: an insertion is rare, and a list in registers would be
    // indexed by a runtime position
    float* lk = S.key[wg][pos];
    int32_t* li = S.id[wg][pos];
    if (live) {
#pragma unroll
        for (int i = 0; i < kTop; ++i) {
            lk[i] = -INFINITY;
            li[i] = kNone;
        }
    }
    float thr = Kp > 0 ? -INFINITY : INFINITY;  // the Kp-th best key so far

    uint32_t parity[2] = {0u, 0u};
    bool ok = true;
    gather(0, 0);
    for (int k = 0; k < nch; ++k) {
        const int buf = k & 1;
        tc::cp_async_wait_all();
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::tc_fence_after();
            const int n = (int)min((int64_t)kBtCols, n_tile - (int64_t)k * kBtCols);
            const uint32_t idesc = idesc_n((n + 15) & ~15);
            const uint32_t dt = tmem + (uint32_t)(buf * 128);
            const uint32_t bh_s = tc::smem_u32(S.b[buf][0]), bl_s = tc::smem_u32(S.b[buf][1]);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_bf16(dt, tc::smem_desc(q_smem + ks * 256, 128, 2048), tc::smem_desc(bh_s + ks * 256, 128, 2048),
                             idesc, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_bf16(dt, tc::smem_desc(q_smem + ks * 256, 128, 2048), tc::smem_desc(bl_s + ks * 256, 128, 2048),
                             idesc, 1u);
            tc::mma_commit(&S.mbar[buf]);
        }
        if (k + 1 < nch) gather(k + 1, buf ^ 1);  // the other buffer's MMAs completed before chunk k - 1's scan
        ok = __syncthreads_and(tc::mbar_wait(&S.mbar[buf], parity[buf], err, 17)) != 0;
        parity[buf] ^= 1u;
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
            const int c0 = wg * 64 + gi * 32;
            const int64_t leaf0 = (int64_t)k * kBtCols + c0;
            if (leaf0 >= n_tile) break;  // uniform: the tile's leaves end here
            float v[32];
            tc::tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(buf * 128 + c0), v);
            tc::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float z = v[j] * p.qscale;
#pragma unroll
                for (int o = 1; o < G; o <<= 1) z += __shfl_xor_sync(kFull, z, o);  // Eq.(11)-style sum over the group
                if (live && z > thr) {  // rare once the list is full
                    const int64_t leaf = leaf0 + j;
                    if (leaf <= c_max && !F.has((int)leaf, 1)) {
                        int i = Kp - 1;
                        while (i > 0 && z > lk[i - 1]) {
                            lk[i] = lk[i - 1];
                            li[i] = li[i - 1];
                            --i;
                        }
                        lk[i] = z;
                        li[i] = (int)leaf;
                        thr = lk[Kp - 1];
                    }
                }
            }
        }
        tc::tc_fence_before();
    }
    tc::cp_async_wait_all();
    __syncthreads();
    if (ok) {
        // one warp per position: merge the two lists, add the forced leaves, sort ascending
        for (int q = warp; q < P; q += kBtThreads / 32) {
            const int tq = t0 + q;
            if (tq >= p.N) continue;
            const Forced Fq(tq, p.C, p.causal, p.forced_mask);
            const int64_t cq = p.causal ? min(M1 - 1, (int64_t)tq / p.C) : M1 - 1;
            float key = S.key[lane >> 4][q][lane & 15];
            int id = S.id[lane >> 4][q][lane & 15];
            warp_sort_desc(key, id, lane);
            // the eligible forced leaves, each once
            int fl[3], nfq = 0;
            {
                const int f[3] = {Fq.f0, Fq.f1, Fq.f2};
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    bool dup = false;
#pragma unroll
                    for (int j = 0; j < i; ++j) dup = dup || f[j] == f[i];
                    fl[i] = -1;
                    if (f[i] >= 0 && f[i] <= cq && !dup) fl[nfq++] = f[i];
                }
            }
            const int kq = p.K - nfq;
            int v = kNone;
            if (lane < kq && key != -INFINITY) v = id;
            const int fi = lane - kq;
            if (fi >= 0 && fi < nfq) v = fi == 0 ? fl[0] : fi == 1 ? fl[1] : fl[2];
            warp_sort_asc(v, lane);
            if (lane < p.K) idx[(bh * p.N + tq) * p.K + lane] = v == kNone ? -1 : v;
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 256);
    }
}

template <int G>
cudaError_t bsa_tc_t(const void* Q, const __nv_bfloat16* hi, const __nv_bfloat16* lo, int32_t* idx, int* err,
                     const SelectParams& sp, cudaStream_t st) {
    constexpr int P = 128 / G;
    const int tiles_per_head = (sp.N + P - 1) / P;
    const size_t smem = sizeof(BtSmem);
    auto kern = bsa_tc_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)sp.B * sp.Hkv * tiles_per_head;
    kern<<<(unsigned)grid, kBtThreads, smem, st>>>((const __nv_bfloat16*)Q, hi, lo, idx, tiles_per_head, err, sp);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bsa_tc(const void* Q, const float* pyr, void* pyr_hl, int32_t* idx, int* err,
                          const SelectParams& sp, int G, int sms, cudaStream_t st) {
    cudaError_t e = launch_split_pyramid(pyr, pyr_hl, (int64_t)sp.B * sp.Hkv * sp.geom.rows * kD, sms, st);
    if (e != cudaSuccess) return e;
    const int64_t elems = (int64_t)sp.B * sp.Hkv * sp.geom.rows * kD;
    const __nv_bfloat16* hi = (const __nv_bfloat16*)pyr_hl;
    const __nv_bfloat16* lo = hi + elems;
    switch (G) {
        case 1: return bsa_tc_t<1>(Q, hi, lo, idx, err, sp, st);
        case 2: return bsa_tc_t<2>(Q, hi, lo, idx, err, sp, st);
        case 4: return bsa_tc_t<4>(Q, hi, lo, idx, err, sp, st);
        case 8: return bsa_tc_t<8>(Q, hi, lo, idx, err, sp, st);
        case 16: return bsa_tc_t<16>(Q, hi, lo, idx, err, sp, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pisa
