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
// the lower leaf. Every row keeps its best keys in a sorted list in registers
// (the list's top slots hold +inf placeholders for the forced leaves, so the
// entry to beat is always the last slot); a 32-column slice of scores marks
// the columns that beat it, and the lanes insert their marked columns in
// lockstep, a branch-free shift per insertion. Warps 0-3 take the first 64
// columns of each chunk and warps 4-7 the last 64, and one warp per position
// merges the two lists at the end. Output rows are sorted ascending, -1
// padded, as from the per-query kernel (bsa.cu).
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
constexpr int kTopPad = 17;   // stride of the lists handed to the merge
constexpr int kZPad = 33;     // stride of a lane's staged scores: a column's 32 lanes hit 32 banks
constexpr int kNone = 0x7fffffff;

struct BtSmem {
    uint8_t q[32768];              // A: 128 rows x 128 bf16, K-major
    uint8_t b[2][2][32768];        // B[buffer][hi, lo]: 128 leaf rows x 128 bf16; after the
                                   // scan, each warpgroup's lists (BtLists)
    float zs[8][32][kZPad];        // per warp and lane: one slice of scores, for the insertions
    uint64_t mbar[2];
    uint32_t tmem_base;
};
struct BtLists {
    float key[2][128][kTopPad];    // per warpgroup and position: its best keys, descending
    int32_t id[2][128][kTopPad];
};
static_assert(sizeof(BtLists) <= sizeof(BtSmem::b), "the lists fit in the tile buffers");

// z into a descending list (ties: the earlier entry stays first), no branches
__device__ __forceinline__ void top_insert(float (&k)[kTop], int (&id)[kTop], float z, int leaf) {
    bool c[kTop];
#pragma unroll
    for (int i = 0; i < kTop; ++i) c[i] = z > k[i];
#pragma unroll
    for (int i = kTop - 1; i > 0; --i) {
        k[i] = c[i - 1] ? k[i - 1] : (c[i] ? z : k[i]);
        id[i] = c[i - 1] ? id[i - 1] : (c[i] ? leaf : id[i]);
    }
    k[0] = c[0] ? z : k[0];
    id[0] = c[0] ? leaf : id[0];
}

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
    // this row's list: kTop - Kp placeholders (+inf, never displaced), then
    // Kp places for the ranked leaves; the entry to beat is k[kTop - 1]
    float lk[kTop];
    int li[kTop];
#pragma unroll
    for (int i = 0; i < kTop; ++i) {
        lk[i] = i < kTop - Kp ? INFINITY : -INFINITY;
        li[i] = kNone;
    }

    uint32_t parity[2] = {0u, 0u};
    bool ok = true;
    // Chunk k's B tile sits in buffer k & 1 of shared memory and its scores in
    // TMEM columns (k & 1) * 128. The MMAs of chunk k + 1 and the gather of
    // chunk k + 2 run while the threads scan chunk k.
    auto issue_mma = [&](int k) {
        if (tid == 0) {
            tc::tc_fence_after();
            const int buf = k & 1;
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
    };
    gather(0, 0);  // the Q tile went out in the group before this one
    if (nch > 1) gather(1, 1);
    if (nch > 1) tc::cp_async_wait_group<1>();
    else tc::cp_async_wait_all();
    tc::fence_async_smem();
    __syncthreads();
    issue_mma(0);
    for (int k = 0; k < nch; ++k) {
        const int buf = k & 1;
        ok = __syncthreads_and(tc::mbar_wait(&S.mbar[buf], parity[buf], err, 17)) != 0;
        parity[buf] ^= 1u;
        if (!ok) break;
        if (k + 2 < nch) gather(k + 2, buf);  // chunk k's MMAs have read this buffer
        if (k + 1 < nch) {
            if (k + 2 < nch) tc::cp_async_wait_group<1>();
            else tc::cp_async_wait_all();
            tc::fence_async_smem();
            __syncthreads();  // chunk k + 1's tile is in place, and chunk k - 1's scan has left TMEM buffer buf ^ 1
            issue_mma(k + 1);
        }
        tc::tc_fence_after();
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
            const int c0 = wg * 64 + gi * 32;
            const int64_t leaf0 = (int64_t)k * kBtCols + c0;
            if (leaf0 >= n_tile) break;  // uniform: the tile's leaves end here
            float v[32];
            tc::tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(buf * 128 + c0), v);
            tc::tmem_ld_wait();
            // eligible columns of this slice: causal, not forced
            const int64_t lim = c_max - leaf0 + 1;
            uint32_t elig = lim >= 32 ? 0xffffffffu : (lim <= 0 ? 0u : (1u << lim) - 1u);
            {
                const int f[3] = {F.f0, F.f1, F.f2};
#pragma unroll
                for (int i = 0; i < 3; ++i)
                    if (f[i] >= leaf0 && f[i] < leaf0 + 32) elig &= ~(1u << (f[i] - leaf0));
            }
            const float thr = lk[kTop - 1];
            uint32_t cm = 0;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float z = v[j] * p.qscale;
#pragma unroll
                for (int o = 1; o < G; o <<= 1) z += __shfl_xor_sync(kFull, z, o);  // Eq.(11)-style sum over the group
                v[j] = z;
                cm |= (z > thr ? 1u : 0u) << j;
            }
            cm = live ? cm & elig : 0u;
            if (__any_sync(kFull, cm != 0u)) {  // rare once the lists are full
                float* zrow = S.zs[warp][lane];
                if (cm) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) zrow[j] = v[j];
                }
                while (cm) {  // the lanes with marked columns take one each per round
                    const int j = __ffs(cm) - 1;
                    cm &= cm - 1u;
                    const float z = zrow[j];
                    if (z > lk[kTop - 1]) top_insert(lk, li, z, (int)(leaf0 + j));
                }
                __syncwarp();
            }
        }
        tc::tc_fence_before();
    }
    tc::cp_async_wait_all();
    __syncthreads();  // every MMA has completed (or the tile gave up): the tile buffers are free
    BtLists& Ls = *reinterpret_cast<BtLists*>(S.b);
    if (ok && live) {
#pragma unroll
        for (int i = 0; i < kTop; ++i) {
            const bool real = lk[i] != INFINITY;  // placeholders rank below every leaf
            Ls.key[wg][pos][i] = real ? lk[i] : -INFINITY;
            Ls.id[wg][pos][i] = real ? li[i] : kNone;
        }
    }
    __syncthreads();
    if (ok) {
        // one warp per position: merge the two lists, add the forced leaves, sort ascending
        for (int q = warp; q < P; q += kBtThreads / 32) {
            const int tq = t0 + q;
            if (tq >= p.N) continue;
            const Forced Fq(tq, p.C, p.causal, p.forced_mask);
            const int64_t cq = p.causal ? min(M1 - 1, (int64_t)tq / p.C) : M1 - 1;
            float key = Ls.key[lane >> 4][q][lane & 15];
            int id = Ls.id[lane >> 4][q][lane & 15];
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
