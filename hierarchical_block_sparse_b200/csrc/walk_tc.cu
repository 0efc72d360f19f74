// walk_tc.cu -- the coarse internal levels of the pyramid walk (Stage 1 of
// close reading §05 Algorithm 1; Eq.(5)-(7), (11); §5.3 forced and causal
// rules) for a tile of consecutive query positions on the tensor cores.
//
// A CTA takes 128 MMA rows: 128/G consecutive positions of one (b, kv-head)
// times the G query heads of the group. Every position walks the pyramid by
// the same rules as the one-warp-per-query walk (pisa_stage1.cuh): at each
// level its candidates are the children of the nodes it kept one level up;
// when it has more than K of them it keeps the forced ones and the best by
// the LSE over each candidate's two children (summed over the G heads), ties
// to the lower index. Consecutive positions keep mostly the same nodes, so
// the dot products are taken for the union of the tile's kept parents: each
// kept parent p at level l+1 contributes its four grandchildren (rows 4p..4p+3
// of level l-1, the children of its candidates 2p and 2p+1), in chunks of 32
// parents (128 columns). S = Q_tile x rows^T runs on tcgen05 into TMEM; the
// fp32 summaries enter as two bf16 parts (hi = bf16(x), lo = bf16(x - hi)),
// and q is bf16 already, so both products are exact and S carries the
// summaries to about 2^-16 of their size (about 1e-5 on a logit). Each row
// reads the four columns of each of its own kept parents (found with a
// bitmask per chunk) and writes its candidates' pair scores to shared memory;
// 2G adjacent lanes per position then rank them with the walk's keep rule.
//
// The levels above the first one where some position of the tile has more
// than K eligible nodes are not walked: there every eligible node is kept.
// Reuse across positions falls towards the leaves (the union grows), so a
// level whose union needs more chunks than tw_handoff_parents allows is left
// to the one-warp walk: each position's kept nodes go to the candidate region
// and its resume level to `resume` (stage1_kernel<..., RESUME> continues). A
// tile that finishes every level writes the level-1 candidates and the
// sibling-pair bucket counts itself, exactly as the one-warp walk does.
//
// Per chunk, the gather of the next chunk's rows (cp.async) runs while the
// current chunk's MMAs and row pick-up run: two B buffers and two 128-column
// TMEM accumulators. Warps 0-3 pick up column groups 0-1 of a chunk, warps
// 4-7 groups 2-3 (warp w reads TMEM lanes 32 (w % 4) ..).
#include <cmath>

#include "pisa_internal.h"
#include "pisa_walk.cuh"
#include "tc.cuh"

namespace pisa {
namespace {

constexpr int kTwThreads = 256;
constexpr int kTwPar = 32;            // union parents per chunk
constexpr int kTwMaxWords = 256;      // bitmap words: parent levels of up to 8192 nodes
constexpr int kTwMaxUnion = 2048;     // 128 positions x 16 kept nodes
// a level whose union needs more chunks than this goes to the one-warp walk:
// a chunk's MMAs serve all 128 rows, so tiles of fewer positions (GQA groups)
// afford fewer chunks per position
__host__ __device__ constexpr int tw_handoff_parents(int positions) { return (positions >= 128 ? 8 : 4) * kTwPar; }
constexpr int kD = 128;
constexpr int kSlots = 32;
constexpr int kPairs = 16;
constexpr int kBig = 0x7fffffff;

constexpr int kRow = 17;  // padded row of the per-position lists (one thread per position reads its own row)

struct TwSmem {
    uint8_t q[32768];        // A: 128 rows x 128 bf16, K-major canonical layout
    uint8_t b[2][2][32768];  // B[buffer][hi, lo]: 128 rows x 128 bf16
    float score[128 * kSlots];  // slot c, MMA row r at score_at<G>(c, r)
    int32_t kept[128][kRow];  // kept nodes of the level above, ascending
    int32_t keptu[128][kRow]; // their index in the union
    int32_t uni[kTwMaxUnion];
    uint32_t bits[kTwMaxWords];
    int32_t pre[kTwMaxWords];
    int32_t nkept[128];
    int32_t need[128];
    int32_t scan[8];
    uint64_t mbar[2];
    uint32_t tmem_base;
};

// Place of (slot c, MMA row r = position * G + head) in TwSmem::score: slot
// major, the row XOR-swizzled by the slot's lane group q = c / SPL (2G lanes
// per position, SPL = 32 / 2G slots per lane). A warp's pick-up stores (32
// consecutive rows, any slots) land in distinct banks but for pairs of rows
// 16 apart; a warp's ranking reads (16 consecutive rows, for a fixed head and
// slot index the 2G lanes of each position in different groups q) flip the
// head bits and bit 4 of the row by q, so they meet 32 distinct banks.
template <int G>
__device__ __forceinline__ int score_swz(int q) { return (q & (G - 1)) | ((q / G) << 4); }
template <int G>
__device__ __forceinline__ int score_at(int c, int r) {
    constexpr int SPL = kSlots / (2 * G);
    return c * 128 + (r ^ score_swz<G>(c / SPL));
}

// exclusive scan of one int per thread over the 256 threads; returns the total
__device__ __forceinline__ int block_exscan(int& v, int32_t* scan) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scan[warp] = x;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kTwThreads / 32; ++w) {
        const int s = scan[w];
        before += w < warp ? s : 0;
        total += s;
    }
    v = before + x - v;
    __syncthreads();
    return total;
}

__device__ __forceinline__ uint32_t idesc_n(int n) {  // kind::f16, bf16 x bf16 -> fp32, both K-major, M = 128
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// One position's candidates at level l are held by LPP = 2G adjacent lanes
// (all 256 threads serve the tile's 128/G positions): lane q of the group owns
// the SPL = 16/G slots q*SPL .. q*SPL + SPL - 1, slot c being child c & 1 of
// the position's (c >> 1)-th kept node one level up (the root alone in slot 0
// at l = L), so the slots ascend with the node index. Bit i of v: slot
// q*SPL + i exists and is eligible (causal: its first key is not after t); of
// f: it is on a forced path (close reading §5.3).
template <int SPL>
struct LaneCands {
    int node[SPL];
    uint32_t v, f;
};

template <int SPL>
__device__ __forceinline__ void lane_cands(const TwSmem& S, int pos, int l, int L, int64_t t, const SelectParams& p,
                                           int q, bool live, LaneCands<SPL>& lc) {
    // node i of level l exists and is eligible iff 0 <= i <= vmax (M_l = ceil(N / span))
    const int64_t span = (int64_t)p.C << (l - 1);
    const int64_t lastn = p.geom.M[l] - 1;
    const int vmax = (int)(p.causal ? min(lastn, t / span) : lastn);
    // the forced leaves' ancestors at level l (-2: none)
    const Forced F(t, p.C, p.causal, p.forced_mask);
    const int s = l - 1;
    const int fa = F.f0 >= 0 ? F.f0 >> s : -2, fb = F.f1 >= 0 ? F.f1 >> s : -2, fc = F.f2 >= 0 ? F.f2 >> s : -2;
    const int nk = (!live || l == L) ? 0 : S.nkept[pos];
    lc.v = lc.f = 0u;
    if constexpr (SPL >= 2) {  // parents q * SPL / 2 .. + SPL / 2 - 1, two slots each
#pragma unroll
        for (int jj = 0; jj < SPL / 2; ++jj) {
            const int j = q * (SPL / 2) + jj;
            const int par = !live ? -1 : l == L ? (j == 0 ? 0 : -1) : (j < nk ? S.kept[pos][j] : -1);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int i = 2 * jj + e;
                const int node = l == L ? (par == 0 && e == 0 ? 0 : -1) : (par >= 0 ? 2 * par + e : -1);
                lc.node[i] = node;
                const bool valid = (unsigned)node <= (unsigned)vmax;
                lc.v |= (valid ? 1u : 0u) << i;
                lc.f |= (valid && (node == fa || node == fb || node == fc) ? 1u : 0u) << i;
            }
        }
    } else {  // one slot: child q & 1 of parent q >> 1
        const int j = q >> 1, e = q & 1;
        const int par = !live ? -1 : l == L ? (j == 0 ? 0 : -1) : (j < nk ? S.kept[pos][j] : -1);
        const int node = l == L ? (par == 0 && e == 0 ? 0 : -1) : (par >= 0 ? 2 * par + e : -1);
        lc.node[0] = node;
        const bool valid = (unsigned)node <= (unsigned)vmax;
        lc.v = valid ? 1u : 0u;
        lc.f = valid && (node == fa || node == fb || node == fc) ? 1u : 0u;
    }
}

// the 32-slot mask of a position from its lanes' SPL-slot parts
template <int SPL>
__device__ __forceinline__ uint32_t group_mask(uint32_t m, int q) {
    constexpr int LPP = kSlots / SPL;
    uint32_t full = m << (q * SPL);
#pragma unroll
    for (int o = 1; o < LPP; o <<= 1) full |= __shfl_xor_sync(kFull, full, o);
    return full;
}

// the kept candidates (bit c of `keep`) in slot order, i.e. ascending node
// order; each lane writes its own slots
template <int SPL>
__device__ __forceinline__ void write_kept(TwSmem& S, int pos, const LaneCands<SPL>& lc, uint32_t keep, int q) {
    int n = __popc(keep & ((1u << (q * SPL)) - 1u));
    const uint32_t mine = (keep >> (q * SPL)) & (SPL == 32 ? 0xffffffffu : ((1u << SPL) - 1u));
#pragma unroll
    for (int i = 0; i < SPL; ++i)
        if ((mine >> i) & 1u) S.kept[pos][n++] = lc.node[i];
    if (q == 0) S.nkept[pos] = __popc(keep);
}

// the lowest k set bits of m
__device__ __forceinline__ uint32_t lowest_bits(uint32_t m, int k) {
    uint32_t r = 0u;
    for (int i = 0; i < k && m; ++i) {
        const uint32_t b = m & (0u - m);
        r |= b;
        m ^= b;
    }
    return r;
}

// order-preserving map of a float onto uint32 (larger float -> larger integer)
__device__ __forceinline__ uint32_t ordered(float x) {
    const uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The keep rule of a ranked level (close reading §04 4.2; Eq.(6)): forced
// candidates first, then the best scores, ties to the lower node (= lower
// slot). Keys are the scores mapped order-preservingly onto uint32 (forced:
// the maximum, not eligible: 0). A bitonic network sorts the 32 keys of a
// position descending, element e = q*SPL + i held by lane q of its group:
// compare-exchanges with partners less than SPL apart are in registers, the
// others exchange with lane q ^ (j / SPL). The K-th largest key tau is then
// known; the kept set is every key above tau and, of the keys equal to tau,
// the lowest slots that fill K. Returns the 32-slot keep mask on every lane.
template <int SPL>
__device__ __forceinline__ uint32_t rank_keep(const float* score, int stride, uint32_t vfull, uint32_t ffull,
                                              int K, int q) {
    constexpr uint32_t kMaskSpl = SPL == 32 ? 0xffffffffu : ((1u << SPL) - 1u);
    const uint32_t vm = (vfull >> (q * SPL)) & kMaskSpl, fm = (ffull >> (q * SPL)) & kMaskSpl;
    uint32_t a[SPL];
#pragma unroll
    for (int i = 0; i < SPL; ++i)
        a[i] = !((vm >> i) & 1u) ? 0u : ((fm >> i) & 1u) ? 0xffffffffu : ordered(score[i * stride]);
#pragma unroll
    for (int k = 2; k <= kSlots; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j < SPL) {
#pragma unroll
                for (int i = 0; i < SPL; ++i) {
                    const int m = i ^ j;
                    if (m > i) {
                        // (q * SPL + i) & k: the lane's part is a multiple of SPL
                        const bool desc = k < SPL ? (i & k) == 0 : ((q * SPL) & k) == 0;
                        const uint32_t x = a[i], y = a[m];
                        a[i] = desc ? max(x, y) : min(x, y);
                        a[m] = desc ? min(x, y) : max(x, y);
                    }
                }
            } else {
                const int lo_lane = (q & (j / SPL)) == 0;  // this lane holds the lower elements of its pairs
#pragma unroll
                for (int i = 0; i < SPL; ++i) {
                    const uint32_t o = __shfl_xor_sync(kFull, a[i], j / SPL);
                    const bool desc = k < SPL ? (i & k) == 0 : ((q * SPL) & k) == 0;
                    a[i] = (desc == (lo_lane != 0)) ? max(a[i], o) : min(a[i], o);
                }
            }
        }
    // element K - 1: lane (K - 1) / SPL of the group, register (K - 1) % SPL
    uint32_t tau = 0u;  // picked with masks (an indexed read would put a[] in local memory)
#pragma unroll
    for (int i = 0; i < SPL; ++i) tau |= a[i] & (0u - (uint32_t)(i == (K - 1) % SPL));
    constexpr int LPP = kSlots / SPL;
    tau = __shfl_sync(kFull, tau, ((threadIdx.x & 31) & ~(LPP - 1)) + (K - 1) / SPL);
    uint32_t gt = 0u, eq = 0u;
#pragma unroll
    for (int i = 0; i < SPL; ++i) {
        const uint32_t k = !((vm >> i) & 1u) ? 0u : ((fm >> i) & 1u) ? 0xffffffffu : ordered(score[i * stride]);
        gt |= (k > tau ? 1u : 0u) << i;
        eq |= (k == tau ? 1u : 0u) << i;
    }
    const uint32_t gt_full = group_mask<SPL>(gt, q), eq_full = group_mask<SPL>(eq, q);
    return (gt_full | lowest_bits(eq_full, K - __popc(gt_full))) & vfull;
}

template <int G>
__global__ void __launch_bounds__(kTwThreads, 1) walk_tc_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ pyr_hi,
    const __nv_bfloat16* __restrict__ pyr_lo, int32_t* __restrict__ cand_out, int32_t* __restrict__ resume,
    int32_t* __restrict__ counts, int32_t* __restrict__ slots, int tiles_per_head, int* __restrict__ err,
    SelectParams p) {
    constexpr int P = 128 / G;       // positions per tile
    constexpr int LPP = 2 * G;       // lanes per position in the per-position phases (LPP * P = 256)
    constexpr int SPL = kSlots / LPP;  // candidate slots per lane
    extern __shared__ __align__(1024) uint8_t dsm[];
    TwSmem& S = *reinterpret_cast<TwSmem*>(dsm);
    const int tid = threadIdx.x, warp = tid >> 5;

    // heaviest tiles (latest positions: the largest unions) first
    const int64_t nbh = (int64_t)p.B * p.Hkv;
    const int64_t bh = blockIdx.x % nbh;
    const int tile = tiles_per_head - 1 - (int)(blockIdx.x / nbh);
    const int64_t b = bh / p.Hkv;
    const int kvh = (int)(bh - b * p.Hkv);
    const int t0 = tile * P;
    const int L = p.geom.L;

    if (warp == 0) tc::tmem_alloc(&S.tmem_base, 256);
    if (tid == 0) {
        tc::mbar_init(&S.mbar[0], 1);
        tc::mbar_init(&S.mbar[1], 1);
        tc::fence_mbar_init();
    }
    // the tile's query rows (row r = position r / G, head r % G) into the A tile
    const uint32_t q_smem = tc::smem_u32(S.q);
    for (int i = tid; i < 128 * 16; i += kTwThreads) {
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
    uint32_t parity[2] = {0u, 0u};
    bool ok = true;

    const __nv_bfloat16* Hh = pyr_hi + bh * p.geom.rows * kD;
    const __nv_bfloat16* Hl = pyr_lo + bh * p.geom.rows * kD;

    // Above the first level where some position of the tile has more than K
    // eligible nodes, every position keeps every eligible node: its kept list
    // one level below that is simply all of its eligible nodes there.
    const int t_hi = min(t0 + P, p.N) - 1;
    int lstart = L;
    while (lstart >= 2) {
        const int64_t span = (int64_t)p.C << (lstart - 1);
        const int64_t n_elig = p.causal ? min(p.geom.M[lstart], (int64_t)t_hi / span + 1) : p.geom.M[lstart];
        if (n_elig > p.K) break;
        --lstart;
    }
    if (lstart < L) {  // kept lists at level lstart + 1 (at most K nodes each)
        const int64_t span = (int64_t)p.C << lstart;
        for (int i = tid; i < P * 16; i += kTwThreads) {
            const int pos = i >> 4, j = i & 15;
            const int64_t t = min(t0 + pos, p.N - 1);
            const int64_t n_elig = p.causal ? min(p.geom.M[lstart + 1], t / span + 1) : p.geom.M[lstart + 1];
            if (j < n_elig) S.kept[pos][j] = j;
            if (j == 0) S.nkept[pos] = (int)n_elig;
        }
        __syncthreads();
    }
    int lstop = 1;  // the level the one-warp walk resumes at (1: only the leaf candidates are left)

    for (int l = lstart; l >= 2 && ok; --l) {
        // ---- level state of every position; those that must rank flag their kept parents
        const int64_t span_par = (int64_t)p.C << l;  // tokens under a node of level l + 1
        const int t_last = min(t0 + P, p.N) - 1;
        // kept parents are eligible nodes: under causal masking none starts after the tile's last position
        const int64_t wnodes = l == L ? 1 : p.causal ? min(p.geom.M[l + 1], (int64_t)t_last / span_par + 1)
                                                      : p.geom.M[l + 1];
        const int words = (int)((wnodes + 31) >> 5);
        for (int i = tid; i < words; i += kTwThreads) S.bits[i] = 0u;
        __syncthreads();
        int any = 0;
        {  // LPP lanes per position
            const int pos = tid / LPP, q = tid % LPP;
            const bool live = t0 + pos < p.N;
            const int64_t t = live ? t0 + pos : 0;
            LaneCands<SPL> lc;
            lane_cands<SPL>(S, pos, l, L, t, p, q, live, lc);
            const uint32_t vfull = group_mask<SPL>(lc.v, q), ffull = group_mask<SPL>(lc.f, q);
            const int n = __popc(vfull), nf = __popc(ffull);
            const bool rank = live && n > p.K && nf < p.K;
            const int nk = live && l < L ? S.nkept[pos] : 0;
            __syncwarp();  // the group's lanes have read the kept nodes they expand
            if (live && !rank)  // all of them, or the forced ones fill the budget: no scores needed
                write_kept<SPL>(S, pos, lc, n <= p.K ? vfull : lowest_bits(ffull, p.K), q);
            if (rank) {  // flag the parents whose grandchildren are needed
                for (int j = q * SPL / 2; j < min(nk, (q + 1) * SPL / 2); ++j) {
                    const int par = S.kept[pos][j];
                    if (par >= 0 && par < wnodes) atomicOr(&S.bits[par >> 5], 1u << (par & 31));
                    else if (err) atomicCAS(err, 0, 16);  // self-check: a kept node past the tile's reach
                }
            }
            if (q == 0) S.need[pos] = rank ? 1 : 0;
            any = rank ? 1 : 0;
        }
        if (!__syncthreads_or(any)) continue;

        // ---- the union of the kept parents (sorted), and each parent's index in it
        int cnt = tid < words ? __popc(S.bits[tid]) : 0;
        const int nU = block_exscan(cnt, S.scan);
        if (tid < words) {
            S.pre[tid] = cnt;
            uint32_t wbits = S.bits[tid];
            int at = cnt;
            while (wbits) {
                const int bit = __ffs(wbits) - 1;
                wbits &= wbits - 1;
                S.uni[at++] = tid * 32 + bit;
            }
        }
        __syncthreads();
        if (S.need[tid / LPP]) {
            const int pos = tid / LPP, q = tid % LPP;
            const int nk = S.nkept[pos];
            for (int j = q * SPL / 2; j < min(nk, (q + 1) * SPL / 2); ++j) {
                const int par = S.kept[pos][j];
                const uint32_t below = S.bits[par >> 5] & ((1u << (par & 31)) - 1u);
                S.keptu[pos][j] = S.pre[par >> 5] + __popc(below);
            }
        }
        __syncthreads();

        // ---- chunks of 32 union parents: gather, MMA, pick-up
        const int64_t child_off = p.geom.off[l - 1];
        const int64_t child_M = p.geom.M[l - 1];
        const int child_rows = (int)child_M;  // rows of level l - 1 (a row exists iff its first key is before N)
        if (nU > tw_handoff_parents(P)) {  // low reuse from here down: the one-warp walk continues at level l
            lstop = l;
            break;
        }
        const int nch = (nU + kTwPar - 1) / kTwPar;
        auto gather = [&](int k, int buf) {
            const int n = min(kTwPar, nU - k * kTwPar);
            const uint32_t dst_hi = tc::smem_u32(S.b[buf][0]), dst_lo = tc::smem_u32(S.b[buf][1]);
            for (int i = tid; i < ((4 * n + 7) & ~7) * 32; i += kTwThreads) {
                // 8 rows of one core-matrix group per 16-byte chunk: each 8 lanes fill 128 contiguous bytes
                const int row = (i >> 8) * 8 + (i & 7), part = (i >> 3) & 31, c = part & 15;
                if (row >= 4 * n) continue;
                const int64_t node = 4 * (int64_t)S.uni[k * kTwPar + (row >> 2)] + (row & 3);
                const bool exists = node < child_M;
                const __nv_bfloat16* base = part < 16 ? Hh : Hl;
                const __nv_bfloat16* src = base + (child_off + (exists ? node : 0)) * kD + c * 8;
                const uint32_t dst = (part < 16 ? dst_hi : dst_lo) + tc::kmajor128_off(row, c);
                if (exists) tc::cp_async16(dst, src);
                else tc::cp_async_zero16(dst, src);
            }
            tc::cp_async_commit();
        };
        // this thread's row and its walk over its position's kept parents
        const int r = tid & 127, wg = tid >> 7;
        const int pos = r / G;
        const bool mine = pos < P && t0 + pos < p.N && S.need[pos];
        const int nk = mine ? S.nkept[pos] : 0;
        int uj[16];  // union index of each of its kept parents (ascending; kBig past the count)
#pragma unroll
        for (int j = 0; j < 16; ++j) uj[j] = j < nk ? S.keptu[pos][j] : kBig;
        gather(0, 0);
        for (int k = 0; k < nch; ++k) {
            const int buf = k & 1;
            tc::cp_async_wait_all();
            tc::fence_async_smem();
            __syncthreads();
            if (tid == 0) {
                tc::tc_fence_after();
                const int n = min(kTwPar, nU - k * kTwPar);
                const uint32_t idesc = idesc_n((4 * n + 15) & ~15);
                const uint32_t dt = tmem + (uint32_t)(buf * 128);
                const uint32_t bh_s = tc::smem_u32(S.b[buf][0]), bl_s = tc::smem_u32(S.b[buf][1]);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc::mma_bf16(dt, tc::smem_desc(q_smem + ks * 256, 128, 2048),
                                 tc::smem_desc(bh_s + ks * 256, 128, 2048), idesc, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc::mma_bf16(dt, tc::smem_desc(q_smem + ks * 256, 128, 2048),
                                 tc::smem_desc(bl_s + ks * 256, 128, 2048), idesc, 1u);
                tc::mma_commit(&S.mbar[buf]);
            }
            // the other buffer was read by chunk k - 1's MMAs, which completed before its pick-up
            if (k + 1 < nch) gather(k + 1, buf ^ 1);
            ok = __syncthreads_and(tc::mbar_wait(&S.mbar[buf], parity[buf], err, 15)) != 0;
            parity[buf] ^= 1u;
            if (!ok) break;
            tc::tc_fence_after();
            // bit i: union parent k * 32 + i is one of this row's kept parents;
            // `base`: how many of its kept parents lie in earlier chunks
            const int c0u = k * kTwPar;
            uint32_t mask = 0u;
            int base = 0;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int dlt = uj[j] - c0u;
                mask |= (dlt >= 0 && dlt < kTwPar) ? (1u << dlt) : 0u;
                base += uj[j] < c0u ? 1 : 0;
            }
            // this warp's two column groups (8 parents each: columns 32 g .. 32 g + 31):
            // both loads go out before the one wait
            const uint32_t m2[2] = {(mask >> (16 * wg)) & 0xffu, (mask >> (16 * wg + 8)) & 0xffu};
            const bool need[2] = {__any_sync(kFull, m2[0] != 0u) != 0, __any_sync(kFull, m2[1] != 0u) != 0};
            if (need[0] || need[1]) {
                float v[2][32];
                const uint32_t ta = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(buf * 128 + 64 * wg);
                if (need[0]) tc::tmem_ld32(ta, v[0]);
                if (need[1]) tc::tmem_ld32(ta + 32u, v[1]);
                tc::tmem_ld_wait();
#pragma unroll
                for (int gi = 0; gi < 2; ++gi) {
                    const int g = 2 * wg + gi;
                    const uint32_t m8 = m2[gi];
                    if (!need[gi]) continue;
                    const int before = base + __popc(mask & ((1u << (8 * g)) - 1u));
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if ((m8 >> i) & 1u) {
                            const int j = before + __popc(m8 & ((1u << i) - 1u));  // its place in the kept list
                            const int par = S.uni[c0u + 8 * g + i];
                            // children 4 par + 1 and 4 par + 3 (the second child of each candidate) may not exist
                            const bool has1 = 4 * par + 1 < child_rows, has3 = 4 * par + 3 < child_rows;
                            const float z0 = v[gi][4 * i] * p.qscale;
                            const float z1 = has1 ? v[gi][4 * i + 1] * p.qscale : -INFINITY;
                            const float z2 = v[gi][4 * i + 2] * p.qscale;
                            const float z3 = has3 ? v[gi][4 * i + 3] * p.qscale : -INFINITY;
                            float* sc0 = S.score + score_at<G>(2 * j, r);
                            float* sc1 = S.score + score_at<G>(2 * j + 1, r);
                            if (p.variant == 0) {  // Eq.(7): the LSE over the two children
                                *sc0 = lse2_pair(z0, z1);
                                *sc1 = lse2_pair(z2, z3);
                            } else {
                                *sc0 = pair_score(z0, z1, p.variant);
                                *sc1 = pair_score(z2, z3, p.variant);
                            }
                        }
                    }
                }
            }
            tc::tc_fence_before();
        }
        tc::cp_async_wait_all();
        __syncthreads();
        if (!ok) break;

        // ---- LPP lanes per ranking position: forced first, then the best by score (lower index on ties)
        {
            const int pos = tid / LPP, q = tid % LPP;
            const bool live = S.need[pos] != 0;
            LaneCands<SPL> lc;
            lane_cands<SPL>(S, pos, l, L, live ? t0 + pos : 0, p, q, live, lc);
            const uint32_t vfull = group_mask<SPL>(lc.v, q), ffull = group_mask<SPL>(lc.f, q);
            // this lane's slots q * SPL + i of the first head: sc[i * 128]
            const int swz = score_swz<G>(q);
            float* sc = S.score + q * SPL * 128 + ((pos * G) ^ swz);
            if (G > 1 && live) {  // Eq.(11): summed over the group, into the first head's entry
#pragma unroll
                for (int i = 0; i < SPL; ++i) {
                    float x = 0.f;
#pragma unroll
                    for (int hh = 0; hh < G; ++hh) x += S.score[(q * SPL + i) * 128 + ((pos * G + hh) ^ swz)];
                    sc[i * 128] = x;
                }
            }
            const uint32_t keep = rank_keep<SPL>(sc, 128, vfull, ffull, p.K, q);
            __syncwarp();  // the group's lanes have read the kept nodes they expand
            if (live) write_kept<SPL>(S, pos, lc, keep, q);
        }
        __syncthreads();
    }

    if (ok && lstop == 1) {
        // ---- every level done: the level-1 candidates and the sibling-pair
        // bucket counts, as the one-warp walk writes them
        const int pos = tid / LPP, q = tid % LPP;
        const bool live = t0 + pos < p.N;
        const int64_t t = live ? t0 + pos : 0;
        const int64_t M1 = p.geom.M[1];
        LaneCands<SPL> lc;
        lane_cands<SPL>(S, pos, 1, L, t, p, q, live, lc);
        uint32_t okm = 0u;  // slots holding a candidate (valid, in range)
        int last = -1;
#pragma unroll
        for (int i = 0; i < SPL; ++i) {
            const bool valid = (lc.v >> i) & 1u;
            const int cand = lc.node[i];
            const bool in_range = cand >= 0 && cand < M1;
            if (live && valid && !in_range && err) atomicCAS(err, 0, 10);  // self-check: never expected
            if (live && valid && last >= 0 && last >= cand && err) atomicCAS(err, 0, 14);  // slots ascend
            if (valid) last = cand;
            okm |= (valid && in_range ? 1u : 0u) << i;
        }
        const uint32_t ok_full = group_mask<SPL>(okm, q);
        const uint32_t free_full = ok_full & ~group_mask<SPL>(lc.f, q);
        // a sibling pair (slots 2i, 2i + 1) whose first slot holds a candidate and
        // has at least one leaf that is not forced counts once in its bucket
        int pnode[SPL];  // the even slots' nodes (odd slots' lanes leave them unused)
#pragma unroll
        for (int i = 0; i < SPL; ++i) pnode[i] = ((okm >> i) & 1u) ? lc.node[i] : -1;
        if (live) {
            const int64_t unit = bh * p.N + t;
#pragma unroll
            for (int i = 0; i < SPL; ++i) cand_out[unit * kSlots + q * SPL + i] = pnode[i];
#pragma unroll
            for (int i = 0; i < SPL; ++i) {
                const int c = q * SPL + i;
                if ((c & 1) == 0 && ((ok_full >> c) & 1u) && ((free_full >> c) & 3u))
                    slots[unit * kPairs + c / 2] = atomicAdd(&counts[bh * ((M1 + 1) / 2) + (pnode[i] >> 1)], 1);
            }
            if (q == 0) resume[unit] = 0;
        }
    } else if (ok) {
        // ---- hand each position's walk over to the one-warp walk: its kept
        // nodes one level above the level it resumes at
        const int pos = tid / LPP, q = tid % LPP;
        if (t0 + pos < p.N) {
            const int64_t unit = bh * p.N + t0 + pos;
            // positions that ranked at the level handed over still hold that level's parents
            const int level = S.need[pos] ? lstop : lstop - 1;
            const int nk = S.nkept[pos];
            for (int j = q * SPL / 2; j < min(nk, (q + 1) * SPL / 2); ++j) cand_out[unit * kSlots + j] = S.kept[pos][j];
            if (q == 0) resume[unit] = (level << 8) | nk;
        }
    }
    tc::cp_async_wait_all();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 256);
    }
}

// fp32 summaries -> bf16 high and low parts: hi = bf16(x), lo = bf16(x - hi)
__global__ void split_pyramid_kernel(const float4* __restrict__ pyr, uint2* __restrict__ hi, uint2* __restrict__ lo,
                                     int64_t n4) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 x = pyr[i];
        const __nv_bfloat162 h01 = __floats2bfloat162_rn(x.x, x.y), h23 = __floats2bfloat162_rn(x.z, x.w);
        const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
        const __nv_bfloat162 l01 = __floats2bfloat162_rn(x.x - f01.x, x.y - f01.y);
        const __nv_bfloat162 l23 = __floats2bfloat162_rn(x.z - f23.x, x.w - f23.y);
        uint2 uh, ul;
        uh.x = *reinterpret_cast<const uint32_t*>(&h01);
        uh.y = *reinterpret_cast<const uint32_t*>(&h23);
        ul.x = *reinterpret_cast<const uint32_t*>(&l01);
        ul.y = *reinterpret_cast<const uint32_t*>(&l23);
        hi[i] = uh;
        lo[i] = ul;
    }
}

cudaError_t launch_split_pyramid_impl(const float* pyr, void* pyr_hl, int64_t elems, int sms, cudaStream_t st) {
    __nv_bfloat16* hi = (__nv_bfloat16*)pyr_hl;
    split_pyramid_kernel<<<sms * 8, 256, 0, st>>>((const float4*)pyr, (uint2*)hi, (uint2*)(hi + elems), elems / 4);
    return cudaGetLastError();
}

template <int G>
cudaError_t walk_tc_t(const void* Q, const float* pyr, void* pyr_hl, int32_t* cand, int32_t* resume, int32_t* counts,
                      int32_t* slots, int* err, const SelectParams& sp, int sms, cudaStream_t st) {
    const int64_t elems = (int64_t)sp.B * sp.Hkv * sp.geom.rows * kD;
    cudaError_t e = launch_split_pyramid(pyr, pyr_hl, elems, sms, st);
    if (e != cudaSuccess) return e;
    const __nv_bfloat16* hi = (const __nv_bfloat16*)pyr_hl;
    const __nv_bfloat16* lo = hi + elems;
    constexpr int P = 128 / G;
    const int tiles_per_head = (sp.N + P - 1) / P;
    const size_t smem = sizeof(TwSmem);
    auto kern = walk_tc_kernel<G>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)sp.B * sp.Hkv * tiles_per_head;
    kern<<<(unsigned)grid, kTwThreads, smem, st>>>((const __nv_bfloat16*)Q, hi, lo, cand, resume, counts, slots,
                                                   tiles_per_head, err, sp);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_split_pyramid(const float* pyr, void* pyr_hl, int64_t elems, int sms, cudaStream_t st) {
    return launch_split_pyramid_impl(pyr, pyr_hl, elems, sms, st);
}

bool walk_tc_fits(const SelectParams& sp) {
    // at least one ranked level below the root's children, and a union bitmap
    // that covers the parent level of every ranked level (at most 8192 nodes)
    return sp.geom.L >= 3 && sp.geom.M[3] <= (int64_t)kTwMaxWords * 32;
}

size_t walk_tc_pyramid_bytes(int64_t units_bh, int64_t rows) { return (size_t)units_bh * rows * kD * 2 * 2; }

cudaError_t launch_walk_tc(const void* Q, const float* pyr, void* pyr_hl, int32_t* cand, int32_t* resume,
                           int32_t* counts, int32_t* slots, int* err, const SelectParams& sp, int G, int sms,
                           cudaStream_t st) {
    switch (G) {
        case 1: return walk_tc_t<1>(Q, pyr, pyr_hl, cand, resume, counts, slots, err, sp, sms, st);
        case 2: return walk_tc_t<2>(Q, pyr, pyr_hl, cand, resume, counts, slots, err, sp, sms, st);
        case 4: return walk_tc_t<4>(Q, pyr, pyr_hl, cand, resume, counts, slots, err, sp, sms, st);
        case 8: return walk_tc_t<8>(Q, pyr, pyr_hl, cand, resume, counts, slots, err, sp, sms, st);
        case 16: return walk_tc_t<16>(Q, pyr, pyr_hl, cand, resume, counts, slots, err, sp, sms, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pisa
