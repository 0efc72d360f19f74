// blockmajor.cu -- the two-stage, key-block-reuse form of PISA prefill on the
// tensor cores (close reading §05 Algorithm 1 and §5.1, Eq.(12)-(13)).
//
// Stage 1 (stage1_kernel): one warp per (b, kv-head, t) walks levels L..2
//   exactly as select_kernel does and writes the eligible leaf candidates
//   (at most 2K) of level 1 -- forced ones included -- to the workspace.
// Grouping (bucket_*): a counting sort turns the (query, slot) pairs of
//   non-forced leaves into one list per (b, kv-head, leaf), cut into tiles of
//   128/G queries.
// Stage 2 (leaf_score_kernel): the level-1 candidates come in sibling pairs
//   (both children of a kept level-2 node), grouped by that node. One tile per
//   step: the queries' rows of every head of the group are gathered into
//   shared memory (cp.async, canonical K-major layout), the pair's 128 keys
//   are loaded once, one tcgen05 MMA (M=128, N=128, K=128) writes the logits
//   to TMEM and the epilogue turns each row into the exact per-head LSE of
//   each leaf (Eq.7 at the leaves).
// Final Top-K (topk_kernel): per query, forced + best-ranked candidates by the
//   LSE summed over the group (Eq.11), written sorted; it also records each
//   head's partial softmax normaliser over the kept non-forced leaves.
// Forced leaves (forced_tile_kernel): the first, previous and current leaves
//   are shared by all queries of a leaf block, so they are scored and attended
//   densely per tile of consecutive queries; this completes each row's
//   normaliser Z and writes the initial fp32 output accumulator. They never go
//   through the grouping, whose atomics would otherwise pile onto a few leaves.
// Attention (attn_tile_kernel): the kept non-forced (query, leaf) pairs are
//   grouped the same way; per tile S = Q K^T (tcgen05, TMEM), P = 2^(S*scale - Z)
//   in bf16, O_part = P V (tcgen05, V as an MN-major operand), and each row of
//   O_part is added into the accumulator with one 512-byte bulk reduction; P
//   is already normalised, so no rescaling is needed.
// finalize_kernel converts the accumulator to the output dtype.
// Backward with the selection fixed (bwd_*): the same leaf grouping plus each
//   leaf's forced section; a statistics pass (S and dP per tile) gives every
//   (query, head) its normaliser and D, then key-major tiles accumulate dK and
//   dV per leaf in TMEM and add dQ rows with bulk reductions.
#include <cmath>
#include <type_traits>

#include "pisa_internal.h"
#include "pisa_stage1.cuh"
#include "pisa_walk.cuh"
#include "tc.cuh"

namespace pisa {

constexpr int kSlots = 32;   // level-1 candidates per query (2K <= 32)
constexpr int kPairs = 16;   // bucket slots recorded per query: sibling pairs, or kept leaves (K <= 16)
constexpr int kBlk = 64;     // leaf size handled by the tensor-core tiles
constexpr int kD = 128;      // head dimension handled by the tensor-core tiles
constexpr int kORowStride = kD * 4 + 16;  // staged fp32 output row: 16-byte pad keeps the row writes conflict-free

// ------------------------------------------------------------------ stage 1 ----

// Walker: Walk4S<G> (4 lanes per child row, q in shared memory) for G <= 2,
// the 32-slot reduce-scatter walker otherwise. Levels with at most K
// candidates keep them all (gather by rank); scored levels keep the forced
// nodes and the best by (score, lower index) through an all-pairs rank.
#ifndef PISA_STAGE1_CARVEOUT
#define PISA_STAGE1_CARVEOUT (-1)  // percent of the shared-memory maximum; -1: the driver's choice
#endif
#ifndef PISA_STAGE1_MINBLOCKS
#define PISA_STAGE1_MINBLOCKS 4  // 64 registers: 32 warps per SM hide the gathers' latency
#endif
// Grid: x = blocks of 8 query positions, y = b * Hkv + kvh. Besides the
// candidates, each lane adds its non-forced candidate to the leaf's bucket
// count (the grouping of stage 2).
// RESUME: the tensor-core tile walk (walk_tc.cu) has done the coarse levels;
// resume[unit] is 0 for a position it finished, else (resume level << 8 |
// count) with the kept nodes in cand_out's row, which this kernel reads
// before it overwrites the row with the level-1 candidates.
// (below the tile walk, the group-of-4+ walker runs faster with the registers
// of 3 CTAs per SM, no spills; the group-of-1-2 one with 4)
template <int G, class W, bool RESUME = false>
__global__ void __launch_bounds__(256, (RESUME && G >= 4) ? 3 : PISA_STAGE1_MINBLOCKS) stage1_kernel(const __nv_bfloat16* __restrict__ Q,
                                                     const float* __restrict__ pyr, int32_t* __restrict__ cand_out,
                                                     int32_t* __restrict__ counts, int32_t* __restrict__ slots,
                                                     int64_t M1, int* __restrict__ err, SelectParams p,
                                                     const int32_t* __restrict__ resume = nullptr) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= p.N) return;
    const int64_t bh = blockIdx.y;
    const int64_t unit = bh * p.N + t;
    if constexpr (RESUME) {
        if (resume[unit] == 0) return;  // the tile walk finished this position
    }
    const int64_t b = bh / p.Hkv;
    const int kvh = (int)(bh - b * p.Hkv);
    W w;
    __shared__ __align__(16) float s_q[8][128 * (G <= 2 ? G : 1)];
    if constexpr (G <= 2) w.qs = s_q[threadIdx.x >> 5];
    {
        const __nv_bfloat16* qrow[G];
#pragma unroll
        for (int h = 0; h < G; ++h) qrow[h] = Q + (((b * p.Hq + (int64_t)kvh * G + h) * p.N) + t) * kD;
        w.load_q(qrow, p.qscale, lane);
    }
    const float* P = pyr + bh * p.geom.rows * kD;
    const Forced F(t, p.C, p.causal, p.forced_mask);
    int cand = lane == 0 ? 0 : -1;
    int lstart = p.geom.L;
    if constexpr (RESUME) {
        const int meta = resume[unit];
        const int nk = meta & 0xff;
        lstart = meta >> 8;
        if (lstart < 1 || lstart >= p.geom.L || nk > p.K) {  // self-check: never expected
            if (lane == 0 && err) atomicCAS(err, 0, 18);
            lstart = 1;
        }
        const int par = lane < nk ? cand_out[unit * kSlots + lane] : -1;
        const int pp = __shfl_sync(kFull, par, lane >> 1);
        cand = lane < 2 * nk && pp >= 0 ? 2 * pp + (lane & 1) : -1;
        __syncwarp();
    }
    for (int l = lstart; l >= 2; --l) {
        const LevelState s = level_state(cand, l, p.C, p.N, t, p.causal, F);
        int parent;
        if (s.n <= p.K) {
            parent = compact_by_rank(cand, s.vmask, lane >> 1);
            cand = lane < 2 * s.n ? 2 * parent + (lane & 1) : -1;
            continue;
        }
        float score = -INFINITY;
        const unsigned fmask = __ballot_sync(kFull, s.forced);
        if (__popc(fmask) < p.K)
            score = w.score_internal(cand, s.vmask & ~fmask, P + p.geom.off[l - 1] * kD,
                                     (int64_t)p.C << (l - 2), p.N, lane, p.variant);
        int id = cand;
        const int kept = keep_topk_lane(id, s.forced ? INFINITY : score, s.valid, p.K, lane);
        parent = __shfl_sync(kFull, id, lane >> 1);
        cand = lane < 2 * kept ? 2 * parent + (lane & 1) : -1;
    }
    const LevelState s = level_state(cand, 1, p.C, p.N, t, p.causal, F);
    const bool in_range = cand >= 0 && cand < M1;
    if (s.valid && !in_range && err) atomicCAS(err, 0, 10);  // self-check: never expected
    // self-check of the lane order the keep relies on: valid candidates ascend
    const int prev = __shfl_up_sync(kFull, cand, 1);
    const bool prev_valid = __shfl_up_sync(kFull, s.valid, 1);
    if (lane > 0 && s.valid && prev_valid && prev >= cand && err) atomicCAS(err, 0, 14);
    const bool ok = s.valid && in_range;
    cand_out[unit * kSlots + lane] = ok ? cand : -1;
    // lanes 2i, 2i+1 hold the two children of one kept level-2 node: the pair
    // is scored together, so the bucket is that node (counted once per pair);
    // the count before this pair's increment is its slot in the bucket
    const bool free_leaf = ok && !s.forced;
    const bool odd_free = __shfl_down_sync(kFull, free_leaf, 1);
    if ((lane & 1) == 0 && ok && (free_leaf || odd_free))
        slots[unit * kPairs + (lane >> 1)] = atomicAdd(&counts[bh * ((M1 + 1) / 2) + (cand >> 1)], 1);
}

// --------------------------------------------------------------- grouping ----

// Grouping of the (query, leaf) pairs that are not forced leaves of the query
// (the forced ones are handled densely by forced_tile_kernel). One warp per
// query position (grid x = blocks of 8 positions, y = b * Hkv + kvh); lane =
// slot of `src` (stride <= 32 leaf ids per query, -1 = none).
struct GroupParams {
    int N, C, causal, forced_mask, stride;
    int64_t M1;
};

__device__ __forceinline__ int free_leaf(const int32_t* src, const GroupParams& g, int64_t unit, int t, int lane) {
    if (lane >= g.stride) return -1;
    const int leaf = src[unit * g.stride + lane];
    if (leaf < 0) return -1;
    const Forced F(t, g.C, g.causal, g.forced_mask);
    return F.has(leaf, 1) ? -1 : leaf;
}

// Counting is also placing: the count a list entry finds in its bucket before
// its own increment is its slot there, recorded in slots[unit * kPairs + lane]
// (g.stride <= kPairs), so the fill after the scan needs no atomics.
__global__ void bucket_count_kernel(const int32_t* __restrict__ src, GroupParams g, int32_t* __restrict__ counts,
                                    int32_t* __restrict__ slots) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= g.N) return;
    const int64_t bh = blockIdx.y;
    const int64_t unit = bh * g.N + t;
    const int leaf = free_leaf(src, g, unit, t, lane);
    if (leaf >= 0) slots[unit * kPairs + lane] = atomicAdd(&counts[bh * g.M1 + leaf], 1);
}

// Exclusive scan of the bucket counts into entry offsets, and the tile list
// (b*Hkv + kvh, leaf, first entry, entries) of every bucket, in two passes
// over blocks of kScanBlock buckets: per-block totals, then each block adds
// the totals of the blocks before it and scans its own buckets.
constexpr int kScanBlock = 1024;

// self-check: a bucket holds at most one entry per query position
__device__ __forceinline__ int bucket_count(const int32_t* counts, int64_t i, int64_t nbuckets, int N, int* err) {
    if (i >= nbuckets) return 0;
    const int c = counts[i];
    if (c < 0 || c > N) {
        if (err) atomicCAS(err, 0, 11);
        return 0;
    }
    return c;
}

// inclusive scan of (a, b) over the block's 1024 threads
__device__ __forceinline__ void block_scan2(long long& a, long long& b, long long* s_a, long long* s_b) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long xa = __shfl_up_sync(kFull, a, o), xb = __shfl_up_sync(kFull, b, o);
        if (lane >= o) {
            a += xa;
            b += xb;
        }
    }
    if (lane == 31) {
        s_a[warp] = a;
        s_b[warp] = b;
    }
    __syncthreads();
    if (warp == 0) {
        long long wa = s_a[lane], wb = s_b[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long xa = __shfl_up_sync(kFull, wa, o), xb = __shfl_up_sync(kFull, wb, o);
            if (lane >= o) {
                wa += xa;
                wb += xb;
            }
        }
        s_a[lane] = wa;  // inclusive totals of warps 0..lane
        s_b[lane] = wb;
    }
    __syncthreads();
    if (warp > 0) {
        a += s_a[warp - 1];
        b += s_b[warp - 1];
    }
}

__global__ void __launch_bounds__(kScanBlock) bucket_total_kernel(const int32_t* __restrict__ counts,
                                                                 int64_t nbuckets, int per_tile, int N,
                                                                 longlong2* __restrict__ bsum, int* __restrict__ err) {
    __shared__ long long s_a[32], s_b[32];
    const int c = bucket_count(counts, (int64_t)blockIdx.x * kScanBlock + threadIdx.x, nbuckets, N, err);
    long long e = c, t = (c + per_tile - 1) / per_tile;
    block_scan2(e, t, s_a, s_b);
    if (threadIdx.x == kScanBlock - 1) bsum[blockIdx.x] = make_longlong2(e, t);
}

__global__ void __launch_bounds__(kScanBlock) bucket_place_kernel(const int32_t* __restrict__ counts,
                                                                 int64_t nbuckets, int64_t M1, int per_tile, int N,
                                                                 const longlong2* __restrict__ bsum,
                                                                 int32_t* __restrict__ offsets,
                                                                 int4* __restrict__ tiles,
                                                                 int32_t* __restrict__ ntiles) {
    __shared__ long long s_a[32], s_b[32];
    __shared__ long long s_pre[2];
    // entries and tiles of the blocks before this one
    long long pe = 0, pt = 0;
    for (int j = threadIdx.x; j < (int)blockIdx.x; j += kScanBlock) {
        pe += bsum[j].x;
        pt += bsum[j].y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        pe += __shfl_xor_sync(kFull, pe, o);
        pt += __shfl_xor_sync(kFull, pt, o);
    }
    if (threadIdx.x == 0) s_pre[0] = s_pre[1] = 0;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(reinterpret_cast<unsigned long long*>(&s_pre[0]), (unsigned long long)pe);
        atomicAdd(reinterpret_cast<unsigned long long*>(&s_pre[1]), (unsigned long long)pt);
    }
    __syncthreads();
    const int64_t i = (int64_t)blockIdx.x * kScanBlock + threadIdx.x;
    const int c = bucket_count(counts, i, nbuckets, N, nullptr);
    const int nt = (c + per_tile - 1) / per_tile;
    long long e = c, t = nt;
    block_scan2(e, t, s_a, s_b);
    const long long be = s_pre[0] + e - c, bt = s_pre[1] + t - nt;  // exclusive
    if (i < nbuckets) {
        offsets[i] = (int32_t)be;
        for (int j = 0; j < nt; ++j)
            tiles[bt + j] = make_int4((int)(i / M1), (int)(i % M1), (int)(be + (int64_t)j * per_tile),
                                      min(per_tile, c - j * per_tile));
    }
    if (blockIdx.x == gridDim.x - 1 && threadIdx.x == kScanBlock - 1) *ntiles = (int32_t)(s_pre[1] + t);
}

// one warp per query position: write (t << 5 | slot) into each bucket
__global__ void bucket_fill_kernel(const int32_t* __restrict__ src, GroupParams g,
                                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ slots,
                                   uint32_t* __restrict__ entries) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= g.N) return;
    const int64_t bh = blockIdx.y;
    const int64_t unit = bh * g.N + t;
    const int leaf = free_leaf(src, g, unit, t, lane);
    if (leaf < 0) return;
    entries[offsets[bh * g.M1 + leaf] + slots[unit * kPairs + lane]] = ((uint32_t)t << 5) | (uint32_t)lane;
}

// Sibling pairs of level-1 candidates (slots 2i, 2i+1, children of one kept
// level-2 node): one entry (t << 5 | i) per pair with at least one non-forced
// leaf, in the bucket of that level-2 node. One warp per query position.
__global__ void bucket_fill_pairs_kernel(const int32_t* __restrict__ cand, GroupParams g,
                                         const int32_t* __restrict__ offsets, const int32_t* __restrict__ slots,
                                         uint32_t* __restrict__ entries) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= g.N) return;
    if (lane >= kSlots / 2) return;
    const int64_t bh = blockIdx.y;
    const int64_t unit = bh * g.N + t;
    const int leaf0 = cand[unit * kSlots + 2 * lane];
    const int leaf1 = cand[unit * kSlots + 2 * lane + 1];
    if (leaf0 < 0) return;
    const Forced F(t, g.C, g.causal, g.forced_mask);
    const bool f0 = !F.has(leaf0, 1), f1 = leaf1 >= 0 && !F.has(leaf1, 1);
    if (!f0 && !f1) return;
    const int64_t key = bh * g.M1 + (leaf0 >> 1);  // g.M1 = level-2 nodes per sequence here
    entries[offsets[key] + slots[unit * kPairs + lane]] = ((uint32_t)t << 5) | (uint32_t)lane;
}

// ---------------------------------------------------------- tile plumbing ----

struct TileRows {
    int t[128];     // query position of each MMA row (-1: empty row)
    int slot[128];  // candidate slot of that query
};

// self-check of a tile descriptor (b*Hkv+kvh, leaf, first entry, entries)
__device__ __forceinline__ bool tile_sane(const int4& td, int64_t bhs, int64_t M1, int per_tile) {
    return td.x >= 0 && td.x < bhs && td.y >= 0 && td.y < M1 && td.z >= 0 && td.w > 0 && td.w <= per_tile;
}

// Row r of a tile is (entry r / G, head r % G). Fills row metadata.
template <int G>
__device__ __forceinline__ void tile_rows(TileRows& tr, const uint32_t* entries, int start, int len, int N,
                                          int* err, int tid) {
    const int e = tid / G;
    tr.t[tid] = -1;
    tr.slot[tid] = 0;
    if (e < len) {
        const uint32_t v = entries[start + e];
        const int t = (int)(v >> 5);
        if (t < N) {
            tr.t[tid] = t;
            tr.slot[tid] = (int)(v & 31u);
        } else if (err) {
            atomicCAS(err, 0, 13);  // self-check: never expected
        }
    }
}

// gather the 128 query rows (head kvh*G + r%G, position t) into the K-major A tile
template <int G>
__device__ __forceinline__ void gather_q(uint32_t a_smem, const TileRows& tr, const __nv_bfloat16* Q, int64_t b,
                                         int kvh, int Hq, int N, int tid) {
    const int i = tid & 7, c = tid >> 3;  // row within the 8-row group, 16-byte chunk
#pragma unroll 4
    for (int g = 0; g < 16; ++g) {
        const int r = g * 8 + i;
        const int t = tr.t[r];
        if (t >= 0) {
            const __nv_bfloat16* src = Q + (((b * Hq + (int64_t)kvh * G + (r % G)) * N) + t) * kD + c * 8;
            tc::cp_async16(a_smem + tc::kmajor128_off(r, c), src);
        }
    }
}

// ROWS key rows (64: one leaf, 128: a sibling pair) into a K-major B tile
// (rows past n_keys are zero)
template <int ROWS = 64>
__device__ __forceinline__ void load_kblock(uint32_t b_smem, const __nv_bfloat16* Kh, int64_t row0, int64_t n_keys,
                                            int tid) {
    const int i = tid & 7, c = tid >> 3;
#pragma unroll
    for (int g = 0; g < ROWS / 8; ++g) {
        const int r = g * 8 + i;
        const int64_t row = row0 + r;
        const __nv_bfloat16* src = Kh + (row < n_keys ? row : row0) * kD + c * 8;
        if (row < n_keys) tc::cp_async16(b_smem + tc::kmajor128_off(r, c), src);
        else tc::cp_async_zero16(b_smem + tc::kmajor128_off(r, c), src);
    }
}

// the leaf's 64 value rows into the MN-major V tile (rows past n_keys are zero)
__device__ __forceinline__ void load_vblock(uint32_t v_smem, const __nv_bfloat16* Vh, int64_t row0, int64_t n_keys,
                                            int tid) {
    const int k = tid & 63, j0 = tid >> 6;  // key, first dim chunk
#pragma unroll
    for (int j = j0; j < 16; j += 2) {
        const int64_t row = row0 + k;
        const __nv_bfloat16* src = Vh + (row < n_keys ? row : row0) * kD + j * 8;
        if (row < n_keys) tc::cp_async16(v_smem + tc::mnmajor_v_off(k, j), src);
        else tc::cp_async_zero16(v_smem + tc::mnmajor_v_off(k, j), src);
    }
}

template <int NK = 64>
__device__ __forceinline__ void issue_qk(uint32_t tmem_s, uint32_t a_smem, uint32_t b_smem) {
    constexpr uint32_t idesc = tc::idesc_bf16(128, NK, 0);
#pragma unroll
    for (int k = 0; k < 8; ++k)
        tc::mma_bf16(tmem_s, tc::smem_desc(a_smem + k * 256, 128, 2048), tc::smem_desc(b_smem + k * 256, 128, 2048),
                     idesc, k > 0);
}

// keys of leaf `leaf` that query t may attend to (0 when none)
__device__ __forceinline__ int visible_keys(int64_t leaf, int64_t t, int N, int causal) {
    int64_t n = min((int64_t)kBlk, (int64_t)N - leaf * kBlk);
    if (causal) n = min(n, t - leaf * kBlk + 1);
    return n > 0 ? (int)n : 0;
}

__device__ __forceinline__ float logaddexp2f(float a, float b) {
    const float m = fmaxf(a, b);
    return m == -INFINITY ? -INFINITY : m + log2f(exp2f(a - m) + exp2f(b - m));
}

// ------------------------------------------------------- stage 2: leaf LSEs ----

struct TileParams {
    int B, Hq, Hkv, N, causal;
    int64_t M1;
    float qscale;  // log2(e) / sqrt(d)
    int max_tiles;  // capacity of the tile list
    int variant;    // enum pisa_score (leaf scoring: PISA-1 / PISA-2 ranking scores when nonzero)
};

// Per-head LSE (log2 units) of every listed (query, candidate leaf):
// lse[(unit * 32 + slot) * G + head]. PAIR: a tile's key is a level-2 node p
// and its entries are sibling-pair slots i; the 128 keys of leaves 2p and 2p+1
// are scored by one N = 128 MMA and each non-forced visible leaf's LSE goes to
// slot 2i or 2i+1.
template <int G, bool PAIR, bool VSCORE = false>
__global__ void __launch_bounds__(128) leaf_score_kernel(const __nv_bfloat16* __restrict__ Q,
                                                         const __nv_bfloat16* __restrict__ Kmat,
                                                         const int4* __restrict__ tiles,
                                                         const int32_t* __restrict__ ntiles_ptr,
                                                         const uint32_t* __restrict__ entries,
                                                         float* __restrict__ lse, float* __restrict__ vscore,
                                                         int* __restrict__ err, TileParams p, int forced_mask) {
    constexpr int NK = PAIR ? 128 : 64;  // keys per tile
    extern __shared__ __align__(1024) uint8_t dsm[];
    uint8_t* sA = dsm;           // 32 KB gathered query rows
    uint8_t* sB = dsm + 32768;   // NK x 256 B key rows
    // Two row tables: while tile i's logits are turned into LSEs, tile i + 1's
    // metadata is read and its query and key rows are gathered into the
    // operand buffers (free once tile i's MMA has completed).
    __shared__ TileRows trs[2];
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5;
    if (warp == 0) tc::tmem_alloc(&tmem_base, NK);
    if (tid == 0) {
        tc::mbar_init(&mbar, 1);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t a_smem = tc::smem_u32(sA), b_smem = tc::smem_u32(sB);
    const int ntiles = min(*ntiles_ptr, p.max_tiles);
    const int64_t nkeys = PAIR ? (p.M1 + 1) / 2 : p.M1;
    uint32_t phase = 0;
    bool ok = true;
    // tile descriptor + the row table; false for a tile past the list or a malformed one
    auto fetch = [&](int tile, int buf, int4& td) {
        if (tile >= ntiles) return false;
        td = tiles[tile];
        if (!tile_sane(td, (int64_t)p.B * p.Hkv, nkeys, 128 / G)) {  // self-check: never expected
            if (tid == 0) atomicCAS(err, 0, 12);
            return false;
        }
        tile_rows<G>(trs[buf], entries, td.z, td.w, p.N, err, tid);
        return true;
    };
    // Consecutive tiles of a bucket share their key block, so each CTA takes
    // runs of kRun consecutive tiles (run r of CTA c is r * gridDim.x + c) and
    // reloads the keys only when the bucket changes.
    constexpr int kRun = 8;
    auto tile_of = [&](int it) { return ((it / kRun) * (int)gridDim.x + (int)blockIdx.x) * kRun + it % kRun; };
    int2 kb_loaded = make_int2(-1, -1);  // (b * Hkv + kvh, key) of the key block in sB
    auto gather = [&](const int4& td, int buf) {
        const int64_t bh = td.x;
        const int64_t b = bh / p.Hkv;
        gather_q<G>(a_smem, trs[buf], Q, b, (int)(bh - b * p.Hkv), p.Hq, p.N, tid);
        if (kb_loaded.x != td.x || kb_loaded.y != td.y) {
            load_kblock<NK>(b_smem, Kmat + bh * p.N * kD, (int64_t)td.y * NK, p.N, tid);
            kb_loaded = make_int2(td.x, td.y);
        }
        tc::cp_async_commit();
    };
    int4 td_next;
    bool have_next = fetch(tile_of(0), 0, td_next);
    __syncthreads();
    if (have_next) gather(td_next, 0);
    int buf = 0;
    for (int it = 0, tile = tile_of(0); tile < ntiles; tile = tile_of(++it), buf ^= 1) {
        const int4 td = td_next;
        const bool have = have_next;
        const int64_t bh = td.x, key = td.y;
        tc::cp_async_wait_all();
        tc::fence_async_smem();
        __syncthreads();
        if (have && tid == 0) {
            tc::tc_fence_after();
            issue_qk<NK>(tmem, a_smem, b_smem);
            tc::mma_commit(&mbar);
        }
        // the next tile's row table goes to the other buffer (read last by tile i - 1's epilogue)
        have_next = fetch(tile_of(it + 1), buf ^ 1, td_next);
        // a CTA-uniform verdict: every thread polls, all agree before moving on
        if (have) {
            ok = __syncthreads_and(tc::mbar_wait(&mbar, phase, err, 1)) != 0;
            phase ^= 1;
        } else {
            __syncthreads();
        }
        if (!ok) break;
        if (have_next) gather(td_next, buf ^ 1);  // the operand buffers are free: this tile's MMA is done
        if (!have) continue;
        tc::tc_fence_after();
        const TileRows& tr = trs[buf];
        const int t = tr.t[tid];
        const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
        for (int half = 0; half < NK / 64; ++half) {
            float v[64];
            tc::tmem_ld32(taddr + half * 64, v);
            tc::tmem_ld32(taddr + half * 64 + 32, v + 32);
            tc::tmem_ld_wait();
            const int64_t leaf = PAIR ? 2 * key + half : key;
            int slot = tr.slot[tid];
            bool write = t >= 0;
            if (PAIR && write) {
                slot = 2 * slot + half;
                const Forced F(t, kBlk, p.causal, forced_mask);
                write = !F.has((int)leaf, 1);
            }
            const int nvalid = write ? visible_keys(leaf, t, p.N, p.causal) : 0;
            if (write && (!PAIR || nvalid > 0)) {
                float m = -INFINITY;
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (j < nvalid) m = fmaxf(m, v[j] * p.qscale);
                float s = 0.f;
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (j < nvalid) s += ex2_approx(v[j] * p.qscale - m);
                const int64_t unit = bh * p.N + t;
                lse[(unit * kSlots + slot) * G + (tid % G)] = m + lg2_approx(s);
                if constexpr (VSCORE) {  // PISA-1 / PISA-2 ranking score: two-pass mean and variance of the logits
                    float sum = 0.f;
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (j < nvalid) sum += v[j];
                    const float mean = sum / (float)nvalid;
                    float m2 = 0.f;
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (j < nvalid) m2 += (v[j] - mean) * (v[j] - mean);
                    const float mean2 = mean * p.qscale, var2 = m2 / (float)nvalid * p.qscale * p.qscale;
                    vscore[(unit * kSlots + slot) * G + (tid % G)] =
                        p.variant == 1 ? mean2 : mean2 + kHalfLn2 * var2;
                }
            }
        }
        tc::tc_fence_before();
    }
    tc::cp_async_wait_all();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, NK);
    }
}

// ----------------------------------------------------------- final Top-K ----

// One warp per kTopkQ consecutive positions of one (b, kv-head); lane =
// candidate slot. Keeps forced + best by the LSE summed over the group (ties:
// lower leaf: valid candidates arrive in ascending order, so the lane order is
// the index order and the kept leaves come out sorted), writes idx and the
// per-head partial normaliser z2[unit * G + h] = log2 sum 2^lse over the kept
// leaves that are not forced (forced_tile_kernel adds the forced ones).
// Each kept free leaf also gets its slot in the attention bucket of its leaf.
// Consecutive positions keep many of the same leaves, so a CTA (8 warps, 32
// positions) first counts its own entries per leaf in a shared-memory hash
// table (local slots), then reserves each leaf's range with one global atomic
// (its base), and an entry's slot is base + local slot.
constexpr int kTopkQ = 4;
constexpr int kTopkHash = 1024;  // > the at most 32 x 16 distinct leaves of a CTA

template <int G>
__global__ void __launch_bounds__(256) topk_kernel(const int32_t* __restrict__ cand, const float* __restrict__ lse,
                                                   const float* __restrict__ vscore,
                                                   int32_t* __restrict__ idx, float* __restrict__ z2,
                                                   int32_t* __restrict__ counts, int32_t* __restrict__ slots,
                                                   int64_t M1, SelectParams p) {
    __shared__ int s_key[kTopkHash], s_cnt[kTopkHash], s_base[kTopkHash];
    for (int e = threadIdx.x; e < kTopkHash; e += blockDim.x) {
        s_key[e] = -1;
        s_cnt[e] = 0;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int t0 = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kTopkQ;
    const int64_t bh = blockIdx.y;
    int out_leaf[kTopkQ];  // lane < K: the lane-th kept leaf that needs a bucket slot, else -1
#pragma unroll
    for (int i = 0; i < kTopkQ; ++i) out_leaf[i] = -1;
    if (t0 < p.N) {  // (warps past the end still take part in the CTA's barriers)
    // all positions' candidates and LSEs are loaded first (independent requests in flight)
    int leaves[kTopkQ];
    float l2s[kTopkQ][G], rank_score[kTopkQ];
#pragma unroll
    for (int i = 0; i < kTopkQ; ++i) {
        const int64_t unit = bh * p.N + t0 + i;
        leaves[i] = t0 + i < p.N ? cand[unit * kSlots + lane] : -1;
        rank_score[i] = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            l2s[i][h] = t0 + i < p.N ? lse[(unit * kSlots + lane) * G + h] : -INFINITY;
            // ranking: the Eq.(7) LSE, or the PISA-1 / PISA-2 score, summed over the group (Eq.11)
            rank_score[i] += vscore ? (t0 + i < p.N ? vscore[(unit * kSlots + lane) * G + h] : -INFINITY) : l2s[i][h];
        }
    }
#pragma unroll
    for (int i = 0; i < kTopkQ; ++i) {
        out_leaf[i] = -1;
        const int t = t0 + i;
        if (t >= p.N) continue;
        const int64_t unit = bh * p.N + t;
        const Forced F(t, p.C, p.causal, p.forced_mask);
        const int leaf = leaves[i];
        float l2[G];
#pragma unroll
        for (int h = 0; h < G; ++h) l2[h] = leaf >= 0 ? l2s[i][h] : -INFINITY;
        const float score = leaf >= 0 ? rank_score[i] : -INFINITY;
        const bool valid = leaf >= 0;
        const bool forced = valid && F.has(leaf, 1);
        const unsigned vmask = __ballot_sync(kFull, valid);
        int id = leaf;
        unsigned kmask;
        int kept;
        if (__popc(vmask) <= p.K) {
            kmask = vmask;
            kept = __popc(vmask);
            id = compact_by_rank(leaf, vmask, lane);
        } else {
            kept = keep_topk_lane(id, forced ? INFINITY : score, valid, p.K, lane, &kmask);
        }
        const bool mine = ((kmask >> lane) & 1u) && !forced;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float x = mine ? l2[h] : -INFINITY;
            float m = x;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
            float e = mine ? exp2f(x - m) : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(kFull, e, o);
            if (lane == 0) z2[unit * G + h] = m + log2f(e);
        }
        const int v = lane < kept ? id : -1;
        if (lane < p.K) idx[unit * p.K + lane] = v;
        if (lane < p.K && v >= 0 && !F.has(v, 1)) out_leaf[i] = v;
    }
    }  // t0 < p.N
    // bucket slots of the kept free leaves: local slots per leaf in the CTA's
    // hash table, one global reservation per distinct leaf, slot = base + local
    int hslot[kTopkQ], local[kTopkQ];
#pragma unroll
    for (int i = 0; i < kTopkQ; ++i) {
        hslot[i] = -1;
        local[i] = 0;
        const int leaf = out_leaf[i];
        if (leaf < 0) continue;
        int h = (int)(((uint32_t)leaf * 2654435761u) >> 22);  // 10 bits
        for (int probe = 0; probe < kTopkHash; ++probe) {
            const int k = atomicCAS(&s_key[h], -1, leaf);
            if (k == -1 || k == leaf) break;
            h = (h + 1) & (kTopkHash - 1);
        }
        hslot[i] = h;
        local[i] = atomicAdd(&s_cnt[h], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kTopkHash; e += blockDim.x) {
        const int leaf = s_key[e];
        if (leaf >= 0) s_base[e] = atomicAdd(&counts[bh * M1 + leaf], s_cnt[e]);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kTopkQ; ++i)
        if (hslot[i] >= 0) slots[(bh * p.N + t0 + i) * kPairs + lane] = s_base[hslot[i]] + local[i];
}

// ------------------------------------------------------ attention tiles ----

// For every listed (query, kept leaf): O_acc[row] += sum_j 2^(s_j*scale - z) v_j
template <int G>
__global__ void __launch_bounds__(128) attn_tile_kernel(const __nv_bfloat16* __restrict__ Q,
                                                        const __nv_bfloat16* __restrict__ Kmat,
                                                        const __nv_bfloat16* __restrict__ Vmat,
                                                        const int4* __restrict__ tiles,
                                                        const int32_t* __restrict__ ntiles_ptr,
                                                        const uint32_t* __restrict__ entries,
                                                        const float* __restrict__ z2, float* __restrict__ oacc,
                                                        int* __restrict__ err, TileParams p) {
    // Shared memory (72 KB): gathered Q rows [0, 32K), later the probabilities P
    // [0, 16K) and the staged output rows (two rounds of 64, [0, 33.8K)); the
    // leaf's value block [40K, 56K) and key block [56K, 72K) outlive a tile, so
    // a run of consecutive tiles of one bucket loads them once.
    extern __shared__ __align__(1024) uint8_t dsm[];
    uint8_t* sA = dsm;                 // 32 KB gathered Q rows
    uint8_t* sP = dsm;                 // 16 KB probabilities (K-major), over Q once S has landed
    uint8_t* sV = dsm + 40960;         // 16 KB value block (MN-major)
    uint8_t* sK = dsm + 57344;         // 16 KB key block
    __shared__ TileRows tr;
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5;
    // S (64 columns) and O (128) share one 128-column allocation: S is read
    // into registers before the PV product starts, and O starts fresh per tile
    if (warp == 0) tc::tmem_alloc(&tmem_base, 128);
    if (tid == 0) {
        tc::mbar_init(&mbar, 1);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_s = tmem_base, tmem_o = tmem_base;
    const uint32_t a_smem = tc::smem_u32(sA), k_smem = tc::smem_u32(sK), v_smem = tc::smem_u32(sV),
                   p_smem = tc::smem_u32(sP);
    const int ntiles = min(*ntiles_ptr, p.max_tiles);
    // runs of kRun consecutive tiles (mostly one bucket: one leaf) per CTA
    constexpr int kRun = 8;
    auto tile_of = [&](int it) { return ((it / kRun) * (int)gridDim.x + (int)blockIdx.x) * kRun + it % kRun; };
    int2 kv_loaded = make_int2(-1, -1);  // (b * Hkv + kvh, leaf) of the blocks in sK / sV
    uint32_t phase = 0;
    bool ok;
    for (int it = 0, tile = tile_of(0); tile < ntiles; tile = tile_of(++it)) {
        const int4 td = tiles[tile];
        const int64_t bh = td.x, leaf = td.y;
        const int64_t b = bh / p.Hkv;
        const int kvh = (int)(bh - b * p.Hkv);
        if (!tile_sane(td, (int64_t)p.B * p.Hkv, p.M1, 128 / G)) {  // self-check: never expected
            if (tid == 0) atomicCAS(err, 0, 12);
            continue;
        }
        tile_rows<G>(tr, entries, td.z, td.w, p.N, err, tid);
        __syncthreads();
        gather_q<G>(a_smem, tr, Q, b, kvh, p.Hq, p.N, tid);
        if (kv_loaded.x != td.x || kv_loaded.y != td.y) {
            load_kblock(k_smem, Kmat + bh * p.N * kD, leaf * kBlk, p.N, tid);
            load_vblock(v_smem, Vmat + bh * p.N * kD, leaf * kBlk, p.N, tid);
            kv_loaded = make_int2(td.x, td.y);
        }
        tc::cp_async_commit();
        tc::cp_async_wait_all();
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::tc_fence_after();
            issue_qk(tmem_s, a_smem, k_smem);
            tc::mma_commit(&mbar);
        }
        ok = __syncthreads_and(tc::mbar_wait(&mbar, phase, err, 2)) != 0;
        phase ^= 1;
        if (!ok) break;
        tc::tc_fence_after();
        // P = 2^(S*scale - z), masked, packed to bf16 in the K-major P tile (over the Q rows, which the MMA has read)
        {
            float v[64];
            const uint32_t taddr = tmem_s + ((uint32_t)(warp * 32) << 16);
            tc::tmem_ld32(taddr, v);
            tc::tmem_ld32(taddr + 32, v + 32);
            tc::tmem_ld_wait();
            const int t = tr.t[tid];
            int nvalid = 0;
            float z = 0.f;
            if (t >= 0) {
                nvalid = visible_keys(leaf, t, p.N, p.causal);
                z = z2[(bh * p.N + t) * G + (tid % G)];
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t w4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j = c * 8 + q * 2;
                    const float p0 = j < nvalid ? ex2_approx(v[j] * p.qscale - z) : 0.f;
                    const float p1 = j + 1 < nvalid ? ex2_approx(v[j + 1] * p.qscale - z) : 0.f;
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                    w4[q] = *reinterpret_cast<uint32_t*>(&h2);
                }
                *reinterpret_cast<uint4*>(sP + tc::kmajor64_off(tid, c)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc::tc_fence_after();
            constexpr uint32_t idesc = tc::idesc_bf16(128, 128, 1);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                tc::mma_bf16(tmem_o, tc::smem_desc(p_smem + k * 256, 128, 1024),
                             tc::smem_desc(v_smem + k * 256, 128, 1024), idesc, k > 0);
            tc::mma_commit(&mbar);
        }
        ok = __syncthreads_and(tc::mbar_wait(&mbar, phase, err, 3)) != 0;
        phase ^= 1;
        if (!ok) break;
        tc::tc_fence_after();
        {
            // Each output row is staged in shared memory (over Q and P, both
            // read by now) and added to the accumulator with one 512-byte bulk
            // reduction: whole-line operations at L2 instead of 32 scattered
            // 16-byte ones. Two rounds of 64 rows leave the K and V blocks intact.
            const int t = tr.t[tid];
            const uint32_t taddr = tmem_o + ((uint32_t)(warp * 32) << 16);
#pragma unroll
            for (int round = 0; round < 2; ++round) {
                const bool mine = (tid >> 6) == round;
                uint8_t* srow = dsm + (tid & 63) * kORowStride;
                if (mine) {
#pragma unroll
                    for (int part = 0; part < 4; ++part) {
                        float v[32];
                        tc::tmem_ld32(taddr + part * 32, v);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 32; q += 4)
                            *reinterpret_cast<float4*>(srow + (part * 32 + q) * 4) =
                                make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
                    }
                    if (t >= 0) {
                        tc::fence_async_smem();
                        tc::bulk_reduce_add_f32(oacc + (((b * p.Hq + (int64_t)kvh * G + (tid % G)) * p.N) + t) * kD,
                                                tc::smem_u32(srow), kD * 4);
                        tc::bulk_commit();
                    }
                }
                tc::bulk_wait_read_all();  // the staged rows have been read: the buffer may be refilled
                __syncthreads();
            }
        }
        tc::tc_fence_before();
    }
    tc::bulk_wait_all();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, 128);
    }
}

// z2[unit * G + h] = log2 sum of 2^lse over the listed leaves that are not
// forced leaves of the query (slot = index in idx); forced_tile_kernel adds the rest.
template <int G>
__global__ void z2_kernel(const int32_t* __restrict__ idx, const float* __restrict__ lse, float* __restrict__ z2,
                          int64_t units, int K, int N, int C, int causal, int forced_mask) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= units * G) return;
    const int64_t unit = i / G;
    const int h = (int)(i - unit * G);
    const Forced F(unit % N, C, causal, forced_mask);
    float m = -INFINITY;
    for (int k = 0; k < K; ++k) {
        const int leaf = idx[unit * K + k];
        if (leaf >= 0 && !F.has(leaf, 1)) m = fmaxf(m, lse[(unit * kSlots + k) * G + h]);
    }
    float e = 0.f;
    for (int k = 0; k < K; ++k) {
        const int leaf = idx[unit * K + k];
        if (leaf >= 0 && !F.has(leaf, 1)) e += exp2f(lse[(unit * kSlots + k) * G + h] - m);
    }
    z2[i] = m + log2f(e);
}

// ---------------------------------------------------- forced leaves, dense ----

// The forced leaves of a query (first, previous, current; close reading §5.3)
// are the same for every query of a leaf block, so they are attended densely:
// a tile holds 128/G consecutive positions (x G heads) of one (b, kv-head),
// whose forced leaves are at most 4 distinct leaves U. Pass 1 runs S = Q K_u^T
// per leaf u (tcgen05, TMEM) and folds each row's masked LSE into the
// normaliser Z = log2(2^z2 + sum_u 2^LSE_u) (z2 holds the non-forced part on
// entry, Z on exit). Pass 2 recomputes S, forms P = 2^(S*scale - Z) and
// accumulates O = sum_u P_u V_u on the tensor cores; the rows are stored into
// the fp32 accumulator as its initial value (the non-forced tiles add to it).
// A leaf counts for a row only if it is a forced leaf of that query and is
// listed in the query's idx row.
struct ForcedParams {
    int B, Hq, Hkv, N, causal, forced_mask, K;
    float qscale;
    int64_t tiles_per_head;
};

__device__ __forceinline__ int forced_union(int64_t t0, int64_t t1, int causal, int mask, int* U) {
    int n = 0;
    auto add = [&](int v) {
        for (int i = 0; i < n; ++i)
            if (U[i] == v) return;
        U[n++] = v;
    };
    for (int64_t c = t0 / kBlk; c <= (t1 - 1) / kBlk; ++c) {
        if (mask & 1) add(0);
        if ((mask & 2) && c >= 1) add((int)c - 1);
        if ((mask & 4) || causal) add((int)c);
    }
    return n;
}

template <int G>
__global__ void __launch_bounds__(128) forced_tile_kernel(const __nv_bfloat16* __restrict__ Q,
                                                          const __nv_bfloat16* __restrict__ Kmat,
                                                          const __nv_bfloat16* __restrict__ Vmat,
                                                          const int32_t* __restrict__ idx, float* __restrict__ z2,
                                                          float* __restrict__ oacc, int* __restrict__ err,
                                                          ForcedParams p) {
    constexpr int QPT = 128 / G;  // query positions per tile
    extern __shared__ __align__(1024) uint8_t dsm[];
    uint8_t* sA = dsm;          // 32 KB query rows
    uint8_t* sK = dsm + 32768;  // 16 KB key block
    uint8_t* sV = dsm + 49152;  // 16 KB value block (MN-major)
    uint8_t* sP = sK;           // 16 KB probabilities, over the keys once S has landed
    __shared__ TileRows tr;
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5;
    if (warp == 0) tc::tmem_alloc(&tmem_base, 256);
    if (tid == 0) {
        tc::mbar_init(&mbar, 1);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_s = tmem_base, tmem_o = tmem_base + 128;
    const uint32_t a_smem = tc::smem_u32(sA), k_smem = tc::smem_u32(sK), v_smem = tc::smem_u32(sV),
                   p_smem = tc::smem_u32(sP);
    const int64_t ntiles = (int64_t)p.B * p.Hkv * p.tiles_per_head;
    uint32_t phase = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int64_t bh = tile / p.tiles_per_head;
        const int64_t t0 = (tile - bh * p.tiles_per_head) * QPT;
        const int64_t t1 = min(t0 + QPT, (int64_t)p.N);
        const int64_t b = bh / p.Hkv;
        const int kvh = (int)(bh - b * p.Hkv);
        const int64_t t = t0 + tid / G;
        const bool row_ok = t < t1;
        tr.t[tid] = row_ok ? (int)t : -1;
        tr.slot[tid] = 0;
        int U[4];
        const int nu = forced_union(t0, t1, p.causal, p.forced_mask, U);
        // which of U count for this row: forced for t and listed in idx[t]
        unsigned member = 0;
        if (row_ok) {
            const Forced F(t, kBlk, p.causal, p.forced_mask);
            const int32_t* row = idx + (bh * p.N + t) * p.K;
            for (int k = 0; k < p.K; ++k) {
                const int leaf = row[k];
                for (int i = 0; i < nu; ++i)
                    if (leaf == U[i] && F.has(leaf, 1)) member |= 1u << i;
            }
        }
        __syncthreads();
        gather_q<G>(a_smem, tr, Q, b, kvh, p.Hq, p.N, tid);
        // pass 1: per-row LSE of every member leaf -> Z
        float lse_f = -INFINITY;
        for (int i = 0; i < nu && ok; ++i) {
            load_kblock(k_smem, Kmat + bh * p.N * kD, (int64_t)U[i] * kBlk, p.N, tid);
            tc::cp_async_commit();
            tc::cp_async_wait_all();
            tc::fence_async_smem();
            __syncthreads();
            if (tid == 0) {
                tc::tc_fence_after();
                issue_qk(tmem_s, a_smem, k_smem);
                tc::mma_commit(&mbar);
            }
            ok = __syncthreads_and(tc::mbar_wait(&mbar, phase, err, 4)) != 0;
            phase ^= 1;
            if (!ok) break;
            tc::tc_fence_after();
            float v[64];
            const uint32_t taddr = tmem_s + ((uint32_t)(warp * 32) << 16);
            tc::tmem_ld32(taddr, v);
            tc::tmem_ld32(taddr + 32, v + 32);
            tc::tmem_ld_wait();
            if ((member >> i) & 1u) {
                const int nvalid = visible_keys(U[i], t, p.N, p.causal);
                float m = -INFINITY;
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (j < nvalid) m = fmaxf(m, v[j] * p.qscale);
                float sum = 0.f;
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (j < nvalid) sum += ex2_approx(v[j] * p.qscale - m);
                lse_f = logaddexp2f(lse_f, m + lg2_approx(sum));
            }
            tc::tc_fence_before();
            __syncthreads();
        }
        if (!ok) break;
        float z = -INFINITY;
        if (row_ok) {
            float* zp = z2 + (bh * p.N + t) * G + (tid % G);
            z = logaddexp2f(*zp, lse_f);
            *zp = z;
        }
        // pass 2: O = sum_u P_u V_u
        for (int i = 0; i < nu && ok; ++i) {
            load_kblock(k_smem, Kmat + bh * p.N * kD, (int64_t)U[i] * kBlk, p.N, tid);
            load_vblock(v_smem, Vmat + bh * p.N * kD, (int64_t)U[i] * kBlk, p.N, tid);
            tc::cp_async_commit();
            tc::cp_async_wait_all();
            tc::fence_async_smem();
            __syncthreads();
            if (tid == 0) {
                tc::tc_fence_after();
                issue_qk(tmem_s, a_smem, k_smem);
                tc::mma_commit(&mbar);
            }
            ok = __syncthreads_and(tc::mbar_wait(&mbar, phase, err, 5)) != 0;
            phase ^= 1;
            if (!ok) break;
            tc::tc_fence_after();
            {
                float v[64];
                const uint32_t taddr = tmem_s + ((uint32_t)(warp * 32) << 16);
                tc::tmem_ld32(taddr, v);
                tc::tmem_ld32(taddr + 32, v + 32);
                tc::tmem_ld_wait();
                const int nvalid = ((member >> i) & 1u) ? visible_keys(U[i], t, p.N, p.causal) : 0;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t w4[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int j = c * 8 + q * 2;
                        const float p0 = j < nvalid ? ex2_approx(v[j] * p.qscale - z) : 0.f;
                        const float p1 = j + 1 < nvalid ? ex2_approx(v[j + 1] * p.qscale - z) : 0.f;
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                        w4[q] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    *reinterpret_cast<uint4*>(sP + tc::kmajor64_off(tid, c)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc::tc_fence_after();
                constexpr uint32_t idesc = tc::idesc_bf16(128, 128, 1);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    tc::mma_bf16(tmem_o, tc::smem_desc(p_smem + k * 256, 128, 1024),
                                 tc::smem_desc(v_smem + k * 256, 128, 1024), idesc, (i > 0 || k > 0) ? 1u : 0u);
                tc::mma_commit(&mbar);
            }
            ok = __syncthreads_and(tc::mbar_wait(&mbar, phase, err, 6)) != 0;
            phase ^= 1;
            if (!ok) break;
            tc::tc_fence_after();
        }
        if (!ok) break;
        // initial value of the output accumulator for these rows: row tid is
        // staged in the tile's (now free) shared memory and stored with one
        // 512-byte bulk copy
        {
            const uint32_t taddr = tmem_o + ((uint32_t)(warp * 32) << 16);
            uint8_t* srow = dsm + tid * kORowStride;
#pragma unroll
            for (int part = 0; part < 4; ++part) {
                float v[32];
                if (nu > 0) {
                    tc::tmem_ld32(taddr + part * 32, v);
                    tc::tmem_ld_wait();
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] = 0.f;
                }
#pragma unroll
                for (int q = 0; q < 32; q += 4)
                    *reinterpret_cast<float4*>(srow + (part * 32 + q) * 4) = make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
            }
            if (row_ok) {
                tc::fence_async_smem();
                tc::bulk_store(oacc + (((b * p.Hq + (int64_t)kvh * G + (tid % G)) * p.N) + t) * kD, tc::smem_u32(srow),
                               kD * 4);
                tc::bulk_commit();
            }
        }
        tc::tc_fence_before();
        tc::bulk_wait_read_all();  // the staged row has been read: the buffers may be refilled
        __syncthreads();
    }
    tc::bulk_wait_all();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, 256);
    }
}

__global__ void finalize_kernel(const float* __restrict__ oacc, __nv_bfloat16* __restrict__ O, int64_t n4) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 v = reinterpret_cast<const float4*>(oacc)[i];
        __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), c = __floats2bfloat162_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t*>(&a);
        u.y = *reinterpret_cast<uint32_t*>(&c);
        reinterpret_cast<uint2*>(O)[i] = u;
    }
}

// ---------------------------------------------------------- backward tiles ----

// Backward of the attention with the selection fixed (close reading §02 Eq.(2)
// differentiated; §5.3: gradients reach only the selected entries), key-major
// on the tensor cores. Per (query row i, selected key j) with the normaliser
// L_i (log2 units) and D_i = dO_i . o_i (from the statistics pass below, or
// from a saved forward):
//   p = 2^(s*scale - L),  dp = dO_i . v_j,  ds = p (dp - D),
//   dV_j += p dO_i,  dK_j += ds q_i / sqrt(d),  dQ_i += ds k_j / sqrt(d).
// Rows are grouped by leaf: bucket (b, kv-head, leaf) holds first the leaf's
// forced section -- the contiguous range of positions for which it is a forced
// leaf (rows whose idx does not list it contribute nothing) -- and then the
// positions that list it freely (the forward's grouping, reused). One tile is
// 128/G positions x G heads of one bucket. Per tile: S = Q K^T and
// dP = dO V^T (M = 128 rows, N = 64 keys), P and dS packed to bf16 in shared
// memory, then dV^T += dO^T P and dK^T += Q^T dS (M = 128 dims, N = 64 keys,
// both operands MN-major views of the row-major tiles) accumulate in TMEM
// across the consecutive tiles of a leaf, and dQ = dS K (K read as an MN-major
// view of its K-major tile) is added to its rows by bulk reductions. The CTAs
// take chunks of consecutive tiles round-robin and add their dK / dV
// accumulators to global memory whenever the leaf changes.

// positions [lo, hi) for which `leaf` is a forced leaf (first: every position;
// current: its own block; previous: the next block), clipped to N
__device__ __forceinline__ void forced_range(int64_t leaf, int N, int causal, int mask, int64_t& lo, int64_t& hi) {
    lo = hi = 0;
    if (leaf == 0 && (mask & 1)) {
        hi = N;
        return;
    }
    const bool cur = (mask & 4) || causal, prev = (mask & 2) != 0;
    const int64_t a = leaf * kBlk;
    if (cur) {
        lo = a;
        hi = a + kBlk;
    }
    if (prev) {
        if (!cur) lo = a + kBlk;
        hi = a + 2 * kBlk;
    }
    lo = min(lo, (int64_t)N);
    hi = min(hi, (int64_t)N);
}

// tiles per bucket = ceil((forced section + free entries) / per_tile): totals per scan block
__global__ void __launch_bounds__(kScanBlock) bwd_total_kernel(const int32_t* __restrict__ counts, int64_t nbuckets,
                                                              int64_t M1, int per_tile, int N, int causal, int mask,
                                                              longlong2* __restrict__ bsum, int* __restrict__ err) {
    __shared__ long long s_a[32], s_b[32];
    const int64_t i = (int64_t)blockIdx.x * kScanBlock + threadIdx.x;
    long long c = bucket_count(counts, i, nbuckets, N, err);
    if (i < nbuckets) {
        int64_t lo, hi;
        forced_range(i % M1, N, causal, mask, lo, hi);
        c += hi - lo;
    }
    long long t = (c + per_tile - 1) / per_tile, z = 0;
    block_scan2(t, z, s_a, s_b);
    if (threadIdx.x == kScanBlock - 1) bsum[blockIdx.x] = make_longlong2(t, 0);
}

// tile list (b*Hkv + kvh, leaf, first row of the bucket, rows)
__global__ void __launch_bounds__(kScanBlock) bwd_place_kernel(const int32_t* __restrict__ counts, int64_t nbuckets,
                                                              int64_t M1, int per_tile, int N, int causal, int mask,
                                                              const longlong2* __restrict__ bsum,
                                                              int4* __restrict__ tiles, int32_t* __restrict__ ntiles) {
    __shared__ long long s_a[32], s_b[32];
    __shared__ long long s_pre;
    long long pt = 0;
    for (int j = threadIdx.x; j < (int)blockIdx.x; j += kScanBlock) pt += bsum[j].x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pt += __shfl_xor_sync(kFull, pt, o);
    if (threadIdx.x == 0) s_pre = 0;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) atomicAdd(reinterpret_cast<unsigned long long*>(&s_pre), (unsigned long long)pt);
    __syncthreads();
    const int64_t i = (int64_t)blockIdx.x * kScanBlock + threadIdx.x;
    long long c = bucket_count(counts, i, nbuckets, N, nullptr);
    if (i < nbuckets) {
        int64_t lo, hi;
        forced_range(i % M1, N, causal, mask, lo, hi);
        c += hi - lo;
    }
    const long long nt = (c + per_tile - 1) / per_tile;
    long long t = nt, z = 0;
    block_scan2(t, z, s_a, s_b);
    const long long bt = s_pre + t - nt;  // exclusive
    if (i < nbuckets)
        for (long long j = 0; j < nt; ++j)
            tiles[bt + j] = make_int4((int)(i / M1), (int)(i % M1), (int)(j * per_tile),
                                      (int)min((long long)per_tile, c - j * per_tile));
    if (blockIdx.x == gridDim.x - 1 && threadIdx.x == kScanBlock - 1) *ntiles = (int32_t)(s_pre + t);
}

// D = dO . O per (query, head), O from the fp32 accumulator a saved forward
// left in the workspace; one warp per row of [B, Hq, N], written as [B, Hkv, N, G]
template <int G>
__global__ void bwd_delta_kernel(const __nv_bfloat16* __restrict__ dO, const float* __restrict__ oacc,
                                 float* __restrict__ Dr, int64_t rows, int N, int Hq) {
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    float a[4], o[4];
    Ld<__nv_bfloat16, 4>::run(dO + r * kD + lane * 4, a);
    const float4 v = *reinterpret_cast<const float4*>(oacc + r * kD + lane * 4);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) s = fmaf(a[e], o[e], s);
#pragma unroll
    for (int w = 16; w > 0; w >>= 1) s += __shfl_xor_sync(kFull, s, w);
    if (lane == 0) {
        const int64_t t = r % N, bq = r / N;
        const int64_t b = bq / Hq, head = bq % Hq;
        const int64_t Hkv = Hq / G;
        Dr[((b * Hkv + head / G) * N + t) * G + head % G] = s;
    }
}

// instruction descriptor (kind::f16, bf16 operands, fp32 accumulator) with
// either operand MN-major
__host__ __device__ constexpr uint32_t idesc_bf16_mn(int M, int N, int a_mn_major, int b_mn_major) {
    return tc::idesc_bf16(M, N, b_mn_major) | ((uint32_t)a_mn_major << 15);
}

struct BwdParams {
    int B, Hq, Hkv, N, causal, forced_mask, K;
    int64_t M1;
    float qscale;      // log2(e) / sqrt(d)
    float inv_sqrt_d;  // 1 / sqrt(d)
    int max_tiles;
};

// gather 128 rows (head kvh*G + r%G, position rt[r]) of X into a K-major tile;
// rows with rt < 0 are zero-filled (they enter the row contractions)
template <int G>
__device__ __forceinline__ void gather_rows_zero(uint32_t smem, const int* rt, const __nv_bfloat16* X, int64_t b,
                                                 int kvh, int Hq, int N, int tid) {
    const int i = tid & 7, c = tid >> 3;  // tid in [0, 128)
#pragma unroll 4
    for (int g = 0; g < 16; ++g) {
        const int r = g * 8 + i;
        const int t = rt[r];
        if (t >= 0)
            tc::cp_async16(smem + tc::kmajor128_off(r, c),
                           X + (((b * Hq + (int64_t)kvh * G + (r % G)) * N) + t) * kD + c * 8);
        else
            tc::cp_async_zero16(smem + tc::kmajor128_off(r, c), X);
    }
}

// Softmax statistics of the backward from Q, K, V, dO and idx alone (no
// forward output needed). Per (row, listed leaf), over the leaf's visible keys
// with x = s * scale (log2 units):
//   lse = log2 sum_j 2^x_j,   dbar = sum_j 2^(x_j - lse) dp_j   (dp = dO . v),
// written per (unit, idx slot, head). bwd_combine_kernel then forms
//   L = log2 sum_l 2^lse_l   and   D = sum_l 2^(lse_l - L) dbar_l = sum_j p_j dp_j,
// which is dO . o. One tile of the backward's tile list per step: S = Q K^T and
// dP = dO V^T on the tensor cores (M = 128 rows, N = 64 keys each).
constexpr size_t kStatsSmem = 96 * 1024;  // Q, dO 32 KB each; K, V 16 KB each

template <int G>
__global__ void __launch_bounds__(128) bwd_stats_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ Kmat,
    const __nv_bfloat16* __restrict__ Vmat, const __nv_bfloat16* __restrict__ dO, const int32_t* __restrict__ idx,
    const int4* __restrict__ tiles, const int32_t* __restrict__ ntiles_ptr, const int32_t* __restrict__ offsets,
    const uint32_t* __restrict__ entries, float* __restrict__ lse_s, float* __restrict__ dbar_s,
    int* __restrict__ err, BwdParams p) {
    extern __shared__ __align__(1024) uint8_t dsm[];
    __shared__ int rt[128], rk[128];  // position and idx slot of each MMA row (rt -1: contributes nothing)
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5;
    if (warp == 0) tc::tmem_alloc(&tmem_base, 128);  // S [0, 64), dP [64, 128)
    if (tid == 0) {
        tc::mbar_init(&mbar, 1);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tm = tmem_base, taddr = tm + ((uint32_t)(warp * 32) << 16);
    const uint32_t q_smem = tc::smem_u32(dsm), o_smem = q_smem + 32768, k_smem = q_smem + 65536,
                   v_smem = q_smem + 81920;
    const int T = min(*ntiles_ptr, p.max_tiles);
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x) {
        const int4 td = tiles[tile];
        if (!tile_sane(td, (int64_t)p.B * p.Hkv, p.M1, 1 << 30) || td.w > 128 / G) {  // self-check: never expected
            if (tid == 0) atomicCAS(err, 0, 12);
            continue;
        }
        const int64_t bh = td.x, leaf = td.y;
        const int64_t b = bh / p.Hkv;
        const int kvh = (int)(bh - b * p.Hkv);
        {
            const int e = tid / G;
            int t = -1, k = -1;
            if (e < td.w) {
                const int64_t q = (int64_t)td.z + e;
                int64_t flo, fhi;
                forced_range(leaf, p.N, p.causal, p.forced_mask, flo, fhi);
                if (q < fhi - flo) {
                    const int64_t tt = flo + q;
                    const int32_t* ir = idx + (bh * p.N + tt) * p.K;
                    for (int j = p.K - 1; j >= 0; --j)
                        if (ir[j] == (int32_t)leaf) k = j;
                    if (k >= 0) t = (int)tt;
                } else {
                    const uint32_t v = entries[offsets[bh * p.M1 + leaf] + (q - (fhi - flo))];
                    if ((int)(v >> 5) < p.N && (int)(v & 31u) < p.K) {
                        t = (int)(v >> 5);
                        k = (int)(v & 31u);
                    } else {
                        atomicCAS(err, 0, 13);  // self-check: never expected
                    }
                }
            }
            rt[tid] = t;
            rk[tid] = k;
        }
        __syncthreads();
        gather_rows_zero<G>(q_smem, rt, Q, b, kvh, p.Hq, p.N, tid);
        gather_rows_zero<G>(o_smem, rt, dO, b, kvh, p.Hq, p.N, tid);
        load_kblock(k_smem, Kmat + bh * p.N * kD, leaf * kBlk, p.N, tid);
        load_kblock(v_smem, Vmat + bh * p.N * kD, leaf * kBlk, p.N, tid);
        tc::cp_async_commit();
        tc::cp_async_wait_all();
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::tc_fence_after();
            constexpr uint32_t id_s = tc::idesc_bf16(128, 64, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tm, tc::smem_desc(q_smem + k * 256, 128, 2048), tc::smem_desc(k_smem + k * 256, 128, 2048),
                             id_s, k > 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tm + 64, tc::smem_desc(o_smem + k * 256, 128, 2048),
                             tc::smem_desc(v_smem + k * 256, 128, 2048), id_s, k > 0);
            tc::mma_commit(&mbar);
        }
        ok = __syncthreads_and(tc::mbar_wait(&mbar, phase, err, 9)) != 0;
        phase ^= 1;
        if (!ok) break;
        tc::tc_fence_after();
        {
            const int t = rt[tid];
            const int nvalid = t >= 0 ? visible_keys(leaf, t, p.N, p.causal) : 0;
            float m = -INFINITY, l = 0.f, dd = 0.f;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float sv[32], dp[32];
                tc::tmem_ld32(taddr + c * 32, sv);
                tc::tmem_ld32(taddr + 64 + c * 32, dp);
                tc::tmem_ld_wait();
                float mc = -INFINITY;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (c * 32 + j < nvalid) mc = fmaxf(mc, sv[j] * p.qscale);
                const float mn = fmaxf(m, mc);
                if (mn != -INFINITY) {
                    const float sc = ex2_approx(m - mn);
                    l *= sc;
                    dd *= sc;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c * 32 + j < nvalid) {
                            const float w = ex2_approx(sv[j] * p.qscale - mn);
                            l += w;
                            dd = fmaf(w, dp[j], dd);
                        }
                    m = mn;
                }
            }
            if (t >= 0) {
                const int64_t o = ((bh * p.N + t) * p.K + rk[tid]) * G + (tid % G);
                lse_s[o] = l > 0.f ? m + lg2_approx(l) : -INFINITY;
                dbar_s[o] = l > 0.f ? dd / l : 0.f;
            }
        }
        tc::tc_fence_before();
        __syncthreads();
    }
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, 128);
    }
}

// L (log2) and D per (unit, head) from the per-leaf statistics of the listed leaves
template <int G>
__global__ void bwd_combine_kernel(const int32_t* __restrict__ idx, const float* __restrict__ lse_s,
                                   const float* __restrict__ dbar_s, float* __restrict__ z2, float* __restrict__ Dr,
                                   int64_t units, int K) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= units * G) return;
    const int64_t unit = i / G;
    const int h = (int)(i - unit * G);
    float m = -INFINITY;
    for (int k = 0; k < K; ++k)
        if (idx[unit * K + k] >= 0) m = fmaxf(m, lse_s[(unit * K + k) * G + h]);
    float l = 0.f, dd = 0.f;
    if (m != -INFINITY)
        for (int k = 0; k < K; ++k)
            if (idx[unit * K + k] >= 0) {
                const float w = exp2f(lse_s[(unit * K + k) * G + h] - m);
                l += w;
                dd = fmaf(w, dbar_s[(unit * K + k) * G + h], dd);
            }
    z2[i] = l > 0.f ? m + log2f(l) : -INFINITY;
    Dr[i] = l > 0.f ? dd / l : 0.f;
}

// Shared memory: K [0, 16K), V [16K, 32K), buffer set 0 = Q0 [32K, 64K) and
// dO0 [64K, 96K), P [96K, 112K), dS [112K, 128K), buffer set 1 = Q1 [128K, 160K)
// and dO1 [160K, 192K). The next tile's rows are gathered into the other set
// while this tile computes. Staged fp32 rows (this tile's dQ rows, or the dV /
// dK rows of a flush; 128 x kORowStride bytes) go to set 0's region
// [32K, 32K + 66K) or set 1's region [96K, 96K + 66K): each covers its own Q,
// dO and parts of P / dS, never the other set's Q and dO.
constexpr size_t kBwdSmem = 192 * 1024;
constexpr int kBwdChunk = 8;  // consecutive tiles per CTA before it moves on by the grid size
__host__ __device__ constexpr uint32_t bwd_q(int st) { return st ? 131072u : 32768u; }
__host__ __device__ constexpr uint32_t bwd_o(int st) { return st ? 163840u : 65536u; }
__host__ __device__ constexpr uint32_t bwd_stage(int st) { return st ? 98304u : 32768u; }
constexpr uint32_t kBwdP = 98304, kBwdS = 114688;
static_assert(bwd_stage(0) + 128 * kORowStride <= bwd_q(1), "set 0 staging stays clear of set 1");
static_assert(bwd_stage(1) >= bwd_o(0) + 32768 && bwd_stage(1) + 128 * kORowStride <= kBwdSmem,
              "set 1 staging stays clear of set 0");

template <int G>
__global__ void __launch_bounds__(256, 1) bwd_tile_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ Kmat,
    const __nv_bfloat16* __restrict__ Vmat, const __nv_bfloat16* __restrict__ dO, const int32_t* __restrict__ idx,
    const int4* __restrict__ tiles, const int32_t* __restrict__ ntiles_ptr, const int32_t* __restrict__ offsets,
    const uint32_t* __restrict__ entries, const float* __restrict__ z2, const float* __restrict__ Dr,
    float* __restrict__ dQ, float* __restrict__ dK, float* __restrict__ dV, int* __restrict__ err, BwdParams p) {
    extern __shared__ __align__(1024) uint8_t dsm[];
    __shared__ int rt[2][128];               // per buffer set: position of each MMA row (-1: contributes nothing)
    __shared__ float rz[2][128], rd[2][128];  // its normaliser (log2) and D
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = (warp & 3) * 32 + lane;  // TMEM lane of this thread
    const int half = warp >> 2;              // which half of the columns it handles
    // TMEM columns: [0, 64) S and [64, 128) dP, then [0, 128) dQ; [128, 192) dV^T; [192, 256) dK^T
    if (warp == 0) tc::tmem_alloc(&tmem_base, 256);
    if (tid == 0) {
        tc::mbar_init(&mbar, 1);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tm = tmem_base, lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t base = tc::smem_u32(dsm), k_smem = base, v_smem = base + 16384, p_smem = base + kBwdP,
                   s_smem = base + kBwdS;
    uint8_t* const sP = dsm + kBwdP;
    uint8_t* const sS = dsm + kBwdS;
    const int64_t T = min((int64_t)*ntiles_ptr, (int64_t)p.max_tiles);
    // the k-th tile of this CTA: chunks of kBwdChunk consecutive tiles dealt
    // round-robin, so that the CTAs work through the list together and the
    // dQ rows they update stay within a window that L2 holds
    auto tile_at = [&](int64_t k) -> int64_t {
        return ((int64_t)blockIdx.x + (k / kBwdChunk) * gridDim.x) * kBwdChunk + k % kBwdChunk;
    };
    const int64_t bhs = (int64_t)p.B * p.Hkv;

    // the tile descriptor, or (-1, -1, 0, 0) for a malformed one (self-check: never expected)
    auto read_tile = [&](int64_t tile) {
        const int4 td = tiles[tile];
        if (tile_sane(td, bhs, p.M1, 1 << 30) && td.w <= 128 / G) return td;
        if (tid == 0) atomicCAS(err, 0, 12);
        return make_int4(-1, -1, 0, 0);
    };
    // rows of a tile into set `st`: forced section first, then the free entries
    auto setup_rows = [&](const int4& td, int st) {
        if (tid >= 128) return;
        const int64_t bh = td.x, leaf = td.y;
        const int e = tid / G;
        int t = -1;
        if (e < td.w) {
            const int64_t q = (int64_t)td.z + e;
            int64_t flo, fhi;
            forced_range(leaf, p.N, p.causal, p.forced_mask, flo, fhi);
            if (q < fhi - flo) {
                const int64_t tt = flo + q;
                const int32_t* ir = idx + (bh * p.N + tt) * p.K;
                bool member = false;
                for (int k = 0; k < p.K; ++k) member |= ir[k] == (int32_t)leaf;
                if (member) t = (int)tt;
            } else {
                const uint32_t v = entries[offsets[bh * p.M1 + leaf] + (q - (fhi - flo))];
                if ((int)(v >> 5) < p.N) t = (int)(v >> 5);
                else atomicCAS(err, 0, 13);  // self-check: never expected
            }
        }
        rt[st][tid] = t;
        float z = 0.f, dd = 0.f;
        if (t >= 0) {
            const int64_t u = (bh * p.N + t) * G + (tid % G);
            z = z2[u];
            dd = Dr[u];
        }
        rz[st][tid] = z;
        rd[st][tid] = dd;
    };
    // gather the tile's Q and dO rows into set `st` (rt[st] must be visible to all threads)
    auto gather = [&](const int4& td, int st) {
        const int64_t b = td.x >= 0 ? td.x / p.Hkv : 0;
        const int kvh = td.x >= 0 ? (int)(td.x - b * p.Hkv) : 0;
        if (tid < 128) gather_rows_zero<G>(base + bwd_q(st), rt[st], Q, b, kvh, p.Hq, p.N, tid);
        else gather_rows_zero<G>(base + bwd_o(st), rt[st], dO, b, kvh, p.Hq, p.N, tid - 128);
    };
    auto load_kv = [&](const int4& td) {
        const int64_t bh = td.x >= 0 ? td.x : 0, leaf = td.y >= 0 ? td.y : 0;
        if (tid < 128) load_kblock(k_smem, Kmat + bh * p.N * kD, leaf * kBlk, p.N, tid);
        else load_kblock(v_smem, Vmat + bh * p.N * kD, leaf * kBlk, p.N, tid - 128);
    };
    // add the leaf's dV / dK accumulators (all MMAs into them have completed) to
    // global memory through the staging region of set `st`
    auto flush = [&](int64_t bh, int64_t leaf, int st) {
        tc::tc_fence_after();
        uint8_t* sbase = dsm + bwd_stage(st) + half * 64 * kORowStride;  // half 0: dV rows, half 1: dK rows
        const float sc = half ? p.inv_sqrt_d : 1.f;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            float v[32];
            tc::tmem_ld32(tm + lane_off + 128 + half * 64 + part * 32, v);
            tc::tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q)
                *reinterpret_cast<float*>(sbase + (part * 32 + q) * kORowStride + row * 4) = v[q] * sc;
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (tid < 128 && bh >= 0) {
            const int key = tid & 63, h = tid >> 6;
            const int64_t krow = leaf * kBlk + key;
            if (krow < p.N) {
                tc::bulk_reduce_add_f32((h ? dK : dV) + (bh * p.N + krow) * kD,
                                        tc::smem_u32(dsm + bwd_stage(st) + (h * 64 + key) * kORowStride), kD * 4);
                tc::bulk_commit();
            }
        }
        tc::bulk_wait_read_all();
        __syncthreads();
    };

    bool have_acc = false, ok = true;
    uint32_t phase = 0;
    int4 td = make_int4(-1, -1, 0, 0);
    int64_t cur_bh = -1, cur_leaf = -1;  // the leaf whose dV / dK are in TMEM
    int cur_st = 0;                      // the buffer set of the last tile processed
    if (tile_at(0) < T) {
        td = read_tile(tile_at(0));
        setup_rows(td, 0);
        __syncthreads();
        load_kv(td);
        gather(td, 0);
        tc::cp_async_commit();
    }
    for (int64_t k = 0; tile_at(k) < T; ++k) {
        const int st = (int)(k & 1);
        const int64_t bh = td.x, leaf = td.y;
        cur_bh = bh;
        cur_leaf = leaf;
        cur_st = st;
        const int64_t b = bh >= 0 ? bh / p.Hkv : 0;
        const int kvh = bh >= 0 ? (int)(bh - b * p.Hkv) : 0;
        const int64_t next = tile_at(k + 1);
        const bool has_next = next < T;
        const int4 tdn = has_next ? read_tile(next) : make_int4(-1, -1, 0, 0);
        // this tile's rows (and, after a leaf change, its K / V) have landed
        tc::cp_async_wait_all();
        tc::fence_async_smem();
        __syncthreads();
        const uint32_t q_smem = base + bwd_q(st), o_smem = base + bwd_o(st);
        if (tid == 0) {
            tc::tc_fence_after();
            constexpr uint32_t id_s = tc::idesc_bf16(128, 64, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tm, tc::smem_desc(q_smem + k * 256, 128, 2048), tc::smem_desc(k_smem + k * 256, 128, 2048),
                             id_s, k > 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tm + 64, tc::smem_desc(o_smem + k * 256, 128, 2048),
                             tc::smem_desc(v_smem + k * 256, 128, 2048), id_s, k > 0);
            tc::mma_commit(&mbar);
        }
        // the next tile's rows, while S and dP are computed
        if (has_next) setup_rows(tdn, st ^ 1);
        ok = __syncthreads_and(tc::mbar_wait(&mbar, phase, err, 7)) != 0;
        phase ^= 1;
        if (!ok) break;
        tc::tc_fence_after();
        // P = 2^(s*scale - L) over the visible keys, dS = P (dP - D), both to bf16
        {
            float sv[32], dp[32];
            tc::tmem_ld32(tm + lane_off + half * 32, sv);
            tc::tmem_ld32(tm + lane_off + 64 + half * 32, dp);
            tc::tmem_ld_wait();
            const int t = rt[st][row];
            const int nvalid = t >= 0 ? visible_keys(leaf, t, p.N, p.causal) : 0;
            const float z = rz[st][row], dd = rd[st][row];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t wp[4], ws[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = c * 8 + q * 2, j = half * 32 + i;
                    const float p0 = j < nvalid ? ex2_approx(sv[i] * p.qscale - z) : 0.f;
                    const float p1 = j + 1 < nvalid ? ex2_approx(sv[i + 1] * p.qscale - z) : 0.f;
                    __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
                    __nv_bfloat162 hs = __floats2bfloat162_rn(p0 * (dp[i] - dd), p1 * (dp[i + 1] - dd));
                    wp[q] = *reinterpret_cast<uint32_t*>(&hp);
                    ws[q] = *reinterpret_cast<uint32_t*>(&hs);
                }
                const uint32_t off = tc::kmajor64_off(row, half * 4 + c);
                *reinterpret_cast<uint4*>(sP + off) = make_uint4(wp[0], wp[1], wp[2], wp[3]);
                *reinterpret_cast<uint4*>(sS + off) = make_uint4(ws[0], ws[1], ws[2], ws[3]);
            }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc::tc_fence_after();
            // dV^T += dO^T P and dK^T += Q^T dS: M = 128 dims, N = 64 keys, K = 128 rows (16 per step)
            constexpr uint32_t id_kv = idesc_bf16_mn(128, 64, 1, 1);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tm + 128, tc::smem_desc(o_smem + k * 4096, 2048, 128),
                             tc::smem_desc(p_smem + k * 2048, 1024, 128), id_kv, (have_acc || k > 0) ? 1u : 0u);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tm + 192, tc::smem_desc(q_smem + k * 4096, 2048, 128),
                             tc::smem_desc(s_smem + k * 2048, 1024, 128), id_kv, (have_acc || k > 0) ? 1u : 0u);
            // dQ = dS K: M = 128 rows, N = 128 dims, K = 64 keys (16 per step)
            constexpr uint32_t id_q = tc::idesc_bf16(128, 128, 1);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                tc::mma_bf16(tm, tc::smem_desc(s_smem + k * 256, 128, 1024),
                             tc::smem_desc(k_smem + k * 4096, 2048, 128), id_q, k > 0);
            tc::mma_commit(&mbar);
        }
        // the next tile's Q and dO rows into the other set, while these MMAs run
        if (has_next) {
            gather(tdn, st ^ 1);
            tc::cp_async_commit();
        }
        ok = __syncthreads_and(tc::mbar_wait(&mbar, phase, err, 8)) != 0;
        phase ^= 1;
        if (!ok) break;
        have_acc = true;
        tc::tc_fence_after();
        // dQ rows: staged in this set's region and added with one 512-byte bulk reduction each
        {
            uint8_t* srow = dsm + bwd_stage(st) + row * kORowStride;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float v[32];
                const int col = half * 64 + part * 32;
                tc::tmem_ld32(tm + lane_off + col, v);
                tc::tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 32; q += 4)
                    *reinterpret_cast<float4*>(srow + (col + q) * 4) =
                        make_float4(v[q] * p.inv_sqrt_d, v[q + 1] * p.inv_sqrt_d, v[q + 2] * p.inv_sqrt_d,
                                    v[q + 3] * p.inv_sqrt_d);
            }
            tc::fence_async_smem();
        }
        tc::tc_fence_before();
        __syncthreads();
        if (tid < 128 && rt[st][tid] >= 0) {
            tc::bulk_reduce_add_f32(dQ + (((b * p.Hq + (int64_t)kvh * G + (tid % G)) * p.N) + rt[st][tid]) * kD,
                                    tc::smem_u32(dsm + bwd_stage(st) + tid * kORowStride), kD * 4);
            tc::bulk_commit();
        }
        tc::bulk_wait_read_all();  // the staged rows have been read: the region may be reused
        __syncthreads();
        // a new leaf next: add this leaf's dV / dK, then load the next K / V
        if (has_next && (tdn.x != bh || tdn.y != leaf)) {
            flush(bh, leaf, st);
            have_acc = false;
            load_kv(tdn);
            tc::cp_async_commit();
        }
        td = tdn;
    }
    if (ok && have_acc) flush(cur_bh, cur_leaf, cur_st);
    tc::cp_async_wait_all();
    tc::bulk_wait_all();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, 256);
    }
}

// -------------------------------------------------------------- host side ----

static int max_tiles_of(const BmShape& s) {
    const int64_t units = (int64_t)s.B * s.Hkv * s.N;
    const int64_t nb = (int64_t)s.B * s.Hkv * s.M1;
    const int per_tile = 128 / s.G;
    return (int)((units * kSlots + per_tile - 1) / per_tile + nb + 1);
}

BmLayout blockmajor_layout(const BmShape& s) {
    const int64_t units = (int64_t)s.B * s.Hkv * s.N;
    const int64_t nb = (int64_t)s.B * s.Hkv * s.M1;
    const int64_t max_tiles = max_tiles_of(s);
    BmLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += (bytes + 255) & ~size_t(255);
        return o;
    };
    L.cand = take(units * kSlots * 4);
    L.lse = take(units * kSlots * s.G * 4);
    L.vscore = take(s.variant ? units * kSlots * s.G * 4 : 0);  // PISA-1 / PISA-2 ranking scores
    L.z2 = take(units * s.G * 4);
    L.counts = take(nb * 4);
    L.slots = take(units * kPairs * 4);
    L.offsets = take(nb * 4);
    L.entries = take(units * kSlots * 4);
    L.tiles = take(max_tiles * 16);
    L.bsum = take(((nb + kScanBlock - 1) / kScanBlock) * 16);
    L.phl = take(walk_tc_pyramid_bytes((int64_t)s.B * s.Hkv, s.rows));  // bf16 high / low parts of the pyramid
    L.resume = take(units * 4);  // where the one-warp walk resumes after the tile walk
    L.misc = take(256);  // [0] tile count, [1] error word
    L.oacc = take((int64_t)s.B * s.Hq * s.N * kD * 4);
    L.total = off;
    return L;
}

static int grid_for(int64_t n, int per) { return (int)((n + per - 1) / per); }

static void mark(const PhaseEvents* ev, int i, cudaStream_t st) {
    if (ev && ev->events && i < ev->n && ev->events[i]) cudaEventRecord((cudaEvent_t)ev->events[i], st);
}

static dim3 unit_grid(const BmShape& s) { return dim3((unsigned)((s.N + 7) / 8), (unsigned)(s.B * s.Hkv)); }

static GroupParams group_params(int stride, const SelectParams& sp, const BmShape& s) {
    return GroupParams{s.N, sp.C, sp.causal, sp.forced_mask, stride, s.M1};
}

static cudaError_t zero_counts(const BmShape& s, uint8_t* ws, const BmLayout& L, cudaStream_t st) {
    const int64_t nb = (int64_t)s.B * s.Hkv * s.M1;
    return cudaMemsetAsync(ws + L.counts, 0, nb * 4, st);
}

// bucket counts and slots of the non-forced entries of `src` must already be
// in place (stage 1 and Top-K record them as they go); scan the counts and
// scatter the entries to their slots.
// pairs: `src` is the candidate list and the buckets are level-2 nodes.
static cudaError_t place_tiles(const int32_t* src, int stride, const SelectParams& sp, const BmShape& s,
                               uint8_t* ws, const BmLayout& L, cudaStream_t st, bool pairs = false) {
    const int64_t nkeys = pairs ? (s.M1 + 1) / 2 : s.M1;
    const int64_t nb = (int64_t)s.B * s.Hkv * nkeys;
    const unsigned nblk = (unsigned)((nb + kScanBlock - 1) / kScanBlock);
    bucket_total_kernel<<<nblk, kScanBlock, 0, st>>>((const int32_t*)(ws + L.counts), nb, 128 / s.G, s.N,
                                                     (longlong2*)(ws + L.bsum), (int*)(ws + L.misc) + 1);
    bucket_place_kernel<<<nblk, kScanBlock, 0, st>>>((const int32_t*)(ws + L.counts), nb, nkeys, 128 / s.G, s.N,
                                                     (const longlong2*)(ws + L.bsum), (int32_t*)(ws + L.offsets),
                                                     (int4*)(ws + L.tiles), (int32_t*)(ws + L.misc));
    GroupParams g = group_params(stride, sp, s);
    if (pairs) {
        g.M1 = nkeys;
        bucket_fill_pairs_kernel<<<unit_grid(s), 256, 0, st>>>(src, g, (const int32_t*)(ws + L.offsets),
                                                               (const int32_t*)(ws + L.slots),
                                                               (uint32_t*)(ws + L.entries));
    } else {
        bucket_fill_kernel<<<unit_grid(s), 256, 0, st>>>(src, g, (const int32_t*)(ws + L.offsets),
                                                         (const int32_t*)(ws + L.slots), (uint32_t*)(ws + L.entries));
    }
    return cudaGetLastError();
}

// count, scan and fill for a caller-provided list (standalone attention)
static cudaError_t build_tiles(const int32_t* src, int stride, const SelectParams& sp, const BmShape& s, uint8_t* ws,
                               const BmLayout& L, cudaStream_t st) {
    cudaError_t e = zero_counts(s, ws, L, st);
    if (e != cudaSuccess) return e;
    bucket_count_kernel<<<unit_grid(s), 256, 0, st>>>(src, group_params(stride, sp, s), (int32_t*)(ws + L.counts),
                                                      (int32_t*)(ws + L.slots));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return place_tiles(src, stride, sp, s, ws, L, st);
}

static int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

// attention tiles: Q (then P, then two rounds of 64 staged output rows) 33.8 KB,
// V 16 KB at 40 KB, K 16 KB at 56 KB: three CTAs per SM. The forced tiles stage
// all 128 rows at once over their Q, K and V buffers.
constexpr size_t kAttnSmem = 72 * 1024;
static_assert(64 * kORowStride <= 40960, "half the staged output tile fits below the value block");
static_assert(128 * kORowStride <= kAttnSmem, "the staged output tile fits in the forced tile's buffers");
constexpr int kAttnCtasPerSm = 3;

template <int G, bool PAIR, bool VSCORE>
static cudaError_t leaf_scores_t(const void* Q, const void* K, const SelectParams& sp, const BmShape& s, uint8_t* ws,
                                 const BmLayout& L, cudaStream_t st) {
    TileParams tp{s.B, s.Hq, s.Hkv, s.N, sp.causal, s.M1, sp.qscale, max_tiles_of(s), sp.variant};
    constexpr size_t smem = 32768 + (PAIR ? 32768 : 16384);
    auto kern = leaf_score_kernel<G, PAIR, VSCORE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<sm_count() * (PAIR ? 3 : 4), 128, smem, st>>>((const __nv_bfloat16*)Q, (const __nv_bfloat16*)K,
                                                          (const int4*)(ws + L.tiles), (const int32_t*)(ws + L.misc),
                                                          (const uint32_t*)(ws + L.entries), (float*)(ws + L.lse),
                                                          VSCORE ? (float*)(ws + L.vscore) : nullptr,
                                                          (int*)(ws + L.misc) + 1, tp, sp.forced_mask);
    return cudaGetLastError();
}

// leaf LSEs (and, for the sibling-pair ranking pass with a PISA-1 / PISA-2
// score, the ranking scores: a separate instantiation, so the default pass
// keeps its registers)
template <int G, bool PAIR>
static cudaError_t leaf_scores(const void* Q, const void* K, const SelectParams& sp, const BmShape& s, uint8_t* ws,
                               const BmLayout& L, cudaStream_t st) {
    if (PAIR && sp.variant) return leaf_scores_t<G, PAIR, true>(Q, K, sp, s, ws, L, st);
    return leaf_scores_t<G, PAIR, false>(Q, K, sp, s, ws, L, st);
}

template <int G>
static cudaError_t select_bm_t(const void* Q, const void* K, const float* pyr, int32_t* idx, const SelectParams& sp,
                               const BmShape& s, uint8_t* ws, const PhaseEvents* ev, cudaStream_t st) {
    const BmLayout L = blockmajor_layout(s);
    int32_t* cand = (int32_t*)(ws + L.cand);
    cudaError_t e = cudaMemsetAsync(ws + L.misc, 0, 256, st);
    if (e != cudaSuccess) return e;
    e = zero_counts(s, ws, L, st);
    if (e != cudaSuccess) return e;
    using W = typename std::conditional<(G <= 2), Walk4S<(G <= 2 ? G : 1)>, Walk<__nv_bfloat16, kD, G>>::type;
    if (walk_tc_fits(sp)) {
        // the coarse levels in tiles of consecutive positions on the tensor cores,
        // the fine ones (little reuse across positions) one warp per position
        e = launch_walk_tc(Q, pyr, ws + L.phl, cand, (int32_t*)(ws + L.resume), (int32_t*)(ws + L.counts),
                           (int32_t*)(ws + L.slots), (int*)(ws + L.misc) + 1, sp, G, sm_count(), st);
        if (e != cudaSuccess) return e;
        stage1_kernel<G, W, true><<<unit_grid(s), 256, 0, st>>>((const __nv_bfloat16*)Q, pyr, cand,
                                                                (int32_t*)(ws + L.counts), (int32_t*)(ws + L.slots),
                                                                s.M1, (int*)(ws + L.misc) + 1, sp,
                                                                (const int32_t*)(ws + L.resume));
    } else {
#if PISA_STAGE1_CARVEOUT >= 0
        // the walk lives on L1 hits of pyramid rows and needs little shared memory
        e = cudaFuncSetAttribute(stage1_kernel<G, W>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 PISA_STAGE1_CARVEOUT);
        if (e != cudaSuccess) return e;
#endif
        stage1_kernel<G, W><<<unit_grid(s), 256, 0, st>>>((const __nv_bfloat16*)Q, pyr, cand,
                                                          (int32_t*)(ws + L.counts), (int32_t*)(ws + L.slots), s.M1,
                                                          (int*)(ws + L.misc) + 1, sp);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    mark(ev, 2, st);
    e = place_tiles(cand, kSlots, sp, s, ws, L, st, /*pairs=*/true);
    if (e != cudaSuccess) return e;
    mark(ev, 3, st);
    e = leaf_scores<G, true>(Q, K, sp, s, ws, L, st);
    if (e != cudaSuccess) return e;
    mark(ev, 4, st);
    e = zero_counts(s, ws, L, st);  // the Top-K counts the kept leaves for the attention grouping
    if (e != cudaSuccess) return e;
    const dim3 topk_grid((unsigned)((s.N + 8 * kTopkQ - 1) / (8 * kTopkQ)), (unsigned)(s.B * s.Hkv));
    topk_kernel<G><<<topk_grid, 256, 0, st>>>(cand, (const float*)(ws + L.lse),
                                              sp.variant ? (const float*)(ws + L.vscore) : nullptr, idx,
                                              (float*)(ws + L.z2),
                                              (int32_t*)(ws + L.counts), (int32_t*)(ws + L.slots), s.M1, sp);
    e = cudaGetLastError();
    mark(ev, 5, st);
    return e;
}

template <int G>
static cudaError_t attn_bm_t(const void* Q, const void* K, const void* V, const int32_t* idx, void* O,
                             const SelectParams& sp, const BmShape& s, uint8_t* ws, bool have_z2,
                             const PhaseEvents* ev, cudaStream_t st) {
    const BmLayout L = blockmajor_layout(s);
    float* oacc = (float*)(ws + L.oacc);
    const int64_t units = (int64_t)s.B * s.Hkv * s.N;
    const int64_t nO = (int64_t)s.B * s.Hq * s.N * kD;
    cudaError_t e;
    if (!have_z2) {
        e = cudaMemsetAsync(ws + L.misc, 0, 256, st);
        if (e != cudaSuccess) return e;
    }
    // the selection leaves the kept leaves' bucket counts in place
    e = have_z2 ? place_tiles(idx, sp.K, sp, s, ws, L, st) : build_tiles(idx, sp.K, sp, s, ws, L, st);
    if (e != cudaSuccess) return e;
    if (!have_z2) {  // per-head LSE of the listed non-forced leaves, then their part of the normaliser
        e = leaf_scores<G, false>(Q, K, sp, s, ws, L, st);
        if (e != cudaSuccess) return e;
        z2_kernel<G><<<grid_for(units * G, 256), 256, 0, st>>>(idx, (const float*)(ws + L.lse),
                                                                (float*)(ws + L.z2), units, sp.K, s.N, sp.C,
                                                                sp.causal, sp.forced_mask);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    mark(ev, 6, st);
    {
        ForcedParams fp{s.B, s.Hq, s.Hkv, s.N, sp.causal, sp.forced_mask, sp.K, sp.qscale,
                        ((int64_t)s.N + 128 / G - 1) / (128 / G)};
        auto fk = forced_tile_kernel<G>;
        e = cudaFuncSetAttribute(fk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmem);
        if (e != cudaSuccess) return e;
        const int64_t ntiles = (int64_t)s.B * s.Hkv * fp.tiles_per_head;
        // 256 TMEM columns each (O accumulates over the leaves while S is recomputed): two per SM
        const int64_t slots = (int64_t)sm_count() * 2;
        const int grid = (int)(ntiles < slots ? ntiles : slots);
        fk<<<grid, 128, kAttnSmem, st>>>((const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
                                         idx, (float*)(ws + L.z2), oacc, (int*)(ws + L.misc) + 1, fp);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    mark(ev, 7, st);
    TileParams tp{s.B, s.Hq, s.Hkv, s.N, sp.causal, s.M1, sp.qscale, max_tiles_of(s), sp.variant};
    auto kern = attn_tile_kernel<G>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmem);
    if (e != cudaSuccess) return e;
    kern<<<sm_count() * kAttnCtasPerSm, 128, kAttnSmem, st>>>((const __nv_bfloat16*)Q, (const __nv_bfloat16*)K,
                                                 (const __nv_bfloat16*)V, (const int4*)(ws + L.tiles),
                                                 (const int32_t*)(ws + L.misc), (const uint32_t*)(ws + L.entries),
                                                 (const float*)(ws + L.z2), oacc, (int*)(ws + L.misc) + 1, tp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    mark(ev, 8, st);
    if (O) {  // without O the fp32 accumulator in the workspace is the result
        finalize_kernel<<<sm_count() * 8, 256, 0, st>>>(oacc, (__nv_bfloat16*)O, nO / 4);
        e = cudaGetLastError();
    }
    mark(ev, 9, st);
    return e;
}

size_t blockmajor_bwd_bytes(const BmShape& s) {
    const int64_t units = (int64_t)s.B * s.Hkv * s.N;
    return blockmajor_layout(s).total + (((size_t)units * s.G * 4 + 255) & ~size_t(255));
}

// Backward with the selection fixed. The softmax statistics L and D per
// (query, head) come either from the stats pass over the same tiles (the free
// (query, leaf) pairs grouped as the forward groups them, plus each leaf's
// forced section) or, when `saved`, from what pisa_forward_ws /
// pisa_sparse_attn_ws left in the workspace (the normaliser, the fp32 output
// for D = dO . O, and the grouping). Then the gradients are zeroed and the
// key-major tiles run.
template <int G>
static cudaError_t attn_bwd_bm_t(const void* Q, const void* K, const void* V, const int32_t* idx, const void* dO,
                                 float* dQ, float* dK, float* dV, const SelectParams& sp, const BmShape& s,
                                 uint8_t* ws, bool saved, const PhaseEvents* ev, cudaStream_t st) {
    const BmLayout L = blockmajor_layout(s);
    float* Dr = (float*)(ws + L.total);
    const int64_t units = (int64_t)s.B * s.Hkv * s.N;
    const int64_t rows = (int64_t)s.B * s.Hq * s.N;
    mark(ev, 0, st);
    cudaError_t e;
    if (saved) {
        bwd_delta_kernel<G><<<grid_for(rows, 8), 256, 0, st>>>((const __nv_bfloat16*)dO, (const float*)(ws + L.oacc),
                                                              Dr, rows, s.N, s.Hq);
    } else {
        if ((e = cudaMemsetAsync(ws + L.misc, 0, 256, st)) != cudaSuccess) return e;
        if ((e = build_tiles(idx, sp.K, sp, s, ws, L, st)) != cudaSuccess) return e;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t nb = (int64_t)s.B * s.Hkv * s.M1;
    const unsigned nblk = (unsigned)((nb + kScanBlock - 1) / kScanBlock);
    bwd_total_kernel<<<nblk, kScanBlock, 0, st>>>((const int32_t*)(ws + L.counts), nb, s.M1, 128 / G, s.N, sp.causal,
                                                  sp.forced_mask, (longlong2*)(ws + L.bsum), (int*)(ws + L.misc) + 1);
    bwd_place_kernel<<<nblk, kScanBlock, 0, st>>>((const int32_t*)(ws + L.counts), nb, s.M1, 128 / G, s.N, sp.causal,
                                                  sp.forced_mask, (const longlong2*)(ws + L.bsum),
                                                  (int4*)(ws + L.tiles), (int32_t*)(ws + L.misc));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    BwdParams bp{s.B, s.Hq, s.Hkv, s.N, sp.causal, sp.forced_mask, sp.K, s.M1, sp.qscale,
                 (float)(1.0 / sqrt((double)kD)), max_tiles_of(s)};
    if (!saved) {
        // per (unit, slot, head) statistics in the leaf-LSE region and the
        // (unused here) output accumulator region, then L into z2 and D
        float* lse_s = (float*)(ws + L.lse);
        float* dbar_s = (float*)(ws + L.oacc);
        auto sk = bwd_stats_kernel<G>;
        if ((e = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStatsSmem)) !=
            cudaSuccess)
            return e;
        sk<<<sm_count() * 2, 128, kStatsSmem, st>>>((const __nv_bfloat16*)Q, (const __nv_bfloat16*)K,
                                                    (const __nv_bfloat16*)V, (const __nv_bfloat16*)dO, idx,
                                                    (const int4*)(ws + L.tiles), (const int32_t*)(ws + L.misc),
                                                    (const int32_t*)(ws + L.offsets),
                                                    (const uint32_t*)(ws + L.entries), lse_s, dbar_s,
                                                    (int*)(ws + L.misc) + 1, bp);
        bwd_combine_kernel<G><<<grid_for(units * G, 256), 256, 0, st>>>(idx, lse_s, dbar_s, (float*)(ws + L.z2), Dr,
                                                                        units, sp.K);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    mark(ev, 1, st);
    const size_t kv_bytes = (size_t)s.B * s.Hkv * s.N * kD * 4;
    if ((e = cudaMemsetAsync(dQ, 0, (size_t)rows * kD * 4, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dK, 0, kv_bytes, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dV, 0, kv_bytes, st)) != cudaSuccess) return e;
    mark(ev, 2, st);
    auto kern = bwd_tile_kernel<G>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBwdSmem);
    if (e != cudaSuccess) return e;
    kern<<<sm_count(), 256, kBwdSmem, st>>>((const __nv_bfloat16*)Q, (const __nv_bfloat16*)K,
                                            (const __nv_bfloat16*)V, (const __nv_bfloat16*)dO, idx,
                                            (const int4*)(ws + L.tiles), (const int32_t*)(ws + L.misc),
                                            (const int32_t*)(ws + L.offsets), (const uint32_t*)(ws + L.entries),
                                            (const float*)(ws + L.z2), Dr, dQ, dK, dV, (int*)(ws + L.misc) + 1, bp);
    e = cudaGetLastError();
    mark(ev, 3, st);
    return e;
}

cudaError_t launch_select_bm(const void* Q, const void* K, const float* pyr, int32_t* idx, const SelectParams& sp,
                             const BmShape& s, void* ws, const PhaseEvents* ev, cudaStream_t st) {
    switch (s.G) {
        case 1: return select_bm_t<1>(Q, K, pyr, idx, sp, s, (uint8_t*)ws, ev, st);
        case 2: return select_bm_t<2>(Q, K, pyr, idx, sp, s, (uint8_t*)ws, ev, st);
        case 4: return select_bm_t<4>(Q, K, pyr, idx, sp, s, (uint8_t*)ws, ev, st);
        case 8: return select_bm_t<8>(Q, K, pyr, idx, sp, s, (uint8_t*)ws, ev, st);
        case 16: return select_bm_t<16>(Q, K, pyr, idx, sp, s, (uint8_t*)ws, ev, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bwd_bm(const void* Q, const void* K, const void* V, const int32_t* idx, const void* dO,
                               float* dQ, float* dK, float* dV, const SelectParams& sp, const BmShape& s, void* ws,
                               bool saved, const PhaseEvents* ev, cudaStream_t st) {
    uint8_t* w = (uint8_t*)ws;
    switch (s.G) {
        case 1: return attn_bwd_bm_t<1>(Q, K, V, idx, dO, dQ, dK, dV, sp, s, w, saved, ev, st);
        case 2: return attn_bwd_bm_t<2>(Q, K, V, idx, dO, dQ, dK, dV, sp, s, w, saved, ev, st);
        case 4: return attn_bwd_bm_t<4>(Q, K, V, idx, dO, dQ, dK, dV, sp, s, w, saved, ev, st);
        case 8: return attn_bwd_bm_t<8>(Q, K, V, idx, dO, dQ, dK, dV, sp, s, w, saved, ev, st);
        case 16: return attn_bwd_bm_t<16>(Q, K, V, idx, dO, dQ, dK, dV, sp, s, w, saved, ev, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bm(const void* Q, const void* K, const void* V, const int32_t* idx, void* O,
                           const SelectParams& sp, const BmShape& s, void* ws, bool have_z2, const PhaseEvents* ev,
                           cudaStream_t st) {
    switch (s.G) {
        case 1: return attn_bm_t<1>(Q, K, V, idx, O, sp, s, (uint8_t*)ws, have_z2, ev, st);
        case 2: return attn_bm_t<2>(Q, K, V, idx, O, sp, s, (uint8_t*)ws, have_z2, ev, st);
        case 4: return attn_bm_t<4>(Q, K, V, idx, O, sp, s, (uint8_t*)ws, have_z2, ev, st);
        case 8: return attn_bm_t<8>(Q, K, V, idx, O, sp, s, (uint8_t*)ws, have_z2, ev, st);
        case 16: return attn_bm_t<16>(Q, K, V, idx, O, sp, s, (uint8_t*)ws, have_z2, ev, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pisa
