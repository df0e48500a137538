// Tensor-core (tcgen05 + TMEM + TMA) tree-ordered GEMM for sm_100a.
//
// Source of the arithmetic: "Deterministic Inference across Tensor Parallel
// Sizes That Eliminates Training-Inference Mismatch" (TBIK summary page),
// sections 核心思路 / 技术框架: the K reduction is one hierarchical binary
// tree shared by the local and the cross-GPU steps.  Here each K leaf is a
// chain of 256xBNx16 bf16 MMAs into an fp32 TMEM accumulator that restarts
// from zero; the leaves are then combined by the halving tree in fp32 in the
// epilogue.  The MMA sequence of a leaf depends only on the leaf's K range,
// never on M, N or T, so a row's bits are the same for every batch size and
// every shard count (and, as measured, for either tile width).
//
// CTA pairs (clusters of 2, cta_group::2): a pair computes a 256 x BN tile,
// BN = 192 (128 for a [K,N] B of at most 128 columns); CTA r holds rows
// [128r, 128r+128) of A and rows/columns [BN/2 r, BN/2 (r+1)) of B in its
// shared memory and its own 128 x BN fp32 accumulators in TMEM.  The leader
// (rank 0) issues the MMAs; commits arrive on both CTAs' barriers.  Each CTA
// (one per SM, persistent over work units):
//   warp 0     TMA producer: its A and B halves, 128 deep (two 64-wide
//              128-byte-swizzle slices), into a ring of 3 stages (up to 8
//              when M is small and only the valid A rows are copied)
//   warp 1     TMEM allocator (both CTAs) + MMA issuer (leader, lane 0)
//   warps 2..  epilogue (8 warps for BN = 128, 12 for 192): drain each leaf
//              from TMEM and apply the tree; warp w reads TMEM lanes
//              32*(w%4).. (its row quadrant) and 64 columns of the tile
//   next warp  waiter (leader): performs every mbarrier wait the issuer needs
//              (stage landed, accumulator drained), then meets the MMA warp on
//              a named barrier.  A barrier wait in the issuing thread costs the
//              tensor pipe a few hundred cycles even when the barrier is
//              already complete; a named barrier between two warps costs
//              nothing, so the issuer only issues MMAs and commits.
// Pending subtree results wait by size (at most one value per on-chip class,
// checked by a host replay of the leaf operation codes for every leaf count
// up to 1100; values of >= 5 leaves go to a per-CTA fp32 scratch stack in
// global memory that stays in L2):
//   BN = 128: TMEM (512 columns) holds three leaf accumulators (columns 0,
//     128, 256) and a 2-leaf slot (384); a single leaf stays in its own
//     accumulator (the next leaf always consumes it); 3-4 leaves in a
//     shared-memory slot.
//   BN = 192: two accumulators (columns 0 and 256); a pending 2-leaf value
//     stays in the epilogue's registers R (64 per thread); the 3-4 leaf slot
//     is the spare TMEM columns [192, 256) and [448, 512) for column groups 0
//     and 1 plus 32 KiB of shared memory for group 2; a single leaf goes to R
//     when R is free, else to the slot when that is free, else it stays in its
//     accumulator (then the MMA waits for the next leaf's first phase).
// The epilogue handles a leaf in two phases: it first drains the leaf (and the
// single leaf it pops) and releases the accumulators, then does the other pops
// and the push, so the MMA does not wait on the rest of the tree work.
// A work unit is (m tile, n tile, frontier node f): the node's subtree of
// leaves is reduced by this pair; with more than one frontier node per tile the
// subtree results go to fp32 partial buffers that a combine kernel reduces
// with the upper levels of the same tree.
#pragma once

#include "device_common.cuh"

namespace tbik {

constexpr int TC_BM = 128;        // rows per CTA
constexpr int TC_PAIR_M = 256;    // rows per CTA pair (one MMA tile)
constexpr int TC_BN = 128;        // columns per pair tile: narrow [K,N] operands (N <= 128)
constexpr int TC_BN_WIDE = 192;   // columns per pair tile otherwise
constexpr int TC_MAX_STAGES = 8;  // ring stages when the A copies are small (small M)
constexpr int TC_BAR_EPI = 1;      // named barrier: the epilogue warps
constexpr int TC_BAR_HANDOFF = 2;  // named barrier: waiter warp + MMA warp, lockstep
constexpr int TC_TMEM_COLS = 512;
constexpr int TC_MAX_F = 64;
constexpr int TC_TAB_MAX = 1024;  // leaves per subtree covered by the shared-memory op table

// Per tile width: the 128-column tile keeps three leaf accumulators and a
// 2-leaf slot in TMEM and its 3-4 leaf slot in shared memory.  The
// 192-column tile keeps two accumulators (columns 0 and 256), holds a pending
// 2-leaf value in the epilogue's registers (12 epilogue warps of 64 columns
// each; 16 warps in all, so a thread may use 128 registers) and splits its
// 3-4 leaf slot: column groups 0 and 1 in the spare TMEM columns [192, 256)
// and [448, 512), group 2 in shared memory.
template <int BN>
struct TcCfg {
    static constexpr bool kWide = BN != TC_BN;
    static constexpr int BK = 128;                // K per ring stage
    static constexpr int KSLICES = BK / 64;       // 64-wide (128-byte) swizzle slices per stage
    static constexpr int KSTEPS = BK / 16;        // MMAs (K = 16) per stage
    static constexpr int STAGES = 3;              // ring stages when A fills its 128 rows
    static constexpr int EPI_WARPS = BN / 16;     // BN/64 column groups per TMEM lane quadrant
    static constexpr int WAITER_WARP = 2 + EPI_WARPS;
    static constexpr int THREADS = kWide ? 512 : 32 * (WAITER_WARP + 1);
    static constexpr int NACC = kWide ? 2 : 3;    // leaf accumulators in TMEM
    static constexpr int ACC_STRIDE = kWide ? 256 : 128;
    static constexpr int A_BYTES = TC_BM * BK * 2;        // this CTA's A rows
    static constexpr int B_BYTES = (BN / 2) * BK * 2;     // this CTA's half of B
    static constexpr int RING_BYTES = STAGES * (A_BYTES + B_BYTES);
    static constexpr int SLOT_FLOATS = TC_BM * BN;                      // one pending value (L2 stack slot)
    static constexpr int SMEM_SLOT_FLOATS = kWide ? TC_BM * 64 : SLOT_FLOATS;  // its shared-memory part
    static constexpr uint32_t TMEM_SPARE0 = 192, TMEM_SPARE1 = 448;    // wide: slot columns of groups 0, 1
    static constexpr size_t SMEM_BYTES = (size_t)RING_BYTES + SMEM_SLOT_FLOATS * 4 + 2 * TC_TAB_MAX * 2 /*op tables*/ +
                                         1024 /*align*/ + 256 /*barriers*/;
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
    static_assert(THREADS / 32 > WAITER_WARP, "warp roles");
};

// EPI_TREE_RES: EPI_TREE whose direct tiles add the bf16 residual to the fp32
// root before the output rounding (a separate instantiation, so the plain
// tree epilogue carries no residual code).
enum { EPI_TREE = 0, EPI_LOGPROB = 1, EPI_TREE_RES = 2 };

struct TcParams {
    int M, N, K;
    int leaf;         // K elements per leaf (multiple of 16)
    int F;            // frontier nodes per output tile
    int tiles_m, tiles_n, group_m;
    int total_units;
    int direct;       // 1: write final C; 0: write partials[f]
    int out_bf16;
    int swiglu;       // 1: C = bf16 SwiGLU of the interleaved gate/up roots, [M, N/2] (direct only)
    void* out;        // C [M,N]
    const uint16_t* residual;  // EPI_TREE_RES: bf16 [M,N] added to the root before the rounding (direct only)
    float* partials;  // [F][M][N]
    float* scratch;   // [gridDim.x][gs][128*BN], layout per slot [col/4][row][4]
    int gs;           // global stack slots per CTA (pending subtrees of >= 5 leaves)
    int b_mn;         // 1: B is [K,N] (MN-major operand)
    // logprob epilogue
    const int32_t* targets;
    float* stats;  // [vocab leaves][M][2]  (max, sum-exp) per row and 64-column vocab leaf
    float* zt;     // [M]  logit of the target
    int* zflag;    // [M] or null: set to 1 where zt is written (vocabulary shard summaries)
    int v0;        // vocabulary index of column 0 of B (a shard's first column; 0 otherwise)
    int V;
    unsigned debug;
    unsigned long long wait_cycles;  // bound of every device-side wait, in SM cycles
    int seq;                         // 1: the leaves form the left-to-right chain, not the tree
    int a_box_rows;                  // rows per A copy: 128, or M rounded up to 8 when M <= 128
    // Ring layout: stage s at s * stage_bytes holds the A slices of a_slice
    // bytes (a_box_rows rows of 128 bytes) and then the B slices;
    // stages = RING_BYTES / stage_bytes, at most TC_MAX_STAGES.
    int stages;
    uint32_t stage_bytes, a_slice;
    int tab_n[2];                    // the (at most two) subtree sizes of the frontier nodes
    // Pacing (null: none): [0] gives up on pacing for the rest of the launch,
    // [e] counts the pairs that reached their unit TC_PACE_UNITS * e.  Zeroed
    // by the host before the launch.
    unsigned int* pace;
    short lo[TC_MAX_F];
    short nl[TC_MAX_F];
};

// Pairs keep in step: every TC_PACE_UNITS work units each pair's producer
// waits, briefly and bounded, until every pair has reached the same unit.
// The pairs of a vocabulary column then fetch its W_lm tile while the others
// still hold it in L2 (left alone they drift apart over a launch and part of
// W_lm is read from DRAM again).  Only timing depends on it, never results.
// A pair that waits longer than TC_PACE_WAIT cycles (CTAs not all resident,
// or one pair far behind) switches pacing off for the whole launch.
constexpr int TC_PACE_UNITS = 16;
constexpr long long TC_PACE_WAIT = 4000000;
__device__ __forceinline__ void tc_pace(unsigned int* pace, int epoch, unsigned int npairs) {
    if (atomicOr(&pace[0], 0u) != 0u) return;
    atomicAdd(&pace[epoch], 1u);
    const long long t0 = clock64();
    while (atomicOr(&pace[epoch], 0u) < npairs) {
        if (clock64() - t0 > TC_PACE_WAIT || atomicOr(&pace[0], 0u) != 0u) {
            atomicExch(&pace[0], 1u);
            return;
        }
        __nanosleep(256);
    }
}

__device__ __forceinline__ void tc_decode(const TcParams& p, int u, int& tm, int& tn, int& f) {
    int tiles = p.tiles_m * p.tiles_n;
    f = u / tiles;
    int t = u - f * tiles;
    int group_size = p.group_m * p.tiles_n;
    int g = t / group_size;
    int first_m = g * p.group_m;
    int gm = min(p.tiles_m - first_m, p.group_m);
    int r = t - g * group_size;
    tm = first_m + r % gm;
    tn = r / gm;
}

template <int BN>
__device__ __forceinline__ float* scratch_slot(const TcParams& p, int slot) {
    return p.scratch + ((size_t)blockIdx.x * p.gs + slot) * TcCfg<BN>::SLOT_FLOATS;
}

// 32 columns (chunk c) of one row of a scratch slot; coalesced across the warp.
__device__ __forceinline__ void scratch_ld(const float* base, int c, int row, float (&w)[32]) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float4 x = *reinterpret_cast<const float4*>(base + ((size_t)(c * 8 + q) * TC_BM + row) * 4);
        w[4 * q + 0] = x.x;
        w[4 * q + 1] = x.y;
        w[4 * q + 2] = x.z;
        w[4 * q + 3] = x.w;
    }
}
__device__ __forceinline__ void scratch_st(float* base, int c, int row, const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(base + ((size_t)(c * 8 + q) * TC_BM + row) * 4) =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// A push onto the L2 stack (the layout of scratch_st), with an evict-last L2
// policy: the lines are read back by the pop a few leaves later, and keeping
// them resident avoids their write-back and re-read (measured 1-2 % faster).
__device__ __forceinline__ void stack_push32(float* base, int c, int row, const float (&v)[32]) {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float* a = base + ((size_t)(c * 8 + q) * TC_BM + row) * 4;
        asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(a), "f"(v[4 * q]),
                     "f"(v[4 * q + 1]), "f"(v[4 * q + 2]), "f"(v[4 * q + 3]), "l"(pol)
                     : "memory");
    }
}

// 16 columns (chunk q) of one row of a slot, as raw bits (the layout of scratch_ld).
__device__ __forceinline__ void scratch_ld16(const float* base, int q, int row, uint32_t (&w)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float4 x = *reinterpret_cast<const float4*>(base + ((size_t)(q * 4 + i) * TC_BM + row) * 4);
        w[4 * i + 0] = __float_as_uint(x.x);
        w[4 * i + 1] = __float_as_uint(x.y);
        w[4 * i + 2] = __float_as_uint(x.z);
        w[4 * i + 3] = __float_as_uint(x.w);
    }
}

// Row `row` (global), columns [col0, col0+32) of the output; N % 8 == 0.
__device__ __forceinline__ void store_row32(void* out, int out_bf16, int M, int N, int row, int col0,
                                            const float (&v)[32]) {
    if (row >= M) return;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        int col = col0 + 8 * q;
        if (col >= N) break;
        size_t off = (size_t)row * N + col;
        if (out_bf16) {
            uint4 w;
            w.x = pack_bf2(v[8 * q + 0], v[8 * q + 1]);
            w.y = pack_bf2(v[8 * q + 2], v[8 * q + 3]);
            w.z = pack_bf2(v[8 * q + 4], v[8 * q + 5]);
            w.w = pack_bf2(v[8 * q + 6], v[8 * q + 7]);
            *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + off) = w;
        } else {
            float* o = reinterpret_cast<float*>(out) + off;
            *reinterpret_cast<float4*>(o) = make_float4(v[8 * q], v[8 * q + 1], v[8 * q + 2], v[8 * q + 3]);
            *reinterpret_cast<float4*>(o + 4) = make_float4(v[8 * q + 4], v[8 * q + 5], v[8 * q + 6], v[8 * q + 7]);
        }
    }
}

// v[k] += f32(R[row, col0 + k]) for the 32 columns of store_row32 (one fp32
// add each, before the output's single rounding); N % 8 == 0.
__device__ __forceinline__ void add_residual32(const uint16_t* R, int M, int N, int row, int col0, float (&v)[32]) {
    if (row >= M) return;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int col = col0 + 8 * q;
        if (col >= N) break;
        float f[8];
        unpack8(*reinterpret_cast<const uint4*>(R + (size_t)row * N + col), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * q + e] = __fadd_rn(v[8 * q + e], f[e]);
    }
}

// Logprob epilogue of one warp's 64 columns, one vocab leaf (index vleaf,
// first column c0 of this call's vocabulary): the max, then the sum of
// exp(z - max) = 2^(z*log2e - max*log2e) as two interleaved partial sums (even
// and odd columns, each ascending) added at the end; (max, sum) go to
// stats[vleaf][row] and the target's logit to zt[row].  Hardware exponential:
// this mode is checked by tolerance; the order is fixed, so the bits are the
// same for every T and M.  v is the fp32 root of the K tree for the 64 columns.
__device__ __forceinline__ void logprob_leaf_stats(const TcParams& p, float (&v)[2][32], int row, int c0,
                                                   int vleaf) {
    if (c0 < p.V) {
        // target column relative to this call's first vocabulary column
        const long long tgt = (row < p.M) ? (long long)p.targets[row] - p.v0 : -1;
        const int ncol = min(64, p.V - c0);
        const long long kt = tgt - c0;  // target column within this leaf
        const bool have_t = kt >= 0 && kt < ncol;
        const int kti = have_t ? (int)kt : -1;
        float zval = 0.0f;
        if (have_t) {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                if (k == kti) zval = v[0][k];
                if (k + 32 == kti) zval = v[1][k];
            }
        }
        if (ncol < 64) {  // the last vocab leaf: columns past V add nothing
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                if (k >= ncol) v[0][k] = -INFINITY;
                if (k + 32 >= ncol) v[1][k] = -INFINITY;
            }
        }
        // the maximum in four independent chains of three-input maxima (max is
        // exact, so the grouping does not change it)
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
#pragma unroll
            for (int k = 0; k < 32; k += 8)
#pragma unroll
                for (int q = 0; q < 4; ++q) mq[q] = fmax3(mq[q], v[cc][k + 2 * q], v[cc][k + 2 * q + 1]);
        const float m = fmax3(fmaxf(mq[0], mq[1]), mq[2], mq[3]);
        const float log2e = 0x1.715476p+0f;
        const float ml = -__fmul_rn(m, log2e);
        float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
                s0 = __fadd_rn(s0, ex2_hw(__fmaf_rn(v[cc][k], log2e, ml)));
                s1 = __fadd_rn(s1, ex2_hw(__fmaf_rn(v[cc][k + 1], log2e, ml)));
            }
        const float s = __fadd_rn(s0, s1);
        if (row < p.M) {
            *reinterpret_cast<float2*>(p.stats + ((size_t)vleaf * p.M + row) * 2) = make_float2(m, s);
            if (have_t) {
                p.zt[row] = zval;
                if (p.zflag) p.zflag[row] = 1;
            }
        }
    }
}

template <int EPI, int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(TcCfg<BN>::THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ TcParams p) {
    using Cfg = TcCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* ring = smem;
    float* sSlot = reinterpret_cast<float*>(smem + Cfg::RING_BYTES);  // pending 3-4 leaf subtree
    uint16_t* leaf_tab = reinterpret_cast<uint16_t*>(sSlot + Cfg::SMEM_SLOT_FLOATS);  // [2][TC_TAB_MAX]
    uint64_t* bars = reinterpret_cast<uint64_t*>(leaf_tab + 2 * TC_TAB_MAX);
    uint64_t* full = bars;                          // [stages] both CTAs' copies landed (leader's)
    uint64_t* empty = bars + TC_MAX_STAGES;         // [stages] MMAs done reading (both CTAs)
    uint64_t* acc_full = bars + 2 * TC_MAX_STAGES;  // [NACC] leaf accumulator ready (both CTAs)
    uint64_t* acc_empty = acc_full + 3;         // [NACC] leaf accumulator drained by both CTAs (leader's)
    uint64_t* done = acc_empty + 3;             // all MMAs retired (both CTAs)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    // Waiter's verdicts, two slots by hand-off parity: the waiter writes the
    // verdict of hand-off h+1 only after hand-off h's barrier, and it reaches
    // hand-off h+2 (same slot as h) only after the issuer has passed hand-off
    // h+1's barrier, so the issuer always reads the verdict of its own step.
    volatile int* handoff_go = abort_flag + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t wait_lim = p.wait_cycles;
    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < TC_MAX_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < Cfg::NACC; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * Cfg::EPI_WARPS);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TC_TMEM_COLS);
        tmem_relinquish_pair();
    }
    const bool use_tab = p.tab_n[0] <= TC_TAB_MAX && p.tab_n[1] <= TC_TAB_MAX;
    if (use_tab)
        for (int i = threadIdx.x; i < p.tab_n[0] + p.tab_n[1]; i += blockDim.x) {
            const int t = i < p.tab_n[0] ? 0 : 1;
            const int j = i - (t ? p.tab_n[0] : 0);
            leaf_tab[t * TC_TAB_MAX + j] = encode_leaf_ops(p.seq ? seq_leaf_ops(p.tab_n[t], j) : leaf_ops(p.tab_n[t], j));
        }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            const bool b_mn = p.b_mn != 0;
            const int stages = p.stages;
            uint32_t q = 0, ph = 0;
            int s = 0;
            // units every pair has (pacing points must be reached by all of them)
            const int common_units = p.total_units / npairs;
            int kunit = 0;
            for (int u = pair; u < p.total_units; u += npairs, ++kunit) {
                if (p.pace != nullptr && rank == 0 && kunit > 0 && kunit % TC_PACE_UNITS == 0 && kunit < common_units)
                    tc_pace(p.pace, kunit / TC_PACE_UNITS, (unsigned)npairs);
                int tm, tn, f;
                tc_decode(p, u, tm, tn, f);
                const int k0 = p.lo[f] * p.leaf;
                const int nkb = (p.nl[f] * p.leaf + Cfg::BK - 1) / Cfg::BK;
                const int arow = tm * TC_PAIR_M + TC_BM * rank;
                const int brow = tn * BN + (BN / 2) * rank;
                // A CTA whose 128 rows are all past M copies no A: the MMA
                // then reads stale shared memory for rows whose results are
                // never stored (rows of an MMA are independent).  Small M also
                // copies only a_box_rows rows.
                const int rows_pair = p.M - tm * TC_PAIR_M;
                const bool a_mine = rows_pair - TC_BM * (int)rank > 0;
                const uint32_t a_copy = p.a_slice * Cfg::KSLICES;  // bytes per CTA and stage
                const uint32_t tx = a_copy * (rows_pair > TC_BM ? 2u : 1u) + 2u * Cfg::B_BYTES;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, wait_lim)) goto producer_out;
                    const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], tx);
                    const int kx = k0 + kb * Cfg::BK;
                    uint8_t* sA = ring + (size_t)s * p.stage_bytes;
                    uint8_t* sB = sA + a_copy;
#pragma unroll
                    for (int h = 0; h < Cfg::KSLICES; ++h) {
                        if (a_mine) tma_load_2d_pair(sA + h * p.a_slice, &tmA, bar, kx + 64 * h, arow);
                        if (!b_mn)
                            tma_load_2d_pair(sB + h * (Cfg::B_BYTES / Cfg::KSLICES), &tmB, bar, kx + 64 * h, brow);
                        else if (!Cfg::kWide)
                            tma_load_2d_pair(sB + h * (Cfg::B_BYTES / Cfg::KSLICES), &tmB, bar, brow, kx + 64 * h);
                    }
                    if (Cfg::kWide && b_mn) {
                        // [K,N] B on the 192-column tile: this CTA's 96 columns as three
                        // 32-column (64-byte swizzle) boxes of the stage's 128 K rows
#pragma unroll
                        for (int j = 0; j < BN / 64; ++j)
                            tma_load_2d_pair(sB + j * (Cfg::BK * 64), &tmB, bar, brow + 32 * j, kx);
                    }
                    ++q;
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
        producer_out:
            // The leader lets the copies of both CTAs land before the pair can exit.
            if (rank == 0)
                for (uint32_t i = (q > (uint32_t)stages ? q - stages : 0u); i < q; ++i)
                    mbar_drain(&full[i % stages], (i / stages) & 1, wait_lim);
        }
    } else if (warp == 1 || warp == Cfg::WAITER_WARP) {
        // ------------------------------------------------ MMA issuer + waiter (leader)
        // Both warps walk the same sequence of k-steps.  A hand-off happens
        // where the issuer needs a condition: a stage start (its copies landed)
        // or a leaf start (its accumulator buffer drained).  The waiter checks
        // the condition(s), stores its verdict, and both warps bar.sync; the
        // issuer then reads the verdict, so the two always stop together.
        // One stage carries BK/16 MMAs of K = 16; descriptors are built once
        // per stage and advanced through the start-address field.
        const bool is_mma = warp == 1;
        if (rank == 0) {
            const uint32_t idesc = idesc_bf16_f32(TC_PAIR_M, BN, 0, p.b_mn);
            const bool b_mn = p.b_mn != 0;
            // MN-major B (a [K,N] operand).  128-column tile: each CTA's 64
            // columns are one 128-byte swizzle atom wide, so the leading (MN)
            // offset spans the whole half tile and the stride between 8-deep K
            // groups is 1024 B.  192-column tile: 64-byte swizzle, the CTA's 96
            // columns are three 32-column atoms 128 K rows (8 KiB) apart, 8-deep
            // K groups 512 B apart, 1 KiB per 16 K rows.
            constexpr uint32_t b_lbo = Cfg::kWide ? (uint32_t)(Cfg::BK * 64) : (uint32_t)Cfg::B_BYTES;
            constexpr uint32_t b_sbo = Cfg::kWide ? 512u : 1024u;
            const uint32_t ring_u = smem_u32(ring);
            const uint32_t stage_bytes = p.stage_bytes, a_slice = p.a_slice;
            const int stages = p.stages;
            const int spl = p.leaf / 16;  // MMAs per leaf
            const uint64_t b_step = b_mn ? ((Cfg::kWide ? 1024u : 2048u) >> 4) : (32u >> 4);
            const bool aligned = (spl % Cfg::KSTEPS) == 0;  // leaf is a whole number of stages
            const int kb_per_leaf = spl / Cfg::KSTEPS;
            uint32_t a = 0, hc = 0, ph = 0;  // ph: phase of the ring (flips when stage 0 comes round)
            int s = 0;
            // The hand-off: waiter lane 0 waits (bounded) for what the issuer needs.
            auto handoff = [&](bool need_full, bool need_acc, uint32_t abuf, uint32_t acount) -> bool {
                volatile int* verdict = handoff_go + (hc & 1);
                ++hc;
                if (!is_mma) {
                    if (lane == 0) {
                        bool ok = true;
                        if (need_full) ok = mbar_wait(&full[s], ph, abort_flag, wait_lim);
                        if (ok && need_acc)
                            ok = mbar_wait(&acc_empty[abuf], ((acount / Cfg::NACC) & 1) ^ 1, abort_flag, wait_lim);
                        *verdict = ok ? 1 : 0;
                    }
                    __syncwarp();
                }
                named_barrier_sync(TC_BAR_HANDOFF, 64);
                const bool go = *verdict != 0;
                if (is_mma) tc_fence_after();
                return go;
            };
            for (int u = pair; u < p.total_units; u += npairs) {
                int tm, tn, f;
                tc_decode(p, u, tm, tn, f);
                const int nsteps = p.nl[f] * spl;
                uint32_t buf = 0;
                int in_leaf = 0, kb_in_leaf = 0;
                for (int st = 0; st < nsteps; st += Cfg::KSTEPS) {
                    // The A slices of a small-M stage are a_box_rows rows apart;
                    // the MMA's other rows read whatever follows (results never
                    // stored), always inside this CTA's shared memory.
                    const uint32_t sa = ring_u + (uint32_t)s * stage_bytes;
                    const uint32_t sb = sa + a_slice * Cfg::KSLICES;
                    const uint64_t adesc = smem_desc_sw128(sa, 16, 1024);
                    const uint64_t bdesc = !b_mn ? smem_desc_sw128(sb, 16, 1024)
                                                 : (Cfg::kWide ? smem_desc_sw64(sb, b_lbo, b_sbo)
                                                               : smem_desc_sw128(sb, b_lbo, b_sbo));
                    // k-step ks: slice ks/4 (advance by a slice's bytes >> 4), step ks%4 within it
                    auto a_at = [&](int ks) {
                        return adesc + (uint64_t)((ks >> 2) * (a_slice >> 4) + (ks & 3) * 2);
                    };
                    auto b_at = [&](int ks) {
                        if (Cfg::kWide && b_mn) return bdesc + b_step * (uint64_t)ks;  // one 128-deep region
                        return bdesc + (uint64_t)((ks >> 2) * ((Cfg::B_BYTES / Cfg::KSLICES) >> 4)) + b_step * (ks & 3);
                    };
                    if (aligned) {
                        if (kb_in_leaf == 0) buf = a % Cfg::NACC;
                        if (!handoff(true, kb_in_leaf == 0, buf, a)) goto mma_out;
                        if (is_mma && lane == 0) {
                            const uint32_t d = tmem_base + buf * Cfg::ACC_STRIDE;
                            tc_mma_pair(d, a_at(0), b_at(0), idesc, kb_in_leaf != 0 ? 1u : 0u);
#pragma unroll
                            for (int ks = 1; ks < Cfg::KSTEPS; ++ks) tc_mma_pair(d, a_at(ks), b_at(ks), idesc, 1u);
                            if (kb_in_leaf + 1 == kb_per_leaf) tc_commit_pair(&acc_full[buf]);
                        }
                        if (++kb_in_leaf == kb_per_leaf) {
                            ++a;
                            kb_in_leaf = 0;
                        }
                    } else {
                        const int nk = min(Cfg::KSTEPS, nsteps - st);
                        for (int ks = 0; ks < nk; ++ks) {
                            if (in_leaf == 0) buf = a % Cfg::NACC;
                            if (ks == 0 || in_leaf == 0)
                                if (!handoff(ks == 0, in_leaf == 0, buf, a)) goto mma_out;
                            if (is_mma && lane == 0) {
                                tc_mma_pair(tmem_base + buf * Cfg::ACC_STRIDE, a_at(ks), b_at(ks), idesc,
                                            in_leaf != 0 ? 1u : 0u);
                                if (in_leaf + 1 == spl) tc_commit_pair(&acc_full[buf]);
                            }
                            if (++in_leaf == spl) {
                                ++a;
                                in_leaf = 0;
                            }
                        }
                    }
                    if (is_mma && lane == 0) tc_commit_pair(&empty[s]);
                    __syncwarp();
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
        mma_out:
            // Every MMA issued by this thread retires before TMEM is released (both CTAs).
            if (is_mma && lane == 0) tc_commit_pair(done);
        }
        if (is_mma && lane == 0) mbar_drain(done, 0, wait_lim);
    } else if (warp < 2 + Cfg::EPI_WARPS) {
        // ------------------------------------------------ epilogue (both CTAs)
      if constexpr (!Cfg::kWide) {
        const int ew = warp & 3;           // TMEM lane quadrant = rows 32*ew .. 32*ew+31
        const int half = (warp - 2) >> 2;  // columns [64*half, 64*half+64)
        const int rt = ew * 32 + lane;     // row within this CTA's 128
        const uint32_t tl = tmem_base + ((uint32_t)(ew * 32) << 16);
        uint32_t a = 0;
        for (int u = pair; u < p.total_units; u += npairs) {
            int tm, tn, f;
            tc_decode(p, u, tm, tn, f);
            const int n = p.nl[f];
            const int row = tm * TC_PAIR_M + TC_BM * rank + rt;
            const uint16_t* tab = leaf_tab + (n == p.tab_n[0] ? 0 : TC_TAB_MAX);
            int gsp = 0;  // pending subtrees of >= 5 leaves in the global scratch
            for (int j = 0; j < n; ++j) {
                const uint32_t buf = a % 3;
                const uint32_t prev = (a + 2) % 3;  // accumulator of leaf j-1 (a retained single leaf)
                // One warp polls the accumulator barrier; the other epilogue
                // warps wait on a hardware barrier, so nothing else polls.  The
                // barrier's OR reduction makes the decision to give up common
                // to all epilogue warps.
                bool ok = true;
                if (warp == 2) ok = mbar_wait(&acc_full[buf], (a / 3) & 1, abort_flag, wait_lim);
                if (named_barrier_or(TC_BAR_EPI, 32 * Cfg::EPI_WARPS, !ok || *abort_flag != 0)) goto epi_out;
                ++a;
                const uint32_t code = use_tab ? tab[j] : encode_leaf_ops(p.seq ? seq_leaf_ops(n, j) : leaf_ops(n, j));
                const bool p1 = code & 1, p2 = (code >> 1) & 1, pm = (code >> 2) & 1;
                const int nb = (code >> 3) & 31;
                const int cls = (code >> 8) & 3;
                const bool final_ = (code >> 10) & 1;
                if (!final_ && cls == 0) continue;  // a single leaf waits in its accumulator
                tc_fence_after();
                // Phase 1: this leaf plus the single leaf it pops, into registers;
                // both accumulators are released before any other tree work, so
                // the MMA never waits on the pops and pushes below.
                float v[2][32];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int c = half * 2 + cc;
                    uint32_t r0[32], r1[32];
                    tmem_ld32_nowait(tl + buf * Cfg::ACC_STRIDE + c * 32, r0);
                    if (p1) tmem_ld32_nowait(tl + prev * Cfg::ACC_STRIDE + c * 32, r1);
                    tmem_wait_ld(r0);
                    if (p1) {
                        tie32(r1);
#pragma unroll
                        for (int k = 0; k < 32; ++k) v[cc][k] = __fadd_rn(__uint_as_float(r1[k]), __uint_as_float(r0[k]));
                    } else {
#pragma unroll
                        for (int k = 0; k < 32; ++k) v[cc][k] = __uint_as_float(r0[k]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0 && !(p.debug & TBIK_DEBUG_WITHHOLD_ACC_ARRIVE)) {
                    mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[buf]), 0));
                    if (p1) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[prev]), 0));
                }
                // Phase 2: the other pops, deepest (smallest) first, both chunks
                // at once, then the push of the result (or the output).
                if (p2) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t r2[32];
                        tmem_ld32_nowait(tl + 384 + (half * 2 + cc) * 32, r2);
                        tmem_wait_ld(r2);
#pragma unroll
                        for (int k = 0; k < 32; ++k) v[cc][k] = __fadd_rn(__uint_as_float(r2[k]), v[cc][k]);
                    }
                }
                if (pm) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        float w[32];
                        scratch_ld(sSlot, half * 2 + cc, rt, w);
#pragma unroll
                        for (int k = 0; k < 32; ++k) v[cc][k] = __fadd_rn(w[k], v[cc][k]);
                    }
                }
                for (int i = 0; i < nb; ++i) {
                    const float* sl = scratch_slot<BN>(p, gsp - 1 - i);
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        float w[32];
                        scratch_ld(sl, half * 2 + cc, rt, w);
#pragma unroll
                        for (int k = 0; k < 32; ++k) v[cc][k] = __fadd_rn(w[k], v[cc][k]);
                    }
                }
                const int g_after = gsp - nb;
                gsp = g_after + ((!final_ && cls == 3) ? 1 : 0);
                if (!final_) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c = half * 2 + cc;
                        if (cls == 1)
                            tmem_st32_nowait(tl + 384 + c * 32, v[cc]);
                        else if (cls == 2)
                            scratch_st(sSlot, c, rt, v[cc]);
                        else
                            stack_push32(scratch_slot<BN>(p, g_after), c, rt, v[cc]);
                    }
                    if (cls == 1) tmem_wait_st();
                } else if (EPI == EPI_TREE && p.swiglu) {
                    // this warp's 64 columns: gate features f0..f0+31 (chunk 0)
                    // and the up values of the same features (chunk 1)
                    if (row < p.M) {
                        const int f0 = tn * (BN / 2) + half * 32;
                        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) +
                                                              (size_t)row * (p.N / 2) + f0);
#pragma unroll
                        for (int q8 = 0; q8 < 4; ++q8) {
                            float o[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) o[e] = swiglu1(v[0][8 * q8 + e], v[1][8 * q8 + e]);
                            if (f0 + 8 * q8 < p.N / 2) dst[q8] = pack8(o);
                        }
                    }
                } else if (EPI != EPI_LOGPROB) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int col = tn * BN + (half * 2 + cc) * 32;
                        if (p.direct) {
                            if (EPI == EPI_TREE_RES) add_residual32(p.residual, p.M, p.N, row, col, v[cc]);
                            store_row32(p.out, p.out_bf16, p.M, p.N, row, col, v[cc]);
                        } else
                            store_row32(p.partials + (size_t)f * p.M * p.N, 0, p.M, p.N, row, col, v[cc]);
                    }
                } else {
                    logprob_leaf_stats(p, v, row, tn * BN + half * 64, 2 * tn + half);
                }
            }
        }
    epi_out:;
      } else {
        // 192-column tile: warp w reads TMEM lanes 32*(w%4).. and owns the 64
        // columns of group (w-2)/4.  R holds this thread's 64 values of the
        // working value, of a pending 2-leaf value, or of a stashed single
        // leaf; the tree-walk replay checks that these never overlap.
        const int ew = warp & 3;
        const int grp = (warp - 2) >> 2;  // columns [64*grp, 64*grp+64)
        const int rt = ew * 32 + lane;
        const uint32_t tl = tmem_base + ((uint32_t)(ew * 32) << 16) + (uint32_t)(grp * 64);
        // this warp's part of the 3-4 leaf slot in TMEM (groups 0, 1; group 2 uses shared memory)
        const uint32_t tslot =
            tmem_base + ((uint32_t)(ew * 32) << 16) + (grp == 0 ? Cfg::TMEM_SPARE0 : Cfg::TMEM_SPARE1);
        float R[2][32];
        uint32_t a = 0;
        for (int u = pair; u < p.total_units; u += npairs) {
            int tm, tn, f;
            tc_decode(p, u, tm, tn, f);
            const int n = p.nl[f];
            const int row = tm * TC_PAIR_M + TC_BM * rank + rt;
            const uint16_t* tab = leaf_tab + (n == p.tab_n[0] ? 0 : TC_TAB_MAX);
            int gsp = 0;
            for (int j = 0; j < n; ++j) {
                const uint32_t buf = a & 1;
                const uint32_t prev = buf ^ 1;  // accumulator of leaf j-1
                bool ok = true;  // as in the 128-column epilogue: one poller, a common decision
                if (warp == 2) ok = mbar_wait(&acc_full[buf], (a >> 1) & 1, abort_flag, wait_lim);
                if (named_barrier_or(TC_BAR_EPI, 32 * Cfg::EPI_WARPS, !ok || *abort_flag != 0)) goto wepi_out;
                ++a;
                const uint32_t code = use_tab ? tab[j] : encode_leaf_ops(p.seq ? seq_leaf_ops(n, j) : leaf_ops(n, j));
                const bool p1 = code & 1, p2 = (code >> 1) & 1, pm = (code >> 2) & 1;
                const int nb = (code >> 3) & 31;
                const int cls = (code >> 8) & 3;
                const bool final_ = (code >> 10) & 1, c2p = (code >> 11) & 1, mp = (code >> 12) & 1;
                const bool single = !final_ && cls == 0;
                // A single leaf goes to R when R is free, else to the 3-4 leaf
                // slot when that is free, else it stays in its accumulator and
                // the next leaf pops it from there.
                if (single && c2p && mp) continue;
                tc_fence_after();
                const uint32_t acc = tl + buf * Cfg::ACC_STRIDE;
                const bool s_tm = p1 && c2p && mp;   // popped single in TMEM (accumulator prev)
                const bool s_slot = p1 && c2p && !mp;  // popped single in the slot
                if (single && c2p) {
                    // park the single in the slot (TMEM spare columns or shared memory)
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t w[32];
                        tmem_ld32_nowait(acc + cc * 32, w);
                        tmem_wait_ld(w);
                        if (grp < 2) {
                            float f[32];
#pragma unroll
                            for (int k = 0; k < 32; ++k) f[k] = __uint_as_float(w[k]);
                            tmem_st32_nowait(tslot + cc * 32, f);
                        } else {
                            float f[32];
#pragma unroll
                            for (int k = 0; k < 32; ++k) f[k] = __uint_as_float(w[k]);
                            scratch_st(sSlot, cc, rt, f);
                        }
                    }
                    if (grp < 2) tmem_wait_st();
                } else if (s_tm || s_slot) {
                    // R = R + (single + leaf), 16 columns at a time
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t l[16], sv[16];
                        tmem_ld16_nowait(acc + q * 16, l);
                        if (s_tm)
                            tmem_ld16_nowait(tl + prev * Cfg::ACC_STRIDE + q * 16, sv);
                        else if (grp < 2)
                            tmem_ld16_nowait(tslot + q * 16, sv);
                        else
                            scratch_ld16(sSlot, q, rt, sv);
                        tmem_wait_ld16(l);
                        tie16(sv);
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            R[q >> 1][(q & 1) * 16 + k] = __fadd_rn(
                                R[q >> 1][(q & 1) * 16 + k], __fadd_rn(__uint_as_float(sv[k]), __uint_as_float(l[k])));
                    }
                } else if (p1 || p2) {
                    // R holds the left operand (a single or the 2-leaf value): R = R + leaf
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t l[32];
                        tmem_ld32_nowait(acc + cc * 32, l);
                        tmem_wait_ld(l);
#pragma unroll
                        for (int k = 0; k < 32; ++k) R[cc][k] = __fadd_rn(R[cc][k], __uint_as_float(l[k]));
                    }
                } else {
                    // R = leaf (a single going to R, or a leaf whose pops are all below)
                    uint32_t l[64];
                    tmem_ld64_nowait(acc, l);
                    tmem_wait_ld64(l);
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        R[0][k] = __uint_as_float(l[k]);
                        R[1][k] = __uint_as_float(l[32 + k]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0 && !(p.debug & TBIK_DEBUG_WITHHOLD_ACC_ARRIVE)) {
                    mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[buf]), 0));
                    if (s_tm) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[prev]), 0));
                }
                if (single) continue;  // held in R or the slot until the next leaf
                // Phase 2: the 3-4 leaf value, then the L2 stack from its top.
                if (pm) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        float w[32];
                        if (grp < 2)
                            tmem_ld32(tslot + cc * 32, w);
                        else
                            scratch_ld(sSlot, cc, rt, w);
#pragma unroll
                        for (int k = 0; k < 32; ++k) R[cc][k] = __fadd_rn(w[k], R[cc][k]);
                    }
                }
                for (int i = 0; i < nb; ++i) {
                    const float* sl = scratch_slot<BN>(p, gsp - 1 - i);
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        float w[32];
                        scratch_ld(sl, grp * 2 + cc, rt, w);
#pragma unroll
                        for (int k = 0; k < 32; ++k) R[cc][k] = __fadd_rn(w[k], R[cc][k]);
                    }
                }
                const int g_after = gsp - nb;
                gsp = g_after + ((!final_ && cls == 3) ? 1 : 0);
                if (!final_) {
                    // a 2-leaf value stays in R
                    if (cls == 2) {
                        if (grp < 2) {
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc) tmem_st32_nowait(tslot + cc * 32, R[cc]);
                            tmem_wait_st();
                        } else {
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc) scratch_st(sSlot, cc, rt, R[cc]);
                        }
                    } else if (cls == 3) {
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) stack_push32(scratch_slot<BN>(p, g_after), grp * 2 + cc, rt, R[cc]);
                    }
                } else if (EPI == EPI_TREE && p.swiglu) {
                    // gate features f0..f0+31 (R[0]) and their up values (R[1])
                    if (row < p.M) {
                        const int f0 = tn * (BN / 2) + grp * 32;
                        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) +
                                                              (size_t)row * (p.N / 2) + f0);
#pragma unroll
                        for (int q8 = 0; q8 < 4; ++q8) {
                            float o[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) o[e] = swiglu1(R[0][8 * q8 + e], R[1][8 * q8 + e]);
                            if (f0 + 8 * q8 < p.N / 2) dst[q8] = pack8(o);
                        }
                    }
                } else if (EPI != EPI_LOGPROB) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int col = tn * BN + (grp * 2 + cc) * 32;
                        if (p.direct) {
                            if (EPI == EPI_TREE_RES) add_residual32(p.residual, p.M, p.N, row, col, R[cc]);
                            store_row32(p.out, p.out_bf16, p.M, p.N, row, col, R[cc]);
                        } else
                            store_row32(p.partials + (size_t)f * p.M * p.N, 0, p.M, p.N, row, col, R[cc]);
                    }
                } else {
                    logprob_leaf_stats(p, R, row, tn * BN + grp * 64, (BN / 64) * tn + grp);
                }
            }
        }
    wepi_out:;
      }
    }

    // A CTA that gave up tells its peer, so the peer's waits end too.
    if (*abort_flag && threadIdx.x == 0) st_cluster_u32(mapa_shared(smem_u32((const void*)abort_flag), rank ^ 1), 1);
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TC_TMEM_COLS);
    }
}

}  // namespace tbik
