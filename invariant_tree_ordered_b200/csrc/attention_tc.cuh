// Tensor-core causal attention with the key reduction in tree order (TC mode).
//
// Source: TBIK summary page, 技术框架 (one hierarchical binary tree for every
// reduction, so the result does not depend on how the work is split).  The
// structure is the exact mode's (attention.cuh): keys in fixed leaves, each
// leaf reduced to a (max, sum, weighted value sum) summary, the summaries of
// the leaves 0..floor(i/128) combined by the halving tree.  What differs is
// the leaf (128 keys, two 64-key tensor-core chunks under one maximum) and how
// it is computed:
//   scores  s_j = fl(S_ij * scale), S = Q K^T on the tensor cores (tcgen05,
//           bf16 operands, fp32 accumulation in TMEM in the hardware's order);
//   leaf    m = max over the leaf's keys j <= i;
//           p_j = bf16(2^(s_j*log2e - m*log2e)) with the hardware exponential,
//           0 for j > i; s = s_lo + s_hi over the rounded p_j, where s_lo
//           covers keys 0..63 of the leaf and s_hi keys 64..127, each
//           (c0 + c1) + (c2 + c3) with c_q the ascending sum over the keys
//           k = q (mod 4) of that half;
//           o = P V on the tensor cores (the bf16 p_j as A, V as B, K = 128);
//   combine M = max, e = 2^(fl(m - M)*log2e) by the hardware exponential (1
//           for the side holding M), s = fma(s', e', fl(s*e)),
//           o = fma(o', e', fl(o*e)) (the left operand's product rounded);
//   output  bf16(o[d] * fl(1/s)).
// A row's result depends only on its query, the keys and values at positions
// <= i and its fixed leaf tree, never on the batch composition, the other
// rows of its tile or how heads are split across devices.
//
// One CTA per SM, persistent over 128-row query tiles of one (batch, head),
// the longest tiles first, dealt out in alternating directions; 320 threads:
//   warp 0     TMA producer: the Q tile (two 64-dim slices, K-major, 128-byte
//              swizzle), per leaf K (same layout, two 64-key chunks) and V
//              (MN-major: per chunk two 64-dim atoms of 64 keys); K of the
//              next leaf is requested as soon as the scores of the current
//              one are done, before V of the current one
//   warp 1     TMEM allocator + MMA issuer: S = Q K^T of the leaf's two chunks
//              (M=128, N=64 each) into S[0], S[1] (as soon as the softmax has
//              read the previous leaf's S into registers), then O_{L-1} = P V
//              of the previous leaf (M=128, N=128, K=128) into O[(L-1)%2]
//   warps 2-9  epilogue: warp w owns rows 32*(w%4).. and half h = (w-2)/4:
//              the softmax of chunk h of each leaf (its maximum taken over
//              both chunks) and head dims [64h, 64h+64) of the tree.  Loop:
//              softmax of leaf L (writes P_L), then the tree step of leaf
//              L-1, so the MMA of O_L runs while the tree of L-1 is evaluated.
// A tile starts at a multiple of 128, so every row of it has the same leaves
// (the tile's own block is the last, the diagonal one) and the tree walk is
// the same for all lanes of a warp.  Pending leaf summaries wait by size: a
// single leaf in its O buffer (the next leaf consumes it), 2 leaves in a TMEM
// slot, 3-4 in shared memory, >= 5 in a per-CTA stack in global memory that
// stays in L2.
#pragma once

#include "device_common.cuh"

namespace tbik {

constexpr int ATC_BM = 128;    // query rows per tile
constexpr int ATC_CH = 64;     // keys per tensor-core chunk
constexpr int ATC_LEAF = 128;  // keys per tree leaf (two chunks)
constexpr int ATC_HD = 128;    // head dimension
constexpr int ATC_EPI_WARPS = 8;
constexpr int ATC_THREADS = 32 * (2 + ATC_EPI_WARPS);
constexpr int ATC_TMEM_COLS = 512;
constexpr uint32_t ATC_S_COL = 0, ATC_O_COL = 128, ATC_SLOT_COL = 384;
constexpr int ATC_VAL_FLOATS = ATC_BM * ATC_HD;  // one pending o value of the tile
constexpr int ATC_MAX_GS = 8;  // L2 stack depth bound (leaf trees of up to 256 leaves need 5)
// shared memory (from a 1024-byte aligned base); V first, so that every
// descriptor-addressed read stays inside the allocation
constexpr int ATC_OFF_V = 0;             // the leaf's 2 chunks x 64 keys x 128 dims bf16, two 8 KiB atoms each
constexpr int ATC_OFF_K = 32768;         // the leaf's 2 chunks x 64 keys x 128 dims, two 8 KiB slices each
constexpr int ATC_OFF_Q = 65536;         // 128 rows x 128 dims, two 16 KiB slices
constexpr int ATC_OFF_P = 98304;         // [2 chunks] 128 rows x 64 keys bf16
constexpr int ATC_OFF_SLOT = 131072;     // pending 3-4 leaf value, fp32 [dim/4][row][4]
constexpr int ATC_OFF_X = 196608;        // [2][2][128] per-row sums exchanged between halves
constexpr int ATC_OFF_BAR = 198656;
constexpr size_t ATC_SMEM_BYTES = ATC_OFF_BAR + 256 + 1024;
static_assert(ATC_SMEM_BYTES <= 232448, "shared memory per CTA");

struct AttTcParams {
    int batch, seq, heads;
    int ntq;           // query tiles per (batch, head) = seq / 128
    int tiles;         // batch * heads * ntq
    float scale;
    uint16_t* out;     // [batch][seq][heads][128] bf16
    float* stack;      // [gridDim.x][gs][ATC_VAL_FLOATS]: o of the pending >= 5-leaf values
    int gs;
    unsigned long long wait_cycles;
    unsigned debug;    // TBIK_DEBUG_* test hooks
};

// 32 dims (chunk c of 4) of one row of a pending value, [dim/4][row][4] layout.
__device__ __forceinline__ void atc_ld32(const float* base, int c, int row, float (&w)[32]) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 x = *reinterpret_cast<const float4*>(base + ((size_t)(c * 8 + q) * ATC_BM + row) * 4);
        w[4 * q] = x.x;
        w[4 * q + 1] = x.y;
        w[4 * q + 2] = x.z;
        w[4 * q + 3] = x.w;
    }
}
__device__ __forceinline__ void atc_st32(float* base, int c, int row, const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(base + ((size_t)(c * 8 + q) * ATC_BM + row) * 4) =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

__device__ __forceinline__ float atc_f(float x) { return x; }
__device__ __forceinline__ float atc_f(uint32_t x) { return __uint_as_float(x); }

// out[k] = fma(b[k], eb, fl(a[k] * ea)): the left operand's product rounded,
// the right one's fused into the add; two lanes per instruction (each lane the
// IEEE result of the scalar operation).
template <typename TA, typename TB>
__device__ __forceinline__ void atc_comb(float (&out)[32], const TA (&a)[32], float ea, const TB (&b)[32], float eb) {
    const f2x ea2 = pk2(ea, ea), eb2 = pk2(eb, eb);
#pragma unroll
    for (int k = 0; k < 32; k += 2) {
        const f2x r = fma2(pk2(atc_f(b[k]), atc_f(b[k + 1])), eb2, mul2(pk2(atc_f(a[k]), atc_f(a[k + 1])), ea2));
        upk2(r, out[k], out[k + 1]);
    }
}
// The same rule for the running sums.
__device__ __forceinline__ float atc_comb1(float a, float ea, float b, float eb) {
    return __fmaf_rn(b, eb, __fmul_rn(a, ea));
}

// Combine factors of two summaries (a is the left operand): M and the two
// exponentials e = 2^(fl(m - M) * log2e) by the hardware exponential (1 for
// the side holding M).
__device__ __forceinline__ void atc_factors(float am, float bm, float& M, float& ea, float& eb) {
    const float log2e = 0x1.715476p+0f;
    M = (bm > am) ? bm : am;
    const bool finite = M != INFINITY;
    ea = (finite && am == M) ? 1.0f : ex2_hw(__fmul_rn(__fsub_rn(am, M), log2e));
    eb = (finite && bm == M) ? 1.0f : ex2_hw(__fmul_rn(__fsub_rn(bm, M), log2e));
}

// The k-th query tile of this CTA: the tiles are dealt out in rounds of
// gridDim.x, in alternating directions, so that every CTA's total of leaves
// stays close to the mean (the tiles are ordered longest first).
__device__ __forceinline__ int atc_sched(int k) {
    const int G = (int)gridDim.x, b = (int)blockIdx.x;
    return k * G + ((k & 1) ? G - 1 - b : b);
}

// Query tile t (longest first): position block qt and (batch, head) bh.
__device__ __forceinline__ void atc_tile(const AttTcParams& p, int t, int& qt, int& bh) {
    const int nbh = p.batch * p.heads;
    qt = p.ntq - 1 - t / nbh;
    bh = t - (t / nbh) * nbh;
}

__global__ void __launch_bounds__(ATC_THREADS, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    float* sSlot = reinterpret_cast<float*>(smem + ATC_OFF_SLOT);
    float* sX = reinterpret_cast<float*>(smem + ATC_OFF_X);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ATC_OFF_BAR);
    uint64_t* q_full = bars;           // Q tile landed
    uint64_t* q_empty = bars + 1;      // the tile's last S MMA retired
    uint64_t* k_full = bars + 2;       // K of a leaf landed
    uint64_t* k_empty = bars + 3;      // the leaf's S MMAs retired
    uint64_t* v_full = bars + 4;       // V of a leaf landed
    uint64_t* v_empty = bars + 5;      // the leaf's P V MMAs retired
    uint64_t* s_full = bars + 6;       // S of a leaf (both chunks) in TMEM
    uint64_t* p_full = bars + 7;       // P of a leaf written by the 8 epilogue warps
    uint64_t* o_full = bars + 8;       // [2] O of a leaf in TMEM
    uint64_t* o_empty = bars + 10;     // [2] O buffer released by the 8 epilogue warps
    uint64_t* done = bars + 12;        // every MMA issued by this CTA retired
    uint64_t* s_empty = bars + 13;     // S of a leaf read by the 8 epilogue warps
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t lim = p.wait_cycles;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        mbar_init(k_full, 1);
        mbar_init(k_empty, 1);
        mbar_init(v_full, 1);
        mbar_init(v_empty, 1);
        mbar_init(s_full, 1);
        mbar_init(p_full, ATC_EPI_WARPS);
        mbar_init(s_empty, ATC_EPI_WARPS);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&o_full[b], 1);
            mbar_init(&o_empty[b], ATC_EPI_WARPS);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, ATC_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            uint32_t gk = 0, gv = 0, nt = 0;  // K leaves, V leaves and tiles loaded so far by this CTA
            for (int t = atc_sched(0); t < p.tiles; t = atc_sched(++nt)) {
                int qt, bh;
                atc_tile(p, t, qt, bh);
                const int b = bh / p.heads, h = bh - b * p.heads;
                const int i0 = qt * ATC_BM;
                const int nl = qt + 1;  // leaves of the tile
                if (nt > 0 && !mbar_wait(q_empty, (nt - 1) & 1, abort_flag, lim)) goto producer_out;
                mbar_arrive_expect_tx(q_full, 2 * ATC_BM * 128);
                for (int sl = 0; sl < 2; ++sl)
                    tma_load_4d(smem + ATC_OFF_Q + sl * 16384, &tmQ, q_full, 64 * sl, h, i0, b);
                for (int l = 0; l <= nl; ++l) {
                    if (l < nl) {  // K of leaf l
                        if (gk >= 1 && !mbar_wait(k_empty, (gk - 1) & 1, abort_flag, lim)) goto producer_out;
                        mbar_arrive_expect_tx(k_full, 2 * 2 * ATC_CH * 128);
                        for (int ch = 0; ch < 2; ++ch)
                            for (int sl = 0; sl < 2; ++sl)
                                tma_load_4d(smem + ATC_OFF_K + ch * 16384 + sl * 8192, &tmK, k_full, 64 * sl, h,
                                            ATC_LEAF * l + ATC_CH * ch, b);
                        ++gk;
                    }
                    if (l >= 1) {  // V of leaf l - 1
                        if (gv >= 1 && !mbar_wait(v_empty, (gv - 1) & 1, abort_flag, lim)) goto producer_out;
                        mbar_arrive_expect_tx(v_full, 2 * 2 * ATC_CH * 128);
                        for (int ch = 0; ch < 2; ++ch)
                            for (int sl = 0; sl < 2; ++sl)
                                tma_load_4d(smem + ATC_OFF_V + ch * 16384 + sl * 8192, &tmV, v_full, 64 * sl, h,
                                            ATC_LEAF * (l - 1) + ATC_CH * ch, b);
                        ++gv;
                    }
                }
            }
        producer_out:
            // let the last copies land before the CTA can exit
            if (gk > 0) mbar_drain(k_full, (gk - 1) & 1, lim);
            if (gv > 0) mbar_drain(v_full, (gv - 1) & 1, lim);
            if (nt > 0) mbar_drain(q_full, (nt - 1) & 1, lim);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(ATC_BM, ATC_CH, 0, 0);
            const uint32_t idesc_o = idesc_bf16_f32(ATC_BM, ATC_HD, 0, 1);
            const uint32_t q_u = smem_u32(smem + ATC_OFF_Q);
            uint32_t g0 = 0, nt = 0;
            for (int t = atc_sched(0); t < p.tiles; t = atc_sched(++nt)) {
                int qt, bh;
                atc_tile(p, t, qt, bh);
                const int nl = qt + 1;
                if (!mbar_wait(q_full, nt & 1, abort_flag, lim)) goto mma_out;
                for (int l = 0; l <= nl; ++l) {
                    if (l < nl) {
                        const uint32_t g = g0 + l;
                        if (!mbar_wait(k_full, g & 1, abort_flag, lim)) goto mma_out;
                        // S was read by the softmax of leaf g - 1
                        if (g >= 1 && !mbar_wait(s_empty, (g - 1) & 1, abort_flag, lim)) goto mma_out;
                        tc_fence_after();
                        const uint64_t adesc = smem_desc_sw128(q_u, 16, 1024);
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch) {
                            const uint64_t bdesc =
                                smem_desc_sw128(smem_u32(smem + ATC_OFF_K + ch * 16384), 16, 1024);
#pragma unroll
                            for (int ks = 0; ks < 8; ++ks)
                                tc_mma(tmem_base + ATC_S_COL + 64 * ch,
                                       adesc + (uint64_t)((ks >> 2) * (16384 >> 4) + (ks & 3) * 2),
                                       bdesc + (uint64_t)((ks >> 2) * (8192 >> 4) + (ks & 3) * 2), idesc_s,
                                       ks ? 1u : 0u);
                        }
                        tc_commit(s_full);
                        tc_commit(k_empty);
                        if (l == nl - 1) tc_commit(q_empty);
                    }
                    if (l >= 1) {
                        const uint32_t g = g0 + l - 1, b = g & 1, ph = (g >> 1) & 1;
                        if (!mbar_wait(v_full, g & 1, abort_flag, lim)) goto mma_out;
                        if (!mbar_wait(p_full, g & 1, abort_flag, lim)) goto mma_out;  // P of leaf g written
                        if (g >= 2 && !mbar_wait(&o_empty[b], ph ^ 1, abort_flag, lim)) goto mma_out;
                        tc_fence_after();
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch) {
                            const uint64_t adesc = smem_desc_sw128(smem_u32(smem + ATC_OFF_P + ch * 16384), 16, 1024);
                            // V: MN-major, the two 64-dim atoms 8 KiB apart, 8-key groups 1 KiB apart
                            const uint64_t bdesc =
                                smem_desc_sw128(smem_u32(smem + ATC_OFF_V + ch * 16384), 8192, 1024);
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                tc_mma(tmem_base + ATC_O_COL + 128 * b, adesc + (uint64_t)(ks * 2),
                                       bdesc + (uint64_t)(ks * (2048 >> 4)), idesc_o, (ch | ks) ? 1u : 0u);
                        }
                        tc_commit(&o_full[b]);
                        tc_commit(v_empty);
                    }
                }
                g0 += nl;
            }
        mma_out:
            // every MMA retires before TMEM is released
            tc_commit(done);
            mbar_drain(done, 0, lim);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int qd = warp & 3;          // row quadrant: rows 32*qd .. 32*qd+31
        const int half = (warp - 2) >> 2;  // chunk h of each leaf, dims [64h, 64h+64)
        const int r = qd * 32 + lane;     // row of the tile
        const uint32_t tl = tmem_base + ((uint32_t)(qd * 32) << 16);
        const float log2e = 0x1.715476p+0f;
        const int bar_pair = 3 + qd;      // named barrier of this quadrant's two warps
        float cm0 = 0.f, cm1 = 0.f, cs0 = 0.f, cs1 = 0.f;  // (m, s) of the leaves in O buffers 0 and 1
        uint32_t g0 = 0;
        // A bounded wait that expires makes this warp skip its work from then
        // on; the pair's barrier (OR reduction) then takes both warps out
        // together, so neither waits there for one that has left.
        bool ab = false;
        float* stack = p.stack + (size_t)blockIdx.x * p.gs * ATC_VAL_FLOATS;
        // (m, s) of the L2 stack's values, per thread: both warps of a row
        // quadrant hold the same values, but a shared copy would race (a leaf
        // that pops a slot and pushes its result into it lets one warp write the
        // new value before the other has read the old one)
        float stk_m[ATC_MAX_GS], stk_s[ATC_MAX_GS];
        for (int k = 0, t = atc_sched(0); t < p.tiles; t = atc_sched(++k)) {
            int qt, bh;
            atc_tile(p, t, qt, bh);
            const int bb = bh / p.heads, hh = bh - bb * p.heads;
            const int i0 = qt * ATC_BM;
            const int i = i0 + r;   // this row's query position
            const int nl = qt + 1;  // leaves of every row of the tile
            // pending summaries: single (its O buffer), 2 (TMEM slot), 3-4 (shared), >= 5 (L2 stack)
            float m1 = 0.f, s1 = 0.f, m2 = 0.f, s2 = 0.f, m34 = 0.f, s34 = 0.f;
            uint32_t single_b = 0;
            int gsp = 0;
            uint32_t lane_code = 0;  // operation code of leaf 32*(l1/32) + lane of this tile's tree
            for (int l = 0; l <= nl; ++l) {
                if (l < nl) {
                    // ---------------- softmax of leaf l (this warp: chunk `half`)
                    const uint32_t g = g0 + l, b = g & 1;
                    uint32_t okw = 1;
                    if (lane == 0 && !ab) okw = mbar_wait(s_full, g & 1, abort_flag, lim) ? 1u : 0u;
                    ab = ab || __shfl_sync(0xffffffffu, okw, 0) == 0;
                    float* xs = sX + (b * 2) * ATC_BM;
                    float m = -INFINITY;
                    if (!ab) {
                    tc_fence_after();
                    const int key0 = ATC_LEAF * l;
                    const int kh = key0 + ATC_CH * half;        // first key of this warp's chunk
                    const int kx = key0 + ATC_CH * (half ^ 1);  // first key of the other chunk
                    // every key of the leaf precedes every row of the tile: no mask
                    const bool full = l < nl - 1;
                    // the other chunk's maximum, on the raw scores: fl(x * scale) is
                    // non-decreasing in x, so scaling the maximum gives the maximum of
                    // the scaled scores exactly
                    {
                        uint32_t sx[64];
                        tmem_ld64_nowait(tl + ATC_S_COL + 64 * (half ^ 1), sx);
                        tmem_wait_ld64(sx);
                        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                        if (full) {
#pragma unroll
                            for (int k = 0; k < 64; k += 8)
#pragma unroll
                                for (int q = 0; q < 4; ++q)
                                    mq[q] = fmax3(mq[q], __uint_as_float(sx[k + 2 * q]), __uint_as_float(sx[k + 2 * q + 1]));
                        } else {
#pragma unroll
                            for (int k = 0; k < 64; ++k)
                                if (kx + k <= i) mq[k & 3] = fmaxf(mq[k & 3], __uint_as_float(sx[k]));
                        }
                        m = __fmul_rn(fmax3(fmaxf(mq[0], mq[1]), mq[2], mq[3]), p.scale);
                    }
                    uint32_t so[64];
                    tmem_ld64_nowait(tl + ATC_S_COL + 64 * half, so);
                    tmem_wait_ld64(so);
                    // S is in registers: the scores of the next leaf may overwrite it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s_empty);
                    float vo[64];
                    const f2x sc2 = pk2(p.scale, p.scale);
#pragma unroll
                    for (int k = 0; k < 64; k += 2)
                        upk2(mul2(pk2(__uint_as_float(so[k]), __uint_as_float(so[k + 1])), sc2), vo[k], vo[k + 1]);
                    {
                        float mq[4] = {m, -INFINITY, -INFINITY, -INFINITY};
                        if (full) {
#pragma unroll
                            for (int k = 0; k < 64; k += 8)
#pragma unroll
                                for (int q = 0; q < 4; ++q) mq[q] = fmax3(mq[q], vo[k + 2 * q], vo[k + 2 * q + 1]);
                        } else {
#pragma unroll
                            for (int k = 0; k < 64; ++k)
                                if (kh + k <= i) mq[k & 3] = fmaxf(mq[k & 3], vo[k]);
                        }
                        m = fmax3(fmaxf(mq[0], mq[1]), mq[2], mq[3]);
                    }
                    const float ml = -__fmul_rn(m, log2e);
                    const f2x l2 = pk2(log2e, log2e), ml2 = pk2(ml, ml);
                    float cq[4] = {0.f, 0.f, 0.f, 0.f};  // sums over the keys k = q (mod 4)
                    uint32_t pk[32];                     // this chunk's 64 bf16 p, packed in pairs
                    // both weights of a pair rounded to bf16 in one conversion; the
                    // sums take the rounded values (0 for a key after the row)
                    if (full) {
#pragma unroll
                        for (int k2 = 0; k2 < 32; ++k2) {
                            const int j = 2 * k2;
                            float y0, y1;
                            upk2(fma2(pk2(vo[j], vo[j + 1]), l2, ml2), y0, y1);
                            const uint32_t w = pack_bf2(ex2_hw(y0), ex2_hw(y1));
                            pk[k2] = w;
                            cq[j & 3] = __fadd_rn(cq[j & 3], __uint_as_float(w << 16));
                            cq[(j + 1) & 3] = __fadd_rn(cq[(j + 1) & 3], __uint_as_float(w & 0xffff0000u));
                        }
                    } else {
#pragma unroll
                        for (int k2 = 0; k2 < 32; ++k2) {
                            const int j = 2 * k2;
                            float y0, y1;
                            upk2(fma2(pk2(vo[j], vo[j + 1]), l2, ml2), y0, y1);
                            uint32_t w = pack_bf2(ex2_hw(y0), ex2_hw(y1));
                            if (kh + j > i) w &= 0xffff0000u;
                            if (kh + j + 1 > i) w &= 0x0000ffffu;
                            pk[k2] = w;
                            cq[j & 3] = __fadd_rn(cq[j & 3], __uint_as_float(w << 16));
                            cq[(j + 1) & 3] = __fadd_rn(cq[(j + 1) & 3], __uint_as_float(w & 0xffff0000u));
                        }
                    }
                    // P of the previous leaf is read by its P V MMA, which is issued
                    // after the scores of this leaf: wait for that MMA before
                    // overwriting P (the same phase the tree step waits for later)
                    if (g >= 1) {
                        const uint32_t gp = g - 1;
                        uint32_t okp = 1;
                        if (lane == 0) okp = mbar_wait(&o_full[gp & 1], (gp >> 1) & 1, abort_flag, lim) ? 1u : 0u;
                        ab = __shfl_sync(0xffffffffu, okp, 0) == 0;
                    }
                    if (!ab) {
                    // P row r of this chunk: eight 16-byte pieces at swizzled positions
                    uint8_t* prow = smem + ATC_OFF_P + half * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint4*>(prow + ((j ^ (r & 7)) * 16)) =
                            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                    xs[half * ATC_BM + r] = __fadd_rn(__fadd_rn(cq[0], cq[1]), __fadd_rn(cq[2], cq[3]));
                    fence_proxy_async_smem();
                    tc_fence_before();
                    }
                    }
                    if (named_barrier_or(bar_pair, 64, ab)) goto epi_out;
                    const float s_l = __fadd_rn(xs[r], xs[ATC_BM + r]);  // keys 0..63, then 64..127
                    if (b) { cm1 = m; cs1 = s_l; } else { cm0 = m; cs0 = s_l; }
                    __syncwarp();
                    if (lane == 0 && !(p.debug & TBIK_DEBUG_WITHHOLD_ACC_ARRIVE)) mbar_arrive(p_full);
                }
                if (l >= 1) {
                    // ---------------- tree step of leaf l - 1
                    const int l1 = l - 1;
                    const uint32_t g = g0 + l1, b = g & 1, ph = (g >> 1) & 1;
                    // O of leaf l - 1 landed: the softmax of leaf l has waited for it
                    // before writing P (or this warp left at the pair's barrier), so
                    // only the tile's last leaf waits here
                    if (l == nl) {
                        uint32_t okw = 1;
                        if (lane == 0 && !ab) okw = mbar_wait(&o_full[b], ph, abort_flag, lim) ? 1u : 0u;
                        ab = ab || __shfl_sync(0xffffffffu, okw, 0) == 0;
                    }
                    if (ab) continue;  // left at the pair's next barrier (or at the end)
                    tc_fence_after();
                    // the lanes walk the tree for 32 leaves at once; each leaf's code
                    // is then one shuffle away
                    if ((l1 & 31) == 0) {
                        const int lj = l1 + lane;
                        lane_code = lj < nl ? encode_leaf_ops(leaf_ops(nl, lj)) : 0u;
                    }
                    const uint32_t code = __shfl_sync(0xffffffffu, lane_code, l1 & 31);
                    const bool p1 = code & 1, p2 = (code >> 1) & 1, pm = (code >> 2) & 1;
                    const int nb = (code >> 3) & 31;
                    const int cls = (code >> 8) & 3;
                    const bool final_ = (code >> 10) & 1;
                    const uint32_t oc = tl + ATC_O_COL + 128 * b + 64 * half;  // this half's 64 dims
                    const float cmb = b ? cm1 : cm0, csb = b ? cs1 : cs0;
                    if (!final_ && cls == 0) {  // a single leaf waits in its O buffer
                        single_b = b;
                        m1 = cmb;
                        s1 = csb;
                        continue;
                    }
                    // phase 1: the leaf (and the single it pops) into v; release the buffers
                    float v[2][32];
                    float vm = cmb, vs = csb;
                    if (p1) {
                        float M, ea, eb;
                        atc_factors(m1, vm, M, ea, eb);
                        const uint32_t os = tl + ATC_O_COL + 128 * single_b + 64 * half;
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            uint32_t ra[32], rb[32];
                            tmem_ld32x2(os + 32 * cc, ra, oc + 32 * cc, rb);
                            atc_comb(v[cc], ra, ea, rb, eb);
                        }
                        vs = atc_comb1(s1, ea, vs, eb);
                        vm = M;
                    } else {
                        uint32_t ro[64];
                        tmem_ld64_nowait(oc, ro);
                        tmem_wait_ld64(ro);
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            v[0][k] = __uint_as_float(ro[k]);
                            v[1][k] = __uint_as_float(ro[32 + k]);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&o_empty[b]);
                        if (p1) mbar_arrive(&o_empty[single_b]);
                    }
                    // phase 2: the other pops (smallest first), each the left operand
                    if (p2) {
                        float M, ea, eb;
                        atc_factors(m2, vm, M, ea, eb);
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            float w[32];
                            tmem_ld32(tl + ATC_SLOT_COL + 64 * half + 32 * cc, w);
                            atc_comb(v[cc], w, ea, v[cc], eb);
                        }
                        vs = atc_comb1(s2, ea, vs, eb);
                        vm = M;
                    }
                    if (pm) {
                        float M, ea, eb;
                        atc_factors(m34, vm, M, ea, eb);
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            float w[32];
                            atc_ld32(sSlot, 2 * half + cc, r, w);
                            atc_comb(v[cc], w, ea, v[cc], eb);
                        }
                        vs = atc_comb1(s34, ea, vs, eb);
                        vm = M;
                    }
                    for (int q = 0; q < nb; ++q) {
                        const int slot = gsp - 1 - q;
                        const float* sl = stack + (size_t)slot * ATC_VAL_FLOATS;
                        float M, ea, eb;
                        atc_factors(stk_m[slot], vm, M, ea, eb);
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            float w[32];
                            atc_ld32(sl, 2 * half + cc, r, w);
                            atc_comb(v[cc], w, ea, v[cc], eb);
                        }
                        vs = atc_comb1(stk_s[slot], ea, vs, eb);
                        vm = M;
                    }
                    gsp -= nb;
                    if (!final_) {
                        if (cls == 1) {
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc) tmem_st32_nowait(tl + ATC_SLOT_COL + 64 * half + 32 * cc, v[cc]);
                            tmem_wait_st();
                            m2 = vm;
                            s2 = vs;
                        } else if (cls == 2) {
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc) atc_st32(sSlot, 2 * half + cc, r, v[cc]);
                            m34 = vm;
                            s34 = vs;
                        } else {
                            float* sl = stack + (size_t)gsp * ATC_VAL_FLOATS;
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc) atc_st32(sl, 2 * half + cc, r, v[cc]);
                            stk_m[gsp] = vm;
                            stk_s[gsp] = vs;
                            ++gsp;
                        }
                    } else if (i < p.seq) {
                        // out[b][i][h][64h .. 64h+63] = bf16(o * fl(1/s))
                        uint16_t* orow = p.out + (((size_t)bb * p.seq + i) * p.heads + hh) * ATC_HD + 64 * half;
                        const float rs = __frcp_rn(vs);
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                            for (int q8 = 0; q8 < 4; ++q8) {
                                float o8[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) o8[e] = __fmul_rn(v[cc][8 * q8 + e], rs);
                                *reinterpret_cast<uint4*>(orow + 32 * cc + 8 * q8) = pack8(o8);
                            }
                    }
                }
            }
            g0 += nl;
        }
    epi_out:;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, ATC_TMEM_COLS);
    }
}

}  // namespace tbik
