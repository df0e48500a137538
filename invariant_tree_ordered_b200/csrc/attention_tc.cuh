// Tensor-core causal attention with the key reduction in tree order (TC mode).
//
// Source: TBIK summary page, 技术框架 (one hierarchical binary tree for every
// reduction, so the result does not depend on how the work is split).  The
// structure is the exact mode's (attention.cuh): keys in chunks of 64
// positions, each chunk reduced to a (max, sum, weighted value sum) summary,
// the summaries of chunks 0..floor(i/64) combined by the halving tree.  What
// differs is how one chunk is computed:
//   scores  s_j = fl(S_ij * scale), S = Q K^T on the tensor cores (tcgen05,
//           bf16 operands, fp32 accumulation in TMEM in the hardware's order);
//   chunk   m = max over the chunk's keys j <= i;
//           p_j = bf16(2^(s_j*log2e - m*log2e)) with the hardware exponential,
//           0 for j > i; s = (ascending sum of p_j over keys 0..31) +
//           (ascending sum over keys 32..63), of the rounded p_j;
//           o = P V on the tensor cores (the bf16 p_j as A, V as B);
//   combine the exact mode's rule: M = max, e = exp(m - M) by the library's
//           exp specification (1 for the side holding M), s = s*e + s'*e',
//           o = o*e + o'*e' (products rounded separately);
//   output  bf16(o[d] / s).
// A row's result depends only on its query, the keys and values at positions
// <= i and its fixed chunk tree, never on the batch composition, the other
// rows of its tile or how heads are split across devices.
//
// One CTA per SM, persistent over 128-row query tiles of one (batch, head),
// the longest tiles first; 320 threads:
//   warp 0     TMA producer: the Q tile (two 64-dim slices, K-major, 128-byte
//              swizzle) and per chunk K (same layout, 64 rows) and V (MN-major:
//              two 64-dim atoms of 64 keys) into a 2-stage ring
//   warp 1     TMEM allocator + MMA issuer: S_c = Q K_c^T (M=128, N=64) into
//              S[c%2], then O_{c-1} = P_{c-1} V_{c-1} (M=128, N=128, K=64)
//              into O[(c-1)%2]
//   warps 2-9  epilogue: warp w owns rows 32*(w%4).. and half h = (w-2)/4:
//              keys [32h, 32h+32) of each chunk's softmax and head dims
//              [64h, 64h+64) of the tree.  Loop: softmax of chunk c (writes
//              P_c), then the tree step of chunk c-1, so the MMA of O_c runs
//              while the tree of chunk c-1 is evaluated.
// A tile starts at a multiple of 128: its rows 0..63 have i0/64 + 1 chunks,
// rows 64..127 one more, so the tree walk is the same for all lanes of a warp.
// Pending chunk summaries wait by size: a single chunk in its O buffer (the
// next chunk consumes it), 2 chunks in a TMEM slot, 3-4 in shared memory,
// >= 5 in a per-CTA stack in global memory that stays in L2.
#pragma once

#include "device_common.cuh"

namespace tbik {

constexpr int ATC_BM = 128;  // query rows per tile
constexpr int ATC_CH = 64;   // keys per chunk
constexpr int ATC_HD = 128;  // head dimension
constexpr int ATC_EPI_WARPS = 8;
constexpr int ATC_THREADS = 32 * (2 + ATC_EPI_WARPS);
constexpr int ATC_TMEM_COLS = 512;
constexpr uint32_t ATC_S_COL = 0, ATC_O_COL = 128, ATC_SLOT_COL = 384;
constexpr int ATC_VAL_FLOATS = ATC_BM * ATC_HD;  // one pending o value of the tile
constexpr int ATC_MAX_GS = 8;  // L2 stack depth bound (chunk trees of up to 256 chunks need 5)
// shared memory (from a 1024-byte aligned base); V first, so that every
// descriptor-addressed read stays inside the allocation
constexpr int ATC_OFF_V = 0;             // [2] 64 keys x 128 dims bf16, two 8 KiB atoms
constexpr int ATC_OFF_K = 32768;         // [2] 64 keys x 128 dims, two 8 KiB slices
constexpr int ATC_OFF_Q = 65536;         // 128 rows x 128 dims, two 16 KiB slices
constexpr int ATC_OFF_P = 98304;         // [2] 128 rows x 64 keys bf16
constexpr int ATC_OFF_SLOT = 131072;     // pending 3-4 chunk value, fp32 [dim/4][row][4]
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
    float* stack;      // [gridDim.x][gs][ATC_VAL_FLOATS]: o of the pending >= 5-chunk values
    int gs;
    unsigned long long wait_cycles;
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

// Combine factors of two summaries (a is the left operand): M and the two
// exponentials of the exact mode's rule.
__device__ __forceinline__ void atc_factors(float am, float bm, float& M, float& ea, float& eb) {
    M = (bm > am) ? bm : am;
    const bool finite = M != INFINITY;
    ea = (finite && am == M) ? 1.0f : exp_spec(__fsub_rn(am, M));
    eb = (finite && bm == M) ? 1.0f : exp_spec(__fsub_rn(bm, M));
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
    uint64_t* kv_full = bars + 2;      // [2] K and V of a chunk landed
    uint64_t* kv_empty = bars + 4;     // [2] the chunk's MMAs retired
    uint64_t* s_full = bars + 6;       // [2] S of a chunk in TMEM
    uint64_t* p_full = bars + 8;       // [2] P of a chunk written (S read) by the 8 epilogue warps
    uint64_t* o_full = bars + 10;      // [2] O of a chunk in TMEM
    uint64_t* o_empty = bars + 12;     // [2] O buffer released by the 8 epilogue warps
    uint64_t* done = bars + 14;        // every MMA issued by this CTA retired
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t lim = p.wait_cycles;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&kv_full[b], 1);
            mbar_init(&kv_empty[b], 1);
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], ATC_EPI_WARPS);
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
            uint32_t g = 0, nt = 0;  // chunks and tiles loaded so far by this CTA
            for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++nt) {
                int qt, bh;
                atc_tile(p, t, qt, bh);
                const int b = bh / p.heads, h = bh - b * p.heads;
                const int i0 = qt * ATC_BM;
                const int nc = i0 / ATC_CH + 2;
                if (nt > 0 && !mbar_wait(q_empty, (nt - 1) & 1, abort_flag, lim)) goto producer_out;
                mbar_arrive_expect_tx(q_full, 2 * ATC_BM * 128);
                for (int sl = 0; sl < 2; ++sl)
                    tma_load_4d(smem + ATC_OFF_Q + sl * 16384, &tmQ, q_full, 64 * sl, h, i0, b);
                for (int c = 0; c < nc; ++c, ++g) {
                    const int s = g & 1;
                    if (g >= 2 && !mbar_wait(&kv_empty[s], ((g >> 1) - 1) & 1, abort_flag, lim)) goto producer_out;
                    mbar_arrive_expect_tx(&kv_full[s], 2 * 2 * ATC_CH * 128);
                    for (int sl = 0; sl < 2; ++sl) {
                        tma_load_4d(smem + ATC_OFF_K + s * 16384 + sl * 8192, &tmK, &kv_full[s], 64 * sl, h,
                                    ATC_CH * c, b);
                        tma_load_4d(smem + ATC_OFF_V + s * 16384 + sl * 8192, &tmV, &kv_full[s], 64 * sl, h,
                                    ATC_CH * c, b);
                    }
                }
            }
        producer_out:
            // let the last copies land before the CTA can exit
            if (g > 0) mbar_drain(&kv_full[(g - 1) & 1], ((g - 1) >> 1) & 1, lim);
            if (g > 1) mbar_drain(&kv_full[(g - 2) & 1], ((g - 2) >> 1) & 1, lim);
            if (nt > 0) mbar_drain(q_full, (nt - 1) & 1, lim);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(ATC_BM, ATC_CH, 0, 0);
            const uint32_t idesc_o = idesc_bf16_f32(ATC_BM, ATC_HD, 0, 1);
            const uint32_t q_u = smem_u32(smem + ATC_OFF_Q);
            uint32_t g0 = 0, nt = 0;
            for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++nt) {
                int qt, bh;
                atc_tile(p, t, qt, bh);
                const int nc = (qt * ATC_BM) / ATC_CH + 2;
                if (!mbar_wait(q_full, nt & 1, abort_flag, lim)) goto mma_out;
                for (int c = 0; c <= nc; ++c) {
                    if (c < nc) {
                        const uint32_t g = g0 + c, b = g & 1, ph = (g >> 1) & 1;
                        if (!mbar_wait(&kv_full[b], ph, abort_flag, lim)) goto mma_out;
                        // S[b] was read by the softmax of chunk g - 2
                        if (g >= 2 && !mbar_wait(&p_full[b], ph ^ 1, abort_flag, lim)) goto mma_out;
                        tc_fence_after();
                        const uint64_t adesc = smem_desc_sw128(q_u, 16, 1024);
                        const uint64_t bdesc = smem_desc_sw128(smem_u32(smem + ATC_OFF_K + b * 16384), 16, 1024);
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks)
                            tc_mma(tmem_base + ATC_S_COL + 64 * b,
                                   adesc + (uint64_t)((ks >> 2) * (16384 >> 4) + (ks & 3) * 2),
                                   bdesc + (uint64_t)((ks >> 2) * (8192 >> 4) + (ks & 3) * 2), idesc_s, ks ? 1u : 0u);
                        tc_commit(&s_full[b]);
                        if (c == nc - 1) tc_commit(q_empty);
                    }
                    if (c >= 1) {
                        const uint32_t g = g0 + c - 1, b = g & 1, ph = (g >> 1) & 1;
                        if (!mbar_wait(&p_full[b], ph, abort_flag, lim)) goto mma_out;
                        if (g >= 2 && !mbar_wait(&o_empty[b], ph ^ 1, abort_flag, lim)) goto mma_out;
                        tc_fence_after();
                        const uint64_t adesc = smem_desc_sw128(smem_u32(smem + ATC_OFF_P + b * 16384), 16, 1024);
                        // V: MN-major, the two 64-dim atoms 8 KiB apart, 8-key groups 1 KiB apart
                        const uint64_t bdesc = smem_desc_sw128(smem_u32(smem + ATC_OFF_V + b * 16384), 8192, 1024);
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            tc_mma(tmem_base + ATC_O_COL + 128 * b, adesc + (uint64_t)(ks * 2),
                                   bdesc + (uint64_t)(ks * (2048 >> 4)), idesc_o, ks ? 1u : 0u);
                        tc_commit(&o_full[b]);
                        tc_commit(&kv_empty[b]);
                    }
                }
                g0 += nc;
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
        const int half = (warp - 2) >> 2;  // keys [32h, 32h+32), dims [64h, 64h+64)
        const int r = qd * 32 + lane;     // row of the tile
        const uint32_t tl = tmem_base + ((uint32_t)(qd * 32) << 16);
        const float log2e = 0x1.715476p+0f;
        const int bar_pair = 3 + qd;      // named barrier of this quadrant's two warps
        float cm0 = 0.f, cm1 = 0.f, cs0 = 0.f, cs1 = 0.f;  // (m, s) of the chunks in buffers 0 and 1
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
        for (int t = blockIdx.x; t < p.tiles; t += gridDim.x) {
            int qt, bh;
            atc_tile(p, t, qt, bh);
            const int bb = bh / p.heads, hh = bh - bb * p.heads;
            const int i0 = qt * ATC_BM;
            const int i = i0 + r;                      // this row's query position
            const int nc = i0 / ATC_CH + 2;            // chunks of the tile
            const int ncr = (qd < 2) ? nc - 1 : nc;    // chunks of this row's tree
            // pending summaries: single (its O buffer), 2 (TMEM slot), 3-4 (shared), >= 5 (L2 stack)
            float m1 = 0.f, s1 = 0.f, m2 = 0.f, s2 = 0.f, m34 = 0.f, s34 = 0.f;
            uint32_t single_b = 0;
            int gsp = 0;
            for (int c = 0; c <= nc; ++c) {
                if (c < nc) {
                    // ---------------- softmax of chunk c
                    const uint32_t g = g0 + c, b = g & 1, ph = (g >> 1) & 1;
                    uint32_t okw = 1;
                    if (lane == 0 && !ab) okw = mbar_wait(&s_full[b], ph, abort_flag, lim) ? 1u : 0u;
                    ab = ab || __shfl_sync(0xffffffffu, okw, 0) == 0;
                    float* xs = sX + (b * 2) * ATC_BM;
                    if (!ab) {
                    tc_fence_after();
                    uint32_t sr[64];
                    tmem_ld64_nowait(tl + ATC_S_COL + 64 * b, sr);
                    tmem_wait_ld64(sr);
                    float m = -INFINITY, sh = 0.0f;
                    uint32_t pk[16];  // this half's 32 bf16 p, packed in pairs
                    if (c < ncr) {
                        const int key0 = ATC_CH * c;
#pragma unroll
                        for (int k = 0; k < 64; ++k) {
                            const float sv = __fmul_rn(__uint_as_float(sr[k]), p.scale);
                            sr[k] = __float_as_uint(sv);
                            if (key0 + k <= i) m = fmaxf(m, sv);
                        }
                        const float ml = -__fmul_rn(m, log2e);
                        const int kh = key0 + 32 * half;  // first key of this half
#pragma unroll
                        for (int k2 = 0; k2 < 16; ++k2) {
                            float pv[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int j = 2 * k2 + e;
                                const float sj = __uint_as_float(half ? sr[32 + j] : sr[j]);
                                const float x = ex2_hw(__fmaf_rn(sj, log2e, ml));
                                pv[e] = (kh + j <= i) ? bf2f(f2bf(x)) : 0.0f;
                                sh = __fadd_rn(sh, pv[e]);
                            }
                            pk[k2] = pack_bf2(pv[0], pv[1]);
                        }
                    } else {
#pragma unroll
                        for (int k2 = 0; k2 < 16; ++k2) pk[k2] = 0u;
                    }
                    // P row r, keys [32h, 32h+32): four 16-byte chunks at swizzled positions
                    uint8_t* prow = smem + ATC_OFF_P + b * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int ch = (4 * half + j) ^ (r & 7);
                        *reinterpret_cast<uint4*>(prow + ch * 16) =
                            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                    }
                    xs[half * ATC_BM + r] = sh;
                    if (b) cm1 = m; else cm0 = m;
                    fence_proxy_async_smem();
                    tc_fence_before();
                    }
                    if (named_barrier_or(bar_pair, 64, ab)) goto epi_out;
                    const float s_c = __fadd_rn(xs[r], xs[ATC_BM + r]);  // keys 0..31, then 32..63
                    if (b) cs1 = s_c; else cs0 = s_c;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&p_full[b]);
                }
                if (c >= 1) {
                    // ---------------- tree step of chunk c - 1
                    const int c1 = c - 1;
                    const uint32_t g = g0 + c1, b = g & 1, ph = (g >> 1) & 1;
                    uint32_t okw = 1;
                    if (lane == 0 && !ab) okw = mbar_wait(&o_full[b], ph, abort_flag, lim) ? 1u : 0u;
                    ab = ab || __shfl_sync(0xffffffffu, okw, 0) == 0;
                    if (ab) continue;  // left at the pair's next barrier (or at the end)
                    tc_fence_after();
                    if (c1 >= ncr) {  // past this row's last chunk: release the buffer only
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&o_empty[b]);
                        continue;
                    }
                    const uint32_t code = encode_leaf_ops(leaf_ops(ncr, c1));
                    const bool p1 = code & 1, p2 = (code >> 1) & 1, pm = (code >> 2) & 1;
                    const int nb = (code >> 3) & 31;
                    const int cls = (code >> 8) & 3;
                    const bool final_ = (code >> 10) & 1;
                    const uint32_t oc = tl + ATC_O_COL + 128 * b + 64 * half;  // this half's 64 dims
                    const float cmb = b ? cm1 : cm0, csb = b ? cs1 : cs0;
                    if (!final_ && cls == 0) {  // a single chunk waits in its O buffer
                        single_b = b;
                        m1 = cmb;
                        s1 = csb;
                        continue;
                    }
                    // phase 1: the chunk (and the single it pops) into v; release the buffers
                    float v[2][32];
                    float vm = cmb, vs = csb;
                    if (p1) {
                        float M, ea, eb;
                        atc_factors(m1, vm, M, ea, eb);
                        const uint32_t os = tl + ATC_O_COL + 128 * single_b + 64 * half;
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            uint32_t ra[32], rb[32];
                            tmem_ld32_nowait(os + 32 * cc, ra);
                            tmem_ld32_nowait(oc + 32 * cc, rb);
                            tmem_wait_ld(ra);
                            tie32(rb);
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                v[cc][k] = __fadd_rn(__fmul_rn(__uint_as_float(ra[k]), ea),
                                                     __fmul_rn(__uint_as_float(rb[k]), eb));
                        }
                        vs = __fadd_rn(__fmul_rn(s1, ea), __fmul_rn(vs, eb));
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
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                v[cc][k] = __fadd_rn(__fmul_rn(w[k], ea), __fmul_rn(v[cc][k], eb));
                        }
                        vs = __fadd_rn(__fmul_rn(s2, ea), __fmul_rn(vs, eb));
                        vm = M;
                    }
                    if (pm) {
                        float M, ea, eb;
                        atc_factors(m34, vm, M, ea, eb);
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            float w[32];
                            atc_ld32(sSlot, 2 * half + cc, r, w);
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                v[cc][k] = __fadd_rn(__fmul_rn(w[k], ea), __fmul_rn(v[cc][k], eb));
                        }
                        vs = __fadd_rn(__fmul_rn(s34, ea), __fmul_rn(vs, eb));
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
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                v[cc][k] = __fadd_rn(__fmul_rn(w[k], ea), __fmul_rn(v[cc][k], eb));
                        }
                        vs = __fadd_rn(__fmul_rn(stk_s[slot], ea), __fmul_rn(vs, eb));
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
                        // out[b][i][h][64h .. 64h+63] = bf16(o / s)
                        uint16_t* orow = p.out + (((size_t)bb * p.seq + i) * p.heads + hh) * ATC_HD + 64 * half;
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                            for (int q8 = 0; q8 < 4; ++q8) {
                                float o8[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) o8[e] = __fdiv_rn(v[cc][8 * q8 + e], vs);
                                *reinterpret_cast<uint4*>(orow + 32 * cc + 8 * q8) = pack8(o8);
                            }
                    }
                }
            }
            g0 += nc;
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
