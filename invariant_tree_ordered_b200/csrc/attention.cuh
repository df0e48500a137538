// Causal attention with the reduction over keys in tree order: the keys of a
// query are cut into fixed chunks of 64 positions, each chunk is reduced to a
// (max, sum of exponentials, weighted value sum) summary, and the summaries are
// combined by the same halving tree as every other reduction here (TBIK
// summary page, 技术框架: one hierarchical binary tree for every reduction, so
// the result does not depend on how the work is split).  Nothing depends on
// the batch composition or on how heads are split across devices.
//
// One warp per query (batch b, head h, position i).  Lane l owns head
// dimensions [DPL*l, DPL*l + DPL) of the value sums and the keys l, l+32 of
// each chunk:
//   score   s_j = fl(dot(q_i, k_j) * scale), the dot accumulated over the head
//           dimension in ascending order with fma from +0;
//   chunk   m = max of its scores (keys <= i); p_j = exp(s_j - m), 0 past i;
//           s = the tree over the chunk's 64 slots of p (xor butterflies over
//           each half of 32 slots, then the two halves); o[d] = ascending sum over the
//           chunk's keys of p_j * v_j[d] by fma from +0;
//   combine (m,s,o) with (m',s',o'): M = max, e = exp(m - M), e' = exp(m' - M),
//           s = s*e + s'*e', o = o*e + o'*e' (products rounded on their own);
//           chunks 0..floor(i/64) by the halving tree, streamed with a stack;
//   output  bf16(o[d] / s).
#pragma once

#include "device_common.cuh"

namespace tbik {

constexpr int ATT_CHUNK = 64;
constexpr int ATT_WARPS = 8;

template <int DPL>
struct AttNode {
    float m, s, o[DPL];
};

template <int DPL>
__device__ __forceinline__ AttNode<DPL> att_combine(const AttNode<DPL>& a, const AttNode<DPL>& b) {
    AttNode<DPL> r;
    r.m = (b.m > a.m) ? b.m : a.m;
    // the side holding the max has the factor exp(+0) = 1 exactly
    const bool finite = r.m != INFINITY;
    const float ea = (finite && a.m == r.m) ? 1.0f : exp_spec(__fsub_rn(a.m, r.m));
    const float eb = (finite && b.m == r.m) ? 1.0f : exp_spec(__fsub_rn(b.m, r.m));
    r.s = __fadd_rn(__fmul_rn(a.s, ea), __fmul_rn(b.s, eb));
#pragma unroll
    for (int d = 0; d < DPL; ++d) r.o[d] = __fadd_rn(__fmul_rn(a.o[d], ea), __fmul_rn(b.o[d], eb));
    return r;
}

// A warp takes QPW consecutive query positions (independent fma chains for
// the same key rows); the ATT_WARPS warps of a CTA take ATT_WARPS * QPW
// consecutive positions of one (b, h) and share each key chunk: its K rows
// (padded to HD/2 + 1 words, so the 32 rows a warp reads at once fall in 32
// different banks) and V rows are staged in shared memory once per CTA.
// Lane l scores keys l and l + 32 of a chunk; the tree over the 64 slots is
// the xor butterfly on each half followed by the top-level add of the halves.
constexpr int ATT_QPW = 2;
constexpr int ATT_QPB = ATT_WARPS * ATT_QPW;  // query positions per CTA

template <int DPL>
__global__ void __launch_bounds__(ATT_WARPS * 32)
    attention_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                     uint16_t* out, int batch, int seq, int heads, float scale) {
    constexpr int HD = 32 * DPL;
    constexpr int WPR = HD / 2;    // 32-bit words (bf16 pairs) per row
    constexpr int KSTR = WPR + 1;  // padded K row stride in words
    constexpr int Q = ATT_QPW;
    __shared__ uint32_t sK[ATT_CHUNK * KSTR];
    __shared__ __align__(16) uint32_t sV[ATT_CHUNK * WPR];
    __shared__ __align__(8) float2 sQ[ATT_WARPS][Q][WPR];  // the queries widened to fp32 (exact), pairs
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int qblocks = (seq + ATT_QPB - 1) / ATT_QPB;
    const int bh = blockIdx.x / qblocks;
    const int i0 = (blockIdx.x - bh * qblocks) * ATT_QPB;
    const int b = bh / heads, h = bh - b * heads;
    const size_t row_stride = (size_t)heads * HD;  // elements between positions
    const size_t base = (size_t)b * seq * row_stride + (size_t)h * HD;
    int qi[Q], nc[Q];
#pragma unroll
    for (int x = 0; x < Q; ++x) {
        qi[x] = i0 + Q * warp + x;
        nc[x] = qi[x] < seq ? qi[x] / ATT_CHUNK + 1 : 0;
        if (qi[x] < seq)
            for (int w = lane; w < WPR; w += 32) {
                const uint32_t qw = __ldg(reinterpret_cast<const uint32_t*>(q + base + (size_t)qi[x] * row_stride) + w);
                sQ[warp][x][w] = make_float2(__uint_as_float(qw << 16), __uint_as_float(qw & 0xffff0000u));
            }
    }
    const int last = min(i0 + ATT_QPB - 1, seq - 1);
    const int nc_all = last / ATT_CHUNK + 1;  // chunks any query of this CTA needs
    const int qlast = min(qi[Q - 1], seq - 1);  // this warp's last position (qi[0] < seq if any is active)
    const int nc_w = qi[0] < seq ? qlast / ATT_CHUNK + 1 : 0;  // chunks this warp needs
    AttNode<DPL> stk[Q][8];
    int sp[Q];
    AttNode<DPL> fin[Q];
#pragma unroll
    for (int x = 0; x < Q; ++x) {
        sp[x] = 0;
        fin[x].m = 0.0f;
        fin[x].s = 1.0f;
#pragma unroll
        for (int d = 0; d < DPL; ++d) fin[x].o[d] = 0.0f;
    }
    // staging: 4 threads per row, WPR/4 words each
    const int sr = threadIdx.x >> 2, sq4 = threadIdx.x & 3;
    for (int c = 0; c < nc_all; ++c) {
        const int j0 = c * ATT_CHUNK;
        __syncthreads();  // the previous chunk's rows are no longer read
        if (j0 + sr < seq) {
            const uint4* kg = reinterpret_cast<const uint4*>(k + base + (size_t)(j0 + sr) * row_stride) + sq4 * (WPR / 16);
            const uint4* vg = reinterpret_cast<const uint4*>(v + base + (size_t)(j0 + sr) * row_stride) + sq4 * (WPR / 16);
#pragma unroll
            for (int e = 0; e < WPR / 16; ++e) {
                const uint4 kw = __ldg(kg + e);
                uint32_t* kd = sK + sr * KSTR + sq4 * (WPR / 4) + 4 * e;
                kd[0] = kw.x, kd[1] = kw.y, kd[2] = kw.z, kd[3] = kw.w;
                reinterpret_cast<uint4*>(sV + sr * WPR + sq4 * (WPR / 4))[e] = __ldg(vg + e);
            }
        }
        __syncthreads();
        if (c >= nc_w) continue;  // warp-uniform: no query of this warp needs this chunk
        float da[Q], db[Q];
#pragma unroll
        for (int x = 0; x < Q; ++x) da[x] = db[x] = 0.0f;
        {
            const uint32_t* ka = sK + lane * KSTR;
            const uint32_t* kb = sK + (lane + 32) * KSTR;
#pragma unroll 8
            for (int w = 0; w < WPR; ++w) {
                const uint32_t a = ka[w], bb = kb[w];
                const float a0 = __uint_as_float(a << 16), a1 = __uint_as_float(a & 0xffff0000u);
                const float b0 = __uint_as_float(bb << 16), b1 = __uint_as_float(bb & 0xffff0000u);
#pragma unroll
                for (int x = 0; x < Q; ++x) {
                    const float2 qf = sQ[warp][x][w];
                    const float q0 = qf.x, q1 = qf.y;
                    da[x] = __fmaf_rn(q0, a0, da[x]);
                    da[x] = __fmaf_rn(q1, a1, da[x]);
                    db[x] = __fmaf_rn(q0, b0, db[x]);
                    db[x] = __fmaf_rn(q1, b1, db[x]);
                }
            }
        }
        float pa[Q], pb[Q];
        AttNode<DPL> cur[Q];
#pragma unroll
        for (int x = 0; x < Q; ++x) {
            const int i = qi[x];
            const bool va = j0 + lane <= i, vb = j0 + lane + 32 <= i;
            const float sa = va ? __fmul_rn(da[x], scale) : -INFINITY;
            const float sb = vb ? __fmul_rn(db[x], scale) : -INFINITY;
            float m = fmaxf(sa, sb);
#pragma unroll
            for (int w = 1; w < 32; w <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, w));
            pa[x] = va ? exp_spec(__fsub_rn(sa, m)) : 0.0f;
            pb[x] = vb ? exp_spec(__fsub_rn(sb, m)) : 0.0f;
            // tree over the 64 slots: slots 0..31 in pa (lane = slot), 32..63 in pb
            float ta = pa[x], tb = pb[x];
#pragma unroll
            for (int w = 1; w < 32; w <<= 1) {
                ta = __fadd_rn(ta, __shfl_xor_sync(0xffffffffu, ta, w));
                tb = __fadd_rn(tb, __shfl_xor_sync(0xffffffffu, tb, w));
            }
            cur[x].m = m;
            cur[x].s = __fadd_rn(ta, tb);
#pragma unroll
            for (int d = 0; d < DPL; ++d) cur[x].o[d] = 0.0f;
        }
        // o: ascending over the chunk's keys; a query whose chunk is partial
        // (or past its position) stops early: keys past i add nothing
        const int nk_max = min(ATT_CHUNK, qlast - j0 + 1);
        for (int t = 0; t < nk_max; ++t) {
            float vf[DPL];
            const uint32_t* vr = sV + t * WPR + (DPL / 2) * lane;
#pragma unroll
            for (int e = 0; e < DPL / 2; ++e) {
                vf[2 * e] = __uint_as_float(vr[e] << 16);
                vf[2 * e + 1] = __uint_as_float(vr[e] & 0xffff0000u);
            }
#pragma unroll
            for (int x = 0; x < Q; ++x) {
                const float pt = __shfl_sync(0xffffffffu, t < 32 ? pa[x] : pb[x], t & 31);
                if (j0 + t <= qi[x]) {
#pragma unroll
                    for (int d = 0; d < DPL; ++d) cur[x].o[d] = __fmaf_rn(pt, vf[d], cur[x].o[d]);
                }
            }
        }
        // the chunk tree of each query, streamed: pop the pending left siblings of every node closing here
#pragma unroll
        for (int x = 0; x < Q; ++x) {
            if (c >= nc[x]) continue;
            const LeafOps ops = leaf_ops(nc[x], c);
            for (int n = leaf_pops(ops); n > 0; --n) cur[x] = att_combine<DPL>(stk[x][--sp[x]], cur[x]);
            if (ops.final_)
                fin[x] = cur[x];
            else
                stk[x][sp[x]++] = cur[x];
        }
    }
#pragma unroll
    for (int x = 0; x < Q; ++x) {
        if (qi[x] >= seq) continue;
        uint16_t* o = out + base + (size_t)qi[x] * row_stride + DPL * lane;
        float r[DPL];
#pragma unroll
        for (int d = 0; d < DPL; ++d) r[d] = __fdiv_rn(fin[x].o[d], fin[x].s);
        if (DPL == 4) {
            *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf2(r[0], r[1]), pack_bf2(r[2], r[3]));
        } else {
            *reinterpret_cast<uint32_t*>(o) = pack_bf2(r[0], r[1]);
        }
    }
}

// out[t] = table[ids[t]], 16-byte vectors; an id outside [0, V) gives zeros.
__global__ void embedding_kernel(const int32_t* __restrict__ ids, const uint16_t* __restrict__ table, uint16_t* out,
                                 int tokens, int V, int d) {
    const int vpr = d >> 3;  // vectors per row
    const long long total = (long long)tokens * vpr;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(e / vpr);
        const int c = (int)(e - (long long)t * vpr);
        const int id = __ldg(ids + t);
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (id >= 0 && id < V)
            w = __ldg(reinterpret_cast<const uint4*>(table + (size_t)id * d) + c);
        else if (c == 0)
            set_error(TBIK_ERR_TARGET);
        reinterpret_cast<uint4*>(out + (size_t)t * d)[c] = w;
    }
}

// bf16 transpose of rows, cols multiples of 8 with 16-byte aligned rows: a
// 64 x 64 tile per CTA of 256 threads, read as 16-byte vectors of 8 columns
// into shared memory (rows padded to 72 elements, so the 16-byte stores and
// the column reads are free of bank conflicts) and written as 32-byte runs of
// 16 consecutive rows of one column (full sectors).
__global__ void __launch_bounds__(256) transpose_vec_kernel(const uint16_t* __restrict__ in, uint16_t* out,
                                                            int rows, int cols) {
    __shared__ __align__(16) uint16_t tile[64][72];
    const int tid = threadIdx.x;
    const int c0 = blockIdx.x * 64, r0 = blockIdx.y * 64;
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
        const int r = (tid >> 3) + 32 * pass, v = tid & 7;  // tile row, 8-column vector
        if (r0 + r < rows && c0 + 8 * v < cols)
            *reinterpret_cast<uint4*>(&tile[r][8 * v]) =
                __ldg(reinterpret_cast<const uint4*>(in + (size_t)(r0 + r) * cols + c0) + v);
    }
    __syncthreads();
    const int c = tid & 63, q = tid >> 6;  // output row c0 + c, input rows r0 + 16q .. r0 + 16q + 15
    if (c0 + c < cols) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int rb = 16 * q + 8 * h;
            if (r0 + rb < rows) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w[e] = (uint32_t)tile[rb + 2 * e][c] | ((uint32_t)tile[rb + 2 * e + 1][c] << 16);
                *reinterpret_cast<uint4*>(out + (size_t)(c0 + c) * rows + r0 + rb) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
}

// bf16 transpose through a 32 x 33 shared-memory tile (block 32 x 8), any shape.
__global__ void transpose_kernel(const uint16_t* __restrict__ in, uint16_t* out, int rows, int cols) {
    __shared__ uint16_t tile[32][33];
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    for (int k = threadIdx.y; k < 32; k += 8) {
        const int r = r0 + k, c = c0 + threadIdx.x;
        if (r < rows && c < cols) tile[k][threadIdx.x] = in[(size_t)r * cols + c];
    }
    __syncthreads();
    for (int k = threadIdx.y; k < 32; k += 8) {
        const int c = c0 + k, r = r0 + threadIdx.x;
        if (r < rows && c < cols) out[(size_t)c * rows + r] = tile[threadIdx.x][k];
    }
}

}  // namespace tbik
