// Causal attention with the reduction over keys in tree order: the keys of a
// query are cut into fixed chunks of 64 positions, each chunk is reduced to a
// (max, sum of exponentials, weighted value sum) summary, and the summaries are
// combined by the same halving tree as every other reduction here (TBIK
// summary page, 技术框架: one hierarchical binary tree for every reduction, so
// the result does not depend on how the work is split).  Nothing depends on
// the batch composition or on how heads are split across devices.
//
// One warp per query (batch b, head h, position i).  Lane l owns head
// dimensions [DPL*l, DPL*l + DPL) of the value sums and the keys 2l, 2l+1 of
// each chunk:
//   score   s_j = fl(dot(q_i, k_j) * scale), the dot accumulated over the head
//           dimension in ascending order with fma from +0;
//   chunk   m = max of its scores (keys <= i); p_j = exp(s_j - m), 0 past i;
//           s = the tree over the chunk's 64 slots of p (slots 2l and 2l+1 in
//           lane l, then xor butterflies); o[d] = ascending sum over the
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
    const float ea = exp_spec(__fsub_rn(a.m, r.m));
    const float eb = exp_spec(__fsub_rn(b.m, r.m));
    r.s = __fadd_rn(__fmul_rn(a.s, ea), __fmul_rn(b.s, eb));
#pragma unroll
    for (int d = 0; d < DPL; ++d) r.o[d] = __fadd_rn(__fmul_rn(a.o[d], ea), __fmul_rn(b.o[d], eb));
    return r;
}

// dot(q, k) over HD = 32*DPL dimensions, ascending, fma from +0; q held as
// HD/2 packed bf16 pairs, k read from global memory in 16-byte vectors.
template <int DPL>
__device__ __forceinline__ float att_dot(const uint32_t (&qp)[16 * DPL], const uint16_t* __restrict__ k) {
    float acc = 0.0f;
    const uint4* kv = reinterpret_cast<const uint4*>(k);
#pragma unroll
    for (int c = 0; c < 4 * DPL; ++c) {
        const uint4 w = __ldg(kv + c);
        const uint32_t kw[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t qw = qp[4 * c + e];
            acc = __fmaf_rn(__uint_as_float(qw << 16), __uint_as_float(kw[e] << 16), acc);
            acc = __fmaf_rn(__uint_as_float(qw & 0xffff0000u), __uint_as_float(kw[e] & 0xffff0000u), acc);
        }
    }
    return acc;
}

template <int DPL>
__global__ void __launch_bounds__(ATT_WARPS * 32)
    attention_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                     uint16_t* out, int batch, int seq, int heads, float scale) {
    constexpr int HD = 32 * DPL;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int qblocks = (seq + ATT_WARPS - 1) / ATT_WARPS;
    const int bh = blockIdx.x / qblocks;
    const int i = (blockIdx.x - bh * qblocks) * ATT_WARPS + warp;
    if (i >= seq) return;
    const int b = bh / heads, h = bh - b * heads;
    const size_t row_stride = (size_t)heads * HD;  // elements between positions
    const size_t base = (size_t)b * seq * row_stride + (size_t)h * HD;
    uint32_t qp[16 * DPL];
    {
        const uint4* qv = reinterpret_cast<const uint4*>(q + base + (size_t)i * row_stride);
#pragma unroll
        for (int c = 0; c < 4 * DPL; ++c) {
            const uint4 w = __ldg(qv + c);
            qp[4 * c] = w.x, qp[4 * c + 1] = w.y, qp[4 * c + 2] = w.z, qp[4 * c + 3] = w.w;
        }
    }
    const int nc = i / ATT_CHUNK + 1;
    AttNode<DPL> stk[8];
    int sp = 0;
    AttNode<DPL> fin;
    for (int c = 0; c < nc; ++c) {
        const int j0 = c * ATT_CHUNK;
        const int ja = j0 + 2 * lane, jb = ja + 1;
        const bool va = ja <= i, vb = jb <= i;
        float sa = -INFINITY, sb = -INFINITY;
        if (va) sa = __fmul_rn(att_dot<DPL>(qp, k + base + (size_t)ja * row_stride), scale);
        if (vb) sb = __fmul_rn(att_dot<DPL>(qp, k + base + (size_t)jb * row_stride), scale);
        float m = fmaxf(sa, sb);
#pragma unroll
        for (int w = 1; w < 32; w <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, w));
        const float pa = va ? exp_spec(__fsub_rn(sa, m)) : 0.0f;
        const float pb = vb ? exp_spec(__fsub_rn(sb, m)) : 0.0f;
        float s = __fadd_rn(pa, pb);  // slots 2l, 2l+1: the bottom level of the tree over 64 slots
#pragma unroll
        for (int w = 1; w < 32; w <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, w));
        AttNode<DPL> cur;
        cur.m = m;
        cur.s = s;
#pragma unroll
        for (int d = 0; d < DPL; ++d) cur.o[d] = 0.0f;
        const int nk = min(ATT_CHUNK, i - j0 + 1);
        const uint16_t* vrow = v + base + (size_t)j0 * row_stride + DPL * lane;
        for (int t = 0; t < nk; ++t) {
            const float pt = __shfl_sync(0xffffffffu, (t & 1) ? pb : pa, t >> 1);
            float vf[DPL];
            if (DPL == 4) {
                const uint2 w = __ldg(reinterpret_cast<const uint2*>(vrow + (size_t)t * row_stride));
                vf[0] = __uint_as_float(w.x << 16);
                vf[1] = __uint_as_float(w.x & 0xffff0000u);
                vf[2] = __uint_as_float(w.y << 16);
                vf[3] = __uint_as_float(w.y & 0xffff0000u);
            } else {
                const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(vrow + (size_t)t * row_stride));
                vf[0] = __uint_as_float(w << 16);
                vf[1] = __uint_as_float(w & 0xffff0000u);
            }
#pragma unroll
            for (int d = 0; d < DPL; ++d) cur.o[d] = __fmaf_rn(pt, vf[d], cur.o[d]);
        }
        // the chunk tree, streamed: pop the pending left siblings of every node closing here
        const LeafOps ops = leaf_ops(nc, c);
        for (int n = leaf_pops(ops); n > 0; --n) cur = att_combine<DPL>(stk[--sp], cur);
        if (ops.final_)
            fin = cur;
        else
            stk[sp++] = cur;
    }
    uint16_t* o = out + base + (size_t)i * row_stride + DPL * lane;
    float r[DPL];
#pragma unroll
    for (int d = 0; d < DPL; ++d) r[d] = __fdiv_rn(fin.o[d], fin.s);
    if (DPL == 4) {
        *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf2(r[0], r[1]), pack_bf2(r[2], r[3]));
    } else {
        *reinterpret_cast<uint32_t*>(o) = pack_bf2(r[0], r[1]);
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

}  // namespace tbik
