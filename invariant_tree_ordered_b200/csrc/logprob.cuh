// Log-softmax over the vocabulary and gather of the target logprob, with the
// vocabulary reduction in tree order (TBIK summary page, 技术框架) and the
// per-token logprob as the compared quantity (IsoExec brief, 壹/叁).
//
//  * vocab_stats_kernel (exact mode only): per (row, vocab leaf of 64
//    columns) the running max in ascending column order and the ascending sum
//    of exp(z - max), from materialised fp32 logits.  The tensor-core mode
//    computes the same summaries inside the GEMM epilogue instead.
//  * logprob_row_kernel: the vocabulary tree per row over the Lv padded
//    leaves: frontier subtrees streamed leaf by leaf with a small stack, then
//    xor-butterfly levels, the T shard summaries taken at their own level.
#pragma once

#include "device_common.cuh"

namespace tbik {

constexpr int VLEAF = 64;  // vocabulary columns per leaf

// v0: vocabulary index of z's column 0 (a shard's first column), so the
// target's column here is targets[row] - v0; zflag (nullable) is set to 1 for
// the rows whose target falls in this call's columns.
__global__ void vocab_stats_kernel(const float* __restrict__ z, const int32_t* __restrict__ targets,
                                   float* __restrict__ stats, float* __restrict__ zt, int* __restrict__ zflag,
                                   int M, int V, int nvt, int v0) {
    const size_t total = (size_t)M * nvt;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const int row = (int)(i / nvt);
        const int j = (int)(i - (size_t)row * nvt);
        const float* zr = z + (size_t)row * V;
        const int c0 = j * VLEAF;
        const int c1 = min(c0 + VLEAF, V);
        float m = zr[c0];
        for (int c = c0 + 1; c < c1; ++c)
            if (zr[c] > m) m = zr[c];
        float s = 0.0f;
        for (int c = c0; c < c1; ++c) s = __fadd_rn(s, exp_spec(__fsub_rn(zr[c], m)));
        *reinterpret_cast<float2*>(stats + ((size_t)j * M + row) * 2) = make_float2(m, s);
        const long long t = (long long)targets[row] - v0;
        if (t >= c0 && t < c1) {
            zt[row] = zr[t];
            if (zflag) zflag[row] = 1;
        }
    }
}

__device__ __forceinline__ MS leaf_ms(const float* stats, int M, int nvt, int row, int j) {
    MS r;
    if (j < nvt) {
        const float2 v = *reinterpret_cast<const float2*>(stats + ((size_t)j * M + row) * 2);
        r.m = v.x;
        r.s = v.y;
    } else {
        r.m = -INFINITY;
        r.s = 0.0f;
    }
    return r;
}

__device__ __forceinline__ MS shfl_ms(MS v, int src_lane_mask) {
    MS o;
    o.m = __shfl_xor_sync(0xffffffffu, v.m, src_lane_mask);
    o.s = __shfl_xor_sync(0xffffffffu, v.s, src_lane_mask);
    return o;
}

// One butterfly level: lanes l and l^w hold sibling subtrees; the lower lane is the left one.
__device__ __forceinline__ MS butterfly_ms(MS v, int lane, int w) {
    const MS o = shfl_ms(v, w);
    return (lane & w) ? ms_combine(o, v) : ms_combine(v, o);
}

constexpr int ROW_BLOCK = 32;  // rows per CTA of the row kernel (one per lane), 32 warps

// The vocabulary tree per row.  Frontier node f (depth d, nf = 2^d <= 32
// whole subtrees) of row r is reduced by lane r of warp f, streaming its
// leaves with a small stack, so a warp's loads of one leaf index cover 32
// consecutive rows (coalesced).  The nf subtree results go through shared
// memory to warp r, whose lane f then holds node f of row r, and the upper
// levels are xor-butterfly levels in which the left operand of every combine
// is the lower lane.  The T shard summaries are taken at their own level,
// written to the shard buffer, read back and combined by the top levels.
__global__ void __launch_bounds__(ROW_BLOCK * 32)
    logprob_row_kernel(const float* __restrict__ stats, const float* __restrict__ zt,
                       const int32_t* __restrict__ targets, float* __restrict__ out, float* shard_ms, int M, int V,
                       int nvt, int Lv, int T, const int* __restrict__ zflag, float4* __restrict__ shard_sum) {
    constexpr int TAB = 512;
    __shared__ uint16_t tab[2][TAB];        // leaf operation codes for the two frontier subtree sizes
    __shared__ float2 part[32][ROW_BLOCK];  // [frontier node][row in block]
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int row0 = blockIdx.x * ROW_BLOCK;
    int d = 0;
    while (d < 5 && (2 << d) <= Lv) ++d;  // largest d <= 5 with 2^d <= Lv
    const int nf = 1 << d;
    // Nodes at depth d of the halving tree hold floor or ceil of Lv / 2^d leaves.
    const int n_hi = (Lv + nf - 1) / nf, n_lo = Lv / nf;
    const bool use_tab = n_hi <= TAB;
    if (use_tab) {
        for (int i = threadIdx.x; i < n_hi + n_lo; i += blockDim.x) {
            const int t = i < n_hi ? 0 : 1;
            const int j = i - (t ? n_hi : 0);
            tab[t][j] = encode_leaf_ops(leaf_ops(t ? n_lo : n_hi, j));
        }
    }
    __syncthreads();
    // Frontier node `warp` of row row0 + lane.
    if (warp < nf) {
        const int row = row0 + lane;
        MS v;
        v.m = -INFINITY;
        v.s = 0.0f;
        if (row < M) {
            int lo = 0, n = Lv;
            for (int lvl = 0; lvl < d; ++lvl) {
                const int h = (n + 1) >> 1;
                if ((warp >> (d - 1 - lvl)) & 1) {
                    lo += h;
                    n -= h;
                } else {
                    n = h;
                }
            }
            MS stk[24];
            int sp = 0;
            const uint16_t* tb = tab[n == n_hi ? 0 : 1];
            // The leaves' summaries are loaded four leaves ahead of their use
            // (a ring of four, unrolled so it stays in registers); the combines
            // run in the same order as without the look-ahead.
            MS ring[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                ring[k].m = -INFINITY;
                ring[k].s = 0.0f;
                if (k < n) ring[k] = leaf_ms(stats, M, nvt, row, lo + k);
            }
            for (int j0 = 0; j0 < n; j0 += 4) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int j = j0 + k;
                    if (j < n) {
                        MS cur = ring[k];
                        if (j + 4 < n) ring[k] = leaf_ms(stats, M, nvt, row, lo + j + 4);
                        const uint32_t code = use_tab ? tb[j] : encode_leaf_ops(leaf_ops(n, j));
                        const int npop = code_pops(code);
                        for (int i = 0; i < npop; ++i) cur = ms_combine(stk[--sp], cur);
                        if (!((code >> 10) & 1)) stk[sp++] = cur;
                        else v = cur;
                    }
                }
            }
        }
        part[warp][lane] = make_float2(v.m, v.s);
    }
    __syncthreads();
    const int row = row0 + warp;
    if (row >= M) return;
    MS v;
    v.m = -INFINITY;
    v.s = 0.0f;
    if (lane < nf) {
        const float2 t2 = part[lane][warp];
        v.m = t2.x;
        v.s = t2.y;
    }
    const int sl = nf / T;  // lanes per shard
    for (int w = 1; w < sl; w <<= 1) v = butterfly_ms(v, lane, w);
    if (lane < nf && (lane % sl) == 0)
        *reinterpret_cast<float2*>(shard_ms + ((size_t)(lane / sl) * M + row) * 2) = make_float2(v.m, v.s);
    __syncwarp();
    // The T shard partials (the emulated cross-GPU exchange), by the same tree.
    MS sv;
    sv.m = -INFINITY;
    sv.s = 0.0f;
    if (lane < T) {
        const float2 t2 = *reinterpret_cast<const float2*>(shard_ms + ((size_t)lane * M + row) * 2);
        sv.m = t2.x;
        sv.s = t2.y;
    }
    for (int w = 1; w < T; w <<= 1) sv = butterfly_ms(sv, lane, w);
    const MS fin = sv;
    if (shard_sum != nullptr) {  // a vocabulary shard's summary (T == 1): (m, s, z_t, owns the target)
        if (lane == 0) {
            const bool own = zflag[row] != 0;
            shard_sum[row] = make_float4(fin.m, fin.s, own ? zt[row] : 0.0f, own ? 1.0f : 0.0f);
        }
        return;
    }
    if (lane == 0) {
        const int t = targets[row];
        if (t < 0 || t >= V) {
            set_error(TBIK_ERR_TARGET);
            out[row] = __int_as_float(0x7fc00000);
        } else {
            out[row] = __fsub_rn(__fsub_rn(zt[row], fin.m), log_spec(fin.s));
        }
    }
}

// The shard level of a vocabulary-parallel logprob: parts [T][M] hold each
// shard's (m, s, z_t, owner) for every row (a shard's summary is the TREE over
// its own contiguous vocabulary leaves).  Per row: TREE over the T summaries
// (T a power of two: adjacent pairs level by level, the lower shard the left
// operand, as in logprob_row_kernel's shard level), z_t from the shard that
// owns the target, out = (z_t - m) - log(s).  A target outside [0, V), or one
// that no shard owns, gives NaN and TBIK_ERR_TARGET.
__global__ void logprob_combine_kernel(const float4* __restrict__ parts, const int32_t* __restrict__ targets,
                                       float* __restrict__ out, int M, int V, int T) {
    for (int row = blockIdx.x * blockDim.x + threadIdx.x; row < M; row += gridDim.x * blockDim.x) {
        MS v[8];
        float z = 0.0f;
        int owners = 0;
        for (int t = 0; t < T; ++t) {
            const float4 q = parts[(size_t)t * M + row];
            v[t].m = q.x;
            v[t].s = q.y;
            if (q.w != 0.0f) {
                z = q.z;
                ++owners;
            }
        }
        for (int w = 1; w < T; w <<= 1)
            for (int i = 0; i + w < T; i += 2 * w) v[i] = ms_combine(v[i], v[i + w]);
        const int tg = targets[row];
        if (tg < 0 || tg >= V || owners != 1) {
            set_error(TBIK_ERR_TARGET);
            out[row] = __int_as_float(0x7fc00000);
        } else {
            out[row] = __fsub_rn(__fsub_rn(z, v[0].m), log_spec(v[0].s));
        }
    }
}

}  // namespace tbik
