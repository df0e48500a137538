// Exact-order CUDA-core GEMM: each output runs, per K leaf, one sequential
// fmaf chain in ascending k from +0.0f, and the leaves are combined by the
// halving tree (TBIK summary page, 技术框架: local then global reduction on one
// binary tree).  This mode is bit-exact to the definition and serves as the
// reference mode of the library; it also yields the non-invariant baseline
// (one leaf per shard) and the logits of the exact logprob mode.
//
// 64x64 output tile per CTA, 256 threads, 4x4 outputs per thread, K staged
// through shared memory 16 deep as fp32 (bf16 widening is exact).  The tree
// stack lives in per-thread local memory (touched once per leaf).
#pragma once

#include "device_common.cuh"

namespace tbik {

constexpr int EX_BM = 64;
constexpr int EX_BN = 64;
constexpr int EX_KC = 16;
constexpr int EX_THREADS = 256;
constexpr int EX_MAXD = 20;
constexpr int EX_MAX_F = 64;

struct ExParams {
    const uint16_t* A;
    const uint16_t* B;
    int M, N, K;
    int leaf;
    int F;
    int tiles_m, tiles_n;
    int total_units;
    int direct;
    int out_bf16;
    void* out;
    const uint16_t* residual;  // bf16 [M,N] added to the fp32 root before the bf16 rounding (direct only)
    float* partials;  // [F][M][N]
    short lo[EX_MAX_F];
    short nl[EX_MAX_F];
};

__device__ __forceinline__ void ex_store(void* out, int bf16, int M, int N, int row, int col, float v,
                                         const uint16_t* residual) {
    if (row >= M || col >= N) return;
    size_t off = (size_t)row * N + col;
    if (residual) v = __fadd_rn(v, bf2f(residual[off]));
    if (bf16)
        reinterpret_cast<uint16_t*>(out)[off] = f2bf(v);
    else
        reinterpret_cast<float*>(out)[off] = v;
}

template <int B_NK>
__global__ void __launch_bounds__(EX_THREADS) gemm_exact_kernel(const __grid_constant__ ExParams p) {
    __shared__ float As[EX_KC][EX_BM];
    __shared__ __align__(16) float Bs[EX_KC][EX_BN];
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    float stk[EX_MAXD][16];

    for (int u = blockIdx.x; u < p.total_units; u += gridDim.x) {
        const int tiles = p.tiles_m * p.tiles_n;
        const int f = u / tiles;
        const int t = u - f * tiles;
        const int tm = t / p.tiles_n, tn = t - (t / p.tiles_n) * p.tiles_n;
        const int m0 = tm * EX_BM, n0 = tn * EX_BN;
        const int n = p.nl[f];
        const int kbeg = p.lo[f] * p.leaf;
        const int kend = kbeg + n * p.leaf;
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
        int sp = 0, j = 0;
        int next_b = kbeg + p.leaf;

        for (int k0 = kbeg; k0 < kend; k0 += EX_KC) {
            __syncthreads();
            {
                const int r = tid >> 2, kk = (tid & 3) * 4;
                const int gm = m0 + r;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int gk = k0 + kk + e;
                    As[kk + e][r] = (gm < p.M && gk < kend) ? bf2f(p.A[(size_t)gm * p.K + gk]) : 0.0f;
                }
            }
            if (B_NK) {
                const int c = tid >> 2, kk = (tid & 3) * 4;
                const int gn = n0 + c;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int gk = k0 + kk + e;
                    Bs[kk + e][c] = (gn < p.N && gk < kend) ? bf2f(p.B[(size_t)gn * p.K + gk]) : 0.0f;
                }
            } else {
                const int kk = tid >> 4, c = (tid & 15) * 4;
                const int gk = k0 + kk;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int gn = n0 + c + e;
                    Bs[kk][c + e] = (gn < p.N && gk < kend) ? bf2f(p.B[(size_t)gk * p.N + gn]) : 0.0f;
                }
            }
            __syncthreads();
            const int kc = min(EX_KC, kend - k0);
            for (int kk = 0; kk < kc; ++kk) {
                float a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
                const float4 bv = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
                b[0] = bv.x;
                b[1] = bv.y;
                b[2] = bv.z;
                b[3] = bv.w;
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[i * 4 + c] = __fmaf_rn(a[i], b[c], acc[i * 4 + c]);
                if (k0 + kk + 1 == next_b) {
                    // leaf j complete: apply the tree
                    const LeafOps ops = leaf_ops(n, j);
                    for (int i = 0; i < leaf_pops(ops); ++i) {
                        --sp;
#pragma unroll
                        for (int e = 0; e < 16; ++e) acc[e] = __fadd_rn(stk[sp][e], acc[e]);
                    }
                    if (ops.final_) {
                        void* dst = p.direct ? p.out : (void*)(p.partials + (size_t)f * p.M * p.N);
                        const int bf = p.direct ? p.out_bf16 : 0;
                        const uint16_t* res = p.direct ? p.residual : nullptr;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                ex_store(dst, bf, p.M, p.N, m0 + ty * 4 + i, n0 + tx * 4 + c, acc[i * 4 + c],
                                         res);
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) stk[sp][e] = acc[e];
                        ++sp;
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
                    ++j;
                    next_b += p.leaf;
                }
            }
        }
    }
}

// --------------------------------------------------------- shard combine

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
    return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z), __fadd_rn(a.w, b.w));
}

// TREE over G (a power of two) partial buffers spaced `stride` floats apart.
template <int G>
struct TreeOf {
    static __device__ __forceinline__ float4 vec(const float* P, size_t stride, size_t idx) {
        return add4(TreeOf<G / 2>::vec(P, stride, idx), TreeOf<G / 2>::vec(P + (G / 2) * stride, stride, idx));
    }
    static __device__ __forceinline__ float one(const float* P, size_t stride, size_t idx) {
        return __fadd_rn(TreeOf<G / 2>::one(P, stride, idx), TreeOf<G / 2>::one(P + (G / 2) * stride, stride, idx));
    }
};
template <>
struct TreeOf<1> {
    static __device__ __forceinline__ float4 vec(const float* P, size_t, size_t idx) {
        return __ldg(reinterpret_cast<const float4*>(P + idx));
    }
    static __device__ __forceinline__ float one(const float* P, size_t, size_t idx) { return __ldg(P + idx); }
};

// out[g] = TREE over P[g*G .. g*G+G) for g < groups; each buffer has MN floats.
// out is fp32 [groups][MN] or, with out_bf16, bf16 [MN] (groups == 1); with
// out_bf16, a non-null R (bf16 [MN], may be `out` itself) is added to the root
// in fp32 before the rounding.  VEC = 1 reads and writes 16-byte vectors and
// needs MN % 4 == 0 (every buffer start P + j*MN and out + g*MN is then
// 16-byte aligned, given 16-byte aligned P and out); VEC = 0 is the element
// loop for any MN.  Same additions in the same order either way.
template <int G, int VEC>
__global__ void tree_combine_kernel(const float* __restrict__ P, size_t MN, int groups, void* out, int out_bf16,
                                    const uint16_t* R) {
    if (VEC) {
        const size_t nvec = MN / 4;
        const size_t total = nvec * groups;
        for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
             i += (size_t)gridDim.x * blockDim.x) {
            const size_t g = i / nvec, e = (i - g * nvec) * 4;
            float4 r = TreeOf<G>::vec(P + g * G * MN, MN, e);
            if (out_bf16 && R) {
                const uint2 q = *reinterpret_cast<const uint2*>(R + e);
                r.x = __fadd_rn(r.x, __uint_as_float(q.x << 16));
                r.y = __fadd_rn(r.y, __uint_as_float(q.x & 0xffff0000u));
                r.z = __fadd_rn(r.z, __uint_as_float(q.y << 16));
                r.w = __fadd_rn(r.w, __uint_as_float(q.y & 0xffff0000u));
            }
            if (out_bf16) {
                uint2 w;
                w.x = pack_bf2(r.x, r.y);
                w.y = pack_bf2(r.z, r.w);
                *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(out) + e) = w;
            } else {
                *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + g * MN + e) = r;
            }
        }
    } else {
        const size_t total = MN * groups;
        for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
             i += (size_t)gridDim.x * blockDim.x) {
            const size_t g = i / MN, e = i - g * MN;
            float r = TreeOf<G>::one(P + g * G * MN, MN, e);
            if (out_bf16 && R) r = __fadd_rn(r, bf2f(R[e]));
            if (out_bf16)
                reinterpret_cast<uint16_t*>(out)[e] = f2bf(r);
            else
                reinterpret_cast<float*>(out)[g * MN + e] = r;
        }
    }
}

// Non-invariant combine: ((P0 + P1) + P2) + ... left to right (then + R, as
// in tree_combine_kernel).
__global__ void seq_combine_kernel(const float* __restrict__ P, size_t MN, int T, void* out, int out_bf16,
                                   const uint16_t* R) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < MN; e += (size_t)gridDim.x * blockDim.x) {
        float acc = P[e];
        for (int t = 1; t < T; ++t) acc = __fadd_rn(acc, P[(size_t)t * MN + e]);
        if (out_bf16 && R) acc = __fadd_rn(acc, bf2f(R[e]));
        if (out_bf16)
            reinterpret_cast<uint16_t*>(out)[e] = f2bf(acc);
        else
            reinterpret_cast<float*>(out)[e] = acc;
    }
}

}  // namespace tbik
