// Exact-order CUDA-core GEMM: each output runs, per K leaf, one sequential
// fmaf chain in ascending k from +0.0f, and the leaves are combined by the
// halving tree (TBIK summary page, 技术框架: local then global reduction on one
// binary tree).  This mode is bit-exact to the definition and serves as the
// reference mode of the library; it also yields the non-invariant baseline
// (one leaf per shard) and the logits of the exact logprob mode.
//
// 128x128 output tile per CTA, 512 threads (16 warps per SM), 8x4 outputs per
// thread: rows 4*ty + {0..3} and 64 + 4*ty + {0..3}, columns 4*tx + {0..3}
// (tx = lane, ty = warp), so each k step reads two 16-byte vectors of A (the
// same for the whole warp: broadcast) and one of B for 32 fmas.  The fmas run
// two columns per instruction (packed f32x2: each lane is the IEEE fmaf of
// that column, so every output is still one scalar fmaf chain).  K is staged
// 16 deep through shared memory as fp32 (bf16 widening is exact), double
// buffered, with the global loads two chunks ahead (held as raw bf16 until
// they are widened into shared memory), one barrier per chunk.  The tree stack lives in per-thread local
// memory (touched once per leaf).
#pragma once

#include "device_common.cuh"

namespace tbik {

constexpr int EX_BM = 128;
constexpr int EX_BN = 128;
constexpr int EX_KC = 16;
constexpr int EX_THREADS = 512;
constexpr int EX_MAXD = 16;
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

// Four consecutive bf16 of one row as raw 16-bit patterns in a uint2 (widened
// only when stored to shared memory); elements at or past `lim` (or a row past
// the matrix) read as 0.  VEC: one 8-byte load (the caller guarantees 8-byte
// alignment and that the row holds all four when k < lim).
template <int VEC>
__device__ __forceinline__ uint2 ld4raw(const uint16_t* row_base, bool row_ok, int k, int lim) {
    if (VEC && row_ok && k + 4 <= lim) return __ldg(reinterpret_cast<const uint2*>(row_base + k));
    uint32_t h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = (row_ok && k + e < lim) ? (uint32_t)row_base[k + e] : 0u;
    return make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
}

__device__ __forceinline__ void widen4(uint2 w, float (&f)[4]) {
    f[0] = __uint_as_float(w.x << 16);
    f[1] = __uint_as_float(w.x & 0xffff0000u);
    f[2] = __uint_as_float(w.y << 16);
    f[3] = __uint_as_float(w.y & 0xffff0000u);
}

// The operands of one 16-deep K chunk [k0, k0+16) of the unit, cut at kend:
// thread t holds 4 values of A (row t/4, k offsets 4*(t%4)..) and 4 of B.
struct ExChunk {
    uint2 a, b;
};

template <int B_NK, int VEC>
__device__ __forceinline__ ExChunk ex_load_chunk(const ExParams& p, int m0, int n0, int k0, int kend) {
    const int t = threadIdx.x;
    ExChunk c;
    {
        const int r = t >> 2, kk = (t & 3) * 4, gm = m0 + r;
        c.a = ld4raw<VEC>(p.A + (size_t)gm * p.K, gm < p.M, k0 + kk, kend);
    }
    if (B_NK) {
        const int col = t >> 2, kk = (t & 3) * 4, gn = n0 + col;
        c.b = ld4raw<VEC>(p.B + (size_t)gn * p.K, gn < p.N, k0 + kk, kend);
    } else {
        const int kk = t >> 5, col = (t & 31) * 4, gk = k0 + kk;
        c.b = ld4raw<VEC>(p.B + (size_t)gk * p.N + n0, gk < kend, col, p.N - n0);
    }
    return c;
}

template <int B_NK>
__device__ __forceinline__ void ex_store_chunk(float (*As)[EX_BM], float (*Bs)[EX_BN], const ExChunk& c) {
    const int t = threadIdx.x;
    float fa[4], fb[4];
    widen4(c.a, fa);
    widen4(c.b, fb);
    {
        const int r = t >> 2, kk = (t & 3) * 4;
#pragma unroll
        for (int e = 0; e < 4; ++e) As[kk + e][r] = fa[e];
    }
    if (B_NK) {
        const int col = t >> 2, kk = (t & 3) * 4;
#pragma unroll
        for (int e = 0; e < 4; ++e) Bs[kk + e][col] = fb[e];
    } else {
        const int kk = t >> 5, col = (t & 31) * 4;
        *reinterpret_cast<float4*>(&Bs[kk][col]) = make_float4(fb[0], fb[1], fb[2], fb[3]);
    }
}

// VEC = 1 needs K % 8 == 0, the leaf length % 8 == 0 (chunk starts are then
// multiples of 8 elements) and, for [K,N] B, N % 8 == 0: every 8-byte load is
// then aligned.  VEC = 0 loads element by element.  Same arithmetic either way.
template <int B_NK, int VEC>
__global__ void __launch_bounds__(EX_THREADS, 1) gemm_exact_kernel(const __grid_constant__ ExParams p) {
    __shared__ __align__(16) float As[2][EX_KC][EX_BM];
    __shared__ __align__(16) float Bs[2][EX_KC][EX_BN];
    const int tid = threadIdx.x;
    const int tx = tid & 31, ty = tid >> 5;
    f2x stk[EX_MAXD][8][2];

    for (int u = blockIdx.x; u < p.total_units; u += gridDim.x) {
        const int tiles = p.tiles_m * p.tiles_n;
        const int f = u / tiles;
        const int t = u - f * tiles;
        const int tm = t / p.tiles_n, tn = t - (t / p.tiles_n) * p.tiles_n;
        const int m0 = tm * EX_BM, n0 = tn * EX_BN;
        const int n = p.nl[f];
        const int kbeg = p.lo[f] * p.leaf;
        const int kend = kbeg + n * p.leaf;
        // acc[i][q]: row i (4*ty + i, then 64 + 4*ty + i - 4) and the column
        // pair q (4*tx + 2q, +1), one packed f32x2 register pair; every lane is
        // the same fmaf chain as a scalar.
        f2x acc[8][2];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int q = 0; q < 2; ++q) acc[i][q] = 0ull;  // (+0.0f, +0.0f)
        int sp = 0, j = 0;
        int next_b = kbeg + p.leaf;
        // Two chunks in flight: chunk i+1's operands were loaded while chunk
        // i-1 was computed, chunk i+2's are loaded while chunk i is computed.
        ex_store_chunk<B_NK>(As[0], Bs[0], ex_load_chunk<B_NK, VEC>(p, m0, n0, kbeg, kend));
        ExChunk next = {make_uint2(0u, 0u), make_uint2(0u, 0u)};
        if (kbeg + EX_KC < kend) next = ex_load_chunk<B_NK, VEC>(p, m0, n0, kbeg + EX_KC, kend);
        __syncthreads();
        int buf = 0;
        for (int k0 = kbeg; k0 < kend; k0 += EX_KC) {
            const bool more = k0 + EX_KC < kend;
            ExChunk after = {make_uint2(0u, 0u), make_uint2(0u, 0u)};
            if (k0 + 2 * EX_KC < kend) after = ex_load_chunk<B_NK, VEC>(p, m0, n0, k0 + 2 * EX_KC, kend);
            const int kc = min(EX_KC, kend - k0);
            // one k step: acc[i][c] = fma(A[row i][k], B[k][col c], acc[i][c]), two columns per instruction
            auto kstep = [&](int kk) {
                const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
                const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
                const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
                const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const f2x b[2] = {pk2(b0.x, b0.y), pk2(b0.z, b0.w)};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const f2x ai = pk2(a[i], a[i]);
#pragma unroll
                    for (int q = 0; q < 2; ++q) acc[i][q] = fma2(ai, b[q], acc[i][q]);
                }
            };
            int kk = 0;
            if (kc == EX_KC && next_b - k0 >= EX_KC) {
                // the whole chunk lies inside one leaf (the common case): straight-line steps
#pragma unroll
                for (int q = 0; q < EX_KC; ++q) kstep(q);
                kk = EX_KC;
            }
            while (kk < kc || k0 + kk == next_b) {
                // k steps up to the next leaf boundary inside this chunk
                const int seg = min(kc, next_b - k0);
#pragma unroll 4
                for (; kk < seg; ++kk) kstep(kk);
                if (k0 + kk == next_b) {
                    // leaf j complete: apply the tree (stack value + this value, per lane)
                    const LeafOps ops = leaf_ops(n, j);
                    for (int i = 0; i < leaf_pops(ops); ++i) {
                        --sp;
#pragma unroll
                        for (int r = 0; r < 8; ++r)
#pragma unroll
                            for (int q = 0; q < 2; ++q) acc[r][q] = add2(stk[sp][r][q], acc[r][q]);
                    }
                    if (ops.final_) {
                        void* dst = p.direct ? p.out : (void*)(p.partials + (size_t)f * p.M * p.N);
                        const int bf = p.direct ? p.out_bf16 : 0;
                        const uint16_t* res = p.direct ? p.residual : nullptr;
#pragma unroll
                        for (int r = 0; r < 8; ++r)
#pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                float lo, hi;
                                upk2(acc[r][q], lo, hi);
                                const int row = m0 + (r >> 2) * 64 + ty * 4 + (r & 3);
                                const int col = n0 + tx * 4 + q * 2;
                                ex_store(dst, bf, p.M, p.N, row, col, lo, res);
                                ex_store(dst, bf, p.M, p.N, row, col + 1, hi, res);
                            }
                    } else {
#pragma unroll
                        for (int r = 0; r < 8; ++r)
#pragma unroll
                            for (int q = 0; q < 2; ++q) stk[sp][r][q] = acc[r][q];
                        ++sp;
                    }
#pragma unroll
                    for (int r = 0; r < 8; ++r)
#pragma unroll
                        for (int q = 0; q < 2; ++q) acc[r][q] = 0ull;
                    ++j;
                    next_b += p.leaf;
                }
            }
            if (more) ex_store_chunk<B_NK>(As[buf ^ 1], Bs[buf ^ 1], next);
            __syncthreads();
            buf ^= 1;
            next = after;
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
