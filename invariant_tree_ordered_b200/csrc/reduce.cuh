// Residual RMSNorm, RoPE and SwiGLU with fp32 intermediates and one bf16
// rounding at the output (rounding-location alignment article, winzheng.jp,
// section "外科手術的な修正：3つのノード"), the RMSNorm sum of squares in tree
// order (TBIK summary page, 技术框架).  All three are HBM-bound: 16-byte
// vector loads and stores, fp32 math with explicit round-to-nearest ops.
#pragma once

#include "device_common.cuh"

namespace tbik {

__device__ __forceinline__ void unpack8(uint4 w, float (&f)[8]) {
    const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(a[i] << 16);
        f[2 * i + 1] = __uint_as_float(a[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    uint4 w;
    w.x = pack_bf2(f[0], f[1]);
    w.y = pack_bf2(f[2], f[3]);
    w.z = pack_bf2(f[4], f[5]);
    w.w = pack_bf2(f[6], f[7]);
    return w;
}

// Pairwise (power-of-two) tree over v[0..n) in place; returns v[0].
__device__ __forceinline__ float pairwise_inplace(float* v, int n) {
    for (int w = 1; w < n; w <<= 1)
        for (int i = 0; i < n; i += 2 * w) v[i] = __fadd_rn(v[i], v[i + w]);
    return v[0];
}

// One CTA per token with NT = H/(8*LPT) threads; thread t owns the LPT
// consecutive leaves [LPT*t, LPT*t + LPT) (leaf = 8 elements, one 16-byte
// vector per tensor).  The leaf sums form a power-of-two pairwise tree: the
// lowest log2(LPT) levels inside the thread, then xor-shuffle levels inside a
// warp (both lanes of a pair add the same two values, and fp32 addition is
// commutative, so they hold the same bits), then shared-memory levels.  With T
// shards, shard t's partial (a whole subtree of (H/8)/T leaves) is taken at its
// own level, written to the shard buffer, and the T partials are combined by
// the same tree.  All of a thread's loads are issued before any arithmetic.
template <int NT, int LPT>
__global__ void __launch_bounds__(NT) rmsnorm_residual_kernel(const uint16_t* __restrict__ x,
                                                              const uint16_t* __restrict__ res,
                                                              const uint16_t* __restrict__ gamma, uint16_t* y,
                                                              uint16_t* res_out, int H, float eps, int T) {
    __shared__ float warp_part[NT / 32 > 0 ? NT / 32 : 1];
    __shared__ float shard[8];
    __shared__ float ss_sh;
    const int tid = threadIdx.x;
    const size_t base = (size_t)blockIdx.x * H;
    uint4 xv[LPT], rv[LPT], gv[LPT];
#pragma unroll
    for (int l = 0; l < LPT; ++l) {
        xv[l] = __ldg(reinterpret_cast<const uint4*>(x + base) + LPT * tid + l);
        rv[l] = __ldg(reinterpret_cast<const uint4*>(res + base) + LPT * tid + l);
        gv[l] = __ldg(reinterpret_cast<const uint4*>(gamma) + LPT * tid + l);
    }
    float r[LPT][8], leafsum[LPT];
#pragma unroll
    for (int l = 0; l < LPT; ++l) {
        float xf[8], rf[8];
        unpack8(xv[l], xf);
        unpack8(rv[l], rf);
        float acc = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            r[l][e] = __fadd_rn(xf[e], rf[e]);
            acc = __fmaf_rn(r[l][e], r[l][e], acc);
        }
        leafsum[l] = acc;
    }
    // in-thread levels of the pairwise tree
#pragma unroll
    for (int w = 1; w < LPT; w <<= 1)
#pragma unroll
        for (int l = 0; l < LPT; l += 2 * w) leafsum[l] = __fadd_rn(leafsum[l], leafsum[l + w]);
    float acc = leafsum[0];
    const int S = NT / T;  // threads per shard (power of two)
    const int lim = S < 32 ? S : 32;
    for (int w = 1; w < lim; w <<= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, w));
    if (S <= 32) {
        if ((tid % S) == 0) shard[tid / S] = acc;
    } else {
        if ((tid & 31) == 0) warp_part[tid >> 5] = acc;
        __syncthreads();
        if (tid < T) shard[tid] = pairwise_inplace(&warp_part[tid * (S / 32)], S / 32);
    }
    __syncthreads();
    if (tid == 0) ss_sh = pairwise_inplace(shard, T);
    __syncthreads();
    const float ss = ss_sh;
    const float ms = __fdiv_rn(ss, (float)H);
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
#pragma unroll
    for (int l = 0; l < LPT; ++l) {
        float gf[8], o[8];
        unpack8(gv[l], gf);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(__fmul_rn(r[l][e], inv), gf[e]);
        reinterpret_cast<uint4*>(y + base)[LPT * tid + l] = pack8(o);
        if (res_out) reinterpret_cast<uint4*>(res_out + base)[LPT * tid + l] = pack8(r[l]);
    }
}

// Rotate-half RoPE: thread = (tensor, token, head, group of 8 pairs).  Each
// product is rounded on its own (no fma), then one bf16 rounding.
__global__ void rope_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, uint16_t* q_out,
                            uint16_t* k_out, const int32_t* __restrict__ pos, const float* __restrict__ table,
                            int tokens, int heads, int head_dim, int max_pos) {
    const uint16_t* x = blockIdx.y == 0 ? q : k;
    uint16_t* o = blockIdx.y == 0 ? q_out : k_out;
    if (x == nullptr) return;
    const int half = head_dim >> 1;
    const int gph = half >> 3;
    const size_t total = (size_t)tokens * heads * gph;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const int g = (int)(i % gph);
        const size_t th = i / gph;
        const int token = (int)(th / heads);
        const size_t hb = th * head_dim;
        const int p = __ldg(pos + token);
        float x1[8], x2[8], o1[8], o2[8];
        unpack8(__ldg(reinterpret_cast<const uint4*>(x + hb + 8 * g)), x1);
        unpack8(__ldg(reinterpret_cast<const uint4*>(x + hb + half + 8 * g)), x2);
        if (p < 0 || p >= max_pos) {
            set_error(TBIK_ERR_POSITION);
#pragma unroll
            for (int e = 0; e < 8; ++e) o1[e] = o2[e] = __int_as_float(0x7fc00000);
        } else {
            const float4* cs = reinterpret_cast<const float4*>(table + ((size_t)p * half + 8 * g) * 2);
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                const float4 t = __ldg(cs + e2);  // (c, s) of two consecutive i
                const float c0 = t.x, s0 = t.y, c1 = t.z, s1 = t.w;
                const int a = 2 * e2, b = 2 * e2 + 1;
                o1[a] = __fsub_rn(__fmul_rn(x1[a], c0), __fmul_rn(x2[a], s0));
                o2[a] = __fadd_rn(__fmul_rn(x2[a], c0), __fmul_rn(x1[a], s0));
                o1[b] = __fsub_rn(__fmul_rn(x1[b], c1), __fmul_rn(x2[b], s1));
                o2[b] = __fadd_rn(__fmul_rn(x2[b], c1), __fmul_rn(x1[b], s1));
            }
        }
        *reinterpret_cast<uint4*>(o + hb + 8 * g) = pack8(o1);
        *reinterpret_cast<uint4*>(o + hb + half + 8 * g) = pack8(o2);
    }
}

__device__ __forceinline__ float swiglu1(float g, float u) {
    const float e = exp_spec(-g);
    const float den = __fadd_rn(1.0f, e);
    const float sg = __fdiv_rn(g, den);
    return __fmul_rn(sg, u);
}

// out = bf16((g / (1 + exp(-g))) * u), two 8-element vectors per thread per
// iteration with all loads issued before the arithmetic.
template <int IN_F32>
__device__ __forceinline__ void load8(const void* p, long long i, float (&f)[8]) {
    if (IN_F32) {
        const float4* q = reinterpret_cast<const float4*>(p) + 2 * i;
        const float4 a = __ldg(q), b = __ldg(q + 1);
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
        unpack8(__ldg(reinterpret_cast<const uint4*>(p) + i), f);
    }
}

template <int IN_F32>
__global__ void swiglu_kernel(const void* __restrict__ g, const void* __restrict__ u, uint16_t* out, long long n) {
    const long long nv = n >> 3;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nv; i += 2 * stride) {
        const long long i2 = i + stride;
        const bool two = i2 < nv;
        float g0[8], u0[8], g1[8], u1[8];
        load8<IN_F32>(g, i, g0);
        load8<IN_F32>(u, i, u0);
        if (two) {
            load8<IN_F32>(g, i2, g1);
            load8<IN_F32>(u, i2, u1);
        }
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = swiglu1(g0[e], u0[e]);
        reinterpret_cast<uint4*>(out)[i] = pack8(o);
        if (two) {
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = swiglu1(g1[e], u1[e]);
            reinterpret_cast<uint4*>(out)[i2] = pack8(o);
        }
    }
}

}  // namespace tbik
