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

// One CTA per token, NT = H/8 threads; thread t owns leaf t = elements [8t, 8t+8).
// The leaf sums form a power-of-two pairwise tree: xor-shuffle levels inside a
// warp (both lanes of a pair add the same two values, and fp32 addition is
// commutative, so they hold the same bits), then shared-memory levels.  With T
// shards, shard t's partial (a whole subtree of NT/T leaves) is taken at its
// own level, written to the shard buffer, and the T partials are combined by
// the same tree.
template <int NT>
__global__ void __launch_bounds__(NT) rmsnorm_residual_kernel(const uint16_t* __restrict__ x,
                                                              const uint16_t* __restrict__ res,
                                                              const uint16_t* __restrict__ gamma, uint16_t* y,
                                                              uint16_t* res_out, int H, float eps, int T) {
    __shared__ float warp_part[NT / 32 > 0 ? NT / 32 : 1];
    __shared__ float shard[8];
    __shared__ float ss_sh;
    const int tid = threadIdx.x;
    const size_t base = (size_t)blockIdx.x * H;
    const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + base) + tid);
    const uint4 rv = __ldg(reinterpret_cast<const uint4*>(res + base) + tid);
    const uint4 gv = __ldg(reinterpret_cast<const uint4*>(gamma) + tid);
    float xf[8], rf[8], gf[8], r[8];
    unpack8(xv, xf);
    unpack8(rv, rf);
    unpack8(gv, gf);
    float acc = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        r[e] = __fadd_rn(xf[e], rf[e]);
        acc = __fmaf_rn(r[e], r[e], acc);
    }
    const int S = NT / T;  // leaves per shard (power of two)
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
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(__fmul_rn(r[e], inv), gf[e]);
    reinterpret_cast<uint4*>(y + base)[tid] = pack8(o);
    if (res_out) reinterpret_cast<uint4*>(res_out + base)[tid] = pack8(r);
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

// out = bf16((g / (1 + exp(-g))) * u), 8 elements per thread.
template <int IN_F32>
__global__ void swiglu_kernel(const void* __restrict__ g, const void* __restrict__ u, uint16_t* out, long long n) {
    const long long nv = n >> 3;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nv;
         i += (long long)gridDim.x * blockDim.x) {
        float gf[8], uf[8], o[8];
        if (IN_F32) {
            const float4* gp = reinterpret_cast<const float4*>(g) + 2 * i;
            const float4* up = reinterpret_cast<const float4*>(u) + 2 * i;
            const float4 g0 = __ldg(gp), g1 = __ldg(gp + 1), u0 = __ldg(up), u1 = __ldg(up + 1);
            gf[0] = g0.x; gf[1] = g0.y; gf[2] = g0.z; gf[3] = g0.w;
            gf[4] = g1.x; gf[5] = g1.y; gf[6] = g1.z; gf[7] = g1.w;
            uf[0] = u0.x; uf[1] = u0.y; uf[2] = u0.z; uf[3] = u0.w;
            uf[4] = u1.x; uf[5] = u1.y; uf[6] = u1.z; uf[7] = u1.w;
        } else {
            unpack8(__ldg(reinterpret_cast<const uint4*>(g) + i), gf);
            unpack8(__ldg(reinterpret_cast<const uint4*>(u) + i), uf);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = swiglu1(gf[e], uf[e]);
        reinterpret_cast<uint4*>(out)[i] = pack8(o);
    }
}

}  // namespace tbik
