// Residual RMSNorm, RoPE and SwiGLU with fp32 intermediates and one bf16
// rounding at the output (rounding-location alignment article, winzheng.jp,
// section "外科手術的な修正：3つのノード"), the RMSNorm sum of squares in tree
// order (TBIK summary page, 技术框架).  All three are HBM-bound: 16-byte
// vector loads and stores, fp32 math with explicit round-to-nearest ops.
#pragma once

#include "device_common.cuh"

namespace tbik {

// NT = H/(8*LPT) threads per token; thread t owns the LPT consecutive leaves
// [LPT*t, LPT*t + LPT) (leaf = 8 elements, one 16-byte vector per tensor).
// The leaf sums form a power-of-two pairwise tree: the lowest log2(LPT)
// levels inside the thread, then xor-shuffle levels inside groups of
// L = min(NT/T, 32) lanes (both lanes of a pair add the same two values, and
// fp32 addition is commutative, so they hold the same bits), then the
// remaining levels over the NT/L group values through shared memory.  With T
// shards each shard (a whole subtree of (H/8)/T leaves) ends at or above the
// group level, so these are the same levels as a per-shard tree followed by
// the tree over the T shard partials.  A CTA loops over tokens and loads the
// next token while it reduces and writes the current one; gamma is loaded once.
// RES = false: no residual input, r = f32(x) (res is not read).
template <int NT, int LPT, bool RES>
__global__ void __launch_bounds__(NT) rmsnorm_residual_kernel(const uint16_t* __restrict__ x,
                                                              const uint16_t* __restrict__ res,
                                                              const uint16_t* __restrict__ gamma, uint16_t* y,
                                                              uint16_t* res_out, int tokens, int H, float eps,
                                                              int T) {
    __shared__ float part[2][32];
    const int tid = threadIdx.x;
    int t = blockIdx.x;
    if (t >= tokens) return;
    const float inv_h = __frcp_rn((float)H);  // exact: H is a power of two
    const int S = NT / T;            // threads per shard (a power of two)
    const int L = S < 32 ? S : 32;   // lanes per shuffle group
    const int G = NT / L;            // group values combined through shared memory
    uint4 gv[LPT], xv[LPT], rv[LPT];
#pragma unroll
    for (int l = 0; l < LPT; ++l) {
        gv[l] = __ldg(reinterpret_cast<const uint4*>(gamma) + LPT * tid + l);
        xv[l] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H) + LPT * tid + l);
        if (RES) rv[l] = __ldg(reinterpret_cast<const uint4*>(res + (size_t)t * H) + LPT * tid + l);
    }
    for (int it = 0;; ++it) {
        const int tn = t + gridDim.x;
        const bool more = tn < tokens;
        uint4 xn[LPT], rn[LPT];
        if (more) {
#pragma unroll
            for (int l = 0; l < LPT; ++l) {
                xn[l] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)tn * H) + LPT * tid + l);
                if (RES) rn[l] = __ldg(reinterpret_cast<const uint4*>(res + (size_t)tn * H) + LPT * tid + l);
            }
        }
        float leafsum[LPT];
#pragma unroll
        for (int l = 0; l < LPT; ++l) {
            float xf[8], rf[8];
            unpack8(xv[l], xf);
            if (RES) unpack8(rv[l], rf);
            float acc = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float r = RES ? __fadd_rn(xf[e], rf[e]) : xf[e];
                acc = __fmaf_rn(r, r, acc);
            }
            leafsum[l] = acc;
        }
#pragma unroll
        for (int w = 1; w < LPT; w <<= 1)
#pragma unroll
            for (int l = 0; l < LPT; l += 2 * w) leafsum[l] = __fadd_rn(leafsum[l], leafsum[l + w]);
        float acc = leafsum[0];
        for (int w = 1; w < L; w <<= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, w));
        if ((tid % L) == 0) part[it & 1][tid / L] = acc;
        __syncthreads();
        // every warp applies the remaining levels to the G group values itself
        float pv = (tid & 31) < G ? part[it & 1][tid & 31] : 0.0f;
        for (int w = 1; w < G; w <<= 1) pv = __fadd_rn(pv, __shfl_xor_sync(0xffffffffu, pv, w));
        const float ss = __shfl_sync(0xffffffffu, pv, 0);
        // H is a power of two (H/8 leaves, a power of two), so ss * (1/H)
        // with 1/H exact is the correctly rounded ss / H: the same bits as the
        // division, without its latency in the per-token chain
        const float ms = __fmul_rn(ss, inv_h);
        const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
#pragma unroll
        for (int l = 0; l < LPT; ++l) {
            float xf[8], rf[8], gf[8], r[8], o[8];
            unpack8(xv[l], xf);
            if (RES) unpack8(rv[l], rf);
            unpack8(gv[l], gf);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                r[e] = RES ? __fadd_rn(xf[e], rf[e]) : xf[e];
                o[e] = __fmul_rn(__fmul_rn(r[e], inv), gf[e]);
            }
            reinterpret_cast<uint4*>(y + (size_t)t * H)[LPT * tid + l] = pack8(o);
            if (res_out) reinterpret_cast<uint4*>(res_out + (size_t)t * H)[LPT * tid + l] = pack8(r);
        }
        if (!more) break;
        t = tn;
#pragma unroll
        for (int l = 0; l < LPT; ++l) {
            xv[l] = xn[l];
            if (RES) rv[l] = rn[l];
        }
    }
}

// Rotate-half RoPE: thread = (token, head, group of 8 pairs) of both q and k,
// grid-stride loop; the table row of the token's position is read once for
// both tensors.  Item indices in IDX (32-bit when they fit, for cheap
// division).  Each product is rounded on its own (no fma), then one bf16
// rounding.
__device__ __forceinline__ void rope8(const uint4& w1, const uint4& w2, const float4 (&cs)[4], uint4& r1, uint4& r2) {
    float x1[8], x2[8], o1[8], o2[8];
    unpack8(w1, x1);
    unpack8(w2, x2);
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
        const float c0 = cs[e2].x, s0 = cs[e2].y, c1 = cs[e2].z, s1 = cs[e2].w;  // (c, s) of two consecutive i
        const int a = 2 * e2, b = 2 * e2 + 1;
        o1[a] = __fsub_rn(__fmul_rn(x1[a], c0), __fmul_rn(x2[a], s0));
        o2[a] = __fadd_rn(__fmul_rn(x2[a], c0), __fmul_rn(x1[a], s0));
        o1[b] = __fsub_rn(__fmul_rn(x1[b], c1), __fmul_rn(x2[b], s1));
        o2[b] = __fadd_rn(__fmul_rn(x2[b], c1), __fmul_rn(x1[b], s1));
    }
    r1 = pack8(o1);
    r2 = pack8(o2);
}

template <typename IDX>
__global__ void rope_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, uint16_t* q_out,
                            uint16_t* k_out, const int32_t* __restrict__ pos, const float* __restrict__ table,
                            int tokens, int heads, int head_dim, int max_pos) {
    const IDX half = (IDX)(head_dim >> 1);
    const IDX gph = half >> 3;
    const IDX total = (IDX)tokens * (IDX)heads * gph;
    const bool hq = q != nullptr, hk = k != nullptr;
    const uint4 nan4 = make_uint4(0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u);
    for (IDX i = blockIdx.x * (IDX)blockDim.x + threadIdx.x; i < total; i += (IDX)gridDim.x * blockDim.x) {
        const IDX th = i / gph;
        const int g = (int)(i - th * gph);
        const int token = (int)(th / (IDX)heads);
        const size_t o1 = (size_t)th * head_dim + 8 * g, o2 = o1 + half;
        uint4 a1, a2, b1, b2;
        if (hq) {
            a1 = __ldg(reinterpret_cast<const uint4*>(q + o1));
            a2 = __ldg(reinterpret_cast<const uint4*>(q + o2));
        }
        if (hk) {
            b1 = __ldg(reinterpret_cast<const uint4*>(k + o1));
            b2 = __ldg(reinterpret_cast<const uint4*>(k + o2));
        }
        const int p = __ldg(pos + token);
        uint4 ra1 = nan4, ra2 = nan4, rb1 = nan4, rb2 = nan4;
        if (p < 0 || p >= max_pos) {
            set_error(TBIK_ERR_POSITION);
        } else {
            const float4* row = reinterpret_cast<const float4*>(table + ((size_t)p * half + 8 * g) * 2);
            float4 cs[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) cs[e2] = __ldg(row + e2);
            if (hq) rope8(a1, a2, cs, ra1, ra2);
            if (hk) rope8(b1, b2, cs, rb1, rb2);
        }
        if (hq) {
            *reinterpret_cast<uint4*>(q_out + o1) = ra1;
            *reinterpret_cast<uint4*>(q_out + o2) = ra2;
        }
        if (hk) {
            *reinterpret_cast<uint4*>(k_out + o1) = rb1;
            *reinterpret_cast<uint4*>(k_out + o2) = rb2;
        }
    }
}


// SwiGLU of bf16 gates through a table: silu(g) = g / (1 + exp(-g)) depends
// only on g's 16 bits, so g_silu_lut[bits] holds the fp32 result of exactly the
// operations of swiglu1 for every bf16 value, and out = bf16(lut[g] * u) has
// the same bits as the computed form (the GPU tests run all 65536 gates).
// Built once per device (silu_lut_kernel) before the first table lookup.
static __device__ float g_silu_lut[65536];

__global__ void silu_lut_kernel() {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= 65536) return;
    const float g = __uint_as_float((uint32_t)t << 16);
    const float e = exp_spec(-g);
    const float den = __fadd_rn(1.0f, e);
    g_silu_lut[t] = __fdiv_rn(g, den);
}

// out = bf16(lut[g] * u) for bf16 g and u, 8 elements per thread per
// iteration of a grid-stride loop (the next vector's loads in flight); the
// table (256 KiB) is read through the read-only cache.
template <typename IDX>
__global__ void swiglu_lut_kernel(const uint16_t* __restrict__ g, const uint16_t* __restrict__ u, uint16_t* out,
                                  long long n) {
    const IDX nv = (IDX)(n >> 3);
    const IDX stride = (IDX)gridDim.x * blockDim.x;
    IDX i = (IDX)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nv) return;
    uint4 cg = __ldg(reinterpret_cast<const uint4*>(g) + i), cu = __ldg(reinterpret_cast<const uint4*>(u) + i);
    while (true) {
        const IDX inext = i + stride;
        const bool more = inext < nv;
        uint4 ng, nu;
        if (more) {
            ng = __ldg(reinterpret_cast<const uint4*>(g) + inext);
            nu = __ldg(reinterpret_cast<const uint4*>(u) + inext);
        }
        const uint32_t gw[4] = {cg.x, cg.y, cg.z, cg.w};
        float sg[8], uf[8], o[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sg[2 * e] = __ldg(g_silu_lut + (gw[e] & 0xffffu));
            sg[2 * e + 1] = __ldg(g_silu_lut + (gw[e] >> 16));
        }
        unpack8(cu, uf);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(sg[e], uf[e]);
        reinterpret_cast<uint4*>(out)[i] = pack8(o);
        if (!more) break;
        i = inext;
        cg = ng;
        cu = nu;
    }
}

// out = bf16((g / (1 + exp(-g))) * u), one 8-element vector per thread per
// iteration of a grid-stride loop; the next iteration's inputs are loaded
// before this one's arithmetic, so loads stay in flight during the (ALU-heavy)
// exp and division.  Elements go through swiglu2 in pairs (packed f32x2
// arithmetic, the same bits as swiglu1).
template <int IN_F32>
struct Vec8;
template <>
struct Vec8<0> {
    uint4 a;
};
template <>
struct Vec8<1> {
    float4 a, b;
};

template <int IN_F32, typename IDX>
__device__ __forceinline__ Vec8<IN_F32> load_vec8(const void* p, IDX i) {
    Vec8<IN_F32> r;
    if constexpr (IN_F32) {
        const float4* q = reinterpret_cast<const float4*>(p) + 2 * i;
        r.a = __ldg(q);
        r.b = __ldg(q + 1);
    } else {
        r.a = __ldg(reinterpret_cast<const uint4*>(p) + i);
    }
    return r;
}

template <int IN_F32>
__device__ __forceinline__ void unpack_vec8(const Vec8<IN_F32>& r, float (&f)[8]) {
    if constexpr (IN_F32) {
        f[0] = r.a.x, f[1] = r.a.y, f[2] = r.a.z, f[3] = r.a.w;
        f[4] = r.b.x, f[5] = r.b.y, f[6] = r.b.z, f[7] = r.b.w;
    } else {
        unpack8(r.a, f);
    }
}

// Grid-stride loop over 8-element vectors, the next vector's loads issued
// before the current one is computed.  Vector indices in IDX (32-bit when
// every index the loop forms fits, for cheaper address arithmetic).
template <int IN_F32, typename IDX>
__global__ void swiglu_kernel(const void* __restrict__ g, const void* __restrict__ u, uint16_t* out, long long n) {
    const IDX nv = (IDX)(n >> 3);
    const IDX stride = (IDX)gridDim.x * blockDim.x;
    IDX i = (IDX)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nv) return;
    Vec8<IN_F32> cg = load_vec8<IN_F32>(g, i), cu = load_vec8<IN_F32>(u, i);
    while (true) {
        const IDX inext = i + stride;
        const bool more = inext < nv;
        Vec8<IN_F32> ng, nu;
        if (more) {
            ng = load_vec8<IN_F32>(g, inext);
            nu = load_vec8<IN_F32>(u, inext);
        }
        float gf[8], uf[8], o[8];
        unpack_vec8<IN_F32>(cg, gf);
        unpack_vec8<IN_F32>(cu, uf);
#pragma unroll
        for (int e = 0; e < 8; e += 2) swiglu2(gf[e], gf[e + 1], uf[e], uf[e + 1], o[e], o[e + 1]);
        reinterpret_cast<uint4*>(out)[i] = pack8(o);
        if (!more) break;
        i = inext;
        cg = ng;
        cu = nu;
    }
}

// SwiGLU over an fp32 [M, 2F] matrix whose columns hold gate and up values
// interleaved in blocks of 32 (the fused gate/up layout); out bf16 [M, F].
// Thread = 8 consecutive features of one row.
__global__ void swiglu_interleaved_kernel(const float* __restrict__ gu, uint16_t* out, int M, int F) {
    const long long per_row = F / 8;
    const long long total = (long long)M * per_row;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(e / per_row);
        const int f0 = (int)(e - (long long)m * per_row) * 8;
        const float* row = gu + (size_t)m * 2 * F;
        const int gcol = (f0 / 32) * 64 + (f0 % 32);
        float g[8], u[8], o[8];
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(row + gcol));
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(row + gcol + 4));
        const float4 u0 = __ldg(reinterpret_cast<const float4*>(row + gcol + 32));
        const float4 u1 = __ldg(reinterpret_cast<const float4*>(row + gcol + 36));
        g[0] = g0.x, g[1] = g0.y, g[2] = g0.z, g[3] = g0.w, g[4] = g1.x, g[5] = g1.y, g[6] = g1.z, g[7] = g1.w;
        u[0] = u0.x, u[1] = u0.y, u[2] = u0.z, u[3] = u0.w, u[4] = u1.x, u[5] = u1.y, u[6] = u1.z, u[7] = u1.w;
#pragma unroll
        for (int k = 0; k < 8; k += 2) swiglu2(g[k], g[k + 1], u[k], u[k + 1], o[k], o[k + 1]);
        *reinterpret_cast<uint4*>(out + (size_t)m * F + f0) = pack8(o);
    }
}

}  // namespace tbik
