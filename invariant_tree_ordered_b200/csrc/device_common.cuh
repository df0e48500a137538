// Device-side helpers shared by the library's kernels: bf16 conversion, the
// error word, bounded waits, the tree walk and thin inline-PTX wrappers for
// mbarrier, TMA (cp.async.bulk.tensor) and tcgen05 (sm_100a), written from the
// PTX ISA description of those instructions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tbik.h"

namespace tbik {

// ------------------------------------------------------------------ errors

// Per-device error word: the first device-detected error wins.
__device__ unsigned int g_err;

__device__ __forceinline__ void set_error(unsigned code) { atomicCAS(&g_err, 0u, code); }

// ------------------------------------------------------------------ bf16

__device__ __forceinline__ float bf2f(uint16_t h) { return __uint_as_float(((uint32_t)h) << 16); }

// fp32 -> bf16 bits, round to nearest even (NaN stays NaN).
__device__ __forceinline__ uint16_t f2bf(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}

// Two values in one instruction (cvt.rn.bf16x2.f32): the same rounding as f2bf.
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}

// eight bf16 values in a 16-byte vector <-> fp32 (exact widening; RNE narrowing)
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

// ----------------------------------------------------- exp / log specs
// Cody-Waite style specifications (W. J. Cody and W. Waite, "Software Manual
// for the Elementary Functions", 1980): additive reduction by a split ln 2 and
// a short polynomial.  Every operation is an explicit round-to-nearest
// intrinsic so the compiler cannot contract or reorder it.

__device__ __forceinline__ float pow2i(int n) { return __uint_as_float((uint32_t)(n + 127) << 23); }

// e^x: clamp to [-104, 89]; k = rint(x*log2e); r = (x - k*ln2hi) - k*ln2lo;
// degree-7 Taylor polynomial of e^r (coefficients: nearest floats to 1/n!);
// scale by 2^(k/2) exactly, then by 2^(k-k/2) (one rounding).
// Instruction choices that keep those bits: rint of y = x*log2e (|y| < 151)
// is (y + 1.5*2^23) - 1.5*2^23 in round-to-nearest-even, and the integer k
// sits in the low bits of that sum.  |r| <= ln2/2 (plus rounding), so p lies
// in [0.70, 1.42] and has exponent -1 or 0; for k in [-125, 127] the product
// p*2^k is then a normal float, exact, and its bits are p's with k added to
// the exponent field (one integer add).  Other k take the two-step scaling.
__device__ __forceinline__ float exp_spec(float x) {
    if (x != x) return __fadd_rn(x, x);
    x = fminf(fmaxf(x, -104.0f), 89.0f);
    const float log2e = 0x1.715476p+0f, ln2hi = 0x1.62e4p-1f, ln2lo = 0x1.7f7d1cp-20f;
    const float t = __fadd_rn(__fmul_rn(x, log2e), 0x1.8p23f);
    const float kf = __fsub_rn(t, 0x1.8p23f);
    const int k = __float_as_int(t) - 0x4b400000;
    float r = __fmaf_rn(-kf, ln2hi, x);
    r = __fmaf_rn(-kf, ln2lo, r);
    float p = 0x1.a01a02p-13f;
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);
    p = __fmaf_rn(p, r, 0x1.111112p-7f);
    p = __fmaf_rn(p, r, 0x1.555556p-5f);
    p = __fmaf_rn(p, r, 0x1.555556p-3f);
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    if (k >= -125 && k <= 127) return __int_as_float(__float_as_int(p) + (int)((uint32_t)k << 23));
    const int k1 = k / 2;
    const int k2 = k - k1;
    return __fmul_rn(__fmul_rn(p, pow2i(k1)), pow2i(k2));
}

// SwiGLU of one element in fp32: (g / (1 + exp(-g))) * u, each step one
// correctly rounded operation (rounding-location alignment article, winzheng.jp,
// section "外科手術的な修正：3つのノード": fp32 intermediates, one rounding at the
// output, which the caller applies).
__device__ __forceinline__ float swiglu1(float g, float u) {
    const float e = exp_spec(-g);
    const float den = __fadd_rn(1.0f, e);
    const float sg = __fdiv_rn(g, den);
    return __fmul_rn(sg, u);
}

// Three-input maximum (max.f32 with three sources, sm_100): the largest of a,
// b, c, exactly (no rounding), NaN inputs ignored as by fmaxf.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// ---- two lanes per instruction (packed f32x2 add / mul / fma, sm_100) ------
// Each lane of a packed operation is the IEEE round-to-nearest-even result of
// the scalar operation on that lane, so the paired forms below return exactly
// the bits of their scalar counterparts while issuing half the instructions.
typedef unsigned long long f2x;

__device__ __forceinline__ f2x pk2(float lo, float hi) {
    f2x d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ void upk2(f2x v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f2x add2(f2x a, f2x b) {
    f2x d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2x mul2(f2x a, f2x b) {
    f2x d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2x fma2(f2x a, f2x b, f2x c) {
    f2x d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// The scaling step of exp_spec for one lane: p * 2^k from the rint sum t.
__device__ __forceinline__ float exp_scale(float p, float t) {
    const int k = __float_as_int(t) - 0x4b400000;
    if (k >= -125 && k <= 127) return __int_as_float(__float_as_int(p) + (int)((uint32_t)k << 23));
    const int k1 = k / 2;
    const int k2 = k - k1;
    return __fmul_rn(__fmul_rn(p, pow2i(k1)), pow2i(k2));
}

// exp_spec of two values with the same operations in the same order: the
// clamp, the rint by 1.5*2^23, the two-fma reduction (fma(-k, c, x) written as
// fma(k, -c, x), the same exact product), the Horner polynomial and the scaling.
__device__ __forceinline__ void exp_spec2(float x0, float x1, float& e0, float& e1) {
    const float c0 = fminf(fmaxf(x0, -104.0f), 89.0f), c1 = fminf(fmaxf(x1, -104.0f), 89.0f);
    const f2x x = pk2(c0, c1);
    const f2x big = pk2(0x1.8p23f, 0x1.8p23f);
    const f2x t = add2(mul2(x, pk2(0x1.715476p+0f, 0x1.715476p+0f)), big);
    const f2x kf = add2(t, pk2(-0x1.8p23f, -0x1.8p23f));
    f2x r = fma2(kf, pk2(-0x1.62e4p-1f, -0x1.62e4p-1f), x);
    r = fma2(kf, pk2(-0x1.7f7d1cp-20f, -0x1.7f7d1cp-20f), r);
    f2x p = pk2(0x1.a01a02p-13f, 0x1.a01a02p-13f);
    p = fma2(p, r, pk2(0x1.6c16c2p-10f, 0x1.6c16c2p-10f));
    p = fma2(p, r, pk2(0x1.111112p-7f, 0x1.111112p-7f));
    p = fma2(p, r, pk2(0x1.555556p-5f, 0x1.555556p-5f));
    p = fma2(p, r, pk2(0x1.555556p-3f, 0x1.555556p-3f));
    p = fma2(p, r, pk2(0.5f, 0.5f));
    p = fma2(p, r, pk2(1.0f, 1.0f));
    p = fma2(p, r, pk2(1.0f, 1.0f));
    float p0, p1, t0, t1;
    upk2(p, p0, p1);
    upk2(t, t0, t1);
    e0 = (x0 != x0) ? __fadd_rn(x0, x0) : exp_scale(p0, t0);
    e1 = (x1 != x1) ? __fadd_rn(x1, x1) : exp_scale(p1, t1);
}

// swiglu1 of two elements: the exponential, the "1 +" and the product by u
// packed; the correctly rounded division stays one per lane.
__device__ __forceinline__ void swiglu2(float g0, float g1, float u0, float u1, float& o0, float& o1) {
    float e0, e1;
    exp_spec2(-g0, -g1, e0, e1);
    float d0, d1;
    upk2(add2(pk2(1.0f, 1.0f), pk2(e0, e1)), d0, d1);
    const f2x sg = pk2(__fdiv_rn(g0, d0), __fdiv_rn(g1, d1));
    upk2(mul2(sg, pk2(u0, u1)), o0, o1);
}

// 2^y through the hardware base-2 exponential (ex2.approx, denormal results
// flushed to zero).  Used where results are compared by tolerance (the
// tensor-core logprob's per-leaf sums of exp(z - max), whose terms are at
// most 1 and whose sum is at least 1, so a flushed term below 2^-126 never
// changes the sum), never in the exact-order path.
__device__ __forceinline__ float ex2_hw(float y) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}

// log x for x > 0: x = 2^e * m, m in [sqrt(1/2), sqrt 2]; t = f/(2+f), f = m-1;
// log m = s + s*w*(1/3 + w/5 + w^2/7 + w^3/9 + w^4/11), s = 2t, w = t^2;
// result = e*ln2hi + (e*ln2lo + log m).
__device__ __forceinline__ float log_spec(float x) {
    if (x != x) return __fadd_rn(x, x);
    if (x < 0.0f) return __int_as_float(0x7fc00000);
    if (x == 0.0f) return -INFINITY;
    if (x == INFINITY) return x;
    int e = 0;
    uint32_t u = __float_as_uint(x);
    if (u < 0x00800000u) {
        x = __fmul_rn(x, 0x1p23f);
        u = __float_as_uint(x);
        e = -23;
    }
    e += (int)(u >> 23) - 127;
    float m = __uint_as_float((u & 0x007fffffu) | 0x3f800000u);
    if (m > 0x1.6a09e6p+0f) {
        m = __fmul_rn(m, 0.5f);
        e += 1;
    }
    float f = __fsub_rn(m, 1.0f);
    float t = __fdiv_rn(f, __fadd_rn(2.0f, f));
    float w = __fmul_rn(t, t);
    float q = 0x1.745d18p-4f;
    q = __fmaf_rn(q, w, 0x1.c71c72p-4f);
    q = __fmaf_rn(q, w, 0x1.24924ap-3f);
    q = __fmaf_rn(q, w, 0x1.99999ap-3f);
    q = __fmaf_rn(q, w, 0x1.555556p-2f);
    float s = __fadd_rn(t, t);
    float lm = __fmaf_rn(__fmul_rn(s, w), q, s);
    float ef = (float)e;
    float r = __fmaf_rn(ef, 0x1.7f7d1cp-20f, lm);
    return __fmaf_rn(ef, 0x1.62e4p-1f, r);
}

// (max, sum-exp) summary and its combine (identity: -inf, 0).  `a` is the left
// operand of the tree; the larger-of rule keeps `a` on ties.
struct MS {
    float m, s;
};

__device__ __forceinline__ MS ms_combine(MS a, MS b) {
    MS r;
    r.m = (b.m > a.m) ? b.m : a.m;
    if (r.m == -INFINITY) {
        r.s = 0.0f;
        return r;
    }
    // the side that holds the max has the factor exp(+0) = 1 exactly (the
    // specification returns 1 for +0), so it is not evaluated
    const bool finite = r.m != INFINITY;
    const float ea = (finite && a.m == r.m) ? 1.0f : exp_spec(__fsub_rn(a.m, r.m));
    const float eb = (finite && b.m == r.m) ? 1.0f : exp_spec(__fsub_rn(b.m, r.m));
    r.s = __fadd_rn(__fmul_rn(a.s, ea), __fmul_rn(b.s, eb));
    return r;
}

// ------------------------------------------------------------- tree walk

// Streaming (post-order) evaluation of TREE over n leaves.  After leaf j
// arrives, the nodes whose last leaf is j close, deepest first; each close adds
// the pending result of that node's left child.  The closing nodes form the
// deepest part of j's root path, and their left children shrink with depth, so
// pending values are popped smallest first.  The shallowest closed node (or the
// leaf itself) is then pushed, unless it is the root.  Pending values are
// counted by size class: 1 leaf, 2 leaves, 3-4 leaves, >= 5 leaves (a pending
// single leaf is always consumed by the very next leaf; at most one value of 2
// and one of 3-4 leaves is ever pending).  Computed in registers only.
struct LeafOps {
    int n1, n2, nm, nb;  // pops per size class (1, 2, 3-4, >= 5 leaves)
    int push_size;       // leaves of the value left after the pops
    bool final_;         // that value is the root of the tree over n leaves
    bool c2_pend;        // a 2-leaf value is pending when leaf j arrives
    bool m_pend;         // a 3-4 leaf value is pending when leaf j arrives
};

__host__ __device__ __forceinline__ LeafOps leaf_ops(int n, int j) {
    LeafOps o;
    o.n1 = o.n2 = o.nm = o.nb = 0;
    o.c2_pend = o.m_pend = false;
    int lo = 0, sz = n, top = 1;
    bool closing = false;
    while (sz > 1) {
        const int h = (sz + 1) >> 1;
        // the left children of the nodes where j lies right are the pending values
        if (j >= lo + h && h == 2) o.c2_pend = true;
        if (j >= lo + h && (h == 3 || h == 4)) o.m_pend = true;
        if (!closing && lo + sz - 1 == j) {
            closing = true;
            top = sz;
        }
        if (closing) {
            if (h == 1)
                ++o.n1;
            else if (h == 2)
                ++o.n2;
            else if (h <= 4)
                ++o.nm;
            else
                ++o.nb;
        }
        if (j < lo + h) {
            sz = h;
        } else {
            lo += h;
            sz -= h;
        }
    }
    o.push_size = top;
    o.final_ = (top == n);
    return o;
}

// The same operations for the left-to-right chain ((L0 + L1) + L2) + ... of
// the non-invariant baseline: leaf j > 0 pops the running sum of j leaves.
__host__ __device__ __forceinline__ LeafOps seq_leaf_ops(int n, int j) {
    LeafOps o;
    o.n1 = o.n2 = o.nm = o.nb = 0;
    o.c2_pend = (j == 2);
    o.m_pend = (j == 3 || j == 4);
    if (j == 1)
        o.n1 = 1;
    else if (j == 2)
        o.n2 = 1;
    else if (j == 3 || j == 4)
        o.nm = 1;
    else if (j >= 5)
        o.nb = 1;
    o.push_size = j + 1;
    o.final_ = (j == n - 1);
    return o;
}

__host__ __device__ __forceinline__ int leaf_pops(const LeafOps& o) { return o.n1 + o.n2 + o.nm + o.nb; }

// A leaf's operations packed in 16 bits, so a table built once per CTA replaces
// the walk (which costs several hundred cycles of dependent branches):
// bit 0 pop of a single leaf, bit 1 pop of a 2-leaf value, bit 2 pop of a 3-4
// leaf value, bits 3-7 pops of >= 5 leaf values, bits 8-9 size class of the
// pushed value (0: 1 leaf, 1: 2, 2: 3-4, 3: >= 5), bit 10 final, bit 11 a
// 2-leaf value is pending when the leaf arrives, bit 12 a 3-4 leaf value is.
__host__ __device__ __forceinline__ uint16_t encode_leaf_ops(const LeafOps& o) {
    const int cls = o.push_size == 1 ? 0 : (o.push_size == 2 ? 1 : (o.push_size <= 4 ? 2 : 3));
    return (uint16_t)(o.n1 | (o.n2 << 1) | (o.nm << 2) | (o.nb << 3) | (cls << 8) | ((o.final_ ? 1 : 0) << 10) |
                      ((o.c2_pend ? 1 : 0) << 11) | ((o.m_pend ? 1 : 0) << 12));
}

__host__ __device__ __forceinline__ int code_pops(uint32_t code) {
    return (code & 1) + ((code >> 1) & 1) + ((code >> 2) & 1) + ((code >> 3) & 31);
}

// ------------------------------------------------------------ PTX: misc

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------ PTX: CTA pairs
// Thread-block clusters of two CTAs run one 256-row MMA tile (cta_group::2):
// rank 0 (the leader) issues the MMAs; each CTA holds its own 128 rows of A
// and 64 of the 128 B rows/columns in shared memory at the same offsets.

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Arrive once on an mbarrier anywhere in the cluster (default semantics; the
// tcgen05 reads it publishes are ordered by tcgen05.fence::before_thread_sync).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

// ---------------------------------------------------------- PTX: mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Named hardware barrier over `count` threads (ids 1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// The same barrier with an OR reduction of a predicate: every participating
// thread gets the same result, so a decision to give up (a bounded wait that
// expired, the abort flag) is taken by all of them together and no thread is
// left waiting at a later barrier for one that has left.
__device__ __forceinline__ bool named_barrier_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on one phase of an mbarrier.  Gives up (returns false) when the
// CTA-wide abort flag is raised by another role, or after limit_cycles SM
// clock cycles, in which case it records TBIK_ERR_TIMEOUT and raises the abort
// flag itself.  The SM-local cycle counter is read only every 64 misses so the
// common path is a bare try_wait.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_cycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((uint64_t)(clock64() - t0) > limit_cycles) {
            *abort_flag = 1;
            set_error(TBIK_ERR_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait used on the way out: no abort check, only the cycle limit.
__device__ __forceinline__ bool mbar_drain(uint64_t* bar, uint32_t parity, uint64_t limit_cycles) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if ((uint64_t)(clock64() - t0) > limit_cycles) {
            set_error(TBIK_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// --------------------------------------------------------------- PTX: TMA

// Pair form: the copy lands in this CTA's shared memory and completes its bytes
// on an mbarrier that may be in the peer CTA (cluster address).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const void* tmap, uint32_t bar_cluster, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 2-D tiled bulk tensor load global -> shared, completion counted in bytes on `bar`.
// x is the innermost coordinate (elements); it must be a multiple of 8 for bf16.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 4-D tiled bulk tensor load (coordinates innermost first); same rules as the 2-D form.
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y, int z,
                                            int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

// Generic-proxy writes to shared memory become visible to the async proxy
// (TMA, tcgen05.mma operand reads) issued after this fence.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ PTX: tcgen05
// (cta_group::2 forms: executed by one warp / thread per the PTX ISA rules;
// alloc, relinquish and dealloc are collective over one warp of each CTA.)

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the mbarrier at this offset in both CTAs of the pair when every
// tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"((uint16_t)3)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// row (lane base + t), columns [col, col+32).  The _nowait form only issues the
// load; tmem_wait_ld() must complete it before the registers are read.
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// Waits for every outstanding tcgen05.ld of this thread; the register
// operands tie the loaded values to the wait so no use is hoisted above it.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&a)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]), "+r"(a[14]), "+r"(a[15]), "+r"(a[16]), "+r"(a[17]), "+r"(a[18]), "+r"(a[19]), "+r"(a[20]), "+r"(a[21]), "+r"(a[22]), "+r"(a[23]), "+r"(a[24]), "+r"(a[25]), "+r"(a[26]), "+r"(a[27]), "+r"(a[28]), "+r"(a[29]), "+r"(a[30]), "+r"(a[31]) :: "memory");
}

// Orders later uses of b after a preceding tmem_wait_ld (volatile asm keeps order).
__device__ __forceinline__ void tie32(uint32_t (&b)[32]) { asm volatile("" : "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]), "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15]), "+r"(b[16]), "+r"(b[17]), "+r"(b[18]), "+r"(b[19]), "+r"(b[20]), "+r"(b[21]), "+r"(b[22]), "+r"(b[23]), "+r"(b[24]), "+r"(b[25]), "+r"(b[26]), "+r"(b[27]), "+r"(b[28]), "+r"(b[29]), "+r"(b[30]), "+r"(b[31])); }

// Two 32-column loads and their wait in one statement: the registers are
// defined only once the data has arrived, so no copy of them can be taken early.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t (&a)[32], uint32_t tb, uint32_t (&b)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31]),
          "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]), "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15]), "=r"(b[16]), "=r"(b[17]), "=r"(b[18]), "=r"(b[19]), "=r"(b[20]), "=r"(b[21]), "=r"(b[22]), "=r"(b[23]), "=r"(b[24]), "=r"(b[25]), "=r"(b[26]), "=r"(b[27]), "=r"(b[28]), "=r"(b[29]), "=r"(b[30]), "=r"(b[31])
        : "r"(ta), "r"(tb)
        : "memory");
}

// 32 lanes x 16 consecutive columns (the x16 shape of the load above).
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&a)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]), "+r"(a[14]), "+r"(a[15]) :: "memory");
}
__device__ __forceinline__ void tie16(uint32_t (&b)[16]) { asm volatile("" : "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]), "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15])); }

// 32 lanes x 64 consecutive columns (the x64 shape), one wait for all of them.
__device__ __forceinline__ void tmem_ld64_nowait(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld64(uint32_t (&a)[64]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]), "+r"(a[14]), "+r"(a[15]), "+r"(a[16]), "+r"(a[17]), "+r"(a[18]), "+r"(a[19]), "+r"(a[20]), "+r"(a[21]), "+r"(a[22]), "+r"(a[23]), "+r"(a[24]), "+r"(a[25]), "+r"(a[26]), "+r"(a[27]), "+r"(a[28]), "+r"(a[29]), "+r"(a[30]), "+r"(a[31]), "+r"(a[32]), "+r"(a[33]), "+r"(a[34]), "+r"(a[35]), "+r"(a[36]), "+r"(a[37]), "+r"(a[38]), "+r"(a[39]), "+r"(a[40]), "+r"(a[41]), "+r"(a[42]), "+r"(a[43]), "+r"(a[44]), "+r"(a[45]), "+r"(a[46]), "+r"(a[47]), "+r"(a[48]), "+r"(a[49]), "+r"(a[50]), "+r"(a[51]), "+r"(a[52]), "+r"(a[53]), "+r"(a[54]), "+r"(a[55]), "+r"(a[56]), "+r"(a[57]), "+r"(a[58]), "+r"(a[59]), "+r"(a[60]), "+r"(a[61]), "+r"(a[62]), "+r"(a[63]) :: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    tmem_ld32_nowait(taddr, r);
    tmem_wait_ld(r);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Issues the store only; tmem_wait_st() completes every outstanding store.
__device__ __forceinline__ void tmem_st32_nowait(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for tcgen05.mma (PTX ISA, "Shared memory
// descriptor"): start address >> 4 in bits [0,14), leading byte offset >> 4 in
// [16,30), stride byte offset >> 4 in [32,46), fixed 0b001 in [46,49), base
// offset 0, swizzle mode in [61,64) (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// The same with the 64-byte swizzle (mode 4): atoms of 8 rows x 64 bytes.
__device__ __forceinline__ uint64_t smem_desc_sw64(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)4 << 61;
    return d;
}

// Instruction descriptor for kind::f16 (PTX ISA, "Instruction descriptor"):
// D format f32 (bits 4-5 = 1), A and B bf16 (bits 7-9 = 1, 10-12 = 1),
// A/B major in bits 15/16 (0 = K-major, 1 = MN-major), N>>3 in bits 17-22,
// M>>4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace tbik
