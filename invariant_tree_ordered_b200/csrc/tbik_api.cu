// Host side of the C ABI declared in include/tbik.h: argument checks, the
// launch plan (frontier split of the tree, workspace carving), TMA tensor
// maps and kernel launches.  One translation unit holds every kernel so the
// device error word is a single symbol per device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "device_common.cuh"
#include "gemm_exact.cuh"
#include "gemm_tc.cuh"
#include "attention_tc.cuh"
#include "logprob.cuh"
#include "attention.cuh"
#include "reduce.cuh"
#include "tbik.h"

namespace {

using namespace tbik;

constexpr unsigned kModeMask = TBIK_EXACT | TBIK_TC | TBIK_NONINV | TBIK_B_NK | TBIK_OUT_BF16 | TBIK_SWIGLU_OUT;
constexpr int kMaxDevices = 64;

unsigned g_debug_flags = 0;
unsigned long long g_wait_ns = 2000000000ull;

struct DeviceInfo {
    bool init = false;
    bool ok = false;
    int sms = 0;
    int clock_khz = 0;
    bool attrs_set = false;
    cudaEvent_t lut_built = nullptr;  // the SwiGLU table's build, recorded on the stream that ran it
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

tbik_status device_info(int& dev, DeviceInfo*& info) {
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TBIK_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.init) {
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return TBIK_ERR_CUDA;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return TBIK_ERR_CUDA;
        if (cudaDeviceGetAttribute(&d.clock_khz, cudaDevAttrClockRate, dev) != cudaSuccess || d.clock_khz <= 0)
            d.clock_khz = 2000000;
        d.ok = (major == 10);
        d.init = true;
    }
    info = &d;
    if (!d.ok) return TBIK_ERR_UNSUPPORTED;
    if (!d.attrs_set) {
        const int s128 = (int)TcCfg<TC_BN>::SMEM_BYTES, s192 = (int)TcCfg<TC_BN_WIDE>::SMEM_BYTES;
        const auto attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
        if (cudaFuncSetAttribute(gemm_tc_kernel<EPI_TREE, TC_BN>, attr, s128) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_tc_kernel<EPI_TREE_RES, TC_BN>, attr, s128) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_tc_kernel<EPI_TREE, TC_BN_WIDE>, attr, s192) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_tc_kernel<EPI_TREE_RES, TC_BN_WIDE>, attr, s192) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_tc_kernel<EPI_LOGPROB, TC_BN_WIDE>, attr, s192) != cudaSuccess ||
            cudaFuncSetAttribute(attention_tc_kernel, attr, (int)ATC_SMEM_BYTES) != cudaSuccess)
            return TBIK_ERR_CUDA;
        d.attrs_set = true;
    }
    return TBIK_OK;
}

// ---------------------------------------------------------------- TMA maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 row-major matrix with `inner` contiguous elements per row and `outer`
// rows; box = box_inner x box_outer elements, 128-byte (or 64-byte) swizzle,
// zero OOB fill.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
              uint32_t box_outer, bool swizzle64 = false) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [batch][seq][heads][head_dim] tensor (head_dim contiguous) as a 4-D map
// {head_dim, heads, seq, batch}; box = 64 dims x 1 head x `rows` positions x 1
// batch, 128-byte swizzle, zero OOB fill.
bool make_map_bshd(CUtensorMap* m, const void* base, int batch, int seq, int heads, int hd, uint32_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)hd, (cuuint64_t)heads, (cuuint64_t)seq, (cuuint64_t)batch};
    cuuint64_t strides[3] = {(cuuint64_t)hd * 2, (cuuint64_t)heads * hd * 2, (cuuint64_t)seq * heads * hd * 2};
    cuuint32_t box[4] = {64, 1, rows, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------- tree plan

// Grid for a kernel that loops over work items (tokens): as many CTAs as are
// resident on the device at once, at most one per item.
template <typename Kernel, typename... Args>
void launch_token_loop(Kernel kernel, int threads, int items, const DeviceInfo* info, cudaStream_t s, Args... args) {
    // resident CTAs per SM, looked up once per (kernel, device)
    struct Entry {
        const void* fn;
        int dev, per_sm;
    };
    static Entry cache[64];
    static int used = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        for (int i = 0; i < used; ++i)
            if (cache[i].fn == reinterpret_cast<const void*>(kernel) && cache[i].dev == dev) per_sm = cache[i].per_sm;
    }
    if (per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        std::lock_guard<std::mutex> lock(g_mu);
        if (used < 64) cache[used++] = Entry{reinterpret_cast<const void*>(kernel), dev, per_sm};
    }
    const long long resident = (long long)per_sm * info->sms;
    const int grid = (int)(items < resident ? items : resident);
    kernel<<<grid, threads, 0, s>>>(args...);
}

// Rows of A per TMA copy in the tensor-core kernel: the whole 128-row half
// tile, or only M rounded up to a whole 8-row swizzle atom when M <= 128.
int a_box_rows(int M) { return M >= TC_BM ? TC_BM : ((M + 7) / 8) * 8; }

// Ring of the tensor-core kernel: with a small A copy (small M) the same
// shared memory holds more stages of B, i.e. more bytes in flight.
template <int BN>
void set_ring(TcParams& prm, int a_box) {
    using Cfg = TcCfg<BN>;
    prm.a_box_rows = a_box;
    prm.a_slice = (uint32_t)a_box * 128u;
    prm.stage_bytes = (uint32_t)Cfg::KSLICES * prm.a_slice + (uint32_t)Cfg::B_BYTES;
    const int st = (int)(Cfg::RING_BYTES / prm.stage_bytes);
    prm.stages = st < TC_MAX_STAGES ? st : TC_MAX_STAGES;
}

// Pair-tile width of the tensor-core GEMM: 192 columns (a [K,N] B in
// 64-byte-swizzle atoms of 32 columns), except for a [K,N] B of at most 128
// columns, which fills one 128-column tile.  It depends on N and the operand
// layout only, never on M or T (and both widths give the same bits).
int tc_tile_n(bool b_nk, int N) {
    if (g_debug_flags & TBIK_DEBUG_TILE128) return TC_BN;
    return (b_nk || N > TC_BN) ? TC_BN_WIDE : TC_BN;
}
size_t tc_slot_bytes(int bn) { return (size_t)TC_BM * bn * sizeof(float); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
int ilog2(int x) {
    int r = 0;
    while ((1 << (r + 1)) <= x) ++r;
    return r;
}
bool valid_T(int T) { return T == 1 || T == 2 || T == 4 || T == 8; }

// Nodes at depth D of the halving tree over [lo, lo+n), left to right.
void frontier(int lo, int n, int D, std::vector<std::pair<int, int>>& out) {
    if (D == 0 || n == 1) {
        out.emplace_back(lo, n);
        return;
    }
    int h = (n + 1) / 2;
    frontier(lo, h, D - 1, out);
    frontier(lo + h, n - h, D - 1, out);
}

// Largest number of simultaneously pending left subtrees of >= 5 leaves while
// streaming the tree over n leaves (they live in the global scratch).
int max_big_pending(int n) {
    if (n <= 1) return 0;
    int h = (n + 1) / 2;
    int l = max_big_pending(h);
    int r = max_big_pending(n - h) + (h >= 5 ? 1 : 0);
    return l > r ? l : r;
}
int max_stack_depth(int n) {
    if (n <= 1) return 0;
    int h = (n + 1) / 2;
    int l = max_stack_depth(h);
    int r = max_stack_depth(n - h) + 1;
    return l > r ? l : r;
}

struct GemmPlan {
    bool tc = false, noninv = false, b_nk = false, out_bf16 = false;
    bool swiglu = false, fused = false;  // SwiGLU output; applied in the TC epilogue when fused
    int M = 0, N = 0, K = 0, T = 1, leaf = 1;
    int L = 0, D = 0, F = 1;
    int tiles_m = 0, tiles_n = 0, units = 0, grid = 0, gs = 0;
    int bn = 0;  // output columns per tile (pair tile in TC mode)
    bool direct = true;
    std::vector<std::pair<int, int>> nodes;  // (first leaf, leaves) per frontier node
    int leaf_eff = 1;                        // K elements per leaf as launched
    size_t off_partials = 0, off_shards = 0, off_scratch = 0, off_gu = 0, total = 0;
};

tbik_status plan_gemm(int M, int N, int K, int T, int leaf, unsigned mode, int sms, GemmPlan& p) {
    if (mode & ~kModeMask) return TBIK_ERR_ARG;
    const bool exact = mode & TBIK_EXACT, tc = mode & TBIK_TC;
    if (exact == tc) return TBIK_ERR_ARG;
    if (M < 0 || N <= 0 || K <= 0 || leaf <= 0) return TBIK_ERR_ARG;
    if (!valid_T(T) || K % leaf) return TBIK_ERR_SHAPE;
    p.tc = tc;
    p.noninv = mode & TBIK_NONINV;
    p.b_nk = mode & TBIK_B_NK;
    p.out_bf16 = mode & TBIK_OUT_BF16;
    p.swiglu = mode & TBIK_SWIGLU_OUT;
    if (p.swiglu && p.noninv) return TBIK_ERR_ARG;
    if (p.swiglu && N % 64) return TBIK_ERR_SHAPE;
    if (p.swiglu) p.out_bf16 = false;  // the tree roots stay fp32 until the SwiGLU
    p.M = M, p.N = N, p.K = K, p.T = T, p.leaf = leaf;
    p.L = K / leaf;
    if (p.L % T) return TBIK_ERR_SHAPE;
    const int bm = tc ? TC_PAIR_M : EX_BM, bn = tc ? tc_tile_n(p.b_nk, N) : EX_BN;
    p.bn = bn;
    if (tc) {
        if (N % 8 || K % 8) return TBIK_ERR_SHAPE;
        if (p.noninv ? (K / T) % 16 : leaf % 16) return TBIK_ERR_SHAPE;
    }
    p.tiles_m = (M + bm - 1) / bm;
    p.tiles_n = (N + bn - 1) / bn;
    const long long tiles = (long long)p.tiles_m * p.tiles_n;
    p.nodes.clear();
    if (p.noninv) {
        p.leaf_eff = K / T;
        p.D = ilog2(T);
        p.F = T;
        for (int t = 0; t < T; ++t) p.nodes.emplace_back(t, 1);
    } else {
        p.leaf_eff = leaf;
        const int d0 = ilog2(T);
        int dmax = ilog2(p.L);
        if (dmax > 6) dmax = 6;
        if (tc ? false : (max_stack_depth(p.L) > EX_MAXD)) return TBIK_ERR_SHAPE;
        const long long want = tc ? sms / 2 : 2LL * sms;  // CTA pairs / CTAs
        int D = d0;
        while (D < dmax && tiles * (1LL << D) < want) ++D;
        p.D = D;
        frontier(0, p.L, D, p.nodes);
        p.F = (int)p.nodes.size();
        if (p.F != (1 << D)) return TBIK_ERR_SHAPE;  // cannot happen for 2^D <= L
    }
    if (p.nodes.size() > (size_t)TC_MAX_F) return TBIK_ERR_SHAPE;
    for (auto& nd : p.nodes)
        if (nd.first > 32767 || nd.second > 32767) return TBIK_ERR_SHAPE;
    p.direct = (p.F == 1);
    const long long units = tiles * p.F;
    if (units > 0x7fffffffLL) return TBIK_ERR_SHAPE;
    p.units = (int)units;
    if (tc) {
        const int pairs = p.units < sms / 2 ? p.units : sms / 2;
        p.grid = 2 * (pairs > 0 ? pairs : 1);
    } else {
        p.grid = p.units < sms ? p.units : sms;
        if (p.grid < 1) p.grid = 1;
    }
    p.gs = 0;
    if (tc)
        for (auto& nd : p.nodes) {
            int g = max_big_pending(nd.second);
            if (g > p.gs) p.gs = g;
        }
    size_t off = 0;
    const size_t mn = (size_t)M * N * sizeof(float);
    if (!p.direct) {
        p.off_partials = off;
        off = align256(off + (size_t)p.F * mn);
        if (!p.noninv && T > 1 && p.F > T) {
            p.off_shards = off;
            off = align256(off + (size_t)T * mn);
        }
    }
    if (tc && p.gs > 0) {
        p.off_scratch = off;
        off = align256(off + (size_t)p.grid * p.gs * tc_slot_bytes(bn));
    }
    p.fused = p.swiglu && tc && p.direct;
    if (p.swiglu && !p.fused) {  // fp32 gate/up roots, then the SwiGLU kernel
        p.off_gu = off;
        off = align256(off + mn);
    }
    p.total = off;
    return TBIK_OK;
}

tbik_status launch_status() { return cudaGetLastError() == cudaSuccess ? TBIK_OK : TBIK_ERR_CUDA; }

// 16-byte vectors when M*N % 4 == 0 (every partial buffer then starts on a
// 16-byte boundary), else the element loop.
template <int G>
void launch_tree_combine(const float* P, size_t MN, int groups, void* out, int bf16, const uint16_t* R,
                         cudaStream_t s, int sms) {
    const bool vec = (MN % 4) == 0;
    const size_t work = (vec ? MN / 4 : MN) * groups;
    size_t blocks = (work + 255) / 256;
    if (blocks > (size_t)sms * 8) blocks = (size_t)sms * 8;
    if (blocks < 1) blocks = 1;
    if (vec)
        tree_combine_kernel<G, 1><<<(int)blocks, 256, 0, s>>>(P, MN, groups, out, bf16, R);
    else
        tree_combine_kernel<G, 0><<<(int)blocks, 256, 0, s>>>(P, MN, groups, out, bf16, R);
}

tbik_status tree_combine(const float* P, size_t MN, int G, int groups, void* out, int bf16, cudaStream_t s,
                         int sms, const uint16_t* R = nullptr) {
    switch (G) {
        case 1: launch_tree_combine<1>(P, MN, groups, out, bf16, R, s, sms); break;
        case 2: launch_tree_combine<2>(P, MN, groups, out, bf16, R, s, sms); break;
        case 4: launch_tree_combine<4>(P, MN, groups, out, bf16, R, s, sms); break;
        case 8: launch_tree_combine<8>(P, MN, groups, out, bf16, R, s, sms); break;
        case 16: launch_tree_combine<16>(P, MN, groups, out, bf16, R, s, sms); break;
        case 32: launch_tree_combine<32>(P, MN, groups, out, bf16, R, s, sms); break;
        case 64: launch_tree_combine<64>(P, MN, groups, out, bf16, R, s, sms); break;
        default: return TBIK_ERR_SHAPE;
    }
    return launch_status();
}

// Upper levels of the tree after the GEMM wrote F frontier partials (and the
// residual R, when given, added to the root before its bf16 rounding).
tbik_status finish_gemm(const GemmPlan& p, uint8_t* ws, void* C, cudaStream_t s, int sms, const uint16_t* R) {
    if (p.direct) return TBIK_OK;
    const float* P = reinterpret_cast<const float*>(ws + p.off_partials);
    const size_t MN = (size_t)p.M * p.N;
    if (p.noninv) {
        int blocks = (int)((MN + 255) / 256);
        if (blocks > sms * 8) blocks = sms * 8;
        seq_combine_kernel<<<blocks, 256, 0, s>>>(P, MN, p.T, C, p.out_bf16, R);
        return launch_status();
    }
    if (p.T == 1 || p.F == p.T) return tree_combine(P, MN, p.F, 1, C, p.out_bf16, s, sms, R);
    // T > 1 and F > T: shard partials first (one fp32 buffer per shard), then
    // the cross-shard levels.
    float* Q = reinterpret_cast<float*>(ws + p.off_shards);
    tbik_status st = tree_combine(P, MN, p.F / p.T, p.T, Q, 0, s, sms);
    if (st != TBIK_OK) return st;
    return tree_combine(Q, MN, p.T, 1, C, p.out_bf16, s, sms, R);
}

// Wait bound in SM cycles at the device's maximum clock (a slower clock only
// lengthens the bound in wall time).
unsigned long long wait_cycles(const DeviceInfo* d) {
    return (unsigned long long)((double)g_wait_ns * (double)d->clock_khz * 1e-6);
}

tbik_status run_gemm(const GemmPlan& p, const uint16_t* A, const uint16_t* B, void* C, uint8_t* ws,
                     cudaStream_t s, const DeviceInfo* info, const uint16_t* R = nullptr) {
    const int sms = info->sms;
    if (p.M == 0) return TBIK_OK;
    void* Cg = (p.swiglu && !p.fused) ? (void*)(ws + p.off_gu) : C;  // where the GEMM writes
    if (p.tc) {
        CUtensorMap ta, tb;
        const int a_box = a_box_rows(p.M);
        if (!make_map(&ta, A, (uint64_t)p.K, (uint64_t)p.M, 64, (uint32_t)a_box)) return TBIK_ERR_CUDA;
        const bool wide = p.bn == TC_BN_WIDE;  // 192-column pair tiles
        bool okb = p.b_nk  ? make_map(&tb, B, (uint64_t)p.K, (uint64_t)p.N, 64, (uint32_t)p.bn / 2)
                   : wide ? make_map(&tb, B, (uint64_t)p.N, (uint64_t)p.K, 32, TcCfg<TC_BN_WIDE>::BK, true)
                          : make_map(&tb, B, (uint64_t)p.N, (uint64_t)p.K, (uint32_t)p.bn / 2, 64);
        if (!okb) return TBIK_ERR_CUDA;
        TcParams prm;
        memset(&prm, 0, sizeof(prm));
        if (wide)
            set_ring<TC_BN_WIDE>(prm, a_box);
        else
            set_ring<TC_BN>(prm, a_box);
        prm.M = p.M, prm.N = p.N, prm.K = p.K;
        prm.leaf = p.leaf_eff;
        prm.F = p.F;
        prm.tiles_m = p.tiles_m, prm.tiles_n = p.tiles_n, prm.group_m = 8;
        prm.total_units = p.units;
        prm.direct = p.direct;
        prm.out_bf16 = p.out_bf16;
        prm.swiglu = p.fused ? 1 : 0;
        prm.out = Cg;
        prm.residual = p.direct ? R : nullptr;
        prm.partials = p.direct ? nullptr : reinterpret_cast<float*>(ws + p.off_partials);
        prm.scratch = p.gs ? reinterpret_cast<float*>(ws + p.off_scratch) : nullptr;
        prm.gs = p.gs;
        prm.b_mn = p.b_nk ? 0 : 1;
        prm.debug = g_debug_flags;
        prm.wait_cycles = wait_cycles(info);
        prm.tab_n[0] = prm.tab_n[1] = p.nodes[0].second;
        for (int f = 0; f < p.F; ++f) {
            prm.lo[f] = (short)p.nodes[f].first;
            prm.nl[f] = (short)p.nodes[f].second;
            if (prm.nl[f] != prm.tab_n[0]) prm.tab_n[1] = prm.nl[f];
        }
        using W = TcCfg<TC_BN_WIDE>;
        using Nw = TcCfg<TC_BN>;
        if (wide && prm.residual)
            gemm_tc_kernel<EPI_TREE_RES, TC_BN_WIDE><<<p.grid, W::THREADS, W::SMEM_BYTES, s>>>(ta, tb, prm);
        else if (wide)
            gemm_tc_kernel<EPI_TREE, TC_BN_WIDE><<<p.grid, W::THREADS, W::SMEM_BYTES, s>>>(ta, tb, prm);
        else if (prm.residual)
            gemm_tc_kernel<EPI_TREE_RES, TC_BN><<<p.grid, Nw::THREADS, Nw::SMEM_BYTES, s>>>(ta, tb, prm);
        else
            gemm_tc_kernel<EPI_TREE, TC_BN><<<p.grid, Nw::THREADS, Nw::SMEM_BYTES, s>>>(ta, tb, prm);
    } else {
        ExParams prm;
        memset(&prm, 0, sizeof(prm));
        prm.A = A, prm.B = B;
        prm.M = p.M, prm.N = p.N, prm.K = p.K;
        prm.leaf = p.leaf_eff;
        prm.F = p.F;
        prm.tiles_m = p.tiles_m, prm.tiles_n = p.tiles_n;
        prm.total_units = p.units;
        prm.direct = p.direct;
        prm.out_bf16 = p.out_bf16;
        prm.out = Cg;
        prm.residual = p.direct ? R : nullptr;
        prm.partials = p.direct ? nullptr : reinterpret_cast<float*>(ws + p.off_partials);
        for (int f = 0; f < p.F; ++f) {
            prm.lo[f] = (short)p.nodes[f].first;
            prm.nl[f] = (short)p.nodes[f].second;
        }
        int grid = p.units < sms ? p.units : sms;  // one resident CTA per SM
        // 16-byte loads when every chunk start and row stride is 8 elements aligned
        const bool vec = (p.K % 8 == 0) && (p.leaf_eff % 8 == 0) && (p.b_nk || p.N % 8 == 0);
        if (p.b_nk) {
            if (vec)
                gemm_exact_kernel<1, 1><<<grid, EX_THREADS, 0, s>>>(prm);
            else
                gemm_exact_kernel<1, 0><<<grid, EX_THREADS, 0, s>>>(prm);
        } else {
            if (vec)
                gemm_exact_kernel<0, 1><<<grid, EX_THREADS, 0, s>>>(prm);
            else
                gemm_exact_kernel<0, 0><<<grid, EX_THREADS, 0, s>>>(prm);
        }
    }
    tbik_status st = launch_status();
    if (st != TBIK_OK) return st;
    st = finish_gemm(p, ws, Cg, s, sms, R);
    if (st != TBIK_OK || !p.swiglu || p.fused) return st;
    const int F = p.N / 2;
    const long long work = (long long)p.M * (F / 8);
    long long blocks = (work + 255) / 256;
    if (blocks > (long long)sms * 8) blocks = (long long)sms * 8;
    swiglu_interleaved_kernel<<<(int)blocks, 256, 0, s>>>(reinterpret_cast<const float*>(Cg),
                                                         reinterpret_cast<uint16_t*>(C), p.M, F);
    return launch_status();
}

// ----------------------------------------------------------- logprob plan

struct LogprobPlan {
    int M = 0, V = 0, H = 0, T = 1, leaf = 256;
    bool tc = false, noninv = false;
    bool part = false;  // a vocabulary shard's summary (tbik_logprob_partial): T = 1, Lv given
    int Vpad = 0, Lv = 0, nvl = 0, nvt = 0, Lk = 0, tiles_m = 0, units = 0, grid = 0, gs = 0;
    size_t off_stats = 0, off_zt = 0, off_shard = 0, off_scratch = 0, off_z = 0, off_zgemm = 0, off_zflag = 0,
           off_pace = 0, total = 0;
    int pace_words = 0;  // tensor-core GEMM's pacing counters (0: no pacing)
    GemmPlan zplan;  // exact mode: the logits GEMM
};

tbik_status zgemm_plan(const LogprobPlan& p, int sms, GemmPlan& z) {
    const int M = p.M > 0 ? p.M : 1;
    if (p.noninv) return plan_gemm(M, p.V, p.H, p.T, p.H / p.T, TBIK_EXACT | TBIK_B_NK | TBIK_NONINV, sms, z);
    return plan_gemm(M, p.V, p.H, 1, p.leaf, TBIK_EXACT | TBIK_B_NK, sms, z);
}

// part_lv > 0: the summary of one vocabulary shard of V columns reduced over
// part_lv leaves (T = 1; leaves past the shard's columns are identities).
tbik_status plan_logprob(int M, int V, int H, int T, int leaf, unsigned mode, int sms, LogprobPlan& p,
                         int part_lv = 0) {
    if (mode & ~(TBIK_EXACT | TBIK_TC | TBIK_NONINV)) return TBIK_ERR_ARG;
    const bool exact = mode & TBIK_EXACT, tc = mode & TBIK_TC;
    if (exact == tc) return TBIK_ERR_ARG;
    if (M < 0 || H <= 0 || leaf <= 0 || (part_lv > 0 ? V < 0 : V <= 0)) return TBIK_ERR_ARG;
    if (!valid_T(T) || H % leaf || H % 8 || leaf % 16) return TBIK_ERR_SHAPE;
    p.M = M, p.V = V, p.H = H, p.T = T, p.leaf = leaf;
    p.tc = tc;
    p.noninv = mode & TBIK_NONINV;
    p.part = part_lv > 0;
    if (p.part) {
        if (T != 1) return TBIK_ERR_SHAPE;
        if ((long long)part_lv * VLEAF < (long long)V || part_lv > (1 << 24)) return TBIK_ERR_SHAPE;
        p.Lv = part_lv;
        p.Vpad = part_lv * VLEAF;
    } else {
        const int step = VLEAF * TBIK_T_MAX;
        p.Vpad = (int)(((long long)V + step - 1) / step * step);
        p.Lv = p.Vpad / VLEAF;
    }
    p.nvl = (V + VLEAF - 1) / VLEAF;        // vocab leaves holding columns
    p.nvt = (V + TC_BN_WIDE - 1) / TC_BN_WIDE;  // 192-column GEMM tiles (three vocab leaves each)
    // The baseline's logits: T chains over H/T each, summed left to right.
    if (p.noninv && (H % T || (tc && (H / T) % 16))) return TBIK_ERR_SHAPE;
    p.Lk = p.noninv ? T : H / leaf;
    if (p.Lk > 32767) return TBIK_ERR_SHAPE;
    p.tiles_m = (M + TC_PAIR_M - 1) / TC_PAIR_M;
    const long long units = (long long)p.tiles_m * p.nvt;
    if (units > 0x7fffffffLL) return TBIK_ERR_SHAPE;
    p.units = (int)units;
    {
        const int pairs = p.units < sms / 2 ? p.units : sms / 2;
        p.grid = 2 * (pairs > 0 ? pairs : 1);
    }
    // pending results of >= 5 leaves: the tree's depth, or one for the chain
    p.gs = tc ? (p.noninv ? (p.Lk >= 6 ? 1 : 0) : max_big_pending(p.Lk)) : 0;
    size_t off = 0;
    p.off_stats = off;
    off = align256(off + (size_t)p.nvl * M * 2 * sizeof(float));
    p.off_zt = off;
    off = align256(off + (size_t)M * sizeof(float));
    p.off_shard = off;
    off = align256(off + (size_t)T * M * 2 * sizeof(float));
    if (tc && p.gs > 0) {
        p.off_scratch = off;
        off = align256(off + (size_t)p.grid * p.gs * tc_slot_bytes(TC_BN_WIDE));
    }
    if (tc) {  // pacing counters: the flag, then one per TC_PACE_UNITS units of every pair
        const int pairs = p.grid / 2;
        p.pace_words = 1 + (p.units / (pairs > 0 ? pairs : 1)) / TC_PACE_UNITS + 1;
        p.off_pace = off;
        off = align256(off + (size_t)p.pace_words * sizeof(unsigned int));
    }
    if (p.part) {  // which rows' targets fall in this shard
        p.off_zflag = off;
        off = align256(off + (size_t)M * sizeof(int));
    }
    if (exact && V > 0) {
        // logits z fp32 [M][V] from the exact GEMM (the K tree, or the baseline's T chains summed in order)
        tbik_status st = zgemm_plan(p, sms, p.zplan);
        if (st != TBIK_OK) return st;
        p.off_z = off;
        off = align256(off + (size_t)M * V * sizeof(float));
        p.off_zgemm = off;
        off = align256(off + p.zplan.total);
    }
    p.total = off;
    return TBIK_OK;
}

// The logprob kernels for a plan: the fused GEMM + vocab statistics (or the
// exact logits GEMM + statistics kernel), then the row tree.  With `part`
// (a vocabulary shard, p.part) the row kernel writes the shard's per-row
// summary instead of the logprob; v0 is the shard's first vocabulary index.
tbik_status run_logprob(const LogprobPlan& p, const uint16_t* hidden, const uint16_t* W, const int32_t* targets,
                        float* out, float4* part, int v0, uint8_t* w8, cudaStream_t s, const DeviceInfo* info) {
    const int M = p.M, V = p.V, H = p.H, T = p.T, leaf = p.leaf;
    tbik_status st;
    float* stats = reinterpret_cast<float*>(w8 + p.off_stats);
    float* zt = reinterpret_cast<float*>(w8 + p.off_zt);
    float* shard = reinterpret_cast<float*>(w8 + p.off_shard);
    int* zflag = p.part ? reinterpret_cast<int*>(w8 + p.off_zflag) : nullptr;
    if (zflag && cudaMemsetAsync(zflag, 0, (size_t)M * sizeof(int), s) != cudaSuccess) return TBIK_ERR_CUDA;
    if (V > 0 && p.tc) {
        CUtensorMap ta, tb;
        const int a_box = a_box_rows(M);
        if (!make_map(&ta, hidden, (uint64_t)H, (uint64_t)M, 64, (uint32_t)a_box)) return TBIK_ERR_CUDA;
        if (!make_map(&tb, W, (uint64_t)H, (uint64_t)V, 64, TC_BN_WIDE / 2)) return TBIK_ERR_CUDA;
        TcParams prm;
        memset(&prm, 0, sizeof(prm));
        set_ring<TC_BN_WIDE>(prm, a_box);
        prm.M = M, prm.N = V, prm.K = H;
        prm.leaf = p.noninv ? H / T : leaf;
        prm.seq = p.noninv ? 1 : 0;
        prm.F = 1;
        prm.tiles_m = p.tiles_m, prm.tiles_n = p.nvt;
        prm.group_m = p.tiles_m;  // all row tiles of a vocab tile run together: W_lm is read once
        prm.pace = reinterpret_cast<unsigned int*>(w8 + p.off_pace);
        if (cudaMemsetAsync(prm.pace, 0, (size_t)p.pace_words * sizeof(unsigned int), s) != cudaSuccess)
            return TBIK_ERR_CUDA;
        prm.total_units = p.units;
        prm.direct = 1;
        prm.scratch = p.gs ? reinterpret_cast<float*>(w8 + p.off_scratch) : nullptr;
        prm.gs = p.gs;
        prm.b_mn = 0;
        prm.targets = targets;
        prm.stats = stats;
        prm.zt = zt;
        prm.zflag = zflag;
        prm.v0 = v0;
        prm.V = V;
        prm.debug = g_debug_flags & ~TBIK_DEBUG_WITHHOLD_ACC_ARRIVE;
        prm.wait_cycles = wait_cycles(info);
        prm.lo[0] = 0;
        prm.nl[0] = (short)p.Lk;
        prm.tab_n[0] = prm.tab_n[1] = prm.nl[0];
        gemm_tc_kernel<EPI_LOGPROB, TC_BN_WIDE>
            <<<p.grid, TcCfg<TC_BN_WIDE>::THREADS, TcCfg<TC_BN_WIDE>::SMEM_BYTES, s>>>(ta, tb, prm);
        if ((st = launch_status()) != TBIK_OK) return st;
    } else if (V > 0) {
        float* z = reinterpret_cast<float*>(w8 + p.off_z);
        GemmPlan zp;
        st = zgemm_plan(p, info->sms, zp);
        if (st != TBIK_OK) return st;
        if (zp.total > p.zplan.total) return TBIK_ERR_WORKSPACE;
        st = run_gemm(zp, hidden, W, z, w8 + p.off_zgemm, s, info);
        if (st != TBIK_OK) return st;
        const size_t work = (size_t)M * p.nvl;
        int blocks = (int)((work + 255) / 256);
        if (blocks > info->sms * 16) blocks = info->sms * 16;
        vocab_stats_kernel<<<blocks, 256, 0, s>>>(z, targets, stats, zt, zflag, M, V, p.nvl, v0);
        if ((st = launch_status()) != TBIK_OK) return st;
    }
    logprob_row_kernel<<<(M + ROW_BLOCK - 1) / ROW_BLOCK, ROW_BLOCK * 32, 0, s>>>(stats, zt, targets, out, shard, M,
                                                                                V, p.nvl, p.Lv, T, zflag, part);
    return launch_status();
}

}  // namespace

// ====================================================================== ABI

// Four leaves (32 elements) per thread when the width allows it: more bytes
// in flight per thread; the tree is the same.
template <bool RES>
void launch_rmsnorm(int nt, const DeviceInfo* info, cudaStream_t s, const uint16_t* x, const uint16_t* res,
                    const uint16_t* gamma, uint16_t* y, uint16_t* res_out, int tokens, int H, float eps, int T) {
    switch (nt) {
        case 32: launch_token_loop(rmsnorm_residual_kernel<32, 1, RES>, 32, tokens, info, s, x, res, gamma, y, res_out, tokens, H, eps, T); break;
        case 64: launch_token_loop(rmsnorm_residual_kernel<64, 1, RES>, 64, tokens, info, s, x, res, gamma, y, res_out, tokens, H, eps, T); break;
        case 128: launch_token_loop(rmsnorm_residual_kernel<32, 4, RES>, 32, tokens, info, s, x, res, gamma, y, res_out, tokens, H, eps, T); break;
        case 256: launch_token_loop(rmsnorm_residual_kernel<64, 4, RES>, 64, tokens, info, s, x, res, gamma, y, res_out, tokens, H, eps, T); break;
        case 512: launch_token_loop(rmsnorm_residual_kernel<128, 4, RES>, 128, tokens, info, s, x, res, gamma, y, res_out, tokens, H, eps, T); break;
        case 1024: launch_token_loop(rmsnorm_residual_kernel<256, 4, RES>, 256, tokens, info, s, x, res, gamma, y, res_out, tokens, H, eps, T); break;
    }
}

extern "C" {

const char* tbik_version(void) { return "tbik-b200 0.1 (sm_100a)"; }

const char* tbik_status_string(tbik_status s) {
    switch (s) {
        case TBIK_OK: return "ok";
        case TBIK_ERR_ARG: return "invalid argument";
        case TBIK_ERR_SHAPE: return "unsupported shape";
        case TBIK_ERR_ALIGN: return "pointer not 16-byte aligned";
        case TBIK_ERR_WORKSPACE: return "workspace missing or too small";
        case TBIK_ERR_CUDA: return "CUDA error";
        case TBIK_ERR_TIMEOUT: return "device wait timed out";
        case TBIK_ERR_TARGET: return "target index out of range";
        case TBIK_ERR_POSITION: return "RoPE position out of range";
        case TBIK_ERR_UNSUPPORTED: return "device is not sm_100";
    }
    return "unknown status";
}

size_t tbik_gemm_workspace(int M, int N, int K, int T, int leaf, unsigned mode) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return (size_t)-1;
    GemmPlan p;
    if (plan_gemm(M, N, K, T, leaf, mode, info->sms, p) != TBIK_OK) return (size_t)-1;
    return p.total;
}

tbik_status tbik_gemm(const uint16_t* A, const uint16_t* B, void* C, int M, int N, int K, int T, int leaf,
                      unsigned mode, void* ws, size_t ws_bytes, void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    GemmPlan p;
    st = plan_gemm(M, N, K, T, leaf, mode, info->sms, p);
    if (st != TBIK_OK) return st;
    if (M == 0) return TBIK_OK;
    if (!A || !B || !C) return TBIK_ERR_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return TBIK_ERR_ALIGN;
    if (p.total > 0 && (!ws || ws_bytes < p.total)) return TBIK_ERR_WORKSPACE;
    if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u)) return TBIK_ERR_ALIGN;
    return run_gemm(p, A, B, C, reinterpret_cast<uint8_t*>(ws), reinterpret_cast<cudaStream_t>(stream), info);
}

tbik_status tbik_gemm_residual(const uint16_t* A, const uint16_t* B, const uint16_t* R, uint16_t* C, int M, int N,
                               int K, int T, int leaf, unsigned mode, void* ws, size_t ws_bytes, void* stream) {
    if (mode & (TBIK_OUT_BF16 | TBIK_SWIGLU_OUT)) return TBIK_ERR_ARG;
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    GemmPlan p;
    st = plan_gemm(M, N, K, T, leaf, mode | TBIK_OUT_BF16, info->sms, p);
    if (st != TBIK_OK) return st;
    if (M == 0) return TBIK_OK;
    if (!A || !B || !C || !R) return TBIK_ERR_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(C) || !aligned16(R)) return TBIK_ERR_ALIGN;
    if (p.total > 0 && (!ws || ws_bytes < p.total)) return TBIK_ERR_WORKSPACE;
    if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u)) return TBIK_ERR_ALIGN;
    return run_gemm(p, A, B, C, reinterpret_cast<uint8_t*>(ws), reinterpret_cast<cudaStream_t>(stream), info, R);
}

tbik_status tbik_rmsnorm_residual(const uint16_t* x, const uint16_t* res, const uint16_t* gamma, uint16_t* y,
                                  uint16_t* res_out, int tokens, int H, float eps, int T, void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    if (tokens < 0 || H <= 0) return TBIK_ERR_ARG;
    if (!valid_T(T) || H % 8) return TBIK_ERR_SHAPE;
    const int nt = H / 8;
    if (nt < 32 || nt > 1024 || (nt & (nt - 1)) || nt % T) return TBIK_ERR_SHAPE;
    if (tokens == 0) return TBIK_OK;
    if (!x || !gamma || !y) return TBIK_ERR_ARG;
    if (!aligned16(x) || (res && !aligned16(res)) || !aligned16(gamma) || !aligned16(y) ||
        (res_out && !aligned16(res_out)))
        return TBIK_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (res)
        launch_rmsnorm<true>(nt, info, s, x, res, gamma, y, res_out, tokens, H, eps, T);
    else
        launch_rmsnorm<false>(nt, info, s, x, res, gamma, y, res_out, tokens, H, eps, T);
    return launch_status();
}

tbik_status tbik_rope_table(float* table, int max_pos, int head_dim, double base, void* stream) {
    if (!table || max_pos <= 0 || head_dim < 2 || head_dim > 512 || (head_dim & 1) || !(base > 0.0))
        return TBIK_ERR_ARG;
    const int half = head_dim / 2;
    std::vector<float> h((size_t)max_pos * half * 2);
    for (int p = 0; p < max_pos; ++p)
        for (int i = 0; i < half; ++i) {
            const double theta = std::pow(base, -(double)(2 * i) / (double)head_dim);
            const double ang = (double)p * theta;
            h[((size_t)p * half + i) * 2 + 0] = (float)std::cos(ang);
            h[((size_t)p * half + i) * 2 + 1] = (float)std::sin(ang);
        }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(table, h.data(), h.size() * sizeof(float), cudaMemcpyHostToDevice, s) != cudaSuccess)
        return TBIK_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return TBIK_ERR_CUDA;
    return TBIK_OK;
}

tbik_status tbik_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, int batch,
                           int seq, int heads, int head_dim, int chunk, void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    if (batch < 0 || seq < 0 || heads <= 0) return TBIK_ERR_ARG;
    if ((head_dim != 64 && head_dim != 128) || chunk != ATT_CHUNK || seq > 256 * ATT_CHUNK) return TBIK_ERR_SHAPE;
    if (batch == 0 || seq == 0) return TBIK_OK;
    if (!q || !k || !v || !out) return TBIK_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return TBIK_ERR_ALIGN;
    const long long blocks = (long long)batch * heads * ((seq + ATT_QPB - 1) / ATT_QPB);
    if (blocks > 0x7fffffffLL) return TBIK_ERR_SHAPE;
    const float scale = (float)(1.0 / std::sqrt((double)head_dim));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (head_dim == 128)
        attention_kernel<4><<<(int)blocks, ATT_WARPS * 32, 0, s>>>(q, k, v, out, batch, seq, heads, scale);
    else
        attention_kernel<2><<<(int)blocks, ATT_WARPS * 32, 0, s>>>(q, k, v, out, batch, seq, heads, scale);
    return launch_status();
}

// Tensor-core mode of the attention: shapes, grid and scratch.
struct AttTcPlan {
    int tiles = 0, grid = 0, gs = 0;
    size_t bytes = 0;
};

tbik_status plan_attention_tc(int batch, int seq, int heads, int head_dim, int chunk, int sms, AttTcPlan& p) {
    if (batch < 0 || seq < 0 || heads <= 0) return TBIK_ERR_ARG;
    if (head_dim != ATC_HD || chunk != ATC_LEAF || seq % ATC_BM || seq > 128 * ATC_LEAF) return TBIK_ERR_SHAPE;
    const long long tiles = (long long)batch * heads * (seq / ATC_BM);
    if (tiles > 0x7fffffffLL) return TBIK_ERR_SHAPE;
    p.tiles = (int)tiles;
    p.grid = p.tiles < sms ? p.tiles : sms;
    // the deepest L2 stack over the leaf trees of every row length
    p.gs = 0;
    for (int n = 1; n <= seq / ATC_LEAF; ++n) {
        const int g = max_big_pending(n);
        if (g > p.gs) p.gs = g;
    }
    if (p.gs > ATC_MAX_GS) return TBIK_ERR_SHAPE;  // cannot happen for seq <= 16384
    p.bytes = (size_t)p.grid * p.gs * ATC_VAL_FLOATS * sizeof(float);
    return TBIK_OK;
}

size_t tbik_attention_tc_workspace(int batch, int seq, int heads, int head_dim, int chunk) {
    int dev;
    DeviceInfo* info;
    if (device_info(dev, info) != TBIK_OK) return (size_t)-1;
    AttTcPlan p;
    if (plan_attention_tc(batch, seq, heads, head_dim, chunk, info->sms, p) != TBIK_OK) return (size_t)-1;
    return p.bytes;
}

tbik_status tbik_attention_tc(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, int batch,
                              int seq, int heads, int head_dim, int chunk, void* workspace, size_t ws_bytes,
                              void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    AttTcPlan p;
    if ((st = plan_attention_tc(batch, seq, heads, head_dim, chunk, info->sms, p)) != TBIK_OK) return st;
    if (p.tiles == 0) return TBIK_OK;
    if (!q || !k || !v || !out) return TBIK_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return TBIK_ERR_ALIGN;
    if (p.bytes > 0 && (!workspace || ws_bytes < p.bytes)) return TBIK_ERR_WORKSPACE;
    if (p.bytes > 0 && !aligned16(workspace)) return TBIK_ERR_ALIGN;
    CUtensorMap tq, tk, tv;
    if (!make_map_bshd(&tq, q, batch, seq, heads, head_dim, ATC_BM) ||
        !make_map_bshd(&tk, k, batch, seq, heads, head_dim, ATC_CH) ||
        !make_map_bshd(&tv, v, batch, seq, heads, head_dim, ATC_CH))
        return TBIK_ERR_CUDA;
    AttTcParams prm;
    memset(&prm, 0, sizeof(prm));
    prm.batch = batch, prm.seq = seq, prm.heads = heads;
    prm.ntq = seq / ATC_BM;
    prm.tiles = p.tiles;
    prm.scale = (float)(1.0 / std::sqrt((double)head_dim));
    prm.out = out;
    prm.stack = reinterpret_cast<float*>(workspace);
    prm.gs = p.gs;
    prm.wait_cycles = wait_cycles(info);
    prm.debug = g_debug_flags;
    attention_tc_kernel<<<p.grid, ATC_THREADS, ATC_SMEM_BYTES, reinterpret_cast<cudaStream_t>(stream)>>>(tq, tk, tv,
                                                                                                           prm);
    return launch_status();
}

tbik_status tbik_transpose(const uint16_t* in, uint16_t* out, int rows, int cols, void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    if (rows < 0 || cols < 0) return TBIK_ERR_ARG;
    if (rows == 0 || cols == 0) return TBIK_OK;
    if (!in || !out) return TBIK_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out)) & 1u) return TBIK_ERR_ALIGN;
    if (rows % 8 == 0 && cols % 8 == 0 && aligned16(in) && aligned16(out) && (rows + 63) / 64 <= 65535) {
        transpose_vec_kernel<<<dim3((unsigned)((cols + 63) / 64), (unsigned)((rows + 63) / 64)), 256, 0,
                               reinterpret_cast<cudaStream_t>(stream)>>>(in, out, rows, cols);
        return launch_status();
    }
    const long long gx = (cols + 31) / 32, gy = (rows + 31) / 32;
    if (gy > 65535) return TBIK_ERR_SHAPE;
    transpose_kernel<<<dim3((unsigned)gx, (unsigned)gy), dim3(32, 8), 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        in, out, rows, cols);
    return launch_status();
}

tbik_status tbik_embedding(const int32_t* ids, const uint16_t* table, uint16_t* out, int tokens, int V, int d,
                           void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    if (tokens < 0 || V <= 0 || d <= 0) return TBIK_ERR_ARG;
    if (d % 8) return TBIK_ERR_SHAPE;
    if (tokens == 0) return TBIK_OK;
    if (!ids || !table || !out) return TBIK_ERR_ARG;
    if (!aligned16(table) || !aligned16(out)) return TBIK_ERR_ALIGN;
    const long long work = (long long)tokens * (d / 8);
    long long blocks = (work + 255) / 256;
    if (blocks > (long long)info->sms * 16) blocks = (long long)info->sms * 16;
    embedding_kernel<<<(int)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(ids, table, out, tokens, V, d);
    return launch_status();
}

tbik_status tbik_rope_swiglu_fp32(const tbik_rope_swiglu_args* a, void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    if (!a) return TBIK_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (a->q || a->k) {
        if (a->tokens < 0 || a->heads <= 0 || a->max_pos <= 0) return TBIK_ERR_ARG;
        if (a->head_dim <= 0 || a->head_dim % 16 || a->head_dim > 512) return TBIK_ERR_SHAPE;
        if (!a->pos || !a->table || (a->q && !a->q_out) || (a->k && !a->k_out)) return TBIK_ERR_ARG;
        if ((a->q && (!aligned16(a->q) || !aligned16(a->q_out))) || (a->k && (!aligned16(a->k) || !aligned16(a->k_out))) ||
            !aligned16(a->table))
            return TBIK_ERR_ALIGN;
    }
    if (a->g) {
        if (!a->u || !a->out || a->n < 0) return TBIK_ERR_ARG;
        if (a->n % 8) return TBIK_ERR_SHAPE;
        if (!aligned16(a->g) || !aligned16(a->u) || !aligned16(a->out)) return TBIK_ERR_ALIGN;
    }
    if ((a->q || a->k) && a->tokens > 0) {
        const size_t work = (size_t)a->tokens * a->heads * (a->head_dim / 16);
        int blocks = (int)((work + 255) / 256);
        if (blocks > info->sms * 16) blocks = info->sms * 16;
        const size_t stride = (size_t)blocks * 256;
        if (work + stride < (1ull << 32))  // every index the loop forms fits 32 bits
            rope_kernel<uint32_t><<<blocks, 256, 0, s>>>(a->q, a->k, a->q_out, a->k_out, a->pos, a->table,
                                                                  a->tokens, a->heads, a->head_dim, a->max_pos);
        else
            rope_kernel<size_t><<<blocks, 256, 0, s>>>(a->q, a->k, a->q_out, a->k_out, a->pos, a->table,
                                                                a->tokens, a->heads, a->head_dim, a->max_pos);
        if ((st = launch_status()) != TBIK_OK) return st;
    }
    if (a->g && a->n > 0) {
        const long long nv = a->n / 8;
        long long blocks = (nv + 255) / 256;
        if (blocks > (long long)info->sms * 16) blocks = (long long)info->sms * 16;
        // 32-bit indices when every index the loop forms, doubled for the fp32
        // inputs' float4 pairs, stays below 2^32
        const bool narrow = (unsigned long long)nv + (unsigned long long)blocks * 256 < (1ull << 31);
        if (a->in_f32) {
            if (narrow)
                swiglu_kernel<1, uint32_t><<<(int)blocks, 256, 0, s>>>(a->g, a->u, a->out, a->n);
            else
                swiglu_kernel<1, long long><<<(int)blocks, 256, 0, s>>>(a->g, a->u, a->out, a->n);
        } else {
            // bf16 gates: the table, built on this device once (on the first
            // caller's stream; later calls on any stream wait for its event)
            {
                std::lock_guard<std::mutex> lk(g_mu);
                if (!info->lut_built) {
                    silu_lut_kernel<<<65536 / 256, 256, 0, s>>>();
                    cudaEvent_t ev;
                    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return TBIK_ERR_CUDA;
                    if (cudaEventRecord(ev, s) != cudaSuccess) return TBIK_ERR_CUDA;
                    info->lut_built = ev;
                }
            }
            if (cudaStreamWaitEvent(s, info->lut_built, 0) != cudaSuccess) return TBIK_ERR_CUDA;
            const uint16_t* g16 = reinterpret_cast<const uint16_t*>(a->g);
            const uint16_t* u16 = reinterpret_cast<const uint16_t*>(a->u);
            if (narrow)
                swiglu_lut_kernel<uint32_t><<<(int)blocks, 256, 0, s>>>(g16, u16, a->out, a->n);
            else
                swiglu_lut_kernel<long long><<<(int)blocks, 256, 0, s>>>(g16, u16, a->out, a->n);
        }
        if ((st = launch_status()) != TBIK_OK) return st;
    }
    return TBIK_OK;
}

size_t tbik_logprob_workspace(int M, int V, int H, int T, int leaf, unsigned mode) {
    int dev;
    DeviceInfo* info;
    if (device_info(dev, info) != TBIK_OK) return (size_t)-1;
    LogprobPlan p;
    if (plan_logprob(M, V, H, T, leaf, mode, info->sms, p) != TBIK_OK) return (size_t)-1;
    return p.total;
}

}  // extern "C"

// Library-internal (hidden visibility, not part of the ABI): the status that
// tbik_logprob's planning gives these arguments on the current device and, when
// it is TBIK_OK, the workspace bytes.  Lets another entry point report the same
// status codes as tbik_logprob (ARG, SHAPE, CUDA, UNSUPPORTED) instead of the
// bare (size_t)-1 of tbik_logprob_workspace.
tbik_status tbik_logprob_plan_status(int M, int V, int H, int T, int leaf, unsigned mode, size_t* bytes) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    LogprobPlan p;
    st = plan_logprob(M, V, H, T, leaf, mode, info->sms, p);
    if (st != TBIK_OK) return st;
    *bytes = p.total;
    return TBIK_OK;
}

extern "C" {

tbik_status tbik_logprob(const uint16_t* hidden, const uint16_t* W, const int32_t* targets, float* out, int M, int V,
                         int H, int T, int leaf, unsigned mode, void* ws, size_t ws_bytes, void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    LogprobPlan p;
    st = plan_logprob(M, V, H, T, leaf, mode, info->sms, p);
    if (st != TBIK_OK) return st;
    if (M == 0) return TBIK_OK;
    if (!hidden || !W || !targets || !out) return TBIK_ERR_ARG;
    if (!aligned16(hidden) || !aligned16(W) || !aligned16(targets) || !aligned16(out)) return TBIK_ERR_ALIGN;
    if (!ws || ws_bytes < p.total) return TBIK_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return TBIK_ERR_ALIGN;
    return run_logprob(p, hidden, W, targets, out, nullptr, 0, reinterpret_cast<uint8_t*>(ws),
                       reinterpret_cast<cudaStream_t>(stream), info);
}

size_t tbik_logprob_partial_workspace(int M, int Vs, int Lvs, int H, int leaf, unsigned mode) {
    int dev;
    DeviceInfo* info;
    if (device_info(dev, info) != TBIK_OK) return (size_t)-1;
    LogprobPlan p;
    if (Lvs <= 0 || (mode & TBIK_NONINV) || plan_logprob(M, Vs, H, 1, leaf, mode, info->sms, p, Lvs) != TBIK_OK)
        return (size_t)-1;
    return p.total;
}

tbik_status tbik_logprob_partial(const uint16_t* hidden, const uint16_t* W_shard, const int32_t* targets, float* part,
                                 int M, int Vs, int v0, int Lvs, int H, int leaf, unsigned mode, void* ws,
                                 size_t ws_bytes, void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    if (mode & TBIK_NONINV) return TBIK_ERR_ARG;
    if (Lvs <= 0 || v0 < 0) return TBIK_ERR_ARG;
    LogprobPlan p;
    st = plan_logprob(M, Vs, H, 1, leaf, mode, info->sms, p, Lvs);
    if (st != TBIK_OK) return st;
    if (M == 0) return TBIK_OK;
    if (!hidden || (Vs > 0 && !W_shard) || !targets || !part) return TBIK_ERR_ARG;
    if (!aligned16(hidden) || (Vs > 0 && !aligned16(W_shard)) || !aligned16(targets) || !aligned16(part))
        return TBIK_ERR_ALIGN;
    if (!ws || ws_bytes < p.total) return TBIK_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return TBIK_ERR_ALIGN;
    return run_logprob(p, hidden, W_shard, targets, nullptr, reinterpret_cast<float4*>(part), v0,
                       reinterpret_cast<uint8_t*>(ws), reinterpret_cast<cudaStream_t>(stream), info);
}

tbik_status tbik_logprob_combine(const float* parts, const int32_t* targets, float* out, int M, int V, int T,
                                 void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    if (M < 0 || V <= 0) return TBIK_ERR_ARG;
    if (!valid_T(T)) return TBIK_ERR_SHAPE;
    if (M == 0) return TBIK_OK;
    if (!parts || !targets || !out) return TBIK_ERR_ARG;
    if (!aligned16(parts) || !aligned16(targets) || !aligned16(out)) return TBIK_ERR_ALIGN;
    int blocks = (M + 255) / 256;
    if (blocks > info->sms * 8) blocks = info->sms * 8;
    logprob_combine_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const float4*>(parts), targets, out, M, V, T);
    return launch_status();
}

tbik_status tbik_tree_combine(const float* partials, void* out, long long MN, int T, unsigned mode, const uint16_t* R,
                              void* stream) {
    int dev;
    DeviceInfo* info;
    tbik_status st = device_info(dev, info);
    if (st != TBIK_OK) return st;
    if (mode & ~(TBIK_NONINV | TBIK_OUT_BF16)) return TBIK_ERR_ARG;
    if (MN < 0) return TBIK_ERR_ARG;
    if (!valid_T(T)) return TBIK_ERR_SHAPE;
    const bool bf16 = mode & TBIK_OUT_BF16;
    if (R && !bf16) return TBIK_ERR_ARG;
    if (MN == 0) return TBIK_OK;
    if (!partials || !out) return TBIK_ERR_ARG;
    if (!aligned16(partials) || !aligned16(out) || (R && !aligned16(R))) return TBIK_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (mode & TBIK_NONINV) {
        size_t blocks = ((size_t)MN + 255) / 256;
        if (blocks > (size_t)info->sms * 8) blocks = (size_t)info->sms * 8;
        seq_combine_kernel<<<(int)blocks, 256, 0, s>>>(partials, (size_t)MN, T, out, bf16 ? 1 : 0, R);
        return launch_status();
    }
    return tree_combine(partials, (size_t)MN, T, 1, out, bf16 ? 1 : 0, s, info->sms, R);
}

tbik_status tbik_get_error(void* stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return TBIK_ERR_CUDA;
    unsigned e = 0;
    if (cudaMemcpyFromSymbol(&e, tbik::g_err, sizeof(e)) != cudaSuccess) return TBIK_ERR_CUDA;
    if (e) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(tbik::g_err, &zero, sizeof(zero)) != cudaSuccess) return TBIK_ERR_CUDA;
    }
    return (tbik_status)e;
}

tbik_status tbik_debug_set(unsigned flags, unsigned long long wait_limit_ns) {
    if (flags & ~(TBIK_DEBUG_WITHHOLD_ACC_ARRIVE | TBIK_DEBUG_TILE128)) return TBIK_ERR_ARG;
    g_debug_flags = flags;
    g_wait_ns = wait_limit_ns ? wait_limit_ns : 2000000000ull;
    return TBIK_OK;
}

}  // extern "C"
