/*
 * CPU oracle for the tree-ordered invariant kernels.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, single-threaded
 * statement of what the library computes.  It shares no code with the CUDA
 * path (no headers, helpers, tables or constants are common to both), and
 * only the tests, smoke() and the benchmark's CPU-baseline leg may load it.
 * Build flags: -O2 -ffp-contract=off -fno-fast-math, x86-64 SSE arithmetic,
 * so every float operation below is one IEEE binary32 round-to-nearest-even
 * operation and fmaf() is the correctly rounded fused multiply-add.  The
 * default build is single-threaded.  The independent outputs of the GEMM and
 * the rows of the logprob carry OpenMP pragmas, which only a second build
 * with -fopenmp (used to time the oracle on all host cores) acts on: each
 * output is still the same serial computation, so both builds give the same
 * bits.
 *
 * Sources (web pages on the subject; cited by title and section):
 *  [TBIK] "Deterministic Inference across Tensor Parallel Sizes That Eliminates
 *         Training-Inference Mismatch" (paper summary page): sections
 *         核心思路, 技术框架 and the English abstract -- one hierarchical binary
 *         tree orders both the local reduction on each GPU and the reduction
 *         across GPUs, so the result is bitwise the same for every TP size.
 *  [RLA]  rounding-location alignment article (winzheng.jp), section
 *         "外科手術的な修正：3つのノード" -- RoPE, SwiGLU and residual RMSNorm keep
 *         FP32 intermediates and round to BF16 once, at the output.
 *  [ISO]  IsoExec executive brief (nxmr.cn), sections 壹/叁/伍 -- the target
 *         token's logprob is the quantity compared bit for bit.
 *  [TP]   distributed-training tutorial (yamichan.com), section 2.1.1 and
 *         figure 5 -- the row-parallel second MLP layer sums per-device partial
 *         contributions.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  R1 TREE(P,lo,n): n == 1 -> P[lo]; else h = ceil(n/2) and the value is
 *     TREE(P,lo,h) + TREE(P,lo+h,n-h).  The pages say "hierarchical binary
 *     tree" only; halving with the left half rounded up is the plainest shape
 *     in which every power-of-two shard count T dividing the leaf count owns
 *     whole subtrees.
 *  R2 Inside a K leaf the products are accumulated in ascending k with
 *     acc = fmaf(a, b, acc), starting from +0.0f.
 *  R3 T shards of the reduced dimension are contiguous leaf ranges; shard
 *     partials are combined with TREE over T.
 *  R4 exp and log are the Cody-Waite style specifications exp_spec/log_spec
 *     below (W. J. Cody and W. Waite, "Software Manual for the Elementary
 *     Functions", 1980: additive argument reduction by a split ln 2, then a
 *     short polynomial), written here from the mathematics.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ bf16 */

static float bf(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary32 -> bfloat16, round to nearest, ties to even; NaN stays a quiet NaN. */
static uint16_t bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u = u + 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

uint16_t oracle_bf16_rne(float f) { return bf16_rne(f); }

void oracle_bf16_rne_array(const float* x, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_rne(x[i]);
}

/* ------------------------------------------------------------------ tree */

/* R1: the halving tree, straight from its definition. */
static float tree_f32(const float* P, int lo, int n) {
    if (n == 1) return P[lo];
    int h = (n + 1) / 2;
    float left = tree_f32(P, lo, h);
    float right = tree_f32(P, lo + h, n - h);
    return left + right;
}

float oracle_tree_sum(const float* P, int n) { return tree_f32(P, 0, n); }

/* Sequential left-to-right sum (the non-invariant combine of shard partials). */
static float seq_f32(const float* P, int lo, int n) {
    float acc = P[lo];
    for (int i = 1; i < n; ++i) acc = acc + P[lo + i];
    return acc;
}

/* ------------------------------------------------------- exp/log (R4) */

static float f_from_bits(uint32_t u) {
    float f;
    memcpy(&f, &u, 4);
    return f;
}
static uint32_t bits_of(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

static const float kLog2e = 0x1.715476p+0f;   /* nearest float to 1/ln 2 */
static const float kLn2Hi = 0x1.62e4p-1f;     /* 45426/65536: ln 2 cut to 16 bits */
static const float kLn2Lo = 0x1.7f7d1cp-20f;  /* nearest float to ln 2 - kLn2Hi */

/* pow2(n) for n in [-126, 127], built from the exponent field (exact). */
static float pow2i(int n) { return f_from_bits((uint32_t)(n + 127) << 23); }

/*
 * exp_spec(x):  clamp x to [-104, 89] (outside, the float result is 0 or inf
 * anyway); k = rint(x * log2e); r = (x - k*ln2hi) - k*ln2lo with two fmas;
 * p = the degree-7 Taylor polynomial of e^r in Horner form (coefficients the
 * nearest floats to 1/n!); result = (p * 2^(k/2)) * 2^(k - k/2), with k/2
 * truncating, so that the one rounding step of the scaling happens last.
 */
static float exp_spec(float x) {
    if (x != x) return x + x;
    if (x > 89.0f) x = 89.0f;
    if (x < -104.0f) x = -104.0f;
    float kf = rintf(x * kLog2e);
    float r = fmaf(-kf, kLn2Hi, x);
    r = fmaf(-kf, kLn2Lo, r);
    float p = 0x1.a01a02p-13f;      /* 1/5040 */
    p = fmaf(p, r, 0x1.6c16c2p-10f); /* 1/720  */
    p = fmaf(p, r, 0x1.111112p-7f);  /* 1/120  */
    p = fmaf(p, r, 0x1.555556p-5f);  /* 1/24   */
    p = fmaf(p, r, 0x1.555556p-3f);  /* 1/6    */
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int k = (int)kf;
    int k1 = k / 2;
    int k2 = k - k1;
    return (p * pow2i(k1)) * pow2i(k2);
}

/*
 * log_spec(x) for x > 0:  x = 2^e * m with m in [sqrt(1/2), sqrt(2)];
 * t = (m-1)/(m+1) computed as f/(2+f), f = m-1 (exact);
 * log m = 2 atanh t = s + s*w*(1/3 + w/5 + w^2/7 + w^3/9 + w^4/11), s = 2t, w = t^2;
 * result = e*ln2lo + log m, then + e*ln2hi (two fmas).
 */
static float log_spec(float x) {
    if (x != x) return x + x;
    if (x < 0.0f) return NAN;
    if (x == 0.0f) return -INFINITY;
    if (x == INFINITY) return x;
    int e = 0;
    uint32_t u = bits_of(x);
    if (u < 0x00800000u) { /* subnormal: scale by 2^23 exactly */
        x = x * 0x1p23f;
        u = bits_of(x);
        e = -23;
    }
    e += (int)(u >> 23) - 127;
    float m = f_from_bits((u & 0x007fffffu) | 0x3f800000u);
    if (m > 0x1.6a09e6p+0f) { /* nearest float to sqrt 2 */
        m = m * 0.5f;
        e += 1;
    }
    float f = m - 1.0f;
    float t = f / (2.0f + f);
    float w = t * t;
    float q = 0x1.745d18p-4f;        /* 1/11 */
    q = fmaf(q, w, 0x1.c71c72p-4f);  /* 1/9  */
    q = fmaf(q, w, 0x1.24924ap-3f);  /* 1/7  */
    q = fmaf(q, w, 0x1.99999ap-3f);  /* 1/5  */
    q = fmaf(q, w, 0x1.555556p-2f);  /* 1/3  */
    float s = t + t;
    float lm = fmaf(s * w, q, s);
    float ef = (float)e;
    float r = fmaf(ef, kLn2Lo, lm);
    return fmaf(ef, kLn2Hi, r);
}

float oracle_exp(float x) { return exp_spec(x); }
float oracle_log(float x) { return log_spec(x); }

/* ------------------------------------------------------------------ GEMM */

/* A [K,N] operand copied to [N,K] so that each output reads one contiguous
   column; a pure data movement, the arithmetic order is untouched. */
static uint16_t* transpose_kn(const uint16_t* B, int K, int N) {
    uint16_t* t = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)K * (size_t)N);
    for (int k = 0; k < K; ++k)
        for (int n = 0; n < N; ++n) t[(size_t)n * K + k] = B[(size_t)k * N + n];
    return t;
}

/*
 * Tree-ordered GEMM (exact-order definition).  [TBIK] 技术框架: each shard
 * reduces locally, then the shard partials are reduced across GPUs, both by one
 * binary tree.  With L = K/leaf leaves and T shards:
 *   P_j      = sum over k in leaf j, ascending, acc = fmaf(A[i,k], B[k,n], acc)   (R2)
 *   Q_t      = TREE(P, t*L/T, L/T)                                          (R1, R3)
 *   C[i,n]   = TREE(Q, 0, T)
 * A is bf16 [M,K] row-major; B is bf16 [K,N] (b_nk = 0) or [N,K] (b_nk = 1).
 * shard_out (nullable) receives Q as fp32 [T][M][N].  Returns 0, or -1 on a
 * shape the definition does not cover.
 */
int oracle_gemm_tree(const uint16_t* A, const uint16_t* B, int b_nk, int M, int N, int K, int T,
                     int leaf, float* C, float* shard_out) {
    if (M < 0 || N < 0 || K <= 0 || leaf <= 0 || T <= 0 || K % leaf) return -1;
    int L = K / leaf;
    if (L % T) return -1;
    int Ls = L / T;
    const uint16_t* Bt = b_nk ? B : transpose_kn(B, K, N);
    /* Every output (i, n) is computed on its own, so a build with OpenMP may
       hand them to several threads, each with its own leaf and shard scratch;
       the computation of each output is the same serial one (the default build
       is single-threaded and ignores the pragmas). */
#pragma omp parallel
    {
        float* P = (float*)malloc(sizeof(float) * (size_t)L);
        float* Q = (float*)malloc(sizeof(float) * (size_t)T);
#pragma omp for schedule(static)
        for (long long o = 0; o < (long long)M * N; ++o) {
            const int i = (int)(o / N), n = (int)(o % N);
            const uint16_t* bcol = Bt + (size_t)n * K;
            for (int j = 0; j < L; ++j) {
                float acc = 0.0f;
                for (int k = j * leaf; k < (j + 1) * leaf; ++k)
                    acc = fmaf(bf(A[(size_t)i * K + k]), bf(bcol[k]), acc);
                P[j] = acc;
            }
            for (int t = 0; t < T; ++t) {
                Q[t] = tree_f32(P, t * Ls, Ls);
                if (shard_out) shard_out[((size_t)t * M + i) * N + n] = Q[t];
            }
            C[(size_t)i * N + n] = tree_f32(Q, 0, T);
        }
        free(P);
        free(Q);
    }
    if (!b_nk) free((void*)Bt);
    return 0;
}

/*
 * Deliberately non-invariant baseline ([TP] 2.1.1 / figure 5; [ISO] 贰): each
 * shard accumulates its whole K range in one fma chain, then the partials are
 * summed left to right: C = ((Q_0 + Q_1) + Q_2) + ...
 */
int oracle_gemm_noninv(const uint16_t* A, const uint16_t* B, int b_nk, int M, int N, int K, int T,
                       float* C, float* shard_out) {
    if (M < 0 || N < 0 || K <= 0 || T <= 0 || K % T) return -1;
    int Ks = K / T;
    float* Q = (float*)malloc(sizeof(float) * (size_t)T);
    const uint16_t* Bt = b_nk ? B : transpose_kn(B, K, N);
    for (int i = 0; i < M; ++i) {
        for (int n = 0; n < N; ++n) {
            const uint16_t* bcol = Bt + (size_t)n * K;
            for (int t = 0; t < T; ++t) {
                float acc = 0.0f;
                for (int k = t * Ks; k < (t + 1) * Ks; ++k)
                    acc = fmaf(bf(A[(size_t)i * K + k]), bf(bcol[k]), acc);
                Q[t] = acc;
                if (shard_out) shard_out[((size_t)t * M + i) * N + n] = acc;
            }
            C[(size_t)i * N + n] = seq_f32(Q, 0, T);
        }
    }
    if (!b_nk) free((void*)Bt);
    free(Q);
    return 0;
}

/* Double-precision product for tolerance checks (sequential binary64 sum). */
void oracle_gemm_f64(const uint16_t* A, const uint16_t* B, int b_nk, int M, int N, int K, double* C) {
    const uint16_t* Bt = b_nk ? B : transpose_kn(B, K, N);
    for (int i = 0; i < M; ++i)
        for (int n = 0; n < N; ++n) {
            const uint16_t* bcol = Bt + (size_t)n * K;
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += (double)bf(A[(size_t)i * K + k]) * (double)bf(bcol[k]);
            C[(size_t)i * N + n] = acc;
        }
    if (!b_nk) free((void*)Bt);
}

/* ------------------------------------------------------- residual RMSNorm */

/*
 * [RLA] residual RMSNorm with FP32 intermediates and one BF16 rounding:
 *   r       = f32(x) + f32(res)
 *   P_j     = sum over the 8 elements of leaf j, ascending, acc = fmaf(r, r, acc)
 *   ss      = TREE(Q, 0, T),  Q_t = TREE(P, t*nl/T, nl/T),  nl = H/8     (R1, R3)
 *   ms      = ss / H;  inv = 1 / sqrt(ms + eps)   (each op correctly rounded)
 *   y       = bf16((r * inv) * gamma);  res_out = bf16(r)
 * res == NULL means no residual input: r = f32(x) (no addition).
 * Returns 0, or -1 when H is not a multiple of 8 or T does not divide H/8.
 */
int oracle_rmsnorm_residual(const uint16_t* x, const uint16_t* res, const uint16_t* gamma,
                            uint16_t* y, uint16_t* res_out, int tokens, int H, float eps, int T) {
    if (H <= 0 || H % 8 || T <= 0 || (H / 8) % T) return -1;
    int nl = H / 8;
    float* r = (float*)malloc(sizeof(float) * (size_t)H);
    float* P = (float*)malloc(sizeof(float) * (size_t)nl);
    float* Q = (float*)malloc(sizeof(float) * (size_t)T);
    for (int t = 0; t < tokens; ++t) {
        const uint16_t* xr = x + (size_t)t * H;
        if (res) {
            const uint16_t* rr = res + (size_t)t * H;
            for (int h = 0; h < H; ++h) r[h] = bf(xr[h]) + bf(rr[h]);
        } else {
            for (int h = 0; h < H; ++h) r[h] = bf(xr[h]);
        }
        for (int j = 0; j < nl; ++j) {
            float acc = 0.0f;
            for (int e = 0; e < 8; ++e) acc = fmaf(r[8 * j + e], r[8 * j + e], acc);
            P[j] = acc;
        }
        for (int s = 0; s < T; ++s) Q[s] = tree_f32(P, s * (nl / T), nl / T);
        float ss = tree_f32(Q, 0, T);
        float ms = ss / (float)H;
        float inv = 1.0f / sqrtf(ms + eps);
        for (int h = 0; h < H; ++h) {
            float v = (r[h] * inv) * bf(gamma[h]);
            y[(size_t)t * H + h] = bf16_rne(v);
            if (res_out) res_out[(size_t)t * H + h] = bf16_rne(r[h]);
        }
    }
    free(r);
    free(P);
    free(Q);
    return 0;
}

/*
 * Residual add at the end of a row-parallel projection ([RLA]: the residual
 * add in fp32, one rounding): C[i] = bf16(root[i] + f32(R[i])), root the fp32
 * result of oracle_gemm_tree (or of oracle_gemm_noninv for the baseline).
 */
void oracle_add_residual_bf16(const float* root, const uint16_t* R, uint16_t* C, size_t n) {
    for (size_t i = 0; i < n; ++i) C[i] = bf16_rne(root[i] + bf(R[i]));
}

/* -------------------------------------------------------------- RoPE */

/*
 * cos/sin table in binary64, rounded to binary32 once ([RLA]: RoPE is the
 * main drift source, so the angle itself is formed in double):
 *   theta_i = base^(-2i/head_dim),  angle = pos * theta_i,
 *   table[pos][i][0] = (float)cos(angle), table[pos][i][1] = (float)sin(angle).
 */
void oracle_rope_table(float* table, int max_pos, int head_dim, double base) {
    int half = head_dim / 2;
    for (int p = 0; p < max_pos; ++p)
        for (int i = 0; i < half; ++i) {
            double theta = pow(base, -(double)(2 * i) / (double)head_dim);
            double ang = (double)p * theta;
            table[((size_t)p * half + i) * 2 + 0] = (float)cos(ang);
            table[((size_t)p * half + i) * 2 + 1] = (float)sin(ang);
        }
}

/*
 * Rotate-half RoPE in FP32, one BF16 rounding per output ([RLA]):
 *   o_i      = x_i * c_i - x_{i+half} * s_i
 *   o_{i+half} = x_{i+half} * c_i + x_i * s_i
 * each product rounded separately (no fma).  x: bf16 [tokens][heads][head_dim].
 */
void oracle_rope(const uint16_t* x, const int32_t* pos, const float* table, uint16_t* out,
                 int tokens, int heads, int head_dim) {
    int half = head_dim / 2;
    for (int t = 0; t < tokens; ++t)
        for (int h = 0; h < heads; ++h) {
            const uint16_t* xv = x + ((size_t)t * heads + h) * head_dim;
            uint16_t* ov = out + ((size_t)t * heads + h) * head_dim;
            const float* cs = table + (size_t)pos[t] * half * 2;
            for (int i = 0; i < half; ++i) {
                float c = cs[2 * i], s = cs[2 * i + 1];
                float x1 = bf(xv[i]), x2 = bf(xv[i + half]);
                float a = x1 * c, b = x2 * s;
                float o1 = a - b;
                float d = x2 * c, e = x1 * s;
                float o2 = d + e;
                ov[i] = bf16_rne(o1);
                ov[i + half] = bf16_rne(o2);
            }
        }
}

/* -------------------------------------------------------------- SwiGLU */

/* [RLA] SwiGLU in FP32, rounded once: o = bf16((g / (1 + exp(-g))) * u). */
static uint16_t swiglu1(float g, float u) {
    float e = exp_spec(-g);
    float den = 1.0f + e;
    float sg = g / den;
    return bf16_rne(sg * u);
}

void oracle_swiglu_bf16(const uint16_t* g, const uint16_t* u, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = swiglu1(bf(g[i]), bf(u[i]));
}

void oracle_swiglu_f32(const float* g, const float* u, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = swiglu1(g[i], u[i]);
}

/* ------------------------------------------------------------ logprob */

typedef struct {
    float m, s;
} ms_t;

/*
 * Combine of two (max, sum-exp) summaries: m = max(ma, mb); if m = -inf the
 * result is the identity (-inf, 0); else s = sa*exp(ma-m) + sb*exp(mb-m) with
 * the two products rounded separately.  The larger-of rule takes the first
 * argument on ties, which is symmetric for the values it can tie on.
 */
static ms_t ms_combine(ms_t a, ms_t b) {
    ms_t r;
    r.m = (b.m > a.m) ? b.m : a.m;
    if (r.m == -INFINITY) {
        r.s = 0.0f;
        return r;
    }
    float ea = exp_spec(a.m - r.m);
    float eb = exp_spec(b.m - r.m);
    float pa = a.s * ea;
    float pb = b.s * eb;
    r.s = pa + pb;
    return r;
}

static ms_t tree_ms(const ms_t* P, int lo, int n) {
    if (n == 1) return P[lo];
    int h = (n + 1) / 2;
    return ms_combine(tree_ms(P, lo, h), tree_ms(P, lo + h, n - h));
}

void oracle_tree_ms(const float* m, const float* s, int n, float* out_m, float* out_s) {
    ms_t* P = (ms_t*)malloc(sizeof(ms_t) * (size_t)n);
    for (int i = 0; i < n; ++i) {
        P[i].m = m[i];
        P[i].s = s[i];
    }
    ms_t r = tree_ms(P, 0, n);
    *out_m = r.m;
    *out_s = r.s;
    free(P);
}

/*
 * Target-token logprob through lm_head ([ISO] 壹/叁 compare exactly this
 * quantity; [TBIK] 技术框架 orders its reductions by the tree):
 *   z[v]       = tree-ordered dot product of hidden row i with W_lm row v over H
 *                (leaves of `leaf`, TREE over all H/leaf leaves); kept in FP32
 *   vocab leaf j covers columns [j*vleaf, (j+1)*vleaf) cut at V; for a leaf
 *     with columns: m_j = running max in ascending column order (a later column
 *     replaces the max only when strictly larger), s_j = sum in ascending order
 *     of exp(z - m_j) starting from 0;  an empty leaf is (-inf, 0)
 *   Lv = vpad/vleaf leaves; shard t owns leaves [t*Lv/T, (t+1)*Lv/T)
 *   (m_t, s_t) = TREE over its leaves; (m, s) = TREE over the T shards
 *   out[i]     = (z[target] - m) - log(s);  a target outside [0, V) gives NaN.
 * noninv != 0 is the non-invariant baseline applied to the lm_head GEMM:
 * H is split into T contiguous shards, each logit is one fma chain per shard
 * and the T partial logits are summed left to right ("per-shard GEMM, then a
 * sequential sum of the partials"); the vocabulary reduction is the tree
 * above, so the baseline differs from the method only in the logits.
 * row_m/row_s (nullable) receive the final (m, s) per row.
 */
int oracle_logprob(const uint16_t* hidden, const uint16_t* W, const int32_t* targets, float* out,
                   int M, int V, int H, int T, int leaf, int vleaf, int vpad, int noninv,
                   float* row_m, float* row_s) {
    if (M < 0 || V <= 0 || H <= 0 || leaf <= 0 || H % leaf || vleaf <= 0 || vpad < V ||
        vpad % vleaf || T <= 0)
        return -1;
    int Lk = H / leaf;
    int Lv = vpad / vleaf;
    if (Lv % T || (noninv && H % T)) return -1;
    int Ls = Lv / T;
    /* Rows are independent: a build with OpenMP may spread them over threads
       (each row with its own scratch, computed exactly as below). */
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < M; ++i) {
        float* z = (float*)malloc(sizeof(float) * (size_t)V);
        float* P = (float*)malloc(sizeof(float) * (size_t)Lk);
        ms_t* leaves = (ms_t*)malloc(sizeof(ms_t) * (size_t)Lv);
        ms_t* shards = (ms_t*)malloc(sizeof(ms_t) * (size_t)T);
        const uint16_t* h = hidden + (size_t)i * H;
        for (int v = 0; v < V; ++v) {
            const uint16_t* w = W + (size_t)v * H;
            if (noninv) {
                int Hs = H / T;
                float sum = 0.0f;
                for (int t = 0; t < T; ++t) {
                    float acc = 0.0f;
                    for (int k = t * Hs; k < (t + 1) * Hs; ++k) acc = fmaf(bf(h[k]), bf(w[k]), acc);
                    sum = t ? sum + acc : acc;
                }
                z[v] = sum;
            } else {
                for (int j = 0; j < Lk; ++j) {
                    float acc = 0.0f;
                    for (int k = j * leaf; k < (j + 1) * leaf; ++k) acc = fmaf(bf(h[k]), bf(w[k]), acc);
                    P[j] = acc;
                }
                z[v] = tree_f32(P, 0, Lk);
            }
        }
        for (int j = 0; j < Lv; ++j) {
            int c0 = j * vleaf, c1 = (j + 1) * vleaf;
            if (c1 > V) c1 = V;
            if (c0 >= c1) {
                leaves[j].m = -INFINITY;
                leaves[j].s = 0.0f;
                continue;
            }
            float m = z[c0];
            for (int c = c0 + 1; c < c1; ++c)
                if (z[c] > m) m = z[c];
            float s = 0.0f;
            for (int c = c0; c < c1; ++c) s = s + exp_spec(z[c] - m);
            leaves[j].m = m;
            leaves[j].s = s;
        }
        for (int t = 0; t < T; ++t) shards[t] = tree_ms(leaves, t * Ls, Ls);
        ms_t fin = tree_ms(shards, 0, T);
        if (row_m) row_m[i] = fin.m;
        if (row_s) row_s[i] = fin.s;
        int tg = targets[i];
        if (tg < 0 || tg >= V) {
            out[i] = NAN;
        } else {
            float d = z[tg] - fin.m;
            out[i] = d - log_spec(fin.s);
        }
        free(z);
        free(P);
        free(leaves);
        free(shards);
    }
    return 0;
}

/* Binary64 log-softmax gather, for tolerance checks: z in double, log-sum-exp in double. */
void oracle_logprob_f64(const uint16_t* hidden, const uint16_t* W, const int32_t* targets,
                        double* out, int M, int V, int H) {
    double* z = (double*)malloc(sizeof(double) * (size_t)V);
    for (int i = 0; i < M; ++i) {
        const uint16_t* h = hidden + (size_t)i * H;
        double mx = -INFINITY;
        for (int v = 0; v < V; ++v) {
            const uint16_t* w = W + (size_t)v * H;
            double acc = 0.0;
            for (int k = 0; k < H; ++k) acc += (double)bf(h[k]) * (double)bf(w[k]);
            z[v] = acc;
            if (acc > mx) mx = acc;
        }
        double s = 0.0;
        for (int v = 0; v < V; ++v) s += exp(z[v] - mx);
        int tg = targets[i];
        out[i] = (tg < 0 || tg >= V) ? NAN : (z[tg] - mx) - log(s);
    }
    free(z);
}

/* ------------------------------------------------------------- attention */
/*
 * Causal attention with the keys in fixed chunks combined by TREE (the
 * end-to-end decoder row; the pages' tree order applied to the reduction over
 * keys).  Readings (listed in the design notes as A1-A4):
 *  A1 score s_j = fl(dot(q_i, k_j) * scale): dot accumulated over the head
 *     dimension in ascending order with fmaf from +0, scale = the binary32
 *     nearest to 1/sqrt(head_dim).  Keys j <= i only.
 *  A2 keys form chunks of `chunk` consecutive positions; chunk c holds keys
 *     [c*chunk, c*chunk + chunk) that are <= i.  Per chunk: m = max of its
 *     scores; p_j = exp(s_j - m) (exp_spec), 0 for a slot past i;
 *     s = TREE over the chunk's `chunk` slots of p; o[d] = ascending sum over
 *     the chunk's keys of p_j * v_j[d] by fmaf from +0.
 *  A3 chunk results combine as (m,s,o) (+) (m',s',o'): M = max(m, m'),
 *     e = exp(m - M), e' = exp(m' - M), s = s*e + s'*e', o[d] = o[d]*e + o'[d]*e'
 *     (products rounded separately); the chunks 0..floor(i/chunk) by TREE.
 *  A4 out[d] = bf16(o[d] / s).
 * Layout: q, k, v, out bf16 [batch][seq][heads][head_dim]; head_dim <= 256.
 */
typedef struct {
    const uint16_t *q, *k, *v;
    int seq, heads, hd, chunk, i;
    size_t b_off;  /* element offset of this sequence */
    int h;
    float scale;
} att_ctx;

static size_t att_at(const att_ctx* c, int pos) {
    return c->b_off + ((size_t)pos * c->heads + c->h) * c->hd;
}

/* one chunk: (m, s, o) */
static void att_chunk(const att_ctx* c, int ci, float* m_out, float* s_out, float* o) {
    int j0 = ci * c->chunk;
    int j1 = j0 + c->chunk - 1;
    if (j1 > c->i) j1 = c->i;
    int n = j1 - j0 + 1;
    float* sc = (float*)malloc(sizeof(float) * (size_t)c->chunk);
    float* p = (float*)malloc(sizeof(float) * (size_t)c->chunk);
    const uint16_t* q = c->q + att_at(c, c->i);
    for (int t = 0; t < n; ++t) {
        const uint16_t* k = c->k + att_at(c, j0 + t);
        float dot = 0.0f;
        for (int d = 0; d < c->hd; ++d) dot = fmaf(bf(q[d]), bf(k[d]), dot);
        sc[t] = dot * c->scale;
    }
    float m = sc[0];
    for (int t = 1; t < n; ++t)
        if (sc[t] > m) m = sc[t];
    for (int t = 0; t < c->chunk; ++t) p[t] = (t < n) ? exp_spec(sc[t] - m) : 0.0f;
    float s = tree_f32(p, 0, c->chunk);
    for (int d = 0; d < c->hd; ++d) {
        float acc = 0.0f;
        for (int t = 0; t < n; ++t) acc = fmaf(p[t], bf(c->v[att_at(c, j0 + t) + d]), acc);
        o[d] = acc;
    }
    *m_out = m;
    *s_out = s;
    free(sc);
    free(p);
}

/* TREE over chunks [lo, lo+n) */
static void att_tree(const att_ctx* c, int lo, int n, float* m_out, float* s_out, float* o) {
    if (n == 1) {
        att_chunk(c, lo, m_out, s_out, o);
        return;
    }
    int h = (n + 1) / 2;
    float ma, sa, mb, sb, ob[256];
    att_tree(c, lo, h, &ma, &sa, o);
    att_tree(c, lo + h, n - h, &mb, &sb, ob);
    float M = (mb > ma) ? mb : ma;
    float ea = exp_spec(ma - M), eb = exp_spec(mb - M);
    float pa = sa * ea, pb = sb * eb;
    *m_out = M;
    *s_out = pa + pb;
    for (int d = 0; d < c->hd; ++d) {
        float xa = o[d] * ea, xb = ob[d] * eb;
        o[d] = xa + xb;
    }
}

int oracle_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, int batch, int seq,
                     int heads, int head_dim, int chunk) {
    if (batch < 0 || seq < 0 || heads <= 0 || head_dim <= 0 || head_dim > 256 || chunk <= 0) return -1;
    att_ctx c;
    c.q = q;
    c.k = k;
    c.v = v;
    c.seq = seq;
    c.heads = heads;
    c.hd = head_dim;
    c.chunk = chunk;
    c.scale = (float)(1.0 / sqrt((double)head_dim));
    float o[256];
    for (int b = 0; b < batch; ++b) {
        c.b_off = (size_t)b * seq * heads * head_dim;
        for (int h = 0; h < heads; ++h) {
            c.h = h;
            for (int i = 0; i < seq; ++i) {
                c.i = i;
                float m, s;
                att_tree(&c, 0, i / chunk + 1, &m, &s, o);
                uint16_t* dst = out + att_at(&c, i);
                for (int d = 0; d < head_dim; ++d) dst[d] = bf16_rne(o[d] / s);
            }
        }
    }
    return 0;
}

/* Binary64 causal softmax attention (no chunks), for tolerance checks. */
void oracle_attention_f64(const uint16_t* q, const uint16_t* k, const uint16_t* v, double* out, int batch, int seq,
                          int heads, int head_dim) {
    double* sc = (double*)malloc(sizeof(double) * (size_t)(seq > 0 ? seq : 1));
    double scale = 1.0 / sqrt((double)head_dim);
    for (int b = 0; b < batch; ++b)
        for (int h = 0; h < heads; ++h)
            for (int i = 0; i < seq; ++i) {
                size_t qi = (((size_t)b * seq + i) * heads + h) * head_dim;
                double mx = -INFINITY;
                for (int j = 0; j <= i; ++j) {
                    size_t kj = (((size_t)b * seq + j) * heads + h) * head_dim;
                    double dot = 0.0;
                    for (int d = 0; d < head_dim; ++d) dot += (double)bf(q[qi + d]) * (double)bf(k[kj + d]);
                    sc[j] = dot * scale;
                    if (sc[j] > mx) mx = sc[j];
                }
                double s = 0.0;
                for (int j = 0; j <= i; ++j) s += exp(sc[j] - mx);
                for (int d = 0; d < head_dim; ++d) {
                    double acc = 0.0;
                    for (int j = 0; j <= i; ++j) {
                        size_t vj = (((size_t)b * seq + j) * heads + h) * head_dim;
                        acc += exp(sc[j] - mx) * (double)bf(v[vj + d]);
                    }
                    out[qi + d] = acc / s;
                }
            }
    free(sc);
}
