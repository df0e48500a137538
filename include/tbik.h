/*
 * tbik.h -- C ABI of the tree-ordered invariant kernels (TBIK-style) for NVIDIA
 * B200 (sm_100a).
 *
 * What the library computes (sources are web pages, cited by title/section):
 *  - "Deterministic Inference across Tensor Parallel Sizes That Eliminates
 *    Training-Inference Mismatch" (paper summary page), sections 核心思路 and
 *    技术框架 and the abstract: matrix multiplication and reduction primitives
 *    whose local (per-GPU) and global (cross-GPU) reductions follow ONE
 *    hierarchical binary tree, so results are bitwise identical for any
 *    tensor-parallel (TP) size.
 *  - Rounding-location alignment article (winzheng.jp), section
 *    "外科手術的な修正：3つのノード": RoPE, SwiGLU and residual RMSNorm keep FP32
 *    intermediates and round to BF16 once, at the output.
 *  - IsoExec executive brief (nxmr.cn), sections 壹, 叁 and 伍: the per-token
 *    logprob is the quantity that must agree bit for bit.
 *
 * The tree.  A reduction over L leaves uses TREE(P, lo, n): n == 1 gives P[lo];
 * otherwise h = ceil(n/2) and the value is TREE(P,lo,h) + TREE(P,lo+h,n-h)
 * (binary32 add, round to nearest even).  T shards of the reduced dimension
 * are contiguous ranges of L/T leaves; for T in {1,2,4,8} with T | L each
 * shard is one whole subtree, so the result does not depend on T.  On one GPU
 * T is emulated: each shard's partial goes to its own fp32 buffer and the
 * partials are combined with TREE over T.
 *
 * Conventions for every entry point:
 *  - bf16 buffers are passed as raw 16-bit patterns (IEEE bfloat16).
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or synchronises on these paths (exceptions are
 *    named: tbik_rope_table and tbik_get_error).  Pointers must be 16-byte
 *    aligned (TBIK_ERR_ALIGN otherwise).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    All work is enqueued on it; results do not depend on the stream or on
 *    other work running concurrently.
 *  - Host-detected errors return a status immediately and enqueue nothing.
 *    Device-detected errors (bad target or position, a bounded wait that
 *    expired) are recorded in a per-device error word read by tbik_get_error.
 *  - Functions are thread-safe; concurrent calls must not share a workspace.
 */
#ifndef TBIK_H
#define TBIK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TBIK_API __attribute__((visibility("default")))
#else
#define TBIK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TBIK_OK = 0,
    TBIK_ERR_ARG = 1,         /* null pointer, negative size, unknown mode bit */
    TBIK_ERR_SHAPE = 2,       /* K % leaf, T not in {1,2,4,8}, T does not divide the leaves ... */
    TBIK_ERR_ALIGN = 3,       /* pointer or row stride not 16-byte aligned */
    TBIK_ERR_WORKSPACE = 4,   /* workspace missing or smaller than the *_workspace() query */
    TBIK_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed */
    TBIK_ERR_TIMEOUT = 6,     /* a device-side bounded wait expired (kernel returned early) */
    TBIK_ERR_TARGET = 7,      /* a logprob target outside [0, V) (its output is NaN) */
    TBIK_ERR_POSITION = 8,    /* a RoPE position outside [0, max_pos) (its outputs are NaN) */
    TBIK_ERR_UNSUPPORTED = 9  /* not a B200-class device (sm_100) */
} tbik_status;

/* ---- mode bits ---------------------------------------------------------- */
/* Arithmetic of the leaf partials (exactly one of the two): */
#define TBIK_EXACT 0x1u  /* CUDA cores: per output, per leaf, acc = fmaf(a, b, acc) in
                            ascending k from +0.0f, then the tree.  Bit-exact to the
                            definition. */
#define TBIK_TC 0x2u     /* tcgen05 tensor cores: each leaf is one chain of 128x128x16
                            bf16 MMAs accumulating in fp32 (TMEM) from zero; leaves are
                            then combined by the same tree in fp32.  The leaf bits are
                            fixed by the hardware and identical for every T and M. */
/* Deliberately non-invariant baseline (with EXACT or TC): each shard
   accumulates its whole K range in one chain and the shard partials are summed
   left to right, ((Q0+Q1)+Q2)+...  In tbik_logprob this applies to the lm_head
   logits (H split into T shards, requires H % T == 0, and (H/T) % 16 == 0 in
   TC mode); the vocabulary reduction stays the tree. */
#define TBIK_NONINV 0x4u
/* Layout of B in tbik_gemm (row-major in both cases): */
#define TBIK_B_KN 0x00u  /* B is [K,N] (N contiguous) */
#define TBIK_B_NK 0x10u  /* B is [N,K] (K contiguous), e.g. an nn.Linear weight */
/* Output type of tbik_gemm: */
#define TBIK_OUT_F32 0x000u  /* C fp32 [M,N] */
#define TBIK_OUT_BF16 0x100u /* C bf16 [M,N], rounded once (RNE) from the fp32 tree root */
/* Gate/up projection fused with SwiGLU: B's N = 2F columns hold the gate and
   up weights interleaved in blocks of 32 (columns [64j, 64j+32) = gate
   features [32j, 32j+32), columns [64j+32, 64j+64) = up features of the same
   features); C is bf16 [M, F] = bf16((g / (1 + exp(-g))) * u) from the fp32
   tree roots g, u (the library's exp specification, no rounding before the
   output).  F % 32 == 0.  Not combinable with TBIK_NONINV; implies bf16 C. */
#define TBIK_SWIGLU_OUT 0x200u

/* Vocabulary columns per logprob leaf, and the largest shard count the vocab
   padding is sized for: V is padded to Vpad = ceil(V / (64*8)) * 64*8 with
   identity leaves (max -inf, sum 0), independent of T. */
#define TBIK_VOCAB_LEAF 64
#define TBIK_T_MAX 8

TBIK_API const char* tbik_version(void);
TBIK_API const char* tbik_status_string(tbik_status s);

/* ---- tree-ordered GEMM -------------------------------------------------- */

/*
 * Bytes of device workspace tbik_gemm needs for these arguments (0 is a valid
 * answer: T = 1 at a size with enough output tiles writes C directly).
 * Returns (size_t)-1 when the arguments would be rejected.
 */
TBIK_API size_t tbik_gemm_workspace(int M, int N, int K, int T, int leaf, unsigned mode);

/*
 * C = A * B with the K reduction in tree order (TBIK summary page, 技术框架:
 * local reduction on each GPU, then a binary-tree reduction across GPUs;
 * tutorial page section 2.1.1 / figure 5: T-way row-parallel split of K).
 *
 *   A  bf16 [M,K] row-major.          B  bf16 [K,N] or [N,K] (mode TBIK_B_*).
 *   C  fp32 or bf16 [M,N] row-major (mode TBIK_OUT_*); may not alias A or B.
 *   leaf  K elements per leaf; K % leaf == 0; L = K/leaf leaves.
 *   T  emulated shard count in {1,2,4,8}; (K/leaf) % T == 0.  Shard t owns
 *      leaves [t*L/T, (t+1)*L/T); its partial is written to its own fp32
 *      buffer in the workspace and the T partials are combined by TREE.
 *   TBIK_TC needs leaf % 16 == 0, N % 8 == 0 and K % 8 == 0 (16-byte TMA
 *   strides); with TBIK_NONINV, (K/T) % 16 == 0 instead of the leaf rule.
 *   ws/ws_bytes  device workspace of at least tbik_gemm_workspace() bytes,
 *      256-byte aligned; may be NULL when that query returns 0.
 * Row i of C depends only on row i of A: any batch size, split or order gives
 * the same bits per row.  M == 0 is a no-op.
 */
TBIK_API tbik_status tbik_gemm(const uint16_t* A, const uint16_t* B, void* C, int M, int N, int K, int T,
                      int leaf, unsigned mode, void* ws, size_t ws_bytes, void* stream);

/*
 * Row-parallel projection with the residual add fused into its last step
 * (the down or output projection of a pre-norm block: the rounding-location
 * article, 3つのノード, keeps the residual add in fp32 and rounds once):
 *   C[i,n] = bf16( root[i,n] + f32(R[i,n]) ),
 * root = the fp32 tree root tbik_gemm computes for the same arguments, one
 * correctly rounded fp32 add, then one RNE rounding.  The add happens where
 * the root is final: the GEMM epilogue when the tiles write C directly, else
 * the kernel that combines the shard partials (the non-invariant baseline
 * adds R after its left-to-right shard sum).
 *   R, C  bf16 [M,N] row-major, 16-byte aligned; C may be R itself (in place)
 *         but may not overlap it otherwise, nor alias A or B.
 *   mode  as tbik_gemm without TBIK_OUT_* bits (the output is bf16) and
 *         without TBIK_SWIGLU_OUT (else TBIK_ERR_ARG).
 *   ws    tbik_gemm_workspace(M, N, K, T, leaf, mode | TBIK_OUT_BF16) bytes.
 * Errors and shape rules are those of tbik_gemm; R == NULL is TBIK_ERR_ARG.
 */
TBIK_API tbik_status tbik_gemm_residual(const uint16_t* A, const uint16_t* B, const uint16_t* R, uint16_t* C,
                               int M, int N, int K, int T, int leaf, unsigned mode, void* ws,
                               size_t ws_bytes, void* stream);

/* ---- residual RMSNorm ---------------------------------------------------- */

/*
 * Residual RMSNorm with fp32 intermediates and one bf16 rounding
 * (rounding-location article, 3つのノード: residual RMSNorm):
 *   r = f32(x) + f32(res);  leaf j = elements [8j, 8j+8), P_j = fmaf(r,r,acc)
 *   ascending from +0;  ss = TREE over the H/8 leaves (T shards of H/(8T)
 *   leaves, shard partials combined by TREE);  ms = ss / H;
 *   inv = 1 / sqrt(ms + eps) (correctly rounded ops);
 *   y = bf16((r * inv) * gamma);  res_out = bf16(r).
 * x, res, y, res_out: bf16 [tokens,H]; gamma bf16 [H]; res_out may be NULL;
 * res may be NULL (r = f32(x): the norm of a residual stream that
 * tbik_gemm_residual already updated); y may alias x.  H % 8 == 0 and H/8 a power of two in [32, 1024]
 * (H in {256, 512, ..., 8192}); T in {1,2,4,8}.
 */
TBIK_API tbik_status tbik_rmsnorm_residual(const uint16_t* x, const uint16_t* res, const uint16_t* gamma,
                                  uint16_t* y, uint16_t* res_out, int tokens, int H, float eps,
                                  int T, void* stream);

/* ---- RoPE + SwiGLU (fp32 intermediates, one rounding) -------------------- */

/*
 * Fills the DEVICE buffer `table` (fp32 [max_pos][head_dim/2][2], cos then
 * sin) from binary64 arithmetic rounded once to fp32:
 *   theta_i = base^(-2i/head_dim),  angle = pos * theta_i.
 * The table is computed on the host and copied synchronously (set-up call,
 * not for the hot path).  head_dim even, 2 <= head_dim <= 512.
 */
TBIK_API tbik_status tbik_rope_table(float* table, int max_pos, int head_dim, double base, void* stream);

typedef struct {
    /* RoPE group, rotate-half form (skipped when q and k are both NULL):
       for i < head_dim/2:  o_i = x_i*c_i - x_{i+half}*s_i,
                            o_{i+half} = x_{i+half}*c_i + x_i*s_i,
       each product rounded separately (no fma), one bf16 rounding.
       q/k bf16 [tokens][heads][head_dim]; outputs may alias inputs; either of
       q or k may be NULL.  head_dim % 16 == 0, head_dim <= 512. */
    const uint16_t* q;
    const uint16_t* k;
    uint16_t* q_out;
    uint16_t* k_out;
    const int32_t* pos;  /* [tokens], each in [0, max_pos) */
    const float* table;  /* from tbik_rope_table */
    int tokens;
    int heads;
    int head_dim;
    int max_pos;
    /* SwiGLU group (skipped when g is NULL): out = bf16((g / (1 + exp(-g))) * u)
       in fp32 with the library's exp specification (Cody-Waite reduction by a
       split ln 2, degree-7 Taylor polynomial, correctly rounded scaling).
       g/u bf16 or fp32 (in_f32 = 1) [n]; out bf16 [n]; n % 8 == 0.
       With bf16 g, silu(g) = g / (1 + exp(-g)) is read from a table of its
       fp32 value for every bf16 g (the same bits): the first such call on a
       device builds the 256 KiB table on its stream and records an event that
       later calls on any stream wait for; make that first call outside a
       stream capture. */
    const void* g;
    const void* u;
    uint16_t* out;
    long long n;
    int in_f32;
} tbik_rope_swiglu_args;

TBIK_API tbik_status tbik_rope_swiglu_fp32(const tbik_rope_swiglu_args* args, void* stream);

/* ---- causal attention with the key reduction in tree order --------------- */

/*
 * Attention of each query position over the keys at positions <= its own,
 * with the reduction over keys in the same halving tree as every other
 * reduction here (TBIK summary page, 技术框架), so the output does not depend
 * on the batch composition or on how heads are split across devices:
 *   s_j = fl(dot(q_i, k_j) * scale), dot ascending over the head dimension by
 *         fma from +0, scale = binary32 nearest to 1/sqrt(head_dim);
 *   keys in chunks of `chunk` = 64 positions; per chunk m = max of its scores,
 *   p_j = exp(s_j - m) (the library's exp specification), s = TREE over the
 *   chunk's 64 slots of p (0 past position i), o[d] = ascending sum of
 *   p_j * v_j[d] by fma from +0;
 *   chunk summaries combined by TREE: M = max, e = exp(m - M),
 *   s = s*e + s'*e', o = o*e + o'*e' (products rounded separately);
 *   out[d] = bf16(o[d] / s).
 * q, k, v, out: bf16 [batch][seq][heads][head_dim] in device memory, 16-byte
 * aligned; out may alias q but not k or v.  head_dim in {64, 128};
 * chunk == 64; seq <= 16384.  Returns TBIK_ERR_SHAPE / _ARG / _ALIGN for
 * violations, without launching.
 */
TBIK_API tbik_status tbik_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, int batch,
                                    int seq, int heads, int head_dim, int chunk, void* stream);

/*
 * The same attention in tensor-core mode (TBIK summary page, 技术框架: the
 * key reduction stays one fixed tree, here of 128-key leaves, each computed
 * as two 64-key tensor-core chunks under one maximum).  Per leaf:
 *   s_j = fl(dot(q_i, k_j) * scale) with the dot product on the tensor cores
 *         (bf16 operands, fp32 accumulation in the hardware's fixed order);
 *   m = max over the leaf's keys j <= i; p_j = bf16(2^(s_j*log2e - m*log2e))
 *   (hardware exponential; 0 for j > i); s = s_lo + s_hi over the rounded
 *   p_j (keys 0..63 and 64..127 of the leaf, each (c0 + c1) + (c2 + c3) with
 *   c_q the ascending sum over its keys k = q mod 4); o = sum of p_j * v_j
 *   on the tensor cores;
 * leaf summaries combined by TREE: M = max, e = 2^(fl(m - M)*log2e) (the
 * hardware exponential; 1 for the side holding M), s = fma(s', e', fl(s*e)),
 * o = fma(o', e', fl(o*e)) (left operand's product rounded);
 * out[d] = bf16(o[d] * fl(1/s)).  Each output row depends only on its query and
 * the keys/values at positions <= i, so it is bitwise the same for any batch
 * composition and head split; it is checked against the binary64 definition
 * by tolerance.
 * q, k, v, out: bf16 [batch][seq][heads][head_dim], device memory, 16-byte
 * aligned; out may alias q but not k or v.  head_dim == 128, chunk == 128
 * (the leaf), seq a multiple of 128 and <= 16384 (else TBIK_ERR_SHAPE);
 * workspace: device memory of at least tbik_attention_tc_workspace() bytes,
 * 16-byte aligned (TBIK_ERR_WORKSPACE / TBIK_ERR_ALIGN otherwise; may be NULL
 * when that is 0), owned by the caller and not used by concurrent calls.  No
 * launch on error.
 */
TBIK_API size_t tbik_attention_tc_workspace(int batch, int seq, int heads, int head_dim, int chunk);
TBIK_API tbik_status tbik_attention_tc(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                                       int batch, int seq, int heads, int head_dim, int chunk, void* workspace,
                                       size_t ws_bytes, void* stream);

/*
 * Embedding rows: out[t] = table[ids[t]] for t < tokens (bf16 rows of d
 * elements, d % 8 == 0, 16-byte aligned).  An id outside [0, V) gives a zero
 * row and records TBIK_ERR_TARGET in the device error word.  Data movement
 * only (the decoder's first step); no counterpart on the pages.
 */
TBIK_API tbik_status tbik_embedding(const int32_t* ids, const uint16_t* table, uint16_t* out, int tokens, int V,
                                    int d, void* stream);

/*
 * out[c][r] = in[r][c] for bf16 [rows, cols] -> [cols, rows] (device memory,
 * 2-byte aligned, no overlap).  Data movement only: it gives the weight
 * gradient dW = X^T dY its A operand, so that dW = tbik_gemm(X^T, dY) reduces
 * over tokens with the same leaf tree (T = data-parallel shards of the
 * tokens).  No counterpart on the pages.
 */
TBIK_API tbik_status tbik_transpose(const uint16_t* in, uint16_t* out, int rows, int cols, void* stream);

/* ---- fused lm_head -> log-softmax -> target logprob ---------------------- */

TBIK_API size_t tbik_logprob_workspace(int M, int V, int H, int T, int leaf, unsigned mode);

/*
 * out[i] = log softmax(hidden[i] . W_lm^T)[targets[i]] (IsoExec brief 壹/叁:
 * the logprob is the compared quantity; TBIK page: tree-ordered reductions),
 * without materialising the logits (TBIK_TC):
 *   z[i,v]  = tree-ordered dot product over H (leaves of `leaf`, TREE over
 *             all H/leaf leaves), kept fp32;
 *   vocab leaf j = columns [64j, 64j+64) cut at V: m_j = max in ascending
 *             column order, s_j = sum in ascending order of exp(z - m_j)
 *             (TBIK_EXACT: the library's exp specification, bit-exact to the
 *             definition; TBIK_TC: the hardware base-2 exponential, a few ulp);
 *   (m,s) combine: m = max(ma,mb); s = sa*exp(ma-m) + sb*exp(mb-m) (products
 *             rounded separately); identity (-inf, 0);
 *   shard t (of T) owns the vocab leaves [t*Lv/T, (t+1)*Lv/T) of the padded
 *             Lv = Vpad/64; shard summaries and then the T shards combine by TREE;
 *   out[i]  = (z[i,target] - m) - log(s)  (library log specification).
 * hidden bf16 [M,H]; W_lm bf16 [V,H] row-major; targets int32 [M]; out fp32 [M].
 * H % leaf == 0, leaf % 16 == 0, H % 8 == 0, T in {1,2,4,8}.  A target outside
 * [0,V) gives NaN and records TBIK_ERR_TARGET.  TBIK_EXACT materialises the
 * fp32 logits in the workspace (CUDA-core reference mode).
 */
TBIK_API tbik_status tbik_logprob(const uint16_t* hidden, const uint16_t* W_lm, const int32_t* targets,
                         float* out, int M, int V, int H, int T, int leaf, unsigned mode, void* ws,
                         size_t ws_bytes, void* stream);

/* ---- tensor parallelism across GPUs: the shard level of the tree ---------- */
/*
 * The TBIK summary page (技术框架) orders the reduction ACROSS GPUs by the same
 * binary tree as the local one.  With T ranks, rank t computes the root of its
 * own subtree (its shard), the T shard results are exchanged into every rank's
 * own memory (for example an NCCL all-gather; never a sum all-reduce, whose
 * order depends on the rank count), and every rank applies the top log2(T)
 * levels of the tree with the calls below.  The result is bitwise the same as
 * tbik_gemm / tbik_logprob on one GPU, for every T.
 *
 * Row-parallel GEMM (K split into T contiguous shards of whole leaves): rank t
 * calls tbik_gemm on its [M, K/T] and [K/T, N] (or [N, K/T]) slices with T = 1
 * and an fp32 output (the root of its subtree: TREE over its L/T leaves; with
 * TBIK_NONINV, its one chain), gathers the T results as fp32 [T][M*N] in rank
 * order, and calls:
 *
 *   out = TREE over t of partials[t] (T in {1,2,4,8}; with TBIK_NONINV the
 *         left-to-right sum ((P0 + P1) + P2) + ... of the baseline instead);
 *   mode  TBIK_OUT_BF16 for a bf16 output rounded once (else fp32), optionally
 *         | TBIK_NONINV; R (bf16 [MN], nullable, needs TBIK_OUT_BF16) is added
 *         to the fp32 root before the rounding, as in tbik_gemm_residual.
 *   partials fp32 [T][MN] and out, R: device memory, 16-byte aligned; out may
 *   be R (in place) but may not overlap partials.
 */
TBIK_API tbik_status tbik_tree_combine(const float* partials, void* out, long long MN, int T, unsigned mode,
                                       const uint16_t* R, void* stream);

/*
 * Vocabulary-parallel logprob.  The padded vocabulary of tbik_logprob
 * (Vpad = ceil(V / 512) * 512 columns, Lv = Vpad / 64 leaves) is split into T
 * contiguous shards of Lv/T leaves: shard t covers vocabulary indices
 * [v0, v0 + Vpad/T) with v0 = t * Vpad / T, of which Vs = clamp(V - v0, 0,
 * Vpad/T) are real columns.  Rank t holds W_shard = rows [v0, v0 + Vs) of W_lm
 * (bf16 [Vs, H]) and calls tbik_logprob_partial with Lvs = Lv / T:
 *   part[i] = (m, s, z, own) as 4 floats: (m, s) = TREE over the shard's Lvs
 *   vocabulary leaves (leaves past its Vs columns are identities); own = 1
 *   and z = the target's logit when targets[i] is in [v0, v0 + Vs), else
 *   own = 0 and z = 0.  Everything else as tbik_logprob in TBIK_TC or
 *   TBIK_EXACT mode (TBIK_NONINV is refused with TBIK_ERR_ARG).  Vs may be 0
 *   (a shard of padding only; W_shard is then not read).
 * Then gather the T part arrays as fp32 [T][M][4] in rank order and call
 * tbik_logprob_combine: per row TREE over the T (m, s), z from the owning
 * shard, out = (z - m) - log(s); a target outside [0, V) (or owned by no
 * shard) gives NaN and records TBIK_ERR_TARGET.
 * part, parts: 16-byte aligned device memory; ws as for tbik_logprob, sized by
 * tbik_logprob_partial_workspace.
 */
TBIK_API size_t tbik_logprob_partial_workspace(int M, int Vs, int Lvs, int H, int leaf, unsigned mode);
TBIK_API tbik_status tbik_logprob_partial(const uint16_t* hidden, const uint16_t* W_shard, const int32_t* targets,
                                          float* part, int M, int Vs, int v0, int Lvs, int H, int leaf,
                                          unsigned mode, void* ws, size_t ws_bytes, void* stream);
TBIK_API tbik_status tbik_logprob_combine(const float* parts, const int32_t* targets, float* out, int M, int V,
                                          int T, void* stream);

/*
 * tbik_logprob_noalloc -- the pages have no counterpart for this entry point.
 *
 * For callers that cannot allocate device memory (code that must not call
 * cudaMalloc, for example while its stream is being captured or under an
 * allocator that forbids side allocations, and plain C callers with no device
 * allocator of their own).  Same arguments and results as tbik_logprob in
 * tensor-core mode (mode = TBIK_TC, optionally | TBIK_NONINV), minus the
 * workspace: the scratch comes from one fixed device array of
 * TBIK_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits.  The caller still passes inputs and
 * outputs.  Nothing is allocated or freed.
 *  - Returns TBIK_ERR_WORKSPACE, and launches nothing, when the arguments need
 *    more scratch than TBIK_NOALLOC_SCRATCH_BYTES (that is, when
 *    tbik_logprob_workspace() for the same arguments is larger).  For the
 *    151936 x 4096 lm_head with leaf 256 on a 148-SM B200 this allows up to
 *    997 rows per call.
 *  - Returns TBIK_ERR_ARG for any mode without TBIK_TC or with TBIK_EXACT;
 *    otherwise the status tbik_logprob would return for the same arguments
 *    (TBIK_ERR_ARG, _SHAPE, _CUDA, _UNSUPPORTED) before the size check.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.  The address is kept for the life of the
 *    process: do not use this entry point across a cudaDeviceReset.
 *  - All calls share the one array, which keeps the last call's contents.
 *    Nothing in it needs clearing (every value read is written earlier in the
 *    same call), but calls that overlap on the GPU (two streams, or two host
 *    threads on one device) race on it: serialise them.
 */
#define TBIK_NOALLOC_SCRATCH_BYTES (32u << 20)
TBIK_API tbik_status tbik_logprob_noalloc(const uint16_t* hidden, const uint16_t* W_lm, const int32_t* targets,
                                          float* out, int M, int V, int H, int T, int leaf, unsigned mode,
                                          void* stream);

/* ---- errors -------------------------------------------------------------- */

/*
 * Synchronises `stream`, then returns and clears the error word of the
 * current device (TBIK_OK when no device-side error was recorded).  Returns
 * TBIK_ERR_CUDA if the synchronisation itself reports an error.
 */
TBIK_API tbik_status tbik_get_error(void* stream);

/*
 * Test hooks.  flags: TBIK_DEBUG_WITHHOLD_ACC_ARRIVE makes the tensor-core GEMM
 * epilogue withhold its "accumulator drained" arrive (and the tensor-core
 * attention's epilogue its "P written" arrive), so the MMA issuer's bounded
 * wait expires: the kernel must record TBIK_ERR_TIMEOUT, drain its own copies
 * in flight, free its TMEM and return.  TBIK_DEBUG_TILE128 runs every
 * tensor-core GEMM on the 128-column pair tile (normally 192 columns unless B
 * is [K,N] with N <= 128), so that tests can compare the two tile designs on
 * the same operands.  wait_limit_ns bounds every device-side wait (0 keeps the
 * default of 2 s).
 */
#define TBIK_DEBUG_WITHHOLD_ACC_ARRIVE 0x1u
#define TBIK_DEBUG_TILE128 0x2u
TBIK_API tbik_status tbik_debug_set(unsigned flags, unsigned long long wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* TBIK_H */
