/*
 * fluxbin.h -- C ABI of the B200 LUT binary GEMV library (libfluxbin.so).
 *
 * The method is the one on the FluxBin page ("FluxBin: Flexible LUT-based
 * Ultra-low-bit LLM Inference by Algorithm-Kernel Synergy"), Methodology:
 *
 *   W_hat = sum_k (alpha_r^(k) alpha_c^(k)^T) (.) B^(k)           [1. Algorithm innovation]
 *         + the same over a salient column subset S with Ks extra bases
 *                                       [Hessian-guided saliency-aware hybrid bases]
 *   y = W_hat x, computed without dequantising W_hat: per-block lookup tables
 *   with alpha_c fused in (LUT-BSF), the salient columns gathered into a dense
 *   compact operand (virtual columnar mapping, VCM), packed uint32 weights
 *   streamed with bit operations extracting pattern indices, and alpha_r
 *   applied in the reduction                                 [2. Kernel innovation]
 *
 * B^(k) entries are +/-1.  Ternary {-1,0,+1} weights (FlashLM v6 page,
 * "Ternary weights and hardware efficiency") are two +/-1 bases with row
 * scales 0.5*alpha_r and alpha_c = 1.
 *
 * Conventions for every entry point:
 *  - All array arguments are DEVICE pointers unless stated otherwise.  The
 *    caller allocates and owns every buffer.  Apart from the calls marked
 *    "synchronous", the library never allocates, frees or synchronises.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Work is enqueued asynchronously; buffers must stay valid until
 *    the stream reaches it.  Launches go to the current CUDA device.
 *  - Argument errors are detected on the host before anything is enqueued and
 *    returned synchronously; nothing is launched in that case.  A launch that
 *    the CUDA runtime rejects returns FB_ERR_CUDA.  No kernel of this library
 *    traps, asserts or waits without a bound.
 *  - Sizes are int; 1 <= M <= 2^24, 32 <= N <= 2^20 with N % 32 == 0,
 *    1 <= K <= 4, 0 <= nS <= N, 1 <= Ks <= 4 when nS > 0, g in {1,2,4,8}.
 */
#ifndef FLUXBIN_H_
#define FLUXBIN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FLUXBIN_ABI_VERSION 1

#if defined(__GNUC__)
#define FB_API __attribute__((visibility("default")))
#else
#define FB_API
#endif

typedef enum {
    FB_OK = 0,
    FB_ERR_INVALID_VALUE = 1, /* a size, pointer, dtype or group width is invalid */
    FB_ERR_UNSUPPORTED = 2,   /* valid request outside what this library implements */
    FB_ERR_MISALIGNED = 3,    /* a pointer breaks the alignment stated below */
    FB_ERR_WORKSPACE = 4,     /* workspace missing, misaligned or too small */
    FB_ERR_CUDA = 5           /* the CUDA runtime reported an error */
} fb_status;

typedef enum { FB_F32 = 0, FB_F16 = 1, FB_BF16 = 2 } fb_dtype;

/*
 * Device layout of packed sign planes ("planes"), produced by fb_pack /
 * fb_pack_bits.  It is the same for every group width g.
 *
 *  - Rows are padded to M_pad = roundup(M, 32) and split into chunks of 32
 *    rows; padded rows hold 0 bits and never reach the output.
 *  - Columns are split into panels of 256 (the last panel holds N mod 256
 *    columns when that is non-zero; always a multiple of 32).  Panel p has
 *    Bp = width/8 "byte groups": byte group q is columns 256p+8q .. 256p+8q+7,
 *    bit t (LSB first) is column 256p+8q+t, set bit = +1, clear bit = -1.
 *  - Base k occupies bytes [k*M_pad*N/8, (k+1)*M_pad*N/8).  Inside it, panel
 *    p starts at byte 32*p*M_pad and holds M_pad/32 chunk blocks of 32*Bp
 *    bytes each (chunk c at 32*Bp*c).
 *  - In a chunk block, row 32c+l ("lane" l) stores its Bp bytes ROTATED:
 *    stored position u (0..Bp-1) holds byte group (l+u) mod Bp.  Position u
 *    of lane l sits at byte  (u/16)*512 + 16*l + u%16  when Bp % 16 == 0,
 *    else at byte           (u/4)*128  + 4*l  + u%4.
 * The rotation lets the 32 lanes of a warp, each walking its own row, read
 * 32 different byte groups at every step, so their table lookups fall in 32
 * different shared-memory banks.
 *
 * fb_packed_words: number of uint32 words of planes for K bases of an M x N
 * matrix (K * M_pad * N / 32); 0 for invalid sizes.  Host only.
 */
FB_API size_t fb_packed_words(int K, int M, int N);

/* fb_pack: signs [K][M][N] int8, each +1 or -1 (any value > 0 counts as +1),
 * row-major -> planes (fb_packed_words(K,M,N) words, 16-byte aligned).
 * Load-time packer (step "a1"): the bit planes B^(k) of the FluxBin page's
 * decomposition, stored as uint32 words ("compressed Uint32 weights",
 * 2. Kernel innovation, execution flow). */
FB_API fb_status fb_pack(const int8_t *signs, int K, int M, int N, uint32_t *planes, void *stream);

/* fb_pack_bits: canonical bit planes [K][M][N/8] uint8 (bit t of byte j of a
 * row = column 8j+t, set = +1) -> planes.  Same output as fb_pack. */
FB_API fb_status fb_pack_bits(const uint8_t *bits, int K, int M, int N, uint32_t *planes, void *stream);

/* fb_unpack: planes -> signs [K][M][N] int8 (+1/-1).  Test aid; inverse of
 * fb_pack. */
FB_API fb_status fb_unpack(const uint32_t *planes, int K, int M, int N, int8_t *signs, void *stream);

/* fb_vcm_gather: virtual columnar mapping (FluxBin page, 2. Kernel
 * innovation, VCM): for v < nvec and t < nS_pad,
 *   dst[v*ld_dst + t] = src[v*ld_src + s_idx[t]]   if t < nS and s_idx[t] < n_src
 *                     = 0                          otherwise.
 * Elements have type t (2 or 4 bytes).  s_idx: nS uint32 column indices.
 * Out-of-range indices read nothing and yield 0.  nS_pad >= nS. */
FB_API fb_status fb_vcm_gather(const void *src, fb_dtype t, int nvec, int n_src, int ld_src,
                        const uint32_t *s_idx, int nS, int nS_pad, void *dst, int ld_dst,
                        void *stream);

/* fb_lut_build: LUT-BSF tables (FluxBin page, 2. Kernel innovation: alpha_c
 * fused into the table entries at build time), in the canonical layout
 *   lut[(k*(N/g) + q) * 2^g + p] = sum_{t<g} (bit t of p ? +1 : -1)
 *                                  * alpha_c[k*N + q*g + t] * x[q*g + t]
 * fp32, the product rounded to fp32 and the g terms added in order t = 0..g-1.
 * alpha_c may be NULL (all ones).  x: N elements of type t.  lut: K*N/g*2^g
 * floats, 4-byte aligned.  The GEMV builds its own tables in shared memory;
 * this call exposes the same step in global memory. */
FB_API fb_status fb_lut_build(const void *x, fb_dtype t, const float *alpha_c, int K, int N, int g,
                       float *lut, void *stream);

/* Weights of one M x N linear layer.  Host struct; every pointer in it is a
 * device pointer owned by the caller. */
typedef struct fb_weights {
    int M, N, K, g;              /* g: LUT group width (1, 2, 4 or 8), checked
                                    but NOT used by the GEMV calls: they always
                                    look up one weight byte (8 columns) per
                                    table access in 256-entry tables, each
                                    entry formed as the sum of the two
                                    4-column tables of its nibbles, so every
                                    g gives the same result bits.  g is the
                                    table width of fb_lut_build */
    const uint32_t *planes;      /* fb_pack(K, M, N) output, 16-byte aligned */
    const float *alpha_r;        /* [K][M] row scales */
    const float *alpha_c;        /* [K][N] column scales, or NULL for all ones */
    int nS, Ks;                  /* salient columns (0 = none) and their bases */
    const uint32_t *s_idx;       /* [nS] salient columns, strictly ascending, < N */
    const uint32_t *s_planes;    /* fb_pack(Ks, M, roundup(nS,32)) of the compact
                                    salient signs: column t is salient column
                                    s_idx[t]; bits past nS are ignored */
    const float *s_alpha_r;      /* [Ks][M] */
    const float *s_alpha_c;      /* [Ks][nS], compact (already gathered) */
} fb_weights;

/* fb_validate_weights: SYNCHRONOUS.  Checks sizes and alignment, then copies
 * s_idx to the host and checks it is strictly ascending and < N.  Returns
 * FB_OK, FB_ERR_INVALID_VALUE, FB_ERR_MISALIGNED or FB_ERR_CUDA.  fb_gemv
 * itself checks only what the host can see without copying; a salient index
 * >= N contributes 0 inside the kernel instead of reading out of bounds. */
FB_API fb_status fb_validate_weights(const fb_weights *W);

/* fb_gemv_workspace_bytes: bytes of workspace fb_gemv / fb_gemv_batched need
 * for W at this batch size.  The current kernels keep every partial sum in
 * on-chip shared memory of a thread-block cluster, so this returns 0 and the
 * ws / ws_bytes arguments may be NULL / 0 (they are kept for kernels that
 * need scratch; a non-NULL ws is ignored).  Host only. */
FB_API size_t fb_gemv_workspace_bytes(const fb_weights *W, int batch);

/* Launch flags. */
#define FB_GEMV_PDL 1u /* programmatic dependent launch: the kernel may start
                          before the previous kernel in the stream ends and
                          loads its weights (planes, scales, s_idx) early; it
                          reads x and writes y only after the previous kernel
                          has completed.  Only valid when no kernel still
                          running writes the weights. */
#define FB_GEMV_INDEPENDENT 2u /* with FB_GEMV_PDL only: the previous kernel in
                          the stream neither writes this call's x nor reads or
                          writes its y, so the whole GEMV may overlap it; the
                          kernel still completes only after the previous one,
                          so ordering with later work is unchanged. */

#define FB_GEMV_TEST_WAIT_TIMEOUT 0x80000000u /* for tests of the failure path
                          (batch-1 calls): no CTA sends its row partials, so
                          every CTA's bounded wait for them runs out (about
                          0.2 s); it then writes NaN into the rows it owns and
                          raises bit 0 of fb_device_errors.  The context stays
                          usable. */

/* fb_gemv: y[i] = sum_j W_hat[i][j] * x[j] for i < M (batch 1), fp32 out,
 * overwriting y (beta = 0).  x: N elements of type t (2- or 4-byte aligned);
 * y: M floats, 4-byte aligned, must not alias x; ws: see
 * fb_gemv_workspace_bytes.  flags: 0 or FB_GEMV_PDL [| FB_GEMV_INDEPENDENT],
 * optionally | FB_GEMV_TEST_WAIT_TIMEOUT; anything else is
 * FB_ERR_INVALID_VALUE.  Table entries and all sums are
 * fp32.  Deterministic: the same inputs give the same bits on every run.
 * The CTAs of a thread-block cluster exchange row partials through shared
 * memory; each waits for its share with a bound (about 0.2 s), and one that
 * gives up writes NaN into the rows it owns and raises bit 0 of
 * fb_device_errors. */
FB_API fb_status fb_gemv(const fb_weights *W, const void *x, fb_dtype t, float *y, void *ws,
                  size_t ws_bytes, unsigned flags, void *stream);

/* fb_gemv_batched: Y[b*ldy + i] = sum_j W_hat[i][j] * X[b*ldx + j] for
 * b < batch (1 <= batch <= 64), i < M.  ldx >= N, ldy >= M.  The tokens are
 * processed in passes (of 2 tokens for matrices of at most 32 MiB of packed
 * planes, whose passes share the weights through L2; else of up to 8):
 * within a pass, each weight word is read from memory once and applied to
 * every token's tables.  Per token the
 * result has the same properties as fb_gemv's (fp32 sums, deterministic,
 * same tolerance). */
FB_API fb_status fb_gemv_batched(const fb_weights *W, const void *X, fb_dtype t, int batch, int ldx,
                          float *Y, int ldy, void *ws, size_t ws_bytes, unsigned flags,
                          void *stream);

/* fb_gemv_grouped: one launch for n (1 <= n <= 4) weight matrices that read
 * the same x -- the q, k, v projections of a decoder layer, or gate and up
 * -- y[m][i] = sum_j W_hat_m[i][j] * x[j] for i < W[m]->M.  The matrices must
 * share one format: N, K, g, nS and Ks (their data, M and salient columns
 * are their own); otherwise FB_ERR_INVALID_VALUE.  W: n host pointers to
 * fb_weights; y: n device pointers, y[m] holding W[m]->M floats (4-byte
 * aligned, not aliasing x or one another).  x and flags as for fb_gemv.  The
 * result of each matrix is the one fb_gemv gives for it with the same plan:
 * deterministic, within the same tolerance.  FB_ERR_UNSUPPORTED if the
 * matrices together need more than 65535 row blocks. */
FB_API fb_status fb_gemv_grouped(const fb_weights *const *W, int n, const void *x, fb_dtype t, float *const *y,
                                 unsigned flags, void *stream);

/* fb_gemv_group_scales: y = W_hat x (batch 1) for the group-wise row-scale
 * format, one row scale per group of G consecutive input columns:
 *   W_hat[i][j] = sum_k alpha_r[k][j / G][i] * alpha_c[k][j] * B^(k)[i][j]
 *                 + the salient term, whose row scales stay per row.
 * The FluxBin page names this variant only through its "2b-s16-g128"
 * setting (Experimental results, the accuracy paragraph) and does not define
 * it; G = 128 is that setting's reading.  W is an ordinary fb_weights except
 * that W->alpha_r holds K * (N / G) row-scale vectors of M floats, laid out
 * [K][N/G][M] (group g of base k at alpha_r + (k * N/G + g) * M).  G = 128,
 * N, or a multiple of 256 dividing N, else FB_ERR_INVALID_VALUE; G = N is the
 * ordinary format (the same result bits as fb_gemv).  x, t, y, flags and the result's properties (fp32 sums,
 * deterministic, tolerance) as for fb_gemv.  With G = 128 every 256-column
 * panel is looked up once per half (the other half's columns contributing
 * exact zeros), so a call costs about twice the table work of fb_gemv. */
FB_API fb_status fb_gemv_group_scales(const fb_weights *W, int G, const void *x, fb_dtype t, float *y,
                                      unsigned flags, void *stream);

/* fb_gemv_launch_plan: diagnostic, host only.  The launch shape fb_gemv /
 * fb_gemv_batched use for W at this batch size and these flags (calls flagged
 * FB_GEMV_INDEPENDENT get a throughput plan, others a latency plan) on a GPU
 * with `sms` SMs:
 * out[0] = CTAs per thread-block cluster, out[1] = chunks of 32 rows per row
 * block, out[2] = row blocks, out[3] = warps per CTA, out[4] = dynamic shared
 * memory bytes per CTA, out[5] = virtual panels (256-column panels x bases).
 * out must hold 6 ints.  Returns FB_OK, or FB_ERR_INVALID_VALUE for invalid
 * weights, batch, sms or flags.  Tuning aid: the environment variable
 * FB_PLAN="C,cpb[,n]", read when a plan is first made for a shape, forces the
 * cluster size and row block (clamped to what the matrix and shared memory
 * allow); the optional n is, for batch-1 calls, 16 to use 16-warp CTAs (one
 * per SM) and, for batched calls, the tokens per pass (even, at most 16; a
 * forced plan uses the kernel variant with two CTAs per SM). */
FB_API fb_status fb_gemv_launch_plan(const fb_weights *W, int batch, unsigned flags, int sms, int *out);

/* fb_device_errors: synchronises the current device, then stores in *flags
 * the error bits GEMV kernels have raised since the last clear (bit 0: a CTA
 * gave up its bounded wait for the row partials of its cluster; the rows it
 * owns were written as NaN), and clears them when clear != 0.  Returns
 * FB_ERR_INVALID_VALUE for a null flags, FB_ERR_CUDA if the device reports an
 * error, else FB_OK. */
FB_API fb_status fb_device_errors(unsigned int *flags, int clear);

/* ---- The fitter: a dense matrix in, the decomposition's factors out ------
 * The step before the GEMV.  The FluxBin page (Methodology, 1. Algorithm
 * innovation: the decoupled row-column binary decomposition and the
 * Hessian-guided saliency-aware hybrid bases) defines the factors of W_hat
 * but no fitting procedure; these two calls implement its plainest reading.
 * Both are asynchronous on `stream`; all pointers are device pointers owned
 * by the caller; sums are accumulated in fp64 in a fixed order, so results
 * are reproducible; argument errors return before anything is enqueued.
 *
 * fb_fit_saliency: the diagonal-Hessian proxy for choosing the salient
 * columns.  W [M][ldw] and calibration activations X [T][ldx], fp32
 * row-major (the first N columns used):
 *   score[j] = (sum_t X[t][j]^2) * (sum_i W[i][j]^2)          j < N, fp32 out
 *   s_idx    = the nS columns of largest score (equal scores: the lower
 *              column first), in ascending order              uint32 [nS] out
 * 1 <= N <= 2^20 (the selection runs in one block: a radix select of the
 * score of rank nS - 1, then one ordered pass placing the selected columns),
 * 0 <= nS <= N, ldw, ldx >= N.  s_idx may be NULL when nS = 0.
 * Returns FB_ERR_INVALID_VALUE / FB_ERR_MISALIGNED (4-byte alignment) for bad
 * arguments, FB_ERR_CUDA if a launch fails. */
FB_API fb_status fb_fit_saliency(const float *W, int M, int N, int ldw, const float *X, int T, int ldx, int nS,
                                 float *score, uint32_t *s_idx, void *stream);

/* fb_fit_base: one greedy base of the decomposition on the residual R
 * [M][ldr] fp32 (updated in place):
 *   signs[i][j] = R[i][j] >= 0 ? +1 : -1 (negative zero gives +1)   int8 [M][lds]
 *   (alpha_r, alpha_c) = the rank-one least-squares fit of |R|, after
 *     `sweeps` alternating sweeps from alpha_c = 1:
 *       alpha_r = |R| alpha_c / ||alpha_c||^2, then alpha_c = |R|^T alpha_r /
 *       ||alpha_r||^2 (a zero norm gives zero scales)     fp32 [M], [N] out
 *   R[i][j] -= (alpha_r[i] * alpha_c[j]) * signs[i][j]   (fp32, the product
 *     rounded once, then the update)
 * Called K times from R = W this yields the global bases; called on the
 * residual's salient columns (gathered with fb_vcm_gather, zero padding
 * included) it yields the salient bases.  1 <= sweeps <= 1000, ldr, lds >= N,
 * M <= 2^24, N <= 2^20.  Errors as fb_fit_saliency. */
FB_API fb_status fb_fit_base(float *R, int M, int N, int ldr, int sweeps, int8_t *signs, int lds, float *alpha_r,
                             float *alpha_c, void *stream);

/* Human-readable name of a status code (static string). */
FB_API const char *fb_status_string(fb_status s);

/* FLUXBIN_ABI_VERSION of the loaded library. */
FB_API int fb_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FLUXBIN_H_ */
