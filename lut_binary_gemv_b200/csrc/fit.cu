// fit.cu -- the fitter: a dense matrix W in, the decomposition's factors out
// (the step before the GEMV).  The FluxBin page (Methodology, 1. Algorithm
// innovation: the decoupled row-column binary decomposition, and the
// Hessian-guided saliency-aware hybrid bases) defines the factors but prints
// no fitting procedure; this file implements its plainest reading:
//
//   saliency  score_j = (sum_t X[t][j]^2) * (sum_i W[i][j]^2): the diagonal of
//             the layer Hessian X^T X times the column's weight energy; the
//             salient set is the nS columns of largest score (equal scores:
//             lower column first), listed ascending;
//   one base  B = sign(R) (R >= 0 gives +1); alpha_r, alpha_c = the rank-one
//             least-squares fit of |R|, by alternating sweeps from alpha_c = 1
//             (alpha_r = |R| alpha_c / ||alpha_c||^2, then alpha_c = |R|^T
//             alpha_r / ||alpha_r||^2; a zero norm gives zero scales); then
//             R -= (alpha_r alpha_c^T) (.) B.
//
// Every sum is accumulated in fp64 in a fixed order (results do not depend
// on scheduling); scales and the residual are stored as fp32.  All of it is
// bandwidth-bound streaming over R, with no tensor-core work.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fb_internal.cuh"

namespace cg = cooperative_groups;

namespace fb {
namespace {

constexpr int kFitMaxN = 65536;        // salient selection runs in one block, a bit per column
constexpr int kFitMaxSweeps = 1000;
constexpr int kSelectThreads = 1024;
constexpr int kColUnroll = 16;   // rows a lane loads before adding them (memory requests in flight)
constexpr int kRowUnroll = 8;    // columns a lane loads before adding them

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sum of squares of n values, by a whole block of 256 threads in a fixed
// order (every block that calls it on the same data gets the same bits).
__device__ double block_norm2(const float *v, int n, double *red) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    double q = 0.0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const double a = v[i];
        q = fma(a, a, q);
    }
    q = warp_sum(q);
    if (lane == 0) red[w] = q;
    __syncthreads();
    double t = 0.0;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) t += red[k];
    __syncthreads();
    return t;
}

// Column passes split the rows over a cluster of kColSplit CTAs: CTA r of
// the cluster sums row slice r of its 32 columns (8 warps, warp w taking rows
// w, w + 8, ... of the slice, the 8 partials added in warp order) and sends
// its 32 sums to rank 0's shared memory; rank 0 adds the kColSplit slices in
// rank order.  A fixed order throughout, so results do not depend on
// scheduling, and no scratch memory.
constexpr int kColSplit = 8;

// Sum over row slice `rank` of f(A[i][j]) * w(i) for this lane's column j, in
// the order described above; returns this CTA's 32 partials' rank-0 total in
// lane order on rank 0 (other ranks return 0).
template <typename Term>
__device__ double cluster_column_sum(int rows, int j, bool valid, Term term) {
    __shared__ double part[8][32];
    __shared__ double inbox[kColSplit][32];
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int rs = (rows + kColSplit - 1) / kColSplit, i0 = rank * rs, i1 = min(rows, i0 + rs);
    double s = 0.0;
    if (valid) {
        int i = i0 + w;
        for (; i + 8 * (kColUnroll - 1) < i1; i += 8 * kColUnroll) {   // same order, loads issued first
            double v[kColUnroll];
#pragma unroll
            for (int u = 0; u < kColUnroll; ++u) v[u] = term.load(i + 8 * u, j);
#pragma unroll
            for (int u = 0; u < kColUnroll; ++u) s = term.add(s, v[u], i + 8 * u);
        }
        for (; i < i1; i += 8) s = term.add(s, term.load(i, j), i);
    }
    part[w][lane] = s;
    __syncthreads();
    if (w == 0) {
        double t = part[0][lane];
        for (int q = 1; q < 8; ++q) t += part[q][lane];
        cl.map_shared_rank(&inbox[0][0], 0)[rank * 32 + lane] = t;
    }
    cl.sync();
    double total = 0.0;
    if (rank == 0 && w == 0) {
        total = inbox[0][lane];
        for (int q = 1; q < kColSplit; ++q) total += inbox[q][lane];
    }
    return total;
}

struct SumSquares {
    const float *A;
    int ld;
    __device__ double load(int i, int j) const { return (double)A[(size_t)i * ld + j]; }
    __device__ double add(double s, double v, int) const { return fma(v, v, s); }
};

// out[j] = sum_i A[i][j]^2 (multiply = 0), or out[j] *= that sum (multiply =
// 1).  grid.x = kColSplit * (column blocks of 32).
__global__ void __cluster_dims__(kColSplit, 1, 1) __launch_bounds__(256)
    colsumsq_kernel(const float *A, int rows, int cols, int ld, float *out, int multiply) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int j = (int)(blockIdx.x / kColSplit) * 32 + lane;
    const double t = cluster_column_sum(rows, j, j < cols, SumSquares{A, ld});
    if (cg::this_cluster().block_rank() == 0 && w == 0 && j < cols)
        out[j] = multiply ? (float)((double)out[j] * t) : (float)t;
}

// Order-preserving key of a float: a larger float has a larger key, and every
// bit pattern (NaN included) has its own place, so ranks below form a total
// order whatever the scores hold.
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The nS columns of largest score, ascending, in one block: every column's
// rank under (score descending, column ascending) is counted against all
// scores (staged through shared memory a tile at a time); rank < nS sets the
// column's bit; a prefix count over the bit words places each selected
// column.  Ranks are a permutation, so exactly nS bits are set.
__global__ void __launch_bounds__(kSelectThreads) select_kernel(const float *score, int N, int nS, uint32_t *s_idx) {
    extern __shared__ uint32_t sm[];
    const int nw = (N + 31) / 32;
    uint32_t *flags = sm, *prefix = sm + nw;
    uint32_t *tile = prefix + nw;
    for (int q = threadIdx.x; q < nw; q += blockDim.x) flags[q] = 0;
    for (int j0 = 0; j0 < N; j0 += blockDim.x) {
        const int j = j0 + (int)threadIdx.x;
        const uint32_t kj = j < N ? order_key(score[j]) : 0u;
        int rank = 0;
        for (int t0 = 0; t0 < N; t0 += blockDim.x) {
            __syncthreads();
            if (t0 + (int)threadIdx.x < N) tile[threadIdx.x] = order_key(score[t0 + threadIdx.x]);
            __syncthreads();
            const int n = min((int)blockDim.x, N - t0);
            for (int u = 0; u < n; ++u) {
                const uint32_t ku = tile[u];
                rank += (ku > kj) || (ku == kj && t0 + u < j);
            }
        }
        if (j < N && rank < nS) atomicOr(&flags[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t run = 0;
        for (int q = 0; q < nw; ++q) {
            prefix[q] = run;
            run += __popc(flags[q]);
        }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < N; j += blockDim.x) {
        const uint32_t f = flags[j >> 5];
        const uint32_t b = (uint32_t)j & 31u;
        const uint32_t pos = prefix[j >> 5] + __popc(f & ((1u << b) - 1u));
        if (((f >> b) & 1u) && pos < (uint32_t)nS) s_idx[pos] = (uint32_t)j;
    }
}

// alpha_r[i] = sum_j |R[i][j]| alpha_c[j] / ||alpha_c||^2 (alpha_c = 1 when
// ones != 0).  One warp per row, lanes striding the columns.
__global__ void __launch_bounds__(256) fit_rows_kernel(const float *R, int M, int N, int ld, const float *ac,
                                                        int ones, float *ar) {
    __shared__ double red[8];
    const double nc = ones ? (double)N : block_norm2(ac, N, red);
    const int lane = threadIdx.x & 31, i = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (i >= M) return;
    const float *row = R + (size_t)i * ld;
    double s = 0.0;
    int j = lane;
    for (; j + 32 * (kRowUnroll - 1) < N; j += 32 * kRowUnroll) {   // same order, loads issued first
        float v[kRowUnroll], c[kRowUnroll];
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
            v[u] = row[j + 32 * u];
            c[u] = ones ? 1.0f : ac[j + 32 * u];
        }
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) s = fma((double)fabsf(v[u]), (double)c[u], s);
    }
    for (; j < N; j += 32) s = fma((double)fabsf(row[j]), ones ? 1.0 : (double)ac[j], s);
    s = warp_sum(s);
    if (lane == 0) ar[i] = nc > 0.0 ? (float)(s / nc) : 0.0f;
}

struct AbsTimesRowScale {
    const float *R;
    int ld;
    const float *ar;
    __device__ double load(int i, int j) const { return (double)fabsf(R[(size_t)i * ld + j]); }
    __device__ double add(double s, double v, int i) const { return fma(v, (double)ar[i], s); }
};

// alpha_c[j] = sum_i |R[i][j]| alpha_r[i] / ||alpha_r||^2, the rows split over
// the cluster as above; rank 0 also forms ||alpha_r||^2 (block_norm2 order).
__global__ void __cluster_dims__(kColSplit, 1, 1) __launch_bounds__(256)
    fit_cols_kernel(const float *R, int M, int N, int ld, const float *ar, float *ac) {
    __shared__ double red[8];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int j = (int)(blockIdx.x / kColSplit) * 32 + lane;
    const double t = cluster_column_sum(M, j, j < N, AbsTimesRowScale{R, ld, ar});
    if (cg::this_cluster().block_rank() != 0) return;
    const double nr = block_norm2(ar, M, red);
    if (w == 0 && j < N) ac[j] = nr > 0.0 ? (float)(t / nr) : 0.0f;
}

// signs = sign(R) (R >= 0 gives +1, -0 included); R -= (alpha_r[i] alpha_c[j])
// * sign, in fp32 with one rounding for the product and one for the update.
__global__ void __launch_bounds__(256) fit_update_kernel(float *R, int M, int N, int ld, const float *ar,
                                                          const float *ac, int8_t *signs, int lds) {
    const int j = blockIdx.x * 256 + threadIdx.x;
    if (j >= N) return;
    const float c = ac[j];
    for (int i = blockIdx.y; i < M; i += gridDim.y) {
        float *p = R + (size_t)i * ld + j;
        const float r = *p;
        const bool pos = r >= 0.0f;
        const float s = __fmul_rn(ar[i], c);
        *p = pos ? __fsub_rn(r, s) : __fadd_rn(r, s);
        signs[(size_t)i * lds + j] = pos ? (int8_t)1 : (int8_t)-1;
    }
}

}  // namespace
}  // namespace fb

using namespace fb;

extern "C" fb_status fb_fit_saliency(const float *W, int M, int N, int ldw, const float *X, int T, int ldx, int nS,
                                     float *score, uint32_t *s_idx, void *stream) {
    if (M < 1 || M > kMaxM || N < 1 || N > kFitMaxN || T < 1 || T > kMaxM || ldw < N || ldx < N || nS < 0 ||
        nS > N || !W || !X || !score || (nS > 0 && !s_idx))
        return FB_ERR_INVALID_VALUE;
    if (!aligned(W, 4) || !aligned(X, 4) || !aligned(score, 4) || (s_idx && !aligned(s_idx, 4)))
        return FB_ERR_MISALIGNED;
    cudaStream_t s = as_stream(stream);
    const dim3 grid(ceil_div(N, 32) * kColSplit), block(256);
    cudaError_t e = launch(colsumsq_kernel, grid, block, 0, s, false, W, M, N, ldw, score, 0);
    if (e == cudaSuccess) e = launch(colsumsq_kernel, grid, block, 0, s, false, X, T, N, ldx, score, 1);
    if (e == cudaSuccess && nS > 0) {
        const size_t smem = (size_t)2 * ceil_div(N, 32) * 4 + (size_t)kSelectThreads * 4;
        e = launch(select_kernel, dim3(1), dim3(kSelectThreads), smem, s, false, (const float *)score, N, nS, s_idx);
    }
    return status_of(e);
}

extern "C" fb_status fb_fit_base(float *R, int M, int N, int ldr, int sweeps, int8_t *signs, int lds,
                                 float *alpha_r, float *alpha_c, void *stream) {
    if (M < 1 || M > kMaxM || N < 1 || N > kMaxN || ldr < N || lds < N || sweeps < 1 || sweeps > kFitMaxSweeps ||
        !R || !signs || !alpha_r || !alpha_c)
        return FB_ERR_INVALID_VALUE;
    if (!aligned(R, 4) || !aligned(alpha_r, 4) || !aligned(alpha_c, 4)) return FB_ERR_MISALIGNED;
    cudaStream_t s = as_stream(stream);
    const dim3 block(256), rows_grid(ceil_div(M, 8)), cols_grid(ceil_div(N, 32) * kColSplit);
    cudaError_t e = cudaSuccess;
    for (int it = 0; it < sweeps && e == cudaSuccess; ++it) {
        e = launch(fit_rows_kernel, rows_grid, block, 0, s, false, (const float *)R, M, N, ldr,
                   (const float *)alpha_c, it == 0 ? 1 : 0, alpha_r);
        if (e == cudaSuccess)
            e = launch(fit_cols_kernel, cols_grid, block, 0, s, false, (const float *)R, M, N, ldr,
                       (const float *)alpha_r, alpha_c);
    }
    if (e == cudaSuccess) {
        const dim3 ugrid(ceil_div(N, 256), M < 8192 ? M : 8192);
        e = launch(fit_update_kernel, ugrid, block, 0, s, false, R, M, N, ldr, (const float *)alpha_r,
                   (const float *)alpha_c, signs, lds);
    }
    return status_of(e);
}
