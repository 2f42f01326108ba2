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

#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "fb_internal.cuh"

namespace cg = cooperative_groups;

namespace fb {
namespace {

constexpr int kFitMaxSweeps = 1000;
constexpr int kSelectThreads = 1024;
constexpr int kRowUnroll = 8;     // float4s a lane loads per row before adding them (row pass)
constexpr int kColSplit = 16;     // CTAs of a column-pass cluster: slices of the rows
constexpr int kColTile = 128;     // columns of a column-pass CTA: a float4 per lane
constexpr int kColUnroll = 8;     // rows a warp loads before adding them (column passes)

// Launched with programmatic dependent launch, every fitter kernel lets the
// next one in the stream start at once and then waits for its predecessor
// before touching memory: the next kernel's CTAs are resident when this one
// ends (no launch gap), and no read or write of this kernel can overtake the
// previous one's.
__device__ __forceinline__ void follow_predecessor() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sum of squares of n values, by a whole block (up to 32 warps) in a fixed
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

__device__ __forceinline__ bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }

// Four consecutive values A[off .. off + valid - 1] (the rest 0): one 16-byte
// load when the row is 16-byte aligned and all four are in range.
__device__ __forceinline__ float4 load4(const float *A, size_t off, int valid, bool vec) {
    if (vec && valid >= 4) return __ldg(reinterpret_cast<const float4 *>(A + off));
    float4 r = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (valid > 0) r.x = __ldg(A + off);
    if (valid > 1) r.y = __ldg(A + off + 1);
    if (valid > 2) r.z = __ldg(A + off + 2);
    if (valid > 3) r.w = __ldg(A + off + 3);
    return r;
}

// Column passes: a CTA of NW warps covers kColTile columns (lane l: columns
// c0 + 4l .. c0 + 4l + 3, read as one float4 per row, so a warp reads 512
// contiguous bytes of a row), and the rows are split over a cluster of
// kColSplit CTAs.  CTA r sums row slice r, warp w taking rows w, w + NW, ...
// of it in increasing order; the NW warps' partials are added in warp order,
// then rank 0 adds the kColSplit slices in rank order (distributed shared
// memory).  A fixed order throughout, so results do not depend on
// scheduling, and no scratch memory.  Returns the column totals on rank 0,
// threads 0 .. kColTile - 1 (thread t: column c0 + t); 0 elsewhere.
template <int NW, typename Term>
__device__ double cluster_column_sums(const float *A, int rows, int cols, int ld, int c0, Term term) {
    __shared__ double part[NW][kColTile];
    __shared__ double inbox[kColSplit][kColTile];
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int rs = (rows + kColSplit - 1) / kColSplit, i0 = rank * rs, i1 = min(rows, i0 + rs);
    const int c = c0 + 4 * lane, valid = max(0, min(4, cols - c));
    const bool vec = (ld % 4 == 0) && aligned16(A);
    double s[4] = {0.0, 0.0, 0.0, 0.0};
    if (valid > 0) {
        int i = i0 + w;
        for (; i + NW * (kColUnroll - 1) < i1; i += NW * kColUnroll) {   // same order, loads issued first
            float4 v[kColUnroll];
#pragma unroll
            for (int u = 0; u < kColUnroll; ++u) v[u] = load4(A, (size_t)(i + NW * u) * ld + c, valid, vec);
#pragma unroll
            for (int u = 0; u < kColUnroll; ++u) term.add(s, v[u], i + NW * u);
        }
        for (; i < i1; i += NW) term.add(s, load4(A, (size_t)i * ld + c, valid, vec), i);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) part[w][4 * lane + k] = s[k];
    __syncthreads();
    if (threadIdx.x < kColTile) {
        double t = part[0][threadIdx.x];
        for (int q = 1; q < NW; ++q) t += part[q][threadIdx.x];
        cl.map_shared_rank(&inbox[0][0], 0)[rank * kColTile + threadIdx.x] = t;
    }
    cl.sync();
    double total = 0.0;
    if (rank == 0 && threadIdx.x < kColTile) {
        total = inbox[0][threadIdx.x];
        for (int q = 1; q < kColSplit; ++q) total += inbox[q][threadIdx.x];
    }
    return total;
}

struct SumSquares {
    __device__ void add(double (&s)[4], float4 v, int) const {
        s[0] = fma((double)v.x, (double)v.x, s[0]);
        s[1] = fma((double)v.y, (double)v.y, s[1]);
        s[2] = fma((double)v.z, (double)v.z, s[2]);
        s[3] = fma((double)v.w, (double)v.w, s[3]);
    }
};

// out[j] = sum_i A[i][j]^2 (multiply = 0), or out[j] *= that sum (multiply =
// 1).  grid.x = kColSplit * (column tiles), clusters of kColSplit.
template <int NW>
__global__ void __launch_bounds__(NW * 32)
    colsumsq_kernel(const float *A, int rows, int cols, int ld, float *out, int multiply) {
    follow_predecessor();
    const int c0 = (int)(blockIdx.x / kColSplit) * kColTile;
    const double t = cluster_column_sums<NW>(A, rows, cols, ld, c0, SumSquares{});
    const int j = c0 + (int)threadIdx.x;
    if (cg::this_cluster().block_rank() == 0 && threadIdx.x < kColTile && j < cols)
        out[j] = multiply ? (float)((double)out[j] * t) : (float)t;
}

// Order-preserving key of a float: a larger float has a larger key, and every
// bit pattern (NaN included) has its own place, so the order below is total
// whatever the scores hold.
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive count of `flag` over the threads of the block below this one (in
// thread order), and the block's total; every thread must call it.
__device__ uint32_t block_exclusive_count(bool flag, uint32_t *warp_cnt, uint32_t &total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const uint32_t b = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) warp_cnt[w] = __popc(b);
    __syncthreads();
    uint32_t before = 0, all = 0;
    for (int q = 0; q < nw; ++q) {
        const uint32_t c = warp_cnt[q];
        before += q < w ? c : 0u;
        all += c;
    }
    __syncthreads();   // warp_cnt is reused by the next call
    total = all;
    return before + __popc(b & ((1u << lane) - 1u));
}

// The nS columns of largest score (equal scores: lower column first),
// ascending, in one block.  The order is (key descending, column ascending)
// with key = order_key(score).  A radix select finds the key T of rank nS - 1
// eight bits at a time from the top (a histogram of the next digit among the
// keys that match the digits found so far; the digit is where the count from
// the top reaches the ranks still wanted), and how many columns of key T
// belong to the set.  A column is selected if its key is above T, or equal to
// T and among the first that many such columns; a running count over the
// columns in order gives each selected column its place.
__global__ void __launch_bounds__(kSelectThreads) select_kernel(const float *score, int N, int nS, uint32_t *s_idx) {
    __shared__ uint32_t hist[256];
    __shared__ uint32_t warp_cnt[32];
    __shared__ uint32_t s_prefix, s_need;
    follow_predecessor();
    const int tid = threadIdx.x;
    uint32_t prefix = 0, mask = 0, need = (uint32_t)nS;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int q = tid; q < 256; q += blockDim.x) hist[q] = 0;
        __syncthreads();
        for (int j = tid; j < N; j += blockDim.x) {
            const uint32_t k = order_key(score[j]);
            if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid == 0) {
            uint32_t above = 0;
            int b = 255;
            for (; b > 0 && above + hist[b] < need; --b) above += hist[b];
            s_prefix = prefix | ((uint32_t)b << shift);
            s_need = need - above;
        }
        __syncthreads();
        prefix = s_prefix;
        need = s_need;
        mask |= 255u << shift;
    }
    uint32_t ties_before = 0, placed = 0;
    for (int j0 = 0; j0 < N; j0 += blockDim.x) {
        const int j = j0 + tid;
        const uint32_t k = j < N ? order_key(score[j]) : 0u;
        const bool tie = j < N && k == prefix, above = j < N && k > prefix;
        uint32_t n_ties, n_sel;
        const uint32_t tie_rank = ties_before + block_exclusive_count(tie, warp_cnt, n_ties);
        const bool sel = above || (tie && tie_rank < need);
        const uint32_t pos = placed + block_exclusive_count(sel, warp_cnt, n_sel);
        if (sel && pos < (uint32_t)nS) s_idx[pos] = (uint32_t)j;
        ties_before += n_ties;
        placed += n_sel;
    }
}

// alpha_r[i] = sum_j |R[i][j]| alpha_c[j] / ||alpha_c||^2 (alpha_c = 1 when
// ones != 0).  One warp per two consecutive rows (each alpha_c load serves
// both): lane l adds columns 4l .. 4l + 3, then 128 further on, and so on
// (float4 loads when the rows are 16-byte aligned), then each row's lane sums
// are added by a butterfly.  grid.x = ceil(M / 16).
__global__ void __launch_bounds__(256) fit_rows_kernel(const float *R, int M, int N, int ld, const float *ac,
                                                        int ones, float *ar) {
    __shared__ double red[32];
    follow_predecessor();
    const double nc = ones ? (double)N : block_norm2(ac, N, red);
    const int lane = threadIdx.x & 31, i = 2 * (blockIdx.x * 8 + (threadIdx.x >> 5));
    if (i >= M) return;
    const bool two = i + 1 < M;
    const float *ra = R + (size_t)i * ld, *rb = two ? ra + ld : ra;
    const bool vec = aligned16(ra) && aligned16(rb) && (ones || aligned16(ac));
    auto add = [&](double s, float4 v, float4 c) {
        s = fma((double)fabsf(v.x), (double)c.x, s);
        s = fma((double)fabsf(v.y), (double)c.y, s);
        s = fma((double)fabsf(v.z), (double)c.z, s);
        return fma((double)fabsf(v.w), (double)c.w, s);
    };
    const float4 one4 = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
    double sa = 0.0, sb = 0.0;
    int j = 4 * lane;
    for (; j + 128 * (kRowUnroll - 1) + 3 < N; j += 128 * kRowUnroll) {   // same order, loads issued first
        float4 va[kRowUnroll], vb[kRowUnroll], c[kRowUnroll];
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
            va[u] = load4(ra, j + 128 * u, 4, vec);
            vb[u] = load4(rb, j + 128 * u, 4, vec);
            c[u] = ones ? one4 : load4(ac, j + 128 * u, 4, vec);
        }
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
            sa = add(sa, va[u], c[u]);
            sb = add(sb, vb[u], c[u]);
        }
    }
    for (; j < N; j += 128) {
        const int valid = min(4, N - j);
        const float4 c = ones ? one4 : load4(ac, j, valid, vec);
        sa = add(sa, load4(ra, j, valid, vec), c);
        sb = add(sb, load4(rb, j, valid, vec), c);
    }
    sa = warp_sum(sa);
    sb = warp_sum(sb);
    if (lane == 0) {
        ar[i] = nc > 0.0 ? (float)(sa / nc) : 0.0f;
        if (two) ar[i + 1] = nc > 0.0 ? (float)(sb / nc) : 0.0f;
    }
}

struct AbsTimesRowScale {
    const float *ar;
    __device__ void add(double (&s)[4], float4 v, int i) const {
        const double r = (double)__ldg(ar + i);
        s[0] = fma((double)fabsf(v.x), r, s[0]);
        s[1] = fma((double)fabsf(v.y), r, s[1]);
        s[2] = fma((double)fabsf(v.z), r, s[2]);
        s[3] = fma((double)fabsf(v.w), r, s[3]);
    }
};

// alpha_c[j] = sum_i |R[i][j]| alpha_r[i] / ||alpha_r||^2, the rows split over
// the cluster as above; rank 0 also forms ||alpha_r||^2 (block_norm2 order).
template <int NW>
__global__ void __launch_bounds__(NW * 32)
    fit_cols_kernel(const float *R, int M, int N, int ld, const float *ar, float *ac) {
    __shared__ double red[32];
    follow_predecessor();
    const int c0 = (int)(blockIdx.x / kColSplit) * kColTile;
    const double t = cluster_column_sums<NW>(R, M, N, ld, c0, AbsTimesRowScale{ar});
    if (cg::this_cluster().block_rank() != 0) return;
    const double nr = block_norm2(ar, M, red);
    const int j = c0 + (int)threadIdx.x;
    if (threadIdx.x < kColTile && j < N) ac[j] = nr > 0.0 ? (float)(t / nr) : 0.0f;
}

// signs = sign(R) (R >= 0 gives +1, -0 included); R -= (alpha_r[i] alpha_c[j])
// * sign, in fp32 with one rounding for the product and one for the update.
// A thread takes four consecutive columns (one float4 and one 4-byte sign
// store when aligned) of rows blockIdx.y * rpb + threadIdx.x / tpr, stepping
// by gridDim.y * rpb; tpr threads cover a row (rpb rows per block).
__global__ void __launch_bounds__(256) fit_update_kernel(float *R, int M, int N, int ld, const float *ar,
                                                          const float *ac, int8_t *signs, int lds, int tpr) {
    follow_predecessor();
    const int rpb = blockDim.x / tpr;
    const int j = 4 * (blockIdx.x * tpr + (int)threadIdx.x % tpr);
    if (j >= N || (int)threadIdx.x >= rpb * tpr) return;
    const int valid = min(4, N - j);
    const bool vec = valid == 4 && ld % 4 == 0 && aligned16(R) && lds % 4 == 0 && ((uintptr_t)signs & 3) == 0;
    float c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) c[k] = k < valid ? ac[j + k] : 0.0f;
    for (int i = blockIdx.y * rpb + (int)threadIdx.x / tpr; i < M; i += gridDim.y * rpb) {
        float *p = R + (size_t)i * ld + j;
        const float a = ar[i];
        float r[4];
        if (vec) {
            const float4 v = *reinterpret_cast<const float4 *>(p);
            r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) r[k] = k < valid ? p[k] : 0.0f;
        }
        uint32_t sg = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const bool pos = r[k] >= 0.0f;
            const float t = __fmul_rn(a, c[k]);
            r[k] = pos ? __fsub_rn(r[k], t) : __fadd_rn(r[k], t);
            sg |= (uint32_t)(uint8_t)(pos ? 1 : -1) << (8 * k);
        }
        int8_t *q = signs + (size_t)i * lds + j;
        if (vec) {
            *reinterpret_cast<float4 *>(p) = make_float4(r[0], r[1], r[2], r[3]);
            *reinterpret_cast<uint32_t *>(q) = sg;
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < valid) {
                    p[k] = r[k];
                    q[k] = (int8_t)(uint8_t)(sg >> (8 * k));
                }
        }
    }
}

// Launch with clusters of kColSplit CTAs (beyond the portable size of 8: the
// kernel's attribute is raised once per kernel and device; the record is
// shared by every kernel of one signature, hence keyed by kernel), with
// programmatic dependent launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster(void (*kernel)(KArgs...), int grid, int block, cudaStream_t stream, Args &&...args) {
    static std::mutex lock;
    static std::vector<std::pair<const void *, int>> done;   // (kernel, device) pairs already raised
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> g(lock);
        const std::pair<const void *, int> key((const void *)kernel, dev);
        if (std::find(done.begin(), done.end(), key) == done.end()) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
            done.push_back(key);
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kColSplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Column passes over `cols` columns: 8-warp CTAs, or 16-warp CTAs when the
// column tiles alone would leave most SMs idle (the rows then supply the
// parallelism).
bool narrow_columns(int cols) { return (long)ceil_div(cols, kColTile) * kColSplit < 2L * sm_count(); }

cudaError_t column_sumsq(const float *A, int rows, int cols, int ld, float *out, int multiply, cudaStream_t s) {
    const int grid = ceil_div(cols, kColTile) * kColSplit;
    return narrow_columns(cols) ? launch_cluster(colsumsq_kernel<16>, grid, 16 * 32, s, A, rows, cols, ld, out, multiply)
                                : launch_cluster(colsumsq_kernel<8>, grid, 8 * 32, s, A, rows, cols, ld, out, multiply);
}

}  // namespace
}  // namespace fb

using namespace fb;

extern "C" fb_status fb_fit_saliency(const float *W, int M, int N, int ldw, const float *X, int T, int ldx, int nS,
                                     float *score, uint32_t *s_idx, void *stream) {
    if (M < 1 || M > kMaxM || N < 1 || N > kMaxN || T < 1 || T > kMaxM || ldw < N || ldx < N || nS < 0 || nS > N ||
        !W || !X || !score || (nS > 0 && !s_idx))
        return FB_ERR_INVALID_VALUE;
    if (!aligned(W, 4) || !aligned(X, 4) || !aligned(score, 4) || (s_idx && !aligned(s_idx, 4)))
        return FB_ERR_MISALIGNED;
    cudaStream_t s = as_stream(stream);
    cudaError_t e = column_sumsq(W, M, N, ldw, score, 0, s);
    if (e == cudaSuccess) e = column_sumsq(X, T, N, ldx, score, 1, s);
    if (e == cudaSuccess && nS > 0)
        e = launch(select_kernel, dim3(1), dim3(kSelectThreads), 0, s, true, (const float *)score, N, nS, s_idx);
    return status_of(e);
}

extern "C" fb_status fb_fit_base(float *R, int M, int N, int ldr, int sweeps, int8_t *signs, int lds,
                                 float *alpha_r, float *alpha_c, void *stream) {
    if (M < 1 || M > kMaxM || N < 1 || N > kMaxN || ldr < N || lds < N || sweeps < 1 || sweeps > kFitMaxSweeps ||
        !R || !signs || !alpha_r || !alpha_c)
        return FB_ERR_INVALID_VALUE;
    if (!aligned(R, 4) || !aligned(alpha_r, 4) || !aligned(alpha_c, 4)) return FB_ERR_MISALIGNED;
    cudaStream_t s = as_stream(stream);
    const int cols_grid = ceil_div(N, kColTile) * kColSplit;
    const bool narrow = narrow_columns(N);
    cudaError_t e = cudaSuccess;
    for (int it = 0; it < sweeps && e == cudaSuccess; ++it) {
        e = launch(fit_rows_kernel, dim3(ceil_div(M, 16)), dim3(256), 0, s, true, (const float *)R, M, N, ldr,
                   (const float *)alpha_c, it == 0 ? 1 : 0, alpha_r);
        if (e == cudaSuccess)
            e = narrow ? launch_cluster(fit_cols_kernel<16>, cols_grid, 16 * 32, s, (const float *)R, M, N, ldr,
                                        (const float *)alpha_r, alpha_c)
                       : launch_cluster(fit_cols_kernel<8>, cols_grid, 8 * 32, s, (const float *)R, M, N, ldr,
                                        (const float *)alpha_r, alpha_c);
    }
    if (e == cudaSuccess) {
        // tpr threads (four columns each) per row, 256 / tpr rows per block
        const int quads = ceil_div(N, 4), tpr = std::min(256, round_up(quads, 32)), rpb = 256 / tpr;
        const dim3 ugrid(ceil_div(quads, tpr), std::min(ceil_div(M, rpb), 2048));
        e = launch(fit_update_kernel, ugrid, dim3(256), 0, s, true, R, M, N, ldr, (const float *)alpha_r,
                   (const float *)alpha_c, signs, lds, tpr);
    }
    return status_of(e);
}
