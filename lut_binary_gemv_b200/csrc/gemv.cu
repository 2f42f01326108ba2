// gemv.cu -- the LUT binary GEMV y = W_hat x of the FluxBin page
// (Methodology, 2. Kernel innovation), written for sm_100a.
//
// W_hat = sum_k (alpha_r^(k) alpha_c^(k)^T) (.) B^(k)  +  salient refinement
// (1. Algorithm innovation; Hessian-guided saliency-aware hybrid bases).
//
// One CTA handles one "virtual panel" -- a panel of <= 256 columns of one
// base, global or salient -- over one block of 32-row chunks:
//   1. before the programmatic-launch wait it issues the loads of its weight
//      words (128-bit, read-only, no L1 allocation), its row scales and its
//      column scales (and, for salient panels, the salient column indices);
//   2. after the wait it reads x, forms z = alpha_c * x (column scales fused
//      here: LUT-BSF) -- salient panels read x[s_idx[t]] directly, which is the
//      virtual columnar mapping -- and builds the panel's 2^g-entry tables in
//      shared memory;
//   3. each lane owns one row of a chunk and walks that row's bytes: one
//      `prmt` turns a weight byte plus the lane's column offset into a table
//      address, one shared load fetches the partial sum, packed fp32x2 adds
//      accumulate (no tensor cores: this is a gather-add, not a contraction);
//   4. the lane multiplies by alpha_r once (alpha_r applied in the reduction)
//      and writes the panel's partial for its row to the workspace;
//   5. the last CTA of a row block to arrive (atomic ticket) sums the partials
//      of all panels in a fixed order and writes y: deterministic, no float
//      atomics, no spinning.
//
// Shared-memory table layout (one panel, one base), byte offsets; q = byte
// group of the panel (0..31), entries fp32:
//   g = 8: T[p][q]              at p*256 + 4q             (p < 256; 64 KiB)
//   g = 4: low nibble T[v][q]   at v*256 + 4q, high nibble at v*256 + 128 + 4q
//   g = 2: T[s][v][q]           at ((s << 2) + v)*128 + 4q (s: 2-bit field of the byte)
//   g = 1: T[s][v][q]           at ((s << 1) + v)*128 + 4q
// Lane l at stored position u reads byte group (l+u) mod Bp (the rotation of
// the packed layout), so a warp's 32 lookups hit 32 different banks.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <new>

#include "fb_internal.cuh"

namespace fb {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kPrefetch = 4;   // chunks per warp whose words are in flight ahead of use
constexpr unsigned kKnownFlags = FB_GEMV_PDL;

struct GemvArgs {
    const uint8_t *planes;
    const float *alpha_r;
    const float *alpha_c;
    const uint8_t *s_planes;
    const float *s_alpha_r;
    const float *s_alpha_c;
    const uint32_t *s_idx;
    const void *x;
    float *y;
    float *partials;      // [batch][V][M_pad]
    unsigned *counters;   // [batch][RB]
    int M, M_pad, N, K, nS, nS_pad, Ks;
    int Pg, Ps, V, nchunks, cpb, RB;
    int ldx, ldy;
};

template <int G>
__host__ __device__ constexpr int table_bytes() {
    return G == 8 ? 65536 : G == 4 ? 4096 : 2048;
}
template <int G>
__host__ __device__ constexpr int smem_bytes() {
    return table_bytes<G>() + 256 * 4;
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint4 ld_stream16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ld_stream4(const void *p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Selector producing (byte j of a) << 8 | (byte j of b), upper bytes zero.
// Byte j of b is a column offset < 128, so replicating its sign bit gives 0.
__host__ __device__ constexpr uint32_t addr_sel(int j) {
    return (uint32_t)(4 + j) | ((uint32_t)j << 4) | ((uint32_t)(12 + j) << 8) | ((uint32_t)(12 + j) << 12);
}

__device__ __forceinline__ float lds(const float *tbl, uint32_t byte_off) {
    return *reinterpret_cast<const float *>(reinterpret_cast<const char *>(tbl) + byte_off);
}

// Packed fp32x2 accumulate (sm_100a).
__device__ __forceinline__ unsigned long long f2pack(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ unsigned long long fadd2(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float f2sum(unsigned long long a) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(a));
    return __fadd_rn(lo, hi);
}

template <int XT>
__device__ __forceinline__ float load_x(const void *x, size_t i) {
    if (XT == FB_F32) return ((const float *)x)[i];
    if (XT == FB_F16) return __half2float(((const __half *)x)[i]);
    return __bfloat162float(((const __nv_bfloat16 *)x)[i]);
}

// sum_{t<4} (bit t of a ? +1 : -1) * z_t, added in order t = 0..3.
__device__ __forceinline__ float sum4(float z0, float z1, float z2, float z3, int a) {
    float s = (a & 1) ? z0 : -z0;
    s = __fadd_rn(s, (a & 2) ? z1 : -z1);
    s = __fadd_rn(s, (a & 4) ? z2 : -z2);
    s = __fadd_rn(s, (a & 8) ? z3 : -z3);
    return s;
}

// LUT-BSF: build this panel's tables from z = alpha_c * x (alpha_c already
// fused into z).  Lane = byte group, warp w writes table rows 2w and 2w+1 of
// the 16 row groups.
template <int G>
__device__ __forceinline__ void build_tables(float *tbl, const float *zbuf, int Bp, int lane, int warp) {
    if (lane >= Bp) return;
    const float4 za = *reinterpret_cast<const float4 *>(zbuf + 8 * lane);
    const float4 zb = *reinterpret_cast<const float4 *>(zbuf + 8 * lane + 4);
    const float z[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
    float *col = tbl + lane;   // + row * (pitch / 4)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = 2 * warp + h;   // 0..15
        if (G == 8) {
            const float hi = sum4(z[4], z[5], z[6], z[7], r);
#pragma unroll
            for (int a = 0; a < 16; ++a)
                col[(r * 16 + a) * 64] = __fadd_rn(sum4(z[0], z[1], z[2], z[3], a), hi);
        } else if (G == 4) {
            col[r * 64] = sum4(z[0], z[1], z[2], z[3], r);
            col[r * 64 + 32] = sum4(z[4], z[5], z[6], z[7], r);
        } else if (G == 2) {
            const int s = r >> 2, v = r & 3;
            float e = (v & 1) ? z[2 * s] : -z[2 * s];
            e = __fadd_rn(e, (v & 2) ? z[2 * s + 1] : -z[2 * s + 1]);
            col[r * 32] = e;
        } else {
            const int s = r >> 1, v = r & 1;
            col[r * 32] = v ? z[s] : -z[s];
        }
    }
}

// Sum of the table entries selected by one row's stored bytes.  w holds the
// row's Bp bytes (position u in byte u%4 of w[u/4]); offp holds, in the same
// places, the byte offset 4*q of the column each position maps to.
template <int G, bool FULL>
__device__ __forceinline__ float lookup_row(const uint32_t (&w)[8], const uint32_t (&offp)[8],
                                            const float *tbl, int nw) {
    unsigned long long acc0 = 0, acc1 = 0;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        if (!FULL && m >= nw) break;
        if (G == 8) {
            const float v0 = lds(tbl, prmt(w[m], offp[m], addr_sel(0)));
            const float v1 = lds(tbl, prmt(w[m], offp[m], addr_sel(1)));
            const float v2 = lds(tbl, prmt(w[m], offp[m], addr_sel(2)));
            const float v3 = lds(tbl, prmt(w[m], offp[m], addr_sel(3)));
            acc0 = fadd2(acc0, f2pack(v0, v1));
            acc1 = fadd2(acc1, f2pack(v2, v3));
        } else if (G == 4) {
            const uint32_t w4 = w[m] >> 4;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float lo = lds(tbl, prmt(w[m], offp[m], addr_sel(j)) & 0x0FFFu);
                const float hi = lds(tbl + 32, prmt(w4, offp[m], addr_sel(j)) & 0x0FFFu);
                if (j & 1)
                    acc1 = fadd2(acc1, f2pack(lo, hi));
                else
                    acc0 = fadd2(acc0, f2pack(lo, hi));
            }
        } else {
            constexpr int kFields = 8 / G, kMask = (1 << G) - 1;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t byte = (w[m] >> (8 * j)) & 0xFFu;
                const uint32_t off = (offp[m] >> (8 * j)) & 0xFFu;
#pragma unroll
                for (int s = 0; s < kFields; s += 2) {
                    const uint32_t v0 = (byte >> (G * s)) & kMask, v1 = (byte >> (G * (s + 1))) & kMask;
                    const float e0 = lds(tbl, (((uint32_t)s << G) + v0) * 128u + off);
                    const float e1 = lds(tbl, (((uint32_t)(s + 1) << G) + v1) * 128u + off);
                    acc0 = fadd2(acc0, f2pack(e0, e1));
                }
            }
        }
    }
    return __fadd_rn(f2sum(acc0), f2sum(acc1));
}

struct PanelView {
    const uint8_t *pl;   // first chunk block of this panel and base
    const float *ar;     // row scales of this base
    int Bp;              // byte groups in the panel
};

__device__ __forceinline__ void load_chunk(const PanelView &pv, int c, int lane, int M, uint32_t (&w)[8],
                                           float &arv) {
    const uint8_t *blk = pv.pl + (size_t)32 * pv.Bp * c;
    if (pv.Bp == 32) {
        const uint4 a = ld_stream16(blk + 16 * lane), b = ld_stream16(blk + 512 + 16 * lane);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else if (pv.Bp == 16) {
        const uint4 a = ld_stream16(blk + 16 * lane);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    } else {
#pragma unroll
        for (int m = 0; m < 7; ++m)
            if (m < pv.Bp / 4) w[m] = ld_stream4(blk + 128 * m + 4 * lane);
    }
    const int row = c * kChunkRows + lane;
    arv = row < M ? __ldg(pv.ar + row) : 0.0f;
}

template <int G, int XT>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const GemvArgs a) {
    extern __shared__ __align__(16) float smem_f[];
    float *tbl = smem_f;
    float *zbuf = smem_f + table_bytes<G>() / 4;
    __shared__ unsigned s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v = blockIdx.x % a.V, rb = blockIdx.x / a.V, b = blockIdx.y;

    // Which virtual panel: global panels of base k first, then salient ones.
    const int nglob = a.Pg * a.K;
    const bool sal = v >= nglob;
    int k, p;
    if (!sal) {
        k = v / a.Pg;
        p = v - k * a.Pg;
    } else {
        k = (v - nglob) / a.Ps;
        p = (v - nglob) - k * a.Ps;
    }
    const int ncols = sal ? a.nS_pad : a.N;
    const int width = panel_width(ncols, p);
    PanelView pv;
    pv.Bp = width >> 3;
    pv.pl = (sal ? a.s_planes : a.planes) + (size_t)k * a.M_pad * (size_t)(ncols / 8) +
            (size_t)32 * p * a.M_pad;
    pv.ar = (sal ? a.s_alpha_r : a.alpha_r) + (size_t)k * a.M;

    const int c_begin = rb * a.cpb;
    const int c_end = min(c_begin + a.cpb, a.nchunks);
    const int n_mine = (c_end - c_begin > warp) ? (c_end - c_begin - warp + kWarps - 1) / kWarps : 0;

    // --- 1. weights and scales: independent of the previous kernel ---------
    float ac = 0.0f;
    uint32_t xcol = 0;
    bool xvalid = false;
    if (tid < width) {
        const int col = p * kPanelCols + tid;
        if (!sal) {
            ac = a.alpha_c ? __ldg(a.alpha_c + (size_t)k * a.N + col) : 1.0f;
            xcol = (uint32_t)col;
            xvalid = true;
        } else if (col < a.nS) {
            ac = __ldg(a.s_alpha_c + (size_t)k * a.nS + col);
            xcol = __ldg(a.s_idx + col);
            xvalid = xcol < (uint32_t)a.N;   // an invalid index contributes 0
        }
    }
    uint32_t wreg[kPrefetch][8];
    float arreg[kPrefetch];
#pragma unroll
    for (int s = 0; s < kPrefetch; ++s)
        if (s < n_mine) load_chunk(pv, c_begin + warp + kWarps * s, lane, a.M, wreg[s], arreg[s]);
    griddep_launch_dependents();

    // --- 2. activations: may be the previous kernel's output ----------------
    griddep_wait();
    if (tid < width) {
        const float xv = xvalid ? load_x<XT>(a.x, (size_t)b * a.ldx + xcol) : 0.0f;
        zbuf[tid] = __fmul_rn(ac, xv);
    }
    __syncthreads();
    build_tables<G>(tbl, zbuf, pv.Bp, lane, warp);

    uint32_t offp[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        uint32_t o = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int u = 4 * m + j;
            const int q = (pv.Bp == 32) ? ((lane + u) & 31) : ((lane + u) % pv.Bp);
            o |= (uint32_t)(4 * q) << (8 * j);
        }
        offp[m] = o;
    }
    __syncthreads();

    // --- 3/4. stream rows through the tables, apply alpha_r ------------------
    float *part = a.partials + ((size_t)b * a.V + v) * a.M_pad;
    const int nw = pv.Bp / 4;
    for (int i0 = 0; i0 < n_mine; i0 += kPrefetch) {
#pragma unroll
        for (int s = 0; s < kPrefetch; ++s) {
            const int i = i0 + s;
            if (i < n_mine) {
                const int c = c_begin + warp + kWarps * i;
                const float sum = (pv.Bp == 32) ? lookup_row<G, true>(wreg[s], offp, tbl, 8)
                                                : lookup_row<G, false>(wreg[s], offp, tbl, nw);
                part[c * kChunkRows + lane] = __fmul_rn(arreg[s], sum);
                if (i + kPrefetch < n_mine)
                    load_chunk(pv, c + kWarps * kPrefetch, lane, a.M, wreg[s], arreg[s]);
            }
        }
    }

    // --- 5. last CTA of this row block sums the panels in a fixed order ------
    __threadfence();
    __syncthreads();
    if (tid == 0)
        s_last = atomicInc(a.counters + (size_t)b * a.RB + rb, (unsigned)(a.V - 1)) == (unsigned)(a.V - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int r0 = c_begin * kChunkRows, r1 = min(c_end * kChunkRows, a.M);
    const float *pb = a.partials + (size_t)b * a.V * a.M_pad;
    for (int row = r0 + tid; row < r1; row += kThreads) {
        float s = 0.0f;
#pragma unroll 8
        for (int vv = 0; vv < a.V; ++vv) s = __fadd_rn(s, __ldcg(pb + (size_t)vv * a.M_pad + row));
        a.y[(size_t)b * a.ldy + row] = s;
    }
}

using KernelFn = void (*)(GemvArgs);

template <int G>
KernelFn pick_xt(fb_dtype t) {
    return t == FB_F32 ? gemv_kernel<G, FB_F32> : t == FB_F16 ? gemv_kernel<G, FB_F16> : gemv_kernel<G, FB_BF16>;
}

KernelFn pick_kernel(int g, fb_dtype t, int *smem) {
    switch (g) {
        case 8: *smem = smem_bytes<8>(); return pick_xt<8>(t);
        case 4: *smem = smem_bytes<4>(); return pick_xt<4>(t);
        case 2: *smem = smem_bytes<2>(); return pick_xt<2>(t);
        default: *smem = smem_bytes<1>(); return pick_xt<1>(t);
    }
}

// Device-independent part of the launch plan.
struct Plan {
    int M_pad, Pg, Ps, nS_pad, V, nchunks;
    size_t part_bytes, ctr_offset, ctr_bytes, total;
};

size_t align256(size_t n) { return (n + 255) / 256 * 256; }

fb_status check_weights(const fb_weights *W) {
    if (!W || !valid_dims(W->K, W->M, W->N) || !(W->g == 1 || W->g == 2 || W->g == 4 || W->g == 8))
        return FB_ERR_INVALID_VALUE;
    if (!W->planes || !W->alpha_r) return FB_ERR_INVALID_VALUE;
    if (W->nS < 0 || W->nS > W->N) return FB_ERR_INVALID_VALUE;
    if (W->nS > 0 && (W->Ks < 1 || W->Ks > kMaxK || !W->s_idx || !W->s_planes || !W->s_alpha_r ||
                      !W->s_alpha_c))
        return FB_ERR_INVALID_VALUE;
    if (!aligned(W->planes, 16) || !aligned(W->alpha_r, 4) || (W->alpha_c && !aligned(W->alpha_c, 4)))
        return FB_ERR_MISALIGNED;
    if (W->nS > 0 && (!aligned(W->s_planes, 16) || !aligned(W->s_idx, 4) || !aligned(W->s_alpha_r, 4) ||
                      !aligned(W->s_alpha_c, 4)))
        return FB_ERR_MISALIGNED;
    return FB_OK;
}

Plan make_plan(const fb_weights *W, int batch) {
    Plan pl;
    pl.M_pad = round_up(W->M, kChunkRows);
    pl.Pg = num_panels(W->N);
    pl.nS_pad = W->nS > 0 ? round_up(W->nS, 32) : 0;
    pl.Ps = W->nS > 0 ? num_panels(pl.nS_pad) : 0;
    pl.V = pl.Pg * W->K + pl.Ps * (W->nS > 0 ? W->Ks : 0);
    pl.nchunks = pl.M_pad / kChunkRows;
    pl.part_bytes = align256((size_t)batch * pl.V * pl.M_pad * sizeof(float));
    pl.ctr_offset = pl.part_bytes;
    pl.ctr_bytes = align256((size_t)batch * pl.nchunks * sizeof(unsigned));
    pl.total = pl.part_bytes + pl.ctr_bytes;
    return pl;
}

// Resident CTAs per SM for a kernel (cached per device and kernel).
int occupancy_of(KernelFn fn, int smem) {
    struct Entry { KernelFn fn; int dev; int occ; };
    static Entry cache[64];
    static int n_cache = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    for (int i = 0; i < n_cache; ++i)
        if (cache[i].fn == fn && cache[i].dev == dev) return cache[i].occ;
    if (smem > 48 * 1024) cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kThreads, smem) != cudaSuccess || occ < 1)
        occ = 1;
    if (n_cache < 64) cache[n_cache++] = {fn, dev, occ};
    return occ;
}

// Split the rows into RB blocks of cpb chunks.  Each CTA (one virtual panel x
// one row block) pays a fixed table build plus work proportional to its rows,
// all of it on the shared-memory pipe, so pick the split that minimises the
// per-SM total: ceil(CTAs / SMs) * (cpb * lookups per chunk + table entries).
void choose_row_blocks(const Plan &pl, int g, int sms, int *RB_out, int *cpb_out) {
    struct Memo { int nchunks, V, g, sms, RB, cpb; };
    thread_local Memo memo[8] = {};
    thread_local int memo_next = 0;
    for (const Memo &m : memo)
        if (m.nchunks == pl.nchunks && m.V == pl.V && m.g == g && m.sms == sms) {
            *RB_out = m.RB;
            *cpb_out = m.cpb;
            return;
        }
    const double per_chunk = 32.0 * 32.0 * (8 / g);
    const double build = g == 8 ? 8192.0 : g == 4 ? 1024.0 : 512.0;
    const int rb_max = std::min(pl.nchunks, 16 * ceil_div(sms, pl.V));
    double best = 1e300;
    int best_rb = 1, best_cpb = pl.nchunks;
    for (int rb = 1; rb <= rb_max; ++rb) {
        const int cpb = ceil_div(pl.nchunks, rb);
        const int RB = ceil_div(pl.nchunks, cpb);
        if (RB != rb) continue;   // the same split is reached by a smaller rb
        const double per_sm = (double)ceil_div(pl.V * RB, sms);
        const double cost = per_sm * (cpb * per_chunk + build);
        if (cost < best * 0.999) {
            best = cost;
            best_rb = RB;
            best_cpb = cpb;
        }
    }
    memo[memo_next] = {pl.nchunks, pl.V, g, sms, best_rb, best_cpb};
    memo_next = (memo_next + 1) % 8;
    *RB_out = best_rb;
    *cpb_out = best_cpb;
}

}  // namespace
}  // namespace fb

using namespace fb;

extern "C" fb_status fb_validate_weights(const fb_weights *W) {
    const fb_status st = check_weights(W);
    if (st != FB_OK || W->nS == 0) return st;
    uint32_t *h = new (std::nothrow) uint32_t[W->nS];
    if (!h) return FB_ERR_INVALID_VALUE;
    fb_status out = FB_OK;
    if (cudaMemcpy(h, W->s_idx, sizeof(uint32_t) * W->nS, cudaMemcpyDeviceToHost) != cudaSuccess) {
        out = FB_ERR_CUDA;
    } else {
        for (int t = 0; t < W->nS; ++t)
            if (h[t] >= (uint32_t)W->N || (t > 0 && h[t] <= h[t - 1])) {
                out = FB_ERR_INVALID_VALUE;
                break;
            }
    }
    delete[] h;
    return out;
}

extern "C" size_t fb_gemv_workspace_bytes(const fb_weights *W, int batch) {
    if (check_weights(W) != FB_OK || batch < 1 || batch > kMaxBatch) return 0;
    return make_plan(W, batch).total;
}

extern "C" fb_status fb_gemv_batched(const fb_weights *W, const void *X, fb_dtype t, int batch, int ldx,
                                     float *Y, int ldy, void *ws, size_t ws_bytes, unsigned flags,
                                     void *stream) {
    fb_status st = check_weights(W);
    if (st != FB_OK) return st;
    const int es = dtype_size(t);
    if (!X || !Y || !es || batch < 1 || batch > kMaxBatch || ldx < W->N || ldy < W->M ||
        (flags & ~kKnownFlags))
        return FB_ERR_INVALID_VALUE;
    if (!aligned(X, es) || !aligned(Y, 4)) return FB_ERR_MISALIGNED;
    const Plan pl = make_plan(W, batch);
    if (!ws || !aligned(ws, 16) || ws_bytes < pl.total) return FB_ERR_WORKSPACE;

    int smem = 0;
    const KernelFn fn = pick_kernel(W->g, t, &smem);
    occupancy_of(fn, smem);   // also raises the kernel's dynamic shared-memory limit once
    int RB, cpb;
    choose_row_blocks(pl, W->g, sm_count(), &RB, &cpb);

    GemvArgs a;
    a.planes = (const uint8_t *)W->planes;
    a.alpha_r = W->alpha_r;
    a.alpha_c = W->alpha_c;
    a.s_planes = (const uint8_t *)W->s_planes;
    a.s_alpha_r = W->s_alpha_r;
    a.s_alpha_c = W->s_alpha_c;
    a.s_idx = W->s_idx;
    a.x = X;
    a.y = Y;
    a.partials = (float *)ws;
    a.counters = (unsigned *)((char *)ws + pl.ctr_offset);
    a.M = W->M;
    a.M_pad = pl.M_pad;
    a.N = W->N;
    a.K = W->K;
    a.nS = W->nS;
    a.nS_pad = pl.nS_pad;
    a.Ks = W->nS > 0 ? W->Ks : 0;
    a.Pg = pl.Pg;
    a.Ps = pl.Ps;
    a.V = pl.V;
    a.nchunks = pl.nchunks;
    a.cpb = cpb;
    a.RB = RB;
    a.ldx = ldx;
    a.ldy = ldy;
    const dim3 grid(pl.V * RB, batch);
    return status_of(launch(fn, grid, dim3(kThreads), smem, as_stream(stream), (flags & FB_GEMV_PDL) != 0, a));
}

extern "C" fb_status fb_gemv(const fb_weights *W, const void *x, fb_dtype t, float *y, void *ws,
                             size_t ws_bytes, unsigned flags, void *stream) {
    if (!W) return FB_ERR_INVALID_VALUE;
    return fb_gemv_batched(W, x, t, 1, W->N, y, W->M, ws, ws_bytes, flags, stream);
}
