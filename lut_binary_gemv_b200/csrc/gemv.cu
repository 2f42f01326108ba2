// gemv.cu -- the LUT binary GEMV y = W_hat x of the FluxBin page
// (Methodology, 2. Kernel innovation), written for sm_100a.
//
// W_hat = sum_k (alpha_r^(k) alpha_c^(k)^T) (.) B^(k)  +  salient refinement
// (1. Algorithm innovation; Hessian-guided saliency-aware hybrid bases).
//
// Work units.  A "virtual panel" is one panel (<= 256 columns) of one base,
// global or salient; the matrix has V of them.  Rows come in chunks of 32,
// one row per lane.  A thread-block cluster of C CTAs owns one block of cpb
// chunks; CTA j of the cluster takes a contiguous, balanced slice of the V
// virtual panels, so the cluster covers every column of its rows.
//
// Per CTA:
//   1. before the programmatic-launch wait: the first weight words of every
//      warp (128-bit, read-only, no L1 allocation) and their row scales, and
//      the column scales and salient indices of the first table group;
//   2. after the wait (or before it, for calls flagged independent): x, then
//      z = alpha_c * x for the group's columns (column scales fused: LUT-BSF;
//      salient panels read x[s_idx[t]] -- the virtual columnar mapping), and
//      the group's tables in shared memory;
//   3. each lane walks its row's bytes: one `prmt` merges a weight byte and
//      the lane's column offset into a table address, one shared load fetches
//      the partial sum, packed fp32x2 adds accumulate (a gather-add, no tensor
//      cores); the sum of each panel is scaled by alpha_r once (alpha_r applied
//      in the reduction) and added to the row's partial;
//   4. the cluster synchronises and each CTA sums the C partials of its share
//      of the rows from distributed shared memory, in a fixed order, and
//      writes y.  No workspace, no atomics, no spin-waits; deterministic.
//
// Shared-memory tables of one virtual panel (byte offsets, q = byte group of
// the panel, entries fp32):
//   g = 8: T[p][q] at p*256 + 4q; two panels share a 64 KiB region, the second
//          at +128 (p < 256)
//   g = 4: low nibble T[v][q] at v*256 + 4q, high nibble at v*256 + 128 + 4q
//   g = 2: T[s][v][q] at ((s << 2) + v)*128 + 4q (s: 2-bit field of the byte)
//   g = 1: T[s][v][q] at ((s << 1) + v)*128 + 4q
// Lane l at stored position u reads byte group (l+u) mod Bp (the rotation of
// the packed layout), so a warp's 32 lookups hit 32 different banks.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <new>

#include "fb_internal.cuh"

namespace cg = cooperative_groups;

namespace fb {
namespace {

constexpr int kMaxCluster = 8;
constexpr int kThreads = 256;           // 8 warps; thread t stages column t of a panel
constexpr int kWarps = kThreads / 32;
constexpr int kRing = 4;                // weight items per warp in flight ahead of use
constexpr int kMaxGroup = 8;            // virtual panels per table group
constexpr int kMaxCpb = 64;             // chunks per row block
constexpr unsigned kKnownFlags = FB_GEMV_PDL | FB_GEMV_INDEPENDENT;

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
    int M, M_pad, N, K, nS, nS_pad, Ks;
    int Pg, Ps;
    int nchunks, cpb, n_my;   // chunks per row block; per warp (cpb = warps * n_my)
    int group_max;            // virtual panels per table group
    int ldx, ldy;
    unsigned flags;
    int C;
    int vsplit[kMaxCluster + 1];   // CTA j of a cluster: virtual panels [vsplit[j], vsplit[j+1])
    int first_sal[kMaxCluster], first_k[kMaxCluster], first_p[kMaxCluster];   // decoded vsplit[j]
    int narrow_mask[kMaxCluster];  // bit 0: rank j has the narrow global tail panel; bit 1: a narrow salient one
};

// Table bytes per virtual panel slot in a group.
__host__ __device__ constexpr int table_stride(int g) { return g == 8 ? 32768 : g == 4 ? 4096 : 2048; }

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

// The stored bits of x[i] (no conversion, so the load does not stall) ...
template <int XT>
__device__ __forceinline__ uint32_t load_x_bits(const void *x, size_t i) {
    if (XT == FB_F32) return __ldg((const unsigned int *)x + i);
    return (uint32_t)__ldg((const unsigned short *)x + i);
}
// ... and their value, exactly.
template <int XT>
__device__ __forceinline__ float x_value(uint32_t bits) {
    if (XT == FB_F32) return __uint_as_float(bits);
    if (XT == FB_F16) return __half2float(__ushort_as_half((unsigned short)bits));
    return __uint_as_float(bits << 16);
}

// sum_{t<4} (bit t of a ? +1 : -1) * z_t, added in order t = 0..3.
__device__ __forceinline__ float sum4(float z0, float z1, float z2, float z3, int a) {
    float s = (a & 1) ? z0 : -z0;
    s = __fadd_rn(s, (a & 2) ? z1 : -z1);
    s = __fadd_rn(s, (a & 4) ? z2 : -z2);
    s = __fadd_rn(s, (a & 8) ? z3 : -z3);
    return s;
}

// The 16 entries sum_{t<4} (bit t of a ? +1 : -1) * z_t, a = 0..15, as
// (+-z0 +- z1) + (+-z2 +- z3).
__device__ __forceinline__ void sums16(float z0, float z1, float z2, float z3, float (&e)[16]) {
    const float p01[4] = {__fadd_rn(-z0, -z1), __fadd_rn(z0, -z1), __fadd_rn(-z0, z1), __fadd_rn(z0, z1)};
    const float p23[4] = {__fadd_rn(-z2, -z3), __fadd_rn(z2, -z3), __fadd_rn(-z2, z3), __fadd_rn(z2, z3)};
#pragma unroll
    for (int a = 0; a < 16; ++a) e[a] = __fadd_rn(p01[a & 3], p23[a >> 2]);
}

// One virtual panel: where its words and row scales live, its width.
struct VPanel {
    const uint8_t *pl;   // chunk block 0 of this panel and base
    const float *ar;     // row scales of this base
    const float *ac;     // column scales of this base, or null (all ones)
    int col0;            // first column of the panel (global, or compact salient)
    int Bp;              // byte groups (width / 8)
    int k, p, sal;       // base, panel, 1 for salient panels
};

__device__ __forceinline__ void vp_set(const GemvArgs &a, VPanel &r, int sal, int k, int p) {
    const int ncols = sal ? a.nS_pad : a.N;
    r.sal = sal;
    r.k = k;
    r.p = p;
    r.col0 = p * kPanelCols;
    r.Bp = panel_width(ncols, p) >> 3;
    r.pl = (sal ? a.s_planes : a.planes) + (size_t)k * a.M_pad * (size_t)(ncols / 8) + (size_t)32 * p * a.M_pad;
    r.ar = (sal ? a.s_alpha_r : a.alpha_r) + (size_t)k * a.M;
    r.ac = sal ? a.s_alpha_c + (size_t)k * a.nS : (a.alpha_c ? a.alpha_c + (size_t)k * a.N : nullptr);
}

// Virtual panel v: global panels of base 0, 1, ... then salient ones.
__device__ __forceinline__ void vp_first(const GemvArgs &a, VPanel &r, int v) {
    const int ng = a.Pg * a.K;
    if (v < ng) {
        const int k = v / a.Pg;
        vp_set(a, r, 0, k, v - k * a.Pg);
    } else {
        const int k = (v - ng) / max(a.Ps, 1);
        vp_set(a, r, 1, k, (v - ng) - k * a.Ps);
    }
}

// The virtual panel after r, without a division.
__device__ __forceinline__ void vp_next(const GemvArgs &a, VPanel &r) {
    int sal = r.sal, k = r.k, p = r.p + 1;
    if (p == (sal ? a.Ps : a.Pg)) {
        p = 0;
        if (++k == (sal ? a.Ks : a.K) && !sal) {
            sal = 1;
            k = 0;
        }
    }
    vp_set(a, r, sal, k, p);
}

// Column c of a panel: its scale alpha_c and the column of x it reads (-1:
// none, including the columns past a narrow panel's width, which therefore
// build all-zero table columns).
__device__ __forceinline__ void column_source(const GemvArgs &a, const VPanel &vp, int c, float &ac, int &xi) {
    ac = 0.0f;
    xi = -1;
    if (c >= vp.Bp * 8) return;
    const int col = vp.col0 + c;
    if (!vp.sal) {
        ac = vp.ac ? __ldg(vp.ac + col) : 1.0f;
        xi = col;
    } else if (col < a.nS) {
        ac = __ldg(vp.ac + col);
        const uint32_t jx = __ldg(a.s_idx + col);
        xi = jx < (uint32_t)a.N ? (int)jx : -1;   // an invalid index contributes 0
    }
}

// The row's words of one chunk of one panel; positions past a narrow
// panel's Bp bytes are zero.
__device__ __forceinline__ void load_item(const VPanel &vp, int c, const GemvArgs &a, int lane, uint32_t (&w)[8],
                                          float &arv) {
#pragma unroll
    for (int m = 0; m < 8; ++m) w[m] = 0;
    arv = 0.0f;
    if (c >= a.nchunks) return;   // padding chunk of the last row block
    const uint8_t *blk = vp.pl + (size_t)32 * vp.Bp * c;
    if (vp.Bp == 32) {
        const uint4 x0 = ld_stream16(blk + 16 * lane), x1 = ld_stream16(blk + 512 + 16 * lane);
        w[0] = x0.x; w[1] = x0.y; w[2] = x0.z; w[3] = x0.w;
        w[4] = x1.x; w[5] = x1.y; w[6] = x1.z; w[7] = x1.w;
    } else if (vp.Bp == 16) {
        const uint4 x0 = ld_stream16(blk + 16 * lane);
        w[0] = x0.x; w[1] = x0.y; w[2] = x0.z; w[3] = x0.w;
    } else {
#pragma unroll
        for (int m = 0; m < 7; ++m)
            if (m < vp.Bp / 4) w[m] = ld_stream4(blk + 128 * m + 4 * lane);
    }
    const int row = c * kChunkRows + lane;
    arv = row < a.M ? __ldg(vp.ar + row) : 0.0f;
}

// Column offsets of a full panel: byte j of offp[m] = 4 * ((lane + 4m + j) mod 32).
__device__ __forceinline__ void full_offsets(int lane, uint32_t (&offp)[8]) {
    const uint32_t L = (uint32_t)(4 * lane) * 0x01010101u;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const uint32_t K = (uint32_t)(16 * m) * 0x01010101u + 0x0C080400u;   // bytes 16m + 4j
        offp[m] = (L + K) & 0x7C7C7C7Cu;                                      // no carry between bytes
    }
}

// Column offsets of a narrow panel (Bp < 32), one word (8 per lane) per
// call: byte j of word m = 4 * ((lane + u) mod Bp) for u = 4m + j < Bp, and
// column 31 (built all zero) for the positions past Bp.
__device__ __forceinline__ uint32_t narrow_offset_word(int lane, int m, int Bp) {
    uint32_t o = 0;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const int u = 4 * m + jj;
        const int q = u < Bp ? (lane + u) % Bp : 31;
        o |= (uint32_t)(4 * q) << (8 * jj);
    }
    return o;
}

// Sum of the table entries selected by one row's 32 stored bytes.  w holds
// position u in byte u%4 of w[u/4]; offp holds, in the same places, the byte
// offset 4*q of the column each position maps to.
template <int G>
__device__ __forceinline__ float lookup_row(const uint32_t (&w)[8], const uint32_t (&offp)[8], const float *tbl) {
    unsigned long long acc0 = 0, acc1 = 0;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
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
            for (int jj = 0; jj < 4; ++jj) {
                const float lo = lds(tbl, prmt(w[m], offp[m], addr_sel(jj)) & 0x0FFFu);
                const float hi = lds(tbl + 32, prmt(w4, offp[m], addr_sel(jj)) & 0x0FFFu);
                if (jj & 1)
                    acc1 = fadd2(acc1, f2pack(lo, hi));
                else
                    acc0 = fadd2(acc0, f2pack(lo, hi));
            }
        } else {
            constexpr int kFields = 8 / G, kMask = (1 << G) - 1;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const uint32_t byte = (w[m] >> (8 * jj)) & 0xFFu;
                const uint32_t off = (offp[m] >> (8 * jj)) & 0xFFu;
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

template <int G>
__device__ __forceinline__ const float *table_of(const float *tbl, int slot) {
    if (G == 8) return tbl + (slot >> 1) * 16384 + (slot & 1) * 32;
    return tbl + slot * (table_stride(G) / 4);
}

// LUT-BSF: the tables of one group of virtual panels from z = alpha_c * x
// (z is 0 past a narrow panel's width, so those table columns are 0).
// Tasks (slot, q, r): q = byte group (consecutive threads -> consecutive
// banks), r = 0..15 a row group of the table.
template <int G>
__device__ __forceinline__ void build_group(float *tbl, const float *zbuf, int gsize, int tid, int nthreads) {
    if (G == 4 || G == 8) {
        // g = 4: task (slot, q, half) writes the 16 entries of one nibble table.
        // g = 8: task (slot, q, hi) writes the 16 entries lo[a] + hi-sum[hi].
        const int ntask = gsize * 32 * (G == 4 ? 2 : 16);
        for (int t = tid; t < ntask; t += nthreads) {
            const int q = t & 31;
            const int r = G == 4 ? (t >> 5) & 1 : (t >> 5) & 15;
            const int slot = G == 4 ? t >> 6 : t >> 9;
            const float *z = zbuf + slot * 256 + 8 * q;
            float *col = const_cast<float *>(table_of<G>(tbl, slot)) + q;
            float e[16];
            if (G == 4) {
                const float4 zz = *reinterpret_cast<const float4 *>(z + 4 * r);
                sums16(zz.x, zz.y, zz.z, zz.w, e);
#pragma unroll
                for (int a = 0; a < 16; ++a) col[a * 64 + 32 * r] = e[a];
            } else {
                const float4 za = *reinterpret_cast<const float4 *>(z);
                const float4 zb = *reinterpret_cast<const float4 *>(z + 4);
                sums16(za.x, za.y, za.z, za.w, e);
                float h[16];
                sums16(zb.x, zb.y, zb.z, zb.w, h);
                float hr = h[0];
#pragma unroll
                for (int a = 1; a < 16; ++a) hr = r == a ? h[a] : hr;
#pragma unroll
                for (int a = 0; a < 16; ++a) col[(r * 16 + a) * 64] = __fadd_rn(e[a], hr);
            }
        }
        return;
    }
    const int ntask = gsize * 32 * 16;
    for (int t = tid; t < ntask; t += nthreads) {
        const int q = t & 31, r = (t >> 5) & 15, slot = t >> 9;
        const float *z = zbuf + slot * 256 + 8 * q;
        const float4 za = *reinterpret_cast<const float4 *>(z);
        const float4 zb = *reinterpret_cast<const float4 *>(z + 4);
        float *col = const_cast<float *>(table_of<G>(tbl, slot)) + q;
        if (G == 2) {
            const int s = r >> 2, v = r & 3;
            const float lo0 = s == 0 ? za.x : s == 1 ? za.z : s == 2 ? zb.x : zb.z;
            const float lo1 = s == 0 ? za.y : s == 1 ? za.w : s == 2 ? zb.y : zb.w;
            float e = (v & 1) ? lo0 : -lo0;
            e = __fadd_rn(e, (v & 2) ? lo1 : -lo1);
            col[r * 32] = e;
        } else {
            const int s = r >> 1, v = r & 1;
            const float zs = s == 0 ? za.x : s == 1 ? za.y : s == 2 ? za.z : s == 3 ? za.w
                           : s == 4 ? zb.x : s == 5 ? zb.y : s == 6 ? zb.z : zb.w;
            col[r * 32] = v ? zs : -zs;
        }
    }
}

template <int G, int XT>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const GemvArgs a) {
    extern __shared__ __align__(16) float smem_f[];
    // offsets of the (at most two) narrow panel widths: global tail, salient tail
    __shared__ __align__(16) uint32_t s_noff[2][32][8];
    cg::cluster_group cluster = cg::this_cluster();
    const int j = (int)cluster.block_rank();
    const int rb = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const int vb = a.vsplit[j], nv = a.vsplit[j + 1] - vb;
    const int GM = a.group_max;
    const int ngroups = (nv + GM - 1) / GM;
    float *tbl = smem_f;
    const int tfloats = G == 8 ? ((GM + 1) / 2) * 16384 : GM * (table_stride(G) / 4);
    float *zbuf = tbl + tfloats;
    float *part = zbuf + GM * 256;
    const bool independent = (a.flags & FB_GEMV_INDEPENDENT) != 0;
    const int c_first = rb * a.cpb;   // first chunk of the row block
    const int n_my = a.n_my;          // chunks per warp: c_first + warp + 8 * ci
    const size_t xoff = (size_t)b * a.ldx;
    const int bp_gtail = panel_width(a.N, a.Pg - 1) >> 3;
    const int bp_stail = a.Ps > 0 ? panel_width(a.nS_pad, a.Ps - 1) >> 3 : 32;

    // ---- 1. weights and first-group column data, before the wait ----------
    // Every warp walks the same padded item sequence: per table group, its
    // real items (panel-major, n_my chunks each) padded to a multiple of kRing.
    uint32_t ring[kRing][8];
    float ring_ar[kRing];
    int p_g = 0, p_pos = 0, p_ci = 0, p_vi = 0;   // producer: group, padded position, chunk, panel
    VPanel p_vp;
    vp_set(a, p_vp, a.first_sal[j], a.first_k[j], a.first_p[j]);
    auto produce = [&](uint32_t (&w)[8], float &arv) {
        if (p_g >= ngroups) return;
        const int n_real = n_my * min(GM, nv - p_g * GM);
        if (p_pos < n_real) {
            load_item(p_vp, c_first + warp + kWarps * p_ci, a, lane, w, arv);
            if (++p_ci == n_my) {
                p_ci = 0;
                if (++p_vi < nv) vp_next(a, p_vp);
            }
        }
        if (++p_pos == (n_real + kRing - 1) / kRing * kRing) {
            p_pos = 0;
            ++p_g;
        }
    };
#pragma unroll
    for (int s = 0; s < kRing; ++s) produce(ring[s], ring_ar[s]);

    // column data of a table group: thread t stages column t of each panel
    float z_ac[kMaxGroup];
    uint32_t z_x[kMaxGroup];
    int z_xi[kMaxGroup];
    auto stage_group = [&](int g0, bool read_x) {
        const int gsize = min(GM, nv - g0);
        VPanel vp;
        if (g0 == 0)
            vp_set(a, vp, a.first_sal[j], a.first_k[j], a.first_p[j]);
        else
            vp_first(a, vp, vb + g0);
#pragma unroll
        for (int gi = 0; gi < kMaxGroup; ++gi) {
            z_ac[gi] = 0.0f;
            z_xi[gi] = -1;
            z_x[gi] = 0;
            if (gi < gsize) {
                if (gi > 0) vp_next(a, vp);
                column_source(a, vp, tid, z_ac[gi], z_xi[gi]);
                if (read_x && z_xi[gi] >= 0) z_x[gi] = load_x_bits<XT>(a.x, xoff + z_xi[gi]);
            }
        }
    };
#pragma unroll
    for (int gi = 0; gi < kMaxGroup; ++gi) {
        z_ac[gi] = 0.0f;
        z_x[gi] = 0;
        z_xi[gi] = -1;
    }
    if (nv > 0) stage_group(0, independent);
    griddep_launch_dependents();
    const int nmask = a.narrow_mask[j];
    if (nmask) {
        for (int t = tid; t < 2 * 32 * 8; t += kThreads) {
            const int which = t >> 8, ln = (t >> 3) & 31, m = t & 7;
            if (nmask & (1 << which)) s_noff[which][ln][m] = narrow_offset_word(ln, m, which == 0 ? bp_gtail : bp_stail);
        }
    }

    // ---- 2. activations (may be the previous kernel's output) --------------
    if (!independent) {
        griddep_wait();
#pragma unroll
        for (int gi = 0; gi < kMaxGroup; ++gi)
            if (z_xi[gi] >= 0) z_x[gi] = load_x_bits<XT>(a.x, xoff + z_xi[gi]);
    }

    // ---- 3. table groups and the item loop ----------------------------------
    VPanel c_vp;                 // consumer: current panel, its chunk index
    vp_set(a, c_vp, a.first_sal[j], a.first_k[j], a.first_p[j]);
    int c_vi = 0, c_ci = 0;
    uint32_t offp[8];
    bool narrow = false;
    float acc1 = 0.0f;           // the row's sum when each warp owns one chunk

    for (int g = 0; g < ngroups; ++g) {
        const int g0 = g * GM, gsize = min(GM, nv - g0);
        __syncthreads();   // the previous group's tables are no longer read
#pragma unroll
        for (int gi = 0; gi < kMaxGroup; ++gi)
            if (gi < gsize) zbuf[gi * 256 + tid] = z_xi[gi] >= 0 ? __fmul_rn(z_ac[gi], x_value<XT>(z_x[gi])) : 0.0f;
        __syncthreads();
        build_group<G>(tbl, zbuf, gsize, tid, kThreads);
        if (g + 1 < ngroups) stage_group(g0 + GM, true);   // x is readable by now
        __syncthreads();
        if (g == 0) {                                      // offsets of the first panel
            narrow = c_vp.Bp != 32;
            if (narrow) {
                const int which = c_vp.sal;
#pragma unroll
                for (int m = 0; m < 8; ++m) offp[m] = s_noff[which][lane][m];
            } else {
                full_offsets(lane, offp);
            }
        }

        const int n_real = n_my * gsize;
        const int n_pad = (n_real + kRing - 1) / kRing * kRing;
        for (int i0 = 0; i0 < n_pad; i0 += kRing) {
#pragma unroll
            for (int s = 0; s < kRing; ++s) {
                if (i0 + s < n_real) {
                    const float sum = lookup_row<G>(ring[s], offp, table_of<G>(tbl, c_vi - g0));
                    const float val = __fmul_rn(ring_ar[s], sum);
                    if (n_my == 1) {
                        acc1 = c_vi == 0 ? val : __fadd_rn(acc1, val);
                    } else {
                        float &pr = part[(warp + kWarps * c_ci) * kChunkRows + lane];
                        pr = c_vi == 0 ? val : __fadd_rn(pr, val);
                    }
                    if (++c_ci == n_my) {
                        c_ci = 0;
                        if (++c_vi < nv) {
                            vp_next(a, c_vp);
                            if (c_vp.Bp != 32) {
                                const int which = c_vp.sal;
#pragma unroll
                                for (int m = 0; m < 8; ++m) offp[m] = s_noff[which][lane][m];
                                narrow = true;
                            } else if (narrow) {
                                full_offsets(lane, offp);
                                narrow = false;
                            }
                        }
                    }
                }
                produce(ring[s], ring_ar[s]);   // the item kRing positions ahead
            }
        }
    }
    if (n_my == 1) {
        part[warp * kChunkRows + lane] = acc1;
    } else if (nv == 0) {
        for (int ci = 0; ci < n_my; ++ci) part[(warp + kWarps * ci) * kChunkRows + lane] = 0.0f;
    }

    // ---- 4. cluster reduction of the row partials --------------------------
    cluster.sync();
    const int R = a.cpb * kChunkRows;
    const int r_lo = (int)((long)R * j / a.C), r_hi = (int)((long)R * (j + 1) / a.C);
    for (int r = r_lo + tid; r < r_hi; r += kThreads) {
        float v[kMaxCluster];
#pragma unroll
        for (int jj = 0; jj < kMaxCluster; ++jj) v[jj] = jj < a.C ? cluster.map_shared_rank(part, jj)[r] : 0.0f;
        float sum = v[0];
#pragma unroll
        for (int jj = 1; jj < kMaxCluster; ++jj)
            if (jj < a.C) sum = __fadd_rn(sum, v[jj]);
        const int row = c_first * kChunkRows + r;
        if (row < a.M) a.y[(size_t)b * a.ldy + row] = sum;
    }
    cluster.sync();   // keep this CTA's partials alive until every reader is done
    if (independent) griddep_wait();   // complete only after the previous kernel
}

using KernelFn = void (*)(GemvArgs);

template <int G>
KernelFn pick_xt(fb_dtype t) {
    return t == FB_F32 ? gemv_kernel<G, FB_F32> : t == FB_F16 ? gemv_kernel<G, FB_F16> : gemv_kernel<G, FB_BF16>;
}

KernelFn pick_kernel(int g, fb_dtype t) {
    switch (g) {
        case 8: return pick_xt<8>(t);
        case 4: return pick_xt<4>(t);
        case 2: return pick_xt<2>(t);
        default: return pick_xt<1>(t);
    }
}

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

// The launch plan: cluster size, split of the virtual panels over the
// cluster, row block size.  Chosen by a cost model of the shared-memory pipe
// (the binding resource): per CTA, lookups (rows x byte groups x 8/g) plus
// table entries built, plus a fixed per-CTA cost; CTAs beyond one per SM form
// further waves.
struct Plan {
    int M_pad, Pg, Ps, nS_pad, V, nchunks;
    int C, cpb, nwarps, n_my, RB, group_max;   // nwarps is always kWarps
    int vsplit[kMaxCluster + 1];
    size_t smem;
};

struct PlanKey {
    int M, N, K, g, nS, Ks, batch, sms;
    bool operator==(const PlanKey &o) const {
        return M == o.M && N == o.N && K == o.K && g == o.g && nS == o.nS && Ks == o.Ks && batch == o.batch &&
               sms == o.sms;
    }
};

// Every virtual panel costs one full 32-position lookup per row (narrow
// panels look up zero columns past their width), so the split over the
// cluster balances panel counts.
void split_panels(int V, int C, int *vsplit, int *max_n) {
    *max_n = 0;
    for (int jj = 0; jj <= C; ++jj) vsplit[jj] = (int)((long)V * jj / C);
    for (int jj = 0; jj < C; ++jj) *max_n = std::max(*max_n, vsplit[jj + 1] - vsplit[jj]);
}

Plan make_plan(const fb_weights *W, int batch, int sms) {
    Plan pl;
    pl.M_pad = round_up(W->M, kChunkRows);
    pl.Pg = num_panels(W->N);
    pl.nS_pad = W->nS > 0 ? round_up(W->nS, 32) : 0;
    pl.Ps = W->nS > 0 ? num_panels(pl.nS_pad) : 0;
    pl.V = pl.Pg * W->K + pl.Ps * (W->nS > 0 ? W->Ks : 0);
    pl.nchunks = pl.M_pad / kChunkRows;
    const int g = W->g;
    const double lookups_per_item = 32.0 * 32.0 * 8.0 / g;   // one chunk of one panel
    const double build_per_panel = g == 8 ? 8192 : g == 4 ? 1024 : 512;
    const double fixed = 6000;   // prologue, syncs, reduce, in lookup units
    double best = 1e300;
    pl.nwarps = kWarps;
    pl.C = 1;
    pl.cpb = std::min(kMaxCpb, round_up(pl.nchunks, kWarps));
    pl.RB = ceil_div(pl.nchunks, pl.cpb);
    pl.vsplit[0] = 0;
    pl.vsplit[1] = pl.V;
    for (int C = 1; C <= std::min(kMaxCluster, pl.V); ++C) {
        int vs[kMaxCluster + 1], max_n;
        split_panels(pl.V, C, vs, &max_n);
        for (int cpb = kWarps; cpb <= kMaxCpb; cpb += kWarps) {
            const int RB = ceil_div(pl.nchunks, cpb);
            if (RB > 65535) continue;   // grid.y limit
            if (cpb > kWarps && ceil_div(pl.nchunks, cpb - kWarps) == RB) continue;   // same split, fewer rows
            const long ctas = (long)C * RB * batch;
            const double work = cpb * max_n * lookups_per_item / 32.0 + max_n * build_per_panel + fixed;
            const double cost = (double)((ctas + sms - 1) / sms) * work;
            if (cost < best * 0.999) {
                best = cost;
                pl.C = C;
                pl.cpb = cpb;
                pl.RB = RB;
                std::copy(vs, vs + C + 1, pl.vsplit);
            }
        }
    }
    pl.n_my = pl.cpb / kWarps;
    pl.group_max = g == 8 ? 2 : kMaxGroup;
    const size_t tbytes = g == 8 ? (size_t)((pl.group_max + 1) / 2) * 65536 : (size_t)pl.group_max * table_stride(g);
    pl.smem = tbytes + (size_t)pl.group_max * 256 * 4 + (size_t)pl.cpb * kChunkRows * 4;
    return pl;
}

const Plan &cached_plan(const fb_weights *W, int batch, int sms) {
    struct Entry {
        PlanKey key;
        Plan plan;
    };
    thread_local Entry memo[16];
    thread_local int used = 0, next = 0;
    const PlanKey key{W->M, W->N, W->K, W->g, W->nS, W->nS > 0 ? W->Ks : 0, batch, sms};
    for (int i = 0; i < used; ++i)
        if (memo[i].key == key) return memo[i].plan;
    Entry &e = memo[next];
    e.key = key;
    e.plan = make_plan(W, batch, sms);
    next = (next + 1) % 16;
    used = std::min(used + 1, 16);
    return e.plan;
}

// Raise the kernel's dynamic shared-memory limit once per kernel and device.
bool prepare_kernel(KernelFn fn, size_t smem) {
    struct Entry {
        KernelFn fn;
        int dev;
        size_t smem;
    };
    static Entry done[64];
    static int n_done = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    for (int i = 0; i < n_done; ++i)
        if (done[i].fn == fn && done[i].dev == dev && done[i].smem >= smem) return true;
    const size_t want = std::max<size_t>(smem, 100 * 1024);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)want) != cudaSuccess)
        return false;
    if (n_done < 64) done[n_done++] = {fn, dev, want};
    return true;
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
    (void)W;
    (void)batch;
    return 0;   // partial sums stay in the cluster's shared memory
}

extern "C" fb_status fb_gemv_batched(const fb_weights *W, const void *X, fb_dtype t, int batch, int ldx,
                                     float *Y, int ldy, void *ws, size_t ws_bytes, unsigned flags,
                                     void *stream) {
    (void)ws;
    (void)ws_bytes;
    fb_status st = check_weights(W);
    if (st != FB_OK) return st;
    const int es = dtype_size(t);
    if (!X || !Y || !es || batch < 1 || batch > kMaxBatch || ldx < W->N || ldy < W->M ||
        (flags & ~kKnownFlags) || ((flags & FB_GEMV_INDEPENDENT) && !(flags & FB_GEMV_PDL)))
        return FB_ERR_INVALID_VALUE;
    if (!aligned(X, es) || !aligned(Y, 4)) return FB_ERR_MISALIGNED;

    const Plan &pl = cached_plan(W, batch, sm_count());
    const KernelFn fn = pick_kernel(W->g, t);
    if (!prepare_kernel(fn, pl.smem)) return FB_ERR_CUDA;

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
    a.M = W->M;
    a.M_pad = pl.M_pad;
    a.N = W->N;
    a.K = W->K;
    a.nS = W->nS;
    a.nS_pad = pl.nS_pad;
    a.Ks = W->nS > 0 ? W->Ks : 0;
    a.Pg = pl.Pg;
    a.Ps = pl.Ps;
    a.nchunks = pl.nchunks;
    a.cpb = pl.cpb;
    a.n_my = pl.n_my;
    a.group_max = pl.group_max;
    a.ldx = ldx;
    a.ldy = ldy;
    a.flags = flags;
    a.C = pl.C;
    std::copy(pl.vsplit, pl.vsplit + kMaxCluster + 1, a.vsplit);
    const int ng = pl.Pg * W->K;
    const bool g_narrow = W->N % kPanelCols != 0, s_narrow = pl.nS_pad % kPanelCols != 0;
    for (int jj = 0; jj < kMaxCluster; ++jj) {
        a.first_sal[jj] = a.first_k[jj] = a.first_p[jj] = 0;
        a.narrow_mask[jj] = 0;
        if (jj >= pl.C) continue;
        const int v0 = pl.vsplit[jj];
        if (v0 < ng) {
            a.first_k[jj] = v0 / pl.Pg;
            a.first_p[jj] = v0 % pl.Pg;
        } else if (pl.Ps > 0) {
            a.first_sal[jj] = 1;
            a.first_k[jj] = (v0 - ng) / pl.Ps;
            a.first_p[jj] = (v0 - ng) % pl.Ps;
        }
        for (int v = pl.vsplit[jj]; v < pl.vsplit[jj + 1]; ++v) {
            if (v < ng && g_narrow && v % pl.Pg == pl.Pg - 1) a.narrow_mask[jj] |= 1;
            if (v >= ng && s_narrow && (v - ng) % pl.Ps == pl.Ps - 1) a.narrow_mask[jj] |= 2;
        }
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.C, pl.RB, batch);
    cfg.blockDim = dim3(pl.nwarps * 32);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = as_stream(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    int na = 1;
    if (flags & FB_GEMV_PDL) {
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        na = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return status_of(cudaLaunchKernelEx(&cfg, fn, a));
}

extern "C" fb_status fb_gemv(const fb_weights *W, const void *x, fb_dtype t, float *y, void *ws,
                             size_t ws_bytes, unsigned flags, void *stream) {
    if (!W) return FB_ERR_INVALID_VALUE;
    return fb_gemv_batched(W, x, t, 1, W->N, y, W->M, ws, ws_bytes, flags, stream);
}
